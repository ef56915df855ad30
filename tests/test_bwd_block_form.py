"""The block form used by the TTT-Linear backward kernel equals the oracle's
token-by-token chain rule (fp64, CPU).

Over a chunk with start weights W_s (rows = tokens, N = diag(eta), E the rows
e_t = k_t W_s - v_t for MSE or -v_t for the inner product, masks inclusive of
the diagonal) the chain rule of the mini-batch rule reads
    dQ = dY W_s^T - tril(dY E^T) N K
    k_t R_t  = K G + triu(K Q^T) dY        (rows)
    R_t e_t^T = E G^T + triu(E dY^T) Q     (rows)
    deta_t = -(k_t R_t) . e_t,  dv_t = eta_t k_t R_t,  de_t = -dv_t,
    dk_t = -eta_t R_t e_t^T (+ de_t W_s^T for MSE),
    dL/dW_s = G + Q^T dY (+ K^T dE for MSE),
with G = dL/dW at the chunk end. The kernel walks each chunk in 16-token
blocks: forward with the running sum of the chunk's updates (for dQ), then in
reverse with R = G + the q^T dy of the later blocks. This restates that walk
in numpy and compares it with the oracle for ragged chunks, chunks shorter
and longer than a block, dk != dv, a W0 per sequence and no final gradient.
"""
import numpy as np
import pytest

from oracle import ttt_oracle as O
from linear_attention_ttt_b200 import synth

TB = 16


def block_form(q, k, v, eta, W0, chunk, mse, dy, G):
    """One (batch, head): q, k [T,dk], v, dy [T,dv], eta [T], W0, G [dk,dv]."""
    T, dk = q.shape
    dv = v.shape[1]
    dq, dkk, dvv = np.zeros((T, dk)), np.zeros((T, dk)), np.zeros((T, dv))
    deta = np.zeros(T)
    nch = (T + chunk - 1) // chunk

    def block(t0, nt):
        Q, K = np.zeros((TB, dk)), np.zeros((TB, dk))
        V, Y, et = np.zeros((TB, dv)), np.zeros((TB, dv)), np.zeros(TB)
        Q[:nt], K[:nt], V[:nt] = q[t0:t0 + nt], k[t0:t0 + nt], v[t0:t0 + nt]
        Y[:nt], et[:nt] = dy[t0:t0 + nt], eta[t0:t0 + nt]
        return Q, K, V, Y, et

    # pass 1: chunk-start weights and dQ
    Ws, starts = W0.copy(), []
    for c in range(nch):
        s0, e0 = c * chunk, min((c + 1) * chunk, T)
        starts.append(Ws.copy())
        acc = np.zeros((dk, dv))
        for t0 in range(s0, e0, TB):
            nt = min(TB, e0 - t0)
            Q, K, V, Y, et = block(t0, nt)
            E = (K @ Ws if mse else 0.0) - V
            S = np.tril(Y @ E.T) * et[None, :]
            S[nt:] = 0.0
            dq[t0:t0 + nt] = (Y @ (Ws - acc).T - S @ K)[:nt]
            acc = acc + K.T @ (et[:, None] * E)
        Ws = Ws - acc
    # pass 2: reverse, R carried over blocks and chunks
    R = G.copy()
    for c in reversed(range(nch)):
        s0, e0 = c * chunk, min((c + 1) * chunk, T)
        Ws, kde = starts[c], np.zeros((dk, dv))
        nb = (e0 - s0 + TB - 1) // TB
        for bi in reversed(range(nb)):
            t0 = s0 + bi * TB
            nt = min(TB, e0 - t0)
            Q, K, V, Y, et = block(t0, nt)
            E = (K @ Ws if mse else 0.0) - V
            mask = np.triu(np.ones((TB, TB)))
            mask[:, nt:] = 0.0
            kR = K @ R + (mask * (K @ Q.T)) @ Y
            Rx = E @ R.T + (mask * (E @ Y.T)) @ Q
            deta[t0:t0 + nt] = -(kR * E).sum(1)[:nt]
            dvb = et[:, None] * kR
            dvv[t0:t0 + nt] = dvb[:nt]
            de = -dvb
            dkk[t0:t0 + nt] = ((de @ Ws.T if mse else 0.0) - et[:, None] * Rx)[:nt]
            R = R + Q.T @ Y
            if mse:
                kde = kde + K.T @ de
        R = R + kde
    return dq, dkk, dvv, deta, R


CASES = [  # (B, H, T, dk, dv, chunk, batched W0, final gradient)
    (1, 2, 40, 32, 48, 16, False, True),
    (1, 2, 37, 32, 48, 5, False, True),
    (1, 1, 16, 16, 24, 1, False, True),
    (1, 2, 50, 32, 32, 64, False, True),
    (1, 1, 70, 24, 16, 32, False, True),
    (2, 2, 33, 16, 16, 8, True, False),
    (1, 1, 0, 16, 16, 4, False, True),
]


@pytest.mark.parametrize("loss", [synth.LOSS_MSE, synth.LOSS_NEG_DOT])
@pytest.mark.parametrize("B,H,T,dk,dv,chunk,batched,with_g", CASES)
def test_block_form_equals_chain_rule(loss, B, H, T, dk, dv, chunk, batched, with_g):
    w = synth.make_ttt_linear(B, H, T, dk, dv, chunk, synth.F32, loss, seed=T + chunk + dk,
                              eta_kind="softplus", eta_scale=0.1, w0_std=0.1,
                              w0_batched=batched)
    rng = np.random.default_rng(T + dv)
    dy = rng.standard_normal((B, H, T, dv))
    G = rng.standard_normal((B, H, dk, dv)) if with_g else None
    want = O.ttt_linear_minibatch_bwd(w.q, w.k, w.v, w.eta, w.W0, chunk, loss, dy, G)
    f = lambda x: np.asarray(x, dtype=np.float64)
    W0 = f(w.W0)
    got = [np.zeros((B, H) + x.shape[2:]) for x in want[:4]] + [np.zeros((B, H, dk, dv))]
    for b in range(B):
        for h in range(H):
            r = block_form(f(w.q[b, h]), f(w.k[b, h]), f(w.v[b, h]), f(w.eta[b, h]),
                           W0[b, h] if W0.ndim == 4 else W0[h], chunk,
                           loss == synth.LOSS_MSE, dy[b, h],
                           G[b, h] if G is not None else np.zeros((dk, dv)))
            for dst, x in zip(got, r):
                dst[b, h] = x
    if W0.ndim == 3:
        got[4] = got[4].sum(axis=0)
    for g, o, n in zip(got, want, ("dq", "dk", "dv", "deta", "dW0")):
        o = f(o)
        assert g.shape == o.shape, n
        if o.size:
            scale = max(np.abs(o).max(), 1e-30)
            assert np.abs(g - o).max() <= 1e-11 * scale, n
