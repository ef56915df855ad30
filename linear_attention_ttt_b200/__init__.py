"""B200-native chunked TTT-layer forward (TTT-Linear MSE, inner-product /
linear attention, LaCT SwiGLU). The compute path is the CUDA library
``libttt_b200.so`` behind the C ABI in ``include/ttt.h``; this package only
marshals arguments to it (``linear_attention_ttt_b200.ops``)."""

__all__ = ["synth"]
