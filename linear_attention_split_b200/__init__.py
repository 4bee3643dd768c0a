"""B200 (sm_100a) Test-Time-Training layer: C-ABI CUDA library + thin Python binding.

    from linear_attention_split_b200 import ttt
    out = ttt.linear_fullbatch(q, k, v, w0)          # TTT-Linear, one full-batch step
    out = ttt.dwconv_fullbatch(q, k, v, taps)        # 3x3 depthwise-conv inner model
    out = ttt.mlp_fullbatch(q, k, v, w1, w2)         # TTT-MLP (tanh-GELU)
    out = ttt.linear_chunked_bidir(q, k, v, w0, 64)  # chunked bidirectional scan
"""
__all__ = ["ttt", "inputs"]
