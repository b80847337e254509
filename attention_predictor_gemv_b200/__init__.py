"""Deja Vu contextual-sparsity decode hot path for B200 (sm_100a).

The CUDA library is loaded by ``attention_predictor_gemv_b200.binding``; this
package import itself does not load it, so the input generators and the byte
accounting work on machines without a GPU.
"""
