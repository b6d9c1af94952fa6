"""Evoformer attention with pair bias on B200 (sm_100a).

``out = sigmoid(g) * softmax(q k^T / sqrt(c) + mask_bias + pair_bias) v`` over
``[B, N_seq, N_res, H, c]`` tensors, forward and backward, computed by
hand-written CUDA kernels behind the C-ABI declared in ``include/evo_attn.h``.
The Python layer (``evoformer_pair_bias_b200.attention``) only marshals
torch tensors into that ABI; it never computes anything itself.
``evoformer_pair_bias_b200.row_shards`` splits one problem's rows over a
process group: the backward's one exchange, d_pair_bias, is all-gathered and
added in rank order by the library's ``evo_sum_partials``.
"""
from . import workloads  # noqa: F401  (seeded synthetic inputs; no arithmetic)

__all__ = ["workloads"]
