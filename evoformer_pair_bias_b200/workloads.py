"""Seeded synthetic workloads for Evoformer pair-bias attention.

This module only draws random inputs and arranges them in memory; it holds
none of the attention arithmetic.  Tests, the oracle checks and ``bench.py``
all take their inputs from here, so the CUDA path and the fp64 oracle see the
same rounded values.

The shapes are the AF2/AF3 training shapes of the pages (MSA-row attention
with pair bias at initial-training and fine-tuning size, triangle attention
around the starting and the ending node, and a long AF3-style triangle case);
no public dataset is involved, every tensor is drawn from N(0, 1) by a seeded
CPU generator.

Recipe (per workload, generator seeded with ``seed``): draw q, k, v, g,
pair_bias and dout in fp32 in that order, scale pair_bias by ``bias_scale``,
then draw the mask permutation; round everything to ``dtype``.  Masks are
additive ``-1e9`` on a residue subset shared by every row s:
``"tail:n"`` masks the last n residues, ``"frac:p"`` masks ``round(p*N)``
residues chosen by a random permutation, ``"none"`` passes no mask.

Layouts.  The op's logical tensors are ``[B, S, N, H, C]`` (row s, residue
n).  ``msa_row`` and ``tri_start`` store them contiguously.  ``tri_end``
(triangle attention around the ending node) stores the pair-derived tensors
in the natural pair layout ``[B, N_i, N_j, H, C]`` and the op reads them
through a transposed view (row s = j, residue n = i), with no copy.
"""
from __future__ import annotations

import dataclasses

import torch

MASK_VALUE = -1e9


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    N: int
    H: int
    C: int
    dtype: str            # "bf16" or "f32"
    layout: str           # "msa_row" | "tri_start" | "tri_end"
    bias_scale: float
    mask: str             # "none" | "tail:n" | "frac:p"
    seed: int
    note: str = ""

    @property
    def torch_dtype(self):
        return {"bf16": torch.bfloat16, "f32": torch.float32}[self.dtype]

    @property
    def logits(self) -> int:
        """Number of attention logits B*S*H*N*N."""
        return self.B * self.S * self.H * self.N * self.N

    @property
    def fwd_flops(self) -> int:
        """FlashAttention convention: QK^T and PV, 2 flops per MAC."""
        return 4 * self.logits * self.C

    @property
    def bwd_flops(self) -> int:
        """FlashAttention convention: 2.5x forward (QK^T recompute, dP, dV, dK, dQ)."""
        return 10 * self.logits * self.C

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five configurations (the fourth has two parts: MSA-row and triangle-end).
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 4, 32, 4, 8, "f32", "msa_row", 1.0, "tail:4", 20261,
                         "tiny oracle case, fp32"),
    "msa_row_256": Workload("msa_row_256", 1, 128, 256, 8, 32, "bf16", "msa_row", 0.5, "frac:0.1",
                            20262, "MSA-row attention with pair bias, AF2 initial training"),
    "tri_start_256": Workload("tri_start_256", 1, 256, 256, 4, 32, "bf16", "tri_start", 1.0, "none",
                              20263, "triangle attention around the starting node"),
    "msa_row_384": Workload("msa_row_384", 1, 512, 384, 8, 32, "bf16", "msa_row", 1.0, "frac:0.05",
                            20264, "MSA-row attention, fine-tuning size"),
    "tri_end_384": Workload("tri_end_384", 1, 384, 384, 4, 32, "bf16", "tri_end", 1.0, "frac:0.05",
                            20265, "triangle attention around the ending node (transposed pair)"),
    "tri_long_1536": Workload("tri_long_1536", 1, 1536, 1536, 4, 32, "bf16", "tri_start", 1.0,
                              "tail:64", 20266, "long AF3-style triangle attention"),
}

#: Bench default: the long AF3-style triangle attention (N_res = 1536), the largest
#: configuration that runs on one GPU and the regime (N_res >= 384) the targets are stated for.
DEFAULT_BENCH = "tri_long_1536"


def mask_columns(w: Workload, gen: torch.Generator) -> torch.Tensor | None:
    """Indices of the masked residues (shared by every row), or None."""
    if w.mask == "none":
        return None
    kind, arg = w.mask.split(":")
    if kind == "tail":
        n = int(arg)
        return torch.arange(w.N - n, w.N)
    if kind == "frac":
        n = int(round(float(arg) * w.N))
        return torch.randperm(w.N, generator=gen)[:n].sort().values
    raise ValueError(f"unknown mask recipe {w.mask!r}")


def _storage_shape(w: Workload):
    if w.layout == "tri_end":
        # natural pair layout [B, N_i, N_j, H, C]; logical row s = j, residue n = i
        return (w.B, w.N, w.S, w.H, w.C)
    return (w.B, w.S, w.N, w.H, w.C)


def logical_view(w: Workload, t: torch.Tensor) -> torch.Tensor:
    """Logical [B, S, N, H, C] view of a tensor stored in the workload's layout."""
    if w.layout == "tri_end":
        return t.permute(0, 2, 1, 3, 4)
    return t


def storage_empty(w: Workload, dtype=None, device="cpu") -> torch.Tensor:
    """An uninitialised per-row tensor in the workload's storage layout (logical view)."""
    t = torch.empty(_storage_shape(w), dtype=dtype or w.torch_dtype, device=device)
    return logical_view(w, t)


def make_inputs(w: Workload, device="cpu", with_dout: bool = True) -> dict:
    """Seeded inputs for workload ``w``.

    Returns q, k, v, g, dout as logical ``[B,S,N,H,C]`` views (strided for
    ``tri_end``), ``mask_bias`` ``[B,S,1,1,N]`` or None, ``pair_bias``
    ``[B,1,H,N,N]``, all rounded to ``w.dtype`` and placed on ``device``.
    """
    if w.layout == "tri_end" and w.S != w.N:
        raise ValueError("triangle attention needs S == N")
    gen = torch.Generator("cpu").manual_seed(w.seed)
    shp = _storage_shape(w)
    out = {}
    for name in ("q", "k", "v", "g"):
        out[name] = torch.randn(shp, generator=gen, dtype=torch.float32)
    pb = torch.randn((w.B, 1, w.H, w.N, w.N), generator=gen, dtype=torch.float32)
    if w.bias_scale != 1.0:
        pb = pb * w.bias_scale
    out["pair_bias"] = pb
    if with_dout:
        out["dout"] = torch.randn(shp, generator=gen, dtype=torch.float32)
    cols = mask_columns(w, gen)
    if cols is not None:
        m = torch.zeros((w.B, w.S, 1, 1, w.N), dtype=torch.float32)
        m[..., cols] = MASK_VALUE
        out["mask_bias"] = m
    else:
        out["mask_bias"] = None
    res = {}
    for name, t in out.items():
        if t is None:
            res[name] = None
            continue
        t = t.to(w.torch_dtype).to(device)
        res[name] = logical_view(w, t) if name in ("q", "k", "v", "g", "dout") else t
    return res


def finite_mask(w: Workload, kind: str, seed: int, device="cpu") -> torch.Tensor:
    """A seeded additive mask ``[B, S, 1, 1, N]`` with finite values that differ per row s.

    ``"gauss3"``: every entry ~ 3 N(0, 1); ``"gauss1"``: ~ N(0, 1).  ``"mixed"``: every entry ~ 2 N(0, 1),
    then a random 20% of the entries of each row s set to ``-1e9`` (at least one
    key of every row stays finite).  Rounded to ``w.dtype``.
    """
    gen = torch.Generator("cpu").manual_seed(seed)
    if kind in ("gauss3", "gauss1"):
        m = (3.0 if kind == "gauss3" else 1.0) * torch.randn((w.B, w.S, 1, 1, w.N), generator=gen)
    elif kind == "mixed":
        m = 2.0 * torch.randn((w.B, w.S, 1, 1, w.N), generator=gen)
        drop = torch.rand((w.B, w.S, 1, 1, w.N), generator=gen) < 0.2
        drop[..., 0] = False
        m[drop] = MASK_VALUE
    else:
        raise ValueError(f"unknown mask kind {kind!r}")
    return m.to(w.torch_dtype).to(device)


def sample_rows(n: int, count: int, seed: int) -> list[int]:
    """A seeded sorted sample of ``count`` distinct indices in [0, n), always with 0 and n-1."""
    gen = torch.Generator("cpu").manual_seed(seed)
    count = min(count, n)
    pick = set(torch.randperm(n, generator=gen)[:count].tolist())
    pick.update({0, n - 1})
    return sorted(pick)


def logits_bytes(n_res: int, heads: int, elem_bytes: int = 2) -> int:
    """Bytes of one layer's triangle-attention logits, N^3 * H * elem (never materialised here)."""
    return n_res ** 3 * heads * elem_bytes


def pair_rep_bytes(n_res: int, c_z: int = 128, elem_bytes: int = 2) -> int:
    """Bytes of the pair representation, N^2 * c_z * elem."""
    return n_res ** 2 * c_z * elem_bytes


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["Workload", "WORKLOADS", "DEFAULT_BENCH", "MASK_VALUE", "make_inputs", "finite_mask",
           "logical_view", "storage_empty", "sample_rows", "logits_bytes", "pair_rep_bytes",
           "mask_columns", "ceil_div", "ProjWorkload", "PROJ_WORKLOADS", "make_proj_inputs",
           "make_pair_bias_params", "TriMulWorkload", "TRI_MUL_WORKLOADS", "make_tri_mul_inputs",
           "OpmWorkload", "OPM_WORKLOADS", "make_opm_inputs"]


# ---------------------------------------------------------------------------
# Fused pre-attention projection (LayerNorm + linear): seeded inputs only.
#
# Recipe (generator seeded with ``seed``): draw x (rows x c_in) ~ N(0, 1),
# then w ~ N(0, 1/c_in), ln_w = 1 + 0.1 N(0, 1), ln_b = 0.1 N(0, 1) and
# bias ~ N(0, 1), in that order, in fp32; x and w are rounded to bf16 (the
# LayerNorm parameters and the bias stay fp32).  Shapes: the MSA
# representation (c_m = 256) projected to q, k, v, g of MSA-row attention
# (4 x 8 heads x 32), and the pair representation (c_z = 128) projected to
# q, k, v, g of triangle attention (4 x 4 heads x 32) and to its pair bias
# (one output per head).


@dataclasses.dataclass(frozen=True)
class ProjWorkload:
    name: str
    B: int
    S: int          # rows of the representation per batch (MSA sequences, or N for the pair)
    N: int
    c_in: int
    H: int          # attention heads
    C: int          # head dim
    seed: int

    @property
    def rows(self) -> int:
        return self.B * self.S * self.N

    @property
    def n_out(self) -> int:
        return 4 * self.H * self.C

    @property
    def flops(self) -> int:
        return 2 * self.rows * self.c_in * self.n_out


PROJ_WORKLOADS = {
    "msa_proj_256": ProjWorkload("msa_proj_256", 1, 128, 256, 256, 8, 32, 20271),
    "pair_proj_256": ProjWorkload("pair_proj_256", 1, 256, 256, 128, 4, 32, 20272),
    "tiny_proj": ProjWorkload("tiny_proj", 1, 3, 50, 64, 1, 32, 20273),
}


def make_proj_inputs(w: ProjWorkload, n_out: int | None = None, device="cpu") -> dict:
    """x [B, S, N, c_in] bf16, w [c_in, n_out] bf16, ln_w / ln_b [c_in] and bias [n_out] fp32."""
    n_out = w.n_out if n_out is None else n_out
    g = torch.Generator("cpu").manual_seed(w.seed)
    x = torch.randn((w.B, w.S, w.N, w.c_in), generator=g)
    wt = torch.randn((w.c_in, n_out), generator=g) / (w.c_in ** 0.5)
    ln_w = 1 + 0.1 * torch.randn(w.c_in, generator=g)
    ln_b = 0.1 * torch.randn(w.c_in, generator=g)
    bias = torch.randn(n_out, generator=g)
    return {"x": x.to(torch.bfloat16).to(device), "w": wt.to(torch.bfloat16).to(device),
            "ln_w": ln_w.to(device), "ln_b": ln_b.to(device), "bias": bias.to(device)}


def make_pair_bias_params(w: ProjWorkload, device="cpu") -> dict:
    """Parameters of the pair-bias projection of a pair representation [B, N, N, c_in]:
    w [c_in, H] ~ N(0, 1/c_in) in bf16, ln_w = 1 + 0.1 N(0, 1), ln_b = 0.1 N(0, 1) and
    bias ~ N(0, 1) in fp32, drawn in that order from a generator seeded with seed + 1."""
    g = torch.Generator("cpu").manual_seed(w.seed + 1)
    wt = torch.randn((w.c_in, w.H), generator=g) / (w.c_in ** 0.5)
    ln_w = 1 + 0.1 * torch.randn(w.c_in, generator=g)
    ln_b = 0.1 * torch.randn(w.c_in, generator=g)
    bias = torch.randn(w.H, generator=g)
    return {"w": wt.to(torch.bfloat16).to(device), "ln_w": ln_w.to(device), "ln_b": ln_b.to(device),
            "bias": bias.to(device)}


# ---------------------------------------------------------------------------
# Triangular multiplicative update (its contraction): seeded inputs only.
#
# Recipe (generator seeded with ``seed``): a then b ~ N(0, 1) drawn as
# [B, C, N, N] (channel-first, the layout the contraction reads), scaled by
# N^(-1/4) so that z = sum_k a b stays O(1) whatever N, rounded to bf16.
# Shapes: the pair representation of N residues with C = 128 hidden channels
# (the update's width in AlphaFold2-style trunks).


@dataclasses.dataclass(frozen=True)
class TriMulWorkload:
    name: str
    B: int
    N: int
    C: int
    seed: int

    @property
    def flops(self) -> int:
        return 2 * self.B * self.C * self.N ** 3


TRI_MUL_WORKLOADS = {
    "tri_mul_256": TriMulWorkload("tri_mul_256", 1, 256, 128, 20281),
    "tri_mul_384": TriMulWorkload("tri_mul_384", 1, 384, 128, 20282),
    "tri_mul_768": TriMulWorkload("tri_mul_768", 1, 768, 128, 20283),
    "tri_mul_tiny": TriMulWorkload("tri_mul_tiny", 2, 40, 3, 20284),
}


def make_tri_mul_inputs(w: TriMulWorkload, device="cpu") -> dict:
    """a, b: bf16 [B, C, N, N] (channel-first)."""
    g = torch.Generator("cpu").manual_seed(w.seed)
    s = w.N ** -0.25
    a = torch.randn((w.B, w.C, w.N, w.N), generator=g) * s
    b = torch.randn((w.B, w.C, w.N, w.N), generator=g) * s
    return {"a": a.to(torch.bfloat16).to(device), "b": b.to(torch.bfloat16).to(device)}


# ---------------------------------------------------------------------------
# Outer product mean: seeded inputs only.
#
# Recipe (generator seeded with ``seed``): a then b ~ N(0, 1) drawn as
# [B, S, N, C] (the MSA representation's layout), rounded to bf16.  Shapes:
# an MSA of S sequences over N residues projected to C = 32 channels, the
# width of the outer product mean in AlphaFold2-style trunks.


@dataclasses.dataclass(frozen=True)
class OpmWorkload:
    name: str
    B: int
    S: int
    N: int
    C: int
    seed: int

    @property
    def flops(self) -> int:
        return 2 * self.B * self.S * (self.N * self.C) ** 2


OPM_WORKLOADS = {
    "opm_256": OpmWorkload("opm_256", 1, 128, 256, 32, 20291),
    "opm_384": OpmWorkload("opm_384", 1, 512, 384, 32, 20292),
    "opm_tiny": OpmWorkload("opm_tiny", 2, 5, 12, 8, 20293),
}


def make_opm_inputs(w: OpmWorkload, device="cpu") -> dict:
    """a, b: bf16 [B, S, N, C]."""
    g = torch.Generator("cpu").manual_seed(w.seed)
    a = torch.randn((w.B, w.S, w.N, w.C), generator=g)
    b = torch.randn((w.B, w.S, w.N, w.C), generator=g)
    return {"a": a.to(torch.bfloat16).to(device), "b": b.to(torch.bfloat16).to(device)}
