"""Plain fp64 CPU oracle for Evoformer attention with pair bias.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference`` arm) may
import this package.  The product path (``evoformer_pair_bias_b200``) never
imports, links or calls it, and it shares no code with the CUDA library.

The arithmetic lives in ``evo_ref.c`` (plain C, fp64, OpenMP over independent
outputs); this module compiles it with gcc on first use and wraps it with
ctypes.  Every function takes numpy arrays of any float dtype and widens them
to fp64 before the call, so a caller that wants the oracle to see bf16 inputs
rounds them to bf16 first and passes the rounded values.  The one exception
is ordered_sum_f32, whose definition is an fp32 sum in a fixed order.

What is computed, per (b, s, h) and query i (see the header of evo_ref.c):

    x[i, j] = q_i . k_j / sqrt(C) + mask_bias[b, s, j] + pair_bias[b, h, i, j]
    out     = sigmoid(g) * softmax_j(x) @ v,   lse = logsumexp_j(x)

This is the attention with an additive broadcast pair-bias term of the
MegaFold summary (section "EvoFlash-3D"), used for MSA-row attention and for
triangle attention around a node ("Evoformer: the memory wall ZeRO cannot
move", section "The three operations").  Pins: tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "evo_ref.c")
_BUILD = os.path.join(_HERE, "_build")
_LOCK = threading.Lock()
_LIBS: dict[int, ctypes.CDLL] = {}

#: Planted mistakes available for mutation tests (id -> what is wrong).
MUTANTS = {
    1: "pair bias dropped",
    2: "mask bias dropped",
    3: "logits scaled by 1/C instead of 1/sqrt(C)",
    4: "sigmoid gate omitted",
    5: "pair bias read transposed (b_ji instead of b_ij)",
    6: "sign of D = sum_j P dP flipped in backward",
    7: "dk missing its 1/sqrt(C) factor",
    8: "LayerNorm divides by the variance instead of its square root",
    9: "projection output columns shifted by one",
    10: "triangular update without its third index (elementwise product of the two edges)",
    11: "triangular update reading the second edge as k-j instead of j-k",
    12: "outer product summed over the sequences instead of averaged",
    13: "outer product mean with its two channel axes swapped",
    14: "partials of d_pair_bias added in reverse rank order",
    15: "last partial of d_pair_bias left out of the sum",
}
#: Which function each planted mistake breaks.
ATTENTION_MUTANTS = (1, 2, 3, 4, 5, 6, 7)
LN_LINEAR_MUTANTS = (8, 9)
TRI_MUL_MUTANTS = (10, 11)
OPM_MUTANTS = (12, 13)
PARTIALS_MUTANTS = (14, 15)


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("B", "S", "Nq", "Nk", "H", "C")]


def lib_path(mutant: int = 0) -> str:
    name = "libevo_ref.so" if mutant == 0 else f"libevo_ref_m{mutant}.so"
    return os.path.join(_BUILD, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile evo_ref.c (optionally with a planted mistake) into a shared object."""
    out = lib_path(mutant)
    with _LOCK:
        if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
            os.makedirs(_BUILD, exist_ok=True)
            tmp = f"{out}.{os.getpid()}.tmp"
            cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                   f"-DEVO_REF_MUTANT={mutant}", "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, out)
    return out


def _lib(mutant: int = 0) -> ctypes.CDLL:
    if mutant not in _LIBS:
        lib = ctypes.CDLL(build(mutant))
        p = ctypes.POINTER(ctypes.c_double)
        lib.evo_ref_forward.argtypes = [ctypes.POINTER(_Dims)] + [p] * 8
        lib.evo_ref_forward.restype = ctypes.c_int
        lib.evo_ref_backward.argtypes = [ctypes.POINTER(_Dims)] + [p] * 12
        lib.evo_ref_backward.restype = ctypes.c_int
        lib.evo_ref_mutant.restype = ctypes.c_int
        lib.evo_ref_ln_linear.argtypes = [ctypes.c_int64] * 3 + [p] * 3 + [ctypes.c_double] + [p] * 3
        lib.evo_ref_ln_linear.restype = ctypes.c_int
        lib.evo_ref_tri_mul.argtypes = [ctypes.c_int64] * 3 + [p] * 2 + [ctypes.c_int, p]
        lib.evo_ref_tri_mul.restype = ctypes.c_int
        lib.evo_ref_outer_product_mean.argtypes = [ctypes.c_int64] * 6 + [p] * 3
        lib.evo_ref_outer_product_mean.restype = ctypes.c_int
        pf = ctypes.POINTER(ctypes.c_float)
        lib.evo_ref_ordered_sum_f32.argtypes = [ctypes.c_int64, ctypes.c_int64, pf, pf]
        lib.evo_ref_ordered_sum_f32.restype = ctypes.c_int
        _LIBS[mutant] = lib
    return _LIBS[mutant]


def _f64(a):
    if a is None:
        return None
    a = np.asarray(a, dtype=np.float64)
    return np.ascontiguousarray(a)


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q, k):
    B, S, Nq, H, C = q.shape
    Bk, Sk, Nk, Hk, Ck = k.shape
    if (B, S, H, C) != (Bk, Sk, Hk, Ck):
        raise ValueError(f"q {q.shape} and k {k.shape} disagree")
    return _Dims(B, S, Nq, Nk, H, C)


def _prep(q, k, v, g, mask_bias, pair_bias):
    q, k, v, g = (_f64(t) for t in (q, k, v, g))
    d = _dims(q, k)
    if v.shape != k.shape or g.shape != q.shape:
        raise ValueError("v must match k and g must match q")
    m = None
    if mask_bias is not None:
        m = _f64(mask_bias).reshape(d.B, d.S, d.Nk)
    pb = None
    if pair_bias is not None:
        pb = _f64(pair_bias).reshape(d.B, d.H, d.Nq, d.Nk)
    return d, q, k, v, g, m, pb


def forward(q, k, v, g, mask_bias=None, pair_bias=None, *, mutant: int = 0):
    """Return (out [B,S,Nq,H,C], lse [B,S,H,Nq]) in fp64.

    q, g: [B,S,Nq,H,C]; k, v: [B,S,Nk,H,C]; mask_bias: [B,S,1,1,Nk] (or
    [B,S,Nk]); pair_bias: [B,1,H,Nq,Nk] (or [B,H,Nq,Nk]); None means zeros.
    """
    d, q, k, v, g, m, pb = _prep(q, k, v, g, mask_bias, pair_bias)
    out = np.empty(q.shape, np.float64)
    lse = np.empty((d.B, d.S, d.H, d.Nq), np.float64)
    rc = _lib(mutant).evo_ref_forward(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                      _ptr(m), _ptr(pb), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("evo_ref_forward rejected its arguments")
    return out, lse


def backward(q, k, v, g, mask_bias, pair_bias, dout, *, mutant: int = 0,
             want=("dq", "dk", "dv", "dg", "d_pair_bias")):
    """Return a dict of fp64 gradients (keys from ``want``).

    d_pair_bias has shape [B,1,H,Nq,Nk] and is the sum over all s of dS.
    dk/dv are only the true gradients when every query row is present.
    """
    d, q, k, v, g, m, pb = _prep(q, k, v, g, mask_bias, pair_bias)
    dout = _f64(dout)
    if dout.shape != q.shape:
        raise ValueError("dout must match q")
    res = {}
    shapes = {"dq": q.shape, "dk": k.shape, "dv": k.shape, "dg": q.shape,
              "d_pair_bias": (d.B, 1, d.H, d.Nq, d.Nk)}
    for name in want:
        res[name] = np.empty(shapes[name], np.float64)
    get = lambda n: _ptr(res.get(n))  # noqa: E731
    rc = _lib(mutant).evo_ref_backward(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                       _ptr(m), _ptr(pb), _ptr(dout), get("dq"), get("dk"),
                                       get("dv"), get("dg"), get("d_pair_bias"))
    if rc != 0:
        raise ValueError("evo_ref_backward rejected its arguments")
    return res


def ln_linear(x, ln_w, ln_b, eps, w, bias=None, *, mutant: int = 0):
    """LayerNorm over the last axis of x, then y = LN(x) @ w + bias, in fp64.

    x: [..., c_in]; ln_w, ln_b: [c_in] (None = ones / zeros); w: [c_in, n_out];
    bias: [n_out] or None.  Returns y with shape x.shape[:-1] + (n_out,).
    This is the fused pre-attention projection (MegaFold summary, section
    "EvoFusion"): q, k, v, g are column blocks of y, and the pair bias is y
    of the pair representation with n_out = H, read as [b, h, i, j].
    """
    x = _f64(x)
    lead, c_in = x.shape[:-1], x.shape[-1]
    w = _f64(w)
    if w.shape[0] != c_in:
        raise ValueError(f"w {w.shape} does not match c_in {c_in}")
    n_out = w.shape[1]
    x2 = x.reshape(-1, c_in)
    y = np.empty((x2.shape[0], n_out), np.float64)
    lw, lb, bb = _f64(ln_w), _f64(ln_b), _f64(bias)
    rc = _lib(mutant).evo_ref_ln_linear(x2.shape[0], c_in, n_out, _ptr(x2), _ptr(lw), _ptr(lb), float(eps),
                                        _ptr(w), _ptr(bb), _ptr(y))
    if rc != 0:
        raise ValueError("evo_ref_ln_linear rejected its arguments")
    return y.reshape(lead + (n_out,))


def tri_mul(a, b, incoming: bool = False, *, mutant: int = 0):
    """The contraction of the triangular multiplicative update, in fp64.

    a, b: [B, N, N, C] (the pair representation's layout).  Outgoing edges
    (default): z[b, i, j, c] = sum_k a[b, i, k, c] * b[b, j, k, c]; incoming:
    z[b, i, j, c] = sum_k a[b, k, i, c] * b[b, k, j, c] ("Evoformer: the memory
    wall ZeRO cannot move", section "The three operations").
    """
    a, b = _f64(a), _f64(b)
    if a.ndim != 4 or a.shape != b.shape or a.shape[1] != a.shape[2]:
        raise ValueError(f"a {a.shape} and b {b.shape} must both be [B, N, N, C]")
    B, N, _, C = a.shape
    z = np.empty_like(a)
    rc = _lib(mutant).evo_ref_tri_mul(B, N, C, _ptr(a), _ptr(b), 1 if incoming else 0, _ptr(z))
    if rc != 0:
        raise ValueError("evo_ref_tri_mul rejected its arguments")
    return z


def outer_product_mean(a, b, *, mutant: int = 0):
    """The outer product mean in fp64: out[b, i, j, c1, c2] = (1/S) sum_s a[b, s, i, c1] b[b, s, j, c2].

    a: [B, S, Na, Ca], b: [B, S, Nb, Cb] (the MSA representation's layout; Na = Nb
    = N for the full operation, Na < N for a subset of columns i); returns
    [B, Na, Nb, Ca, Cb] ("Evoformer: the memory wall ZeRO cannot move", section
    "The three operations": the outer product of MSA columns i and j averaged
    over the sequences).
    """
    a, b = _f64(a), _f64(b)
    if a.ndim != 4 or b.ndim != 4 or a.shape[:2] != b.shape[:2]:
        raise ValueError(f"a {a.shape} and b {b.shape} must be [B, S, N, C] with the same B, S")
    B, S, Na, Ca = a.shape
    Nb, Cb = b.shape[2], b.shape[3]
    out = np.empty((B, Na, Nb, Ca, Cb), np.float64)
    rc = _lib(mutant).evo_ref_outer_product_mean(B, S, Na, Nb, Ca, Cb, _ptr(a), _ptr(b), _ptr(out))
    if rc != 0:
        raise ValueError("evo_ref_outer_product_mean rejected its arguments")
    return out


def ordered_sum_f32(parts, *, mutant: int = 0):
    """Rank-ordered fp32 sum: out = (...((parts[0] + parts[1]) + parts[2]) ...) + parts[-1].

    Unlike the other functions this one works in fp32, each addition rounded
    to nearest: it is the exact expected value of the fixed-order exchange of
    d_pair_bias when the rows s of one problem are split over GPUs (the sum
    over s of the backward's dS, grouped by GPU).  parts: [count, ...] array
    (converted to fp32); returns an fp32 array of parts.shape[1:].
    """
    p = np.ascontiguousarray(parts, dtype=np.float32)
    if p.ndim < 1 or p.shape[0] < 1:
        raise ValueError("ordered_sum_f32 needs at least one partial")
    out = np.empty(p.shape[1:], np.float32)
    pf = ctypes.POINTER(ctypes.c_float)
    rc = _lib(mutant).evo_ref_ordered_sum_f32(p.shape[0], out.size, p.ctypes.data_as(pf),
                                              out.ctypes.data_as(pf))
    if rc != 0:
        raise ValueError("evo_ref_ordered_sum_f32 rejected its arguments")
    return out


def mutant_id(mutant: int) -> int:
    """The planted-mistake id compiled into that build (sanity check for tests)."""
    return int(_lib(mutant).evo_ref_mutant())
