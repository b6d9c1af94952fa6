"""Python binding of libevo_attn.so (include/evo_attn.h).

Argument marshalling only: these functions turn torch tensors into the
pointers, sizes and strides of the C-ABI and call it on the current CUDA
stream.  Every step of the computation runs in the library's CUDA kernels;
there is no fallback of any kind -- if the library is missing or rejects a
call, an exception says why.

    out, lse, out_lo = evo_attn_fwd(q, k, v, g, mask_bias, pair_bias, out_lo=True)
    grads = evo_attn_bwd(q, k, v, g, mask_bias, pair_bias, out, lse, dout, out_lo=out_lo)

Per-row tensors (q, k, v, g, out, dout and the gradients) are logical
``[B, S, N, H, C]`` views with a contiguous C axis; any other strides are
passed through, so the triangle attention around the ending node is the same
call on a transposed view.  ``mask_bias`` is ``[B, S, 1, 1, N]`` and
``pair_bias`` ``[B, 1, H, N, N]`` (both contiguous, or None).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libevo_attn.so")

EVO_OK = 0
STATUS = {0: "EVO_OK", 1: "EVO_ERR_INVALID_ARG", 2: "EVO_ERR_UNSUPPORTED", 3: "EVO_ERR_WORKSPACE_TOO_SMALL",
          4: "EVO_ERR_CUDA", 5: "EVO_ERR_DEVICE_TIMEOUT"}
DTYPES = {torch.bfloat16: 0, torch.float32: 1}

#: Every symbol include/evo_attn.h declares.
EXPORTS = ("evo_attn_fwd", "evo_attn_bwd", "evo_attn_bwd_workspace_bytes", "evo_status_string",
           "evo_attn_device_status", "evo_attn_version", "evo_attn_launch_count", "evo_attn_bwd_noalloc",
           "evo_attn_timing_enable", "evo_attn_timing_collect", "evo_ln_linear", "evo_ln_pair_bias",
           "evo_tri_mul", "evo_outer_product_mean", "evo_sum_partials", "evo_attn_set_wait_limit_ns",
           "evo_exp2_fma")

#: Default limit of the kernels' bounded waits (EVO_WAIT_LIMIT_NS), nanoseconds.
DEFAULT_WAIT_LIMIT_NS = 2_000_000_000

#: Most partials one evo_sum_partials call adds (EVO_MAX_PARTIALS).
MAX_PARTIALS = 64

#: Size of the library's fixed scratch area used by evo_attn_bwd_noalloc (bytes).
NOALLOC_WORKSPACE_BYTES = 32 << 20


class EvoError(RuntimeError):
    def __init__(self, where: str, code: int):
        super().__init__(f"{where} failed: {STATUS.get(code, code)}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("B", "S", "N", "H", "C")]


class Strides(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("b", "s", "n", "h")]


#: Timing phases (evo_timing_t indices).
PHASES = ("fwd_main", "bwd_main", "bwd_all", "proj", "pair_bias", "tri_mul", "opm", "bwd_dbias")


class Timing(ctypes.Structure):
    _fields_ = [("calls", ctypes.c_uint64 * len(PHASES)), ("ms", ctypes.c_double * len(PHASES))]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libevo_attn.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m evoformer_pair_bias_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sp, stp = ctypes.c_void_p, ctypes.POINTER(Shape), ctypes.POINTER(Strides)
    lib.evo_attn_fwd.argtypes = [sp, ctypes.c_int, vp, vp, vp, vp, stp, vp, vp, vp, vp, stp, vp, vp]
    lib.evo_attn_fwd.restype = ctypes.c_int
    lib.evo_attn_bwd.argtypes = [sp, ctypes.c_int, vp, vp, vp, vp, stp, vp, vp, vp, vp, vp, stp, vp,
                                 vp, vp, vp, vp, stp, vp, vp, ctypes.c_size_t, vp]
    lib.evo_attn_bwd.restype = ctypes.c_int
    lib.evo_attn_bwd_workspace_bytes.argtypes = [sp, ctypes.c_int]
    lib.evo_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.evo_status_string.argtypes = [ctypes.c_int]
    lib.evo_status_string.restype = ctypes.c_char_p
    lib.evo_attn_device_status.argtypes = [ctypes.c_int]
    lib.evo_attn_device_status.restype = ctypes.c_int
    lib.evo_attn_version.restype = ctypes.c_int
    lib.evo_attn_launch_count.restype = ctypes.c_uint64
    lib.evo_attn_bwd_noalloc.argtypes = [sp, ctypes.c_int, vp, vp, vp, vp, stp, vp, vp, vp, vp, vp, stp, vp,
                                         vp, vp, vp, vp, stp, vp, vp]
    lib.evo_attn_bwd_noalloc.restype = ctypes.c_int
    lib.evo_attn_timing_enable.argtypes = [ctypes.c_int]
    lib.evo_attn_timing_enable.restype = ctypes.c_int
    lib.evo_attn_timing_collect.argtypes = [ctypes.POINTER(Timing)]
    lib.evo_attn_timing_collect.restype = ctypes.c_int
    i64, f32 = ctypes.c_int64, ctypes.c_float
    lib.evo_ln_linear.argtypes = [i64, i64, i64, vp, vp, vp, f32, vp, vp, vp, i64, vp]
    lib.evo_ln_linear.restype = ctypes.c_int
    lib.evo_ln_pair_bias.argtypes = [i64, i64, i64, i64, vp, vp, vp, f32, vp, vp, vp, vp]
    lib.evo_ln_pair_bias.restype = ctypes.c_int
    lib.evo_tri_mul.argtypes = [i64, i64, i64, vp, vp, ctypes.c_int, vp, vp]
    lib.evo_tri_mul.restype = ctypes.c_int
    lib.evo_outer_product_mean.argtypes = [i64, i64, i64, i64, i64, vp, vp, vp, vp]
    lib.evo_outer_product_mean.restype = ctypes.c_int
    lib.evo_sum_partials.argtypes = [i64, ctypes.POINTER(ctypes.c_void_p), i64, vp, vp]
    lib.evo_sum_partials.restype = ctypes.c_int
    lib.evo_attn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.evo_attn_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.evo_exp2_fma.argtypes = [vp, vp, i64, vp]
    lib.evo_exp2_fma.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _shape(q) -> Shape:
    if q.dim() != 5:
        raise ValueError(f"expected a [B,S,N,H,C] tensor, got shape {tuple(q.shape)}")
    return Shape(*q.shape)


def _strides(t) -> Strides:
    st = t.stride()
    if t.shape[4] > 1 and st[4] != 1:
        raise ValueError("the C axis must be contiguous")
    return Strides(st[0], st[1], st[2], st[3])


def _same_strides(*ts):
    ref = ts[0].stride()
    for t in ts[1:]:
        if t.stride() != ref:
            raise ValueError("q, k, v and g (and out/dout, and the gradients) must share strides")


def _check(where: str, rc: int):
    if rc != EVO_OK:
        raise EvoError(where, rc)


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check_biases(q, mask_bias, pair_bias):
    """mask_bias [B,S,1,1,N] and pair_bias [B,1,H,N,N]: contiguous, of q's dtype, on q's device.

    The library reads both as dense arrays of those shapes, so a strided view
    (a slice of a larger mask over rows s, say) or another dtype would be read
    as the wrong values; such arguments are refused here instead.
    """
    B, S, N, H, _ = q.shape
    for name, t, shape in (("mask_bias", mask_bias, (B, S, 1, 1, N)), ("pair_bias", pair_bias, (B, 1, H, N, N))):
        if t is None:
            continue
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous (pass .contiguous() of a strided view)")
        if t.dtype != q.dtype or t.device != q.device:
            raise ValueError(f"{name} must be of q's dtype and device")


def _check_lse(q, lse):
    """lse [B,S,H,N]: contiguous fp32 on q's device."""
    B, S, N, H, _ = q.shape
    if tuple(lse.shape) != (B, S, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous() \
            or lse.device != q.device:
        raise ValueError(f"lse must be a contiguous fp32 tensor of shape {(B, S, H, N)} on q's device")


def empty_like_rows(t: torch.Tensor, dtype=None) -> torch.Tensor:
    """Uninitialised tensor with t's shape and strides (keeps the transposed-pair layout)."""
    return torch.empty_strided(t.shape, t.stride(), dtype=dtype or t.dtype, device=t.device)


def workspace_bytes(q: torch.Tensor) -> int:
    lib = load_library()
    return int(lib.evo_attn_bwd_workspace_bytes(ctypes.byref(_shape(q)), DTYPES[q.dtype]))


def evo_attn_fwd(q, k, v, g, mask_bias=None, pair_bias=None, out=None, lse=None, out_lo=None):
    """Forward pass; returns (out, lse), or (out, lse, out_lo) when ``out_lo`` is given.

    out/lse may be passed in preallocated.  ``out_lo`` (bf16 only): True to
    allocate, or a tensor shaped and strided like out, that receives the
    rounding residual of out (pass it on to evo_attn_bwd for an accurate D_i,
    which is what keeps d_pair_bias's error small at large N_seq).
    """
    lib = load_library()
    _same_strides(q, k, v, g)
    sh = _shape(q)
    B, S, N, H, C = q.shape
    if out is None:
        out = empty_like_rows(q)
    _check_biases(q, mask_bias, pair_bias)
    if lse is None:
        lse = torch.empty((B, S, H, N), dtype=torch.float32, device=q.device)
    _check_lse(q, lse)
    want_lo = out_lo is not None and out_lo is not False
    if out_lo is True:
        out_lo = empty_like_rows(out)
    if want_lo and (out_lo.stride() != out.stride() or out_lo.dtype != out.dtype or out_lo.shape != out.shape):
        raise ValueError("out_lo must have out's shape, strides and dtype")
    rc = lib.evo_attn_fwd(ctypes.byref(sh), DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                          ctypes.byref(_strides(q)), _ptr(mask_bias), _ptr(pair_bias), _ptr(out),
                          _ptr(out_lo) if want_lo else None, ctypes.byref(_strides(out)), _ptr(lse),
                          _stream(q.device))
    _check("evo_attn_fwd", rc)
    return (out, lse, out_lo) if want_lo else (out, lse)


def _check_out_lo(out, out_lo):
    if out_lo is not None and (out_lo.stride() != out.stride() or out_lo.dtype != out.dtype
                               or out_lo.shape != out.shape or out_lo.device != out.device):
        raise ValueError("out_lo must have out's shape, strides, dtype and device")


def evo_attn_bwd(q, k, v, g, mask_bias, pair_bias, out, lse, dout, grads=None, workspace=None, out_lo=None):
    """Backward pass; returns dict(dq, dk, dv, dg, d_pair_bias).

    d_pair_bias is fp32 ``[B, 1, H, N, N]``.  ``grads`` may hold preallocated
    outputs, ``workspace`` a preallocated uint8 buffer of ``workspace_bytes(q)``,
    ``out_lo`` the forward's rounding residual of out (or None).
    """
    lib = load_library()
    _same_strides(q, k, v, g)
    _same_strides(out, dout)
    sh = _shape(q)
    B, S, N, H, C = q.shape
    _check_biases(q, mask_bias, pair_bias)
    _check_lse(q, lse)
    _check_out_lo(out, out_lo)
    grads = dict(grads or {})
    for n in ("dq", "dk", "dv", "dg"):
        if grads.get(n) is None:
            grads[n] = empty_like_rows(q)
    if grads.get("d_pair_bias") is None:
        grads["d_pair_bias"] = torch.empty((B, 1, H, N, N), dtype=torch.float32, device=q.device)
    _same_strides(grads["dq"], grads["dk"], grads["dv"], grads["dg"])
    need = int(lib.evo_attn_bwd_workspace_bytes(ctypes.byref(sh), DTYPES[q.dtype]))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    rc = lib.evo_attn_bwd(ctypes.byref(sh), DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                          ctypes.byref(_strides(q)), _ptr(mask_bias), _ptr(pair_bias), _ptr(out), _ptr(out_lo),
                          _ptr(dout), ctypes.byref(_strides(out)), _ptr(lse), _ptr(grads["dq"]), _ptr(grads["dk"]),
                          _ptr(grads["dv"]), _ptr(grads["dg"]), ctypes.byref(_strides(grads["dq"])),
                          _ptr(grads["d_pair_bias"]), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                          _stream(q.device))
    _check("evo_attn_bwd", rc)
    return grads


def evo_attn_bwd_noalloc(q, k, v, g, mask_bias, pair_bias, out, lse, dout, grads=None, out_lo=None):
    """Backward pass through evo_attn_bwd_noalloc: no workspace is passed or allocated.

    For callers that must not allocate device memory: the library uses its own
    fixed scratch area (NOALLOC_WORKSPACE_BYTES per device), shared by every call,
    so calls must not overlap on the GPU.  Output tensors may be passed in
    ``grads``; any that are missing are allocated here by torch, as plumbing.
    """
    lib = load_library()
    _same_strides(q, k, v, g)
    _same_strides(out, dout)
    sh = _shape(q)
    B, S, N, H, C = q.shape
    _check_biases(q, mask_bias, pair_bias)
    _check_lse(q, lse)
    _check_out_lo(out, out_lo)
    grads = dict(grads or {})
    for n in ("dq", "dk", "dv", "dg"):
        if grads.get(n) is None:
            grads[n] = empty_like_rows(q)
    if grads.get("d_pair_bias") is None:
        grads["d_pair_bias"] = torch.empty((B, 1, H, N, N), dtype=torch.float32, device=q.device)
    _same_strides(grads["dq"], grads["dk"], grads["dv"], grads["dg"])
    rc = lib.evo_attn_bwd_noalloc(ctypes.byref(sh), DTYPES[q.dtype], _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                  ctypes.byref(_strides(q)), _ptr(mask_bias), _ptr(pair_bias), _ptr(out),
                                  _ptr(out_lo), _ptr(dout), ctypes.byref(_strides(out)), _ptr(lse), _ptr(grads["dq"]),
                                  _ptr(grads["dk"]), _ptr(grads["dv"]), _ptr(grads["dg"]),
                                  ctypes.byref(_strides(grads["dq"])), _ptr(grads["d_pair_bias"]),
                                  _stream(q.device))
    _check("evo_attn_bwd_noalloc", rc)
    return grads


def launch_count() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(load_library().evo_attn_launch_count())


def _opt_f32(t, n, device):
    if t is None:
        return None
    t = t.to(device=device, dtype=torch.float32).contiguous()
    if t.numel() != n:
        raise ValueError(f"expected {n} values, got {t.numel()}")
    return t


def ln_linear(x, ln_w, ln_b, eps, w, bias=None, y=None):
    """Fused LayerNorm + linear: y = LayerNorm(x) @ w + bias (bf16 in and out).

    x: bf16 [..., c_in] (rows contiguous); ln_w, ln_b, bias: any float tensors
    (None = ones / zeros / zeros); w: bf16 [c_in, n_out].  Returns y with shape
    x.shape[:-1] + (n_out,).  With w = [w_q | w_k | w_v | w_g], qkvg_views(y, H)
    gives q, k, v, g as attention inputs without a copy.
    """
    lib = load_library()
    c_in = x.shape[-1]
    xc = x.contiguous().view(-1, c_in)
    n_out = w.shape[1]
    if w.shape[0] != c_in:
        raise ValueError(f"w {tuple(w.shape)} does not match c_in {c_in}")
    wc = w.contiguous()
    if y is None:
        y = torch.empty(x.shape[:-1] + (n_out,), dtype=torch.bfloat16, device=x.device)
    lw, lb, bb = (_opt_f32(t, n, x.device) for t, n in ((ln_w, c_in), (ln_b, c_in), (bias, n_out)))
    rc = lib.evo_ln_linear(xc.shape[0], c_in, n_out, _ptr(xc), _ptr(lw), _ptr(lb), float(eps), _ptr(wc),
                           _ptr(bb), _ptr(y), n_out, _stream(x.device))
    _check("evo_ln_linear", rc)
    return y


def qkvg_views(y, H: int):
    """q, k, v, g as [B, S, N, H, C] views of a ln_linear output [B, S, N, 4*H*C]."""
    B, S, N, F = y.shape
    C = F // (4 * H)
    if 4 * H * C != F:
        raise ValueError(f"last axis {F} is not 4 * H * C")
    y5 = y.view(B, S, N, 4, H, C)
    return tuple(y5[:, :, :, m] for m in range(4))


def ln_pair_bias(z, ln_w, ln_b, eps, w, bias=None, out=None):
    """Pair-bias projection: pair_bias[b, 0, h, i, j] = LayerNorm(z[b, i, j]) @ w[:, h] + bias[h].

    z: bf16 [B, N, N, c_z]; w: bf16 [c_z, H].  Returns bf16 [B, 1, H, N, N].
    """
    lib = load_library()
    B, N, N2, c_z = z.shape
    if N2 != N or w.shape[0] != c_z:
        raise ValueError("z must be [B, N, N, c_z] and w [c_z, H]")
    H = w.shape[1]
    zc, wc = z.contiguous(), w.contiguous()
    if out is None:
        out = torch.empty((B, 1, H, N, N), dtype=torch.bfloat16, device=z.device)
    lw, lb, bb = (_opt_f32(t, n, z.device) for t, n in ((ln_w, c_z), (ln_b, c_z), (bias, H)))
    rc = lib.evo_ln_pair_bias(B, N, c_z, H, _ptr(zc), _ptr(lw), _ptr(lb), float(eps), _ptr(wc), _ptr(bb),
                              _ptr(out), _stream(z.device))
    _check("evo_ln_pair_bias", rc)
    return out


def tri_mul(a, b, incoming: bool = False, z=None):
    """Triangular multiplicative update contraction on channel-first bf16 [B, C, N, N] tensors.

    Outgoing edges: z[b, c, i, j] = sum_k a[b, c, i, k] * b[b, c, j, k]; incoming:
    z[b, c, i, j] = sum_k a[b, c, k, i] * b[b, c, k, j].  Returns z (bf16, same shape).
    """
    lib = load_library()
    if a.dim() != 4 or a.shape != b.shape or a.shape[2] != a.shape[3]:
        raise ValueError("a and b must both be [B, C, N, N]")
    B, C, N, _ = a.shape
    ac, bc = a.contiguous(), b.contiguous()
    if z is None:
        z = torch.empty_like(ac)
    rc = lib.evo_tri_mul(B, C, N, _ptr(ac), _ptr(bc), 1 if incoming else 0, _ptr(z), _stream(a.device))
    _check("evo_tri_mul", rc)
    return z


def outer_product_mean(a, b, out=None):
    """Outer product mean: out[b, i, c1, j, c2] = (1/S) sum_s a[b, s, i, c1] b[b, s, j, c2].

    a: bf16 [B, S, N, Ca], b: bf16 [B, S, N, Cb].  Returns bf16 [B, N, Ca, N, Cb];
    opm_pair_view(out) is the same data as the pair layout [B, N, N, Ca, Cb].
    """
    lib = load_library()
    if a.dim() != 4 or b.dim() != 4 or a.shape[:3] != b.shape[:3]:
        raise ValueError("a and b must be [B, S, N, C] with the same B, S, N")
    B, S, N, Ca = a.shape
    Cb = b.shape[3]
    ac, bc = a.contiguous(), b.contiguous()
    if out is None:
        out = torch.empty((B, N, Ca, N, Cb), dtype=torch.bfloat16, device=a.device)
    rc = lib.evo_outer_product_mean(B, S, N, Ca, Cb, _ptr(ac), _ptr(bc), _ptr(out), _stream(a.device))
    _check("evo_outer_product_mean", rc)
    return out


def sum_partials(parts, out=None):
    """Fixed-order fp32 sum: out = (...((parts[0] + parts[1]) + parts[2]) ...) + parts[-1].

    ``parts`` is a sequence of contiguous fp32 CUDA tensors with one number of
    elements, or one tensor whose first axis indexes the partials (an
    all-gathered buffer).  Callers that pass the same partials in the same
    order get the same bits.  Returns ``out`` (shaped like one partial,
    allocated when None; it may be one of the partials).
    """
    lib = load_library()
    if isinstance(parts, torch.Tensor):
        parts = list(parts.unbind(0))
    parts = list(parts)
    if not parts:
        raise ValueError("sum_partials needs at least one partial")
    n = parts[0].numel()
    for t in parts:
        if t.dtype != torch.float32 or not t.is_contiguous() or t.numel() != n or t.device != parts[0].device:
            raise ValueError("partials must be contiguous fp32 tensors of one size on one device")
    if out is None:
        out = torch.empty_like(parts[0])
    if out.dtype != torch.float32 or not out.is_contiguous() or out.numel() != n:
        raise ValueError("out must be a contiguous fp32 tensor with as many elements as a partial")
    if n == 0:
        return out                                   # the empty sum: nothing to add
    arr = (ctypes.c_void_p * len(parts))(*[t.data_ptr() for t in parts])
    rc = lib.evo_sum_partials(len(parts), arr, n, _ptr(out), _stream(out.device))
    _check("evo_sum_partials", rc)
    return out


def opm_pair_view(out):
    """[B, N, Ca, N, Cb] outer-product-mean output as the pair layout [B, N, N, Ca, Cb] (a view)."""
    return out.permute(0, 1, 3, 2, 4)


def timing_enable(on: bool = True) -> None:
    """Switch the library's per-kernel event timing on or off."""
    _check("evo_attn_timing_enable", load_library().evo_attn_timing_enable(1 if on else 0))


def timing_collect() -> dict:
    """Wait for the recorded phases; {phase: (calls, total ms)} since the last collect."""
    t = Timing()
    _check("evo_attn_timing_collect", load_library().evo_attn_timing_collect(ctypes.byref(t)))
    return {name: (int(t.calls[i]), float(t.ms[i])) for i, name in enumerate(PHASES)}


def set_wait_limit_ns(ns: int) -> int:
    """Limit of the forward kernels' bounded waits from now on (nanoseconds); returns the previous one."""
    return int(load_library().evo_attn_set_wait_limit_ns(int(ns)))


def exp2_fma(x, y=None):
    """2^x for a contiguous fp32 CUDA tensor, by the kernels' FMA-pipe exponential."""
    if x.dtype != torch.float32 or not x.is_contiguous() or not x.is_cuda:
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    if y is None:
        y = torch.empty_like(x)
    _check("evo_exp2_fma", load_library().evo_exp2_fma(_ptr(x), _ptr(y), x.numel(), _stream(x.device)))
    return y


def device_status(clear: bool = True) -> int:
    """Synchronises and returns the library's device status (0 = EVO_OK, 5 = a wait timed out)."""
    return int(load_library().evo_attn_device_status(1 if clear else 0))


class EvoformerAttention(torch.autograd.Function):
    """autograd wrapper: out = sigmoid(g) * softmax(q k^T/sqrt(C) + mask_bias + pair_bias) v."""

    @staticmethod
    def forward(ctx, q, k, v, g, mask_bias, pair_bias):
        if q.dtype == torch.bfloat16:
            out, lse, out_lo = evo_attn_fwd(q, k, v, g, mask_bias, pair_bias, out_lo=True)
        else:
            (out, lse), out_lo = evo_attn_fwd(q, k, v, g, mask_bias, pair_bias), None
        ctx.save_for_backward(q, k, v, g, mask_bias, pair_bias, out, lse, out_lo)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, g, mask_bias, pair_bias, out, lse, out_lo = ctx.saved_tensors
        dout = dout if dout.stride() == out.stride() else empty_like_rows(out).copy_(dout)
        gr = evo_attn_bwd(q, k, v, g, mask_bias, pair_bias, out, lse, dout, out_lo=out_lo)
        dpb = None
        if pair_bias is not None and ctx.needs_input_grad[5]:
            dpb = gr["d_pair_bias"].to(pair_bias.dtype)
        return gr["dq"], gr["dk"], gr["dv"], gr["dg"], None, dpb


def evoformer_attention(q, k, v, g, mask_bias=None, pair_bias=None):
    return EvoformerAttention.apply(q, k, v, g, mask_bias, pair_bias)
