// evo_attn.cu -- C-ABI entry points, argument validation and launch layer.
//
// The whole library is one translation unit (it includes every kernel
// header), so the device status word and all kernels share one module.
//
// Call shapes handled here (all through strides, no copies):
//   MSA-row attention          rows s = MSA sequences
//   triangle, starting node    rows s = pair rows
//   triangle, ending node      transposed pair: s and n strides swapped
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "evo_attn.h"
#include "common.cuh"
#include "simt.cuh"
#include "sm100.cuh"
#include "tma_maps.cuh"
#include "timing.cuh"
#include "fwd_sm100.cuh"
#include "bwd_sm100.cuh"
#include "proj_sm100.cuh"
#include "trimul_sm100.cuh"
#include "partials.cuh"

#define EVO_VERSION 10000

namespace {

using evo::Strides;

std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_limit_ns{EVO_WAIT_LIMIT_NS};

// 2^x through the FMA-pipe exponential of the attention kernels, two values per call.
__global__ void exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
    for (int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n;
         i += 2 * (int64_t)gridDim.x * blockDim.x) {
        const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.0f;
        const uint64_t r = evo::sm100::exp2_poly2(evo::sm100::f2(a, b));
        y[i] = evo::sm100::f2lo(r);
        if (i + 1 < n) y[i + 1] = evo::sm100::f2hi(r);
    }
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

Strides to_strides(const evo_strides_t& s) { return Strides{s.b, s.s, s.n, s.h}; }

bool strides_ok(const evo_strides_t* s) {
    return s && s->b >= 0 && s->s >= 0 && s->n >= 0 && s->h >= 0;
}

bool strides_mult(const evo_strides_t* s, int64_t m) {
    return s->b % m == 0 && s->s % m == 0 && s->n % m == 0 && s->h % m == 0;
}

// Every element of a [B,S,N,H,C] view must be addressed at most once: the
// strides must not make two logical rows of the output overlap.  (Inputs may
// alias freely.)  Checked by sorting the four (extent, stride) pairs.
bool non_overlapping(const evo_shape_t& sh, const evo_strides_t& st) {
    struct D { int64_t n, s; };
    D d[5] = {{sh.B, st.b}, {sh.S, st.s}, {sh.N, st.n}, {sh.H, st.h}, {sh.C, 1}};
    std::sort(d, d + 5, [](const D& a, const D& b) { return a.s < b.s; });
    int64_t span = 1;  // elements covered by the inner dims so far
    for (auto& e : d) {
        if (e.n == 1) continue;
        if (e.s < span) return false;
        span = e.s * e.n;
    }
    return true;
}

evo_status_t check_shape(const evo_shape_t* sh) {
    if (!sh) return EVO_ERR_INVALID_ARG;
    if (sh->B < 0 || sh->S < 0 || sh->N < 0 || sh->H < 0 || sh->C < 1) return EVO_ERR_INVALID_ARG;
    if (sh->B > 65535 || sh->S > (1 << 30) || sh->N > (1 << 30) || sh->H > 65535) return EVO_ERR_UNSUPPORTED;
    if (sh->B * sh->H > 65535) return EVO_ERR_UNSUPPORTED;
    return EVO_OK;
}

bool empty_call(const evo_shape_t* sh) { return sh->B == 0 || sh->S == 0 || sh->N == 0 || sh->H == 0; }

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// ---------------------------------------------------------------- forward
evo_status_t fwd_f32(const evo_shape_t& sh, const void* q, const void* k, const void* v, const void* g,
                     const evo_strides_t& in, const void* mask, const void* bias, void* out,
                     const evo_strides_t& os, float* lse, cudaStream_t stream) {
    evo::simt::Args a{};
    a.B = (int)sh.B; a.S = (int)sh.S; a.N = (int)sh.N; a.H = (int)sh.H; a.C = (int)sh.C;
    a.q = q; a.k = k; a.v = v; a.g = g; a.in = to_strides(in);
    a.mask = mask; a.bias = bias; a.out_w = out; a.os = to_strides(os); a.lse = lse;
    dim3 grid((unsigned)((sh.N + evo::simt::kRowsPerCta - 1) / evo::simt::kRowsPerCta), (unsigned)sh.S,
              (unsigned)(sh.B * sh.H));
    {
        evo::timing::Scope t(EVO_PHASE_FWD_MAIN, stream);
        evo::simt::fwd_kernel<float><<<grid, evo::simt::kWarps * 32, 0, stream>>>(a);
    }
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

template <int NSUB, bool HM, bool HB>
evo_status_t launch_fwd_bf16(const CUtensorMap* maps, const evo::fwd::Params& p, cudaStream_t stream) {
    using L = evo::fwd::Layout<NSUB>;
    auto kern = evo::fwd::fwd_bf16_kernel<NSUB, HM, HB>;
    static cudaError_t attr = set_smem(kern, L::bytes);
    if (attr != cudaSuccess) return EVO_ERR_CUDA;
    // The kernel's setmaxnreg split assumes exactly L::launch_regs registers per
    // thread at launch; any other count could make the increase wait forever.
    static int regs = [&] {
        cudaFuncAttributes fa{};
        return cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : -1;
    }();
    if (regs != L::launch_regs) return EVO_ERR_UNSUPPORTED;
    const int grid = std::min(p.n_items, sm_count());
    {
        evo::timing::Scope t(EVO_PHASE_FWD_MAIN, stream);
        kern<<<grid, L::threads, L::bytes, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
    }
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

constexpr int kFwdNsub = 2;

evo_status_t fwd_bf16(const evo_shape_t& sh, const void* q, const void* k, const void* v, const void* g,
                      const evo_strides_t& in, const void* mask, const void* bias, void* out, void* out_lo,
                      const evo_strides_t& os, float* lse, cudaStream_t stream) {
    if (sh.C != evo::fwd::HD || sh.N % 8 != 0) return EVO_ERR_UNSUPPORTED;
    if (!strides_mult(&in, 8) || !strides_mult(&os, 8)) return EVO_ERR_UNSUPPORTED;
    for (const void* ptr : {q, k, v, g, (const void*)out}) if (!aligned(ptr, 16)) return EVO_ERR_UNSUPPORTED;
    if (out_lo && !aligned(out_lo, 16)) return EVO_ERR_UNSUPPORTED;
    if ((mask && !aligned(mask, 16)) || (bias && !aligned(bias, 16))) return EVO_ERR_UNSUPPORTED;
    const int64_t n_it = (sh.N + evo::fwd::BM - 1) / evo::fwd::BM;
    const int64_t n_sg = (sh.S + kFwdNsub - 1) / kFwdNsub;
    const int64_t n_items = sh.B * sh.H * n_sg * n_it;
    if (n_items > (int64_t)1 << 30) return EVO_ERR_UNSUPPORTED;
    CUtensorMap maps[6];
    std::memset(maps, 0, sizeof(maps));
    if (!evo::tma::rows_bf16(&maps[0], q, sh, in, evo::fwd::BM, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !evo::tma::rows_bf16(&maps[1], k, sh, in, evo::fwd::BN, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !evo::tma::rows_bf16(&maps[2], v, sh, in, evo::fwd::BN, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !evo::tma::rows_bf16(&maps[5], g, sh, in, evo::fwd::BM, CU_TENSOR_MAP_SWIZZLE_64B))
        return EVO_ERR_CUDA;
    if (bias && !evo::tma::square_bf16(&maps[3], bias, sh, evo::fwd::BM)) return EVO_ERR_CUDA;
    if (mask && !evo::tma::mask_bf16(&maps[4], mask, sh, 64)) return EVO_ERR_CUDA;
    evo::fwd::Params p{};
    p.B = (int)sh.B; p.S = (int)sh.S; p.N = (int)sh.N; p.H = (int)sh.H;
    p.n_kv = (int)((sh.N + evo::fwd::BN - 1) / evo::fwd::BN);
    p.n_it = (int)n_it;
    p.n_sg = (int)n_sg;
    p.n_items = (int)n_items;
    p.scale = 1.0f / sqrtf((float)sh.C);
    p.r_bf16 = __bfloat162float(__float2bfloat16_rn(sqrtf((float)sh.C)));
    p.r2_bf16 = __bfloat162float(__float2bfloat16_rn(sqrtf((float)sh.C) - p.r_bf16));
    p.g = static_cast<const __nv_bfloat16*>(g);
    p.in = to_strides(in);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.out_lo = static_cast<__nv_bfloat16*>(out_lo);
    p.os = to_strides(os);
    p.lse = lse;
    p.wait_ns = g_wait_limit_ns.load();
    if (mask && bias) return launch_fwd_bf16<kFwdNsub, true, true>(maps, p, stream);
    if (mask) return launch_fwd_bf16<kFwdNsub, true, false>(maps, p, stream);
    if (bias) return launch_fwd_bf16<kFwdNsub, false, true>(maps, p, stream);
    return launch_fwd_bf16<kFwdNsub, false, false>(maps, p, stream);
}

// ---------------------------------------------------------------- backward
struct BwdWorkspace {
    size_t d_off, nl_off, doa_off, dol_off, dqacc_off, biast_off, part_off, total;
    int groups, db_groups;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

BwdWorkspace bwd_workspace(const evo_shape_t& sh, evo_dtype_t dt) {
    BwdWorkspace w{};
    const size_t rows = (size_t)sh.B * sh.S * sh.H * sh.N;       // logit rows
    const size_t T = rows * (size_t)sh.C;                         // elements of a per-row tensor
    const size_t pair = (size_t)sh.B * sh.H * sh.N * sh.N;
    size_t off = 0;
    w.d_off = off;
    off = align256(off + rows * 4);
    if (dt == EVO_DTYPE_BF16) {
        // row terms -D and nl are stored with the query axis padded to whole tiles
        const size_t padded_rows = (size_t)sh.B * sh.S * sh.H * (size_t)((sh.N + 127) / 128 * 128);
        off = align256(w.d_off + padded_rows * 4);
        w.groups = evo::bwd::num_groups(sh.B, sh.S, sh.N, sh.H);
        // the d_pair_bias kernel's row groups, chosen for a 148-SM B200 (a pure function
        // of the shape, so that the workspace size never depends on the device)
        w.db_groups = evo::dbias::num_groups(sh.B, sh.S, sh.N, sh.H, 148);
        w.nl_off = off;
        off = align256(off + padded_rows * 4);
        w.doa_off = off;
        off = align256(off + T * 2);
        w.dol_off = off;
        off = align256(off + T * 2);
        w.dqacc_off = off;
        off = align256(off + T * 4);
        w.biast_off = off;
        off = align256(off + pair * 2);
        w.part_off = off;
        off = align256(off + pair * 4 * (size_t)(w.db_groups > 1 ? w.db_groups : 0));
    }
    w.total = off;
    return w;
}

evo_status_t bwd_f32(const evo_shape_t& sh, evo::simt::Args a, cudaStream_t stream) {
    (void)sh;
    const int64_t rows = (int64_t)a.B * a.S * a.N * a.H;
    evo::simt::bwd_pre_kernel<float><<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(a);
    const dim3 grid((unsigned)((a.N + evo::simt::kRowsPerCta - 1) / evo::simt::kRowsPerCta), (unsigned)a.S,
                    (unsigned)(a.B * a.H));
    evo::simt::bwd_dq_kernel<float><<<grid, evo::simt::kWarps * 32, 0, stream>>>(a);
    evo::simt::bwd_dkdv_kernel<float><<<grid, evo::simt::kWarps * 32, 0, stream>>>(a);
    const dim3 gb((unsigned)((a.N + 127) / 128), (unsigned)a.N, (unsigned)(a.B * a.H));
    evo::simt::bwd_dbias_kernel<float><<<gb, 128, 0, stream>>>(a);
    g_launches += 4;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

// ---------------------------------------------------------------- fused pre-attention projection
// maps[0]: w [c_in, n_out], boxes of 64 columns x 64 rows; maps[1]: y [rows, n_out] (pitch ldy),
// boxes of 64 columns x 32 rows.  Persistent grid: n_groups x (CTAs per group), at most one per SM.
template <int BNO, int CIN>
evo_status_t launch_ln_linear(const CUtensorMap* maps, const evo::proj::LnParams& p, cudaStream_t stream) {
    using L = evo::proj::PLayout<BNO, CIN>;
    auto kern = evo::proj::ln_linear_kernel<BNO, CIN>;
    static cudaError_t attr = set_smem(kern, L::bytes);
    if (attr != cudaSuccess) return EVO_ERR_CUDA;
    const int64_t nrb = (p.rows + evo::proj::BM - 1) / evo::proj::BM;
    // the widest column group whose w chunks stay resident; else all columns in one group
    const int nsl = p.n_out / BNO, kc = CIN / evo::proj::KBOX;
    int gsl = nsl;
    if (nsl * kc > L::NW) {
        for (int g = nsl; g >= 1; --g)
            if (nsl % g == 0 && g * kc <= L::NW) { gsl = g; break; }
    }
    evo::proj::LnParams q = p;
    q.gsl = gsl;
    const int64_t ngr = nsl / gsl;
    const int64_t grid = ngr * std::min<int64_t>(nrb, std::max<int64_t>(1, sm_count() / ngr));
    if (grid > 0x7fffffff) return EVO_ERR_UNSUPPORTED;
    {
        evo::timing::Scope t(EVO_PHASE_PROJ, stream);
        kern<<<(unsigned)grid, evo::proj::THREADS, L::bytes, stream>>>(maps[0], maps[1], q);
    }
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

template <int BNO>
evo_status_t launch_ln_linear_cin(const CUtensorMap* maps, const evo::proj::LnParams& p, cudaStream_t stream) {
    switch (p.c_in) {
        case 64: return launch_ln_linear<BNO, 64>(maps, p, stream);
        case 128: return launch_ln_linear<BNO, 128>(maps, p, stream);
        case 192: return launch_ln_linear<BNO, 192>(maps, p, stream);
        case 256: return launch_ln_linear<BNO, 256>(maps, p, stream);
    }
    return EVO_ERR_UNSUPPORTED;
}

template <int CPL, int LPR, int HQ>
evo_status_t launch_pair_bias(const evo::proj::PbParams& p, int64_t total, cudaStream_t stream) {
    auto kern = evo::proj::pair_bias_kernel<CPL, LPR, HQ>;
    static cudaError_t attr = set_smem(kern, evo::proj::PB_SMEM);
    if (attr != cudaSuccess) return EVO_ERR_CUDA;
    const int64_t blocks = (total + evo::proj::PB_ROWS - 1) / evo::proj::PB_ROWS;
    const size_t shm = (size_t)p.c_z * 4 * HQ * sizeof(float) + (size_t)4 * HQ * evo::proj::PB_ROWS * 2;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, evo::proj::PB_THREADS, shm) != cudaSuccess)
        return EVO_ERR_CUDA;
    const int grid = (int)std::min<int64_t>(blocks, (int64_t)sm_count() * std::max(per_sm, 1));
    {
        evo::timing::Scope t(EVO_PHASE_PAIR_BIAS, stream);
        kern<<<grid, evo::proj::PB_THREADS, shm, stream>>>(p);
    }
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

template <int HQ>
evo_status_t launch_pair_bias_rows(const evo::proj::PbParams& p, int64_t total, cudaStream_t stream) {
    auto kern = evo::proj::pair_bias_rows_kernel<HQ>;
    static cudaError_t attr = set_smem(kern, evo::proj::PBR_SMEM);
    if (attr != cudaSuccess) return EVO_ERR_CUDA;
    const int64_t ch = p.c_z / 8;
    const size_t shm = (size_t)evo::proj::PBR_THREADS * (ch | 1) * 16 + (size_t)p.c_z * 4 * HQ * 4 +
                       (size_t)(1 + evo::proj::PBR_THREADS / 32) * 4 * HQ * 4;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, evo::proj::PBR_THREADS, shm) != cudaSuccess)
        return EVO_ERR_CUDA;
    const int64_t blocks = (total + evo::proj::PBR_THREADS - 1) / evo::proj::PBR_THREADS;
    const int grid = (int)std::min<int64_t>(blocks, (int64_t)sm_count() * std::max(per_sm, 1));
    {
        evo::timing::Scope t(EVO_PHASE_PAIR_BIAS, stream);
        kern<<<grid, evo::proj::PBR_THREADS, shm, stream>>>(p);
    }
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

template <int CPL, int LPR>
evo_status_t launch_pair_bias_h(const evo::proj::PbParams& p, int64_t total, cudaStream_t stream) {
    switch ((p.H + 3) / 4) {
        case 1: return launch_pair_bias<CPL, LPR, 1>(p, total, stream);
        case 2: return launch_pair_bias<CPL, LPR, 2>(p, total, stream);
        case 3: return launch_pair_bias<CPL, LPR, 3>(p, total, stream);
        case 4: return launch_pair_bias<CPL, LPR, 4>(p, total, stream);
    }
    return EVO_ERR_UNSUPPORTED;
}

// z[m] (M x Nc) = scale * a[m]^T b[m] (incoming: a, b are K x M, K x Nc) or a[m] b[m]^T
// (outgoing: a, b are M x K, Nc x K) for the `batch` matrices m, on the tri_mul kernel.
evo_status_t launch_contraction(const void* a, const void* bb, void* z, int64_t M, int64_t Nc, int64_t K,
                                int64_t batch, bool incoming, float scale, int phase, cudaStream_t stream) {
    using namespace evo::trimul;
    CUtensorMap maps[3];
    std::memset(maps, 0, sizeof(maps));
    const bool ok = incoming ? (evo::tma::batch_bf16(&maps[0], a, M, K, batch, 64, 64) &&
                                evo::tma::batch_bf16(&maps[1], bb, Nc, K, batch, 64, 64))
                             : (evo::tma::batch_bf16(&maps[0], a, K, M, batch, 64, BM) &&
                                evo::tma::batch_bf16(&maps[1], bb, K, Nc, batch, 64, BN));
    if (!ok || !evo::tma::batch_bf16(&maps[2], z, Nc, M, batch, 64, 32)) return EVO_ERR_CUDA;
    TriParams p{};
    p.M = (int)M; p.Nc = (int)Nc; p.K = (int)K; p.BC = (int)batch; p.incoming = incoming ? 1 : 0; p.scale = scale;
    p.tiles_i = (int)((M + BM - 1) / BM); p.tiles_j = (int)((Nc + BN - 1) / BN);
    const int64_t tiles = batch * p.tiles_i * p.tiles_j;
    static cudaError_t attr = set_smem(tri_mul_kernel, TLayout::bytes);
    if (attr != cudaSuccess) return EVO_ERR_CUDA;
    const int grid = (int)std::min<int64_t>(tiles, sm_count());
    {
        evo::timing::Scope t(phase, stream);
        tri_mul_kernel<<<grid, THREADS, TLayout::bytes, stream>>>(maps[0], maps[1], maps[2], p);
    }
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* evo_status_string(evo_status_t s) {
    switch (s) {
        case EVO_OK: return "EVO_OK";
        case EVO_ERR_INVALID_ARG: return "EVO_ERR_INVALID_ARG";
        case EVO_ERR_UNSUPPORTED: return "EVO_ERR_UNSUPPORTED";
        case EVO_ERR_WORKSPACE_TOO_SMALL: return "EVO_ERR_WORKSPACE_TOO_SMALL";
        case EVO_ERR_CUDA: return "EVO_ERR_CUDA";
        case EVO_ERR_DEVICE_TIMEOUT: return "EVO_ERR_DEVICE_TIMEOUT";
    }
    return "EVO_ERR_UNKNOWN";
}

int evo_attn_version(void) { return EVO_VERSION; }

uint64_t evo_attn_set_wait_limit_ns(uint64_t ns) { return g_wait_limit_ns.exchange(ns); }

evo_status_t evo_exp2_fma(const float* x, float* y, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (!x || !y))) return EVO_ERR_INVALID_ARG;
    if (n == 0) return EVO_OK;
    if (!aligned(x, 4) || !aligned(y, 4)) return EVO_ERR_INVALID_ARG;
    const int blocks = (int)std::min<int64_t>((n + 511) / 512, 148 * 8);
    exp2_fma_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

uint64_t evo_attn_launch_count(void) { return g_launches.load(); }

evo_status_t evo_attn_timing_enable(int on) { return evo::timing::enable(on); }

evo_status_t evo_attn_timing_collect(evo_timing_t* out) { return evo::timing::collect(out); }

evo_status_t evo_attn_device_status(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return EVO_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_evo_status, sizeof(v)) != cudaSuccess) return EVO_ERR_CUDA;
    if (clear) {
        const unsigned int z = 0;
        if (cudaMemcpyToSymbol(g_evo_status, &z, sizeof(z)) != cudaSuccess) return EVO_ERR_CUDA;
    }
    return v == 0 ? EVO_OK : EVO_ERR_DEVICE_TIMEOUT;
}

size_t evo_attn_bwd_workspace_bytes(const evo_shape_t* shape, evo_dtype_t dtype) {
    if (check_shape(shape) != EVO_OK) return 0;
    if (dtype != EVO_DTYPE_BF16 && dtype != EVO_DTYPE_F32) return 0;
    return bwd_workspace(*shape, dtype).total;
}

evo_status_t evo_attn_fwd(const evo_shape_t* shape, evo_dtype_t dtype, const void* q, const void* k,
                          const void* v, const void* g, const evo_strides_t* in_str, const void* mask_bias,
                          const void* pair_bias, void* out, void* out_lo, const evo_strides_t* out_str, float* lse,
                          void* stream) {
    evo_status_t st = check_shape(shape);
    if (st != EVO_OK) return st;
    if (dtype != EVO_DTYPE_BF16 && dtype != EVO_DTYPE_F32) return EVO_ERR_INVALID_ARG;
    if (!strides_ok(in_str) || !strides_ok(out_str)) return EVO_ERR_INVALID_ARG;
    if (empty_call(shape)) return EVO_OK;
    if (!q || !k || !v || !g || !out || !lse) return EVO_ERR_INVALID_ARG;
    if (!non_overlapping(*shape, *out_str)) return EVO_ERR_INVALID_ARG;
    if (!aligned(lse, 4)) return EVO_ERR_INVALID_ARG;
    if (out_lo && out_lo == out) return EVO_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == EVO_DTYPE_F32) {
        if (shape->C > evo::simt::kMaxC) return EVO_ERR_UNSUPPORTED;
        for (const void* p : {q, k, v, g, (const void*)out})
            if (!aligned(p, 4)) return EVO_ERR_INVALID_ARG;
        if (shape->S > 65535) return EVO_ERR_UNSUPPORTED;
        return fwd_f32(*shape, q, k, v, g, *in_str, mask_bias, pair_bias, out, *out_str, lse, s);
    }
    return fwd_bf16(*shape, q, k, v, g, *in_str, mask_bias, pair_bias, out, out_lo, *out_str, lse, s);
}

evo_status_t evo_attn_bwd(const evo_shape_t* shape, evo_dtype_t dtype, const void* q, const void* k,
                          const void* v, const void* g, const evo_strides_t* in_str, const void* mask_bias,
                          const void* pair_bias, const void* out, const void* out_lo, const void* dout,
                          const evo_strides_t* out_str, const float* lse, void* dq, void* dk, void* dv,
                          void* dg, const evo_strides_t* grad_str, float* d_pair_bias, void* workspace,
                          size_t workspace_bytes, void* stream) {
    evo_status_t st = check_shape(shape);
    if (st != EVO_OK) return st;
    if (dtype != EVO_DTYPE_BF16 && dtype != EVO_DTYPE_F32) return EVO_ERR_INVALID_ARG;
    if (!strides_ok(in_str) || !strides_ok(out_str) || !strides_ok(grad_str)) return EVO_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (shape->B == 0 || shape->H == 0 || shape->N == 0) return EVO_OK;
    if (!d_pair_bias || !aligned(d_pair_bias, 4)) return EVO_ERR_INVALID_ARG;
    const size_t pair_bytes = (size_t)shape->B * shape->H * shape->N * shape->N * sizeof(float);
    if (shape->S == 0) {
        return cudaMemsetAsync(d_pair_bias, 0, pair_bytes, s) == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
    }
    if (!q || !k || !v || !g || !out || !dout || !lse || !dq || !dk || !dv || !dg) return EVO_ERR_INVALID_ARG;
    if (!non_overlapping(*shape, *grad_str)) return EVO_ERR_INVALID_ARG;
    const BwdWorkspace ws = bwd_workspace(*shape, dtype);
    if (ws.total > 0 && (!workspace || workspace_bytes < ws.total)) return EVO_ERR_WORKSPACE_TOO_SMALL;
    if (workspace && !aligned(workspace, 256)) return EVO_ERR_INVALID_ARG;
    if (!aligned(lse, 4)) return EVO_ERR_INVALID_ARG;

    evo::simt::Args a{};
    a.B = (int)shape->B; a.S = (int)shape->S; a.N = (int)shape->N; a.H = (int)shape->H; a.C = (int)shape->C;
    a.q = q; a.k = k; a.v = v; a.g = g; a.in = to_strides(*in_str);
    a.mask = mask_bias; a.bias = pair_bias; a.out = out; a.dout = dout; a.os = to_strides(*out_str);
    a.lse = const_cast<float*>(lse);
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.gs = to_strides(*grad_str);
    a.dbias = d_pair_bias;
    a.D = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws.d_off);
    if (dtype == EVO_DTYPE_F32) {
        if (shape->C > evo::simt::kMaxC) return EVO_ERR_UNSUPPORTED;
        for (const void* p : {q, k, v, g, out, dout, (const void*)dq, (const void*)dk, (const void*)dv,
                              (const void*)dg})
            if (!aligned(p, 4)) return EVO_ERR_INVALID_ARG;
        if (shape->S > 65535 || shape->N > 65535) return EVO_ERR_UNSUPPORTED;
        evo::timing::Scope t(EVO_PHASE_BWD_ALL, s);
        return bwd_f32(*shape, a, s);
    }
    evo::bwd::Call c{};
    c.shape = *shape;
    c.q = q; c.k = k; c.v = v; c.g = g; c.in = *in_str;
    c.mask = mask_bias; c.bias = pair_bias; c.out = out; c.out_lo = out_lo; c.dout = dout; c.os = *out_str;
    c.lse = lse;
    c.dq = dq; c.dk = dk; c.dv = dv; c.dg = dg; c.gs = *grad_str; c.dbias = d_pair_bias;
    c.ws = static_cast<char*>(workspace);
    c.d_off = ws.d_off; c.nl_off = ws.nl_off; c.doa_off = ws.doa_off; c.dol_off = ws.dol_off;
    c.dqacc_off = ws.dqacc_off;
    c.biast_off = ws.biast_off; c.part_off = ws.part_off; c.groups = ws.groups; c.db_groups = ws.db_groups;
    c.wait_ns = g_wait_limit_ns.load();
    int launched = 0;
    evo_status_t rs;
    {
        evo::timing::Scope t(EVO_PHASE_BWD_ALL, s);
        rs = evo::bwd::run(c, s, &launched);
    }
    g_launches += (uint64_t)launched;
    return rs;
}

// ---------------------------------------------------------------- no-allocation backward
// Scratch area of evo_attn_bwd_noalloc.  Host code must not pass the array's
// name to a kernel: on the host it is only a stand-in for the device object,
// whose address is looked up once per device below.
static __device__ __align__(256) unsigned char g_evo_noalloc_ws[EVO_ATTN_NOALLOC_WORKSPACE_BYTES];

static std::mutex g_noalloc_mu;
struct NoallocSlot {
    unsigned long long ctx_id;   // the context the address belongs to (0: none yet)
    void* addr;
};
static NoallocSlot g_noalloc_slot[256] = {};

// Identifier of the calling thread's current context, unique among the
// contexts this process creates (cuCtxGetId), or 0 when it cannot be had.  A
// context created after cudaDeviceReset gets a new identifier, so an address
// cached for the old context is never reused.
static unsigned long long current_ctx_id() {
    static std::once_flag once;
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array in the current device's context.  It
// is looked up (cudaGetSymbolAddress, with that device current) on the first
// call in each context and cached; a later call in the same context reuses
// it, a call in a new context (after cudaDeviceReset) looks it up again.
// Without a context identifier it is looked up on every call.
static evo_status_t noalloc_workspace(void** addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return EVO_ERR_CUDA;
    if (dev < 0 || dev >= 256) return EVO_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    unsigned long long id = current_ctx_id();
    NoallocSlot& slot = g_noalloc_slot[dev];
    if (id == 0 || slot.ctx_id != id || !slot.addr) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_evo_noalloc_ws) != cudaSuccess || !a) return EVO_ERR_CUDA;
        if (id == 0) id = current_ctx_id();      // the lookup may have made the context current
        slot.ctx_id = id;
        slot.addr = a;
    }
    *addr = slot.addr;
    return EVO_OK;
}

evo_status_t evo_ln_linear(int64_t rows, int64_t c_in, int64_t n_out, const void* x, const float* ln_w,
                           const float* ln_b, float eps, const void* w, const float* bias, void* y, int64_t ldy,
                           void* stream) {
    if (rows < 0 || c_in <= 0 || n_out <= 0 || ldy < n_out || !(eps >= 0.f)) return EVO_ERR_INVALID_ARG;
    if (rows == 0) return EVO_OK;
    if (!x || !w || !y) return EVO_ERR_INVALID_ARG;
    if (c_in % evo::proj::KBOX != 0 || c_in > evo::proj::MAX_CIN || n_out % 128 != 0 || ldy % 8 != 0)
        return EVO_ERR_UNSUPPORTED;
    if (rows > (int64_t)0x7fffffff - evo::proj::BM || n_out > (int64_t)0x7fffffff) return EVO_ERR_UNSUPPORTED;
    for (const void* q : {x, w, (const void*)y})
        if (!aligned(q, 16)) return EVO_ERR_UNSUPPORTED;
    if (bias && !aligned(bias, 16)) return EVO_ERR_UNSUPPORTED;      // read as float4
    for (const void* q : {(const void*)ln_w, (const void*)ln_b})
        if (q && !aligned(q, 4)) return EVO_ERR_INVALID_ARG;
    CUtensorMap maps[2];
    std::memset(maps, 0, sizeof(maps));
    if (!evo::tma::matrix_bf16(&maps[0], w, c_in, n_out, n_out, 64) ||
        !evo::tma::matrix_bf16(&maps[1], y, rows, n_out, ldy, 32))
        return EVO_ERR_CUDA;
    evo::proj::LnParams p{};
    p.rows = (int)rows; p.c_in = (int)c_in; p.n_out = (int)n_out; p.eps = eps;
    p.x = static_cast<const __nv_bfloat16*>(x); p.ln_w = ln_w; p.ln_b = ln_b; p.bias = bias;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return n_out % 256 == 0 ? launch_ln_linear_cin<256>(maps, p, s) : launch_ln_linear_cin<128>(maps, p, s);
}

evo_status_t evo_ln_pair_bias(int64_t B, int64_t N, int64_t c_z, int64_t H, const void* z, const float* ln_w,
                              const float* ln_b, float eps, const void* w, const float* bias, void* pair_bias,
                              void* stream) {
    if (B < 0 || N < 0 || c_z <= 0 || H <= 0 || !(eps >= 0.f)) return EVO_ERR_INVALID_ARG;
    if (B == 0 || N == 0) return EVO_OK;
    if (!z || !w || !pair_bias) return EVO_ERR_INVALID_ARG;
    if (c_z % 8 != 0 || c_z > 1024 || H > evo::proj::PB_MAX_H) return EVO_ERR_UNSUPPORTED;
    if (!aligned(z, 16) || !aligned(w, 2) || !aligned(pair_bias, 2)) return EVO_ERR_UNSUPPORTED;
    evo::proj::PbParams p{};
    p.B = (int)B; p.N = (int)N; p.c_z = (int)c_z; p.H = (int)H; p.eps = eps;
    p.z = static_cast<const __nv_bfloat16*>(z); p.ln_w = ln_w; p.ln_b = ln_b;
    p.w = static_cast<const __nv_bfloat16*>(w); p.bias = bias;
    p.out = static_cast<__nv_bfloat16*>(pair_bias);
    const int64_t total = B * N * N;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t chunks = c_z / 8;
    if (c_z <= evo::proj::PBR_MAX_CZ) {
        switch ((H + 3) / 4) {
            case 1: return launch_pair_bias_rows<1>(p, total, s);
            case 2: return launch_pair_bias_rows<2>(p, total, s);
            case 3: return launch_pair_bias_rows<3>(p, total, s);
            default: return launch_pair_bias_rows<4>(p, total, s);
        }
    }
    if (chunks > 64) return launch_pair_bias_h<4, 32>(p, total, s);
    if (chunks > 32) return launch_pair_bias_h<2, 32>(p, total, s);
    if (chunks > 16) return launch_pair_bias_h<1, 32>(p, total, s);
    if (chunks > 8) return launch_pair_bias_h<1, 16>(p, total, s);
    if (chunks > 4) return launch_pair_bias_h<1, 8>(p, total, s);
    if (chunks > 2) return launch_pair_bias_h<1, 4>(p, total, s);
    return launch_pair_bias_h<1, 2>(p, total, s);    // at least 2 lanes per row: 16 rows per warp step
}

evo_status_t evo_tri_mul(int64_t B, int64_t C, int64_t N, const void* a, const void* bb, int incoming,
                         void* z, void* stream) {
    if (B < 0 || C < 0 || N < 0) return EVO_ERR_INVALID_ARG;
    if (B == 0 || C == 0 || N == 0) return EVO_OK;
    if (!a || !bb || !z) return EVO_ERR_INVALID_ARG;
    const int64_t BC = B * C;
    if (N % 8 != 0 || BC > (int64_t)0x7fffffff || N > (int64_t)0x7fffffff / 2) return EVO_ERR_UNSUPPORTED;
    for (const void* q : {a, bb, (const void*)z})
        if (!aligned(q, 16)) return EVO_ERR_UNSUPPORTED;
    const bool in = incoming != 0;
    return launch_contraction(a, bb, z, N, N, N, BC, in, 1.f, EVO_PHASE_TRI_MUL, static_cast<cudaStream_t>(stream));
}

evo_status_t evo_outer_product_mean(int64_t B, int64_t S, int64_t N, int64_t Ca, int64_t Cb, const void* a,
                                    const void* bb, void* out, void* stream) {
    if (B < 0 || S < 0 || N < 0 || Ca <= 0 || Cb <= 0) return EVO_ERR_INVALID_ARG;
    if (B == 0 || N == 0) return EVO_OK;
    if (S == 0 || !a || !bb || !out) return EVO_ERR_INVALID_ARG;
    const int64_t M = N * Ca, Nc = N * Cb;
    if (M % 8 != 0 || Nc % 8 != 0 || M > (int64_t)0x7fffffff / 2 || Nc > (int64_t)0x7fffffff / 2 ||
        S > (int64_t)0x7fffffff || B > (int64_t)0x7fffffff)
        return EVO_ERR_UNSUPPORTED;
    for (const void* q : {a, bb, (const void*)out})
        if (!aligned(q, 16)) return EVO_ERR_UNSUPPORTED;
    // out[b, (i, c1), (j, c2)] = (1/S) sum_s a[b, s, (i, c1)] bb[b, s, (j, c2)]: the MN-major contraction
    return launch_contraction(a, bb, out, M, Nc, S, B, true, (float)(1.0 / (double)S), EVO_PHASE_OPM,
                              static_cast<cudaStream_t>(stream));
}

evo_status_t evo_sum_partials(int64_t count, const float* const* parts, int64_t n, float* out, void* stream) {
    static_assert(EVO_MAX_PARTIALS == evo::partials::MAX_PARTS, "partials limit");
    if (count < 1 || n < 0 || !parts || !out) return EVO_ERR_INVALID_ARG;
    if (count > EVO_MAX_PARTIALS) return EVO_ERR_UNSUPPORTED;
    evo::partials::Params p{};
    bool vec = aligned(out, 16);
    for (int64_t r = 0; r < count; ++r) {
        if (!parts[r]) return EVO_ERR_INVALID_ARG;
        if (!aligned(parts[r], 4)) return EVO_ERR_UNSUPPORTED;
        vec = vec && aligned(parts[r], 16);
        p.part[r] = parts[r];
    }
    if (!aligned(out, 4)) return EVO_ERR_UNSUPPORTED;
    if (n == 0) return EVO_OK;
    p.out = out;
    p.n = n;
    p.count = (int)count;
    p.vec = vec ? 1 : 0;
    const int64_t items = vec ? n / 4 + n % 4 : n;
    const int blocks = (int)std::min<int64_t>((items + 255) / 256, 148 * 8);
    evo::partials::sum_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    g_launches += 1;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

evo_status_t evo_attn_bwd_noalloc(const evo_shape_t* shape, evo_dtype_t dtype, const void* q, const void* k,
                                  const void* v, const void* g, const evo_strides_t* in_str, const void* mask_bias,
                                  const void* pair_bias, const void* out, const void* out_lo, const void* dout,
                                  const evo_strides_t* out_str, const float* lse, void* dq, void* dk, void* dv,
                                  void* dg, const evo_strides_t* grad_str, float* d_pair_bias, void* stream) {
    const evo_status_t st = check_shape(shape);
    if (st != EVO_OK) return st;
    if (dtype != EVO_DTYPE_BF16 && dtype != EVO_DTYPE_F32) return EVO_ERR_INVALID_ARG;
    if (evo_attn_bwd_workspace_bytes(shape, dtype) > EVO_ATTN_NOALLOC_WORKSPACE_BYTES)
        return EVO_ERR_WORKSPACE_TOO_SMALL;
    void* ws = nullptr;
    const evo_status_t wst = noalloc_workspace(&ws);
    if (wst != EVO_OK) return wst;
    return evo_attn_bwd(shape, dtype, q, k, v, g, in_str, mask_bias, pair_bias, out, out_lo, dout, out_str, lse,
                        dq, dk, dv, dg, grad_str, d_pair_bias, ws, EVO_ATTN_NOALLOC_WORKSPACE_BYTES, stream);
}

}  // extern "C"
