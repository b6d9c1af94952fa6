// proj_sm100.cuh -- fused pre-attention projection on sm_100a:
//   y = LayerNorm(x) @ w + bias
// over the rows of the MSA or pair representation, without writing the
// normalised tensor to memory: the LayerNorm + linear pair that the MegaFold
// summary's EvoFusion section fuses ("EvoFusion : Pile d'Operateurs
// Fusionnes").  With w = [w_q | w_k | w_v | w_g] the four column blocks of y
// are q, k, v and g in the attention's [B, S, N, H, c] layout (row stride
// 4*H*c, which the attention kernels take as strides); with one output per
// head over the pair representation, y is the pair bias.
//
// ln_linear_kernel (tensor cores), persistent, one CTA per SM.  The n_out
// columns are cut into slices of BNO; CTA c keeps slice c % n_slices of w
// resident in shared memory (loaded once by TMA, an MN-major B operand) and
// walks the 128-row blocks rb = c / n_slices, + grid / n_slices, ...  Roles:
//   warp 0      one thread loads w and issues the MMAs (M = 128, N = BNO,
//               K = 16) of row block j into TMEM accumulator j % 2;
//   warps 1-4   epilogue: TMEM -> + bias -> bf16 -> shared staging (128B
//               swizzle) -> TMA store, 32 rows x 64 columns per store;
//   warps 5-12  LayerNorm: coalesced 16-byte loads of x rows from global
//               memory (a row's c_in channels spread over up to 32 lanes),
//               fp32 statistics by warp shuffles, normalised bf16 written
//               into the A tile (K-major, 128B swizzle) the MMA reads.
// The A tile is double-buffered when shared memory allows it; otherwise
// (c_in = 256 with 256-column slices) its two K halves have their own
// full/empty barriers, so the LayerNorm warps refill one half while the
// MMAs still read the other.  Every wait is bounded; on expiry the CTA
// records a status code and winds down.
//
// pair_bias_kernel (SIMT, H <= 16 outputs per row): block = 8 warps, 128
// consecutive pair rows (b, i, j) per step; a row's c_z channels spread over
// up to 32 lanes (16-byte loads), LayerNorm and the H dot products reduced by
// warp shuffles, outputs staged per head so that out[b, h, i, j] is written
// in runs of consecutive j.
#pragma once

#include "sm100.cuh"
#include "tma_maps.cuh"

namespace evo {
namespace proj {

using namespace evo::sm100;

constexpr int BM = 128;
constexpr int KBOX = 64;                       // K elements per 128-byte swizzled box
constexpr int MAX_CIN = 256;
constexpr int LN_WARPS = 8;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 32 * (1 + EPI_WARPS + LN_WARPS);
constexpr int STG_TILE = 32 * 128;             // 32 rows x 64 bf16 columns
constexpr int STG_BYTES = EPI_WARPS * 2 * STG_TILE;
constexpr int SMEM_LIMIT = 232448;             // opt-in dynamic shared memory per CTA
constexpr int SMEM_MIN = 120 * 1024;           // > half an SM: one CTA (and one TMEM owner) per SM

template <int BNO, int CIN>
struct PLayout {
    static constexpr int w_bytes = BNO / 64 * CIN * 128;          // BNO/64 boxes of CIN rows x 128 B
    static constexpr int a_bytes = CIN / KBOX * BM * 128;         // CIN/64 boxes of 128 rows x 128 B
    static constexpr int fixed = STG_BYTES + BNO * 4 + 256;
    static constexpr int NA = (w_bytes + 2 * a_bytes + fixed + 1024 <= SMEM_LIMIT) ? 2 : 1;
    static constexpr int KS = NA == 1 ? 2 : 1;                    // K parts with their own barriers
    static constexpr int a_off = w_bytes;
    static constexpr int stg_off = a_off + NA * a_bytes;
    static constexpr int bias_off = stg_off + STG_BYTES;
    static constexpr int bar_off = bias_off + BNO * 4;
    // w_full, a_full[NA*KS], a_empty[NA*KS], acc_full[2], acc_empty[2], done
    static constexpr int n_bars = 1 + 2 * NA * KS + 4 + 1;
    static constexpr int misc_off = bar_off + n_bars * 8;         // TMEM slot, abort flag
    static constexpr int used = misc_off + 16;
    static constexpr int bytes = used + 1024 > SMEM_MIN ? used + 1024 : SMEM_MIN;
    static_assert(used + 1024 <= SMEM_LIMIT, "shared memory budget");
    static_assert(KS == 1 || (CIN / KBOX) % 2 == 0, "K halves must be whole boxes");
};

struct LnParams {
    int rows, c_in, n_out;
    float eps;
    const __nv_bfloat16* x;   // [rows, c_in], rows contiguous
    const float* ln_w;        // [c_in] or null (ones)
    const float* ln_b;        // [c_in] or null (zeros)
    const float* bias;        // [n_out] or null (zeros)
};

enum : unsigned int { kTimeoutBase = 0x3000u };

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = bf16lo(w4[e]);
        f[2 * e + 1] = bf16hi(w4[e]);
    }
}

// Registers are granted per group of four warps, so the 13 warps count as 16:
// 128 registers a thread at most.
template <int BNO, int CIN>
__global__ void __launch_bounds__(THREADS, 1)
    ln_linear_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_y,
                     const LnParams p) {
    using L = PLayout<BNO, CIN>;
    constexpr int NA = L::NA, KS = L::KS, NB = CIN / KBOX, KSTEPS = CIN / 16;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nsl = p.n_out / BNO;
    const int n0 = (int)(blockIdx.x % nsl) * BNO;
    const int rb_first = (int)(blockIdx.x / nsl), rb_step = (int)(gridDim.x / nsl);
    const int nrb = (p.rows + BM - 1) / BM;
    const uint32_t bar_w = base + L::bar_off;
    auto bar_afull = [&](int i) { return base + L::bar_off + 8u * (1 + i); };
    auto bar_aempty = [&](int i) { return base + L::bar_off + 8u * (1 + NA * KS + i); };
    auto bar_accf = [&](int b) { return base + L::bar_off + 8u * (1 + 2 * NA * KS + b); };
    auto bar_acce = [&](int b) { return base + L::bar_off + 8u * (3 + 2 * NA * KS + b); };
    const uint32_t bar_done = base + L::bar_off + 8u * (5 + 2 * NA * KS);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + L::misc_off);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::misc_off + 4);
    float* bias_s = reinterpret_cast<float*>(gbase + L::bias_off);

    if (threadIdx.x == 0) {
        mbar_init(bar_w, 1);
        for (int i = 0; i < NA * KS; ++i) {
            mbar_init(bar_afull(i), LN_WARPS);
            mbar_init(bar_aempty(i), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_accf(b), 1);
            mbar_init(bar_acce(b), EPI_WARPS);
        }
        mbar_init(bar_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < BNO; i += THREADS) bias_s[i] = p.bias ? __ldg(p.bias + n0 + i) : 0.f;
    if (warp == 0) {
        tmem_alloc(base + L::misc_off, 2 * BNO);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ w slice + MMA issue
        if (lane == 0) {
            prefetch_tmap(&tm_w);
            mbar_arrive_expect_tx(bar_w, (uint32_t)L::w_bytes);
            for (int nb = 0; nb < BNO / 64; ++nb) tma_load_2d(base + nb * CIN * 128, &tm_w, bar_w, n0 + nb * 64, 0);
            const bool w_ok = mbar_wait(bar_w, 0, abort_flag, kTimeoutBase | 0x01);
            bool ok = w_ok;
            constexpr uint32_t IDESC = idesc_bf16(BM, BNO, false, true);   // B operand MN-major
            int j = 0;
            for (int rb = rb_first; ok && rb < nrb; rb += rb_step, ++j) {
                const int s = j % NA, n = j / NA, buf = j & 1, m = j >> 1;
                ok = mbar_wait(bar_acce(buf), (m & 1) ^ 1, abort_flag, kTimeoutBase | 0x02);
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * BNO);
                const uint32_t a_base = base + L::a_off + s * L::a_bytes;
                for (int part = 0; ok && part < KS; ++part) {
                    ok = mbar_wait(bar_afull(s * KS + part), n & 1, abort_flag, kTimeoutBase | 0x03);
                    if (!ok) break;
                    tc_fence_after();
                    for (int kk = part * KSTEPS / KS; kk < (part + 1) * KSTEPS / KS; ++kk) {
                        const uint64_t ad = smem_desc(a_base + (kk >> 2) * BM * 128 + (kk & 3) * 32, 16, 1024, kSw128);
                        const uint64_t bd = smem_desc(base + kk * 2048, CIN * 128, 1024, kSw128);
                        mma_ss(d, ad, bd, IDESC, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar_aempty(s * KS + part));
                }
                if (ok) mma_commit(bar_accf(buf));
            }
            // every MMA issued above, and the w load, complete before TMEM and
            // shared memory are released
            volatile int no_abort = 0;
            mma_commit(bar_done);
            mbar_wait(bar_done, 0, &no_abort, kTimeoutBase | 0x04);
            if (!w_ok) mbar_wait(bar_w, 0, &no_abort, kTimeoutBase | 0x05);
        }
    } else if (warp <= EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                        // the TMEM lane quarter this warp may read
        const uint32_t stg = base + L::stg_off + (uint32_t)((warp - 1) * 2 * STG_TILE);
        if (lane == 0) prefetch_tmap(&tm_y);
        int j = 0;
        for (int rb = rb_first; rb < nrb; rb += rb_step, ++j) {
            const int buf = j & 1, m = j >> 1;
            const bool ok = mbar_wait(bar_accf(buf), m & 1, abort_flag, kTimeoutBase | 0x06);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int row0 = rb * BM + 32 * q;
            const uint32_t taddr = tmem + (uint32_t)(buf * BNO) + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
            for (int g = 0; g < BNO / 64; ++g) {
                uint32_t v[64];
                tmem_ld32x2_sync(taddr + 64 * g, taddr + 64 * g + 32, v);
                const uint32_t sb = stg + (uint32_t)((g & 1) * STG_TILE);
                if (lane == 0) bulk_wait_read<1>();    // the store that last read this buffer is done with it
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 b0 = *reinterpret_cast<const float4*>(bias_s + 64 * g + 8 * c);
                    const float4 b1 = *reinterpret_cast<const float4*>(bias_s + 64 * g + 8 * c + 4);
                    const uint32_t* vc = v + 8 * c;
                    sts128(sb + lane * 128 + ((c ^ (lane & 7)) << 4),
                           pack_bf16(__uint_as_float(vc[0]) + b0.x, __uint_as_float(vc[1]) + b0.y),
                           pack_bf16(__uint_as_float(vc[2]) + b0.z, __uint_as_float(vc[3]) + b0.w),
                           pack_bf16(__uint_as_float(vc[4]) + b1.x, __uint_as_float(vc[5]) + b1.y),
                           pack_bf16(__uint_as_float(vc[6]) + b1.z, __uint_as_float(vc[7]) + b1.w));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && row0 < p.rows) {     // rows past the end are clipped by the tensor map
                    tma_store_2d(&tm_y, sb, n0 + 64 * g, row0);
                    bulk_commit();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_acce(buf));
        }
        if (lane == 0) bulk_wait<0>();
    } else {
        // ----------------------------------------------------------- LayerNorm
        constexpr int CH = CIN / 8;                    // 16-byte chunks per row
        constexpr int LPR = CH == 24 ? 32 : CH;        // lanes per row
        constexpr int RPI = 32 / LPR;                  // rows per warp-wide load
        constexpr int ROWS_W = BM / LN_WARPS;          // rows of a block per warp
        constexpr int ITERS = ROWS_W / RPI;
        static_assert(32 % LPR == 0 && ROWS_W % RPI == 0, "lane mapping");
        const int lw = warp - 1 - EPI_WARPS;
        const int cidx = lane % LPR, sub = lane / LPR;
        const bool active = cidx < CH;
        const int kb = cidx >> 3, cc = cidx & 7;
        const int mypart = KS == 2 ? (kb >= NB / 2 ? 1 : 0) : 0;
        float gw[8], gb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int k = cidx * 8 + e;
            gw[e] = (active && p.ln_w) ? __ldg(p.ln_w + k) : 1.f;
            gb[e] = (active && p.ln_b) ? __ldg(p.ln_b + k) : 0.f;
        }
        const uint4* xg = reinterpret_cast<const uint4*>(p.x);
        const float inv_c = 1.f / (float)CIN;
        int j = 0;
        for (int rb = rb_first; rb < nrb; rb += rb_step, ++j) {
            const int s = j % NA, n = j / NA;
            uint4 xv[ITERS];
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                const int r = rb * BM + lw * ROWS_W + it * RPI + sub;
                xv[it] = (active && r < p.rows) ? __ldg(xg + (int64_t)r * CH + cidx) : make_uint4(0, 0, 0, 0);
            }
            // the next block's rows into L2 while this one is normalised
            const int rb_next = rb + rb_step;
            if (rb_next < nrb && active && (cidx & 7) == 0) {
#pragma unroll
                for (int it = 0; it < ITERS; ++it) {
                    const int r = rb_next * BM + lw * ROWS_W + it * RPI + sub;
                    if (r < p.rows) prefetch_l2(xg + (int64_t)r * CH + cidx);
                }
            }
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                float f[8];
                unpack8(xv[it], f);
                float sum = ((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]));
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                const float mean = sum * inv_c;
                float sq = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float dlt = f[e] - mean;
                    sq = fmaf(dlt, dlt, sq);
                }
                if (!active) sq = 0.f;
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
                const float rstd = rsqrtf(sq * inv_c + p.eps);
                uint32_t o4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o4[e] = pack_bf16(fmaf((f[2 * e] - mean) * rstd, gw[2 * e], gb[2 * e]),
                                      fmaf((f[2 * e + 1] - mean) * rstd, gw[2 * e + 1], gb[2 * e + 1]));
                xv[it] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
            }
            const uint32_t a_base = base + L::a_off + s * L::a_bytes;
            bool ok = true;
#pragma unroll
            for (int part = 0; part < KS; ++part) {
                ok = mbar_wait(bar_aempty(s * KS + part), (n & 1) ^ 1, abort_flag, kTimeoutBase | 0x07);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                if (active && mypart == part) {
#pragma unroll
                    for (int it = 0; it < ITERS; ++it) {
                        const int rr = lw * ROWS_W + it * RPI + sub;
                        sts128(a_base + kb * BM * 128 + rr * 128 + ((cc ^ (rr & 7)) << 4), xv[it].x, xv[it].y,
                               xv[it].z, xv[it].w);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_afull(s * KS + part));
            }
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 2 * BNO);
    }
}

// ---------------------------------------------------------------- pair bias
struct PbParams {
    int B, N, c_z, H;
    float eps;
    const __nv_bfloat16* z;   // [B, N, N, c_z]
    const float* ln_w;        // [c_z] or null
    const float* ln_b;        // [c_z] or null
    const __nv_bfloat16* w;   // [c_z, H]
    const float* bias;        // [H] or null
    __nv_bfloat16* out;       // [B, H, N, N]
};
constexpr int PB_MAX_H = 16;
constexpr int PB_MAX_CZ = 1024;
constexpr int PB_ROWS = 128;                   // pair rows per block step
constexpr int PB_THREADS = 256;
constexpr int PB_SMEM = PB_MAX_CZ * PB_MAX_H * 4 + PB_MAX_H * PB_ROWS * 2;   // w (fp32, heads padded to 4) + outputs

// CPL = 16-byte chunks per lane (chunk c = lane % LPR + LPR * t), LPR = lanes
// per row, HQ = heads / 4 rounded up (the head loops are unrolled exactly).
template <int CPL, int LPR, int HQ>
__global__ void __launch_bounds__(PB_THREADS) pair_bias_kernel(const PbParams p) {
    constexpr int HP = 4 * HQ;
    extern __shared__ float pb_smem[];
    const int H = p.H;
    const int ch = p.c_z / 8;
    // w[k][h] at ((k % 8) * ch + k / 8) * HP + h: for a fixed k % 8 the lanes of a
    // row, which hold consecutive chunks k / 8, read consecutive 16-byte words
    float* wsh = pb_smem;
    __nv_bfloat16* osh = reinterpret_cast<__nv_bfloat16*>(pb_smem + p.c_z * HP);   // [HP][PB_ROWS]
    for (int o = threadIdx.x; o < p.c_z * HP; o += PB_THREADS) {
        const int k = o / HP, h = o - k * HP;
        wsh[((k & 7) * ch + (k >> 3)) * HP + h] = h < H ? __bfloat162float(p.w[k * H + h]) : 0.f;
    }
    constexpr int RPI = 32 / LPR;
    constexpr int ROWS_W = PB_ROWS / (PB_THREADS / 32);
    constexpr int ITERS = ROWS_W / RPI;
    constexpr int BATCH = (8 / CPL) < ITERS ? (8 / CPL) : ITERS;
    static_assert(ITERS % BATCH == 0, "batching");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cl = lane % LPR, sub = lane / LPR;
    const int64_t nn = (int64_t)p.N * p.N, total = (int64_t)p.B * nn;
    const float inv_c = 1.f / (float)p.c_z;
    const uint4* zg = reinterpret_cast<const uint4*>(p.z);
    float gw[CPL * 8], gb[CPL * 8];
#pragma unroll
    for (int t = 0; t < CPL; ++t)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int c = cl + LPR * t, k = c * 8 + e;
            gw[t * 8 + e] = (c < ch && p.ln_w) ? __ldg(p.ln_w + k) : 1.f;
            gb[t * 8 + e] = (c < ch && p.ln_b) ? __ldg(p.ln_b + k) : 0.f;
        }
    float bh[HP];
#pragma unroll
    for (int h = 0; h < HP; ++h) bh[h] = (h < H && p.bias) ? __ldg(p.bias + h) : 0.f;
    __syncthreads();
    for (int64_t r0 = (int64_t)blockIdx.x * PB_ROWS; r0 < total; r0 += (int64_t)gridDim.x * PB_ROWS) {
#pragma unroll 1
        for (int ib = 0; ib < ITERS; ib += BATCH) {
            uint4 v[BATCH][CPL];
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                const int64_t r = r0 + warp * ROWS_W + (ib + b) * RPI + sub;
#pragma unroll
                for (int t = 0; t < CPL; ++t) {
                    const int c = cl + LPR * t;
                    v[b][t] = (r < total && c < ch) ? __ldg(zg + r * ch + c) : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                const int rloc = warp * ROWS_W + (ib + b) * RPI + sub;
                float f[CPL * 8];
#pragma unroll
                for (int t = 0; t < CPL; ++t) unpack8(v[b][t], f + 8 * t);
                float sum = 0.f;
#pragma unroll
                for (int e = 0; e < CPL * 8; ++e) sum += f[e];
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                const float mean = sum * inv_c;
                float sq = 0.f;
#pragma unroll
                for (int t = 0; t < CPL; ++t)
                    if (cl + LPR * t < ch) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) sq = fmaf(f[8 * t + e] - mean, f[8 * t + e] - mean, sq);
                    }
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
                const float rstd = rsqrtf(sq * inv_c + p.eps);
                float acc[HP];
#pragma unroll
                for (int h = 0; h < HP; ++h) acc[h] = 0.f;
#pragma unroll
                for (int t = 0; t < CPL; ++t) {
                    const int c = cl + LPR * t;
                    if (c < ch) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float nv = fmaf((f[8 * t + e] - mean) * rstd, gw[8 * t + e], gb[8 * t + e]);
                            const float4* w4 = reinterpret_cast<const float4*>(wsh + (e * ch + c) * HP);
#pragma unroll
                            for (int hq = 0; hq < HQ; ++hq) {
                                const float4 wv = w4[hq];
                                acc[4 * hq] = fmaf(nv, wv.x, acc[4 * hq]);
                                acc[4 * hq + 1] = fmaf(nv, wv.y, acc[4 * hq + 1]);
                                acc[4 * hq + 2] = fmaf(nv, wv.z, acc[4 * hq + 2]);
                                acc[4 * hq + 3] = fmaf(nv, wv.w, acc[4 * hq + 3]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < HP; ++h) {
#pragma unroll
                    for (int o = LPR / 2; o >= 1; o >>= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
                }
                if (cl == 0) {
#pragma unroll
                    for (int h = 0; h < HP; ++h) osh[h * PB_ROWS + rloc] = __float2bfloat16_rn(acc[h] + bh[h]);
                }
            }
        }
        __syncthreads();
        for (int o = threadIdx.x; o < H * PB_ROWS; o += PB_THREADS) {
            const int h = o / PB_ROWS, rloc = o - h * PB_ROWS;
            const int64_t r = r0 + rloc;
            if (r < total) {
                const int64_t b = r / nn, ij = r - b * nn;
                p.out[(b * H + h) * nn + ij] = osh[o];
            }
        }
        __syncthreads();
    }
}

}  // namespace proj
}  // namespace evo
