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
// columns are cut into slices of BNO and the slices into column groups; CTA c
// takes group c % n_groups and walks the 128-row blocks c / n_groups,
// + grid / n_groups, ..., producing the group's columns of each.  w is cut
// into chunks of 64 k-rows x BNO columns (an MN-major B operand, TMA with
// 128B swizzle), which stay resident in shared memory when a group's chunks
// fit and otherwise stream from L2 through a ring of stages.  The host picks
// the widest group whose w fits (each row is then normalised once per group),
// else one group of all columns (each row normalised once).  Roles:
//   warp 0      one thread issues the MMAs (M = 128, N = BNO, K = 16) of
//               each slice into TMEM accumulator (slice count) % 2;
//   warps 1-4   epilogue: TMEM -> + bias -> bf16 -> shared staging (128B
//               swizzle) -> TMA store, 32 rows x 64 columns per store;
//   warps 5-12  LayerNorm: coalesced 16-byte loads of x rows from global
//               memory (a row's c_in channels spread over up to 32 lanes),
//               fp32 statistics by warp shuffles, normalised bf16 written
//               into the A tile (K-major, 128B swizzle) the MMA reads;
//   warp 13     one thread: TMA loads of the w chunks.
// The A tile is double-buffered unless that leaves fewer than four w stages
// (c_in = 256 and 192 with 256-column slices); the LayerNorm warps load and
// normalise the next block in registers while the MMAs read the current one.
// Every wait is bounded; on expiry the CTA records a status code and winds
// down.
//
// pair_bias_rows_kernel (SIMT, c_z <= 256, H <= 16): one pair row per thread
// from a shared-memory tile (described at the kernel).
// pair_bias_kernel (SIMT, any c_z <= 1024, H <= 16): block = 8 warps, 128
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
constexpr int THREADS = 32 * (2 + EPI_WARPS + LN_WARPS);   // + MMA warp + w producer warp
constexpr int STG_TILE = 32 * 128;             // 32 rows x 64 bf16 columns
constexpr int STG_BYTES = EPI_WARPS * 2 * STG_TILE;
constexpr int SMEM_LIMIT = 232448;             // opt-in dynamic shared memory per CTA
constexpr int SMEM_MIN = 120 * 1024;           // > half an SM: one CTA (and one TMEM owner) per SM

constexpr int BIAS_CACHE = 1024;               // bias floats kept in shared memory (larger n_out: read from L1/L2)

template <int BNO, int CIN>
struct PLayout {
    static constexpr int w_chunk = BNO * 64 * 2;                  // 64 k-rows x BNO columns (BNO/64 boxes of 8 KB)
    static constexpr int a_bytes = CIN / KBOX * BM * 128;         // CIN/64 boxes of 128 rows x 128 B
    static constexpr int fixed = STG_BYTES + BIAS_CACHE * 4 + 512 + 1024;   // staging, bias, barriers, slack
    static constexpr int region(int na) { return SMEM_LIMIT - fixed - na * a_bytes; }
    static constexpr int cap(int na) { return region(na) / w_chunk > 8 ? 8 : region(na) / w_chunk; }
    // double-buffer the A tile unless that leaves fewer than three w stages
    static constexpr int NA = cap(2) >= 3 ? 2 : 1;
    static constexpr int NW = cap(NA);                            // w stages (ring, or all chunks when they fit)
    static constexpr int w_off = 0;
    static constexpr int a_off = NW * w_chunk;
    static constexpr int stg_off = a_off + NA * a_bytes;
    static constexpr int bias_off = stg_off + STG_BYTES;
    static constexpr int bar_off = bias_off + BIAS_CACHE * 4;
    // w_full[NW], w_empty[NW], a_full[NA], a_empty[NA], acc_full[2], acc_empty[2], done
    static constexpr int n_bars = 2 * NW + 2 * NA + 5;
    static constexpr int misc_off = bar_off + n_bars * 8;         // TMEM slot, abort flag
    static constexpr int used = misc_off + 16;
    static constexpr int bytes = used + 1024 > SMEM_MIN ? used + 1024 : SMEM_MIN;
    static_assert(NW >= 2, "w ring");
    static_assert(n_bars * 8 + 16 <= 512, "barrier area");
    static_assert(used + 1024 <= SMEM_LIMIT, "shared memory budget");
};

struct LnParams {
    int rows, c_in, n_out;
    int gsl;                  // column slices per CTA (a column group); n_out / BNO / gsl groups
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

// Registers are granted per group of four warps, so the 14 warps count as 16:
// 128 registers a thread at most.
template <int BNO, int CIN>
__global__ void __launch_bounds__(THREADS, 1)
    ln_linear_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_y,
                     const LnParams p) {
    using L = PLayout<BNO, CIN>;
    constexpr int NA = L::NA, NW = L::NW, KC = CIN / KBOX;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gsl = p.gsl;                            // column slices this CTA produces per row block
    const int ngr = p.n_out / BNO / gsl;              // column groups
    const int sl0 = (int)(blockIdx.x % ngr) * gsl;    // first slice of this CTA's group
    const int rb0 = (int)(blockIdx.x / ngr), rbs = (int)(gridDim.x / ngr);
    const int total_chunks = gsl * KC;                // w chunks of one row block of the group
    const bool resident = total_chunks <= NW;         // the group's w stays in shared memory
    const int nrb = (p.rows + BM - 1) / BM;
    auto bar_wfull = [&](int i) { return base + L::bar_off + 8u * i; };
    auto bar_wempty = [&](int i) { return base + L::bar_off + 8u * (NW + i); };
    auto bar_afull = [&](int i) { return base + L::bar_off + 8u * (2 * NW + i); };
    auto bar_aempty = [&](int i) { return base + L::bar_off + 8u * (2 * NW + NA + i); };
    auto bar_accf = [&](int b) { return base + L::bar_off + 8u * (2 * NW + 2 * NA + b); };
    auto bar_acce = [&](int b) { return base + L::bar_off + 8u * (2 * NW + 2 * NA + 2 + b); };
    const uint32_t bar_done = base + L::bar_off + 8u * (2 * NW + 2 * NA + 4);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + L::misc_off);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::misc_off + 4);
    float* bias_s = reinterpret_cast<float*>(gbase + L::bias_off);
    const bool bias_cached = p.n_out <= BIAS_CACHE;
    if (bias_cached)
        for (int i = threadIdx.x; i < p.n_out; i += THREADS) bias_s[i] = p.bias ? __ldg(p.bias + i) : 0.f;
    // the bias the epilogue reads: shared memory, or global memory (L1-cached) for wide outputs
    const float* bias_src = bias_cached ? bias_s : p.bias;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NW; ++i) {
            mbar_init(bar_wfull(i), 1);
            mbar_init(bar_wempty(i), 1);
        }
        for (int i = 0; i < NA; ++i) {
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
    if (warp == 0) {
        tmem_alloc(base + L::misc_off, 2 * BNO);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16(BM, BNO, false, true);   // B operand MN-major
            bool ok = true;
            int64_t it = 0;                            // w chunks consumed (ring mode)
            int sl = 0;                                // slices accumulated (TMEM buffer rotation)
            int j = 0;
            for (int rb = rb0; ok && rb < nrb; rb += rbs, ++j) {
                const int s = j % NA, n = j / NA;
                ok = mbar_wait(bar_afull(s), n & 1, abort_flag, kTimeoutBase | 0x03);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_base = base + L::a_off + s * L::a_bytes;
                for (int si = 0; ok && si < gsl; ++si, ++sl) {
                    const int buf = sl & 1, m = sl >> 1;
                    ok = mbar_wait(bar_acce(buf), (m & 1) ^ 1, abort_flag, kTimeoutBase | 0x02);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(buf * BNO);
                    for (int kc = 0; kc < KC; ++kc) {
                        int st;
                        if (resident) {
                            st = si * KC + kc;
                            ok = mbar_wait(bar_wfull(st), 0, abort_flag, kTimeoutBase | 0x08);
                        } else {
                            st = (int)(it % NW);
                            ok = mbar_wait(bar_wfull(st), (uint32_t)((it / NW) & 1), abort_flag, kTimeoutBase | 0x08);
                        }
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t w_base = base + L::w_off + st * L::w_chunk;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = smem_desc(a_base + kc * BM * 128 + kk * 32, 16, 1024, kSw128);
                            const uint64_t bd = smem_desc(w_base + kk * 2048, 8192, 1024, kSw128);
                            mma_ss(d, ad, bd, IDESC, (kc > 0 || kk > 0) ? 1u : 0u);
                        }
                        if (!resident) {
                            mma_commit(bar_wempty(st));     // the w stage may be refilled
                            ++it;
                        }
                    }
                    if (ok) mma_commit(bar_accf(buf));
                }
                if (ok) mma_commit(bar_aempty(s));          // the A stage may be rewritten
            }
            // every MMA issued above completes before TMEM and shared memory are released
            volatile int no_abort = 0;
            mma_commit(bar_done);
            mbar_wait(bar_done, 0, &no_abort, kTimeoutBase | 0x04);
        }
    } else if (warp == 1 + EPI_WARPS + LN_WARPS) {
        // ---------------------------------------------------------- w producer
        if (lane == 0) {
            prefetch_tmap(&tm_w);
            bool ok = true;
            int64_t it = 0;
            for (int rb = rb0; ok && rb < nrb; rb += rbs) {
                for (int c = 0; ok && c < total_chunks; ++c) {
                    const int si = c / KC, kc = c % KC;
                    int st;
                    if (resident) {
                        st = c;
                    } else {
                        st = (int)(it % NW);
                        ok = mbar_wait(bar_wempty(st), (uint32_t)(((it / NW) & 1) ^ 1), abort_flag, kTimeoutBase | 0x09);
                        if (!ok) break;
                        ++it;
                    }
                    const uint32_t fb = bar_wfull(st), dst = base + L::w_off + st * L::w_chunk;
                    mbar_arrive_expect_tx(fb, (uint32_t)L::w_chunk);
                    for (int nb = 0; nb < BNO / 64; ++nb)
                        tma_load_2d(dst + nb * 8192, &tm_w, fb, (sl0 + si) * BNO + nb * 64, kc * 64);
                }
                if (resident) break;                        // loaded once for every block
            }
            // the loads still in flight land before shared memory is released
            volatile int no_abort = 0;
            if (resident) {
                for (int c = 0; c < total_chunks; ++c) mbar_wait(bar_wfull(c), 0, &no_abort, kTimeoutBase | 0x0a);
            } else {
                for (int64_t u = it - NW > 0 ? it - NW : 0; u < it; ++u)
                    mbar_wait(bar_wfull((int)(u % NW)), (uint32_t)((u / NW) & 1), &no_abort, kTimeoutBase | 0x0a);
            }
        }
    } else if (warp <= EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                        // the TMEM lane quarter this warp may read
        const uint32_t stg = base + L::stg_off + (uint32_t)((warp - 1) * 2 * STG_TILE);
        if (lane == 0) prefetch_tmap(&tm_y);
        int sl = 0;
        bool ok = true;
        for (int rb = rb0; ok && rb < nrb; rb += rbs) {
            const int row0 = rb * BM + 32 * q;
            for (int si = 0; si < gsl; ++si, ++sl) {
                const int buf = sl & 1, m = sl >> 1;
                ok = mbar_wait(bar_accf(buf), m & 1, abort_flag, kTimeoutBase | 0x06);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int n0 = (sl0 + si) * BNO;
                const uint32_t taddr = tmem + (uint32_t)(buf * BNO) + ((uint32_t)(32 * q) << 16);
                // TMEM columns 64g .. 64g+31 arrive in va, 64g+32 .. 64g+63 in vb (each load
                // waited for in the same statement that issues it)
                uint32_t va[32], vb[32];
                const bool has_bias = bias_src != nullptr;
#pragma unroll 1
                for (int g = 0; g < BNO / 64; ++g) {
                    const uint32_t sb = stg + (uint32_t)((g & 1) * STG_TILE);
                    const float* bg = has_bias ? bias_src + n0 + 64 * g : nullptr;
                    tmem_ld32_sync(taddr + 64 * g, va);
                    if (lane == 0) bulk_wait_read<1>();    // the store that last read this buffer is done with it
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f), b1 = b0;
                        if (has_bias) {
                            b0 = *reinterpret_cast<const float4*>(bg + 8 * c);
                            b1 = *reinterpret_cast<const float4*>(bg + 8 * c + 4);
                        }
                        const uint32_t* vc = va + 8 * c;
                        sts128(sb + lane * 128 + ((c ^ (lane & 7)) << 4),
                               pack_bf16(__uint_as_float(vc[0]) + b0.x, __uint_as_float(vc[1]) + b0.y),
                               pack_bf16(__uint_as_float(vc[2]) + b0.z, __uint_as_float(vc[3]) + b0.w),
                               pack_bf16(__uint_as_float(vc[4]) + b1.x, __uint_as_float(vc[5]) + b1.y),
                               pack_bf16(__uint_as_float(vc[6]) + b1.z, __uint_as_float(vc[7]) + b1.w));
                    }
                    tmem_ld32_sync(taddr + 64 * g + 32, vb);
#pragma unroll
                    for (int c = 4; c < 8; ++c) {
                        float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f), b1 = b0;
                        if (has_bias) {
                            b0 = *reinterpret_cast<const float4*>(bg + 8 * c);
                            b1 = *reinterpret_cast<const float4*>(bg + 8 * c + 4);
                        }
                        const uint32_t* vc = vb + 8 * (c - 4);
                        sts128(sb + lane * 128 + ((c ^ (lane & 7)) << 4),
                               pack_bf16(__uint_as_float(vc[0]) + b0.x, __uint_as_float(vc[1]) + b0.y),
                               pack_bf16(__uint_as_float(vc[2]) + b0.z, __uint_as_float(vc[3]) + b0.w),
                               pack_bf16(__uint_as_float(vc[4]) + b1.x, __uint_as_float(vc[5]) + b1.y),
                               pack_bf16(__uint_as_float(vc[6]) + b1.z, __uint_as_float(vc[7]) + b1.w));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    // rows past the end are clipped by the tensor map; a box wholly past them is
                    // not stored, but its group is still committed so that the wait above keeps
                    // covering the store that last read each buffer
                    if (lane == 0) {
                        if (row0 < p.rows) tma_store_2d(&tm_y, sb, n0 + 64 * g, row0);
                        bulk_commit();
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acce(buf));
            }
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
        for (int rb = rb0; rb < nrb; rb += rbs, ++j) {
            const int s = j % NA, n = j / NA;
            uint4 xv[ITERS];
#pragma unroll
            for (int it = 0; it < ITERS; ++it) {
                const int r = rb * BM + lw * ROWS_W + it * RPI + sub;
                xv[it] = (active && r < p.rows) ? __ldg(xg + (int64_t)r * CH + cidx) : make_uint4(0, 0, 0, 0);
            }
            // the next block's rows into L2 while this one is normalised
            const int rb_next = rb + rbs;
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
            const bool ok = mbar_wait(bar_aempty(s), (n & 1) ^ 1, abort_flag, kTimeoutBase | 0x07);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (active) {
#pragma unroll
                for (int it = 0; it < ITERS; ++it) {
                    const int rr = lw * ROWS_W + it * RPI + sub;
                    sts128(a_base + kb * BM * 128 + rr * 128 + ((cc ^ (rr & 7)) << 4), xv[it].x, xv[it].y, xv[it].z,
                           xv[it].w);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_afull(s));
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

// pair_bias_rows_kernel (c_z <= 256): block = 128 threads, one pair row per
// thread and 128 consecutive rows per step.  The rows are staged in shared
// memory by cp.async (coalesced 16-byte copies; row pitch padded to an odd
// number of 16-byte units, so the 32 rows a warp reads at one offset fall in
// distinct bank groups).  Each thread then normalises its own row (no
// shuffles) and forms the H outputs as
//   out_h = rstd * sum_k (x_k - mean) * (ln_w_k w_kh) + (sum_k ln_b_k w_kh + bias_h),
// the same sum as sum_k LN(x)_k w_kh regrouped in fp32, with ln_w_k w_kh and
// the constant term computed once per block (shared memory, read by
// broadcast).  Outputs go straight to out[b, h, i, j], consecutive threads
// writing consecutive j.
constexpr int PBR_THREADS = 128;
constexpr int PBR_MAX_CZ = 256;
constexpr int PBR_SMEM = PBR_THREADS * (PBR_MAX_CZ / 8 + 1) * 16 + PBR_MAX_CZ * PB_MAX_H * 4 +
                         (1 + PBR_THREADS / 32) * PB_MAX_H * 4;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

template <int HQ>
__global__ void __launch_bounds__(PBR_THREADS) pair_bias_rows_kernel(const PbParams p) {
    constexpr int HP = 4 * HQ;
    extern __shared__ __align__(16) uint8_t pbr_smem[];
    const int ch = p.c_z / 8;
    const int pitch = ch | 1;                                      // row pitch in 16-byte units (odd)
    uint8_t* zt = pbr_smem;                                        // [PBR_THREADS][pitch] x 16 B
    float* wsh = reinterpret_cast<float*>(pbr_smem + PBR_THREADS * pitch * 16);   // [c_z][HP]: ln_w_k w_kh
    float* csh = wsh + p.c_z * HP;                                 // [HP]: sum_k ln_b_k w_kh + bias_h
    const int H = p.H, t = threadIdx.x;
    for (int o = t; o < p.c_z * HP; o += PBR_THREADS) {
        const int k = o / HP, h = o - k * HP;
        const float g = p.ln_w ? __ldg(p.ln_w + k) : 1.f;
        wsh[o] = h < H ? g * __bfloat162float(p.w[k * H + h]) : 0.f;
    }
    // sum_k ln_b_k w_kh: every thread takes channels k = t, t + 128, reduced by warp
    // shuffles and then over the warps in a fixed order (deterministic)
    float* part = csh + HP;                                         // [PBR_THREADS / 32][HP]
    {
        float pc[HP];
#pragma unroll
        for (int h = 0; h < HP; ++h) pc[h] = 0.f;
        if (p.ln_b)
            for (int k = t; k < p.c_z; k += PBR_THREADS) {
                const float bk = __ldg(p.ln_b + k);
#pragma unroll
                for (int h = 0; h < HP; ++h)
                    if (h < H) pc[h] = fmaf(bk, __bfloat162float(p.w[k * H + h]), pc[h]);
            }
#pragma unroll
        for (int h = 0; h < HP; ++h) {
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) pc[h] += __shfl_xor_sync(0xffffffffu, pc[h], o);
        }
        if ((t & 31) == 0)
#pragma unroll
            for (int h = 0; h < HP; ++h) part[(t >> 5) * HP + h] = pc[h];
    }
    __syncthreads();
    if (t < HP) {
        float c = (t < H && p.bias) ? __ldg(p.bias + t) : 0.f;
        for (int w = 0; w < PBR_THREADS / 32; ++w) c += part[w * HP + t];
        csh[t] = c;
    }
    const int64_t nn = (int64_t)p.N * p.N, total = (int64_t)p.B * nn;
    const float inv_c = 1.f / (float)p.c_z;
    const uint4* zg = reinterpret_cast<const uint4*>(p.z);
    const uint32_t zt_s = smem_u32(zt);
    for (int64_t r0 = (int64_t)blockIdx.x * PBR_THREADS; r0 < total; r0 += (int64_t)gridDim.x * PBR_THREADS) {
        const int rows = (int)(total - r0 < PBR_THREADS ? total - r0 : PBR_THREADS);
        for (int idx = t; idx < rows * ch; idx += PBR_THREADS) {
            const int row = idx / ch, c = idx - row * ch;
            cp_async16(zt_s + (uint32_t)((row * pitch + c) * 16), zg + (r0 + row) * ch + c);
        }
        cp_async_wait_all();
        __syncthreads();
        if (t < rows) {
            const uint4* zr = reinterpret_cast<const uint4*>(zt + t * pitch * 16);
            float sum = 0.f;
            for (int c = 0; c < ch; ++c) {
                float f[8];
                unpack8(zr[c], f);
                sum += ((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]));
            }
            const float mean = sum * inv_c;
            float sq = 0.f;
            for (int c = 0; c < ch; ++c) {
                float f[8];
                unpack8(zr[c], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) sq = fmaf(f[e] - mean, f[e] - mean, sq);
            }
            const float rstd = rsqrtf(sq * inv_c + p.eps);
            float acc[HP];
#pragma unroll
            for (int h = 0; h < HP; ++h) acc[h] = 0.f;
            for (int c = 0; c < ch; ++c) {
                float f[8];
                unpack8(zr[c], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float d = f[e] - mean;
                    const float4* w4 = reinterpret_cast<const float4*>(wsh + (c * 8 + e) * HP);
#pragma unroll
                    for (int hq = 0; hq < HQ; ++hq) {
                        const float4 wv = w4[hq];
                        acc[4 * hq] = fmaf(d, wv.x, acc[4 * hq]);
                        acc[4 * hq + 1] = fmaf(d, wv.y, acc[4 * hq + 1]);
                        acc[4 * hq + 2] = fmaf(d, wv.z, acc[4 * hq + 2]);
                        acc[4 * hq + 3] = fmaf(d, wv.w, acc[4 * hq + 3]);
                    }
                }
            }
            const int64_t r = r0 + t, b = r / nn, ij = r - b * nn;
#pragma unroll
            for (int h = 0; h < HP; ++h)
                if (h < H) p.out[(b * H + h) * nn + ij] = __float2bfloat16_rn(fmaf(rstd, acc[h], csh[h]));
        }
        __syncthreads();                                           // the tile is free for the next copy
    }
}

}  // namespace proj
}  // namespace evo
