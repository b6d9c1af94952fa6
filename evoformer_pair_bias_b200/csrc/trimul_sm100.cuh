// trimul_sm100.cuh -- the contraction of the triangular multiplicative update
// on sm_100a ("Evoformer: the memory wall ZeRO cannot move", section "The
// three operations"): edge (i, j) is updated from every third residue k,
// channel by channel,
//
//   outgoing edges:  z[b, c, i, j] = sum_k a[b, c, i, k] * bb[b, c, j, k]
//   incoming edges:  z[b, c, i, j] = sum_k a[b, c, k, i] * bb[b, c, k, j]
//
// i.e. one N x N x N matrix product per (batch, channel): a dense contraction
// for the tensor cores.  The kernel takes rectangular products (z is M x Nc,
// the sum runs over K) and a scale on z, which the outer product mean uses:
// out[(i, c1), (j, c2)] = (1/S) sum_s a[s, (i, c1)] b[s, (j, c2)] is the
// MN-major form with M = N Ca, Nc = N Cb, K = S.  The operands are channel-first [B, C, N, N] bf16
// (the per-channel matrices contiguous); outgoing reads both operands
// K-major (k contiguous), incoming reads the same layout MN-major (i or j
// contiguous), so neither direction needs a transposed copy.  fp32
// accumulation in TMEM, bf16 output [B, C, N, N].
//
// tri_mul_kernel, persistent, one CTA per SM, 192 threads:
//   warp 0     one thread: TMA loads of 64-wide k chunks of the a tile
//              (128 rows i) and the b tile (256 rows j) into a 4-stage ring;
//   warp 1     one thread: tcgen05 MMAs (M = 128, N = 256, K = 16) into TMEM
//              accumulator t % 2 of its t-th tile;
//   warps 2-5  epilogue: TMEM -> bf16 -> shared staging (128B swizzle) ->
//              TMA store, 32 rows x 64 columns per store.
// Tiles (matrix, 128-row block of i, 256-column block of j) go round-robin
// to the CTAs.  3D tensor maps (inner, rows, matrices) zero-fill rows and k
// past the ends, so a ragged size never reads the next matrix.  Every wait is
// bounded.
#pragma once

#include "sm100.cuh"
#include "tma_maps.cuh"

namespace evo {
namespace trimul {

using namespace evo::sm100;

constexpr int BM = 128;                        // rows i of a tile
constexpr int BN = 256;                        // columns j of a tile
constexpr int BK = 64;                         // k per stage (one 128-byte swizzle span)
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int STG_TILE = 32 * 128;

struct TLayout {
    static constexpr int a_stage = BM * BK * 2;                    // 16 KB
    static constexpr int b_stage = BN * BK * 2;                    // 32 KB
    static constexpr int a_off = 0;
    static constexpr int b_off = STAGES * a_stage;
    static constexpr int stg_off = b_off + STAGES * b_stage;
    static constexpr int bar_off = stg_off + EPI_WARPS * 2 * STG_TILE;
    // full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], done
    static constexpr int n_bars = 2 * STAGES + 5;
    static constexpr int misc_off = bar_off + n_bars * 8;          // TMEM slot, abort flag
    static constexpr int bytes = misc_off + 16 + 1024;
    static_assert(bytes <= 232448, "shared memory budget");
};

struct TriParams {
    int M, Nc, K;       // z is M x Nc per matrix, the contraction runs over K
    int BC;             // independent matrices (B * C for the triangular update)
    int incoming;       // 0: a[i][k], b[j][k] (K-major); 1: a[k][i], b[k][j] (MN-major)
    float scale;        // z is multiplied by it before the bf16 rounding
    int tiles_i, tiles_j;
};

enum : unsigned int { kTimeoutBase = 0x4000u };

__global__ void __launch_bounds__(THREADS, 1)
    tri_mul_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_z, const TriParams p) {
    using L = TLayout;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_mat = p.tiles_i * p.tiles_j;
    const int64_t n_tiles = (int64_t)p.BC * per_mat;
    const int nk = (p.K + BK - 1) / BK;
    auto bar_full = [&](int s) { return base + L::bar_off + 8u * s; };
    auto bar_empty = [&](int s) { return base + L::bar_off + 8u * (STAGES + s); };
    auto bar_accf = [&](int b) { return base + L::bar_off + 8u * (2 * STAGES + b); };
    auto bar_acce = [&](int b) { return base + L::bar_off + 8u * (2 * STAGES + 2 + b); };
    const uint32_t bar_done = base + L::bar_off + 8u * (2 * STAGES + 4);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + L::misc_off);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::misc_off + 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_accf(b), 1);
            mbar_init(bar_acce(b), EPI_WARPS);
        }
        mbar_init(bar_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(base + L::misc_off, 2 * BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_a);
            prefetch_tmap(&tm_b);
            bool ok = true;
            int64_t it = 0;                                  // stage uses so far
            for (int64_t t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
                const int bc = (int)(t / per_mat), r = (int)(t % per_mat);
                const int i0 = (r / p.tiles_j) * BM, j0 = (r % p.tiles_j) * BN;
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int s = (int)(it % STAGES);
                    const uint32_t use = (uint32_t)(it / STAGES);
                    ok = mbar_wait(bar_empty(s), (use & 1) ^ 1, abort_flag, kTimeoutBase | 0x01);
                    if (!ok) break;
                    const uint32_t fb = bar_full(s);
                    mbar_arrive_expect_tx(fb, (uint32_t)(L::a_stage + L::b_stage));
                    const uint32_t sa = base + L::a_off + s * L::a_stage, sb = base + L::b_off + s * L::b_stage;
                    const int k0 = kc * BK;
                    if (!p.incoming) {
                        // a[i][k], b[j][k]: one box of 64 k x rows each (K-major)
                        tma_load_3d(sa, &tm_a, fb, k0, i0, bc);
                        tma_load_3d(sb, &tm_b, fb, k0, j0, bc);
                    } else {
                        // a[k][i], b[k][j]: boxes of 64 i (or j) x 64 k (MN-major)
                        for (int h = 0; h < BM / 64; ++h) tma_load_3d(sa + h * 8192, &tm_a, fb, i0 + 64 * h, k0, bc);
                        for (int h = 0; h < BN / 64; ++h) tma_load_3d(sb + h * 8192, &tm_b, fb, j0 + 64 * h, k0, bc);
                    }
                }
            }
            // the loads still in flight land before shared memory is released
            volatile int no_abort = 0;
            for (int64_t u = it - STAGES > 0 ? it - STAGES : 0; u < it; ++u)
                mbar_wait(bar_full((int)(u % STAGES)), (uint32_t)((u / STAGES) & 1), &no_abort, kTimeoutBase | 0x02);
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t IDESC = p.incoming ? idesc_bf16(BM, BN, true, true) : idesc_bf16(BM, BN, false, false);
            bool ok = true;
            int64_t it = 0;
            int tl = 0;                                      // tiles of this CTA so far
            for (int64_t t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++tl) {
                const int buf = tl & 1, m = tl >> 1;
                ok = mbar_wait(bar_acce(buf), (m & 1) ^ 1, abort_flag, kTimeoutBase | 0x03);
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * BN);
                for (int kc = 0; ok && kc < nk; ++kc, ++it) {
                    const int s = (int)(it % STAGES);
                    ok = mbar_wait(bar_full(s), (uint32_t)((it / STAGES) & 1), abort_flag, kTimeoutBase | 0x04);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t sa = base + L::a_off + s * L::a_stage, sb = base + L::b_off + s * L::b_stage;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        uint64_t ad, bd;
                        if (!p.incoming) {
                            ad = smem_desc(sa + kk * 32, 16, 1024, kSw128);
                            bd = smem_desc(sb + kk * 32, 16, 1024, kSw128);
                        } else {
                            ad = smem_desc(sa + kk * 2048, 8192, 1024, kSw128);
                            bd = smem_desc(sb + kk * 2048, 8192, 1024, kSw128);
                        }
                        mma_ss(d, ad, bd, IDESC, (kc > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar_empty(s));
                }
                if (ok) mma_commit(bar_accf(buf));
            }
            volatile int no_abort = 0;
            mma_commit(bar_done);
            mbar_wait(bar_done, 0, &no_abort, kTimeoutBase | 0x05);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                          // the TMEM lane quarter this warp may read
        const uint32_t stg = base + L::stg_off + (uint32_t)((warp - 2) * 2 * STG_TILE);
        if (lane == 0) prefetch_tmap(&tm_z);
        int tl = 0;
        for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tl) {
            const int buf = tl & 1, m = tl >> 1;
            const bool ok = mbar_wait(bar_accf(buf), m & 1, abort_flag, kTimeoutBase | 0x06);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int bc = (int)(t / per_mat), r = (int)(t % per_mat);
            const int row0 = (r / p.tiles_j) * BM + 32 * q, j0 = (r % p.tiles_j) * BN;
            const uint32_t taddr = tmem + (uint32_t)(buf * BN) + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
            for (int g = 0; g < BN / 64; ++g) {
                uint32_t v[64];
                tmem_ld32x2_sync(taddr + 64 * g, taddr + 64 * g + 32, v);
                if (p.scale != 1.f) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * p.scale);
                }
                const uint32_t sb = stg + (uint32_t)((g & 1) * STG_TILE);
                if (lane == 0) bulk_wait_read<1>();      // the store that last read this buffer is done with it
                __syncwarp();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t* vc = v + 8 * c;
                    sts128(sb + lane * 128 + ((c ^ (lane & 7)) << 4),
                           pack_bf16(__uint_as_float(vc[0]), __uint_as_float(vc[1])),
                           pack_bf16(__uint_as_float(vc[2]), __uint_as_float(vc[3])),
                           pack_bf16(__uint_as_float(vc[4]), __uint_as_float(vc[5])),
                           pack_bf16(__uint_as_float(vc[6]), __uint_as_float(vc[7])));
                }
                fence_proxy_async_smem();
                __syncwarp();
                // partial boxes are clipped; a box wholly outside z is not stored, but its
                // group is still committed: "every group but the newest is done" must
                // keep meaning "the store that last read the other buffer is done"
                if (lane == 0) {
                    if (row0 < p.M && j0 + 64 * g < p.Nc) tma_store_3d(&tm_z, sb, j0 + 64 * g, row0, bc);
                    bulk_commit();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_acce(buf));
        }
        if (lane == 0) bulk_wait<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 2 * BN);
    }
}

}  // namespace trimul
}  // namespace evo
