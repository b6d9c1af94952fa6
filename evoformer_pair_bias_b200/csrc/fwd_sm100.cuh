// fwd_sm100.cuh -- bf16 forward of Evoformer pair-bias attention on sm_100a.
//
// One CTA owns a 128-row query tile i0..i0+127 of head h in batch b, for
// NSUB consecutive rows s (MSA sequences or pair rows).  It streams the key
// axis in 128-key tiles and never stores a logit outside TMEM/registers
// (the flash-style, online-softmax treatment EvoFlash-3D gives this op in
// the MegaFold summary, section "EvoFlash-3D"); the pair-bias tile of
// (h, i-tile, j-tile) is the same for every row s, so it is loaded once per
// CTA and read by all NSUB softmax warpgroups.
//
// Warp roles (64 + 128*NSUB threads):
//   warp 0        TMA producer: Q once, then per key tile K, V (per row s),
//                 the pair-bias tile and the mask row into a 2-stage ring.
//   warp 1        TMEM owner and MMA issuer (one lane):
//                   S_u  = Q_u K_u^T          (M=128, N=128, K=32)  -> TMEM
//                   O_u += P_u V_u            (M=128, N=32,  K=128, P read from TMEM)
//   warps 2..     one 4-warp softmax group per row s (thread = query row):
//                 load S from TMEM, add scale/bias/mask, online max/sum in
//                 fp32, rescale O in TMEM when the max moves, write P (bf16)
//                 back to TMEM, and finally out = sigmoid(g) * O / l and
//                 lse = m + log l.
// TMEM per row s: S 128 columns, P 64 columns (bf16 pairs), O 32 columns.
#pragma once

#include "sm100.cuh"

namespace evo {
namespace fwd {

using namespace evo::sm100;

constexpr int BM = 128;                 // query rows per tile (TMEM lanes)
constexpr int BN = 128;                 // keys per tile
constexpr int HD = 32;                  // head dim C
constexpr int STAGES = 2;
constexpr int Q_BYTES = BM * HD * 2;    // 8 KB, 64-byte rows, 64B swizzle
constexpr int KV_BYTES = BN * HD * 2;   // 8 KB each for K and V
constexpr int BIAS_BOX = BM * 64 * 2;   // 16 KB: 128 rows x 64 keys, 128B swizzle
constexpr int BIAS_BYTES = 2 * BIAS_BOX;
constexpr int MASK_BYTES = BN * 2;
constexpr uint32_t COL_S = 0, COL_P = 128, COL_O = 192, SUBCOLS = 256;

__host__ __device__ constexpr int round_up(int x, int a) { return (x + a - 1) / a * a; }

template <int NSUB>
struct Layout {
    static constexpr int q = 0;
    static constexpr int stage0 = NSUB * Q_BYTES;
    static constexpr int k_off(int u) { return u * KV_BYTES; }
    static constexpr int v_off(int u) { return (NSUB + u) * KV_BYTES; }
    static constexpr int bias_off = 2 * NSUB * KV_BYTES;
    static constexpr int mask_off(int u) { return bias_off + BIAS_BYTES + u * MASK_BYTES; }
    static constexpr int stage_bytes = round_up(bias_off + BIAS_BYTES + NSUB * MASK_BYTES, 1024);
    static constexpr int bars = stage0 + STAGES * stage_bytes;
    // q_full, kv_full[2], kv_empty[2], s_full[u], s_free[u], p_full[u], o_full[u], mma_done
    static constexpr int nbars = 1 + 2 * STAGES + 4 * NSUB + 1;
    static constexpr int misc = bars + nbars * 8;   // tmem base (u32), abort flag (u32)
    static constexpr int bytes = misc + 16 + 1024;  // + slack to align the base to 1024
    static constexpr uint32_t tmem_cols = NSUB == 1 ? 256 : 512;
    static constexpr int threads = 64 + 128 * NSUB;
    static constexpr int min_blocks = NSUB == 1 ? 2 : 1;
};

struct Params {
    int B, S, N, H;
    int n_kv;                 // ceil(N / BN)
    float scale;              // 1/sqrt(C)
    const __nv_bfloat16* g;   // gate, strides `in`
    Strides in;
    __nv_bfloat16* out;       // strides `os`
    Strides os;
    float* lse;               // [B,S,H,N]
};

// Status codes recorded when a wait gives up: 0x1RRB (role R, barrier B).
enum : unsigned int { kTimeoutBase = 0x1000u };

template <int NSUB, bool HAS_MASK, bool HAS_BIAS>
__global__ void __launch_bounds__(Layout<NSUB>::threads, Layout<NSUB>::min_blocks)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_bias,
                    const __grid_constant__ CUtensorMap tm_mask, const Params p) {
    using L = Layout<NSUB>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * BM;
    const int s0 = blockIdx.y * NSUB;
    const int b = blockIdx.z / p.H, h = blockIdx.z % p.H;

    const uint32_t bar0 = base + L::bars;
    const uint32_t bar_q = bar0;
    auto bar_kv_full = [&](int st) { return bar0 + 8u * (1 + st); };
    auto bar_kv_empty = [&](int st) { return bar0 + 8u * (1 + STAGES + st); };
    auto bar_s_full = [&](int u) { return bar0 + 8u * (1 + 2 * STAGES + u); };
    auto bar_s_free = [&](int u) { return bar0 + 8u * (1 + 2 * STAGES + NSUB + u); };
    auto bar_p_full = [&](int u) { return bar0 + 8u * (1 + 2 * STAGES + 2 * NSUB + u); };
    auto bar_o_full = [&](int u) { return bar0 + 8u * (1 + 2 * STAGES + 3 * NSUB + u); };
    const uint32_t bar_mma_done = bar0 + 8u * (1 + 2 * STAGES + 4 * NSUB);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + L::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::misc + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(bar_kv_full(st), 1);
            mbar_init(bar_kv_empty(st), 1 + 4 * NSUB);
        }
        for (int u = 0; u < NSUB; ++u) {
            mbar_init(bar_s_full(u), 1);
            mbar_init(bar_s_free(u), 4);
            mbar_init(bar_p_full(u), 4);
            mbar_init(bar_o_full(u), 1);
        }
        mbar_init(bar_mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        if (HAS_BIAS) prefetch_tmap(&tm_bias);
        if (HAS_MASK) prefetch_tmap(&tm_mask);
    }
    if (warp == 1) {
        tmem_alloc(base + L::misc, L::tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int s_ld[NSUB];
#pragma unroll
            for (int u = 0; u < NSUB; ++u) s_ld[u] = min(s0 + u, p.S - 1);
            mbar_arrive_expect_tx(bar_q, NSUB * Q_BYTES);
#pragma unroll
            for (int u = 0; u < NSUB; ++u) tma_load_5d(base + L::q + u * Q_BYTES, &tm_q, bar_q, 0, i0, h, s_ld[u], b);
            constexpr uint32_t tx = 2 * NSUB * KV_BYTES + (HAS_BIAS ? BIAS_BYTES : 0) + (HAS_MASK ? NSUB * MASK_BYTES : 0);
            int issued[STAGES] = {};
            for (int j = 0; j < p.n_kv; ++j) {
                const int st = j % STAGES;
                const uint32_t sb = base + L::stage0 + st * L::stage_bytes;
                if (j >= STAGES && !mbar_wait(bar_kv_empty(st), ((j / STAGES) - 1) & 1, abort_flag, kTimeoutBase | 0x001))
                    break;
                mbar_arrive_expect_tx(bar_kv_full(st), tx);
#pragma unroll
                for (int u = 0; u < NSUB; ++u) {
                    tma_load_5d(sb + L::k_off(u), &tm_k, bar_kv_full(st), 0, j * BN, h, s_ld[u], b);
                    tma_load_5d(sb + L::v_off(u), &tm_v, bar_kv_full(st), 0, j * BN, h, s_ld[u], b);
                }
                if (HAS_BIAS) {
                    tma_load_4d(sb + L::bias_off, &tm_bias, bar_kv_full(st), j * BN, i0, h, b);
                    tma_load_4d(sb + L::bias_off + BIAS_BOX, &tm_bias, bar_kv_full(st), j * BN + 64, i0, h, b);
                }
                if (HAS_MASK) {
#pragma unroll
                    for (int u = 0; u < NSUB; ++u)
                        tma_load_3d(sb + L::mask_off(u), &tm_mask, bar_kv_full(st), j * BN, s_ld[u], b);
                }
                ++issued[st];
            }
            // Never leave with copies in flight: wait (bounded) for the last fill of each stage.
            volatile int no_abort = 0;
            mbar_wait(bar_q, 0, &no_abort, kTimeoutBase | 0x002);
            for (int st = 0; st < STAGES; ++st)
                if (issued[st] > 0) mbar_wait(bar_kv_full(st), (issued[st] - 1) & 1, &no_abort, kTimeoutBase | 0x003);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false, false);
            constexpr uint32_t IDESC_PV = idesc_bf16(BM, HD, false, true);
            bool ok = mbar_wait(bar_q, 0, abort_flag, kTimeoutBase | 0x101);
            const uint32_t qa = base + L::q;
            for (int j = 0; ok && j <= p.n_kv; ++j) {
                if (j < p.n_kv) {
                    const int st = j % STAGES;
                    const uint32_t sb = base + L::stage0 + st * L::stage_bytes;
                    ok = mbar_wait(bar_kv_full(st), (j / STAGES) & 1, abort_flag, kTimeoutBase | 0x102);
#pragma unroll
                    for (int u = 0; u < NSUB && ok; ++u) {
                        if (j > 0) ok = mbar_wait(bar_s_free(u), (j - 1) & 1, abort_flag, kTimeoutBase | 0x103);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk) {
                            const uint64_t ad = smem_desc(qa + u * Q_BYTES + kk * 32, 16, 512, kSw64);
                            const uint64_t bd = smem_desc(sb + L::k_off(u) + kk * 32, 16, 512, kSw64);
                            mma_ss(tmem + u * SUBCOLS + COL_S, ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(bar_s_full(u));
                    }
                }
                if (ok && j > 0) {
                    const int jp = j - 1, st = jp % STAGES;
                    const uint32_t sb = base + L::stage0 + st * L::stage_bytes;
#pragma unroll
                    for (int u = 0; u < NSUB && ok; ++u) {
                        ok = mbar_wait(bar_p_full(u), jp & 1, abort_flag, kTimeoutBase | 0x104);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk) {
                            const uint64_t bd = smem_desc(sb + L::v_off(u) + kk * 1024, KV_BYTES, 512, kSw64);
                            mma_ts(tmem + u * SUBCOLS + COL_O, tmem + u * SUBCOLS + COL_P + kk * 8, bd, IDESC_PV,
                                   (jp > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(bar_o_full(u));
                    }
                    if (ok) mma_commit(bar_kv_empty(st));
                }
            }
            // Drain: every MMA issued by this thread has finished before TMEM is released.
            mma_commit(bar_mma_done);
            volatile int no_abort = 0;
            mbar_wait(bar_mma_done, 0, &no_abort, kTimeoutBase | 0x105);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int u = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;          // query row within the tile = TMEM lane
        const int s = s0 + u;
        const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + u * SUBCOLS;
        const float scale = p.scale;
        // Running max in log2 units (ms = max * log2 e, exactly the value that is
        // subtracted inside exp2) and running sum l of exp2(x * log2 e - ms).
        float ms = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < p.n_kv; ++j) {
            const int st = j % STAGES;
            const uint32_t sb = base + L::stage0 + st * L::stage_bytes;
            ok = mbar_wait(bar_s_full(u), j & 1, abort_flag, kTimeoutBase | 0x201);
            if (!ok) break;
            tc_fence_after();
            uint32_t xr[BN];
            tmem_ld128_sync(lane_addr + COL_S, xr);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_s_free(u));
            ok = mbar_wait(bar_kv_full(st), (j / STAGES) & 1, abort_flag, kTimeoutBase | 0x202);
            if (!ok) break;

            // x = S/sqrt(C) + pair_bias[i, j] + mask_bias[s, j]   (natural-log units)
            // Row max over 4 independent partial maxima (short dependency chains).
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int q = 0; q < BN / 8; ++q) {
                float add[8];
                if (HAS_BIAS) {
                    const uint32_t chunk = (uint32_t)(q & 7) ^ (uint32_t)(r & 7);
                    const uint4 w = lds128(sb + L::bias_off + (q >> 3) * BIAS_BOX + r * 128 + (chunk << 4));
                    add[0] = bf16lo(w.x); add[1] = bf16hi(w.x); add[2] = bf16lo(w.y); add[3] = bf16hi(w.y);
                    add[4] = bf16lo(w.z); add[5] = bf16hi(w.z); add[6] = bf16lo(w.w); add[7] = bf16hi(w.w);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) add[e] = 0.f;
                }
                if (HAS_MASK) {
                    const uint4 w = lds128(sb + L::mask_off(u) + q * 16);
                    add[0] += bf16lo(w.x); add[1] += bf16hi(w.x); add[2] += bf16lo(w.y); add[3] += bf16hi(w.y);
                    add[4] += bf16lo(w.z); add[5] += bf16hi(w.z); add[6] += bf16lo(w.w); add[7] += bf16hi(w.w);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xv = fmaf(__uint_as_float(xr[q * 8 + e]), scale, add[e]);
                    xr[q * 8 + e] = __float_as_uint(xv);
                    mq[e & 3] = fmaxf(mq[e & 3], xv);
                }
            }
            float mloc = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            const int valid = p.N - j * BN;      // keys beyond N are padding: exclude them
            if (valid < BN) {
                mloc = -INFINITY;
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    if (c >= valid) xr[c] = __float_as_uint(-INFINITY);
                    mloc = fmaxf(mloc, __uint_as_float(xr[c]));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_kv_empty(st));   // done reading bias / mask of this stage

            const float ms_new = fmaxf(ms, mloc * EVO_LOG2E);
            const float alpha = ex2(ms - ms_new);       // 0 on the first tile, exactly 1 if the max stays
            float rq[4] = {0.f, 0.f, 0.f, 0.f};     // 4 independent partial sums
            uint32_t pk[BN / 2];
#pragma unroll
            for (int c = 0; c < BN / 2; ++c) {
                const float p0 = ex2(fmaf(__uint_as_float(xr[2 * c]), EVO_LOG2E, -ms_new));
                const float p1 = ex2(fmaf(__uint_as_float(xr[2 * c + 1]), EVO_LOG2E, -ms_new));
                rq[c & 3] += p0 + p1;
                pk[c] = pack_bf16(p0, p1);
            }
            const float rs = (rq[0] + rq[1]) + (rq[2] + rq[3]);
            l = l * alpha + rs;
            ms = ms_new;
            if (j > 0) {
                // O must hold PV of tile j-1 before it is rescaled and P is overwritten.
                ok = mbar_wait(bar_o_full(u), (j - 1) & 1, abort_flag, kTimeoutBase | 0x203);
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.0f)) {
                    uint32_t o[HD];
                    tmem_ld32_sync(lane_addr + COL_O, o);
#pragma unroll
                    for (int c = 0; c < HD; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st32(lane_addr + COL_O, o);
                }
            }
            tmem_st32(lane_addr + COL_P, pk);
            tmem_st32(lane_addr + COL_P + 32, pk + 32);
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_p_full(u));
        }
        if (ok) ok = mbar_wait(bar_o_full(u), (p.n_kv - 1) & 1, abort_flag, kTimeoutBase | 0x204);
        if (ok) {
            tc_fence_after();
            uint32_t o[HD];
            tmem_ld32_sync(lane_addr + COL_O, o);
            const int i = i0 + r;
            if (s < p.S && i < p.N) {
                const float inv_l = 1.0f / l;
                const __nv_bfloat16* gp = p.g + p.in.off(b, s, i, h);
                __nv_bfloat16* op = p.out + p.os.off(b, s, i, h);
#pragma unroll
                for (int q = 0; q < HD / 8; ++q) {
                    const uint4 gw = *reinterpret_cast<const uint4*>(gp + q * 8);
                    const uint32_t gv[4] = {gw.x, gw.y, gw.z, gw.w};
                    uint32_t ov[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float g0 = bf16lo(gv[e]), g1 = bf16hi(gv[e]);
                        const float o0 = __uint_as_float(o[q * 8 + 2 * e]) * inv_l / (1.0f + __expf(-g0));
                        const float o1 = __uint_as_float(o[q * 8 + 2 * e + 1]) * inv_l / (1.0f + __expf(-g1));
                        ov[e] = pack_bf16(o0, o1);
                    }
                    *reinterpret_cast<uint4*>(op + q * 8) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
                }
                p.lse[((int64_t)(b * p.S + s) * p.H + h) * p.N + i] = (ms + __log2f(l)) * EVO_LN2;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::tmem_cols);
    }
}

}  // namespace fwd
}  // namespace evo
