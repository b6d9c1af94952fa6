// dbias_sm100.cuh -- d_pair_bias of the bf16 backward on sm_100a, summed over
// the rows s on chip.
//
// d_pair_bias[b,h,i,j] = sum_s dS[b,s,h,i,j] is one number per (i, j) pair
// summed over every row s: the pair bias is a single term broadcast over the
// rows (MegaFold summary, section "EvoFlash-3D"), so its gradient is the sum
// of the rows' logit gradients.  This kernel gives each CTA a fixed
// 128-key x 128-query tile of one (b, h) and a group of rows s, streams the
// rows through it and keeps the running sum in registers, so each element of
// the result is written once per row group instead of once per row.
// P and dP are recomputed per row from the saved log-sum-exp, exactly as in
// the main backward kernel (the logits never leave the chip):
//   S^T  = K_j Q_i^T - lse_i sqrt(C) + (r1 + r2) mask_j      (tcgen05, TMEM)
//   dP^T = V_j (dOa_hi + dOa_lo)_i^T - D_i                    (tcgen05, TMEM)
//   P^T  = exp2(S^T log2(e)/sqrt(C) + bias^T log2(e) r1/sqrt(C)),   dS^T = P^T dP^T
//          (r1 = bf16(sqrt(C)): the bias with the forward's scale, see fwd_sm100.cuh)
//   acc[j, i] += dS^T    (fp32 registers, rows s in order)
// The row terms (-lse sqrt(C), -D as bf16 high/low pairs), the gated output
// gradient split into two bf16 parts and the transposed pair bias are the
// ones the backward's preparation pass writes for the main kernel.
//
// Work item = (b*H + h, query tile, key tile, row group g).  Persistent
// grid: one CTA per SM walks the items in a static round-robin.  Each item's
// sums are stored (plain stores, one writer per address) into the partial
// slab of its row group, or straight into d_pair_bias when there is one
// group; the finishing pass adds the slabs in group order.  The result is
// therefore bitwise reproducible.
//
// Warp roles (640 threads):
//   warps 0..15 four dS warpgroups (queries 0..31, 32..63, 64..95, 96..127 of
//               the tile); thread = key row j of the tile (TMEM lane), 32 sums each
//   warp 16     TMA producer: per item the transposed bias tile (double
//               buffered by item parity), per row s K, V, Q, dOa high/low,
//               the mask and the two row terms into a 2-stage ring
//   warp 17     MMA issuer of S^T; warp 18 MMA issuer of dP^T, both into a
//               double-buffered TMEM pair (S^T, dP^T), so the MMAs of row
//               s + 1 run while the dS warps work on row s
#pragma once

#include "sm100.cuh"
#include "tma_maps.cuh"

namespace evo {
namespace dbias {

using namespace evo::sm100;

constexpr int BQ = 128;   // query tile (columns of S^T)
constexpr int BK = 128;   // key tile (TMEM lanes)
constexpr int HD = 32;
constexpr int TILE_BYTES = 128 * HD * 2;          // 8 KB, 64-byte rows, 64B swizzle
constexpr int BT_BOX = 128 * 64 * 2;              // 16 KB: 128 key rows x 64 queries, 128B swizzle
constexpr int RT_BYTES = 4096;                    // 16 x 128 bf16 block, 128B swizzle
constexpr int CONST_BYTES = 4096;                 // 128 x 16 bf16 constant block, no swizzle
// one stage per row s (two stages): K, V, Q, dOa high, dOa low, the mask block
// (rows 0 and 8 = mask row of s; MN-major A operand), the nl block (rows 0, 1 =
// high/low of -lse*sqrt(C)) and the -D block (rows 0, 1 = high/low of -D)
constexpr int ST_K = 0, ST_V = TILE_BYTES, ST_Q = 2 * TILE_BYTES, ST_DOH = 3 * TILE_BYTES,
              ST_DOL = 4 * TILE_BYTES, ST_MASK = 5 * TILE_BYTES, ST_NL = ST_MASK + RT_BYTES,
              ST_ND = ST_NL + RT_BYTES, STB = ST_ND + RT_BYTES;
constexpr int OFF_ST = 0;
constexpr int OFF_BT = 2 * STB;                   // transposed bias tile, per item parity
constexpr int OFF_ONES = OFF_BT + 2 * 2 * BT_BOX; // A operand: columns 0 and 1 equal to 1
constexpr int OFF_RROW = OFF_ONES + CONST_BYTES;  // B operand: columns k = 0, 8 equal to r1, r2
constexpr int OFF_BAR = OFF_RROW + CONST_BYTES;
// st_full[2] st_empty[2] bt_full[2] bt_empty[2] s_full[2] dp_full[2] sdp_free[2] mma_done[2]
constexpr int NBARS = 16;
constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory");
// Four dS warpgroups, 32 queries each (more warps per SM hide the latency of the
// per-row chain of TMEM loads, exponentials and sums), then the control warpgroup.
constexpr int NWG = 4;
constexpr int QW = BQ / NWG;                      // queries per dS warpgroup
constexpr int THREADS = 128 * NWG + 128;
constexpr int LAUNCH_REGS = (65536 / THREADS) / 8 * 8;
// The control warpgroup hands registers to the dS warpgroups (with one setmaxnreg per
// warpgroup; the same split without setmaxnreg measured 5-8 % slower).
constexpr uint32_t DS_REGS = 104, CONTROL_REGS = 56;
static_assert((NWG * DS_REGS + CONTROL_REGS) * 128 <= LAUNCH_REGS * THREADS, "register split");
// TMEM: buffer x holds S^T at 256 x and dP^T at 256 x + 128
constexpr uint32_t TM_COLS = 512;
// Every POLY_EVERY-th pair of exponentials runs on the FMA pipe (exp2_poly2)
// instead of the MUFU unit; 0 keeps all of them on MUFU.  The kernel's dS warps are
// bound by instruction issue, not by MUFU: every 2nd, 3rd, 4th or 6th pair on the FMA
// pipe measured 19, 3, 3 and 2 % slower than none.
#ifndef EVO_DBIAS_POLY_EVERY
#define EVO_DBIAS_POLY_EVERY 0
#endif
constexpr int POLY_EVERY = EVO_DBIAS_POLY_EVERY;

// Row groups.  More groups spread a problem with few (b, h, tile) pairs over
// more SMs, but every group beyond the first adds a partial slab that is
// written once and read once more by the finishing pass.  The count is the
// one that minimises a time model of the two, in cycles of a 148-SM B200 at
// its nominal clock: each CTA runs ceil(items / sms) items of ceil(S / g)
// rows at about 1,800 cycles a row, and the slabs move at about 6.5 TB/s;
// more groups are taken only for a gain above 2%.
inline int num_groups(int64_t B, int64_t S, int64_t N, int64_t H, int sms) {
    const int64_t nt = (N + BQ - 1) / BQ;
    const int64_t base = B * H * nt * nt;
    if (base <= 0 || S <= 0 || sms <= 0) return 1;
    const double kRowCycles = 1800.0, kClockHz = 1.965e9, kBytesPerS = 6.5e12;
    const double slab = 4.0 * (double)(B * H) * (double)N * (double)N;
    int best = 1;
    double best_t = 0.0;
    const int64_t gmax = std::min<int64_t>(S, 64);
    for (int64_t g = 1; g <= gmax; ++g) {
        const int64_t gsz = (S + g - 1) / g;
        if ((S + gsz - 1) / gsz != g) continue;        // a group would be empty
        const int64_t waves = (base * g + sms - 1) / sms;
        double t = (double)waves * (double)gsz * kRowCycles / kClockHz;
        if (g > 1) t += (2.0 * (double)g + 1.0) * slab / kBytesPerS;   // slabs written, read, sum written
        if (g == 1 || t < 0.98 * best_t) {              // more slabs only for a real gain
            best_t = t;
            best = (int)g;
        }
    }
    return best;
}

struct Params {
    int B, S, N, H;
    int n_t;             // tiles along the query (= key) axis
    int gsz, groups;     // rows s per group, groups
    int n_items;         // B * H * n_t * n_t * groups
    float sc2;           // log2(e) / sqrt(C)
    float bsc;           // log2(e) * r1 / sqrt(C): the pair bias enters as the forward's tensor core adds it
    float r_bf16, r2_bf16;
    float* out;          // [groups, B, H, N, N] partial slabs, or d_pair_bias when groups == 1
    uint64_t wait_ns;
};

struct Item {
    int b, h, it, jt, g;
};
// Items are numbered with the key tile fastest, then the query tile, then the
// row group, then (b, h): CTAs running side by side share the rows' K, V, Q and
// output-gradient tiles in L2.
__device__ __forceinline__ Item decode(const Params& p, int item) {
    Item x;
    x.jt = item % p.n_t;
    int r = item / p.n_t;
    x.it = r % p.n_t;
    r /= p.n_t;
    x.g = r % p.groups;
    const int bh = r / p.groups;
    x.b = bh / p.H;
    x.h = bh % p.H;
    return x;
}

enum : unsigned int { kTimeoutBase = 0x3000u };

template <bool HAS_MASK, bool HAS_BIAS>
__global__ void __launch_bounds__(THREADS, 1)
    dbias_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_doa,
                 const __grid_constant__ CUtensorMap tm_dol, const __grid_constant__ CUtensorMap tm_bt,
                 const __grid_constant__ CUtensorMap tm_mask, const __grid_constant__ CUtensorMap tm_nl,
                 const __grid_constant__ CUtensorMap tm_d, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kDsWarps = 4 * NWG, kProducer = kDsWarps, kMmaS = kDsWarps + 1, kMmaD = kDsWarps + 2;

    const uint32_t bar0 = base + OFF_BAR;
    auto st_full = [&](int x) { return bar0 + 8u * (0 + x); };
    auto st_empty = [&](int x) { return bar0 + 8u * (2 + x); };
    auto bt_full = [&](int x) { return bar0 + 8u * (4 + x); };
    auto bt_empty = [&](int x) { return bar0 + 8u * (6 + x); };
    auto s_full = [&](int x) { return bar0 + 8u * (8 + x); };
    auto dp_full = [&](int x) { return bar0 + 8u * (10 + x); };
    auto sdp_free = [&](int x) { return bar0 + 8u * (12 + x); };
    auto mma_done = [&](int x) { return bar0 + 8u * (14 + x); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(st_full(x), 1);
            mbar_init(st_empty(x), 2);      // one commit per MMA issuer
            mbar_init(bt_full(x), 1);
            mbar_init(bt_empty(x), kDsWarps);   // one arrival per dS warp
            mbar_init(s_full(x), 1);
            mbar_init(dp_full(x), 1);
            mbar_init(sdp_free(x), kDsWarps);
            mbar_init(mma_done(x), 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kProducer && lane == 0) {
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_doa);
        prefetch_tmap(&tm_dol); prefetch_tmap(&tm_nl); prefetch_tmap(&tm_d);
        if (HAS_BIAS) prefetch_tmap(&tm_bt);
        if (HAS_MASK) prefetch_tmap(&tm_mask);
    }
    if (warp == kMmaS) {
        tmem_alloc(base + OFF_MISC, TM_COLS);
        tmem_relinquish();
    }
    if (warp < kDsWarps) {
        // Constant operands, and the zero rows of the per-stage blocks (the TMA
        // writes only rows 0..1 of the nl / -D blocks and rows 0, 8 of the mask
        // block).  No-swizzle K-major element (row, k) sits at
        // (row%8)*16 + (row/8)*256 + (k/8)*128 + (k%8)*2.
        const int t = threadIdx.x;
        constexpr int nt = 32 * kDsWarps;
        auto zero = [&](int off, int bytes) {
            for (int o = t * 16; o < bytes; o += nt * 16)
                *reinterpret_cast<uint4*>(gbase + off + o) = make_uint4(0u, 0u, 0u, 0u);
        };
        zero(OFF_ONES, CONST_BYTES);
        zero(OFF_RROW, CONST_BYTES);
        for (int x = 0; x < 2; ++x) {
            zero(OFF_ST + x * STB + ST_MASK, RT_BYTES);
            zero(OFF_ST + x * STB + ST_NL, RT_BYTES);
            zero(OFF_ST + x * STB + ST_ND, RT_BYTES);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(nt) : "memory");
        if (t < 128) {
            const uint16_t one = 0x3F80u;
            const uint16_t rb = (uint16_t)(__float_as_uint(p.r_bf16) >> 16);
            const uint16_t rb2 = (uint16_t)(__float_as_uint(p.r2_bf16) >> 16);
            uint8_t* o = gbase + OFF_ONES + (t % 8) * 16 + (t / 8) * 256;
            reinterpret_cast<uint16_t*>(o)[0] = one;   // k = 0
            reinterpret_cast<uint16_t*>(o)[1] = one;   // k = 1
            uint8_t* rr = gbase + OFF_RROW + (t % 8) * 16 + (t / 8) * 256;
            *reinterpret_cast<uint16_t*>(rr) = rb;          // k = 0
            *reinterpret_cast<uint16_t*>(rr + 128) = rb2;   // k = 8
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // setmaxnreg is warpgroup-wide: all four warps of a warpgroup execute the same
    // instruction, so each warpgroup changes its count before its warps' roles split.
    if (warp >= kDsWarps) {
        regs_decrease<CONTROL_REGS>();
        if (warp == kProducer) {
            // ---------------------------------------------------------------- producer
            if (lane == 0) {
                constexpr uint32_t tx = 5 * TILE_BYTES + 4 * 256 + (HAS_MASK ? 4 * 128 : 0);
                int st_issued[2] = {0, 0}, bt_issued[2] = {0, 0};
                int tg = 0;
                bool ok = true;
                for (int item = blockIdx.x, k = 0; ok && item < p.n_items; item += gridDim.x, ++k) {
                    const Item x = decode(p, item);
                    const int i0 = x.it * BQ, j0 = x.jt * BK;
                    const int s0 = x.g * p.gsz, ns = min(p.gsz, p.S - s0);
                    if (HAS_BIAS) {
                        const int bb = k & 1;
                        if (k >= 2) ok = mbar_wait(bt_empty(bb), ((k >> 1) - 1) & 1, abort_flag, kTimeoutBase | 0x01, p.wait_ns);
                        if (!ok) break;
                        mbar_arrive_expect_tx(bt_full(bb), 2 * BT_BOX);
                        const uint32_t bt = base + OFF_BT + bb * 2 * BT_BOX;
                        tma_load_4d(bt, &tm_bt, bt_full(bb), i0, j0, x.h, x.b);
                        tma_load_4d(bt + BT_BOX, &tm_bt, bt_full(bb), i0 + 64, j0, x.h, x.b);
                        ++bt_issued[bb];
                    }
                    for (int si = 0; si < ns; ++si, ++tg) {
                        const int s = s0 + si, st = tg & 1;
                        const uint32_t sb = base + OFF_ST + st * STB;
                        if (tg >= 2) ok = mbar_wait(st_empty(st), ((tg >> 1) - 1) & 1, abort_flag, kTimeoutBase | 0x02, p.wait_ns);
                        if (!ok) break;
                        mbar_arrive_expect_tx(st_full(st), tx);
                        tma_load_5d(sb + ST_K, &tm_k, st_full(st), 0, j0, x.h, s, x.b);
                        tma_load_5d(sb + ST_V, &tm_v, st_full(st), 0, j0, x.h, s, x.b);
                        tma_load_5d(sb + ST_Q, &tm_q, st_full(st), 0, i0, x.h, s, x.b);
                        tma_load_5d(sb + ST_DOH, &tm_doa, st_full(st), 0, i0, x.h, s, x.b);
                        tma_load_5d(sb + ST_DOL, &tm_dol, st_full(st), 0, i0, x.h, s, x.b);
                        if (HAS_MASK) {   // rows 0 and 8 of the two 64-key halves of the A block
                            tma_load_3d(sb + ST_MASK, &tm_mask, st_full(st), j0, s, x.b);
                            tma_load_3d(sb + ST_MASK + 1024, &tm_mask, st_full(st), j0, s, x.b);
                            tma_load_3d(sb + ST_MASK + 2048, &tm_mask, st_full(st), j0 + 64, s, x.b);
                            tma_load_3d(sb + ST_MASK + 3072, &tm_mask, st_full(st), j0 + 64, s, x.b);
                        }
                        // rows 0..1 (high, low) of the two 64-query atoms of the nl and -D blocks
                        tma_load_5d(sb + ST_NL, &tm_nl, st_full(st), i0, 0, x.h, s, x.b);
                        tma_load_5d(sb + ST_NL + 2048, &tm_nl, st_full(st), i0 + 64, 0, x.h, s, x.b);
                        tma_load_5d(sb + ST_ND, &tm_d, st_full(st), i0, 0, x.h, s, x.b);
                        tma_load_5d(sb + ST_ND + 2048, &tm_d, st_full(st), i0 + 64, 0, x.h, s, x.b);
                        ++st_issued[st];
                    }
                }
                // Never leave with copies in flight: wait (bounded) for the last fill of every buffer.
                volatile int no_abort = 0;
                for (int x = 0; x < 2; ++x) {
                    if (st_issued[x]) mbar_wait(st_full(x), (st_issued[x] - 1) & 1, &no_abort, kTimeoutBase | 0x03);
                    if (bt_issued[x]) mbar_wait(bt_full(x), (bt_issued[x] - 1) & 1, &no_abort, kTimeoutBase | 0x04);
                }
            }
        } else if (warp == kMmaS || warp == kMmaD) {
            // ---------------------------------------------------------------- MMA issuers
            const int role = warp - kMmaS;   // 0: S^T, 1: dP^T
            if (lane == 0) {
                constexpr uint32_t ID_SS = idesc_bf16(BK, BQ, false, false);   // K Q^T, V dOa^T
                constexpr uint32_t ID_RT = idesc_bf16(BK, BQ, false, true);    // ones x row-term block
                constexpr uint32_t ID_MK = idesc_bf16(BK, BQ, true, false);    // mask block x r-row
                bool ok = true;
                int tg = 0;
                for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
                    const Item x = decode(p, item);
                    const int ns = min(p.gsz, p.S - x.g * p.gsz);
                    for (int si = 0; si < ns; ++si, ++tg) {
                        const int st = tg & 1, buf = tg & 1;
                        ok = mbar_wait(st_full(st), (tg >> 1) & 1, abort_flag, kTimeoutBase | (0x11 + role), p.wait_ns);
                        if (ok && tg >= 2)
                            ok = mbar_wait(sdp_free(buf), ((tg >> 1) - 1) & 1, abort_flag, kTimeoutBase | (0x13 + role), p.wait_ns);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t sb = base + OFF_ST + st * STB;
                        const uint32_t d = tmem + 256u * (uint32_t)buf + (role == 0 ? 0u : 128u);
                        if (role == 0) {
                            // S^T = K Q^T - lse*sqrt(C) (+ (r1 + r2) * mask_j)
#pragma unroll
                            for (int kk = 0; kk < HD / 16; ++kk)
                                mma_ss(d, smem_desc(sb + ST_K + kk * 32, 16, 512, kSw64),
                                       smem_desc(sb + ST_Q + kk * 32, 16, 512, kSw64), ID_SS, kk > 0);
                            mma_ss(d, smem_desc(base + OFF_ONES, 128, 256, kSwNone),
                                   smem_desc(sb + ST_NL, 2048, 1024, kSw128), ID_RT, 1u);
                            if (HAS_MASK)
                                mma_ss(d, smem_desc(sb + ST_MASK, 2048, 1024, kSw128),
                                       smem_desc(base + OFF_RROW, 128, 256, kSwNone), ID_MK, 1u);
                            mma_commit(s_full(buf));
                        } else {
                            // dP^T = V (dOa_hi + dOa_lo)^T - D
#pragma unroll
                            for (int kk = 0; kk < HD / 16; ++kk)
                                mma_ss(d, smem_desc(sb + ST_V + kk * 32, 16, 512, kSw64),
                                       smem_desc(sb + ST_DOH + kk * 32, 16, 512, kSw64), ID_SS, kk > 0);
#pragma unroll
                            for (int kk = 0; kk < HD / 16; ++kk)
                                mma_ss(d, smem_desc(sb + ST_V + kk * 32, 16, 512, kSw64),
                                       smem_desc(sb + ST_DOL + kk * 32, 16, 512, kSw64), ID_SS, 1u);
                            mma_ss(d, smem_desc(base + OFF_ONES, 128, 256, kSwNone),
                                   smem_desc(sb + ST_ND, 2048, 1024, kSw128), ID_RT, 1u);
                            mma_commit(dp_full(buf));
                        }
                        mma_commit(st_empty(st));    // this issuer no longer reads the stage
                    }
                }
                // Drain: every MMA issued by this thread has finished before TMEM is released.
                mma_commit(mma_done(role));
                volatile int no_abort = 0;
                mbar_wait(mma_done(role), 0, &no_abort, kTimeoutBase | (0x15 + role));
            }
        }
    } else {
        regs_increase<DS_REGS>();
        // ---------------------------------------------------------------- dS warpgroups
        const int wg = warp >> 2;                // queries 32 wg .. 32 wg + 31 of the tile
        const int quad = warp & 3;
        const int r = quad * 32 + lane;          // key row within the tile = TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(wg * QW);
        const uint64_t SC2 = f2(p.sc2, p.sc2);
        const uint64_t L2E2 = f2(p.bsc, p.bsc);
        bool ok = true;
        int tg = 0;
        for (int item = blockIdx.x, k = 0; ok && item < p.n_items; item += gridDim.x, ++k) {
            const Item x = decode(p, item);
            const int i0 = x.it * BQ, j0 = x.jt * BK;
            const int ns = min(p.gsz, p.S - x.g * p.gsz);
            const int j = j0 + r;
            const bool jvalid = j < p.N;
            const int bb = k & 1;
            if (HAS_BIAS) {
                ok = mbar_wait(bt_full(bb), (k >> 1) & 1, abort_flag, kTimeoutBase | 0x21, p.wait_ns);
                if (!ok) break;
            }
            // this warpgroup's 32 queries: 64-query box wg / 2, 16-byte chunks 4 (wg % 2) .. + 3
            const uint8_t* bt_ptr = gbase + OFF_BT + bb * 2 * BT_BOX + (wg >> 1) * BT_BOX + r * 128;
            uint64_t acc[QW / 2];
#pragma unroll
            for (int c = 0; c < QW / 2; ++c) acc[c] = 0;
            for (int si = 0; si < ns; ++si, ++tg) {
                const int buf = tg & 1;
                ok = mbar_wait(s_full(buf), (tg >> 1) & 1, abort_flag, kTimeoutBase | 0x22, p.wait_ns);
                if (ok) ok = mbar_wait(dp_full(buf), (tg >> 1) & 1, abort_flag, kTimeoutBase | 0x23, p.wait_ns);
                if (!ok) break;
                tc_fence_after();
                const uint32_t ts = lane_addr + 256u * (uint32_t)buf;
                // 16 queries at a time: cur[0,16) S^T columns, cur[16,32) dP^T columns
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t cur[32];
                    tmem_ld16x2_sync(ts + 16 * hf, ts + 128 + 16 * hf, cur);
                    if (hf == 1) {                       // both halves of this buffer in registers
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(sdp_free(buf));
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {        // 8 queries (one 16-byte bias chunk) at a time
                        uint32_t bw[4] = {0u, 0u, 0u, 0u};
                        if (HAS_BIAS) {
                            const int ch = (wg & 1) * 4 + hf * 2 + q;
                            const uint4 w = *reinterpret_cast<const uint4*>(
                                bt_ptr + (((uint32_t)ch ^ (uint32_t)(r & 7)) << 4));
                            bw[0] = w.x; bw[1] = w.y; bw[2] = w.z; bw[3] = w.w;
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = q * 8 + 2 * e;          // column within the half
                            const int pr = hf * 8 + q * 4 + e;    // column pair within the 32
                            uint64_t y2 = fmul2(f2(__uint_as_float(cur[c]), __uint_as_float(cur[c + 1])), SC2);
                            if (HAS_BIAS) y2 = ffma2(bf16x2_to_f2(bw[e]), L2E2, y2);
                            uint64_t p2;
                            if (POLY_EVERY > 0 && pr % (POLY_EVERY > 0 ? POLY_EVERY : 1) == POLY_EVERY - 1)
                                p2 = exp2_poly2(y2);
                            else
                                p2 = f2(ex2(f2lo(y2)), ex2(f2hi(y2)));
                            const uint64_t ds2 =
                                fmul2(p2, f2(__uint_as_float(cur[16 + c]), __uint_as_float(cur[17 + c])));
                            acc[pr] = fadd2(acc[pr], ds2);
                        }
                    }
                }
            }
            if (!ok) break;
            if (HAS_BIAS) {                      // the item's bias tile is no longer read
                fence_proxy_async_smem();        // generic reads before the TMA's refill of the buffer
                __syncwarp();
                if (lane == 0) mbar_arrive(bt_empty(bb));
            }
            // d_pair_bias[b, h, i, j] for i = i0 + 32 wg + c: one column j per thread, so each
            // store of the warp covers 32 consecutive j (128 bytes).
            if (jvalid) {
                float* dst = p.out + ((int64_t)x.g * p.B * p.H + (int64_t)x.b * p.H + x.h) * p.N * p.N +
                             (int64_t)(i0 + wg * QW) * p.N + j;
                const int ivalid = min(QW, p.N - i0 - wg * QW);
#pragma unroll
                for (int c = 0; c < QW / 2; ++c) {
                    if (2 * c < ivalid) dst[(int64_t)(2 * c) * p.N] = f2lo(acc[c]);
                    if (2 * c + 1 < ivalid) dst[(int64_t)(2 * c + 1) * p.N] = f2hi(acc[c]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaS) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

}  // namespace dbias
}  // namespace evo
