// bwd_sm100.cuh -- bf16 backward of Evoformer pair-bias attention on sm_100a.
//
// Like the forward, the backward never stores a logit: P is recomputed tile
// by tile from q, k, the biases and the saved log-sum-exp, which is how
// EvoFlash-3D treats the backward pass (MegaFold summary, section
// "EvoFlash-3D": logits computed incrementally in on-chip memory in the
// forward and the backward passes).
//
// Kernels (one stream, in order):
//   bwd_prep       one launch, by block range:
//                  per logit row: D_i = sum_c dout*out, dOa = dout*sigmoid(g)
//                  split into a bf16 high part and a bf16 low part (their sum
//                  carries ~16 mantissa bits into dP), dg = dout*out*(1-sigmoid(g)),
//                  nl_i = -lse_i*sqrt(C); zeroes the fp32 dq accumulator.  Four
//                  threads per row, 16-byte accesses.  The row terms nl and -D
//                  are stored with the query axis padded to whole tiles, padding
//                  nl = -1e30, so padded queries get P = 0;
//                  pair_bias[b,h,i,j] -> biasT[b,h,j,i] (bf16), so that the
//                  main kernel reads bias rows along its TMEM lanes (keys);
//   bwd_main       CTA = (key tile j, row group g, b*H + h); loops over the
//                  group's rows s (outer) and query tiles i (inner):
//                    S^T  = K_j Q_i^T      dP^T = V_j (dOa_hi + dOa_lo)_i^T  (TMEM)
//                    P^T  = exp2(S^T*scale*log2e + bias*log2e*r1/sqrt(C) + mask + nl_i)
//                    (the pair bias with the scale the forward's tensor core gives it,
//                    r1 = bf16(sqrt(C)), so that P matches the forward's lse)
//                    dS^T = P^T (dP^T - D_i)
//                    dV_j += P^T dOa_hi_i  dK_j += dS^T Q_i         (TMEM)
//                    dQ_i  = dS K_j  -> fp32 atomic add into the accumulator
//                  The P^T TMEM tile is double-buffered by step parity, so the dS
//                  warps write step t while dV of step t-1 still reads the other
//                  buffer; the dS^T tile in shared memory is single-buffered (dK and
//                  dQ of step t-1 finish before the dS warps store step t's).
//   dbias          d_pair_bias, summed over the rows s on chip (dbias_sm100.cuh):
//                  one partial slab per row group, plain stores.
//   bwd_post       one launch: dq = bf16(accumulator); d_pair_bias = sum over
//                  the row groups' slabs in group order (when there are several).
// The result of d_pair_bias is therefore bitwise reproducible; dq's last bits
// depend on the order of the atomic adds.
#pragma once

#include "sm100.cuh"
#include "tma_maps.cuh"
#include "dbias_sm100.cuh"

namespace evo {
namespace bwd {

using namespace evo::sm100;

constexpr int BQ = 128;   // query tile (columns of S^T)
constexpr int BK = 128;   // key tile (TMEM lanes)
constexpr int HD = 32;
constexpr int TILE_BYTES = 128 * HD * 2;          // 8 KB, 64-byte rows, 64B swizzle
constexpr int BT_BOX = 128 * 64 * 2;              // 16 KB: 128 key rows x 64 queries, 128B swizzle
constexpr int RT_BYTES = 4096;                    // 16 x 128 bf16 rank-term block, 128B swizzle
constexpr int CONST_BYTES = 4096;                 // 128 x 16 bf16 constant block, no swizzle
// per row s (double-buffered): K, V, mask block (row 0 = mask row of s; MN-major A operand)
constexpr int KV_K = 0, KV_V = TILE_BYTES, KV_MASK = 2 * TILE_BYTES, KVB = 2 * TILE_BYTES + RT_BYTES;
// Per step (query tile of a row s), two rings with different lifetimes, so that
// the next steps' loads are not held back by the last products of this one:
//   ring X (2 stages): transposed bias tile, dOa low part, nl block (rows 0,1 =
//     high/low of -lse*sqrt(C)) and -D block (rows 0,1 = high/low of -D); read
//     by the S^T / dP^T products and the dS warps' bias adds, released early
//   ring Y (3 stages): Q and dOa high part; read also by dK and dV, released late
constexpr int X_BT = 0, X_DOL = 2 * BT_BOX, X_NL = X_DOL + TILE_BYTES, X_ND = X_NL + RT_BYTES,
              XB = X_ND + RT_BYTES;
constexpr int Y_Q = 0, Y_DOH = TILE_BYTES, YB = 2 * TILE_BYTES;
constexpr int X_STAGES = 2, Y_STAGES = 3;
constexpr int OFF_KV = 0;
constexpr int OFF_X = 2 * KVB;
constexpr int OFF_Y = OFF_X + X_STAGES * XB;
constexpr int OFF_DS = OFF_Y + Y_STAGES * YB;      // dS^T tile, 2 boxes of 128 rows x 128 B
constexpr int DS_BYTES = 2 * BT_BOX;
constexpr int OFF_ONES = OFF_DS + DS_BYTES;        // A operand: columns 0 and 1 equal to 1
constexpr int OFF_RROW = OFF_ONES + CONST_BYTES;   // B operand: columns k = 0, 8 equal to r1, r2 (sum sqrt(C))
constexpr int OFF_BAR = OFF_RROW + CONST_BYTES;
// kv_full[2] kv_empty[2] x_full[2] x_empty[2] y_full[3] y_empty[3] sdp_full sdp_free ds_full[2]
// (18, 19 unused) ds_free dq_full dq_free dkv_full dkv_free mma_done[3]
constexpr int NBARS = 28;
constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory");
// Warps 0..15: four dS warpgroups, warpgroup w taking queries 32 w .. 32 w + 31 of the
// tile (each dS warp's per-step chain of waits, loads, exponentials and stores is
// mostly latency, which more warps per SM overlap); warp 16 TMA; three MMA issuers,
// so that no single issuing thread serialises a step's 33 instructions: warp 17 S^T
// and dP^T of the next step, warp 18 dV and dK, warp 19 dQ.  Warps 20..23 drain: each
// step's 128 x 32 fp32 dQ goes from TMEM into the global fp32 accumulator with vector
// reductions, and each row's dK and dV into their outputs, off the dS warps' path.
// Registers: 4*128*96 + 128*56 + 128*40 = 768*80, the launch's register pool (no spills).
constexpr int NWG = 4;                       // dS warpgroups
constexpr int QW = BQ / NWG;                 // queries per dS warpgroup
constexpr int DS_WARPS = 4 * NWG;
constexpr int THREADS = 128 * NWG + 256;
constexpr int LAUNCH_REGS = (65536 / THREADS) / 8 * 8;
constexpr uint32_t DS_REGS = 96, CONTROL_REGS = 56, DRAIN_REGS = 40;
static_assert((NWG * DS_REGS + CONTROL_REGS + DRAIN_REGS) * 128 <= LAUNCH_REGS * THREADS, "register split");
// TMEM columns: S^T, dP^T, two P^T buffers (bf16 pairs), dV, dK, dQ accumulators
constexpr uint32_t TM_ST = 0, TM_DPT = 128, TM_PT = 256, TM_DV = 384, TM_DK = 416, TM_DQ = 448, TM_COLS = 512;

// Row groups of the main kernel: about one CTA (key tile x head x batch x
// group) per SM of a 148-SM B200, in one wave.
inline int num_groups(int64_t B, int64_t S, int64_t N, int64_t H) {
    const int64_t njt = (N + BK - 1) / BK;
    const int64_t base = njt * B * H;
    if (base <= 0 || S <= 0) return 1;
    int64_t g = 148 / base;
    if (g > S) g = S;
    if (g < 1) g = 1;
    const int64_t gsz = (S + g - 1) / g;       // rows per group; drop groups left empty
    return (int)((S + gsz - 1) / gsz);
}

struct MainParams {
    int B, S, N, H;
    int n_it;            // query tiles
    int gsz;             // rows s per group
    float sc2;           // log2(e) / sqrt(C)
    float bsc;           // log2(e) * r1 / sqrt(C): the pair bias enters as the forward's tensor core adds it
    float rs;            // 1 / sqrt(C)
    float r_bf16;        // r1 = bf16(sqrt(C))
    float r2_bf16;       // r2 = bf16(sqrt(C) - r1): the mask enters as (r1 + r2) * mask
    float* dq_acc;       // [B,S,N,H,C] fp32, contiguous
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    Strides gs;
};

enum : unsigned int { kTimeoutBase = 0x2000u };

template <bool HAS_MASK, bool HAS_BIAS>
__global__ void __launch_bounds__(THREADS, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_doa,
                    const __grid_constant__ CUtensorMap tm_dol, const __grid_constant__ CUtensorMap tm_bt,
                    const __grid_constant__ CUtensorMap tm_mask, const __grid_constant__ CUtensorMap tm_nl,
                    const __grid_constant__ CUtensorMap tm_d, const MainParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kProducer = DS_WARPS, kMma = DS_WARPS + 1;   // issuers: kMma (S^T, dP^T), + 1 (dV, dK), + 2 (dQ)
    const int j0 = blockIdx.x * BK;
    const int grp = blockIdx.y;
    const int b = blockIdx.z / p.H, h = blockIdx.z % p.H;
    const int s_begin = grp * p.gsz;
    const int ns = min(p.gsz, p.S - s_begin);
    const int ni = p.n_it;
    const int T = ns * ni;

    const uint32_t bar0 = base + OFF_BAR;
    auto kv_full = [&](int x) { return bar0 + 8u * (0 + x); };
    auto kv_empty = [&](int x) { return bar0 + 8u * (2 + x); };
    auto x_full = [&](int x) { return bar0 + 8u * (4 + x); };
    auto x_empty = [&](int x) { return bar0 + 8u * (6 + x); };
    auto y_full = [&](int x) { return bar0 + 8u * (8 + x); };
    auto y_empty = [&](int x) { return bar0 + 8u * (11 + x); };
    const uint32_t sdp_full = bar0 + 8u * 14, sdp_free = bar0 + 8u * 15;
    // ds_full[t & 1]: dS^T of step t in shared memory and P^T in TMEM (one barrier per step
    // parity, because two issuers consume it and the dS warps may run a step ahead of one)
    auto ds_full = [&](int x) { return bar0 + 8u * (16 + x); };
    const uint32_t ds_free = bar0 + 8u * 20;
    const uint32_t dq_full = bar0 + 8u * 21, dq_free = bar0 + 8u * 22;
    const uint32_t dkv_full = bar0 + 8u * 23, dkv_free = bar0 + 8u * 24;
    auto mma_done = [&](int x) { return bar0 + 8u * (25 + x); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_MISC + 4);

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(kv_full(x), 1);
            mbar_init(kv_empty(x), 2);            // K and V read by the S^T / dP^T issuer and the dQ issuer
            mbar_init(x_full(x), 1);
            mbar_init(x_empty(x), 1 + DS_WARPS);  // the S^T / dP^T issuer and the dS warps (bias)
            mbar_init(ds_full(x), DS_WARPS);
        }
        for (int x = 0; x < Y_STAGES; ++x) {
            mbar_init(y_full(x), 1);
            mbar_init(y_empty(x), 2);             // the S^T / dP^T and the dV / dK issuers
        }
        mbar_init(sdp_full, 1);
        mbar_init(sdp_free, DS_WARPS);
        mbar_init(ds_free, 2);                    // dK and dQ read the dS^T tile
        mbar_init(dq_full, 1);
        mbar_init(dq_free, 4);                    // the dQ drain warps
        mbar_init(dkv_full, 1);
        mbar_init(dkv_free, 4);                   // the drain warps
        for (int x = 0; x < 3; ++x) mbar_init(mma_done(x), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kProducer && lane == 0) {
        prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); prefetch_tmap(&tm_doa);
        prefetch_tmap(&tm_dol); prefetch_tmap(&tm_nl); prefetch_tmap(&tm_d);
        if (HAS_BIAS) prefetch_tmap(&tm_bt);
        if (HAS_MASK) prefetch_tmap(&tm_mask);
    }
    if (warp == kMma) {
        tmem_alloc(base + OFF_MISC, TM_COLS);
        tmem_relinquish();
    }
    if (warp < 8) {
        // Constant operands and the zero rows of the rank-term blocks (the TMA
        // writes only rows 0..1 of the nl / -D blocks and row 0 of a mask block).
        // No-swizzle K-major element (row, k): (row%8)*16 + (row/8)*256 + (k/8)*128 + (k%8)*2.
        const int t = threadIdx.x;
        auto zero = [&](int off, int bytes) {
            for (int o = t * 16; o < bytes; o += 256 * 16)
                *reinterpret_cast<uint4*>(gbase + off + o) = make_uint4(0u, 0u, 0u, 0u);
        };
        zero(OFF_ONES, CONST_BYTES);
        zero(OFF_RROW, CONST_BYTES);
        for (int x = 0; x < 2; ++x) {
            zero(OFF_KV + x * KVB + KV_MASK, RT_BYTES);
            zero(OFF_X + x * XB + X_NL, RT_BYTES);
            zero(OFF_X + x * XB + X_ND, RT_BYTES);
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (t < 128) {
            const uint16_t one = 0x3F80u;
            const uint16_t rb = (uint16_t)(__float_as_uint(p.r_bf16) >> 16);
            const uint16_t rb2 = (uint16_t)(__float_as_uint(p.r2_bf16) >> 16);
            uint8_t* o = gbase + OFF_ONES + (t % 8) * 16 + (t / 8) * 256;
            reinterpret_cast<uint16_t*>(o)[0] = one;   // k = 0
            reinterpret_cast<uint16_t*>(o)[1] = one;   // k = 1
            *reinterpret_cast<uint16_t*>(gbase + OFF_RROW + (t % 8) * 16 + (t / 8) * 256) = rb;
            *reinterpret_cast<uint16_t*>(gbase + OFF_RROW + (t % 8) * 16 + (t / 8) * 256 + 128) = rb2;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // setmaxnreg is warpgroup-wide: all four warps of a warpgroup execute the same
    // instruction, so each warpgroup changes its count before its warps' roles split.
    if (warp >= DS_WARPS + 4) {
        regs_decrease<DRAIN_REGS>();
        // ---------------------------------------------------------------- drain warps
        // dQ_i of step t (lanes = queries) into the fp32 accumulator, scaled by 1/sqrt(C);
        // at the end of each row s, dK_j and dV_j (lanes = keys) into their bf16 outputs.
        // The reductions are the kernel's heaviest traffic (one per element of dQ per key
        // tile): a 16-byte reduction that covers half of a 32-byte sector costs the L2 about
        // as much as a whole sector, so neighbouring lanes first trade halves (see below).
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int j = j0 + r;
        const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
        // dK / dV rows 16 columns (32 bytes) at a time, 8 columns per TMEM load (the drain warps
        // run on 40 registers; the accumulators are released once their last columns are in
        // registers); lanes 2m, 2m+1 (key rows 2m, 2m+1) trade halves, so each store of the
        // warp writes whole 32-byte sectors of 16 rows
        auto drain_dkv = [&](int si) -> bool {
            if (!mbar_wait(dkv_full, si & 1, abort_flag, kTimeoutBase | 0x22)) return false;
            tc_fence_after();
            const bool odd = (lane & 1) != 0;
            const int j_even = j & ~1;
            const bool ok_e = j_even < p.N, ok_o = j_even + 1 < p.N;
            const int64_t rs_n = p.gs.n;
#pragma unroll
            for (int part = 0; part < 4; ++part) {   // dK columns 0..15, 16..31, then dV's
                const float f = part < 2 ? p.rs : 1.0f;
                uint32_t w[2][4];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t v[8];
                    tmem_ld8_sync(lane_addr + (part < 2 ? TM_DK : TM_DV) + (part & 1) * 16 + 8 * q, v);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[q][e] = pack_bf16(__uint_as_float(v[2 * e]) * f, __uint_as_float(v[2 * e + 1]) * f);
                }
                if (part == 3) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(dkv_free);
                }
                uint32_t rcv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) rcv[e] = __shfl_xor_sync(0xffffffffu, odd ? w[0][e] : w[1][e], 1);
                __nv_bfloat16* row_even = (part < 2 ? p.dk : p.dv) + p.gs.off(b, s_begin + si, ok_e ? j_even : 0, h) +
                                          (part & 1) * 16 + (odd ? 8 : 0);
                if (ok_e)                            // even row: low half from the even lane, high from the odd
                    *reinterpret_cast<uint4*>(row_even) = odd ? make_uint4(rcv[0], rcv[1], rcv[2], rcv[3])
                                                              : make_uint4(w[0][0], w[0][1], w[0][2], w[0][3]);
                if (ok_o)                            // odd row
                    *reinterpret_cast<uint4*>(row_even + rs_n) = odd ? make_uint4(w[1][0], w[1][1], w[1][2], w[1][3])
                                                                     : make_uint4(rcv[0], rcv[1], rcv[2], rcv[3]);
            }
            return true;
        };
        for (int t = 0; t < T; ++t) {
            if (!mbar_wait(dq_full, t & 1, abort_flag, kTimeoutBase | 0x21)) break;
            tc_fence_after();
            const int si = t / ni, it = t - si * ni;
            const int i = it * BQ + r, s = s_begin + si;
            const bool odd = (lane & 1) != 0;
            const int i_even = i & ~1;
            const int64_t row_stride = (int64_t)p.H * HD;
            float* dst_even = p.dq_acc + ((((int64_t)b * p.S + s) * p.N + (i_even < p.N ? i_even : 0)) * p.H + h) * HD;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t v[16];
                tmem_ld16_sync(lane_addr + TM_DQ + hf * 16, v);
                if (hf == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(dq_free);
                }
                // lanes 2m and 2m+1 hold query rows 2m and 2m+1; they trade half of each 32-byte
                // sector of their rows, so that each vector reduction of the warp covers whole
                // sectors of 16 rows: the even lane reduces low halves, the odd lane high halves
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float lo[4], hi[4], recv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        lo[e] = __uint_as_float(v[8 * k + e]) * p.rs;
                        hi[e] = __uint_as_float(v[8 * k + 4 + e]) * p.rs;
                        recv[e] = __shfl_xor_sync(0xffffffffu, odd ? lo[e] : hi[e], 1);
                    }
                    const int col = hf * 16 + 8 * k + (odd ? 4 : 0);
                    if (i_even < p.N)        // even row: its low half from the even lane, high half from the odd
                        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst_even + col),
                                     "f"(odd ? recv[0] : lo[0]), "f"(odd ? recv[1] : lo[1]),
                                     "f"(odd ? recv[2] : lo[2]), "f"(odd ? recv[3] : lo[3]) : "memory");
                    if (i_even + 1 < p.N)    // odd row: its low half from the even lane, high half from the odd
                        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst_even + row_stride + col),
                                     "f"(odd ? hi[0] : recv[0]), "f"(odd ? hi[1] : recv[1]),
                                     "f"(odd ? hi[2] : recv[2]), "f"(odd ? hi[3] : recv[3]) : "memory");
                }
            }
            if (it == ni - 1 && !drain_dkv(si)) break;
        }
    } else if (warp >= DS_WARPS) {
        regs_decrease<CONTROL_REGS>();
        if (warp == kProducer) {
            // ---------------------------------------------------------------- producer
            if (lane == 0 && T > 0) {
                int kv_issued[2] = {0, 0}, x_issued[X_STAGES] = {}, y_issued[Y_STAGES] = {};
                bool ok = true;
                for (int si = 0; si < ns && ok; ++si) {
                    const int s = s_begin + si, x = si & 1;
                    const uint32_t kb = base + OFF_KV + x * KVB;
                    if (si >= 2) ok = mbar_wait(kv_empty(x), ((si >> 1) - 1) & 1, abort_flag, kTimeoutBase | 0x01);
                    if (!ok) break;
                    mbar_arrive_expect_tx(kv_full(x), 2 * TILE_BYTES + (HAS_MASK ? 512 : 0));
                    tma_load_5d(kb + KV_K, &tm_k, kv_full(x), 0, j0, h, s, b);
                    tma_load_5d(kb + KV_V, &tm_v, kv_full(x), 0, j0, h, s, b);
                    if (HAS_MASK) {   // mask row of s into rows 0 and 8 of the two 64-key halves of the A block
                        tma_load_3d(kb + KV_MASK, &tm_mask, kv_full(x), j0, s, b);
                        tma_load_3d(kb + KV_MASK + 1024, &tm_mask, kv_full(x), j0, s, b);
                        tma_load_3d(kb + KV_MASK + 2048, &tm_mask, kv_full(x), j0 + 64, s, b);
                        tma_load_3d(kb + KV_MASK + 3072, &tm_mask, kv_full(x), j0 + 64, s, b);
                    }
                    ++kv_issued[x];
                    for (int it = 0; it < ni; ++it) {
                        const int t = si * ni + it, i0 = it * BQ;
                        const int xs = t % X_STAGES, ys = t % Y_STAGES;
                        const uint32_t xb = base + OFF_X + xs * XB, yb = base + OFF_Y + ys * YB;
                        if (t >= X_STAGES)
                            ok = mbar_wait(x_empty(xs), ((t / X_STAGES) - 1) & 1, abort_flag, kTimeoutBase | 0x02);
                        if (!ok) break;
                        mbar_arrive_expect_tx(x_full(xs), TILE_BYTES + (HAS_BIAS ? 2 * BT_BOX : 0) + 4 * 256);
                        if (HAS_BIAS) {
                            tma_load_4d(xb + X_BT, &tm_bt, x_full(xs), i0, j0, h, b);
                            tma_load_4d(xb + X_BT + BT_BOX, &tm_bt, x_full(xs), i0 + 64, j0, h, b);
                        }
                        tma_load_5d(xb + X_DOL, &tm_dol, x_full(xs), 0, i0, h, s, b);
                        // rows 0..1 (high, low) of the two 64-query atoms of the nl and -D blocks
                        tma_load_5d(xb + X_NL, &tm_nl, x_full(xs), i0, 0, h, s, b);
                        tma_load_5d(xb + X_NL + 2048, &tm_nl, x_full(xs), i0 + 64, 0, h, s, b);
                        tma_load_5d(xb + X_ND, &tm_d, x_full(xs), i0, 0, h, s, b);
                        tma_load_5d(xb + X_ND + 2048, &tm_d, x_full(xs), i0 + 64, 0, h, s, b);
                        ++x_issued[xs];
                        if (t >= Y_STAGES)
                            ok = mbar_wait(y_empty(ys), ((t / Y_STAGES) - 1) & 1, abort_flag, kTimeoutBase | 0x05);
                        if (!ok) break;
                        mbar_arrive_expect_tx(y_full(ys), 2 * TILE_BYTES);
                        tma_load_5d(yb + Y_Q, &tm_q, y_full(ys), 0, i0, h, s, b);
                        tma_load_5d(yb + Y_DOH, &tm_doa, y_full(ys), 0, i0, h, s, b);
                        ++y_issued[ys];
                    }
                }
                volatile int no_abort = 0;
                for (int x = 0; x < 2; ++x)
                    if (kv_issued[x]) mbar_wait(kv_full(x), (kv_issued[x] - 1) & 1, &no_abort, kTimeoutBase | 0x03);
                for (int x = 0; x < X_STAGES; ++x)
                    if (x_issued[x]) mbar_wait(x_full(x), (x_issued[x] - 1) & 1, &no_abort, kTimeoutBase | 0x04);
                for (int x = 0; x < Y_STAGES; ++x)
                    if (y_issued[x]) mbar_wait(y_full(x), (y_issued[x] - 1) & 1, &no_abort, kTimeoutBase | 0x06);
            }
        } else {
            // ---------------------------------------------------------------- MMA issuers
            const int role = warp - kMma;            // 0: S^T, dP^T   1: dV, dK   2: dQ
            if (lane == 0 && T > 0) {
                constexpr uint32_t ID_SS = idesc_bf16(BK, BQ, false, false);   // S^T, dP^T
                constexpr uint32_t ID_RT = idesc_bf16(BK, BQ, false, true);    // ones x rank-term block
                constexpr uint32_t ID_MK = idesc_bf16(BK, BQ, true, false);    // mask block x r-row
                constexpr uint32_t ID_KV = idesc_bf16(BK, HD, false, true);    // dV, dK (B MN-major)
                constexpr uint32_t ID_Q = idesc_bf16(BQ, HD, true, true);      // dQ (A and B MN-major)
                bool ok = true;
                const uint32_t ds = base + OFF_DS;
                for (int t = 0; ok && t < T; ++t) {
                    const int si = t / ni, it = t - si * ni, x = si & 1, st = t & 1;
                    const int xs = t % X_STAGES, ys = t % Y_STAGES;
                    const uint32_t kb = base + OFF_KV + x * KVB, xb = base + OFF_X + xs * XB, yb = base + OFF_Y + ys * YB;
                    if (role == 0) {
                        // S^T = K Q^T - lse*sqrt(C) (+ (r1 + r2) * mask_j);  dP^T = V (dOa_hi + dOa_lo)^T - D.
                        // Step t's products are issued as soon as the dS warps hold step t-1's in registers.
                        if (it == 0) ok = mbar_wait(kv_full(x), (si >> 1) & 1, abort_flag, kTimeoutBase | 0x11);
                        if (ok) ok = mbar_wait(x_full(xs), (t / X_STAGES) & 1, abort_flag, kTimeoutBase | 0x12);
                        if (ok) ok = mbar_wait(y_full(ys), (t / Y_STAGES) & 1, abort_flag, kTimeoutBase | 0x1D);
                        if (ok && t > 0) ok = mbar_wait(sdp_free, (t - 1) & 1, abort_flag, kTimeoutBase | 0x13);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk)
                            mma_ss(tmem + TM_ST, smem_desc(kb + KV_K + kk * 32, 16, 512, kSw64),
                                   smem_desc(yb + Y_Q + kk * 32, 16, 512, kSw64), ID_SS, kk > 0);
                        mma_ss(tmem + TM_ST, smem_desc(base + OFF_ONES, 128, 256, kSwNone),
                               smem_desc(xb + X_NL, 2048, 1024, kSw128), ID_RT, 1u);
                        if (HAS_MASK)
                            mma_ss(tmem + TM_ST, smem_desc(kb + KV_MASK, 2048, 1024, kSw128),
                                   smem_desc(base + OFF_RROW, 128, 256, kSwNone), ID_MK, 1u);
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk)
                            mma_ss(tmem + TM_DPT, smem_desc(kb + KV_V + kk * 32, 16, 512, kSw64),
                                   smem_desc(yb + Y_DOH + kk * 32, 16, 512, kSw64), ID_SS, kk > 0);
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk)
                            mma_ss(tmem + TM_DPT, smem_desc(kb + KV_V + kk * 32, 16, 512, kSw64),
                                   smem_desc(xb + X_DOL + kk * 32, 16, 512, kSw64), ID_SS, 1u);
                        mma_ss(tmem + TM_DPT, smem_desc(base + OFF_ONES, 128, 256, kSwNone),
                               smem_desc(xb + X_ND, 2048, 1024, kSw128), ID_RT, 1u);
                        mma_commit(sdp_full);
                        mma_commit(x_empty(xs));
                        mma_commit(y_empty(ys));
                        if (it == ni - 1) mma_commit(kv_empty(x));
                    } else if (role == 1) {
                        // dV_j += P^T dOa_hi;  dK_j += dS^T Q
                        ok = mbar_wait(y_full(ys), (t / Y_STAGES) & 1, abort_flag, kTimeoutBase | 0x14);
                        if (ok) ok = mbar_wait(ds_full(st), (t >> 1) & 1, abort_flag, kTimeoutBase | 0x15);
                        if (ok && it == 0 && si > 0) ok = mbar_wait(dkv_free, (si - 1) & 1, abort_flag, kTimeoutBase | 0x16);
                        if (!ok) break;
                        tc_fence_after();
                        const int pb = t & 1;                // P^T buffer of this step
#pragma unroll
                        for (int kk = 0; kk < BQ / 16; ++kk)
                            mma_ts(tmem + TM_DV, tmem + TM_PT + pb * 64 + kk * 8,
                                   smem_desc(yb + Y_DOH + kk * 1024, TILE_BYTES, 512, kSw64), ID_KV,
                                   (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < BQ / 16; ++kk) {
                            const uint32_t a = ds + (kk >> 2) * BT_BOX + (kk & 3) * 32;
                            mma_ss(tmem + TM_DK, smem_desc(a, 16, 1024, kSw128),
                                   smem_desc(yb + Y_Q + kk * 1024, TILE_BYTES, 512, kSw64), ID_KV,
                                   (it > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(ds_free);
                        mma_commit(y_empty(ys));
                        if (it == ni - 1) mma_commit(dkv_full);
                    } else {
                        // dQ_i = dS K_j
                        if (it == 0) ok = mbar_wait(kv_full(x), (si >> 1) & 1, abort_flag, kTimeoutBase | 0x17);
                        if (ok) ok = mbar_wait(ds_full(st), (t >> 1) & 1, abort_flag, kTimeoutBase | 0x18);
                        if (ok && t > 0) ok = mbar_wait(dq_free, (t - 1) & 1, abort_flag, kTimeoutBase | 0x19);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            mma_ss(tmem + TM_DQ, smem_desc(ds + kk * 2048, BT_BOX, 1024, kSw128),
                                   smem_desc(kb + KV_K + kk * 1024, TILE_BYTES, 512, kSw64), ID_Q, kk > 0 ? 1u : 0u);
                        mma_commit(ds_free);
                        mma_commit(dq_full);
                        if (it == ni - 1) mma_commit(kv_empty(x));
                    }
                }
                // Drain: every MMA issued by this thread has finished before TMEM is released.
                mma_commit(mma_done(role));
                volatile int no_abort = 0;
                mbar_wait(mma_done(role), 0, &no_abort, kTimeoutBase | (0x1A + role));
            }
        }
    } else {
        regs_increase<DS_REGS>();
        if (T > 0) {
        // ---------------------------------------------------------------- dS warpgroups
        const int wg = warp >> 2;                // queries QW wg .. QW wg + QW - 1 of the tile
        const int quad = warp & 3;
        const int r = quad * 32 + lane;          // key row within the tile = TMEM lane
        const int j = j0 + r;
        const bool jvalid = j < p.N;
        const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
        const uint64_t SC2 = f2(p.sc2, p.sc2);
        const uint64_t L2E2 = f2(p.bsc, p.bsc);
        bool ok = true;

        for (int t = 0; t < T; ++t) {
            const int st = t & 1;
            ok = mbar_wait(sdp_full, t & 1, abort_flag, kTimeoutBase | 0x24);
            if (!ok) break;
            tc_fence_after();
            // this thread's bias row for the warpgroup's 32 queries (64-query box wg / 2,
            // 16-byte chunks 4 (wg % 2) .. + 3) into registers at once, so the stage of ring X
            // is released early
            const int xs = t % X_STAGES;
            ok = mbar_wait(x_full(xs), (t / X_STAGES) & 1, abort_flag, kTimeoutBase | 0x25);
            uint32_t bw[QW / 2];
            if (HAS_BIAS) {
                const uint8_t* bt_ptr = gbase + OFF_X + xs * XB + X_BT + (wg >> 1) * BT_BOX + r * 128;
#pragma unroll
                for (int q = 0; q < QW / 8; ++q) {
                    const uint32_t ch = (uint32_t)((wg & 1) * 4 + q);
                    const uint4 w = *reinterpret_cast<const uint4*>(bt_ptr + ((ch ^ (uint32_t)(r & 7)) << 4));
                    bw[4 * q] = w.x; bw[4 * q + 1] = w.y; bw[4 * q + 2] = w.z; bw[4 * q + 3] = w.w;
                }
            }
            // the TMA refills this stage once it is released: order the generic-proxy reads above
            // before that async-proxy write (without the fence the refill can overtake them)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(x_empty(xs));           // bias tile of this stage consumed
            // P^T buffer of this step.  Its last reader, dV of step t - 2, is complete: the dS
            // warps waited for ds_free of step t - 2 before their dS stores of step t - 1, and
            // that barrier's dV/dK commit covers every earlier MMA of the same issuer.
            const int pb = t & 1;
            if (!ok) break;
            const uint32_t ts = lane_addr + TM_ST + wg * QW, td = lane_addr + TM_DPT + wg * QW;
            const uint32_t pt_addr = lane_addr + TM_PT + pb * 64 + wg * (QW / 2);
            // S^T and dP^T 16 queries at a time (v[0,16): S^T columns, v[16,32): dP^T columns).
            // P = exp2(S^T * sc2 + bias * bsc) (S^T already holds -lse and the mask),
            // dS = P * dP^T (dP^T already holds -D); two columns per op
            uint32_t dk2[QW / 2];
#pragma unroll
            for (int hf = 0; hf < QW / 16; ++hf) {
                uint32_t v[32];
                tmem_ld16x2_sync(ts + hf * 16, td + hf * 16, v);
                if (hf == QW / 16 - 1) {         // every S^T / dP^T column of this step is in registers
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sdp_free);
                }
                if (!jvalid) {                   // padded key rows: P = 0
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] = __float_as_uint(-INFINITY);
                }
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {                // 8 columns (one bias chunk) at a time
                    const int ch = hf * 2 + q2;
                    uint32_t pk4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = q2 * 8 + 2 * e;             // column within the 16
                        uint64_t y2 = fmul2(f2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), SC2);
                        if (HAS_BIAS) y2 = ffma2(bf16x2_to_f2(bw[ch * 4 + e]), L2E2, y2);
                        const float p0 = ex2(f2lo(y2)), p1 = ex2(f2hi(y2));
                        const uint64_t ds2 =
                            fmul2(f2(p0, p1), f2(__uint_as_float(v[16 + c]), __uint_as_float(v[17 + c])));
                        pk4[e] = pack_bf16(p0, p1);
                        dk2[ch * 4 + e] = pack_bf16(f2lo(ds2), f2hi(ds2));
                    }
                    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pt_addr + ch * 4),
                                 "r"(pk4[0]), "r"(pk4[1]), "r"(pk4[2]), "r"(pk4[3]));
                }
            }
            if (t > 0) ok = mbar_wait(ds_free, (t - 1) & 1, abort_flag, kTimeoutBase | 0x27);
            if (!ok) break;
            const uint32_t ds_row = base + OFF_DS + (wg >> 1) * BT_BOX + r * 128;
#pragma unroll
            for (int q = 0; q < QW / 8; ++q) {
                const uint32_t addr = ds_row + ((((uint32_t)((wg & 1) * 4 + q)) ^ (uint32_t)(r & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dk2[4 * q]),
                             "r"(dk2[4 * q + 1]), "r"(dk2[4 * q + 2]), "r"(dk2[4 * q + 3])
                             : "memory");
            }
            tc_wait_st();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_full(st));
        }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMma) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ------------------------------------------------------------------ elementwise kernels
struct PreParams {
    int B, S, N, H, n_pad;
    float sqrt_c;
    const __nv_bfloat16* out; const __nv_bfloat16* dout; Strides os;
    const __nv_bfloat16* out_lo;   // the forward's rounding residual of out (strides os), or null
    const __nv_bfloat16* g; Strides in;
    const float* lse;
    __nv_bfloat16* dg; Strides gs;
    __nv_bfloat16* doa_hi;  // contiguous [B,S,N,H,C]
    __nv_bfloat16* doa_lo;  // contiguous [B,S,N,H,C]: dOa - float(doa_hi), rounded
    __nv_bfloat16* nl;      // [B,S,H,2,n_pad]: high / low rows of -lse*sqrt(C); padding -1e30 / 0
    __nv_bfloat16* nd;      // [B,S,H,2,n_pad]: high / low rows of -D; padding 0
    float* dq_acc;          // contiguous [B,S,N,H,C] fp32
};

__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16* hi, __nv_bfloat16* lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    *hi = h;
    *lo = __float2bfloat16_rn(v - __bfloat162float(h));
}

constexpr int PRE_LANES = HD / 8;   // threads per logit row, 8 channels (16 bytes) each

__device__ __forceinline__ void pre_rows(const PreParams& p, int blk, int nblk) {
    const int64_t rows = (int64_t)p.B * p.S * p.N * p.H;
    const int64_t pads = (int64_t)p.B * p.S * p.H * (p.n_pad - p.N);
    const int part = threadIdx.x % PRE_LANES;
    const int64_t step = (int64_t)nblk * (blockDim.x / PRE_LANES);
    for (int64_t t = (int64_t)blk * (blockDim.x / PRE_LANES) + threadIdx.x / PRE_LANES; t < rows + pads;
         t += step) {
        if (t >= rows) {   // padded query slots of the rank-term rows: P must come out 0
            if (part == 0) {
                const int64_t u = t - rows;
                const int w = p.n_pad - p.N;
                const int64_t bsh = u / w;
                const int i = p.N + (int)(u % w);
                const int64_t o = bsh * 2 * p.n_pad + i;
                p.nl[o] = __float2bfloat16_rn(-1e30f);
                p.nl[o + p.n_pad] = __float2bfloat16_rn(0.f);
                p.nd[o] = __float2bfloat16_rn(0.f);
                p.nd[o + p.n_pad] = __float2bfloat16_rn(0.f);
            }
            continue;
        }
        int h, i, s, b;
        if (rows < 0x7fffffff) {             // 32-bit index arithmetic: a fraction of the 64-bit cost
            const uint32_t u = (uint32_t)t, q1 = u / (uint32_t)p.H, q2 = q1 / (uint32_t)p.N;
            h = (int)(u - q1 * (uint32_t)p.H);
            i = (int)(q1 - q2 * (uint32_t)p.N);
            b = (int)(q2 / (uint32_t)p.S);
            s = (int)(q2 - (uint32_t)b * (uint32_t)p.S);
        } else {
            h = (int)(t % p.H);
            i = (int)((t / p.H) % p.N);
            s = (int)((t / ((int64_t)p.H * p.N)) % p.S);
            b = (int)(t / ((int64_t)p.H * p.N * p.S));
        }
        const int64_t oo = p.os.off(b, s, i, h);
        const uint4 ow = reinterpret_cast<const uint4*>(p.out + oo)[part];
        const uint4 lw = p.out_lo ? reinterpret_cast<const uint4*>(p.out_lo + oo)[part] : make_uint4(0u, 0u, 0u, 0u);
        const uint4 dw = reinterpret_cast<const uint4*>(p.dout + p.os.off(b, s, i, h))[part];
        const uint4 gw = reinterpret_cast<const uint4*>(p.g + p.in.off(b, s, i, h))[part];
        const uint32_t ov[4] = {ow.x, ow.y, ow.z, ow.w}, dv[4] = {dw.x, dw.y, dw.z, dw.w},
                       gv[4] = {gw.x, gw.y, gw.z, gw.w}, lov[4] = {lw.x, lw.y, lw.z, lw.w};
        uint32_t dgv[4], hv[4], lv[4];
        float D = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // out as the forward computed it in fp32: the stored bf16 plus its rounding residual
            const float o0 = bf16lo(ov[e]) + bf16lo(lov[e]), o1 = bf16hi(ov[e]) + bf16hi(lov[e]);
            const float d0 = bf16lo(dv[e]), d1 = bf16hi(dv[e]);
            const float s0 = __fdividef(1.0f, 1.0f + __expf(-bf16lo(gv[e]))),
                        s1 = __fdividef(1.0f, 1.0f + __expf(-bf16hi(gv[e])));
            D = fmaf(d0, o0, D);
            D = fmaf(d1, o1, D);
            dgv[e] = pack_bf16(d0 * o0 * (1.0f - s0), d1 * o1 * (1.0f - s1));
            const float a0 = d0 * s0, a1 = d1 * s1;
            hv[e] = pack_bf16(a0, a1);
            lv[e] = pack_bf16(a0 - bf16lo(hv[e]), a1 - bf16hi(hv[e]));
        }
        reinterpret_cast<uint4*>(p.dg + p.gs.off(b, s, i, h))[part] = make_uint4(dgv[0], dgv[1], dgv[2], dgv[3]);
        reinterpret_cast<uint4*>(p.doa_hi + t * HD)[part] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        reinterpret_cast<uint4*>(p.doa_lo + t * HD)[part] = make_uint4(lv[0], lv[1], lv[2], lv[3]);
        float4* acc = reinterpret_cast<float4*>(p.dq_acc + t * HD) + 2 * part;
        acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 1; m < PRE_LANES; m <<= 1) D += __shfl_xor_sync(0xffffffffu, D, m);
        if (part == 0) {
            const int64_t bsh = ((int64_t)b * p.S + s) * p.H + h;
            const int64_t o = bsh * 2 * p.n_pad + i;
            split_bf16(-D, p.nd + o, p.nd + o + p.n_pad);
            split_bf16(-p.lse[bsh * p.N + i] * p.sqrt_c, p.nl + o, p.nl + o + p.n_pad);
        }
    }
}

// biasT[b,h,j,i] = pair_bias[b,h,i,j]: one 32x32 tile through shared memory
// (256 threads as 32 x 8).
__device__ __forceinline__ void transpose_tile(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                               int N, int tile) {
    __shared__ __nv_bfloat16 buf[32][33];
    const int nt = (N + 31) / 32;
    const int64_t plane = (int64_t)(tile / (nt * nt)) * N * N;
    const int bx = (tile % nt) * 32, by = ((tile / nt) % nt) * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int y = ty; y < 32; y += 8) {
        const int i = by + y, jj = bx + tx;
        if (i < N && jj < N) buf[y][tx] = src[plane + (int64_t)i * N + jj];
    }
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
        const int jj = bx + y, i = by + tx;
        if (i < N && jj < N) dst[plane + (int64_t)jj * N + i] = buf[tx][y];
    }
}

// The backward's preparation in one launch, by block range: the per-row pass
// (pre_rows) and the pair-bias transpose (one tile per block).
struct PrepParams {
    PreParams pre;
    int nb_pre;
    const __nv_bfloat16* bias;
    __nv_bfloat16* biast;
    int nb_tr;                // transpose tiles (0 without a pair bias)
};

__global__ void __launch_bounds__(256) bwd_prep_kernel(const PrepParams pp) {
    const int blk = blockIdx.x;
    if (blk < pp.nb_pre) {
        pre_rows(pp.pre, blk, pp.nb_pre);
        return;
    }
    transpose_tile(pp.bias, pp.biast, pp.pre.N, blk - pp.nb_pre);
}

struct PostParams {
    int B, S, N, H;
    const float* dq_acc;  // contiguous fp32
    __nv_bfloat16* dq; Strides gs;
    const float* part; int groups;
    float* dbias;
};

// The backward's finishing pass in one launch: dq (bf16, caller strides) from
// the fp32 accumulator, four threads per row converting 8 channels each; then
// (several row groups only) d_pair_bias = sum over groups g = 0, 1, ... of the
// partial slabs, in that order, 4 elements per thread.
__global__ void __launch_bounds__(256) bwd_post_kernel(const PostParams p) {
    const int64_t rows = (int64_t)p.B * p.S * p.N * p.H;
    const int64_t nq = rows * PRE_LANES;
    const int64_t n4 = p.groups > 1 ? (int64_t)p.B * p.H * p.N * p.N / 4 : 0;
    const int64_t stride = (int64_t)p.B * p.H * p.N * p.N;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nq + n4; g += (int64_t)gridDim.x * blockDim.x) {
        if (g < nq) {
            const int64_t t = g / PRE_LANES;
            const int part = (int)(g % PRE_LANES);
            int h, i, s, b;
            if (rows < 0x7fffffff) {         // 32-bit index arithmetic: a fraction of the 64-bit cost
                const uint32_t u = (uint32_t)t, q1 = u / (uint32_t)p.H, q2 = q1 / (uint32_t)p.N;
                h = (int)(u - q1 * (uint32_t)p.H);
                i = (int)(q1 - q2 * (uint32_t)p.N);
                b = (int)(q2 / (uint32_t)p.S);
                s = (int)(q2 - (uint32_t)b * (uint32_t)p.S);
            } else {
                h = (int)(t % p.H);
                i = (int)((t / p.H) % p.N);
                s = (int)((t / ((int64_t)p.H * p.N)) % p.S);
                b = (int)(t / ((int64_t)p.H * p.N * p.S));
            }
            const float4* a = reinterpret_cast<const float4*>(p.dq_acc + t * HD) + 2 * part;
            const float4 x = a[0], y = a[1];
            reinterpret_cast<uint4*>(p.dq + p.gs.off(b, s, i, h))[part] =
                make_uint4(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w), pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
        } else {
            const int64_t t = g - nq;
            float4 acc = reinterpret_cast<const float4*>(p.part)[t];
            for (int k = 1; k < p.groups; ++k) {
                const float4 v = reinterpret_cast<const float4*>(p.part + k * stride)[t];
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            reinterpret_cast<float4*>(p.dbias)[t] = acc;
        }
    }
}

// ------------------------------------------------------------------ host side
struct Call {
    evo_shape_t shape;
    const void *q, *k, *v, *g;
    evo_strides_t in;
    const void *mask, *bias, *out, *out_lo, *dout;
    evo_strides_t os;
    const float* lse;
    void *dq, *dk, *dv, *dg;
    evo_strides_t gs;
    float* dbias;
    char* ws;
    size_t d_off, nl_off, doa_off, dol_off, dqacc_off, biast_off, part_off;
    int groups;        // row groups of the main kernel (parallelism only)
    int db_groups;     // row groups of the d_pair_bias kernel: partial slabs at part_off when > 1
    uint64_t wait_ns;  // limit of the d_pair_bias kernel's waits
};

inline bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

inline int grid_for(int64_t items, int per_block) {
    const int64_t blocks = (items + per_block - 1) / per_block;
    return (int)std::min<int64_t>(std::max<int64_t>(blocks, 1), 148 * 16);
}

template <bool HM, bool HB>
inline cudaError_t launch_main(const CUtensorMap* m, const MainParams& mp, dim3 grid, cudaStream_t stream) {
    auto kern = bwd_main_kernel<HM, HB>;
    static cudaError_t attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (attr != cudaSuccess) return attr;
    // The setmaxnreg split assumes exactly LAUNCH_REGS registers per thread at
    // launch; with any other count an increase could wait forever.
    static int regs = [&] {
        cudaFuncAttributes fa{};
        return cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : -1;
    }();
    if (regs != LAUNCH_REGS) return cudaErrorInvalidConfiguration;
    {
        timing::Scope t(EVO_PHASE_BWD_MAIN, stream);
        kern<<<grid, THREADS, SMEM_BYTES, stream>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], m[8], mp);
    }
    return cudaGetLastError();
}

template <bool HM, bool HB>
inline cudaError_t launch_dbias(const CUtensorMap* m, const dbias::Params& dp, int grid, cudaStream_t stream) {
    auto kern = dbias::dbias_kernel<HM, HB>;
    static cudaError_t attr =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dbias::SMEM_BYTES);
    if (attr != cudaSuccess) return attr;
    static int regs = [&] {
        cudaFuncAttributes fa{};
        return cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : -1;
    }();
    if (regs != dbias::LAUNCH_REGS) return cudaErrorInvalidConfiguration;   // the setmaxnreg split assumes it
    {
        timing::Scope t(EVO_PHASE_BWD_DBIAS, stream);
        kern<<<grid, dbias::THREADS, dbias::SMEM_BYTES, stream>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7],
                                                                  m[8], dp);
    }
    return cudaGetLastError();
}

inline evo_status_t run(const Call& c, cudaStream_t stream, int* launched) {
    const evo_shape_t& sh = c.shape;
    *launched = 0;
    if (sh.C != HD || sh.N % 8 != 0) return EVO_ERR_UNSUPPORTED;
    const evo_strides_t* strs[3] = {&c.in, &c.os, &c.gs};
    for (auto s : strs)
        if (s->b % 8 || s->s % 8 || s->n % 8 || s->h % 8) return EVO_ERR_UNSUPPORTED;
    for (const void* ptr : {c.q, c.k, c.v, c.g, c.out, c.dout, (const void*)c.dq, (const void*)c.dk,
                            (const void*)c.dv, (const void*)c.dg})
        if (!aligned16(ptr)) return EVO_ERR_UNSUPPORTED;
    if (c.out_lo && !aligned16(c.out_lo)) return EVO_ERR_UNSUPPORTED;
    if ((c.mask && !aligned16(c.mask)) || (c.bias && !aligned16(c.bias)) || !aligned16(c.dbias))
        return EVO_ERR_UNSUPPORTED;

    const int B = (int)sh.B, S = (int)sh.S, N = (int)sh.N, H = (int)sh.H;
    const int n_pad = (N + BQ - 1) / BQ * BQ;
    __nv_bfloat16* nd = reinterpret_cast<__nv_bfloat16*>(c.ws + c.d_off);
    __nv_bfloat16* nl = reinterpret_cast<__nv_bfloat16*>(c.ws + c.nl_off);
    __nv_bfloat16* doa = reinterpret_cast<__nv_bfloat16*>(c.ws + c.doa_off);
    __nv_bfloat16* dol = reinterpret_cast<__nv_bfloat16*>(c.ws + c.dol_off);
    float* dq_acc = reinterpret_cast<float*>(c.ws + c.dqacc_off);
    __nv_bfloat16* biasT = reinterpret_cast<__nv_bfloat16*>(c.ws + c.biast_off);
    float* part = c.db_groups > 1 ? reinterpret_cast<float*>(c.ws + c.part_off) : c.dbias;

    const int64_t rows = (int64_t)B * S * N * H;
    PreParams pp{};
    pp.B = B; pp.S = S; pp.N = N; pp.H = H; pp.n_pad = n_pad;
    pp.sqrt_c = sqrtf((float)HD);
    pp.out = static_cast<const __nv_bfloat16*>(c.out); pp.dout = static_cast<const __nv_bfloat16*>(c.dout);
    pp.out_lo = static_cast<const __nv_bfloat16*>(c.out_lo);
    pp.os = Strides{c.os.b, c.os.s, c.os.n, c.os.h};
    pp.g = static_cast<const __nv_bfloat16*>(c.g); pp.in = Strides{c.in.b, c.in.s, c.in.n, c.in.h};
    pp.lse = c.lse; pp.dg = static_cast<__nv_bfloat16*>(c.dg); pp.gs = Strides{c.gs.b, c.gs.s, c.gs.n, c.gs.h};
    pp.doa_hi = doa; pp.doa_lo = dol; pp.nl = nl; pp.nd = nd; pp.dq_acc = dq_acc;
    // one launch: per-row pass and pair-bias transpose
    PrepParams prep{};
    prep.pre = pp;
    prep.nb_pre = grid_for((rows + (int64_t)B * S * H * (n_pad - N)) * PRE_LANES, 256);
    prep.bias = static_cast<const __nv_bfloat16*>(c.bias);
    prep.biast = biasT;
    const int nt = (N + 31) / 32;
    prep.nb_tr = c.bias ? nt * nt * B * H : 0;
    bwd_prep_kernel<<<prep.nb_pre + prep.nb_tr, 256, 0, stream>>>(prep);
    ++*launched;

    // tensor maps: q, k, v, dOa high, dOa low, transposed bias, mask, nl rows, -D rows
    const evo_strides_t contig{(int64_t)S * N * H * HD, (int64_t)N * H * HD, (int64_t)H * HD, (int64_t)HD};
    CUtensorMap m[9];
    std::memset(m, 0, sizeof(m));
    const evo_shape_t& s5 = sh;
    if (!tma::rows_bf16(&m[0], c.q, s5, c.in, BQ, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !tma::rows_bf16(&m[1], c.k, s5, c.in, BK, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !tma::rows_bf16(&m[2], c.v, s5, c.in, BK, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !tma::rows_bf16(&m[3], doa, s5, contig, BQ, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !tma::rows_bf16(&m[4], dol, s5, contig, BQ, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !tma::rowterm_bf16(&m[7], nl, s5, n_pad) || !tma::rowterm_bf16(&m[8], nd, s5, n_pad))
        return EVO_ERR_CUDA;
    if (c.bias && !tma::square_bf16(&m[5], biasT, s5, BK)) return EVO_ERR_CUDA;
    if (c.mask && !tma::mask_bf16(&m[6], c.mask, s5, 64)) return EVO_ERR_CUDA;

    MainParams mp{};
    mp.B = B; mp.S = S; mp.N = N; mp.H = H;
    mp.n_it = (N + BQ - 1) / BQ;
    const int G = c.groups;
    mp.gsz = (S + G - 1) / G;
    mp.sc2 = EVO_LOG2E / sqrtf((float)HD);
    mp.rs = 1.0f / sqrtf((float)HD);
    mp.r_bf16 = __bfloat162float(__float2bfloat16_rn(sqrtf((float)HD)));
    mp.r2_bf16 = __bfloat162float(__float2bfloat16_rn(sqrtf((float)HD) - mp.r_bf16));
    mp.bsc = mp.sc2 * mp.r_bf16;
    mp.dq_acc = dq_acc;
    mp.dk = static_cast<__nv_bfloat16*>(c.dk);
    mp.dv = static_cast<__nv_bfloat16*>(c.dv);
    mp.gs = Strides{c.gs.b, c.gs.s, c.gs.n, c.gs.h};
    const dim3 grid((unsigned)((N + BK - 1) / BK), (unsigned)G, (unsigned)(B * H));
    cudaError_t e;
    if (c.mask && c.bias) e = launch_main<true, true>(m, mp, grid, stream);
    else if (c.mask) e = launch_main<true, false>(m, mp, grid, stream);
    else if (c.bias) e = launch_main<false, true>(m, mp, grid, stream);
    else e = launch_main<false, false>(m, mp, grid, stream);
    if (e == cudaErrorInvalidConfiguration) return EVO_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return EVO_ERR_CUDA;
    ++*launched;

    // d_pair_bias: row sums on chip, one slab per row group (or the output itself)
    dbias::Params dp{};
    dp.B = B; dp.S = S; dp.N = N; dp.H = H;
    dp.n_t = (N + dbias::BQ - 1) / dbias::BQ;
    const int GD = c.db_groups;
    dp.gsz = (S + GD - 1) / GD;
    dp.groups = (S + dp.gsz - 1) / dp.gsz;
    if (dp.groups != GD) return EVO_ERR_UNSUPPORTED;      // the workspace was sized for GD slabs
    const int64_t items = (int64_t)B * H * dp.n_t * dp.n_t * GD;
    if (items > 0x7fffffff) return EVO_ERR_UNSUPPORTED;
    dp.n_items = (int)items;
    dp.sc2 = mp.sc2;
    dp.bsc = mp.bsc;
    dp.r_bf16 = mp.r_bf16;
    dp.r2_bf16 = mp.r2_bf16;
    dp.out = part;
    dp.wait_ns = c.wait_ns;
    int sms = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    const int dgrid = (int)std::min<int64_t>(items, sms);
    if (c.mask && c.bias) e = launch_dbias<true, true>(m, dp, dgrid, stream);
    else if (c.mask) e = launch_dbias<true, false>(m, dp, dgrid, stream);
    else if (c.bias) e = launch_dbias<false, true>(m, dp, dgrid, stream);
    else e = launch_dbias<false, false>(m, dp, dgrid, stream);
    if (e == cudaErrorInvalidConfiguration) return EVO_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return EVO_ERR_CUDA;
    ++*launched;

    PostParams qp{};
    qp.B = B; qp.S = S; qp.N = N; qp.H = H;
    qp.dq_acc = dq_acc; qp.dq = static_cast<__nv_bfloat16*>(c.dq); qp.gs = mp.gs;
    qp.part = part; qp.groups = GD; qp.dbias = c.dbias;
    bwd_post_kernel<<<grid_for(rows * PRE_LANES + (GD > 1 ? (int64_t)B * H * N * N / 4 : 0), 256), 256, 0, stream>>>(qp);
    ++*launched;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

}  // namespace bwd
}  // namespace evo
