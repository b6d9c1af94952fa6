// fwd_sm100.cuh -- bf16 forward of Evoformer pair-bias attention on sm_100a.
//
// Persistent kernel: one CTA per SM walks a static round-robin list of work
// items.  An item is a 128-row query tile i0..i0+127 of head h in batch b for
// NSUB consecutive rows s (MSA sequences or pair rows).  The key axis is
// streamed in 128-key tiles; no logit ever leaves TMEM/registers (the
// flash-style, online-softmax treatment EvoFlash-3D gives this op in the
// MegaFold summary, section "EvoFlash-3D").
//
// The mask row is added by the tensor core:
//   S_u = Q_u K_u^T + (r1 e_0 + r2 e_8) m_u^T,   r1 = bf16(sqrt(C)), r2 = bf16(sqrt(C) - r1)
// accumulates, in fp32 TMEM, sqrt(C) times the logit without the pair bias:
// the last term is one 16-deep K step whose B block carries the mask row of
// row s in its rows 0 and 8 (exact products in fp32; r1 + r2 equals sqrt(C)
// to 3e-7 relative, so the mask enters exactly up to that and fp32 rounding).
// The pair-bias tile (TMA-loaded once per key tile and shared by all NSUB rows
// s -- it is the same for every s) is added by the tensor core too, as
// (r1 I) B with I the identity: eight more 16-deep K steps whose A blocks are
// shifted 16 x 16 identities, all read from one small constant block (see
// Layout::ident).  The bias therefore enters as (r1 / sqrt(C)) bias, scaled by
// 1 - 1.07e-4 for C = 32 -- eighteen times below the 2^-9 rounding of the bf16
// bias itself; the backward adds it with the same factor, so its recomputed P
// matches this pass's log-sum-exp.  The softmax threads only scale, take
// maxima and exponentiate.
//
// Warp roles (128*NSUB + 256 threads; the two control warpgroups give up
// registers to the softmax warpgroups with setmaxnreg, one site per warpgroup):
//   warps 0 .. 4*NSUB-1   one 4-warp softmax group per row s (see below)
//   warp 4*NSUB           TMA producer: per item Q and the gate tiles (each
//            double-buffered by item parity), then per key tile K and the mask
//            row (per row s) and the pair-bias tile into a 2-stage ring ("A")
//            that runs across items, released by the S MMAs' commits (K, mask
//            and bias are MMA operands only)
//   warps 4*NSUB+1+u      S issuer of row group u (one lane; the first also
//            owns TMEM): S_u = Q K^T + (r1 e_0 + r2 e_8) m^T + (r1 I) bias,
//            2 + 1 + 8 MMAs of M = 128, N = 128
//   warp 4*NSUB+NSUB+1    TMA producer of V (per row s) into its own 2-stage
//            ring ("B"), released when the P V products of the tile are done
//   warps 4*NSUB+NSUB+2+u P V issuer of row group u: O_u += P_u V_u (M = 128,
//            N = 32, K = 128, P read from TMEM), O double-buffered by item
//   softmax: thread = query row.  Load S from TMEM, online max and sum in fp32
//            with a lazy rescale (the running max moves only when a tile's
//            max exceeds it by more than 2^8), P (bf16) back to TMEM, and at
//            the end of the item out = sigmoid(g) * O / l (the gate read from
//            its TMA-loaded tile; out's bf16 rounding residual written too when
//            asked), lse = log(l) + max.  The two row groups take turns on the
//            exponentials (the MUFU unit is the scarce resource at C = 32):
//            each group's loads and maxima overlap the other group's
//            exponentials.
// TMEM per row s: S 128 columns, P 64 columns (bf16 pairs), O 2 x 32 columns.
#pragma once

#include "sm100.cuh"

namespace evo {
namespace fwd {

using namespace evo::sm100;

constexpr int BM = 128;                 // query rows per tile (TMEM lanes)
constexpr int BN = 128;                 // keys per tile
constexpr int HD = 32;                  // head dim C
constexpr int STAGES_A = 2;             // K, pair-bias tile, mask blocks
constexpr int STAGES_B = 2;             // V
constexpr int Q_BYTES = BM * HD * 2;    // 8 KB, 64-byte rows, 64B swizzle
constexpr int KV_BYTES = BN * HD * 2;   // 8 KB each for K and V
constexpr int BIAS_BOX = BM * 64 * 2;   // 16 KB: 128 rows x 64 keys, 128B swizzle
constexpr int BIAS_BYTES = 2 * BIAS_BOX;
constexpr int MASKB_BYTES = 4096;       // 16 x 128 bf16 B block (rows 0 and 8 = mask row), 128B swizzle
constexpr int ONES_BYTES = 128 * 16 * 2;     // r1 e_0 + r2 e_8 columns, K-major, no swizzle
// The A operands of the bias MMAs, 128 x 16 blocks (r1 I)[:, 16 kk : 16 kk + 16], kk = 0..7,
// all read from one array of 45 no-swizzle core matrices (8 x 8 bf16, 128 bytes each) that
// is zero except r1 I_8 in cores IDENT_C0 and IDENT_C0 + 16.  K-step kk starts at core
// IDENT_C0 - 2 kk with 8-row groups one core apart (SBO 128 B) and the second 8-wide K group
// 15 cores further (LBO 1920 B): row group g, K group h reads core IDENT_C0 - 2 kk + g + 15 h,
// which is an identity core exactly for (g, h) = (2 kk, 0) and (2 kk + 1, 1).
constexpr int IDENT_C0 = 14;
constexpr int IDENT_BYTES = 6144;            // 45 cores = 5760 bytes, rounded up
constexpr uint32_t IDENT_SBO = 128, IDENT_LBO = 15 * 128;
// per row group: S, P, and two O accumulators (items alternate between them,
// so an item's epilogue can run after the next item's first tile)
constexpr uint32_t COL_S = 0, COL_P = 128, COL_O = 192, SUBCOLS = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units
// Every POLY_EVERY-th pair of exponentials of a row runs on the FMA pipe
// (exp2_poly2) instead of the MUFU unit, which at C = 32 is the scarcest unit;
// 0 keeps every exponential on MUFU.
#ifndef EVO_FWD_POLY_EVERY
#define EVO_FWD_POLY_EVERY 0
#endif
constexpr int POLY_EVERY = EVO_FWD_POLY_EVERY;

__host__ __device__ constexpr int round_up(int x, int a) { return (x + a - 1) / a * a; }

template <int NSUB>
struct Layout {
    static constexpr int qbuf(int k, int u) { return (k * NSUB + u) * Q_BYTES; }   // per item parity k
    // the gate tile of each row s, read by the item's epilogue (same box and swizzle as Q)
    static constexpr int gbuf(int k, int u) { return (2 * NSUB + k * NSUB + u) * Q_BYTES; }
    static constexpr int ones = 4 * NSUB * Q_BYTES;
    static constexpr int ident = ones + ONES_BYTES;
    // ring A: per stage K (per row), the pair-bias tile, the mask blocks (per row)
    static constexpr int stage0 = round_up(ident + IDENT_BYTES, 1024);
    static constexpr int k_off(int u) { return u * KV_BYTES; }
    static constexpr int bias_off = NSUB * KV_BYTES;
    static constexpr int maskb_off(int u) { return bias_off + BIAS_BYTES + u * MASKB_BYTES; }
    static constexpr int stage_bytes = round_up(bias_off + BIAS_BYTES + NSUB * MASKB_BYTES, 1024);
    // ring B: per stage V (per row)
    static constexpr int vstage0 = stage0 + STAGES_A * stage_bytes;
    static constexpr int v_off(int u) { return u * KV_BYTES; }
    static constexpr int vstage_bytes = round_up(NSUB * KV_BYTES, 1024);
    static constexpr int bars = vstage0 + STAGES_B * vstage_bytes;
    // q_full[2], q_empty[2], ka_full[SA], ka_empty[SA], v_full[SB], v_empty[SB], s_full[u], s_free[u],
    // p_full[u], o_full[u], mma_done[2 NSUB], exp_turn[u], g_full[2], g_empty[2]
    static constexpr int nbars = 4 + 2 * STAGES_A + 2 * STAGES_B + 7 * NSUB + 4;
    static constexpr int misc = bars + nbars * 8;   // tmem base (u32), abort flag (u32)
    static constexpr int bytes = misc + 16 + 1024;  // + slack to align the base to 1024
    static constexpr uint32_t tmem_cols = NSUB == 1 ? 256 : 512;
    // softmax warpgroups, then two control warpgroups (producers, S issuers, P V issuers)
    static constexpr int threads = 128 * NSUB + 256;
    // register split: launch count (65536 / threads, rounded down to 8) and the
    // per-warpgroup counts after setmaxnreg; softmax + control <= launch pool
    static constexpr int launch_regs = (65536 / threads) / 8 * 8;
    static constexpr uint32_t softmax_regs = NSUB == 2 ? 208 : 240;
    static constexpr uint32_t control_regs = NSUB == 2 ? 48 : 64;
    static_assert((int)(NSUB * softmax_regs + 2 * control_regs) * 128 <= launch_regs * threads, "register split");
};

struct Params {
    int B, S, N, H;
    int n_kv;                 // ceil(N / BN)
    int n_it;                 // query tiles per (b, h, s)
    int n_sg;                 // row groups of NSUB rows
    int n_items;              // B * H * n_sg * n_it
    float scale;              // 1/sqrt(C)
    float r_bf16;             // r1 = bf16(sqrt(C)) and r2 = bf16(sqrt(C) - r1): the mask MMA's
    float r2_bf16;            //   two nonzero columns, whose sum is sqrt(C) to 3e-7
    const __nv_bfloat16* g;   // gate, strides `in`
    Strides in;
    __nv_bfloat16* out;       // strides `os`
    __nv_bfloat16* out_lo;    // strides `os`: bf16(out_fp32 - out), or null
    Strides os;
    float* lse;               // [B,S,H,N]
    uint64_t wait_ns;         // limit of every wait but the final drains (EVO_WAIT_LIMIT_NS by default)
};

struct Item {
    int b, h, sg, i0;
};
// Items are numbered with the query tile fastest, then the row group, then
// (b, h): the CTAs running side by side share K/V tiles and pair-bias tiles in L2.
__device__ __forceinline__ Item decode(const Params& p, int item) {
    Item it;
    const int ti = item % p.n_it;
    const int rest = item / p.n_it;
    it.sg = rest % p.n_sg;
    const int bh = rest / p.n_sg;
    it.i0 = ti * BM;
    it.b = bh / p.H;
    it.h = bh % p.H;
    return it;
}

// Status codes recorded when a wait gives up: 0x1RRB (role R, barrier B).
enum : unsigned int { kTimeoutBase = 0x1000u };

template <int NSUB, bool HAS_MASK, bool HAS_BIAS>
__global__ void __launch_bounds__(Layout<NSUB>::threads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_bias,
                    const __grid_constant__ CUtensorMap tm_mask, const __grid_constant__ CUtensorMap tm_g,
                    const Params p) {
    using L = Layout<NSUB>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // S issuers: warps kMma .. kMma+NSUB-1; P V issuers: warps kMmaPV .. kMmaPV+NSUB-1
    constexpr int kProducer = 4 * NSUB, kMma = 4 * NSUB + 1;
    constexpr int kProducerV = kMma + NSUB, kMmaPV = kProducerV + 1;
    static_assert(kMmaPV + NSUB <= L::threads / 32, "warp roles");

    const uint32_t bar0 = base + L::bars;
    constexpr int kS = 4 + 2 * STAGES_A + 2 * STAGES_B;        // first per-row-group barrier
    auto q_full = [&](int x) { return bar0 + 8u * (0 + x); };
    auto q_empty = [&](int x) { return bar0 + 8u * (2 + x); };
    auto ka_full = [&](int st) { return bar0 + 8u * (4 + st); };
    auto ka_empty = [&](int st) { return bar0 + 8u * (4 + STAGES_A + st); };
    auto v_full = [&](int st) { return bar0 + 8u * (4 + 2 * STAGES_A + st); };
    auto v_empty = [&](int st) { return bar0 + 8u * (4 + 2 * STAGES_A + STAGES_B + st); };
    auto s_full = [&](int u) { return bar0 + 8u * (kS + u); };
    auto s_free = [&](int u) { return bar0 + 8u * (kS + NSUB + u); };
    auto p_full = [&](int u) { return bar0 + 8u * (kS + 2 * NSUB + u); };
    auto o_full = [&](int u) { return bar0 + 8u * (kS + 3 * NSUB + u); };
    auto mma_done = [&](int x) { return bar0 + 8u * (kS + 4 * NSUB + x); };      // x < 2 * NSUB
    // exp_turn[u]: row group u may start the exponentials of its next tile
    auto exp_turn = [&](int u) { return bar0 + 8u * (kS + 6 * NSUB + u); };
    // g_full[x] / g_empty[x]: the gate tiles of the item with parity x loaded / read by its epilogue
    auto g_full = [&](int x) { return bar0 + 8u * (kS + 7 * NSUB + x); };
    auto g_empty = [&](int x) { return bar0 + 8u * (kS + 7 * NSUB + 2 + x); };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + L::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::misc + 4);

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(q_full(x), 1);
            mbar_init(q_empty(x), NSUB);           // one commit per MMA issuer
            mbar_init(g_full(x), 1);
            mbar_init(g_empty(x), 4 * NSUB);       // one arrival per softmax warp, after its epilogue
        }
        for (int st = 0; st < STAGES_A; ++st) {
            mbar_init(ka_full(st), 1);
            mbar_init(ka_empty(st), NSUB);              // the S MMAs' commits (K, mask and bias are MMA operands)
        }
        for (int st = 0; st < STAGES_B; ++st) {
            mbar_init(v_full(st), 1);
            mbar_init(v_empty(st), NSUB);               // the P V MMAs' commits
        }
        for (int u = 0; u < NSUB; ++u) {
            mbar_init(s_full(u), 1);
            mbar_init(s_free(u), 4);
            mbar_init(p_full(u), 4);
            mbar_init(o_full(u), 1);
            mbar_init(mma_done(u), 1);
            mbar_init(mma_done(NSUB + u), 1);
            mbar_init(exp_turn(u), 4);             // one arrival per warp of the other group
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kProducer && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_g);
        if (HAS_BIAS) prefetch_tmap(&tm_bias);
        if (HAS_MASK) prefetch_tmap(&tm_mask);
    }
    if (warp == kMma) {
        tmem_alloc(base + L::misc, L::tmem_cols);
        tmem_relinquish();
    }
    if (warp < 4 * NSUB) {
        // Constant MMA operand (element (row, k) of a no-swizzle K-major tile is
        // at (row % 8) * 16 + (row / 8) * SBO + (k / 8) * 128 + (k % 8) * 2):
        //   columns r1 e_0 + r2 e_8 (SBO 256), and every mask block zero but
        //   its rows 0 and 8 (the TMA writes those each stage).
        const int t = threadIdx.x;
        const int nt = 128 * NSUB;
        const uint16_t rb = (uint16_t)(__float_as_uint(p.r_bf16) >> 16);
        const uint16_t rb2 = (uint16_t)(__float_as_uint(p.r2_bf16) >> 16);
        for (int o = t * 16; o < ONES_BYTES + IDENT_BYTES; o += nt * 16)   // ones and ident are adjacent
            *reinterpret_cast<uint4*>(gbase + L::ones + o) = make_uint4(0u, 0u, 0u, 0u);
        for (int st = 0; st < STAGES_A; ++st)
            for (int u = 0; u < NSUB; ++u)
                for (int o = t * 16; o < MASKB_BYTES; o += nt * 16)
                    *reinterpret_cast<uint4*>(gbase + L::stage0 + st * L::stage_bytes + L::maskb_off(u) + o) =
                        make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
        asm volatile("bar.sync 1, %0;" ::"r"(nt) : "memory");
        if (t < 128) {
            const int rr = t;
            *reinterpret_cast<uint16_t*>(gbase + L::ones + (rr % 8) * 16 + (rr / 8) * 256) = rb;
            *reinterpret_cast<uint16_t*>(gbase + L::ones + (rr % 8) * 16 + (rr / 8) * 256 + 128) = rb2;
        }
        if (t < 16) {   // the diagonals of the two identity cores: element (m, m) at 18 m bytes
            const int core = IDENT_C0 + (t >> 3) * 16, m = t & 7;
            *reinterpret_cast<uint16_t*>(gbase + L::ident + core * 128 + 18 * m) = rb;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // setmaxnreg is warpgroup-wide: all four warps of a warpgroup execute the same
    // instruction, so each warpgroup changes its count before its warps' roles split.
    if (warp >= 4 * NSUB) {
        regs_decrease<L::control_regs>();
        if (warp == kProducer) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                constexpr uint32_t tx = NSUB * KV_BYTES + (HAS_BIAS ? BIAS_BYTES : 0) + (HAS_MASK ? NSUB * 512 : 0);
                int q_issued[2] = {0, 0}, g_issued[2] = {0, 0}, kv_issued[STAGES_A] = {};
                int tg = 0;
                bool ok = true;
                for (int item = blockIdx.x, k = 0; ok && item < p.n_items; item += gridDim.x, ++k) {
                    const Item itm = decode(p, item);
                    const int s0 = itm.sg * NSUB;
                    int s_ld[NSUB];
#pragma unroll
                    for (int u = 0; u < NSUB; ++u) s_ld[u] = min(s0 + u, p.S - 1);
                    const int qb = k & 1;
                    if (k >= 2) ok = mbar_wait(q_empty(qb), ((k >> 1) - 1) & 1, abort_flag, kTimeoutBase | 0x001, p.wait_ns);
                    if (!ok) break;
                    mbar_arrive_expect_tx(q_full(qb), NSUB * Q_BYTES);
#pragma unroll
                    for (int u = 0; u < NSUB; ++u)
                        tma_load_5d(base + L::qbuf(qb, u), &tm_q, q_full(qb), 0, itm.i0, itm.h, s_ld[u], itm.b);
                    ++q_issued[qb];
                    // the gate tiles of this item (buffer qb is free once item k-2's epilogue has read it)
                    if (k >= 2) ok = mbar_wait(g_empty(qb), ((k >> 1) - 1) & 1, abort_flag, kTimeoutBase | 0x008, p.wait_ns);
                    if (!ok) break;
                    mbar_arrive_expect_tx(g_full(qb), NSUB * Q_BYTES);
#pragma unroll
                    for (int u = 0; u < NSUB; ++u)
                        tma_load_5d(base + L::gbuf(qb, u), &tm_g, g_full(qb), 0, itm.i0, itm.h, s_ld[u], itm.b);
                    ++g_issued[qb];
                    for (int j = 0; j < p.n_kv; ++j, ++tg) {
                        const int st = tg % STAGES_A;
                        const uint32_t sb = base + L::stage0 + st * L::stage_bytes;
                        if (tg >= STAGES_A)
                            ok = mbar_wait(ka_empty(st), ((tg / STAGES_A) - 1) & 1, abort_flag, kTimeoutBase | 0x002, p.wait_ns);
                        if (!ok) break;
                        mbar_arrive_expect_tx(ka_full(st), tx);
#pragma unroll
                        for (int u = 0; u < NSUB; ++u)
                            tma_load_5d(sb + L::k_off(u), &tm_k, ka_full(st), 0, j * BN, itm.h, s_ld[u], itm.b);
                        if (HAS_BIAS) {
                            tma_load_4d(sb + L::bias_off, &tm_bias, ka_full(st), j * BN, itm.i0, itm.h, itm.b);
                            tma_load_4d(sb + L::bias_off + BIAS_BOX, &tm_bias, ka_full(st), j * BN + 64, itm.i0, itm.h, itm.b);
                        }
                        if (HAS_MASK) {
#pragma unroll
                            for (int u = 0; u < NSUB; ++u) {
                                // rows 0 and 8 of the two 64-key halves (rows 0 and 8 both start a
                                // 128B-swizzle atom, so the unswizzled row lands as the MMA reads it)
                                tma_load_3d(sb + L::maskb_off(u), &tm_mask, ka_full(st), j * BN, s_ld[u], itm.b);
                                tma_load_3d(sb + L::maskb_off(u) + 1024, &tm_mask, ka_full(st), j * BN, s_ld[u], itm.b);
                                tma_load_3d(sb + L::maskb_off(u) + 2048, &tm_mask, ka_full(st), j * BN + 64, s_ld[u], itm.b);
                                tma_load_3d(sb + L::maskb_off(u) + 3072, &tm_mask, ka_full(st), j * BN + 64, s_ld[u], itm.b);
                            }
                        }
                        ++kv_issued[st];
                    }
                }
                // Never leave with copies in flight: wait (bounded) for the last fill of every buffer.
                volatile int no_abort = 0;
                for (int x = 0; x < 2; ++x) {
                    if (q_issued[x]) mbar_wait(q_full(x), (q_issued[x] - 1) & 1, &no_abort, kTimeoutBase | 0x003);
                    if (g_issued[x]) mbar_wait(g_full(x), (g_issued[x] - 1) & 1, &no_abort, kTimeoutBase | 0x009);
                }
                for (int st = 0; st < STAGES_A; ++st)
                    if (kv_issued[st]) mbar_wait(ka_full(st), (kv_issued[st] - 1) & 1, &no_abort, kTimeoutBase | 0x004);
            }
        } else if (warp == kProducerV) {
            // ------------------------------------------------------------ producer of V
            if (lane == 0) {
                int v_issued[STAGES_B] = {};
                int tg = 0;
                bool ok = true;
                for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
                    const Item itm = decode(p, item);
                    const int s0 = itm.sg * NSUB;
                    for (int j = 0; j < p.n_kv; ++j, ++tg) {
                        const int st = tg % STAGES_B;
                        const uint32_t vb = base + L::vstage0 + st * L::vstage_bytes;
                        if (tg >= STAGES_B)
                            ok = mbar_wait(v_empty(st), ((tg / STAGES_B) - 1) & 1, abort_flag, kTimeoutBase | 0x006, p.wait_ns);
                        if (!ok) break;
                        mbar_arrive_expect_tx(v_full(st), NSUB * KV_BYTES);
#pragma unroll
                        for (int u = 0; u < NSUB; ++u)
                            tma_load_5d(vb + L::v_off(u), &tm_v, v_full(st), 0, j * BN, itm.h, min(s0 + u, p.S - 1), itm.b);
                        ++v_issued[st];
                    }
                }
                volatile int no_abort = 0;
                for (int st = 0; st < STAGES_B; ++st)
                    if (v_issued[st]) mbar_wait(v_full(st), (v_issued[st] - 1) & 1, &no_abort, kTimeoutBase | 0x007);
            }
        } else if (warp >= kMma && warp < kMma + NSUB) {
            // ------------------------------------------------------------ S issuer of row group u
            const int u = warp - kMma;
            if (lane == 0) {
                constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false, false);
                constexpr uint32_t IDESC_MASK = idesc_bf16(BM, BN, false, true);   // B operand MN-major
                const uint32_t t_s = tmem + u * SUBCOLS + COL_S;
                // descriptors that depend only on the stage are built once; per MMA only the
                // start-address field (address / 16, in the low bits) moves
                const uint64_t d_ones = smem_desc(base + L::ones, 128, 256, kSwNone);
                const uint64_t d_id0 = smem_desc(base + L::ident + IDENT_C0 * 128, IDENT_LBO, IDENT_SBO, kSwNone);
                bool ok = true;
                int tg = 0;
                for (int item = blockIdx.x, k = 0; ok && item < p.n_items; item += gridDim.x, ++k) {
                    const int qb = k & 1;
                    ok = mbar_wait(q_full(qb), (k >> 1) & 1, abort_flag, kTimeoutBase | 0x101, p.wait_ns);
                    const uint64_t d_q = smem_desc(base + L::qbuf(qb, u), 16, 512, kSw64);
                    for (int j = 0; ok && j < p.n_kv; ++j, ++tg) {
                        const int st = tg % STAGES_A;
                        const uint32_t sb = base + L::stage0 + st * L::stage_bytes;
                        ok = mbar_wait(ka_full(st), (tg / STAGES_A) & 1, abort_flag, kTimeoutBase | 0x102, p.wait_ns);
                        if (ok && tg > 0) ok = mbar_wait(s_free(u), (tg - 1) & 1, abort_flag, kTimeoutBase | 0x103, p.wait_ns);
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t d_k = smem_desc(sb + L::k_off(u), 16, 512, kSw64);
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk)               // 32 bytes = 2 in the address field
                            mma_ss(t_s, d_q + 2 * kk, d_k + 2 * kk, IDESC_QK, kk > 0 ? 1u : 0u);
                        if (HAS_MASK)                                     // + (r1 + r2) * mask[s, j]
                            mma_ss(t_s, d_ones, smem_desc(sb + L::maskb_off(u), 2048, 1024, kSw128), IDESC_MASK, 1u);
                        if (HAS_BIAS) {                                   // + r1 * bias[i, j]: (r1 I) times the bias tile
                            const uint64_t d_b = smem_desc(sb + L::bias_off, BIAS_BOX, 1024, kSw128);
#pragma unroll
                            for (int kk = 0; kk < BM / 16; ++kk)          // A: 2 cores (256 B) back, B: 2048 B on
                                mma_ss(t_s, d_id0 - (uint64_t)(16 * kk), d_b + (uint64_t)(128 * kk), IDESC_MASK, 1u);
                        }
                        mma_commit(s_full(u));
                        mma_commit(ka_empty(st));                         // K, mask and bias read
                    }
                    if (ok) mma_commit(q_empty(qb));   // Q of this item no longer read once these MMAs finish
                }
                // Drain: every MMA issued by this thread has finished before TMEM is released.
                mma_commit(mma_done(u));
                volatile int no_abort = 0;
                mbar_wait(mma_done(u), 0, &no_abort, kTimeoutBase | 0x105);
            }
        } else if (warp >= kMmaPV && warp < kMmaPV + NSUB) {
            // ------------------------------------------------------------ P V issuer of row group u
            const int u = warp - kMmaPV;
            if (lane == 0) {
                constexpr uint32_t IDESC_PV = idesc_bf16(BM, HD, false, true);
                const uint32_t t_p = tmem + u * SUBCOLS + COL_P, t_o = tmem + u * SUBCOLS + COL_O;
                bool ok = true;
                int tg = 0;
                for (int item = blockIdx.x, k = 0; ok && item < p.n_items; item += gridDim.x, ++k) {
                    for (int j = 0; ok && j < p.n_kv; ++j, ++tg) {
                        const int vs = tg % STAGES_B;
                        ok = mbar_wait(p_full(u), tg & 1, abort_flag, kTimeoutBase | 0x104, p.wait_ns);
                        if (ok) ok = mbar_wait(v_full(vs), (tg / STAGES_B) & 1, abort_flag, kTimeoutBase | 0x106, p.wait_ns);
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t d_v = smem_desc(base + L::vstage0 + vs * L::vstage_bytes + L::v_off(u), KV_BYTES, 512,
                                                       kSw64);
                        const uint32_t o = t_o + (uint32_t)(k & 1) * HD;
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk)               // 16 keys = 1024 B = 64 in the address field
                            mma_ts(o, t_p + kk * 8, d_v + (uint64_t)(64 * kk), IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(o_full(u));
                        mma_commit(v_empty(vs));
                    }
                }
                mma_commit(mma_done(NSUB + u));
                volatile int no_abort = 0;
                mbar_wait(mma_done(NSUB + u), 0, &no_abort, kTimeoutBase | 0x107);
            }
        }
    } else {
        regs_increase<L::softmax_regs>();
        // ------------------------------------------------------------ softmax
        const int u = warp >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;          // query row within the tile = TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + u * SUBCOLS;
        // S holds sqrt(C) times the logit; the logit in log2 units is y = S * sc2,
        // sc2 = log2(e)/sqrt(C); exponents are exp2(y - ms)
        const float sc2 = p.scale * EVO_LOG2E;
        const uint64_t SC2 = f2(sc2, sc2);
        bool ok = true;
        int tg = 0;
        // The epilogue of an item (out = sigmoid(g) * O / l, lse) is deferred to
        // after the first tile of the next item: by then the item's last PV is
        // complete (that tile waited for it), so no thread idles on it.
        struct Epi {
            bool pending, row_ok;
            int b, s, i, h, obuf, k;
            float l, ms;
        } epi;
        epi.pending = false;
        auto run_epilogue = [&]() -> bool {
            // the gate row from the item's gate tile in shared memory (64B swizzle: 16-byte
            // chunk c of row r sits at chunk c ^ ((r >> 1) & 3))
            const int gb = epi.k & 1;
            if (!mbar_wait(g_full(gb), (epi.k >> 1) & 1, abort_flag, kTimeoutBase | 0x207, p.wait_ns)) return false;
            uint4 gw[HD / 8];
            const uint8_t* grow = gbase + L::gbuf(gb, u) + r * 64;
#pragma unroll
            for (int q = 0; q < HD / 8; ++q)
                gw[q] = *reinterpret_cast<const uint4*>(grow + ((((uint32_t)q ^ (uint32_t)((r >> 1) & 3))) << 4));
            fence_proxy_async_smem();            // generic reads before the TMA's refill of the buffer
            __syncwarp();
            if (lane == 0) mbar_arrive(g_empty(gb));
            uint32_t o[HD];
            tmem_ld32_sync(lane_addr + COL_O + (uint32_t)epi.obuf * HD, o);
            if (epi.row_ok) {
                const int64_t oo = p.os.off(epi.b, epi.s, epi.i, epi.h);
                __nv_bfloat16* op = p.out + oo;
#pragma unroll
                for (int q = 0; q < HD / 8; ++q) {
                    const uint32_t gv[4] = {gw[q].x, gw[q].y, gw[q].z, gw[q].w};
                    uint32_t ov[4], lv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // out = O / (l * (1 + exp(-g))), exp(-g) from the MUFU unit (a few ulp:
                        // the backward's D = sum(dout * out) feeds a cancellation, so the gate is
                        // taken in full fp32; arguments clamped to the exponent range)
                        const float e0 = ex2(fminf(-EVO_LOG2E * bf16lo(gv[e]), 126.0f));
                        const float e1 = ex2(fminf(-EVO_LOG2E * bf16hi(gv[e]), 126.0f));
                        const float o0 = __fdividef(__uint_as_float(o[q * 8 + 2 * e]), epi.l * (1.0f + e0));
                        const float o1 = __fdividef(__uint_as_float(o[q * 8 + 2 * e + 1]), epi.l * (1.0f + e1));
                        ov[e] = pack_bf16(o0, o1);
                        lv[e] = pack_bf16(o0 - bf16lo(ov[e]), o1 - bf16hi(ov[e]));   // rounding residual
                    }
                    *reinterpret_cast<uint4*>(op + q * 8) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
                    if (p.out_lo)
                        *reinterpret_cast<uint4*>(p.out_lo + oo + q * 8) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
                }
                p.lse[((int64_t)(epi.b * p.S + epi.s) * p.H + epi.h) * p.N + epi.i] =
                    (epi.ms + __log2f(epi.l)) * EVO_LN2;
            }
            epi.pending = false;
            return true;
        };
        for (int item = blockIdx.x, k = 0; ok && item < p.n_items; item += gridDim.x, ++k) {
            const Item itm = decode(p, item);
            const int s = itm.sg * NSUB + u;
            const int i = itm.i0 + r;
            const bool row_ok = s < p.S && i < p.N;
            const uint32_t col_o = COL_O + (uint32_t)(k & 1) * HD;
            // ms: running max in log2 units (the value subtracted inside exp2);
            // l: running sum of exp2(S * sc2 - ms)
            float ms = -INFINITY, l = 0.f;
            for (int j = 0; j < p.n_kv; ++j, ++tg) {
                ok = mbar_wait(s_full(u), tg & 1, abort_flag, kTimeoutBase | 0x201, p.wait_ns);
                if (!ok) break;
                tc_fence_after();
                uint32_t xr[BN];
                tmem_ld128_sync(lane_addr + COL_S, xr);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_free(u));

                // S already holds sqrt(C) times the whole logit (q.k, mask and bias); the
                // logit in log2 units is y = S * sc2, taken inside the exponent's FMA below
                const int valid = p.N - j * BN;      // keys beyond N are padding: exclude them
                if (valid < BN) {
#pragma unroll
                    for (int c = 0; c < BN; ++c)
                        if (c >= valid) xr[c] = __float_as_uint(-INFINITY);
                }
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < BN; c += 2) {
                    float m3;
                    asm("max.f32 %0, %1, %2, %3;" : "=f"(m3)
                        : "f"(mx[(c >> 1) & 3]), "f"(__uint_as_float(xr[c])), "f"(__uint_as_float(xr[c + 1])));
                    mx[(c >> 1) & 3] = m3;
                }
                const float mloc = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sc2;   // sc2 > 0

                // lazy rescale: move the running max only when this tile's max exceeds it by > 2^8
                const float mcand = mloc;
                const bool move = mcand > ms + RESCALE_THRESHOLD;
                const float ms_new = move ? mcand : ms;
                const float alpha = move ? ex2(ms - ms_new) : 1.0f;   // 0 on an item's first tile
                if (tg > 0) {
                    // PV of the previous tile must be done before P is overwritten and O rescaled.
                    ok = mbar_wait(o_full(u), (tg - 1) & 1, abort_flag, kTimeoutBase | 0x203, p.wait_ns);
                    if (!ok) break;
                    tc_fence_after();
                }
                if (j > 0 && __any_sync(0xffffffffu, move)) {
                    uint32_t o[HD];
                    tmem_ld32_sync(lane_addr + col_o, o);
#pragma unroll
                    for (int c = 0; c < HD; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st32(lane_addr + col_o, o);
                }
                // The two row groups take turns on the exponentials (MUFU): group 1
                // runs tile t after group 0's tile t, group 0 runs tile t+1 after
                // group 1's tile t, so one group's exponentials overlap the other's
                // loads, maxima and waits instead of competing with its exponentials.
                if (NSUB == 2) {
                    if (u == 1) ok = mbar_wait(exp_turn(1), tg & 1, abort_flag, kTimeoutBase | 0x205, p.wait_ns);
                    else if (tg > 0) ok = mbar_wait(exp_turn(0), (tg - 1) & 1, abort_flag, kTimeoutBase | 0x205, p.wait_ns);
                    if (!ok) break;
                }
                const uint64_t NEG_MS2 = f2(-ms_new, -ms_new);
                uint64_t rs2[2] = {0, 0};
#pragma unroll
                for (int half = 0; half < 2; ++half) {     // P stored 32 columns (64 keys) at a time
                    uint32_t pk[BN / 4];
#pragma unroll
                    for (int cc = 0; cc < BN / 4; ++cc) {
                        const int c = half * (BN / 4) + cc;
                        const uint64_t y2 =
                            ffma2(f2(__uint_as_float(xr[2 * c]), __uint_as_float(xr[2 * c + 1])), SC2, NEG_MS2);
                        uint64_t pp;
                        if (POLY_EVERY > 0 && c % (POLY_EVERY > 0 ? POLY_EVERY : 1) == POLY_EVERY - 1)
                            pp = exp2_poly2(y2);
                        else
                            pp = f2(ex2(f2lo(y2)), ex2(f2hi(y2)));
                        const float p0 = f2lo(pp), p1 = f2hi(pp);
                        rs2[c & 1] = (c < 2) ? pp : fadd2(rs2[c & 1], pp);
                        pk[cc] = pack_bf16(p0, p1);
                    }
                    tmem_st32(lane_addr + COL_P + half * 32, pk);
                }
                if (NSUB == 2) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(exp_turn(1 - u));
                }
                const uint64_t rsum = fadd2(rs2[0], rs2[1]);
                l = fmaf(l, alpha, f2lo(rsum) + f2hi(rsum));
                ms = ms_new;
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full(u));
                // the previous item's epilogue: its last PV finished before this
                // tile's P was written (the o_full wait above)
                if (j == 0 && epi.pending && !run_epilogue()) {
                    ok = false;
                    break;
                }
            }
            if (!ok) break;
            epi.pending = true;
            epi.row_ok = row_ok;
            epi.b = itm.b; epi.s = s; epi.i = i; epi.h = itm.h; epi.obuf = k & 1; epi.k = k;
            epi.l = l; epi.ms = ms;
        }
        if (ok && epi.pending) {   // the last item: wait for its last PV
            ok = mbar_wait(o_full(u), (tg - 1) & 1, abort_flag, kTimeoutBase | 0x204, p.wait_ns);
            if (ok) {
                tc_fence_after();
                ok = run_epilogue();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMma) {
        tc_fence_after();
        tmem_dealloc(tmem, L::tmem_cols);
    }
}

}  // namespace fwd
}  // namespace evo
