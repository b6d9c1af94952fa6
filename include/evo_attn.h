/*
 * evo_attn.h -- C-ABI of the B200 (sm_100a) Evoformer attention with pair bias.
 *
 * The operation.  For batch b, row s (an MSA sequence for MSA-row attention,
 * a pair row for triangle attention), head h, query residue i and key j:
 *
 *   x[i,j] = (q[b,s,i,h,:] . k[b,s,j,h,:]) / sqrt(C)
 *            + mask_bias[b,s,0,0,j] + pair_bias[b,0,h,i,j]
 *   out[b,s,i,h,:] = sigmoid(g[b,s,i,h,:]) * sum_j softmax_j(x[i,:])[j] * v[b,s,j,h,:]
 *   lse[b,s,h,i]   = log sum_j exp(x[i,j])            (natural log, fp32)
 *
 * This is the attention whose additive, broadcast pair-bias term MegaFold's
 * EvoFlash-3D handles with an online, numerically stable softmax computed
 * tile by tile in on-chip memory (MegaFold summary, section "EvoFlash-3D :
 * Attention 3D Econome en Memoire"), and the triangle attention around a node
 * whose logits are O(N_res^3 * n_heads) ("Evoformer: the memory wall ZeRO
 * cannot move", sections "Where the memory goes" and "The three operations").
 * The library never materialises those logits: peak extra memory is linear in
 * B*H*N^2 and in the per-row tensors.
 *
 * Call shapes.  All per-row tensors are logical [B, S, N, H, C] with the C
 * axis contiguous and the other four axes given by element strides:
 *   - MSA-row attention:       rows s = MSA sequences, contiguous strides;
 *   - triangle, starting node: rows s = pair rows i, contiguous strides;
 *   - triangle, ending node:   the same op on the transposed pair, expressed by
 *     swapping the s and n strides of a tensor stored as [B, N, N, H, C]
 *     (no copy).
 *
 * Ownership and execution.  The caller allocates every buffer (device
 * memory), including the backward workspace.  The library never allocates,
 * frees or synchronises in evo_attn_fwd / evo_attn_bwd: they validate the
 * arguments on the host, enqueue kernels on `stream` and return.  Outputs are
 * overwritten, never accumulated into.
 *
 * Errors.  Argument problems are found on the host before any launch and
 * returned as a status (nothing is enqueued then).  A launch failure returns
 * EVO_ERR_CUDA.  There is no fallback: a shape the kernels do not cover is
 * EVO_ERR_UNSUPPORTED, never a silent slower path and never a CPU path.
 * Every wait inside a kernel is bounded; a wait that runs out sets a device
 * status word, the kernel returns early, and evo_attn_device_status() reports
 * EVO_ERR_DEVICE_TIMEOUT.
 */
#ifndef EVO_ATTN_H_
#define EVO_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EVO_OK = 0,
    EVO_ERR_INVALID_ARG = 1,         /* null pointer, negative size, shape mismatch      */
    EVO_ERR_UNSUPPORTED = 2,         /* valid, but outside what the kernels implement    */
    EVO_ERR_WORKSPACE_TOO_SMALL = 3, /* backward workspace smaller than the query says   */
    EVO_ERR_CUDA = 4,                /* a CUDA runtime/driver call or launch failed      */
    EVO_ERR_DEVICE_TIMEOUT = 5       /* a bounded in-kernel wait ran out (see below)     */
} evo_status_t;

typedef enum {
    EVO_DTYPE_BF16 = 0,  /* bf16 storage, fp32 accumulation, tcgen05 tensor cores    */
    EVO_DTYPE_F32 = 1    /* fp32 storage and arithmetic on the FMA pipe (no TF32)    */
} evo_dtype_t;

/* Logical sizes: batch B, rows S (N_seq), residues N (N_res), heads H, head dim C. */
typedef struct {
    int64_t B, S, N, H, C;
} evo_shape_t;

/* Element strides of a logical [B, S, N, H, C] tensor; the C stride is 1. */
typedef struct {
    int64_t b, s, n, h;
} evo_strides_t;

/* Limits of the kernels (EVO_ERR_UNSUPPORTED outside them).
 *   bf16: C == 32; N % 8 == 0; every stride a multiple of 8 elements; every
 *         pointer 16-byte aligned.
 *   f32:  1 <= C <= 64; any N >= 1; pointers 4-byte aligned.
 * Sizes B, S, N or H equal to 0 are an empty call: EVO_OK, nothing launched
 * except that evo_attn_bwd zero-fills d_pair_bias when S == 0.               */

/*
 * Bytes of device workspace evo_attn_bwd needs for this shape and dtype
 * (a pure function of its arguments).  Returns 0 for a null or invalid shape.
 * The workspace holds the gated output gradient, the row sums D_i, the fp32
 * dq accumulator, a transposed copy of pair_bias and the per-row-group
 * partial sums of d_pair_bias; all of it is linear in the per-row tensors and
 * in B*H*N^2.
 */
size_t evo_attn_bwd_workspace_bytes(const evo_shape_t* shape, evo_dtype_t dtype);

/*
 * Forward pass.
 *   shape        logical sizes (see above).
 *   dtype        element type of q, k, v, g, mask_bias, pair_bias and out.
 *   q, k, v, g   device pointers, logical [B,S,N,H,C] with strides `in_str`.
 *   in_str       element strides shared by q, k, v and g.
 *   mask_bias    device pointer, contiguous [B,S,1,1,N] additive mask over the
 *                keys (e.g. -1e9 for padding), or NULL for none.
 *   pair_bias    device pointer, contiguous [B,1,H,N,N] indexed [b,h,i,j]
 *                (query i, key j), or NULL for none.
 *   out          device pointer, logical [B,S,N,H,C] with strides `out_str`.
 *   out_lo       bf16 only, optional (NULL = not written): device pointer with
 *                `out`'s layout and strides that receives the rounding residual
 *                of out, bf16(out_fp32 - out), so that out + out_lo carries
 *                about 16 significant bits of the fp32 result.  Passed back to
 *                evo_attn_bwd, it makes the row sums D_i = sum_c dout*out exact
 *                to that precision; d_pair_bias adds the error of D_i over all
 *                rows s, so this is what keeps its error small at large N_seq.
 *                Ignored (may be NULL) on the fp32 path.
 *   lse          device pointer, contiguous fp32 [B,S,H,N]: the natural-log
 *                sum-exp of each logit row, saved for the backward pass.
 *   stream       cudaStream_t to enqueue on (NULL = legacy default stream).
 */
evo_status_t evo_attn_fwd(const evo_shape_t* shape, evo_dtype_t dtype,
                          const void* q, const void* k, const void* v, const void* g,
                          const evo_strides_t* in_str,
                          const void* mask_bias, const void* pair_bias,
                          void* out, void* out_lo, const evo_strides_t* out_str,
                          float* lse, void* stream);

/*
 * Backward pass.  Recomputes the softmax from q, k, the biases and the saved
 * lse (no logits are stored), and returns every input gradient:
 *   dq, dk, dv, dg    device pointers, logical [B,S,N,H,C] with strides
 *                     `grad_str`, same dtype as the inputs.
 *   d_pair_bias       device pointer, contiguous fp32 [B,1,H,N,N]: the sum over
 *                     all rows s of dL/dx.  It is bitwise reproducible: partial
 *                     sums over fixed row groups are added in a fixed order,
 *                     with no floating-point atomics.
 *   out, dout         the forward output and its gradient (strides `out_str`).
 *   out_lo            the forward's out_lo (bf16 only), or NULL: without it D_i
 *                     is taken from the bf16 out alone.
 *   lse               the forward's saved lse.
 *   workspace         device buffer of at least evo_attn_bwd_workspace_bytes()
 *                     bytes, 256-byte aligned; contents need not be initialised.
 * mask_bias gets no gradient (it is a constant).  dq is accumulated in fp32
 * across key tiles with atomic adds, so its last bits may vary run to run;
 * every other output is deterministic.
 */
evo_status_t evo_attn_bwd(const evo_shape_t* shape, evo_dtype_t dtype,
                          const void* q, const void* k, const void* v, const void* g,
                          const evo_strides_t* in_str,
                          const void* mask_bias, const void* pair_bias,
                          const void* out, const void* out_lo, const void* dout,
                          const evo_strides_t* out_str, const float* lse,
                          void* dq, void* dk, void* dv, void* dg, const evo_strides_t* grad_str,
                          float* d_pair_bias,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass that allocates nothing and takes no workspace argument.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot call cudaMalloc and have no device buffer of their own to lend
 * as workspace -- for example a plug-in that runs inside a host framework
 * which owns all device memory and forbids its extensions to allocate, or a
 * service whose device memory footprint is fixed when it starts.
 *
 * Same arguments and results as evo_attn_bwd, minus the workspace.  Instead
 * the library uses a fixed scratch area of EVO_ATTN_NOALLOC_WORKSPACE_BYTES
 * (32 MiB) in device memory that exists from the moment the library is loaded
 * on a device until the process exits; every GPU that loads the library holds
 * it.  A shape whose workspace (evo_attn_bwd_workspace_bytes) is larger than
 * that is rejected with EVO_ERR_WORKSPACE_TOO_SMALL before anything is
 * enqueued -- for instance bf16 with B=1, S=32, N=256, H=4, C=32 fits, the
 * 128-row, 8-head MSA-row shape at N=256 does not.
 *
 * The first call on a device looks up the scratch area's device address (a
 * host-side query that allocates nothing) and caches it for the device's
 * current context; make that first call before any stream capture on that
 * device.  After cudaDeviceReset the next call runs in a new context and
 * looks the address up again (again before any stream capture).  All calls share the one scratch
 * area and it keeps the last call's contents; every part of it that must
 * start at zero is cleared by the call itself.  Calls whose kernels overlap
 * on the GPU (different streams, or different host threads, with no ordering
 * between them) race on the scratch area and corrupt each other's results:
 * order them on one stream, or use evo_attn_bwd with separate workspaces.
 */
#define EVO_ATTN_NOALLOC_WORKSPACE_BYTES ((size_t)32 << 20)
evo_status_t evo_attn_bwd_noalloc(const evo_shape_t* shape, evo_dtype_t dtype,
                                  const void* q, const void* k, const void* v, const void* g,
                                  const evo_strides_t* in_str,
                                  const void* mask_bias, const void* pair_bias,
                                  const void* out, const void* out_lo, const void* dout,
                                  const evo_strides_t* out_str, const float* lse,
                                  void* dq, void* dk, void* dv, void* dg, const evo_strides_t* grad_str,
                                  float* d_pair_bias, void* stream);

/*
 * Fused pre-attention projection: y = LayerNorm(x) @ w + bias, for every row
 * of a representation, without writing the normalised rows to memory -- the
 * LayerNorm + linear pair that EvoFusion fuses (MegaFold summary, section
 * "EvoFusion : Pile d'Operateurs Fusionnes").
 *
 *   mean_r = (1/c_in) sum_k x[r,k],  var_r = (1/c_in) sum_k (x[r,k] - mean_r)^2
 *   y[r,o] = sum_k ((x[r,k] - mean_r) / sqrt(var_r + eps) * ln_w[k] + ln_b[k]) * w[k,o] + bias[o]
 *
 * x: bf16 [rows, c_in], rows contiguous (pitch c_in); ln_w, ln_b: fp32 [c_in]
 * (NULL = ones / zeros); w: bf16 [c_in, n_out] row-major; bias: fp32 [n_out]
 * or NULL; y: bf16 [rows, n_out] with row pitch ldy >= n_out (elements).
 * LayerNorm statistics and the products accumulate in fp32 (tensor cores).
 * With w = [w_q | w_k | w_v | w_g] (each H*c wide) the column blocks of y are
 * q, k, v and g of the attention, as [B, S, N, H, c] views with row stride
 * 4*H*c that evo_attn_fwd / evo_attn_bwd take through their strides.
 * Supported: c_in a multiple of 64 up to 256, n_out a multiple of 128, ldy a
 * multiple of 8, x / w / y / bias 16-byte aligned (else EVO_ERR_UNSUPPORTED); rows
 * == 0 is a no-op.  Only y[0:rows, 0:n_out] is written (columns n_out..ldy-1
 * keep their contents).  The normalised activations are rounded to bf16
 * before the product, y to bf16 on the store.  Stream-ordered, no
 * allocation, no synchronisation; the kernel's waits are bounded, and one
 * that gives up is reported by evo_attn_device_status.
 */
evo_status_t evo_ln_linear(int64_t rows, int64_t c_in, int64_t n_out, const void* x,
                           const float* ln_w, const float* ln_b, float eps,
                           const void* w, const float* bias, void* y, int64_t ldy, void* stream);

/*
 * Pair-bias projection of the pair representation: the same LayerNorm +
 * linear with one output per head, written in the layout the attention reads,
 *   pair_bias[b, h, i, j] = sum_k LN(z[b, i, j, :])[k] * w[k, h] + bias[h].
 * z: bf16 [B, N, N, c_z] contiguous; ln_w, ln_b: fp32 [c_z] (NULL = ones /
 * zeros); w: bf16 [c_z, H]; bias: fp32 [H] or NULL; pair_bias: bf16
 * [B, 1, H, N, N] contiguous.  Supported: c_z a multiple of 8 up to 1024,
 * H <= 16, z 16-byte aligned.  Stream-ordered, no allocation.
 */
evo_status_t evo_ln_pair_bias(int64_t B, int64_t N, int64_t c_z, int64_t H, const void* z,
                              const float* ln_w, const float* ln_b, float eps,
                              const void* w, const float* bias, void* pair_bias, void* stream);

/*
 * The contraction of the triangular multiplicative update ("Evoformer: the
 * memory wall ZeRO cannot move", section "The three operations"): every edge
 * (i, j) gathers the third residues k, channel by channel,
 *
 *   outgoing (incoming == 0):  z[b,c,i,j] = sum_k a[b,c,i,k] * bb[b,c,j,k]
 *   incoming (incoming != 0):  z[b,c,i,j] = sum_k a[b,c,k,i] * bb[b,c,k,j]
 *
 * one N x N x N matrix product per (b, c).  a, bb, z: bf16 [B, C, N, N]
 * contiguous (channel-first: the matrix of each (b, c) contiguous); products
 * accumulate in fp32 on the tensor cores and z is rounded to bf16 on the
 * store.  Supported: N a multiple of 8, a / bb / z 16-byte aligned, B*C and
 * N below 2^31 (else EVO_ERR_UNSUPPORTED); B, C or N == 0 is a no-op.
 * Stream-ordered, no allocation, no synchronisation; the kernel's waits are
 * bounded, and one that gives up is reported by evo_attn_device_status.
 */
evo_status_t evo_tri_mul(int64_t B, int64_t C, int64_t N, const void* a, const void* bb, int incoming,
                         void* z, void* stream);

/*
 * Outer product mean, the bridge from the MSA to the pair representation
 * ("Evoformer: the memory wall ZeRO cannot move", section "The three
 * operations"): the outer product of MSA columns i and j averaged over the S
 * sequences,
 *
 *   out[b, i, c1, j, c2] = (1/S) sum_s a[b, s, i, c1] * bb[b, s, j, c2]
 *
 * a: bf16 [B, S, N, Ca], bb: bf16 [B, S, N, Cb], both contiguous (the MSA
 * representation's layout); out: bf16 [B, N, Ca, N, Cb] contiguous, i.e. for
 * each b the (N Ca) x (N Cb) matrix a^T bb / S -- the pair layout
 * [B, N, N, Ca, Cb] is its view with axes 2 and 3 swapped.  Products
 * accumulate in fp32 on the tensor cores; the 1/S scale is applied in fp32
 * before the bf16 rounding.  Supported: N*Ca and N*Cb multiples of 8,
 * pointers 16-byte aligned, sizes below 2^31 (else EVO_ERR_UNSUPPORTED);
 * B or N == 0 is a no-op; S == 0 is EVO_ERR_INVALID_ARG (no mean).
 * Stream-ordered, no allocation, no synchronisation; the kernel's waits are
 * bounded, and one that gives up is reported by evo_attn_device_status.
 */
evo_status_t evo_outer_product_mean(int64_t B, int64_t S, int64_t N, int64_t Ca, int64_t Cb, const void* a,
                                    const void* bb, void* out, void* stream);

/*
 * Fixed-order sum of fp32 partial results: the exchange step of a backward
 * pass whose rows s are split over several GPUs, the way a sequence-parallel
 * group partitions the pair tensor (MegaFold summary, section "EvoSP-3D").
 * Rows s are independent problems that share the additive pair bias, which
 * is broadcast over them (same page, section "EvoFlash-3D"), so every input
 * gradient but d_pair_bias stays on the GPU that holds its row, and
 * d_pair_bias -- the sum over all s of dL/dx -- is the sum of the per-GPU
 * partials that evo_attn_bwd returns for each GPU's rows:
 *
 *   out[i] = (...((parts[0][i] + parts[1][i]) + parts[2][i]) ...) + parts[count-1][i]
 *
 * in fp32, each addition rounded to nearest, left to right: every caller that
 * passes the same partials in the same (rank) order gets the same bits.
 *   count   number of partials, 1 <= count <= EVO_MAX_PARTIALS
 *           (EVO_ERR_INVALID_ARG below 1, EVO_ERR_UNSUPPORTED above).
 *   parts   HOST array of `count` device pointers, each to n fp32 values; it
 *           is read during the call only.  The pointers may be slices of
 *           one all-gathered buffer, or any memory this device can load from.
 *   n       elements per partial; 0 is a no-op, negative EVO_ERR_INVALID_ARG.
 *   out     device pointer to n fp32 values.  It may be one of parts[r]
 *           (element-wise in place); any other overlap is undefined.
 * NULL pointers are EVO_ERR_INVALID_ARG; pointers not 4-byte aligned are
 * EVO_ERR_UNSUPPORTED.  All 16-byte aligned pointers take 16-byte loads.
 * Stream-ordered, no allocation, no synchronisation, no waits.
 */
#define EVO_MAX_PARTIALS 64
evo_status_t evo_sum_partials(int64_t count, const float* const* parts, int64_t n, float* out, void* stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char* evo_status_string(evo_status_t status);

/*
 * Reports whether any kernel on the current device gave up on a bounded wait
 * since the last clear.  Synchronises the current device first.  Returns
 * EVO_OK or EVO_ERR_DEVICE_TIMEOUT (EVO_ERR_CUDA if the device cannot be
 * queried).  If `clear` is non-zero the status word is reset to zero.
 */
evo_status_t evo_attn_device_status(int clear);

/*
 * Limit, in nanoseconds, of the bounded in-kernel waits of the forward kernel
 * and of the backward's d_pair_bias kernel launched after this call (default
 * 2e9, i.e. 2 s); returns the previous limit.  It exists so that the timeout path can be exercised without
 * breaking anything: with a limit of 0 every wait that is not satisfied at
 * once gives up, the kernel drains its own copies and tensor-core work (those
 * drains always keep the 2 s default) and returns, and
 * evo_attn_device_status() reports EVO_ERR_DEVICE_TIMEOUT.  The outputs of
 * such a call are undefined; the context stays usable.  Affects every device;
 * not for use while other threads launch attention kernels.
 */
uint64_t evo_attn_set_wait_limit_ns(uint64_t ns);

/*
 * y[i] = 2^x[i] for n fp32 values (device pointers, 4-byte aligned), computed
 * by the FMA-pipe exponential that the attention kernels can take in place of
 * the MUFU unit for a share of their exponentials (build switches
 * EVO_FWD_POLY_EVERY and EVO_DBIAS_POLY_EVERY, off by default): a cubic in the
 * fraction after a round-to-nearest split of x, relative error below 8e-5 for
 * -125 <= x <= 126;
 * arguments below -125 give 2^-125.  Exported so that the device function
 * itself can be checked against 2^x on the GPU.  Returns EVO_ERR_INVALID_ARG
 * for n < 0 or a null pointer with n > 0.
 */
evo_status_t evo_exp2_fma(const float* x, float* y, int64_t n, void* stream);

/* ABI version, major * 10000 + minor * 100 + patch. */
int evo_attn_version(void);

/* Number of CUDA kernels this library has enqueued in this process so far
 * (all devices, all streams).  Host-side counter; never synchronises. */
uint64_t evo_attn_launch_count(void);

/*
 * Per-kernel device timing (off by default).  While switched on, each
 * evo_attn_fwd / evo_attn_bwd / evo_ln_linear / evo_ln_pair_bias / evo_tri_mul /
 * evo_outer_product_mean call records
 * a pair of CUDA events on its own `stream` around its main kernel, and
 * evo_attn_bwd a second pair around all of its kernels, so that a caller can
 * see how a step's device time splits between the kernels without a
 * profiler.  The events come from a pool kept
 * by the library (created on first use, reused afterwards); recording them
 * adds no kernel and no synchronisation.  Recording is best-effort: if an
 * event cannot be created or recorded that call simply goes untimed.
 *
 * evo_attn_timing_collect blocks until every phase recorded since the last
 * collect has completed, adds up the elapsed times per phase into *out
 * (calls and milliseconds) and forgets them.  It returns EVO_ERR_INVALID_ARG
 * for a NULL `out` and EVO_ERR_CUDA if an event could not be waited on or
 * read (that phase is then left out of the sums).  Both functions are safe to
 * call from several host threads.
 */
#define EVO_TIMING_PHASES 8
enum {
    EVO_PHASE_FWD_MAIN = 0,   /* the forward kernel                         */
    EVO_PHASE_BWD_MAIN = 1,   /* the backward's dq, dk, dv kernel            */
    EVO_PHASE_BWD_ALL = 2,    /* every kernel and memset of one evo_attn_bwd */
    EVO_PHASE_PROJ = 3,       /* the evo_ln_linear kernel                    */
    EVO_PHASE_PAIR_BIAS = 4,  /* the evo_ln_pair_bias kernel                 */
    EVO_PHASE_TRI_MUL = 5,    /* the evo_tri_mul kernel                      */
    EVO_PHASE_OPM = 6,        /* the evo_outer_product_mean kernel           */
    EVO_PHASE_BWD_DBIAS = 7   /* the backward's d_pair_bias kernel           */
};
typedef struct {
    uint64_t calls[EVO_TIMING_PHASES];
    double ms[EVO_TIMING_PHASES];
} evo_timing_t;
evo_status_t evo_attn_timing_enable(int on);
evo_status_t evo_attn_timing_collect(evo_timing_t* out);

#ifdef __cplusplus
}
#endif

#endif /* EVO_ATTN_H_ */
