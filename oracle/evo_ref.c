/*
 * evo_ref.c -- plain fp64 CPU oracle for Evoformer attention with pair bias.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (per batch b, row s, head h, query i, key j):
 *
 *   x[i,j]  = (sum_c q[b,s,i,h,c] * k[b,s,j,h,c]) / sqrt(C)
 *             + mask_bias[b,s,j] + pair_bias[b,h,i,j]
 *   lse[i]  = log(sum_j exp(x[i,j]))          (computed as m + log(sum exp(x - m)))
 *   P[i,j]  = exp(x[i,j] - lse[i])
 *   A[i,:]  = sum_j P[i,j] * v[b,s,j,h,:]
 *   out     = sigmoid(g) * A
 *
 * This is the attention with an additive, broadcast pair-bias term that the
 * MegaFold summary describes for EvoFlash-3D ("EvoFlash-3D : Attention 3D
 * Econome en Memoire"), and the triangle attention of "Evoformer: the memory
 * wall ZeRO cannot move" (section "The three operations"), whose logits are
 * O(N_res^3 * n_heads) (section "Where the memory goes", first equation).
 * The oracle materialises one logit row at a time in fp64: it is the plain
 * definition, not a tiled or online-softmax rewrite.
 *
 * Backward, given dout (chain rule of the definition above):
 *   sig   = sigmoid(g);   dA = dout * sig;   dg = dout * A * sig * (1 - sig)
 *   dP[i,j] = sum_c dA[i,c] * v[j,c];        D[i] = sum_j P[i,j] * dP[i,j]
 *   dS[i,j] = P[i,j] * (dP[i,j] - D[i])
 *   dv[j] = sum_i P[i,j] dA[i];   dq[i] = sum_j dS[i,j] k[j] / sqrt(C);
 *   dk[j] = sum_i dS[i,j] q[i] / sqrt(C)
 *   d_pair_bias[b,h,i,j] = sum_s dS^{(b,s,h)}[i,j]     (mask_bias is a constant)
 *
 * Layouts (all contiguous, fp64):
 *   q, g, out, dout, dq, dg : [B, S, Nq, H, C]
 *   k, v, dk, dv            : [B, S, Nk, H, C]
 *   mask_bias               : [B, S, Nk]        (NULL = zeros)
 *   pair_bias, d_pair_bias  : [B, H, Nq, Nk]    (NULL = zeros)
 *   lse                     : [B, S, H, Nq]
 * Nq may differ from Nk so that a caller can evaluate the definition at a
 * subset of query rows (a smaller, equally valid problem).
 *
 * The file also holds the fused pre-attention projection (LayerNorm + linear,
 * evo_ref_ln_linear below) that produces q, k, v, g and the pair bias, and
 * the contraction of the triangular multiplicative update (evo_ref_tri_mul),
 * and the outer product mean (evo_ref_outer_product_mean).
 *
 * Planted mistakes (mutation testing of the pins): building with
 * -DEVO_REF_MUTANT=n swaps in one deliberate error, see mutant_* below.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef EVO_REF_MUTANT
#define EVO_REF_MUTANT 0
#endif

typedef struct {
    int64_t B, S, Nq, Nk, H, C;
} evo_ref_dims;

/* Index helpers for the layouts above. */
static inline int64_t ix_q(const evo_ref_dims* d, int64_t b, int64_t s, int64_t i, int64_t h) {
    return (((b * d->S + s) * d->Nq + i) * d->H + h) * d->C;
}
static inline int64_t ix_k(const evo_ref_dims* d, int64_t b, int64_t s, int64_t j, int64_t h) {
    return (((b * d->S + s) * d->Nk + j) * d->H + h) * d->C;
}
static inline int64_t ix_mask(const evo_ref_dims* d, int64_t b, int64_t s, int64_t j) {
    return (b * d->S + s) * d->Nk + j;
}
static inline int64_t ix_bias(const evo_ref_dims* d, int64_t b, int64_t h, int64_t i, int64_t j) {
    return ((b * d->H + h) * d->Nq + i) * d->Nk + j;
}
static inline int64_t ix_lse(const evo_ref_dims* d, int64_t b, int64_t s, int64_t h, int64_t i) {
    return ((b * d->S + s) * d->H + h) * d->Nq + i;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* Logit row x[0..Nk) for (b, s, h, query i), straight from the definition. */
static void logit_row(const evo_ref_dims* d, const double* q, const double* k,
                      const double* mask, const double* bias,
                      int64_t b, int64_t s, int64_t h, int64_t i, double* x) {
    const double* qi = q + ix_q(d, b, s, i, h);
#if EVO_REF_MUTANT == 3
    const double scale = 1.0 / (double)d->C;           /* mutant: 1/C instead of 1/sqrt(C) */
#else
    const double scale = 1.0 / sqrt((double)d->C);
#endif
    for (int64_t j = 0; j < d->Nk; ++j) {
        const double* kj = k + ix_k(d, b, s, j, h);
        double dot = 0.0;
        for (int64_t c = 0; c < d->C; ++c) dot += qi[c] * kj[c];
        double xij = dot * scale;
#if EVO_REF_MUTANT != 2                                /* mutant 2: mask dropped */
        if (mask) xij += mask[ix_mask(d, b, s, j)];
#endif
#if EVO_REF_MUTANT == 5                                /* mutant 5: bias read transposed */
        if (bias) xij += bias[ix_bias(d, b, h, j, i)];
#elif EVO_REF_MUTANT != 1                              /* mutant 1: pair bias dropped */
        if (bias) xij += bias[ix_bias(d, b, h, i, j)];
#endif
        x[j] = xij;
    }
}

/* In place: x <- softmax(x); returns lse = m + log(sum exp(x - m)). */
static double softmax_row(int64_t n, double* x) {
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) m = x[j] > m ? x[j] : m;
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) l += exp(x[j] - m);
    const double lse = m + log(l);
    for (int64_t j = 0; j < n; ++j) x[j] = exp(x[j] - lse);
    return lse;
}

static double gate(double g) {
#if EVO_REF_MUTANT == 4
    (void)g;
    return 1.0;                                        /* mutant 4: gate omitted */
#else
    return sigmoid(g);
#endif
}

/* Everything one query row contributes to the backward pass.
 * In:  the row's P (from logit_row + softmax_row).
 * Out: A[C], dA[C], dP/dS row (dS written over dp), D.                  */
static void backward_row(const evo_ref_dims* d, const double* v, const double* g,
                         const double* dout, int64_t b, int64_t s, int64_t h, int64_t i,
                         const double* p, double* A, double* dA, double* ds, double* dg_row) {
    const int64_t C = d->C;
    const double* gi = g + ix_q(d, b, s, i, h);
    const double* doi = dout + ix_q(d, b, s, i, h);
    for (int64_t c = 0; c < C; ++c) A[c] = 0.0;
    for (int64_t j = 0; j < d->Nk; ++j) {
        const double* vj = v + ix_k(d, b, s, j, h);
        for (int64_t c = 0; c < C; ++c) A[c] += p[j] * vj[c];
    }
    for (int64_t c = 0; c < C; ++c) {
        const double sg = gate(gi[c]);
        dA[c] = doi[c] * sg;
        if (dg_row) dg_row[c] = doi[c] * A[c] * sg * (1.0 - sg);
    }
    double D = 0.0;
    for (int64_t j = 0; j < d->Nk; ++j) {
        const double* vj = v + ix_k(d, b, s, j, h);
        double dp = 0.0;
        for (int64_t c = 0; c < C; ++c) dp += dA[c] * vj[c];
        ds[j] = dp;                                    /* dP for now */
        D += p[j] * dp;
    }
#if EVO_REF_MUTANT == 6
    D = -D;                                            /* mutant 6: sign of D flipped */
#endif
    for (int64_t j = 0; j < d->Nk; ++j) ds[j] = p[j] * (ds[j] - D);
}

int evo_ref_forward(const evo_ref_dims* d, const double* q, const double* k, const double* v,
                    const double* g, const double* mask, const double* bias,
                    double* out, double* lse) {
    if (!d || d->B < 0 || d->S < 0 || d->Nq < 0 || d->Nk < 1 || d->H < 0 || d->C < 1) return 1;
    const int64_t nslice = d->B * d->S * d->H;
#pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)d->Nk);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < nslice; ++t) {
            const int64_t h = t % d->H, s = (t / d->H) % d->S, b = t / (d->H * d->S);
            for (int64_t i = 0; i < d->Nq; ++i) {
                logit_row(d, q, k, mask, bias, b, s, h, i, x);
                const double l = softmax_row(d->Nk, x);
                if (lse) lse[ix_lse(d, b, s, h, i)] = l;
                const double* gi = g + ix_q(d, b, s, i, h);
                double* oi = out + ix_q(d, b, s, i, h);
                for (int64_t c = 0; c < d->C; ++c) {
                    double a = 0.0;
                    for (int64_t j = 0; j < d->Nk; ++j) a += x[j] * v[ix_k(d, b, s, j, h) + c];
                    oi[c] = gate(gi[c]) * a;
                }
            }
        }
        free(x);
    }
    return 0;
}

/* Gradients of the definition above.  Any output pointer may be NULL.
 * dk and dv are sums over all Nq query rows, so they are only the true
 * gradients when the caller passes every query row (Nq == Nk problem). */
int evo_ref_backward(const evo_ref_dims* d, const double* q, const double* k, const double* v,
                     const double* g, const double* mask, const double* bias,
                     const double* dout, double* dq, double* dk, double* dv, double* dg,
                     double* d_pair_bias) {
    if (!d || d->B < 0 || d->S < 0 || d->Nq < 0 || d->Nk < 1 || d->H < 0 || d->C < 1) return 1;
    const int64_t C = d->C;
    const double rs = 1.0 / sqrt((double)C);
    const int64_t nslice = d->B * d->S * d->H;

    /* Pass 1: per (b, s, h) slice -- dq, dg (row-local) and dk, dv (sums over i). */
    const int pass1 = dq || dk || dv || dg;
#pragma omp parallel if (pass1)
    if (pass1) {
        double* p = (double*)malloc(sizeof(double) * (size_t)d->Nk);
        double* ds = (double*)malloc(sizeof(double) * (size_t)d->Nk);
        double* A = (double*)malloc(sizeof(double) * (size_t)C);
        double* dA = (double*)malloc(sizeof(double) * (size_t)C);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < nslice; ++t) {
            const int64_t h = t % d->H, s = (t / d->H) % d->S, b = t / (d->H * d->S);
            for (int64_t j = 0; j < d->Nk; ++j) {
                if (dk) memset(dk + ix_k(d, b, s, j, h), 0, sizeof(double) * (size_t)C);
                if (dv) memset(dv + ix_k(d, b, s, j, h), 0, sizeof(double) * (size_t)C);
            }
            for (int64_t i = 0; i < d->Nq; ++i) {
                logit_row(d, q, k, mask, bias, b, s, h, i, p);
                softmax_row(d->Nk, p);
                backward_row(d, v, g, dout, b, s, h, i, p, A, dA,
                             ds, dg ? dg + ix_q(d, b, s, i, h) : NULL);
                const double* qi = q + ix_q(d, b, s, i, h);
                double* dqi = dq ? dq + ix_q(d, b, s, i, h) : NULL;
                if (dqi) for (int64_t c = 0; c < C; ++c) dqi[c] = 0.0;
                for (int64_t j = 0; j < d->Nk; ++j) {
                    const double* kj = k + ix_k(d, b, s, j, h);
                    if (dqi) for (int64_t c = 0; c < C; ++c) dqi[c] += ds[j] * kj[c] * rs;
                    if (dk) {
                        double* dkj = dk + ix_k(d, b, s, j, h);
#if EVO_REF_MUTANT == 7
                        for (int64_t c = 0; c < C; ++c) dkj[c] += ds[j] * qi[c];     /* mutant 7: no 1/sqrt(C) */
#else
                        for (int64_t c = 0; c < C; ++c) dkj[c] += ds[j] * qi[c] * rs;
#endif
                    }
                    if (dv) {
                        double* dvj = dv + ix_k(d, b, s, j, h);
                        for (int64_t c = 0; c < C; ++c) dvj[c] += p[j] * dA[c];
                    }
                }
            }
        }
        free(p); free(ds); free(A); free(dA);
    }

    /* Pass 2: d_pair_bias rows, summed over s in order, one (b, h, i) per task. */
    if (d_pair_bias) {
        const int64_t nrow = d->B * d->H * d->Nq;
#pragma omp parallel
        {
            double* p = (double*)malloc(sizeof(double) * (size_t)d->Nk);
            double* ds = (double*)malloc(sizeof(double) * (size_t)d->Nk);
            double* A = (double*)malloc(sizeof(double) * (size_t)C);
            double* dA = (double*)malloc(sizeof(double) * (size_t)C);
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < nrow; ++t) {
                const int64_t i = t % d->Nq, h = (t / d->Nq) % d->H, b = t / (d->Nq * d->H);
                double* row = d_pair_bias + ix_bias(d, b, h, i, 0);
                for (int64_t j = 0; j < d->Nk; ++j) row[j] = 0.0;
                for (int64_t s = 0; s < d->S; ++s) {
                    logit_row(d, q, k, mask, bias, b, s, h, i, p);
                    softmax_row(d->Nk, p);
                    backward_row(d, v, g, dout, b, s, h, i, p, A, dA, ds, NULL);
                    for (int64_t j = 0; j < d->Nk; ++j) row[j] += ds[j];
                }
            }
            free(p); free(ds); free(A); free(dA);
        }
    }
    return 0;
}

/*
 * Fused pre-attention projection: the LayerNorm of every row of a
 * representation (MSA or pair) followed by its linear projections, the pair
 * of operators that EvoFusion computes without writing the normalised tensor
 * to memory (MegaFold summary, section "EvoFusion : Pile d'Operateurs
 * Fusionnes").  For each row r of x [rows, c_in]:
 *
 *   mu      = (1/c_in) sum_k x[r,k]
 *   var     = (1/c_in) sum_k (x[r,k] - mu)^2            (biased, as LayerNorm)
 *   n[k]    = (x[r,k] - mu) / sqrt(var + eps) * ln_w[k] + ln_b[k]
 *   y[r,o]  = sum_k n[k] * w[k,o] + bias[o]               (w: [c_in, n_out])
 *
 * ln_w NULL means ones, ln_b and bias NULL mean zeros.  Returns 0, or -1 for
 * a bad size.
 */
int evo_ref_ln_linear(int64_t rows, int64_t c_in, int64_t n_out, const double* x, const double* ln_w,
                      const double* ln_b, double eps, const double* w, const double* bias, double* y) {
    if (rows < 0 || c_in <= 0 || n_out <= 0) return -1;
#pragma omp parallel
    {
        double* n = (double*)malloc(sizeof(double) * (size_t)c_in);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            const double* xr = x + r * c_in;
            double mu = 0.0;
            for (int64_t k = 0; k < c_in; ++k) mu += xr[k];
            mu /= (double)c_in;
            double var = 0.0;
            for (int64_t k = 0; k < c_in; ++k) var += (xr[k] - mu) * (xr[k] - mu);
            var /= (double)c_in;
#if EVO_REF_MUTANT == 8
            const double inv = 1.0 / var;          /* mutant: missing square root */
#else
            const double inv = 1.0 / sqrt(var + eps);
#endif
            for (int64_t k = 0; k < c_in; ++k)
                n[k] = (xr[k] - mu) * inv * (ln_w ? ln_w[k] : 1.0) + (ln_b ? ln_b[k] : 0.0);
            double* yr = y + r * n_out;
            for (int64_t o = 0; o < n_out; ++o) yr[o] = bias ? bias[o] : 0.0;
            for (int64_t k = 0; k < c_in; ++k) {
                const double nk = n[k];
                const double* wk = w + k * n_out;
#if EVO_REF_MUTANT == 9
                /* mutant: output columns shifted by one */
                for (int64_t o = 0; o < n_out; ++o) yr[o] += nk * wk[(o + 1) % n_out];
#else
                for (int64_t o = 0; o < n_out; ++o) yr[o] += nk * wk[o];
#endif
            }
        }
        free(n);
    }
    return 0;
}

/*
 * Triangular multiplicative update, the contraction at its core ("Evoformer:
 * the memory wall ZeRO cannot move", section "The three operations"): edge
 * (i, j) is updated from every third residue k, channel by channel,
 *
 *   outgoing edges (i-k and j-k):  z[b,i,j,c] = sum_k a[b,i,k,c] * bb[b,j,k,c]
 *   incoming edges (k-i and k-j):  z[b,i,j,c] = sum_k a[b,k,i,c] * bb[b,k,j,c]
 *
 * a, bb, z: [B, N, N, C] contiguous fp64, the layout of the pair
 * representation.  O(N^3 C) time; the sum over k contracts as it goes.
 * Returns 0, or -1 for a bad size.
 */
int evo_ref_tri_mul(int64_t B, int64_t N, int64_t C, const double* a, const double* bb, int incoming,
                    double* z) {
    if (B < 0 || N < 0 || C <= 0) return -1;
    const int64_t nn = N * N;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t i = 0; i < N; ++i) {
            const double* ab = a + b * nn * C;
            const double* bbb = bb + b * nn * C;
            for (int64_t j = 0; j < N; ++j) {
                double* zr = z + ((b * N + i) * N + j) * C;
                for (int64_t c = 0; c < C; ++c) zr[c] = 0.0;
#if EVO_REF_MUTANT == 10
                /* mutant: no third index -- the elementwise product of the two edges */
                for (int64_t c = 0; c < C; ++c) zr[c] = ab[(i * N + j) * C + c] * bbb[(i * N + j) * C + c];
#else
                for (int64_t k = 0; k < N; ++k) {
                    const double* ar = incoming ? ab + (k * N + i) * C : ab + (i * N + k) * C;
#if EVO_REF_MUTANT == 11
                    /* mutant: second operand read as the edge k-j in outgoing mode */
                    const double* br = incoming ? bbb + (k * N + j) * C : bbb + (k * N + j) * C;
#else
                    const double* br = incoming ? bbb + (k * N + j) * C : bbb + (j * N + k) * C;
#endif
                    for (int64_t c = 0; c < C; ++c) zr[c] += ar[c] * br[c];
                }
#endif
            }
        }
    }
    return 0;
}

/*
 * Outer product mean, the bridge from the MSA to the pair representation
 * ("Evoformer: the memory wall ZeRO cannot move", section "The three
 * operations"): the outer product of MSA columns i and j averaged over the
 * S sequences,
 *
 *   out[b,i,j,c1,c2] = (1/S) sum_s a[b,s,i,c1] * bb[b,s,j,c2]
 *
 * a: [B, S, Na, Ca], bb: [B, S, Nb, Cb], out: [B, Na, Nb, Ca, Cb],
 * contiguous fp64.  Na = Nb = N for the full operation; Na < N evaluates the
 * definition at a subset of columns i (a smaller, equally valid problem).
 * Returns 0, or -1 for a bad size.
 */
int evo_ref_outer_product_mean(int64_t B, int64_t S, int64_t Na, int64_t Nb, int64_t Ca, int64_t Cb,
                               const double* a, const double* bb, double* out) {
    if (B < 0 || S <= 0 || Na < 0 || Nb < 0 || Ca <= 0 || Cb <= 0) return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t i = 0; i < Na; ++i) {
            for (int64_t j = 0; j < Nb; ++j) {
                double* o = out + (((b * Na + i) * Nb + j) * Ca) * Cb;
                for (int64_t e = 0; e < Ca * Cb; ++e) o[e] = 0.0;
                for (int64_t s = 0; s < S; ++s) {
                    const double* ar = a + ((b * S + s) * Na + i) * Ca;
                    const double* br = bb + ((b * S + s) * Nb + j) * Cb;
                    for (int64_t c1 = 0; c1 < Ca; ++c1)
                        for (int64_t c2 = 0; c2 < Cb; ++c2) o[c1 * Cb + c2] += ar[c1] * br[c2];
                }
#if EVO_REF_MUTANT == 12
                /* mutant: the sum over sequences, not its mean */
#else
                for (int64_t e = 0; e < Ca * Cb; ++e) o[e] /= (double)S;
#endif
#if EVO_REF_MUTANT == 13
                /* mutant: the two channel axes swapped (Ca == Cb only) */
                if (Ca == Cb)
                    for (int64_t c1 = 0; c1 < Ca; ++c1)
                        for (int64_t c2 = c1 + 1; c2 < Cb; ++c2) {
                            const double t = o[c1 * Cb + c2];
                            o[c1 * Cb + c2] = o[c2 * Cb + c1];
                            o[c2 * Cb + c1] = t;
                        }
#endif
            }
        }
    }
    return 0;
}

/*
 * Rank-ordered sum of fp32 partials, every addition rounded to fp32:
 *
 *   out[i] = (...((parts[0][i] + parts[1][i]) + parts[2][i]) ...) + parts[count-1][i]
 *
 * When the rows s of one problem are split over GPUs, d_pair_bias -- the sum
 * over s of dS (backward, above) -- is the sum of each GPU's partial over its
 * own rows.  The library adds those partials left to right in fp32, so this
 * function is held to the same precision (not fp64): its result is the
 * exchange's exact expected value, compared bit for bit.
 * parts: [count, n] contiguous fp32; out: [n].  Returns 0, or -1 for a bad size.
 */
int evo_ref_ordered_sum_f32(int64_t count, int64_t n, const float* parts, float* out) {
    if (count < 1 || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
#if EVO_REF_MUTANT == 14
        /* mutant: the partials added in reverse order */
        float acc = parts[(count - 1) * n + i];
        for (int64_t r = count - 2; r >= 0; --r) acc = acc + parts[r * n + i];
#elif EVO_REF_MUTANT == 15
        /* mutant: the last partial left out */
        float acc = parts[i];
        for (int64_t r = 1; r < count - 1; ++r) acc = acc + parts[r * n + i];
#else
        float acc = parts[i];
        for (int64_t r = 1; r < count; ++r) acc = acc + parts[r * n + i];
#endif
        out[i] = acc;
    }
    return 0;
}

/* Which planted mistake this build carries (0 = none). */
int evo_ref_mutant(void) { return EVO_REF_MUTANT; }
