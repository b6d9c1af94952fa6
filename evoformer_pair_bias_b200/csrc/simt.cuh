// simt.cuh -- fp32 path of Evoformer pair-bias attention on the FMA pipe.
//
// The fp32 contract (relative L2 error 1e-4) rules out TF32 tensor cores, so
// this path multiplies in plain fp32.  It follows the same flash-style plan as
// the tensor-core path -- logits live only in registers, the softmax is online
// with warp-shuffle row reductions, nothing of size N^2 per row is stored --
// but uses one warp per logit row (lanes across keys), which suits the small
// head dims (C <= 64) and sizes it serves.
//
// Backward is split so that every output element has exactly one writer
// (deterministic, no atomics):
//   bwd_pre   D_i = sum_c dout*out, dg = dout*out*(1-sigmoid(g))
//   bwd_dq    one warp per query row, loops over keys
//   bwd_dkdv  one warp per key row, loops over queries
//   bwd_dbias one thread per (b, h, i, j), loops over rows s in order
// Each recomputes P = exp(x - lse) from the saved lse.
#pragma once

#include <math.h>

#include "common.cuh"

namespace evo {
namespace simt {

constexpr int kWarps = 4;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;  // 16 logit rows per CTA
constexpr int kChunk = 32;                          // keys (or queries) staged per step
constexpr int kMaxC = 64;

struct Args {
    int B, S, N, H, C;
    const void *q, *k, *v, *g;
    Strides in;
    const void* mask;  // [B,S,N] or null
    const void* bias;  // [B,H,N,N] or null
    const void* out;
    const void* dout;
    Strides os;
    float* lse;        // [B,S,H,N]
    void *dq, *dk, *dv, *dg;
    Strides gs;
    float* dbias;      // [B,H,N,N]
    float* D;          // workspace [B,S,H,N]
    void* out_w;       // forward output (writable)
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ int64_t row_index(const Args& a, int b, int s, int h, int i) {
    return ((int64_t)(b * a.S + s) * a.H + h) * a.N + i;  // [B,S,H,N]
}

template <typename T>
__device__ __forceinline__ float mask_at(const Args& a, int b, int s, int j) {
    return a.mask ? Elem<T>::load((const T*)a.mask + (int64_t)(b * a.S + s) * a.N + j) : 0.f;
}
template <typename T>
__device__ __forceinline__ float bias_at(const Args& a, int b, int h, int i, int j) {
    return a.bias ? Elem<T>::load((const T*)a.bias + ((int64_t)(b * a.H + h) * a.N + i) * a.N + j) : 0.f;
}

// ---------------------------------------------------------------- forward
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) fwd_kernel(Args a) {
    __shared__ float ks[kChunk][kMaxC + 1];
    __shared__ float vs[kChunk][kMaxC + 1];
    __shared__ float qs[kRowsPerCta][kMaxC];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * kRowsPerCta, s = blockIdx.y;
    const int b = blockIdx.z / a.H, h = blockIdx.z % a.H;
    const int C = a.C, N = a.N;
    const T* q = (const T*)a.q;
    const T* k = (const T*)a.k;
    const T* v = (const T*)a.v;
    const float scale = 1.0f / sqrtf((float)C);

    for (int t = threadIdx.x; t < kRowsPerCta * C; t += blockDim.x) {
        const int r = t / C, c = t % C, i = i0 + r;
        qs[r][c] = (i < N) ? Elem<T>::load(q + a.in.off(b, s, i, h) + c) : 0.f;
    }
    float m[kRowsPerWarp], l[kRowsPerWarp], acc0[kRowsPerWarp], acc1[kRowsPerWarp];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        m[rr] = -INFINITY; l[rr] = 0.f; acc0[rr] = 0.f; acc1[rr] = 0.f;
    }
    for (int j0 = 0; j0 < N; j0 += kChunk) {
        __syncthreads();
        for (int t = threadIdx.x; t < kChunk * C; t += blockDim.x) {
            const int jj = t / C, c = t % C, j = j0 + jj;
            float kv = 0.f, vv = 0.f;
            if (j < N) {
                kv = Elem<T>::load(k + a.in.off(b, s, j, h) + c);
                vv = Elem<T>::load(v + a.in.off(b, s, j, h) + c);
            }
            ks[jj][c] = kv;
            vs[jj][c] = vv;
        }
        __syncthreads();
        const int j = j0 + lane;
        const float mj = (j < N) ? mask_at<T>(a, b, s, j) : 0.f;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const int r = warp * kRowsPerWarp + rr, i = i0 + r;
            float dot = 0.f;
            for (int c = 0; c < C; ++c) dot += qs[r][c] * ks[lane][c];
            float x = dot * scale + mj;
            if (i < N && j < N) x += bias_at<T>(a, b, h, i, j);
            if (j >= N) x = -INFINITY;
            const float mnew = fmaxf(m[rr], warp_max(x));
            const float p = expf(x - mnew);
            const float alpha = expf(m[rr] - mnew);
            l[rr] = l[rr] * alpha + warp_sum(p);
            float a0 = acc0[rr] * alpha, a1 = acc1[rr] * alpha;
            for (int jj = 0; jj < kChunk; ++jj) {
                const float pj = __shfl_sync(0xffffffffu, p, jj);
                if (lane < C) a0 += pj * vs[jj][lane];
                if (lane + 32 < C) a1 += pj * vs[jj][lane + 32];
            }
            acc0[rr] = a0; acc1[rr] = a1; m[rr] = mnew;
        }
    }
    T* out = (T*)a.out_w;
    const T* g = (const T*)a.g;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int i = i0 + warp * kRowsPerWarp + rr;
        if (i >= N) continue;
        const float inv = 1.0f / l[rr];
        if (lane < C) {
            const float gg = Elem<T>::load(g + a.in.off(b, s, i, h) + lane);
            Elem<T>::store(out + a.os.off(b, s, i, h) + lane, acc0[rr] * inv / (1.0f + expf(-gg)));
        }
        if (lane + 32 < C) {
            const float gg = Elem<T>::load(g + a.in.off(b, s, i, h) + lane + 32);
            Elem<T>::store(out + a.os.off(b, s, i, h) + lane + 32, acc1[rr] * inv / (1.0f + expf(-gg)));
        }
        if (lane == 0) a.lse[row_index(a, b, s, h, i)] = m[rr] + logf(l[rr]);
    }
}

// ---------------------------------------------------------------- backward
// D_i = sum_c dout * out (= sum_c dA * A since out = sigmoid(g) * A),
// dg = dout * out * (1 - sigmoid(g)).  One thread per (b, s, i, h) row.
template <typename T>
__global__ void __launch_bounds__(256) bwd_pre_kernel(Args a) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t rows = (int64_t)a.B * a.S * a.N * a.H;
    if (t >= rows) return;
    const int h = (int)(t % a.H);
    const int i = (int)((t / a.H) % a.N);
    const int s = (int)((t / ((int64_t)a.H * a.N)) % a.S);
    const int b = (int)(t / ((int64_t)a.H * a.N * a.S));
    const T* o = (const T*)a.out + a.os.off(b, s, i, h);
    const T* d = (const T*)a.dout + a.os.off(b, s, i, h);
    const T* g = (const T*)a.g + a.in.off(b, s, i, h);
    T* dg = (T*)a.dg + a.gs.off(b, s, i, h);
    float D = 0.f;
    for (int c = 0; c < a.C; ++c) {
        const float oc = Elem<T>::load(o + c), dc = Elem<T>::load(d + c);
        const float sg = 1.0f / (1.0f + expf(-Elem<T>::load(g + c)));
        D += dc * oc;
        Elem<T>::store(dg + c, dc * oc * (1.0f - sg));
    }
    a.D[row_index(a, b, s, h, i)] = D;
}

// dq: one warp per query row; dq_i = sum_j P_ij (dP_ij - D_i) k_j / sqrt(C).
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) bwd_dq_kernel(Args a) {
    __shared__ float ks[kChunk][kMaxC + 1];
    __shared__ float vs[kChunk][kMaxC + 1];
    __shared__ float qs[kRowsPerCta][kMaxC];
    __shared__ float das[kRowsPerCta][kMaxC];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i0 = blockIdx.x * kRowsPerCta, s = blockIdx.y;
    const int b = blockIdx.z / a.H, h = blockIdx.z % a.H;
    const int C = a.C, N = a.N;
    const float scale = 1.0f / sqrtf((float)C);
    for (int t = threadIdx.x; t < kRowsPerCta * C; t += blockDim.x) {
        const int r = t / C, c = t % C, i = i0 + r;
        float qv = 0.f, dav = 0.f;
        if (i < N) {
            qv = Elem<T>::load((const T*)a.q + a.in.off(b, s, i, h) + c);
            const float gg = Elem<T>::load((const T*)a.g + a.in.off(b, s, i, h) + c);
            dav = Elem<T>::load((const T*)a.dout + a.os.off(b, s, i, h) + c) / (1.0f + expf(-gg));
        }
        qs[r][c] = qv;
        das[r][c] = dav;
    }
    float lse[kRowsPerWarp], Dr[kRowsPerWarp], acc0[kRowsPerWarp], acc1[kRowsPerWarp];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int i = i0 + warp * kRowsPerWarp + rr;
        lse[rr] = (i < N) ? a.lse[row_index(a, b, s, h, i)] : 0.f;
        Dr[rr] = (i < N) ? a.D[row_index(a, b, s, h, i)] : 0.f;
        acc0[rr] = 0.f; acc1[rr] = 0.f;
    }
    for (int j0 = 0; j0 < N; j0 += kChunk) {
        __syncthreads();
        for (int t = threadIdx.x; t < kChunk * C; t += blockDim.x) {
            const int jj = t / C, c = t % C, j = j0 + jj;
            float kv = 0.f, vv = 0.f;
            if (j < N) {
                kv = Elem<T>::load((const T*)a.k + a.in.off(b, s, j, h) + c);
                vv = Elem<T>::load((const T*)a.v + a.in.off(b, s, j, h) + c);
            }
            ks[jj][c] = kv;
            vs[jj][c] = vv;
        }
        __syncthreads();
        const int j = j0 + lane;
        const float mj = (j < N) ? mask_at<T>(a, b, s, j) : 0.f;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const int r = warp * kRowsPerWarp + rr, i = i0 + r;
            float dot = 0.f, dp = 0.f;
            for (int c = 0; c < C; ++c) {
                dot += qs[r][c] * ks[lane][c];
                dp += das[r][c] * vs[lane][c];
            }
            float x = dot * scale + mj;
            if (i < N && j < N) x += bias_at<T>(a, b, h, i, j);
            const float p = (j < N && i < N) ? expf(x - lse[rr]) : 0.f;
            const float ds = p * (dp - Dr[rr]);
            float a0 = acc0[rr], a1 = acc1[rr];
            for (int jj = 0; jj < kChunk; ++jj) {
                const float dj = __shfl_sync(0xffffffffu, ds, jj);
                if (lane < C) a0 += dj * ks[jj][lane];
                if (lane + 32 < C) a1 += dj * ks[jj][lane + 32];
            }
            acc0[rr] = a0; acc1[rr] = a1;
        }
    }
    T* dq = (T*)a.dq;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int i = i0 + warp * kRowsPerWarp + rr;
        if (i >= N) continue;
        if (lane < C) Elem<T>::store(dq + a.gs.off(b, s, i, h) + lane, acc0[rr] * scale);
        if (lane + 32 < C) Elem<T>::store(dq + a.gs.off(b, s, i, h) + lane + 32, acc1[rr] * scale);
    }
}

// dk, dv: one warp per key row; dv_j = sum_i P_ij dA_i, dk_j = sum_i dS_ij q_i / sqrt(C).
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) bwd_dkdv_kernel(Args a) {
    __shared__ float qs[kChunk][kMaxC + 1];
    __shared__ float das[kChunk][kMaxC + 1];
    __shared__ float lses[kChunk], Ds[kChunk];
    __shared__ float kr[kRowsPerCta][kMaxC];
    __shared__ float vr[kRowsPerCta][kMaxC];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = blockIdx.x * kRowsPerCta, s = blockIdx.y;
    const int b = blockIdx.z / a.H, h = blockIdx.z % a.H;
    const int C = a.C, N = a.N;
    const float scale = 1.0f / sqrtf((float)C);
    for (int t = threadIdx.x; t < kRowsPerCta * C; t += blockDim.x) {
        const int r = t / C, c = t % C, j = j0 + r;
        float kv = 0.f, vv = 0.f;
        if (j < N) {
            kv = Elem<T>::load((const T*)a.k + a.in.off(b, s, j, h) + c);
            vv = Elem<T>::load((const T*)a.v + a.in.off(b, s, j, h) + c);
        }
        kr[r][c] = kv;
        vr[r][c] = vv;
    }
    float mjr[kRowsPerWarp], dk0[kRowsPerWarp], dk1[kRowsPerWarp], dv0[kRowsPerWarp], dv1[kRowsPerWarp];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int j = j0 + warp * kRowsPerWarp + rr;
        mjr[rr] = (j < N) ? mask_at<T>(a, b, s, j) : 0.f;
        dk0[rr] = dk1[rr] = dv0[rr] = dv1[rr] = 0.f;
    }
    for (int ib = 0; ib < N; ib += kChunk) {
        __syncthreads();
        for (int t = threadIdx.x; t < kChunk * C; t += blockDim.x) {
            const int ii = t / C, c = t % C, i = ib + ii;
            float qv = 0.f, dav = 0.f;
            if (i < N) {
                qv = Elem<T>::load((const T*)a.q + a.in.off(b, s, i, h) + c);
                const float gg = Elem<T>::load((const T*)a.g + a.in.off(b, s, i, h) + c);
                dav = Elem<T>::load((const T*)a.dout + a.os.off(b, s, i, h) + c) / (1.0f + expf(-gg));
            }
            qs[ii][c] = qv;
            das[ii][c] = dav;
        }
        if (threadIdx.x < kChunk) {
            const int i = ib + threadIdx.x;
            lses[threadIdx.x] = (i < N) ? a.lse[row_index(a, b, s, h, i)] : 0.f;
            Ds[threadIdx.x] = (i < N) ? a.D[row_index(a, b, s, h, i)] : 0.f;
        }
        __syncthreads();
        const int i = ib + lane;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const int r = warp * kRowsPerWarp + rr, j = j0 + r;
            float dot = 0.f, dp = 0.f;
            for (int c = 0; c < C; ++c) {
                dot += qs[lane][c] * kr[r][c];
                dp += das[lane][c] * vr[r][c];
            }
            float x = dot * scale + mjr[rr];
            if (i < N && j < N) x += bias_at<T>(a, b, h, i, j);
            const float p = (i < N && j < N) ? expf(x - lses[lane]) : 0.f;
            const float ds = p * (dp - Ds[lane]);
            float k0 = dk0[rr], k1 = dk1[rr], v0 = dv0[rr], v1 = dv1[rr];
            for (int ii = 0; ii < kChunk; ++ii) {
                const float pi = __shfl_sync(0xffffffffu, p, ii);
                const float di = __shfl_sync(0xffffffffu, ds, ii);
                if (lane < C) { v0 += pi * das[ii][lane]; k0 += di * qs[ii][lane]; }
                if (lane + 32 < C) { v1 += pi * das[ii][lane + 32]; k1 += di * qs[ii][lane + 32]; }
            }
            dk0[rr] = k0; dk1[rr] = k1; dv0[rr] = v0; dv1[rr] = v1;
        }
    }
    T* dk = (T*)a.dk;
    T* dv = (T*)a.dv;
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int j = j0 + warp * kRowsPerWarp + rr;
        if (j >= N) continue;
        if (lane < C) {
            Elem<T>::store(dk + a.gs.off(b, s, j, h) + lane, dk0[rr] * scale);
            Elem<T>::store(dv + a.gs.off(b, s, j, h) + lane, dv0[rr]);
        }
        if (lane + 32 < C) {
            Elem<T>::store(dk + a.gs.off(b, s, j, h) + lane + 32, dk1[rr] * scale);
            Elem<T>::store(dv + a.gs.off(b, s, j, h) + lane + 32, dv1[rr]);
        }
    }
}

// d_pair_bias[b,h,i,j] = sum_s dS: one thread per key j, one CTA per (b,h,i) and
// key block; rows s are visited in order, so the sum is deterministic.
template <typename T>
__global__ void __launch_bounds__(128) bwd_dbias_kernel(Args a) {
    __shared__ float qi[kMaxC], dai[kMaxC];
    __shared__ float lse_i, D_i;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    const int i = blockIdx.y;
    const int b = blockIdx.z / a.H, h = blockIdx.z % a.H;
    const int C = a.C, N = a.N;
    const float scale = 1.0f / sqrtf((float)C);
    const float bij = (j < N) ? bias_at<T>(a, b, h, i, j) : 0.f;
    float acc = 0.f;
    for (int s = 0; s < a.S; ++s) {
        __syncthreads();
        for (int c = threadIdx.x; c < C; c += blockDim.x) {
            qi[c] = Elem<T>::load((const T*)a.q + a.in.off(b, s, i, h) + c);
            const float gg = Elem<T>::load((const T*)a.g + a.in.off(b, s, i, h) + c);
            dai[c] = Elem<T>::load((const T*)a.dout + a.os.off(b, s, i, h) + c) / (1.0f + expf(-gg));
        }
        if (threadIdx.x == 0) {
            lse_i = a.lse[row_index(a, b, s, h, i)];
            D_i = a.D[row_index(a, b, s, h, i)];
        }
        __syncthreads();
        if (j < N) {
            const T* kj = (const T*)a.k + a.in.off(b, s, j, h);
            const T* vj = (const T*)a.v + a.in.off(b, s, j, h);
            float dot = 0.f, dp = 0.f;
            for (int c = 0; c < C; ++c) {
                dot += qi[c] * Elem<T>::load(kj + c);
                dp += dai[c] * Elem<T>::load(vj + c);
            }
            const float x = dot * scale + mask_at<T>(a, b, s, j) + bij;
            const float p = expf(x - lse_i);
            acc += p * (dp - D_i);
        }
    }
    if (j < N) a.dbias[((int64_t)(b * a.H + h) * N + i) * N + j] = acc;
}

}  // namespace simt
}  // namespace evo
