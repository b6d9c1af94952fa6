// common.cuh -- small device helpers shared by the kernels of libevo_attn.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "evo_attn.h"

#define EVO_LOG2E 1.4426950408889634f
#define EVO_LN2 0.6931471805599453f

// Device status word: 0 = fine.  A kernel that gives up on a bounded wait
// stores a non-zero code describing where (first writer wins) and returns.
// Read and cleared by evo_attn_device_status().  The library is built as one
// translation unit, so this definition is the only one.
static __device__ unsigned int g_evo_status = 0u;

// Longest a kernel thread spins on one barrier before it declares a timeout.
#ifndef EVO_WAIT_LIMIT_NS
#define EVO_WAIT_LIMIT_NS 2000000000ull
#endif

namespace evo {

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void report_timeout(unsigned int code) {
    atomicCAS(&g_evo_status, 0u, code);
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + __expf(-z)); }

struct Strides {  // element strides of a logical [B,S,N,H,C] tensor
    int64_t b, s, n, h;
    __host__ __device__ __forceinline__ int64_t off(int64_t bb, int64_t ss, int64_t nn, int64_t hh) const {
        return bb * b + ss * s + nn * n + hh * h;
    }
};

}  // namespace evo
