// partials.cuh -- fixed-order sum of fp32 partials (evo_sum_partials).
//
// When the rows s of one attention problem are split over several GPUs, each
// GPU's backward returns the part of d_pair_bias that its rows contribute;
// the full gradient is their sum.  The partials are added left to right in
// the order given (rank order), so the result does not depend on which GPU
// computes it.  HBM-bound: (count + 1) * 4 bytes per element.
#pragma once

#include <cstdint>

namespace evo {
namespace partials {

constexpr int MAX_PARTS = 64;

struct Params {
    const float* part[MAX_PARTS];
    float* out;
    int64_t n;
    int count;
    int vec;   // every pointer 16-byte aligned: float4 groups first, scalar tail
};

// One thread per float4 group (or per element of the tail).  Each output
// element is read from every partial and written by the same thread, after
// its reads, so out may be one of the partials.
__global__ void __launch_bounds__(256) sum_kernel(const Params p) {
    const int64_t n4 = p.vec ? p.n / 4 : 0;
    const int64_t items = n4 + (p.n - 4 * n4);
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < items;
         t += (int64_t)gridDim.x * blockDim.x) {
        if (t < n4) {
            float4 acc = reinterpret_cast<const float4*>(p.part[0])[t];
#pragma unroll 4
            for (int r = 1; r < p.count; ++r) {
                const float4 v = reinterpret_cast<const float4*>(p.part[r])[t];
                acc.x = __fadd_rn(acc.x, v.x);
                acc.y = __fadd_rn(acc.y, v.y);
                acc.z = __fadd_rn(acc.z, v.z);
                acc.w = __fadd_rn(acc.w, v.w);
            }
            reinterpret_cast<float4*>(p.out)[t] = acc;
        } else {
            const int64_t i = 4 * n4 + (t - n4);
            float acc = p.part[0][i];
#pragma unroll 4
            for (int r = 1; r < p.count; ++r) acc = __fadd_rn(acc, p.part[r][i]);
            p.out[i] = acc;
        }
    }
}

}  // namespace partials
}  // namespace evo
