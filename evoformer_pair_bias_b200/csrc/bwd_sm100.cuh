// bwd_sm100.cuh -- bf16 backward of Evoformer pair-bias attention.
#pragma once

#include "sm100.cuh"
#include "simt.cuh"

namespace evo {
namespace bwd {

// Row groups for the deterministic d_pair_bias reduction: enough CTAs
// (key tiles x heads x batch x groups) for about two per SM of a 148-SM B200.
inline int num_groups(int64_t B, int64_t S, int64_t N, int64_t H) {
    const int64_t njt = (N + 127) / 128;
    const int64_t base = njt * B * H;
    if (base <= 0) return 1;
    int64_t g = (2 * 148 + base - 1) / base;
    if (g > S) g = S;
    if (g < 1) g = 1;
    return (int)g;
}

struct Call {
    evo_shape_t shape;
    const void *q, *k, *v, *g;
    evo_strides_t in;
    const void *mask, *bias, *out, *dout;
    evo_strides_t os;
    const float* lse;
    void *dq, *dk, *dv, *dg;
    evo_strides_t gs;
    float* dbias;
    char* ws;
    size_t d_off, doa_off, dqacc_off, biast_off, part_off;
    int groups;
};

inline evo_status_t run(const Call& c, cudaStream_t stream, int* launched) {
    const evo_shape_t& sh = c.shape;
    simt::Args a{};
    a.B = (int)sh.B; a.S = (int)sh.S; a.N = (int)sh.N; a.H = (int)sh.H; a.C = (int)sh.C;
    if (sh.C > simt::kMaxC || sh.S > 65535 || sh.N > 65535) return EVO_ERR_UNSUPPORTED;
    a.q = c.q; a.k = c.k; a.v = c.v; a.g = c.g; a.in = Strides{c.in.b, c.in.s, c.in.n, c.in.h};
    a.mask = c.mask; a.bias = c.bias; a.out = c.out; a.dout = c.dout;
    a.os = Strides{c.os.b, c.os.s, c.os.n, c.os.h};
    a.lse = const_cast<float*>(c.lse);
    a.dq = c.dq; a.dk = c.dk; a.dv = c.dv; a.dg = c.dg; a.gs = Strides{c.gs.b, c.gs.s, c.gs.n, c.gs.h};
    a.dbias = c.dbias;
    a.D = reinterpret_cast<float*>(c.ws + c.d_off);
    using T = __nv_bfloat16;
    const int64_t rows = (int64_t)a.B * a.S * a.N * a.H;
    simt::bwd_pre_kernel<T><<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(a);
    const dim3 grid((unsigned)((a.N + simt::kRowsPerCta - 1) / simt::kRowsPerCta), (unsigned)a.S,
                    (unsigned)(a.B * a.H));
    simt::bwd_dq_kernel<T><<<grid, simt::kWarps * 32, 0, stream>>>(a);
    simt::bwd_dkdv_kernel<T><<<grid, simt::kWarps * 32, 0, stream>>>(a);
    const dim3 gb((unsigned)((a.N + 127) / 128), (unsigned)a.N, (unsigned)(a.B * a.H));
    simt::bwd_dbias_kernel<T><<<gb, 128, 0, stream>>>(a);
    *launched = 4;
    return cudaGetLastError() == cudaSuccess ? EVO_OK : EVO_ERR_CUDA;
}

}  // namespace bwd
}  // namespace evo
