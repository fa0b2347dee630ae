// Offline calibration: per (layer, query head, pair f) complex mean of the
// pre-RoPE queries and mean magnitude ("TriAttention：基于三角函数 KV 压缩的高效长
// 推理", 流程详解 step 1: centres are extracted ahead of time).
//
// One CTA per (layer, query head); 4F threads = 4 groups x F pairs (F = d/2).
// Thread (grp, f) walks queries t = grp, grp+4, ... reading the two dims of
// pair f - (f, f+F) with rotate-half RoPE, (2f, 2f+1) with interleaved RoPE,
// coalesced across the warp either way - and accumulates in fp64 (x^2 + y^2 of
// two bf16 values is exact in fp64).  The four partial sums are combined in a
// fixed order, so results are deterministic.  Runs once, offline; it is not on
// the per-token path.
#include "tri_internal.cuh"

namespace tri {

template <int F, bool IL>
__global__ void __launch_bounds__(4 * F) calib_kernel(const CalibParams p) {
    constexpr int D = 2 * F;
    __shared__ double part[3][4][F];
    const int head = blockIdx.x;
    const int f = threadIdx.x % F;
    const int grp = threadIdx.x / F;
    const uint16_t *base = p.q + (int64_t)head * p.nq * D;
    const int ia = IL ? 2 * f : f, ib = IL ? 2 * f + 1 : f + F;
    double sr = 0.0, si = 0.0, sn = 0.0;
    for (int64_t t = grp; t < p.nq; t += 4) {
        const double x = (double)__uint_as_float((uint32_t)base[t * D + ia] << 16);
        const double y = (double)__uint_as_float((uint32_t)base[t * D + ib] << 16);
        sr += x;
        si += y;
        sn += sqrt(x * x + y * y);
    }
    part[0][grp][f] = sr;
    part[1][grp][f] = si;
    part[2][grp][f] = sn;
    __syncthreads();
    if (grp == 0) {
        const double n = (double)p.nq;
        double a = 0.0, b = 0.0, c = 0.0;
        for (int k = 0; k < 4; k++) {
            a += part[0][k][f];
            b += part[1][k][f];
            c += part[2][k][f];
        }
        p.centres[((int64_t)head * F + f) * 2] = (float)(a / n);
        p.centres[((int64_t)head * F + f) * 2 + 1] = (float)(b / n);
        p.mean_norm[(int64_t)head * F + f] = (float)(c / n);
    }
}

template <int F>
static cudaError_t launch_calib_f(const CalibParams &p, cudaStream_t s) {
    if (p.il) calib_kernel<F, true><<<p.n_heads, 4 * F, 0, s>>>(p);
    else calib_kernel<F, false><<<p.n_heads, 4 * F, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_calib(const CalibParams &p, cudaStream_t s) {
    if (p.n_heads <= 0) return cudaSuccess;
    switch (p.D) {
        case 64: return launch_calib_f<32>(p, s);
        case 128: return launch_calib_f<64>(p, s);
        case 256: return launch_calib_f<128>(p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tri
