// Offline calibration: per (layer, query head, pair f) complex mean of the
// pre-RoPE queries and mean magnitude ("TriAttention：基于三角函数 KV 压缩的高效长
// 推理", 流程详解 step 1: centres are extracted ahead of time).
//
// One CTA per (layer, query head); 256 threads = 4 groups x 64 pairs.  Thread
// (grp, f) walks queries t = grp, grp+4, ... reading dims f and f+64 (coalesced
// 128-byte half-rows per warp pair), accumulating in fp64 (x^2 + y^2 of two
// bf16 values is exact in fp64).  The four partial sums are combined in a
// fixed order, so results are deterministic.  Runs once, offline; it is not on
// the per-token path.
#include "tri_internal.cuh"

namespace tri {

constexpr int kCalibThreads = 256;

__global__ void __launch_bounds__(kCalibThreads) calib_kernel(const CalibParams p) {
    __shared__ double part[3][4][kF];
    const int head = blockIdx.x;
    const int f = threadIdx.x & (kF - 1);
    const int grp = threadIdx.x >> 6;
    const uint16_t *base = p.q + (int64_t)head * p.nq * kD;
    double sr = 0.0, si = 0.0, sn = 0.0;
    for (int64_t t = grp; t < p.nq; t += 4) {
        const double x = (double)__uint_as_float((uint32_t)base[t * kD + f] << 16);
        const double y = (double)__uint_as_float((uint32_t)base[t * kD + kF + f] << 16);
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
        p.centres[((int64_t)head * kF + f) * 2] = (float)(a / n);
        p.centres[((int64_t)head * kF + f) * 2 + 1] = (float)(b / n);
        p.mean_norm[(int64_t)head * kF + f] = (float)(c / n);
    }
}

cudaError_t launch_calib(const CalibParams &p, cudaStream_t s) {
    if (p.n_heads <= 0) return cudaSuccess;
    calib_kernel<<<p.n_heads, kCalibThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tri
