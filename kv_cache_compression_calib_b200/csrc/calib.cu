// Offline calibration: per (layer, query head, pair f) complex mean of the
// pre-RoPE queries and mean magnitude ("TriAttention：基于三角函数 KV 压缩的高效长
// 推理", 流程详解 step 1: centres are extracted ahead of time).
//
// One CTA per (layer, query head); 4F threads = 4 groups x F pairs (F = d/2).
// Thread (grp, f) walks queries t = grp, grp+4, ... reading the two dims of
// pair f - (f, f+F) with rotate-half RoPE, (2f, 2f+1) with interleaved RoPE,
// coalesced across the warp either way - and accumulates in fp64 (x^2 + y^2 of
// two bf16 values is exact in fp64).  The loads of 8 consecutive queries of a
// thread are issued before their sums (the sums still run in query order), so
// each thread keeps 16 loads in flight.  The four partial sums are combined in
// a fixed order, so results are deterministic.  Runs once, offline; it is not
// on the per-token path.
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
    constexpr int kBatch = 8;  // queries per thread whose loads are in flight together
    int64_t t = grp;
    for (; t + 4 * (kBatch - 1) < p.nq; t += 4 * kBatch) {
        uint16_t xa[kBatch], ya[kBatch];
#pragma unroll
        for (int k = 0; k < kBatch; k++) {
            xa[k] = __ldg(base + (t + 4 * k) * D + ia);
            ya[k] = __ldg(base + (t + 4 * k) * D + ib);
        }
#pragma unroll
        for (int k = 0; k < kBatch; k++) {
            const double x = (double)__uint_as_float((uint32_t)xa[k] << 16);
            const double y = (double)__uint_as_float((uint32_t)ya[k] << 16);
            sr += x;
            si += y;
            sn += sqrt(x * x + y * y);
        }
    }
    for (; t < p.nq; t += 4) {
        const double x = (double)__uint_as_float((uint32_t)__ldg(base + t * D + ia) << 16);
        const double y = (double)__uint_as_float((uint32_t)__ldg(base + t * D + ib) << 16);
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

// Online update of the same statistics: every call multiplies the running sums
// and the running query weight of each head by `decay`, then adds this call's
// queries, and writes the centres of the updated state.  Same thread layout and
// fixed summation order as calib_kernel, so a stream of updates is
// deterministic.
template <int F, bool IL>
__global__ void __launch_bounds__(4 * F) calib_update_kernel(const CalibUpdateParams u) {
    constexpr int D = 2 * F;
    const CalibParams &p = u.c;
    __shared__ double part[3][4][F];
    const int head = blockIdx.x;
    const int f = threadIdx.x % F;
    const int grp = threadIdx.x / F;
    const double w_old = u.weight[head];  // read by every thread before thread 0 rewrites it
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
    if (grp != 0) return;
    double a = 0.0, b = 0.0, c = 0.0;
    for (int k = 0; k < 4; k++) {
        a += part[0][k][f];
        b += part[1][k][f];
        c += part[2][k][f];
    }
    double *st = u.sums + ((int64_t)head * F + f) * 3;
    a += u.decay * st[0];
    b += u.decay * st[1];
    c += u.decay * st[2];
    st[0] = a;
    st[1] = b;
    st[2] = c;
    const double w = u.decay * w_old + (double)p.nq;
    if (f == 0) u.weight[head] = w;
    p.centres[((int64_t)head * F + f) * 2] = (float)(a / w);
    p.centres[((int64_t)head * F + f) * 2 + 1] = (float)(b / w);
    p.mean_norm[(int64_t)head * F + f] = (float)(c / w);
}

template <int F>
static cudaError_t launch_update_f(const CalibUpdateParams &p, cudaStream_t s) {
    if (p.c.il) calib_update_kernel<F, true><<<p.c.n_heads, 4 * F, 0, s>>>(p);
    else calib_update_kernel<F, false><<<p.c.n_heads, 4 * F, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_calib_update(const CalibUpdateParams &p, cudaStream_t s) {
    if (p.c.n_heads <= 0) return cudaSuccess;
    switch (p.c.D) {
        case 64: return launch_update_f<32>(p, s);
        case 128: return launch_update_f<64>(p, s);
        case 256: return launch_update_f<128>(p, s);
    }
    return cudaErrorInvalidValue;
}

// Concentration and drift of each head's statistics, one warp per head (fp64,
// fixed reduction order):
//   concentration[f] = |centre_f| / mean_norm_f (0 where mean_norm_f = 0),
//   head_stats[0]    = sum_f |centre_f| / sum_f mean_norm_f,
//   head_stats[1]    = sum_f (|centre_f - ref_f| + |mean_norm_f - ref_norm_f|) / sum_f ref_norm_f
//                      (0 without a reference).
constexpr int kStatsThreads = 256;

__global__ void __launch_bounds__(kStatsThreads) stats_kernel(const StatsParams p) {
    const int64_t head = (int64_t)blockIdx.x * (kStatsThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (head >= p.n_heads) return;
    const float2 *c = reinterpret_cast<const float2 *>(p.centres) + head * p.F;
    const float *m = p.mean_norm + head * p.F;
    const float2 *rc = p.ref_centres ? reinterpret_cast<const float2 *>(p.ref_centres) + head * p.F : nullptr;
    const float *rm = p.ref_mean_norm ? p.ref_mean_norm + head * p.F : nullptr;
    double sc = 0.0, sm = 0.0, dd = 0.0, sr = 0.0;
    for (int f = lane; f < p.F; f += 32) {
        const float2 cf = c[f];
        const double a = hypot((double)cf.x, (double)cf.y);
        const double mf = m[f];
        if (p.concentration) p.concentration[head * p.F + f] = mf > 0.0 ? (float)(a / mf) : 0.f;
        sc += a;
        sm += mf;
        if (rc) {
            const float2 r = rc[f];
            dd += hypot((double)cf.x - (double)r.x, (double)cf.y - (double)r.y) + fabs(mf - (double)rm[f]);
            sr += rm[f];
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        sc += __shfl_xor_sync(0xffffffffu, sc, o);
        sm += __shfl_xor_sync(0xffffffffu, sm, o);
        dd += __shfl_xor_sync(0xffffffffu, dd, o);
        sr += __shfl_xor_sync(0xffffffffu, sr, o);
    }
    if (lane == 0 && p.head_stats) {
        p.head_stats[head * 2] = sm > 0.0 ? (float)(sc / sm) : 0.f;
        p.head_stats[head * 2 + 1] = (rc && sr > 0.0) ? (float)(dd / sr) : 0.f;
    }
}

cudaError_t launch_stats(const StatsParams &p, cudaStream_t s) {
    if (p.n_heads <= 0) return cudaSuccess;
    const int64_t grid = (p.n_heads + (kStatsThreads / 32) - 1) / (kStatsThreads / 32);
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    stats_kernel<<<(unsigned)grid, kStatsThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tri
