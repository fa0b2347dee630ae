// Per-row score coefficients ("TriAttention：基于三角函数 KV 压缩的高效长推理",
// 流程详解 steps 2-3): for the row of KV head h of sequence s,
//   A_f = (1/G) sum_g qbar_f^g * e^{i w_f p_now} * sum_delta e^{i w_f delta}
//         (without the e^{i w_f p_now} factor for a pre-RoPE cache),
//   c_f = (1/G) sum_g (E|q_f^g| - |qbar_f^g|),
// formed in fp64 and stored fp32 in the workspace ([R][d/16][24]: for lane
// group g, pairs 8g..8g+7 as Re A, Im A, c), plus the table T_f = w_f / 2pi in
// 0.64 fixed point that the score kernel uses for per-key phases.  Every phase
// w_f * n is reduced exactly as (n * T_f) mod 2^64 and evaluated in fp64.
#include "tri_internal.cuh"

namespace tri {

constexpr int kPrepParts = 4;
constexpr double kTurnScale = 2.9358905032820014e+18;    // 2^64 / (2 pi)
constexpr double kTurnToRad64 = 3.4061215800865545e-19;  // 2 pi / 2^64

// sin/cos of the angle 2 pi * t / 2^64 (t a fixed-point fraction of a turn,
// taken as signed so the angle is in [-pi, pi)): always a small argument.
__device__ __forceinline__ void sincos_turns(unsigned long long t, double *sn, double *cs) {
    sincos((double)(long long)t * kTurnToRad64, sn, cs);
}

// One CTA of 4F threads per row (F = d/2 pairs); thread (part, f) sums the
// offsets e = part, part+4, ... of pair f, then the F threads of part 0 finish
// the row's coefficients.  All phases w_f * n are reduced exactly as
// (n * T_f) mod 2^64, T_f = w_f / 2pi in 0.64 fixed point, and evaluated in fp64.
template <int F>
__global__ void __launch_bounds__(kPrepParts * F) prep_kernel(const PrepParams p) {
    __shared__ double part_re[kPrepParts][F], part_im[kPrepParts][F];
    const Geometry &geo = p.geo;
    const int r = blockIdx.x;
    const int f = threadIdx.x % F;
    const int part = threadIdx.x / F;
    const int h = r % geo.H;
    const int s = (r / geo.H) % geo.S;
    const int l = r / (geo.H * geo.S);
    const int64_t qh0 = (int64_t)l * geo.Hq + (int64_t)h * geo.G;
    // The offsets' phasor sums depend on kernel parameters only: form them before
    // waiting for the preceding kernel on the stream.
    const double w = pow(p.theta, -2.0 * (double)f / (double)(2 * F));
    const unsigned long long T = __double2ull_rn(w * kTurnScale);
    double sr = 0.0, si = 0.0;
    for (int e = part; e < p.n_off; e += kPrepParts) {
        double sn, cs;
        sincos_turns((unsigned long long)(long long)p.offsets[e] * T, &sn, &cs);
        sr += cs;
        si += sn;
    }
    grid_dependency_wait();
    grid_dependents_launch();
    float2 qv[8];
    float mv[8];
    long long pnow = 0;
    if (part == 0) {
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if (j < geo.G) {
                qv[j] = reinterpret_cast<const float2 *>(p.centres)[(qh0 + j) * F + f];
                mv[j] = p.mean_norm[(qh0 + j) * F + f];
            }
        }
        pnow = p.p_now[s];
    }
    part_re[part][f] = sr;
    part_im[part][f] = si;
    __syncthreads();
    if (part != 0) return;
    sr = 0.0;
    si = 0.0;
#pragma unroll
    for (int k = 0; k < kPrepParts; k++) {
        sr += part_re[k][f];
        si += part_im[k][f];
    }
    double mr = 0.0, mi = 0.0, cf = 0.0;
    for (int g0 = 0; g0 < geo.G; g0 += 8) {
        if (g0 > 0) {
#pragma unroll
            for (int j = 0; j < 8; j++) {
                if (g0 + j < geo.G) {
                    qv[j] = reinterpret_cast<const float2 *>(p.centres)[(qh0 + g0 + j) * F + f];
                    mv[j] = p.mean_norm[(qh0 + g0 + j) * F + f];
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if (g0 + j < geo.G) {
                const double qr = qv[j].x, qi = qv[j].y;
                mr += qr;
                mi += qi;
                cf += (double)mv[j] - hypot(qr, qi);
            }
        }
    }
    mr /= (double)geo.G;
    mi /= (double)geo.G;
    cf /= (double)geo.G;
    const double tr = mr * sr - mi * si, ti = mr * si + mi * sr;
    double ar = tr, ai = ti;
    if (!p.pre_rope) {
        double sn, cs;
        sincos_turns((unsigned long long)pnow * T, &sn, &cs);
        ar = tr * cs - ti * sn;
        ai = tr * sn + ti * cs;
    }
    float *c = p.coef + (int64_t)r * (3 * F) + (f >> 3) * kCoefPerGroup;
    c[f & 7] = (float)ar;
    c[8 + (f & 7)] = (float)ai;
    c[16 + (f & 7)] = (float)cf;
    if (r == 0) {
        p.turns[f] = T;
        if (f == 0) {
            const int64_t R = (int64_t)geo.L * geo.S * geo.H;
            if (geo.row_off[0] != 0 || geo.row_off[R] != geo.total) atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
        }
    }
}

cudaError_t launch_prep(const PrepParams &p, cudaStream_t s) {
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    switch (p.geo.D) {
        case 64: return launch_pdl(prep_kernel<32>, dim3((unsigned)R), dim3(kPrepParts * 32), 0, s, p);
        case 128: return launch_pdl(prep_kernel<64>, dim3((unsigned)R), dim3(kPrepParts * 64), 0, s, p);
        case 256: return launch_pdl(prep_kernel<128>, dim3((unsigned)R), dim3(kPrepParts * 128), 0, s, p);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tri
