// Per-row score coefficients ("TriAttention：基于三角函数 KV 压缩的高效长推理",
// 流程详解 steps 2-3), in the steps both the prep kernel and the fused
// score-and-select kernel run, so the two produce the same bits:
//   A_f = (1/G) sum_g qbar_f^g * e^{i w_f p_now} * sum_delta e^{i w_f delta}
//         (without the e^{i w_f p_now} factor for a pre-RoPE cache),
//   c_f = (1/G) sum_g (E|q_f^g| - |qbar_f^g|),
// formed in fp64 and stored fp32 ([d/16][24] per row: for lane group g, pairs
// 8g..8g+7 as Re A, Im A, c), plus T_f = w_f / 2pi in 0.64 fixed point.  Every
// phase w_f * n is reduced exactly as (n * T_f) mod 2^64 and evaluated in fp64.
// kPrepParts * F threads take part: thread (part, f) sums the offsets e = part,
// part + kPrepParts, ... of pair f; then the F threads of part 0 finish.
#pragma once

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

// Step 1 (kernel parameters only, so it may run before the kernel waits for its
// predecessor): T_f and this thread's partial sum of the offsets' phasors.
template <int F>
__device__ __forceinline__ void coef_offsets(const PrepParams &p, int f, int part, unsigned long long &T, double &sr,
                                             double &si) {
    const double w = pow(p.theta, -2.0 * (double)f / (double)(2 * F));
    T = __double2ull_rn(w * kTurnScale);
    sr = 0.0;
    si = 0.0;
    for (int e = part; e < p.n_off; e += kPrepParts) {
        double sn, cs;
        sincos_turns((unsigned long long)(long long)p.offsets[e] * T, &sn, &cs);
        sr += cs;
        si += sn;
    }
}

// Step 2, by the F threads of part 0 after every part's sums are in
// part_re/part_im ([kPrepParts][F]): the row's coefficients of pair f into
// coef_row (the row's [d/16][24] block).
template <int F>
__device__ __forceinline__ void coef_finish(const PrepParams &p, int r, int f, unsigned long long T,
                                            const double (*part_re)[F], const double (*part_im)[F], float *coef_row) {
    const Geometry &geo = p.geo;
    const int h = r % geo.H;
    const int s = (r / geo.H) % geo.S;
    const int l = r / (geo.H * geo.S);
    const int64_t qh0 = (int64_t)l * geo.Hq + (int64_t)h * geo.G;
    double sr = 0.0, si = 0.0;
#pragma unroll
    for (int k = 0; k < kPrepParts; k++) {
        sr += part_re[k][f];
        si += part_im[k][f];
    }
    double mr = 0.0, mi = 0.0, cf = 0.0;
    for (int g0 = 0; g0 < geo.G; g0 += 8) {
        float2 qv[8];
        float mv[8];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if (g0 + j < geo.G) {
                qv[j] = reinterpret_cast<const float2 *>(p.centres)[(qh0 + g0 + j) * F + f];
                mv[j] = p.mean_norm[(qh0 + g0 + j) * F + f];
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
        sincos_turns((unsigned long long)p.p_now[s] * T, &sn, &cs);
        ar = tr * cs - ti * sn;
        ai = tr * sn + ti * cs;
    }
    float *c = coef_row + (f >> 3) * kCoefPerGroup;
    c[f & 7] = (float)ar;
    c[8 + (f & 7)] = (float)ai;
    c[16 + (f & 7)] = (float)cf;
}

}  // namespace tri
