// Per-row score coefficients ("TriAttention：基于三角函数 KV 压缩的高效长推理",
// 流程详解 steps 2-3): for the row of KV head h of sequence s,
//   A_f = (1/G) sum_g qbar_f^g * e^{i w_f p_now} * sum_delta e^{i w_f delta}
//         (without the e^{i w_f p_now} factor for a pre-RoPE cache),
//   c_f = (1/G) sum_g (E|q_f^g| - |qbar_f^g|),
// formed in fp64 and stored fp32 in the workspace ([R][d/16][24]: for lane
// group g, pairs 8g..8g+7 as Re A, Im A, c), plus the table T_f = w_f / 2pi in
// 0.64 fixed point that the score kernel uses for per-key phases.  The steps
// live in coef.cuh (the fused kernel runs them too).
#include "coef.cuh"

namespace tri {

// One CTA of kPrepParts * F threads per row (F = d/2 pairs), the steps of
// coef.cuh; row 0 also stores the T_f table and checks the row offsets' ends.
template <int F>
__global__ void __launch_bounds__(kPrepParts * F) prep_kernel(const PrepParams p) {
    __shared__ double part_re[kPrepParts][F], part_im[kPrepParts][F];
    const Geometry &geo = p.geo;
    const int r = blockIdx.x;
    const int f = threadIdx.x % F;
    const int part = threadIdx.x / F;
    unsigned long long T;
    double sr, si;
    coef_offsets<F>(p, f, part, T, sr, si);
    grid_dependency_wait();
    grid_dependents_launch();
    part_re[part][f] = sr;
    part_im[part][f] = si;
    __syncthreads();
    if (part != 0) return;
    coef_finish<F>(p, r, f, T, part_re, part_im, p.coef + (int64_t)r * (3 * F));
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
