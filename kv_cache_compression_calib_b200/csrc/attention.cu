// Decode attention over the compressed cache ("TriAttention：基于三角函数 KV 压缩的
// 高效长推理", 流程详解 step 5: every later attention step reads only the
// compressed cache, with the model's weights unchanged).  For each (layer l,
// sequence s, query head g of KV head h), with the row's kept keys k_j, values v_j:
//   s_j = scale * (q . k_j),  out = sum_j e^{s_j} v_j / sum_j e^{s_j},  lse = log sum_j e^{s_j}.
//
// A batched GEMV with G = Hq/H queries per KV head: 4 G flops per 2 d bytes of
// K and V, bound by HBM, so CUDA cores, not tensor cores.  Pass 1: kAttnChunks
// CTAs per row, each over a contiguous slice of the row's keys in tiles of 32
// keys.  K and V tiles are staged in shared memory with cp.async (16-byte
// copies, double-buffered, rows padded by 16 bytes so lane-per-key reads hit
// distinct banks).  QK: lane = key, each warp a slice of the head dims, partial
// dot products for all G queries (q pre-scaled by scale * log2 e, broadcast
// from shared memory), added over the warps in a fixed order.  Online softmax
// in base 2, one warp per query.  PV: each thread owns a pair of dims for all G
// queries over a group of the tile's keys.  The slice's unnormalised output,
// running maximum and sum go to the workspace.  Pass 2 merges a row's slices.
#include "keys.cuh"

namespace tri {

constexpr int kAttnThreads = 256;
constexpr int kAttnTile = 32;

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Record index of slot j of a paged row (-1 if the table cannot place it).
__device__ __forceinline__ int64_t paged_record(const Geometry &geo, const int32_t *table, int64_t layer_blk, int h,
                                                int64_t j) {
    const int64_t bi = j >> geo.block_shift;
    if (j < 0 || bi >= geo.max_blocks) return -1;
    const int32_t blk = __ldg(table + bi);
    if (blk < 0 || blk >= geo.n_blocks) return -1;
    return ((((layer_blk + blk) << geo.block_shift) | (j & ((1 << geo.block_shift) - 1))) * geo.H) + h;
}

// 8 elements of a record (bf16: 16 bytes, fp8: 8 bytes) from shared memory, as floats.
template <int ELEM>
__device__ __forceinline__ void smem_elems8(const char *p, float (&x)[8]) {
    if (ELEM == 2) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        unpack_bf16x8(v, x);
    } else {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        unpack_e4m3x8(v, x);
    }
}

// Two adjacent elements (dims 2i, 2i+1) of a record in shared memory.
template <int ELEM>
__device__ __forceinline__ float2 smem_elems2(const char *p) {
    if (ELEM == 2) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
        return make_float2(bf16lo(w), bf16hi(w));
    }
    return e4m3x2_to_float2(*reinterpret_cast<const uint16_t *>(p));
}

template <int ELEM, int D, int GB>
struct AttnSmem {
    static constexpr int RB = D * ELEM;           // record bytes
    static constexpr int RS = RB + 16;            // padded row stride
    static constexpr int KV = kAttnTile * RS;     // one tile of K or V
    static constexpr int off_k = 0;               // [2][KV]
    static constexpr int off_v = 2 * KV;          // [2][KV]
    static constexpr int off_q = 4 * KV;          // float [GB][D]
    static constexpr int off_red = off_q + GB * D * 4;            // float [8][GB][32] (also [G][D] at the end)
    static constexpr int off_sc = off_red + 8 * GB * kAttnTile * 4;  // float [GB][32]
    static constexpr int off_alpha = off_sc + GB * kAttnTile * 4;    // float [GB]
    static constexpr int bytes = off_alpha + GB * 4;
};

template <int ELEM, int D, int GB, bool PAGED>
__global__ void __launch_bounds__(kAttnThreads) attn_partial_kernel(const AttnParams p) {
    using SM = AttnSmem<ELEM, D, GB>;
    constexpr int RB = SM::RB, RS = SM::RS;
    constexpr int CPR = RB / 16;              // 16-byte chunks per record
    constexpr int DW = D / 8;                 // dims per warp in QK
    constexpr int NDP = D / 2;                // dim pairs
    constexpr int NKG = kAttnThreads / NDP;   // key groups in PV
    constexpr int KPG = kAttnTile / NKG;      // keys per group per tile
    extern __shared__ __align__(16) char smem[];
    char *sK = smem + SM::off_k;
    char *sV = smem + SM::off_v;
    float *qs = reinterpret_cast<float *>(smem + SM::off_q);
    float *red = reinterpret_cast<float *>(smem + SM::off_red);
    float *sc = reinterpret_cast<float *>(smem + SM::off_sc);
    float *alpha = reinterpret_cast<float *>(smem + SM::off_alpha);

    const Geometry &geo = p.geo;
    const int G = geo.G;
    const int64_t r = blockIdx.x / kAttnChunks;
    const int chunk = (int)(blockIdx.x % kAttnChunks);
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int h = (int)(r % geo.H);
    const int s = (int)((r / geo.H) % geo.S);
    const int l = (int)(r / ((int64_t)geo.H * geo.S));
    int64_t lo = geo.row_off[r], hi = geo.row_off[r + 1];
    if (lo < 0 || hi < lo || hi > geo.total) {
        if (t == 0 && chunk == 0) atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
        lo = hi = 0;
    }
    const int64_t n = hi - lo;
    const int64_t beg = n * chunk / kAttnChunks, end = n * (chunk + 1) / kAttnChunks;  // slots in the row
    const int32_t *table = geo.block_table + (int64_t)s * geo.max_blocks;
    const int64_t layer_blk = (int64_t)l * geo.n_blocks;

    // Scaled queries of this KV head's G query heads.
    const uint16_t *qrow = p.q + (((int64_t)l * geo.S + s) * geo.Hq + (int64_t)h * G) * D;
    for (int i = t; i < G * D; i += kAttnThreads)
        qs[i] = __uint_as_float((uint32_t)qrow[i] << 16) * p.scale_log2;

    // Issue the cp.async copies of the tile starting at slot j0 into buffer b.
    auto load_tile = [&](int64_t j0, int b) {
        const int cnt = (int)min((int64_t)kAttnTile, end - j0);
        for (int i = t; i < 2 * kAttnTile * CPR; i += kAttnThreads) {
            const int rec = i / CPR, part = i % CPR;
            const int key = rec % kAttnTile;
            const bool isv = rec >= kAttnTile;
            if (key >= cnt) continue;
            const int64_t j = j0 + key;
            int64_t src = PAGED ? paged_record(geo, table, layer_blk, h, j) : lo + j;
            if (src < 0) {
                if (part == 0 && !isv) atomicOr(p.flags, TRI_FLAG_BLOCK_TABLE);
                src = -1;
            }
            char *dst = (isv ? sV : sK) + b * SM::KV + key * RS + 16 * part;
            if (src >= 0) cp_async16(dst, (isv ? p.V : p.K) + src * RB + 16 * part);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        cp_async_commit();
    };

    float acc[GB][2];
#pragma unroll
    for (int g = 0; g < GB; g++) acc[g][0] = acc[g][1] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;  // of query `warp` (and warp + 8), kept by that warp
    float m_run2 = -INFINITY, l_run2 = 0.f;

    const int ntiles = (int)((end - beg + kAttnTile - 1) / kAttnTile);
    if (ntiles > 0) load_tile(beg, 0);
    for (int it = 0; it < ntiles; it++) {
        const int b = it & 1;
        const int64_t j0 = beg + (int64_t)it * kAttnTile;
        const int cnt = (int)min((int64_t)kAttnTile, end - j0);
        if (it + 1 < ntiles) {
            load_tile(j0 + kAttnTile, b ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        // QK partials: lane = key, warp = dims [warp * DW, (warp + 1) * DW).
        {
            float sp[GB];
#pragma unroll
            for (int g = 0; g < GB; g++) sp[g] = 0.f;
            const char *krow = sK + b * SM::KV + lane * RS;
#pragma unroll
            for (int c = 0; c < DW / 8; c++) {
                const int d0 = warp * DW + 8 * c;
                float x[8];
                smem_elems8<ELEM>(krow + d0 * ELEM, x);
#pragma unroll
                for (int g = 0; g < GB; g++) {
                    if (g < G) {
                        const float4 qa = *reinterpret_cast<const float4 *>(qs + g * D + d0);
                        const float4 qb = *reinterpret_cast<const float4 *>(qs + g * D + d0 + 4);
                        float a = sp[g];
                        a = fmaf(x[0], qa.x, a); a = fmaf(x[1], qa.y, a); a = fmaf(x[2], qa.z, a); a = fmaf(x[3], qa.w, a);
                        a = fmaf(x[4], qb.x, a); a = fmaf(x[5], qb.y, a); a = fmaf(x[6], qb.z, a); a = fmaf(x[7], qb.w, a);
                        sp[g] = a;
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < GB; g++)
                if (g < G) red[(warp * GB + g) * kAttnTile + lane] = sp[g];
        }
        __syncthreads();
        for (int i = t; i < G * kAttnTile; i += kAttnThreads) {
            const int g = i / kAttnTile, key = i % kAttnTile;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < 8; w++) v += red[(w * GB + g) * kAttnTile + key];
            sc[g * kAttnTile + key] = key < cnt ? v : -INFINITY;
        }
        __syncthreads();
        // Online softmax, base 2: warp w handles queries w and w + 8.
#pragma unroll
        for (int rep = 0; rep < 2; rep++) {
            const int g = warp + 8 * rep;
            if (g < G) {
                const float v = sc[g * kAttnTile + lane];
                float mt = v;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
                float &mr = rep ? m_run2 : m_run;
                float &lr = rep ? l_run2 : l_run;
                const float mn = fmaxf(mr, mt);
                const float pv = exp2f(v - mn);
                float ps = pv;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
                const float a = exp2f(mr - mn);
                lr = lr * a + ps;
                mr = mn;
                sc[g * kAttnTile + lane] = pv;
                if (lane == 0) alpha[g] = a;
            }
        }
        __syncthreads();
        // PV: thread = (key group kg, dim pair dp) over the group's keys of the tile.
        {
            const int dp = t % NDP, kg = t / NDP;
#pragma unroll
            for (int g = 0; g < GB; g++) {
                if (g < G) {
                    const float a = alpha[g];
                    acc[g][0] *= a;
                    acc[g][1] *= a;
                }
            }
            const char *vb = sV + b * SM::KV + 2 * dp * ELEM;
            for (int kk = 0; kk < KPG; kk++) {
                const int key = kg * KPG + kk;
                if (key >= cnt) break;
                const float2 v2 = smem_elems2<ELEM>(vb + key * RS);
#pragma unroll
                for (int g = 0; g < GB; g++) {
                    if (g < G) {
                        const float pr = sc[g * kAttnTile + key];
                        acc[g][0] = fmaf(pr, v2.x, acc[g][0]);
                        acc[g][1] = fmaf(pr, v2.y, acc[g][1]);
                    }
                }
            }
        }
        __syncthreads();  // buffer b is refilled by the load issued in the next iteration
    }

    // Add the key groups' accumulators in order (group 0 first), then write the slice.
    {
        const int dp = t % NDP, kg = t / NDP;
        float *buf = red;  // [G][D]
        for (int k = 0; k < NKG; k++) {
            if (kg == k) {
#pragma unroll
                for (int g = 0; g < GB; g++) {
                    if (g < G) {
                        if (k == 0) {
                            buf[g * D + 2 * dp] = acc[g][0];
                            buf[g * D + 2 * dp + 1] = acc[g][1];
                        } else {
                            buf[g * D + 2 * dp] += acc[g][0];
                            buf[g * D + 2 * dp + 1] += acc[g][1];
                        }
                    }
                }
            }
            __syncthreads();
        }
        float *out = p.part + ((r * kAttnChunks + chunk) * (int64_t)G) * (D + 2);
        for (int i = t; i < G * D; i += kAttnThreads) out[(i / D) * (D + 2) + (i % D)] = buf[i];
#pragma unroll
        for (int rep = 0; rep < 2; rep++) {
            const int g = warp + 8 * rep;
            if (g < G && lane == 0) {
                out[g * (D + 2) + D] = rep ? m_run2 : m_run;
                out[g * (D + 2) + D + 1] = rep ? l_run2 : l_run;
            }
        }
    }
}

// Merge a row's slices: one CTA of D threads per (row, query of the group).
template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(const AttnParams p) {
    const Geometry &geo = p.geo;
    const int G = geo.G;
    const int64_t r = blockIdx.x / G;
    const int g = (int)(blockIdx.x % G);
    const int dim = threadIdx.x;
    const float *part = p.part + (r * kAttnChunks * (int64_t)G + g) * (D + 2);
    float m = -INFINITY;
    for (int c = 0; c < kAttnChunks; c++) m = fmaxf(m, part[(int64_t)c * G * (D + 2) + D]);
    float num = 0.f, den = 0.f;
    if (m != -INFINITY) {
        for (int c = 0; c < kAttnChunks; c++) {
            const float *pc = part + (int64_t)c * G * (D + 2);
            const float mc = pc[D];
            if (mc == -INFINITY) continue;
            const float w = exp2f(mc - m);
            num = fmaf(w, pc[dim], num);
            den = fmaf(w, pc[D + 1], den);
        }
    }
    const int h = (int)(r % geo.H);
    const int s = (int)((r / geo.H) % geo.S);
    const int l = (int)(r / ((int64_t)geo.H * geo.S));
    const int64_t qi = ((int64_t)l * geo.S + s) * geo.Hq + (int64_t)h * G + g;
    p.out[qi * D + dim] = den > 0.f ? num / den : 0.f;
    if (p.lse && dim == 0) p.lse[qi] = den > 0.f ? (m + log2f(den)) * 0.6931471805599453f : -INFINITY;
}

template <int ELEM, int D, int GB, bool PAGED>
static cudaError_t launch_attn_t(const AttnParams &p, int64_t R, cudaStream_t s) {
    using SM = AttnSmem<ELEM, D, GB>;
    auto kern = attn_partial_kernel<ELEM, D, GB, PAGED>;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::bytes);
        if (e != cudaSuccess) return e;
        attr_set[dev & 63] = true;
    }
    kern<<<(unsigned)(R * kAttnChunks), kAttnThreads, SM::bytes, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_combine_kernel<D><<<(unsigned)(R * p.geo.G), D, 0, s>>>(p);
    return cudaGetLastError();
}

template <int ELEM, int D, bool PAGED>
static cudaError_t launch_attn_g(const AttnParams &p, int64_t R, cudaStream_t s) {
    if (p.geo.G <= 4) return launch_attn_t<ELEM, D, 4, PAGED>(p, R, s);
    if (p.geo.G <= 8) return launch_attn_t<ELEM, D, 8, PAGED>(p, R, s);
    return launch_attn_t<ELEM, D, 16, PAGED>(p, R, s);
}

template <int ELEM, bool PAGED>
static cudaError_t launch_attn_d(const AttnParams &p, int64_t R, cudaStream_t s) {
    switch (p.geo.D) {
        case 64: return launch_attn_g<ELEM, 64, PAGED>(p, R, s);
        case 128: return launch_attn_g<ELEM, 128, PAGED>(p, R, s);
        case 256: return launch_attn_g<ELEM, 256, PAGED>(p, R, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_attention(const AttnParams &p, cudaStream_t s) {
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    if (R * kAttnChunks > 0x7fffffffLL || R * p.geo.G > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const bool paged = p.geo.layout == TRI_KV_PAGED;
    if (p.geo.elem_bytes == 1) return paged ? launch_attn_d<1, true>(p, R, s) : launch_attn_d<1, false>(p, R, s);
    return paged ? launch_attn_d<2, true>(p, R, s) : launch_attn_d<2, false>(p, R, s);
}

}  // namespace tri
