// Decode attention over the compressed cache ("TriAttention：基于三角函数 KV 压缩的
// 高效长推理", 流程详解 step 5: every later attention step reads only the
// compressed cache, with the model's weights unchanged).  For each (layer l,
// sequence s, query head g of KV head h), with the row's kept keys k_j, values v_j:
//   s_j = scale * (q . k_j),  out = sum_j e^{s_j} v_j / sum_j e^{s_j},  lse = log sum_j e^{s_j}.
//
// A batched GEMV with G = Hq/H queries per KV head: 4 G flops per 2 d bytes of
// K and V, bound by HBM.  Pass 1 cuts every row into slices and writes each
// slice's unnormalised output, running maximum and sum to the workspace; pass 2
// (attn_combine_kernel) merges a row's slices.  Pass 1 has two kernels:
// attn_partial_mma (d <= 128, warp-level tensor-core MMAs, below) and
// attn_partial_simt (d = 256, CUDA cores), described here.  `chunks` CTAs per
// row (about one wave over the SMs), each over a contiguous slice of the row's
// keys in tiles of TK keys (64, or 32 for 512-byte records).  K and V tiles are
// staged in shared memory with cp.async (16-byte copies, double-buffered, rows
// padded by 16 bytes so lane-per-key reads hit distinct banks).  QK: lane =
// key, warps split the tile's keys into 32-key halves and the head dims into
// slices, partial dot products for all G queries (q pre-scaled by scale * log2
// e, broadcast from shared memory), added over the dim slices in a fixed order.
// Online softmax in base 2, one warp per query.  PV: each thread owns a pair of
// dims for all G queries over a group of the tile's keys.
#include <algorithm>

#include <cuda_bf16.h>

#include "keys.cuh"

namespace tri {

constexpr int kAttnThreads = 256;

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
    static constexpr int TK = RB <= 256 ? 64 : 32;  // keys per tile
    static constexpr int NKH = TK / 32;           // 32-key halves of a tile (QK)
    static constexpr int NDQ = 8 / NKH;           // head-dim slices (QK)
    static constexpr int KV = TK * RS;            // one tile of K or V
    static constexpr int off_k = 0;               // [2][KV]
    static constexpr int off_v = 2 * KV;          // [2][KV]
    static constexpr int off_q = 4 * KV;          // float [GB][D]
    static constexpr int off_red = off_q + GB * D * 4;            // float [NDQ][GB][TK] (also [G][D] at the end)
    static constexpr int off_sc = off_red + NDQ * GB * TK * 4;    // float [GB][TK]
    static constexpr int off_alpha = off_sc + GB * TK * 4;        // float [GB]
    static constexpr int bytes = off_alpha + GB * 4;
    static_assert(NDQ * GB * TK >= GB * D, "the final [G][D] sum reuses the QK partial buffer");
};

template <int ELEM, int D, int GB, bool PAGED>
__global__ void __launch_bounds__(kAttnThreads) attn_partial_simt(const AttnParams p) {
    using SM = AttnSmem<ELEM, D, GB>;
    constexpr int RB = SM::RB, RS = SM::RS, TK = SM::TK, NDQ = SM::NDQ;
    constexpr int CPR = RB / 16;              // 16-byte chunks per record
    constexpr int DW = D / NDQ;               // dims per warp in QK
    constexpr int NDP = D / 2;                // dim pairs
    constexpr int NKG = kAttnThreads / NDP;   // key groups in PV
    constexpr int KPG = TK / NKG;             // keys per group per tile
    extern __shared__ __align__(16) char smem[];
    char *sK = smem + SM::off_k;
    char *sV = smem + SM::off_v;
    float *qs = reinterpret_cast<float *>(smem + SM::off_q);
    float *red = reinterpret_cast<float *>(smem + SM::off_red);
    float *sc = reinterpret_cast<float *>(smem + SM::off_sc);
    float *alpha = reinterpret_cast<float *>(smem + SM::off_alpha);

    const Geometry &geo = p.geo;
    const int G = geo.G;
    const int nc = p.chunks;
    const int64_t r = blockIdx.x / nc;
    const int chunk = (int)(blockIdx.x % nc);
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
    const int64_t beg = n * chunk / nc, end = n * (chunk + 1) / nc;  // slots in the row
    const int32_t *table = geo.block_table + (int64_t)s * geo.max_blocks;
    const int64_t layer_blk = (int64_t)l * geo.n_blocks;

    // Scaled queries of this KV head's G query heads.
    const uint16_t *qrow = p.q + (((int64_t)l * geo.S + s) * geo.Hq + (int64_t)h * G) * D;
    for (int i = t; i < G * D; i += kAttnThreads)
        qs[i] = __uint_as_float((uint32_t)qrow[i] << 16) * p.scale_log2;

    // Issue the cp.async copies of the tile starting at slot j0 into buffer b.
    auto load_tile = [&](int64_t j0, int b) {
        const int cnt = (int)min((int64_t)TK, end - j0);
        for (int i = t; i < 2 * TK * CPR; i += kAttnThreads) {
            const int rec = i / CPR, part = i % CPR;
            const int key = rec % TK;
            const bool isv = rec >= TK;
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

    const int ntiles = (int)((end - beg + TK - 1) / TK);
    if (ntiles > 0) load_tile(beg, 0);
    for (int it = 0; it < ntiles; it++) {
        const int b = it & 1;
        const int64_t j0 = beg + (int64_t)it * TK;
        const int cnt = (int)min((int64_t)TK, end - j0);
        if (it + 1 < ntiles) {
            load_tile(j0 + TK, b ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        // QK partials: key = 32 * (warp % NKH) + lane, dims [dq * DW, (dq + 1) * DW).
        {
            const int key = 32 * (warp % SM::NKH) + lane, dq = warp / SM::NKH;
            float sp[GB];
#pragma unroll
            for (int g = 0; g < GB; g++) sp[g] = 0.f;
            const char *krow = sK + b * SM::KV + key * RS;
#pragma unroll
            for (int c = 0; c < DW / 8; c++) {
                const int d0 = dq * DW + 8 * c;
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
                if (g < G) red[(dq * GB + g) * TK + key] = sp[g];
        }
        __syncthreads();
        for (int i = t; i < G * TK; i += kAttnThreads) {
            const int g = i / TK, key = i % TK;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < NDQ; w++) v += red[(w * GB + g) * TK + key];
            sc[g * TK + key] = key < cnt ? v : -INFINITY;
        }
        __syncthreads();
        // Online softmax, base 2: warp w handles queries w and w + 8.
#pragma unroll
        for (int rep = 0; rep < 2; rep++) {
            const int g = warp + 8 * rep;
            if (g < G) {
                float v[SM::NKH];
                float mt = -INFINITY;
#pragma unroll
                for (int k = 0; k < SM::NKH; k++) {
                    v[k] = sc[g * TK + 32 * k + lane];
                    mt = fmaxf(mt, v[k]);
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
                float &mr = rep ? m_run2 : m_run;
                float &lr = rep ? l_run2 : l_run;
                const float mn = fmaxf(mr, mt);
                float ps = 0.f;
#pragma unroll
                for (int k = 0; k < SM::NKH; k++) {
                    const float pv = exp2f(v[k] - mn);
                    sc[g * TK + 32 * k + lane] = pv;
                    ps += pv;
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
                const float a = exp2f(mr - mn);
                lr = lr * a + ps;
                mr = mn;
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
                        const float pr = sc[g * TK + key];
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
        float *out = p.part + ((r * nc + chunk) * (int64_t)G) * (D + 2);
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

// ------------------------------------------------ tensor-core slice kernel
//
// For d <= 128: warp-level MMAs (mma.sync m16n8k16, fp32 accumulation) with the
// G <= 16 queries as the 16 rows of the A operand.  The op is HBM-bound, so the
// tensor pipe only takes the multiply-adds off the CUDA cores.  (The transposed
// form, keys on the 128-row M side of tcgen05.mma and the queries on N, is the
// kernel of attention_tc.cu; on the same caches it is slower than this one,
// because each 128-key tile's softmax sits between its two MMAs in one
// warpgroup's chain.)  bf16 caches use bf16 MMAs (the q and key
// products are exact in fp32); fp8 caches use f16 MMAs with e4m3 converted to
// f16 exactly and q rounded to f16 (exact for |q| in [2^-14, 65504]).  A
// persistent grid of the resident CTAs (4 warps each): every warp is a worker
// that takes work items (row, slice) wid, wid + workers, ... and streams their
// 16-key tiles through a private double buffer, prefetching across the end of
// one item into the next, so there is no CTA barrier anywhere.
//   S = Q K^T: K rows as the col-major B operand (ldmatrix, or e4m3 pairs
//     converted in registers); scores scaled into base 2, masked past the slice.
//   Online softmax per query row (4 lanes per row, shuffles).
//   O += P V: the S accumulator fragments are the A fragments of the PV MMA;
//     P is split into hi + lo halves (two MMAs) so P keeps ~16 bits; V via
//     ldmatrix.trans (or e4m3 pairs gathered by key).
// At the end of an item its worker writes the slice's (O, m, l) for the G rows.
constexpr int kMmaWarps = 4;
constexpr int kMmaThreads = 32 * kMmaWarps;
constexpr int kMmaKeys = 16;  // keys per warp tile

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *smem) {
    const unsigned a = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *smem) {
    const unsigned a = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}

// d += a * b for one m16n8k16 tile: bf16 (F16 = false) or f16 operands, fp32 accumulators.
template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if (F16)
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    else
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats as a packed pair of the MMA element type (low half = first), rounded to nearest.
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float x, float y) {
    if (F16) {
        const __half2 h = __floats2half2_rn(x, y);
        return *reinterpret_cast<const uint32_t *>(&h);
    }
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<const uint32_t *>(&h);
}
template <bool F16>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
    if (F16) return __half22float2(*reinterpret_cast<const __half2 *>(&w));
    return make_float2(bf16lo(w), bf16hi(w));
}

// Two e4m3 bytes (low byte first) as an f16 pair.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

template <int ELEM, int D>
struct MmaSmem {
    static constexpr int RB = D * ELEM;                  // record bytes
    static constexpr int RS = RB + 16;                   // padded row stride of a K/V tile
    static constexpr int TILE = kMmaKeys * RS;           // one 16-key tile of K or V
    static constexpr int WARP = 2 * 2 * TILE;            // per warp: 2 stages x (K, V)
    static constexpr int bytes = kMmaWarps * WARP;
};

// One work item: slice `c` of row `r`, keys [beg, end) of the row.
struct AttnItem {
    int64_t r, lo, beg, end;
    int h, s, l;
    int ntiles;
};

__device__ __forceinline__ AttnItem attn_item(const AttnParams &p, int64_t item, unsigned *flags, bool report) {
    const Geometry &geo = p.geo;
    AttnItem it;
    it.r = item / p.chunks;
    const int c = (int)(item % p.chunks);
    it.h = (int)(it.r % geo.H);
    it.s = (int)((it.r / geo.H) % geo.S);
    it.l = (int)(it.r / ((int64_t)geo.H * geo.S));
    int64_t lo = geo.row_off[it.r], hi = geo.row_off[it.r + 1];
    if (lo < 0 || hi < lo || hi > geo.total) {
        if (report) atomicOr(flags, TRI_FLAG_ROW_OFFSETS);
        lo = hi = 0;
    }
    const int64_t n = hi - lo;
    it.lo = lo;
    it.beg = n * c / p.chunks;
    it.end = n * (c + 1) / p.chunks;
    it.ntiles = (int)((it.end - it.beg + kMmaKeys - 1) / kMmaKeys);
    return it;
}

template <int ELEM, int D, bool PAGED>
__global__ void __launch_bounds__(kMmaThreads) attn_partial_mma(const AttnParams p) {
    using SM = MmaSmem<ELEM, D>;
    constexpr bool F16 = ELEM == 1;
    constexpr int RB = SM::RB, RS = SM::RS, CPR = RB / 16;
    constexpr int KS = D / 16;  // k-steps of QK
    constexpr int NT = D / 8;   // output n-tiles of PV
    constexpr int KPI = 16 / CPR;  // keys per copy instruction (K and V of each)
    extern __shared__ __align__(16) char smem[];
    const Geometry &geo = p.geo;
    const int G = geo.G;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t nwork = (int64_t)gridDim.x * kMmaWarps;
    const int64_t items = (int64_t)geo.L * geo.S * geo.H * p.chunks;
    char *wbuf = smem + warp * SM::WARP;  // [stage][K, V][16 keys][RS]
    const float sl2 = p.scale_log2;

    // Copy tile `ti` of item `a` into stage `st`: lane i < 16 finds the record of
    // key i once; every instruction then moves whole records, half the warp on K
    // and half on V (16-byte chunks, consecutive lanes on consecutive chunks).
    auto load_tile = [&](const AttnItem &a, int ti, int st) {
        const int64_t j0 = a.beg + (int64_t)ti * kMmaKeys;
        const int cnt = (int)min((int64_t)kMmaKeys, a.end - j0);
        int64_t my_rec = -1;
        if (lane < kMmaKeys && lane < cnt) {
            if (PAGED) {
                const int32_t *table = geo.block_table + (int64_t)a.s * geo.max_blocks;
                my_rec = paged_record(geo, table, (int64_t)a.l * geo.n_blocks, a.h, j0 + lane);
                if (my_rec < 0) atomicOr(p.flags, TRI_FLAG_BLOCK_TABLE);
            } else {
                my_rec = a.lo + j0 + lane;
            }
        }
        const int half = lane >> 4, c16 = lane & 15;
        const int sub = c16 / CPR, part = c16 % CPR;
        const char *base = half ? p.V : p.K;
#pragma unroll
        for (int i = 0; i < kMmaKeys / KPI; i++) {
            const int key = i * KPI + sub;
            const int64_t rec = __shfl_sync(0xffffffffu, my_rec, key);
            char *dst = wbuf + (st * 2 + half) * SM::TILE + key * RS + 16 * part;
            if (rec >= 0) cp_async16(dst, base + rec * RB + 16 * part);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);  // finite zeros past the end
        }
        cp_async_commit();
    };

    // The warp's stream of (item, tile) pairs: items wid, wid + nwork, ...
    int64_t item = (int64_t)blockIdx.x * kMmaWarps + warp;
    AttnItem cur;
    cur.ntiles = 0;
    // Advance `item` to the next one with tiles, writing empty results for empty items.
    auto next_nonempty = [&](int64_t from, AttnItem &a) -> int64_t {
        for (int64_t i = from; i < items; i += nwork) {
            a = attn_item(p, i, p.flags, lane == 0 && (i % p.chunks) == 0);
            if (a.ntiles > 0) return i;
            float *out = p.part + (i * (int64_t)G) * (D + 2);  // an empty slice: m = -inf, l = 0, O = 0
            for (int k = lane; k < G * (D + 2); k += 32) out[k] = (k % (D + 2)) == D ? -INFINITY : 0.f;
        }
        return items;
    };
    item = next_nonempty(item, cur);
    if (item >= items) return;
    int tile = 0, st = 0;
    load_tile(cur, 0, 0);

    uint32_t qf[KS][4];
    float o[NT][4];
    float m0 = -INFINITY, m1 = -INFINITY;  // rows lane/4 and lane/4 + 8
    float l0 = 0.f, l1 = 0.f;              // this lane's share of the row sums
    for (;;) {
        if (tile == 0) {
            // Query fragments of this item's row: A operand rows g = lane/4 (+8), k = dims.
            const uint16_t *qrow = p.q + (((int64_t)cur.l * geo.S + cur.s) * geo.Hq + (int64_t)cur.h * G) * D;
            const int g0 = lane >> 2, g1 = g0 + 8, kc = 2 * (lane & 3);
#pragma unroll
            for (int ks = 0; ks < KS; ks++) {
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int g = (e & 1) ? g1 : g0;
                    const int dim = ks * 16 + kc + ((e & 2) ? 8 : 0);
                    uint32_t w = 0u;
                    if (g < G) {
                        const uint32_t raw = (uint32_t)qrow[(int64_t)g * D + dim] | ((uint32_t)qrow[(int64_t)g * D + dim + 1] << 16);
                        w = F16 ? pack2<true>(bf16lo(raw), bf16hi(raw)) : raw;
                    }
                    qf[ks][e] = w;
                }
            }
#pragma unroll
            for (int i = 0; i < NT; i++) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
        }
        // Prefetch the next tile of the stream (this item's next, or the next item's first).
        AttnItem nxt = cur;
        int64_t nitem = item;
        int ntile = tile + 1;
        if (ntile >= cur.ntiles) {
            nitem = next_nonempty(item + nwork, nxt);
            ntile = 0;
        }
        const bool more = nitem < items;
        if (more) {
            load_tile(nxt, ntile, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        const int cnt = (int)min((int64_t)kMmaKeys, cur.end - (cur.beg + (int64_t)tile * kMmaKeys));
        const char *kt = wbuf + (st * 2) * SM::TILE;
        const char *vt = wbuf + (st * 2 + 1) * SM::TILE;
        // ---- S = Q K^T for keys 0-7 (sc[0]) and 8-15 (sc[1])
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < KS; ks++) {
            uint32_t b[4];  // b0, b1 of keys 0-7, then of keys 8-15
            if (!F16) {
                const int mi = lane >> 3, i = lane & 7;
                const int key = i + 8 * (mi >> 1), dim = ks * 16 + 8 * (mi & 1);
                ldsm_x4(b, kt + key * RS + dim * 2);
            } else {
                const int key = lane >> 2, dim = ks * 16 + 2 * (lane & 3);
                b[0] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t *>(kt + key * RS + dim));
                b[1] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t *>(kt + key * RS + dim + 8));
                b[2] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t *>(kt + (key + 8) * RS + dim));
                b[3] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t *>(kt + (key + 8) * RS + dim + 8));
            }
            mma16816<F16>(sc[0], qf[ks], b[0], b[1]);
            mma16816<F16>(sc[1], qf[ks], b[2], b[3]);
        }
        // ---- scale to base 2, mask keys past the slice (partial tiles only), online softmax per row
        const int kc = 2 * (lane & 3);
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; nt++) {
#pragma unroll
            for (int e = 0; e < 2; e++) {
                sc[nt][e] *= sl2;
                sc[nt][2 + e] *= sl2;
                if (cnt < kMmaKeys && nt * 8 + kc + e >= cnt) sc[nt][e] = sc[nt][2 + e] = -INFINITY;
                mx0 = fmaxf(mx0, sc[nt][e]);
                mx1 = fmaxf(mx1, sc[nt][2 + e]);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float a0 = exp2f(m0 - mn0), a1 = exp2f(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; nt++) {
#pragma unroll
            for (int e = 0; e < 2; e++) {
                sc[nt][e] = exp2f(sc[nt][e] - mn0);
                sc[nt][2 + e] = exp2f(sc[nt][2 + e] - mn1);
                ps0 += sc[nt][e];
                ps1 += sc[nt][2 + e];
            }
        }
        l0 = l0 * a0 + ps0;
        l1 = l1 * a1 + ps1;
        if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {  // some row's maximum moved
#pragma unroll
            for (int i = 0; i < NT; i++) {
                o[i][0] *= a0;
                o[i][1] *= a0;
                o[i][2] *= a1;
                o[i][3] *= a1;
            }
        }
        // ---- P as A fragments (rows = queries, k = the 16 keys), hi + lo
        uint32_t ph[4], pl[4];
        {
            const float src[4][2] = {{sc[0][0], sc[0][1]}, {sc[0][2], sc[0][3]}, {sc[1][0], sc[1][1]},
                                     {sc[1][2], sc[1][3]}};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                ph[i] = pack2<F16>(src[i][0], src[i][1]);
                const float2 back = unpack2<F16>(ph[i]);
                pl[i] = pack2<F16>(src[i][0] - back.x, src[i][1] - back.y);
            }
        }
        // ---- O += P V, two n-tiles of 8 dims per step
#pragma unroll
        for (int dt = 0; dt < NT; dt += 2) {
            uint32_t b[4];  // b0, b1 of dims dt*8.., then of dims (dt+1)*8..
            if (!F16) {
                const int mi = lane >> 3, i = lane & 7;
                const int key = i + 8 * (mi & 1), dim = (dt + (mi >> 1)) * 8;
                ldsm_x4_t(b, vt + key * RS + dim * 2);
            } else {
                const int key = 2 * (lane & 3), dim = lane >> 2;
#pragma unroll
                for (int hh = 0; hh < 2; hh++) {
                    const int dd = (dt + hh) * 8 + dim;
                    const uint32_t k0 = (uint8_t)vt[key * RS + dd], k1 = (uint8_t)vt[(key + 1) * RS + dd];
                    const uint32_t k8 = (uint8_t)vt[(key + 8) * RS + dd], k9 = (uint8_t)vt[(key + 9) * RS + dd];
                    b[2 * hh] = e4m3x2_to_f16x2(k0 | (k1 << 8));
                    b[2 * hh + 1] = e4m3x2_to_f16x2(k8 | (k9 << 8));
                }
            }
            mma16816<F16>(o[dt], ph, b[0], b[1]);
            mma16816<F16>(o[dt], pl, b[0], b[1]);
            mma16816<F16>(o[dt + 1], ph, b[2], b[3]);
            mma16816<F16>(o[dt + 1], pl, b[2], b[3]);
        }
        __syncwarp();  // this stage is refilled by the prefetch after next
        if (tile + 1 == cur.ntiles) {
            // Item done: row sums over the 4 lanes of each row, then (O, m, l) of rows < G.
            float s0 = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
            s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
            float s1 = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
            float *out = p.part + (item * (int64_t)G) * (D + 2);
            const int g0 = lane >> 2, g1 = g0 + 8, c0 = 2 * (lane & 3);
#pragma unroll
            for (int i = 0; i < NT; i++) {
                if (g0 < G) {
                    out[g0 * (D + 2) + i * 8 + c0] = o[i][0];
                    out[g0 * (D + 2) + i * 8 + c0 + 1] = o[i][1];
                }
                if (g1 < G) {
                    out[g1 * (D + 2) + i * 8 + c0] = o[i][2];
                    out[g1 * (D + 2) + i * 8 + c0 + 1] = o[i][3];
                }
            }
            if ((lane & 3) == 0) {
                if (g0 < G) {
                    out[g0 * (D + 2) + D] = m0;
                    out[g0 * (D + 2) + D + 1] = s0;
                }
                if (g1 < G) {
                    out[g1 * (D + 2) + D] = m1;
                    out[g1 * (D + 2) + D + 1] = s1;
                }
            }
        }
        if (!more) break;
        item = nitem;
        cur = nxt;
        tile = ntile;
        st ^= 1;
    }
    cp_async_wait<0>();
}

// Merge a row's slices: one CTA of D threads per (row, query of the group).
template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(const AttnParams p) {
    const Geometry &geo = p.geo;
    const int G = geo.G;
    const int nc = p.chunks;
    const int64_t r = blockIdx.x / G;
    const int g = (int)(blockIdx.x % G);
    const int dim = threadIdx.x;
    const float *part = p.part + (r * nc * (int64_t)G + g) * (D + 2);
    float m = -INFINITY;
    for (int c = 0; c < nc; c++) m = fmaxf(m, part[(int64_t)c * G * (D + 2) + D]);
    float num = 0.f, den = 0.f;
    if (m != -INFINITY) {
        for (int c = 0; c < nc; c++) {
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
static cudaError_t launch_attn_t(const AttnParams &p0, int64_t R, cudaStream_t s) {
    using SM = AttnSmem<ELEM, D, GB>;
    auto kern = attn_partial_simt<ELEM, D, GB, PAGED>;
    static int occ[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int &o = occ[dev & 63];
    if (o == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::bytes);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, kAttnThreads, SM::bytes);
        if (e != cudaSuccess) return e;
        if (o < 1) o = 1;
    }
    // About one wave: enough slices per row to give every SM its resident CTAs.
    AttnParams p = p0;
    const int64_t slots = (int64_t)sm_count() * o;
    p.chunks = (int)std::min<int64_t>(kAttnMaxChunks, std::max<int64_t>(1, (slots + R - 1) / R));
    kern<<<(unsigned)(R * p.chunks), kAttnThreads, SM::bytes, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_combine_kernel<D><<<(unsigned)(R * p.geo.G), D, 0, s>>>(p);
    return cudaGetLastError();
}

template <int ELEM, int D, bool PAGED>
static cudaError_t launch_attn_mma(const AttnParams &p0, int64_t R, cudaStream_t s) {
    using SM = MmaSmem<ELEM, D>;
    auto kern = attn_partial_mma<ELEM, D, PAGED>;
    static int occ[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int &o = occ[dev & 63];
    if (o == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::bytes);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, kMmaThreads, SM::bytes);
        if (e != cudaSuccess) return e;
        if (o < 1) o = 1;
    }
    // Persistent grid of the resident CTAs; rows cut into enough slices that every
    // warp gets about two work items (each slice costs (d + 2) G floats written
    // and read back, so more slices than that only add traffic).
    AttnParams p = p0;
    const int64_t ctas = (int64_t)sm_count() * o;
    const int64_t workers = ctas * kMmaWarps;
    p.chunks = (int)std::min<int64_t>(kAttnMaxChunks, std::max<int64_t>(1, (2 * workers + R - 1) / R));
    const int64_t grid = std::min<int64_t>(ctas, (R * p.chunks + kMmaWarps - 1) / kMmaWarps);
    kern<<<(unsigned)grid, kMmaThreads, SM::bytes, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_combine_kernel<D><<<(unsigned)(R * p.geo.G), D, 0, s>>>(p);
    return cudaGetLastError();
}

template <int ELEM, int D, bool PAGED>
static cudaError_t launch_attn_g(const AttnParams &p, int64_t R, cudaStream_t s) {
    if (D <= 128) return launch_attn_mma<ELEM, (D <= 128 ? D : 128), PAGED>(p, R, s);
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

cudaError_t launch_attn_combine(const AttnParams &p, int64_t R, cudaStream_t s) {
    switch (p.geo.D) {
        case 64: attn_combine_kernel<64><<<(unsigned)(R * p.geo.G), 64, 0, s>>>(p); break;
        case 128: attn_combine_kernel<128><<<(unsigned)(R * p.geo.G), 128, 0, s>>>(p); break;
        case 256: attn_combine_kernel<256><<<(unsigned)(R * p.geo.G), 256, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_attention(const AttnParams &p, cudaStream_t s) {
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    if (R * kAttnMaxChunks > 0x7fffffffLL || R * p.geo.G > 0x7fffffffLL) return cudaErrorInvalidConfiguration;

    const bool paged = p.geo.layout == TRI_KV_PAGED;
    if (p.geo.elem_bytes == 1) return paged ? launch_attn_d<1, true>(p, R, s) : launch_attn_d<1, false>(p, R, s);
    return paged ? launch_attn_d<2, true>(p, R, s) : launch_attn_d<2, false>(p, R, s);
}

}  // namespace tri
