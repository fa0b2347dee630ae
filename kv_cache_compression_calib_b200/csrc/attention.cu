// Decode attention over the compressed cache ("TriAttention：基于三角函数 KV 压缩的
// 高效长推理", 流程详解 step 5: every later attention step reads only the
// compressed cache, with the model's weights unchanged).  For each (layer l,
// sequence s, query head g of KV head h), with the row's kept keys k_j, values v_j:
//   s_j = scale * (q . k_j),  out = sum_j e^{s_j} v_j / sum_j e^{s_j},  lse = log sum_j e^{s_j}.
//
// A batched GEMV with G = Hq/H queries per KV head: 4 G flops per 2 d bytes of
// K and V, bound by HBM.  Pass 1 cuts every row into slices and writes each
// slice's unnormalised output, running maximum and sum to the workspace
// (attn_partial_mma, warp-level tensor-core MMAs, below; head dims 64, 128 and
// 256); pass 2 (attn_combine_kernel) merges a row's slices.
#include <algorithm>

#include <cuda_bf16.h>

#include "keys.cuh"

namespace tri {

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

// ------------------------------------------------ tensor-core slice kernel
//
// Warp-level MMAs (mma.sync m16n8k16, fp32 accumulation) with the G <= 16
// queries as the 16 rows of the A operand (head dim 256: a warp pair per item,
// see MmaSmem).  The op is HBM-bound, so the
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

// Head dim 256: a pair of warps shares each work item, warp h of the pair
// holding dims [128 h, 128 h + 128) of Q, K, V and O (so its fragments are those
// of a d = 128 warp); the two halves of every S tile are added through shared
// memory (a 64-thread named barrier per tile) before the softmax, which both
// warps then run on the same values.
template <int ELEM, int D>
struct MmaSmem {
    static constexpr bool PAIR = D > 128;                // two warps per item
    static constexpr int DW = PAIR ? D / 2 : D;          // dims per warp
    static constexpr int RB = DW * ELEM;                 // a warp's bytes of a record
    static constexpr int RS = RB + 16;                   // padded row stride of a K/V tile
    static constexpr int TILE = kMmaKeys * RS;           // one 16-key tile of K or V
    // Tiles in flight per warp (one computed, STAGES - 1 loading).  Deeper rings
    // measured no faster, for fp8 too (its tiles are half as long, but its time
    // goes to the per-tile arithmetic, which is the same as for bf16).
    static constexpr int STAGES = 2;
    static constexpr int WARP = STAGES * 2 * TILE;       // per warp: STAGES x (K, V)
    static constexpr int XCH = PAIR ? 2 * 32 * 8 * 4 : 0;  // per warp: S halves [2 tiles][32 lanes][8]
    static constexpr int WPI = PAIR ? 2 : 1;             // warps per work item
    static constexpr int bytes = kMmaWarps * (WARP + XCH);
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
__global__ void __launch_bounds__(kMmaThreads, 3) attn_partial_mma(const AttnParams p) {
    using SM = MmaSmem<ELEM, D>;
    constexpr bool F16 = ELEM == 1;
    constexpr bool PAIR = SM::PAIR;
    constexpr int DW = SM::DW, WPI = SM::WPI;
    constexpr int RB = SM::RB, RS = SM::RS, CPR = RB / 16;
    constexpr int RBG = D * ELEM;   // record bytes in the cache
    constexpr int KS = DW / 16;     // k-steps of QK (this warp's dims)
    constexpr int NT = DW / 8;      // output n-tiles of PV (this warp's dims)
    constexpr int KPI = 16 / CPR;   // keys per copy instruction (K and V of each)
    extern __shared__ __align__(16) char smem[];
    const Geometry &geo = p.geo;
    const int G = geo.G;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = PAIR ? (warp & 1) : 0;  // which dims of the item this warp holds
    const int dw0 = half * DW;               // its first dim
    const int64_t nwork = (int64_t)gridDim.x * (kMmaWarps / WPI);
    const int64_t items = (int64_t)geo.L * geo.S * geo.H * p.chunks;
    char *wbuf = smem + warp * SM::WARP;  // [stage][K, V][16 keys][RS]
    float *xch = reinterpret_cast<float *>(smem + kMmaWarps * SM::WARP);  // [warp][2][32][8]
    const float sl2 = p.scale_log2;
    grid_dependency_wait();  // the cache may come from the compaction just before
    grid_dependents_launch();

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
        const int kv = lane >> 4, c16 = lane & 15;
        const int sub = c16 / CPR, part = c16 % CPR;
        const char *base = (kv ? p.V : p.K) + dw0 * ELEM;
#pragma unroll
        for (int i = 0; i < kMmaKeys / KPI; i++) {
            const int key = i * KPI + sub;
            const int64_t rec = __shfl_sync(0xffffffffu, my_rec, key);
            char *dst = wbuf + (st * 2 + kv) * SM::TILE + key * RS + 16 * part;
            if (rec >= 0) cp_async16(dst, base + rec * RBG + 16 * part);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);  // finite zeros past the end
        }
        cp_async_commit();
    };

    // The warp's stream of (item, tile) pairs: items wid, wid + nwork, ... (both
    // warps of a pair take the same stream, so their control flow is the same).
    int64_t item = (int64_t)blockIdx.x * (kMmaWarps / WPI) + warp / WPI;
    AttnItem cur;
    cur.ntiles = 0;
    // Advance `item` to the next one with tiles; the prefetch cursor (first) writes
    // the empty results of empty items on the way.
    auto next_nonempty = [&](int64_t from, AttnItem &a, bool write_empty) -> int64_t {
        for (int64_t i = from; i < items; i += nwork) {
            a = attn_item(p, i, p.flags, write_empty && lane == 0 && (i % p.chunks) == 0);
            if (a.ntiles > 0) return i;
            float *out = p.part + (i * (int64_t)G) * (D + 2);  // an empty slice: m = -inf, l = 0, O = 0
            if (write_empty && half == 0)
                for (int k = lane; k < G * (D + 2); k += 32) out[k] = (k % (D + 2)) == D ? -INFINITY : 0.f;
        }
        return items;
    };
    // The next (item, tile) of the stream; false at its end.
    auto advance = [&](int64_t &it, AttnItem &a, int &t, bool write_empty) -> bool {
        if (t + 1 < a.ntiles) {
            t++;
            return true;
        }
        it = next_nonempty(it + nwork, a, write_empty);
        t = 0;
        return it < items;
    };
    item = next_nonempty(item, cur, true);
    if (item >= items) return;
    int tile = 0;
    // The prefetch cursor runs NS - 1 tiles ahead of the compute cursor, one
    // cp.async group per tile (an empty group past the stream's end, so that
    // waiting for all but the newest NS - 1 groups always means "this tile").
    constexpr int NS = SM::STAGES;
    int64_t pitem = item;
    AttnItem pcur = cur;
    int ptile = 0;
    bool pmore = true;
#pragma unroll
    for (int k = 0; k < NS - 1; k++) {
        if (pmore) {
            load_tile(pcur, ptile, k);
            pmore = advance(pitem, pcur, ptile, true);
        } else {
            cp_async_commit();
        }
    }
    int ci = 0;  // tiles computed so far

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
                    // fp8 caches: k index 2c + e' (+8) of k-step ks holds dim
                    // c DW/4 + 4 ks + e' (+2), c = lane % 4 (see the fp8 fragments below)
                    const int dim = F16 ? dw0 + (lane & 3) * (DW / 4) + 4 * ks + ((e & 2) ? 2 : 0)
                                        : dw0 + ks * 16 + kc + ((e & 2) ? 8 : 0);
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
        // Prefetch NS - 1 tiles ahead, into the stage computed in the previous step.
        const int st = ci % NS;
        if (pmore) {
            load_tile(pcur, ptile, (ci + NS - 1) % NS);
            pmore = advance(pitem, pcur, ptile, true);
        } else {
            cp_async_commit();
        }
        cp_async_wait<NS - 1>();
        __syncwarp();
        const int cnt = (int)min((int64_t)kMmaKeys, cur.end - (cur.beg + (int64_t)tile * kMmaKeys));
        const char *kt = wbuf + (st * 2) * SM::TILE;
        const char *vt = wbuf + (st * 2 + 1) * SM::TILE;
        // ---- S = Q K^T for keys 0-7 (sc[0]) and 8-15 (sc[1])
        // fp8 caches take the dims of the contraction in a permuted order (the sum
        // is the same for any order that Q and K share): lane c = lane % 4 holds,
        // over all k-steps, the DW/4 consecutive dims c DW/4 .. of its keys, so it
        // reads them with 16-byte loads; k-step ks uses the key's bytes 4 ks .. 4 ks + 3.
        uint32_t kw[2][F16 ? DW / 16 : 1];
        if constexpr (F16) {
            const char *k0p = kt + (lane >> 2) * RS + (lane & 3) * (DW / 4);
#pragma unroll
            for (int kk = 0; kk < 2; kk++)
#pragma unroll
                for (int v = 0; v < DW / 64; v++) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(k0p + kk * 8 * RS + 16 * v);
                    kw[kk][4 * v] = w.x;
                    kw[kk][4 * v + 1] = w.y;
                    kw[kk][4 * v + 2] = w.z;
                    kw[kk][4 * v + 3] = w.w;
                }
        }
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < KS; ks++) {
            uint32_t b[4];  // b0, b1 of keys 0-7, then of keys 8-15
            if constexpr (!F16) {
                const int mi = lane >> 3, i = lane & 7;
                const int key = i + 8 * (mi >> 1), dim = ks * 16 + 8 * (mi & 1);
                ldsm_x4(b, kt + key * RS + dim * 2);
            } else {
                b[0] = e4m3x2_to_f16x2(kw[0][ks]);
                b[1] = e4m3x2_to_f16x2(kw[0][ks] >> 16);
                b[2] = e4m3x2_to_f16x2(kw[1][ks]);
                b[3] = e4m3x2_to_f16x2(kw[1][ks] >> 16);
            }
            mma16816<F16>(sc[0], qf[ks], b[0], b[1]);
            mma16816<F16>(sc[1], qf[ks], b[2], b[3]);
        }
        if constexpr (PAIR) {
            // S = (dims 0-127 part) + (dims 128-255 part), added in that order by both
            // warps of the pair: the halves meet in shared memory (double-buffered by
            // tile parity, so one barrier per tile keeps a buffer from being rewritten
            // before the partner has read it).
            float *mine = xch + ((warp * 2 + (ci & 1)) * 32 + lane) * 8;
            const float *other = xch + (((warp ^ 1) * 2 + (ci & 1)) * 32 + lane) * 8;
#pragma unroll
            for (int e = 0; e < 8; e++) mine[e] = sc[e >> 2][e & 3];
            asm volatile("bar.sync %0, 64;" ::"r"(1 + (warp >> 1)) : "memory");
#pragma unroll
            for (int e = 0; e < 8; e++) {
                const float ov = other[e];
                sc[e >> 2][e & 3] = half == 0 ? sc[e >> 2][e & 3] + ov : ov + sc[e >> 2][e & 3];
            }
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
        // ---- O += P V
        if constexpr (!F16) {
            // two n-tiles of 8 dims per step
#pragma unroll
            for (int dt = 0; dt < NT; dt += 2) {
                uint32_t b[4];  // b0, b1 of dims dt*8.., then of dims (dt+1)*8..
                const int mi = lane >> 3, i = lane & 7;
                const int key = i + 8 * (mi & 1), dim = (dt + (mi >> 1)) * 8;
                ldsm_x4_t(b, vt + key * RS + dim * 2);
                mma16816<F16>(o[dt], ph, b[0], b[1]);
                mma16816<F16>(o[dt], pl, b[0], b[1]);
                mma16816<F16>(o[dt + 1], ph, b[2], b[3]);
                mma16816<F16>(o[dt + 1], pl, b[2], b[3]);
            }
        } else {
            // fp8: column n of n-tile j is dim n NT + j, so lane (n = lane / 4) reads
            // the NT consecutive bytes n NT .. of each of its keys 2c, 2c+1, 2c+8,
            // 2c+9 once, and pairs the keys' bytes of dim n NT + j with a byte permute.
            uint32_t vw[4][NT / 4];
            const int key = 2 * (lane & 3);
            const char *vp = vt + key * RS + (lane >> 2) * NT;
#pragma unroll
            for (int r = 0; r < 4; r++) {
                const char *row = vp + ((r & 1) + 8 * (r >> 1)) * RS;
                if constexpr (NT == 16) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(row);
                    vw[r][0] = w.x;
                    vw[r][1] = w.y;
                    vw[r][2] = w.z;
                    vw[r][3] = w.w;
                } else {
                    const uint2 w = *reinterpret_cast<const uint2 *>(row);
                    vw[r][0] = w.x;
                    vw[r][1] = w.y;
                }
            }
#pragma unroll
            for (int j = 0; j < NT; j++) {
                const uint32_t sel = (uint32_t)(j & 3) | ((uint32_t)(4 + (j & 3)) << 4);
                const uint32_t b0 = e4m3x2_to_f16x2(__byte_perm(vw[0][j >> 2], vw[1][j >> 2], sel));
                const uint32_t b1 = e4m3x2_to_f16x2(__byte_perm(vw[2][j >> 2], vw[3][j >> 2], sel));
                mma16816<F16>(o[j], ph, b0, b1);
                mma16816<F16>(o[j], pl, b0, b1);
            }
        }
        __syncwarp();  // this stage is refilled by the next step's prefetch
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
                // column c of n-tile i: dim i 8 + c (bf16), dim c NT + i (fp8, permuted)
                const int d0 = dw0 + (F16 ? c0 * NT + i : i * 8 + c0);
                const int d1 = dw0 + (F16 ? (c0 + 1) * NT + i : i * 8 + c0 + 1);
                if (g0 < G) {
                    out[g0 * (D + 2) + d0] = o[i][0];
                    out[g0 * (D + 2) + d1] = o[i][1];
                }
                if (g1 < G) {
                    out[g1 * (D + 2) + d0] = o[i][2];
                    out[g1 * (D + 2) + d1] = o[i][3];
                }
            }
            if ((lane & 3) == 0 && half == 0) {
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
        if (!advance(item, cur, tile, false)) break;
        ci++;
    }
    cp_async_wait<0>();
}

// Merge a row's slices: one CTA of D threads per (row, query of the group).
template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(const AttnParams p) {
    grid_dependency_wait();
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
    // Persistent grid of the resident CTAs; rows cut into c slices, the workers
    // taking items round-robin.  At most about two items per worker (each slice
    // adds (d + 2) G floats written and read back, and a few dependent loads per
    // item); within that, the slowest worker streams ceil(R c / workers) items of
    // about keys/(R c) keys each plus a fixed cost per item, and c minimises that
    // (the smallest such c): a last round that keeps few workers busy is avoided.
    AttnParams p = p0;
    const int64_t ctas = (int64_t)sm_count() * o;
    const int64_t per_cta = kMmaWarps / SM::WPI;  // workers per CTA (a warp, or a warp pair)
    const int64_t workers = ctas * per_cta;
    const int64_t keys_per_row = std::max<int64_t>(1, p.geo.total / R);
    const int c_max = (int)std::min<int64_t>(kAttnMaxChunks, std::max<int64_t>(1, (2 * workers + R - 1) / R));
    int64_t best = -1;
    p.chunks = 1;
    for (int c = 1; c <= c_max; c++) {
        const int64_t rounds = (R * c + workers - 1) / workers;
        const int64_t tiles = (keys_per_row + (int64_t)c * kMmaKeys - 1) / ((int64_t)c * kMmaKeys);
        const int64_t cost = rounds * (tiles + 2);
        if (best < 0 || cost < best) {
            best = cost;
            p.chunks = c;
        }
    }
    const int64_t grid = std::min<int64_t>(ctas, (R * p.chunks + per_cta - 1) / per_cta);
    cudaError_t e = launch_pdl(kern, dim3((unsigned)grid), dim3(kMmaThreads), SM::bytes, s, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_combine_kernel<D>, dim3((unsigned)(R * p.geo.G)), dim3(D), 0, s, p);
}

template <int ELEM, int D, bool PAGED>
static cudaError_t launch_attn_g(const AttnParams &p, int64_t R, cudaStream_t s) {
    return launch_attn_mma<ELEM, D, PAGED>(p, R, s);
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
