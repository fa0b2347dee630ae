// Decode attention on the 5th-generation tensor cores ("TriAttention：基于三角函数
// KV 压缩的高效长推理", 流程详解 step 5: later attention steps read only the
// compressed cache).  For bf16 caches of head dim 128 in the contiguous layout
// (the [R][B] output of tri_compact, or any contiguous cache) and G <= 16
// queries per KV head (tri_decode_attention_tc); tri_decode_attention runs
// attn_partial_mma, which serves every case and measured faster on these.
//
// The contraction is transposed so the keys, not the few queries, fill the
// 128-row tile of tcgen05.mma:
//   S^T [128 keys x 16]  = K_tile [128 keys x 128 dims] . Q^T [128 dims x 16 queries]
//   O^T [128 dims x 16] += V_tile^T [128 dims x 128 keys] . P^T [128 keys x 16 queries]
// (queries G..15 are zero).  K and V tiles are brought into shared memory by
// TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast) on transaction-
// counting mbarriers; both products run as tcgen05.mma kind::f16 issued by one
// thread, with their fp32 accumulators in tensor memory (S in two 16-column
// buffers, O in two more), read back with tcgen05.ld.  One warpgroup per CTA:
// thread t owns TMEM lane t, i.e. key t of a tile for S and dim t for O.
//   - K tiles: K-major A operand (dims contiguous per key), 128-byte swizzle.
//   - V tiles: the same bytes read as an MN-major A operand (V^T, dims contiguous).
//   - Q and P: K-major B operands without swizzle, 8 x 16-byte core matrices.
// Softmax is online in base 2: per tile, the tile maximum of every query over
// the 128 keys (a warp reduce-scatter, then 4 warps through shared memory),
// p = 2^(s - m) in fp32, split into bf16 hi + lo parts for two PV products
// (~16-bit weights), per-thread fp32 partial sums rescaled as the maximum
// grows.  The output of tile i is read from TMEM and added to the registers
// while tile i+1 runs (O double-buffered), and the QK product of tile i+1 is
// issued before tile i's softmax (S double-buffered); K and V tiles are fetched
// up to three tiles ahead (three stages each).  A persistent grid of one CTA per SM takes (row,
// slice) items in turn and writes each slice's unnormalised output, maximum and
// sum; attn_combine_kernel merges a row's slices.  Every wait is bounded
// (TRI_FLAG_STAGE_TIMEOUT); tensor memory is released before the CTA exits.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "stage.cuh"

namespace tri {

cudaError_t launch_attn_combine(const AttnParams &p, int64_t R, cudaStream_t s);

namespace {

constexpr int kTcThreads = 128;  // one warpgroup: thread t <-> TMEM lane t
constexpr int kTcKeys = 128;     // keys per tile: M of the QK product
constexpr int kTcN = 16;         // query columns (G <= 16, padded with zeros)
constexpr int kTcD = 128;        // head dim: M of the PV product
constexpr int kTcBoxDims = 64;   // dims per TMA box: one 128-byte swizzle row
constexpr int kTcBoxBytes = kTcKeys * kTcBoxDims * 2;  // 16 KB
constexpr int kTcTileBytes = 2 * kTcBoxBytes;          // 32 KB: a K or V tile
constexpr int kTcBBytes = kTcN * kTcD * 2;             // 4 KB: Q, or one P part
constexpr int kTcTmemCols = 64;                        // S[2], O[2]: 16 columns each

// P (a B operand, [16 queries][128 keys]) uses a padded core-matrix layout: the
// core matrices of 8 keys are 144 bytes apart (not 128), so the four key groups a
// warp's 32 lanes write for one query fall on different banks.
constexpr int kPLbo = 144;               // between core matrices along the keys
constexpr int kPSbo = 16 * kPLbo;        // between the two groups of 8 queries
constexpr int kPBytes = 2 * kPSbo;       // one P part: 4608 bytes
constexpr int kTcStages = 3;             // K and V tiles in flight per CTA

// Shared memory, from a 1024-byte aligned base (swizzle atoms need it).
constexpr int kSmK = 0;                                 // K tiles [kTcStages]
constexpr int kSmV = kSmK + kTcStages * kTcTileBytes;   // V tiles [kTcStages]
constexpr int kSmP = kSmV + kTcStages * kTcTileBytes;   // P [2 buffers][hi, lo]
constexpr int kSmQ = kSmP + 4 * kPBytes;                // Q
constexpr int kSmRed = kSmQ + kTcBBytes;                // float [16][4] per-warp reductions
constexpr int kSmBar = kSmRed + kTcN * 4 * 4;           // 10 mbarriers
constexpr int kSmTmem = kSmBar + 10 * 8;                // allocated TMEM base
constexpr int kSmAbort = kSmTmem + 4;                   // 1 after a wait ran out
constexpr size_t kTcSmem = kSmAbort + 4 + 1024;         // + alignment slack

// ---------------------------------------------------------------- descriptors

// Shared-memory matrix descriptor of tcgen05.mma: start address, leading and
// stride byte offsets (all in 16-byte units), descriptor version 1 at bit 46,
// swizzle mode at bits 61-63 (0: none, 2: 128-byte).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t swizzle) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)swizzle << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), bf16 A
// and B (bits 7-9, 10-12 = 1), A major-ness (bit 15: 0 K, 1 MN), B K-major, N/8
// at bits 17-22, M/16 at bits 24-28.
constexpr uint32_t idesc_bf16(int M, int N, int a_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdescQK = idesc_bf16(kTcKeys, kTcN, 0);
constexpr uint32_t kIdescPV = idesc_bf16(kTcD, kTcN, 1);

// K-major B operand without swizzle: core matrix (row group i of 8 rows, column
// group j of 8 elements) at i * sbo + j * lbo bytes, its rows 16 bytes apart.
__device__ __forceinline__ uint32_t b_core_offset(int row, int col, int lbo = 128, int sbo = 2048) {
    return (uint32_t)((row >> 3) * sbo + (col >> 3) * lbo + (row & 7) * 16 + (col & 7) * 2);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// Arrive on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes 32w..32w+31).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}

// One 64-dim x 128-key box of a K or V tile: TMA from the tensor map at
// (x = dims, y = key), completing `bar`'s transaction count.  No multicast.
__device__ __forceinline__ void tma_box(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_tile(unsigned char *dst, const CUtensorMap *map, int64_t key0, uint64_t *bar) {
    mbar_arrive_expect_tx(bar, (uint32_t)kTcTileBytes);
    tma_box(dst, map, 0, (int)key0, bar);
    tma_box(dst + kTcBoxBytes, map, kTcBoxDims, (int)key0, bar);
}

// Maximum (MAX = true) or sum over the warp of each of the first N values (N =
// 4, 8 or 16): a reduce-scatter over the top log2(N) lane bits (lane bit 16 >> s
// decides which half of the remaining values a lane keeps at stage s), then
// butterflies over the other lane bits.  Lane l ends with the result for value
// index reduced_index<N>(l), which is returned.
template <int N, bool MAX>
__device__ __forceinline__ float warp_reduce(const float (&v)[16]) {
    float a[N];
#pragma unroll
    for (int i = 0; i < N; i++) a[i] = v[i];
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = N / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < half; i++) {
            const float send = up ? a[i] : a[i + half];
            const float keep = up ? a[i + half] : a[i];
            const float other = __shfl_xor_sync(0xffffffffu, send, bit);
            a[i] = MAX ? fmaxf(keep, other) : keep + other;
        }
    }
#pragma unroll
    for (int bit = 32 / N / 2; bit >= 1; bit >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, a[0], bit);
        a[0] = MAX ? fmaxf(a[0], o) : a[0] + o;
    }
    return a[0];
}

template <int N>
__device__ __forceinline__ int reduced_index(int lane) {
    int idx = 0;
#pragma unroll
    for (int half = N / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1)
        if (lane & bit) idx += half;
    return idx;
}

// Waits on bar[st] for the parity in bit st of ph (then flips that bit); false,
// with the abort flag and TRI_FLAG_STAGE_TIMEOUT set, if the wait ran out.
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t &ph, int st, volatile uint32_t *abort_flag,
                                        unsigned *flags) {
    const bool ok = mbar_wait(bar + st, (ph >> st) & 1u);
    ph ^= 1u << st;
    if (!ok) {
        *abort_flag = 1u;
        atomicOr(flags, TRI_FLAG_STAGE_TIMEOUT);
    }
    return ok;
}

// The QK product of a tile (one thread): K stage ks against Q, into TMEM
// columns t_s, once the stage's copy has landed (bar_k[ks]); completion
// arrives on bar_s[sb].
__device__ __forceinline__ void tc_issue_qk(int ks, int sb, uint32_t sm_base, uint32_t t_s, uint64_t *bar_k,
                                            uint64_t *bar_s, uint32_t &ph_k, volatile uint32_t *abort_flag,
                                            unsigned *flags) {
    if (!tc_wait(bar_k, ph_k, ks, abort_flag, flags)) return;
    tc_fence_after();
    const uint32_t kb = sm_base + kSmK + ks * kTcTileBytes;
#pragma unroll
    for (int k = 0; k < kTcD / 16; k++) {
        const uint64_t a = smem_desc(kb + (k >> 2) * kTcBoxBytes + (k & 3) * 32, 16, 1024, 2);
        const uint64_t b = smem_desc(sm_base + kSmQ + k * 256, 128, 2048, 0);
        mma_bf16(t_s, a, b, kIdescQK, k > 0);
    }
    mma_commit(&bar_s[sb]);
}

}  // namespace

// GQ: the query columns the softmax works on (4, 8 or 16; G <= GQ).  The MMAs
// always run 16 columns; P rows GQ..15 stay zero.
template <int GQ>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_partial_tc(const AttnParams p, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV) {
    extern __shared__ unsigned char smraw[];
    unsigned char *sm = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
    uint64_t *bar_k = reinterpret_cast<uint64_t *>(sm + kSmBar);  // K tile landed [kTcStages]
    uint64_t *bar_v = bar_k + kTcStages;                            // V tile landed [kTcStages]
    uint64_t *bar_s = bar_v + kTcStages;                            // QK product done [2]
    uint64_t *bar_o = bar_s + 2;                                    // PV product done [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kSmTmem);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + kSmAbort);
    float *red = reinterpret_cast<float *>(sm + kSmRed);  // [16][4]
    const Geometry &geo = p.geo;
    const int G = geo.G;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;

    if (t == 0) {
        for (int i = 0; i < 2 * kTcStages + 4; i++) mbar_init(&bar_k[i], 1);
        mbar_init_fence();
        *abort_flag = 0u;
    }
    // P rows of the padded queries are read by the PV products and must be zero.
    for (int e = t; e < 4 * kPBytes / 16; e += kTcThreads)
        reinterpret_cast<uint4 *>(sm + kSmP)[e] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTcTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    // TMEM columns: S of stage st at tbase + 16 st, O of stage st at tbase + 32 + 16 st.
#define t_s(st) (tbase + 16u * (uint32_t)(st))
#define t_o(st) (tbase + 32u + 16u * (uint32_t)(st))
    // Parities of the next phase to wait for: bit st of each word, per barrier pair
    // (thread 0 alone waits on bar_k).
    uint32_t ph_k = 0u, ph_v = 0u, ph_s = 0u, ph_o = 0u;
    const uint32_t sm_base = smem_u32(sm);
    const int64_t n_items = (int64_t)geo.L * geo.S * geo.H * p.chunks;

    for (int64_t item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x) {
        const int64_t r = item / p.chunks;
        const int c = (int)(item % p.chunks);
        const int h = (int)(r % geo.H);
        const int s = (int)((r / geo.H) % geo.S);
        const int l = (int)(r / ((int64_t)geo.H * geo.S));
        int64_t lo = geo.row_off[r], hi = geo.row_off[r + 1];
        if (lo < 0 || hi < lo || hi > geo.total) {
            if (t == 0 && c == 0) atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
            lo = hi = 0;
        }
        const int64_t n = hi - lo;
        const int64_t beg = n * c / p.chunks, end = n * (c + 1) / p.chunks;
        const int ntiles = (int)((end - beg + kTcKeys - 1) / kTcKeys);

        // Q into the B-operand layout: thread t takes query t/8, dims 16 (t%8) .. +15.
        {
            const int q = t >> 3, d0 = (t & 7) * 16;
            uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
            if (q < G) {
                const uint16_t *qrow = p.q + ((((int64_t)l * geo.S + s) * geo.Hq + (int64_t)h * G + q) * kTcD + d0);
                uint32_t x[8];  // the queries are only 2-byte aligned
#pragma unroll
                for (int i = 0; i < 8; i++) x[i] = (uint32_t)qrow[2 * i] | ((uint32_t)qrow[2 * i + 1] << 16);
                a = make_uint4(x[0], x[1], x[2], x[3]);
                b = make_uint4(x[4], x[5], x[6], x[7]);
            }
            *reinterpret_cast<uint4 *>(sm + kSmQ + b_core_offset(q, d0)) = a;
            *reinterpret_cast<uint4 *>(sm + kSmQ + b_core_offset(q, d0 + 8)) = b;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        float o_acc[16], l_part[16], m_run[16], alpha_prev[16];
#pragma unroll
        for (int i = 0; i < 16; i++) {
            o_acc[i] = 0.f;
            l_part[i] = 0.f;
            m_run[i] = -INFINITY;
            alpha_prev[i] = 1.f;
        }
        const int64_t key0 = lo + beg;

        // Prologue: K and V of tiles 0 and 1, then the QK product of tile 0.
        if (t == 0 && ntiles > 0) {
            for (int j = 0; j < kTcStages && j < ntiles; j++) {
                tma_tile(sm + kSmK + j * kTcTileBytes, &tmK, key0 + (int64_t)j * kTcKeys, &bar_k[j]);
                tma_tile(sm + kSmV + j * kTcTileBytes, &tmV, key0 + (int64_t)j * kTcKeys, &bar_v[j]);
            }
        }

        if (t == 0 && ntiles > 0) tc_issue_qk(0, 0, sm_base, t_s(0), bar_k, bar_s, ph_k, abort_flag, p.flags);

        for (int i = 0; i < ntiles; i++) {
            const int st = i & 1;          // S, O and P buffers
            const int ks = i % kTcStages;  // K and V stages
            if (t == 0 && i + 1 < ntiles)
                tc_issue_qk((i + 1) % kTcStages, (i + 1) & 1, sm_base, t_s((i + 1) & 1), bar_k, bar_s, ph_k,
                            abort_flag, p.flags);
            // ---- scores of tile i
            tc_wait(bar_s, ph_s, st, abort_flag, p.flags);
            tc_fence_after();
            if (t == 0 && i + kTcStages < ntiles)  // K stage ks is free once the QK product of tile i is done
                tma_tile(sm + kSmK + ks * kTcTileBytes, &tmK, key0 + (int64_t)(i + kTcStages) * kTcKeys, &bar_k[ks]);
            float x[16];
            tmem_ld16(t_s(st) + lane_off, x);
            const int64_t tile_beg = beg + (int64_t)i * kTcKeys;
            const int valid = (int)std::min<int64_t>(kTcKeys, end - tile_beg);
#pragma unroll
            for (int q = 0; q < GQ; q++) x[q] = t < valid ? x[q] * p.scale_log2 : -INFINITY;
            // V of tile i has landed; the rows past the slice's end are zeroed (a
            // zero weight times whatever the box read there must give zero).
            tc_wait(bar_v, ph_v, ks, abort_flag, p.flags);
            if (valid < kTcKeys && t >= valid) {
                unsigned char *vrow = sm + kSmV + ks * kTcTileBytes + t * 128;
#pragma unroll
                for (int b = 0; b < 2; b++)
#pragma unroll
                    for (int k = 0; k < 8; k++)
                        *reinterpret_cast<uint4 *>(vrow + b * kTcBoxBytes + 16 * k) = make_uint4(0u, 0u, 0u, 0u);
            }
            // tile maximum of every query over the 128 keys
            {
                const float wm = warp_reduce<GQ, true>(x);
                if ((lane & (32 / GQ - 1)) == 0) red[reduced_index<GQ>(lane) * 4 + warp] = wm;
            }
            __syncthreads();
            float pw[16];
#pragma unroll
            for (int q = 0; q < GQ; q++) {
                const float4 mv = *reinterpret_cast<const float4 *>(red + q * 4);
                const float tm = fmaxf(fmaxf(mv.x, mv.y), fmaxf(mv.z, mv.w));
                const float mn = fmaxf(m_run[q], tm);
                const float a = mn == -INFINITY ? 1.f : exp2f(m_run[q] - mn);
                pw[q] = mn == -INFINITY ? 0.f : exp2f(x[q] - mn);
                l_part[q] = fmaf(l_part[q], a, pw[q]);
                m_run[q] = mn;
                x[q] = a;  // this tile's rescale factor, kept for its output
            }
            // P^T of tile i as bf16 hi + lo parts (B operands [16 queries][128 keys]).
            unsigned char *ph = sm + kSmP + (2 * st) * kPBytes;
            unsigned char *pl = ph + kPBytes;
#pragma unroll
            for (int q = 0; q < GQ; q++) {
                const __nv_bfloat16 hb = __float2bfloat16_rn(pw[q]);
                const __nv_bfloat16 lb = __float2bfloat16_rn(pw[q] - __bfloat162float(hb));
                *reinterpret_cast<__nv_bfloat16 *>(ph + b_core_offset(q, t, kPLbo, kPSbo)) = hb;
                *reinterpret_cast<__nv_bfloat16 *>(pl + b_core_offset(q, t, kPLbo, kPSbo)) = lb;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            // Leaving is decided here, by the whole block at once: a wait that ran out
            // anywhere before (its thread set the flag) ends the item for every thread.
            if (__syncthreads_or(*abort_flag)) break;
            tc_fence_after();
            // ---- PV product of tile i into O[st] (fresh), hi then lo weights
            if (t == 0) {
                const uint32_t vb = sm_base + kSmV + ks * kTcTileBytes;
                const uint32_t pb = sm_base + kSmP + (2 * st) * kPBytes;
#pragma unroll
                for (int part = 0; part < 2; part++)
#pragma unroll
                    for (int k = 0; k < kTcKeys / 16; k++) {
                        const uint64_t a = smem_desc(vb + k * 2048, kTcBoxBytes, 1024, 2);
                        const uint64_t b = smem_desc(pb + part * kPBytes + k * 2 * kPLbo, kPLbo, kPSbo, 0);
                        mma_bf16(t_o(st), a, b, kIdescPV, part > 0 || k > 0);
                    }
                mma_commit(&bar_o[st]);
            }
            // ---- output of tile i-1 (its PV product ran while this tile's scores were formed)
            if (i >= 1) {
                const int sp = st ^ 1;
                tc_wait(bar_o, ph_o, sp, abort_flag, p.flags);
                tc_fence_after();
                // V stage (i-1) % kTcStages is free once the PV product of tile i-1 is
                // done: it takes the tile kTcStages - 1 ahead of this one.
                const int vs = (i - 1) % kTcStages;
                if (t == 0 && i - 1 + kTcStages < ntiles)
                    tma_tile(sm + kSmV + vs * kTcTileBytes, &tmV, key0 + (int64_t)(i - 1 + kTcStages) * kTcKeys,
                             &bar_v[vs]);
                float ot[16];
                tmem_ld16(t_o(sp) + lane_off, ot);
#pragma unroll
                for (int q = 0; q < GQ; q++) o_acc[q] = fmaf(o_acc[q], alpha_prev[q], ot[q]);
            }
#pragma unroll
            for (int q = 0; q < GQ; q++) alpha_prev[q] = x[q];
            tc_fence_before();
        }
        if (__syncthreads_or(*abort_flag)) break;
        // ---- the last tile's output, then (O, m, l) of queries < G
        if (ntiles > 0) {
            const int sp = (ntiles - 1) & 1;
            tc_wait(bar_o, ph_o, sp, abort_flag, p.flags);
            tc_fence_after();
            float ot[16];
            tmem_ld16(t_o(sp) + lane_off, ot);
#pragma unroll
            for (int q = 0; q < GQ; q++) o_acc[q] = fmaf(o_acc[q], alpha_prev[q], ot[q]);
        }
        {
            const float ws = warp_reduce<GQ, false>(l_part);
            __syncthreads();  // red[] of the last tile maximum has been read
            if ((lane & (32 / GQ - 1)) == 0) red[reduced_index<GQ>(lane) * 4 + warp] = ws;
            __syncthreads();
        }
        float *out = p.part + item * (int64_t)G * (kTcD + 2);
        for (int q = 0; q < G; q++) out[q * (kTcD + 2) + t] = o_acc[q];
        if (t < G) {
            const float4 lv = *reinterpret_cast<const float4 *>(red + t * 4);
            out[t * (kTcD + 2) + kTcD] = m_run[t];
            out[t * (kTcD + 2) + kTcD + 1] = (lv.x + lv.y) + (lv.z + lv.w);
        }
        tc_fence_before();
        __syncthreads();  // red[] and Q are rewritten by the next item
        tc_fence_after();
    }
    // Teardown: after a wait ran out, give every copy and product still in flight
    // one more bounded wait, so nothing lands in memory that is released below.
    if (*abort_flag && t == 0) {
        for (int b = 0; b < kTcStages; b++) {
            mbar_wait(&bar_k[b], (ph_k >> b) & 1u);
            mbar_wait(&bar_v[b], (ph_v >> b) & 1u);
        }
        for (int b = 0; b < 2; b++) {
            mbar_wait(&bar_s[b], (ph_s >> b) & 1u);
            mbar_wait(&bar_o[b], (ph_o >> b) & 1u);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTcTmemCols) : "memory");
#undef t_s
#undef t_o
}

namespace {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// A [total][128] bf16 matrix as 64-dim x 128-key boxes, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int64_t total) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kTcD, (cuuint64_t)total};
    const cuuint64_t strides[1] = {(cuuint64_t)kTcD * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTcBoxDims, (cuuint32_t)kTcKeys};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// The tensor-core path applies to bf16 contiguous caches of head dim 128 with
// G <= 16 and at most 2^31 - 1 keys; returns cudaErrorNotSupported otherwise
// (the caller then takes the other kernels).
cudaError_t launch_attention_tc(const AttnParams &p0, int64_t R, cudaStream_t s) {
    const Geometry &geo = p0.geo;
    if (geo.elem_bytes != 2 || geo.D != kTcD || geo.layout != TRI_KV_CONTIG || geo.G > kTcN || geo.total < 1 ||
        geo.total > 0x7fffffffLL)
        return cudaErrorNotSupported;
    CUtensorMap mk, mv;
    if (!make_map(&mk, p0.K, geo.total) || !make_map(&mv, p0.V, geo.total)) return cudaErrorNotSupported;
    auto kern = geo.G <= 4 ? attn_partial_tc<4> : geo.G <= 8 ? attn_partial_tc<8> : attn_partial_tc<16>;
    static bool attr[3][64] = {{false}};
    int dev = 0;
    cudaGetDevice(&dev);
    const int ki = geo.G <= 4 ? 0 : geo.G <= 8 ? 1 : 2;
    if (!attr[ki][dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmem);
        if (e != cudaSuccess) return e;
        attr[ki][dev & 63] = true;
    }
    // Persistent grid, one CTA per SM; rows cut into slices so that every CTA
    // gets about four items (each slice costs (d + 2) G floats written and read back).
    AttnParams p = p0;
    const int64_t ctas = sm_count();
    p.chunks = (int)std::min<int64_t>(kAttnMaxChunks, std::max<int64_t>(1, (4 * ctas + R - 1) / R));
    const int64_t grid = std::min<int64_t>(ctas, R * p.chunks);
    kern<<<(unsigned)grid, kTcThreads, kTcSmem, s>>>(p, mk, mv);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_attn_combine(p, R, s);
}

}  // namespace tri
