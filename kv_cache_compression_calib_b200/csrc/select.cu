// Per-row top-B selection with a protected recent window ("TriAttention：基于三角
// 函数 KV 压缩的高效长推理", 流程详解 step 4: keep only the most important KV pairs).
//
// Row of N keys, budget B, window W:
//   N <= B: keep every slot;
//   N >  B: keep slots N-W .. N-1, plus the K = B-W best of slots 0 .. M-1
//           (M = N-W) under (score desc, slot desc); emit slots ascending.
//
// One CTA per row.  Scores map to order-preserving uint32 keys.  The K-th
// largest key is found exactly by an adaptive radix search: pass 0 takes the
// row's min/max key; each further pass histograms the candidates' keys
// (u - lo) >> shift into 2048 bins, with shift chosen so the candidates'
// remaining range fills the bins (skipping bits that are constant across the
// row), walks the bins from the top to the one holding the K-th key, and
// narrows to that bin.  It ends when the range is a single key value thr:
// then `above` keys are > thr, and the K - above kept ties at thr are the
// ones in the most recent slots.  A last pass walks the row in slot order:
// one block scan of packed (greater, equal) counts per chunk gives every
// thread both its output offset and its ties' ranks, so the kept slots are
// written ascending with no sort.  All passes re-read the row's scores, which
// stay in L2 between the score kernel and here for rows of moderate length.
// Blocks never wait on other blocks.
#include "tri_internal.cuh"

namespace tri {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 2048;
constexpr int kBinsPerThread = kBins / kSelThreads;  // 4
constexpr int kChunkPerThread = 16;

// Exclusive scan over the block in thread order; *total receives the sum.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *sm, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < kSelWarps ? sm[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kSelWarps) sm[lane] = w;
    }
    __syncthreads();
    const uint32_t base = warp ? sm[warp - 1] : 0u;
    *total = sm[kSelWarps - 1];
    __syncthreads();
    return base + x - v;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelectParams p) {
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t scan_sm[32];
    __shared__ uint32_t red_min[kSelWarps], red_max[kSelWarps];
    __shared__ uint32_t sh_bin, sh_above;
    __shared__ int sh_nan;

    const int tid = threadIdx.x;
    const int r = blockIdx.x;
    const int64_t row_lo = p.geo.row_off[r];
    const int64_t N = p.geo.row_off[r + 1] - row_lo;
    const int32_t B = p.B, W = p.W;
    int32_t *out = p.kept + (int64_t)r * B;
    if (N < 0 || N > 0x7fffffffLL || row_lo < 0 || row_lo + N > p.geo.total) {
        if (tid == 0) {
            atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
            if (p.kept_count) p.kept_count[r] = 0;
        }
        return;
    }
    if (N <= B) {
        for (int64_t i = tid; i < N; i += kSelThreads) out[i] = (int32_t)i;
        if (tid == 0 && p.kept_count) p.kept_count[r] = (int32_t)N;
        return;
    }
    const int64_t M = N - W;
    const uint32_t K = (uint32_t)(B - W);
    for (int i = tid; i < W; i += kSelThreads) out[K + i] = (int32_t)(M + i);
    if (tid == 0 && p.kept_count) p.kept_count[r] = B;
    if (K == 0) return;
    const float *sc = p.scores + row_lo;
    if (tid == 0) {
        sh_bin = 0;
        sh_above = 0;
    }

    // Pass 0: range of keys over the candidate slots.
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    int has_nan = 0;
    for (int64_t i = tid; i < M; i += kSelThreads) {
        const float s = sc[i];
        has_nan |= (s != s);
        const uint32_t u = order_key(s);
        kmin = min(kmin, u);
        kmax = max(kmax, u);
    }
    if (tid == 0) sh_nan = 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if ((tid & 31) == 0) {
        red_min[tid >> 5] = kmin;
        red_max[tid >> 5] = kmax;
    }
    __syncthreads();
    if (has_nan) sh_nan = 1;
    if (tid < 32) {
        uint32_t a = tid < kSelWarps ? red_min[tid] : 0xffffffffu;
        uint32_t b = tid < kSelWarps ? red_max[tid] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
            b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
        }
        if (tid == 0) {
            red_min[0] = a;
            red_max[0] = b;
        }
    }
    __syncthreads();
    uint32_t lo = red_min[0], hi = red_max[0];
    if (tid == 0 && sh_nan) atomicOr(p.flags, TRI_FLAG_NONFINITE);

    // Radix narrowing to the single key value `thr` of the K-th best slot.
    uint32_t need = K;           // still to pick at or below the current range
    uint32_t cand = (uint32_t)M; // keys inside [lo, hi]
    for (;;) {
        const uint32_t range = hi - lo;
        if (range == 0) break;
        const int nbits = 32 - __clz(range);
        const int shift = nbits > 11 ? nbits - 11 : 0;
        for (int i = tid; i < kBins; i += kSelThreads) hist[i] = 0u;
        __syncthreads();
        for (int64_t i = tid; i < M; i += kSelThreads) {
            const uint32_t u = order_key(sc[i]);
            if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> shift], 1u);
        }
        __syncthreads();
        // Thread t owns bins kBins-1-4t .. kBins-4-4t (top first).
        const int top = kBins - 1 - kBinsPerThread * tid;
        uint32_t mine = 0;
#pragma unroll
        for (int b = 0; b < kBinsPerThread; b++) mine += hist[top - b];
        uint32_t tot;
        const uint32_t above_me = block_exclusive_scan(mine, scan_sm, &tot);
        if (above_me < need && above_me + mine >= need) {
            uint32_t c = above_me;
            for (int b = 0; b < kBinsPerThread; b++) {
                const uint32_t hb = hist[top - b];
                if (c + hb >= need) {
                    sh_bin = (uint32_t)(top - b);
                    sh_above = c;
                    break;
                }
                c += hb;
            }
        }
        __syncthreads();
        const uint32_t bin = sh_bin & (kBins - 1);
        need -= sh_above;
        cand = hist[bin];
        const uint32_t nlo = lo + (bin << shift);
        const unsigned long long nhi = (unsigned long long)nlo + ((1ull << shift) - 1ull);
        hi = nhi < (unsigned long long)hi ? (uint32_t)nhi : hi;
        lo = nlo;
        __syncthreads();
        if (shift == 0) break;
    }
    const uint32_t thr = lo;
    const uint32_t tie_skip = cand - need;  // ties at thr in the oldest slots that are dropped

    // Emit kept slots of [0, M) in ascending order.
    uint32_t gt_base = 0, tie_base = 0;
    for (int64_t c0 = 0; c0 < M; c0 += (int64_t)kSelThreads * kChunkPerThread) {
        const int64_t s0 = c0 + (int64_t)tid * kChunkPerThread;
        uint32_t gt_bits = 0, eq_bits = 0;
#pragma unroll
        for (int e = 0; e < kChunkPerThread; e++) {
            const int64_t i = s0 + e;
            if (i < M) {
                const uint32_t u = order_key(sc[i]);
                gt_bits |= (uint32_t)(u > thr) << e;
                eq_bits |= (uint32_t)(u == thr) << e;
            }
        }
        const uint32_t packed = ((uint32_t)__popc(gt_bits) << 16) | (uint32_t)__popc(eq_bits);
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan(packed, scan_sm, &tot);
        uint32_t tie_rank = tie_base + (ex & 0xffffu);
        uint32_t o = gt_base + (ex >> 16) + (tie_rank > tie_skip ? tie_rank - tie_skip : 0u);
#pragma unroll
        for (int e = 0; e < kChunkPerThread; e++) {
            const bool keep = ((gt_bits >> e) & 1u) || (((eq_bits >> e) & 1u) && tie_rank >= tie_skip);
            tie_rank += (eq_bits >> e) & 1u;
            if (keep && o < K) out[o] = (int32_t)(s0 + e);
            o += keep;
        }
        gt_base += tot >> 16;
        tie_base += tot & 0xffffu;
    }
}

cudaError_t launch_select(const SelectParams &p, cudaStream_t s) {
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    select_kernel<<<(unsigned)R, kSelThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tri
