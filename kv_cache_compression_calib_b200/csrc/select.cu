// Per-row top-B selection with a protected recent window ("TriAttention：基于三角
// 函数 KV 压缩的高效长推理", 流程详解 step 4: keep only the most important KV pairs).
//
// Row of N keys, budget B, window W:
//   N <= B: keep every slot;
//   N >  B: keep slots N-W .. N-1, plus the K = B-W best of slots 0 .. M-1
//           (M = N-W) under (score desc, slot desc); emit slots ascending.
//
// One CTA of 512 threads per row, in 32768-slot chunks (one chunk covers rows
// up to 32K keys).  Streaming passes read the scores coalesced (a warp reads
// 512 contiguous bytes per instruction); the passes that must walk slots in
// order give thread t the range 64t .. 64t+63 and read its bins from shared
// memory.  Scores are compared
// through order-preserving uint32 keys (-0 folded onto +0, NaN lowest).
// Exact threshold search:
//  0. one streaming pass takes the row's finite min/max (and whether a NaN or
//     an infinity is present);
//  1. a second pass maps every score to one of 2048 bins by a monotone map -
//     linear in value over [min, max] when all scores are finite, else the
//     adaptive key-space map (u - min) >> shift - keeps the bin index (2 B per
//     slot, shared memory) and histograms it; one block scan finds the bin
//     holding the K-th best score (higher bins outrank it entirely, lower bins
//     are outranked entirely);
//  2. that bin's members (typically a few dozen) are gathered and the K-th
//     best key value thr is found by counting, per candidate, how many others
//     are greater / not smaller; a crowded bin instead narrows in key space
//     with further 2048-bin passes over its members until one value remains;
//  3. a last pass in slot order keeps the higher bins, the bin's keys above
//     thr and the most recent of the ties at thr: one block scan of packed
//     (greater, equal) counts gives every thread its output offset and its
//     ties' ranks, so kept slots are written ascending with no sort.
// Only bin indices live in shared memory (64 KB), so two rows share an SM;
// scores are re-read from global memory (L2) by the streaming passes and by
// the candidate lookups.  Rows longer than one chunk recompute the bins of
// non-resident chunks.  Blocks never wait on other blocks.
#include "tri_internal.cuh"

namespace tri {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kItems = 64;  // slots per thread per chunk
constexpr int64_t kChunk = (int64_t)kSelThreads * kItems;
constexpr int kBins = 2048;
constexpr int kBinsPerThread = kBins / kSelThreads;
constexpr int kCandMax = kSelThreads / 4;  // candidates resolved by counting
constexpr size_t kSelDynSmem = (size_t)kItems * kSelThreads * sizeof(uint16_t);  // 64 KiB

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

template <typename T>
__device__ __forceinline__ void block_minmax(T &mn, T &mx, T *red_min, T *red_max) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    __syncthreads();  // red_* may still be read from a previous use
    if ((threadIdx.x & 31) == 0) {
        red_min[threadIdx.x >> 5] = mn;
        red_max[threadIdx.x >> 5] = mx;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        T a = threadIdx.x < kSelWarps ? red_min[threadIdx.x] : red_min[0];
        T b = threadIdx.x < kSelWarps ? red_max[threadIdx.x] : red_max[0];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
            b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
        }
        __syncwarp();
        if (threadIdx.x == 0) {
            red_min[0] = a;
            red_max[0] = b;
        }
    }
    __syncthreads();
    mn = red_min[0];
    mx = red_max[0];
}

// Calls fn(j, score) for the chunk's valid slots j (relative to c0) in a
// coalesced order: 16-byte vector v = k*512 + t covers slots 4v .. 4v+3, so a
// warp reads 512 contiguous bytes per instruction (4-byte loads, slot
// k*512 + t, when the row is not 16-byte aligned).
template <typename Fn>
__device__ __forceinline__ void for_each_score(const float *sc, int64_t M, int64_t c0, bool vec, Fn &&fn) {
    const int t = threadIdx.x;
    const int64_t rem = M - c0;
    const int n = rem >= kChunk ? (int)kChunk : (int)rem;
    if (vec) {
        const float4 *q = reinterpret_cast<const float4 *>(sc + c0);
        const int nvec = n >> 2;
#pragma unroll 4
        for (int k = 0; k < kItems / 4; k++) {
            const int v = k * kSelThreads + t;
            if (v < nvec) {
                const float4 x = __ldg(q + v);
                fn(4 * v + 0, x.x);
                fn(4 * v + 1, x.y);
                fn(4 * v + 2, x.z);
                fn(4 * v + 3, x.w);
            }
        }
        const int j = 4 * nvec + t;  // ragged tail: at most 3 slots
        if (j < n) fn(j, __ldg(sc + c0 + j));
    } else {
#pragma unroll 4
        for (int k = 0; k < kItems; k++) {
            const int j = k * kSelThreads + t;
            if (j < n) fn(j, __ldg(sc + c0 + j));
        }
    }
}

// Shared-memory position (in uint16 units) of the bin of chunk slot j.  Slot
// j = 64t + e belongs to thread t's range; its 32 words are stored XOR-swizzled
// (word w at w ^ (t mod 32)), so a warp reading word w of each lane's range
// touches 32 distinct banks.
__device__ __forceinline__ int bin_pos(int j) {
    const int t = j >> 6, e = j & 63;
    return (((t << 5) | ((e >> 1) ^ (t & 31))) << 1) | (e & 1);
}

// Number of valid slots of chunk c0 in this thread's range 64t .. 64t+63.
__device__ __forceinline__ int range_count(int64_t M, int64_t c0) {
    const int64_t rem = M - c0 - (int64_t)threadIdx.x * kItems;
    return rem <= 0 ? 0 : (rem >= kItems ? kItems : (int)rem);
}

// Monotone map of a score to one of kBins bins (uniform over the row).
struct BinMap {
    int by_value;  // 1: linear in value from vmin; 0: key space from lo
    float vmin, scale;
    uint32_t lo;
    int shift;
    __device__ __forceinline__ int operator()(float s) const {
        if (by_value) return min((int)((s - vmin) * scale), kBins - 1);
        return (int)((order_key(s) - lo) >> shift);
    }
};

// After a histogram pass: the bin (top first) holding the need-th best key and
// the number of keys in higher bins.
__device__ __forceinline__ void find_bin(const uint32_t *hist, uint32_t need, uint32_t *scan_sm, uint32_t *sh_bin,
                                         uint32_t *sh_above, uint32_t &bin, uint32_t &above) {
    const int top = kBins - 1 - kBinsPerThread * threadIdx.x;
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
                *sh_bin = (uint32_t)(top - b);
                *sh_above = c;
                break;
            }
            c += hb;
        }
    }
    __syncthreads();
    bin = *sh_bin & (kBins - 1);
    above = *sh_above;
}

__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(const SelectParams p) {
    extern __shared__ __align__(16) uint16_t bins[];  // [kChunk], bin of each slot of the resident chunk
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t scan_sm[kSelWarps];
    __shared__ uint32_t red_a[kSelWarps], red_b[kSelWarps];
    __shared__ float red_fa[kSelWarps], red_fb[kSelWarps];
    __shared__ uint32_t cand_key[kCandMax];
    __shared__ uint32_t sh_bin, sh_above, sh_count, sh_thr, sh_ge;

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
    const bool vec = (((uintptr_t)sc) & 15) == 0;
    const int nchunks = (int)((M + kChunk - 1) / kChunk);
    if (tid == 0) {
        sh_bin = 0;
        sh_above = 0;
        sh_count = 0;
        sh_thr = 0;
        sh_ge = 0;
    }

    // Pass 0: finite value range; NaN / infinity present.
    float fmn = INFINITY, fmx = -INFINITY;
    int nan = 0, inf = 0;
    for (int c = 0; c < nchunks; c++) {
        for_each_score(sc, M, (int64_t)c * kChunk, vec, [&](int, float s) {
            fmn = fminf(fmn, s);
            fmx = fmaxf(fmx, s);
            nan |= s != s;
            inf |= fabsf(s) == INFINITY;
        });
    }
    if (__syncthreads_or(nan) && tid == 0) atomicOr(p.flags, TRI_FLAG_NONFINITE);
    const int any_nonfinite = __syncthreads_or(nan | inf);
    block_minmax(fmn, fmx, red_fa, red_fb);

    BinMap bm;
    bm.vmin = fmn;
    const float vspan = fmx - fmn;
    bm.scale = vspan > 0.f ? (float)kBins / vspan : 0.f;
    bm.by_value = !any_nonfinite && isfinite(vspan) && vspan > 0.f && isfinite(bm.scale);
    uint32_t umn = 0u, umx = 0xffffffffu;
    bm.lo = 0u;
    bm.shift = 21;
    if (!bm.by_value) {
        // key-space bins over the row's key range
        umn = 0xffffffffu;
        umx = 0u;
        for (int c = 0; c < nchunks; c++) {
            for_each_score(sc, M, (int64_t)c * kChunk, vec, [&](int, float s) {
                const uint32_t u = order_key(s);
                umn = min(umn, u);
                umx = max(umx, u);
            });
        }
        block_minmax(umn, umx, red_a, red_b);
        const uint32_t range = umx - umn;
        const int nbits = range ? 32 - __clz(range) : 0;
        bm.lo = umn;
        bm.shift = nbits > 11 ? nbits - 11 : 0;
    }

    // Pass 1: bin every score (kept in shared memory) and histogram the bins.
    for (int b = 0; b < kBinsPerThread; b++) hist[tid * kBinsPerThread + b] = 0u;
    __syncthreads();
    int resident = 0;
    for (int c = 0; c < nchunks; c++) {
        __syncthreads();  // bins of the previous chunk are no longer read
        for_each_score(sc, M, (int64_t)c * kChunk, vec, [&](int j, float s) {
            const int b = bm(s);
            bins[bin_pos(j)] = (uint16_t)b;
            atomicAdd(&hist[b], 1u);
        });
        resident = c;
    }
    __syncthreads();
    uint32_t bin, above;
    find_bin(hist, K, scan_sm, &sh_bin, &sh_above, bin, above);
    uint32_t need = K - above;  // keys still to keep from `bin`
    uint32_t cand = hist[bin];  // keys in `bin`
    uint32_t thr, tie_skip;

    // Make chunk c's bins resident (recomputed from the scores if needed); nv is
    // then this thread's count in its slot range 64t .. 64t+63 of the chunk.
    int nv = range_count(M, (int64_t)resident * kChunk);
    auto ensure = [&](int c) {
        if (c != resident) {
            __syncthreads();
            for_each_score(sc, M, (int64_t)c * kChunk, vec, [&](int j, float s) { bins[bin_pos(j)] = (uint16_t)bm(s); });
            __syncthreads();
            resident = c;
        }
        nv = range_count(M, (int64_t)c * kChunk);
    };

    // Calls fn(e, bin) for this thread's valid range slots 64t + e, e < nv.
    const uint32_t *bins32 = reinterpret_cast<const uint32_t *>(bins);
    auto for_range = [&](auto &&fn) {
#pragma unroll 4
        for (int w = 0; w < kItems / 2; w++) {
            if (2 * w < nv) {
                const uint32_t pair = bins32[(tid << 5) | (w ^ (tid & 31))];
                fn(2 * w, pair & 0xffffu);
                if (2 * w + 1 < nv) fn(2 * w + 1, pair >> 16);
            }
        }
    };

    if (cand <= (uint32_t)kCandMax) {
        // Gather the bin's keys; the need-th largest is thr.
        for (int k = 0; k < nchunks; k++) {
            const int c = (resident + k) % nchunks;
            ensure(c);
            const int64_t s0 = (int64_t)c * kChunk + (int64_t)tid * kItems;
            for_range([&](int e, uint32_t b) {
                if (b == bin) {
                    const uint32_t slot = atomicAdd(&sh_count, 1u);
                    if (slot < (uint32_t)kCandMax) cand_key[slot] = order_key(__ldg(sc + s0 + e));
                }
            });
        }
        __syncthreads();
        // 4 threads per candidate count the candidates greater / not smaller.
        const int i = tid >> 2, q = tid & 3;
        uint32_t gt = 0, ge = 0, ui = 0;
        if (i < (int)cand) {
            ui = cand_key[i];
            for (int j = q; j < (int)cand; j += 4) {
                const uint32_t uj = cand_key[j];
                gt += uj > ui;
                ge += uj >= ui;
            }
        }
        gt += __shfl_xor_sync(0xffffffffu, gt, 1);
        gt += __shfl_xor_sync(0xffffffffu, gt, 2);
        ge += __shfl_xor_sync(0xffffffffu, ge, 1);
        ge += __shfl_xor_sync(0xffffffffu, ge, 2);
        if (i < (int)cand && q == 0 && gt < need && ge >= need) {
            sh_thr = ui;  // every such candidate holds the same key value
            sh_ge = ge;
        }
        __syncthreads();
        thr = sh_thr;
        tie_skip = sh_ge - need;
    } else {
        // Crowded bin: narrow in key space over its members, whose keys form the
        // contiguous range [lo, hi].
        uint32_t lo, hi;
        if (bm.by_value) {
            uint32_t cmn = 0xffffffffu, cmx = 0u;
            for (int k = 0; k < nchunks; k++) {
                const int c = (resident + k) % nchunks;
                ensure(c);
                const int64_t s0 = (int64_t)c * kChunk + (int64_t)tid * kItems;
                for_range([&](int e, uint32_t b) {
                    if (b == bin) {
                        const uint32_t u = order_key(__ldg(sc + s0 + e));
                        cmn = min(cmn, u);
                        cmx = max(cmx, u);
                    }
                });
            }
            block_minmax(cmn, cmx, red_a, red_b);
            lo = cmn;
            hi = cmx;
        } else {
            lo = bm.lo + (bin << bm.shift);
            const unsigned long long h = (unsigned long long)lo + ((1ull << bm.shift) - 1ull);
            hi = h < (unsigned long long)umx ? (uint32_t)h : umx;
        }
        for (;;) {
            const uint32_t range = hi - lo;
            if (range == 0) break;
            const int nbits = 32 - __clz(range);
            const int shift = nbits > 11 ? nbits - 11 : 0;
            for (int b = 0; b < kBinsPerThread; b++) hist[tid * kBinsPerThread + b] = 0u;
            __syncthreads();
            for (int k = 0; k < nchunks; k++) {
                const int c = (resident + k) % nchunks;
                ensure(c);
                const int64_t s0 = (int64_t)c * kChunk + (int64_t)tid * kItems;
                for_range([&](int e, uint32_t b) {
                    if (b == bin) {
                        const uint32_t u = order_key(__ldg(sc + s0 + e));
                        if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> shift], 1u);
                    }
                });
            }
            __syncthreads();
            uint32_t b2, ab2;
            find_bin(hist, need, scan_sm, &sh_bin, &sh_above, b2, ab2);
            need -= ab2;
            cand = hist[b2];
            const uint32_t nlo = lo + (b2 << shift);
            const unsigned long long nhi = (unsigned long long)nlo + ((1ull << shift) - 1ull);
            hi = nhi < (unsigned long long)hi ? (uint32_t)nhi : hi;
            lo = nlo;
            __syncthreads();
            if (shift == 0) break;
        }
        thr = lo;
        tie_skip = cand - need;
    }

    // Last pass: emit kept slots of [0, M) in ascending order, chunk by chunk.
    uint32_t gt_base = 0, tie_base = 0;
    for (int c = 0; c < nchunks; c++) {
        ensure(c);
        const int64_t s0 = (int64_t)c * kChunk + (int64_t)tid * kItems;
        unsigned long long gt_bits = 0, eq_bits = 0;
        for_range([&](int e, uint32_t b) {
            if (b > bin) {
                gt_bits |= 1ull << e;
            } else if (b == bin) {
                const uint32_t u = order_key(__ldg(sc + s0 + e));
                gt_bits |= (unsigned long long)(u > thr) << e;
                eq_bits |= (unsigned long long)(u == thr) << e;
            }
        });
        const uint32_t packed = ((uint32_t)__popcll(gt_bits) << 16) | (uint32_t)__popcll(eq_bits);
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan(packed, scan_sm, &tot);
        uint32_t tie_rank = tie_base + (ex & 0xffffu);
        uint32_t o = gt_base + (ex >> 16) + (tie_rank > tie_skip ? tie_rank - tie_skip : 0u);
        unsigned long long any = gt_bits | eq_bits;
        while (any) {
            const int e = __ffsll((long long)any) - 1;
            any &= any - 1;
            const bool eq = (eq_bits >> e) & 1ull;
            const bool keep = !eq || tie_rank >= tie_skip;
            tie_rank += eq;
            if (keep) {
                if (o < K) out[o] = (int32_t)(s0 + e);
                o++;
            }
        }
        gt_base += tot >> 16;
        tie_base += tot & 0xffffu;
    }
}

cudaError_t launch_select(const SelectParams &p, cudaStream_t s) {
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    static bool configured[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSelDynSmem);
        if (e != cudaSuccess) return e;
        configured[dev & 63] = true;
    }
    select_kernel<<<(unsigned)R, kSelThreads, kSelDynSmem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tri
