// Per-row top-B selection with a protected recent window ("TriAttention：基于三角
// 函数 KV 压缩的高效长推理", 流程详解 step 4: keep only the most important KV pairs).
//
// Row of N keys, budget B, window W:
//   N <= B: keep every slot;
//   N >  B: keep slots N-W .. N-1, plus the K = B-W best of slots 0 .. M-1
//           (M = N-W) under (score desc, slot desc); emit slots ascending.
//
// One CTA of 512 threads per row, walking the row in 32768-slot chunks (one
// chunk covers rows up to 32K keys).  Scores are compared through
// order-preserving uint32 keys (-0 folded onto +0, NaN lowest).  Streaming
// passes read the scores coalesced (a warp reads 512 contiguous bytes per
// instruction, from L2 while the scores are resident there):
//  0. the value range of an evenly spaced 1024-slot sample, widened by 1/16 of
//     its span on each side;
//  1. a monotone map of every score to one of 2048 bins - linear in value over
//     that range and clamped at both ends (NaN to the lowest bin, as it ranks
//     lowest), or, when the sample is constant or non-finite, the adaptive
//     key-space map (u - min) >> shift over the row's key range - is
//     histogrammed; one block scan finds the bin b* holding the K-th best
//     score.  Any monotone map keeps the search exact: higher bins are kept
//     whole, lower bins dropped whole; the spread only decides how many keys
//     share b*;
//  2. each chunk's keep-bitmap (1 bit per slot, shared memory) gets the slots
//     of higher bins, assembled with warp shuffles, and b*'s members (a few
//     dozen at the workloads' score spreads) are gathered;
//  3. the members are ranked exactly by (key desc, slot desc) by counting, and
//     the best ones needed set their bits;
//  4. the kept slots are emitted ascending from the bitmap: one block scan of
//     per-thread popcounts gives every thread its output offset.
// A crowded b* (many ties, outliers, constant rows) instead narrows in key
// space with further 2048-bin passes over its members to the single key value
// thr of the K-th best, then an in-order pass with one block scan of packed
// (greater, equal) counts marks the keys above thr and the most recent ties.
// Blocks never wait on other blocks.
#include "tri_internal.cuh"

namespace tri {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kItems = 64;  // slots per thread per chunk
constexpr int64_t kChunk = (int64_t)kSelThreads * kItems;
constexpr int kWords = (int)(kChunk / 32);  // bitmap words per chunk
constexpr int kBins = 2048;
constexpr int kBinsPerThread = kBins / kSelThreads;
constexpr int kCandMax = kSelThreads / 4;  // members of b* resolved by counting

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
        T a = red_min[threadIdx.x < kSelWarps ? threadIdx.x : 0];
        T b = red_max[threadIdx.x < kSelWarps ? threadIdx.x : 0];
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

// Monotone map of a score to one of kBins bins (uniform over the row).
struct BinMap {
    int by_value;  // 1: linear in value from vmin; 0: key space from lo
    float vmin, scale;
    uint32_t lo;
    int shift;
    __device__ __forceinline__ int operator()(float s) const {
        // Clamped at both ends: values outside [vmin, vmin + kBins/scale) go to
        // the end bins and NaN (fmaxf returns the non-NaN operand) to bin 0, where
        // it ranks lowest; subtract, multiply and clamps all keep the order.
        // Adding 2^23 to a value in [0, 2047] rounds it to an integer held in the
        // low mantissa bits: a monotone float-to-bin step on the FMA/ALU pipes.
        if (by_value)
            return __float_as_int(fminf(fmaxf((s - vmin) * scale, 0.f), (float)(kBins - 1)) + 8388608.f) -
                   0x4B000000;
        return (int)((order_key(s) - lo) >> shift);
    }
};

// Number of slots of the chunk starting at c0 (at most kChunk).
__device__ __forceinline__ int chunk_len(int64_t M, int64_t c0) {
    const int64_t rem = M - c0;
    return rem >= kChunk ? (int)kChunk : (int)rem;
}

// Calls fn(j, score) for every slot j < n of the chunk at `base`, coalesced:
// 16-byte vector v = k*512 + t covers slots 4v .. 4v+3 (4-byte loads of slot
// k*512 + t when the row is not 16-byte aligned).
template <typename Fn>
__device__ __forceinline__ void for_each_score(const float *base, int n, bool vec, Fn &&fn) {
    const int t = threadIdx.x;
    if (vec) {
        const float4 *q = reinterpret_cast<const float4 *>(base);
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
        if (j < n) fn(j, __ldg(base + j));
    } else {
#pragma unroll 4
        for (int k = 0; k < kItems; k++) {
            const int j = k * kSelThreads + t;
            if (j < n) fn(j, __ldg(base + j));
        }
    }
}

// Writes the chunk's bitmap words with bit j = pred(j, score of slot j), j < n
// (bits past n are 0).  Every word is written once, without atomics: in the
// vector layout lane l holds slots 4l .. 4l+3 of its warp's 128-slot span, so
// the 8 lanes of a word OR their nibbles together with shuffles.
template <typename Pred>
__device__ __forceinline__ void build_bitmap(const float *base, int n, bool vec, uint32_t *bm_words, Pred &&pred) {
    const int t = threadIdx.x, lane = t & 31;
    if (vec) {
        const float4 *q = reinterpret_cast<const float4 *>(base);
#pragma unroll 4
        for (int k = 0; k < kItems / 4; k++) {
            const int v = k * kSelThreads + t;
            uint32_t nib = 0;
            if (4 * v + 3 < n) {
                const float4 x = __ldg(q + v);
                nib = (uint32_t)pred(4 * v, x.x) | ((uint32_t)pred(4 * v + 1, x.y) << 1) |
                      ((uint32_t)pred(4 * v + 2, x.z) << 2) | ((uint32_t)pred(4 * v + 3, x.w) << 3);
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++)
                    if (4 * v + i < n) nib |= (uint32_t)pred(4 * v + i, __ldg(base + 4 * v + i)) << i;
            }
            uint32_t w = nib << (4 * (lane & 7));
            w |= __shfl_xor_sync(0xffffffffu, w, 1);
            w |= __shfl_xor_sync(0xffffffffu, w, 2);
            w |= __shfl_xor_sync(0xffffffffu, w, 4);
            if ((lane & 7) == 0) bm_words[(4 * v) >> 5] = w;
        }
    } else {
#pragma unroll 4
        for (int k = 0; k < kItems; k++) {
            const int j = k * kSelThreads + t;
            const uint32_t w = __ballot_sync(0xffffffffu, j < n && pred(j, __ldg(base + j)));
            if (lane == 0) bm_words[j >> 5] = w;
        }
    }
}

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

// Emits the set bits of a chunk's bitmap as ascending slots c0 + j into
// out[*base ...] (positions >= K are never written).
__device__ __forceinline__ void emit_bitmap(const uint32_t *bm_words, int64_t c0, int32_t *out, uint32_t K,
                                            uint32_t &base, uint32_t *scan_sm) {
    const int t = threadIdx.x;
    const uint32_t w0 = bm_words[2 * t], w1 = bm_words[2 * t + 1];
    uint32_t tot;
    uint32_t o = base + block_exclusive_scan((uint32_t)(__popc(w0) + __popc(w1)), scan_sm, &tot);
    unsigned long long bits = ((unsigned long long)w1 << 32) | w0;
    while (bits) {
        const int e = __ffsll((long long)bits) - 1;
        bits &= bits - 1;
        if (o < K) out[o] = (int32_t)(c0 + 64 * t + e);
        o++;
    }
    base += tot;
}

__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(const SelectParams p) {
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t bmw[kWords];  // keep-bitmap of the current chunk
    __shared__ uint32_t scan_sm[kSelWarps];
    __shared__ uint32_t red_a[kSelWarps], red_b[kSelWarps];
    __shared__ float red_fa[kSelWarps], red_fb[kSelWarps];
    __shared__ uint32_t cand_key[kCandMax];
    __shared__ int64_t cand_slot[kCandMax];
    __shared__ uint8_t cand_keep[kCandMax];
    __shared__ uint32_t sh_bin, sh_above, sh_count;

    grid_dependency_wait();
    grid_dependents_launch();
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
    }

    // Value range of an evenly spaced 1024-slot sample of the row, widened by
    // 1/16 of its span on each side (two 4-byte loads per thread).
    float fmn = INFINITY, fmx = -INFINITY;
    int snan = 0;
#pragma unroll
    for (int k = 0; k < 2; k++) {
        const int64_t j = ((int64_t)(2 * tid + k) * M) / (2 * kSelThreads);  // < M
        const float s = __ldg(sc + j);
        fmn = fminf(fmn, s);
        fmx = fmaxf(fmx, s);
        snan |= s != s;
    }
    const int any_snan = __syncthreads_or(snan);
    block_minmax(fmn, fmx, red_fa, red_fb);

    BinMap bm;
    const float vspan = fmx - fmn;
    const float vlo = fmn - 0.0625f * vspan, vhi = fmx + 0.0625f * vspan;
    bm.vmin = vlo;
    bm.scale = vhi > vlo ? (float)kBins / (vhi - vlo) : 0.f;
    bm.by_value = !any_snan && isfinite(vspan) && vspan > 0.f && isfinite(vlo) && isfinite(vhi) &&
                  isfinite(bm.scale) && bm.scale > 0.f;
    uint32_t umx = 0xffffffffu;
    bm.lo = 0u;
    bm.shift = 21;
    if (!bm.by_value) {  // key-space bins over the row's key range
        uint32_t umn = 0xffffffffu;
        umx = 0u;
        for (int c = 0; c < nchunks; c++) {
            const int64_t c0 = (int64_t)c * kChunk;
            for_each_score(sc + c0, chunk_len(M, c0), vec, [&](int, float s) {
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

    // Pass 1: histogram of the bins; b* and the keys above it.
    for (int b = 0; b < kBinsPerThread; b++) hist[tid * kBinsPerThread + b] = 0u;
    __syncthreads();
    int nan = 0;
    for (int c = 0; c < nchunks; c++) {
        const int64_t c0 = (int64_t)c * kChunk;
        for_each_score(sc + c0, chunk_len(M, c0), vec, [&](int, float s) {
            atomicAdd(&hist[bm(s)], 1u);
            nan |= s != s;
        });
    }
    if (__syncthreads_or(nan) && tid == 0) atomicOr(p.flags, TRI_FLAG_NONFINITE);
    uint32_t bin, above;
    find_bin(hist, K, scan_sm, &sh_bin, &sh_above, bin, above);
    const uint32_t need = K - above;  // keys to keep from b*
    const uint32_t cand = hist[bin];  // keys in b*
    const int ibin = (int)bin;
    uint32_t out_base = 0;

    if (cand <= (uint32_t)kCandMax) {
        // Pass 2: gather b*'s members (and, for a one-chunk row, the bitmap of
        // the higher bins on the same read).
        for (int c = 0; c < nchunks; c++) {
            const int64_t c0 = (int64_t)c * kChunk;
            const int n = chunk_len(M, c0);
            if (nchunks == 1) {
                build_bitmap(sc, n, vec, bmw, [&](int j, float s) {
                    const int b = bm(s);
                    if (b == ibin) {
                        const uint32_t i = atomicAdd(&sh_count, 1u);
                        if (i < (uint32_t)kCandMax) {
                            cand_key[i] = order_key(s);
                            cand_slot[i] = j;
                        }
                    }
                    return b > ibin;
                });
            } else {
                for_each_score(sc + c0, n, vec, [&](int j, float s) {
                    if (bm(s) == ibin) {
                        const uint32_t i = atomicAdd(&sh_count, 1u);
                        if (i < (uint32_t)kCandMax) {
                            cand_key[i] = order_key(s);
                            cand_slot[i] = c0 + j;
                        }
                    }
                });
            }
        }
        __syncthreads();
        // Rank each member by (key desc, slot desc), 4 threads per member.
        const int i = tid >> 2, q = tid & 3;
        uint32_t rank = 0;
        uint32_t ui = 0;
        int64_t si = 0;
        if (i < (int)cand) {
            ui = cand_key[i];
            si = cand_slot[i];
            for (int j = q; j < (int)cand; j += 4) {
                const uint32_t uj = cand_key[j];
                rank += (uj > ui) | ((uj == ui) & (cand_slot[j] > si));
            }
        }
        rank += __shfl_xor_sync(0xffffffffu, rank, 1);
        rank += __shfl_xor_sync(0xffffffffu, rank, 2);
        if (i < (int)cand && q == 0) cand_keep[i] = rank < need;
        __syncthreads();
        for (int c = 0; c < nchunks; c++) {
            const int64_t c0 = (int64_t)c * kChunk;
            const int n = chunk_len(M, c0);
            if (nchunks > 1) build_bitmap(sc + c0, n, vec, bmw, [&](int, float s) { return bm(s) > ibin; });
            __syncthreads();
            if (tid < (int)cand && cand_keep[tid] && cand_slot[tid] >= c0 && cand_slot[tid] < c0 + n) {
                const int j = (int)(cand_slot[tid] - c0);
                atomicOr(&bmw[j >> 5], 1u << (j & 31));
            }
            __syncthreads();
            emit_bitmap(bmw, c0, out, K, out_base, scan_sm);
        }
        return;
    }

    // Crowded b*: narrow in key space over its members, whose keys form the
    // contiguous range [lo, hi], to the single key value thr.
    uint32_t lo, hi;
    if (bm.by_value) {
        uint32_t cmn = 0xffffffffu, cmx = 0u;
        for (int c = 0; c < nchunks; c++) {
            const int64_t c0 = (int64_t)c * kChunk;
            for_each_score(sc + c0, chunk_len(M, c0), vec, [&](int, float s) {
                if (bm(s) == ibin) {
                    const uint32_t u = order_key(s);
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
    uint32_t need2 = need, cand2 = cand;
    for (;;) {
        const uint32_t range = hi - lo;
        if (range == 0) break;
        const int nbits = 32 - __clz(range);
        const int shift = nbits > 11 ? nbits - 11 : 0;
        for (int b = 0; b < kBinsPerThread; b++) hist[tid * kBinsPerThread + b] = 0u;
        __syncthreads();
        for (int c = 0; c < nchunks; c++) {
            const int64_t c0 = (int64_t)c * kChunk;
            for_each_score(sc + c0, chunk_len(M, c0), vec, [&](int, float s) {
                if (bm(s) == ibin) {
                    const uint32_t u = order_key(s);
                    if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> shift], 1u);
                }
            });
        }
        __syncthreads();
        uint32_t b2, ab2;
        find_bin(hist, need2, scan_sm, &sh_bin, &sh_above, b2, ab2);
        need2 -= ab2;
        cand2 = hist[b2];
        const uint32_t nlo = lo + (b2 << shift);
        const unsigned long long nhi = (unsigned long long)nlo + ((1ull << shift) - 1ull);
        hi = nhi < (unsigned long long)hi ? (uint32_t)nhi : hi;
        lo = nlo;
        __syncthreads();
        if (shift == 0) break;
    }
    const uint32_t thr = lo;
    const uint32_t tie_skip = cand2 - need2;  // ties at thr in the oldest slots are dropped
    // In slot order (thread t: slots 64t .. 64t+63), mark the keys above thr and
    // the ties whose rank from the oldest is at least tie_skip.
    uint32_t tie_base = 0;
    for (int c = 0; c < nchunks; c++) {
        const int64_t c0 = (int64_t)c * kChunk;
        const int n = chunk_len(M, c0);
        const int j0 = tid * kItems;
        unsigned long long gt_bits = 0, eq_bits = 0;
        for (int e = 0; e < kItems; e++) {
            const int j = j0 + e;
            if (j < n) {
                const float s = __ldg(sc + c0 + j);
                const int b = bm(s);
                if (b > ibin) {
                    gt_bits |= 1ull << e;
                } else if (b == ibin) {
                    const uint32_t u = order_key(s);
                    gt_bits |= (unsigned long long)(u > thr) << e;
                    eq_bits |= (unsigned long long)(u == thr) << e;
                }
            }
        }
        uint32_t tot;
        uint32_t rank = tie_base + block_exclusive_scan((uint32_t)__popcll(eq_bits), scan_sm, &tot);
        unsigned long long keep = gt_bits, eqs = eq_bits;
        while (eqs) {
            const int e = __ffsll((long long)eqs) - 1;
            eqs &= eqs - 1;
            if (rank >= tie_skip) keep |= 1ull << e;
            rank++;
        }
        tie_base += tot;
        bmw[2 * tid] = (uint32_t)keep;
        bmw[2 * tid + 1] = (uint32_t)(keep >> 32);
        __syncthreads();
        emit_bitmap(bmw, c0, out, K, out_base, scan_sm);
    }
}

cudaError_t launch_select(const SelectParams &p, cudaStream_t s) {
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    return launch_pdl(select_kernel, dim3((unsigned)R), dim3(kSelThreads), 0, s, p);
}

}  // namespace tri
