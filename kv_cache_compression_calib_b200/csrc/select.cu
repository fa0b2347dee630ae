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
#include "gather_chunk.cuh"

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

// All kept records of row r (cnt of them), moved by the whole CTA in chunks of
// GatherChunk<RB, kSelThreads, 2>::kSlots slots (two K and two V vectors in flight per
// thread: 64 KB per SM with two CTAs, within the select path's registers).
template <int RB>
__device__ __forceinline__ void gather_row(const GatherParams &g, int64_t r, int64_t row_lo, int64_t N, int cnt,
                                           unsigned char *stage) {
    GatherStaged<RB, kSelThreads, 3>::copy(g, r, row_lo, N, cnt, stage);
}

// ------------------------------------------------------------------ one pass
//
// Rows of more than one chunk and at most kOpMaxRow candidate slots first try
// a single streaming pass (the general passes re-read a multi-chunk row, whose
// scores no longer sit in L2, three times).  The value range of a sample (512 runs of 8 consecutive slots, evenly
// spaced) sets the same clamped linear 2048-bin map as above; the sample's own
// histogram gives a band of bins [b_lo, b_hi] that holds the K-th best key
// unless the sample misleads by more than kOpZ standard deviations of a
// binomial count (bins above b_hi hold fewer than pS - kOpZ sd sampled keys,
// bins from b_lo up more than pS + kOpZ sd, p = K/M, S = 4096).  One pass over
// the row then sets the keep-bit of every key above the band (bitmap words
// assembled with shuffles, each written once) and appends the band's keys and
// slots to a shared-memory list (one warp scan per 16 slots a thread reads);
// the band is held as two fp32 values, so a slot costs three comparisons.  If the band did hold the
// K-th best key (A keys above it, A <= K <= A + C with the C band keys all
// held), the rest runs on chip: radix narrowing of the C keys to the exact
// threshold key thr, keep-bits for keys above thr, tie-bits for keys equal to
// it, the most recent ties chosen by a block scan in slot order, and the kept
// slots emitted ascending by a block scan of the keep words.  Otherwise nothing
// has been written and the general passes run.  The result is identical
// either way: the band only decides which keys are resolved on chip.
constexpr int kOpRuns = kSelThreads;             // sample runs, one per thread
constexpr int kOpRun = 8;                        // consecutive slots per run
constexpr int kOpSample = kOpRuns * kOpRun;      // 4096 sampled slots
constexpr int64_t kOpMinRow = kChunk + 1;        // one-chunk rows: the general passes (from L2, cheaper)
constexpr int64_t kOpMaxRow = 4 * kChunk;        // 131072 slots: the bitmaps' capacity
constexpr int kOpWords = (int)(kOpMaxRow / 32);  // words per bitmap
constexpr int kOpCand = 8192;                    // band keys held on chip
constexpr float kOpZ = 5.f;                      // band half-width in binomial standard deviations
constexpr int kOpUnroll = 8;                     // 16-byte loads in flight per thread
constexpr size_t kSelDynSmem = (size_t)(2 * kOpWords + 2 * kOpCand) * sizeof(uint32_t);
static_assert(GatherStaged<64, kSelThreads, 3>::kStageBytes <= (int)kSelDynSmem &&
                  GatherStaged<128, kSelThreads, 3>::kStageBytes <= (int)kSelDynSmem &&
                  GatherStaged<256, kSelThreads, 3>::kStageBytes <= (int)kSelDynSmem &&
                  GatherStaged<512, kSelThreads, 3>::kStageBytes <= (int)kSelDynSmem,
              "the copy stages fit the selection's dynamic shared memory");

__device__ __forceinline__ bool one_pass_select(const float *sc, int M, uint32_t K, bool vec, int32_t *out,
                                                unsigned *flags, uint32_t *dyn, uint32_t *hist, uint32_t *scan_sm,
                                                uint32_t *sh_bin, uint32_t *sh_above, uint32_t *sh_count,
                                                float *red_fa, float *red_fb, uint32_t *red_a, uint32_t *red_b) {
    const int tid = threadIdx.x, lane = tid & 31;
    uint32_t *keepw = dyn;                     // [kOpWords] keep-bits of the row
    uint32_t *tiew = dyn + kOpWords;           // [kOpWords] keys equal to thr
    uint32_t *cand_u = dyn + 2 * kOpWords;     // [kOpCand] band keys
    uint32_t *cand_s = cand_u + kOpCand;       // [kOpCand] their slots
    const int nwords = (M + 31) >> 5;

    // Sample: run `tid` starts at slot (tid * M / 512) rounded down to a multiple
    // of 8, and ends at most at M - 8 (M >= kOpMinRow).
    const int r0 = (int)(((int64_t)tid * M / kOpRuns) & ~(int64_t)7);
    float x[kOpRun];
    float fmn = INFINITY, fmx = -INFINITY;
    int snan = 0;
#pragma unroll
    for (int i = 0; i < kOpRun; i++) {
        x[i] = __ldg(sc + r0 + i);
        fmn = fminf(fmn, x[i]);
        fmx = fmaxf(fmx, x[i]);
        snan |= x[i] != x[i];
    }
    snan = __syncthreads_or(snan);
    block_minmax(fmn, fmx, red_fa, red_fb);
    BinMap bm;
    const float vspan = fmx - fmn;
    const float vlo = fmn - 0.0625f * vspan, vhi = fmx + 0.0625f * vspan;
    bm.vmin = vlo;
    bm.scale = vhi > vlo ? (float)kBins / (vhi - vlo) : 0.f;
    bm.by_value = 1;
    bm.lo = 0u;
    bm.shift = 0;
    if (snan || !isfinite(vspan) || !(vspan > 0.f) || !isfinite(vlo) || !isfinite(vhi) || !isfinite(bm.scale) ||
        !(bm.scale > 0.f))
        return false;  // no usable value range (block-uniform)

    for (int b = 0; b < kBinsPerThread; b++) hist[tid * kBinsPerThread + b] = 0u;
    for (int w = tid; w < nwords; w += kSelThreads) tiew[w] = 0u;
    if (tid == 0) *sh_count = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kOpRun; i++) atomicAdd(&hist[bm(x[i])], 1u);
    __syncthreads();
    const float pk = (float)K / (float)M;
    const float ps = pk * (float)kOpSample;
    const float sd = sqrtf(ps * (1.f - pk));
    const int r_hi = max(0, (int)floorf(ps - kOpZ * sd) - 1);        // sampled keys allowed above the band
    const int r_lo = min(kOpSample, (int)ceilf(ps + kOpZ * sd) + 1);  // sampled keys from the band's low bin up
    uint32_t b_hi = kBins - 1, b_lo, dummy;
    if (r_hi > 0) find_bin(hist, (uint32_t)r_hi, scan_sm, sh_bin, sh_above, b_hi, dummy);
    find_bin(hist, (uint32_t)r_lo, scan_sm, sh_bin, sh_above, b_lo, dummy);
    // The band in value terms: T_hi = the largest sampled value in bin b_hi (no
    // sampled value above it lies outside the bins above b_hi; +inf when nothing
    // may be above), T_lo = the smallest sampled value in bin b_lo.  The map is
    // monotone, so exactly the sampled keys of bins > b_hi exceed T_hi and those
    // of bins >= b_lo are >= T_lo.  Comparisons in fp32 rank -0 with +0 and put
    // NaN (every comparison false) below the band, as the order keys do.
    float hmax = -INFINITY, lmin = INFINITY;
#pragma unroll
    for (int i = 0; i < kOpRun; i++) {
        const int b = bm(x[i]);
        if (b == (int)b_hi) hmax = fmaxf(hmax, x[i]);
        if (b == (int)b_lo) lmin = fminf(lmin, x[i]);
    }
    block_minmax(lmin, hmax, red_fa, red_fb);
    const float t_hi = r_hi > 0 ? hmax : INFINITY, t_lo = lmin;

    // The pass: thread t takes slots 4v .. 4v+3 for v = k * 512 + t, kOpUnroll
    // 16-byte loads in flight (4-byte loads when the row is not 16-byte aligned).
    // Keep-bits of the keys above the band go to the bitmap; the band's slots of a
    // group of kOpUnroll vectors are appended with one warp scan per group (their
    // values are read again, from L1, when stored).
    uint32_t above = 0;
    int nan = 0;
    const int nv = (M + 3) >> 2;
    const int iters = (nv + kSelThreads - 1) / kSelThreads;
    for (int k0 = 0; k0 < iters; k0 += kOpUnroll) {
        float sv[kOpUnroll][4];
#pragma unroll
        for (int u = 0; u < kOpUnroll; u++) {
            const int v = (k0 + u) * kSelThreads + tid;
            if (vec && 4 * v + 3 < M) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(sc) + v);
                sv[u][0] = f.x;
                sv[u][1] = f.y;
                sv[u][2] = f.z;
                sv[u][3] = f.w;
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++) sv[u][i] = 4 * v + i < M ? __ldg(sc + 4 * v + i) : 0.f;
            }
        }
        uint32_t cmask = 0;  // bit 4u + i: slot 4 v_u + i lies in the band
#pragma unroll
        for (int u = 0; u < kOpUnroll; u++) {
            const int v = (k0 + u) * kSelThreads + tid;
            const int lim = M - 4 * v;  // valid slots of this vector (<= 0: none)
            uint32_t nib = 0;
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float sx = sv[u][i];
                const bool valid = i < lim;
                nib |= (uint32_t)(valid && sx > t_hi) << i;
                cmask |= (uint32_t)(valid && sx >= t_lo && sx <= t_hi) << (4 * u + i);
                nan |= valid && sx != sx;
            }
            above += __popc(nib);
            uint32_t w = nib << (4 * (lane & 7));
            w |= __shfl_xor_sync(0xffffffffu, w, 1);
            w |= __shfl_xor_sync(0xffffffffu, w, 2);
            w |= __shfl_xor_sync(0xffffffffu, w, 4);
            if ((lane & 7) == 0 && lim > 0) keepw[v >> 3] = w;
        }
        const uint32_t c = __popc(cmask);
        if (__ballot_sync(0xffffffffu, c != 0u)) {
            uint32_t incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t base = 0;
            if (lane == 31) base = atomicAdd(sh_count, incl);
            base = __shfl_sync(0xffffffffu, base, 31) + incl - c;
            while (cmask) {
                const int e = __ffs(cmask) - 1;
                cmask &= cmask - 1;
                const int j = 4 * ((k0 + (e >> 2)) * kSelThreads + tid) + (e & 3);
                if (base < (uint32_t)kOpCand) {
                    cand_u[base] = order_key(__ldg(sc + j));
                    cand_s[base] = (uint32_t)j;
                }
                base++;
            }
        }
    }
    if (__syncthreads_or(nan) && tid == 0) atomicOr(flags, TRI_FLAG_NONFINITE);
    uint32_t A;
    block_exclusive_scan(above, scan_sm, &A);
    const uint32_t C = *sh_count;
    if (!(A <= K && A + C >= K && C <= (uint32_t)kOpCand)) return false;  // block-uniform

    // The K - A best band keys: exact threshold key thr by radix narrowing over
    // the band keys' range; need2 of the cand2 keys equal to thr are kept.
    const uint32_t need = K - A;
    uint32_t thr = 0xffffffffu, need2 = 0, cand2 = 0;
    if (need > 0) {
        uint32_t lo = 0xffffffffu, hi = 0u;
        for (int i = tid; i < (int)C; i += kSelThreads) {
            lo = min(lo, cand_u[i]);
            hi = max(hi, cand_u[i]);
        }
        block_minmax(lo, hi, red_a, red_b);
        need2 = need;
        cand2 = C;
        for (;;) {
            const uint32_t range = hi - lo;
            if (range == 0) break;
            const int nbits = 32 - __clz(range);
            const int shift = nbits > 11 ? nbits - 11 : 0;
            for (int b = 0; b < kBinsPerThread; b++) hist[tid * kBinsPerThread + b] = 0u;
            __syncthreads();
            for (int i = tid; i < (int)C; i += kSelThreads) {
                const uint32_t u = cand_u[i];
                if (u >= lo && u <= hi) atomicAdd(&hist[(u - lo) >> shift], 1u);
            }
            __syncthreads();
            uint32_t b2, ab2;
            find_bin(hist, need2, scan_sm, sh_bin, sh_above, b2, ab2);
            need2 -= ab2;
            cand2 = hist[b2];
            const uint32_t nlo = lo + (b2 << shift);
            const unsigned long long nhi = (unsigned long long)nlo + ((1ull << shift) - 1ull);
            hi = nhi < (unsigned long long)hi ? (uint32_t)nhi : hi;
            lo = nlo;
            __syncthreads();
            if (shift == 0) break;
        }
        thr = lo;
        for (int i = tid; i < (int)C; i += kSelThreads) {
            const uint32_t u = cand_u[i], j = cand_s[i];
            if (u > thr) atomicOr(&keepw[j >> 5], 1u << (j & 31));
            else if (u == thr) atomicOr(&tiew[j >> 5], 1u << (j & 31));
        }
    }
    __syncthreads();

    // Thread t owns words t*wpt .. t*wpt+wpt-1: keep the ties whose rank from the
    // oldest is at least cand2 - need2, then emit the kept slots ascending.
    const int wpt = (nwords + kSelThreads - 1) / kSelThreads;
    const int w0 = tid * wpt;
    uint32_t tcnt = 0;
    for (int j = 0; j < wpt; j++)
        if (w0 + j < nwords) tcnt += __popc(tiew[w0 + j]);
    uint32_t ttot;
    uint32_t trank = block_exclusive_scan(tcnt, scan_sm, &ttot);
    const uint32_t tie_skip = cand2 - need2;
    uint32_t kcnt = 0;
    for (int j = 0; j < wpt; j++) {
        if (w0 + j >= nwords) break;
        uint32_t kw = keepw[w0 + j], tw = tiew[w0 + j];
        while (tw) {
            const int e = __ffs(tw) - 1;
            tw &= tw - 1;
            if (trank >= tie_skip) kw |= 1u << e;
            trank++;
        }
        keepw[w0 + j] = kw;
        kcnt += __popc(kw);
    }
    uint32_t ktot;
    uint32_t o = block_exclusive_scan(kcnt, scan_sm, &ktot);
    for (int j = 0; j < wpt; j++) {
        if (w0 + j >= nwords) break;
        uint32_t kw = keepw[w0 + j];
        while (kw) {
            const int e = __ffs(kw) - 1;
            kw &= kw - 1;
            if (o < K) out[o] = (w0 + j) * 32 + e;
            o++;
        }
    }
    return true;
}

// LONG: rows average more than one chunk.  Then multi-chunk rows try the single
// pass (its 96 KB of dynamic shared memory are reserved) and the kernel copies
// its row's records; otherwise neither, and the launch reserves no dynamic shared
// memory, leaving the L1 its passes' re-reads use.
template <bool LONG>
__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(const SelectParams p, const GatherParams g) {
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
    // Selection (every exit is block-uniform and leaves the loop), then the
    // row's kept records are copied by the same CTA: rows whose selection is
    // latency-bound overlap other rows' copies, which keep HBM busy.
    bool row_ok = true;
    do {
        if (N < 0 || N > 0x7fffffffLL || row_lo < 0 || row_lo + N > p.geo.total) {
            if (tid == 0) {
                atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
                if (p.kept_count) p.kept_count[r] = 0;
            }
            row_ok = false;
            break;
        }
        if (N <= B) {
            for (int64_t i = tid; i < N; i += kSelThreads) out[i] = (int32_t)i;
            if (tid == 0 && p.kept_count) p.kept_count[r] = (int32_t)N;
            break;
        }
        const int64_t M = N - W;
        const uint32_t K = (uint32_t)(B - W);
        for (int i = tid; i < W; i += kSelThreads) out[K + i] = (int32_t)(M + i);
        if (tid == 0 && p.kept_count) p.kept_count[r] = B;
        if (K == 0) break;
        const float *sc = p.scores + row_lo;
        const bool vec = (((uintptr_t)sc) & 15) == 0;
        const int nchunks = (int)((M + kChunk - 1) / kChunk);
        if (LONG && M >= kOpMinRow && M <= kOpMaxRow) {
            extern __shared__ uint32_t sel_dyn[];
            if (one_pass_select(sc, (int)M, K, vec, out, p.flags, sel_dyn, hist, scan_sm, &sh_bin, &sh_above, &sh_count,
                                red_fa, red_fb, red_a, red_b))
                break;
            __syncthreads();  // every thread has read sh_count before it is cleared below
        }
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
            break;
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
    } while (0);
    if (!LONG || !row_ok) return;
    __syncthreads();  // out[] of this row is complete and visible to the block; the
                      // selection's dynamic shared memory is free for the copy stages
    const int cnt = (int)(N < (int64_t)B ? N : (int64_t)B);
    extern __shared__ __align__(16) uint32_t sel_dyn[];
    unsigned char *stage = reinterpret_cast<unsigned char *>(sel_dyn);
    switch (g.geo.D * g.geo.elem_bytes) {
        case 64: gather_row<64>(g, r, row_lo, N, cnt, stage); break;
        case 128: gather_row<128>(g, r, row_lo, N, cnt, stage); break;
        case 256: gather_row<256>(g, r, row_lo, N, cnt, stage); break;
        case 512: gather_row<512>(g, r, row_lo, N, cnt, stage); break;
    }
}

template <bool LONG>
static cudaError_t launch_select_t(const SelectParams &p, const GatherParams &g, cudaStream_t s) {
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    const size_t dyn = LONG ? kSelDynSmem : 0;
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (LONG && !attr[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSelDynSmem);
        if (e != cudaSuccess) return e;
        attr[dev & 63] = true;
    }
    return launch_pdl(select_kernel<LONG>, dim3((unsigned)R), dim3(kSelThreads), dyn, s, p, g);
}

// Rows longer than one selection chunk on average: the single pass for
// multi-chunk rows, and the selection kernel copies its row's records itself
// (rows still selecting overlap rows already copying, over several waves).
// Shorter rows all select in one wave, where the gather kernel, with more bytes
// in flight per thread, moves the records faster.  The results are identical
// either way.
cudaError_t launch_select_gather(const SelectParams &p, const GatherParams &g, cudaStream_t s) {
    const int rb = g.geo.D * g.geo.elem_bytes;
    if (rb != 64 && rb != 128 && rb != 256 && rb != 512) return cudaErrorInvalidValue;
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R > 0 && p.geo.total > R * kChunk) return launch_select_t<true>(p, g, s);
    const cudaError_t e = launch_select_t<false>(p, g, s);
    if (e != cudaSuccess) return e;
    return launch_gather(g, s);
}

}  // namespace tri
