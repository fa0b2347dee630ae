// Fused scoring and selection for rows of at most kFusedMaxRow keys
// ("TriAttention：基于三角函数 KV 压缩的高效长推理", 流程详解 steps 2-4: score every
// key, keep the most important ones).  One CTA of 512 threads per row keeps the
// row's scores on chip, as order-preserving uint32 keys in shared memory
// (128 KB for 32768 keys), so neither the scores' round trip through HBM nor
// the selection's re-reads happen, and no separate selection launch is made.
//
//  A. Scores: the streaming score kernel's lane layout and arithmetic (the same
//     device functions, the same reduction order, and batches of KB keys on the
//     same grid of multiples of KB in the concatenated key space, so the scores
//     are bit-identical), the 16 warps taking the row's batches in turn.
//     Optionally the fp32 scores are also written to global memory.
//  B. Threshold: for N > B, the exact (B-W)-th best key value thr of slots
//     0 .. M-1 (M = N-W) by radix narrowing over the row's key range: at most
//     three passes of 2048-bin shared-memory histograms, each over the keys
//     still in range, one block scan per pass to find the bin.
//  C. Marking and emission: thread t owns slots ipt*t .. ipt*t+ipt-1, ipt =
//     ceil(N / 512) (read in a rotated order; for ipt = 64 a warp's reads hit 32
//     distinct banks); keys above thr and the window are kept, and of the keys
//     equal to thr the most recent ones (a block scan ranks the ties in slot
//     order); a second block scan of the per-thread kept counts places every
//     kept slot, ascending.  Every pass is bounded by the row's length, so a
//     short row costs little.
// Blocks never wait on other blocks.  Rows longer than kFusedMaxRow are not
// processed here: they are flagged and their kept entries set to -1 (the host
// routes calls whose bound on the row length exceeds kFusedMaxRow to the
// unfused kernels, so only a caller's understated bound gets here).
#include "coef.cuh"
#include "score_common.cuh"

namespace tri {

constexpr int kFThreads = 512;
constexpr int kFWarps = kFThreads / 32;
constexpr int kFItems = kFusedMaxRow / kFThreads;  // most slots per thread (64)
static_assert(kFusedMaxRow % kFThreads == 0 && kFItems <= 64, "a thread's slots fit its 64-bit masks");
constexpr int kFBins = 2048;
constexpr int kFBinsPerThread = kFBins / kFThreads;
constexpr size_t kFusedSmem = (size_t)kFusedMaxRow * 4 + kFBins * 4;

// Exclusive scan over the block in thread order; *total receives the sum.
__device__ __forceinline__ uint32_t fused_scan(uint32_t v, uint32_t *sm, uint32_t *total) {
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
        uint32_t w = lane < kFWarps ? sm[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < kFWarps) sm[lane] = w;
    }
    __syncthreads();
    const uint32_t base = warp ? sm[warp - 1] : 0u;
    *total = sm[kFWarps - 1];
    __syncthreads();
    return base + x - v;
}

template <bool PAGED, bool PRE, int ELEM, bool IL, int LPK>
__global__ void __launch_bounds__(kFThreads, 1) fused_kernel(const FusedParams fp) {
    using Sh = Shape<LPK, PRE>;
    constexpr int NG = Sh::NG, U = Sh::U, KB = Sh::KB, F = Sh::F;
    constexpr int RB = 2 * F * ELEM;
    extern __shared__ __align__(16) uint32_t fsm[];
    uint32_t *keys = fsm;                  // [kFusedMaxRow]
    uint32_t *hist = fsm + kFusedMaxRow;  // [kFBins]
    __shared__ uint32_t scan_sm[kFWarps];
    __shared__ uint32_t red_a[kFWarps], red_b[kFWarps];
    __shared__ uint32_t sh_bin, sh_above;

    const ScoreParams &p = fp.sp;
    const Geometry &geo = p.geo;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = blockIdx.x;
    // The row's coefficients, step 1 (kernel parameters only) before the wait
    // for the preceding kernel: threads tid < kPrepParts * F, as in the prep kernel.
    constexpr int kCoefThreads = kPrepParts * F;
    static_assert(kCoefThreads <= kFThreads, "the coefficient steps fit the block");
    unsigned long long Tf = 0;
    double osr = 0.0, osi = 0.0;
    if (tid < kCoefThreads) coef_offsets<F>(fp.pp, tid % F, tid / F, Tf, osr, osi);
    grid_dependency_wait();
    grid_dependents_launch();
    const int64_t lo = geo.row_off[r], hi = geo.row_off[r + 1];
    const int64_t N64 = hi - lo;
    const int32_t B = fp.B, W = fp.W;
    int32_t *out = fp.kept + (int64_t)r * B;
    if (lo < 0 || N64 < 0 || hi > geo.total || N64 > kFusedMaxRow) {
        if (tid == 0) {
            atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
            if (fp.kept_count) fp.kept_count[r] = 0;
        }
        // The row keeps nothing: every kept entry is marked empty (-1), so the
        // gather that follows leaves the row's output records untouched.
        for (int i = tid; i < B; i += kFThreads) out[i] = -1;
        return;
    }
    const int N = (int)N64;
    const int M = N > B ? N - W : N;       // candidate slots (all slots when N <= B)
    const uint32_t K = N > B ? (uint32_t)(B - W) : 0u;

    // Step 2 of the coefficients, staged in shared memory before the keys use it:
    // partial sums in the histogram's space, the row's [d/16][24] coefficients and
    // the T_f table at the start of the keys' space.
    double(*part_re)[F] = reinterpret_cast<double(*)[F]>(hist);
    double(*part_im)[F] = reinterpret_cast<double(*)[F]>(hist + 2 * kPrepParts * F);
    float *coef_sm = reinterpret_cast<float *>(keys);
    unsigned long long *turns_sm = reinterpret_cast<unsigned long long *>(keys + 3 * F);
    if (tid < kCoefThreads) {
        part_re[tid / F][tid % F] = osr;
        part_im[tid / F][tid % F] = osi;
    }
    __syncthreads();
    if (tid < F) {
        coef_finish<F>(fp.pp, r, tid, Tf, part_re, part_im, coef_sm);
        turns_sm[tid] = Tf;
        if (r == 0 && tid == 0) {
            const int64_t R = (int64_t)geo.L * geo.S * geo.H;
            if (geo.row_off[0] != 0 || geo.row_off[R] != geo.total) atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
        }
    }
    __syncthreads();

    // ---- A. scores of the row into shared memory (and optionally global)
    const int q = lane / LPK, gl = lane % LPK;
    unsigned long long T[8];
#pragma unroll
    for (int i = 0; i < 8; i++) T[i] = PRE ? turns_sm[8 * gl + i] : 0ull;
    unsigned long long TC[4], TS[4];
    if (PRE) step_phasors(T, NG, TC, TS);
    const unsigned long long pol = policy_evict_first();
    RowCtx c;
    set_row_coef(c, p, r, gl, coef_sm + gl * kCoefPerGroup);
    __syncthreads();  // the keys' space is rewritten below
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    int nan = 0;
    // Batches on the same grid as the score kernel's (multiples of KB in the
    // concatenated key space), so every key sees the same batch and the same
    // per-lane arithmetic: bit-identical scores, pre-RoPE phasor chains included.
    const int64_t grid0 = lo - lo % KB;
    for (int64_t b0 = grid0 + (int64_t)warp * KB; b0 < hi; b0 += (int64_t)kFWarps * KB) {
        float part[U];
        if (b0 >= lo && b0 + KB <= hi) {
            KeyChunk<ELEM, IL, F> kc[U];
            int32_t kpos[U];
            bool ok[U];
            if constexpr (PAGED && !PRE) {
                // key_slot's address in 32-bit steps where they fit: the row has at
                // most kFusedMaxRow keys, so a key's place in the row and its block
                // index are small; only the block's byte offset needs 64 bits.
                // Byte address: the layer's head-h record of block 0, plus blk blocks,
                // plus the slot within the block.
                const int j0 = (int)(b0 - lo) + q;
                const char *kb = p.K + (((c.layer_blk << geo.block_shift) * geo.H) + c.h) * RB;
                const int64_t blk_bytes = ((int64_t)geo.H * RB) << geo.block_shift;
                const int64_t slot_bytes = (int64_t)geo.H * RB;
#pragma unroll
                for (int u = 0; u < U; u++) {
                    const int j = j0 + NG * u;
                    const int bi = j >> geo.block_shift;
                    const int32_t blk = bi < geo.max_blocks ? __ldg(c.table + bi) : -1;
                    ok[u] = blk >= 0 && blk < geo.n_blocks;
                    kpos[u] = 0;
                    if (ok[u]) kc[u].load(kb + blk * blk_bytes + (j & ((1 << geo.block_shift) - 1)) * slot_bytes, gl, pol);
                    else kc[u].zero();
                }
            } else {
                int64_t slot[U];
#pragma unroll
                for (int u = 0; u < U; u++) {
                    slot[u] = key_slot<PAGED>(p, c, b0 + NG * u + q);
                    if (slot[u] >= 0) {
                        kc[u].load(p.K + slot[u] * RB, gl, pol);
                        kpos[u] = PRE ? __ldg(p.pos + slot[u]) : 0;
                    } else {
                        kc[u].zero();
                        kpos[u] = 0;
                    }
                }
#pragma unroll
                for (int u = 0; u < U; u++) ok[u] = !PAGED || slot[u] >= 0;
            }
#pragma unroll
            for (int u = 0; u < U; u++)
                if (!ok[u]) atomicOr(p.flags, TRI_FLAG_BLOCK_TABLE);
            batch_partials<PRE, U, NG>(kc, kpos, ok, c, T, TC, TS, part);
        } else {
#pragma unroll
            for (int u = 0; u < U; u++) {
                const int64_t k = b0 + NG * u + q;
                part[u] = (k >= lo && k < hi) ? key_partial<PAGED, PRE, ELEM, IL, LPK>(p, c, k, gl, pol, T) : 0.f;
            }
        }
        // The score kernel's reduce-scatter, in the same order.
#pragma unroll
        for (int half = U / 2; half >= 1; half >>= 1) {
            const bool up = (gl & half) != 0;
#pragma unroll
            for (int i = 0; i < half; i++) {
                const float send = up ? part[i] : part[i + half];
                const float keep = up ? part[i + half] : part[i];
                part[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
            }
        }
#pragma unroll
        for (int o = U; o < LPK; o <<= 1) part[0] += __shfl_xor_sync(0xffffffffu, part[0], o);
        const int src = lane < KB ? (lane % NG) * LPK + lane / NG : lane;
        const float v = __shfl_sync(0xffffffffu, part[0], src);
        if (lane < KB && b0 + lane >= lo && b0 + lane < hi) {
            const int j = (int)(b0 + lane - lo);
            const uint32_t u = order_key(v);
            keys[j] = u;
            if (p.scores) p.scores[b0 + lane] = v;
            nan |= v != v;
            if (j < M) {
                kmin = min(kmin, u);
                kmax = max(kmax, u);
            }
        }
    }
    if (__syncthreads_or(nan) && tid == 0) atomicOr(p.flags, TRI_FLAG_NONFINITE);
    if (tid == 0 && fp.kept_count) fp.kept_count[r] = N < B ? N : B;

    // ---- B. the exact K-th best key value thr among slots 0 .. M-1
    uint32_t thr = 0xffffffffu, tie_skip = 0u;
    if (K > 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        }
        if (lane == 0) {
            red_a[warp] = kmin;
            red_b[warp] = kmax;
        }
        __syncthreads();
        uint32_t klo = 0xffffffffu, khi = 0u;
        for (int w = 0; w < kFWarps; w++) {
            klo = min(klo, red_a[w]);
            khi = max(khi, red_b[w]);
        }
        uint32_t need = K, cand = (uint32_t)M;
        for (int pass = 0; pass < 3; pass++) {
            const uint32_t range = khi - klo;
            if (range == 0) break;
            const int nbits = 32 - __clz(range);
            const int shift = nbits > 11 ? nbits - 11 : 0;
            for (int b = 0; b < kFBinsPerThread; b++) hist[tid * kFBinsPerThread + b] = 0u;
            __syncthreads();
            const int passes = (M + kFThreads - 1) / kFThreads;
            for (int e = 0; e < passes; e++) {
                const int j = e * kFThreads + tid;
                if (j < M) {
                    const uint32_t u = keys[j];
                    if (u >= klo && u <= khi) atomicAdd(&hist[(u - klo) >> shift], 1u);
                }
            }
            __syncthreads();
            // The bin (from the top) holding the need-th best key, and the keys above it.
            const int top = kFBins - 1 - kFBinsPerThread * tid;
            uint32_t mine = 0;
#pragma unroll
            for (int b = 0; b < kFBinsPerThread; b++) mine += hist[top - b];
            uint32_t tot;
            const uint32_t above_me = fused_scan(mine, scan_sm, &tot);
            if (above_me < need && above_me + mine >= need) {
                uint32_t acc = above_me;
                for (int b = 0; b < kFBinsPerThread; b++) {
                    const uint32_t hb = hist[top - b];
                    if (acc + hb >= need) {
                        sh_bin = (uint32_t)(top - b);
                        sh_above = acc;
                        break;
                    }
                    acc += hb;
                }
            }
            __syncthreads();
            const uint32_t bin = sh_bin, above = sh_above;
            need -= above;
            cand = hist[bin];
            const uint32_t nlo = klo + (bin << shift);
            const unsigned long long nhi = (unsigned long long)nlo + ((1ull << shift) - 1ull);
            khi = nhi < (unsigned long long)khi ? (uint32_t)nhi : khi;
            klo = nlo;
            __syncthreads();  // hist and sh_* are rewritten by the next pass
            if (shift == 0) break;
        }
        thr = klo;
        tie_skip = cand - need;  // ties at thr in the oldest slots are dropped
    }

    // ---- C. mark kept slots (rotated reads: lane l of a warp reads bank (e + l) % 32) and emit them ascending
    unsigned long long gt = 0, eq = 0, keep = 0;
    const int ipt = (N + kFThreads - 1) / kFThreads;  // 1 .. kFItems slots per thread
    const int rot = ipt ? tid % ipt : 0;               // rotation of the read order
    for (int e = 0; e < ipt; e++) {
        int pos = e + rot;
        if (pos >= ipt) pos -= ipt;
        const int j = ipt * tid + pos;
        if (j < N) {
            if (j >= M || K == 0 && N <= B) {
                keep |= 1ull << pos;  // window slots, or every slot when N <= B
            } else if (K > 0) {
                const uint32_t u = keys[j];
                gt |= (unsigned long long)(u > thr) << pos;
                eq |= (unsigned long long)(u == thr) << pos;
            }
        }
    }
    uint32_t tot;
    uint32_t rank = fused_scan((uint32_t)__popcll(eq), scan_sm, &tot);
    unsigned long long eqs = eq;
    while (eqs) {
        const int e = __ffsll((long long)eqs) - 1;
        eqs &= eqs - 1;
        if (rank >= tie_skip) keep |= 1ull << e;
        rank++;
    }
    keep |= gt;
    uint32_t o = fused_scan((uint32_t)__popcll(keep), scan_sm, &tot);
    unsigned long long bits = keep;
    while (bits) {
        const int e = __ffsll((long long)bits) - 1;
        bits &= bits - 1;
        if (o < (uint32_t)B) out[o] = ipt * tid + e;
        o++;
    }
}

template <bool PAGED, bool PRE, int ELEM, bool IL, int LPK>
static cudaError_t launch_fused_t(const FusedParams &p, cudaStream_t s) {
    auto kern = fused_kernel<PAGED, PRE, ELEM, IL, LPK>;
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFusedSmem);
        if (e != cudaSuccess) return e;
        attr[dev & 63] = true;
    }
    const int64_t R = (int64_t)p.sp.geo.L * p.sp.geo.S * p.sp.geo.H;
    return launch_pdl(kern, dim3((unsigned)R), dim3(kFThreads), kFusedSmem, s, p);
}

template <int ELEM, bool IL, int LPK>
static cudaError_t launch_fused_d(const FusedParams &p, int pre, cudaStream_t s) {
    if (p.sp.geo.layout == TRI_KV_PAGED)
        return pre ? launch_fused_t<true, true, ELEM, IL, LPK>(p, s) : launch_fused_t<true, false, ELEM, IL, LPK>(p, s);
    return pre ? launch_fused_t<false, true, ELEM, IL, LPK>(p, s) : launch_fused_t<false, false, ELEM, IL, LPK>(p, s);
}

template <int ELEM, bool IL>
static cudaError_t launch_fused_l(const FusedParams &p, int pre, cudaStream_t s) {
    switch (p.sp.geo.D) {
        case 64: return launch_fused_d<ELEM, IL, 4>(p, pre, s);
        case 128: return launch_fused_d<ELEM, IL, 8>(p, pre, s);
        case 256: return launch_fused_d<ELEM, IL, 16>(p, pre, s);
    }
    return cudaErrorInvalidValue;
}

template <int ELEM>
static cudaError_t launch_fused_e(const FusedParams &p, int pre, cudaStream_t s) {
    return p.sp.geo.il ? launch_fused_l<ELEM, true>(p, pre, s) : launch_fused_l<ELEM, false>(p, pre, s);
}

cudaError_t launch_fused(const FusedParams &p, int pre_rope, cudaStream_t s) {
    const int64_t R = (int64_t)p.sp.geo.L * p.sp.geo.S * p.sp.geo.H;
    if (R <= 0) return cudaSuccess;
    if (R > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return p.sp.geo.elem_bytes == 1 ? launch_fused_e<1>(p, pre_rope, s) : launch_fused_e<2>(p, pre_rope, s);
}

}  // namespace tri
