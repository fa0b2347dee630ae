// Key scoring ("TriAttention：基于三角函数 KV 压缩的高效长推理", 流程详解 steps 2-3;
// "WeianMao/triattention", How it works).
//
// For the row of KV head h the score of a cached key is
//   S_j = (1/G) sum_g sum_f [ |qbar_f^g||k_f| sum_delta cos(w_f (p_now + delta - j) + phi_f^g)
//                             + (E|q_f^g| - |qbar_f^g|) |k_f| ].
// With q.conj(k) written as complex pairs, each cosine term is
// Re(qbar_f conj(k_f^pre) e^{i w_f (p_now + delta - j)}), and a RoPE cache holds
// k_f^post = k_f^pre e^{i w_f j}, so the key's own rotation cancels the -j:
//   S_j = sum_f Re(A_f conj(k_f^post)) + c_f |k_f|,
//   A_f = (1/G) sum_g qbar_f^g * e^{i w_f p_now} * sum_delta e^{i w_f delta},
//   c_f = (1/G) sum_g (E|q_f^g| - |qbar_f^g|).
// The delta sum collapses by angle addition into one complex constant per f,
// and the GQA mean into A_f (the score is linear in the per-head terms).  The
// per-key work is then a d/2-pair dot product plus d/2 magnitudes against
// per-row constants: d x 2 bytes of bf16 (d bytes of fp8) read per key, ~6 FP32
// ops per pair - bound by HBM, not arithmetic, so no tensor cores (there is no
// dense contraction here).
//
// For a cache of pre-RoPE keys, the literal one-(sin, cos)-per-(key, pair)
// form is used instead: A'_f = (1/G) sum_g qbar_f^g sum_delta e^{i w_f delta}
// and S_j = sum_f Re(A'_f e^{i w_f (p_now - j)} conj(k_f)) + c_f |k_f|, with the
// phase w_f (p_now - j) reduced exactly as a 64-bit fixed-point fraction of a
// turn (integer multiply mod 2^64), so fp32 never holds a large angle.
//
// prep_kernel (prep.cu) forms A_f, c_f per row in fp64 and stores fp32.
// score_kernel streams the keys: each warp owns a contiguous span of the
// concatenated key space (all rows end to end, so ragged rows balance across
// the whole grid).  A key of head dim d is shared by d/16 lanes, each owning 8
// frequency pairs (with rotate-half RoPE: 8 consecutive real parts and the 8
// matching imaginary parts d/2 elements later; with interleaved RoPE: 16
// consecutive elements), so a warp instruction covers 32 / (d/16) keys'
// records.  Every lane keeps U keys' loads in flight (U = 4 for d = 64 and for
// pre-RoPE caches, else 8), accumulates its 8 pairs in fp32, and a butterfly
// reduce-scatter over the lanes of a key leaves one full score per lane; a
// shuffle orders them for one coalesced store per batch (KB = 32 / (d/16) x U
// keys).  Contiguous pre-RoPE and fp8 caches take score_staged_kernel (below),
// which stages the same batches in shared memory.
#include "score_common.cuh"
#include "stage.cuh"

namespace tri {

constexpr int kScoreThreads = 256;

template <bool PAGED, bool PRE, int ELEM, bool IL, int LPK>
__global__ void __launch_bounds__(kScoreThreads, (ELEM == 1 && !PRE && !PAGED) ? 3 : 2) score_kernel(const ScoreParams p) {
    using Sh = Shape<LPK, PRE>;
    constexpr int NG = Sh::NG, U = Sh::U, KB = Sh::KB, F = Sh::F;
    constexpr int RB = 2 * F * ELEM;  // record bytes
    grid_dependency_wait();
    grid_dependents_launch();
    const Geometry &geo = p.geo;
    const int lane = threadIdx.x & 31;
    const int q = lane / LPK;   // key of the NG-key group
    const int gl = lane % LPK;  // pairs 8gl .. 8gl+7
    const int64_t nwarps = (int64_t)gridDim.x * (kScoreThreads / 32);
    const int64_t wid = (int64_t)blockIdx.x * (kScoreThreads / 32) + (threadIdx.x >> 5);
    const int64_t total = geo.total;
    int64_t per = (total + nwarps - 1) / nwarps;
    per = (per + KB - 1) / KB * KB;
    const int64_t beg = wid * per;
    const int64_t end = min(total, beg + per);
    if (beg >= end) return;
    const int R = geo.L * geo.S * geo.H;
    const int cpr = LPK * kCoefPerGroup;

    unsigned long long T[8];
#pragma unroll
    for (int i = 0; i < 8; i++) T[i] = PRE ? p.turns[8 * gl + i] : 0ull;
    unsigned long long TC[4], TS[4];  // e^{-i w NG}: from one key's rotated coefficients to the next one's
    if (PRE) step_phasors(T, NG, TC, TS);
    const unsigned long long pol = policy_evict_first();

    // Row holding key `beg`: the last r with row_off[r] <= beg.
    int rl = 0, rh = R;
    while (rh - rl > 1) {
        const int mid = (rl + rh) >> 1;
        if (geo.row_off[mid] <= beg) rl = mid;
        else rh = mid;
    }
    int r0 = rl;
    while (r0 < R - 1 && geo.row_off[r0 + 1] <= beg) r0++;
    RowCtx c;
    set_row(c, p, r0, gl, cpr);

    for (int64_t b0 = beg; b0 < end; b0 += KB) {
        const int64_t bend = min(b0 + KB, end);
        if (b0 >= c.hi && c.r < R - 1) {  // the batch starts in a later row: move there first
            int r = c.r + 1;
            while (r < R - 1 && geo.row_off[r + 1] <= b0) r++;
            set_row(c, p, r, gl, cpr);
        }
        float part[U];
        if (bend == b0 + KB && b0 >= c.lo && bend <= c.hi) {
            // Whole batch inside the current row: issue all loads, then compute.
            KeyChunk<ELEM, IL, F> kc[U];
            int64_t slot[U];
            int32_t kpos[U];
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
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; u++) {
                ok[u] = !PAGED || slot[u] >= 0;
                if (!ok[u]) atomicOr(p.flags, TRI_FLAG_BLOCK_TABLE);
            }
            batch_partials<PRE, U, NG>(kc, kpos, ok, c, T, TC, TS, part);
        } else {
            // Batch crosses a row boundary or the span end: one segment per row.
#pragma unroll
            for (int u = 0; u < U; u++) part[u] = 0.f;
            int64_t k0 = b0;
            for (;;) {
                const int64_t seg_end = min(bend, c.hi);
#pragma unroll
                for (int u = 0; u < U; u++) {
                    const int64_t k = b0 + NG * u + q;
                    if (k >= k0 && k < seg_end) part[u] += key_partial<PAGED, PRE, ELEM, IL, LPK>(p, c, k, gl, pol, T);
                }
                if (bend <= c.hi) break;
                k0 = max(k0, c.hi);
                int r = c.r + 1;
                while (r < R && geo.row_off[r + 1] <= k0) r++;
                if (r >= R) {
                    atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
                    break;
                }
                set_row(c, p, r, gl, cpr);
                if (c.lo != k0) atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
            }
        }
        // Butterfly reduce-scatter over the lanes sharing a key: at the stage of
        // lane bit `half`, a lane keeps the upper or lower half of its partials
        // and adds its partner's copy of that half.  Afterwards lane (q, gl) holds
        // key NG * (gl % U) + q summed over the lanes that differ from it in the
        // low log2(U) bits of gl; when LPK > U, plain exchanges over the remaining
        // lane bits add the other lanes' pairs.
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
        // Lane i < KB stores key b0 + i, held by lane (i % NG) * LPK + i / NG.
        const int src = lane < KB ? (lane % NG) * LPK + lane / NG : lane;
        const float v = __shfl_sync(0xffffffffu, part[0], src);
        if (lane < KB && b0 + lane < bend) p.scores[b0 + lane] = v;
    }
}

// ------------------------------------------------------------ staged variant
//
// Contiguous caches: a warp's span is consecutive records, so each of its
// batches (KB keys) is one run of KB x RB bytes (and KB positions for a
// pre-RoPE cache).  The warp stages its batches in a private ring of STAGES
// slots of shared memory, one bulk copy per batch, issued STAGES batches
// ahead, so the bytes in flight no longer depend on registers; each lane then
// reads its share of a key from the slot.  A slot is refilled only after the
// batch's arithmetic has consumed it.  Span partition, batch grid, row
// advance, fast/slow path and arithmetic are those of score_kernel: the scores
// are bit-identical.
template <bool PRE, int ELEM, int LPK>
struct Staging {
    using Sh = Shape<LPK, PRE>;
    static constexpr int kWarps = kScoreThreads / 32;
    static constexpr int RB = 2 * Sh::F * ELEM;                     // record bytes
    static constexpr int KEY_BYTES = Sh::KB * RB;                   // a batch's records
    static constexpr int SLOT = KEY_BYTES + (PRE ? Sh::KB * 4 : 0);  // then its positions
    static constexpr int BUDGET = PRE ? 13312 : 8192;               // shared bytes per warp
    static constexpr int STAGES = BUDGET / SLOT < 2 ? 2 : (BUDGET / SLOT > 4 ? 4 : BUDGET / SLOT);
    static constexpr int HEADER = (kWarps * STAGES * 8 + 127) / 128 * 128;  // the barriers
    static constexpr size_t SMEM = (size_t)HEADER + (size_t)kWarps * STAGES * SLOT;
    static_assert(SLOT % 16 == 0 && KEY_BYTES % 16 == 0 && HEADER % 128 == 0, "bulk copies need 16-byte units");
    static_assert(Sh::KB % 4 == 0, "a batch's positions start on a 16-byte boundary");
};

// Issues batch i of a warp's span (keys b0 .. min(b0 + KB, end) - 1) into slot
// i % STAGES of the warp's ring: one bulk copy of the records and, when the
// positions array is 16-byte aligned, one of the positions in whole groups of
// four (the remaining ones are read from global memory).  One thread per warp.
template <typename St>
__device__ __forceinline__ void stage_batch(const ScoreParams &p, int64_t b0, int64_t end, unsigned char *ring,
                                            uint64_t *bar, int64_t i, bool pos_bulk, unsigned long long pol) {
    const int n = (int)min((int64_t)St::Sh::KB, end - b0);
    unsigned char *slot = ring + (int)(i % St::STAGES) * St::SLOT;
    uint64_t *b = &bar[i % St::STAGES];
    const uint32_t kbytes = (uint32_t)n * St::RB;
    const uint32_t pbytes = pos_bulk ? (uint32_t)(n & ~3) * 4u : 0u;
    mbar_arrive_expect_tx(b, kbytes + pbytes);
    bulk_load(slot, p.K + b0 * St::RB, kbytes, b, pol);
    if (pbytes) bulk_load(slot + St::KEY_BYTES, p.pos + b0, pbytes, b, pol);
}

template <bool PRE, int ELEM, bool IL, int LPK>
__global__ void __launch_bounds__(kScoreThreads, (ELEM == 1 && !PRE) ? 3 : 2) score_staged_kernel(const ScoreParams p) {
    using Sh = Shape<LPK, PRE>;
    using St = Staging<PRE, ELEM, LPK>;
    constexpr int NG = Sh::NG, U = Sh::U, KB = Sh::KB, F = Sh::F;
    constexpr int RB = St::RB, SLOT = St::SLOT, STAGES = St::STAGES;
    extern __shared__ __align__(128) unsigned char smem[];
    grid_dependency_wait();
    grid_dependents_launch();
    const Geometry &geo = p.geo;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int q = lane / LPK;
    const int gl = lane % LPK;
    const int64_t nwarps = (int64_t)gridDim.x * (kScoreThreads / 32);
    const int64_t wid = (int64_t)blockIdx.x * (kScoreThreads / 32) + warp;
    const int64_t total = geo.total;
    int64_t per = (total + nwarps - 1) / nwarps;
    per = (per + KB - 1) / KB * KB;
    const int64_t beg = wid * per;
    const int64_t end = min(total, beg + per);
    if (beg >= end) return;
    const int R = geo.L * geo.S * geo.H;
    const int cpr = LPK * kCoefPerGroup;

    uint64_t *bar = reinterpret_cast<uint64_t *>(smem) + warp * STAGES;
    unsigned char *ring = smem + St::HEADER + (size_t)warp * STAGES * SLOT;
    const unsigned long long pol = policy_evict_first();
    const bool pos_bulk = PRE && (reinterpret_cast<uintptr_t>(p.pos) & 15) == 0;
    const int64_t nb = (end - beg + KB - 1) / KB;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; s++) mbar_init(&bar[s], 1);
        mbar_init_fence();
    }
    __syncwarp();
    const int64_t first = nb < STAGES ? nb : STAGES;
    if (lane == 0)
        for (int64_t i = 0; i < first; i++) stage_batch<St>(p, beg + i * KB, end, ring, bar, i, pos_bulk, pol);

    unsigned long long T[8];
#pragma unroll
    for (int i = 0; i < 8; i++) T[i] = PRE ? p.turns[8 * gl + i] : 0ull;
    unsigned long long TC[4], TS[4];
    if (PRE) step_phasors(T, NG, TC, TS);

    int rl = 0, rh = R;
    while (rh - rl > 1) {
        const int mid = (rl + rh) >> 1;
        if (geo.row_off[mid] <= beg) rl = mid;
        else rh = mid;
    }
    int r0 = rl;
    while (r0 < R - 1 && geo.row_off[r0 + 1] <= beg) r0++;
    RowCtx c;
    set_row(c, p, r0, gl, cpr);

    for (int64_t i = 0; i < nb; i++) {
        const int64_t b0 = beg + i * KB;
        const int64_t bend = min(b0 + KB, end);
        const int si = (int)(i % STAGES);
        if (!__all_sync(0xffffffffu, mbar_wait(&bar[si], (uint32_t)(i / STAGES) & 1u))) {
            // A copy did not land: flag it, wait once more (bounded) for every
            // copy still in flight into this warp's ring - batches i .. i +
            // STAGES - 1 - and leave the rest of the span.
            if (lane == 0) atomicOr(p.flags, TRI_FLAG_STAGE_TIMEOUT);
            const int64_t last = min(nb, i + STAGES);
            for (int64_t j = i; j < last; j++) mbar_wait(&bar[j % STAGES], (uint32_t)(j / STAGES) & 1u);
            return;
        }
        const unsigned char *slot = ring + si * SLOT;
        const int32_t *spos = reinterpret_cast<const int32_t *>(slot + St::KEY_BYTES);
        const int npos = pos_bulk ? ((int)(bend - b0) & ~3) : 0;
        if (b0 >= c.hi && c.r < R - 1) {
            int r = c.r + 1;
            while (r < R - 1 && geo.row_off[r + 1] <= b0) r++;
            set_row(c, p, r, gl, cpr);
        }
        float part[U];
        if (bend == b0 + KB && b0 >= c.lo && bend <= c.hi) {
            // Whole batch inside the current row (npos = KB when positions were staged):
            // each key is read from the slot as it is scored.
            int32_t kpos[U];
#pragma unroll
            for (int u = 0; u < U; u++) {
                const int idx = NG * u + q;
                kpos[u] = PRE ? (pos_bulk ? spos[idx] : __ldg(p.pos + b0 + idx)) : 0;
            }
            batch_partials_lazy<PRE, U, NG, KeyChunk<ELEM, IL, F>>(
                [&](int u, KeyChunk<ELEM, IL, F> &kc) { kc.lds(slot + (NG * u + q) * RB, gl); }, kpos, c, T, TC,
                TS, part);
        } else {
            // Batch crosses a row boundary or the span end: one segment per row,
            // each key read from the slot as it is scored.
#pragma unroll
            for (int u = 0; u < U; u++) part[u] = 0.f;
            int64_t k0 = b0;
            for (;;) {
                const int64_t seg_end = min(bend, c.hi);
#pragma unroll
                for (int u = 0; u < U; u++) {
                    const int idx = NG * u + q;
                    const int64_t k = b0 + idx;
                    if (k >= k0 && k < seg_end) {
                        KeyChunk<ELEM, IL, F> kc;
                        kc.lds(slot + idx * RB, gl);
                        const int64_t delta =
                            PRE ? c.p_now - (int64_t)(idx < npos ? spos[idx] : __ldg(p.pos + k)) : 0;
                        part[u] += chunk_partial<PRE>(kc, c, T, delta);
                    }
                }
                if (bend <= c.hi) break;
                k0 = max(k0, c.hi);
                int r = c.r + 1;
                while (r < R && geo.row_off[r + 1] <= k0) r++;
                if (r >= R) {
                    atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
                    break;
                }
                set_row(c, p, r, gl, cpr);
                if (c.lo != k0) atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
            }
        }
        if (i + STAGES < nb) {  // the slot's bytes are consumed: refill it
            fence_async_smem();
            __syncwarp();
            if (lane == 0) stage_batch<St>(p, b0 + STAGES * KB, end, ring, bar, i + STAGES, pos_bulk, pol);
        }
#pragma unroll
        for (int half = U / 2; half >= 1; half >>= 1) {
            const bool up = (gl & half) != 0;
#pragma unroll
            for (int j = 0; j < half; j++) {
                const float send = up ? part[j] : part[j + half];
                const float keep = up ? part[j + half] : part[j];
                part[j] = keep + __shfl_xor_sync(0xffffffffu, send, half);
            }
        }
#pragma unroll
        for (int o = U; o < LPK; o <<= 1) part[0] += __shfl_xor_sync(0xffffffffu, part[0], o);
        const int src = lane < KB ? (lane % NG) * LPK + lane / NG : lane;
        const float v = __shfl_sync(0xffffffffu, part[0], src);
        if (lane < KB && b0 + lane < bend) p.scores[b0 + lane] = v;
    }
}

template <bool PAGED, bool PRE, int ELEM, bool IL, int LPK>
static cudaError_t launch_score_t(const ScoreParams &p, cudaStream_t s) {
    auto kern = score_kernel<PAGED, PRE, ELEM, IL, LPK>;
    static int occ[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int &o = occ[dev & 63];
    if (o == 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, kScoreThreads, 0);
        if (e != cudaSuccess) return e;
        if (o < 1) o = 1;
    }
    constexpr int KB = Shape<LPK, PRE>::KB;
    const int64_t want = (p.geo.total + KB * (kScoreThreads / 32) - 1) / (KB * (kScoreThreads / 32));
    int64_t grid = (int64_t)sm_count() * o;
    if (want < grid) grid = want;
    if (grid < 1) grid = 1;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kScoreThreads), 0, s, p);
}

template <bool PRE, int ELEM, bool IL, int LPK>
static cudaError_t launch_score_staged_t(const ScoreParams &p, cudaStream_t s) {
    using St = Staging<PRE, ELEM, LPK>;
    auto kern = score_staged_kernel<PRE, ELEM, IL, LPK>;
    static int occ[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int &o = occ[dev & 63];
    if (o == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)St::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, kScoreThreads, St::SMEM);
        if (e != cudaSuccess) return e;
        if (o < 1) return cudaErrorInvalidConfiguration;
    }
    constexpr int KB = Shape<LPK, PRE>::KB;
    const int64_t want = (p.geo.total + KB * (kScoreThreads / 32) - 1) / (KB * (kScoreThreads / 32));
    int64_t grid = (int64_t)sm_count() * o;
    if (want < grid) grid = want;
    if (grid < 1) grid = 1;
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kScoreThreads), St::SMEM, s, p);
}

// Contiguous caches whose keys the registers alone cannot keep enough of in
// flight (pre-RoPE keys: four per lane; fp8 records: half the bytes per
// load) stream through the staged kernel; the rest through score_kernel.
template <int ELEM, bool IL, int LPK>
static cudaError_t launch_score_d(const ScoreParams &p, int pre_rope, cudaStream_t s) {
    if (p.geo.layout == TRI_KV_PAGED)
        return pre_rope ? launch_score_t<true, true, ELEM, IL, LPK>(p, s) : launch_score_t<true, false, ELEM, IL, LPK>(p, s);
    if (pre_rope) return launch_score_staged_t<true, ELEM, IL, LPK>(p, s);
    if constexpr (ELEM == 1) return launch_score_staged_t<false, ELEM, IL, LPK>(p, s);
    else return launch_score_t<false, false, ELEM, IL, LPK>(p, s);
}

template <int ELEM, bool IL>
static cudaError_t launch_score_l(const ScoreParams &p, int pre_rope, cudaStream_t s) {
    switch (p.geo.D) {
        case 64: return launch_score_d<ELEM, IL, 4>(p, pre_rope, s);
        case 128: return launch_score_d<ELEM, IL, 8>(p, pre_rope, s);
        case 256: return launch_score_d<ELEM, IL, 16>(p, pre_rope, s);
    }
    return cudaErrorInvalidValue;
}

template <int ELEM>
static cudaError_t launch_score_e(const ScoreParams &p, int pre_rope, cudaStream_t s) {
    return p.geo.il ? launch_score_l<ELEM, true>(p, pre_rope, s) : launch_score_l<ELEM, false>(p, pre_rope, s);
}

cudaError_t launch_score(const ScoreParams &p, int pre_rope, cudaStream_t s) {
    if (p.geo.total <= 0) return cudaSuccess;
    return p.geo.elem_bytes == 1 ? launch_score_e<1>(p, pre_rope, s) : launch_score_e<2>(p, pre_rope, s);
}

}  // namespace tri
