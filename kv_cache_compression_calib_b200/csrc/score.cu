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
// records.  Every lane keeps U keys' loads in flight (U = 4 for d = 64, else
// 8), accumulates its 8 pairs in fp32, and a butterfly reduce-scatter over the
// lanes of a key leaves one full score per lane; a shuffle orders them for one
// coalesced store per batch (32 keys, 16 for d = 256).
#include "score_common.cuh"

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
    float stc[8], sts[8];  // e^{-i w NG}: from one key's rotation to the next one's in a batch
    if (PRE) phasors(T, -(int64_t)NG, stc, sts);
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
            batch_partials<PRE, U, NG>(kc, kpos, ok, c, T, stc, sts, part);
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

template <int ELEM, bool IL, int LPK>
static cudaError_t launch_score_d(const ScoreParams &p, int pre_rope, cudaStream_t s) {
    if (p.geo.layout == TRI_KV_PAGED)
        return pre_rope ? launch_score_t<true, true, ELEM, IL, LPK>(p, s) : launch_score_t<true, false, ELEM, IL, LPK>(p, s);
    return pre_rope ? launch_score_t<false, true, ELEM, IL, LPK>(p, s) : launch_score_t<false, false, ELEM, IL, LPK>(p, s);
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
