// Pre-RoPE key centres of every cache row ("TriAttention：基于三角函数 KV 压缩的高效
// 长推理", 流程详解 step 1: the pre-RoPE centres of Q and K; section 核心洞见: both
// cluster around fixed centres).  For the row of (layer, sequence, KV head) and
// pair f:
//   centre_f = (1/N) sum_j k_f^pre(j),   mean_norm_f = (1/N) sum_j |k_f(j)|,
// where a RoPE cache is de-rotated by each key's own position,
// k_f^pre = k_f^post e^{-i w_f pos}, with the phase w_f pos reduced exactly as a
// 64-bit fixed-point fraction of a turn (as the pre-RoPE scoring path does).
//
// Pass 1: kKeyCentreChunks CTAs per row, each streaming a contiguous slice of the
// row's keys with the scoring kernel's lane layout (d/16 lanes per key, 8 pairs
// per lane, U keys per lane in flight), summing each run of kFlush batches in
// fp32 and folding the run into fp64, and writing one partial (sum re, sum im,
// sum |k|) per pair.  Pass 2: one CTA per row adds its
// chunks' partials in chunk order and divides.  Both passes sum in a fixed order,
// so results are deterministic.  It reads every key once: an HBM-bound pass like
// the scoring one (plus one sin/cos per (key, pair) for a RoPE cache).
#include "score_common.cuh"

namespace tri {

constexpr int kKcThreads = 256;
constexpr double kKcTurnScale = 2.9358905032820014e+18;  // 2^64 / (2 pi)

constexpr int kFlush = 8;  // batches summed in fp32 before folding into fp64

// Each thread folds its fp32 runs into its own fp64 column of `acc` (element-major,
// so a warp's 8-byte accesses are consecutive); after the loop the CTA adds the
// columns of every pair in a fixed order.
template <bool PAGED, bool POST, int ELEM, bool IL, int LPK>
__global__ void __launch_bounds__(kKcThreads, 2) key_centre_kernel(const KeyCentreParams p) {
    constexpr int NG = 32 / LPK;
    constexpr int U = 4;
    constexpr int F = 8 * LPK;
    constexpr int RB = 2 * F * ELEM;
    constexpr int W = kKcThreads / 32;
    __shared__ double acc[24][kKcThreads];
    const Geometry &geo = p.geo;
    const int64_t r = blockIdx.x / kKeyCentreChunks;
    const int chunk = (int)(blockIdx.x % kKeyCentreChunks);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int q = lane / LPK, gl = lane % LPK;
    const int h = (int)(r % geo.H);
    const int s = (int)((r / geo.H) % geo.S);
    const int l = (int)(r / ((int64_t)geo.H * geo.S));
    int64_t lo = geo.row_off[r], hi = geo.row_off[r + 1];
    if (lo < 0 || hi < lo || hi > geo.total) {
        if (threadIdx.x == 0 && chunk == 0) atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
        lo = hi = 0;
    }
    const int64_t n = hi - lo;
    const int64_t beg = lo + n * chunk / kKeyCentreChunks;
    const int64_t end = lo + n * (chunk + 1) / kKeyCentreChunks;

    unsigned long long T[8];
#pragma unroll
    for (int i = 0; i < 8; i++)
        T[i] = POST ? __double2ull_rn(pow(p.theta, -2.0 * (double)(8 * gl + i) / (double)(2 * F)) * kKcTurnScale)
                    : 0ull;
    float stc[8], sts[8];  // e^{+i w NG}: from one key's rotation to the next one's in a batch
    if (POST) phasors(T, (int64_t)NG, stc, sts);
    const unsigned long long pol = policy_evict_first();
    const int32_t *table = geo.block_table + (int64_t)s * geo.max_blocks;
    const int64_t layer_blk = (int64_t)l * geo.n_blocks;

#pragma unroll
    for (int i = 0; i < 24; i++) acc[i][threadIdx.x] = 0.0;
    float fr[8], fi[8], fn[8];
#pragma unroll
    for (int i = 0; i < 8; i++) fr[i] = fi[i] = fn[i] = 0.f;

    int run = 0;
    for (int64_t b0 = beg + (int64_t)warp * NG * U; b0 < end; b0 += (int64_t)W * NG * U) {
        KeyChunk<ELEM, IL, F> kc[U];
        int64_t slot[U];
        int32_t kpos[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int64_t k = b0 + NG * u + q;
            slot[u] = -1;
            kpos[u] = 0;
            if (k < end) {
                if (PAGED) {
                    const int64_t j = k - lo, bi = j >> geo.block_shift;
                    const int32_t blk = bi < geo.max_blocks ? __ldg(table + bi) : -1;
                    if (blk >= 0 && blk < geo.n_blocks)
                        slot[u] = ((((layer_blk + blk) << geo.block_shift) | (j & ((1 << geo.block_shift) - 1))) *
                                   geo.H) + h;
                    else if (gl == 0)
                        atomicOr(p.flags, TRI_FLAG_BLOCK_TABLE);
                } else {
                    slot[u] = k;
                }
            }
            if (slot[u] >= 0) {
                kc[u].load(p.K + slot[u] * RB, gl, pol);
                if (POST) kpos[u] = __ldg(p.pos + slot[u]);
            } else {
                kc[u].zero();
            }
        }
        // Rotation phasors e^{i w pos} of the lane's keys: the first from its reduced
        // phase, each next one by one complex step when positions advance by NG.
        float cs[8], sn[8];
        if (POST) phasors(T, (int64_t)kpos[0], cs, sn);
#pragma unroll
        for (int u = 0; u < U; u++) {
            if (POST && u > 0) {
                if (kpos[u] == kpos[u - 1] + NG) advance_phasors(cs, sn, stc, sts);
                else phasors(T, (int64_t)kpos[u], cs, sn);
            }
            if (slot[u] < 0) continue;
            float x[8], y[8];
            kc[u].unpack(x, y);
#pragma unroll
            for (int i = 0; i < 8; i++) {
                float xr = x[i], xi = y[i];
                if (POST) {
                    xr = x[i] * cs[i] + y[i] * sn[i];
                    xi = y[i] * cs[i] - x[i] * sn[i];
                }
                fr[i] += xr;
                fi[i] += xi;
                fn[i] += sqrt_approx(fmaf(x[i], x[i], y[i] * y[i]));
            }
        }
        if (++run == kFlush) {
            run = 0;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                acc[i][threadIdx.x] += (double)fr[i];
                acc[8 + i][threadIdx.x] += (double)fi[i];
                acc[16 + i][threadIdx.x] += (double)fn[i];
                fr[i] = fi[i] = fn[i] = 0.f;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; i++) {
        acc[i][threadIdx.x] += (double)fr[i];
        acc[8 + i][threadIdx.x] += (double)fi[i];
        acc[16 + i][threadIdx.x] += (double)fn[i];
    }
    __syncthreads();
    // Pair f = 8 gl + i lives in the columns of the threads with that gl (every warp,
    // every key group): add them in thread order.
    for (int e = threadIdx.x; e < 3 * F; e += kKcThreads) {
        const int f = e % F, comp = e / F;
        const int g = f >> 3, i = f & 7;
        double v = 0.0;
        for (int t = g; t < kKcThreads; t += LPK) v += acc[comp * 8 + i][t];
        p.partial[((r * kKeyCentreChunks + chunk) * F + f) * 3 + comp] = v;
    }
}

template <int F>
__global__ void __launch_bounds__(F) key_centre_finalize(const KeyCentreParams p) {
    const int64_t r = blockIdx.x;
    const int f = threadIdx.x;
    int64_t n = p.geo.row_off[r + 1] - p.geo.row_off[r];
    if (p.geo.row_off[r] < 0 || n < 0 || p.geo.row_off[r + 1] > p.geo.total) n = 0;
    double a = 0.0, b = 0.0, c = 0.0;
    for (int k = 0; k < kKeyCentreChunks; k++) {
        const double *in = p.partial + ((r * kKeyCentreChunks + k) * F + f) * 3;
        a += in[0];
        b += in[1];
        c += in[2];
    }
    const double inv = n > 0 ? 1.0 / (double)n : 0.0;
    p.centres[(r * F + f) * 2] = (float)(a * inv);
    p.centres[(r * F + f) * 2 + 1] = (float)(b * inv);
    p.mean_norm[r * F + f] = (float)(c * inv);
}

template <bool PAGED, bool POST, int ELEM, bool IL, int LPK>
static cudaError_t launch_kc_t(const KeyCentreParams &p, int64_t R, cudaStream_t s) {
    key_centre_kernel<PAGED, POST, ELEM, IL, LPK><<<(unsigned)(R * kKeyCentreChunks), kKcThreads, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    key_centre_finalize<8 * LPK><<<(unsigned)R, 8 * LPK, 0, s>>>(p);
    return cudaGetLastError();
}

template <int ELEM, bool IL, int LPK>
static cudaError_t launch_kc_d(const KeyCentreParams &p, int64_t R, cudaStream_t s) {
    const bool paged = p.geo.layout == TRI_KV_PAGED;
    if (paged) return p.post_rope ? launch_kc_t<true, true, ELEM, IL, LPK>(p, R, s) : launch_kc_t<true, false, ELEM, IL, LPK>(p, R, s);
    return p.post_rope ? launch_kc_t<false, true, ELEM, IL, LPK>(p, R, s) : launch_kc_t<false, false, ELEM, IL, LPK>(p, R, s);
}

template <int ELEM, bool IL>
static cudaError_t launch_kc_l(const KeyCentreParams &p, int64_t R, cudaStream_t s) {
    switch (p.geo.D) {
        case 64: return launch_kc_d<ELEM, IL, 4>(p, R, s);
        case 128: return launch_kc_d<ELEM, IL, 8>(p, R, s);
        case 256: return launch_kc_d<ELEM, IL, 16>(p, R, s);
    }
    return cudaErrorInvalidValue;
}

template <int ELEM>
static cudaError_t launch_kc_e(const KeyCentreParams &p, int64_t R, cudaStream_t s) {
    return p.geo.il ? launch_kc_l<ELEM, true>(p, R, s) : launch_kc_l<ELEM, false>(p, R, s);
}

cudaError_t launch_key_centres(const KeyCentreParams &p, cudaStream_t s) {
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    if (R * kKeyCentreChunks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return p.geo.elem_bytes == 1 ? launch_kc_e<1>(p, R, s) : launch_kc_e<2>(p, R, s);
}

}  // namespace tri
