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
// the scoring one.
//
// RoPE caches: the de-rotated sum of a lane's keys is accumulated in Horner form
// along the lane's keys, H = sum_i k_i e^{i w (p - p_i)} with p the position of
// the lane's last key, so a key whose position is a fixed step D past the last
// one costs H <- H e^{i w D} + k: one complex multiply-add per pair, with two
// constant steps (the next key of a lane's batch, NG positions on, and the first
// key of the lane's next batch).  Any other key, and the end of every run of
// kFlush batches, first settles H into the run sums as H e^{-i w p} (one sin/cos
// per pair of the exactly reduced phase) and restarts it.
#include "score_common.cuh"
#include "stage.cuh"

namespace tri {

constexpr int kKcThreads = 256;
constexpr double kKcTurnScale = 2.9358905032820014e+18;  // 2^64 / (2 pi)

constexpr int kFlush = 8;  // batches summed in fp32 before folding into fp64

// Turn rates T_f = w_f / 2 pi in 0.64 fixed point, w_f = theta^(-2f/d), of the F
// pairs into t[f]: one fp64 power per pair, by the block's first F threads.
template <int F>
__device__ __forceinline__ void kc_turns(double theta, unsigned long long *t) {
    for (int f = threadIdx.x; f < F; f += blockDim.x)
        t[f] = __double2ull_rn(pow(theta, -2.0 * (double)f / (double)(2 * F)) * kKcTurnScale);
}

// e^{i w delta} of the lane's 8 pairs, two pairs per register: C = cos, S = sin, NS = -sin.
__device__ __forceinline__ void kc_step(const unsigned long long (&T)[8], int64_t delta, unsigned long long (&C)[4],
                                        unsigned long long (&S)[4], unsigned long long (&NS)[4]) {
    float cs[8], sn[8];
    phasors(T, delta, cs, sn);
#pragma unroll
    for (int k = 0; k < 4; k++) {
        C[k] = f2(cs[2 * k], cs[2 * k + 1]);
        S[k] = f2(sn[2 * k], sn[2 * k + 1]);
        NS[k] = neg2(S[k]);
    }
}

// Settles the Horner sum H (relative to position p) into the run sums,
// fr + i fi += H e^{-i w p}, and clears it.  Tg: the lane group's 8 turn rates in
// shared memory (read only here, so they hold no registers in the key loop).
__device__ __forceinline__ void kc_settle(const unsigned long long *Tg, int32_t p, unsigned long long (&HR)[4],
                                          unsigned long long (&HI)[4], unsigned long long (&fr)[4],
                                          unsigned long long (&fi)[4]) {
    unsigned long long T[8];
#pragma unroll
    for (int i = 0; i < 8; i++) T[i] = Tg[i];
    float cs[8], sn[8];
    phasors(T, (int64_t)p, cs, sn);
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const unsigned long long CS = f2(cs[2 * k], cs[2 * k + 1]), SN = f2(sn[2 * k], sn[2 * k + 1]);
        fr[k] = add2(fr[k], fma2(HR[k], CS, mul2(HI[k], SN)));        // HR cos + HI sin
        fi[k] = add2(fi[k], fma2(HI[k], CS, mul2(neg2(HR[k]), SN)));  // HI cos - HR sin
        HR[k] = HI[k] = 0ull;
    }
}

// H <- H e^{i w D} + (X + i Y) for the step (C, S, NS) of D, two pairs per register.
__device__ __forceinline__ void kc_horner(unsigned long long (&HR)[4], unsigned long long (&HI)[4], int k,
                                          unsigned long long X, unsigned long long Y, const unsigned long long (&C)[4],
                                          const unsigned long long (&S)[4], const unsigned long long (&NS)[4]) {
    const unsigned long long re = fma2(HR[k], C[k], fma2(HI[k], NS[k], X));
    HI[k] = fma2(HR[k], S[k], fma2(HI[k], C[k], Y));
    HR[k] = re;
}

// Each run of kFlush batches is folded in fp64 across the lanes of a warp that
// hold the same pairs (a fixed shuffle tree) into one column per (warp, lane
// group); after the loop the CTA adds the columns of every pair in warp order.
template <bool PAGED, bool POST, int ELEM, bool IL, int LPK>
__global__ void __launch_bounds__(kKcThreads, 2) key_centre_kernel(const KeyCentreParams p) {
    constexpr int NG = 32 / LPK;
    constexpr int U = 4;
    constexpr int F = 8 * LPK;
    constexpr int RB = 2 * F * ELEM;
    constexpr int W = kKcThreads / 32;
    __shared__ double acc[24 * W * LPK];          // [24][W * LPK]: one column per (warp, lane group)
    __shared__ unsigned long long t_sm[8 * LPK];  // turn rates of the pairs, [gl][i]
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

    if (POST) kc_turns<F>(p.theta, t_sm);
    for (int e = threadIdx.x; e < 24 * W * LPK; e += kKcThreads) acc[e] = 0.0;
    __syncthreads();  // t_sm and acc written
    const unsigned long long *Tg = t_sm + 8 * gl;
    // Horner steps: the lane's next key in a batch (NG positions on) and the first
    // key of its next batch (W KB - (U - 1) NG positions after the batch's last).
    constexpr int DB = W * NG * U - (U - 1) * NG;
    unsigned long long ZC[4], ZS[4], ZN[4], BC[4], BS[4], BN[4];
    if (POST) {
        unsigned long long T[8];
#pragma unroll
        for (int i = 0; i < 8; i++) T[i] = Tg[i];
        kc_step(T, NG, ZC, ZS, ZN);
        kc_step(T, DB, BC, BS, BN);
    }
    const unsigned long long pol = policy_evict_first();
    const int32_t *table = geo.block_table + (int64_t)s * geo.max_blocks;
    const int64_t layer_blk = (int64_t)l * geo.n_blocks;
    unsigned long long fr2[4], fi2[4], fn2[4], HR[4], HI[4];  // pairs (2k, 2k+1) packed
#pragma unroll
    for (int i = 0; i < 4; i++) fr2[i] = fi2[i] = fn2[i] = HR[i] = HI[i] = 0ull;
    int32_t plast = 0;  // position of the lane's last key (H is relative to it)
    // Adds the lanes' runs into this warp's columns: fp64 tree over the NG lanes
    // of each lane group, then lane group gl's column.
    auto flush = [&]() {
        if (POST) kc_settle(Tg, plast, HR, HI, fr2, fi2);
#pragma unroll
        for (int c3 = 0; c3 < 3; c3++)
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float2 pr = f2split(c3 == 0 ? fr2[i >> 1] : c3 == 1 ? fi2[i >> 1] : fn2[i >> 1]);
                double v = (double)((i & 1) ? pr.y : pr.x);
#pragma unroll
                for (int o = LPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (q == 0) acc[(c3 * 8 + i) * (W * LPK) + warp * LPK + gl] += v;
            }
#pragma unroll
        for (int i = 0; i < 4; i++) fr2[i] = fi2[i] = fn2[i] = 0ull;
    };

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
#pragma unroll
        for (int u = 0; u < U; u++) {
            if (slot[u] < 0) continue;
            float x[8], y[8];
            kc[u].unpack(x, y);
            if (POST && !pos_follows(kpos[u], plast, u == 0 ? DB : NG)) kc_settle(Tg, plast, HR, HI, fr2, fi2);
#pragma unroll
            for (int k2 = 0; k2 < 4; k2++) {
                const unsigned long long X = f2(x[2 * k2], x[2 * k2 + 1]), Y = f2(y[2 * k2], y[2 * k2 + 1]);
                if (POST) {
                    if (u == 0) kc_horner(HR, HI, k2, X, Y, BC, BS, BN);
                    else kc_horner(HR, HI, k2, X, Y, ZC, ZS, ZN);
                } else {
                    fr2[k2] = add2(fr2[k2], X);
                    fi2[k2] = add2(fi2[k2], Y);
                }
                const float2 qq = f2split(fma2(X, X, mul2(Y, Y)));
                fn2[k2] = add2(fn2[k2], f2(sqrt_approx(qq.x), sqrt_approx(qq.y)));
            }
            if (POST) plast = kpos[u];
        }
        if (++run == kFlush) {
            run = 0;
            flush();
        }
    }
    flush();
    __syncthreads();
    // Pair f = 8 gl + i lives in the column of lane group gl of every warp: add
    // them in warp order.
    for (int e = threadIdx.x; e < 3 * F; e += kKcThreads) {
        const int f = e % F, comp = e / F;
        const int g = f >> 3, i = f & 7;
        double v = 0.0;
        for (int w = 0; w < W; w++) v += acc[(comp * 8 + i) * (W * LPK) + w * LPK + g];
        p.partial[((r * kKeyCentreChunks + chunk) * F + f) * 3 + comp] = v;
    }
}

// Contiguous caches: the same pass with each warp's batches staged in shared
// memory by bulk copies, STAGES batches ahead (see stage.cuh), so the bytes in
// flight do not depend on registers.  A chunk may start at any key, so each
// batch also stages the 16-byte-aligned window of positions around its keys.
// To leave room for the ring, a flush folds the lanes' fp32 runs in fp64
// across the lanes of the warp that hold the same pairs (a fixed shuffle
// tree) into one column per (warp, lane group); the final sum runs over warps
// in order.  Deterministic, like the unstaged pass.
template <bool POST, int ELEM, int LPK>
struct KcStaging {
    static constexpr int kWarps = kKcThreads / 32;
    static constexpr int NG = 32 / LPK, U = 4, KB = NG * U, F = 8 * LPK;
    static constexpr int RB = 2 * F * ELEM;
    static constexpr int KEY_BYTES = KB * RB;
    static constexpr int POS_CAP = POST ? KB + 4 : 0;  // aligned window of a batch's positions
    static constexpr int SLOT = KEY_BYTES + POS_CAP * 4;
    static constexpr int ACC_BYTES = 24 * kWarps * LPK * 8;
    static constexpr int HEADER = 256;  // the barriers (at most 8 warps x 4 stages)
    // Two CTAs per SM: 228 KB less 1 KB reserved per CTA.
    static constexpr int PER_CTA = (228 * 1024 - 2 * 1024) / 2;
    static constexpr int FIT = (PER_CTA - ACC_BYTES - HEADER) / (kWarps * SLOT);
    static constexpr int STAGES = FIT < 2 ? 2 : (FIT > 4 ? 4 : FIT);
    static constexpr size_t SMEM = (size_t)HEADER + ACC_BYTES + (size_t)kWarps * STAGES * SLOT;
    static_assert(KB % 4 == 0 && SLOT % 16 == 0 && KEY_BYTES % 16 == 0 && ACC_BYTES % 16 == 0, "16-byte units");
    static_assert(kWarps * STAGES * 8 <= HEADER, "barriers fit the header");
    static_assert(2 * (SMEM + 8 * 8 * LPK + 1024) <= 228 * 1024, "two CTAs per SM");
};

// Issues batch t of a warp (keys b0 .. b0 + n - 1) into slot t % STAGES: its
// records, and the positions [a0, a1) of the 16-byte-aligned window around
// them that lies inside the array.  One thread per warp.
template <typename St>
__device__ __forceinline__ void kc_stage_batch(const KeyCentreParams &p, int64_t b0, int n, unsigned char *ring,
                                               uint64_t *bar, int t, unsigned long long pol) {
    unsigned char *slot = ring + (t % St::STAGES) * St::SLOT;
    uint64_t *b = &bar[t % St::STAGES];
    const uint32_t kbytes = (uint32_t)n * St::RB;
    uint32_t pbytes = 0;
    int64_t a0 = 0;
    if (St::POS_CAP) {
        a0 = b0 & ~int64_t(3);
        const int64_t a1 = min((b0 + n + 3) & ~int64_t(3), p.geo.total & ~int64_t(3));
        if (a1 > a0) pbytes = (uint32_t)(a1 - a0) * 4u;
    }
    mbar_arrive_expect_tx(b, kbytes + pbytes);
    bulk_load(slot, p.K + b0 * St::RB, kbytes, b, pol);
    if (pbytes) bulk_load(slot + St::KEY_BYTES, p.pos + a0, pbytes, b, pol);
}

template <bool POST, int ELEM, bool IL, int LPK>
__global__ void __launch_bounds__(kKcThreads, 2) key_centre_staged_kernel(const KeyCentreParams p) {
    using St = KcStaging<POST, ELEM, LPK>;
    constexpr int NG = St::NG, U = St::U, KB = St::KB, F = St::F, RB = St::RB, W = St::kWarps;
    constexpr int STAGES = St::STAGES;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ unsigned long long t_sm[8 * LPK];  // turn rates of the pairs, [gl][i]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    double *acc = reinterpret_cast<double *>(smem + St::HEADER);  // [24][W * LPK]
    unsigned char *rings = smem + St::HEADER + St::ACC_BYTES;
    const Geometry &geo = p.geo;
    const int64_t r = blockIdx.x / kKeyCentreChunks;
    const int chunk = (int)(blockIdx.x % kKeyCentreChunks);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int q = lane / LPK, gl = lane % LPK;
    int64_t lo = geo.row_off[r], hi = geo.row_off[r + 1];
    if (lo < 0 || hi < lo || hi > geo.total) {
        if (threadIdx.x == 0 && chunk == 0) atomicOr(p.flags, TRI_FLAG_ROW_OFFSETS);
        lo = hi = 0;
    }
    const int64_t n = hi - lo;
    const int64_t beg = lo + n * chunk / kKeyCentreChunks;
    const int64_t end = lo + n * (chunk + 1) / kKeyCentreChunks;
    // This warp's batches: keys beg + (warp + t W) KB ..., t = 0 .. nbw - 1.
    const int64_t first0 = beg + (int64_t)warp * KB;
    const int nbw = first0 < end ? (int)((end - first0 + (int64_t)W * KB - 1) / ((int64_t)W * KB)) : 0;

    const unsigned long long pol = policy_evict_first();
    uint64_t *bar = bars + warp * STAGES;
    unsigned char *ring = rings + (size_t)warp * STAGES * St::SLOT;

    if (POST) kc_turns<F>(p.theta, t_sm);
    for (int e = threadIdx.x; e < 24 * W * LPK; e += kKcThreads) acc[e] = 0.0;
    if (lane == 0) {
#pragma unroll
        for (int k = 0; k < STAGES; k++) mbar_init(&bar[k], 1);
        mbar_init_fence();
    }
    __syncthreads();  // t_sm, acc and the barriers are ready
    const unsigned long long *Tg = t_sm + 8 * gl;
    constexpr int DB = W * KB - (U - 1) * NG;  // a lane's last key of a batch -> its first of the next
    unsigned long long ZC[4], ZS[4], ZN[4], BC[4], BS[4], BN[4];
    if (POST) {
        unsigned long long T[8];
#pragma unroll
        for (int i = 0; i < 8; i++) T[i] = Tg[i];
        kc_step(T, NG, ZC, ZS, ZN);
        kc_step(T, DB, BC, BS, BN);
    }
    if (lane == 0)
        for (int t = 0; t < min(nbw, STAGES); t++) {
            const int64_t b0 = first0 + (int64_t)t * W * KB;
            kc_stage_batch<St>(p, b0, (int)min((int64_t)KB, end - b0), ring, bar, t, pol);
        }

    unsigned long long fr2[4], fi2[4], fn2[4], HR[4], HI[4];  // fp32 runs, pairs (2k, 2k+1) packed
#pragma unroll
    for (int i = 0; i < 4; i++) fr2[i] = fi2[i] = fn2[i] = HR[i] = HI[i] = 0ull;
    int32_t plast = 0;  // position of the lane's last key (H is relative to it)
    // Adds the lanes' runs into this warp's columns: fp64 tree over the NG lanes
    // of each lane group, then lane group gl's column.
    auto fold = [&]() {
        if (POST) kc_settle(Tg, plast, HR, HI, fr2, fi2);
#pragma unroll
        for (int c3 = 0; c3 < 3; c3++)
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const float2 pr = f2split(c3 == 0 ? fr2[i >> 1] : c3 == 1 ? fi2[i >> 1] : fn2[i >> 1]);
                double v = (double)((i & 1) ? pr.y : pr.x);
#pragma unroll
                for (int o = LPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (q == 0) acc[(c3 * 8 + i) * (W * LPK) + warp * LPK + gl] += v;
            }
#pragma unroll
        for (int i = 0; i < 4; i++) fr2[i] = fi2[i] = fn2[i] = 0ull;
    };

    int run = 0;
    for (int t = 0; t < nbw; t++) {
        const int64_t b0 = first0 + (int64_t)t * W * KB;
        const int nk = (int)min((int64_t)KB, end - b0);
        if (!__all_sync(0xffffffffu, mbar_wait(&bar[t % STAGES], (uint32_t)(t / STAGES) & 1u))) {
            // A copy did not land: flag it, wait once more (bounded) for every copy
            // still in flight into this warp's ring, and skip the warp's other keys.
            if (lane == 0) atomicOr(p.flags, TRI_FLAG_STAGE_TIMEOUT);
            for (int j = t; j < min(nbw, t + STAGES); j++) mbar_wait(&bar[j % STAGES], (uint32_t)(j / STAGES) & 1u);
            break;
        }
        const unsigned char *slot = ring + (t % STAGES) * St::SLOT;
        const int32_t *spos = reinterpret_cast<const int32_t *>(slot + St::KEY_BYTES);
        const int64_t a0 = b0 & ~int64_t(3);
        const int64_t a1 = POST ? min((b0 + nk + 3) & ~int64_t(3), geo.total & ~int64_t(3)) : 0;
        int32_t kpos[U];
        bool valid[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int idx = NG * u + q;
            const int64_t k = b0 + idx;
            valid[u] = idx < nk;
            kpos[u] = 0;
            if (valid[u] && POST) kpos[u] = k < a1 ? spos[k - a0] : __ldg(p.pos + k);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            if (!valid[u]) continue;
            KeyChunk<ELEM, IL, F> kc;  // read from the slot as it is used
            kc.lds(slot + (NG * u + q) * RB, gl);
            float x[8], y[8];
            kc.unpack(x, y);
            if (POST && !pos_follows(kpos[u], plast, u == 0 ? DB : NG)) kc_settle(Tg, plast, HR, HI, fr2, fi2);
            // Two pairs per packed instruction: the Horner step (RoPE caches) or
            // the plain sums, and the magnitudes.
#pragma unroll
            for (int k2 = 0; k2 < 4; k2++) {
                const unsigned long long X = f2(x[2 * k2], x[2 * k2 + 1]), Y = f2(y[2 * k2], y[2 * k2 + 1]);
                if (POST) {
                    if (u == 0) kc_horner(HR, HI, k2, X, Y, BC, BS, BN);
                    else kc_horner(HR, HI, k2, X, Y, ZC, ZS, ZN);
                } else {
                    fr2[k2] = add2(fr2[k2], X);
                    fi2[k2] = add2(fi2[k2], Y);
                }
                const float2 qq = f2split(fma2(X, X, mul2(Y, Y)));
                fn2[k2] = add2(fn2[k2], f2(sqrt_approx(qq.x), sqrt_approx(qq.y)));
            }
            if (POST) plast = kpos[u];
        }
        if (t + STAGES < nbw) {  // the slot's bytes are consumed: refill it
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int64_t bn = first0 + (int64_t)(t + STAGES) * W * KB;
                kc_stage_batch<St>(p, bn, (int)min((int64_t)KB, end - bn), ring, bar, t + STAGES, pol);
            }
        }
        if (++run == kFlush) {
            run = 0;
            fold();
        }
    }
    fold();
    __syncthreads();
    for (int e = threadIdx.x; e < 3 * F; e += kKcThreads) {
        const int f = e % F, comp = e / F;
        const int g = f >> 3, i = f & 7;
        double v = 0.0;
        for (int w = 0; w < W; w++) v += acc[(comp * 8 + i) * (W * LPK) + w * LPK + g];
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

template <bool POST, int ELEM, bool IL, int LPK>
static cudaError_t launch_kc_staged_t(const KeyCentreParams &p, int64_t R, cudaStream_t s) {
    using St = KcStaging<POST, ELEM, LPK>;
    auto kern = key_centre_staged_kernel<POST, ELEM, IL, LPK>;
    static bool set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!set[dev & 63]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)St::SMEM);
        if (e != cudaSuccess) return e;
        set[dev & 63] = true;
    }
    kern<<<(unsigned)(R * kKeyCentreChunks), kKcThreads, St::SMEM, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    key_centre_finalize<8 * LPK><<<(unsigned)R, 8 * LPK, 0, s>>>(p);
    return cudaGetLastError();
}

template <int ELEM, bool IL, int LPK>
static cudaError_t launch_kc_d(const KeyCentreParams &p, int64_t R, cudaStream_t s) {
    const bool paged = p.geo.layout == TRI_KV_PAGED;
    if (paged) return p.post_rope ? launch_kc_t<true, true, ELEM, IL, LPK>(p, R, s) : launch_kc_t<true, false, ELEM, IL, LPK>(p, R, s);
    return p.post_rope ? launch_kc_staged_t<true, ELEM, IL, LPK>(p, R, s) : launch_kc_staged_t<false, ELEM, IL, LPK>(p, R, s);
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
