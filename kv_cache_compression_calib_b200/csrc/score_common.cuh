// Per-key scoring pieces shared by the streaming score kernel and the fused
// score-and-select kernel: row context, record addressing, the per-lane partial
// sums for post- and pre-RoPE caches, and the compile-time lane layout.
#pragma once

#include "keys.cuh"

namespace tri {

struct RowCtx {
    int r;
    int64_t lo, hi;
    // paged addressing
    const int32_t *table;
    int64_t layer_blk;  // l * n_blocks
    int h;
    int64_t p_now;
    float ar[8], ai[8], cc[8];
};

// Row context of row r with lane group gl's 24 coefficients at `cg` (global or
// shared memory, 16-byte aligned).
__device__ __forceinline__ void set_row_coef(RowCtx &c, const ScoreParams &p, int r, int gl, const float *cg) {
    const Geometry &geo = p.geo;
    c.r = r;
    c.lo = geo.row_off[r];
    c.hi = geo.row_off[r + 1];
    const int h = r % geo.H;
    const int s = (r / geo.H) % geo.S;
    const int l = r / (geo.H * geo.S);
    c.h = h;
    c.table = geo.block_table + (int64_t)s * geo.max_blocks;
    c.layer_blk = (int64_t)l * geo.n_blocks;
    c.p_now = p.p_now[s];
    const float4 *cp = reinterpret_cast<const float4 *>(cg);
    const float4 v0 = cp[0], v1 = cp[1], v2 = cp[2], v3 = cp[3], v4 = cp[4], v5 = cp[5];
    c.ar[0] = v0.x; c.ar[1] = v0.y; c.ar[2] = v0.z; c.ar[3] = v0.w;
    c.ar[4] = v1.x; c.ar[5] = v1.y; c.ar[6] = v1.z; c.ar[7] = v1.w;
    c.ai[0] = v2.x; c.ai[1] = v2.y; c.ai[2] = v2.z; c.ai[3] = v2.w;
    c.ai[4] = v3.x; c.ai[5] = v3.y; c.ai[6] = v3.z; c.ai[7] = v3.w;
    c.cc[0] = v4.x; c.cc[1] = v4.y; c.cc[2] = v4.z; c.cc[3] = v4.w;
    c.cc[4] = v5.x; c.cc[5] = v5.y; c.cc[6] = v5.z; c.cc[7] = v5.w;
}

__device__ __forceinline__ void set_row(RowCtx &c, const ScoreParams &p, int r, int gl, int coef_per_row) {
    set_row_coef(c, p, r, gl, p.coef + (int64_t)r * coef_per_row + gl * kCoefPerGroup);
}

// Slot index (in units of one (slot, head) record) of global key k in row c,
// or -1 if the paged table cannot place it.
template <bool PAGED>
__device__ __forceinline__ int64_t key_slot(const ScoreParams &p, const RowCtx &c, int64_t k) {
    if (!PAGED) return k;
    const Geometry &geo = p.geo;
    const int64_t j = k - c.lo;
    const int64_t bi = j >> geo.block_shift;
    if (j < 0 || bi >= geo.max_blocks) return -1;
    const int32_t blk = __ldg(c.table + bi);
    if (blk < 0 || blk >= geo.n_blocks) return -1;
    return ((((c.layer_blk + blk) << geo.block_shift) | (j & ((1 << geo.block_shift) - 1))) * geo.H) + c.h;
}

// Partial score of 8 pairs: sum_i Re(A_i conj k_i) + c_i |k_i|.
// Two fp32 lanes in one 64-bit register pair, for the packed fp32 instructions of
// sm_100 (fma/mul .rn.f32x2: each lane rounds exactly as the scalar instruction).
__device__ __forceinline__ unsigned long long f2(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 f2split(unsigned long long r) {
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// Both lanes negated (sign bits flipped: exact).
__device__ __forceinline__ unsigned long long neg2(unsigned long long a) { return a ^ 0x8000000080000000ull; }
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The same two-lane operations as scalar fp32 instructions on the register pair's
// halves (each rounds exactly as the packed form, so the results are the same
// bits), for the pre-RoPE steps, where the compiler can then fold sign flips
// into the multiply-adds.
__device__ __forceinline__ unsigned long long fma2s(unsigned long long a, unsigned long long b, unsigned long long c) {
    const float2 A = f2split(a), B = f2split(b), C = f2split(c);
    return f2(__fmaf_rn(A.x, B.x, C.x), __fmaf_rn(A.y, B.y, C.y));
}
__device__ __forceinline__ unsigned long long mul2s(unsigned long long a, unsigned long long b) {
    const float2 A = f2split(a), B = f2split(b);
    return f2(__fmul_rn(A.x, B.x), __fmul_rn(A.y, B.y));
}

// Partial score of 8 pairs: sum_i Re(A_i conj k_i) + c_i |k_i|, two pairs (i, i+1)
// per packed instruction: the dot product and the squared norms in f32x2, one
// square root per pair.
__device__ __forceinline__ float partial_post(const float (&x)[8], const float (&y)[8], const RowCtx &c) {
    unsigned long long d = 0ull, e = 0ull;  // (even, odd) lanes of the dot product and the norm term
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const unsigned long long X = f2(x[2 * k], x[2 * k + 1]), Y = f2(y[2 * k], y[2 * k + 1]);
        d = fma2(f2(c.ar[2 * k], c.ar[2 * k + 1]), X, d);
        d = fma2(f2(c.ai[2 * k], c.ai[2 * k + 1]), Y, d);
        const float2 q = f2split(fma2(X, X, mul2(Y, Y)));
        e = fma2(f2(c.cc[2 * k], c.cc[2 * k + 1]), f2(sqrt_approx(q.x), sqrt_approx(q.y)), e);
    }
    const float2 dd = f2split(d), ee = f2split(e);
    return (dd.x + dd.y) + (ee.x + ee.y);
}

// Pre-RoPE cache: rotate A'_i by w_i (p_now - pos) first.  The phase in turns
// is (delta * T_i) mod 2^64 with T_i = w_i / 2pi in 0.64 fixed point; its top
// 23 bits, read as signed, give the angle in [-pi, pi).
__device__ __forceinline__ void phasors(const unsigned long long (&T)[8], int64_t delta, float (&cs)[8],
                                        float (&sn)[8]) {
#pragma unroll
    for (int i = 0; i < 8; i++)
        __sincosf(turn_units23((unsigned long long)delta * T[i]) * kTurn23ToRad, &sn[i], &cs[i]);
}

// Partial score of a pre-RoPE key given its rotation phasors e^{i w_i delta}: the
// rotation, the dot product and the squared norms two pairs per packed instruction.
__device__ __forceinline__ float partial_pre_rot(const float (&x)[8], const float (&y)[8], const RowCtx &c,
                                                 const float (&cs)[8], const float (&sn)[8]) {
    unsigned long long d = 0ull, e = 0ull;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const unsigned long long AR = f2(c.ar[2 * k], c.ar[2 * k + 1]), AI = f2(c.ai[2 * k], c.ai[2 * k + 1]);
        const unsigned long long CS = f2(cs[2 * k], cs[2 * k + 1]), SN = f2(sn[2 * k], sn[2 * k + 1]);
        const unsigned long long BR = fma2(AR, CS, mul2(f2(-c.ai[2 * k], -c.ai[2 * k + 1]), SN));
        const unsigned long long BI = fma2(AR, SN, mul2(AI, CS));
        const unsigned long long X = f2(x[2 * k], x[2 * k + 1]), Y = f2(y[2 * k], y[2 * k + 1]);
        d = fma2(BR, X, d);
        d = fma2(BI, Y, d);
        const float2 q = f2split(fma2(X, X, mul2(Y, Y)));
        e = fma2(f2(c.cc[2 * k], c.cc[2 * k + 1]), f2(sqrt_approx(q.x), sqrt_approx(q.y)), e);
    }
    const float2 dd = f2split(d), ee = f2split(e);
    return (dd.x + dd.y) + (ee.x + ee.y);
}

__device__ __forceinline__ float partial_pre(const float (&x)[8], const float (&y)[8], const RowCtx &c,
                                             const unsigned long long (&T)[8], int64_t delta) {
    float cs[8], sn[8];
    phasors(T, delta, cs, sn);
    return partial_pre_rot(x, y, c, cs, sn);
}

// The step e^{-i w NG} from one key of a lane's batch to the next (pre-RoPE),
// two pairs per register: TC = cos, TS = sin.
__device__ __forceinline__ void step_phasors(const unsigned long long (&T)[8], int NG, unsigned long long (&TC)[4],
                                             unsigned long long (&TS)[4]) {
    float cs[8], sn[8];
    phasors(T, -(int64_t)NG, cs, sn);
#pragma unroll
    for (int k = 0; k < 4; k++) {
        TC[k] = f2(cs[2 * k], cs[2 * k + 1]);
        TS[k] = f2(sn[2 * k], sn[2 * k + 1]);
    }
}

// Pre-RoPE, rotated coefficients of 8 pairs, two pairs per register:
// B_i = A'_i (cs_i + i sn_i), formed exactly as partial_pre_rot forms them.
__device__ __forceinline__ void rotate_coef(const RowCtx &c, const float (&cs)[8], const float (&sn)[8],
                                            unsigned long long (&BR)[4], unsigned long long (&BI)[4]) {
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const unsigned long long AR = f2(c.ar[2 * k], c.ar[2 * k + 1]), AI = f2(c.ai[2 * k], c.ai[2 * k + 1]);
        const unsigned long long CS = f2(cs[2 * k], cs[2 * k + 1]), SN = f2(sn[2 * k], sn[2 * k + 1]);
        BR[k] = fma2s(AR, CS, mul2s(neg2(AI), SN));
        BI[k] = fma2s(AR, SN, mul2s(AI, CS));
    }
}

// B <- B * e^{-i w NG} (TC, TS the step's cos and sin): the rotated
// coefficients of the key NG slots further on.
__device__ __forceinline__ void advance_coef(unsigned long long (&BR)[4], unsigned long long (&BI)[4],
                                             const unsigned long long (&TC)[4], const unsigned long long (&TS)[4]) {
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const unsigned long long r = fma2s(BR[k], TC[k], mul2s(BI[k], neg2(TS[k])));
        BI[k] = fma2s(BR[k], TS[k], mul2s(BI[k], TC[k]));
        BR[k] = r;
    }
}

// Partial score of 8 pre-RoPE pairs given their rotated coefficients: the dot
// product and the norm term in the order of partial_pre_rot.
__device__ __forceinline__ float partial_rotated(const float (&x)[8], const float (&y)[8],
                                                 const unsigned long long (&BR)[4],
                                                 const unsigned long long (&BI)[4], const RowCtx &c) {
    unsigned long long d = 0ull, e = 0ull;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const unsigned long long X = f2(x[2 * k], x[2 * k + 1]), Y = f2(y[2 * k], y[2 * k + 1]);
        d = fma2s(BR[k], X, d);
        d = fma2s(BI[k], Y, d);
        const float2 q = f2split(fma2s(X, X, mul2s(Y, Y)));
        e = fma2s(f2(c.cc[2 * k], c.cc[2 * k + 1]), f2(sqrt_approx(q.x), sqrt_approx(q.y)), e);
    }
    const float2 dd = f2split(d), ee = f2split(e);
    return (dd.x + dd.y) + (ee.x + ee.y);
}

// True when position `pos` lies exactly `step` past `last` (positions are int32:
// no wrap-around across the int32 range counts as a step).
__device__ __forceinline__ bool pos_follows(int32_t pos, int32_t last, int step) {
    return pos > last && (uint32_t)pos - (uint32_t)last == (uint32_t)step;
}

// Pre-RoPE partials of a lane's U keys (NG slots apart): the first key's rotated
// coefficients from its exactly reduced phase, each next key's by one complex
// step of the coefficients themselves when the positions advance by NG (any
// gap: from the key's own reduced phase).  key(u, x, y) unpacks key u.
template <int U, int NG, typename Key>
__device__ __forceinline__ void pre_partials(Key &&key, const int32_t (&kpos)[U], const bool (&ok)[U],
                                             const RowCtx &c, const unsigned long long (&T)[8],
                                             const unsigned long long (&TC)[4], const unsigned long long (&TS)[4],
                                             float (&part)[U]) {
    unsigned long long BR[4], BI[4];
    {
        float cs[8], sn[8];
        phasors(T, c.p_now - (int64_t)kpos[0], cs, sn);
        rotate_coef(c, cs, sn, BR, BI);
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
        if (u > 0) {
            if (pos_follows(kpos[u], kpos[u - 1], NG)) {
                advance_coef(BR, BI, TC, TS);
            } else {
                float cs[8], sn[8];
                phasors(T, c.p_now - (int64_t)kpos[u], cs, sn);
                rotate_coef(c, cs, sn, BR, BI);
            }
        }
        float x[8], y[8];
        key(u, x, y);
        part[u] = ok[u] ? partial_rotated(x, y, BR, BI, c) : 0.f;
    }
}

// Partials of one lane's U keys of a whole batch (keys NG slots apart); pre-RoPE
// keys through pre_partials.  Invalid (unplaceable) keys give 0.
template <bool PRE, int U, int NG, typename Chunk>
__device__ __forceinline__ void batch_partials(const Chunk (&kc)[U], const int32_t (&kpos)[U], const bool (&ok)[U],
                                               const RowCtx &c, const unsigned long long (&T)[8],
                                               const unsigned long long (&TC)[4], const unsigned long long (&TS)[4],
                                               float (&part)[U]) {
    if (!PRE) {
#pragma unroll
        for (int u = 0; u < U; u++) {
            float x[8], y[8];
            kc[u].unpack(x, y);
            part[u] = ok[u] ? partial_post(x, y, c) : 0.f;
        }
        return;
    }
    pre_partials<U, NG>([&](int u, float(&x)[8], float(&y)[8]) { kc[u].unpack(x, y); }, kpos, ok, c, T, TC, TS,
                        part);
}

// batch_partials for keys read as they are scored (from shared memory, where a
// staged batch already sits), so no key waits in registers: load(u, chunk)
// fetches key u.  The same arithmetic in the same order, so the same bits.
template <bool PRE, int U, int NG, typename Chunk, typename Load>
__device__ __forceinline__ void batch_partials_lazy(Load &&load, const int32_t (&kpos)[U], const RowCtx &c,
                                                    const unsigned long long (&T)[8],
                                                    const unsigned long long (&TC)[4],
                                                    const unsigned long long (&TS)[4], float (&part)[U]) {
    if constexpr (!PRE) {
#pragma unroll
        for (int u = 0; u < U; u++) {
            Chunk kc;
            load(u, kc);
            float x[8], y[8];
            kc.unpack(x, y);
            part[u] = partial_post(x, y, c);
        }
    } else {
        bool ok[U];
#pragma unroll
        for (int u = 0; u < U; u++) ok[u] = true;
        pre_partials<U, NG>(
            [&](int u, float(&x)[8], float(&y)[8]) {
                Chunk kc;
                load(u, kc);
                kc.unpack(x, y);
            },
            kpos, ok, c, T, TC, TS, part);
    }
}

template <bool PRE, typename Chunk>
__device__ __forceinline__ float chunk_partial(const Chunk &kc, const RowCtx &c, const unsigned long long (&T)[8],
                                               int64_t delta) {
    float x[8], y[8];
    kc.unpack(x, y);
    return PRE ? partial_pre(x, y, c, T, delta) : partial_post(x, y, c);
}

// Compile-time shape of one instantiation: LPK lanes per key (d / 16), NG keys
// per warp instruction, U keys per lane per batch, KB keys per batch.  The
// pre-RoPE mode keeps 4 keys per lane in flight (its per-pair sin/cos needs the
// registers; two CTAs per SM still keep enough bytes in flight).
template <int LPK, bool PRE>
struct Shape {
    static constexpr int NG = 32 / LPK;
    static constexpr int U = (LPK == 4 || PRE) ? 4 : 8;
    static constexpr int KB = NG * U;
    static constexpr int F = 8 * LPK;
};

template <bool PAGED, bool PRE, int ELEM, bool IL, int LPK>
__device__ __forceinline__ float key_partial(const ScoreParams &p, const RowCtx &c, int64_t k, int gl,
                                             unsigned long long pol, const unsigned long long (&T)[8]) {
    constexpr int F = Shape<LPK, PRE>::F;
    const int64_t slot = key_slot<PAGED>(p, c, k);
    if (slot < 0) {
        atomicOr(p.flags, TRI_FLAG_BLOCK_TABLE);
        return 0.f;
    }
    KeyChunk<ELEM, IL, F> kc;
    kc.load(p.K + slot * (2 * F * ELEM), gl, pol);
    const int64_t delta = PRE ? c.p_now - (int64_t)__ldg(p.pos + slot) : 0;
    return chunk_partial<PRE>(kc, c, T, delta);
}

}  // namespace tri
