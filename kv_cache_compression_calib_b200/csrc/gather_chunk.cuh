// Copying the kept records of one row ("TriAttention：基于三角函数 KV 压缩的高效长
// 推理", 流程详解 step 4: later attention reads only the compressed cache): K, V
// and pos of kept slot i of row r go, bit for bit, to output slot i.  Shared by
// the standalone gather kernel and the select-and-gather kernel.
#pragma once

#include "tri_internal.cuh"

namespace tri {

// Layer l, sequence s and KV head h of row r = (l S + s) H + h, in 32-bit
// arithmetic (a 64-bit division is a long instruction sequence, paid by every
// thread of every gather CTA): r < 2^31, since every launch over rows keeps its
// grid within one grid dimension.
__device__ __forceinline__ void row_lsh(const Geometry &geo, int64_t r, int &l, int &s, int &h) {
    const uint32_t ru = (uint32_t)r, H = (uint32_t)geo.H, S = (uint32_t)geo.S;
    const uint32_t q = ru / H;
    h = (int)(ru - q * H);
    l = (int)(q / S);
    s = (int)(q - (uint32_t)l * S);
}

// Source and destination records of kept slot i of row r (layer l, sequence
// s, KV head h).  False for an entry the fused kernel emptied (-1) and for a
// slot a block table cannot place (flagged by the lane with c == 0).
__device__ __forceinline__ bool kept_record(const GatherParams &p, int64_t r, int64_t row_lo, int64_t N, int i, int h,
                                            int s, int l, int c, int64_t &src, int64_t &dst) {
    const Geometry &geo = p.geo;
    const int64_t j = p.kept[r * p.B + i];
    if (j == -1) return false;  // an entry the fused kernel emptied (its row was flagged there)
    // Paged records: (layer l, block blk, slot t, head h) is record
    // (l n_blocks + blk) bs H + t H + h; j < N < 2^31 and i < B, so a slot's place
    // and block index are 32-bit and only the block term needs 64 bits.
    src = -1;
    if (j >= 0 && j < N) {
        if (geo.layout == TRI_KV_PAGED) {
            const int jj = (int)j;
            const int bi = jj >> geo.block_shift;
            const int32_t blk = bi < geo.max_blocks ? __ldg(geo.block_table + (int64_t)s * geo.max_blocks + bi) : -1;
            if (blk >= 0 && blk < geo.n_blocks)
                src = ((int64_t)l * geo.n_blocks + blk) * ((int64_t)geo.H << geo.block_shift) +
                      (int64_t)(jj & ((1 << geo.block_shift) - 1)) * geo.H + h;
        } else {
            src = row_lo + j;
        }
    }
    dst = -1;
    if (p.out_layout == TRI_KV_PAGED) {
        const int bi = i >> p.out_block_shift;
        const int32_t blk = bi < p.out_max_blocks ? __ldg(p.out_table + (int64_t)s * p.out_max_blocks + bi) : -1;
        if (blk >= 0 && blk < p.out_n_blocks)
            dst = ((int64_t)l * p.out_n_blocks + blk) * ((int64_t)geo.H << p.out_block_shift) +
                  (int64_t)(i & ((1 << p.out_block_shift) - 1)) * geo.H + h;
    } else {
        dst = r * p.B + i;
    }
    if (src < 0 || dst < 0) {
        if (c == 0) atomicOr(p.flags, TRI_FLAG_BLOCK_TABLE);
        return false;
    }
    return true;
}

// THREADS threads move CHUNK consecutive kept slots, base .. base + kSlots - 1
// (those below cnt): a record of RB bytes is RB/16 16-byte vectors, one per
// lane, so a warp instruction moves 32/(RB/16) whole records; each thread keeps
// ITERS K and ITERS V vectors in flight before storing them.  kept[] is read
// with plain loads (the select-and-gather kernel has just written it).
template <int RB, int THREADS, int ITERS>
struct GatherChunk {
    static constexpr int kLanes = RB / 16;        // lanes per record
    static constexpr int kPerWarp = 32 / kLanes;  // records per instruction
    static constexpr int kSlots = (THREADS / 32) * ITERS * kPerWarp;

    __device__ __forceinline__ static void move(const GatherParams &p, int64_t r, int64_t row_lo, int64_t N, int cnt,
                                                int base) {
        const Geometry &geo = p.geo;
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int sub = lane / kLanes, c = lane % kLanes;
        int l, s, h;
        row_lsh(geo, r, l, s, h);
        uint4 kv[ITERS], vv[ITERS];
        int64_t dst[ITERS];
        int32_t pv[ITERS];
#pragma unroll
        for (int it = 0; it < ITERS; it++) {
            const int i = base + (warp * ITERS + it) * kPerWarp + sub;
            dst[it] = -1;
            pv[it] = 0;
            int64_t src, d;
            if (i >= cnt || !kept_record(p, r, row_lo, N, i, h, s, l, c, src, d)) continue;
            dst[it] = d;
            kv[it] = ld_nc16(p.K + src * RB + 16 * c);
            vv[it] = ld_nc16(p.V + src * RB + 16 * c);
            if (p.pos && c == 0) pv[it] = __ldg(p.pos + src);
        }
#pragma unroll
        for (int it = 0; it < ITERS; it++) {
            if (dst[it] < 0) continue;
            st_stream16(p.K_out + dst[it] * RB + 16 * c, kv[it]);
            st_stream16(p.V_out + dst[it] * RB + 16 * c, vv[it]);
            if (p.pos_out && c == 0) p.pos_out[dst[it]] = pv[it];
        }
    }
};

__device__ __forceinline__ void gc_cp_async16(void *smem, const void *gmem) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void gc_cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void gc_cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// A whole row's kept records through shared memory: the records are moved in
// groups of kSlots (K and V of each, ITERS vectors of each per thread) with
// asynchronous 16-byte copies into one half of `stage` while the other half,
// which the same threads filled before, is written out.  No register holds a
// record while it is in flight, so a group's 2 kSlots RB bytes are all in
// flight at once; every thread stores exactly the vectors it copied, so no
// barrier is needed.  `stage`: kStageBytes of shared memory, 16-byte aligned.
template <int RB, int THREADS, int ITERS>
struct GatherStaged {
    static constexpr int kLanes = RB / 16;
    static constexpr int kPerWarp = 32 / kLanes;
    static constexpr int kSlots = (THREADS / 32) * ITERS * kPerWarp;  // records per half
    static constexpr int kHalfBytes = kSlots * 2 * RB;
    static constexpr int kStageBytes = 2 * kHalfBytes;

    __device__ __forceinline__ static void copy(const GatherParams &p, int64_t r, int64_t row_lo, int64_t N, int cnt,
                                                unsigned char *stage) {
        const Geometry &geo = p.geo;
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int sub = lane / kLanes, c = lane % kLanes;
        int l, s, h;
        row_lsh(geo, r, l, s, h);
        int64_t dst0[ITERS], dst1[ITERS];
        int32_t pv0[ITERS], pv1[ITERS];
        // Records base .. base + kSlots - 1 into half `hf` (one commit group).
        auto issue = [&](unsigned char *buf, int base, int64_t (&dst)[ITERS], int32_t (&pv)[ITERS]) {
#pragma unroll
            for (int it = 0; it < ITERS; it++) {
                const int k = (warp * ITERS + it) * kPerWarp + sub;
                const int i = base + k;
                dst[it] = -1;
                pv[it] = 0;
                int64_t src, d;
                if (i >= cnt || !kept_record(p, r, row_lo, N, i, h, s, l, c, src, d)) continue;
                dst[it] = d;
                gc_cp_async16(buf + k * 2 * RB + 16 * c, p.K + src * RB + 16 * c);
                gc_cp_async16(buf + k * 2 * RB + RB + 16 * c, p.V + src * RB + 16 * c);
                if (p.pos && c == 0) pv[it] = __ldg(p.pos + src);
            }
            gc_cp_async_commit();
        };
        auto drain = [&](const unsigned char *buf, const int64_t (&dst)[ITERS], const int32_t (&pv)[ITERS]) {
#pragma unroll
            for (int it = 0; it < ITERS; it++) {
                if (dst[it] < 0) continue;
                const int k = (warp * ITERS + it) * kPerWarp + sub;
                const uint4 a = *reinterpret_cast<const uint4 *>(buf + k * 2 * RB + 16 * c);
                const uint4 b = *reinterpret_cast<const uint4 *>(buf + k * 2 * RB + RB + 16 * c);
                st_stream16(p.K_out + dst[it] * RB + 16 * c, a);
                st_stream16(p.V_out + dst[it] * RB + 16 * c, b);
                if (p.pos_out && c == 0) p.pos_out[dst[it]] = pv[it];
            }
        };
        if (cnt <= 0) return;
        unsigned char *b0 = stage, *b1 = stage + kHalfBytes;
        issue(b0, 0, dst0, pv0);
        for (int base = 0;;) {
            if (base + kSlots < cnt) issue(b1, base + kSlots, dst1, pv1);
            else gc_cp_async_commit();
            gc_cp_async_wait<1>();
            drain(b0, dst0, pv0);
            base += kSlots;
            if (base >= cnt) break;
            if (base + kSlots < cnt) issue(b0, base + kSlots, dst0, pv0);
            else gc_cp_async_commit();
            gc_cp_async_wait<1>();
            drain(b1, dst1, pv1);
            base += kSlots;
            if (base >= cnt) break;
        }
        gc_cp_async_wait<0>();
    }
};

}  // namespace tri
