// Copying the kept records of one row ("TriAttention：基于三角函数 KV 压缩的高效长
// 推理", 流程详解 step 4: later attention reads only the compressed cache): K, V
// and pos of kept slot i of row r go, bit for bit, to output slot i.  Shared by
// the standalone gather kernel and the select-and-gather kernel.
#pragma once

#include "tri_internal.cuh"

namespace tri {

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
        const int h = (int)(r % geo.H);
        const int s = (int)((r / geo.H) % geo.S);
        const int l = (int)(r / ((int64_t)geo.H * geo.S));
        uint4 kv[ITERS], vv[ITERS];
        int64_t dst[ITERS];
        int32_t pv[ITERS];
#pragma unroll
        for (int it = 0; it < ITERS; it++) {
            const int i = base + (warp * ITERS + it) * kPerWarp + sub;
            dst[it] = -1;
            pv[it] = 0;
            if (i >= cnt) continue;
            const int64_t j = p.kept[r * p.B + i];
            if (j == -1) continue;  // an entry the fused kernel emptied (its row was flagged there)
            int64_t src = -1;
            if (j >= 0 && j < N) {
                if (geo.layout == TRI_KV_PAGED) {
                    const int64_t bi = j >> geo.block_shift;
                    const int32_t blk =
                        bi < geo.max_blocks ? __ldg(geo.block_table + (int64_t)s * geo.max_blocks + bi) : -1;
                    if (blk >= 0 && blk < geo.n_blocks)
                        src = ((((int64_t)l * geo.n_blocks + blk) << geo.block_shift) |
                               (j & ((1 << geo.block_shift) - 1))) * geo.H + h;
                } else {
                    src = row_lo + j;
                }
            }
            int64_t d = -1;
            if (p.out_layout == TRI_KV_PAGED) {
                const int64_t bi = (int64_t)i >> p.out_block_shift;
                const int32_t blk =
                    bi < p.out_max_blocks ? __ldg(p.out_table + (int64_t)s * p.out_max_blocks + bi) : -1;
                if (blk >= 0 && blk < p.out_n_blocks)
                    d = ((((int64_t)l * p.out_n_blocks + blk) << p.out_block_shift) |
                         (i & ((1 << p.out_block_shift) - 1))) * geo.H + h;
            } else {
                d = r * p.B + i;
            }
            if (src < 0 || d < 0) {
                if (c == 0) atomicOr(p.flags, TRI_FLAG_BLOCK_TABLE);
                continue;
            }
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

}  // namespace tri
