// Stable compaction: copy K, V (and pos) of every kept slot, in ascending slot
// order, into the output cache ("TriAttention：基于三角函数 KV 压缩的高效长推理",
// 流程详解 step 4: later attention reads only the compressed cache).
//
// Flat grid over (row, chunk of kept slots).  A record (one key or value: d
// elements, 64 to 512 bytes) is moved as 16-byte vectors by record/16 lanes,
// so each warp instruction copies 512 bytes of whole records; every thread
// keeps 4 K and 4 V vectors in flight.  Source reads
// bypass L1; destination writes are streaming stores (not re-read here).
// Paged input and/or output addresses go through the block tables.
#include "tri_internal.cuh"

namespace tri {

constexpr int kGatherThreads = 256;
constexpr int kGatherIters = 4;

// RB: record bytes (d x element size).  A record is moved as RB/16
// 16-byte vectors by RB/16 lanes, so a warp instruction moves 512 bytes.
template <int RB>
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const GatherParams p) {
    constexpr int kLanes = RB / 16;                                       // lanes per record
    constexpr int kPerWarp = 32 / kLanes;                                 // records per instruction
    constexpr int kSlotsPerCta = (kGatherThreads / 32) * kGatherIters * kPerWarp;
    grid_dependency_wait();
    grid_dependents_launch();
    const Geometry &geo = p.geo;
    const int64_t chunks = (p.B + kSlotsPerCta - 1) / kSlotsPerCta;
    const int64_t r = blockIdx.x / chunks;
    const int base = (int)(blockIdx.x % chunks) * kSlotsPerCta;
    const int64_t row_lo = geo.row_off[r];
    const int64_t N = geo.row_off[r + 1] - row_lo;
    if (N < 0 || N > 0x7fffffffLL || row_lo < 0 || row_lo + N > geo.total) return;  // flagged by the selection
    const int cnt = (int)min(N, (int64_t)p.B);
    if (base >= cnt) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / kLanes, c = lane % kLanes;
    const int h = (int)(r % geo.H);
    const int s = (int)((r / geo.H) % geo.S);
    const int l = (int)(r / ((int64_t)geo.H * geo.S));

    uint4 kv[kGatherIters], vv[kGatherIters];
    int64_t dst[kGatherIters];
    int32_t pv[kGatherIters];
#pragma unroll
    for (int it = 0; it < kGatherIters; it++) {
        const int i = base + (warp * kGatherIters + it) * kPerWarp + sub;
        dst[it] = -1;
        pv[it] = 0;
        if (i >= cnt) continue;
        const int64_t j = p.kept[r * p.B + i];
        if (j == -1) continue;  // an entry the fused kernel emptied (its row was flagged there)
        int64_t src = -1;
        if (j >= 0 && j < N) {
            if (geo.layout == TRI_KV_PAGED) {
                const int64_t bi = j >> geo.block_shift;
                const int32_t blk = bi < geo.max_blocks ? __ldg(geo.block_table + (int64_t)s * geo.max_blocks + bi) : -1;
                if (blk >= 0 && blk < geo.n_blocks)
                    src = ((((int64_t)l * geo.n_blocks + blk) << geo.block_shift) | (j & ((1 << geo.block_shift) - 1))) * geo.H + h;
            } else {
                src = row_lo + j;
            }
        }
        int64_t d = -1;
        if (p.out_layout == TRI_KV_PAGED) {
            const int64_t bi = (int64_t)i >> p.out_block_shift;
            const int32_t blk = bi < p.out_max_blocks ? __ldg(p.out_table + (int64_t)s * p.out_max_blocks + bi) : -1;
            if (blk >= 0 && blk < p.out_n_blocks)
                d = ((((int64_t)l * p.out_n_blocks + blk) << p.out_block_shift) | (i & ((1 << p.out_block_shift) - 1))) * geo.H + h;
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
    for (int it = 0; it < kGatherIters; it++) {
        if (dst[it] < 0) continue;
        st_stream16(p.K_out + dst[it] * RB + 16 * c, kv[it]);
        st_stream16(p.V_out + dst[it] * RB + 16 * c, vv[it]);
        if (p.pos_out && c == 0) p.pos_out[dst[it]] = pv[it];
    }
}

template <int RB>
static cudaError_t launch_gather_t(const GatherParams &p, cudaStream_t s) {
    constexpr int kSlotsPerCta = (kGatherThreads / 32) * kGatherIters * (32 / (RB / 16));
    const int64_t R = (int64_t)p.geo.L * p.geo.S * p.geo.H;
    if (R <= 0) return cudaSuccess;
    const int64_t chunks = (p.B + kSlotsPerCta - 1) / kSlotsPerCta;
    const int64_t grid = R * chunks;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return launch_pdl(gather_kernel<RB>, dim3((unsigned)grid), dim3(kGatherThreads), 0, s, p);
}

cudaError_t launch_gather(const GatherParams &p, cudaStream_t s) {
    switch (p.geo.D * p.geo.elem_bytes) {
        case 64: return launch_gather_t<64>(p, s);
        case 128: return launch_gather_t<128>(p, s);
        case 256: return launch_gather_t<256>(p, s);
        case 512: return launch_gather_t<512>(p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tri
