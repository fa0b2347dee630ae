// Stable compaction: copy K, V (and pos) of every kept slot, in ascending slot
// order, into the output cache ("TriAttention：基于三角函数 KV 压缩的高效长推理",
// 流程详解 step 4: later attention reads only the compressed cache).
//
// Flat grid over (row, chunk of kept slots), for the fused score-and-select
// call (tri_compact gathers inside its selection kernel).  A record (one key or
// value: d elements, 64 to 512 bytes) is moved as 16-byte vectors by record/16
// lanes, so each warp instruction copies 512 bytes of whole records; every
// thread keeps 4 K and 4 V vectors in flight.  Source reads bypass L1;
// destination writes are streaming stores (not re-read here).  Paged input
// and/or output addresses go through the block tables.
#include "gather_chunk.cuh"

namespace tri {

constexpr int kGatherThreads = 256;
constexpr int kGatherIters = 4;

// RB: record bytes (d x element size).  A record is moved as RB/16 16-byte
// vectors by RB/16 lanes, so a warp instruction moves 512 bytes.  One CTA of
// kGatherThreads moves one chunk of kept slots (gather_chunk, shared with the
// select-and-gather kernel).
template <int RB>
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const GatherParams p) {
    constexpr int kSlotsPerCta = GatherChunk<RB, kGatherThreads, kGatherIters>::kSlots;
    grid_dependency_wait();
    grid_dependents_launch();
    const Geometry &geo = p.geo;
    const uint32_t chunks = (uint32_t)((p.B + kSlotsPerCta - 1) / kSlotsPerCta);  // grid = rows x chunks < 2^31
    const int64_t r = blockIdx.x / chunks;
    const int base = (int)(blockIdx.x % chunks) * kSlotsPerCta;
    const int64_t row_lo = geo.row_off[r];
    const int64_t N = geo.row_off[r + 1] - row_lo;
    if (N < 0 || N > 0x7fffffffLL || row_lo < 0 || row_lo + N > geo.total) return;  // flagged by the selection
    const int cnt = (int)min(N, (int64_t)p.B);
    if (base >= cnt) return;
    GatherChunk<RB, kGatherThreads, kGatherIters>::move(p, r, row_lo, N, cnt, base);
}

template <int RB>
static cudaError_t launch_gather_t(const GatherParams &p, cudaStream_t s) {
    constexpr int kSlotsPerCta = GatherChunk<RB, kGatherThreads, kGatherIters>::kSlots;
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
