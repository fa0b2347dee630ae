// tri_score_noalloc: tri_score for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they score a cache: code running inside another framework's memory pool
// that forbids foreign allocations, plugins whose host process owns every
// device allocation, and hard real-time or pre-sized serving loops that
// allocate everything once at start-up.  Such a caller has the cache, the
// calibration and a score buffer, but no workspace.  This entry point gives it
// the same computation as tri_score with the workspace replaced by a fixed
// scratch array compiled into the library.
//
// The scratch is one file-scope __device__ array of kNoAllocBytes: exactly the
// workspace tri_score asks for with TRI_NOALLOC_MAX_ROWS = 4096 rows at the
// largest head dim, 256 (1.25 KiB of flag word and turn table plus 1536 B of
// coefficients per row - 6 B per head dim - about 6 MiB).  Every GPU that loads
// the library holds its own copy until the process exits.  In host code the
// array's name only stands in for it: the device address is looked up with
// cudaGetSymbolAddress, with the calling device current, on every call made
// outside a stream capture (so a device reset, which moves the array, is
// followed), and the last address found on that device is used while the
// stream is being captured.
#include <mutex>

#include "tri_internal.cuh"

namespace {

constexpr int64_t kNoAllocMaxRows = TRI_NOALLOC_MAX_ROWS;
constexpr size_t kNoAllocBytes = tri::ws_idx_offset(kNoAllocMaxRows, tri::kMaxD);
static_assert(kNoAllocBytes % 256 == 0, "the scratch keeps the workspace's 256-byte granularity");
static_assert(tri::ws_idx_offset(kNoAllocMaxRows, 64) <= kNoAllocBytes &&
                  tri::ws_idx_offset(kNoAllocMaxRows, 128) <= kNoAllocBytes,
              "every head dim fits the scratch at the row limit");

static __device__ __align__(256) unsigned char g_score_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of this device's scratch array: looked up afresh outside a
// stream capture, the last address found on this device during one.
tri_status scratch_address(cudaStream_t stream, void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TRI_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TRI_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return TRI_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (cap == cudaStreamCaptureStatusNone || !g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_score_scratch) != cudaSuccess || !p) return TRI_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return TRI_OK;
}

}  // namespace

extern "C" tri_status tri_score_noalloc(const tri_model *m, const tri_kv_desc *kv, const void *K,
                                        const int32_t *pos, const float *centres, const float *mean_norm,
                                        const int64_t *p_now, const int32_t *offsets, int32_t n_offsets,
                                        int32_t key_mode, float *scores, tri_stream_t stream) {
    if (!m || !kv || kv->n_seqs < 1 || m->n_layers < 1 || m->n_kv_heads < 1) return TRI_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)m->n_layers * kv->n_seqs * m->n_kv_heads;
    if (rows > kNoAllocMaxRows) return TRI_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    tri_status st = scratch_address((cudaStream_t)stream, &scratch);
    if (st != TRI_OK) return st;
    // The scratch keeps the previous call's contents.  Nothing in it has to start
    // at zero: the prep kernel rewrites the turn table and every coefficient row
    // the score kernel reads in this call.  The flag word there is only OR-ed
    // into and is never reported by this entry point.
    return tri_score(m, kv, K, pos, centres, mean_norm, p_now, offsets, n_offsets, key_mode, scores, scratch,
                     kNoAllocBytes, stream);
}
