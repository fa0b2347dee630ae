// Internal launch interface and device helpers of libtri.so (not installed).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <utility>

#include "tri.h"

namespace tri {

constexpr int kMaxD = 256;            // largest supported head dim
constexpr int kMaxF = kMaxD / 2;      // its frequency pairs
constexpr int kCoefPerGroup = 24;     // 8 pairs x (Re A, Im A, c)
constexpr int coef_per_row(int D) { return (D / 16) * kCoefPerGroup; }  // 3 floats per pair

// Workspace layout (byte offsets from the 256-byte aligned base).
constexpr size_t kWsFlags = 0;       // uint32 flag word
constexpr size_t kWsTurns = 256;     // uint64 [d/2 <= 128]: w_f / 2pi in 0.64 fixed point
constexpr size_t kWsCoef = 1280;     // float [R][d/16][24]
constexpr size_t ws_coef_bytes(int64_t R, int D) { return ((size_t)R * coef_per_row(D) * 4 + 255) & ~size_t(255); }
constexpr size_t ws_idx_offset(int64_t R, int D) { return kWsCoef + ws_coef_bytes(R, D); }  // what tri_score needs
constexpr size_t ws_total(int64_t R, int64_t B, int D) {
    return ws_idx_offset(R, D) + (((size_t)R * (size_t)B * 4 + 255) & ~size_t(255));
}

struct Geometry {  // row numbering and cache addressing
    int32_t L, S, H, Hq, G;
    int32_t layout;
    int32_t D;           // head dim: 64, 128 or 256
    int32_t il;          // 1: interleaved RoPE pairs (2f, 2f+1); 0: rotate-half (f, f+D/2)
    int32_t elem_bytes;  // 2: bf16, 1: fp8 e4m3
    int32_t max_blocks, block_shift;  // paged: block_size = 1 << block_shift
    int64_t n_blocks;
    int64_t total;
    const int64_t *row_off;
    const int32_t *block_table;
};

struct PrepParams {
    Geometry geo;
    const float *centres;
    const float *mean_norm;
    const int64_t *p_now;
    double theta;
    int32_t n_off;
    int32_t pre_rope;
    int32_t offsets[TRI_MAX_OFFSETS];
    float *coef;
    unsigned long long *turns;
    unsigned *flags;
};

struct ScoreParams {
    Geometry geo;
    const char *K;
    const int32_t *pos;
    const int64_t *p_now;
    const float *coef;
    const unsigned long long *turns;
    float *scores;
    unsigned *flags;
};

struct SelectParams {
    Geometry geo;
    const float *scores;
    int32_t B, W;
    int32_t *kept;        // [R][B]
    int32_t *kept_count;  // [R] or null
    unsigned *flags;
};

struct GatherParams {
    Geometry geo;
    // output paging (layout TRI_KV_PAGED) or contiguous [R][B]
    int32_t out_layout, out_max_blocks, out_block_shift;
    int64_t out_n_blocks;
    const int32_t *out_table;
    int32_t B;
    const int32_t *kept;
    const char *K, *V;
    const int32_t *pos;
    char *K_out, *V_out;
    int32_t *pos_out;
    unsigned *flags;
};

struct CalibParams {
    int32_t D, il;
    const uint16_t *q;
    int64_t nq;
    int32_t n_heads;  // L * Hq
    float *centres, *mean_norm;
};

struct CalibUpdateParams {
    CalibParams c;
    double decay;
    double *sums;    // [n_heads][F][3]: decayed sums of re, im, |q|
    double *weight;  // [n_heads]: decayed query count
};

struct StatsParams {
    int32_t F;
    int64_t n_heads;
    const float *centres, *mean_norm;          // [n][F][2], [n][F]
    const float *ref_centres, *ref_mean_norm;  // same shapes, or null
    float *concentration;                      // [n][F] or null
    float *head_stats;                         // [n][2] or null
};

constexpr int kKeyCentreChunks = 16;  // CTAs per row of the key-centre pass

struct KeyCentreParams {
    Geometry geo;
    const char *K;
    const int32_t *pos;
    int32_t post_rope;
    double theta;
    double *partial;  // [R][kKeyCentreChunks][F][3]
    float *centres, *mean_norm;
    unsigned *flags;
};

constexpr int kAttnMaxChunks = 32;  // most slices per cache row in decode attention

struct AttnParams {
    Geometry geo;        // the (compressed) cache: layout, head dim, element type
    const char *K, *V;
    const uint16_t *q;   // bf16 [L][S][Hq][D], RoPE'd at the decode position
    float scale_log2;    // softmax scale * log2(e)
    int32_t chunks;      // CTAs per row (1 .. kAttnMaxChunks), set at launch
    float *part;         // [R][chunks][G][D + 2]: unnormalised output, running max, running sum
    float *out;          // [L][S][Hq][D]
    float *lse;          // [L][S][Hq] or null
    unsigned *flags;
};

constexpr int kFusedMaxRow = TRI_FUSED_MAX_ROW;  // longest row the fused score-and-select kernel holds on chip

struct FusedParams {
    PrepParams pp;        // calibration, positions, offsets: each CTA forms its row's coefficients
    ScoreParams sp;       // cache, scores (may be null: kept on chip only)
    int32_t B, W;
    int32_t *kept;        // [R][B]
    int32_t *kept_count;  // [R] or null
};

cudaError_t launch_calib(const CalibParams &p, cudaStream_t s);
cudaError_t launch_fused(const FusedParams &p, int pre_rope, cudaStream_t s);
cudaError_t launch_attention(const AttnParams &p, cudaStream_t s);
cudaError_t launch_attention_tc(const AttnParams &p, int64_t R, cudaStream_t s);  // cudaErrorNotSupported outside its case
cudaError_t launch_calib_update(const CalibUpdateParams &p, cudaStream_t s);
cudaError_t launch_stats(const StatsParams &p, cudaStream_t s);
cudaError_t launch_key_centres(const KeyCentreParams &p, cudaStream_t s);
cudaError_t launch_prep(const PrepParams &p, cudaStream_t s);
cudaError_t launch_score(const ScoreParams &p, int pre_rope, cudaStream_t s);
cudaError_t launch_select_gather(const SelectParams &p, const GatherParams &g, cudaStream_t s);
cudaError_t launch_gather(const GatherParams &p, cudaStream_t s);

int sm_count();  // SMs of the current device (cached per device)

// Launch with programmatic stream serialization: the kernel may be scheduled
// while its predecessor on the stream finishes.  Every kernel launched this
// way calls grid_dependency_wait() before its first access to global memory
// and grid_dependents_launch() only after that wait, so each kernel still
// starts its memory work after every earlier kernel on the stream completed.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Wait until the grids this one depends on have completed and their memory is
// visible (returns at once when launched without programmatic serialization).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next kernel on the stream to be scheduled.
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

// ------------------------------------------------------------ device helpers

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float sqrt_approx(float x) {
    float r;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// L2 policy that marks lines for early eviction: streamed-once data.
__device__ __forceinline__ unsigned long long policy_evict_first() {
    unsigned long long pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 16-byte read-only load that bypasses L1 and carries an L2 eviction policy.
__device__ __forceinline__ uint4 ld_stream16(const void *ptr, unsigned long long pol) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr), "l"(pol));
    return v;
}

// 8-byte variant of ld_stream16.
__device__ __forceinline__ uint2 ld_stream8(const void *ptr, unsigned long long pol) {
    uint2 v;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;"
        : "=r"(v.x), "=r"(v.y)
        : "l"(ptr), "l"(pol));
    return v;
}

__device__ __forceinline__ uint4 ld_nc16(const void *ptr) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr));
    return v;
}

__device__ __forceinline__ void st_stream16(void *ptr, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// A phase held as a 0.64 fixed-point fraction of a turn, as a float count of
// 2^-23 turns in [-2^22, 2^22): the top 23 bits, re-centred by flipping their top
// bit, placed in the mantissa of 2^23 (exact for any 23-bit integer) and the bias
// 1.5 * 2^23 subtracted - integer and FP32-pipe operations only, no conversion
// instruction.  Multiply by 2 pi / 2^23 for radians (step 7.5e-7 rad).
constexpr float kTurn23ToRad = 7.490140565847157e-07f;  // 2 pi / 2^23
__device__ __forceinline__ float turn_units23(unsigned long long t) {
    const uint32_t u = (uint32_t)(t >> 41);
    return __uint_as_float(0x4B000000u | (u ^ 0x400000u)) - 12582912.0f;
}

// Order-preserving map of fp32 scores to uint32: larger score -> larger key.
// -0 is folded onto +0 (they compare equal); NaN maps to 0, below -inf.
__device__ __forceinline__ uint32_t order_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (s != s) return 0u;
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace tri
