// Loading a lane's share of one cached key record (bf16 or fp8 e4m3, rotate-half
// or interleaved RoPE pairs) and widening it to fp32 pairs.  Shared by the
// scoring and key-centre kernels.
#pragma once

#include "tri_internal.cuh"

namespace tri {

__device__ __forceinline__ void unpack_bf16x8(const uint4 v, float (&x)[8]) {
    x[0] = bf16lo(v.x); x[1] = bf16hi(v.x); x[2] = bf16lo(v.y); x[3] = bf16hi(v.y);
    x[4] = bf16lo(v.z); x[5] = bf16hi(v.z); x[6] = bf16lo(v.w); x[7] = bf16hi(v.w);
}

// Two packed e4m3 values (low byte first) to floats: exact via f16.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    return __half22float2(__half2(h));
}

__device__ __forceinline__ void unpack_e4m3x8(const uint2 v, float (&x)[8]) {
    const float2 a = e4m3x2_to_float2(v.x), b = e4m3x2_to_float2(v.x >> 16);
    const float2 c = e4m3x2_to_float2(v.y), d = e4m3x2_to_float2(v.y >> 16);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
}

__device__ __forceinline__ void unpack_bf16_pairs(const uint4 a, const uint4 b, float (&x)[8], float (&y)[8]) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; i++) {
        x[i] = bf16lo(w[i]);
        y[i] = bf16hi(w[i]);
    }
}

// Lane gl's share of one key record, as stored: the 8 pairs 8gl .. 8gl+7 of a
// key with F = d/2 pairs.  Rotate-half (IL = false): real parts at dims
// 8gl..8gl+7, imaginary parts F dims later - 2 x 16 bytes for bf16, 2 x 8 bytes
// for fp8.  Interleaved (IL = true): dims 16gl..16gl+15, (re, im) adjacent -
// 32 bytes for bf16, 16 for fp8.  Every load is naturally aligned: records are
// 64..512 bytes long and start at multiples of their length from K.  `lds`
// reads the same bytes of a record staged in shared memory.
template <int ELEM, bool IL, int F>
struct KeyChunk;

template <int F>
struct KeyChunk<2, false, F> {
    uint4 re, im;
    __device__ __forceinline__ void load(const char *key, int gl, unsigned long long pol) {
        re = ld_stream16(key + 16 * gl, pol);
        im = ld_stream16(key + 2 * F + 16 * gl, pol);
    }
    __device__ __forceinline__ void lds(const unsigned char *key, int gl) {
        re = *reinterpret_cast<const uint4 *>(key + 16 * gl);
        im = *reinterpret_cast<const uint4 *>(key + 2 * F + 16 * gl);
    }
    __device__ __forceinline__ void zero() { re = im = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[8], float (&y)[8]) const {
        unpack_bf16x8(re, x);
        unpack_bf16x8(im, y);
    }
};

template <int F>
struct KeyChunk<1, false, F> {
    uint2 re, im;
    __device__ __forceinline__ void load(const char *key, int gl, unsigned long long pol) {
        re = ld_stream8(key + 8 * gl, pol);
        im = ld_stream8(key + F + 8 * gl, pol);
    }
    __device__ __forceinline__ void lds(const unsigned char *key, int gl) {
        re = *reinterpret_cast<const uint2 *>(key + 8 * gl);
        im = *reinterpret_cast<const uint2 *>(key + F + 8 * gl);
    }
    __device__ __forceinline__ void zero() { re = im = make_uint2(0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[8], float (&y)[8]) const {
        unpack_e4m3x8(re, x);
        unpack_e4m3x8(im, y);
    }
};

template <int F>
struct KeyChunk<2, true, F> {
    uint4 a, b;
    __device__ __forceinline__ void load(const char *key, int gl, unsigned long long pol) {
        a = ld_stream16(key + 32 * gl, pol);
        b = ld_stream16(key + 32 * gl + 16, pol);
    }
    __device__ __forceinline__ void lds(const unsigned char *key, int gl) {
        a = *reinterpret_cast<const uint4 *>(key + 32 * gl);
        b = *reinterpret_cast<const uint4 *>(key + 32 * gl + 16);
    }
    __device__ __forceinline__ void zero() { a = b = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[8], float (&y)[8]) const { unpack_bf16_pairs(a, b, x, y); }
};

template <int F>
struct KeyChunk<1, true, F> {
    uint4 v;
    __device__ __forceinline__ void load(const char *key, int gl, unsigned long long pol) {
        v = ld_stream16(key + 16 * gl, pol);
    }
    __device__ __forceinline__ void lds(const unsigned char *key, int gl) {
        v = *reinterpret_cast<const uint4 *>(key + 16 * gl);
    }
    __device__ __forceinline__ void zero() { v = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void unpack(float (&x)[8], float (&y)[8]) const {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float2 p0 = e4m3x2_to_float2(w[i]), p1 = e4m3x2_to_float2(w[i] >> 16);
            x[2 * i] = p0.x;
            y[2 * i] = p0.y;
            x[2 * i + 1] = p1.x;
            y[2 * i + 1] = p1.y;
        }
    }
};

}  // namespace tri
