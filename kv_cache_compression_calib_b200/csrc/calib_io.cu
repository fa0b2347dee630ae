// Calibration artefact on disk ("TriAttention：基于三角函数 KV 压缩的高效长推理",
// 流程详解 step 1: the pre-RoPE query centres are extracted offline, ahead of
// serving; 复现注意事项: they depend on the calibration data, so the file
// records the model shape and the number of queries that produced them).
//
// Host code only (file I/O on caller-owned host buffers; no kernel, no device
// memory).  Layout, every field little-endian:
//    0  char[8]  magic "TRICALIB"
//    8  u32      format version (TRI_CALIB_FILE_VERSION)
//   12  u32      header bytes (64)
//   16  i32      head_dim
//   20  i32      n_layers
//   24  i32      n_q_heads
//   28  i32      n_kv_heads
//   32  i32      rope_style
//   36  i32      reserved (0)
//   40  f64      rope_theta (IEEE binary64 bits)
//   48  i64      calibration queries per head
//   56  u64      FNV-1a 64-bit hash of the payload bytes
//   64  payload: centres f32 [n_layers][n_q_heads][d/2][2], then
//                mean_norm f32 [n_layers][n_q_heads][d/2] (IEEE binary32 bits)
#include <cstdio>
#include <cstring>
#include <vector>

#include "tri.h"

namespace {

constexpr char kMagic[8] = {'T', 'R', 'I', 'C', 'A', 'L', 'I', 'B'};
constexpr uint32_t kHeaderBytes = 64;

void put_u32(unsigned char *p, uint32_t v) {
    for (int i = 0; i < 4; i++) p[i] = (unsigned char)(v >> (8 * i));
}
void put_u64(unsigned char *p, uint64_t v) {
    for (int i = 0; i < 8; i++) p[i] = (unsigned char)(v >> (8 * i));
}
uint32_t get_u32(const unsigned char *p) {
    uint32_t v = 0;
    for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
    return v;
}
uint64_t get_u64(const unsigned char *p) {
    uint64_t v = 0;
    for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
    return v;
}

// FNV-1a, 64-bit (offset basis 0xcbf29ce484222325, prime 0x100000001b3).
uint64_t fnv1a64(const unsigned char *p, size_t n, uint64_t h = 0xcbf29ce484222325ull) {
    for (size_t i = 0; i < n; i++) {
        h ^= p[i];
        h *= 0x100000001b3ull;
    }
    return h;
}

bool model_ok(const tri_model *m) {
    return m && (m->head_dim == 64 || m->head_dim == 128 || m->head_dim == 256) && m->n_layers >= 1 &&
           m->n_q_heads >= 1 && m->n_kv_heads >= 1 && m->n_q_heads % m->n_kv_heads == 0 &&
           (m->rope_style == TRI_ROPE_HALF || m->rope_style == TRI_ROPE_INTERLEAVED) && m->rope_theta > 1.0 &&
           m->rope_theta < 1e300;
}

// Pairs (layer, query head, frequency pair) of a model, or 0 if it overflows.
uint64_t n_pairs(const tri_model *m) {
    const uint64_t n = (uint64_t)m->n_layers * (uint64_t)m->n_q_heads * (uint64_t)(m->head_dim / 2);
    return n > (1ull << 40) ? 0 : n;
}

// Payload bytes of `pairs` pairs: 3 floats each, little-endian.
void encode_payload(const float *centres, const float *mean_norm, uint64_t pairs, std::vector<unsigned char> &out) {
    out.resize(pairs * 12);
    unsigned char *p = out.data();
    for (uint64_t i = 0; i < 2 * pairs; i++, p += 4) {
        uint32_t b;
        std::memcpy(&b, centres + i, 4);
        put_u32(p, b);
    }
    for (uint64_t i = 0; i < pairs; i++, p += 4) {
        uint32_t b;
        std::memcpy(&b, mean_norm + i, 4);
        put_u32(p, b);
    }
}

}  // namespace

extern "C" {

tri_status tri_calib_save(const char *path, const tri_model *m, int64_t nq, const float *centres,
                          const float *mean_norm) {
    if (!path || !centres || !mean_norm || nq < 1 || !model_ok(m)) return TRI_ERR_INVALID_ARG;
    const uint64_t pairs = n_pairs(m);
    if (!pairs) return TRI_ERR_UNSUPPORTED;
    std::vector<unsigned char> payload;
    encode_payload(centres, mean_norm, pairs, payload);
    unsigned char h[kHeaderBytes] = {0};
    std::memcpy(h, kMagic, 8);
    put_u32(h + 8, TRI_CALIB_FILE_VERSION);
    put_u32(h + 12, kHeaderBytes);
    put_u32(h + 16, (uint32_t)m->head_dim);
    put_u32(h + 20, (uint32_t)m->n_layers);
    put_u32(h + 24, (uint32_t)m->n_q_heads);
    put_u32(h + 28, (uint32_t)m->n_kv_heads);
    put_u32(h + 32, (uint32_t)m->rope_style);
    uint64_t tb;
    std::memcpy(&tb, &m->rope_theta, 8);
    put_u64(h + 40, tb);
    put_u64(h + 48, (uint64_t)nq);
    put_u64(h + 56, fnv1a64(payload.data(), payload.size()));
    FILE *f = std::fopen(path, "wb");
    if (!f) return TRI_ERR_IO;
    bool ok = std::fwrite(h, 1, kHeaderBytes, f) == kHeaderBytes &&
              std::fwrite(payload.data(), 1, payload.size(), f) == payload.size();
    ok = (std::fclose(f) == 0) && ok;
    return ok ? TRI_OK : TRI_ERR_IO;
}

tri_status tri_calib_load(const char *path, tri_model *m, int64_t *nq, float *centres, float *mean_norm,
                          size_t capacity_pairs) {
    if (!path || !m || !nq || ((centres == nullptr) != (mean_norm == nullptr))) return TRI_ERR_INVALID_ARG;
    FILE *f = std::fopen(path, "rb");
    if (!f) return TRI_ERR_IO;
    unsigned char h[kHeaderBytes];
    if (std::fread(h, 1, kHeaderBytes, f) != kHeaderBytes || std::memcmp(h, kMagic, 8) != 0 ||
        get_u32(h + 8) != TRI_CALIB_FILE_VERSION || get_u32(h + 12) != kHeaderBytes || get_u32(h + 36) != 0) {
        std::fclose(f);
        return TRI_ERR_IO;
    }
    tri_model fm;
    std::memset(&fm, 0, sizeof(fm));
    fm.head_dim = (int32_t)get_u32(h + 16);
    fm.n_layers = (int32_t)get_u32(h + 20);
    fm.n_q_heads = (int32_t)get_u32(h + 24);
    fm.n_kv_heads = (int32_t)get_u32(h + 28);
    fm.rope_style = (int32_t)get_u32(h + 32);
    const uint64_t tb = get_u64(h + 40);
    std::memcpy(&fm.rope_theta, &tb, 8);
    const int64_t fnq = (int64_t)get_u64(h + 48);
    const uint64_t pairs = model_ok(&fm) ? n_pairs(&fm) : 0;
    if (!pairs || fnq < 1) {
        std::fclose(f);
        return TRI_ERR_IO;
    }
    if (!centres) {  // header only
        std::fclose(f);
        *m = fm;
        *nq = fnq;
        return TRI_OK;
    }
    if (capacity_pairs < pairs) {
        std::fclose(f);
        return TRI_ERR_WORKSPACE_TOO_SMALL;
    }
    std::vector<unsigned char> payload(pairs * 12);
    const bool got = std::fread(payload.data(), 1, payload.size(), f) == payload.size();
    const bool at_end = got && std::fgetc(f) == EOF;
    std::fclose(f);
    if (!got || !at_end || fnv1a64(payload.data(), payload.size()) != get_u64(h + 56)) return TRI_ERR_IO;
    const unsigned char *p = payload.data();
    for (uint64_t i = 0; i < 2 * pairs; i++, p += 4) {
        const uint32_t b = get_u32(p);
        std::memcpy(centres + i, &b, 4);
    }
    for (uint64_t i = 0; i < pairs; i++, p += 4) {
        const uint32_t b = get_u32(p);
        std::memcpy(mean_norm + i, &b, 4);
    }
    *m = fm;
    *nq = fnq;
    return TRI_OK;
}

}  // extern "C"
