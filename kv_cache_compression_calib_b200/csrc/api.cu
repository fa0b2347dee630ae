// extern "C" entry points of libtri.so: argument checks, workspace carving and
// kernel dispatch.  See include/tri.h for the contract of every call.
#include <cmath>
#include <cstdio>
#include <cstring>

#include "tri_internal.cuh"

namespace tri {

int sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    int &c = cache[dev & 63];
    if (c == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 1;
        c = v;
    }
    return c;
}

}  // namespace tri

using namespace tri;

namespace {

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

int pow2_shift(int32_t x) {
    if (x < 1 || x > 1024 || (x & (x - 1))) return -1;
    int s = 0;
    while ((1 << s) != x) s++;
    return s;
}

tri_status check_model(const tri_model *m) {
    if (!m) return TRI_ERR_INVALID_ARG;
    if (m->head_dim != 64 && m->head_dim != 128 && m->head_dim != 256) return TRI_ERR_UNSUPPORTED;
    if (m->rope_style != TRI_ROPE_HALF && m->rope_style != TRI_ROPE_INTERLEAVED) return TRI_ERR_INVALID_ARG;
    if (m->n_layers < 1 || m->n_q_heads < 1 || m->n_kv_heads < 1) return TRI_ERR_INVALID_ARG;
    if (m->n_q_heads % m->n_kv_heads) return TRI_ERR_INVALID_ARG;
    if (!std::isfinite(m->rope_theta) || !(m->rope_theta > 1.0)) return TRI_ERR_INVALID_ARG;
    return TRI_OK;
}

int64_t rows_of(const tri_model *m, int32_t S) { return (int64_t)m->n_layers * S * m->n_kv_heads; }

tri_status check_kv(const tri_model *m, const tri_kv_desc *kv, Geometry *geo) {
    if (!kv || !kv->row_off || kv->n_seqs < 1 || kv->total_keys < 0) return TRI_ERR_INVALID_ARG;
    if (!aligned(kv->row_off, 8)) return TRI_ERR_ALIGNMENT;
    const int64_t R = rows_of(m, kv->n_seqs);
    if (R > 0x7fffffffLL || kv->total_keys > (1LL << 56)) return TRI_ERR_UNSUPPORTED;
    std::memset(geo, 0, sizeof(*geo));
    geo->L = m->n_layers;
    geo->S = kv->n_seqs;
    geo->H = m->n_kv_heads;
    geo->Hq = m->n_q_heads;
    geo->G = m->n_q_heads / m->n_kv_heads;
    geo->layout = kv->layout;
    geo->D = m->head_dim;
    geo->il = m->rope_style == TRI_ROPE_INTERLEAVED;
    geo->total = kv->total_keys;
    geo->row_off = kv->row_off;
    if (kv->elem_type == TRI_ELEM_BF16) geo->elem_bytes = 2;
    else if (kv->elem_type == TRI_ELEM_FP8_E4M3) geo->elem_bytes = 1;
    else return TRI_ERR_INVALID_ARG;
    if (kv->layout == TRI_KV_PAGED) {
        if (!kv->block_table || kv->max_blocks < 1 || kv->n_blocks < 1) return TRI_ERR_INVALID_ARG;
        if (!aligned(kv->block_table, 4)) return TRI_ERR_ALIGNMENT;
        const int sh = pow2_shift(kv->block_size);
        if (sh < 0) return TRI_ERR_UNSUPPORTED;
        geo->block_table = kv->block_table;
        geo->max_blocks = kv->max_blocks;
        geo->block_shift = sh;
        geo->n_blocks = kv->n_blocks;
    } else if (kv->layout != TRI_KV_CONTIG) {
        return TRI_ERR_INVALID_ARG;
    }
    return TRI_OK;
}

tri_status check_ws(const void *ws, size_t have, size_t need) {
    if (!ws) return TRI_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return TRI_ERR_ALIGNMENT;
    if (have < need) return TRI_ERR_WORKSPACE_TOO_SMALL;
    return TRI_OK;
}

thread_local char g_last_error[256] = "";

// Maps a CUDA result to a status, recording the failing call for tri_last_error.
tri_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return TRI_OK;
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    return TRI_ERR_CUDA;
}

}  // namespace

extern "C" {

const char *tri_status_str(tri_status s) {
    switch (s) {
        case TRI_OK: return "TRI_OK";
        case TRI_ERR_INVALID_ARG: return "TRI_ERR_INVALID_ARG";
        case TRI_ERR_UNSUPPORTED: return "TRI_ERR_UNSUPPORTED";
        case TRI_ERR_ALIGNMENT: return "TRI_ERR_ALIGNMENT";
        case TRI_ERR_WORKSPACE_TOO_SMALL: return "TRI_ERR_WORKSPACE_TOO_SMALL";
        case TRI_ERR_CUDA: return "TRI_ERR_CUDA";
        case TRI_ERR_DEVICE_FLAG: return "TRI_ERR_DEVICE_FLAG";
        case TRI_ERR_IO: return "TRI_ERR_IO";
    }
    return "TRI_ERR_UNKNOWN";
}

uint32_t tri_version(void) { return (0u << 16) | 3u; }

const char *tri_last_error(void) { return g_last_error; }

size_t tri_workspace_size(const tri_model *m, int32_t n_seqs, int32_t B) {
    if (check_model(m) != TRI_OK || n_seqs < 1 || B < 1) return 0;
    return ws_total(rows_of(m, n_seqs), B, m->head_dim);
}

tri_status tri_workspace_init(void *ws, size_t ws_bytes, tri_stream_t stream) {
    tri_status st = check_ws(ws, ws_bytes, 256);
    if (st != TRI_OK) return st;
    return cuda_status(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream), "tri_workspace_init");
}

tri_status tri_calib(const tri_model *m, const void *qpre, int64_t nq, float *centres, float *mean_norm,
                     tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    if (!qpre || !centres || !mean_norm || nq < 1) return TRI_ERR_INVALID_ARG;
    if (!aligned(qpre, 16) || !aligned(centres, 4) || !aligned(mean_norm, 4)) return TRI_ERR_ALIGNMENT;
    const int64_t heads = (int64_t)m->n_layers * m->n_q_heads;
    if (heads > 0x7fffffffLL) return TRI_ERR_UNSUPPORTED;
    CalibParams p;
    p.D = m->head_dim;
    p.il = m->rope_style == TRI_ROPE_INTERLEAVED;
    p.q = (const uint16_t *)qpre;
    p.nq = nq;
    p.n_heads = (int32_t)heads;
    p.centres = centres;
    p.mean_norm = mean_norm;
    return cuda_status(launch_calib(p, (cudaStream_t)stream), "calib_kernel launch");
}

tri_status tri_score(const tri_model *m, const tri_kv_desc *kv, const void *K, const int32_t *pos,
                     const float *centres, const float *mean_norm, const int64_t *p_now,
                     const int32_t *offsets, int32_t n_offsets, int32_t key_mode, float *scores, void *ws,
                     size_t ws_bytes, tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    Geometry geo;
    if ((st = check_kv(m, kv, &geo)) != TRI_OK) return st;
    if (!K || !centres || !mean_norm || !p_now || !offsets || !scores) return TRI_ERR_INVALID_ARG;
    if (n_offsets < 1 || n_offsets > TRI_MAX_OFFSETS) return TRI_ERR_INVALID_ARG;
    if (key_mode != TRI_KEYS_POST_ROPE && key_mode != TRI_KEYS_PRE_ROPE) return TRI_ERR_INVALID_ARG;
    if (key_mode == TRI_KEYS_PRE_ROPE && !pos) return TRI_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(scores, 4) || !aligned(centres, 8) || !aligned(mean_norm, 4) ||
        !aligned(p_now, 8) || (pos && !aligned(pos, 4)))
        return TRI_ERR_ALIGNMENT;
    const int64_t R = rows_of(m, kv->n_seqs);
    if ((st = check_ws(ws, ws_bytes, ws_idx_offset(R, m->head_dim))) != TRI_OK) return st;
    char *w = (char *)ws;
    cudaStream_t s = (cudaStream_t)stream;

    PrepParams pp;
    std::memset(&pp, 0, sizeof(pp));
    pp.geo = geo;
    pp.centres = centres;
    pp.mean_norm = mean_norm;
    pp.p_now = p_now;
    pp.theta = m->rope_theta;
    pp.n_off = n_offsets;
    pp.pre_rope = key_mode == TRI_KEYS_PRE_ROPE;
    for (int i = 0; i < n_offsets; i++) pp.offsets[i] = offsets[i];
    pp.coef = (float *)(w + kWsCoef);
    pp.turns = (unsigned long long *)(w + kWsTurns);
    pp.flags = (unsigned *)(w + kWsFlags);
    if ((st = cuda_status(launch_prep(pp, s), "prep_kernel launch")) != TRI_OK) return st;

    ScoreParams sp;
    sp.geo = geo;
    sp.K = (const char *)K;
    sp.pos = pos;
    sp.p_now = p_now;
    sp.coef = pp.coef;
    sp.turns = pp.turns;
    sp.scores = scores;
    sp.flags = pp.flags;
    return cuda_status(launch_score(sp, pp.pre_rope, s), "score_kernel launch");
}

tri_status tri_compact(const tri_model *m, const tri_kv_desc *kv, const float *scores, int32_t B, int32_t W,
                       const void *K, const void *V, const int32_t *pos, const tri_out_desc *out, void *K_out,
                       void *V_out, int32_t *pos_out, int32_t *kept_idx, int32_t *kept_count, void *ws,
                       size_t ws_bytes, tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    Geometry geo;
    if ((st = check_kv(m, kv, &geo)) != TRI_OK) return st;
    if (B < 1 || W < 0 || W > B) return TRI_ERR_INVALID_ARG;
    if (!scores || !K || !V || !out || !K_out || !V_out) return TRI_ERR_INVALID_ARG;
    if (pos_out && !pos) return TRI_ERR_INVALID_ARG;
    if (K_out == K || V_out == V || K_out == V || V_out == K) return TRI_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(K, 16) || !aligned(V, 16) || !aligned(K_out, 16) || !aligned(V_out, 16) ||
        (pos && !aligned(pos, 4)) || (pos_out && !aligned(pos_out, 4)) || (kept_idx && !aligned(kept_idx, 4)) ||
        (kept_count && !aligned(kept_count, 4)))
        return TRI_ERR_ALIGNMENT;
    int out_shift = 0;
    if (out->layout == TRI_KV_PAGED) {
        if (!out->block_table || out->max_blocks < 1 || out->n_blocks < 1) return TRI_ERR_INVALID_ARG;
        if (!aligned(out->block_table, 4)) return TRI_ERR_ALIGNMENT;
        out_shift = pow2_shift(out->block_size);
        if (out_shift < 0) return TRI_ERR_UNSUPPORTED;
    } else if (out->layout != TRI_KV_CONTIG) {
        return TRI_ERR_INVALID_ARG;
    }
    const int64_t R = rows_of(m, kv->n_seqs);
    if ((st = check_ws(ws, ws_bytes, kept_idx ? 256 : ws_total(R, B, m->head_dim))) != TRI_OK) return st;
    char *w = (char *)ws;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t *kept = kept_idx ? kept_idx : (int32_t *)(w + ws_idx_offset(R, m->head_dim));

    SelectParams sp;
    sp.geo = geo;
    sp.scores = scores;
    sp.B = B;
    sp.W = W;
    sp.kept = kept;
    sp.kept_count = kept_count;
    sp.flags = (unsigned *)(w + kWsFlags);

    GatherParams gp;
    std::memset(&gp, 0, sizeof(gp));
    gp.geo = geo;
    gp.out_layout = out->layout;
    gp.out_max_blocks = out->max_blocks;
    gp.out_block_shift = out_shift;
    gp.out_n_blocks = out->n_blocks;
    gp.out_table = out->block_table;
    gp.B = B;
    gp.kept = kept;
    gp.K = (const char *)K;
    gp.V = (const char *)V;
    gp.pos = pos_out ? pos : nullptr;
    gp.K_out = (char *)K_out;
    gp.V_out = (char *)V_out;
    gp.pos_out = pos_out;
    gp.flags = sp.flags;
    return cuda_status(launch_select_gather(sp, gp, s), "select_kernel launch");
}

tri_status tri_calib_update(const tri_model *m, const void *qpre, int64_t nq, double decay, double *sums,
                            double *weight, float *centres, float *mean_norm, tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    if (!qpre || !sums || !weight || !centres || !mean_norm || nq < 1) return TRI_ERR_INVALID_ARG;
    if (!std::isfinite(decay) || !(decay > 0.0) || decay > 1.0) return TRI_ERR_INVALID_ARG;
    if (!aligned(qpre, 16) || !aligned(sums, 8) || !aligned(weight, 8) || !aligned(centres, 4) ||
        !aligned(mean_norm, 4))
        return TRI_ERR_ALIGNMENT;
    const int64_t heads = (int64_t)m->n_layers * m->n_q_heads;
    if (heads > 0x7fffffffLL) return TRI_ERR_UNSUPPORTED;
    CalibUpdateParams p;
    p.c.D = m->head_dim;
    p.c.il = m->rope_style == TRI_ROPE_INTERLEAVED;
    p.c.q = (const uint16_t *)qpre;
    p.c.nq = nq;
    p.c.n_heads = (int32_t)heads;
    p.c.centres = centres;
    p.c.mean_norm = mean_norm;
    p.decay = decay;
    p.sums = sums;
    p.weight = weight;
    return cuda_status(launch_calib_update(p, (cudaStream_t)stream), "calib_update_kernel launch");
}

tri_status tri_calib_stats(const tri_model *m, int64_t n_heads, const float *centres, const float *mean_norm,
                           const float *ref_centres, const float *ref_mean_norm, float *concentration,
                           float *head_stats, tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    if (n_heads < 1 || !centres || !mean_norm || (!concentration && !head_stats)) return TRI_ERR_INVALID_ARG;
    if ((ref_centres == nullptr) != (ref_mean_norm == nullptr)) return TRI_ERR_INVALID_ARG;
    if (!aligned(centres, 8) || !aligned(mean_norm, 4) || (ref_centres && !aligned(ref_centres, 8)) ||
        (ref_mean_norm && !aligned(ref_mean_norm, 4)) || (concentration && !aligned(concentration, 4)) ||
        (head_stats && !aligned(head_stats, 4)))
        return TRI_ERR_ALIGNMENT;
    StatsParams p;
    p.F = m->head_dim / 2;
    p.n_heads = n_heads;
    p.centres = centres;
    p.mean_norm = mean_norm;
    p.ref_centres = ref_centres;
    p.ref_mean_norm = ref_mean_norm;
    p.concentration = concentration;
    p.head_stats = head_stats;
    return cuda_status(launch_stats(p, (cudaStream_t)stream), "stats_kernel launch");
}

size_t tri_key_centres_ws_size(const tri_model *m, int32_t n_seqs) {
    if (check_model(m) != TRI_OK || n_seqs < 1) return 0;
    const size_t R = (size_t)rows_of(m, n_seqs);
    return 256 + ((R * kKeyCentreChunks * (size_t)(m->head_dim / 2) * 3 * sizeof(double) + 255) & ~size_t(255));
}

tri_status tri_key_centres(const tri_model *m, const tri_kv_desc *kv, const void *K, const int32_t *pos,
                           int32_t key_mode, float *centres, float *mean_norm, void *ws, size_t ws_bytes,
                           tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    Geometry geo;
    if ((st = check_kv(m, kv, &geo)) != TRI_OK) return st;
    if (!K || !centres || !mean_norm) return TRI_ERR_INVALID_ARG;
    if (key_mode != TRI_KEYS_POST_ROPE && key_mode != TRI_KEYS_PRE_ROPE) return TRI_ERR_INVALID_ARG;
    if (key_mode == TRI_KEYS_POST_ROPE && !pos) return TRI_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(centres, 4) || !aligned(mean_norm, 4) || (pos && !aligned(pos, 4)))
        return TRI_ERR_ALIGNMENT;
    if ((st = check_ws(ws, ws_bytes, tri_key_centres_ws_size(m, kv->n_seqs))) != TRI_OK) return st;
    KeyCentreParams p;
    p.geo = geo;
    p.K = (const char *)K;
    p.pos = pos;
    p.post_rope = key_mode == TRI_KEYS_POST_ROPE;
    p.theta = m->rope_theta;
    p.partial = (double *)((char *)ws + 256);
    p.centres = centres;
    p.mean_norm = mean_norm;
    p.flags = (unsigned *)((char *)ws + kWsFlags);
    return cuda_status(launch_key_centres(p, (cudaStream_t)stream), "key_centre_kernel launch");
}

tri_status tri_score_compact(const tri_model *m, const tri_kv_desc *kv, const void *K, const void *V,
                             const int32_t *pos, const float *centres, const float *mean_norm, const int64_t *p_now,
                             const int32_t *offsets, int32_t n_offsets, int32_t key_mode, int32_t B, int32_t W,
                             int32_t max_row_len, const tri_out_desc *out, void *K_out, void *V_out,
                             int32_t *pos_out, int32_t *kept_idx, int32_t *kept_count, float *scores, void *ws,
                             size_t ws_bytes, tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    Geometry geo;
    if ((st = check_kv(m, kv, &geo)) != TRI_OK) return st;
    if (max_row_len < 0) return TRI_ERR_INVALID_ARG;
    // Fused for short rows (one CTA per row streams little and the selection
    // launch is saved) and whenever no score buffer is given; long rows with a
    // score buffer take the two-call path, which spreads a long row over many SMs.
    const bool fused = max_row_len <= kFusedMaxRow && (max_row_len <= TRI_FUSED_PREFER_ROW || !scores);
    if (!fused) {
        if (!scores) return TRI_ERR_INVALID_ARG;
        if ((st = tri_score(m, kv, K, pos, centres, mean_norm, p_now, offsets, n_offsets, key_mode, scores, ws,
                            ws_bytes, stream)) != TRI_OK)
            return st;
        return tri_compact(m, kv, scores, B, W, K, V, pos, out, K_out, V_out, pos_out, kept_idx, kept_count, ws,
                           ws_bytes, stream);
    }
    // Checks of tri_score ...
    if (!K || !centres || !mean_norm || !p_now || !offsets) return TRI_ERR_INVALID_ARG;
    if (n_offsets < 1 || n_offsets > TRI_MAX_OFFSETS) return TRI_ERR_INVALID_ARG;
    if (key_mode != TRI_KEYS_POST_ROPE && key_mode != TRI_KEYS_PRE_ROPE) return TRI_ERR_INVALID_ARG;
    if (key_mode == TRI_KEYS_PRE_ROPE && !pos) return TRI_ERR_INVALID_ARG;
    if (!aligned(K, 16) || (scores && !aligned(scores, 4)) || !aligned(centres, 8) || !aligned(mean_norm, 4) ||
        !aligned(p_now, 8) || (pos && !aligned(pos, 4)))
        return TRI_ERR_ALIGNMENT;
    // ... and of tri_compact.
    if (B < 1 || W < 0 || W > B) return TRI_ERR_INVALID_ARG;
    if (!V || !out || !K_out || !V_out) return TRI_ERR_INVALID_ARG;
    if (pos_out && !pos) return TRI_ERR_INVALID_ARG;
    if (K_out == K || V_out == V || K_out == V || V_out == K) return TRI_ERR_INVALID_ARG;
    if (!aligned(V, 16) || !aligned(K_out, 16) || !aligned(V_out, 16) || (pos_out && !aligned(pos_out, 4)) ||
        (kept_idx && !aligned(kept_idx, 4)) || (kept_count && !aligned(kept_count, 4)))
        return TRI_ERR_ALIGNMENT;
    int out_shift = 0;
    if (out->layout == TRI_KV_PAGED) {
        if (!out->block_table || out->max_blocks < 1 || out->n_blocks < 1) return TRI_ERR_INVALID_ARG;
        if (!aligned(out->block_table, 4)) return TRI_ERR_ALIGNMENT;
        out_shift = pow2_shift(out->block_size);
        if (out_shift < 0) return TRI_ERR_UNSUPPORTED;
    } else if (out->layout != TRI_KV_CONTIG) {
        return TRI_ERR_INVALID_ARG;
    }
    const int64_t R = rows_of(m, kv->n_seqs);
    if ((st = check_ws(ws, ws_bytes, kept_idx ? ws_idx_offset(R, m->head_dim) : ws_total(R, B, m->head_dim))) !=
        TRI_OK)
        return st;
    char *w = (char *)ws;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t *kept = kept_idx ? kept_idx : (int32_t *)(w + ws_idx_offset(R, m->head_dim));

    PrepParams pp;
    std::memset(&pp, 0, sizeof(pp));
    pp.geo = geo;
    pp.centres = centres;
    pp.mean_norm = mean_norm;
    pp.p_now = p_now;
    pp.theta = m->rope_theta;
    pp.n_off = n_offsets;
    pp.pre_rope = key_mode == TRI_KEYS_PRE_ROPE;
    for (int i = 0; i < n_offsets; i++) pp.offsets[i] = offsets[i];
    pp.flags = (unsigned *)(w + kWsFlags);

    // No prep launch: every CTA of the fused kernel forms its own row's
    // coefficients with the prep kernel's steps.
    FusedParams fp;
    std::memset(&fp, 0, sizeof(fp));
    fp.pp = pp;
    fp.sp.geo = geo;
    fp.sp.K = (const char *)K;
    fp.sp.pos = pos;
    fp.sp.p_now = p_now;
    fp.sp.scores = scores;
    fp.sp.flags = pp.flags;
    fp.B = B;
    fp.W = W;
    fp.kept = kept;
    fp.kept_count = kept_count;
    if ((st = cuda_status(launch_fused(fp, pp.pre_rope, s), "fused_kernel launch")) != TRI_OK) return st;

    GatherParams gp;
    std::memset(&gp, 0, sizeof(gp));
    gp.geo = geo;
    gp.out_layout = out->layout;
    gp.out_max_blocks = out->max_blocks;
    gp.out_block_shift = out_shift;
    gp.out_n_blocks = out->n_blocks;
    gp.out_table = out->block_table;
    gp.B = B;
    gp.kept = kept;
    gp.K = (const char *)K;
    gp.V = (const char *)V;
    gp.pos = pos_out ? pos : nullptr;
    gp.K_out = (char *)K_out;
    gp.V_out = (char *)V_out;
    gp.pos_out = pos_out;
    gp.flags = pp.flags;
    return cuda_status(launch_gather(gp, s), "gather_kernel launch");
}

size_t tri_attention_ws_size(const tri_model *m, int32_t n_seqs) {
    if (check_model(m) != TRI_OK || n_seqs < 1) return 0;
    const size_t R = (size_t)rows_of(m, n_seqs);
    const size_t G = (size_t)(m->n_q_heads / m->n_kv_heads);
    return 256 + ((R * kAttnMaxChunks * G * (size_t)(m->head_dim + 2) * sizeof(float) + 255) & ~size_t(255));
}

tri_status tri_decode_attention(const tri_model *m, const tri_kv_desc *kv, const void *K, const void *V,
                                const void *q, float softmax_scale, float *out, float *lse, void *ws,
                                size_t ws_bytes, tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    Geometry geo;
    if ((st = check_kv(m, kv, &geo)) != TRI_OK) return st;
    if (geo.G > 16) return TRI_ERR_UNSUPPORTED;
    if (!K || !V || !q || !out) return TRI_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.f)) return TRI_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(q, 2) || !aligned(out, 4) || (lse && !aligned(lse, 4)))
        return TRI_ERR_ALIGNMENT;
    if ((st = check_ws(ws, ws_bytes, tri_attention_ws_size(m, kv->n_seqs))) != TRI_OK) return st;
    AttnParams p;
    p.geo = geo;
    p.K = (const char *)K;
    p.V = (const char *)V;
    p.q = (const uint16_t *)q;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.part = (float *)((char *)ws + 256);
    p.out = out;
    p.lse = lse;
    p.flags = (unsigned *)((char *)ws + kWsFlags);
    return cuda_status(launch_attention(p, (cudaStream_t)stream), "attention kernel launch");
}

tri_status tri_decode_attention_tc(const tri_model *m, const tri_kv_desc *kv, const void *K, const void *V,
                                   const void *q, float softmax_scale, float *out, float *lse, void *ws,
                                   size_t ws_bytes, tri_stream_t stream) {
    tri_status st = check_model(m);
    if (st != TRI_OK) return st;
    Geometry geo;
    if ((st = check_kv(m, kv, &geo)) != TRI_OK) return st;
    if (geo.G > 16 || geo.D != 128 || geo.elem_bytes != 2 || geo.layout != TRI_KV_CONTIG) return TRI_ERR_UNSUPPORTED;
    if (kv->total_keys < 1 || kv->total_keys > 0x7fffffffLL) return TRI_ERR_UNSUPPORTED;
    if (!K || !V || !q || !out) return TRI_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.f)) return TRI_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(V, 16) || !aligned(q, 2) || !aligned(out, 4) || (lse && !aligned(lse, 4)))
        return TRI_ERR_ALIGNMENT;
    if ((st = check_ws(ws, ws_bytes, tri_attention_ws_size(m, kv->n_seqs))) != TRI_OK) return st;
    const int64_t R = rows_of(m, kv->n_seqs);
    if (R * kAttnMaxChunks > 0x7fffffffLL || R * geo.G > 0x7fffffffLL) return TRI_ERR_UNSUPPORTED;
    AttnParams p;
    p.geo = geo;
    p.K = (const char *)K;
    p.V = (const char *)V;
    p.q = (const uint16_t *)q;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.part = (float *)((char *)ws + 256);
    p.out = out;
    p.lse = lse;
    p.flags = (unsigned *)((char *)ws + kWsFlags);
    const cudaError_t e = launch_attention_tc(p, R, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return TRI_ERR_UNSUPPORTED;
    return cuda_status(e, "tensor-memory attention kernel launch");
}

tri_status tri_status_check(void *ws, uint32_t *flags, tri_stream_t stream) {
    tri_status st = check_ws(ws, 256, 256);
    if (st != TRI_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t host = 0;
    if ((st = cuda_status(cudaMemcpyAsync(&host, ws, sizeof(host), cudaMemcpyDeviceToHost, s), "flag read")) != TRI_OK)
        return st;
    if ((st = cuda_status(cudaStreamSynchronize(s), "stream synchronize")) != TRI_OK) return st;
    if ((st = cuda_status(cudaMemsetAsync(ws, 0, sizeof(host), s), "flag clear")) != TRI_OK) return st;
    if (flags) *flags = host;
    return host ? TRI_ERR_DEVICE_FLAG : TRI_OK;
}

}  // extern "C"
