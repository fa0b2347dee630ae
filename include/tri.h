/*
 * tri.h - C ABI of libtri.so: TriAttention KV-cache key scoring, per-head top-B
 * selection and K/V compaction on NVIDIA B200 (sm_100a).
 *
 * The method ("TriAttention：基于三角函数 KV 压缩的高效长推理", whatsmy.fun paper
 * digest, section 流程详解 steps 1-4; "WeianMao/triattention" project card,
 * "How it works"): pre-RoPE query centres are calibrated offline (step 1);
 * every cached key is scored by a trigonometric series in its RoPE distance to
 * the future positions p_now + delta (step 2) plus a norm term (step 3); each
 * KV head keeps its B best keys, the W most recent always among them, and the
 * cache is compacted to those keys (step 4).  The score of the key at position
 * j in the cache row of KV head h is
 *
 *   S_j = (1/G) sum_{g in group(h)} [ sum_f |qbar_f^g| |k_f| sum_delta cos(w_f (p_now + delta - j) + phi_f^g)
 *                                    + sum_f (E|q_f^g| - |qbar_f^g|) |k_f| ],
 *   w_f = rope_theta^(-2f/d),  phi_f^g = arg qbar_f^g - arg k_f,
 *
 * k the pre-RoPE key, f = 0 .. d/2-1 over frequency pairs: dims (f, f + d/2) with
 * rotate-half RoPE (Qwen3 / Llama-HF / GPT-NeoX), dims (2f, 2f + 1) with
 * interleaved RoPE (GPT-J / Meta-Llama); group(h) = query heads h*G .. h*G+G-1,
 * G = n_q_heads/n_kv_heads.
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers on the current device, allocated
 *    and owned by the caller; the library allocates nothing and keeps no state
 *    besides per-device caches (SM counts, and the fixed scratch array of
 *    tri_score_noalloc with its address).  Every call is asynchronous on
 *    `stream` (a cudaStream_t; NULL = the legacy default stream) and returns
 *    after enqueuing its kernels.
 *  - bf16 tensors are passed as `void*` and hold IEEE bfloat16 bit patterns.
 *  - Arguments are checked on the host before anything is launched; a failed
 *    check returns its status and launches nothing.  Kernels never trap and
 *    never wait on other blocks: data anomalies they detect (see TRI_FLAG_*)
 *    are OR-ed into a flag word in the workspace, read by tri_status_check.
 *  - A "row" is one (layer l, sequence s, KV head h), numbered
 *    r = (l * n_seqs + s) * n_kv_heads + h; R = n_layers * n_seqs * n_kv_heads.
 */
#ifndef TRI_H
#define TRI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *tri_stream_t; /* same type as cudaStream_t */

typedef enum {
    TRI_OK = 0,
    TRI_ERR_INVALID_ARG = 1,         /* null pointer, negative size, inconsistent shapes */
    TRI_ERR_UNSUPPORTED = 2,         /* head_dim not 64/128/256, block size not a power of two, ... */
    TRI_ERR_ALIGNMENT = 3,           /* a pointer is not aligned as documented */
    TRI_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes < tri_workspace_size(...) */
    TRI_ERR_CUDA = 5,                /* a CUDA launch or copy failed */
    TRI_ERR_DEVICE_FLAG = 6,         /* tri_status_check found a flag set by a kernel */
    TRI_ERR_IO = 7                   /* a file could not be opened, read or written, or is not a valid calibration file */
} tri_status;

/* Flag bits that kernels OR into the workspace flag word. */
#define TRI_FLAG_ROW_OFFSETS 0x1u /* row_off not non-decreasing from 0 to total_keys */
#define TRI_FLAG_NONFINITE 0x2u   /* a NaN score reached selection (ranked last) */
#define TRI_FLAG_BLOCK_TABLE 0x4u /* paged: block id out of [0, n_blocks) or row too long for the table; the key is skipped */
#define TRI_FLAG_STAGE_TIMEOUT 0x8u /* a staged copy of keys did not land within 2 s; the warp that waited skipped its remaining keys */

#define TRI_MAX_OFFSETS 64

enum { TRI_KV_CONTIG = 0, TRI_KV_PAGED = 1 };
enum { TRI_ROPE_HALF = 0, TRI_ROPE_INTERLEAVED = 1 }; /* pair f = dims (f, f+d/2) or (2f, 2f+1) */
enum { TRI_ELEM_BF16 = 0, TRI_ELEM_FP8_E4M3 = 1 }; /* K/V element type */
enum { TRI_KEYS_POST_ROPE = 0, TRI_KEYS_PRE_ROPE = 1 };

typedef struct {
    int32_t head_dim;   /* d: 64, 128 or 256 */
    int32_t n_layers;   /* L >= 1 */
    int32_t n_q_heads;  /* Hq >= 1 */
    int32_t n_kv_heads; /* H >= 1, Hq % H == 0 */
    double rope_theta;  /* theta > 1 */
    int32_t rope_style; /* TRI_ROPE_HALF (0, the default of a zeroed struct) or TRI_ROPE_INTERLEAVED */
    int32_t pad_;       /* zero */
} tri_model;

/*
 * Where the cached keys of each row live.
 *  TRI_KV_CONTIG: K is [total_keys][d] (elem_type) and pos is [total_keys] int32; row r
 *    is entries row_off[r] .. row_off[r+1]-1 (rows of any length, in row order).
 *  TRI_KV_PAGED (vLLM block layout): K is [n_layers][n_blocks][block_size][H][d]
 *    (elem_type) and pos is [n_layers][n_blocks][block_size][H] int32; slot j of
 *    sequence s is slot j % block_size of block block_table[s][j / block_size],
 *    the same table for every layer.  row_off then only describes the score
 *    buffer (row r's scores are entries row_off[r] .. row_off[r+1]-1) and the
 *    row lengths.
 * In both layouts the score buffer is float [total_keys], indexed like row_off.
 */
typedef struct {
    int32_t layout;         /* TRI_KV_CONTIG or TRI_KV_PAGED */
    int32_t n_seqs;         /* S >= 1 */
    int64_t total_keys;     /* must equal row_off[R] */
    const int64_t *row_off; /* device [R + 1], row_off[0] = 0, non-decreasing */
    /* TRI_KV_PAGED only (ignored for TRI_KV_CONTIG): */
    const int32_t *block_table; /* device [n_seqs][max_blocks] */
    int32_t max_blocks;         /* >= 1 */
    int32_t block_size;         /* power of two, 1 .. 1024 (vLLM: 16) */
    int64_t n_blocks;           /* blocks per layer in the pool, >= 1 */
    /* Element type of K and V (and of the compacted outputs): TRI_ELEM_BF16
     * (2 bytes, the default of a zeroed descriptor) or TRI_ELEM_FP8_E4M3 (1 byte,
     * OCP e4m3 "fn": no infinities, 0x7f/0xff are NaN).  fp8 values are scored as
     * stored: a per-tensor dequantisation scale multiplies every score of a row
     * equally and leaves the selection unchanged. */
    int32_t elem_type;
    int32_t pad_;
} tri_kv_desc;

/*
 * Where tri_compact writes the kept keys.
 *  TRI_KV_CONTIG: K_out/V_out are [R][B][d], pos_out [R][B]: kept slot i of row
 *    r goes to entry r * B + i.
 *  TRI_KV_PAGED: K_out/V_out are [n_layers][n_blocks][block_size][H][d] and
 *    pos_out [n_layers][n_blocks][block_size][H]; kept slot i of row (l, s, h)
 *    goes to slot i % block_size of block block_table[s][i / block_size] -
 *    a fresh table chosen by the caller's block allocator, which needs
 *    ceil(min(N, B) / block_size) <= max_blocks entries per sequence.
 */
typedef struct {
    int32_t layout;
    int32_t max_blocks;
    const int32_t *block_table;
    int32_t block_size;
    int32_t pad_;
    int64_t n_blocks;
} tri_out_desc;

/* Human-readable name of a status code (static string). */
const char *tri_status_str(tri_status s);

/* Library version, (major << 16) | minor.  0.2: tri_model carries rope_style and
 * tri_kv_desc elem_type (both zero by default: rotate-half RoPE, bf16).  0.3:
 * calibration files (tri_calib_save / tri_calib_load) and TRI_ERR_IO. */
uint32_t tri_version(void);

/* After a call returned TRI_ERR_CUDA: which CUDA call failed on this thread,
 * with the CUDA error name and text (a thread-local string, "" if none). */
const char *tri_last_error(void);

/*
 * Bytes of workspace that tri_score and tri_compact need for `m` and `n_seqs`
 * sequences with budget B.  One buffer may serve both calls (they run in
 * stream order).  The workspace must be 256-byte aligned device memory.
 */
size_t tri_workspace_size(const tri_model *m, int32_t n_seqs, int32_t B);

/* Clear the workspace flag word (enqueued on `stream`).  Call once after
 * allocating a workspace; tri_status_check clears it again after reading. */
tri_status tri_workspace_init(void *ws, size_t ws_bytes, tri_stream_t stream);

/*
 * Offline calibration (digest, 流程详解 step 1): for every (layer l, query head g)
 * and pair f, the complex mean of the pre-RoPE queries and the mean of their
 * magnitudes,
 *   centres[l][g][f] = (1/nq) sum_t (q[t][a_f] + i q[t][b_f])          (re, im)
 *   mean_norm[l][g][f] = (1/nq) sum_t |q[t][a_f] + i q[t][b_f]|,
 * with (a_f, b_f) the dims of pair f under m->rope_style, accumulated in fp64,
 * stored fp32.
 *   qpre:      bf16 [n_layers][n_q_heads][nq][d], 16-byte aligned
 *   nq:        queries per head, >= 1
 *   centres:   float [n_layers][n_q_heads][d/2][2]
 *   mean_norm: float [n_layers][n_q_heads][d/2]
 */
tri_status tri_calib(const tri_model *m, const void *qpre, int64_t nq, float *centres,
                     float *mean_norm, tri_stream_t stream);

/*
 * Calibration artefact on disk (digest, 流程详解 step 1: the centres are
 * computed offline, ahead of serving; 复现注意事项: they depend on the
 * calibration data, so the file records the model shape and the number of
 * queries per head that produced them).  HOST pointers: the caller copies the
 * centres from or to the device (they are tri_calib's outputs and
 * tri_score's inputs).  The file is a 64-byte little-endian header (magic
 * "TRICALIB", format version TRI_CALIB_FILE_VERSION, header size, head_dim,
 * n_layers, n_q_heads, n_kv_heads, rope_style, a zero word, rope_theta as
 * binary64, nq, and the FNV-1a 64-bit hash of the payload) followed by the
 * payload: centres then mean_norm as little-endian binary32, in tri_calib's
 * layouts.  Values are stored bit for bit.
 *
 * tri_calib_save: writes (or replaces) `path`.
 *   m, nq:     the model and the calibration queries per head (>= 1)
 *   centres:   host float [n_layers][n_q_heads][d/2][2]
 *   mean_norm: host float [n_layers][n_q_heads][d/2]
 *   Returns TRI_ERR_INVALID_ARG for null pointers, nq < 1 or an invalid
 *   model, TRI_ERR_IO if the file cannot be written.
 *
 * tri_calib_load: reads `path` into *m and *nq and, when centres and mean_norm
 *   are not NULL, the payload into them (capacity_pairs = the number of
 *   (layer, query head, pair) entries they hold; it must be at least
 *   n_layers * n_q_heads * d/2 of the file, else TRI_ERR_WORKSPACE_TOO_SMALL).
 *   With both NULL only the header is read and checked, so a caller can size
 *   its buffers first.  A missing or unreadable file, a wrong magic, version or
 *   header, an invalid model, a truncated or over-long payload or a hash
 *   mismatch return TRI_ERR_IO; nothing is written to the outputs then.
 */
#define TRI_CALIB_FILE_VERSION 1
tri_status tri_calib_save(const char *path, const tri_model *m, int64_t nq, const float *centres,
                          const float *mean_norm);
tri_status tri_calib_load(const char *path, tri_model *m, int64_t *nq, float *centres, float *mean_norm,
                          size_t capacity_pairs);

/*
 * Score every cached key (digest, 流程详解 steps 2-3) with the rule in the
 * header comment, the GQA mean taken over the query heads of each KV head.
 *   kv:        layout and row offsets of the cache
 *   K:         keys (kv->elem_type) in kv's layout, 16-byte aligned
 *   pos:       int32 position of every cached slot (kv's layout).  Read only
 *              for TRI_KEYS_PRE_ROPE; may be NULL for TRI_KEYS_POST_ROPE.
 *   centres, mean_norm: calibration of tri_calib, [n_layers][n_q_heads][d/2](x2);
 *              centres 8-byte aligned, mean_norm 4-byte aligned
 *   p_now:     device int64 [n_seqs], the position of each sequence's next token
 *   offsets:   HOST int32 [n_offsets], the future offsets delta, 1 <= n_offsets
 *              <= TRI_MAX_OFFSETS (copied into the launch; not kept)
 *   key_mode:  TRI_KEYS_POST_ROPE: K holds RoPE-rotated keys (as an inference
 *              cache does): the key's own rotation cancels the -j of the
 *              distance, so pos is not needed and no per-key sin/cos is taken.
 *              TRI_KEYS_PRE_ROPE: K holds pre-RoPE keys; one sin/cos per
 *              (key, pair) of w_f (p_now - pos) is taken, with the phase
 *              reduced exactly in 64-bit fixed-point turns.
 *   scores:    float [kv->total_keys], 4-byte aligned
 *   ws:        workspace of tri_workspace_size bytes
 * Scores are fp32 with fp32 accumulation; per-row coefficients are formed in
 * fp64.
 */
tri_status tri_score(const tri_model *m, const tri_kv_desc *kv, const void *K, const int32_t *pos,
                     const float *centres, const float *mean_norm, const int64_t *p_now,
                     const int32_t *offsets, int32_t n_offsets, int32_t key_mode, float *scores,
                     void *ws, size_t ws_bytes, tri_stream_t stream);

/*
 * Per-row top-B selection and stable compaction (digest, 流程详解 step 4).
 * For a row of N keys:
 *   N <= B: every slot is kept (identity compaction);
 *   N >  B: the last W slots are kept, plus the B - W best of slots
 *           0 .. N-W-1 under the order (score descending, slot descending),
 *           so exactly B keys survive and equal scores favour recent slots.
 *           NaN scores rank last (and set TRI_FLAG_NONFINITE).
 * Kept slots are emitted in ascending slot order, and K, V and pos of each
 * kept slot are copied bit for bit to the output.
 *   scores:     float, as written by tri_score for the same kv
 *   B, W:       1 <= B, 0 <= W <= B
 *   K, V, pos:  the cache in kv's layout (pos may be NULL if pos_out is NULL)
 *   out:        layout of the outputs; K_out/V_out 16-byte aligned, must not
 *               overlap K/V
 *   kept_idx:   optional int32 [R][B]: kept slots of row r at r*B .. r*B+cnt-1
 *   kept_count: optional int32 [R]: min(N, B) per row
 *   ws:         workspace of tri_workspace_size bytes
 * V, K_out, V_out and pos_out may also be page-locked host memory that the
 * device addresses at the same pointer (cudaHostAlloc, or cudaHostRegister
 * with cudaHostRegisterMapped, under unified addressing): only the kept
 * records of V then cross the host link, and the compacted cache is written
 * straight to host memory.  Pageable host memory must not be passed; the
 * library cannot tell it from device memory.
 */
tri_status tri_compact(const tri_model *m, const tri_kv_desc *kv, const float *scores, int32_t B,
                       int32_t W, const void *K, const void *V, const int32_t *pos,
                       const tri_out_desc *out, void *K_out, void *V_out, int32_t *pos_out,
                       int32_t *kept_idx, int32_t *kept_count, void *ws, size_t ws_bytes,
                       tri_stream_t stream);

/*
 * Synchronise `stream`, read the workspace flag word into *flags (may be
 * NULL), clear it, and return TRI_ERR_DEVICE_FLAG if any bit was set.
 */
tri_status tri_status_check(void *ws, uint32_t *flags, tri_stream_t stream);

/*
 * Online (decode-time) calibration update (digest, 流程详解 step 1, with the
 * calibration/deployment shift the digest flags as a risk in sections 不足 and
 * 复现注意事项): the centres of tri_calib maintained over a stream of query
 * batches.  Each call, per (layer l, query head g):
 *   sums   <- decay * sums + sum over this call's queries of (re q_f, im q_f, |q_f|)
 *   weight <- decay * weight + nq
 *   centres = sums[0..1] / weight,  mean_norm = sums[2] / weight
 * so a query that arrived k calls ago carries weight decay^k (decay = 1: the
 * plain mean of every query seen).  fp64 state and accumulation, fp32 outputs;
 * deterministic.
 *   qpre:      bf16 [n_layers][n_q_heads][nq][d] new pre-RoPE queries, 16-byte aligned
 *   nq:        queries per head in this call, >= 1
 *   decay:     0 < decay <= 1
 *   sums:      device double [n_layers][n_q_heads][d/2][3], caller-owned state,
 *              zeroed by the caller before the first call; updated in place
 *   weight:    device double [n_layers][n_q_heads], same ownership
 *   centres, mean_norm: outputs as for tri_calib
 */
tri_status tri_calib_update(const tri_model *m, const void *qpre, int64_t nq, double decay, double *sums,
                            double *weight, float *centres, float *mean_norm, tri_stream_t stream);

/*
 * Concentration and drift diagnostics of n_heads sets of centre statistics
 * (query heads from tri_calib / tri_calib_update, or cache rows from
 * tri_key_centres).  The premise of the method is that pre-RoPE Q/K
 * concentrate around their centres (digest, section 核心洞见); the digest flags
 * the sensitivity to calibration/deployment shift as open (sections 不足,
 * 复现注意事项).  Per head, in fp64:
 *   concentration[f] = |centre_f| / mean_norm_f   (0 where mean_norm_f = 0)
 *   head_stats[0]    = sum_f |centre_f| / sum_f mean_norm_f
 *   head_stats[1]    = sum_f (|centre_f - ref_f| + |mean_norm_f - ref_norm_f|) / sum_f ref_norm_f
 *                      (relative L1 drift; 0 when ref_centres is NULL)
 *   centres, mean_norm:         float [n_heads][d/2][2] (8-byte aligned), [n_heads][d/2]
 *   ref_centres, ref_mean_norm: the same shapes, or both NULL
 *   concentration:              float [n_heads][d/2] or NULL
 *   head_stats:                 float [n_heads][2] or NULL (not both NULL)
 */
tri_status tri_calib_stats(const tri_model *m, int64_t n_heads, const float *centres, const float *mean_norm,
                           const float *ref_centres, const float *ref_mean_norm, float *concentration,
                           float *head_stats, tri_stream_t stream);

/*
 * Pre-RoPE key centres of every cache row (digest, 流程详解 step 1 extracts the
 * centres of Q and K): per row r and pair f,
 *   centres[r][f]   = (1/N_r) sum_j k_f^pre(j)      (re, im)
 *   mean_norm[r][f] = (1/N_r) sum_j |k_f(j)|
 * (0 for an empty row).  key_mode TRI_KEYS_POST_ROPE: the cache holds RoPE'd
 * keys and each is de-rotated by e^{-i w_f pos} (pos required; phase reduced
 * exactly in 64-bit fixed-point turns); TRI_KEYS_PRE_ROPE: keys are used as
 * stored (pos may be NULL).  fp64 accumulation in a fixed order.
 *   kv, K, pos: the cache as for tri_score (bf16 or fp8, contiguous or paged)
 *   centres:    float [R][d/2][2];  mean_norm: float [R][d/2]
 *   ws:         tri_key_centres_ws_size bytes, 256-byte aligned; its first
 *               word is a flag word (TRI_FLAG_ROW_OFFSETS, TRI_FLAG_BLOCK_TABLE)
 *               read by tri_status_check
 */
size_t tri_key_centres_ws_size(const tri_model *m, int32_t n_seqs);
tri_status tri_key_centres(const tri_model *m, const tri_kv_desc *kv, const void *K, const int32_t *pos,
                           int32_t key_mode, float *centres, float *mean_norm, void *ws, size_t ws_bytes,
                           tri_stream_t stream);

/*
 * tri_score followed by tri_compact in one call (digest, 流程详解 steps 2-4),
 * with the scoring and the selection fused on chip where that pays:
 *   fused (max_row_len <= TRI_FUSED_PREFER_ROW, or `scores` NULL and
 *     max_row_len <= TRI_FUSED_MAX_ROW): one CTA per row keeps the row's
 *     scores in shared memory, selects from there and writes the kept slots;
 *     K, V and pos are then gathered.  `scores`, when given, receives the
 *     scores; when NULL they never leave the chip.  A row longer than
 *     TRI_FUSED_MAX_ROW keys (possible only when max_row_len understates the
 *     longest row) sets TRI_FLAG_ROW_OFFSETS and keeps nothing: its kept_count
 *     is 0, its kept_idx entries are -1 and its output records are left
 *     untouched.  Rows longer than max_row_len but within TRI_FUSED_MAX_ROW
 *     are processed normally.
 *   otherwise: exactly tri_score then tri_compact, `scores` (float
 *     [total_keys]) required.
 * Both ways give the same results bit for bit (the fused kernel runs the
 * score kernel's arithmetic in the same order), so the choice is only speed.
 * Arguments as for tri_score and tri_compact (V and the outputs may be mapped
 * page-locked host memory, as there); max_row_len is the caller's bound on the
 * longest row (for the compacted rounds of a serving loop, min(N, B) + the new
 * tokens).  Same workspace as tri_compact.
 */
#define TRI_FUSED_MAX_ROW 32768
#define TRI_FUSED_PREFER_ROW 8192
tri_status tri_score_compact(const tri_model *m, const tri_kv_desc *kv, const void *K, const void *V,
                             const int32_t *pos, const float *centres, const float *mean_norm, const int64_t *p_now,
                             const int32_t *offsets, int32_t n_offsets, int32_t key_mode, int32_t B, int32_t W,
                             int32_t max_row_len, const tri_out_desc *out, void *K_out, void *V_out,
                             int32_t *pos_out, int32_t *kept_idx, int32_t *kept_count, float *scores, void *ws,
                             size_t ws_bytes, tri_stream_t stream);

/*
 * Decode attention over a (compressed) cache (digest, 流程详解 step 5: every
 * later attention step reads only the compressed cache; weights unchanged).
 * For every layer l, sequence s and query head g (KV head h = g / G), over the
 * keys k_j and values v_j of row (l, s, h):
 *   s_j = softmax_scale * (q . k_j)
 *   out = sum_j e^{s_j} v_j / sum_j e^{s_j},   lse = log sum_j e^{s_j}
 * (out = 0 and lse = -inf for an empty row).  fp32 arithmetic: exact products
 * of the stored elements, fp32 sums, online softmax in base 2.
 *   kv, K, V:  the cache in either layout and element type; for the compacted
 *              cache of tri_compact, row_off holds the kept counts' prefix sums
 *              (contiguous [R][B] output with every row full: row_off[r] = r*B;
 *              paged output: the fresh block table, row r holding min(N_r, B) keys)
 *   q:         bf16 [n_layers][n_seqs][n_q_heads][d], RoPE'd at the position
 *              being decoded (2-byte aligned)
 *   softmax_scale: > 0 (usually 1/sqrt(d))
 *   out:       float [n_layers][n_seqs][n_q_heads][d]
 *   lse:       float [n_layers][n_seqs][n_q_heads] or NULL
 *   ws:        tri_attention_ws_size bytes, 256-byte aligned; first word is a
 *              flag word (TRI_FLAG_ROW_OFFSETS, TRI_FLAG_BLOCK_TABLE)
 * G = n_q_heads / n_kv_heads must be <= 16 (else TRI_ERR_UNSUPPORTED).
 */
size_t tri_attention_ws_size(const tri_model *m, int32_t n_seqs);
tri_status tri_decode_attention(const tri_model *m, const tri_kv_desc *kv, const void *K, const void *V,
                                const void *q, float softmax_scale, float *out, float *lse, void *ws,
                                size_t ws_bytes, tri_stream_t stream);

/*
 * tri_decode_attention on the 5th-generation tensor cores: the same result
 * (within fp32 rounding of a different summation order), for bf16 caches of
 * head dim 128 in the contiguous layout with G <= 16 and total_keys < 2^31;
 * anything else returns TRI_ERR_UNSUPPORTED before any launch.  Per 128-key
 * tile the keys fill the M side of tcgen05.mma (S^T = K Q^T, then O^T = V^T P^T
 * with the head dims on M, the queries padded to 16 columns on N), accumulators
 * in tensor memory, K and V tiles brought by TMA; softmax, its maximum and sums
 * as in tri_decode_attention.  On the workloads measured here it is slower than
 * tri_decode_attention (one 4-warp CTA per SM keeps too few tiles in flight;
 * the warp-level kernel runs 12 independent warps per SM), so
 * tri_decode_attention does not use it.  Same arguments, workspace and flags;
 * a copy or product that does not complete within 2 s sets
 * TRI_FLAG_STAGE_TIMEOUT.
 */
tri_status tri_decode_attention_tc(const tri_model *m, const tri_kv_desc *kv, const void *K, const void *V,
                                   const void *q, float softmax_scale, float *out, float *lse, void *ws,
                                   size_t ws_bytes, tri_stream_t stream);

/*
 * tri_score without a workspace argument, for callers that cannot allocate
 * device memory where they score: code running inside another framework's
 * memory pool that forbids foreign allocations, plugins whose host process
 * owns every device allocation, and serving loops that allocate everything
 * once at start-up.  The method pages have no counterpart to this call; it is
 * an interface convenience.
 *
 * Same arguments and results as tri_score, minus ws/ws_bytes.  The scratch is
 * a fixed array inside the library (about 6 MiB on every GPU that loads it,
 * held until the process exits), enough for at most TRI_NOALLOC_MAX_ROWS rows
 * (n_layers * n_seqs * n_kv_heads); more rows return
 * TRI_ERR_WORKSPACE_TOO_SMALL before anything is launched.  The call
 * allocates nothing.
 *  - Each call made outside a stream capture looks up the scratch's device
 *    address (cudaGetSymbolAddress) with the calling device current; a call
 *    made while `stream` is being captured reuses the last address found on
 *    that device.  Make the first call on each device before any stream
 *    capture there, and again after a cudaDeviceReset.
 *  - All calls on a device share the one scratch array: calls whose kernels
 *    can overlap on the GPU (other streams, other threads) race and must be
 *    serialised by the caller.
 *  - Data anomalies detected by the kernels are not reported (there is no
 *    workspace flag word to read); use tri_score with a workspace for those.
 */
#define TRI_NOALLOC_MAX_ROWS 4096
tri_status tri_score_noalloc(const tri_model *m, const tri_kv_desc *kv, const void *K, const int32_t *pos,
                             const float *centres, const float *mean_norm, const int64_t *p_now,
                             const int32_t *offsets, int32_t n_offsets, int32_t key_mode, float *scores,
                             tri_stream_t stream);

/*
 * tri_selftest_wait_timeout - exercises the bounded wait of the staged kernels.
 *
 * Kernels that stage keys in shared memory wait on a barrier that their bulk
 * copies complete; the wait gives up after a time limit and the kernel sets
 * TRI_FLAG_STAGE_TIMEOUT instead of hanging.  This call launches one warp that
 * waits on a barrier nothing ever completes, with the same wait and the limit
 * given here, so a caller can see that path end: after the stream reaches it,
 * tri_status_check(ws) returns TRI_ERR_DEVICE_FLAG with TRI_FLAG_STAGE_TIMEOUT
 * set, and the context remains usable.  No memory is accessed out of bounds
 * and nothing faults.
 *   ws, ws_bytes: a workspace of at least 256 bytes, 256-byte aligned (only its
 *             flag word is written).
 *   limit_ns:  the wait's limit, 1 us .. 10 s.
 * Returns TRI_OK once the kernel is enqueued; TRI_ERR_INVALID_ARG,
 * TRI_ERR_ALIGNMENT or TRI_ERR_WORKSPACE_TOO_SMALL for bad arguments (nothing
 * launched); TRI_ERR_CUDA when the launch fails.
 */
tri_status tri_selftest_wait_timeout(void *ws, size_t ws_bytes, uint64_t limit_ns, tri_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TRI_H */
