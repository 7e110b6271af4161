/*
 * qi21.h — C ABI of the B200 (sm_100a) cached Flow-Matching Euler step of a
 * single-stream, Qwen-Image-2.1-style diffusion transformer with a prefix K/V
 * cache.
 *
 * Sources (course pages on Qwen-Image-2.1; section names as on the pages):
 *   [LAB]  "Bài Lab tổng hợp — Qwen-Image-2.1 Architecture": the 1:1 mapping
 *          table and the NumPy lab qwen-image-21.py, blocks [1A] .. [6B].
 *   [E2E]  "Lab tổng hợp Qwen-Image-2.1 — chạy toàn trình 1A → 6B bằng NumPy",
 *          §1 Định nghĩa, §3 Giải pháp, §4 Profiling.
 *   [6B]   "6B · Scale-Only Final AdaLN, Dự đoán vận tốc v_θ & Vòng lặp 8-Step Euler".
 *   [3B]   "3B · Điều kiện nhân quả (t=0 vs t) & Bộ điều biến dùng chung".
 *   [2A]   "2A · Mở rộng 4× Slot ảnh & Ghép chuỗi đồng nhất".
 *
 * Conventions for every entry point
 *   - Device pointers are plain CUDA device addresses owned by the caller. The
 *     library never allocates or frees device memory; scratch comes from the
 *     caller's workspace (see qi21_workspace_bytes).
 *   - Work is enqueued on the given cudaStream_t (passed as void*; NULL is the
 *     legacy default stream). No call synchronises the host except
 *     qi21_check_device_error.
 *   - Matrices are row-major. Weights use the torch.nn.Linear order
 *     [out][in]; per-layer weights are stacked on a leading layer axis.
 *   - Every device pointer must be 16-byte aligned; otherwise QI21_ERR_INVALID_ARG.
 *   - Host-detectable errors return before anything is enqueued. A device-side
 *     bounded wait that expires sets an error word in the workspace, the
 *     kernel returns, and qi21_check_device_error reports QI21_ERR_DEVICE_TIMEOUT.
 *   - Every function is thread-compatible (no hidden global state besides the
 *     optional per-kernel timing of qi21_profile_*).
 */
#ifndef QI21_H
#define QI21_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t qi21_status;
enum {
    QI21_OK = 0,
    QI21_ERR_INVALID_ARG = 1,      /* null / misaligned pointer, bad enum value */
    QI21_ERR_SHAPE = 2,            /* inconsistent sizes (d != H*Dh, N == 0 ...) */
    QI21_ERR_METADATA = 3,         /* target not last, empty segment, bad coords */
    QI21_ERR_CACHE_STATE = 4,      /* cached step before extract, or cache shape mismatch */
    QI21_ERR_UNSUPPORTED = 5,      /* shape the selected kernel family does not cover */
    QI21_ERR_CUDA = 6,             /* a CUDA runtime / driver call failed */
    QI21_ERR_DEVICE_TIMEOUT = 7,   /* a bounded device wait expired */
    QI21_ERR_WORKSPACE_TOO_SMALL = 8,
    QI21_ERR_DEVICE_CHECK = 9      /* a kernel's own layout check failed; it returned without work */
};

/* Storage dtype of weights, activations and the K/V cache. The residual
 * stream, LayerNorm statistics, softmax and all accumulators are fp32 in
 * both modes. F32 runs CUDA-core kernels (the parity mode); BF16 runs the
 * tcgen05 tensor-core GEMMs and attention (the throughput mode). */
enum { QI21_DTYPE_F32 = 0, QI21_DTYPE_BF16 = 1 };

/* Model configuration.
 *   d_model = n_heads * head_dim; mlp_hidden = SwiGLU width; latent_ch = C
 *   (64 in production, [LAB] 1A); time_dim = width of the sin-cos timestep
 *   embedding ([3B] §1).
 *   use_shift = 0: modulation rows hold 4 chunks [scale1, gate1, scale2, gate2]
 *   ([3B] §1-§2, scale-only AdaLN). use_shift = 1: 6 chunks
 *   [shift1, scale1, gate1, shift2, scale2, gate2] as in the NumPy lab
 *   ([LAB] 3B); the modulated LayerNorm then adds the shift.
 *   ln_eps: LayerNorm epsilon; qk_eps: QK-RMSNorm epsilon (1e-6 in [LAB]). */
typedef struct {
    int32_t d_model, n_heads, head_dim, n_layers, mlp_hidden, latent_ch, time_dim;
    int32_t dtype;
    int32_t use_shift;
    float ln_eps, qk_eps;
} qi21_config;

/* One segment of the packed sequence ([2A] §1-§2): TEXT with n_text tokens,
 * or IMAGE with an h x w latent grid (patch size 1, row-major). Condition
 * images take ids 0..K-1 in order; the LAST segment must be the target image. */
enum { QI21_SEG_TEXT = 0, QI21_SEG_IMAGE = 1 };
typedef struct {
    int32_t kind;
    int32_t n_text;
    int32_t h, w;
} qi21_segment;

/* Device weights (dtype of the config unless stated), [out][in] order.
 *   w_img_in [d][C]        img_in, latent -> token ([LAB] 1A, patch size 1)
 *   w_out    [C][d]        proj_out -> v_theta ([6B] §1)
 *   w_t1     [d][time_dim], w_t2 [d][d]   timestep MLP ([3B] §1; shape is a reading)
 *   w_mod    [chunks*d][d] shared modulation Linear ([3B] §1)
 *   w_fin    [d][d]        final AdaLN scale Linear ([6B] §3)
 *   w_q, w_k, w_v, w_o     [L][d][d]
 *   w_gate, w_up           [L][F][d]
 *   w_down                 [L][d][F]
 *   q_norm, k_norm         [L][head_dim] float32: QK-RMSNorm weights w, applied as (1 + w). */
typedef struct {
    const void *w_img_in, *w_out;
    const void *w_t1, *w_t2, *w_mod, *w_fin;
    const void *w_q, *w_k, *w_v, *w_o;
    const void *w_gate, *w_up, *w_down;
    const float *q_norm, *k_norm;
} qi21_weights;

/* The same weights as row-major [in][out] matrices (the lab's y = x @ W), device
 * pointers in the config dtype, per-layer tensors stacked on a leading layer axis:
 *   w_img_in [C][d], w_out [d][C], w_t1 [time_dim][d], w_t2 [d][d],
 *   w_mod [d][chunks*d], w_fin [d][d], w_q/w_k/w_v/w_o [L][d][d],
 *   w_gate/w_up [L][d][F], w_down [L][F][d]; q_norm, k_norm [L][head_dim] float32. */
typedef struct {
    const void *w_img_in, *w_out;
    const void *w_t1, *w_t2, *w_mod, *w_fin;
    const void *w_q, *w_k, *w_v, *w_o;
    const void *w_gate, *w_up, *w_down;
    const float *q_norm, *k_norm;
} qi21_weights_canonical;

/* Prefix K/V cache ([LAB] 6A; [E2E] §6 "kv_cache_mode"): one caller-owned
 * device buffer of qi21_kv_cache_bytes(), laid out [L][2 (K,V)][B][P+N][d]
 * in the config dtype. For layer l, item b, row r, head h, dim j the K value
 * sits at ((l*2 + 0)*B + b)*(P+N)*d + r*d + h*head_dim + j. Rows [0, P) hold
 * the prefix K (after QK-RMSNorm and RoPE) and raw V written by
 * qi21_prefix_extract; rows [P, P+N) are rewritten by every cached step with
 * that step's target K/V. state: QI21_CACHE_EMPTY until an extract succeeds. */
enum { QI21_CACHE_EMPTY = 0, QI21_CACHE_EXTRACTED = 1 };

/* Shared-prefix layout (denoise batching: several requests with the same text
 * and reference images, [LAB] 6A "prefix K/V computed once, used by every
 * step"): one prefix for all `batch` target requests. Per layer
 * [2 (K,V)][Pp + batch*N][d], Pp = P rounded up to QI21_ATTN_KEY_TILE: rows
 * [0, P) hold the prefix K/V written by one extract (prefix_hidden [1][P][d]),
 * rows [P, Pp) are never read, and rows [Pp + b*N, Pp + (b+1)*N) hold request
 * b's target K/V of the current step. Every request's attention reads the one
 * copy of the prefix rows. Built by qi21_kv_cache_init_shared. */
#define QI21_ATTN_KEY_TILE 128
typedef struct {
    void *base;
    int32_t batch, n_prefix, n_target;
    int32_t n_layers, d_model, dtype;
    int32_t state;
    int32_t shared_prefix;   /* 0: [L][2][B][P+N][d]; 1: the shared-prefix layout above */
} qi21_kv_cache;

/* ---------------------------------------------------------------- host helpers */

/* Packing metadata of a segment list ([2A] §1 build_token_metadata; [LAB] 3A,
 * 3C). Host-only and pure. Outputs (each caller-allocated host array of S
 * entries, any may be NULL): image_ids (-1 text, 0..K-1 condition images, K
 * target), target_mask (1 on target tokens), coords [S][3] = (frame, h, w)
 * (text (i,i,i) counting text tokens; images frame 0 — or the image id when
 * frame_mode = 1 — and grid r - H/2, c - W/2), kv_limit (row q may attend to
 * keys [0, kv_limit[q]): q+1 for text, the end of its image's run otherwise;
 * exactly the block-causal rule (q >= kv) or same image id).
 * Pass image_ids = NULL etc. with capacity 0 to query S, P, N first.
 * Returns QI21_ERR_METADATA if the last segment is not an image, a segment is
 * empty, or capacity < S. */
qi21_status qi21_build_metadata(const qi21_segment *segments, int32_t n_segments,
                                int32_t frame_mode, int32_t capacity,
                                int32_t *image_ids, uint8_t *target_mask,
                                int32_t *coords, int32_t *kv_limit,
                                int32_t *S, int32_t *P, int32_t *N);

/* Axial RoPE frequencies omega [head_dim/2][3] (host). Production split
 * ([LAB] 3A notes): head_dim 128 -> (frame 16, height 56, width 56) dims,
 * i.e. 8 + 28 + 28 pairs, omega = base^(-2j/dim_axis); other head dims scale
 * the split by head_dim/128 (head_dim % 16 == 0). */
qi21_status qi21_rope_omega_axial(int32_t head_dim, double base, double *omega);

/* cos/sin table [S][head_dim/2][2] float32 (host, computed in fp64): angle of
 * pair j at token s = sum_a coords[s][a] * omega[j][a]; entry = (cos, sin).
 * The kernels rotate adjacent pairs (2j, 2j+1) as in [LAB] 3A. */
qi21_status qi21_rope_table(int32_t head_dim, const int32_t *coords, int32_t S,
                            const double *omega, float *cos_sin);

/* Latent cells per VLM image slot: one slot stands for a 2x2 block ([2A]). */
#define QI21_IMG_TOKENS_PER_SLOT 4

/* Index tables of the joint packing of the prefix values ([2A] mechanisms (1)
 * and (2); [LAB] 2A repeats = where(img_mask, 4, 1)). Host-only and pure.
 * Over the prefix (every segment but the last, the target): a text token is
 * one VLM slot; an image of h*w latent cells (h*w divisible by 4) has h*w/4
 * slots, each written at 4 consecutive positions of the image's run.
 *   slot_of [P]: the slot each prefix token expands (index into ctx rows)
 *   img_row [P]: row of the img_in token table at image positions (reference
 *                images in order, raster order inside each), -1 at text positions
 * Host arrays of capacity entries, either may be NULL; pass both NULL to query
 * P, n_slots (rows of ctx) and n_img (rows of the img_in token table).
 * Returns QI21_ERR_METADATA for an empty segment, an image whose cell count is
 * not a multiple of 4, a last segment that is not an image, or capacity < P. */
qi21_status qi21_build_packing(const qi21_segment *segments, int32_t n_segments, int32_t capacity,
                               int32_t *slot_of, int32_t *img_row, int32_t *P,
                               int32_t *n_slots, int32_t *n_img);

/* The lab's micro RoPE split for head_dim 4 ([LAB] 3A), omega [2][3] (host):
 * pair 0 turns with the frame axis at rate 1; pair 1 is shared by height
 * (rate base^-1) and width (rate base^-1.5), the two angles adding. */
qi21_status qi21_rope_omega_lab(double base, double *omega);

/* Timestep of a noise level: t = QI21_T_PER_SIGMA * sigma ([3B] §1; [6B] §3). */
#define QI21_T_PER_SIGMA 1000.0

/* Sin-cos timestep embedding [time_dim] (host, fp64 math, float result):
 * [cos(t f_i) ..., sin(t f_i) ...], f_i = 10000^(-2i/time_dim), t = 1000*sigma
 * ([LAB] 3B, [3B] §1). */
qi21_status qi21_timestep_embedding(double t, int32_t time_dim, float *emb);

/* Bytes of the packed weight buffer of qi21_pack_weights (every tensor in the
 * [out][in] layout of qi21_weights, each starting on a 256-byte boundary). */
size_t qi21_packed_weights_bytes(const qi21_config *cfg);

/* Sizes in bytes of the caller-allocated buffers. */
size_t qi21_kv_cache_bytes(const qi21_config *cfg, int32_t batch, int32_t n_prefix, int32_t n_target);
/* Workspace large enough for every entry point with these sizes
 * (the full recompute over S = P + N tokens is the largest). */
size_t qi21_workspace_bytes(const qi21_config *cfg, int32_t batch, int32_t n_prefix, int32_t n_target);

/* Initialise a cache descriptor over caller memory (state EMPTY). */
qi21_status qi21_kv_cache_init(qi21_kv_cache *cache, void *base, const qi21_config *cfg,
                               int32_t batch, int32_t n_prefix, int32_t n_target);
/* The shared-prefix layout: bytes, and a descriptor (shared_prefix = 1). */
size_t qi21_kv_cache_bytes_shared(const qi21_config *cfg, int32_t batch, int32_t n_prefix, int32_t n_target);
qi21_status qi21_kv_cache_init_shared(qi21_kv_cache *cache, void *base, const qi21_config *cfg,
                                      int32_t batch, int32_t n_prefix, int32_t n_target);

/* ---------------------------------------------------------------- device entry points */

/* Shared modulation ([3B] §1-§2; [6B] §3): for timestep t (= 1000*sigma),
 *   e = w_t2 . silu(w_t1 . emb(t)),  mod_row = w_mod . silu(e)  [chunks*d],
 *   scale_final = w_fin . silu(e)  [d]   (device float32 outputs).
 * The prefix row is mod_row at t = 0 (computed once per image); the target
 * row is recomputed every step. ws: workspace of >= qi21_workspace_bytes. */
qi21_status qi21_modulation(const qi21_config *cfg, const qi21_weights *w, double t,
                            float *mod_row, float *scale_final,
                            void *ws, size_t ws_bytes, void *stream);

/* qi21_modulation at the timestep of noise level sigma, t = QI21_T_PER_SIGMA * sigma
 * (formed on the host in fp64). */
qi21_status qi21_modulation_sigma(const qi21_config *cfg, const qi21_weights *w, double sigma,
                                  float *mod_row, float *scale_final,
                                  void *ws, size_t ws_bytes, void *stream);

/* Largest d_model qi21_modulation_noalloc accepts: its scratch is a fixed
 * device array of 2 * QI21_NOALLOC_MAX_D floats (64 KB on every GPU that
 * loads the library, held until the process exits). */
#define QI21_NOALLOC_MAX_D 8192

/* The pages have no counterpart to this call; it exists for callers of the
 * library that cannot allocate device memory (their device memory is owned by
 * another allocator, or they must never call cudaMalloc because it can block).
 * Same result as qi21_modulation, but takes no workspace: its two
 * timestep-MLP intermediate vectors live in a fixed file-scope device array of
 * 2 * QI21_NOALLOC_MAX_D floats instead. Applies the shape checks of
 * qi21_modulation and returns QI21_ERR_UNSUPPORTED when d_model >
 * QI21_NOALLOC_MAX_D, before anything is enqueued; a failed launch returns
 * QI21_ERR_CUDA. Allocates nothing and calls no allocating routine. The first call
 * on a device looks up that device's address of the array
 * (cudaGetSymbolAddress, with the device current), so make that first call
 * before any stream capture. Every call on a device shares the one array and
 * overwrites what the previous call left there: calls that overlap on the GPU
 * (for instance on two streams) race and must be serialised by the caller. */
qi21_status qi21_modulation_noalloc(const qi21_config *cfg, const qi21_weights *w, double t,
                                    float *mod_row, float *scale_final, void *stream);

/* Prefix extract ([LAB] 6A mode "extract"; [E2E] §3): run the L blocks over
 * the P prefix rows of every batch item with the prefix modulation row (t = 0
 * under causal_condition, [3B] §1) and the block-causal mask given as
 * kv_limit_prefix [P] (device int32, from qi21_build_metadata), writing K
 * (post QK-RMSNorm, post RoPE) and V of every layer into cache rows [0, P).
 *   prefix_hidden  [B][P][d] float32 device (joint hidden states of the prefix)
 *   cos_sin_prefix [P][head_dim/2][2] float32 device
 *   mod_row_prefix [chunks*d] float32 device
 * With a shared-prefix cache (qi21_kv_cache_init_shared) there is one prefix
 * for all requests: prefix_hidden is [1][P][d] and rows [0, P) of the single
 * prefix block are written.
 * On success cache->state = QI21_CACHE_EXTRACTED. */
qi21_status qi21_prefix_extract(const qi21_config *cfg, const qi21_weights *w,
                                qi21_kv_cache *cache, const float *prefix_hidden,
                                const float *cos_sin_prefix, const int32_t *kv_limit_prefix,
                                const float *mod_row_prefix,
                                void *ws, size_t ws_bytes, void *stream);

/* Cached step ([LAB] 6A mode "cached", 6B; [E2E] §3): v_theta for the N
 * target tokens of every item. Only target rows run the blocks: img_in(x_k),
 * then per block LN(h)(1+scale1) -> Q,K,V -> QK-RMSNorm -> RoPE -> attention
 * over [cached prefix K/V; this step's target K/V] (all P+N keys: the target
 * is last) -> h += tanh(gate1)(o Wo) -> LN(h)(1+scale2) -> SwiGLU ->
 * h += tanh(gate2)(. Wdown); then v = (LN(h)(1+scale_final)) Wout.
 *   x_k            [B][N][C] float32 device (current latent, standardised space)
 *   cos_sin_target [N][head_dim/2][2] float32 device
 *   mod_row_target [chunks*d], scale_final [d] float32 device (from qi21_modulation)
 *   v_out          [B][N][C] float32 device
 * Returns QI21_ERR_CACHE_STATE unless the cache was extracted with matching
 * sizes. Writes cache rows [P, P+N) (target K/V of this step); with a
 * shared-prefix cache, request b's rows [Pp + b*N, Pp + (b+1)*N), and every
 * request's attention reads the one copy of the prefix rows. */
qi21_status qi21_cached_step(const qi21_config *cfg, const qi21_weights *w,
                             const qi21_kv_cache *cache, const float *x_k,
                             const float *cos_sin_target, const float *mod_row_target,
                             const float *scale_final, float *v_out,
                             void *ws, size_t ws_bytes, void *stream);

/* Full recomputation ([LAB] run_pipeline with use_cache=False; [E2E] §4):
 * every one of the S = P + N tokens runs every block with the block-causal
 * mask (kv_limit_all [S] device int32); prefix rows read mod_row_prefix,
 * target rows mod_row_target ([3B] _select_modulation_rows). No cache is
 * read or written (K/V live in the workspace). Used to check the cache path.
 *   prefix_hidden [B][P][d] f32, x_k [B][N][C] f32, cos_sin_all [S][Dh/2][2] f32,
 *   v_out [B][N][C] f32. */
qi21_status qi21_full_recompute_step(const qi21_config *cfg, const qi21_weights *w,
                                     int32_t batch, int32_t n_prefix, int32_t n_target,
                                     const float *prefix_hidden, const float *x_k,
                                     const float *cos_sin_all, const int32_t *kv_limit_all,
                                     const float *mod_row_prefix, const float *mod_row_target,
                                     const float *scale_final, float *v_out,
                                     void *ws, size_t ws_bytes, void *stream);

/* Flow-Match Euler update ([6B] §1): x_out = x_k + (sigma_k1 - sigma_k) * v,
 * n float32 elements; the difference is formed in fp64 on the host.
 * x_out may alias x_k. */
qi21_status qi21_euler_update(const float *x_k, const float *v, double sigma_k, double sigma_k1,
                              float *x_out, int64_t n, void *stream);

/* Pack canonical [in][out] weights into the layout the kernels read: every
 * matrix transposed to [out][in] (layer by layer for stacked tensors) into the
 * caller's device buffer `packed` (qi21_packed_weights_bytes bytes, 256-byte
 * aligned), the QK-norm vectors copied; *w receives pointers into `packed`.
 * Data movement only: exact. Returns QI21_ERR_INVALID_ARG for null or
 * misaligned pointers, QI21_ERR_WORKSPACE_TOO_SMALL if packed_bytes is short. */
qi21_status qi21_pack_weights(const qi21_config *cfg, const qi21_weights_canonical *canonical,
                              void *packed, size_t packed_bytes, qi21_weights *w, void *stream);

/* Joint packing of the prefix values on the device ([2A] mechanisms (1)-(2);
 * [LAB] 2A). For item b and prefix token s:
 *   mode QI21_PACK_SUBSTITUTE (the 2A page): out = img_row[s] >= 0 ?
 *       img_tokens[b][img_row[s]] : ctx[b][slot_of[s]]
 *   mode QI21_PACK_ADD (the lab's COND_TOKENS): out = ctx[b][slot_of[s]]
 *       (+ img_tokens[b][img_row[s]] at image positions, one float32 add)
 *   ctx [B][n_slots][d] f32 device: VLM slot vectors (text slots after txt_in)
 *   img_tokens [B][n_img][d] f32 device: img_in tokens of the reference images
 *   slot_of, img_row [P] int32 device (from qi21_build_packing; the indices
 *       are trusted: they must lie in [0, n_slots) and [-1, n_img))
 *   out [B][P][d] f32 device: prefix_hidden for qi21_prefix_extract.
 * Pure data movement (plus the add): bit-exact. Returns QI21_ERR_INVALID_ARG
 * for null or misaligned pointers, d % 4 != 0 or a bad mode. */
#define QI21_PACK_SUBSTITUTE 0
#define QI21_PACK_ADD 1
qi21_status qi21_pack_prefix(int32_t batch, int32_t P, int32_t d, int32_t n_slots, int32_t n_img,
                             const float *ctx, const float *img_tokens, const int32_t *slot_of,
                             const int32_t *img_row, int32_t mode, float *out, void *stream);

/* img_in of latents on the device ([LAB] 1A, patch size 1): out [rows][d] f32 =
 * latents [rows][C] f32 x w_img_in^T, the projection the cached step applies to
 * the target latent; here for the reference images' latents before packing. */
qi21_status qi21_img_in_tokens(const qi21_config *cfg, const qi21_weights *w, const float *latents,
                               int32_t rows, float *out, void *stream);

/* Device-indexed forms for captured sequences (CUDA graphs): the sigma of a
 * step is read on the device from sigmas, a table of float64 values in device
 * memory (8-byte aligned, caller-owned, at least step + 2 entries), so one
 * captured sequence serves any sigma schedule written into the table before a
 * replay. qi21_modulation_at computes the embedding of t = t_per_sigma *
 * sigmas[step] on the device in fp64 (the pages use t = 1000 * sigma, [3B] §1;
 * [6B] §3) and otherwise equals qi21_modulation; qi21_euler_update_at applies
 * x_out = x_k + (sigmas[step+1] - sigmas[step]) * v with the difference formed
 * in fp64 on the device ([6B] §1). Invalid pointers or step < 0 return
 * QI21_ERR_INVALID_ARG before anything is enqueued; the table is not bounds-
 * checked on the device. */
qi21_status qi21_modulation_at(const qi21_config *cfg, const qi21_weights *w, const double *sigmas,
                               int32_t step, double t_per_sigma, float *mod_row, float *scale_final,
                               void *ws, size_t ws_bytes, void *stream);
qi21_status qi21_euler_update_at(const float *x_k, const float *v, const double *sigmas, int32_t step,
                                 float *x_out, int64_t n, void *stream);

/* Whole image ([6B] §4 the 8-step Euler loop; [E2E] §3 extract once, then
 * cached steps): enqueues, on one stream and with no host synchronisation,
 *   mod_row_prefix = modulation(t = 0); qi21_prefix_extract;
 *   for k in [0, n_steps): modulation_at(k) -> mod_row_target, scale_final;
 *                          qi21_cached_step(x) -> v; x = euler_update_at(k)
 * so that the whole call can be captured once into a CUDA graph and replayed
 * per image (make one uncaptured call first: it sets kernel attributes).
 *   prefix_hidden [B][P][d] f32; cos_sin_prefix [P][Dh/2][2], kv_limit_prefix [P],
 *   cos_sin_target [N][Dh/2][2]; sigmas [n_steps+1] f64 device;
 *   x [B][N][C] f32: x_0 in, x_{n_steps} out; v [B][N][C] f32 scratch (last v);
 *   mod_row_prefix, mod_row_target [chunks*d], scale_final [d] f32 scratch.
 * All device buffers are the caller's. Stops at the first failing call and
 * returns its status. */
qi21_status qi21_denoise_image(const qi21_config *cfg, const qi21_weights *w, qi21_kv_cache *cache,
                               const float *prefix_hidden, const float *cos_sin_prefix,
                               const int32_t *kv_limit_prefix, const float *cos_sin_target,
                               const double *sigmas, int32_t n_steps, double t_per_sigma, float *x,
                               float *v, float *mod_row_prefix, float *mod_row_target,
                               float *scale_final, void *ws, size_t ws_bytes, void *stream);

/* Synchronise the stream, then read and clear the device error word of the
 * workspace. Returns QI21_OK, QI21_ERR_DEVICE_TIMEOUT, QI21_ERR_DEVICE_CHECK or
 * QI21_ERR_CUDA. */
qi21_status qi21_check_device_error(void *ws, size_t ws_bytes, void *stream);

const char *qi21_status_string(qi21_status s);

/* Self test of the failure path (not part of the pages' method): launches a
 * kernel whose single bounded wait can never be satisfied, with a limit of
 * limit_ns nanoseconds (1 .. 10^9). The wait gives up, sets the workspace's
 * device error word and the kernel returns normally, so
 * qi21_check_device_error must then report QI21_ERR_DEVICE_TIMEOUT (and clear
 * the word). Nothing traps, faults or hangs. */
qi21_status qi21_selftest_wait_timeout(void *ws, size_t ws_bytes, int64_t limit_ns, void *stream);

/* ---------------------------------------------------------------- per-kernel timing */

/* When enabled, the entry points record a CUDA event pair on their stream
 * around every kernel launch, grouped by kernel name. qi21_profile_read
 * synchronises the recorded events and returns, for each kernel name, the
 * launch count and total milliseconds (names are static strings).
 * Returns the number of entries written. Off by default. */
typedef struct {
    const char *name;
    int64_t launches;
    double total_ms;
} qi21_kernel_time;
void qi21_profile_enable(int32_t enable);
int32_t qi21_profile_read(qi21_kernel_time *out, int32_t max_entries);
void qi21_profile_reset(void);

/* Kernel family of the BF16 mode: 1 (default) the tcgen05 tensor-core GEMMs
 * and attention; 0 the CUDA-core kernels of the F32 mode run on bf16 storage
 * (differential testing of the two families). Process-wide. */
void qi21_set_tensor_cores(int32_t enable);

/* Kernel family the block stack of cfg runs on under the current setting:
 * QI21_FAMILY_TENSOR_CORES (BF16 with tensor cores enabled and a supported
 * shape), QI21_FAMILY_CUDA_CORES (F32, or BF16 with tensor cores switched
 * off), or QI21_FAMILY_NONE when the entry points refuse cfg (an invalid
 * config, or a BF16 shape the tensor-core kernels do not cover: d_model a
 * multiple of 256, head_dim 64 or 128, mlp_hidden a multiple of 128). BF16
 * never falls back to the CUDA-core kernels on its own: such a config returns
 * QI21_ERR_UNSUPPORTED from every device entry point. */
enum { QI21_FAMILY_NONE = -1, QI21_FAMILY_CUDA_CORES = 0, QI21_FAMILY_TENSOR_CORES = 1 };
int32_t qi21_kernel_family(const qi21_config *cfg);

/* Library version string and the number of kernels the last entry point call
 * enqueued (for launch accounting). */
const char *qi21_version(void);
int32_t qi21_last_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* QI21_H */
