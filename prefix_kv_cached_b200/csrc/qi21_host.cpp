// Host-side helpers of the C ABI: packing metadata, RoPE tables, timestep
// embedding, buffer sizes. Pure C++ (no CUDA); see include/qi21.h.
#include "qi21.h"
#include "qi21_internal.h"

#include <cmath>
#include <cstring>

bool qi21_config_ok(const qi21_config *c);

extern "C" qi21_status qi21_build_metadata(const qi21_segment *seg, int32_t n_seg, int32_t frame_mode,
                                           int32_t capacity, int32_t *image_ids, uint8_t *target_mask,
                                           int32_t *coords, int32_t *kv_limit, int32_t *S_out,
                                           int32_t *P_out, int32_t *N_out) {
    // 2A page §1 (build_token_metadata) and the lab's [3A]/[3C] blocks.
    if (!seg || n_seg <= 0) return QI21_ERR_INVALID_ARG;
    if (frame_mode != 0 && frame_mode != 1) return QI21_ERR_INVALID_ARG;
    if (seg[n_seg - 1].kind != QI21_SEG_IMAGE) return QI21_ERR_METADATA;
    int64_t S = 0, n_img = 0;
    for (int i = 0; i < n_seg; ++i) {
        if (seg[i].kind == QI21_SEG_TEXT) {
            if (seg[i].n_text <= 0) return QI21_ERR_METADATA;
            S += seg[i].n_text;
        } else if (seg[i].kind == QI21_SEG_IMAGE) {
            if (seg[i].h <= 0 || seg[i].w <= 0) return QI21_ERR_METADATA;
            S += (int64_t)seg[i].h * seg[i].w;
            ++n_img;
        } else {
            return QI21_ERR_INVALID_ARG;
        }
    }
    if (S > INT32_MAX / 4) return QI21_ERR_SHAPE;
    const int64_t N = (int64_t)seg[n_seg - 1].h * seg[n_seg - 1].w;
    if (S_out) *S_out = (int32_t)S;
    if (P_out) *P_out = (int32_t)(S - N);
    if (N_out) *N_out = (int32_t)N;
    const bool want = image_ids || target_mask || coords || kv_limit;
    if (!want) return QI21_OK;
    if (capacity < S) return QI21_ERR_METADATA;
    int64_t pos = 0, text_i = 0, img = 0;
    for (int i = 0; i < n_seg; ++i) {
        if (seg[i].kind == QI21_SEG_TEXT) {
            for (int t = 0; t < seg[i].n_text; ++t, ++pos, ++text_i) {
                if (image_ids) image_ids[pos] = -1;
                if (target_mask) target_mask[pos] = 0;
                if (coords) {
                    coords[pos * 3 + 0] = (int32_t)text_i;
                    coords[pos * 3 + 1] = (int32_t)text_i;
                    coords[pos * 3 + 2] = (int32_t)text_i;
                }
                if (kv_limit) kv_limit[pos] = (int32_t)(pos + 1);      // causal text row
            }
        } else {
            const int H = seg[i].h, W = seg[i].w;
            const int64_t run_end = pos + (int64_t)H * W;
            for (int r = 0; r < H; ++r)
                for (int c = 0; c < W; ++c, ++pos) {
                    if (image_ids) image_ids[pos] = (int32_t)img;
                    if (target_mask) target_mask[pos] = (img == n_img - 1) ? 1 : 0;
                    if (coords) {
                        coords[pos * 3 + 0] = frame_mode == 1 ? (int32_t)img : 0;
                        coords[pos * 3 + 1] = r - H / 2;
                        coords[pos * 3 + 2] = c - W / 2;
                    }
                    // (q >= kv) or same image: the allowed keys are [0, end of this run)
                    if (kv_limit) kv_limit[pos] = (int32_t)run_end;
                }
            ++img;
        }
    }
    return QI21_OK;
}

extern "C" qi21_status qi21_rope_omega_axial(int32_t head_dim, double base, double *omega) {
    if (!omega || head_dim <= 0 || head_dim % 16 != 0 || !(base > 1.0)) return QI21_ERR_INVALID_ARG;
    const int dims[3] = {head_dim / 8, head_dim * 7 / 16, head_dim * 7 / 16};
    std::memset(omega, 0, sizeof(double) * (size_t)(head_dim / 2) * 3);
    int p = 0;
    for (int a = 0; a < 3; ++a)
        for (int j = 0; j < dims[a] / 2; ++j, ++p) omega[p * 3 + a] = std::pow(base, -2.0 * j / dims[a]);
    return p == head_dim / 2 ? QI21_OK : QI21_ERR_SHAPE;
}

extern "C" qi21_status qi21_rope_omega_lab(double base, double *omega) {
    // [LAB] 3A micro split: pair 0 = frame at rate 1; pair 1 = height at
    // base^-1 plus width at base^-1.5.
    if (!omega || !(base > 1.0)) return QI21_ERR_INVALID_ARG;
    const double v[6] = {1.0, 0.0, 0.0, 0.0, std::pow(base, -1.0), std::pow(base, -1.5)};
    std::memcpy(omega, v, sizeof(v));
    return QI21_OK;
}

extern "C" qi21_status qi21_rope_table(int32_t head_dim, const int32_t *coords, int32_t S,
                                       const double *omega, float *cos_sin) {
    if (!coords || !omega || !cos_sin || head_dim <= 0 || head_dim % 2 || S < 0) return QI21_ERR_INVALID_ARG;
    const int half = head_dim / 2;
    for (int64_t s = 0; s < S; ++s)
        for (int j = 0; j < half; ++j) {
            double ang = 0.0;
            for (int a = 0; a < 3; ++a) ang += (double)coords[s * 3 + a] * omega[j * 3 + a];
            cos_sin[(s * half + j) * 2 + 0] = (float)std::cos(ang);
            cos_sin[(s * half + j) * 2 + 1] = (float)std::sin(ang);
        }
    return QI21_OK;
}

extern "C" qi21_status qi21_timestep_embedding(double t, int32_t time_dim, float *emb) {
    if (!emb || time_dim <= 0 || time_dim % 2) return QI21_ERR_INVALID_ARG;
    const int half = time_dim / 2;
    for (int i = 0; i < half; ++i) {
        const double f = std::pow(10000.0, -2.0 * i / time_dim);
        emb[i] = (float)std::cos(t * f);
        emb[half + i] = (float)std::sin(t * f);
    }
    return QI21_OK;
}

extern "C" qi21_status qi21_build_packing(const qi21_segment *seg, int32_t n_seg, int32_t capacity,
                                          int32_t *slot_of, int32_t *img_row, int32_t *P_out,
                                          int32_t *n_slots_out, int32_t *n_img_out) {
    // 2A page, mechanisms (1) and (2): each text token is one VLM slot; an image of
    // h*w latent cells has h*w/4 slots, each repeated at 4 consecutive positions
    // (repeat_interleave); image positions also index the table of img_in tokens
    // (reference images in order, raster order inside an image).
    if (!seg || n_seg <= 0) return QI21_ERR_INVALID_ARG;
    if (seg[n_seg - 1].kind != QI21_SEG_IMAGE) return QI21_ERR_METADATA;
    int64_t P = 0, slots = 0, cells_total = 0;
    for (int i = 0; i < n_seg - 1; ++i) {
        if (seg[i].kind == QI21_SEG_TEXT) {
            if (seg[i].n_text <= 0) return QI21_ERR_METADATA;
            P += seg[i].n_text;
            slots += seg[i].n_text;
        } else if (seg[i].kind == QI21_SEG_IMAGE) {
            if (seg[i].h <= 0 || seg[i].w <= 0) return QI21_ERR_METADATA;
            const int64_t cells = (int64_t)seg[i].h * seg[i].w;
            if (cells % QI21_IMG_TOKENS_PER_SLOT) return QI21_ERR_METADATA;
            P += cells;
            slots += cells / QI21_IMG_TOKENS_PER_SLOT;
            cells_total += cells;
        } else {
            return QI21_ERR_INVALID_ARG;
        }
    }
    if (P > INT32_MAX / 4) return QI21_ERR_SHAPE;
    if (P_out) *P_out = (int32_t)P;
    if (n_slots_out) *n_slots_out = (int32_t)slots;
    if (n_img_out) *n_img_out = (int32_t)cells_total;
    if (!slot_of && !img_row) return QI21_OK;
    if (capacity < P) return QI21_ERR_METADATA;
    int64_t pos = 0, slot = 0, row = 0;
    for (int i = 0; i < n_seg - 1; ++i) {
        if (seg[i].kind == QI21_SEG_TEXT) {
            for (int t = 0; t < seg[i].n_text; ++t, ++pos, ++slot) {
                if (slot_of) slot_of[pos] = (int32_t)slot;
                if (img_row) img_row[pos] = -1;
            }
        } else {
            const int64_t cells = (int64_t)seg[i].h * seg[i].w;
            for (int64_t c = 0; c < cells; ++c, ++pos, ++row) {
                if (slot_of) slot_of[pos] = (int32_t)(slot + c / QI21_IMG_TOKENS_PER_SLOT);
                if (img_row) img_row[pos] = (int32_t)row;
            }
            slot += cells / QI21_IMG_TOKENS_PER_SLOT;
        }
    }
    return QI21_OK;
}

extern "C" const char *qi21_status_string(qi21_status s) {
    switch (s) {
        case QI21_OK: return "ok";
        case QI21_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad enum)";
        case QI21_ERR_SHAPE: return "inconsistent shape";
        case QI21_ERR_METADATA: return "invalid segment metadata";
        case QI21_ERR_CACHE_STATE: return "kv cache not extracted or shape mismatch";
        case QI21_ERR_UNSUPPORTED: return "shape not supported by the selected kernels";
        case QI21_ERR_CUDA: return "CUDA error";
        case QI21_ERR_DEVICE_TIMEOUT: return "device wait timed out";
        case QI21_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case QI21_ERR_DEVICE_CHECK: return "a kernel's device-side layout check failed";
        default: return "unknown status";
    }
}

extern "C" const char *qi21_version(void) { return "qi21 0.1 sm_100a"; }

static bool g_tc_enabled = true;
bool qi21::tc_enabled() { return g_tc_enabled; }
extern "C" void qi21_set_tensor_cores(int32_t enable) { g_tc_enabled = enable != 0; }

bool qi21_config_ok(const qi21_config *c) {
    return c && c->d_model > 0 && c->n_heads > 0 && c->head_dim > 0 && c->n_layers > 0 &&
           c->mlp_hidden > 0 && c->latent_ch > 0 && c->time_dim > 0 && c->time_dim % 2 == 0 &&
           c->d_model == c->n_heads * c->head_dim && c->head_dim % 2 == 0 &&
           (c->dtype == QI21_DTYPE_F32 || c->dtype == QI21_DTYPE_BF16) &&
           (c->use_shift == 0 || c->use_shift == 1);
}

extern "C" size_t qi21_kv_cache_bytes(const qi21_config *c, int32_t B, int32_t P, int32_t N) {
    if (!qi21_config_ok(c) || B <= 0 || P < 0 || N <= 0) return 0;
    return qi21::dtype_bytes(c->dtype) * (size_t)c->n_layers * 2 * (size_t)B * ((size_t)P + N) *
           (size_t)c->d_model;
}

static int64_t padded_prefix(int32_t P) {
    return ((int64_t)P + QI21_ATTN_KEY_TILE - 1) / QI21_ATTN_KEY_TILE * QI21_ATTN_KEY_TILE;
}

extern "C" size_t qi21_kv_cache_bytes_shared(const qi21_config *c, int32_t B, int32_t P, int32_t N) {
    if (!qi21_config_ok(c) || B <= 0 || P <= 0 || N <= 0) return 0;
    return qi21::dtype_bytes(c->dtype) * (size_t)c->n_layers * 2 * (size_t)(padded_prefix(P) + (int64_t)B * N) *
           (size_t)c->d_model;
}

extern "C" size_t qi21_packed_weights_bytes(const qi21_config *c) {
    if (!qi21_config_ok(c)) return 0;
    return qi21::packed_layout(*c).total;
}

extern "C" size_t qi21_workspace_bytes(const qi21_config *c, int32_t B, int32_t P, int32_t N) {
    if (!qi21_config_ok(c) || B <= 0 || P < 0 || N <= 0) return 0;
    return qi21::ws_layout(*c, B, P, N).total;
}

extern "C" qi21_status qi21_kv_cache_init(qi21_kv_cache *cache, void *base, const qi21_config *c,
                                          int32_t B, int32_t P, int32_t N) {
    if (!cache || !base || !qi21_config_ok(c)) return QI21_ERR_INVALID_ARG;
    if (((uintptr_t)base) & 15) return QI21_ERR_INVALID_ARG;
    if (B <= 0 || P <= 0 || N <= 0) return QI21_ERR_SHAPE;
    cache->base = base;
    cache->batch = B;
    cache->n_prefix = P;
    cache->n_target = N;
    cache->n_layers = c->n_layers;
    cache->d_model = c->d_model;
    cache->dtype = c->dtype;
    cache->state = QI21_CACHE_EMPTY;
    cache->shared_prefix = 0;
    return QI21_OK;
}

extern "C" qi21_status qi21_kv_cache_init_shared(qi21_kv_cache *cache, void *base, const qi21_config *c,
                                                 int32_t B, int32_t P, int32_t N) {
    qi21_status s = qi21_kv_cache_init(cache, base, c, B, P, N);
    if (s == QI21_OK) cache->shared_prefix = 1;
    return s;
}
