// C-ABI entry points: argument validation, workspace carve-up and the per-layer
// launch sequence of the prefix extract, the cached step and the full
// recomputation (see include/qi21.h for the contract of each call).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>
#include <type_traits>

#include "qi21.h"
#include "qi21_internal.h"
#include "qi21_simt.cuh"
#include "qi21_gemm_tc.cuh"
#include "qi21_attn_tc.cuh"
#include "qi21_final_tc.cuh"

bool qi21_config_ok(const qi21_config *c);

namespace qi21 {

// ------------------------------------------------------------------ per-kernel timing
struct ProfRec {
    const char *name;
    cudaEvent_t a, b;
};
static std::mutex g_prof_mu;
static bool g_prof_on = false;
static std::vector<cudaEvent_t> g_event_pool;
static size_t g_event_next = 0;
static std::vector<ProfRec> g_prof_recs;
static int g_last_launches = 0;

static cudaEvent_t prof_event() {
    if (g_event_next == g_event_pool.size()) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
        g_event_pool.push_back(e);
    }
    return g_event_pool[g_event_next++];
}

struct Launcher {
    cudaStream_t st;
    int count = 0;
    qi21_status status = QI21_OK;
    explicit Launcher(cudaStream_t s) : st(s) {}
    template <typename F>
    void run(const char *name, F &&f) {
        if (status != QI21_OK) return;
        cudaEvent_t a = nullptr, b = nullptr;
        if (g_prof_on) {
            std::lock_guard<std::mutex> lk(g_prof_mu);
            a = prof_event();
            b = prof_event();
        }
        if (a) cudaEventRecord(a, st);
        nvtxRangePushA(name);     // one NVTX range per launch, named as in qi21_profile_read
        f();
        nvtxRangePop();
        ++count;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) {
            fprintf(stderr, "qi21: launch of %s failed: %s\n", name, cudaGetErrorString(e));
            status = QI21_ERR_CUDA;
            return;
        }
#ifdef QI21_DEBUG
        // debug build: wait for every kernel and name the one that failed (not
        // while the stream is being captured, where synchronising is illegal)
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(st, &cap) == cudaSuccess && cap == cudaStreamCaptureStatusNone) {
            e = cudaStreamSynchronize(st);
            if (e != cudaSuccess) {
                fprintf(stderr, "qi21: kernel %s failed: %s\n", name, cudaGetErrorString(e));
                status = QI21_ERR_CUDA;
                return;
            }
        }
#endif
        if (b) {
            cudaEventRecord(b, st);
            std::lock_guard<std::mutex> lk(g_prof_mu);
            g_prof_recs.push_back({name, a, b});
        }
    }
    ~Launcher() { g_last_launches = count; }
};

static inline bool al16(const void *p) { return p && ((uintptr_t)p & 15) == 0; }

#ifndef QI21_PDL
#define QI21_PDL 1
#endif

// Launch a kernel that calls pdl_wait() before its first global-memory access
// with programmatic stream serialisation, so that it may be scheduled (and run
// its prologue) while the previous kernel in the stream finishes. Optional
// extra attribute (the GEMM's cluster shape). Same-GPU A/B, steps without
// per-launch timing events: single-block workload 1.845 -> 1.808 ms per step,
// mid (d 1024, 8 blocks, 2048 rows) 1.152 -> 1.014 ms. A timing event recorded
// between two kernels (qi21_profile_enable) keeps them from overlapping.
template <typename... KArgs, typename... Args>
static cudaError_t launch_dep(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              const cudaLaunchAttribute *extra, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    int n = 0;
    if (QI21_PDL) {
        at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (extra) at[n++] = *extra;
    cfg.attrs = at;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The dynamic shared-memory opt-in above 48 KB is a per-device attribute of a
// kernel: each call site keeps one flag per device and sets it on the current
// device the first time (the call is not a stream operation, so this also
// works while a stream is being captured).
constexpr int kMaxDevices = 64;
using DeviceFlags = std::atomic<int>[kMaxDevices];

template <typename K>
static void smem_opt_in(K *kernel, int bytes, DeviceFlags &done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return;   // the launch reports the error
    if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire) >= bytes) return;
    if (cudaFuncSetAttribute((const void *)kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
            cudaSuccess &&
        dev >= 0 && dev < kMaxDevices)
        done[dev].store(bytes, std::memory_order_release);
}

static inline int grid_for(int64_t n, int threads, int cap = 148 * 16) {
    int64_t g = (n + threads - 1) / threads;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return (int)g;
}


// ------------------------------------------------------------------ tensor-core family (BF16 mode)
static bool tc_supported(const qi21_config &c) {
    return c.dtype == QI21_DTYPE_BF16 && c.d_model % TC_BN == 0 && c.mlp_hidden % 128 == 0 &&
           (c.head_dim == 64 || c.head_dim == 128) && c.d_model >= TC_BN;
}

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

static bool get_encode() {
    if (g_encode) return true;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return false;
    g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    return true;
}

// 3-D bf16 tensor map over [depth][rows][inner] with a box of 64 x box_rows x 1,
// 128-byte swizzle, zero fill outside the tensor.
static bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t depth,
                     uint32_t box_rows) {
    if (!get_encode()) return false;
    cuuint64_t dims[3] = {inner, rows, depth};
    cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static int num_sms() {
    static std::atomic<int> count[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && count[dev].load() > 0) return count[dev].load();
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (dev >= 0 && dev < kMaxDevices) count[dev].store(n);
    return n;
}

#ifndef QI21_GEMM_PAIRS
#define QI21_GEMM_PAIRS 1
#endif

// Row blocks per band of the GEMM tile order (0: one band). Up to 4096 rows one
// band keeps the whole activation in L2 and reads each weight tile once per wave;
// beyond that, bands of 2048 rows keep each wave's A rows in L2 (same-GPU A/B at
// 16384 rows: gate/up -15 %, down -11 %, QKV -7 %; at 4096 rows banding cost
// gate/up 3 %).
static int gemm_group_m(int rows, int tile_rows) { return rows > 4096 ? 2048 / tile_rows : 0; }

// The persistent tcgen05 GEMM over p.R rows. Work units are 256 x 256 tiles of a
// CTA pair (cluster of 2) from 4096 rows on, else 128 x 256 tiles of single CTAs;
// one worker (pair or CTA) per pair of SMs or SM. Same-GPU A/B at 4096 rows
// (d 4096): pairs took QKV 300 -> 252 us, gate/up 554 -> 497, down 311 -> 275,
// out-proj 111 -> 97; at 2048 rows (d 1024) they were 3-11 % slower (half as
// many work units), and for img_in (K = 64) 27 vs 21 us. stream_k (residual
// epilogue): the tiles of the last, partial wave are shared stream-K style so
// that every worker gets the same number of K blocks and only about one extra
// partial tile per worker is reduce-added into h.
template <int EPI>
static void launch_gemm_tc(Launcher &L, const char *name, const CUtensorMap &a, const CUtensorMap &b0,
                           const CUtensorMap &b1, const CUtensorMap &b2, GemmParams p, bool stream_k = false) {
    const bool pair = QI21_GEMM_PAIRS && EPI != EPI_STORE && p.R >= 4096;
    const int tile_rows = pair ? 2 * TC_BM : TC_BM;
    p.m_blocks = (p.R + tile_rows - 1) / tile_rows;
    p.group_m = gemm_group_m(p.R, tile_rows);
    const int workers = pair ? num_sms() / 2 : num_sms();
    const int tiles = p.m_blocks * p.n_blocks;
    p.sk_tiles = (stream_k && p.ksplit == 1) ? tiles % workers : 0;
    const int units = tiles * p.ksplit;
    const int active = (units < workers && p.sk_tiles == 0) ? units : workers;
    if (pair) {
        constexpr size_t smem = tc_smem_bytes<EPI, true>();
        static DeviceFlags attr;
        smem_opt_in(k_gemm_tc<EPI, true>, (int)smem, attr);
        cudaLaunchAttribute cl;
        cl.id = cudaLaunchAttributeClusterDimension;
        cl.val.clusterDim.x = 2;
        cl.val.clusterDim.y = 1;
        cl.val.clusterDim.z = 1;
        L.run(name, [&] { launch_dep(k_gemm_tc<EPI, true>, dim3(2 * active), dim3(TC_THREADS), smem, L.st, &cl, a, b0, b1, b2, p); });
    } else {
        constexpr size_t smem = tc_smem_bytes<EPI, false>();
        static DeviceFlags attr;
        smem_opt_in(k_gemm_tc<EPI, false>, (int)smem, attr);
        L.run(name, [&] { launch_dep(k_gemm_tc<EPI, false>, dim3(active), dim3(TC_THREADS), smem, L.st, nullptr, a, b0, b1, b2, p); });
    }
}

// 2-D fp32 tensor map [rows][inner] with a 32 x 32 box and 128-byte swizzle:
// the target of the residual epilogue's TMA reduce-add.
static bool make_map_f32(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows) {
    if (!get_encode()) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 4};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D tensor map [rows][inner] of bf16 or fp32 with a box of box_inner x
// box_rows elements, 128-byte swizzle, zero fill outside the tensor.
static bool make_map2d(CUtensorMap *m, const void *base, bool f32, uint64_t inner, uint64_t rows,
                       uint32_t box_inner, uint32_t box_rows) {
    if (!get_encode()) return false;
    const uint64_t eb = f32 ? 4 : 2;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * eb};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                          const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4-D bf16 tensor map [w][z][rows][inner] (strides in elements), box 64 x 128 x 1 x 1.
static bool make_map4(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t zn, uint64_t wn,
                      uint64_t row_stride, uint64_t z_stride, uint64_t w_stride) {
    if (!get_encode()) return false;
    cuuint64_t dims[4] = {inner, rows, zn, wn};
    cuuint64_t strides[3] = {row_stride * 2, z_stride * 2, w_stride * 2};
    cuuint32_t box[4] = {64, 128, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int DH>
static void launch_attn_tc(Launcher &L, const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                           const AttnParams &p, int B) {
    using Cf = AttnCfg<DH>;
    static DeviceFlags attr;
    smem_opt_in(k_attn_tc<DH>, (int)Cf::SMEM, attr);
    dim3 grid((p.Mq + Cf::BQ - 1) / Cf::BQ, p.H, B);
    L.run("attn", [&] { launch_dep(k_attn_tc<DH>, grid, dim3(Cf::THREADS), Cf::SMEM, L.st, nullptr, q, k, v, p); });
}

struct TcMaps {
    CUtensorMap xn, o, hid, wq, wk, wv, wo, wg, wu, wd, q4, k4, v4, h32;
};

static bool build_tc_maps(TcMaps &t, const qi21_config &c, const qi21_weights &w, const void *xn, const void *o,
                          const void *hid, int R) {
    const uint64_t d = c.d_model, F = c.mlp_hidden, L = c.n_layers;
    bool ok = true;
    ok &= make_map(&t.xn, xn, d, R, 1, 128);
    ok &= make_map(&t.o, o, d, R, 1, 128);
    ok &= make_map(&t.hid, hid, F, R, 1, 128);
    ok &= make_map(&t.wq, w.w_q, d, d, L, 128);
    ok &= make_map(&t.wk, w.w_k, d, d, L, 128);
    ok &= make_map(&t.wv, w.w_v, d, d, L, 128);
    ok &= make_map(&t.wo, w.w_o, d, d, L, 128);
    ok &= make_map(&t.wg, w.w_gate, d, F, L, 128);
    ok &= make_map(&t.wu, w.w_up, d, F, L, 128);
    ok &= make_map(&t.wd, w.w_down, F, d, L, 128);
    return ok;
}

// ------------------------------------------------------------------ block stack
struct StackArgs {
    int B, M, split;          // items, rows per item in this call, rows < split read the prefix row
    int P, N;                 // prefix / target sizes of the sequence
    float *h;                 // fp32 [B*M][d]
    void *xn, *q, *o, *hid;   // T buffers
    float *gemm;              // fp32 scratch (F32 mode)
    float *gates;             // [4][d]
    uint32_t *err;
    const float *mod_lo, *mod_hi;
    const float *cos_sin;     // [M][Dh/2][2]
    char *kv_k0, *kv_v0;      // K / V base of layer 0 (bytes)
    int64_t kv_layer_stride;  // elements between layers (0: one buffer reused)
    int64_t kv_bstride;       // elements between items
    int row_off;              // K/V row of token 0 of this call
    int kv_len;               // keys visible (rows of the K/V buffer per item)
    const int *kv_limit;      // [M] or null
    bool kv_only_last;        // extract: the last layer only needs K/V
    // shared-prefix cache: the prefix rows [0, P) are one copy read by every item;
    // item b's target rows start at Pp + b*N (kv_bstride = N*d, row_off = Pp)
    bool shared;
    int shared_P, shared_Pp;
};

template <typename T>
static void launch_modln(Launcher &L, const qi21_config &c, const float *h, T *out, int rows, int M, int split,
                         const float *sc_lo, const float *sc_hi, const float *sh_lo, const float *sh_hi) {
    const int d = c.d_model;
    if (d % 4 == 0 && d <= 4 * 256 * 8) {
        const int vpt = (d / 4 + 255) / 256;
        // one row per block: measured alone at 4096 x 4096 it moves 4.9 TB/s (a
        // plain fp32 -> bf16 copy of the same bytes: 5.6 TB/s); 128-thread blocks
        // are as fast, 512 or 1024 threads, a warp per row, a one-pass
        // (shifted) variance and a row-looping grid with the next row prefetched
        // were slower
        L.run("modln", [&] {
#define QI21_LN(V)                                                                                           \
    launch_dep(k_modln_vec<T, V>, dim3(rows), dim3(256), 0, L.st, nullptr, h, out, d, M, split, sc_lo, sc_hi, sh_lo, \
               sh_hi, c.ln_eps)
            if (vpt <= 1) QI21_LN(1);
            else if (vpt <= 2) QI21_LN(2);
            else if (vpt <= 4) QI21_LN(4);
            else QI21_LN(8);
#undef QI21_LN
        });
    } else {
        L.run("modln", [&] {
            k_modln_any<T><<<rows, 256, 0, L.st>>>(h, out, d, M, split, sc_lo, sc_hi, sh_lo, sh_hi, c.ln_eps);
        });
    }
}

template <typename T>
static void launch_gemm_simt(Launcher &L, const T *A, int lda, const T *W, int ldw, float *Cm, int ldc, int M,
                             int N, int K) {
    dim3 grid((N + 63) / 64, (M + 63) / 64);
    L.run("gemm_simt", [&] { k_gemm_simt<T><<<grid, 256, 0, L.st>>>(A, lda, W, ldw, Cm, ldc, M, N, K); });
}

template <typename T>
static void run_stack(Launcher &L, const qi21_config &c, const qi21_weights &w, const StackArgs &a) {
    const int d = c.d_model, F = c.mlp_hidden, H = c.n_heads, Dh = c.head_dim;
    const int R = a.B * a.M;
    const int ch_scale1 = c.use_shift ? 1 : 0, ch_scale2 = c.use_shift ? 4 : 2;
    const float *sc1_lo = a.mod_lo + (size_t)ch_scale1 * d, *sc1_hi = a.mod_hi + (size_t)ch_scale1 * d;
    const float *sc2_lo = a.mod_lo + (size_t)ch_scale2 * d, *sc2_hi = a.mod_hi + (size_t)ch_scale2 * d;
    const float *sh1_lo = c.use_shift ? a.mod_lo : nullptr, *sh1_hi = c.use_shift ? a.mod_hi : nullptr;
    const float *sh2_lo = c.use_shift ? a.mod_lo + 3 * (size_t)d : nullptr;
    const float *sh2_hi = c.use_shift ? a.mod_hi + 3 * (size_t)d : nullptr;
    const float *tg1_lo = a.gates, *tg1_hi = a.gates + d, *tg2_lo = a.gates + 2 * d, *tg2_hi = a.gates + 3 * d;
    T *xn = (T *)a.xn, *q = (T *)a.q, *o = (T *)a.o, *hid = (T *)a.hid;
    const bool tc = std::is_same<T, bf16>::value && tc_enabled() && tc_supported(c);
    const float scale = 1.0f / sqrtf((float)Dh);

    TcMaps maps;
    GemmParams gp{};
    if (tc) {
        if (!build_tc_maps(maps, c, w, a.xn, a.o, a.hid, R)) {
            L.status = QI21_ERR_CUDA;
            return;
        }
        // attention operands: q [R][d]; K and V [layer][item][kv_len rows][d]
        const uint64_t nl = a.kv_layer_stride ? (uint64_t)c.n_layers : 1;
        const uint64_t lstride = a.kv_layer_stride ? (uint64_t)a.kv_layer_stride : (uint64_t)a.kv_bstride * a.B;
        bool ok = make_map4(&maps.q4, a.q, d, R, 1, 1, d, (uint64_t)R * d, (uint64_t)R * d);
        if (a.shared) {   // one item of Pp + B*N rows per layer
            const uint64_t rows_all = (uint64_t)a.shared_Pp + (uint64_t)a.B * a.N;
            ok &= make_map4(&maps.k4, a.kv_k0, d, rows_all, 1, nl, d, rows_all * d, lstride);
            ok &= make_map4(&maps.v4, a.kv_v0, d, rows_all, 1, nl, d, rows_all * d, lstride);
        } else {
            ok &= make_map4(&maps.k4, a.kv_k0, d, a.kv_len, a.B, nl, d, a.kv_bstride, lstride);
            ok &= make_map4(&maps.v4, a.kv_v0, d, a.kv_len, a.B, nl, d, a.kv_bstride, lstride);
        }
        ok &= make_map_f32(&maps.h32, a.h, d, R);
        if (!ok) {
            L.status = QI21_ERR_CUDA;
            return;
        }
        gp.R = R;
        gp.ksplit = 1;
        gp.M = a.M;
        gp.split = a.split;
        gp.h = a.h;
        gp.ldh = d;
        gp.F = F;
        gp.hid = (bf16 *)a.hid;
        gp.d = d;
        gp.Dh = Dh;
        gp.qk_eps = c.qk_eps;
        gp.cos_sin = a.cos_sin;
        gp.q_out = (bf16 *)a.q;
        gp.kv_bstride = a.kv_bstride;
        gp.row_off = a.row_off;
        gp.err = a.err;
    }

    L.run("prep_gates", [&] {
        launch_dep(k_prep_gates, dim3(grid_for(d, 256)), dim3(256), 0, L.st, nullptr, a.mod_lo, a.mod_hi, d, c.use_shift,
                   a.gates);
    });
    for (int l = 0; l < c.n_layers; ++l) {
        const T *Wq = (const T *)w.w_q + (size_t)l * d * d, *Wk = (const T *)w.w_k + (size_t)l * d * d;
        const T *Wv = (const T *)w.w_v + (size_t)l * d * d, *Wo = (const T *)w.w_o + (size_t)l * d * d;
        const T *Wg = (const T *)w.w_gate + (size_t)l * F * d, *Wu = (const T *)w.w_up + (size_t)l * F * d;
        const T *Wd = (const T *)w.w_down + (size_t)l * d * F;
        const float *qn = w.q_norm + (size_t)l * Dh, *kn = w.k_norm + (size_t)l * Dh;
        T *kdst = (T *)(a.kv_k0) + (size_t)l * a.kv_layer_stride;
        T *vdst = (T *)(a.kv_v0) + (size_t)l * a.kv_layer_stride;
        gp.layer = l;

        launch_modln<T>(L, c, a.h, xn, R, a.M, a.split, sc1_lo, sc1_hi, sh1_lo, sh1_hi);
        if (tc) {
            GemmParams g = gp;
            g.K = d;
            g.n_blocks = 3 * d / TC_BN;
            g.qn = qn;
            g.kn = kn;
            g.k_base = (bf16 *)kdst;
            g.v_base = (bf16 *)vdst;
            launch_gemm_tc<EPI_QKV>(L, "gemm_qkv", maps.xn, maps.wq, maps.wk, maps.wv, g);
        } else {
            launch_gemm_simt<T>(L, xn, d, Wq, d, a.gemm, 3 * d, R, d, d);
            launch_gemm_simt<T>(L, xn, d, Wk, d, a.gemm + d, 3 * d, R, d, d);
            launch_gemm_simt<T>(L, xn, d, Wv, d, a.gemm + 2 * d, 3 * d, R, d, d);
            L.run("qkv_post", [&] {
                k_qkv_post<T><<<(R * H + 3) / 4, 128, 0, L.st>>>(a.gemm, R, a.M, d, H, Dh, qn, kn, c.qk_eps,
                                                               a.cos_sin, q, kdst, vdst, a.kv_bstride, a.row_off);
            });
        }
        if (a.kv_only_last && l == c.n_layers - 1) break;

        if (tc) {
            AttnParams ap{};
            ap.Mq = a.M;
            ap.kv_len = a.kv_len;
            ap.H = H;
            ap.d = d;
            ap.kv_limit = a.kv_limit;
            ap.out = (bf16 *)a.o;
            ap.scale_log2 = 1.4426950408889634f / sqrtf((float)Dh);
            ap.layer = a.kv_layer_stride ? l : 0;
            ap.err = a.err;
            if (a.shared) {
                ap.shared_tiles = a.shared_Pp / QI21_ATTN_KEY_TILE;
                ap.prefix_len = a.shared_P;
                ap.tgt_len = a.N;
                ap.tgt_row0 = a.shared_Pp;
            }
            if (Dh == 128)
                launch_attn_tc<128>(L, maps.q4, maps.k4, maps.v4, ap, a.B);
            else
                launch_attn_tc<64>(L, maps.q4, maps.k4, maps.v4, ap, a.B);
        } else {
            const size_t smem = sizeof(float) * (3 * 32 * (Dh + 1) + 32 * 33);
            static DeviceFlags attr;
            smem_opt_in(k_attn_simt<T>, 64 * 1024, attr);
            dim3 grid((a.M + 31) / 32, H, a.B);
            L.run("attn_simt", [&] {
                if (a.shared)
                    k_attn_simt<T><<<grid, 128, smem, L.st>>>(q, (int64_t)a.M * d, a.M, d, kdst, vdst, 0, d, a.kv_len,
                                                             a.kv_limit, o, Dh, scale, a.shared_P,
                                                             (int64_t)a.shared_Pp * d, a.kv_bstride);
                else
                    k_attn_simt<T><<<grid, 128, smem, L.st>>>(q, (int64_t)a.M * d, a.M, d, kdst, vdst, a.kv_bstride, d,
                                                             a.kv_len, a.kv_limit, o, Dh, scale, a.kv_len, 0, 0);
            });
        }
        if (tc) {
            GemmParams g = gp;
            g.K = d;
            g.n_blocks = d / TC_BN;
            g.g_lo = tg1_lo;
            g.g_hi = tg1_hi;
            launch_gemm_tc<EPI_RESIDUAL>(L, "gemm_o", maps.o, maps.wo, maps.wo, maps.h32, g, true);
        } else {
            launch_gemm_simt<T>(L, o, d, Wo, d, a.gemm, d, R, d, d);
            L.run("gated_residual", [&] {
                k_gated_residual<<<grid_for((int64_t)R * d, 256), 256, 0, L.st>>>(a.h, a.gemm, d, R, d, a.M, a.split,
                                                                                   tg1_lo, tg1_hi);
            });
        }
        launch_modln<T>(L, c, a.h, xn, R, a.M, a.split, sc2_lo, sc2_hi, sh2_lo, sh2_hi);
        if (tc) {
            GemmParams g = gp;
            g.K = d;
            g.n_blocks = F / 128;
            launch_gemm_tc<EPI_SWIGLU>(L, "gemm_gateup", maps.xn, maps.wg, maps.wu, maps.wu, g);
            GemmParams g2 = gp;
            g2.K = F;
            g2.n_blocks = d / TC_BN;
            g2.g_lo = tg2_lo;
            g2.g_hi = tg2_hi;
            launch_gemm_tc<EPI_RESIDUAL>(L, "gemm_down", maps.hid, maps.wd, maps.wd, maps.h32, g2, true);
        } else {
            launch_gemm_simt<T>(L, xn, d, Wg, d, a.gemm, 2 * F, R, F, d);
            launch_gemm_simt<T>(L, xn, d, Wu, d, a.gemm + F, 2 * F, R, F, d);
            L.run("swiglu", [&] {
                k_swiglu<T><<<grid_for((int64_t)R * F, 256), 256, 0, L.st>>>(a.gemm, hid, R, F);
            });
            launch_gemm_simt<T>(L, hid, F, Wd, F, a.gemm, d, R, d, F);
            L.run("gated_residual", [&] {
                k_gated_residual<<<grid_for((int64_t)R * d, 256), 256, 0, L.st>>>(a.h, a.gemm, d, R, d, a.M, a.split,
                                                                                   tg2_lo, tg2_hi);
            });
        }
    }
}

// Tensor-core forms of img_in and of the final AdaLN + proj_out for the BF16
// cached step (target rows contiguous in h): 64 latent channels, d a multiple
// of 256 (every shape tc_supported() accepts).
static bool tc_head_supported(const qi21_config &c) {
    return c.dtype == QI21_DTYPE_BF16 && tc_enabled() && tc_supported(c) && c.latent_ch == 64;
}

static __global__ void k_to_bf16(const float *__restrict__ x, bf16 *__restrict__ y, int64_t n4) {
    pdl_launch_dependents();
    pdl_wait();
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 f = reinterpret_cast<const float4 *>(x)[i];
        reinterpret_cast<uint2 *>(y)[i] = make_uint2(pack_bf16x2(f.x, f.y), pack_bf16x2(f.z, f.w));
    }
}

// h[r][:] = x[r][:] W_img_in^T for rows [0, rows): the latent rounded to bf16,
// then the tcgen05 GEMM with K = 64 whose epilogue stores fp32 rows of h.
static void launch_img_in_tc(Launcher &L, const qi21_config &c, const float *x, const void *w_img_in, float *h,
                             int rows, bf16 *xin, uint32_t *err) {
    const int d = c.d_model, C = c.latent_ch;
    const int64_t n4 = (int64_t)rows * C / 4;
    L.run("img_in_cvt", [&] { launch_dep(k_to_bf16, dim3(grid_for(n4, 256)), dim3(256), 0, L.st, nullptr, x, xin, n4); });
    CUtensorMap ma, mb, mh;
    if (!make_map(&ma, xin, C, rows, 1, 128) || !make_map(&mb, w_img_in, C, d, 1, 128) ||
        !make_map_f32(&mh, h, d, rows)) {
        L.status = QI21_ERR_CUDA;
        return;
    }
    GemmParams g{};
    g.R = rows;
    g.K = C;
    g.n_blocks = d / TC_BN;
    g.ksplit = 1;
    g.M = rows;
    g.split = 0;
    g.layer = 0;
    g.err = err;
    launch_gemm_tc<EPI_STORE>(L, "img_in", ma, mb, mb, mh, g);
}

// v[r][:] = (LN(h[r]) (1 + scale_final)) W_out^T for rows [0, rows) of h.
static void launch_final_tc(Launcher &L, const qi21_config &c, const float *h, int rows, const float *sf,
                            const void *w_out, float *v, char *wsb, const WsLayout &lay, uint32_t *err) {
    const int d = c.d_model;
    bf16 *wp = (bf16 *)(wsb + lay.fwp);
    float *u = (float *)(wsb + lay.fu), *part = (float *)(wsb + lay.fpart);
    L.run("final_prep", [&] {
        launch_dep(k_final_prep, dim3(FT_C), dim3(256), 0, L.st, nullptr, (const bf16 *)w_out, sf, d, wp, u);
    });
    CUtensorMap mh, mw;
    if (!make_map2d(&mh, h, true, d, rows, 32, FT_BM) || !make_map2d(&mw, wp, false, d, FT_C, FT_BK, FT_C)) {
        L.status = QI21_ERR_CUDA;
        return;
    }
    const int mb = (rows + FT_BM - 1) / FT_BM, kblocks = d / FT_BK;
    int ks = num_sms() / mb;
    if (ks > FINAL_MAX_KSPLIT) ks = FINAL_MAX_KSPLIT;
    if (ks > kblocks) ks = kblocks;
    if (ks < 1) ks = 1;
    FinalParams fp{rows, d, kblocks, ks, part, err};
    static DeviceFlags attr;
    smem_opt_in(k_final_tc, (int)FT_SMEM, attr);
    L.run("final", [&] { launch_dep(k_final_tc, dim3(mb, ks), dim3(FT_THREADS), FT_SMEM, L.st, nullptr, mh, mw, fp); });
    L.run("final_reduce", [&] {
        launch_dep(k_final_reduce, dim3((int)(((int64_t)rows * 16 + 255) / 256)), dim3(256), 0, L.st, nullptr, part,
                   ks, rows, d, u, c.ln_eps, v);
    });
}

template <typename T>
static void launch_img_in(Launcher &L, const qi21_config &c, const float *x, const void *w_img_in, float *h, int B,
                          int N, int M_out, int off) {
    const int rows = B * N, C = c.latent_ch, d = c.d_model;
    dim3 grid((rows + 15) / 16, (d + 255) / 256);
    if (C == 64) {
        L.run("img_in", [&] {
            k_img_in64<T><<<grid, 256, 0, L.st>>>(x, (const T *)w_img_in, h, rows, d, N, M_out, off);
        });
        return;
    }
    L.run("img_in", [&] {
        k_img_in<T><<<grid, 256, sizeof(float) * 16 * C, L.st>>>(x, (const T *)w_img_in, h, rows, C, d, N, M_out, off);
    });
}

template <typename T>
static void launch_final(Launcher &L, const qi21_config &c, const float *h, int M, int off, int B, int N,
                         const float *sf, const void *w_out, float *v) {
    const int rows = B * N, d = c.d_model;
    if (c.latent_ch == 64 && d % 128 == 0) {
        L.run("final", [&] {
            k_final64<T><<<(rows + 15) / 16, 256, 0, L.st>>>(h, M, off, N, d, sf, (const T *)w_out, c.ln_eps, v, rows);
        });
        return;
    }
    const size_t smem = sizeof(float) * 4 * d;
    static DeviceFlags attr;
    if (smem > 48 * 1024) smem_opt_in(k_final<T>, 200 * 1024, attr);
    L.run("final", [&] {
        k_final<T><<<(rows + 3) / 4, 256, smem, L.st>>>(h, M, off, N, d, sf, (const T *)w_out, c.latent_ch, c.ln_eps,
                                                       v, rows);
    });
}

// ------------------------------------------------------------------ validation helpers
static qi21_status check_weights(const qi21_weights *w, bool need_time) {
    if (!w) return QI21_ERR_INVALID_ARG;
    const void *ps[] = {w->w_img_in, w->w_out, w->w_q, w->w_k, w->w_v, w->w_o, w->w_gate, w->w_up, w->w_down,
                        w->q_norm, w->k_norm};
    for (const void *p : ps)
        if (!al16(p)) return QI21_ERR_INVALID_ARG;
    if (need_time) {
        const void *ts[] = {w->w_t1, w->w_t2, w->w_mod, w->w_fin};
        for (const void *p : ts)
            if (!al16(p)) return QI21_ERR_INVALID_ARG;
    }
    return QI21_OK;
}

static qi21_status check_shapes(const qi21_config *c) {
    if (!c) return QI21_ERR_INVALID_ARG;
    if (!qi21_config_ok(c)) return QI21_ERR_SHAPE;
    // 16-byte row alignment of every activation row and cos/sin row
    if (c->d_model % 8 || c->mlp_hidden % 8 || c->latent_ch % 4 || c->head_dim % 4) return QI21_ERR_UNSUPPORTED;
    if (c->head_dim > 128 || c->time_dim > 512) return QI21_ERR_UNSUPPORTED;
    if (c->dtype == QI21_DTYPE_BF16 && tc_enabled() && !tc_supported(*c)) return QI21_ERR_UNSUPPORTED;
    return QI21_OK;
}

qi21_status check_config_shapes(const qi21_config *c) { return check_shapes(c); }

static qi21_status finish(Launcher &L) { return L.status; }

// Shared-prefix cache: prefix rows padded to the attention key tile, then batch*N target rows.
static int64_t padded_prefix_rows(int P) {
    return ((int64_t)P + QI21_ATTN_KEY_TILE - 1) / QI21_ATTN_KEY_TILE * QI21_ATTN_KEY_TILE;
}
static int64_t shared_rows(int P, int N, int B) { return padded_prefix_rows(P) + (int64_t)B * N; }

}  // namespace qi21

using namespace qi21;

// ------------------------------------------------------------------ entry points
// Modulation rows for the timestep embedding given either on the host
// (emb != null) or as a device table of sigmas (sigmas[step] * t_per_sigma).
static qi21_status modulation_impl(const qi21_config *c, const qi21_weights *w, const TembArg *emb,
                                   const double *sigmas, int step, double t_per_sigma, float *mod_row,
                                   float *scale_final, void *ws, size_t ws_bytes, void *stream) {
    qi21_status s = check_shapes(c);
    if (s) return s;
    if (!w || !al16(w->w_t1) || !al16(w->w_t2) || !al16(w->w_mod) || !al16(w->w_fin)) return QI21_ERR_INVALID_ARG;
    if (!al16(mod_row) || !al16(scale_final) || !al16(ws)) return QI21_ERR_INVALID_ARG;
    const WsLayout lay = ws_layout(*c, 1, 0, 1);
    if (ws_bytes < lay.modtmp + align256(sizeof(float) * 2 * c->d_model)) return QI21_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    const int d = c->d_model, K0 = c->time_dim, nch = c->use_shift ? 6 : 4;
    float *a1 = (float *)((char *)ws + lay.modtmp), *e = a1 + d;
    const size_t xs = sizeof(float) * d;
    auto run = [&](auto *wt) {
        using T = std::remove_const_t<std::remove_pointer_t<decltype(wt)>>;
        static DeviceFlags attr;
        smem_opt_in(k_gemv2<T>, 64 * 1024, attr);
        if (emb)
            L.run("temb_in", [&] {
                launch_dep(k_temb_in<T>, dim3((d + 7) / 8), dim3(256), 0, st, nullptr, (const T *)w->w_t1, *emb, K0, d,
                           a1);
            });
        else
            L.run("temb_in", [&] {
                launch_dep(k_temb_in_sigma<T>, dim3((d + 7) / 8), dim3(256), 0, st, nullptr, (const T *)w->w_t1, sigmas,
                           step, t_per_sigma, K0, d, a1);
            });
        L.run("gemv", [&] {
            launch_dep(k_gemv2<T>, dim3((d + 7) / 8), dim3(256), xs, st, nullptr, (const T *)w->w_t2, d, e,
                       (const T *)w->w_t2, 0, e, (const float *)a1, d, 0);
        });
        L.run("gemv", [&] {
            launch_dep(k_gemv2<T>, dim3((nch * d + d + 7) / 8), dim3(256), xs, st, nullptr, (const T *)w->w_mod,
                       nch * d, mod_row, (const T *)w->w_fin, d, scale_final, (const float *)e, d, 1);
        });
    };
    if (c->dtype == QI21_DTYPE_BF16)
        run((const bf16 *)nullptr);
    else
        run((const float *)nullptr);
    return finish(L);
}

extern "C" qi21_status qi21_modulation(const qi21_config *c, const qi21_weights *w, double t, float *mod_row,
                                       float *scale_final, void *ws, size_t ws_bytes, void *stream) {
    if (!std::isfinite(t)) return QI21_ERR_INVALID_ARG;
    qi21_status s = check_shapes(c);
    if (s) return s;
    TembArg emb;
    qi21_timestep_embedding(t, c->time_dim, emb.v);
    return modulation_impl(c, w, &emb, nullptr, 0, 0.0, mod_row, scale_final, ws, ws_bytes, stream);
}

extern "C" qi21_status qi21_modulation_sigma(const qi21_config *c, const qi21_weights *w, double sigma,
                                             float *mod_row, float *scale_final, void *ws, size_t ws_bytes,
                                             void *stream) {
    if (!std::isfinite(sigma)) return QI21_ERR_INVALID_ARG;
    return qi21_modulation(c, w, QI21_T_PER_SIGMA * sigma, mod_row, scale_final, ws, ws_bytes, stream);
}

extern "C" int32_t qi21_kernel_family(const qi21_config *c) {
    if (check_shapes(c) != QI21_OK) return QI21_FAMILY_NONE;
    return uses_cuda_core_gemm(*c) ? QI21_FAMILY_CUDA_CORES : QI21_FAMILY_TENSOR_CORES;
}

extern "C" qi21_status qi21_modulation_at(const qi21_config *c, const qi21_weights *w, const double *sigmas,
                                          int32_t step, double t_per_sigma, float *mod_row, float *scale_final,
                                          void *ws, size_t ws_bytes, void *stream) {
    if (!sigmas || ((uintptr_t)sigmas & 7) || step < 0 || !std::isfinite(t_per_sigma)) return QI21_ERR_INVALID_ARG;
    return modulation_impl(c, w, nullptr, sigmas, step, t_per_sigma, mod_row, scale_final, ws, ws_bytes, stream);
}

extern "C" qi21_status qi21_prefix_extract(const qi21_config *c, const qi21_weights *w, qi21_kv_cache *cache,
                                           const float *prefix_hidden, const float *cos_sin_prefix,
                                           const int32_t *kv_limit_prefix, const float *mod_row_prefix, void *ws,
                                           size_t ws_bytes, void *stream) {
    qi21_status s = check_shapes(c);
    if (s) return s;
    if ((s = check_weights(w, false))) return s;
    if (!cache || !al16(cache->base)) return QI21_ERR_INVALID_ARG;
    if (!al16(prefix_hidden) || !al16(cos_sin_prefix) || !al16(kv_limit_prefix) || !al16(mod_row_prefix) ||
        !al16(ws))
        return QI21_ERR_INVALID_ARG;
    const int P = cache->n_prefix, N = cache->n_target;
    const bool shared = cache->shared_prefix != 0;
    const int B = shared ? 1 : cache->batch;          // a shared prefix is extracted once
    if (cache->n_layers != c->n_layers || cache->d_model != c->d_model || cache->dtype != c->dtype ||
        cache->batch <= 0 || P <= 0 || N <= 0)
        return QI21_ERR_CACHE_STATE;
    const WsLayout lay = ws_layout(*c, B, P, N);
    if (ws_bytes < lay.total) return QI21_ERR_WORKSPACE_TOO_SMALL;
    char *wsb = (char *)ws;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    const int d = c->d_model;
    const size_t eb = dtype_bytes(c->dtype);
    cache->state = QI21_CACHE_EMPTY;
    StackArgs a{};
    a.B = B; a.M = P; a.split = P; a.P = P; a.N = N;
    a.h = (float *)(wsb + lay.h);
    a.xn = wsb + lay.xn; a.q = wsb + lay.q; a.o = wsb + lay.o; a.hid = wsb + lay.hid;
    a.gemm = (float *)(wsb + lay.gemm); a.gates = (float *)(wsb + lay.gates); a.err = (uint32_t *)(wsb + lay.err);
    a.mod_lo = mod_row_prefix; a.mod_hi = mod_row_prefix;
    a.cos_sin = cos_sin_prefix;
    // rows per (layer, K|V) block: one item of Pp + batch*N rows (shared), else batch items of P + N rows
    const int64_t rows = shared ? shared_rows(P, N, cache->batch) : (int64_t)P + N;
    a.kv_k0 = (char *)cache->base;
    a.kv_v0 = (char *)cache->base + eb * (size_t)B * rows * d;
    a.kv_layer_stride = 2 * (int64_t)B * rows * d;
    a.kv_bstride = rows * d;
    a.row_off = 0;
    a.kv_len = P;
    a.kv_limit = kv_limit_prefix;
    a.kv_only_last = true;
    L.run("copy_prefix", [&] {
        const int64_t tot = (int64_t)B * P * d;
        k_copy_rows<<<grid_for(tot, 256), 256, 0, st>>>(prefix_hidden, a.h, P, d, P, tot);
    });
    if (c->dtype == QI21_DTYPE_BF16) run_stack<bf16>(L, *c, *w, a);
    else run_stack<float>(L, *c, *w, a);
    s = finish(L);
    if (s == QI21_OK) cache->state = QI21_CACHE_EXTRACTED;
    return s;
}

extern "C" qi21_status qi21_cached_step(const qi21_config *c, const qi21_weights *w, const qi21_kv_cache *cache,
                                        const float *x_k, const float *cos_sin_target, const float *mod_row_target,
                                        const float *scale_final, float *v_out, void *ws, size_t ws_bytes,
                                        void *stream) {
    qi21_status s = check_shapes(c);
    if (s) return s;
    if ((s = check_weights(w, false))) return s;
    if (!cache || !al16(cache->base)) return QI21_ERR_INVALID_ARG;
    if (!al16(x_k) || !al16(cos_sin_target) || !al16(mod_row_target) || !al16(scale_final) || !al16(v_out) ||
        !al16(ws))
        return QI21_ERR_INVALID_ARG;
    if (cache->state != QI21_CACHE_EXTRACTED || cache->n_layers != c->n_layers || cache->d_model != c->d_model ||
        cache->dtype != c->dtype)
        return QI21_ERR_CACHE_STATE;
    const int B = cache->batch, P = cache->n_prefix, N = cache->n_target;
    const bool shared = cache->shared_prefix != 0;
    const WsLayout lay = ws_layout(*c, B, P, N);
    if (ws_bytes < lay.total) return QI21_ERR_WORKSPACE_TOO_SMALL;
    char *wsb = (char *)ws;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    const int d = c->d_model;
    const size_t eb = dtype_bytes(c->dtype);
    StackArgs a{};
    a.B = B; a.M = N; a.split = 0; a.P = P; a.N = N;
    a.h = (float *)(wsb + lay.h);
    a.xn = wsb + lay.xn; a.q = wsb + lay.q; a.o = wsb + lay.o; a.hid = wsb + lay.hid;
    a.gemm = (float *)(wsb + lay.gemm); a.gates = (float *)(wsb + lay.gates); a.err = (uint32_t *)(wsb + lay.err);
    a.mod_lo = mod_row_target; a.mod_hi = mod_row_target;
    a.cos_sin = cos_sin_target;
    if (shared) {
        const int64_t rows_all = shared_rows(P, N, B);
        a.kv_k0 = (char *)cache->base;
        a.kv_v0 = (char *)cache->base + eb * (size_t)rows_all * d;
        a.kv_layer_stride = 2 * rows_all * d;
        a.kv_bstride = (int64_t)N * d;            // item b's target rows start at Pp + b*N
        a.row_off = (int)padded_prefix_rows(P);
        a.kv_len = P + N;                         // keys each target row sees
        a.shared = true;
        a.shared_P = P;
        a.shared_Pp = (int)padded_prefix_rows(P);
    } else {
        const int64_t rows = (int64_t)P + N;
        a.kv_k0 = (char *)cache->base;
        a.kv_v0 = (char *)cache->base + eb * (size_t)B * rows * d;
        a.kv_layer_stride = 2 * (int64_t)B * rows * d;
        a.kv_bstride = rows * d;
        a.row_off = P;
        a.kv_len = (int)rows;
    }
    a.kv_limit = nullptr;
    a.kv_only_last = false;
    if (c->dtype == QI21_DTYPE_BF16 && tc_head_supported(*c)) {
        launch_img_in_tc(L, *c, x_k, w->w_img_in, a.h, B * N, (bf16 *)(wsb + lay.xin), a.err);
        run_stack<bf16>(L, *c, *w, a);
        launch_final_tc(L, *c, a.h, B * N, scale_final, w->w_out, v_out, wsb, lay, a.err);
    } else if (c->dtype == QI21_DTYPE_BF16) {
        launch_img_in<bf16>(L, *c, x_k, w->w_img_in, a.h, B, N, N, 0);
        run_stack<bf16>(L, *c, *w, a);
        launch_final<bf16>(L, *c, a.h, N, 0, B, N, scale_final, w->w_out, v_out);
    } else {
        launch_img_in<float>(L, *c, x_k, w->w_img_in, a.h, B, N, N, 0);
        run_stack<float>(L, *c, *w, a);
        launch_final<float>(L, *c, a.h, N, 0, B, N, scale_final, w->w_out, v_out);
    }
    return finish(L);
}

extern "C" qi21_status qi21_full_recompute_step(const qi21_config *c, const qi21_weights *w, int32_t B, int32_t P,
                                                int32_t N, const float *prefix_hidden, const float *x_k,
                                                const float *cos_sin_all, const int32_t *kv_limit_all,
                                                const float *mod_row_prefix, const float *mod_row_target,
                                                const float *scale_final, float *v_out, void *ws, size_t ws_bytes,
                                                void *stream) {
    qi21_status s = check_shapes(c);
    if (s) return s;
    if ((s = check_weights(w, false))) return s;
    if (B <= 0 || P <= 0 || N <= 0) return QI21_ERR_SHAPE;
    if (!al16(prefix_hidden) || !al16(x_k) || !al16(cos_sin_all) || !al16(kv_limit_all) || !al16(mod_row_prefix) ||
        !al16(mod_row_target) || !al16(scale_final) || !al16(v_out) || !al16(ws))
        return QI21_ERR_INVALID_ARG;
    const WsLayout lay = ws_layout(*c, B, P, N);
    if (ws_bytes < lay.total) return QI21_ERR_WORKSPACE_TOO_SMALL;
    char *wsb = (char *)ws;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    const int d = c->d_model, S = P + N;
    const size_t eb = dtype_bytes(c->dtype);
    StackArgs a{};
    a.B = B; a.M = S; a.split = P; a.P = P; a.N = N;
    a.h = (float *)(wsb + lay.h);
    a.xn = wsb + lay.xn; a.q = wsb + lay.q; a.o = wsb + lay.o; a.hid = wsb + lay.hid;
    a.gemm = (float *)(wsb + lay.gemm); a.gates = (float *)(wsb + lay.gates); a.err = (uint32_t *)(wsb + lay.err);
    a.mod_lo = mod_row_prefix; a.mod_hi = mod_row_target;
    a.cos_sin = cos_sin_all;
    a.kv_k0 = wsb + lay.kvf;
    a.kv_v0 = wsb + lay.kvf + eb * (size_t)B * S * d;
    a.kv_layer_stride = 0;
    a.kv_bstride = (int64_t)S * d;
    a.row_off = 0;
    a.kv_len = S;
    a.kv_limit = kv_limit_all;
    a.kv_only_last = false;
    L.run("copy_prefix", [&] {
        const int64_t tot = (int64_t)B * P * d;
        k_copy_rows<<<grid_for(tot, 256), 256, 0, st>>>(prefix_hidden, a.h, P, d, S, tot);
    });
    if (c->dtype == QI21_DTYPE_BF16) {
        launch_img_in<bf16>(L, *c, x_k, w->w_img_in, a.h, B, N, S, P);
        run_stack<bf16>(L, *c, *w, a);
        launch_final<bf16>(L, *c, a.h, S, P, B, N, scale_final, w->w_out, v_out);
    } else {
        launch_img_in<float>(L, *c, x_k, w->w_img_in, a.h, B, N, S, P);
        run_stack<float>(L, *c, *w, a);
        launch_final<float>(L, *c, a.h, S, P, B, N, scale_final, w->w_out, v_out);
    }
    return finish(L);
}

extern "C" qi21_status qi21_euler_update(const float *x_k, const float *v, double sigma_k, double sigma_k1,
                                         float *x_out, int64_t n, void *stream) {
    if (!al16(x_k) || !al16(v) || !al16(x_out) || n < 0) return QI21_ERR_INVALID_ARG;
    if (!std::isfinite(sigma_k) || !std::isfinite(sigma_k1)) return QI21_ERR_INVALID_ARG;
    if (n == 0) return QI21_OK;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    const float dsig = (float)(sigma_k1 - sigma_k);
    L.run("euler", [&] { launch_dep(k_euler, dim3(grid_for((n + 3) / 4, 256)), dim3(256), 0, st, nullptr, x_k, v, dsig, x_out, n); });
    return finish(L);
}

extern "C" qi21_status qi21_pack_weights(const qi21_config *c, const qi21_weights_canonical *cw, void *packed,
                                         size_t packed_bytes, qi21_weights *w, void *stream) {
    qi21_status s = check_shapes(c);
    if (s) return s;
    if (!cw || !w || !al16(packed)) return QI21_ERR_INVALID_ARG;
    const void *src[15] = {cw->w_img_in, cw->w_out, cw->w_t1,   cw->w_t2,   cw->w_mod, cw->w_fin, cw->w_q,     cw->w_k,
                           cw->w_v,      cw->w_o,   cw->w_gate, cw->w_up,   cw->w_down, cw->q_norm, cw->k_norm};
    for (const void *p : src)
        if (!al16(p)) return QI21_ERR_INVALID_ARG;
    const PackedLayout lay = packed_layout(*c);
    if (packed_bytes < lay.total) return QI21_ERR_WORKSPACE_TOO_SMALL;
    const int d = c->d_model, C = c->latent_ch, T = c->time_dim, F = c->mlp_hidden, L = c->n_layers;
    const int nch = c->use_shift ? 6 : 4;
    // canonical [in][out] (rows = in, cols = out) per matrix, and how many are stacked
    const int rows[13] = {C, d, T, d, d, d, d, d, d, d, d, d, F};
    const int cols[13] = {d, C, d, d, nch * d, d, d, d, d, d, F, F, d};
    const int nmat[13] = {1, 1, 1, 1, 1, 1, L, L, L, L, L, L, L};
    char *base = (char *)packed;
    void *dst[15];
    for (int i = 0; i < 15; ++i) dst[i] = base + lay.off[i];
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L_(st);
    for (int i = 0; i < 13; ++i) {
        dim3 grid((cols[i] + 31) / 32, (rows[i] + 31) / 32, nmat[i]);
        if (c->dtype == QI21_DTYPE_BF16)
            L_.run("transpose", [&] {
                k_transpose<bf16><<<grid, 256, 0, st>>>((const bf16 *)src[i], (bf16 *)dst[i], rows[i], cols[i]);
            });
        else
            L_.run("transpose", [&] {
                k_transpose<float><<<grid, 256, 0, st>>>((const float *)src[i], (float *)dst[i], rows[i], cols[i]);
            });
    }
    for (int i = 13; i < 15; ++i)
        if (cudaMemcpyAsync(dst[i], src[i], sizeof(float) * (size_t)L * c->head_dim, cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess)
            return QI21_ERR_CUDA;
    const qi21_status fs = finish(L_);
    if (fs) return fs;
    w->w_img_in = dst[0]; w->w_out = dst[1]; w->w_t1 = dst[2]; w->w_t2 = dst[3]; w->w_mod = dst[4];
    w->w_fin = dst[5]; w->w_q = dst[6]; w->w_k = dst[7]; w->w_v = dst[8]; w->w_o = dst[9];
    w->w_gate = dst[10]; w->w_up = dst[11]; w->w_down = dst[12];
    w->q_norm = (const float *)dst[13]; w->k_norm = (const float *)dst[14];
    return QI21_OK;
}

extern "C" qi21_status qi21_pack_prefix(int32_t B, int32_t P, int32_t d, int32_t n_slots, int32_t n_img,
                                        const float *ctx, const float *img_tokens, const int32_t *slot_of,
                                        const int32_t *img_row, int32_t mode, float *out, void *stream) {
    if (B <= 0 || P <= 0 || d <= 0 || d % 4 || n_slots <= 0 || n_img < 0) return QI21_ERR_INVALID_ARG;
    if (mode != QI21_PACK_SUBSTITUTE && mode != QI21_PACK_ADD) return QI21_ERR_INVALID_ARG;
    if (!al16(ctx) || !al16(out) || !slot_of || !img_row || (n_img > 0 && !al16(img_tokens)))
        return QI21_ERR_INVALID_ARG;
    if ((int64_t)B > 65535) return QI21_ERR_SHAPE;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    L.run("pack", [&] {
        k_pack_prefix<<<dim3(P, B), 256, 0, st>>>(ctx, img_tokens, slot_of, img_row, P, d, n_slots, n_img, mode, out);
    });
    return finish(L);
}

extern "C" qi21_status qi21_img_in_tokens(const qi21_config *c, const qi21_weights *w, const float *latents,
                                          int32_t rows, float *out, void *stream) {
    qi21_status s = check_shapes(c);
    if (s) return s;
    if (!w || !al16(w->w_img_in) || !al16(latents) || !al16(out) || rows <= 0) return QI21_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    if (c->dtype == QI21_DTYPE_BF16)
        launch_img_in<bf16>(L, *c, latents, w->w_img_in, out, 1, rows, rows, 0);
    else
        launch_img_in<float>(L, *c, latents, w->w_img_in, out, 1, rows, rows, 0);
    return finish(L);
}

extern "C" qi21_status qi21_euler_update_at(const float *x_k, const float *v, const double *sigmas, int32_t step,
                                            float *x_out, int64_t n, void *stream) {
    if (!al16(x_k) || !al16(v) || !al16(x_out) || n < 0) return QI21_ERR_INVALID_ARG;
    if (!sigmas || ((uintptr_t)sigmas & 7) || step < 0) return QI21_ERR_INVALID_ARG;
    if (n == 0) return QI21_OK;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    L.run("euler", [&] {
        launch_dep(k_euler_sigma, dim3(grid_for((n + 3) / 4, 256)), dim3(256), 0, st, nullptr, x_k, v, sigmas, step, x_out,
                   n);
    });
    return finish(L);
}

extern "C" qi21_status qi21_denoise_image(const qi21_config *c, const qi21_weights *w, qi21_kv_cache *cache,
                                          const float *prefix_hidden, const float *cos_sin_prefix,
                                          const int32_t *kv_limit_prefix, const float *cos_sin_target,
                                          const double *sigmas, int32_t n_steps, double t_per_sigma, float *x,
                                          float *v, float *mod_row_prefix, float *mod_row_target,
                                          float *scale_final, void *ws, size_t ws_bytes, void *stream) {
    if (!cache || n_steps < 1 || !sigmas) return QI21_ERR_INVALID_ARG;
    int launches = 0;
    qi21_status s = qi21_modulation(c, w, 0.0, mod_row_prefix, scale_final, ws, ws_bytes, stream);
    launches += g_last_launches;
    if (!s) s = qi21_prefix_extract(c, w, cache, prefix_hidden, cos_sin_prefix, kv_limit_prefix, mod_row_prefix, ws,
                                    ws_bytes, stream);
    launches += g_last_launches;
    const int64_t n = (int64_t)cache->batch * cache->n_target * c->latent_ch;
    for (int k = 0; k < n_steps && !s; ++k) {
        s = qi21_modulation_at(c, w, sigmas, k, t_per_sigma, mod_row_target, scale_final, ws, ws_bytes, stream);
        launches += g_last_launches;
        if (!s) s = qi21_cached_step(c, w, cache, x, cos_sin_target, mod_row_target, scale_final, v, ws, ws_bytes,
                                     stream);
        launches += g_last_launches;
        if (!s) s = qi21_euler_update_at(x, v, sigmas, k, x, n, stream);
        launches += g_last_launches;
    }
    g_last_launches = launches;
    return s;
}

extern "C" qi21_status qi21_check_device_error(void *ws, size_t ws_bytes, void *stream) {
    if (!al16(ws) || ws_bytes < 64) return QI21_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return QI21_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return QI21_ERR_CUDA;
    if (word != 0) {
        if (cudaMemsetAsync(ws, 0, sizeof(word), st) != cudaSuccess) return QI21_ERR_CUDA;
        cudaStreamSynchronize(st);
        return word == DEV_ERR_TIMEOUT ? QI21_ERR_DEVICE_TIMEOUT : QI21_ERR_DEVICE_CHECK;
    }
    return QI21_OK;
}

extern "C" qi21_status qi21_selftest_wait_timeout(void *ws, size_t ws_bytes, int64_t limit_ns, void *stream) {
    if (!al16(ws) || ws_bytes < 64) return QI21_ERR_INVALID_ARG;
    if (limit_ns < 1 || limit_ns > 1000000000) return QI21_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    Launcher L(st);
    L.run("selftest_wait_timeout", [&] {
        sm100::k_selftest_wait_timeout<<<1, 32, 0, st>>>((uint32_t *)ws, (uint64_t)limit_ns);
    });
    return finish(L);
}

extern "C" void qi21_profile_enable(int32_t enable) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = enable != 0;
}

extern "C" void qi21_profile_reset(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_recs.clear();
    g_event_next = 0;
}

extern "C" int32_t qi21_profile_read(qi21_kernel_time *out, int32_t max_entries) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    std::vector<qi21_kernel_time> acc;
    for (const ProfRec &r : g_prof_recs) {
        cudaEventSynchronize(r.b);
        float ms = 0.f;
        cudaEventElapsedTime(&ms, r.a, r.b);
        bool found = false;
        for (auto &k : acc)
            if (strcmp(k.name, r.name) == 0) {
                k.launches += 1;
                k.total_ms += ms;
                found = true;
                break;
            }
        if (!found) acc.push_back({r.name, 1, (double)ms});
    }
    int32_t n = 0;
    for (auto &k : acc) {
        if (n >= max_entries || !out) break;
        out[n++] = k;
    }
    return n;
}

extern "C" int32_t qi21_last_launch_count(void) { return g_last_launches; }
