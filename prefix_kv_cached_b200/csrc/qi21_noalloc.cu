// qi21_modulation_noalloc: the shared-modulation computation for callers that
// cannot allocate device memory, with its scratch in a fixed device array.
//
// Some callers cannot hand the library a workspace: a host application whose
// device memory is entirely owned by another allocator (a framework's
// fixed-size memory pool, or a plug-in host that forbids device allocations
// from plug-ins), or a latency-critical loop that must never call cudaMalloc
// because it can block and synchronise the device. For them this entry point
// takes only its inputs and outputs; the two timestep-MLP intermediate vectors
// live in g_modulation_scratch below, a file-scope __device__ array that every
// GPU which loads the library keeps until the process exits.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "qi21.h"
#include "qi21_internal.h"
#include "qi21_simt.cuh"

namespace qi21 {

// [0, d): silu(w_t1 . emb(t));  [d, 2d): e = w_t2 . (first half).
// Both halves are fully written before they are read on every call, so
// nothing in the array has to start at zero.
static __device__ __align__(256) float g_modulation_scratch[2 * QI21_NOALLOC_MAX_D];

// Device address of g_modulation_scratch per device. In host code the
// symbol's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, called with the device current.
static constexpr int kMaxDevices = 64;
static float *g_scratch_addr[kMaxDevices] = {};
static std::mutex g_scratch_mu;

static float *scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_modulation_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_addr[dev] = static_cast<float *>(p);
    }
    return g_scratch_addr[dev];
}

static inline bool aligned16(const void *p) { return p && ((uintptr_t)p & 15) == 0; }

}  // namespace qi21

using namespace qi21;

extern "C" qi21_status qi21_modulation_noalloc(const qi21_config *c, const qi21_weights *w, double t,
                                               float *mod_row, float *scale_final, void *stream) {
    if (!c || !w) return QI21_ERR_INVALID_ARG;
    // the same shape checks as qi21_modulation, then this entry point's own limit
    const qi21_status shape = check_config_shapes(c);
    if (shape != QI21_OK) return shape;
    if (c->d_model > QI21_NOALLOC_MAX_D) return QI21_ERR_UNSUPPORTED;   // scratch holds 2 * QI21_NOALLOC_MAX_D floats
    if (!aligned16(w->w_t1) || !aligned16(w->w_t2) || !aligned16(w->w_mod) || !aligned16(w->w_fin) ||
        !aligned16(mod_row) || !aligned16(scale_final))
        return QI21_ERR_INVALID_ARG;
    if (!std::isfinite(t)) return QI21_ERR_INVALID_ARG;
    float *scratch = scratch_for_current_device();
    if (!scratch) return QI21_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    const int d = c->d_model, K0 = c->time_dim, nch = c->use_shift ? 6 : 4;
    TembArg emb;
    qi21_timestep_embedding(t, K0, emb.v);
    float *a1 = scratch, *e = scratch + d;
    const size_t xs = sizeof(float) * d;     // <= 32 KB: no opt-in above the 48 KB default needed
    // each launch's own status is read right after it, as the other entry points do
    auto launched = [] { return cudaGetLastError() == cudaSuccess; };
    if (c->dtype == QI21_DTYPE_BF16) {
        k_temb_in<bf16><<<(d + 7) / 8, 256, 0, st>>>((const bf16 *)w->w_t1, emb, K0, d, a1);
        if (!launched()) return QI21_ERR_CUDA;
        k_gemv2<bf16><<<(d + 7) / 8, 256, xs, st>>>((const bf16 *)w->w_t2, d, e, (const bf16 *)w->w_t2, 0, e, a1,
                                                     d, 0);
        if (!launched()) return QI21_ERR_CUDA;
        k_gemv2<bf16><<<(nch * d + d + 7) / 8, 256, xs, st>>>((const bf16 *)w->w_mod, nch * d, mod_row,
                                                              (const bf16 *)w->w_fin, d, scale_final, e, d, 1);
        if (!launched()) return QI21_ERR_CUDA;
    } else {
        k_temb_in<float><<<(d + 7) / 8, 256, 0, st>>>((const float *)w->w_t1, emb, K0, d, a1);
        if (!launched()) return QI21_ERR_CUDA;
        k_gemv2<float><<<(d + 7) / 8, 256, xs, st>>>((const float *)w->w_t2, d, e, (const float *)w->w_t2, 0, e,
                                                      a1, d, 0);
        if (!launched()) return QI21_ERR_CUDA;
        k_gemv2<float><<<(nch * d + d + 7) / 8, 256, xs, st>>>((const float *)w->w_mod, nch * d, mod_row,
                                                               (const float *)w->w_fin, d, scale_final, e, d, 1);
        if (!launched()) return QI21_ERR_CUDA;
    }
    return QI21_OK;
}
