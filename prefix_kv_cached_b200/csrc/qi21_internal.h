// Internal declarations shared by the host helpers and the CUDA entry points.
#pragma once
#include <stddef.h>
#include <stdint.h>

#include "qi21.h"

namespace qi21 {

// Workspace carve-up. Every region starts on a 256-byte boundary.
//   err     : device error words (uint32 [8])
//   gates   : fp32 [4][d]  tanh(gate1) prefix row, tanh(gate1) target row,
//                          tanh(gate2) prefix row, tanh(gate2) target row
//   modtmp  : fp32 [2][d]  timestep-MLP intermediates
//   h       : fp32 [R][d]  residual stream (R = B * S rows at most)
//   xn      : T [R][d]     modulated LayerNorm output (LN1 and LN2 share it)
//   q       : T [R][d]     queries after QK-RMSNorm and RoPE
//   o       : T [R][d]     attention output
//   hid     : T [R][F]     SwiGLU activation
//   kvf     : T [2][B][S][d]  K/V of the full recomputation
//   gemm    : fp32 [R][max(3d, 2F)]  outputs of the CUDA-core GEMMs (present when
//             they run: F32 mode, or BF16 mode with the tensor cores switched off)
//   xin     : bf16 [B*N][C]   the latent rounded for the tensor-core img_in
//   fwp, fu : bf16 [C][d], fp32 [C]  W_out scaled by (1 + scale_final) and its row
//             sums (tensor-core final AdaLN + proj_out)
//   fpart   : fp32 [FINAL_MAX_KSPLIT][B*N][68]  its per-K-slice partial sums
constexpr int FINAL_MAX_KSPLIT = 8;
struct WsLayout {
    size_t err, gates, modtmp, h, xn, q, o, hid, kvf, gemm, xin, fwp, fu, fpart, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline size_t dtype_bytes(int32_t dtype) { return dtype == QI21_DTYPE_BF16 ? 2 : 4; }

// Kernel family of the BF16 mode (process-wide; qi21_set_tensor_cores).
bool tc_enabled();

// The shape checks every device entry point applies before enqueueing work:
// QI21_ERR_INVALID_ARG / SHAPE / UNSUPPORTED, or QI21_OK.
qi21_status check_config_shapes(const qi21_config *c);

// Packed weight buffer of qi21_pack_weights: the 15 tensors of qi21_weights in
// struct order, [out][in] (stacked [L][out][in]), each on a 256-byte boundary.
struct PackedLayout {
    size_t off[15];
    size_t total;
};
inline PackedLayout packed_layout(const qi21_config &c) {
    const size_t eb = dtype_bytes(c.dtype);
    const size_t d = c.d_model, C = c.latent_ch, T = c.time_dim, F = c.mlp_hidden, L = c.n_layers;
    const size_t nch = c.use_shift ? 6 : 4, dh = c.head_dim;
    const size_t sizes[15] = {d * C * eb,     C * d * eb,     d * T * eb,     d * d * eb,     nch * d * d * eb,
                              d * d * eb,     L * d * d * eb, L * d * d * eb, L * d * d * eb, L * d * d * eb,
                              L * F * d * eb, L * F * d * eb, L * d * F * eb, L * dh * 4,     L * dh * 4};
    PackedLayout p{};
    size_t o = 0;
    for (int i = 0; i < 15; ++i) {
        p.off[i] = o;
        o += align256(sizes[i]);
    }
    p.total = o;
    return p;
}

inline bool uses_cuda_core_gemm(const qi21_config &c) { return c.dtype == QI21_DTYPE_F32 || !tc_enabled(); }

inline WsLayout ws_layout(const qi21_config &c, int64_t B, int64_t P, int64_t N) {
    const int64_t S = P + N, R = B * S, d = c.d_model, F = c.mlp_hidden;
    const size_t eb = dtype_bytes(c.dtype);
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += align256(bytes);
        return o;
    };
    L.err = take(64);
    L.gates = take(sizeof(float) * 4 * d);
    L.modtmp = take(sizeof(float) * 2 * d);
    L.h = take(sizeof(float) * R * d);
    L.xn = take(eb * R * d);
    L.q = take(eb * R * d);
    L.o = take(eb * R * d);
    L.hid = take(eb * R * F);
    L.kvf = take(eb * 2 * B * S * d);
    const int64_t gw = (3 * d > 2 * F) ? 3 * d : 2 * F;
    L.gemm = take(uses_cuda_core_gemm(c) ? sizeof(float) * R * gw : 0);
    const int64_t C = c.latent_ch;
    L.xin = take(2 * B * N * C);
    L.fwp = take(2 * C * d);
    L.fu = take(sizeof(float) * C);
    L.fpart = take(sizeof(float) * FINAL_MAX_KSPLIT * B * N * 68);
    L.total = off;
    return L;
}

}  // namespace qi21
