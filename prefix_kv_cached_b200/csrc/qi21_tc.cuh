// tcgen05 / TMA tensor-core kernels for the BF16 mode (GEMMs with fused
// epilogues, attention). Declarations used by qi21_api.cu.
#pragma once
#include "qi21_common.cuh"

namespace qi21 {
struct Launcher;
inline bool tc_supported(const qi21_config &c) { (void)c; return false; }
static void tc_gemm_qkv(Launcher &, const qi21_config &, const bf16 *, int, int, const bf16 *, const bf16 *,
                        const bf16 *, const float *, const float *, const float *, bf16 *, bf16 *, bf16 *, int64_t,
                        int, uint32_t *) {}
static void tc_attention(Launcher &, const qi21_config &, const bf16 *, int64_t, int, const bf16 *, const bf16 *,
                         int64_t, int, const int *, bf16 *, int, uint32_t *) {}
static void tc_gemm_residual(Launcher &, const qi21_config &, const bf16 *, int, int, const bf16 *, int, float *,
                             int, int, const float *, const float *, uint32_t *, const char *) {}
static void tc_gemm_swiglu(Launcher &, const qi21_config &, const bf16 *, int, const bf16 *, const bf16 *, bf16 *,
                           uint32_t *) {}
}  // namespace qi21
