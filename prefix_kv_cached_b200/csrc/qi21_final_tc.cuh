// Final scale-only AdaLN + proj_out on tcgen05 (BF16 mode, cached step; 6B
// page §1 and §3): v[r][c] = sum_k LN(h)[r][k] (1 + s[k]) W_out[c][k].
//
// Written so that h (fp32, the largest tensor) is read from HBM once:
//   v[r][c] = rstd_r * (sum_k h[r][k] W'[c][k] - mean_r u[c]),
//   W'[c][k] = (1 + s[k]) W_out[c][k] (rounded to bf16), u[c] = sum_k W'[c][k],
// so the LayerNorm statistics (CUDA cores) and the contraction (tensor cores)
// come from the same pass.
//   k_final_prep   W' and u for this step's scale_final (one block per output c)
//   k_final_tc     one CTA per (128 rows, K slice): TMA streams fp32 h boxes and
//                  W' tiles into shared memory; four converter warps (one row per
//                  thread) accumulate the row's sum and sum of squares, round the
//                  row to bf16 into a swizzled K-major A tile; one elected lane
//                  issues tcgen05.mma (M 128, N 64, K 16) into a TMEM accumulator;
//                  the same warps write the partial sums of the slice
//   k_final_reduce adds the K slices and applies rstd (x - mean u)
// Latent channels C = 64 (the MMA's N); d a multiple of 64.
#pragma once
#include "qi21_gemm_tc.cuh"
#include "qi21_sm100.cuh"

namespace qi21 {

constexpr int FT_BM = 128, FT_C = 64, FT_BK = 64, FT_STAGES = 4;
constexpr int FT_H_BOX = FT_BM * 128;                  // one 32-float-wide fp32 box of 128 rows (16 KB)
constexpr int FT_H_BYTES = 2 * FT_H_BOX;               // 64 columns of h (32 KB)
constexpr int FT_W_BYTES = FT_C * FT_BK * 2;           // 64 x 64 bf16 (8 KB)
constexpr int FT_STAGE_BYTES = FT_H_BYTES + FT_W_BYTES;
constexpr int FT_A_BYTES = FT_BM * FT_BK * 2;          // 128 x 64 bf16 (16 KB)
constexpr int FT_PART = 68;                            // floats per row of a partial: 64 sums, sum h, sum h^2
constexpr size_t FT_SMEM = 1024 + (size_t)FT_STAGES * FT_STAGE_BYTES + 2 * FT_A_BYTES + 256;
constexpr int FT_THREADS = 192;

struct FinalParams {
    int R, d;
    int kblocks;     // d / 64
    int ksplit;      // K slices (gridDim.y)
    float *part;     // [ksplit][R][FT_PART]
    uint32_t *err;
};

// W'[c][k] = bf16((1 + s[k]) W_out[c][k]); u[c] = sum_k W'[c][k] (fp32 sum of the
// rounded values). One block per output c; each thread takes 8 consecutive k
// (16-byte loads and stores), d % 8 == 0.
static __global__ void __launch_bounds__(256) k_final_prep(const bf16 *__restrict__ w_out, const float *__restrict__ sf,
                                                           int d, bf16 *__restrict__ wp, float *__restrict__ u) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ float red[32];
    const int c = blockIdx.x;
    const uint4 *w8 = reinterpret_cast<const uint4 *>(w_out + (size_t)c * d);
    uint4 *o8 = reinterpret_cast<uint4 *>(wp + (size_t)c * d);
    const float4 *s4 = reinterpret_cast<const float4 *>(sf);
    float acc = 0.f;
    for (int k8 = threadIdx.x; k8 < d / 8; k8 += blockDim.x) {
        const uint4 wv = w8[k8];
        const float4 sa = s4[2 * k8], sb = s4[2 * k8 + 1];
        const float sc[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        const uint32_t win[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t wout[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&win[i]));
            const __nv_bfloat162 r = __floats2bfloat162_rn((1.f + sc[2 * i]) * f.x, (1.f + sc[2 * i + 1]) * f.y);
            const float2 g = __bfloat1622float2(r);
            acc += g.x + g.y;
            wout[i] = *reinterpret_cast<const uint32_t *>(&r);
        }
        o8[k8] = make_uint4(wout[0], wout[1], wout[2], wout[3]);
    }
    acc = block_sum(acc, red);
    if (threadIdx.x == 0) u[c] = acc;
}

__global__ void __launch_bounds__(FT_THREADS, 1)
    k_final_tc(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW, FinalParams p) {
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *stages = smem;                                              // [S][h box 0 | h box 1 | W']
    uint8_t *abuf = smem + (size_t)FT_STAGES * FT_STAGE_BYTES;           // [2][128 rows x 128 B]
    uint64_t *bars = reinterpret_cast<uint64_t *>(abuf + 2 * FT_A_BYTES);
    uint64_t *full = bars;                      // [S] TMA bytes landed
    uint64_t *empty = full + FT_STAGES;         // [S] converters read h (128) + MMAs read W' (1)
    uint64_t *afull = empty + FT_STAGES;        // [2] converters wrote the A tile (128)
    uint64_t *aempty = afull + 2;               // [2] MMAs that read the A tile are done
    uint64_t *dfull = aempty + 2;               // every MMA done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(dfull + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    static_assert((2 * FT_STAGES + 2 * 2 + 1) * 8 + 16 <= 256, "barrier region");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.x * FT_BM, ks = blockIdx.y;
    const int kb0 = (int)((int64_t)p.kblocks * ks / p.ksplit), kb1 = (int)((int64_t)p.kblocks * (ks + 1) / p.ksplit);
    const int nk = kb1 - kb0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < FT_STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), FT_BM + 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(smem_u32(&afull[j]), FT_BM);
            mbar_init(smem_u32(&aempty[j]), 1);
        }
        mbar_init(smem_u32(dfull), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), FT_C);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int i = 0; i < nk; ++i) {
                const int s = i % FT_STAGES, kb = kb0 + i;
                if (!mbar_wait(smem_u32(&empty[s]), ((i / FT_STAGES) & 1) ^ 1, abort_flag, p.err)) break;
                const uint32_t fb = smem_u32(&full[s]);
                mbar_arrive_expect_tx(fb, FT_STAGE_BYTES);
                uint8_t *st = stages + (size_t)s * FT_STAGE_BYTES;
                tma_load_2d(smem_u32(st), &tmH, fb, kb * FT_BK, r0);
                tma_load_2d(smem_u32(st + FT_H_BOX), &tmH, fb, kb * FT_BK + 32, r0);
                tma_load_2d(smem_u32(st + FT_H_BYTES), &tmW, fb, kb * FT_BK, 0);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ UMMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(FT_BM, FT_C);
        const bool leader = elect_one();
        auto wait_warp = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, abort_flag, p.err) ? 1 : 0) != 0;
        };
        bool ok = true;
        for (int i = 0; i < nk && ok; ++i) {
            const int s = i % FT_STAGES, j = i & 1;
            ok = wait_warp(&afull[j], (i >> 1) & 1) && wait_warp(&full[s], (i / FT_STAGES) & 1);
            if (!ok) break;
            tc_fence_after();
            if (leader) {
                const uint64_t da = sdesc_kmajor_sw128(smem_u32(abuf + (size_t)j * FT_A_BYTES));
                const uint64_t db = sdesc_kmajor_sw128(smem_u32(stages + (size_t)s * FT_STAGE_BYTES + FT_H_BYTES));
#pragma unroll
                for (int k = 0; k < FT_BK / 16; ++k)
                    umma_f16(tmem_base, da + 2 * k, db + 2 * k, idesc, (i > 0 || k > 0) ? 1u : 0u);
                umma_commit(smem_u32(&aempty[j]));
                umma_commit(smem_u32(&empty[s]));
            }
            __syncwarp();
        }
        if (ok && leader) umma_commit(smem_u32(dfull));
        __syncwarp();
    } else {
        // ------------------------------------------------------------ converters, then epilogue
        const int quad = warp & 3;                 // TMEM lane quadrant of this warp
        const int r = quad * 32 + lane;            // row within the tile
        const uint32_t sw = (uint32_t)(r & 7);
        float sum = 0.f, sumsq = 0.f;
        bool ok = true;
        for (int i = 0; i < nk; ++i) {
            const int s = i % FT_STAGES, j = i & 1;
            if (!mbar_wait(smem_u32(&full[s]), (i / FT_STAGES) & 1, abort_flag, p.err)) {
                ok = false;
                break;
            }
            const uint8_t *hs = stages + (size_t)s * FT_STAGE_BYTES + (size_t)r * 128;
            uint32_t packed[32];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 f = *reinterpret_cast<const float4 *>(hs + b * FT_H_BOX + ((q ^ sw) << 4));
                    sum += (f.x + f.y) + (f.z + f.w);
                    sumsq += (f.x * f.x + f.y * f.y) + (f.z * f.z + f.w * f.w);
                    packed[b * 16 + q * 2] = pack_bf16x2(f.x, f.y);
                    packed[b * 16 + q * 2 + 1] = pack_bf16x2(f.z, f.w);
                }
            }
            mbar_arrive(smem_u32(&empty[s]));      // this row of h has been read
            if (!mbar_wait(smem_u32(&aempty[j]), ((i >> 1) & 1) ^ 1, abort_flag, p.err)) {
                ok = false;
                break;
            }
            uint8_t *ar = abuf + (size_t)j * FT_A_BYTES + (size_t)r * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<uint4 *>(ar + ((q ^ sw) << 4)) =
                    make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
            fence_proxy_async_shared();
            mbar_arrive(smem_u32(&afull[j]));
        }
        // every lane of the warp takes the same branch: the TMEM loads are warp-collective
        if (__all_sync(0xffffffffu, ok ? 1 : 0) && nk > 0 &&
            __all_sync(0xffffffffu, mbar_wait(smem_u32(dfull), 0, abort_flag, p.err) ? 1 : 0)) {
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16);
            float d0[32], d1[32];
            tmem_ld32(taddr, d0);
            tmem_ld32(taddr + 32, d1);
            tmem_wait_ld();
            const int row = r0 + r;
            if (row < p.R) {
                float4 *dst = reinterpret_cast<float4 *>(p.part + ((size_t)ks * p.R + row) * FT_PART);
#pragma unroll
                for (int q = 0; q < 8; ++q) dst[q] = make_float4(d0[4 * q], d0[4 * q + 1], d0[4 * q + 2], d0[4 * q + 3]);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    dst[8 + q] = make_float4(d1[4 * q], d1[4 * q + 1], d1[4 * q + 2], d1[4 * q + 3]);
                dst[16] = make_float4(sum, sumsq, 0.f, 0.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, FT_C);
    }
}

// v[r][c] = rstd (sum_ks D[c] - mean u[c]); 16 threads per row, 4 outputs each.
static __global__ void __launch_bounds__(256) k_final_reduce(const float *__restrict__ part, int ksplit, int R, int d,
                                                             const float *__restrict__ u, float eps,
                                                             float *__restrict__ v) {
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int row = t >> 4, g = t & 15;
    if (row >= R) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float sum = 0.f, sumsq = 0.f;
    for (int ks = 0; ks < ksplit; ++ks) {
        const float4 *pr = reinterpret_cast<const float4 *>(part + ((size_t)ks * R + row) * FT_PART);
        const float4 a = pr[g];
        acc.x += a.x;
        acc.y += a.y;
        acc.z += a.z;
        acc.w += a.w;
        const float4 st = pr[16];
        sum += st.x;
        sumsq += st.y;
    }
    const float mean = sum / d;
    const float var = fmaxf(sumsq / d - mean * mean, 0.f);
    const float rstd = 1.0f / sqrtf(var + eps);
    const float4 u4 = reinterpret_cast<const float4 *>(u)[g];
    reinterpret_cast<float4 *>(v + (size_t)row * FT_C)[g] =
        make_float4(rstd * (acc.x - mean * u4.x), rstd * (acc.y - mean * u4.y), rstd * (acc.z - mean * u4.z),
                    rstd * (acc.w - mean * u4.w));
}

}  // namespace qi21
