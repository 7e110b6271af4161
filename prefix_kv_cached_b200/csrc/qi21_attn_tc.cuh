// Flash attention on tcgen05 tensor cores (BF16 mode):
//   o = softmax(q k^T / sqrt(Dh)) v over keys [0, limit(row)) of each query row,
// limit = kv_limit[row] (block-causal prefix extract, full recompute) or every
// one of the kv_len keys (cached target rows: the target is last, so they see
// the whole prefix cache and all target keys).
//
// One CTA per (item, head, 128 query rows); K/V tiles of 128 keys stream
// through a 2-stage TMA ring (128-byte swizzle, no multicast).
//   warp 0     : TMA producer (Q once, then K_j and V_j)
//   warp 1     : TMEM allocator + UMMA issuer:
//                S_j = Q K_j^T  (M 128, N 128, K Dh)   -> TMEM S[j % 2]
//                O_j = P_j V_j  (M 128, N Dh, K 128)  -> TMEM O[j % 2]
//                P_j is read from shared memory (K-major), V_j as an MN-major operand.
//   warps 2..5 : softmax, one query row per thread (TMEM lane): two passes over
//                S_j (row max, then exp2 and the bf16 P row written swizzled to
//                shared memory); O_{j-1} is folded into fp32 registers one tile
//                late so that PV(j-1) runs under the softmax of tile j.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+Dh), O1 [384,384+Dh).
#pragma once
#include "qi21_sm100.cuh"

namespace qi21 {

struct AttnParams {
    int Mq;               // query rows per item
    int kv_len;           // key rows per item
    int H;
    int d;
    const int *kv_limit;  // [Mq] or null
    bf16 *out;            // [B*Mq][d]
    float scale_log2;     // log2(e) / sqrt(Dh)
    int layer;            // 4th coordinate of the K/V tensor maps
    uint32_t *err;
};

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *m, uint32_t bar, int x, int y, int z,
                                            int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
        "[%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

template <int DH>
struct AttnCfg {
    static constexpr int BQ = 128, BK = 128;
    static constexpr int BOXES = DH / 64;                  // 64-element (128-byte) swizzle boxes per row
    static constexpr int Q_BYTES = BQ * DH * 2;
    static constexpr int KV_BYTES = BK * DH * 2;           // one K or V tile
    static constexpr int P_BYTES = BQ * BK * 2;            // 32 KB
    static constexpr int STAGES = 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
    static constexpr int OFF_P = OFF_V + STAGES * KV_BYTES;
    static constexpr int OFF_BAR = OFF_P + P_BYTES;
    static constexpr size_t SMEM = 1024 + (size_t)OFF_BAR + 256;
    static constexpr int THREADS = 192;
};

template <int DH>
__global__ void __launch_bounds__(192, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, AttnParams p) {
    using namespace sm100;
    using C = AttnCfg<DH>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = bars + 1;      // [2]
    uint64_t *v_full = bars + 3;      // [2]
    uint64_t *kv_empty = bars + 5;    // [2]
    uint64_t *s_full = bars + 7;      // [2]
    uint64_t *s_empty = bars + 9;     // [2]
    uint64_t *p_full = bars + 11;
    uint64_t *o_full = bars + 12;     // [2]
    uint64_t *o_empty = bars + 14;    // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *kv_end_s = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * C::BQ, hh = blockIdx.y, b = blockIdx.z;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(q_full), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&k_full[i]), 1);
            mbar_init(smem_u32(&v_full[i]), 1);
            mbar_init(smem_u32(&kv_empty[i]), 1);
            mbar_init(smem_u32(&s_full[i]), 1);
            mbar_init(smem_u32(&s_empty[i]), 128);
            mbar_init(smem_u32(&o_full[i]), 1);
            mbar_init(smem_u32(&o_empty[i]), 128);
        }
        mbar_init(smem_u32(p_full), 128);
        *abort_flag = 0;
        *kv_end_s = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // keys this CTA needs: the largest limit over its query rows
    if (threadIdx.x >= 64) {
        const int row = q0 + (threadIdx.x - 64);
        int lim = 0;
        if (row < p.Mq) lim = p.kv_limit ? min(p.kv_limit[row], p.kv_len) : p.kv_len;
        atomicMax(kv_end_s, lim);
    }
    __syncthreads();
    const uint32_t tmem_base = *tmem_slot;
    const int kv_end = *kv_end_s;
    const int T = (kv_end + C::BK - 1) / C::BK;

    if (warp == 0) {
        if (lane == 0 && T > 0) {
            // ------------------------------------------------------------ TMA producer
            const uint32_t qb = smem_u32(q_full);
            mbar_arrive_expect_tx(qb, C::Q_BYTES);
            for (int x = 0; x < C::BOXES; ++x)
                tma_load_4d(smem_u32(smem + C::OFF_Q + x * (C::BQ * 128)), &tmQ, qb, hh * DH + x * 64,
                            b * p.Mq + q0, 0, 0);
            for (int j = 0; j < T; ++j) {
                const int s = j & 1;
                if (!mbar_wait(smem_u32(&kv_empty[s]), ((j >> 1) & 1) ^ 1, abort_flag, p.err)) break;
                const uint32_t kb = smem_u32(&k_full[s]), vb = smem_u32(&v_full[s]);
                mbar_arrive_expect_tx(kb, C::KV_BYTES);
                for (int x = 0; x < C::BOXES; ++x)
                    tma_load_4d(smem_u32(smem + C::OFF_K + s * C::KV_BYTES + x * (C::BK * 128)), &tmK, kb,
                                hh * DH + x * 64, j * C::BK, b, p.layer);
                mbar_arrive_expect_tx(vb, C::KV_BYTES);
                for (int x = 0; x < C::BOXES; ++x)
                    tma_load_4d(smem_u32(smem + C::OFF_V + s * C::KV_BYTES + x * (C::BK * 128)), &tmV, vb,
                                hh * DH + x * 64, j * C::BK, b, p.layer);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && T > 0) {
            // ------------------------------------------------------------ UMMA issuer
            constexpr uint32_t idesc_s = idesc_bf16_f32(C::BQ, C::BK);
            constexpr uint32_t idesc_o = idesc_bf16_f32(C::BQ, DH, true);
            const uint32_t sq = smem_u32(smem + C::OFF_Q);
            const uint32_t sp = smem_u32(smem + C::OFF_P);
            bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag, p.err);
            auto issue_pv = [&](int jj) -> bool {
                const int s = jj & 1, ob = jj & 1;
                if (!mbar_wait(smem_u32(p_full), jj & 1, abort_flag, p.err)) return false;
                if (!mbar_wait(smem_u32(&v_full[s]), (jj >> 1) & 1, abort_flag, p.err)) return false;
                if (!mbar_wait(smem_u32(&o_empty[ob]), ((jj >> 1) & 1) ^ 1, abort_flag, p.err)) return false;
                tc_fence_after();
                const uint32_t sv = smem_u32(smem + C::OFF_V + s * C::KV_BYTES);
                const uint32_t d_tmem = tmem_base + 256 + ob * 128;
#pragma unroll
                for (int k = 0; k < C::BK / 16; ++k) {
                    const uint64_t adesc = sdesc_kmajor_sw128(sp + (k >> 2) * (C::BQ * 128) + (k & 3) * 32);
                    const uint64_t bdesc = sdesc_mnmajor_sw128(sv + k * 2048, C::BK * 128);
                    umma_f16(d_tmem, adesc, bdesc, idesc_o, k > 0 ? 1u : 0u);
                }
                umma_commit(smem_u32(&o_full[ob]));
                umma_commit(smem_u32(&kv_empty[s]));
                return true;
            };
            for (int j = 0; j < T && ok; ++j) {
                const int s = j & 1, sb = j & 1;
                if (!mbar_wait(smem_u32(&k_full[s]), (j >> 1) & 1, abort_flag, p.err)) break;
                if (!mbar_wait(smem_u32(&s_empty[sb]), ((j >> 1) & 1) ^ 1, abort_flag, p.err)) break;
                tc_fence_after();
                const uint32_t sk = smem_u32(smem + C::OFF_K + s * C::KV_BYTES);
                const uint32_t d_tmem = tmem_base + sb * 128;
#pragma unroll
                for (int k = 0; k < DH / 16; ++k) {
                    const uint32_t off = (k >> 2) * (C::BQ * 128) + (k & 3) * 32;
                    umma_f16(d_tmem, sdesc_kmajor_sw128(sq + off), sdesc_kmajor_sw128(sk + (k >> 2) * (C::BK * 128) +
                                                                                     (k & 3) * 32),
                             idesc_s, k > 0 ? 1u : 0u);
                }
                umma_commit(smem_u32(&s_full[sb]));
                if (j >= 1 && !issue_pv(j - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) issue_pv(T - 1);
        }
    } else {
        // ---------------------------------------------------------------- softmax warps
        const int quad = warp & 3;
        const int r = quad * 32 + lane;                  // row within the tile = TMEM lane
        const int row = q0 + r;
        int lim = p.kv_len;
        if (p.kv_limit && row < p.Mq) lim = min(p.kv_limit[row], p.kv_len);
        const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
        uint8_t *prow = smem + C::OFF_P + r * 128;       // row r of each 64-key box
        const int sw = r & 7;
        float o[DH];
#pragma unroll
        for (int i = 0; i < DH; ++i) o[i] = 0.f;
        float m_run = -INFINITY, l_run = 0.f, alpha_prev = 0.f;
        const float c = p.scale_log2;
        bool ok = true;
        float v[32];
        for (int j = 0; j < T && ok; ++j) {
            const int sb = j & 1;
            if (!mbar_wait(smem_u32(&s_full[sb]), (j >> 1) & 1, abort_flag, p.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int key0 = j * C::BK;
            // pass 1: row max over the allowed keys
            float mx = -INFINITY;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                tmem_ld32(t_lane + sb * 128 + cc * 32, v);
                tmem_wait_ld();
                const int kb = key0 + cc * 32;
                if (kb + 32 <= lim) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, v[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (kb + i < lim) mx = fmaxf(mx, v[i]);
                }
            }
            const float m_new = fmaxf(m_run, mx);
            const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx((m_run - m_new) * c);
            const float mc = (m_new == -INFINITY) ? 0.f : m_new * c;
            // P buffer is free once PV(j-1) finished; O_{j-1} is then ready too
            if (j >= 1) {
                if (!mbar_wait(smem_u32(&o_full[(j - 1) & 1]), ((j - 1) >> 1) & 1, abort_flag, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            // pass 2: p = exp2(s c - m c), bf16 P row into shared memory (128B swizzle)
            float rs = 0.f;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                tmem_ld32(t_lane + sb * 128 + cc * 32, v);
                tmem_wait_ld();
                const int kb = key0 + cc * 32;
                if (kb + 32 <= lim) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        v[i] = ex2_approx(fmaf(v[i], c, -mc));
                        rs += v[i];
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        v[i] = (kb + i < lim) ? ex2_approx(fmaf(v[i], c, -mc)) : 0.f;
                        rs += v[i];
                    }
                }
                // keys cc*32 .. cc*32+31 live in box cc/2, 16-byte chunks (cc%2)*4 .. +3
                uint8_t *box = prow + (cc >> 1) * (C::BQ * 128);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int chunk = (cc & 1) * 4 + q;
                    uint4 u;
                    u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
                    u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
                    u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
                    u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
                    *reinterpret_cast<uint4 *>(box + ((chunk ^ sw) << 4)) = u;
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&s_empty[sb]));
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(p_full));
            l_run = l_run * alpha + rs;
            m_run = m_new;
            // fold O_{j-1} (scale m_{j-1}) into o (scale m_{j-2})
            if (j >= 1) {
                const int ob = (j - 1) & 1;
#pragma unroll
                for (int cc = 0; cc < DH / 32; ++cc) {
                    tmem_ld32(t_lane + 256 + ob * 128 + cc * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[cc * 32 + i] = fmaf(o[cc * 32 + i], alpha_prev, v[i]);
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&o_empty[ob]));
            }
            alpha_prev = alpha;
        }
        if (ok && T > 0) {
            const int ob = (T - 1) & 1;
            if (mbar_wait(smem_u32(&o_full[ob]), ((T - 1) >> 1) & 1, abort_flag, p.err)) {
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < DH / 32; ++cc) {
                    tmem_ld32(t_lane + 256 + ob * 128 + cc * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[cc * 32 + i] = fmaf(o[cc * 32 + i], alpha_prev, v[i]);
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&o_empty[ob]));
                if (row < p.Mq) {
                    const float inv = 1.f / l_run;
                    bf16 *dst = p.out + ((size_t)b * p.Mq + row) * p.d + hh * DH;
#pragma unroll
                    for (int cc = 0; cc < DH / 32; ++cc) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = o[cc * 32 + i] * inv;
                        store_bf16x32(dst + cc * 32, v);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace qi21
