// Flash attention on tcgen05 tensor cores (BF16 mode):
//   o = softmax(q k^T / sqrt(Dh)) v over keys [0, limit(row)) of each query row,
// limit = kv_limit[row] (block-causal prefix extract, full recompute) or every
// one of the kv_len keys (cached target rows: the target is last, so they see
// the whole prefix cache and all target keys).
//
// One CTA per (item, head, 128 query rows); K and V tiles of 128 keys stream
// through two 2-stage TMA rings (128-byte swizzle, no multicast).
//   warp 0     : TMA producers: lane 0 loads Q once, then K_j (a K stage is
//                released as soon as its S MMA completes); lane 1 loads V_j (a
//                V stage is released when its PV MMA completes)
//   warp 1     : TMEM allocator + UMMA issuer:
//                S_j = Q K_j^T   (M 128, N 128, K Dh)  -> TMEM S[j % 2]
//                O  += P_j V_j   (M 128, N Dh, K 128)  -> TMEM O (accumulated across tiles)
//                P_j (bf16) is read from TMEM, V_j from shared memory as an
//                MN-major operand.
//   warps 2..9 : softmax, two threads per query row: each warp owns 16 TMEM
//                lanes (16 rows) and reads them with the 16x32bx2 shape, so
//                threads t and t+16 hold key columns 0..63 / 64..127 of the
//                same row and the matching halves of its O row; the halves
//                combine their row max by a shuffle. The row keeps a running
//                max m and only when a tile
//                raises it by more than 2^8 (in the exp2 domain) do the two
//                threads rescale their O halves in TMEM (after PV(j-1) has
//                landed) — otherwise P_j = exp2(S_j c - m c) <= 256 is formed
//                against the stale max, exactly as the final 1/l normalisation
//                expects. S_{j+1} and PV(j-1) run under softmax(j).
// TMEM columns: S0 [0,128), S1 [128,256), O [256,256+Dh), P0 [384,448),
// P1 [448,512) (P rows as bf16 pairs: key k of row r at lane r, column k/2).
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
    static constexpr int STAGES = 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
    // The dynamic shared-memory window is checked to start on a 1024-byte
    // boundary (the swizzled tiles need it), so no alignment slack is requested.
    static constexpr size_t SMEM = (size_t)OFF_BAR + 256;
    static constexpr int THREADS = 320;
    static constexpr int SOFTMAX_THREADS = 256;
};

// Rescale the O row only when the running max grows by more than this (log2 units).
constexpr float kRescaleLog2 = 8.0f;

template <int DH>
__global__ void __launch_bounds__(320, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, AttnParams p) {
    using namespace sm100;
    using C = AttnCfg<DH>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (smem_u32(smem_raw) & 1023) {           // never expected; refuse rather than overrun
        if (threadIdx.x == 0) raise_device_error(p.err, DEV_ERR_LAYOUT);
        return;
    }
    uint8_t *smem = smem_raw;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = bars + 1;      // [2]
    uint64_t *v_full = bars + 3;      // [2]
    uint64_t *k_empty = bars + 5;     // [2]  (S MMA of that K stage done)
    uint64_t *s_full = bars + 7;      // [2]
    uint64_t *s_empty = bars + 9;     // [2]
    uint64_t *p_full = bars + 11;     // [2]
    uint64_t *p_empty = bars + 13;    // [2]  (PV of that P buffer done)
    uint64_t *v_empty = bars + 15;    // [2]  (PV MMA of that V stage done)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 17);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *kv_end_s = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * C::BQ, hh = blockIdx.y, b = blockIdx.z;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(q_full), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&k_full[i]), 1);
            mbar_init(smem_u32(&v_full[i]), 1);
            mbar_init(smem_u32(&k_empty[i]), 1);
            mbar_init(smem_u32(&v_empty[i]), 1);
            mbar_init(smem_u32(&s_full[i]), 1);
            mbar_init(smem_u32(&s_empty[i]), C::SOFTMAX_THREADS);
            mbar_init(smem_u32(&p_full[i]), C::SOFTMAX_THREADS);
            mbar_init(smem_u32(&p_empty[i]), 1);
        }
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
    if (threadIdx.x >= 64 && threadIdx.x < 64 + C::BQ) {
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
        // ---------------------------------------------------------------- TMA producers
        // lane 0 streams K (a stage frees as soon as its S MMA is done, so K runs
        // two tiles ahead); lane 1 streams V (a stage frees after its PV MMA).
        if (lane == 0 && T > 0) {
            const uint32_t qb = smem_u32(q_full);
            mbar_arrive_expect_tx(qb, C::Q_BYTES);
            for (int x = 0; x < C::BOXES; ++x)
                tma_load_4d(smem_u32(smem + C::OFF_Q + x * (C::BQ * 128)), &tmQ, qb, hh * DH + x * 64,
                            b * p.Mq + q0, 0, 0);
            for (int j = 0; j < T; ++j) {
                const int s = j & 1;
                if (!mbar_wait(smem_u32(&k_empty[s]), ((j >> 1) & 1) ^ 1, abort_flag, p.err)) break;
                const uint32_t kb = smem_u32(&k_full[s]);
                mbar_arrive_expect_tx(kb, C::KV_BYTES);
                for (int x = 0; x < C::BOXES; ++x)
                    tma_load_4d(smem_u32(smem + C::OFF_K + s * C::KV_BYTES + x * (C::BK * 128)), &tmK, kb,
                                hh * DH + x * 64, j * C::BK, b, p.layer);
            }
        } else if (lane == 1 && T > 0) {
            for (int j = 0; j < T; ++j) {
                const int s = j & 1;
                if (!mbar_wait(smem_u32(&v_empty[s]), ((j >> 1) & 1) ^ 1, abort_flag, p.err)) break;
                const uint32_t vb = smem_u32(&v_full[s]);
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
            const uint32_t o_tmem = tmem_base + 256;
            bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag, p.err);
            auto issue_pv = [&](int i) -> bool {
                const int s = i & 1;
                if (!mbar_wait(smem_u32(&p_full[s]), (i >> 1) & 1, abort_flag, p.err)) return false;
                if (!mbar_wait(smem_u32(&v_full[s]), (i >> 1) & 1, abort_flag, p.err)) return false;
                tc_fence_after();
                const uint32_t p_tmem = tmem_base + 384 + s * 64;
                const uint32_t sv = smem_u32(smem + C::OFF_V + s * C::KV_BYTES);
#pragma unroll
                for (int k = 0; k < C::BK / 16; ++k) {
                    const uint64_t bdesc = sdesc_mnmajor_sw128(sv + k * 2048, C::BK * 128);
                    umma_f16_ts(o_tmem, p_tmem + k * 8, bdesc, idesc_o, (i > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(smem_u32(&p_empty[s]));
                umma_commit(smem_u32(&v_empty[s]));
                return true;
            };
            for (int j = 0; j < T && ok; ++j) {
                const int s = j & 1;
                if (!mbar_wait(smem_u32(&k_full[s]), (j >> 1) & 1, abort_flag, p.err)) break;
                if (!mbar_wait(smem_u32(&s_empty[s]), ((j >> 1) & 1) ^ 1, abort_flag, p.err)) break;
                tc_fence_after();
                const uint32_t sk = smem_u32(smem + C::OFF_K + s * C::KV_BYTES);
                const uint32_t d_tmem = tmem_base + s * 128;
#pragma unroll
                for (int k = 0; k < DH / 16; ++k) {
                    const uint32_t off = (k >> 2) * (C::BQ * 128) + (k & 3) * 32;
                    umma_f16(d_tmem, sdesc_kmajor_sw128(sq + off),
                             sdesc_kmajor_sw128(sk + (k >> 2) * (C::BK * 128) + (k & 3) * 32), idesc_s,
                             k > 0 ? 1u : 0u);
                }
                umma_commit(smem_u32(&s_full[s]));
                umma_commit(smem_u32(&k_empty[s]));
                if (j >= 1 && !issue_pv(j - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) issue_pv(T - 1);
        }
    } else {
        // ---------------------------------------------------------------- softmax warps (2..9)
        // Warp w owns 16 rows (TMEM lanes 32*(w%4) + 16*((w-2)/4) ..); thread t holds
        // row t%16, key half t/16 (keys 64h .. 64h+63 of S, O columns h*Dh/2 ..),
        // loaded with the 16x32bx2 shape, so the two halves of a row meet by shuffle.
        const int quad = warp & 3;
        const int sub = (warp - 2) >> 2;
        const int rr = lane & 15, half = lane >> 4;
        const int r = quad * 32 + sub * 16 + rr;          // row within the tile = TMEM lane
        const int row = q0 + r;
        int lim = p.kv_len;
        if (p.kv_limit && row < p.Mq) lim = min(p.kv_limit[row], p.kv_len);
        const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32 + sub * 16) << 16);
        const uint32_t t_o = t_lane + 256;
        const float c = p.scale_log2;
        float m_run = -INFINITY, l_half = 0.f;
        bool ok = true;
        float sv[64];
        // tcgen05.ld / tcgen05.st are warp-collective (.sync.aligned): every
        // decision that guards one is made uniform across the warp.
        auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, abort_flag, p.err) ? 1 : 0) != 0;
        };
        for (int j = 0; j < T && ok; ++j) {
            const int s = j & 1;
            if (!wait_all(&s_full[s], (j >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_ld16x2_32<64>(t_lane + s * 128, *reinterpret_cast<float(*)[32]>(&sv[0]));
            tmem_ld16x2_32<64>(t_lane + s * 128 + 32, *reinterpret_cast<float(*)[32]>(&sv[32]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(smem_u32(&s_empty[s]));
            const int key0 = j * C::BK + half * 64;
            if (key0 + 64 > lim) {
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (key0 + i >= lim) sv[i] = -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = sv[i];
#pragma unroll
            for (int i = 8; i < 64; ++i) m8[i & 7] = fmaxf(m8[i & 7], sv[i]);
            float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));      // the row's other half
            // per row: move the running max only when this tile raises it by more than 2^8
            const bool first = (m_run == -INFINITY);
            const bool grow = first || (mx - m_run) * c > kRescaleLog2;
            const float m_new = grow ? fmaxf(m_run, mx) : m_run;
            const float alpha = (grow && !first) ? ex2_approx((m_run - m_new) * c) : 1.f;
            if (__any_sync(0xffffffffu, grow && !first)) {
                // O holds PV(0..j-1) against the old max: the whole warp rescales its
                // O rows (alpha = 1 where the row's max did not move) once PV(j-1) landed
                if (!wait_all(&p_empty[(j - 1) & 1], ((j - 1) >> 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float ov[32];
#pragma unroll
                for (int cc = 0; cc < DH / 64; ++cc) {
                    tmem_ld16x2_32<DH / 2>(t_o + cc * 32, ov);
                    tmem_wait_ld();
                    uint32_t u[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(ov[i] * alpha);
                    tmem_st16x2_32<DH / 2>(t_o + cc * 32, u);
                }
                tmem_wait_st();
            }
            l_half *= alpha;
            m_run = m_new;
            const float mc = m_run * c;
            float s8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) s8[i] = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                sv[i] = ex2_approx(fmaf(sv[i], c, -mc));    // masked: exp2(-inf) = 0
                s8[i & 7] += sv[i];
            }
            l_half += ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
            // P buffer s is free once PV(j-2) has completed
            if (!wait_all(&p_empty[s], ((j >> 1) & 1) ^ 1)) {
                ok = false;
                break;
            }
            // this half's 64 keys -> 32 TMEM columns of P[s] (bf16 pairs, lower key in the low half)
            {
                uint32_t u[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) u[q] = pack_bf16x2(sv[2 * q], sv[2 * q + 1]);
                tmem_st16x2_32<32>(t_lane + 384 + s * 64, u);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&p_full[s]));
        }
        if (ok && T > 0) {
            const float l_row = l_half + __shfl_xor_sync(0xffffffffu, l_half, 16);
            if (wait_all(&p_empty[(T - 1) & 1], ((T - 1) >> 1) & 1)) {
                tc_fence_after();
                const float inv = 1.f / l_row;
                bf16 *dst = p.out + ((size_t)b * p.Mq + row) * p.d + hh * DH + half * (DH / 2);
                float ov[32];
#pragma unroll
                for (int cc = 0; cc < DH / 64; ++cc) {
                    tmem_ld16x2_32<DH / 2>(t_o + cc * 32, ov);   // every lane: the load is warp-collective
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] *= inv;
                    if (row < p.Mq) store_bf16x32(dst + cc * 32, ov);
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
