// Flash attention on tcgen05 tensor cores (BF16 mode):
//   o = softmax(q k^T / sqrt(Dh)) v over keys [0, limit(row)) of each query row,
// limit = kv_limit[row] (block-causal prefix extract, full recompute) or every
// one of the kv_len keys (cached target rows: the target is last, so they see
// the whole prefix cache and all target keys).
//
// One CTA per (item, head, 128 query rows). The CTA's T key tiles (128 keys
// each) are split into two halves, A = tiles [0, TA) and B = tiles [TA, T),
// TA = ceil(T/2). Each half has its own S and O accumulators in TMEM and its
// own softmax warpgroup, so the single MMA issuer alternates between them:
// while half A's softmax turns S_A into P_A, the tensor pipe runs half B's PV
// and next S, and the other way round. Each half keeps its own running max m
// and row sum l; the epilogue merges the two partial results,
//   o = (2^{(m_A-m)c} O_A + 2^{(m_B-m)c} O_B) / (2^{(m_A-m)c} l_A + 2^{(m_B-m)c} l_B),
// m = max(m_A, m_B) — the standard combination of two softmax partials over
// disjoint key sets.
//   warp 0     : TMA producers: lane 0 loads Q once, then the K tiles, lane 1
//                the V tiles, both in the order A0 B0 A1 B1 ... in which the
//                MMAs consume them (2-stage rings, 128-byte swizzle, no multicast)
//   warp 1     : TMEM allocator + UMMA issuer (warp-uniform schedule, one elected lane issues):
//                S_X = Q K^T   (M 128, N 128, K Dh)  -> TMEM S_X
//                O_X += P_X V  (M 128, N Dh, K 128)  -> TMEM O_X, P_X read from
//                TMEM, V from shared memory as an MN-major operand
//   warps 2..5 : softmax of half A, one thread per query row (= TMEM lane)
//   warps 6..9 : softmax of half B
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+Dh), O_B [256+Dh,256+2Dh).
// P_X (bf16 pairs: key k of row r at lane r, column k/2) overwrites the first 64
// columns of S_X after the softmax has read all of S_X into registers. The next
// S_X MMA is issued after the PV MMA that reads P_X; the tcgen05.mma operations
// of one issuing thread execute in issue order, so that PV reads P_X before the
// next S_X overwrites it. A commit tracks every earlier MMA of the thread, so
// when S_X(j) is complete, PV_X(j-1) is too: the softmax may then rescale O_X
// and write P_X(j) without a further wait. The softmax signals P_X(j) in two
// parts (keys 0..63, then 64..127; any O rescale before the first), and the MMA
// warp issues the first half of PV_X(j) on the first signal, so it runs while
// the second half of the exponentials is computed.
// The running max of a row moves only when a tile raises it by more than 2^8
// (exp2 domain); otherwise P = exp2(S c - m c) <= 256 is formed against the
// stale max, which the final 1/l normalisation absorbs.
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
    // Shared-prefix cache (one prefix for every item): key tiles [0, shared_tiles)
    // are prefix rows t*BK (keys >= prefix_len masked), the rest item b's target
    // rows tgt_row0 + b*tgt_len + (t - shared_tiles)*BK (keys >= tgt_len masked).
    // shared_tiles == 0: every item's keys are rows [0, kv_len) of its own block.
    int shared_tiles, prefix_len, tgt_len, tgt_row0;
};

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed pairs of fp32 (sm_100a f32x2 arithmetic: one instruction for two lanes).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x for a pair on the FMA pipe: x = n + f, n = rint(x), f in [-1/2, 1/2];
// 2^f from a cubic with constant term 1 (least-squares relative-error fit on
// [-1/2, 1/2], max relative error 1.1e-4; the coefficients are printed by
// exp2_poly_fit.py beside this file; P is rounded to bf16 afterwards, relative
// step 2^-8) and 2^n added to the exponent field. Inputs are clamped
// at -127, where f = 0 and the result is exactly +0 (masked keys: -inf).
__device__ __forceinline__ void ex2_poly2(float x0, float x1, float &e0, float &e1) {
    const uint64_t x = f2_pack(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
    const uint64_t magic = f2_pack(12582912.f, 12582912.f);   // 1.5 * 2^23: t's low bits hold rint(x)
    const uint64_t t = f2_add(x, magic);
    const uint64_t f = f2_sub(x, f2_sub(t, magic));
    uint64_t q = f2_fma(f2_pack(0.054592825f, 0.054592825f), f, f2_pack(0.24221784f, 0.24221784f));
    q = f2_fma(q, f, f2_pack(0.6933686f, 0.6933686f));
    q = f2_fma(q, f, f2_pack(1.0f, 1.0f));
    float p0, p1, t0, t1;
    f2_unpack(q, p0, p1);
    f2_unpack(t, t0, t1);
    e0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
    e1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
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

// Named barrier over the 256 softmax threads (id 1; id 0 is __syncthreads).
__device__ __forceinline__ void softmax_bar_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

static_assert(QI21_ATTN_KEY_TILE == 128, "the shared-prefix padding is the attention key tile");

template <int DH>
struct AttnCfg {
    static constexpr int BQ = 128, BK = 128;
    static constexpr int BOXES = DH / 64;                  // 64-element (128-byte) swizzle boxes per row
    static constexpr int Q_BYTES = BQ * DH * 2;
    static constexpr int KV_BYTES = BK * DH * 2;           // one K or V tile
    static constexpr int SK = 2, SV = 2;                   // K and V ring stages
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + SK * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + SV * KV_BYTES;
    static constexpr int OFF_STATS = OFF_BAR + 256;        // [2 halves][m, l][128 rows] floats
    // The dynamic shared-memory window is checked to start on a 1024-byte
    // boundary (the swizzled tiles need it), so no alignment slack is requested.
    static constexpr size_t SMEM = (size_t)OFF_STATS + 2 * 2 * BQ * 4;
    static constexpr int THREADS = 320;                    // warps: 0 loads, 1 MMA, 2..9 softmax
    static constexpr int HALF_THREADS = 128;               // softmax threads of one half
};

// Rescale the O row only when the running max grows by more than this (log2 units).
constexpr float kRescaleLog2 = 8.0f;

// Every kPolyEvery-th pair of exponentials of a row runs on the FMA pipe
// (ex2_poly2), the rest on the MUFU unit, which would otherwise take as long as
// the MMAs per key tile. Same-GPU A/B on the single-block workload (attention
// time over the gate/up GEMM's, interleaved runs): every 8th pair -6 %, every
// 4th -5 %, every 2nd +6 %, against the scalar MUFU-only softmax.
constexpr int kPolyEvery = 8;

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
    uint64_t *k_full = q_full + 1;     // [SK] ring stages
    uint64_t *k_empty = k_full + C::SK;   // [SK] (the S MMA reading that stage is done)
    uint64_t *v_full = k_empty + C::SK;   // [SV]
    uint64_t *v_empty = v_full + C::SV;   // [SV] (the PV MMA reading that stage is done)
    uint64_t *s_full = v_empty + C::SV;   // [2 halves]
    uint64_t *p_full = s_full + 2;        // [half][part]: softmax wrote P (keys 64*part ..) and finished with O
    uint64_t *o_full = p_full + 4;        // every MMA done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(o_full + 1);
    static_assert((1 + 2 * C::SK + 2 * C::SV + 5) * 8 + 16 <= 256, "barrier region");
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *kv_end_s = reinterpret_cast<int *>(tmem_slot + 2);
    float *stats = reinterpret_cast<float *>(smem + C::OFF_STATS);   // [half][m | l][row]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * C::BQ, hh = blockIdx.y, b = blockIdx.z;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(q_full), 1);
        for (int i = 0; i < C::SK; ++i) {
            mbar_init(smem_u32(&k_full[i]), 1);
            mbar_init(smem_u32(&k_empty[i]), 1);
        }
        for (int i = 0; i < C::SV; ++i) {
            mbar_init(smem_u32(&v_full[i]), 1);
            mbar_init(smem_u32(&v_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&s_full[i]), 1);
            mbar_init(smem_u32(&p_full[2 * i]), C::HALF_THREADS);
            mbar_init(smem_u32(&p_full[2 * i + 1]), C::HALF_THREADS);
        }
        mbar_init(smem_u32(o_full), 1);
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
    pdl_launch_dependents();
    pdl_wait();
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
    const int T = p.shared_tiles > 0 ? p.shared_tiles + (p.tgt_len + C::BK - 1) / C::BK
                                     : (kv_end + C::BK - 1) / C::BK;
    const int TA = (T + 1) >> 1, TB = T >> 1;     // tiles of half A and half B
    // row and item coordinates of key tile t in the K/V tensor maps
    auto tile_row = [&](int t) -> int {
        if (p.shared_tiles == 0) return t * C::BK;
        return t < p.shared_tiles ? t * C::BK : p.tgt_row0 + b * p.tgt_len + (t - p.shared_tiles) * C::BK;
    };
    const int kv_item = p.shared_tiles > 0 ? 0 : b;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producers
        // Load n of either ring is key tile A(n/2) for even n, B(n/2) for odd n.
        if (lane == 0 && T > 0) {
            const uint32_t qb = smem_u32(q_full);
            mbar_arrive_expect_tx(qb, C::Q_BYTES);
            for (int x = 0; x < C::BOXES; ++x)
                tma_load_4d(smem_u32(smem + C::OFF_Q + x * (C::BQ * 128)), &tmQ, qb, hh * DH + x * 64,
                            b * p.Mq + q0, 0, 0);
            for (int n = 0; n < T; ++n) {
                const int s = n % C::SK, tile = (n & 1) ? TA + (n >> 1) : (n >> 1);
                if (!mbar_wait(smem_u32(&k_empty[s]), ((n / C::SK) & 1) ^ 1, abort_flag, p.err)) break;
                const uint32_t kb = smem_u32(&k_full[s]);
                mbar_arrive_expect_tx(kb, C::KV_BYTES);
                for (int x = 0; x < C::BOXES; ++x)
                    tma_load_4d(smem_u32(smem + C::OFF_K + s * C::KV_BYTES + x * (C::BK * 128)), &tmK, kb,
                                hh * DH + x * 64, tile_row(tile), kv_item, p.layer);
            }
        } else if (lane == 1 && T > 0) {
            for (int n = 0; n < T; ++n) {
                const int s = n % C::SV, tile = (n & 1) ? TA + (n >> 1) : (n >> 1);
                if (!mbar_wait(smem_u32(&v_empty[s]), ((n / C::SV) & 1) ^ 1, abort_flag, p.err)) break;
                const uint32_t vb = smem_u32(&v_full[s]);
                mbar_arrive_expect_tx(vb, C::KV_BYTES);
                for (int x = 0; x < C::BOXES; ++x)
                    tma_load_4d(smem_u32(smem + C::OFF_V + s * C::KV_BYTES + x * (C::BK * 128)), &tmV, vb,
                                hh * DH + x * 64, tile_row(tile), kv_item, p.layer);
            }
        }
    } else if (warp == 1) {
        if (T > 0) {
            // ------------------------------------------------------------ UMMA issuer
            // order: S_A0 S_B0 | PV_A0 S_A1 PV_B0 S_B1 | PV_A1 S_A2 PV_B1 S_B2 | ...
            // The whole warp runs the schedule (its values stay warp-uniform) and one
            // elected lane issues each group of MMAs. Descriptors are built once; a
            // K=16 step inside a 64-element swizzle box adds 32 B (2 units of the
            // start-address field), a new box adds rows * 128 B, a new V K-step 2 KB.
            constexpr uint32_t idesc_s = idesc_bf16_f32(C::BQ, C::BK);
            constexpr uint32_t idesc_o = idesc_bf16_f32(C::BQ, DH, true);
            constexpr uint32_t BOX_UNITS = (C::BK * 128) >> 4;     // Q (BQ == BK) and K boxes
            constexpr uint32_t KV_UNITS = C::KV_BYTES >> 4;
            const uint64_t dq0 = sdesc_kmajor_sw128(smem_u32(smem + C::OFF_Q));
            const uint64_t dk0 = sdesc_kmajor_sw128(smem_u32(smem + C::OFF_K));
            const uint64_t dv0 = sdesc_mnmajor_sw128(smem_u32(smem + C::OFF_V), C::BK * 128);
            const bool leader = elect_one();
            auto wait_warp = [&](uint64_t *bar, uint32_t parity) -> bool {
                return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, abort_flag, p.err) ? 1 : 0) != 0;
            };
            int nk = 0, nv = 0;                      // loads consumed from the K and V rings
            auto issue_s = [&](int h) -> bool {
                const int s = nk % C::SK;
                if (!wait_warp(&k_full[s], (nk / C::SK) & 1)) return false;
                tc_fence_after();
                if (leader) {
                    const uint64_t dk = dk0 + s * KV_UNITS;
#pragma unroll
                    for (int k = 0; k < DH / 16; ++k) {
                        const uint32_t off = (k >> 2) * BOX_UNITS + (k & 3) * 2;
                        umma_f16(tmem_base + h * 128, dq0 + off, dk + off, idesc_s, k > 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&s_full[h]));
                    umma_commit(smem_u32(&k_empty[s]));
                }
                __syncwarp();
                ++nk;
                return true;
            };
            auto issue_pv = [&](int h, int j) -> bool {
                if (!wait_warp(&p_full[2 * h], j & 1)) return false;
                const int s = nv % C::SV;
                if (!wait_warp(&v_full[s], (nv / C::SV) & 1)) return false;
                tc_fence_after();
                // keys 0..63 of P as soon as they are written, keys 64..127 after the
                // second signal: the first half of PV runs under the rest of the softmax
                const uint64_t dv = dv0 + s * KV_UNITS;
                constexpr int KSTEPS = C::BK / 16;
                if (leader) {
#pragma unroll
                    for (int k = 0; k < KSTEPS / 2; ++k)
                        umma_f16_ts(tmem_base + 256 + h * DH, tmem_base + h * 128 + k * 8, dv + k * 128, idesc_o,
                                    (j > 0 || k > 0) ? 1u : 0u);
                }
                __syncwarp();
                if (!wait_warp(&p_full[2 * h + 1], j & 1)) return false;
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int k = KSTEPS / 2; k < KSTEPS; ++k)
                        umma_f16_ts(tmem_base + 256 + h * DH, tmem_base + h * 128 + k * 8, dv + k * 128, idesc_o,
                                    1u);
                    umma_commit(smem_u32(&v_empty[s]));
                }
                __syncwarp();
                ++nv;
                return true;
            };
            bool ok = wait_warp(q_full, 0);
            ok = ok && issue_s(0);
            if (TB > 0) ok = ok && issue_s(1);
            for (int j = 0; j < TA && ok; ++j) {
                ok = issue_pv(0, j);
                if (ok && j + 1 < TA) ok = issue_s(0);
                if (ok && j < TB) {
                    ok = issue_pv(1, j);
                    if (ok && j + 1 < TB) ok = issue_s(1);
                }
            }
            if (ok && leader) umma_commit(smem_u32(o_full));
            __syncwarp();
        }
    } else {
        // ---------------------------------------------------------------- softmax warps (2..9)
        const int h = (warp - 2) >> 2;                 // half: 0 = A (warps 2..5), 1 = B (warps 6..9)
        const int quad = warp & 3;                     // the TMEM lane quadrant this warp may access
        const int r = quad * 32 + lane;                // row within the tile = TMEM lane
        const int row = q0 + r;
        int lim = p.kv_len;
        if (p.kv_limit && row < p.Mq) lim = min(p.kv_limit[row], p.kv_len);
        const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
        const uint32_t t_s = t_lane + h * 128;         // S_h, later P_h in its first 64 columns
        const uint32_t t_o = t_lane + 256 + h * DH;    // O_h
        const int nt = h ? TB : TA, tile0 = h ? TA : 0;
        const float c = p.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        // tcgen05.ld / tcgen05.st are warp-collective (.sync.aligned): every
        // decision that guards one is made uniform across the warp.
        auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, abort_flag, p.err) ? 1 : 0) != 0;
        };
        for (int j = 0; j < nt && ok; ++j) {
            if (!wait_all(&s_full[h], j & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[4][32];                          // S row: key 32a+b in sv[a][b]
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tmem_ld32(t_s + cc * 32, sv[cc]);
            tmem_wait_ld();
            // keys of this tile and the first masked one
            const int t = tile0 + j;
            int key0 = t * C::BK, klim = lim;
            if (p.shared_tiles > 0) {
                if (t < p.shared_tiles) {
                    klim = min(lim, p.prefix_len);
                } else {
                    key0 = (t - p.shared_tiles) * C::BK;
                    klim = p.tgt_len;
                }
            }
            if (key0 + C::BK > klim) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (key0 + i >= klim) sv[i >> 5][i & 31] = -INFINITY;
            }
            // row max: three-input max over pairs, four independent chains
            float m4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) m4[i] = fmaxf(sv[0][2 * i], sv[0][2 * i + 1]);
#pragma unroll
            for (int i = 8; i < 128; i += 2) m4[(i >> 1) & 3] = fmax3(m4[(i >> 1) & 3], sv[i >> 5][i & 31],
                                                                      sv[i >> 5][(i + 1) & 31]);
            const float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
            // move the running max only when this tile raises it by more than 2^8
            const bool first = (m_run == -INFINITY);
            const bool grow = first || (mx - m_run) * c > kRescaleLog2;
            const float m_new = grow ? fmaxf(m_run, mx) : m_run;
            const float alpha = (grow && !first) ? ex2_approx((m_run - m_new) * c) : 1.f;
            l_run *= alpha;
            m_run = m_new;
            // a row with no allowed key so far (half B past its limit) keeps m = -inf: P = 0
            const float mc = m_run == -INFINITY ? 0.f : m_run * c;
            // row sum in packed pairs (f32x2 adds), four independent chains
            uint64_t s4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) s4[i] = 0ull;      // pairs of +0.f
            const uint64_t c2 = f2_pack(c, c), nmc2 = f2_pack(-mc, -mc);
            // P ready for the PV MMA, in two parts: keys 0..63, then 64..127
            auto signal_p = [&](int part) {
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(smem_u32(&p_full[2 * h + part]));
            };
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t u[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    float x0, x1, e0, e1;     // x = S c - m c, one f32x2 FMA for the pair (masked: -inf -> 0)
                    f2_unpack(f2_fma(f2_pack(sv[cc][2 * q], sv[cc][2 * q + 1]), c2, nmc2), x0, x1);
                    if ((cc * 16 + q) % kPolyEvery == kPolyEvery - 1) {
                        ex2_poly2(x0, x1, e0, e1);
                    } else {
                        e0 = ex2_approx(x0);
                        e1 = ex2_approx(x1);
                    }
                    s4[q & 3] = f2_add(s4[q & 3], f2_pack(e0, e1));
                    u[q] = pack_bf16x2(e0, e1);
                }
                tmem_st16(t_s + cc * 16, u);               // P_h: keys 32cc .. 32cc+31
                if (cc == 1) {
                    // O rescale (rare) before the first P signal, so that PV_h(j) sees the
                    // rescaled O. O_h holds PV_h(0..j-1) against the old max (complete: S_h(j)
                    // was issued after PV_h(j-1)); alpha = 1 on rows whose max did not move.
                    if (__any_sync(0xffffffffu, grow && !first)) {
                        float ov[32];
#pragma unroll
                        for (int oc = 0; oc < DH / 32; ++oc) {
                            tmem_ld32(t_o + oc * 32, ov);
                            tmem_wait_ld();
                            uint32_t w32[32];
#pragma unroll
                            for (int i = 0; i < 32; ++i) w32[i] = __float_as_uint(ov[i] * alpha);
                            tmem_st32(t_o + oc * 32, w32);
                        }
                    }
                    signal_p(0);
                }
            }
            signal_p(1);
            const uint64_t s2 = f2_add(f2_add(s4[0], s4[1]), f2_add(s4[2], s4[3]));
            float sa, sb;
            f2_unpack(s2, sa, sb);
            l_run += sa + sb;
        }
        // merge the halves: each publishes its (m, l) per row; half h then writes
        // output columns [h Dh/2, (h+1) Dh/2) of its rows from O_A and O_B
        stats[(2 * h + 0) * C::BQ + r] = m_run;
        stats[(2 * h + 1) * C::BQ + r] = l_run;
        softmax_bar_sync();
        if (ok && T > 0 && wait_all(o_full, 0)) {
            tc_fence_after();
            const float mA = stats[0 * C::BQ + r], lA = stats[1 * C::BQ + r];
            const float mB = stats[2 * C::BQ + r], lB = stats[3 * C::BQ + r];
            float m = fmaxf(mA, mB);
            if (m == -INFINITY) m = 0.f;
            const float wA = ex2_approx((mA - m) * c);
            const float wB = TB > 0 ? ex2_approx((mB - m) * c) : 0.f;
            const float inv = 1.f / (lA * wA + lB * wB);
            const float fA = wA * inv, fB = wB * inv;
            bf16 *dst = p.out + ((size_t)b * p.Mq + row) * p.d + hh * DH + h * (DH / 2);
#pragma unroll
            for (int cc = 0; cc < DH / 64; ++cc) {
                const int col = h * (DH / 2) + cc * 32;
                float oa[32], ob[32];
                tmem_ld32(t_lane + 256 + col, oa);            // every lane: the loads are warp-collective
                if (TB > 0) tmem_ld32(t_lane + 256 + DH + col, ob);
                tmem_wait_ld();
                if (TB > 0) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) oa[i] = fmaf(fA, oa[i], fB * ob[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) oa[i] *= fA;
                }
                if (row < p.Mq) store_bf16x32(dst + cc * 32, oa);
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
