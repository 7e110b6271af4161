// Persistent warp-specialised tcgen05 GEMM with fused epilogues (BF16 mode).
//
//   D[r][n] = sum_k A[r][k] * W[n][k]      A: activations [R][K] bf16 (K-major)
//                                          W: weights [N][K] bf16 (K-major, [out][in])
// Tile 128 x 256 x 64, 4-stage TMA -> shared memory pipeline, fp32
// accumulators double-buffered in TMEM (2 x 256 columns), one CTA per SM.
//   warp 0      : TMA producer (one elected lane)
//   warp 1      : TMEM allocator + UMMA issuer (one lane)
//   warps 2..5  : epilogue; warp w reads TMEM lanes 32*(w%4) .. +31, i.e. one
//                 output row per thread, 32 columns per tcgen05.ld.
// Epilogues (the lab's [4A]/[5A] block):
//   EPI_QKV      per-head zero-centred RMSNorm (1 + w) of q and k, RoPE on the
//                adjacent pairs, q -> q buffer, k / v -> K/V rows of the cache
//   EPI_RESIDUAL h[r][n] += tanh(gate)[n] * D[r][n]   (fp32 residual stream)
//   EPI_SWIGLU   hid[r][j] = silu(D[r][j]) * D[r][F + j]   (gate and up halves
//                of one 256-column tile come from W_gate and W_up rows j0..j0+127)
//   EPI_STORE    out[r][n] = D[r][n] as fp32 through a TMA tensor store (img_in:
//                the residual stream's first value, h = x W_img_in^T)
#pragma once
#include "qi21_sm100.cuh"

namespace qi21 {

enum { EPI_QKV = 0, EPI_RESIDUAL = 1, EPI_SWIGLU = 2, EPI_STORE = 3 };

constexpr int TC_BM = 128, TC_BN = 256, TC_BK = 64;
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;          // 16 KB: a CTA's 128 rows of A per K block
constexpr int TC_THREADS = 192;
// EPI_RESIDUAL and EPI_STORE stage each epilogue warp's 32 x 32 fp32 box in
// shared memory (two buffers per warp) for the TMA reduce-add into the
// residual stream, or the TMA store.
constexpr int TC_RED_BUF = 32 * 32 * 4;
// staging boxes per epilogue warp: 2 for the residual (its GEMMs are bound by the
// MMAs), 6 for the store epilogue (img_in, K = 64: bound by the stores; each box
// waits for the TMA engine to read it before it is written again)
template <int EPI>
__host__ __device__ constexpr int tc_red_nbuf() {
    return EPI == EPI_STORE ? 6 : 2;
}
template <int EPI>
__host__ __device__ constexpr int tc_red_bytes() {
    return 4 * tc_red_nbuf<EPI>() * TC_RED_BUF;
}
template <int EPI>
__host__ __device__ constexpr bool tc_boxed_epilogue() {
    return EPI == EPI_RESIDUAL || EPI == EPI_STORE;
}

// Shared-memory pipeline of one CTA. PAIR = false: the CTA computes a 128 x 256
// tile alone and loads all 256 W rows of a K block. PAIR = true: two CTAs (a
// cluster) compute a 256 x 256 tile with cta_group::2 MMAs; each loads its own
// 128 rows of A and 128 of the 256 W rows, so a stage is 32 KB instead of 48 KB
// and the shared-memory and L2 traffic per MMA drop by a third.
template <int EPI, bool PAIR>
struct TcCfg {
    static constexpr int B_ROWS = PAIR ? 128 : 256;                 // W rows a CTA loads per K block
    static constexpr int B_BYTES = B_ROWS * TC_BK * 2;
    static constexpr int STAGE_BYTES = TC_A_BYTES + B_BYTES;
    static constexpr int STAGES = EPI == EPI_STORE ? 2 : (PAIR ? (tc_boxed_epilogue<EPI>() ? 5 : 6) : 4);
    static constexpr int TILE_ROWS = PAIR ? 256 : 128;              // output rows of a work unit
    static constexpr size_t SMEM =
        1024 + (size_t)STAGES * STAGE_BYTES + (tc_boxed_epilogue<EPI>() ? tc_red_bytes<EPI>() : 0) + 256;
};
template <int EPI, bool PAIR>
constexpr size_t tc_smem_bytes() {
    return TcCfg<EPI, PAIR>::SMEM;
}

struct GemmParams {
    int R;             // rows of A (tokens of all items)
    int K;             // reduction length
    int m_blocks;      // ceil(R / 128)
    int n_blocks;      // output tiles along N
    int ksplit;        // EPI_RESIDUAL: K slices per output tile, each reduce-added into h (1 otherwise)
    int sk_tiles;      // EPI_RESIDUAL with ksplit 1: the last sk_tiles tiles are shared stream-K style
    int group_m;       // row blocks per band of the tile order (0: all of them)
    int M, split;      // rows per item; rows m < split read the prefix modulation row
    // EPI_RESIDUAL
    float *h;
    int ldh;
    const float *g_lo, *g_hi;
    // EPI_SWIGLU
    bf16 *hid;
    int F;
    // EPI_QKV
    int d, Dh;
    const float *qn, *kn;
    float qk_eps;
    const float *cos_sin;
    bf16 *q_out, *k_base, *v_base;
    int64_t kv_bstride;
    int row_off;
    int layer;         // z coordinate of the stacked weight tensor maps
    uint32_t *err;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&p);
}

// out[box] += smem box, element-wise in L2 (2-D fp32 tensor map, 128B swizzle).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap *m, uint32_t src, int x, int y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
// out[box] = smem box (2-D fp32 tensor map, 128B swizzle); rows past the
// tensor's extent are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *m, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Store 32 fp32 values as bf16 (64 contiguous bytes, 16-byte aligned).
__device__ __forceinline__ void store_bf16x32(bf16 *dst, const float (&v)[32]) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 u;
        u.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
        u.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
        u.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
        u.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
        d4[i] = u;
    }
}

// Work unit -> (row block, column block, K slice). m fastest: CTAs running
// together share a weight tile while the activations stay in L2. With
// ksplit > 1 (residual epilogue only) a unit covers K blocks [kb0, kb1); its
// partial product is reduce-added into h like a whole tile's.
__device__ __forceinline__ void tile_coords(const GemmParams &p, int tile, int kblocks, int &m_blk, int &n_blk,
                                            int &kb0, int &kb1) {
    // K slice outermost; inside a slice, bands of group_m row blocks, and inside a
    // band the row block varies fastest, so the CTAs running together read a band
    // of A rows and a run of B rows instead of all of A.
    const int per_slice = p.m_blocks * p.n_blocks;
    const int ks = tile / per_slice;
    const int t = tile - ks * per_slice;
    const int gm = p.group_m > 0 ? p.group_m : p.m_blocks;
    const int band = t / (gm * p.n_blocks);
    const int m0 = band * gm;
    const int rows = min(gm, p.m_blocks - m0);
    const int local = t - band * gm * p.n_blocks;
    m_blk = m0 + local % rows;
    n_blk = local / rows;
    kb0 = (int)((int64_t)kblocks * ks / p.ksplit);
    kb1 = (int)((int64_t)kblocks * (ks + 1) / p.ksplit);
}

// The work of one CTA: first the data-parallel units blockIdx.x, +gridDim.x, ...
// (whole tiles, or K slices of them when ksplit > 1); then, when sk_tiles > 0
// (residual epilogue, ksplit 1), this CTA's equal contiguous share of the K
// blocks of the last sk_tiles tiles (stream-K: a share may start or end inside
// a tile; every piece is reduce-added into h like a K slice). The data-parallel
// units fill whole waves, so every CTA ends with the same number of K blocks.
struct WorkCursor {
    int unit;          // next data-parallel unit
    int64_t it, end;   // stream-K iterations [it, end) of this CTA
};

// `worker` / `workers`: this CTA (or CTA pair) and how many there are.
__device__ __forceinline__ void work_begin(const GemmParams &p, int kblocks, int worker, int workers, WorkCursor &c) {
    c.unit = worker;
    const int64_t W = (int64_t)p.sk_tiles * kblocks;
    c.it = W * worker / workers;
    c.end = W * (worker + 1) / workers;
}

__device__ __forceinline__ bool work_next(const GemmParams &p, int kblocks, int workers, WorkCursor &c, int &m_blk,
                                          int &n_blk, int &kb0, int &kb1) {
    const int dp_units = p.m_blocks * p.n_blocks * p.ksplit - p.sk_tiles;
    if (c.unit < dp_units) {
        tile_coords(p, c.unit, kblocks, m_blk, n_blk, kb0, kb1);
        c.unit += workers;
        return true;
    }
    if (c.it >= c.end) return false;
    const int tile = dp_units + (int)(c.it / kblocks);
    const int k0 = (int)(c.it % kblocks);
    const int64_t left = c.end - c.it;
    const int k1 = (left < (int64_t)(kblocks - k0)) ? k0 + (int)left : kblocks;
    int unused0, unused1;
    tile_coords(p, tile, kblocks, m_blk, n_blk, unused0, unused1);
    kb0 = k0;
    kb1 = k1;
    c.it += k1 - k0;
    return true;
}

template <int EPI, bool PAIR>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2, GemmParams p) {
    using namespace sm100;
    using Cfg = TcCfg<EPI, PAIR>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *stage_base = smem;
    uint8_t *red_base = smem + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(red_base + (tc_boxed_epilogue<EPI>() ? tc_red_bytes<EPI>() : 0));
    uint64_t *full = bars, *empty = bars + Cfg::STAGES, *tfull = bars + 2 * Cfg::STAGES, *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    static_assert((2 * Cfg::STAGES + 4) * 8 + 8 <= 256, "barrier region");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kblocks = p.K / TC_BK;
    // CTA pair: rank 0 (the leader) issues every MMA of the pair; each CTA owns
    // rows [rank * 128, rank * 128 + 128) of the 256-row tile.
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const int worker = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int workers = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    const bool mma_cta = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), PAIR ? 8 : 4);     // one arrival per epilogue warp of the tile
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        tma_prefetch_desc(&tmB1);
        if (EPI != EPI_SWIGLU) tma_prefetch_desc(&tmB2);
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_u32(tmem_slot), 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_slot), 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // the peer's barriers are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            WorkCursor wc;
            work_begin(p, kblocks, worker, workers, wc);
            int m_blk, n_blk, kb0, kb1;
            while (ok && work_next(p, kblocks, workers, wc, m_blk, n_blk, kb0, kb1)) {
                // this CTA's W rows of the tile: all 256 (single CTA) or half of them (pair)
                const CUtensorMap *b0 = &tmB0, *b1 = &tmB1;
                int rb0, rb1;
                if (EPI == EPI_SWIGLU) {
                    // columns 0..127 of the tile from W_gate, 128..255 from W_up, rows j0..j0+127
                    rb0 = rb1 = n_blk * 128;
                    if (PAIR && rank == 1) b0 = &tmB1;
                } else if (EPI == EPI_QKV) {
                    const int n0 = n_blk * TC_BN, part = n0 / p.d;
                    const CUtensorMap *bm = part == 0 ? &tmB0 : (part == 1 ? &tmB1 : &tmB2);
                    b0 = b1 = bm;
                    rb0 = n0 - part * p.d + (int)rank * 128;
                    rb1 = rb0 + 128;
                } else {
                    rb0 = n_blk * TC_BN + (int)rank * 128;
                    rb1 = rb0 + 128;
                }
                const int arow = m_blk * Cfg::TILE_ROWS + (int)rank * TC_BM;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = smem_u32(stage_base + (size_t)stage * Cfg::STAGE_BYTES);
                    const uint32_t sb = sa + TC_A_BYTES;
                    if constexpr (PAIR) {
                        // both CTAs' loads complete on the leader's full barrier
                        const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
                        if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full[stage]), 2 * Cfg::STAGE_BYTES);
                        tma_load_3d_pair(sa, &tmA, fb, kb * TC_BK, arow, 0);
                        tma_load_3d_pair(sb, b0, fb, kb * TC_BK, rb0, p.layer);
                    } else {
                        const uint32_t fb = smem_u32(&full[stage]);
                        mbar_arrive_expect_tx(fb, Cfg::STAGE_BYTES);
                        tma_load_3d(sa, &tmA, fb, kb * TC_BK, arow, 0);
                        tma_load_3d(sb, b0, fb, kb * TC_BK, rb0, p.layer);
                        tma_load_3d(sb + Cfg::B_BYTES / 2, b1, fb, kb * TC_BK, rb1, p.layer);
                    }
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- UMMA issuer (the leader CTA's)
        // The whole warp runs the schedule and one elected lane issues; the
        // operand descriptors are built once and advanced by adding to the
        // start-address field (16-byte units: 32 B per K=16 step).
        if (mma_cta) {
            constexpr uint32_t idesc = idesc_bf16_f32(Cfg::TILE_ROWS, TC_BN);
            constexpr uint32_t STAGE_UNITS = Cfg::STAGE_BYTES >> 4, A_UNITS = TC_A_BYTES >> 4;
            const uint64_t d0 = sdesc_kmajor_sw128(smem_u32(stage_base));
            const bool leader = elect_one();
            auto wait_warp = [&](uint64_t *bar, uint32_t parity) -> bool {
                return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, abort_flag, p.err) ? 1 : 0) != 0;
            };
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            WorkCursor wc;
            work_begin(p, kblocks, worker, workers, wc);
            int m_blk, n_blk, kb0, kb1;
            for (; ok && work_next(p, kblocks, workers, wc, m_blk, n_blk, kb0, kb1); ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!wait_warp(&tempty[acc], acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TC_BN);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_warp(&full[stage], phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (leader) {
                        const uint64_t da = d0 + (uint32_t)stage * STAGE_UNITS;
#pragma unroll
                        for (int k = 0; k < TC_BK / 16; ++k) {
                            if constexpr (PAIR)
                                umma_f16_pair(d_tmem, da + 2 * k, da + A_UNITS + 2 * k, idesc,
                                              (kb > kb0 || k > 0) ? 1u : 0u);
                            else
                                umma_f16(d_tmem, da + 2 * k, da + A_UNITS + 2 * k, idesc,
                                         (kb > kb0 || k > 0) ? 1u : 0u);
                        }
                        if constexpr (PAIR)
                            umma_commit_pair(smem_u32(&empty[stage]), 0x3);
                        else
                            umma_commit(smem_u32(&empty[stage]));
                    }
                    __syncwarp();
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (ok && leader) {
                    if constexpr (PAIR)
                        umma_commit_pair(smem_u32(&tfull[acc]), 0x3);
                    else
                        umma_commit(smem_u32(&tfull[acc]));
                }
                __syncwarp();
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue (warps 2..5)
        const int quad = warp & 3;
        const int row_in_tile = (int)rank * TC_BM + quad * 32 + lane;
        int it = 0;
        int red_count = 0;   // boxed epilogues: reduce-add / store boxes issued by this warp
        WorkCursor wc;
        work_begin(p, kblocks, worker, workers, wc);
        int m_blk, n_blk, kb0, kb1;
        for (; work_next(p, kblocks, workers, wc, m_blk, n_blk, kb0, kb1); ++it) {
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            // warp-uniform: the tcgen05.ld below is warp-collective
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.err) ? 1 : 0))
                break;
            tc_fence_after();
            // this warp is done with the accumulator: tell the leader's MMA warp
            auto release_acc = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR)
                        mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
                    else
                        mbar_arrive(smem_u32(&tempty[acc]));
                }
            };
            const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * TC_BN);
            const int r = m_blk * Cfg::TILE_ROWS + row_in_tile;
            const bool live = r < p.R;
            const int m = live ? r % p.M : 0;
            const int b = live ? r / p.M : 0;
            float v[32];
            if (tc_boxed_epilogue<EPI>()) {
                // EPI_RESIDUAL: h[r][n] += tanh(gate)[n] * acc; EPI_STORE: out[r][n] = acc.
                // Each warp writes its 32 rows x 32 columns into a swizzled shared box
                // and one lane reduce-adds (or stores) the box.
                const int n0 = n_blk * TC_BN;
                const float *g = EPI == EPI_RESIDUAL ? (m < p.split ? p.g_lo : p.g_hi) + n0 : nullptr;
                constexpr int NBUF = tc_red_nbuf<EPI>();
                uint8_t *stg = red_base + (size_t)(warp - 2) * NBUF * TC_RED_BUF;
                const int sw = lane & 7;
                const int box_row = m_blk * Cfg::TILE_ROWS + (int)rank * TC_BM + quad * 32;
#pragma unroll 1
                for (int cc = 0; cc < TC_BN / 32; ++cc, ++red_count) {
                    tmem_ld32(t_row + cc * 32, v);
                    tmem_wait_ld();
                    if (cc == TC_BN / 32 - 1) release_acc();
                    if (EPI == EPI_RESIDUAL && live) {
                        const float4 *g4 = reinterpret_cast<const float4 *>(g + cc * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 gv = g4[i];
                            v[4 * i + 0] *= gv.x;
                            v[4 * i + 1] *= gv.y;
                            v[4 * i + 2] *= gv.z;
                            v[4 * i + 3] *= gv.w;
                        }
                    }
                    uint8_t *buf = stg + (red_count % NBUF) * TC_RED_BUF;
                    if (red_count >= NBUF) {
                        if (lane == 0) bulk_wait_group_read<NBUF - 1>();   // the copy that used `buf` has read it
                        __syncwarp();
                    }
                    uint8_t *rowp = buf + lane * 128;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4 *>(rowp + ((q ^ sw) << 4)) =
                            make_float4(v[4 * q + 0], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    fence_proxy_async_shared();
                    __syncwarp();
                    if (lane == 0) {
                        if (EPI == EPI_RESIDUAL)
                            tma_reduce_add_2d(&tmB2, smem_u32(buf), n0 + cc * 32, box_row);
                        else
                            tma_store_2d(&tmB2, smem_u32(buf), n0 + cc * 32, box_row);
                        bulk_commit_group();
                    }
                }
                continue;   // accumulator already released
            } else if (EPI == EPI_SWIGLU) {
                const int j0 = n_blk * 128;
                float u[32];
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    tmem_ld32(t_row + cc * 32, v);
                    tmem_ld32(t_row + 128 + cc * 32, u);
                    tmem_wait_ld();
                    if (live) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = v[i] / (1.0f + __expf(-v[i])) * u[i];
                        store_bf16x32(p.hid + (size_t)r * p.F + j0 + cc * 32, v);
                    }
                }
            } else {  // EPI_QKV
                const int n0 = n_blk * TC_BN, part = n0 / p.d, c0 = n0 - part * p.d;
                const int nch = p.Dh / 32;
                if (part == 2) {
                    bf16 *dst = p.v_base + (size_t)b * p.kv_bstride + (size_t)(p.row_off + m) * p.d + c0;
#pragma unroll 1
                    for (int cc = 0; cc < TC_BN / 32; ++cc) {
                        tmem_ld32(t_row + cc * 32, v);
                        tmem_wait_ld();
                        if (live) store_bf16x32(dst + cc * 32, v);
                    }
                } else {
                    const float *wn = part == 0 ? p.qn : p.kn;
                    bf16 *dst_row = part == 0 ? p.q_out + (size_t)r * p.d
                                              : p.k_base + (size_t)b * p.kv_bstride + (size_t)(p.row_off + m) * p.d;
                    const float *cs_row = p.cos_sin + (size_t)m * p.Dh;   // [Dh/2][2] floats = Dh floats
#pragma unroll 1
                    for (int hh = 0; hh < TC_BN / p.Dh; ++hh) {
                        float ss = 0.f;
#pragma unroll 1
                        for (int cc = 0; cc < nch; ++cc) {
                            tmem_ld32(t_row + hh * p.Dh + cc * 32, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
                        }
                        const float inv = rsqrtf(ss / (float)p.Dh + p.qk_eps);
#pragma unroll 1
                        for (int cc = 0; cc < nch; ++cc) {
                            tmem_ld32(t_row + hh * p.Dh + cc * 32, v);
                            tmem_wait_ld();
                            if (live) {
                                const float4 *w4 = reinterpret_cast<const float4 *>(wn + cc * 32);
                                const float4 *cs4 = reinterpret_cast<const float4 *>(cs_row + cc * 32);
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const float4 w = w4[i];
                                    const float4 cs = cs4[i];   // (cos, sin) of two pairs
                                    const float y0 = v[4 * i + 0] * inv * (1.f + w.x);
                                    const float y1 = v[4 * i + 1] * inv * (1.f + w.y);
                                    const float y2 = v[4 * i + 2] * inv * (1.f + w.z);
                                    const float y3 = v[4 * i + 3] * inv * (1.f + w.w);
                                    v[4 * i + 0] = y0 * cs.x - y1 * cs.y;
                                    v[4 * i + 1] = y0 * cs.y + y1 * cs.x;
                                    v[4 * i + 2] = y2 * cs.z - y3 * cs.w;
                                    v[4 * i + 3] = y2 * cs.w + y3 * cs.z;
                                }
                                store_bf16x32(dst_row + c0 + hh * p.Dh + cc * 32, v);
                            }
                        }
                    }
                }
            }
            release_acc();
        }
        if (tc_boxed_epilogue<EPI>() && lane == 0) bulk_wait_group0();
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // neither CTA frees the pair's TMEM while the other still uses it
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR)
            tmem_dealloc_pair(tmem_base, 512);
        else
            tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace qi21
