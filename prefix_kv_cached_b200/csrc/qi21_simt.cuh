// CUDA-core kernels: the memory-bound steps shared by both modes (modulated
// LayerNorm, img_in, final AdaLN + proj_out, Euler, modulation GEMVs) and the
// unfused fp32 path (GEMM, QK-norm/RoPE scatter, gated residual, SwiGLU,
// attention) that the F32 mode runs for parity with the fp64 oracle.
#pragma once
#include "qi21_common.cuh"

namespace qi21 {

// ---------------------------------------------------------------------------
// tanh of the two gate chunks of the prefix and target modulation rows.
// Chunk order [scale1, gate1, scale2, gate2] (3B page §1) or, with shifts,
// [shift1, scale1, gate1, shift2, scale2, gate2] (lab [3B]).
// gates = [tanh g1 prefix | tanh g1 target | tanh g2 prefix | tanh g2 target].
// ---------------------------------------------------------------------------
static __global__ void k_prep_gates(const float *__restrict__ mod_lo, const float *__restrict__ mod_hi, int d,
                             int use_shift, float *__restrict__ gates) {
    pdl_launch_dependents();
    pdl_wait();
    const int g1 = use_shift ? 2 : 1, g2 = use_shift ? 5 : 3;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < d; c += gridDim.x * blockDim.x) {
        gates[0 * d + c] = tanhf(mod_lo[g1 * d + c]);
        gates[1 * d + c] = tanhf(mod_hi[g1 * d + c]);
        gates[2 * d + c] = tanhf(mod_lo[g2 * d + c]);
        gates[3 * d + c] = tanhf(mod_hi[g2 * d + c]);
    }
}

// ---------------------------------------------------------------------------
// Modulated LayerNorm: out = LN(h) * (1 + scale) (+ shift), one row per block.
// Row r is token m = r % M of its item; m < split reads the prefix row (lo),
// otherwise the target row (hi) — the per-token row selection of the 3B page.
// Two-pass mean/variance in fp32 over a register copy of the row.
// ---------------------------------------------------------------------------
template <typename T, int VPT>
__global__ void __launch_bounds__(256) k_modln_vec(const float *__restrict__ h, T *__restrict__ out, int d, int M,
                                                   int split, const float *__restrict__ scale_lo,
                                                   const float *__restrict__ scale_hi,
                                                   const float *__restrict__ shift_lo,
                                                   const float *__restrict__ shift_hi, float eps) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ float red[32];
    const int r = blockIdx.x;
    const int m = r % M;
    const float *sc = m < split ? scale_lo : scale_hi;
    const float *sh = m < split ? shift_lo : shift_hi;
    const float4 *x4 = reinterpret_cast<const float4 *>(h + (size_t)r * d);
    const int n4 = d >> 2;
    float4 v[VPT];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int c4 = threadIdx.x + i * 256;
        v[i] = c4 < n4 ? x4[c4] : make_float4(0.f, 0.f, 0.f, 0.f);
        s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
    const float mean = block_sum(s, red) / d;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int c4 = threadIdx.x + i * 256;
        if (c4 < n4) {
            const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, e = v[i].w - mean;
            q += (a * a + b * b) + (c * c + e * e);
        }
    }
    const float var = block_sum(q, red) / d;
    const float rstd = 1.0f / sqrtf(var + eps);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int c4 = threadIdx.x + i * 256;
        if (c4 < n4) {
            const float4 s4 = reinterpret_cast<const float4 *>(sc)[c4];
            float4 b4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (sh) b4 = reinterpret_cast<const float4 *>(sh)[c4];
            float y0 = (v[i].x - mean) * rstd * (1.f + s4.x) + b4.x;
            float y1 = (v[i].y - mean) * rstd * (1.f + s4.y) + b4.y;
            float y2 = (v[i].z - mean) * rstd * (1.f + s4.z) + b4.z;
            float y3 = (v[i].w - mean) * rstd * (1.f + s4.w) + b4.w;
            T *o = out + (size_t)r * d + 4 * c4;
            if constexpr (sizeof(T) == 2) {
                __nv_bfloat162 p0 = __floats2bfloat162_rn(y0, y1), p1 = __floats2bfloat162_rn(y2, y3);
                uint2 pk;
                pk.x = *reinterpret_cast<uint32_t *>(&p0);
                pk.y = *reinterpret_cast<uint32_t *>(&p1);
                *reinterpret_cast<uint2 *>(o) = pk;
            } else {
                *reinterpret_cast<float4 *>(o) = make_float4(y0, y1, y2, y3);
            }
        }
    }
}

// Generic fallback (any d): three passes over the row.
template <typename T>
__global__ void __launch_bounds__(256) k_modln_any(const float *__restrict__ h, T *__restrict__ out, int d, int M,
                                                   int split, const float *__restrict__ scale_lo,
                                                   const float *__restrict__ scale_hi,
                                                   const float *__restrict__ shift_lo,
                                                   const float *__restrict__ shift_hi, float eps) {
    __shared__ float red[32];
    const int r = blockIdx.x;
    const int m = r % M;
    const float *sc = m < split ? scale_lo : scale_hi;
    const float *sh = m < split ? shift_lo : shift_hi;
    const float *x = h + (size_t)r * d;
    float s = 0.f;
    for (int c = threadIdx.x; c < d; c += blockDim.x) s += x[c];
    const float mean = block_sum(s, red) / d;
    float q = 0.f;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        const float a = x[c] - mean;
        q += a * a;
    }
    const float var = block_sum(q, red) / d;
    const float rstd = 1.0f / sqrtf(var + eps);
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float y = (x[c] - mean) * rstd * (1.f + sc[c]);
        if (sh) y += sh[c];
        out[(size_t)r * d + c] = from_f<T>(y);
    }
}

// ---------------------------------------------------------------------------
// img_in: h[out_row(r)][c] = sum_k x[r][k] * W[c][k]  (lab [1A], patch size 1).
// Input row r = b*N + n goes to residual row b*M_out + off + n.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_img_in(const float *__restrict__ x, const T *__restrict__ W,
                                                float *__restrict__ h, int rows, int C, int d, int N, int M_out,
                                                int off) {
    extern __shared__ float xs[];   // [16][C]
    const int r0 = blockIdx.x * 16;
    for (int e = threadIdx.x; e < 16 * C; e += blockDim.x) {
        const int i = e / C, k = e % C;
        xs[e] = (r0 + i < rows) ? x[(size_t)(r0 + i) * C + k] : 0.f;
    }
    __syncthreads();
    const int c = blockIdx.y * 256 + threadIdx.x;
    if (c >= d) return;
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    const T *w = W + (size_t)c * C;
    for (int k = 0; k < C; ++k) {
        const float wk = to_f(w[k]);
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = fmaf(xs[i * C + k], wk, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int r = r0 + i;
        if (r < rows) {
            const int b = r / N, n = r % N;
            h[((size_t)b * M_out + off + n) * d + c] = acc[i];
        }
    }
}

// img_in for 64 latent channels: each thread keeps its output column's 64
// weights in registers (eight 16-byte loads) and produces 16 rows.
template <typename T>
__global__ void __launch_bounds__(256) k_img_in64(const float *__restrict__ x, const T *__restrict__ W,
                                                  float *__restrict__ h, int rows, int d, int N, int M_out, int off) {
    constexpr int C = 64;
    __shared__ float xs[16][C];
    const int r0 = blockIdx.x * 16;
    for (int e = threadIdx.x; e < 16 * C; e += blockDim.x) {
        const int i = e / C, k = e % C;
        xs[i][k] = (r0 + i < rows) ? x[(size_t)(r0 + i) * C + k] : 0.f;
    }
    const int c = blockIdx.y * 256 + threadIdx.x;
    float w[C];
    if (c < d) {
        if constexpr (sizeof(T) == 2) {
            const uint4 *w8 = reinterpret_cast<const uint4 *>(W + (size_t)c * C);
#pragma unroll
            for (int q = 0; q < C / 8; ++q) {
                const uint4 u = w8[q];
                const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 f = __bfloat1622float2(p2[t]);
                    w[8 * q + 2 * t] = f.x;
                    w[8 * q + 2 * t + 1] = f.y;
                }
            }
        } else {
            const float4 *w4 = reinterpret_cast<const float4 *>(W + (size_t)c * C);
#pragma unroll
            for (int q = 0; q < C / 4; ++q) {
                const float4 f = w4[q];
                w[4 * q] = f.x;
                w[4 * q + 1] = f.y;
                w[4 * q + 2] = f.z;
                w[4 * q + 3] = f.w;
            }
        }
    }
    __syncthreads();
    if (c >= d) return;
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
        const int r = r0 + i;
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < C; ++k) acc = fmaf(xs[i][k], w[k], acc);
        if (r < rows) {
            const int b = r / N, n = r % N;
            h[((size_t)b * M_out + off + n) * d + c] = acc;
        }
    }
}

// Copy the prefix hidden states [B][P][d] into residual rows b*M_out + n.
// out[z][c][r] = in[z][r][c] (one matrix per blockIdx.z), 32x32 tiles through
// shared memory so that both the reads and the writes are coalesced.
template <typename T>
__global__ void __launch_bounds__(256) k_transpose(const T *__restrict__ in, T *__restrict__ out, int rows, int cols) {
    __shared__ T tile[32][33];
    const size_t mat = (size_t)rows * cols * blockIdx.z;
    const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
    for (int i = ty; i < 32; i += 8) {
        const int r = r0 + i, c = c0 + tx;
        if (r < rows && c < cols) tile[i][tx] = in[mat + (size_t)r * cols + c];
    }
    __syncthreads();
    for (int i = ty; i < 32; i += 8) {
        const int c = c0 + i, r = r0 + tx;
        if (r < rows && c < cols) out[mat + (size_t)c * rows + r] = tile[tx][i];
    }
}

static __global__ void k_copy_rows(const float *__restrict__ src, float *__restrict__ dst, int rows_per_item, int d,
                            int M_out, int64_t total) {
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = e / d, c = e % d;
        const int64_t b = row / rows_per_item, n = row % rows_per_item;
        dst[(b * M_out + n) * d + c] = src[e];
    }
}

// ---------------------------------------------------------------------------
// CUDA-core GEMM: Cm[m][n] = sum_k A[m][k] * W[n][k], fp32 accumulate, fp32 out.
// 64x64 tile, BK 16, 256 threads, 4x4 outputs per thread, bounds-checked.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(const T *__restrict__ A, int lda, const T *__restrict__ W,
                                                   int ldw, float *__restrict__ Cm, int ldc, int M, int N, int K) {
    __shared__ float As[16][68];
    __shared__ float Ws[16][68];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + i * 256, row = e >> 4, kk = e & 15;
            const int gk = k0 + kk;
            As[kk][row] = (m0 + row < M && gk < K) ? to_f(A[(size_t)(m0 + row) * lda + gk]) : 0.f;
            Ws[kk][row] = (n0 + row < N && gk < K) ? to_f(W[(size_t)(n0 + row) * ldw + gk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) Cm[(size_t)m * ldc + n] = acc[i][j];
        }
    }
}

// ---------------------------------------------------------------------------
// QK-RMSNorm + RoPE + scatter of one (row, head) per warp (lab [4A]):
// q, k <- x * rsqrt(mean x^2 + eps) * (1 + w) over the head dims, then the
// adjacent pairs (2j, 2j+1) rotate by the token's angle (cos_sin[m][j]).
// Queries go to q_out[r]; K and V go to the K/V buffer rows row_off + m of item b.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) k_qkv_post(const float *__restrict__ Cm, int R, int M, int d, int H, int Dh,
                                                  const float *__restrict__ q_norm, const float *__restrict__ k_norm,
                                                  float eps, const float *__restrict__ cos_sin,
                                                  T *__restrict__ q_out, T *__restrict__ k_base,
                                                  T *__restrict__ v_base, int64_t kv_bstride, int row_off) {
    const int warp = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (warp >= R * H) return;
    const int r = warp / H, hh = warp % H;
    const int b = r / M, m = r % M;
    const float *row = Cm + (size_t)r * 3 * d;
    const int nper = (Dh + 31) / 32;
    T *kdst = k_base + (size_t)b * kv_bstride + (size_t)(row_off + m) * d + hh * Dh;
    T *vdst = v_base + (size_t)b * kv_bstride + (size_t)(row_off + m) * d + hh * Dh;
    T *qdst = q_out + (size_t)r * d + hh * Dh;
    for (int part = 0; part < 2; ++part) {
        const float *src = row + part * d + hh * Dh;
        const float *w = part == 0 ? q_norm : k_norm;
        T *dst = part == 0 ? qdst : kdst;
        float ss = 0.f;
        for (int i = 0; i < nper; ++i) {
            const int j = lane + 32 * i;
            if (j < Dh) ss += src[j] * src[j];
        }
        ss = warp_sum(ss);
        const float inv = 1.0f / sqrtf(ss / Dh + eps);
        for (int i = 0; i < nper; ++i) {
            const int j = lane + 32 * i;
            const float y = j < Dh ? src[j] * inv * (1.f + w[j]) : 0.f;
            const float partner = __shfl_xor_sync(0xffffffffu, y, 1);
            if (j < Dh) {
                const float c = cos_sin[((size_t)m * (Dh / 2) + j / 2) * 2 + 0];
                const float s = cos_sin[((size_t)m * (Dh / 2) + j / 2) * 2 + 1];
                const float o = (j & 1) ? (partner * s + y * c) : (y * c - partner * s);
                dst[j] = from_f<T>(o);
            }
        }
    }
    const float *src = row + 2 * d + hh * Dh;
    for (int j = lane; j < Dh; j += 32) vdst[j] = from_f<T>(src[j]);
}

// h[r][c] += g[c] * Y[r][c], g = tanh(gate) of the row's modulation (lo/hi).
static __global__ void k_gated_residual(float *__restrict__ h, const float *__restrict__ Y, int ldy, int R, int d, int M,
                                 int split, const float *__restrict__ g_lo, const float *__restrict__ g_hi) {
    const int64_t total = (int64_t)R * d;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e / d;
        const int c = (int)(e % d);
        const float g = ((r % M) < split ? g_lo : g_hi)[c];
        h[e] += g * Y[r * ldy + c];
    }
}

// hid[r][j] = silu(G[r][j]) * U[r][j] with G = Cm[:, 0:F], U = Cm[:, F:2F] (lab [5A]).
template <typename T>
__global__ void k_swiglu(const float *__restrict__ Cm, T *__restrict__ hid, int R, int F) {
    const int64_t total = (int64_t)R * F;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e / F;
        const int j = (int)(e % F);
        const float g = Cm[r * 2 * F + j], u = Cm[r * 2 * F + F + j];
        hid[e] = from_f<T>(silu_f(g) * u);
    }
}

// ---------------------------------------------------------------------------
// Attention on CUDA cores: softmax(q k^T / sqrt(Dh)) v over keys [0, limit)
// of the query row (kv_limit, or all kv_len keys), online softmax in fp32.
// Block = 32 query rows of one (item, head); tiles of 32 keys in shared memory.
// Thread t of warp w owns row 8w + lane/4 and the dims (lane % 4) + 4i.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) k_attn_simt(const T *__restrict__ q, int64_t q_bstride, int q_rows, int ldq,
                                                   const T *__restrict__ kb, const T *__restrict__ vb,
                                                   int64_t kv_bstride, int ldkv, int kv_len,
                                                   const int *__restrict__ kv_limit, T *__restrict__ out, int Dh,
                                                   float scale, int split, int64_t tgt_off, int64_t tgt_bstride) {
    // keys [0, split) are rows of kb + b*kv_bstride; keys k >= split are rows
    // k - split of kb + tgt_off + b*tgt_bstride (the shared-prefix cache; split =
    // kv_len otherwise)
    extern __shared__ float sm[];
    const int DP = Dh + 1;
    float *Qs = sm;                 // [32][DP]
    float *Ks = Qs + 32 * DP;       // [32][DP]
    float *Vs = Ks + 32 * DP;       // [32][DP]
    float *Ps = Vs + 32 * DP;       // [32][33]
    __shared__ int lim_max;
    const int hh = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * 32;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int row = wid * 8 + (lane >> 2), sub = lane & 3;
    const T *qb = q + (size_t)b * q_bstride + hh * Dh;
    const T *kbb = kb + (size_t)b * kv_bstride + hh * Dh;
    const T *vbb = vb + (size_t)b * kv_bstride + hh * Dh;
    for (int e = tid; e < 32 * Dh; e += 128) {
        const int i = e / Dh, j = e % Dh;
        Qs[i * DP + j] = (q0 + i < q_rows) ? to_f(qb[(size_t)(q0 + i) * ldq + j]) : 0.f;
    }
    const int qrow = q0 + row;
    int my_lim = kv_len;
    if (kv_limit) my_lim = (qrow < q_rows) ? kv_limit[qrow] : 1;
    if (my_lim > kv_len) my_lim = kv_len;
    if (tid == 0) lim_max = 0;
    __syncthreads();
    atomicMax(&lim_max, my_lim);
    __syncthreads();
    const int kv_end = lim_max;
    const int nd = (Dh + 3) / 4;
    float o[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    for (int t0 = 0; t0 < kv_end; t0 += 32) {
        __syncthreads();
        for (int e = tid; e < 32 * Dh; e += 128) {
            const int i = e / Dh, j = e % Dh;
            const int key = t0 + i;
            const bool ok = key < kv_len;
            const size_t off = key < split ? (size_t)key * ldkv : (size_t)(tgt_off - (int64_t)b * kv_bstride) +
                                                                     (size_t)b * tgt_bstride +
                                                                     (size_t)(key - split) * ldkv;
            Ks[i * DP + j] = ok ? to_f(kbb[off + j]) : 0.f;
            Vs[i * DP + j] = ok ? to_f(vbb[off + j]) : 0.f;
        }
        __syncthreads();
        float s[8];
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = sub * 8 + i;
            float acc = 0.f;
            for (int j = 0; j < Dh; ++j) acc = fmaf(Qs[row * DP + j], Ks[c * DP + j], acc);
            s[i] = (t0 + c < my_lim) ? acc * scale : -INFINITY;
            mx = fmaxf(mx, s[i]);
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = (m_new == -INFINITY) ? 1.f : expf(m_run - m_new);
        float rs = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float p = (s[i] == -INFINITY) ? 0.f : expf(s[i] - m_new);
            Ps[row * 33 + sub * 8 + i] = p;
            rs += p;
        }
        rs += __shfl_xor_sync(0xffffffffu, rs, 1);
        rs += __shfl_xor_sync(0xffffffffu, rs, 2);
        l_run = l_run * alpha + rs;
        m_run = m_new;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i < nd) {
                const int j = sub + 4 * i;
                if (j < Dh) {
                    float acc = o[i] * alpha;
                    for (int c = 0; c < 32; ++c) acc = fmaf(Ps[row * 33 + c], Vs[c * DP + j], acc);
                    o[i] = acc;
                }
            }
        }
    }
    if (qrow < q_rows) {
        T *ob = out + (size_t)b * q_bstride + (size_t)qrow * ldq + hh * Dh;
        const float inv = 1.f / l_run;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int j = sub + 4 * i;
            if (i < nd && j < Dh) ob[j] = from_f<T>(o[i] * inv);
        }
    }
}

// ---------------------------------------------------------------------------
// Final scale-only AdaLN + proj_out (6B page §1): v[b][n][c] =
// sum_k LN(h)[k] (1 + scale_final[k]) Wout[c][k] for the N target rows of each
// item (residual rows b*M + off + n). 4 rows per block, rows staged in smem.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_final(const float *__restrict__ h, int M, int off, int N, int d,
                                               const float *__restrict__ sf, const T *__restrict__ Wout, int C,
                                               float eps, float *__restrict__ v, int rows) {
    extern __shared__ float xs[];   // [4][d]
    __shared__ float red[32];
    const int r0 = blockIdx.x * 4;
    for (int i = 0; i < 4; ++i) {
        const int r = r0 + i;
        if (r >= rows) {
            for (int c = threadIdx.x; c < d; c += blockDim.x) xs[i * d + c] = 0.f;
            continue;
        }
        const int b = r / N, n = r % N;
        const float *x = h + ((size_t)b * M + off + n) * d;
        float s = 0.f;
        for (int c = threadIdx.x; c < d; c += blockDim.x) s += x[c];
        const float mean = block_sum(s, red) / d;
        float q = 0.f;
        for (int c = threadIdx.x; c < d; c += blockDim.x) {
            const float a = x[c] - mean;
            q += a * a;
        }
        const float rstd = 1.0f / sqrtf(block_sum(q, red) / d + eps);
        for (int c = threadIdx.x; c < d; c += blockDim.x) xs[i * d + c] = (x[c] - mean) * rstd * (1.f + sf[c]);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int o = wid; o < 4 * C; o += 8) {
        const int i = o / C, c = o % C;
        const T *w = Wout + (size_t)c * d;
        float acc = 0.f;
        for (int k = lane; k < d; k += 32) acc = fmaf(xs[i * d + k], to_f(w[k]), acc);
        acc = warp_sum(acc);
        if (lane == 0 && r0 + i < rows) v[(size_t)(r0 + i) * C + c] = acc;
    }
}

// Final AdaLN + proj_out for 64 latent channels and d % 128 == 0, tiled:
// 16 rows x 64 outputs per block. Row statistics first (one warp per two
// rows, two-pass), then K chunks of 128: the normalised, scaled rows and the
// matching W_out columns are staged in shared memory and each thread
// accumulates one row x four outputs.
template <typename T>
__global__ void __launch_bounds__(256) k_final64(const float *__restrict__ h, int M, int off, int N, int d,
                                                 const float *__restrict__ sf, const T *__restrict__ Wout, float eps,
                                                 float *__restrict__ v, int rows) {
    constexpr int RB = 16, C = 64, KC = 128;
    __shared__ float mean_s[RB], rstd_s[RB];
    __shared__ float xs[RB][KC];
    __shared__ float ws[C][KC + 1];
    const int r0 = blockIdx.x * RB;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int i = wid; i < RB; i += 8) {
        const int r = r0 + i;
        float mean = 0.f, rstd = 0.f;
        if (r < rows) {
            const int b = r / N, n = r % N;
            const float4 *x4 = reinterpret_cast<const float4 *>(h + ((size_t)b * M + off + n) * d);
            float s = 0.f;
            for (int c4 = lane; c4 < d / 4; c4 += 32) {
                const float4 a = x4[c4];
                s += (a.x + a.y) + (a.z + a.w);
            }
            mean = warp_sum(s) / d;
            float q = 0.f;
            for (int c4 = lane; c4 < d / 4; c4 += 32) {
                const float4 a = x4[c4];
                const float e0 = a.x - mean, e1 = a.y - mean, e2 = a.z - mean, e3 = a.w - mean;
                q += (e0 * e0 + e1 * e1) + (e2 * e2 + e3 * e3);
            }
            rstd = 1.0f / sqrtf(warp_sum(q) / d + eps);
        }
        if (lane == 0) {
            mean_s[i] = mean;
            rstd_s[i] = rstd;
        }
    }
    __syncthreads();
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;     // row ty, outputs 4tx .. 4tx+3
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < d; k0 += KC) {
        for (int e = threadIdx.x; e < RB * KC; e += 256) {
            const int i = e / KC, k = e % KC;
            const int r = r0 + i;
            float val = 0.f;
            if (r < rows) {
                const int b = r / N, n = r % N;
                val = (h[((size_t)b * M + off + n) * d + k0 + k] - mean_s[i]) * rstd_s[i] * (1.f + sf[k0 + k]);
            }
            xs[i][k] = val;
        }
        for (int e = threadIdx.x; e < C * KC; e += 256) {
            const int cc = e / KC, k = e % KC;
            ws[cc][k] = to_f(Wout[(size_t)cc * d + k0 + k]);
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < KC; ++k) {
            const float xv = xs[ty][k];
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = fmaf(xv, ws[4 * tx + j][k], acc[j]);
        }
        __syncthreads();
    }
    const int r = r0 + ty;
    if (r < rows) {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[(size_t)r * C + 4 * tx + j] = acc[j];
    }
}

// x_out = x + dsig * v  (6B page §1).
// Joint packing of the prefix values (2A page, mechanisms (1)-(2)): one block
// per (prefix token, item) copies its slot vector (text) or its img_in token
// (image, mode 0) — or adds the two (mode 1, the lab's COND_TOKENS) — with
// 16-byte loads. Rows whose index tables point outside ctx / img are skipped.
static __global__ void k_pack_prefix(const float *__restrict__ ctx, const float *__restrict__ img,
                                     const int32_t *__restrict__ slot_of, const int32_t *__restrict__ img_row,
                                     int P, int d, int n_slots, int n_img, int mode, float *__restrict__ out) {
    const int s = blockIdx.x, b = blockIdx.y;
    const int slot = slot_of[s], ir = img_row[s];
    if (slot < 0 || slot >= n_slots || ir < -1 || ir >= n_img) return;
    const float4 *c4 = reinterpret_cast<const float4 *>(ctx + ((size_t)b * n_slots + slot) * d);
    const float4 *i4 = ir >= 0 ? reinterpret_cast<const float4 *>(img + ((size_t)b * n_img + ir) * d) : nullptr;
    float4 *o4 = reinterpret_cast<float4 *>(out + ((size_t)b * P + s) * d);
    for (int i = threadIdx.x; i < d / 4; i += blockDim.x) {
        float4 v;
        if (mode == 0) {
            v = i4 ? i4[i] : c4[i];
        } else {
            v = c4[i];
            if (i4) {
                const float4 t = i4[i];
                v.x += t.x;
                v.y += t.y;
                v.z += t.z;
                v.w += t.w;
            }
        }
        o4[i] = v;
    }
}

__device__ __forceinline__ void euler_body(const float *__restrict__ x, const float *__restrict__ v, float dsig,
                                           float *__restrict__ xo, int64_t n) {
    const int64_t n4 = n >> 2;
    const float4 *x4 = reinterpret_cast<const float4 *>(x);
    const float4 *v4 = reinterpret_cast<const float4 *>(v);
    float4 *o4 = reinterpret_cast<float4 *>(xo);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = x4[i], b = v4[i];
        o4[i] = make_float4(fmaf(dsig, b.x, a.x), fmaf(dsig, b.y, a.y), fmaf(dsig, b.z, a.z), fmaf(dsig, b.w, a.w));
    }
    for (int64_t i = (n4 << 2) + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        xo[i] = fmaf(dsig, v[i], x[i]);
}

static __global__ void k_euler(const float *__restrict__ x, const float *__restrict__ v, float dsig,
                        float *__restrict__ xo, int64_t n) {
    pdl_launch_dependents();
    pdl_wait();
    euler_body(x, v, dsig, xo, n);
}

// Euler update with the step read from a device table of sigmas; the
// difference is formed in fp64 and rounded once, as on the host path.
static __global__ void k_euler_sigma(const float *__restrict__ x, const float *__restrict__ v,
                                     const double *__restrict__ sigmas, int step, float *__restrict__ xo, int64_t n) {
    pdl_launch_dependents();
    pdl_wait();
    euler_body(x, v, (float)(sigmas[step + 1] - sigmas[step]), xo, n);
}

// ---------------------------------------------------------------------------
// Modulation GEMVs (3B page §1): y[n] = act_out( sum_k W[n][k] act_in(x[k]) ).
// One warp per output row, K-contiguous weight rows streamed with 16-byte loads.
// ---------------------------------------------------------------------------
struct TembArg {
    float v[512];
};

template <typename T>
__device__ __forceinline__ float dot_row(const T *__restrict__ w, const float *__restrict__ xs, int K, int lane) {
    float acc = 0.f;
    if constexpr (sizeof(T) == 2) {
        if ((K & 7) == 0) {
            const uint4 *w8 = reinterpret_cast<const uint4 *>(w);
            for (int k8 = lane; k8 < K / 8; k8 += 32) {
                const uint4 u = w8[k8];
                const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 f = __bfloat1622float2(p[t]);
                    acc = fmaf(f.x, xs[k8 * 8 + 2 * t], acc);
                    acc = fmaf(f.y, xs[k8 * 8 + 2 * t + 1], acc);
                }
            }
            return acc;
        }
    } else {
        if ((K & 3) == 0) {
            const float4 *w4 = reinterpret_cast<const float4 *>(w);
            for (int k4 = lane; k4 < K / 4; k4 += 32) {
                const float4 f = w4[k4];
                acc = fmaf(f.x, xs[k4 * 4 + 0], acc);
                acc = fmaf(f.y, xs[k4 * 4 + 1], acc);
                acc = fmaf(f.z, xs[k4 * 4 + 2], acc);
                acc = fmaf(f.w, xs[k4 * 4 + 3], acc);
            }
            return acc;
        }
    }
    for (int k = lane; k < K; k += 32) acc = fmaf(to_f(w[k]), xs[k], acc);
    return acc;
}

// First layer of the timestep MLP: y = silu(W x), x = the sin-cos embedding
// passed by value (computed on the host in fp64).
template <typename T>
__global__ void __launch_bounds__(256) k_temb_in(const T *__restrict__ W, TembArg emb, int K, int N,
                                                 float *__restrict__ y) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ float xs[512];
    for (int k = threadIdx.x; k < K; k += blockDim.x) xs[k] = emb.v[k];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (n >= N) return;
    const float acc = warp_sum(dot_row(W + (size_t)n * K, xs, K, lane));
    if (lane == 0) y[n] = silu_f(acc);
}

// As k_temb_in, with the embedding formed on the device from a device table of
// sigmas (so that a captured sequence of steps reads its sigma at run time):
// t = t_per_sigma * sigmas[step], emb = [cos(t f_i) | sin(t f_i)],
// f_i = 10000^(-2i/K), in fp64 rounded once to fp32 (the host helper
// qi21_timestep_embedding does the same arithmetic).
template <typename T>
__global__ void __launch_bounds__(256) k_temb_in_sigma(const T *__restrict__ W, const double *__restrict__ sigmas,
                                                       int step, double t_per_sigma, int K, int N,
                                                       float *__restrict__ y) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ float xs[512];
    const int half = K / 2;
    const double t = t_per_sigma * sigmas[step];
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        const double f = pow(10000.0, -2.0 * i / K);
        xs[i] = (float)cos(t * f);
        xs[half + i] = (float)sin(t * f);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (n >= N) return;
    const float acc = warp_sum(dot_row(W + (size_t)n * K, xs, K, lane));
    if (lane == 0) y[n] = silu_f(acc);
}

// y[n] = W[n] . act_in(x), act_in = silu when silu_in; rows [0, N1) come from
// W1 into y1, rows [N1, N1+N2) from W2 into y2 (one launch for mod and final scale).
template <typename T>
__global__ void __launch_bounds__(256) k_gemv2(const T *__restrict__ W1, int N1, float *__restrict__ y1,
                                               const T *__restrict__ W2, int N2, float *__restrict__ y2,
                                               const float *__restrict__ x, int K, int silu_in) {
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ float xs[];
    for (int k = threadIdx.x; k < K; k += blockDim.x) xs[k] = silu_in ? silu_f(x[k]) : x[k];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (n >= N1 + N2) return;
    const bool first = n < N1;
    const T *w = first ? W1 + (size_t)n * K : W2 + (size_t)(n - N1) * K;
    const float acc = warp_sum(dot_row(w, xs, K, lane));
    if (lane == 0) {
        if (first)
            y1[n] = acc;
        else
            y2[n - N1] = acc;
    }
}

}  // namespace qi21
