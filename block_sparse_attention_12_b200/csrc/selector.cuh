// IBCS selector kernels: mean keys, intra-block k-means and block scores.
//
// Follows the IBCS paragraph of the AB-Attention news page (hamidun, Arabic),
// section "three techniques in AB-Attention": 128-query blocks, 8 clusters
// per block weighted by their share of the block's queries, and a KV block
// score equal to the weighted attention of the centroids to the block's mean
// key.  The clusters only estimate importance; no token is reordered.
#pragma once

#include "common.cuh"

namespace abattn {

// ---------------------------------------------------------------- mean keys
// One thread per (KV block, 8-column group): 16-byte bf16 loads, fp32 sums,
// two 16-byte fp32 stores.  HBM bound: reads K once, writes Kbar once.
template <int D>
__global__ void __launch_bounds__(256) meanpool_kernel(const __nv_bfloat16 *__restrict__ K,
                                                       int64_t BH, int64_t N, int kb,
                                                       int64_t nkvb, float *__restrict__ Kbar) {
    constexpr int G = D / 8;
    const int64_t total = BH * nkvb * G;
    for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += int64_t(gridDim.x) * blockDim.x) {
        const int c8 = int(e % G);
        const int64_t blk = e / G;
        const int64_t bh = blk / nkvb, j = blk % nkvb;
        const int64_t t0 = j * kb;
        const int64_t t1 = min(N, t0 + kb);
        float acc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = 0.f;
        const __nv_bfloat16 *src = K + (bh * N + t0) * D + c8 * 8;
#pragma unroll 4
        for (int64_t t = t0; t < t1; ++t, src += D) {
            uint4 v = __ldg(reinterpret_cast<const uint4 *>(src));
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float2 f = __bfloat1622float2(h[u]);
                acc[2 * u] += f.x;
                acc[2 * u + 1] += f.y;
            }
        }
        const float cnt = float(t1 - t0);
        float4 o0 = make_float4(acc[0] / cnt, acc[1] / cnt, acc[2] / cnt, acc[3] / cnt);
        float4 o1 = make_float4(acc[4] / cnt, acc[5] / cnt, acc[6] / cnt, acc[7] / cnt);
        float4 *dst = reinterpret_cast<float4 *>(Kbar + blk * D + c8 * 8);
        dst[0] = o0;
        dst[1] = o1;
    }
}

// ---------------------------------------------------------------- k-means
// One CTA (256 threads) per q-block.  The block's queries sit in shared
// memory transposed, Qs[k][i] (row stride 129 floats: conflict-free column
// and row walks); centroids interleaved, Cs[k][8].
constexpr int KM_THREADS = 256;
constexpr int KM_QS = 129;

template <int D>
constexpr size_t kmeans_smem_bytes() {
    return sizeof(float) * (size_t(D) * KM_QS + size_t(D) * 8 + 128 * 9) + sizeof(int) * (128 + 8);
}

template <int D>
__global__ void __launch_bounds__(KM_THREADS) kmeans_kernel(
    const __nv_bfloat16 *__restrict__ Q, int64_t N, int64_t nqb, int nc, int iters,
    float *__restrict__ Cout, float *__restrict__ wout, int32_t *__restrict__ labels_out) {
    extern __shared__ float km_smem[];
    float *Qs = km_smem;                 // [D][KM_QS]
    float *Cs = Qs + D * KM_QS;          // [D][8]
    float *dist = Cs + D * 8;            // [128][9]
    int *lab = reinterpret_cast<int *>(dist + 128 * 9);  // [128]
    int *cnt_s = lab + 128;                               // [8]

    const int tid = threadIdx.x;
    const int64_t row = blockIdx.x;
    const int64_t bh = row / nqb, qb = row % nqb;
    const int64_t q0 = qb * 128;
    const int M = int(N - q0 < 128 ? N - q0 : 128);

    // load + transpose (bf16 -> fp32)
    constexpr int G = D / 8;
    const __nv_bfloat16 *src = Q + (bh * N + q0) * D;
    for (int e = tid; e < M * G; e += KM_THREADS) {
        const int i = e / G, c8 = e % G;
        uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + size_t(i) * D + c8 * 8));
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float2 f = __bfloat1622float2(h[u]);
            Qs[(c8 * 8 + 2 * u) * KM_QS + i] = f.x;
            Qs[(c8 * 8 + 2 * u + 1) * KM_QS + i] = f.y;
        }
    }
    __syncthreads();
    // init: centroid c = query floor(c*M/nc); unused centroid slots are zero
    for (int e = tid; e < D * 8; e += KM_THREADS) {
        const int k = e / 8, c = e % 8;
        Cs[e] = c < nc ? Qs[k * KM_QS + (c * M) / nc] : 0.f;
    }
    if (tid < 8) cnt_s[tid] = 0;
    __syncthreads();

    for (int it = 0; it < iters; ++it) {
        // squared distances: thread -> (query i, centroids 4g .. 4g+3)
        {
            const int i = tid & 127, g = tid >> 7;
            if (i < M && 4 * g < nc) {
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
                for (int k = 0; k < D; ++k) {
                    const float q = Qs[k * KM_QS + i];
                    const float4 c = *reinterpret_cast<const float4 *>(Cs + k * 8 + 4 * g);
                    float t;
                    t = q - c.x; a0 = fmaf(t, t, a0);
                    t = q - c.y; a1 = fmaf(t, t, a1);
                    t = q - c.z; a2 = fmaf(t, t, a2);
                    t = q - c.w; a3 = fmaf(t, t, a3);
                }
                dist[i * 9 + 4 * g + 0] = a0;
                dist[i * 9 + 4 * g + 1] = a1;
                dist[i * 9 + 4 * g + 2] = a2;
                dist[i * 9 + 4 * g + 3] = a3;
            }
        }
        __syncthreads();
        if (tid < M) {
            int best = 0;
            float bd = dist[tid * 9];
            for (int c = 1; c < nc; ++c) {
                const float v = dist[tid * 9 + c];
                if (v < bd) { bd = v; best = c; }
            }
            lab[tid] = best;
        }
        __syncthreads();
        // centroid update: thread -> (column k, CPT centroids)
        {
            constexpr int GROUPS = KM_THREADS / D;  // 2 for d=128, 4 for d=64
            constexpr int CPT = 8 / GROUPS;
            const int k = tid % D, grp = tid / D, c0 = grp * CPT;
            float acc[CPT];
            int n[CPT];
#pragma unroll
            for (int u = 0; u < CPT; ++u) { acc[u] = 0.f; n[u] = 0; }
            for (int i = 0; i < M; ++i) {
                const int l = lab[i];
                const float v = Qs[k * KM_QS + i];
#pragma unroll
                for (int u = 0; u < CPT; ++u)
                    if (l == c0 + u) { acc[u] += v; n[u] += 1; }
            }
#pragma unroll
            for (int u = 0; u < CPT; ++u) {
                const int c = c0 + u;
                if (c < nc && n[u] > 0) Cs[k * 8 + c] = acc[u] / float(n[u]);
                if (k == 0 && c < 8) cnt_s[c] = n[u];
            }
        }
        __syncthreads();
    }

    const int64_t r = row;
    for (int e = tid; e < nc * D; e += KM_THREADS) {
        const int c = e / D, k = e % D;
        Cout[(r * nc + c) * D + k] = Cs[k * 8 + c];
    }
    if (tid < nc) wout[r * nc + tid] = iters > 0 ? float(cnt_s[tid]) / float(M) : 1.f / float(nc);
    if (labels_out != nullptr && tid < 128)
        labels_out[r * 128 + tid] = (iters > 0 && tid < M) ? lab[tid] : -1;
}

// ---------------------------------------------------------------- scores
// Per head, the centroids of all q-blocks against all mean keys form a GEMM
// [nqb*nc, d] x [d, nkvb].  A CTA computes a tile of 8 q-blocks (their nc <= 8
// centroids each, 64 rows) x 128 KV blocks in fp32 on the CUDA cores: warp w
// owns q-block w of the tile, lane l owns KV blocks l, l+32, l+64, l+96.
// Pass 1 writes per-tile (max, sum exp) of every centroid row; a combine
// kernel folds them into (m_c, Z_c); pass 2 recomputes the tile and writes
// s_j = sum_c (w_c / Z_c) exp(L_cj - m_c).  Logits are kept in log2 units.
constexpr int SC_QB = 8;
constexpr int SC_TN = 128;

template <int D>
constexpr size_t score_smem_bytes() {
    return sizeof(float) * size_t(SC_QB * 8 + SC_TN) * (D + 4);
}

template <int D>
__device__ __forceinline__ void score_tile(const float *__restrict__ C, const float *__restrict__ Kbar,
                                           int64_t bh, int64_t nqb, int64_t nkvb, int nc,
                                           int64_t qb0, int64_t j0, float scale_log2,
                                           float *smem, float (&L)[8][4]) {
    constexpr int LD = D + 4;
    float *Cs = smem;              // [64][LD]
    float *Ks = smem + 64 * LD;    // [128][LD]
    const int tid = threadIdx.x;
    constexpr int V4 = D / 4;
    for (int e = tid; e < 64 * V4; e += 256) {
        const int r = e / V4, k4 = e % V4;
        const int64_t qb = qb0 + r / 8;
        const int c = r % 8;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (qb < nqb && c < nc)
            v = __ldg(reinterpret_cast<const float4 *>(C + ((bh * nqb + qb) * nc + c) * D) + k4);
        *reinterpret_cast<float4 *>(Cs + r * LD + 4 * k4) = v;
    }
    for (int e = tid; e < SC_TN * V4; e += 256) {
        const int r = e / V4, k4 = e % V4;
        const int64_t j = j0 + r;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j < nkvb) v = __ldg(reinterpret_cast<const float4 *>(Kbar + (bh * nkvb + j) * D) + k4);
        *reinterpret_cast<float4 *>(Ks + r * LD + 4 * k4) = v;
    }
    __syncthreads();
    const int w = tid >> 5, lane = tid & 31;
    float acc[8][4];
#pragma unroll
    for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[c][i] = 0.f;
    const float *crow = Cs + (w * 8) * LD;
#pragma unroll 2
    for (int k = 0; k < D; k += 4) {
        float4 kv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) kv[i] = *reinterpret_cast<const float4 *>(Ks + (lane + 32 * i) * LD + k);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 cv = *reinterpret_cast<const float4 *>(crow + c * LD + k);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[c][i] = fmaf(cv.x, kv[i].x, acc[c][i]);
                acc[c][i] = fmaf(cv.y, kv[i].y, acc[c][i]);
                acc[c][i] = fmaf(cv.z, kv[i].z, acc[c][i]);
                acc[c][i] = fmaf(cv.w, kv[i].w, acc[c][i]);
            }
        }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            L[c][i] = (j0 + lane + 32 * i < nkvb) ? acc[c][i] * scale_log2 : -INFINITY;
}

template <int D>
__global__ void __launch_bounds__(256) score_pass1_kernel(
    const float *__restrict__ C, const float *__restrict__ Kbar, int64_t nqb, int64_t nkvb, int nc,
    float scale_log2, float2 *__restrict__ partials, int ntiles) {
    extern __shared__ float sc_smem[];
    const int64_t bh = blockIdx.z, qb0 = int64_t(blockIdx.y) * SC_QB, j0 = int64_t(blockIdx.x) * SC_TN;
    float L[8][4];
    score_tile<D>(C, Kbar, bh, nqb, nkvb, nc, qb0, j0, scale_log2, sc_smem, L);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t qb = qb0 + w;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float m = fmaxf(fmaxf(L[c][0], L[c][1]), fmaxf(L[c][2], L[c][3]));
        m = warp_max(m);
        float z = 0.f;
        if (m != -INFINITY) {
#pragma unroll
            for (int i = 0; i < 4; ++i) z += exp2f(L[c][i] - m);
        }
        z = warp_sum(z);
        if (lane == 0 && qb < nqb && c < nc)
            partials[((bh * nqb + qb) * nc + c) * ntiles + blockIdx.x] = make_float2(m, z);
    }
}

// (m_c, Z_c) = fold of the per-tile partials, one thread per centroid row.
__global__ void score_combine_kernel(const float2 *__restrict__ partials, int64_t nrows, int ntiles,
                                     float2 *__restrict__ stats) {
    const int64_t r = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (r >= nrows) return;
    const float2 *p = partials + r * ntiles;
    float m = -INFINITY;
    for (int t = 0; t < ntiles; ++t) m = fmaxf(m, p[t].x);
    float z = 0.f;
    if (m != -INFINITY)
        for (int t = 0; t < ntiles; ++t)
            if (p[t].x != -INFINITY) z += p[t].y * exp2f(p[t].x - m);
    stats[r] = make_float2(m, z);
}

template <int D>
__global__ void __launch_bounds__(256) score_pass2_kernel(
    const float *__restrict__ C, const float *__restrict__ w, const float *__restrict__ Kbar,
    int64_t nqb, int64_t nkvb, int nc, float scale_log2, const float2 *__restrict__ stats,
    float *__restrict__ S) {
    extern __shared__ float sc_smem[];
    const int64_t bh = blockIdx.z, qb0 = int64_t(blockIdx.y) * SC_QB, j0 = int64_t(blockIdx.x) * SC_TN;
    float L[8][4];
    score_tile<D>(C, Kbar, bh, nqb, nkvb, nc, qb0, j0, scale_log2, sc_smem, L);
    const int wq = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t qb = qb0 + wq;
    if (qb >= nqb) return;
    const int64_t r = bh * nqb + qb;
    float out[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        if (c < nc) {
            const float2 st = stats[r * nc + c];
            const float wc = __ldg(w + r * nc + c);
            if (wc > 0.f && st.y > 0.f) {
                const float coef = wc / st.y;
#pragma unroll
                for (int i = 0; i < 4; ++i) out[i] = fmaf(coef, exp2f(L[c][i] - st.x), out[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t j = j0 + lane + 32 * i;
        if (j < nkvb) S[r * nkvb + j] = out[i];
    }
}

}  // namespace abattn
