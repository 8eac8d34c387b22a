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
// 16-byte stores.  HBM bound: reads K once, writes the mean keys once, either
// as fp32 (Kbar) or as a bf16 pair hi + lo with hi = bf16(x), lo = bf16(x - hi)
// (the operand format of the tensor-core score kernel), or both.
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

template <int D>
__global__ void __launch_bounds__(256) meanpool_kernel(const __nv_bfloat16 *__restrict__ K,
                                                       int64_t BH, int64_t N, int kb,
                                                       int64_t nkvb, float *__restrict__ Kbar,
                                                       __nv_bfloat16 *__restrict__ Khi,
                                                       __nv_bfloat16 *__restrict__ Klo) {
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
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = acc[u] / cnt;
        if (Kbar != nullptr) {
            float4 *dst = reinterpret_cast<float4 *>(Kbar + blk * D + c8 * 8);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        if (Khi != nullptr) {
            alignas(16) __nv_bfloat16 h[8], l[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) split_bf16(acc[u], h[u], l[u]);
            *reinterpret_cast<uint4 *>(Khi + blk * D + c8 * 8) = *reinterpret_cast<const uint4 *>(h);
            *reinterpret_cast<uint4 *>(Klo + blk * D + c8 * 8) = *reinterpret_cast<const uint4 *>(l);
        }
    }
}

// fp32 rows -> bf16 hi/lo pairs (used when the score stage gets fp32 inputs).
// src rows of D floats, grouped n_in per block and padded to n_out rows per
// block in the destination (the padding rows are zero).
template <int D>
__global__ void split_rows_kernel(const float *__restrict__ src, int64_t nblk, int n_in, int n_out,
                                  __nv_bfloat16 *__restrict__ hi, __nv_bfloat16 *__restrict__ lo) {
    const int64_t total = nblk * n_out * D;
    for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += int64_t(gridDim.x) * blockDim.x) {
        const int k = int(e % D);
        const int64_t r = e / D;
        const int c = int(r % n_out);
        const int64_t b = r / n_out;
        const float x = c < n_in ? src[(b * n_in + c) * D + k] : 0.f;
        split_bf16(x, hi[e], lo[e]);
    }
}

// ---------------------------------------------------------------- k-means
// One CTA (128 threads) per q-block.  The block's queries sit in shared
// memory transposed and in their own bf16 precision, Qs[k][i] (row stride
// 130 bf16: conflict-free column and row walks); centroids fp32,
// interleaved, Cs[k][8].
//   assignment: thread i scores its query against all 8 centroids as
//               |c|^2 - 2 q.c (the same argmin as |q - c|^2; |q|^2 is
//               common), ties to the lower index;
//   update:     a stable counting sort of the labels (warp ballots) gives
//               each cluster's members in ascending query order; thread k
//               sums column k over each cluster's members.
constexpr int KM_THREADS = 128;
constexpr int KM_QS = 130;  // bf16 elements per Qs row (65 words: odd stride)

template <int D>
constexpr size_t kmeans_smem_bytes() {
    return sizeof(__nv_bfloat16) * size_t(D) * KM_QS + sizeof(float) * (size_t(D) * 8 + 8 + 4 * 8) +
           sizeof(int) * (128 + 128 + 8 + 9 + 4 * 8);
}

template <int D>
__global__ void __launch_bounds__(KM_THREADS) kmeans_kernel(
    const __nv_bfloat16 *__restrict__ Q, int64_t N, int64_t nqb, int nc, int iters,
    float *__restrict__ Cout, float *__restrict__ wout, int32_t *__restrict__ labels_out,
    __nv_bfloat16 *__restrict__ Chi, __nv_bfloat16 *__restrict__ Clo) {
    extern __shared__ float km_smem[];
    __nv_bfloat16 *Qs = reinterpret_cast<__nv_bfloat16 *>(km_smem);               // [D][KM_QS]
    float *Cs = km_smem + (D * KM_QS) / 2;                                         // [D][8]
    float *cn = Cs + D * 8;                       // [8]     |c|^2
    float *cn_part = cn + 8;                      // [4][8]  per-warp partial |c|^2
    int *lab = reinterpret_cast<int *>(cn_part + 32);  // [128]
    int *order = lab + 128;                        // [128]   queries sorted by cluster
    int *cnt_s = order + 128;                      // [8]
    int *start = cnt_s + 8;                        // [9]
    int *wcnt = start + 9;                         // [4][8]  per-warp cluster counts

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t row = blockIdx.x;
    const int64_t bh = row / nqb, qb = row % nqb;
    const int64_t q0 = qb * 128;
    const int M = int(N - q0 < 128 ? N - q0 : 128);

    // load (all 16-byte loads in flight first) + transpose
    constexpr int G = D / 8;
    constexpr int PER = (128 * G) / KM_THREADS;  // 16-byte chunks per thread
    const __nv_bfloat16 *src = Q + (bh * N + q0) * D;
    {
        uint4 v[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = tid + u * KM_THREADS, i = e / G, c8 = e % G;
            v[u] = i < M ? __ldg(reinterpret_cast<const uint4 *>(src + size_t(i) * D + c8 * 8)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = tid + u * KM_THREADS, i = e / G, c8 = e % G;
            const __nv_bfloat16 *hv = reinterpret_cast<const __nv_bfloat16 *>(&v[u]);
#pragma unroll
            for (int x = 0; x < 8; ++x) Qs[(c8 * 8 + x) * KM_QS + i] = hv[x];
        }
    }
    __syncthreads();
    // init: centroid c = query floor(c*M/nc); unused centroid slots are zero
    for (int e = tid; e < D * 8; e += KM_THREADS) {
        const int k = e / 8, c = e % 8;
        Cs[e] = c < nc ? __bfloat162float(Qs[k * KM_QS + (c * M) / nc]) : 0.f;
    }
    if (tid < 8) cnt_s[tid] = 0;
    __syncthreads();

    auto centroid_norms = [&]() {
        float part[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) part[c] = 0.f;
        for (int k = tid; k < D; k += KM_THREADS) {
#pragma unroll
            for (int c = 0; c < 8; ++c) part[c] = fmaf(Cs[k * 8 + c], Cs[k * 8 + c], part[c]);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float v = warp_sum(part[c]);
            if (lane == 0) cn_part[wid * 8 + c] = v;
        }
        __syncthreads();
        if (tid < 8) cn[tid] = (cn_part[tid] + cn_part[8 + tid]) + (cn_part[16 + tid] + cn_part[24 + tid]);
        __syncthreads();
    };
    if (iters > 0) centroid_norms();

    for (int it = 0; it < iters; ++it) {
        // assignment
        int best = 0;
        if (tid < M) {
            float a[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) a[c] = 0.f;
#pragma unroll 4
            for (int k = 0; k < D; ++k) {
                const float q = __bfloat162float(Qs[k * KM_QS + tid]);
                const float4 c0 = *reinterpret_cast<const float4 *>(Cs + k * 8);
                const float4 c1 = *reinterpret_cast<const float4 *>(Cs + k * 8 + 4);
                a[0] = fmaf(q, c0.x, a[0]);
                a[1] = fmaf(q, c0.y, a[1]);
                a[2] = fmaf(q, c0.z, a[2]);
                a[3] = fmaf(q, c0.w, a[3]);
                a[4] = fmaf(q, c1.x, a[4]);
                a[5] = fmaf(q, c1.y, a[5]);
                a[6] = fmaf(q, c1.z, a[6]);
                a[7] = fmaf(q, c1.w, a[7]);
            }
            float bd = fmaf(-2.f, a[0], cn[0]);
#pragma unroll
            for (int c = 1; c < 8; ++c) {
                const float v = fmaf(-2.f, a[c], cn[c]);
                if (c < nc && v < bd) { bd = v; best = c; }
            }
        }
        // a fixed point (no label changed) repeats itself in every remaining
        // iteration: stop, the result is the same as running them all
        const bool moved = tid < M && (it == 0 || lab[tid] != best);
        if (it > 0 && !__syncthreads_or(moved)) break;
        if (tid < M) lab[tid] = best;
        // stable counting sort of the labels
        unsigned my_rank = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const unsigned m = __ballot_sync(0xffffffffu, tid < M && best == c);
            if (best == c) my_rank = __popc(m & ((1u << lane) - 1u));
            if (lane == 0) wcnt[wid * 8 + c] = __popc(m);
        }
        __syncthreads();
        if (tid == 0) {
            int acc = 0;
            for (int c = 0; c < 8; ++c) {
                start[c] = acc;
                const int n = wcnt[c] + wcnt[8 + c] + wcnt[16 + c] + wcnt[24 + c];
                cnt_s[c] = n;
                acc += n;
            }
            start[8] = acc;
        }
        __syncthreads();
        if (tid < M) {
            int pos = start[best] + int(my_rank);
            for (int w = 0; w < wid; ++w) pos += wcnt[w * 8 + best];
            order[pos] = tid;
        }
        __syncthreads();
        // update: thread k sums column k over each cluster's members (ascending order)
        for (int k = tid; k < D; k += KM_THREADS) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int n = cnt_s[c];
                if (c < nc && n > 0) {
                    float acc = 0.f;
                    for (int p = start[c]; p < start[c + 1]; ++p) acc += __bfloat162float(Qs[k * KM_QS + order[p]]);
                    Cs[k * 8 + c] = acc / float(n);
                }
            }
        }
        __syncthreads();
        if (it + 1 < iters) centroid_norms();
    }

    const int64_t r = row;
    if (Cout != nullptr)
        for (int e = tid; e < nc * D; e += KM_THREADS) {
            const int c = e / D, k = e % D;
            Cout[(r * nc + c) * D + k] = Cs[k * 8 + c];
        }
    if (Chi != nullptr)  // [rows][8][D], clusters past nc zero
        for (int e = tid; e < 8 * D; e += KM_THREADS) {
            const int c = e / D, k = e % D;
            split_bf16(c < nc ? Cs[k * 8 + c] : 0.f, Chi[(r * 8 + c) * D + k], Clo[(r * 8 + c) * D + k]);
        }
    if (tid < nc) wout[r * nc + tid] = iters > 0 ? float(cnt_s[tid]) / float(M) : 1.f / float(nc);
    if (labels_out != nullptr && tid < 128)
        labels_out[r * 128 + tid] = (iters > 0 && tid < M) ? lab[tid] : -1;
}

// ---------------------------------------------------------------- scores
// Per head, the centroids of all q-blocks against all mean keys form the GEMM
// L = C Kbar^T ([nqb*8, d] x [d, nkvb]), evaluated on the tensor cores with
// each fp32 operand split into a bf16 pair: C.K ~ Chi.Khi + Chi.Klo + Clo.Khi
// (three kind::f16 MMAs into one fp32 TMEM accumulator; relative error about
// 2^-16 of |C||K|).  One CTA owns 16 q-blocks (128 centroid rows) of one head
// and sweeps the head's KV blocks twice:
//   pass 1, rows = centroids: each epilogue thread owns one centroid row and
//           keeps its running max m_c and normaliser Z_c = sum_j 2^(L_cj - m_c);
//   pass 2, operands swapped, rows = KV blocks: each thread owns one KV block
//           j and writes s_j = sum_c (w_c / Z_c) 2^(L_cj - m_c) for the 16
//           q-blocks (the 8 clusters of a q-block are 8 columns of its row).
// Warps 0..7 are two epilogue warpgroups taking alternate tiles (TMEM
// accumulator u % 2); at the end of pass 1 they merge their per-centroid
// (max, normaliser).  Warp 8 streams the Kbar tiles by TMA (2 stages), warp 9
// issues the MMAs.  Logits are in log2 units.
constexpr int SC_THREADS = 384;
constexpr int SC_EPI_REGS = 216;    // setmaxnreg of the two epilogue warpgroups
constexpr int SC_OTHER_REGS = 64;   // producer / MMA warpgroup
static_assert(2 * 128 * SC_EPI_REGS + 128 * SC_OTHER_REGS <= SC_THREADS * 168,
              "setmaxnreg split exceeds the launch register budget");
constexpr int SC_QBT = 16;  // q-blocks per CTA (x 8 cluster slots = 128 rows)

template <int D>
struct ScoreLayout {
    static constexpr int HALVES = D / 64;
    static constexpr int TILE = HALVES * 16384;  // 128 rows x D bf16
    static constexpr int C_HI = 0;
    static constexpr int C_LO = TILE;
    static constexpr int STAGE0 = 2 * TILE;  // stage s: hi at STAGE0 + 2*s*TILE, lo right after
    static constexpr int MC_OFF = STAGE0 + 4 * TILE;       // m[128], coef[128]
    static constexpr int XCH_OFF = MC_OFF + 2 * 128 * 4;   // odd warpgroup's pass-1 (m, z)[128]
    static constexpr int BAR_OFF = XCH_OFF + 2 * 128 * 4;
    static constexpr int NBARS = 9;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;
};

struct ScoreParams {
    const float *w;  // [rows][nc]
    float *S;        // [rows][nkvb]
    int nqb;
    int nkvb;
    int nc;
    float scale_log2;
};

__device__ __forceinline__ void epi_bar_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }


template <int D>
__global__ void __launch_bounds__(SC_THREADS, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmChi, const __grid_constant__ CUtensorMap tmClo,
                    const __grid_constant__ CUtensorMap tmKhi, const __grid_constant__ CUtensorMap tmKlo,
                    const ScoreParams p) {
    using L = ScoreLayout<D>;
    extern __shared__ uint8_t sc_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(sc_smem_raw) + 1023) & ~uintptr_t(1023));
    float *sm_m = reinterpret_cast<float *>(smem + L::MC_OFF);
    float *sm_coef = sm_m + 128;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *c_full = bars, *kv_full = bars + 1, *kv_empty = bars + 3, *acc_full = bars + 5,
             *acc_free = bars + 7;
    float *xch = reinterpret_cast<float *>(smem + L::XCH_OFF);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ct = blockIdx.x, bh = blockIdx.y;  // centroid tile (16 q-blocks), head
    const int NT = (p.nkvb + 127) / 128;
    const int U = 2 * NT;  // tile visits over both passes

    if (threadIdx.x == 0) {
        mbar_init(c_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_free[i], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(SC_OTHER_REGS) : "memory");
        if (lane == 0) {
            mbar_arrive_expect_tx(c_full, 2 * L::TILE);
#pragma unroll
            for (int h = 0; h < L::HALVES; ++h) {
                tma_load_3d(smem + L::C_HI + h * 16384, &tmChi, c_full, h * 64, ct * 128, bh);
                tma_load_3d(smem + L::C_LO + h * 16384, &tmClo, c_full, h * 64, ct * 128, bh);
            }
            int issued = 0;
            for (int u = 0; u < U; ++u) {
                const int s = u & 1, t = u < NT ? u : u - NT;
                if (u >= 2 && !mbar_wait(&kv_empty[s], ((u >> 1) - 1) & 1, abort_flag)) break;
                uint8_t *dst = smem + L::STAGE0 + 2 * s * L::TILE;
                mbar_arrive_expect_tx(&kv_full[s], 2 * L::TILE);
#pragma unroll
                for (int h = 0; h < L::HALVES; ++h) {
                    tma_load_3d(dst + h * 16384, &tmKhi, &kv_full[s], h * 64, t * 128, bh);
                    tma_load_3d(dst + L::TILE + h * 16384, &tmKlo, &kv_full[s], h * 64, t * 128, bh);
                }
                ++issued;
            }
            if (*abort_flag) {
                mbar_drain(c_full, 0);
                for (int u = issued - 2 < 0 ? 0 : issued - 2; u < issued; ++u) mbar_drain(&kv_full[u & 1], (u >> 1) & 1);
            }
        }
        __syncwarp();
    } else if (warp >= 9) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(SC_OTHER_REGS) : "memory");
        if (warp == 9 && lane == 0) {
            constexpr uint32_t idesc = make_idesc_bf16(128, 128, 0, 0);
            const uint32_t cb = smem_u32(smem);
            bool ok = mbar_wait(c_full, 0, abort_flag);
            for (int u = 0; ok && u < U; ++u) {
                const int s = u & 1, b = u & 1;
                if (!mbar_wait(&kv_full[s], (u >> 1) & 1, abort_flag)) break;
                if (u >= 2 && !mbar_wait(&acc_free[b], ((u >> 1) - 1) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t kb = cb + L::STAGE0 + 2 * s * L::TILE;
                const uint32_t cbase = cb + L::C_HI;
                // pass 1: A = centroids, B = mean keys; pass 2: swapped
                const uint32_t a_hi = u < NT ? cbase : kb, a_lo = a_hi + L::TILE;
                const uint32_t b_hi = u < NT ? kb : cbase, b_lo = b_hi + L::TILE;
                const uint32_t dt = tmem + b * 128;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    umma_f16_ss(dt, make_sdesc_sw128(a_hi + off, 16, 1024), make_sdesc_sw128(b_hi + off, 16, 1024), idesc, k > 0);
                    umma_f16_ss(dt, make_sdesc_sw128(a_hi + off, 16, 1024), make_sdesc_sw128(b_lo + off, 16, 1024), idesc, 1u);
                    umma_f16_ss(dt, make_sdesc_sw128(a_lo + off, 16, 1024), make_sdesc_sw128(b_hi + off, 16, 1024), idesc, 1u);
                }
                umma_commit(&kv_empty[s]);
                umma_commit(&acc_full[b]);
            }
        }
        __syncwarp();
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(SC_EPI_REGS) : "memory");
        const int eg = warp >> 2;  // this warpgroup takes tiles u with u % 2 == eg
        const int wq = warp & 3, rr = wq * 32 + lane;
        const uint32_t t_lane = tmem + (uint32_t(wq * 32) << 16) + eg * 128;
        float m = -INFINITY, z = 0.f;  // pass 1: raw-accumulator max and sum of 2^(s*(L - m))
        bool ok = true;
        const float sl2 = p.scale_log2;
        // reads this warpgroup's accumulator of tile u into x; false on abort
        auto fetch_acc = [&](int u, uint32_t (&x)[4][32]) -> bool {
            if (!ok || !mbar_wait(&acc_full[eg], (u >> 1) & 1, abort_flag)) { ok = false; return false; }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(t_lane + c * 32, x[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_free[eg]);
            return true;
        };
        // ---- pass 1: columns are KV blocks u*128 + col
        for (int u = eg; u < NT; u += 2) {
            uint32_t x[4][32];
            if (!fetch_acc(u, x)) continue;
            const int j0 = u * 128;
            if (j0 + 128 > p.nkvb) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (j0 + c * 32 + i >= p.nkvb) x[c][i] = __float_as_uint(-INFINITY);
            }
            float mt0 = -INFINITY, mt1 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    mt0 = fmaxf(mt0, __uint_as_float(x[c][i]));
                    mt1 = fmaxf(mt1, __uint_as_float(x[c][i + 1]));
                }
            const float mn = fmaxf(m, fmaxf(mt0, mt1));
            if (mn != -INFINITY) {
                const float neg = -mn * sl2;
                float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i) a[i & 3] += fast_exp2(fmaf(__uint_as_float(x[c][i]), sl2, neg));
                z = (m == -INFINITY ? 0.f : z * fast_exp2((m - mn) * sl2)) + ((a[0] + a[1]) + (a[2] + a[3]));
                m = mn;
            }
        }
        // ---- merge of the two warpgroups' statistics (every epilogue thread
        // reaches both barriers, whatever its number of tiles)
        if (eg == 1) {
            xch[rr] = m;
            xch[128 + rr] = z;
        }
        epi_bar_sync();
        if (eg == 0) {
            const float m1 = xch[rr], z1 = xch[128 + rr];
            const float mm = fmaxf(m, m1);
            float zz = 0.f;
            if (mm != -INFINITY) {
                if (m != -INFINITY) zz += z * fast_exp2((m - mm) * sl2);
                if (m1 != -INFINITY) zz += z1 * fast_exp2((m1 - mm) * sl2);
            }
            const int qb = ct * SC_QBT + (rr >> 3), c = rr & 7;
            float coef = 0.f, mlog = 0.f;  // a padding slot: weight 0 against 2^(s*L)
            if (qb < p.nqb && c < p.nc && zz > 0.f) {
                const float wc = p.w[(int64_t(bh) * p.nqb + qb) * p.nc + c];
                coef = wc / zz;
                mlog = mm * sl2;
            }
            sm_m[rr] = mlog;
            sm_coef[rr] = coef;
        }
        epi_bar_sync();
        // ---- pass 2: this thread's row is KV block j; columns are centroid rows
        for (int u = NT + ((eg - NT) & 1); u < U; u += 2) {
            uint32_t x[4][32];
            if (!fetch_acc(u, x)) continue;
            const int j = (u - NT) * 128 + rr;
#pragma unroll
            for (int q = 0; q < SC_QBT; ++q) {
                const float4 m0 = *reinterpret_cast<const float4 *>(sm_m + q * 8);
                const float4 m1 = *reinterpret_cast<const float4 *>(sm_m + q * 8 + 4);
                const float4 k0 = *reinterpret_cast<const float4 *>(sm_coef + q * 8);
                const float4 k1 = *reinterpret_cast<const float4 *>(sm_coef + q * 8 + 4);
                const float mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
                const float kk[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
                float sv = 0.f;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    sv = fmaf(kk[c], fast_exp2(fmaf(__uint_as_float(x[q >> 2][(q & 3) * 8 + c]), sl2, -mm[c])), sv);
                const int qb = ct * SC_QBT + q;
                if (j < p.nkvb && qb < p.nqb) p.S[(int64_t(bh) * p.nqb + qb) * p.nkvb + j] = sv;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace abattn
