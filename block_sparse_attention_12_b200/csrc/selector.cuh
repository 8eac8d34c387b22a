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
// One CTA (128 threads, one warpgroup) per q-block; both Lloyd steps run on
// the tensor cores, with the block's queries staged once by TMA in the
// 128-byte-swizzled K-major layout:
//   assignment: D_a[query][c] = q . c for 16 centroid slots (8 used); the
//               queries are exactly bf16 and the fp32 centroids are split
//               into a bf16 pair hi + lo, stacked as the 32 rows of one B
//               operand (rows 0..15 hi, 16..31 lo), so each k-step is one
//               N = 32 MMA and columns c and 16 + c of the fp32 TMEM
//               accumulator hold q . c_hi and q . c_lo; thread i (TMEM lane
//               i) adds the two and takes argmin_c |c|^2 - 2 q.c (the same
//               argmin as |q - c|^2), ties to the lower index;
//   update:     D_u[k][c] = sum of dimension k over cluster c's members as
//               Q^T [d x 128] times a one-hot [128 x 16] assignment matrix;
//               the same shared-memory tile of Q is read as an MN-major
//               operand; thread k divides by the member counts (ballots).
// Products are exact (bf16 x bf16, or x 0/1) and accumulate in fp32.  An
// empty cluster keeps its centroid; a fixed point (no label moved) ends the
// iterations early with the same result.  For d = 64 the tile's second
// 64-column half is zero, so the update still has M = 128 rows.  Thread k
// keeps the fp32 centroids of dimension k in registers, and the one-hot
// operand takes the rows of the centroids' lo part (the assignment has read
// those before the one-hot is written, the update has read the one-hot before
// the new centroids are), so five CTAs fit an SM.  The kernel is bound by the
// latency of its two dependent MMA round trips per iteration; the stacked
// hi/lo operand halves the first one (8 MMAs a k-sweep instead of 16).
constexpr int KM_THREADS = 128;

struct KmLayout {
    static constexpr int Q_OFF = 0;          // [2 halves][128 rows][128 B]
    static constexpr int C_HALF = 4096;      // bytes between the 64-column halves of the centroid operand
    static constexpr int CHI_OFF = 32768;    // [2 halves][32 rows][128 B]: rows 0..15 hi, 16..31 lo
    static constexpr int CLO_OFF = CHI_OFF + 2048;  // rows 16..31 of each half
    static constexpr int OH_OFF = CLO_OFF;   // or the one-hot [2 query halves][16 rows][128 B] in those rows
    static constexpr int CN_OFF = CHI_OFF + 2 * C_HALF;  // |c|^2 [8], partials [4][8]
    static constexpr int INT_OFF = CN_OFF + 40 * 4;      // lab[128], cnt[8], wcnt[4][8]
    static constexpr int BAR_OFF = INT_OFF + (128 + 8 + 32) * 4;  // q_bar, mma_bar
    static constexpr int MISC_OFF = BAR_OFF + 16;         // tmem slot
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;
};

// Byte offset of element (r, k) in a 128-byte-swizzled K-major tile whose
// 64-column halves are `hs` bytes apart (rows of 128 bytes).
__device__ __forceinline__ uint32_t sw128_off(int r, int k, uint32_t hs) {
    const int cc = k & 63;
    return uint32_t(k >> 6) * hs + uint32_t(r) * 128u + (uint32_t(((cc >> 3) ^ (r & 7))) << 4) + uint32_t(cc & 7) * 2u;
}

template <int D>
__global__ void __launch_bounds__(KM_THREADS, 5) kmeans_kernel(
    const __grid_constant__ CUtensorMap tmQ, int64_t N, int64_t nqb, int nc, int iters,
    float *__restrict__ Cout, float *__restrict__ wout, int32_t *__restrict__ labels_out,
    __nv_bfloat16 *__restrict__ Chi, __nv_bfloat16 *__restrict__ Clo) {
    using L = KmLayout;
    extern __shared__ uint8_t km_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(km_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::Q_OFF;
    uint8_t *sChi = smem + L::CHI_OFF, *sClo = smem + L::CLO_OFF, *sOH = smem + L::OH_OFF;
    float *cn = reinterpret_cast<float *>(smem + L::CN_OFF);   // [8]
    float *cn_part = cn + 8;                                    // [4][8]
    int *lab = reinterpret_cast<int *>(smem + L::INT_OFF);     // [128]
    int *cnt_s = lab + 128;                                     // [8]
    int *wcnt = cnt_s + 8;                                      // [4][8]
    uint64_t *q_bar = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *mma_bar = q_bar + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 4);

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t row = blockIdx.x;
    const int64_t bh = row / nqb, qb = row % nqb;
    const int q0 = int(qb * 128);
    const int M = int(N - q0 < 128 ? N - q0 : 128);

    if (wid == 0) {
        tmem_alloc(tmem_slot, 64);  // D_a: columns [0, 32), D_u: [32, 48)
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(q_bar, 1);
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // zero the centroid and one-hot operands (their unused rows stay zero)
    // and, for d = 64, the tile's second half
    {
        uint4 *z = reinterpret_cast<uint4 *>(smem + L::CHI_OFF);
        for (int e = tid; e < (2 * L::C_HALF) / 16; e += KM_THREADS) z[e] = make_uint4(0, 0, 0, 0);
        if (D == 64) {
            uint4 *zq = reinterpret_cast<uint4 *>(sQ + 16384);
            for (int e = tid; e < 16384 / 16; e += KM_THREADS) zq[e] = make_uint4(0, 0, 0, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_lane = tmem + (uint32_t(wid * 32) << 16);

    bool ok = true;
    if (tid == 0) {
        mbar_arrive_expect_tx(q_bar, 128 * D * 2);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) tma_load_3d(sQ + h * 16384, &tmQ, q_bar, h * 64, q0, int(bh));
    }
    ok = mbar_wait(q_bar, 0, abort_flag);
    ok = __syncthreads_and(ok) != 0;

    auto qval = [&](int r, int k) {
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sQ + sw128_off(r, k, 16384)));
    };
    float cs[8];  // thread k < D: the fp32 centroids' dimension k
    // centroid c of dimension k (thread k) into cs and the bf16 hi/lo operand
    // tiles; returns its square for |c|^2
    auto set_centroid = [&](int c, int k, float v) {
        cs[c] = v;
        __nv_bfloat16 hi, lo;
        split_bf16(v, hi, lo);
        const uint32_t o = sw128_off(c, k, L::C_HALF);
        *reinterpret_cast<__nv_bfloat16 *>(sChi + o) = hi;
        *reinterpret_cast<__nv_bfloat16 *>(sClo + o) = lo;
        return v * v;
    };
    // |c|^2 from each thread's dimension: warp sums, then across the warps
    auto centroid_norms = [&](const float (&part)[8]) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float v = warp_sum(part[c]);
            if (lane == 0) cn_part[wid * 8 + c] = v;
        }
        __syncthreads();
        if (tid < 8) cn[tid] = (cn_part[tid] + cn_part[8 + tid]) + (cn_part[16 + tid] + cn_part[24 + tid]);
    };

    // init: centroid c = query floor(c*M/nc); unused centroid slots are zero
    {
        float part[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float v = (tid < D && c < nc) ? qval((c * M) / nc, tid < D ? tid : 0) : 0.f;
            part[c] = tid < D ? set_centroid(c, tid, v) : 0.f;
        }
        fence_proxy_async_smem();
        centroid_norms(part);
    }
    if (tid < 8) cnt_s[tid] = 0;

    constexpr uint32_t idesc_a = make_idesc_bf16(128, 32, 0, 0);  // Q . [C_hi; C_lo]^T
    constexpr uint32_t idesc_u = make_idesc_bf16(128, 16, 1, 0);  // Q^T . onehot, A MN-major
    uint32_t phase = 0;
    for (int it = 0; ok && it < iters; ++it) {
        __syncthreads();  // centroid operands, |c|^2 and the last one-hot reads are done
        if (tid == 0) {
            tc_fence_after();
            const uint32_t q_lo = sdesc_lo(smem_u32(sQ), 16);
            const uint32_t c_lo = sdesc_lo(smem_u32(sChi), 16);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint32_t qo = ((k >> 2) * 16384 + (k & 3) * 32) >> 4,
                               co = ((k >> 2) * L::C_HALF + (k & 3) * 32) >> 4;
                umma_ss_lo(tmem, q_lo + qo, c_lo + co, idesc_a, k > 0 ? 1u : 0u);
            }
            umma_commit(mma_bar);
        }
        ok = mbar_wait(mma_bar, phase, abort_flag);
        phase ^= 1;
        tc_fence_after();
        uint32_t a32[32];
        tmem_ld32(t_lane, a32);
        tmem_wait_ld();
        int best = 0;
        {
            // q . c = (q . c_hi) + (q . c_lo), columns c and 16 + c
            float bd = fmaf(-2.f, __uint_as_float(a32[0]) + __uint_as_float(a32[16]), cn[0]);
#pragma unroll
            for (int c = 1; c < 8; ++c) {
                const float v = fmaf(-2.f, __uint_as_float(a32[c]) + __uint_as_float(a32[16 + c]), cn[c]);
                if (c < nc && v < bd) { bd = v; best = c; }
            }
        }
        // a fixed point (no label changed) repeats itself in every remaining
        // iteration: stop, the result is the same as running them all
        const bool moved = tid < M && (it == 0 || lab[tid] != best);
        const int flags = __syncthreads_or((moved ? 1 : 0) | (ok ? 0 : 2));
        if (flags & 2) { ok = false; break; }
        if (it > 0 && !(flags & 1)) break;
        if (tid < M) lab[tid] = best;
        // member counts and the one-hot operand (column tid)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const unsigned m = __ballot_sync(0xffffffffu, tid < M && best == c);
            if (lane == 0) wcnt[wid * 8 + c] = __popc(m);
            const __nv_bfloat16 one = __float2bfloat16(tid < M && best == c ? 1.f : 0.f);
            *reinterpret_cast<__nv_bfloat16 *>(sOH + sw128_off(c, tid, L::C_HALF)) = one;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid < 8) cnt_s[tid] = wcnt[tid] + wcnt[8 + tid] + wcnt[16 + tid] + wcnt[24 + tid];
        if (tid == 0) {
            tc_fence_after();
            const uint32_t qt_lo = sdesc_lo(smem_u32(sQ), 16384), oh_lo = sdesc_lo(smem_u32(sOH), 16);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t oo = ((k >> 2) * L::C_HALF + (k & 3) * 32) >> 4;
                umma_ss_lo(tmem + 32, qt_lo + k * (2048 >> 4), oh_lo + oo, idesc_u, k > 0 ? 1u : 0u);
            }
            umma_commit(mma_bar);
        }
        ok = mbar_wait(mma_bar, phase, abort_flag);
        phase ^= 1;
        tc_fence_after();
        uint32_t s16[16];
        tmem_ld16(t_lane + 32, s16);
        tmem_wait_ld();
        ok = __syncthreads_and(ok) != 0;  // (also publishes cnt_s)
        if (!ok) break;
        float part[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            part[c] = 0.f;
            if (tid < D) {
                const int n = cnt_s[c];
                const float v = (c < nc && n > 0) ? __uint_as_float(s16[c]) / float(n) : cs[c];
                part[c] = set_centroid(c, tid, v);
            }
        }
        fence_proxy_async_smem();
        centroid_norms(part);
    }
    __syncthreads();

    if (tid < D) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            if (Cout != nullptr && c < nc) Cout[(row * nc + c) * D + tid] = cs[c];
            if (Chi != nullptr)  // [rows][8][D], clusters past nc zero
                split_bf16(c < nc ? cs[c] : 0.f, Chi[(row * 8 + c) * D + tid], Clo[(row * 8 + c) * D + tid]);
        }
    }
    if (tid < nc) wout[row * nc + tid] = iters > 0 ? float(cnt_s[tid]) / float(M) : 1.f / float(nc);
    if (labels_out != nullptr)
        labels_out[row * 128 + tid] = (iters > 0 && tid < M) ? lab[tid] : -1;

    tc_fence_before();
    __syncthreads();
    if (wid == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
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
