// SIP planner kernels: inclusion probabilities, counter-based Poisson
// sampling and per-row compaction; plus the top-k truncation baseline.
//
// Follows the SIP bullet of the AB-Attention summary page (edumints, section
// "AB-Attention ve Uc Temel Yeniligi") and the SIP paragraph of the news page
// (hamidun, section "three techniques in AB-Attention"): a block enters the
// sample with probability proportional to its score, the most important
// blocks always enter, and each selected block is later weighted by the
// inverse of its probability.  Top-k truncation is the weakness described in
// the "where earlier sparse schemes fail" section of the news page.
//
// One CTA per q-block row; the row's scores (or probabilities) live in
// shared memory; reductions use warp shuffles and a block-wide scan
// compacts the selected indices in ascending order.
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int PL_THREADS = 512;
constexpr int PL_WARPS = PL_THREADS / 32;
constexpr int PL_ITEMS = 4;  // consecutive blocks per thread per chunk (one Philox block)
constexpr int PL_CHUNK = PL_THREADS * PL_ITEMS;

enum PlanMode : int { kPlanSip = 0, kPlanTopk = 1, kPlanFromPi = 2 };

// Philox4x64 with 10 rounds (Salmon, Moraes, Dror and Shaw, SC'11): per round,
// two 64x64->128-bit products of words 0 and 2 with fixed odd multipliers;
// the high halves are xored with words 1 / 3 and the round key, the low
// halves move to words 1 / 3; the key advances by two Weyl increments.
__device__ __forceinline__ void philox4x64_10(uint64_t &x0, uint64_t &x1, uint64_t &x2, uint64_t &x3,
                                              uint64_t k0, uint64_t k1) {
    constexpr uint64_t kMulA = 0xD2E7470EE14C6C93ull, kMulB = 0xCA5A826395121157ull;
    constexpr uint64_t kWeylA = 0x9E3779B97F4A7C15ull, kWeylB = 0xBB67AE8584CAA73Bull;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t hA = __umul64hi(kMulA, x0), lA = kMulA * x0;
        const uint64_t hB = __umul64hi(kMulB, x2), lB = kMulB * x2;
        const uint64_t n0 = hB ^ x1 ^ k0, n2 = hA ^ x3 ^ k1;
        x0 = n0;
        x1 = lB;
        x2 = n2;
        x3 = lA;
        k0 += kWeylA;
        k1 += kWeylB;
    }
}

// Uniforms for blocks 4m .. 4m+3 of row (b, h, qb): counter (m, qb, h, b),
// key (seed, 0); each 64-bit word gives its top 24 bits times 2^-24.
__device__ __forceinline__ void row_uniforms(uint64_t seed, int64_t b, int64_t h, int64_t qb,
                                             int64_t m, float (&u)[4]) {
    uint64_t x0 = uint64_t(m), x1 = uint64_t(qb), x2 = uint64_t(h), x3 = uint64_t(b);
    philox4x64_10(x0, x1, x2, x3, seed, 0ull);
    u[0] = float(uint32_t(x0 >> 40)) * 5.9604644775390625e-8f;  // 2^-24
    u[1] = float(uint32_t(x1 >> 40)) * 5.9604644775390625e-8f;
    u[2] = float(uint32_t(x2 >> 40)) * 5.9604644775390625e-8f;
    u[3] = float(uint32_t(x3 >> 40)) * 5.9604644775390625e-8f;
}

struct PlanScratch {
    int iwarp[PL_WARPS];
    double dwarp[PL_WARPS];
    int bcast[4];
    double dbcast;
    int hist[256];
};

// Block-wide sum; every thread gets the result.
template <typename T>
__device__ __forceinline__ T block_sum(T v, T *warp_buf, T *bcast) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) warp_buf[wid] = v;
    __syncthreads();
    if (wid == 0) {
        T x = lane < PL_WARPS ? warp_buf[lane] : T(0);
        x = warp_sum(x);
        if (lane == 0) *bcast = x;
    }
    __syncthreads();
    const T r = *bcast;
    __syncthreads();
    return r;
}

// Block-wide exclusive scan of per-thread counts; *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int *warp_buf, int *total_out, int &total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_buf[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int x = lane < PL_WARPS ? warp_buf[lane] : 0;
        int xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) xi += y;
        }
        if (lane < PL_WARPS) warp_buf[lane] = xi - x;  // exclusive warp offsets
        if (lane == PL_WARPS - 1) *total_out = xi;
    }
    __syncthreads();
    const int r = warp_buf[wid] + incl - v;
    total = *total_out;
    __syncthreads();
    return r;
}

template <int MODE>
__global__ void __launch_bounds__(PL_THREADS) plan_kernel(
    const float *__restrict__ in, int64_t H, int64_t nqb, int64_t nkvb, double Bblk, int64_t k_top,
    uint64_t seed, int64_t cap, int32_t *__restrict__ counts, int32_t *__restrict__ idx_out,
    float *__restrict__ pi_sel, float *__restrict__ pi_out) {
    extern __shared__ float pl_smem[];
    __shared__ PlanScratch sc;
    float *vals = pl_smem;                                                   // [nkvb]
    unsigned char *capped = reinterpret_cast<unsigned char *>(vals + nkvb);  // [nkvb] (SIP)
    const int tid = threadIdx.x;
    const int64_t row = blockIdx.x;
    const int64_t b = row / (H * nqb), h = (row / nqb) % H, qb = row % nqb;
    const float *src = in + row * nkvb;
    for (int64_t j = tid; j < nkvb; j += PL_THREADS) vals[j] = __ldg(src + j);
    __syncthreads();

    if (MODE == kPlanSip) {
        int npos_l = 0;
        for (int64_t j = tid; j < nkvb; j += PL_THREADS) npos_l += vals[j] > 0.f;
        const int npos = block_sum<int>(npos_l, sc.iwarp, &sc.bcast[0]);
        if (Bblk >= double(npos)) {
            for (int64_t j = tid; j < nkvb; j += PL_THREADS) vals[j] = vals[j] > 0.f ? 1.f : 0.f;
        } else {
            for (int64_t j = tid; j < nkvb; j += PL_THREADS) capped[j] = 0;
            __syncthreads();
            int64_t ncap = 0;
            double lam = 0.0;
            for (int64_t round = 0; round <= nkvb; ++round) {
                double rest_l = 0.0;
                for (int64_t j = tid; j < nkvb; j += PL_THREADS)
                    if (!capped[j]) rest_l += double(vals[j]);
                const double rest = block_sum<double>(rest_l, sc.dwarp, &sc.dbcast);
                lam = (Bblk - double(ncap)) / rest;
                int added_l = 0;
                for (int64_t j = tid; j < nkvb; j += PL_THREADS)
                    if (!capped[j] && lam * double(vals[j]) >= 1.0) { capped[j] = 1; ++added_l; }
                const int added = block_sum<int>(added_l, sc.iwarp, &sc.bcast[0]);
                if (added == 0) break;
                ncap += added;
            }
            for (int64_t j = tid; j < nkvb; j += PL_THREADS)
                vals[j] = capped[j] ? 1.f : __double2float_rn(lam * double(vals[j]));
        }
        __syncthreads();
        if (pi_out != nullptr)
            for (int64_t j = tid; j < nkvb; j += PL_THREADS) pi_out[row * nkvb + j] = vals[j];
    }

    // threshold of the top-k (radix select on the fp32 bit patterns of the
    // non-negative scores, 8 bits per pass, most significant first)
    uint32_t thr = 0;
    int need_eq = 0;
    if (MODE == kPlanTopk) {
        uint32_t prefix = 0, pmask = 0;
        int kk = int(k_top);
        if (kk > 0) {
            for (int shift = 24; shift >= 0; shift -= 8) {
                for (int i = tid; i < 256; i += PL_THREADS) sc.hist[i] = 0;
                __syncthreads();
                for (int64_t j = tid; j < nkvb; j += PL_THREADS) {
                    const uint32_t bits = __float_as_uint(vals[j]);
                    if ((bits & pmask) == prefix) atomicAdd(&sc.hist[(bits >> shift) & 255u], 1);
                }
                __syncthreads();
                if (tid == 0) {
                    int cum = 0, digit = 0;
                    for (int dg = 255; dg >= 0; --dg) {
                        if (cum + sc.hist[dg] >= kk) { digit = dg; break; }
                        cum += sc.hist[dg];
                    }
                    sc.bcast[1] = digit;
                    sc.bcast[2] = kk - cum;
                }
                __syncthreads();
                prefix |= uint32_t(sc.bcast[1]) << shift;
                pmask |= 255u << shift;
                kk = sc.bcast[2];
                __syncthreads();
            }
            thr = prefix;
            need_eq = kk;
        }
    }

    // sampling / selection and compaction in ascending index order
    int64_t base = 0, eq_base = 0;
    for (int64_t c0 = 0; c0 < nkvb; c0 += PL_CHUNK) {
        const int64_t j0 = c0 + int64_t(tid) * PL_ITEMS;
        bool take[PL_ITEMS];
        if (MODE == kPlanTopk) {
            bool gt[PL_ITEMS], eq[PL_ITEMS];
            int neq = 0;
#pragma unroll
            for (int u = 0; u < PL_ITEMS; ++u) {
                const int64_t j = j0 + u;
                const uint32_t bits = j < nkvb ? __float_as_uint(vals[j]) : 0u;
                gt[u] = j < nkvb && k_top > 0 && bits > thr;
                eq[u] = j < nkvb && k_top > 0 && bits == thr;
                neq += eq[u];
            }
            int eq_tot;
            const int eq_excl = block_excl_scan(neq, sc.iwarp, &sc.bcast[3], eq_tot);
            int64_t rank = eq_base + eq_excl;
#pragma unroll
            for (int u = 0; u < PL_ITEMS; ++u) {
                take[u] = gt[u] || (eq[u] && rank < need_eq);
                rank += eq[u];
            }
            eq_base += eq_tot;
        } else {
            float u4[4];
            row_uniforms(seed, b, h, qb, j0 >> 2, u4);
#pragma unroll
            for (int u = 0; u < PL_ITEMS; ++u) {
                const int64_t j = j0 + u;
                take[u] = j < nkvb && u4[u] < vals[j];
            }
        }
        int nt = 0;
#pragma unroll
        for (int u = 0; u < PL_ITEMS; ++u) nt += take[u];
        int tot;
        const int excl = block_excl_scan(nt, sc.iwarp, &sc.bcast[3], tot);
        int64_t pos = base + excl;
#pragma unroll
        for (int u = 0; u < PL_ITEMS; ++u) {
            if (take[u]) {
                if (pos < cap) {
                    idx_out[row * cap + pos] = int32_t(j0 + u);
                    pi_sel[row * cap + pos] = MODE == kPlanTopk ? 1.f : vals[j0 + u];
                }
                ++pos;
            }
        }
        base += tot;
    }
    if (tid == 0) {
        if (base > cap) raise_error(kErrOverflow);
        counts[row] = int32_t(base < cap ? base : cap);
    }
}

}  // namespace abattn
