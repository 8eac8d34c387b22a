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
// shared memory; reductions use warp shuffles; each warp compacts its own
// contiguous segment of the row, so the indices come out in ascending order
// with a single block-wide exchange of per-warp counts.
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int PL_THREADS = 512;
constexpr int PL_WARPS = PL_THREADS / 32;

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
    int wcount[PL_WARPS];   // per-warp selected (or tie) counts
    int wcount2[PL_WARPS];
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

// One CTA per q-block row.  The row's scores (or probabilities) sit in
// shared memory; warp w owns the contiguous segment [seg*w, seg*(w+1)) of
// blocks (seg a multiple of 128), so selections are compacted per warp with
// ballots and only the per-warp counts need a block-wide prefix.
template <int MODE>
__global__ void __launch_bounds__(PL_THREADS) plan_kernel(
    const float *__restrict__ in, int64_t H, int64_t nqb, int64_t nkvb, double Bblk, int64_t k_top,
    uint64_t seed, int64_t cap, int32_t *__restrict__ counts, int32_t *__restrict__ idx_out,
    float *__restrict__ pi_sel, float *__restrict__ pi_out) {
    extern __shared__ float pl_smem[];
    __shared__ PlanScratch sc;
    float *vals = pl_smem;                                                   // [nkvb]
    uint32_t *bits = reinterpret_cast<uint32_t *>(vals + nkvb);              // [ceil(nkvb/32)] flags
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t row = blockIdx.x;
    const int64_t b = row / (H * nqb), h = (row / nqb) % H, qb = row % nqb;
    const float *src = in + row * nkvb;
    const int nwords = int((nkvb + 31) / 32);

    // load (8 independent loads in flight per thread); SIP also counts
    // positive scores and sums them
    int npos_l = 0;
    double sum_l = 0.0;
    for (int64_t j0 = tid; j0 < nkvb; j0 += 8 * PL_THREADS) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t j = j0 + int64_t(u) * PL_THREADS;
            v[u] = j < nkvb ? __ldg(src + j) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int64_t j = j0 + int64_t(u) * PL_THREADS;
            if (j < nkvb) {
                vals[j] = v[u];
                if (MODE == kPlanSip) {
                    npos_l += v[u] > 0.f;
                    sum_l += double(v[u]);
                }
            }
        }
    }
    for (int w = tid; w < nwords; w += PL_THREADS) bits[w] = 0u;  // SIP: capped flags

    if (MODE == kPlanSip) {
        const int npos = block_sum<int>(npos_l, sc.iwarp, &sc.bcast[0]);  // (also orders the loads)
        if (Bblk >= double(npos)) {
            for (int64_t j = tid; j < nkvb; j += PL_THREADS) vals[j] = vals[j] > 0.f ? 1.f : 0.f;
        } else {
            // capping rounds: lambda = (Bblk - |C|) / sum_{j not in C} s_j; C grows by
            // {j : lambda s_j >= 1}; each pass also sums the scores left uncapped
            double rest = block_sum<double>(sum_l, sc.dwarp, &sc.dbcast);
            int64_t ncap = 0;
            double lam = (Bblk - double(ncap)) / rest;
            for (int64_t round = 0; round <= nkvb; ++round) {
                int added_l = 0;
                double rest_l = 0.0;
                for (int64_t j = tid; j < nkvb; j += PL_THREADS) {
                    const int w = int(j >> 5);
                    const uint32_t bit = 1u << (j & 31);
                    if (bits[w] & bit) continue;
                    const double sv = double(vals[j]);
                    if (lam * sv >= 1.0) {
                        atomicOr(&bits[w], bit);
                        ++added_l;
                    } else {
                        rest_l += sv;
                    }
                }
                const int added = block_sum<int>(added_l, sc.iwarp, &sc.bcast[0]);
                if (added == 0) break;
                rest = block_sum<double>(rest_l, sc.dwarp, &sc.dbcast);
                ncap += added;
                lam = (Bblk - double(ncap)) / rest;
            }
            for (int64_t j = tid; j < nkvb; j += PL_THREADS)
                vals[j] = (bits[j >> 5] >> (j & 31)) & 1u ? 1.f : __double2float_rn(lam * double(vals[j]));
        }
        __syncthreads();
        if (pi_out != nullptr)
            for (int64_t j = tid; j < nkvb; j += PL_THREADS) pi_out[row * nkvb + j] = vals[j];
    } else {
        __syncthreads();
    }

    // top-k threshold: radix select on the fp32 bit patterns of the
    // non-negative scores, 8 bits per pass, most significant first
    uint32_t thr = 0;
    int need_eq = 0;
    if (MODE == kPlanTopk && k_top > 0) {
        uint32_t prefix = 0, pmask = 0;
        int kk = int(k_top);
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += PL_THREADS) sc.hist[i] = 0;
            __syncthreads();
            for (int64_t j = tid; j < nkvb; j += PL_THREADS) {
                const uint32_t bv = __float_as_uint(vals[j]);
                if ((bv & pmask) == prefix) atomicAdd(&sc.hist[(bv >> shift) & 255u], 1);
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

    // ---- selection flags and per-warp counts (warp w owns a contiguous segment)
    // Sampled modes keep their take flags as bits (the capping flags are done).
    if (MODE != kPlanTopk) {
        for (int w = tid; w < nwords; w += PL_THREADS) bits[w] = 0u;
        __syncthreads();
    }
    const int64_t seg = ((nkvb + PL_WARPS * 128 - 1) / (PL_WARPS * 128)) * 128;
    const int64_t w0 = int64_t(wid) * seg;
    const int64_t w1 = w0 + seg < nkvb ? w0 + seg : nkvb;
    int nsel_w = 0, neq_w = 0;
    for (int64_t base = w0; base < w1; base += 128) {
        const int64_t j0 = base + 4 * lane;
        uint32_t tk = 0, ek = 0;
        if (MODE == kPlanTopk) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t j = j0 + u;
                const uint32_t bv = j < w1 ? __float_as_uint(vals[j]) : 0u;
                tk |= uint32_t(k_top > 0 && j < w1 && bv > thr) << u;
                ek |= uint32_t(k_top > 0 && j < w1 && bv == thr) << u;
            }
        } else if (j0 < w1) {
            float u4[4];
            row_uniforms(seed, b, h, qb, j0 >> 2, u4);
#pragma unroll
            for (int u = 0; u < 4; ++u) tk |= uint32_t(j0 + u < w1 && u4[u] < vals[j0 + u]) << u;
            if (tk) atomicOr(&bits[j0 >> 5], tk << (j0 & 31));
        }
        nsel_w += __popc(tk);
        neq_w += __popc(ek);
    }
    nsel_w = warp_sum(nsel_w);
    neq_w = warp_sum(neq_w);
    if (lane == 0) {
        sc.wcount[wid] = nsel_w;
        sc.wcount2[wid] = neq_w;
    }
    __syncthreads();
    int64_t pos = 0, eq_rank = 0, total = 0, eq_total = 0;
    for (int w = 0; w < PL_WARPS; ++w) {
        if (w < wid) {
            pos += sc.wcount[w];
            eq_rank += sc.wcount2[w];
        }
        total += sc.wcount[w];
        eq_total += sc.wcount2[w];
    }
    if (MODE == kPlanTopk) {
        // ties at the threshold are taken in ascending index order until k
        const int64_t from_eq = eq_total < need_eq ? eq_total : need_eq;
        pos += eq_rank < need_eq ? eq_rank : need_eq;  // ties of earlier warps taken before us
        total += from_eq;
    }

    // ---- compaction in ascending index order, warp by warp
    for (int64_t base = w0; base < w1; base += 128) {
        const int64_t j0 = base + 4 * lane;
        uint32_t tk = 0;
        if (MODE == kPlanTopk) {
            uint32_t ek = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t j = j0 + u;
                const uint32_t bv = j < w1 ? __float_as_uint(vals[j]) : 0u;
                tk |= uint32_t(k_top > 0 && j < w1 && bv > thr) << u;
                ek |= uint32_t(k_top > 0 && j < w1 && bv == thr) << u;
            }
            const int neq = __popc(ek);
            int incl = neq;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int64_t r = eq_rank + (incl - neq);  // rank of this lane's first tie
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if ((ek >> u) & 1u) {
                    if (r < need_eq) tk |= 1u << u;
                    ++r;
                }
            }
            eq_rank += __shfl_sync(0xffffffffu, incl, 31);
        } else if (j0 < w1) {
            tk = (bits[j0 >> 5] >> (j0 & 31)) & 15u;
        }
        const int nt = __popc(tk);
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int64_t p = pos + (incl - nt);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if ((tk >> u) & 1u) {
                if (p < cap) {
                    idx_out[row * cap + p] = int32_t(j0 + u);
                    pi_sel[row * cap + p] = MODE == kPlanTopk ? 1.f : vals[j0 + u];
                }
                ++p;
            }
        }
        pos += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (tid == 0) {
        if (total > cap) raise_error(kErrOverflow);
        counts[row] = int32_t(total < cap ? total : cap);
    }
}

}  // namespace abattn
