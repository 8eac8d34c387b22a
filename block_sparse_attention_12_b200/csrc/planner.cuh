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
// Capping candidates: blocks whose score is within a factor PL_CAND_ALPHA of
// the first threshold 1 / lambda_0, listed while the row loads (or, for rows
// that sum to less than 0.9, by a first round over the whole row).  The
// rounds test only these while lambda stays below PL_CAND_ALPHA lambda_0 (so
// no other block can reach the threshold); otherwise, or when a warp lists
// more than PL_CAND_W blocks, every round scans the whole row.  On the
// workloads' score rows lambda ends 6 to 22 times above lambda_0.
constexpr int PL_CAND = 2048;
constexpr int PL_CAND_W = PL_CAND / (PL_THREADS / 32);  // per-warp region of the list
constexpr double PL_CAND_ALPHA = 32.0;

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

// Uniforms for blocks 8m .. 8m+7 of row (b, h, qb): counter (m, qb, h, b),
// key (seed, 0); 64-bit word i gives blocks 8m+2i (its high 32-bit half) and
// 8m+2i+1 (its low half), each as the half's top 24 bits times 2^-24.
__device__ __forceinline__ void row_uniforms8(uint64_t seed, int64_t b, int64_t h, int64_t qb,
                                              int64_t m, float (&u)[8]) {
    uint64_t x[4] = {uint64_t(m), uint64_t(qb), uint64_t(h), uint64_t(b)};
    philox4x64_10(x[0], x[1], x[2], x[3], seed, 0ull);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        u[2 * i] = float(uint32_t(x[i] >> 40)) * 5.9604644775390625e-8f;                 // 2^-24
        u[2 * i + 1] = float(uint32_t(x[i] & 0xFFFFFFFFull) >> 8) * 5.9604644775390625e-8f;
    }
}

// vals[j0 .. j0+7] (zero past `end`); two 16-byte shared loads when the
// eight lie inside the row (j0 is a multiple of 8, so they are aligned).
__device__ __forceinline__ void load8(const float *vals, int j0, int end, float (&r)[8]) {
    if (j0 + 8 <= end) {
        const float4 a = *reinterpret_cast<const float4 *>(vals + j0);
        const float4 b = *reinterpret_cast<const float4 *>(vals + j0 + 4);
        r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
        r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
    } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) r[u] = j0 + u < end ? vals[j0 + u] : 0.f;
    }
}

// vals[j0 .. j0+7] = r (only the entries below `end`).
__device__ __forceinline__ void store8(float *vals, int j0, int end, const float (&r)[8]) {
    if (j0 + 8 <= end) {
        *reinterpret_cast<float4 *>(vals + j0) = make_float4(r[0], r[1], r[2], r[3]);
        *reinterpret_cast<float4 *>(vals + j0 + 4) = make_float4(r[4], r[5], r[6], r[7]);
    } else {
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (j0 + u < end) vals[j0 + u] = r[u];
    }
}

struct PlanScratch {
    int iwarp[PL_WARPS];
    double dwarp[PL_WARPS];
    int iwarp2[2][PL_WARPS];
    double dwarp2[2][PL_WARPS];
    int wcount[PL_WARPS];   // per-warp selected (or tie) counts
    int wcount2[PL_WARPS];
    int bcast[4];
    double dbcast;
    int hist[256];
    int wcand[PL_WARPS];      // candidates listed by each warp (may exceed PL_CAND_W)
    uint16_t cand[PL_CAND];   // warp w's candidates at [w * PL_CAND_W, ...)
};

// Block-wide sums of one int and one double in a single exchange, with one
// barrier: the warp partials alternate between two buffers (flipped by
// `parity`), so a round's writes never meet the previous round's reads.
__device__ __forceinline__ void block_sum2(int vi, double vd, PlanScratch &sc, int &parity, int &si, double &sd) {
    vi = warp_sum(vi);
    vd = warp_sum(vd);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) {
        sc.iwarp2[parity][wid] = vi;
        sc.dwarp2[parity][wid] = vd;
    }
    __syncthreads();
    int ti = 0;
    double td = 0.0;
#pragma unroll
    for (int w = 0; w < PL_WARPS; ++w) {
        ti += sc.iwarp2[parity][w];
        td += sc.dwarp2[parity][w];
    }
    si = ti;
    sd = td;
    parity ^= 1;
}

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
// blocks (seg a multiple of 256) and each lane 8 consecutive blocks at a
// time, whose flags (capped, then taken) form one byte of `flags`.  Sampled
// indices are compacted per warp with shuffles; only the per-warp counts
// need a block-wide exchange, so they come out in ascending order.
template <int MODE>
__global__ void __launch_bounds__(PL_THREADS) plan_kernel(
    const float *__restrict__ in, int64_t H, int64_t h_off, int64_t nqb, int64_t nkvb, double Bblk, int64_t k_top,
    uint64_t seed, int64_t cap, int32_t *__restrict__ counts, int32_t *__restrict__ idx_out,
    float *__restrict__ pi_sel, float *__restrict__ pi_out) {
    extern __shared__ float pl_smem[];
    __shared__ PlanScratch sc;
    float *vals = pl_smem;                                                   // [nkvb]
    uint8_t *flags = reinterpret_cast<uint8_t *>(vals + nkvb);               // [ceil(nkvb/32) words]
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t row = blockIdx.x;
    // h is the head's global index (the tensors may hold a slice of a layer's heads)
    const int64_t b = row / (H * nqb), h = (row / nqb) % H + h_off, qb = row % nqb;
    const float *src = in + row * nkvb;
    int32_t *ridx = idx_out + row * cap;
    float *rpis = pi_sel + row * cap;
    const int n = int(nkvb);  // row length (at most kMaxPlanBlocks), 32-bit loop indices below
    const int ncap_out = int(cap);
    const int nbytes = ((n + 31) / 32) * 4;

    // load (8 independent loads in flight per thread); SIP also counts
    // positive scores, sums them and lists the capping candidates: the
    // blocks with s >= 0.9 / (PL_CAND_ALPHA Bblk).  When the row sums to at
    // least 0.9 (scores sum to 1) that bound is below 1 / (PL_CAND_ALPHA
    // lambda_0), so the list holds every block that a lambda up to
    // PL_CAND_ALPHA lambda_0 can cap.
    int npos_l = 0;
    double sum_l = 0.0;
    const float cand_thr = MODE == kPlanSip ? float(0.9 / (PL_CAND_ALPHA * Bblk)) * (1.f - 1e-5f) : 0.f;
    int ncw = 0;  // candidates this warp has listed (warp-uniform)
    uint16_t *wcand_list = sc.cand + wid * PL_CAND_W;
    for (int j0 = tid; j0 - lane < n; j0 += 8 * PL_THREADS) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = j0 + u * PL_THREADS;
            v[u] = j < n ? __ldg(src + j) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = j0 + u * PL_THREADS;
            if (j < n) {
                vals[j] = v[u];
                if (MODE == kPlanSip) {
                    npos_l += v[u] > 0.f;
                    sum_l += double(v[u]);
                }
            }
            if (MODE == kPlanSip) {
                // appended to this warp's region of the list, no atomics
                const bool c = j < n && v[u] >= cand_thr;
                const uint32_t cm = __ballot_sync(0xffffffffu, c);
                const int at = ncw + __popc(cm & ((1u << lane) - 1u));
                if (c && at < PL_CAND_W) wcand_list[at] = uint16_t(j);
                ncw += __popc(cm);
            }
        }
    }
    for (int i = tid; i < nbytes; i += PL_THREADS) flags[i] = 0;
    if (MODE == kPlanSip && lane == 0) sc.wcand[wid] = ncw;

    // this warp's segment; lane works on blocks j0 .. j0+7 of each 256-block step
    const int seg = ((n + PL_WARPS * 256 - 1) / (PL_WARPS * 256)) * 256;
    const int w0 = wid * seg;
    const int w1 = w0 + seg < n ? w0 + seg : n;

    // SIP: after the capping rounds vals still holds the scores; the sampling
    // pass takes pi = 1 for capped blocks (their flag bits) and
    // fp32(lambda s) for the others
    bool pi_from_s = false;
    double lam_final = 0.0;
    if (MODE == kPlanSip) {
        const int npos = block_sum<int>(npos_l, sc.iwarp, &sc.bcast[0]);  // (also orders the loads)
        if (Bblk >= double(npos)) {
            for (int j = tid; j < n; j += PL_THREADS) vals[j] = vals[j] > 0.f ? 1.f : 0.f;
        } else {
            // capping rounds: lambda = (Bblk - |C|) / sum_{j not in C} s_j; C
            // grows by {j : lambda s_j >= 1}, tested exactly in fp64 for the
            // blocks an fp32 product puts near the threshold; the uncapped sum
            // is updated by subtracting the newly capped scores.  Lane-strided
            // walk (conflict-free shared loads); the capped flags of 32
            // consecutive blocks form one word, rebuilt by ballot.
            uint32_t *fw = reinterpret_cast<uint32_t *>(flags);
            double rest = block_sum<double>(sum_l, sc.dwarp, &sc.dbcast);  // (also publishes wcand)
            auto cand_fit = [&]() {
                bool fit = true;
#pragma unroll
                for (int w = 0; w < PL_WARPS; ++w) fit &= sc.wcand[w] <= PL_CAND_W;
                return fit;
            };
            // the load pass's list serves when it is complete and the row sums
            // to at least 0.9; otherwise the first round scans the whole row
            // and lists the candidates itself
            const bool pre_ok = rest >= 0.9 && cand_fit();
            int ncap = 0;
            int rpar = 0;  // buffer parity of block_sum2
            double lam = Bblk / rest;
            const double lam_lim = PL_CAND_ALPHA * lam;
            // one round over the whole row; the first one also collects the candidates
            auto full_round = [&](bool collect, int &added, double &capped) {
                const float near = float(lam) * (1.f + 1e-5f);
                const float cand_near = float(lam_lim) * (1.f + 1e-5f);
                int added_l = 0;
                double capped_l = 0.0;
                int nc = 0;  // candidates this warp has listed (warp-uniform)
                // four words (128 blocks) per step: four independent chains
                for (int j128 = w0; j128 < w1; j128 += 128) {
                    uint32_t word[4];
                    float sv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j = j128 + 32 * q + lane;
                        word[q] = j128 + 32 * q < w1 ? fw[(j128 >> 5) + q] : 0xFFFFFFFFu;
                        sv[q] = j < w1 ? vals[j] : 0.f;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int j = j128 + 32 * q + lane;
                        const bool open = j < w1 && !((word[q] >> lane) & 1u);
                        bool cap_now = false;
                        if (open && sv[q] * near >= 1.f && lam * double(sv[q]) >= 1.0) {
                            cap_now = true;
                            ++added_l;
                            capped_l += double(sv[q]);
                        }
                        const uint32_t nb = __ballot_sync(0xffffffffu, cap_now);
                        if (nb != 0u && lane == 0) fw[(j128 >> 5) + q] = word[q] | nb;
                        if (collect) {
                            const bool c = open && !cap_now && sv[q] * cand_near >= 1.f;
                            const uint32_t cm = __ballot_sync(0xffffffffu, c);
                            const int at = nc + __popc(cm & ((1u << lane) - 1u));
                            if (c && at < PL_CAND_W) wcand_list[at] = uint16_t(j);
                            nc += __popc(cm);
                        }
                    }
                }
                if (collect && lane == 0) sc.wcand[wid] = nc;
                block_sum2(added_l, capped_l, sc, rpar, added, capped);
            };
            // a round over the candidates only, each warp over its own list
            auto cand_round = [&](int &added, double &capped) {
                const float near = float(lam) * (1.f + 1e-5f);
                int added_l = 0;
                double capped_l = 0.0;
                const int cw = sc.wcand[wid];
                for (int i = lane; i < cw; i += 32) {
                    const int j = wcand_list[i];
                    const float sj = vals[j];
                    const uint32_t bit = 1u << (j & 31);
                    if (!(fw[j >> 5] & bit) && sj * near >= 1.f && lam * double(sj) >= 1.0) {
                        atomicOr(&fw[j >> 5], bit);
                        ++added_l;
                        capped_l += double(sj);
                    }
                }
                block_sum2(added_l, capped_l, sc, rpar, added, capped);
            };
            int added;
            double capped;
            bool scan_all;
            if (pre_ok) {
                scan_all = false;
                cand_round(added, capped);
            } else {
                __syncthreads();  // every thread has read wcand before the first round relists
                full_round(true, added, capped);
                scan_all = !cand_fit();  // wcand read after block_sum2's barriers
            }
            while (added != 0) {
                rest -= capped;
                ncap += added;
                lam = (Bblk - double(ncap)) / rest;
                if (lam > lam_lim) scan_all = true;
                if (scan_all) {
                    full_round(false, added, capped);
                } else {
                    cand_round(added, capped);
                }
            }
            pi_from_s = true;
            lam_final = lam;
        }
    }
    __syncthreads();

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
            for (int j = tid; j < n; j += PL_THREADS) {
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

    // ---- pass 1: (SIP) final pi; flags <- taken blocks; per-warp counts
    int nsel_w = 0, neq_w = 0;
    for (int j0 = w0 + 8 * lane; j0 < w1; j0 += 256) {
        uint32_t tk = 0, ek = 0;
        if (MODE == kPlanTopk) {
            float raw[8];
            load8(vals, j0, w1, raw);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u;
                const uint32_t bv = __float_as_uint(raw[u]);
                tk |= uint32_t(k_top > 0 && j < w1 && bv > thr) << u;
                ek |= uint32_t(k_top > 0 && j < w1 && bv == thr) << u;
            }
        } else {
            float pv[8];
            load8(vals, j0, w1, pv);
            if (pi_from_s) {
                // this lane's 8 blocks: pi from the capped bits and lambda
                const uint32_t cb = flags[j0 >> 3];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    pv[u] = ((cb >> u) & 1u) ? 1.f : __double2float_rn(lam_final * double(pv[u]));
                store8(vals, j0, w1, pv);
            }
            float u8[8];
            row_uniforms8(seed, b, h, qb, j0 >> 3, u8);
#pragma unroll
            for (int u = 0; u < 8; ++u) tk |= uint32_t(j0 + u < w1 && u8[u] < pv[u]) << u;
            flags[j0 >> 3] = uint8_t(tk);
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
    if (MODE == kPlanSip && pi_out != nullptr)
        for (int j = tid; j < n; j += PL_THREADS) pi_out[row * nkvb + j] = vals[j];
    int pos = 0, eq_rank = 0, total = 0, eq_total = 0;
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
        pos += eq_rank < need_eq ? eq_rank : need_eq;  // ties of earlier warps taken before ours
        total += eq_total < need_eq ? eq_total : need_eq;
    }

    // ---- pass 2: compaction in ascending index order within the warp's segment
    for (int j0 = w0 + 8 * lane; j0 < w1; j0 += 256) {
        uint32_t tk = 0;
        if (MODE == kPlanTopk) {
            uint32_t ek = 0;
            float raw[8];
            load8(vals, j0, w1, raw);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u;
                const uint32_t bv = __float_as_uint(raw[u]);
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
            int r = eq_rank + (incl - neq);  // rank of this lane's first tie
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if ((ek >> u) & 1u) {
                    if (r < need_eq) tk |= 1u << u;
                    ++r;
                }
            }
            eq_rank += __shfl_sync(0xffffffffu, incl, 31);
        } else {
            tk = flags[j0 >> 3];
        }
        const int nt = __popc(tk);
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int p = pos + (incl - nt);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if ((tk >> u) & 1u) {
                if (p < ncap_out) {
                    ridx[p] = j0 + u;
                    rpis[p] = MODE == kPlanTopk ? 1.f : vals[j0 + u];
                }
                ++p;
            }
        }
        pos += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (tid == 0) {
        if (total > ncap_out) raise_error(kErrOverflow);
        counts[row] = total < ncap_out ? total : ncap_out;
    }
}

}  // namespace abattn
