// Gathered block-sparse attention forward (and the dense reference) on the
// 5th-generation tensor cores.
//
// The AB-Attention news page (hamidun, Arabic), section "three techniques in
// AB-Attention", fine-grained kernel paragraph: KV blocks are only 4 tokens,
// but the kernel gathers the selected blocks by index into full-size
// tensor-core tiles, with no token reordering and no redundant copies; SIP
// paragraph: each selected block counts 1/pi times, realised as a shift of
// the logits inside an ordinary softmax.
//
// One CTA per 128-query block, 192 threads, warp-specialised:
//   warp 0      producer: TMA of the Q tile once; per 128-key tile, the
//               selected KV blocks' K and V rows (one kb-row box per block and
//               64-column half, 128-byte swizzle) and the tile's per-key
//               log2(1/pi) bias into shared memory;
//   warp 1      TMEM owner and MMA issuer: S = Q K^T into one of two TMEM
//               buffers (128 columns each), O += P V into a third (d columns),
//               tcgen05.commit to mbarriers;
//   warps 2..5  softmax: one query row per thread (TMEM lane); logits
//               t = s * scale * log2(e) + log2(1/pi); running max with lazy
//               O rescaling (only when the max grows by more than 2^8);
//               P = exp2(t - m) as bf16 into a swizzled shared-memory tile;
//               the epilogue normalises O and writes O (bf16) and the
//               natural-log LSE.
// The MMA warp issues QK^T of tile t+1 before PV of tile t, so the softmax
// of one tile overlaps the tensor-core work of its neighbours.
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int FWD_THREADS = 192;
constexpr int FWD_NS = 2;  // K/V stages
constexpr uint32_t FWD_TMEM_COLS = 512;
constexpr uint32_t FWD_TMEM_O = 256;  // O accumulator column offset

struct FwdParams {
    const int32_t *counts;
    const int32_t *idx;
    const float *pi_sel;
    int64_t cap;
    __nv_bfloat16 *O;
    float *lse;
    int N;
    int nqb;
    int kb;
    int nkvb;
    float scale_log2;
};

template <int HD>
struct FwdLayout {
    static constexpr int HALVES = HD / 64;
    static constexpr int TILE = HALVES * 16384;  // 128 rows x HD bf16, per 64-col half 16 KB
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + TILE;
    static constexpr int V_OFF = K_OFF + FWD_NS * TILE;
    static constexpr int P_OFF = V_OFF + FWD_NS * TILE;
    static constexpr int BIAS_OFF = P_OFF + 32768;
    static constexpr int BAR_OFF = BIAS_OFF + FWD_NS * 128 * 4;
    static constexpr int NBARS = 1 + 2 * FWD_NS + 6;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
};

// Waits without looking at the abort flag (used to drain in-flight copies
// before the CTA exits); bounded like mbar_wait.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity) {
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) { raise_error(kErrTimeout); return; }
    }
}

template <int HD, bool DENSE>
__global__ void __launch_bounds__(FWD_THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using L = FwdLayout<HD>;
    extern __shared__ uint8_t fwd_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(fwd_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::Q_OFF;
    uint8_t *sK = smem + L::K_OFF;
    uint8_t *sV = smem + L::V_OFF;
    uint8_t *sP = smem + L::P_OFF;
    float *sBias = reinterpret_cast<float *>(smem + L::BIAS_OFF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *q_full = bars;
    uint64_t *kv_full = bars + 1;
    uint64_t *kv_empty = bars + 1 + FWD_NS;
    uint64_t *s_full = bars + 1 + 2 * FWD_NS;
    uint64_t *s_free = s_full + 2;
    uint64_t *p_full = s_free + 2;
    uint64_t *pv_done = p_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x;
    const int bh = row / p.nqb, qb = row % p.nqb;
    const int q0 = qb * 128;

    int cnt = 0, T = 0;
    if (DENSE) {
        T = (p.N + 127) / 128;
    } else {
        int64_t c = p.counts[row];
        c = c < 0 ? 0 : (c > p.cap ? p.cap : c);
        cnt = int(c);
        T = int((int64_t(cnt) * p.kb + 127) / 128);
    }

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < FWD_NS; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 4);
        }
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, FWD_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        int issued = 0;
        if (T > 0) {
            if (lane == 0) {
                mbar_arrive_expect_tx(q_full, 128 * HD * 2);
#pragma unroll
                for (int h = 0; h < L::HALVES; ++h) tma_load_3d(sQ + h * 16384, &tmQ, q_full, h * 64, q0, bh);
            }
            const int32_t *ridx = DENSE ? nullptr : p.idx + int64_t(row) * p.cap;
            const float *rpi = DENSE ? nullptr : p.pi_sel + int64_t(row) * p.cap;
            const int spt = DENSE ? 1 : 128 / p.kb;  // KV blocks per 128-key tile
            int fill_blk = 0;                       // a valid block to load into padding slots
            if (!DENSE) {
                const int b0 = ridx[0];
                fill_blk = (b0 >= 0 && b0 < p.nkvb) ? b0 : 0;
            }
            for (int t = 0; t < T; ++t) {
                const int s = t % FWD_NS;
                if (t >= FWD_NS && !mbar_wait(&kv_empty[s], ((t / FWD_NS) - 1) & 1, abort_flag)) break;
                // per-key bias of this tile: log2(1/pi) of the key's block, -inf if absent
                float bv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int pos = lane * 4 + i;
                    if (DENSE) {
                        bv[i] = (t * 128 + pos < p.N) ? 0.f : -INFINITY;
                    } else {
                        const int slot = t * spt + pos / p.kb;
                        bv[i] = -INFINITY;
                        if (slot < cnt) {
                            const int blk = ridx[slot];
                            const float pi = rpi[slot];
                            if (blk < 0 || blk >= p.nkvb || !(pi > 0.f)) {
                                raise_error(kErrBounds);
                            } else {
                                const int key = blk * p.kb + pos % p.kb;
                                if (key < p.N) bv[i] = -log2f(pi);
                            }
                        }
                    }
                }
                *reinterpret_cast<float4 *>(sBias + s * 128 + lane * 4) = make_float4(bv[0], bv[1], bv[2], bv[3]);
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(&kv_full[s], 2 * 128 * HD * 2);
                __syncwarp();
                uint8_t *dK = sK + s * L::TILE;
                uint8_t *dV = sV + s * L::TILE;
                if (DENSE) {
                    if (lane == 0) {
#pragma unroll
                        for (int h = 0; h < L::HALVES; ++h) {
                            tma_load_3d(dK + h * 16384, &tmK, &kv_full[s], h * 64, t * 128, bh);
                            tma_load_3d(dV + h * 16384, &tmV, &kv_full[s], h * 64, t * 128, bh);
                        }
                    }
                } else {
                    for (int q = lane; q < spt; q += 32) {
                        const int slot = t * spt + q;
                        int blk = slot < cnt ? ridx[slot] : fill_blk;
                        if (blk < 0 || blk >= p.nkvb) blk = fill_blk;
                        const int r0 = blk * p.kb;
                        const int off = q * p.kb * 128;  // kb rows of 128 bytes per half
#pragma unroll
                        for (int h = 0; h < L::HALVES; ++h) {
                            tma_load_3d(dK + h * 16384 + off, &tmK, &kv_full[s], h * 64, r0, bh);
                            tma_load_3d(dV + h * 16384 + off, &tmV, &kv_full[s], h * 64, r0, bh);
                        }
                    }
                }
                ++issued;
            }
            // drain: every issued copy lands before the CTA may exit
            if (*abort_flag) {
                if (lane == 0) {
                    mbar_drain(q_full, 0);
                    for (int t = issued - FWD_NS < 0 ? 0 : issued - FWD_NS; t < issued; ++t)
                        mbar_drain(&kv_full[t % FWD_NS], (t / FWD_NS) & 1);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && T > 0) {
            constexpr uint32_t idesc_qk = make_idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = make_idesc_bf16(128, HD, 0, 1);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
            bool ok = mbar_wait(q_full, 0, abort_flag);
            auto issue_qk = [&](int t) -> bool {
                const int s = t % FWD_NS, sb = t & 1;
                if (!mbar_wait(&kv_full[s], (t / FWD_NS) & 1, abort_flag)) return false;
                if (t >= 2 && !mbar_wait(&s_free[sb], ((t >> 1) - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t kbase = aK + s * L::TILE;
#pragma unroll
                for (int k = 0; k < HD / 16; ++k) {
                    const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
                    umma_f16_ss(tmem + sb * 128, make_sdesc_sw128(aQ + off, 16, 1024),
                                make_sdesc_sw128(kbase + off, 16, 1024), idesc_qk, k > 0);
                }
                umma_commit(&s_full[sb]);
                return true;
            };
            if (ok) ok = issue_qk(0);
            for (int t = 0; ok && t < T; ++t) {
                if (t + 1 < T && !issue_qk(t + 1)) break;
                if (!mbar_wait(p_full, t & 1, abort_flag)) break;
                tc_fence_after();
                const int s = t % FWD_NS;
                const uint32_t vbase = aV + s * L::TILE;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    umma_f16_ss(tmem + FWD_TMEM_O,
                                make_sdesc_sw128(aP + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                                make_sdesc_sw128(vbase + k * 2048, 16384, 1024), idesc_pv,
                                (t > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&kv_empty[s]);
                umma_commit(pv_done);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int wq = warp & 3;
        const int rr = wq * 32 + lane;
        const uint32_t t_lane = tmem + (uint32_t(wq * 32) << 16);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int t = 0; t < T; ++t) {
            const int s = t % FWD_NS, sb = t & 1;
            if (!mbar_wait(&s_full[sb], (t >> 1) & 1, abort_flag) ||
                !mbar_wait(&kv_full[s], (t / FWD_NS) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t x[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(t_lane + sb * 128 + c * 32, x[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sb]);

            const float *bias = sBias + s * 128;
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 bb = *reinterpret_cast<const float4 *>(bias + c * 32 + i);
                    float v0 = fmaf(__uint_as_float(x[c][i + 0]), p.scale_log2, bb.x);
                    float v1 = fmaf(__uint_as_float(x[c][i + 1]), p.scale_log2, bb.y);
                    float v2 = fmaf(__uint_as_float(x[c][i + 2]), p.scale_log2, bb.z);
                    float v3 = fmaf(__uint_as_float(x[c][i + 3]), p.scale_log2, bb.w);
                    x[c][i + 0] = __float_as_uint(v0);
                    x[c][i + 1] = __float_as_uint(v1);
                    x[c][i + 2] = __float_as_uint(v2);
                    x[c][i + 3] = __float_as_uint(v3);
                    mt = fmaxf(mt, fmaxf(fmaxf(v0, v1), fmaxf(v2, v3)));
                }
            }
            const float m_new = fmaxf(m, mt);
            const bool need = m_new > m + 8.f;
            float alpha = 1.f;
            if (need) {
                alpha = exp2f(m - m_new);
                l *= alpha;
                m = m_new;
            }
            const bool any = __any_sync(0xffffffffu, need);
            const float m_use = (m == -INFINITY) ? 0.f : m;
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float e = exp2f(__uint_as_float(x[c][i]) - m_use);
                    rs += e;
                    x[c][i] = __float_as_uint(e);
                }
            }
            l += rs;
            if (t > 0) {
                if (!mbar_wait(pv_done, (t - 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (any) {
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(t_lane + FWD_TMEM_O + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(t_lane + FWD_TMEM_O + c * 32, o);
                    }
                    tmem_wait_st();
                }
            }
            // P row -> shared memory, K-major 128-byte-swizzled (two 64-key halves)
            uint8_t *prow = sP + (rr >> 3) * 1024 + (rr & 7) * 128;
#pragma unroll
            for (int c8 = 0; c8 < 16; ++c8) {
                const int c = c8 >> 2, i0 = (c8 & 3) * 8;
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(x[c][i0 + 0]), __uint_as_float(x[c][i0 + 1]));
                v.y = pack_bf16x2(__uint_as_float(x[c][i0 + 2]), __uint_as_float(x[c][i0 + 3]));
                v.z = pack_bf16x2(__uint_as_float(x[c][i0 + 4]), __uint_as_float(x[c][i0 + 5]));
                v.w = pack_bf16x2(__uint_as_float(x[c][i0 + 6]), __uint_as_float(x[c][i0 + 7]));
                const int h = c8 >> 3, cc = c8 & 7;
                *reinterpret_cast<uint4 *>(prow + h * 16384 + ((cc ^ (rr & 7)) << 4)) = v;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ------------------------------------------------------------ epilogue
        const int M = min(128, p.N - q0);
        const bool write = rr < M;
        __nv_bfloat16 *orow = p.O + (int64_t(bh) * p.N + q0 + rr) * HD;
        if (ok && T > 0 && mbar_wait(pv_done, (T - 1) & 1, abort_flag)) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(t_lane + FWD_TMEM_O + c * 32, o);
                tmem_wait_ld();
                if (write) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + i) = v;
                    }
                }
            }
            if (write && p.lse != nullptr)
                p.lse[int64_t(bh) * p.N + q0 + rr] =
                    l > 0.f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
        } else if (write && (T == 0 || !ok)) {
#pragma unroll
            for (int i = 0; i < HD; i += 8) *reinterpret_cast<uint4 *>(orow + i) = make_uint4(0, 0, 0, 0);
            if (p.lse != nullptr) p.lse[int64_t(bh) * p.N + q0 + rr] = -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, FWD_TMEM_COLS);
    }
}

}  // namespace abattn
