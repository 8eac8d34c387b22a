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
// One CTA per 128-query block, 512 threads in four warpgroups:
//   warps 0..7  softmax, two warpgroups (setmaxnreg raised): warpgroup g takes
//               the KV tiles t = g, g+2, g+4, ... with its own S buffer and
//               its own O accumulator in TMEM, so the two run side by side
//               and hide each other's latencies.  One query row per thread
//               (TMEM lane); logits t = s * scale * log2(e) + log2(1/pi);
//               running max with lazy O rescaling (only when the max grows by
//               more than 2^32); P = exp2(t - m), packed to bf16 as it is
//               computed and stored back to TMEM over the first 64 columns of
//               its S buffer (the dense kernel hands keys 0..63 of P to the
//               MMA warp before it computes the exponentials of keys 64..127,
//               so that half of PV starts early).  At the end the two partial
//               softmaxes are merged
//               (max, sums, O) and O (bf16) and the natural-log LSE are written;
//   warps 8..11, 13..15  producers (setmaxnreg lowered): warp 8 loads the Q
//               tile once by TMA.  Sparse kernel: the 32 quads of 4 rows of a
//               128-key tile are gathered with cp.async, 16 bytes per lane,
//               into the 128-byte-swizzled layout (warp w takes quads w,
//               w+7, ...), with the bias log2(1/pi) of each quad; dense kernel:
//               one TMA box of 32 rows per 64-column half and tensor.  K and V
//               share a ring of 3 stages.  The lanes prefetch the plan entries
//               two tiles ahead;
//   warp 12     TMEM owner and MMA issuer (setmaxnreg lowered): S = Q K^T
//               (both operands in shared memory) into S buffer t % 2;
//               O_{t%2} += P V with P read from TMEM and V from shared memory;
//               tcgen05.commit to mbarriers.
// TMEM: S0 [0,128), S1 [128,256), O_even [256,256+d), O_odd [384,384+d).
// The MMA warp issues QK^T of tile t+1 before PV of tile t; MMAs issued by
// one thread run in order, so QK^T of tile t+2 cannot overwrite P(t) before
// PV(t) has read it.
#pragma once

#include "common.cuh"

namespace abattn {

constexpr int FWD_THREADS = 512;
// setmaxnreg split (per thread): two softmax warpgroups take FWD_SOFTMAX_REGS,
// the producer and MMA warpgroups FWD_OTHER_REGS; 2*128*S + 2*128*O must not
// exceed the 512 x 128 registers the CTA launches with.
#ifndef ABATTN_FWD_SOFTMAX_REGS
#define ABATTN_FWD_SOFTMAX_REGS 200
#endif
#ifndef ABATTN_FWD_OTHER_REGS
#define ABATTN_FWD_OTHER_REGS 56
#endif
constexpr int FWD_SOFTMAX_REGS = ABATTN_FWD_SOFTMAX_REGS;
constexpr int FWD_OTHER_REGS = ABATTN_FWD_OTHER_REGS;
static_assert(2 * 128 * FWD_SOFTMAX_REGS + 2 * 128 * FWD_OTHER_REGS <= FWD_THREADS * 128,
              "setmaxnreg split exceeds the launch register budget");
constexpr int FWD_PRODUCERS = 7;  // producer warps (8..11, 13..15); producer w gathers the quads q = w mod 7 of a tile
constexpr int FWD_NS = 3;  // K/V stages
// O and the row sum are rescaled only when a tile's max exceeds the running
// reference max by more than this (log2 units).  Probabilities then stay
// below 2^FWD_RESCALE_LOG2, so O <= keys * 2^32 * max|V| and l stay far
// inside the fp32 range, and bf16 P keeps its relative precision.
#ifndef ABATTN_FWD_RESCALE_LOG2
#define ABATTN_FWD_RESCALE_LOG2 32
#endif
constexpr float FWD_RESCALE_LOG2 = ABATTN_FWD_RESCALE_LOG2;
constexpr uint32_t FWD_TMEM_COLS = 512;
constexpr uint32_t FWD_TMEM_O = 256;  // O accumulators: even tiles at 256, odd tiles at 384

struct FwdParams {
    const __nv_bfloat16 *K;  // [B*H][N][HD], gathered by the sparse kernel
    const __nv_bfloat16 *V;
    const int32_t *counts;
    const int32_t *idx;
    const float *pi_sel;
    int64_t cap;
    __nv_bfloat16 *O;
    float *lse;
    int N;
    int nqb;
    int kb;
    int box_rows;  // dense kernel: rows per K/V TMA box (32)
    int nkvb;
    float scale_log2;
    // E4M3 forward only: the scale of each 128-query block [rows] and of each
    // KV block [B*H][nkvb]; K then holds E4M3 codes [B*H][N][128]
    const float *q_scale;
    const float *k_scale;
};

// FP8: Q and K as E4M3 codes (d = 128: one 128-byte row per query or key, so
// a 16 KB tile), V bf16; the smaller tiles leave room for a fourth stage.
template <int HD, bool FP8 = false>
struct FwdLayout {
    static constexpr int HALVES = HD / 64;
    static constexpr int TILE = HALVES * 16384;  // 128 rows x HD bf16, per 64-col half 16 KB
    static constexpr int NS = FP8 ? 4 : FWD_NS;  // K/V stages
    static constexpr int QT = FP8 ? 16384 : TILE;
    static constexpr int KT = FP8 ? 16384 : TILE;
    static constexpr int VT = TILE;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + QT;
    static constexpr int V_OFF = K_OFF + NS * KT;
    // per-key bias [NS][128] (N % 4 != 0) or per-group bias [NS][32]: one
    // kernel uses one of the two, so they share the area
    static constexpr int BIAS_OFF = V_OFF + NS * VT;
    static constexpr int GBIAS_OFF = BIAS_OFF;
    // FP8: each 4-key group's logit multiplier (query-block scale x KV-block
    // scale x softmax scale) [NS][32]
    static constexpr int MUL_OFF = BIAS_OFF + NS * 128 * 4;
    static constexpr int BAR_OFF = MUL_OFF + (FP8 ? NS * 32 * 4 : 0);
    static constexpr int NBARS = 1 + 2 * NS + 8;
    // (m, l) of both softmax warpgroups, [2][2][128] floats, exchanged in the
    // epilogue through the first K stage: by then every QK^T MMA has completed
    // and every K load has landed
    static constexpr int XCH_OFF = K_OFF;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
};

// GROUPED (N % 4 == 0): every 4-key group of a tile shares one bias, since
// block boundaries are multiples of 4 keys and so is N; the softmax then adds
// the bias once per group.  Otherwise the bias is kept per key.
//
// FP8 (sparse, grouped, d = 128 only): Q and K are E4M3 codes with one scale per
// 128-query block and per KV block (the VC-Attention pages' 8-bit attention on
// B200); QK^T runs as E4M3 MMAs and each group's logits are multiplied by its
// block's scales; P and V stay bf16.
template <int HD, bool DENSE, bool GROUPED, bool FP8 = false>
__global__ void __launch_bounds__(FWD_THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    static_assert(!FP8 || (!DENSE && GROUPED && HD == 128), "E4M3 forward: sparse, grouped, d = 128");
    using L = FwdLayout<HD, FP8>;
    constexpr int NS = L::NS;
    extern __shared__ uint8_t fwd_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(fwd_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + L::Q_OFF;
    uint8_t *sK = smem + L::K_OFF;
    uint8_t *sV = smem + L::V_OFF;
    float *sBias = reinterpret_cast<float *>(smem + L::BIAS_OFF);
    float *sGBias = reinterpret_cast<float *>(smem + L::GBIAS_OFF);
    float *sMul = reinterpret_cast<float *>(smem + L::MUL_OFF);  // FP8 only
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *q_full = bars;
    uint64_t *kv_full = bars + 1;
    uint64_t *kv_empty = bars + 1 + NS;
    uint64_t *s_full = bars + 1 + 2 * NS;  // [2]
    uint64_t *p_full = s_full + 2;              // [2 warpgroups][2 key halves]
    uint64_t *pv_done = p_full + 4;             // [2]
    float *xch = reinterpret_cast<float *>(smem + L::XCH_OFF);
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
        for (int s = 0; s < NS; ++s) {
            // dense: one expect_tx arrival per producer warp (TMA bytes);
            // sparse: one cp.async completion arrival per producer thread plus
            // one release arrival per warp for the biases
            mbar_init(&kv_full[s], DENSE ? FWD_PRODUCERS : FWD_PRODUCERS * 33);
            mbar_init(&kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[2 * i], 4);
            mbar_init(&p_full[2 * i + 1], 4);
            mbar_init(&pv_done[i], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 12) {
        tmem_alloc(tmem_slot, FWD_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8 && warp != 12) {
        // ------------------------------------------------------------ producers
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(FWD_OTHER_REGS) : "memory");
        const int pw = warp < 12 ? warp - 8 : warp - 9;  // 0..6
        if (lane == 0 && pw == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        int issued = 0;
        if (T > 0) {
            if (lane == 0 && pw == 0) {
                mbar_arrive_expect_tx(q_full, L::QT);
                if constexpr (FP8) {
                    tma_load_3d(sQ, &tmQ, q_full, 0, q0, bh);  // 128 rows x 128 E4M3 codes
                } else {
#pragma unroll
                    for (int h = 0; h < L::HALVES; ++h) tma_load_3d(sQ + h * 16384, &tmQ, q_full, h * 64, q0, bh);
                }
            }
            const int32_t *ridx = DENSE ? nullptr : p.idx + int64_t(row) * p.cap;
            const float *rpi = DENSE ? nullptr : p.pi_sel + int64_t(row) * p.cap;
            const int kb = p.kb;                      // rows per block (128 for the dense kernel)
            const int spt = 128 / kb;                 // block slots per tile
            if constexpr (DENSE) {
                // whole 128-key tiles: units of R = 32 rows, one TMA box per
                // unit, 64-column half and tensor
                const int R = p.box_rows;
                const int nunits = 128 / R;
                const int unit = pw + FWD_PRODUCERS * lane;  // this lane's unit in every tile
                const bool owner = unit < nunits;
                const int ro = (unit * R) % kb;       // the unit's first row inside its tile
                const int nown = nunits > pw ? (nunits - pw + FWD_PRODUCERS - 1) / FWD_PRODUCERS : 0;
                const uint32_t tx_bytes = uint32_t(nown) * R * HD * 2 * 2;
                for (int t = 0; t < T; ++t) {
                    const int s = t % NS;
                    if (t >= NS && !mbar_wait(&kv_empty[s], ((t / NS) - 1) & 1, abort_flag)) break;
                    if (owner) {
                        const int key0 = t * kb + ro;
                        if constexpr (GROUPED) {
                            float *gdst = sGBias + s * 32 + unit * (R / 4);
                            for (int i = 0; i < R; i += 4) gdst[i / 4] = key0 + i < p.N ? 0.f : -INFINITY;
                        } else {
                            float *bdst = sBias + s * 128 + unit * R;
                            for (int i = 0; i < R; ++i) bdst[i] = key0 + i < p.N ? 0.f : -INFINITY;
                        }
                        __syncwarp(__activemask());
                        if (lane == 0) mbar_arrive_expect_tx(&kv_full[s], tx_bytes);
                        __syncwarp(__activemask());
                        uint8_t *dK = sK + s * L::KT + unit * R * 128;
                        uint8_t *dV = sV + s * L::VT + unit * R * 128;
#pragma unroll
                        for (int h = 0; h < L::HALVES; ++h) {
                            tma_load_3d(dK + h * 16384, &tmK, &kv_full[s], h * 64, key0, bh);
                            tma_load_3d(dV + h * 16384, &tmV, &kv_full[s], h * 64, key0, bh);
                        }
                    } else if (lane == 0) {
                        mbar_arrive_expect_tx(&kv_full[s], 0);  // a warp without units still arrives
                    }
                    __syncwarp();
                    ++issued;
                }
            } else {
                // Selected blocks: the tile's 32 quads of 4 rows (a quad lies in
                // one block since kb >= 4); warp pw gathers quads pw, pw+7, ...
                // with cp.async, 16 bytes per lane (row r = lane / 8 of the quad,
                // chunk c = lane % 8 of a 64-column half), written straight into
                // the 128-byte-swizzled layout the MMAs read.  Small TMA boxes
                // would cost the issuing warps tens of cycles each (128 per
                // tile); cp.async issues one warp instruction per quad, half and
                // tensor.  kv_full counts one completion arrival per producer
                // thread (cp.async.mbarrier.arrive.noinc) and one release
                // arrival per warp after its bias stores.
                const int nown = (32 - pw + FWD_PRODUCERS - 1) / FWD_PRODUCERS;  // quads of this warp
                const bool owner = lane < nown;       // lane j fetches the plan entry of quad pw + 7j
                const int my_q = pw + FWD_PRODUCERS * lane;
                const int sl = owner ? (my_q * 4) / kb : 0;  // the quad's block slot in the tile
                const int ro = owner ? (my_q * 4) % kb : 0;  // the quad's first row inside its block
                const int r = lane >> 3, c = lane & 7;
                const __nv_bfloat16 *Kbh = p.K + int64_t(bh) * p.N * HD;
                const __nv_bfloat16 *Vbh = p.V + int64_t(bh) * p.N * HD;
                int fill_blk = 0;                     // a valid block to load into padding slots
                {
                    const int b0 = ridx[0];
                    fill_blk = (b0 >= 0 && b0 < p.nkvb) ? b0 : 0;
                }
                auto fetch = [&](int t, int &blk, float &pi) {
                    const int e = t * spt + sl;
                    blk = -1;
                    pi = 0.f;
                    if (owner && e < cnt) {
                        blk = __ldg(ridx + e);
                        pi = __ldg(rpi + e);
                    }
                };
                {
                    // the plan row is read once per tile by the producer lanes:
                    // bring it into L1 up front
                    const int lines = (cnt * 4 + 127) / 128;
                    for (int i = pw * 32 + lane; i < 2 * lines; i += FWD_PRODUCERS * 32)
                        prefetch_l1(i < lines ? reinterpret_cast<const char *>(ridx) + i * 128
                                              : reinterpret_cast<const char *>(rpi) + (i - lines) * 128);
                }
                // plan entries of tiles t (cur) and t+1 (nxt); the entry of tile
                // t+2 is fetched at the top of iteration t
                int cur_blk, nxt_blk;
                float cur_pi, nxt_pi;
                fetch(0, cur_blk, cur_pi);
                fetch(1, nxt_blk, nxt_pi);
                // FP8: the KV-block scale of the entries of tiles t (cur) and
                // t+1 (nxt, loaded at the top of iteration t), and the query
                // block's scale times the softmax scale
                auto fetch_ks = [&](int blk) -> float {
                    return (owner && blk >= 0 && blk < p.nkvb) ? __ldg(p.k_scale + int64_t(bh) * p.nkvb + blk) : 0.f;
                };
                const float qmul = FP8 ? __ldg(p.q_scale + row) * p.scale_log2 : 0.f;
                float cur_ks = FP8 ? fetch_ks(cur_blk) : 0.f, nxt_ks = 0.f;
                for (int t = 0; t < T; ++t) {
                    const int s = t % NS;
                    int x_blk;
                    float x_pi;
                    fetch(t + 2, x_blk, x_pi);
                    if constexpr (FP8) nxt_ks = fetch_ks(nxt_blk);
                    if (t >= NS && !mbar_wait(&kv_empty[s], ((t / NS) - 1) & 1, abort_flag)) break;
                    // this lane's quad: block, first key, bias and (FP8) multiplier
                    int key0 = 0;
                    float b = -INFINITY, mq = 0.f;
                    if (owner) {
                        int blk = fill_blk;  // padding slot: loaded, weighted zero
                        if (t * spt + sl < cnt) {
                            if (cur_blk >= 0 && cur_blk < p.nkvb && cur_pi > 0.f) {
                                blk = cur_blk;
                                b = -log2f(cur_pi);
                                if constexpr (FP8) mq = qmul * cur_ks;
                            } else if (ro == 0) {
                                raise_error(kErrBounds);
                            }
                        }
                        key0 = blk * kb + ro;
                    }
                    for (int j = 0; j < nown; ++j) {
                        const int q = pw + FWD_PRODUCERS * j;
                        const int k0 = __shfl_sync(0xffffffffu, key0, j);
                        const float bj = __shfl_sync(0xffffffffu, b, j);
                        const int key = k0 + r;
                        const bool valid = key < p.N;  // rows past N (ragged last block) read as zero
                        const int srow = q * 4 + r;
                        const uint32_t roff = uint32_t(srow * 128 + ((c ^ (srow & 7)) << 4));
                        const int64_t goff = int64_t(valid ? key : 0) * HD + c * 8;
                        if constexpr (FP8) {
                            // the K row is 128 E4M3 codes: one 16-byte chunk per lane
                            const uint8_t *K8bh = reinterpret_cast<const uint8_t *>(p.K) + int64_t(bh) * p.N * 128;
                            cp_async16(sK + s * L::KT + roff, K8bh + int64_t(valid ? key : 0) * 128 + c * 16, valid);
                        }
#pragma unroll
                        for (int h = 0; h < L::HALVES; ++h) {
                            if constexpr (!FP8) cp_async16(sK + s * L::KT + roff + h * 16384, Kbh + goff + h * 64, valid);
                            cp_async16(sV + s * L::VT + roff + h * 16384, Vbh + goff + h * 64, valid);
                        }
                        if constexpr (GROUPED) {
                            if constexpr (FP8) {
                                const float mj = __shfl_sync(0xffffffffu, mq, j);
                                if (lane == 0) sMul[s * 32 + q] = mj;
                            }
                            if (lane == 0) sGBias[s * 32 + q] = k0 < p.N ? bj : -INFINITY;
                        } else {
                            if (c == 0) sBias[s * 128 + q * 4 + r] = valid ? bj : -INFINITY;
                        }
                    }
                    cp_async_mbar_arrive_noinc(&kv_full[s]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&kv_full[s]);
                    cur_blk = nxt_blk;
                    cur_pi = nxt_pi;
                    nxt_blk = x_blk;
                    nxt_pi = x_pi;
                    cur_ks = nxt_ks;
                    ++issued;
                }
                cp_async_wait_all();
            }
            // drain: every issued copy lands before the CTA may exit
            if (*abort_flag) {
                if (lane == 0) {
                    if (pw == 0) mbar_drain(q_full, 0);
                    if (DENSE)
                        for (int t = issued - NS < 0 ? 0 : issued - NS; t < issued; ++t)
                            mbar_drain(&kv_full[t % NS], (t / NS) & 1);
                }
            }
        }
    } else if (warp == 12) {
        // ------------------------------------------------------------ MMA issuer
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(FWD_OTHER_REGS) : "memory");
        if (lane == 0 && T > 0) {
            constexpr uint32_t idesc_qk = make_idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = make_idesc_bf16(128, HD, 0, 1);
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait(q_full, 0, abort_flag);
            // descriptor low words (see umma_ss_lo): K-major operands have LBO 16,
            // V as an MN-major operand LBO 16384 (its second 64-column half)
            const uint32_t q_lo = sdesc_lo(aQ, 16), k_lo = sdesc_lo(aK, 16), v_lo = sdesc_lo(aV, 16384);
            auto issue_qk = [&](int t) -> bool {
                const int s = t % NS, sb = t & 1;
                if (!mbar_wait(&kv_full[s], (t / NS) & 1, abort_flag)) return false;
                // the sparse tile was written by cp.async (generic proxy): order
                // those writes, observed through the barrier, before the MMAs'
                // async-proxy reads
                if (!DENSE) fence_proxy_async_smem();
                tc_fence_after();
                const uint32_t kb_lo = k_lo + uint32_t(s) * (L::KT >> 4);
                if constexpr (FP8) {
                    // E4M3: 32 codes (32 bytes) of the 128-byte rows per MMA
                    constexpr uint32_t idesc_qk8 = make_idesc_e4m3(128, 128);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f8_ss_lo(tmem + sb * 128, q_lo + k * 2, kb_lo + k * 2, idesc_qk8, k > 0 ? 1u : 0u);
                } else {
#pragma unroll
                    for (int k = 0; k < HD / 16; ++k) {
                        const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
                        umma_ss_lo(tmem + sb * 128, q_lo + off, kb_lo + off, idesc_qk, k > 0 ? 1u : 0u);
                    }
                }
                umma_commit(&s_full[sb]);
                return true;
            };
            if (ok) ok = issue_qk(0);
            for (int t = 0; ok && t < T; ++t) {
                if (t + 1 < T && !issue_qk(t + 1)) break;
                const int g = t & 1;  // softmax warpgroup / S buffer / O accumulator of this tile
                const int s = t % NS;
                const uint32_t vb_lo = v_lo + uint32_t(s) * (L::VT >> 4);
                const uint32_t pbase = tmem + g * 128;
                const uint32_t acc0 = t >= 2 ? 1u : 0u;
                if constexpr (DENSE) {
                    // PV in two key halves: the softmax releases keys 0..63 of P
                    // before it computes the exponentials of keys 64..127
                    bool got = true;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if (!mbar_wait(&p_full[2 * g + hh], (t >> 1) & 1, abort_flag)) { got = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int k = 4 * hh; k < 4 * hh + 4; ++k)
                            umma_ts_lo(tmem + FWD_TMEM_O + g * 128, pbase + k * 8, vb_lo + k * (2048 >> 4),
                                       idesc_pv, k > 0 ? 1u : acc0);
                    }
                    if (!got) break;
                } else {
                    // one release of the whole P row (the split measured no
                    // gain on the sparse kernel)
                    if (!mbar_wait(&p_full[2 * g + 1], (t >> 1) & 1, abort_flag)) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        umma_ts_lo(tmem + FWD_TMEM_O + g * 128, pbase + k * 8, vb_lo + k * (2048 >> 4), idesc_pv,
                                   k > 0 ? 1u : acc0);
                }
                umma_commit(&kv_empty[s]);
                umma_commit(&pv_done[g]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(FWD_SOFTMAX_REGS) : "memory");
        const int g = warp >> 2;  // 0: even tiles, 1: odd tiles
        const int wq = warp & 3;
        const int rr = wq * 32 + lane;
        const uint32_t t_lane = tmem + (uint32_t(wq * 32) << 16);
        const uint32_t t_S = t_lane + g * 128;
        const uint32_t t_O = t_lane + FWD_TMEM_O + g * 128;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        int ntiles = 0;
        for (int t = g; t < T; t += 2, ++ntiles) {
            const int s = t % NS;
            if (!mbar_wait(&s_full[g], (t >> 1) & 1, abort_flag) ||
                !mbar_wait(&kv_full[s], (t / NS) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t x[4][32];  // the S row
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(t_S + c * 32, x[c]);
            tmem_wait_ld();
            const float *gbias = sGBias + s * 32;
            const float *gmul = sMul + s * 32;  // FP8: each group's logit multiplier
            const float *bias = sBias + s * 128;
            const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
            float2 rs01 = make_float2(0.f, 0.f), rs23 = make_float2(0.f, 0.f);
            // P as packed bf16 pairs: column j of the row holds keys 2j, 2j+1
            uint32_t pk[64];
            // 2^(a*mul + off) for the four keys of group q (two packed pairs):
            // packed FFMA for the logit shift, SFU exponentials, packed adds
            // into the row sum, bf16 packing into pk
            auto exp_group = [&](int q, float2 a, float2 b, float2 mul2, float2 off_a, float2 off_b) {
                a = __ffma2_rn(a, mul2, off_a);
                b = __ffma2_rn(b, mul2, off_b);
                a = make_float2(fast_exp2(a.x), fast_exp2(a.y));
                b = make_float2(fast_exp2(b.x), fast_exp2(b.y));
                rs01 = __fadd2_rn(rs01, a);
                rs23 = __fadd2_rn(rs23, b);
                pk[2 * q] = pack_bf16x2(a.x, a.y);
                pk[2 * q + 1] = pack_bf16x2(b.x, b.y);
            };
            auto xa = [&](int q) {
                const int c = q >> 3, i = (q & 7) * 4;
                return make_float2(__uint_as_float(x[c][i]), __uint_as_float(x[c][i + 1]));
            };
            auto xb = [&](int q) {
                const int c = q >> 3, i = (q & 7) * 4;
                return make_float2(__uint_as_float(x[c][i + 2]), __uint_as_float(x[c][i + 3]));
            };
            // largest raw logit of group q
            auto gmax = [&](int q) {
                const int c = q >> 3, i = (q & 7) * 4;
                return fmaxf(fmax3(__uint_as_float(x[c][i]), __uint_as_float(x[c][i + 1]),
                                   __uint_as_float(x[c][i + 2])),
                             __uint_as_float(x[c][i + 3]));
            };
            // The tile's largest biased logit.  With GROUPED it is taken on the raw
            // group maxima (scale > 0), one FFMA per group; otherwise per key,
            // and x then holds the biased logits.
            auto max_pass = [&]() -> float {
                float mt0 = -INFINITY, mt1 = -INFINITY;
#pragma unroll
                for (int q0 = 0; q0 < 32; q0 += 4) {
                    if constexpr (GROUPED) {
                        const float4 g4 = *reinterpret_cast<const float4 *>(gbias + q0);
                        float gm[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) gm[j] = gmax(q0 + j);
                        float2 m01 = sc2, m23 = sc2;  // (FP8: the groups' multipliers, all positive)
                        if constexpr (FP8) {
                            const float4 u4 = *reinterpret_cast<const float4 *>(gmul + q0);
                            m01 = make_float2(u4.x, u4.y);
                            m23 = make_float2(u4.z, u4.w);
                        }
                        const float2 v01 = __ffma2_rn(make_float2(gm[0], gm[1]), m01, make_float2(g4.x, g4.y));
                        const float2 v23 = __ffma2_rn(make_float2(gm[2], gm[3]), m23, make_float2(g4.z, g4.w));
                        mt0 = fmax3(mt0, v01.x, v01.y);
                        mt1 = fmax3(mt1, v23.x, v23.y);
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int q = q0 + j;
                            const float4 bb = *reinterpret_cast<const float4 *>(bias + 4 * q);
                            const float2 va = __ffma2_rn(xa(q), sc2, make_float2(bb.x, bb.y));
                            const float2 vb = __ffma2_rn(xb(q), sc2, make_float2(bb.z, bb.w));
                            mt0 = fmax3(mt0, va.x, va.y);
                            mt1 = fmax3(mt1, vb.x, vb.y);
                            // keep the biased logit for the exponentials
                            const int c = q >> 3, i = (q & 7) * 4;
                            x[c][i + 0] = __float_as_uint(va.x);
                            x[c][i + 1] = __float_as_uint(va.y);
                            x[c][i + 2] = __float_as_uint(vb.x);
                            x[c][i + 3] = __float_as_uint(vb.y);
                        }
                    }
                }
                return fmaxf(mt0, mt1);
            };
            // P = 2^(logit - m_ref) into pk for the groups [qa, qa+16) (keys
            // 4qa .. 4qa+63), and the row sum
            auto exp_pass = [&](float m_ref, int qa) {
#pragma unroll
                for (int q0 = qa; q0 < qa + 16; q0 += 4) {
                    float4 g4, u4;
                    if constexpr (GROUPED) g4 = *reinterpret_cast<const float4 *>(gbias + q0);
                    if constexpr (FP8) u4 = *reinterpret_cast<const float4 *>(gmul + q0);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int q = q0 + j;
                        if constexpr (GROUPED) {
                            const float gb = j == 0 ? g4.x : j == 1 ? g4.y : j == 2 ? g4.z : g4.w;
                            const float2 off = make_float2(gb - m_ref, gb - m_ref);
                            float2 mul = sc2;
                            if constexpr (FP8) {
                                const float mu = j == 0 ? u4.x : j == 1 ? u4.y : j == 2 ? u4.z : u4.w;
                                mul = make_float2(mu, mu);
                            }
                            exp_group(q, xa(q), xb(q), mul, off, off);
                        } else {
                            const float2 neg_m = make_float2(-m_ref, -m_ref);
                            exp_group(q, xa(q), xb(q), make_float2(1.f, 1.f), neg_m, neg_m);
                        }
                    }
                }
            };
            // half hh of the P row (keys 64hh .. 64hh+63) -> TMEM columns
            // [32hh, 32hh+32) of this S buffer
            auto store_p = [&](int hh) {
                tmem_st32(t_S + 32 * hh, *reinterpret_cast<const uint32_t(*)[32]>(pk + 32 * hh));
            };
            // this warp's P writes (and O rescaling) done: release half hh
            auto release_p = [&](int hh) {
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[2 * g + hh]);
            };
            // Lazy rescaling: O and l keep the reference max m until a tile's
            // max exceeds it by more than FWD_RESCALE_LOG2.
            const float m_new = fmaxf(m, max_pass());
            const bool need = m_new > m + FWD_RESCALE_LOG2;
            float alpha = 1.f;
            if (need) {
                alpha = fast_exp2(m - m_new);
                l *= alpha;
                m = m_new;
            }
            const bool any = __any_sync(0xffffffffu, need);
            const bool rescale = ntiles > 0 && any;
            const float m_ref = m == -INFINITY ? 0.f : m;
            auto rescale_o = [&]() -> bool {
                // this warpgroup's O must be complete before it is rescaled
                // (PV(t) waits for our release of P(t)).  Waiting only when
                // rescaling is safe: PV(t) needs that release, so the barrier
                // is never more than one phase past the one waited for.
                if (!mbar_wait(&pv_done[g], ((t >> 1) - 1) & 1, abort_flag)) return false;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(t_O + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(t_O + c * 32, o);
                }
                return true;
            };
            if constexpr (DENSE) {
                // keys 0..63 of P go to the MMA warp before the exponentials of
                // keys 64..127, unless this warp's rows of O are to be rescaled
                // first (PV(t) must add to the rescaled O)
                exp_pass(m_ref, 0);
                if (!rescale) {
                    store_p(0);
                    release_p(0);
                }
                exp_pass(m_ref, 16);
                if (rescale) store_p(0);
                store_p(1);
                if (rescale) {
                    if (!rescale_o()) { ok = false; break; }
                    release_p(0);
                }
                release_p(1);
                l += (rs01.x + rs01.y) + (rs23.x + rs23.y);
            } else {
                exp_pass(m_ref, 0);
                exp_pass(m_ref, 16);
                store_p(0);
                store_p(1);
                l += (rs01.x + rs01.y) + (rs23.x + rs23.y);
                if (rescale && !rescale_o()) { ok = false; break; }
                release_p(1);
            }
        }
        // ------------------------------------------------------------ epilogue
        // wait for this warpgroup's last PV, swap (m, l) with the other
        // warpgroup, then each warpgroup merges and writes half of the columns
        bool done = ok && ntiles > 0;
        if (done) {
            const int t_last = g + 2 * (ntiles - 1);
            done = mbar_wait(&pv_done[g], (t_last >> 1) & 1, abort_flag);
        } else if (ok && T > 0) {
            // no tile of our own (T == 1): the exchange area is K stage 0, so
            // wait until QK^T of tile 0 has read it
            mbar_wait(&s_full[0], 0, abort_flag);
        }
        xch[(g * 2 + 0) * 128 + rr] = done ? m : -INFINITY;
        xch[(g * 2 + 1) * 128 + rr] = done ? l : 0.f;
        tc_fence_before();
        named_bar_sync(1, 256);
        tc_fence_after();
        const float m0 = xch[0 * 128 + rr], l0 = xch[1 * 128 + rr];
        const float m1 = xch[2 * 128 + rr], l1 = xch[3 * 128 + rr];
        const bool has0 = m0 != -INFINITY, has1 = m1 != -INFINITY;
        const float mm = fmaxf(m0, m1);
        const float a0 = has0 ? fast_exp2(m0 - mm) : 0.f;
        const float a1 = has1 ? fast_exp2(m1 - mm) : 0.f;
        const float lt = l0 * a0 + l1 * a1;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float s0 = a0 * inv, s1 = a1 * inv;
        const int M = min(128, p.N - q0);
        const bool write = rr < M;
        __nv_bfloat16 *orow = p.O + (int64_t(bh) * p.N + q0 + rr) * HD;
        const uint32_t o0 = t_lane + FWD_TMEM_O, o1 = t_lane + FWD_TMEM_O + 128;
        // this warpgroup writes columns [g*HD/2, (g+1)*HD/2); an accumulator
        // that no tile reached is never read
#pragma unroll
        for (int c = 0; c < HD / 64; ++c) {
            const int col = g * (HD / 2) + c * 32;
            uint32_t va[32], vb[32];
            if (has0) tmem_ld32(o0 + col, va);
            if (has1) tmem_ld32(o1 + col, vb);
            tmem_wait_ld();
            if (write) {
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                    float f[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        f[u] = (has0 ? __uint_as_float(va[i + u]) * s0 : 0.f) +
                               (has1 ? __uint_as_float(vb[i + u]) * s1 : 0.f);
                    uint4 v;
                    v.x = pack_bf16x2(f[0], f[1]);
                    v.y = pack_bf16x2(f[2], f[3]);
                    v.z = pack_bf16x2(f[4], f[5]);
                    v.w = pack_bf16x2(f[6], f[7]);
                    *reinterpret_cast<uint4 *>(orow + col + i) = v;
                }
            }
        }
        if (g == 0 && write && p.lse != nullptr)
            p.lse[int64_t(bh) * p.N + q0 + rr] = lt > 0.f ? (mm + log2f(lt)) * 0.69314718055994530942f : -INFINITY;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc(tmem, FWD_TMEM_COLS);
    }
}

}  // namespace abattn
