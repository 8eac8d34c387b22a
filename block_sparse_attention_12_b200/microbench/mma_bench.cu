// Microbenchmark of the 5th-generation tensor cores' issue and execution
// rate: one thread per CTA (one CTA per SM) issues back-to-back bf16
// tcgen05.mma instructions of M = 128, K = 16 (accumulators in TMEM) and
// times them with clock64 up to the completion of the last one.  Operand
// values are zeros (the rate does not depend on them).  Modes:
//   0: both operands in shared memory, N = 128, one accumulator;
//   1: both operands in shared memory, N = 256;
//   2: A in TMEM, B in shared memory, N = 128;
//   3: both operands in shared memory, N = 64;
//   4: the score kernel's issue: per 128-key tile, three MMAs per k-step
//      (hi.hi, hi.lo, lo.hi) with their 64-bit shared-memory descriptors
//      built per MMA, eight k-steps, two commits;
//   5: the forward kernel's issue: per tile, QK^T as eight shared-memory
//      MMAs into an S buffer, PV as eight MMAs with P read from TMEM into an
//      O accumulator, two commits after each;
//   6, 7: modes 0 and 2 while four other warps load 16 bytes per lane from
//      another 64 KB of shared memory as fast as they can;
//   8: mode 0 while those warps store instead.
// Modes 6-8 also report the other warps' shared-memory bytes per cycle.
// Not part of the attention path: built beside the library for the
// benchmark's --mma-bench mode.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../csrc/common.cuh"

namespace {

using namespace abattn;

constexpr int kA = 16384;       // A: 128 rows x 128 bytes
constexpr int kB = 32768;       // B: 256 rows x 128 bytes
constexpr int kT = 65536;       // the traffic warps' region
constexpr int kSmem = kA + kB + kT + 64 + 1024;
constexpr int kThreads = 160;   // the issuing warp and four traffic warps

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) mma_bench_kernel(int iters, long long *cycles, long long *traffic) {
    extern __shared__ uint8_t raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem, *sB = smem + kA;
    uint4 *sT = reinterpret_cast<uint4 *>(smem + kA + kB);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kA + kB + kT);  // done, and two commit targets
    uint32_t *slot = reinterpret_cast<uint32_t *>(smem + kA + kB + kT + 32);
    volatile int *stop = reinterpret_cast<volatile int *>(smem + kA + kB + kT + 48);
    for (int i = threadIdx.x; i < (kA + kB + kT) / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
        *stop = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *slot;
    if (warp == 0 && lane == 0) {
        const uint32_t a_lo = sdesc_lo(smem_u32(sA), 16), b_lo = sdesc_lo(smem_u32(sB), 16);
        constexpr int N = MODE == 1 ? 256 : MODE == 3 ? 64 : 128;
        constexpr bool kTmemA = MODE == 2 || MODE == 7;
        constexpr uint32_t idesc = make_idesc_bf16(128, N, 0, 0);
        const long long t0 = clock64();
        if constexpr (MODE == 4) {
            const uint32_t base = smem_u32(smem);
            for (int it = 0; it < iters; ++it) {
                const uint32_t a_hi = base, a_l = base + 8192;
                const uint32_t b_hi = base + kA + (it & 1) * 8192, b_l = b_hi + 4096;
                const uint32_t d = tmem + (it & 1) * 128;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = (k & 3) * 32;
                    umma_f16_ss(d, make_sdesc_sw128(a_hi + off, 16, 1024), make_sdesc_sw128(b_hi + off, 16, 1024), idesc, k > 0);
                    umma_f16_ss(d, make_sdesc_sw128(a_hi + off, 16, 1024), make_sdesc_sw128(b_l + off, 16, 1024), idesc, 1u);
                    umma_f16_ss(d, make_sdesc_sw128(a_l + off, 16, 1024), make_sdesc_sw128(b_hi + off, 16, 1024), idesc, 1u);
                }
                umma_commit(&bars[1]);
                umma_commit(&bars[2]);
            }
        } else if constexpr (MODE == 5) {
            for (int it = 0; it < iters; ++it) {
                const uint32_t s = tmem + (it & 1) * 128;
#pragma unroll
                for (int k = 0; k < 8; ++k) umma_ss_lo(s, a_lo + (k & 3) * 2, b_lo + (k & 3) * 2, idesc, k > 0 ? 1u : 0u);
                umma_commit(&bars[1]);
                umma_commit(&bars[2]);
#pragma unroll
                for (int k = 0; k < 8; ++k) umma_ts_lo(tmem + 256 + (it & 1) * 128, s + k * 8, b_lo + (k & 3) * 2, idesc, 1u);
                umma_commit(&bars[1]);
                umma_commit(&bars[2]);
            }
        } else {
            for (int it = 0; it < iters; ++it) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int k = j & 3;
                    if constexpr (kTmemA) umma_ts_lo(tmem, tmem + 256 + k * 8, b_lo + k * 2, idesc, 1u);
                    else umma_ss_lo(tmem, a_lo + k * 2, b_lo + k * 2, idesc, 1u);
                }
            }
        }
        umma_commit(&bars[0]);
        const long long w0 = clock64();
        bool done = false;
        while (!(done = mbar_try_wait(&bars[0], 0)) && clock64() - w0 < 2000000000ll) {
        }
        cycles[blockIdx.x] = done ? clock64() - t0 : -1;
        *stop = 1;
    } else if (MODE >= 6 && warp >= 1) {
        // shared-memory traffic beside the MMAs, until they have completed
        // (bounded by an iteration count)
        long long n = 0;
        uint32_t acc = 0;
        const long long t0 = clock64();
        for (int it = 0; it < 4000000 && !*stop; ++it) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int idx = ((it * 8 + u) * 32 + lane + warp * 256) & (kT / 16 - 1);
                if constexpr (MODE == 8) {
                    sT[idx] = make_uint4(uint32_t(it), uint32_t(u), uint32_t(lane), uint32_t(warp));
                } else {
                    acc ^= sT[idx].x;
                }
            }
            n += 8;
        }
        const long long dt = clock64() - t0;
        if (acc == 0x9e3779b9u) n = -n;  // keeps the loads
        if (lane == 0) {
            atomicAdd(reinterpret_cast<unsigned long long *>(&traffic[2 * blockIdx.x]),
                      static_cast<unsigned long long>(n * 512));
            if (warp == 1) traffic[2 * blockIdx.x + 1] = dt;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int MODE>
int launch(int iters, int ctas, long long *d, long long *t) {
    if (cudaFuncSetAttribute(mma_bench_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
        return -3;
    mma_bench_kernel<MODE><<<ctas, kThreads, kSmem>>>(iters, d, t);
    return int(cudaDeviceSynchronize());
}

}  // namespace

// Runs `ctas` CTAs (one per SM) of `iters` iterations of the mode's pattern
// and stores the median over CTAs of clock cycles per MMA instruction (the
// score pattern counts 24 MMAs per iteration, the others 16) and, for modes
// 6-8, the median of the other warps' shared-memory bytes per cycle (else 0).
// Returns 0, a CUDA error code, -1 (allocation), -2 (unknown mode) or -4 (a
// CTA's wait for the last MMA ran out).
extern "C" int abattn_mma_bench(int mode, int iters, int ctas, double *cycles_per_mma,
                                double *traffic_bytes_per_cycle) {
    long long *d = nullptr, *t = nullptr;
    if (ctas <= 0 || iters <= 0 || cudaMalloc(&d, sizeof(long long) * ctas) != cudaSuccess) return -1;
    if (cudaMalloc(&t, sizeof(long long) * 2 * ctas) != cudaSuccess) {
        cudaFree(d);
        return -1;
    }
    cudaMemset(t, 0, sizeof(long long) * 2 * ctas);
    int rc = -2;
    switch (mode) {
        case 0: rc = launch<0>(iters, ctas, d, t); break;
        case 1: rc = launch<1>(iters, ctas, d, t); break;
        case 2: rc = launch<2>(iters, ctas, d, t); break;
        case 3: rc = launch<3>(iters, ctas, d, t); break;
        case 4: rc = launch<4>(iters, ctas, d, t); break;
        case 5: rc = launch<5>(iters, ctas, d, t); break;
        case 6: rc = launch<6>(iters, ctas, d, t); break;
        case 7: rc = launch<7>(iters, ctas, d, t); break;
        case 8: rc = launch<8>(iters, ctas, d, t); break;
    }
    *traffic_bytes_per_cycle = 0.0;
    if (rc == 0 && mode >= 6) {
        long long *h = new long long[2 * ctas];
        rc = int(cudaMemcpy(h, t, sizeof(long long) * 2 * ctas, cudaMemcpyDeviceToHost));
        if (rc == 0) {
            double *r = new double[ctas];
            for (int i = 0; i < ctas; ++i) r[i] = h[2 * i + 1] > 0 ? double(h[2 * i] < 0 ? -h[2 * i] : h[2 * i]) / double(h[2 * i + 1]) : 0.0;
            for (int i = 1; i < ctas; ++i)
                for (int j = i; j > 0 && r[j] < r[j - 1]; --j) {
                    const double x = r[j]; r[j] = r[j - 1]; r[j - 1] = x;
                }
            *traffic_bytes_per_cycle = r[ctas / 2];
            delete[] r;
        }
        delete[] h;
    }
    if (rc == 0) {
        long long *h = new long long[ctas];
        rc = int(cudaMemcpy(h, d, sizeof(long long) * ctas, cudaMemcpyDeviceToHost));
        if (rc == 0) {
            for (int i = 1; i < ctas; ++i)  // insertion sort for the median
                for (int j = i; j > 0 && h[j] < h[j - 1]; --j) {
                    const long long t = h[j]; h[j] = h[j - 1]; h[j - 1] = t;
                }
            if (h[0] < 0) rc = -4;
            *cycles_per_mma = double(h[ctas / 2]) / (double(iters) * (mode == 4 ? 24 : 16));
        }
        delete[] h;
    }
    cudaFree(d);
    cudaFree(t);
    return rc;
}
