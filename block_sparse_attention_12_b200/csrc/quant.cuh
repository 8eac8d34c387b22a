// E4M3 block quantisation of the 8-bit forward's Q and K (the VC-Attention
// pages, B200 results: 8-bit attention on Blackwell).  E4M3 is the OCP 8-bit
// float (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite
// value 448).  Consecutive rows are grouped in blocks that share one scale:
// scale = amax / 448 over the block, so that its largest element takes the
// largest code, and each element is encoded from fp32(x * fp32(448 / amax)),
// rounded to nearest even and saturated at +-448; a block of zeros takes
// scale 1.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace abattn {

constexpr int QZ_THREADS = 128;

// One thread per row of a bf16 [batches][n][128] tensor, 128 rows per CTA
// (grid: row tiles x batches); rows_per_block is a power of two that divides
// 128, so no block crosses a CTA.  codes [batches][n][128]; scale
// [batches][nblk].
__global__ void __launch_bounds__(QZ_THREADS) quant_e4m3_kernel(const __nv_bfloat16 *__restrict__ X, int64_t n,
                                                                int rows_per_block, int64_t nblk,
                                                                uint8_t *__restrict__ codes,
                                                                float *__restrict__ scale) {
    __shared__ float s_amax[QZ_THREADS];
    const int64_t b = blockIdx.y;
    const int64_t r = int64_t(blockIdx.x) * QZ_THREADS + threadIdx.x;
    const bool live = r < n;
    // the row: 128 bf16 as 16 chunks of 8
    uint4 v[16];
    const uint4 *src = reinterpret_cast<const uint4 *>(X + (b * n + (live ? r : 0)) * 128);
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        v[i] = live ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(h[j]);
            am = fmaxf(am, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
    s_amax[threadIdx.x] = am;
    __syncthreads();
    const int b0 = (int(threadIdx.x) / rows_per_block) * rows_per_block;
    float bmax = 0.f;
    for (int i = 0; i < rows_per_block; ++i) bmax = fmaxf(bmax, s_amax[b0 + i]);
    const float inv = bmax > 0.f ? __fdiv_rn(448.f, bmax) : 1.f;
    if (live) {
        uint4 *dst = reinterpret_cast<uint4 *>(codes + (b * n + r) * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // 16 codes per 16-byte store
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v[2 * c + k / 2]);
                const float2 f0 = __bfloat1622float2(h[(k & 1) * 2]);
                const float2 f1 = __bfloat1622float2(h[(k & 1) * 2 + 1]);
                const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fmul_rn(f0.x, inv), __fmul_rn(f0.y, inv)), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fmul_rn(f1.x, inv), __fmul_rn(f1.y, inv)), __NV_SATFINITE, __NV_E4M3);
                w[k] = uint32_t(lo) | (uint32_t(hi) << 16);
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if ((int(threadIdx.x) % rows_per_block) == 0)
            scale[b * nblk + r / rows_per_block] = bmax > 0.f ? __fdiv_rn(bmax, 448.f) : 1.f;
    }
}

}  // namespace abattn
