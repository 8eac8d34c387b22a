// Microbenchmark of the sparse forward's gather: the 32 selected 4-row blocks
// of a 128-key tile, both 64-column halves of K and of V (64 KB), copied into
// a 3-stage ring in shared memory by W issuing warps, in the 128-byte-swizzled
// layout the tensor cores read; one consumer thread releases each stage as
// soon as it has landed, so the measured cycles per tile are the issue and
// landing cost alone.  One CTA per SM.  Three ways to copy a block's rows:
//   mode 0: a TMA tiled box of 4 rows x 64 columns per half and tensor;
//   mode 1: cp.async, 16 bytes per lane (row lane / 8, chunk lane % 8);
//   mode 2: a TMA tile::gather4 load per half and tensor (2D tensor map over
//           [rows][d] with a box one row high; four row coordinates).
// The consumer also checks the last tile's bytes against global memory.
// Not part of the attention path: built beside the library for the
// benchmark's --gather-bench mode.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kStages = 3;
constexpr int kTile = 32768;  // 128 rows x 128 bf16
constexpr long long kWaitLimit = 2000000000ll;

__device__ int g_bench_err;

__device__ __forceinline__ uint32_t sa(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void bar_init(uint64_t *b, uint32_t n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sa(b)), "r"(n));
}
__device__ __forceinline__ void bar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(sa(b)) : "memory");
}
__device__ __forceinline__ void bar_expect(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(sa(b)), "r"(bytes) : "memory");
}
// bounded wait; false (and the error flag) when it runs out
__device__ __forceinline__ bool bar_wait(uint64_t *b, uint32_t parity) {
    const long long t0 = clock64();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(sa(b)), "r"(parity)
            : "memory");
        if (ok) return true;
        if (clock64() - t0 > kWaitLimit) {
            atomicExch(&g_bench_err, 1);
            return false;
        }
    }
}

// block of quad u of tile t in CTA c (deterministic, spread over the head)
__device__ __forceinline__ int block_of(int t, int u, int c, int nblk) {
    const uint32_t h = uint32_t(t) * 2654435761u ^ (uint32_t(u) * 40503u + uint32_t(c) * 2246822519u);
    return int((h ^ (h >> 15)) % uint32_t(nblk));
}

__global__ void gather_bench_kernel(const __grid_constant__ CUtensorMap boxK, const __grid_constant__ CUtensorMap boxV,
                                    const __grid_constant__ CUtensorMap rowsK, const __grid_constant__ CUtensorMap rowsV,
                                    const __nv_bfloat16 *K, const __nv_bfloat16 *V, int BH, int N, int mode, int W,
                                    int T, long long *cycles, int *mism) {
    extern __shared__ uint8_t raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = sm, *sV = sm + kStages * kTile;
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + 2 * kStages * kTile), *empty = full + kStages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x % BH, nblk = N / 4;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            bar_init(&full[s], mode == 1 ? W * 32 : W);
            bar_init(&empty[s], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp < W) {
        const int nown = (32 - warp + W - 1) / W;  // quads of this warp: warp, warp + W, ...
        for (int t = 0; t < T; ++t) {
            const int s = t % kStages;
            if (t >= kStages && !bar_wait(&empty[s], ((t / kStages) - 1) & 1)) return;
            if (mode == 1) {
                const int r = lane >> 3, c = lane & 7;
                for (int j = 0; j < nown; ++j) {
                    const int u = warp + W * j;
                    const int key = block_of(t, u, blockIdx.x, nblk) * 4 + r;
                    const int srow = u * 4 + r;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t so = uint32_t(s * kTile + h * 16384 + srow * 128 + ((c ^ (srow & 7)) << 4));
                        const int64_t go = (int64_t(bh) * N + key) * 128 + h * 64 + c * 8;
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa(sK + so)), "l"(K + go) : "memory");
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa(sV + so)), "l"(V + go) : "memory");
                    }
                }
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(sa(&full[s])) : "memory");
            } else {
                // lane j issues quad warp + W j: 4 copies of 512 bytes each
                if (lane == 0) bar_expect(&full[s], uint32_t(nown) * 4 * 512);
                __syncwarp();
                const int u = warp + W * lane;
                if (lane < nown) {
                    const int key0 = block_of(t, u, blockIdx.x, nblk) * 4;
                    const uint32_t mb = sa(&full[s]);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t dk = sa(sK + s * kTile + h * 16384 + u * 512);
                        const uint32_t dv = sa(sV + s * kTile + h * 16384 + u * 512);
                        if (mode == 0) {
                            asm volatile(
                                "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
                                " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dk),
                                "l"(reinterpret_cast<uint64_t>(&boxK)), "r"(mb), "r"(h * 64), "r"(key0), "r"(bh)
                                : "memory");
                            asm volatile(
                                "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
                                " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dv),
                                "l"(reinterpret_cast<uint64_t>(&boxV)), "r"(mb), "r"(h * 64),
                                "r"(key0), "r"(bh)
                                : "memory");
                        } else {
                            const int r0 = bh * N + key0;
                            asm volatile(
                                "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
                                " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dk),
                                "l"(reinterpret_cast<uint64_t>(&rowsK)), "r"(mb), "r"(h * 64), "r"(r0), "r"(r0 + 1),
                                "r"(r0 + 2), "r"(r0 + 3)
                                : "memory");
                            asm volatile(
                                "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
                                " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dv),
                                "l"(reinterpret_cast<uint64_t>(&rowsV)), "r"(mb), "r"(h * 64),
                                "r"(r0), "r"(r0 + 1), "r"(r0 + 2), "r"(r0 + 3)
                                : "memory");
                        }
                    }
                }
                __syncwarp();
            }
        }
        if (mode == 1) asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == W) {
        long long t0 = 0;
        const int warm = T / 10;
        int bad = 0;
        for (int t = 0; t < T; ++t) {
            const int s = t % kStages;
            if (!bar_wait(&full[s], (t / kStages) & 1)) return;
            if (t == warm) t0 = clock64();
            if (t == T - 1) {
                // the last tile: every row of K and V, chunks lane % 8 of both halves
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                for (int row = lane >> 3; row < 128; row += 4) {
                    const int u = row >> 2, key = block_of(t, u, blockIdx.x, nblk) * 4 + (row & 3), c = lane & 7;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t so = uint32_t(s * kTile + h * 16384 + row * 128 + ((c ^ (row & 7)) << 4));
                        const int64_t go = (int64_t(bh) * N + key) * 128 + h * 64 + c * 8;
                        const uint4 a = *reinterpret_cast<const uint4 *>(sK + so), b = *reinterpret_cast<const uint4 *>(K + go);
                        const uint4 e = *reinterpret_cast<const uint4 *>(sV + so), f = *reinterpret_cast<const uint4 *>(V + go);
                        bad += (a.x != b.x || a.y != b.y || a.z != b.z || a.w != b.w) + (e.x != f.x || e.y != f.y || e.z != f.z || e.w != f.w);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) bar_arrive(&empty[s]);
        }
        bad = __reduce_add_sync(0xffffffffu, bad);
        if (lane == 0) {
            cycles[blockIdx.x] = (clock64() - t0) / (T - warm);
            if (bad) atomicAdd(mism, bad);
        }
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

}  // namespace

// Runs one configuration: K, V are bf16 [BH][N][128] device arrays (N a
// multiple of 4); mode 0 (TMA 4-row boxes), 1 (cp.async) or 2 (TMA gather4);
// W issuing warps (1..16); T tiles per CTA.  Writes the mean cycles per tile
// over the CTAs and the number of mismatching 16-byte chunks of the last tile.
// Returns 0, or -1 (bad arguments), -2 (CUDA error), -3 (a wait ran out).
extern "C" int abattn_gather_bench(const void *K, const void *V, int BH, int N, int mode, int W, int T,
                                   double *cycles_per_tile, long long *mismatches) {
    if (K == nullptr || V == nullptr || BH < 1 || N < 4 || N % 4 != 0 || mode < 0 || mode > 2 || W < 1 || W > 16 ||
        T < 20 || cycles_per_tile == nullptr || mismatches == nullptr)
        return -1;
    auto enc = encoder();
    if (enc == nullptr) return -2;
    // maps 0/1: K/V as {128, N, BH} with a 64 x 4 box; maps 2/3: K/V as {128, BH*N} with a 64 x 1 box
    CUtensorMap m[4];
    for (int i = 0; i < 2; ++i) {
        void *base = const_cast<void *>(i == 0 ? K : V);
        cuuint64_t d3[3] = {128, cuuint64_t(N), cuuint64_t(BH)}, s3[2] = {256, cuuint64_t(N) * 256};
        cuuint32_t b3[3] = {64, 4, 1}, e3[3] = {1, 1, 1};
        if (enc(&m[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, d3, s3, b3, e3, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return -2;
        cuuint64_t d2[2] = {128, cuuint64_t(BH) * N}, s2[1] = {256};
        cuuint32_t b2[2] = {64, 1}, e2[2] = {1, 1};
        if (enc(&m[2 + i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, d2, s2, b2, e2, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return -2;
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long *cyc = nullptr;
    int *bad = nullptr;
    if (cudaMalloc(&cyc, sizeof(long long) * sms) != cudaSuccess) return -2;
    if (cudaMalloc(&bad, sizeof(int)) != cudaSuccess) { cudaFree(cyc); return -2; }
    cudaMemset(bad, 0, sizeof(int));
    int zero = 0;
    cudaMemcpyToSymbol(g_bench_err, &zero, sizeof(int));
    const int smem = 2 * kStages * kTile + 2 * kStages * 8 + 1024;
    cudaFuncSetAttribute(gather_bench_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    gather_bench_kernel<<<sms, (W + 1) * 32, smem>>>(m[0], m[1], m[2], m[3], static_cast<const __nv_bfloat16 *>(K),
                                                     static_cast<const __nv_bfloat16 *>(V), BH, N, mode, W, T, cyc, bad);
    int rc = cudaGetLastError() == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess ? 0 : -2;
    long long h[1024] = {};
    int hb = 0, herr = 0;
    if (rc == 0) {
        cudaMemcpy(h, cyc, sizeof(long long) * (sms < 1024 ? sms : 1024), cudaMemcpyDeviceToHost);
        cudaMemcpy(&hb, bad, sizeof(int), cudaMemcpyDeviceToHost);
        cudaMemcpyFromSymbol(&herr, g_bench_err, sizeof(int));
        double sum = 0;
        for (int i = 0; i < sms; ++i) sum += double(h[i]);
        *cycles_per_tile = sum / sms;
        *mismatches = hb;
        if (herr) rc = -3;
    }
    cudaFree(cyc);
    cudaFree(bad);
    return rc;
}
