// Host side of the AB-Attention C ABI (include/abattn.h): argument checks,
// TMA tensor maps, workspace carving and kernel launches.  Every check runs
// before the first CUDA call, so a rejected call launches nothing.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>

#include <mutex>

#include "../../include/abattn.h"
#include "common.cuh"
#include "forward.cuh"
#include "planner.cuh"
#include "quant.cuh"
#include "selector.cuh"

using namespace abattn;

namespace {

constexpr int64_t kMaxPlanBlocks = 40960;  // per-row score / probability row held in shared memory

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const abattn_dims *d) {
    if (d == nullptr) return ABATTN_ERR_NULL;
    if (d->B < 1 || d->H < 1 || d->N < 1) return ABATTN_ERR_SHAPE;
    if (d->d != 64 && d->d != 128) return ABATTN_ERR_SHAPE;
    if (d->N > (int64_t(1) << 30)) return ABATTN_ERR_SHAPE;
    const int64_t rows = d->B * d->H * cdiv(d->N, 128);
    if (rows >= (int64_t(1) << 31) || d->B * d->H >= (int64_t(1) << 31)) return ABATTN_ERR_SHAPE;
    return ABATTN_OK;
}

bool valid_kb(int kb) { return kb == 4 || kb == 8 || kb == 16 || kb == 32 || kb == 64 || kb == 128; }

int check_params(const abattn_params *p, bool need_planner) {
    if (p == nullptr) return ABATTN_ERR_NULL;
    if (!valid_kb(p->kv_block)) return ABATTN_ERR_PARAM;
    if (!(p->scale >= 0.f) || isinf(p->scale)) return ABATTN_ERR_PARAM;
    if (!need_planner) return ABATTN_OK;
    if (p->q_block != 128) return ABATTN_ERR_PARAM;
    if (p->n_clusters < 1 || p->n_clusters > 8) return ABATTN_ERR_PARAM;
    if (p->kmeans_iters < 0 || p->kmeans_iters > 64) return ABATTN_ERR_PARAM;
    if (!(p->budget > 0.f && p->budget <= 1.f)) return ABATTN_ERR_PARAM;
    if (p->mode != ABATTN_MODE_SIP && p->mode != ABATTN_MODE_TOPK) return ABATTN_ERR_PARAM;
    if (p->head_offset < 0) return ABATTN_ERR_PARAM;
    return ABATTN_OK;
}

float resolve_scale(float scale, int64_t d) { return scale > 0.f ? scale : 1.f / sqrtf(float(d)); }

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return ABATTN_OK;
    fprintf(stderr, "abattn: CUDA error %s\n", cudaGetErrorString(e));
    return ABATTN_ERR_CUDA;
}

int launch_status() { return cuda_status(cudaGetLastError()); }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3D view {d, rows, batches} of a bf16 [batches][rows][d] tensor; box
// {64, box_rows, 1}, 128-byte swizzle, zero fill outside the tensor (so a
// tile past the last row never reads the next batch).
int make_map_rows(CUtensorMap *m, const void *base, int64_t d, int64_t rows, int64_t batches, int box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return ABATTN_ERR_DEVICE;
    cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(rows), cuuint64_t(batches)};
    cuuint64_t strides[2] = {cuuint64_t(d * 2), cuuint64_t(rows * d * 2)};
    cuuint32_t box[3] = {64u, cuuint32_t(box_rows), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ABATTN_OK : ABATTN_ERR_CUDA;
}

// Q, K, V [B][H][N][d] as {d, N, B*H}.
int make_map(CUtensorMap *m, const void *base, const abattn_dims *d, int box_rows) {
    return make_map_rows(m, base, d->d, d->N, d->B * d->H, box_rows);
}

// E4M3 codes [B][H][N][128] as a byte tensor {128, N, B*H}; box {128, 128, 1}
// (one 128-byte row per query), 128-byte swizzle, zero fill.
int make_map_e4m3(CUtensorMap *m, const void *base, const abattn_dims *d) {
    auto fn = encode_fn();
    if (fn == nullptr) return ABATTN_ERR_DEVICE;
    cuuint64_t dims[3] = {128u, cuuint64_t(d->N), cuuint64_t(d->B * d->H)};
    cuuint64_t strides[2] = {128u, cuuint64_t(d->N * 128)};
    cuuint32_t box[3] = {128u, 128u, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ABATTN_OK : ABATTN_ERR_CUDA;
}

int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ABATTN_ERR_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return ABATTN_ERR_DEVICE;
    return major == 10 ? ABATTN_OK : ABATTN_ERR_DEVICE;
}

int sm_count() {
    int dev = 0, n = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// Plan workspace: mean keys and centroids as bf16 hi/lo pairs (the score
// kernel's operands), cluster weights, scores.
struct PlanWs {
    __nv_bfloat16 *Khi, *Klo, *Chi, *Clo;
    float *w, *S;
    size_t bytes;
};

PlanWs carve(void *ws, const abattn_dims *d, const abattn_params *p) {
    const int64_t nqb = cdiv(d->N, 128), nkvb = cdiv(d->N, p->kv_block);
    const int64_t BH = d->B * d->H, rows = BH * nqb;
    PlanWs w{};
    uint8_t *b = static_cast<uint8_t *>(ws);
    size_t off = 0;
    auto take = [&](size_t n) {
        uint8_t *r = b ? b + off : nullptr;
        off += align256(n);
        return r;
    };
    w.Khi = reinterpret_cast<__nv_bfloat16 *>(take(2 * BH * nkvb * d->d));
    w.Klo = reinterpret_cast<__nv_bfloat16 *>(take(2 * BH * nkvb * d->d));
    w.Chi = reinterpret_cast<__nv_bfloat16 *>(take(2 * rows * 8 * d->d));
    w.Clo = reinterpret_cast<__nv_bfloat16 *>(take(2 * rows * 8 * d->d));
    w.w = reinterpret_cast<float *>(take(sizeof(float) * rows * p->n_clusters));
    w.S = reinterpret_cast<float *>(take(sizeof(float) * rows * nkvb));
    w.bytes = off;
    return w;
}

// abattn_score workspace: the bf16 hi/lo operands made from the fp32 inputs.
size_t score_ws_bytes(const abattn_dims *d, const abattn_params *p) {
    const int64_t nqb = cdiv(d->N, 128), nkvb = cdiv(d->N, p->kv_block);
    const int64_t BH = d->B * d->H, rows = BH * nqb;
    return 2 * align256(2 * BH * nkvb * d->d) + 2 * align256(2 * rows * 8 * d->d);
}

int64_t capacity(int64_t nkvb, float budget) {
    const double B = double(budget) * double(nkvb);
    const double c = ceil(B + 8.0 * sqrt(B) + 32.0);
    return c < double(nkvb) ? int64_t(c) : nkvb;
}

// ---------------------------------------------------------------- launchers
int launch_meanpool(const void *K, const abattn_dims *d, int kb, float *Kbar, __nv_bfloat16 *Khi,
                    __nv_bfloat16 *Klo, cudaStream_t st) {
    const int64_t nkvb = cdiv(d->N, kb), BH = d->B * d->H;
    const int64_t total = BH * nkvb * (d->d / 8);
    const int64_t want = cdiv(total, 256);
    const int grid = int(want < int64_t(sm_count()) * 32 ? want : int64_t(sm_count()) * 32);
    if (d->d == 128)
        meanpool_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(K), BH, d->N, kb, nkvb, Kbar, Khi, Klo);
    else
        meanpool_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(K), BH, d->N, kb, nkvb, Kbar, Khi, Klo);
    return launch_status();
}

template <int D>
int launch_kmeans_t(const void *Q, const abattn_dims *d, const abattn_params *p, float *C, float *w,
                    int32_t *labels, __nv_bfloat16 *Chi, __nv_bfloat16 *Clo, cudaStream_t st) {
    const int64_t nqb = cdiv(d->N, 128), rows = d->B * d->H * nqb;
    constexpr int smem = KmLayout::ALLOC;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(kmeans_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e);
        attr = true;
    }
    CUtensorMap mQ;
    int rc = make_map(&mQ, Q, d, 128);
    if (rc) return rc;
    kmeans_kernel<D><<<unsigned(rows), KM_THREADS, smem, st>>>(mQ, d->N, nqb, p->n_clusters, p->kmeans_iters, C, w,
                                                               labels, Chi, Clo);
    return launch_status();
}

template <int D>
int launch_score_t(const __nv_bfloat16 *Chi, const __nv_bfloat16 *Clo, const __nv_bfloat16 *Khi,
                   const __nv_bfloat16 *Klo, const float *w, const abattn_dims *d, const abattn_params *p,
                   float *S, cudaStream_t st) {
    const int64_t nqb = cdiv(d->N, 128), nkvb = cdiv(d->N, p->kv_block), BH = d->B * d->H;
    CUtensorMap mChi, mClo, mKhi, mKlo;
    int rc;
    if ((rc = make_map_rows(&mChi, Chi, D, nqb * 8, BH, 128)) || (rc = make_map_rows(&mClo, Clo, D, nqb * 8, BH, 128)) ||
        (rc = make_map_rows(&mKhi, Khi, D, nkvb, BH, 128)) || (rc = make_map_rows(&mKlo, Klo, D, nkvb, BH, 128)))
        return rc;
    ScoreParams sp;
    sp.w = w;
    sp.S = S;
    sp.nqb = int(nqb);
    sp.nkvb = int(nkvb);
    sp.nc = p->n_clusters;
    sp.scale_log2 = resolve_scale(p->scale, d->d) * 1.4426950408889634f;
    constexpr int smem = ScoreLayout<D>::ALLOC;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e);
        attr = true;
    }
    dim3 grid(unsigned(cdiv(nqb, SC_QBT)), unsigned(BH));
    score_tc_kernel<D><<<grid, SC_THREADS, smem, st>>>(mChi, mClo, mKhi, mKlo, sp);
    return launch_status();
}

int launch_score(const __nv_bfloat16 *Chi, const __nv_bfloat16 *Clo, const __nv_bfloat16 *Khi,
                 const __nv_bfloat16 *Klo, const float *w, const abattn_dims *d, const abattn_params *p, float *S,
                 cudaStream_t st) {
    return d->d == 128 ? launch_score_t<128>(Chi, Clo, Khi, Klo, w, d, p, S, st)
                       : launch_score_t<64>(Chi, Clo, Khi, Klo, w, d, p, S, st);
}

int launch_plan(int mode, const float *in, const abattn_dims *d, const abattn_params *p, int32_t *counts,
                int32_t *idx, float *pi_sel, int64_t cap, float *pi_out, cudaStream_t st) {
    const int64_t nqb = cdiv(d->N, 128), nkvb = cdiv(d->N, p->kv_block);
    const int64_t rows = d->B * d->H * nqb;
    const double Bblk = double(p->budget) * double(nkvb);
    int64_t k_top = int64_t(floor(Bblk + 0.5));
    if (k_top > nkvb) k_top = nkvb;
    const size_t smem = sizeof(float) * nkvb + 4 * size_t((nkvb + 31) / 32);  // scores, flag words
    cudaError_t e;
    switch (mode) {
        case kPlanSip:
            e = cudaFuncSetAttribute(plan_kernel<kPlanSip>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (e != cudaSuccess) return cuda_status(e);
            plan_kernel<kPlanSip><<<unsigned(rows), PL_THREADS, smem, st>>>(in, d->H, p->head_offset, nqb, nkvb, Bblk, k_top, p->seed, cap, counts, idx, pi_sel, pi_out);
            break;
        case kPlanTopk:
            e = cudaFuncSetAttribute(plan_kernel<kPlanTopk>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (e != cudaSuccess) return cuda_status(e);
            plan_kernel<kPlanTopk><<<unsigned(rows), PL_THREADS, smem, st>>>(in, d->H, p->head_offset, nqb, nkvb, Bblk, k_top, p->seed, cap, counts, idx, pi_sel, nullptr);
            break;
        default:
            e = cudaFuncSetAttribute(plan_kernel<kPlanFromPi>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (e != cudaSuccess) return cuda_status(e);
            plan_kernel<kPlanFromPi><<<unsigned(rows), PL_THREADS, smem, st>>>(in, d->H, p->head_offset, nqb, nkvb, Bblk, k_top, p->seed, cap, counts, idx, pi_sel, nullptr);
            break;
    }
    return launch_status();
}

template <int HD, bool DENSE, bool GROUPED>
int launch_fwd_t(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mV, const FwdParams &fp,
                 int64_t rows, cudaStream_t st) {
    constexpr int smem = FwdLayout<HD>::ALLOC;
    static bool attr = false;
    if (!attr) {
        cudaError_t e =
            cudaFuncSetAttribute(fwd_kernel<HD, DENSE, GROUPED>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e);
        attr = true;
    }
    fwd_kernel<HD, DENSE, GROUPED><<<unsigned(rows), FWD_THREADS, smem, st>>>(mQ, mK, mV, fp);
    return launch_status();
}

template <int HD>
int launch_fwd_hd(bool dense, bool grouped, const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mV,
                  const FwdParams &fp, int64_t rows, cudaStream_t st) {
    if (dense)
        return grouped ? launch_fwd_t<HD, true, true>(mQ, mK, mV, fp, rows, st)
                       : launch_fwd_t<HD, true, false>(mQ, mK, mV, fp, rows, st);
    return grouped ? launch_fwd_t<HD, false, true>(mQ, mK, mV, fp, rows, st)
                   : launch_fwd_t<HD, false, false>(mQ, mK, mV, fp, rows, st);
}

int run_forward(bool dense, const void *Q, const void *K, const void *V, const abattn_dims *d, int kb,
                float scale, const int32_t *counts, const int32_t *idx, const float *pi_sel, int64_t cap,
                void *O, float *lse, cudaStream_t st) {
    int rc = check_device();
    if (rc) return rc;
    CUtensorMap mQ, mK, mV;
    const int box = 32;  // K/V TMA boxes of the dense kernel (the sparse kernel gathers with cp.async)
    if ((rc = make_map(&mQ, Q, d, 128)) || (rc = make_map(&mK, K, d, box)) || (rc = make_map(&mV, V, d, box)))
        return rc;
    FwdParams fp;
    fp.K = static_cast<const __nv_bfloat16 *>(K);
    fp.V = static_cast<const __nv_bfloat16 *>(V);
    fp.counts = counts;
    fp.idx = idx;
    fp.pi_sel = pi_sel;
    fp.cap = cap;
    fp.O = static_cast<__nv_bfloat16 *>(O);
    fp.lse = lse;
    fp.N = int(d->N);
    fp.nqb = int(cdiv(d->N, 128));
    fp.kb = dense ? 128 : kb;
    fp.box_rows = box;
    fp.nkvb = int(cdiv(d->N, fp.kb));
    fp.scale_log2 = resolve_scale(scale, d->d) * 1.4426950408889634f;
    fp.q_scale = nullptr;
    fp.k_scale = nullptr;
    const int64_t rows = d->B * d->H * fp.nqb;
    // every kv block starts at a multiple of 4 keys (kb is 4, 8, ..., 128), so
    // with N % 4 == 0 each 4-key group of a tile is entirely valid or entirely past N
    const bool grouped = (d->N % 4) == 0;
    if (d->d == 128) return launch_fwd_hd<128>(dense, grouped, mQ, mK, mV, fp, rows, st);
    return launch_fwd_hd<64>(dense, grouped, mQ, mK, mV, fp, rows, st);
}

// The E4M3 forward: sparse, grouped (N % 4 == 0), d = 128.
int run_forward_e4m3(const void *Q8, const float *q_scale, const void *K8, const float *k_scale, const void *V,
                     const abattn_dims *d, int kb, float scale, const int32_t *counts, const int32_t *idx,
                     const float *pi_sel, int64_t cap, void *O, float *lse, cudaStream_t st) {
    int rc = check_device();
    if (rc) return rc;
    CUtensorMap mQ, mV;
    if ((rc = make_map_e4m3(&mQ, Q8, d)) || (rc = make_map(&mV, V, d, 32))) return rc;
    FwdParams fp;
    fp.K = static_cast<const __nv_bfloat16 *>(K8);  // E4M3 codes, read as bytes
    fp.V = static_cast<const __nv_bfloat16 *>(V);
    fp.counts = counts;
    fp.idx = idx;
    fp.pi_sel = pi_sel;
    fp.cap = cap;
    fp.O = static_cast<__nv_bfloat16 *>(O);
    fp.lse = lse;
    fp.N = int(d->N);
    fp.nqb = int(cdiv(d->N, 128));
    fp.kb = kb;
    fp.box_rows = 32;
    fp.nkvb = int(cdiv(d->N, kb));
    fp.scale_log2 = resolve_scale(scale, d->d) * 1.4426950408889634f;
    fp.q_scale = q_scale;
    fp.k_scale = k_scale;
    const int64_t rows = d->B * d->H * fp.nqb;
    constexpr int smem = FwdLayout<128, true>::ALLOC;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(fwd_kernel<128, false, true, true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_status(e);
        attr = true;
    }
    fwd_kernel<128, false, true, true><<<unsigned(rows), FWD_THREADS, smem, st>>>(mQ, mQ, mV, fp);
    return launch_status();
}

int check_plan_shape(const abattn_dims *d, const abattn_params *p) {
    const int64_t nkvb = cdiv(d->N, p->kv_block);
    return nkvb > kMaxPlanBlocks ? ABATTN_ERR_SHAPE : ABATTN_OK;
}

}  // namespace

// ====================================================================== ABI
extern "C" {

const char *abattn_version(void) { return "abattn 0.1 (sm_100a, tcgen05 forward)"; }

const char *abattn_strerror(int code) {
    switch (code) {
        case ABATTN_OK: return "ok";
        case ABATTN_ERR_NULL: return "a required pointer is NULL";
        case ABATTN_ERR_SHAPE: return "shape out of range";
        case ABATTN_ERR_PARAM: return "parameter out of range";
        case ABATTN_ERR_ALIGN: return "pointer not 16-byte aligned";
        case ABATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case ABATTN_ERR_PLAN_OVERFLOW: return "a plan row selected more blocks than its capacity";
        case ABATTN_ERR_TIMEOUT: return "a bounded device wait ran out";
        case ABATTN_ERR_BOUNDS: return "a plan index or probability was out of range and skipped";
        case ABATTN_ERR_CUDA: return "CUDA call failed";
        case ABATTN_ERR_DEVICE: return "no sm_100 device or driver entry point";
        default: return "unknown status";
    }
}

int abattn_check(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(e);
    uint32_t word = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word));
    if (e != cudaSuccess) return cuda_status(e);
    if (word != 0) {
        e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_status(e);
    }
    if (word & kErrTimeout) return ABATTN_ERR_TIMEOUT;
    if (word & kErrOverflow) return ABATTN_ERR_PLAN_OVERFLOW;
    if (word & kErrBounds) return ABATTN_ERR_BOUNDS;
    return ABATTN_OK;
}

int abattn_plan_capacity(const abattn_dims *dims, const abattn_params *p, int64_t *cap) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if (cap == nullptr) return ABATTN_ERR_NULL;
    *cap = capacity(cdiv(dims->N, p->kv_block), p->budget);
    return ABATTN_OK;
}

int abattn_plan_workspace_size(const abattn_dims *dims, const abattn_params *p, size_t *bytes) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if (bytes == nullptr) return ABATTN_ERR_NULL;
    *bytes = carve(nullptr, dims, p).bytes;
    return ABATTN_OK;
}

int abattn_score_workspace_size(const abattn_dims *dims, const abattn_params *p, size_t *bytes) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if (bytes == nullptr) return ABATTN_ERR_NULL;
    *bytes = score_ws_bytes(dims, p);
    return ABATTN_OK;
}

int abattn_meanpool(const void *K, const abattn_dims *dims, int32_t kv_block, float *Kbar, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!valid_kb(kv_block)) return ABATTN_ERR_PARAM;
    if (K == nullptr || Kbar == nullptr) return ABATTN_ERR_NULL;
    if (!aligned16(K) || !aligned16(Kbar)) return ABATTN_ERR_ALIGN;
    if ((rc = check_device())) return rc;
    return launch_meanpool(K, dims, kv_block, Kbar, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

int abattn_kmeans(const void *Q, const abattn_dims *dims, const abattn_params *p, float *C, float *w,
                  int32_t *labels, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if (Q == nullptr || C == nullptr || w == nullptr) return ABATTN_ERR_NULL;
    if (!aligned16(Q)) return ABATTN_ERR_ALIGN;
    if ((rc = check_device())) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dims->d == 128 ? launch_kmeans_t<128>(Q, dims, p, C, w, labels, nullptr, nullptr, st)
                          : launch_kmeans_t<64>(Q, dims, p, C, w, labels, nullptr, nullptr, st);
}

int abattn_score(const float *C, const float *w, const float *Kbar, const abattn_dims *dims,
                 const abattn_params *p, float *S, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if (C == nullptr || w == nullptr || Kbar == nullptr || S == nullptr) return ABATTN_ERR_NULL;
    if (!aligned16(C) || !aligned16(Kbar)) return ABATTN_ERR_ALIGN;
    const size_t need = score_ws_bytes(dims, p);
    if (ws == nullptr || ws_bytes < need) return ABATTN_ERR_WORKSPACE;
    if (!aligned16(ws)) return ABATTN_ERR_ALIGN;
    if ((rc = check_device())) return rc;
    const int64_t nqb = cdiv(dims->N, 128), nkvb = cdiv(dims->N, p->kv_block);
    const int64_t BH = dims->B * dims->H, rows = BH * nqb;
    uint8_t *b = static_cast<uint8_t *>(ws);
    __nv_bfloat16 *Khi = reinterpret_cast<__nv_bfloat16 *>(b);
    __nv_bfloat16 *Klo = reinterpret_cast<__nv_bfloat16 *>(b + align256(2 * BH * nkvb * dims->d));
    __nv_bfloat16 *Chi = reinterpret_cast<__nv_bfloat16 *>(b + 2 * align256(2 * BH * nkvb * dims->d));
    __nv_bfloat16 *Clo = reinterpret_cast<__nv_bfloat16 *>(b + 2 * align256(2 * BH * nkvb * dims->d) +
                                                           align256(2 * rows * 8 * dims->d));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int grid = sm_count() * 8;
    if (dims->d == 128) {
        split_rows_kernel<128><<<grid, 256, 0, st>>>(Kbar, BH * nkvb, 1, 1, Khi, Klo);
        split_rows_kernel<128><<<grid, 256, 0, st>>>(C, rows, p->n_clusters, 8, Chi, Clo);
    } else {
        split_rows_kernel<64><<<grid, 256, 0, st>>>(Kbar, BH * nkvb, 1, 1, Khi, Klo);
        split_rows_kernel<64><<<grid, 256, 0, st>>>(C, rows, p->n_clusters, 8, Chi, Clo);
    }
    if ((rc = launch_status())) return rc;
    return launch_score(Chi, Clo, Khi, Klo, w, dims, p, S, st);
}

int abattn_plan_from_scores(const float *S, const abattn_dims *dims, const abattn_params *p, int32_t *counts,
                            int32_t *idx, float *pi_sel, int64_t cap, float *pi_out, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if ((rc = check_plan_shape(dims, p))) return rc;
    if (S == nullptr || counts == nullptr || idx == nullptr || pi_sel == nullptr) return ABATTN_ERR_NULL;
    if (cap < 1 || cap > cdiv(dims->N, p->kv_block)) return ABATTN_ERR_SHAPE;
    if ((rc = check_device())) return rc;
    return launch_plan(p->mode == ABATTN_MODE_TOPK ? kPlanTopk : kPlanSip, S, dims, p, counts, idx, pi_sel,
                       cap, pi_out, static_cast<cudaStream_t>(stream));
}

int abattn_plan_from_pi(const float *pi, const abattn_dims *dims, const abattn_params *p, int32_t *counts,
                        int32_t *idx, float *pi_sel, int64_t cap, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if ((rc = check_plan_shape(dims, p))) return rc;
    if (pi == nullptr || counts == nullptr || idx == nullptr || pi_sel == nullptr) return ABATTN_ERR_NULL;
    if (cap < 1 || cap > cdiv(dims->N, p->kv_block)) return ABATTN_ERR_SHAPE;
    if ((rc = check_device())) return rc;
    return launch_plan(kPlanFromPi, pi, dims, p, counts, idx, pi_sel, cap, nullptr,
                       static_cast<cudaStream_t>(stream));
}

int abattn_plan(const void *Q, const void *K, const abattn_dims *dims, const abattn_params *p, int32_t *counts,
                int32_t *idx, float *pi_sel, int64_t cap, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if ((rc = check_plan_shape(dims, p))) return rc;
    if (Q == nullptr || K == nullptr || counts == nullptr || idx == nullptr || pi_sel == nullptr)
        return ABATTN_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K)) return ABATTN_ERR_ALIGN;
    if (cap < 1 || cap > cdiv(dims->N, p->kv_block)) return ABATTN_ERR_SHAPE;
    PlanWs w = carve(ws, dims, p);
    if (ws == nullptr || ws_bytes < w.bytes) return ABATTN_ERR_WORKSPACE;
    if (!aligned16(ws)) return ABATTN_ERR_ALIGN;
    if ((rc = check_device())) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = launch_meanpool(K, dims, p->kv_block, nullptr, w.Khi, w.Klo, st))) return rc;
    rc = dims->d == 128 ? launch_kmeans_t<128>(Q, dims, p, nullptr, w.w, nullptr, w.Chi, w.Clo, st)
                        : launch_kmeans_t<64>(Q, dims, p, nullptr, w.w, nullptr, w.Chi, w.Clo, st);
    if (rc) return rc;
    if ((rc = launch_score(w.Chi, w.Clo, w.Khi, w.Klo, w.w, dims, p, w.S, st))) return rc;
    return launch_plan(p->mode == ABATTN_MODE_TOPK ? kPlanTopk : kPlanSip, w.S, dims, p, counts, idx, pi_sel,
                       cap, nullptr, st);
}

int abattn_forward(const void *Q, const void *K, const void *V, const abattn_dims *dims, const abattn_params *p,
                   const int32_t *counts, const int32_t *idx, const float *pi_sel, int64_t cap, void *O,
                   float *lse, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, false))) return rc;
    if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr || counts == nullptr || idx == nullptr ||
        pi_sel == nullptr)
        return ABATTN_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return ABATTN_ERR_ALIGN;
    if (cap < 1 || cap > cdiv(dims->N, p->kv_block)) return ABATTN_ERR_SHAPE;
    return run_forward(false, Q, K, V, dims, p->kv_block, p->scale, counts, idx, pi_sel, cap, O, lse,
                       static_cast<cudaStream_t>(stream));
}

int abattn_quantize_e4m3(const void *X, const abattn_dims *dims, int rows_per_block, void *codes, float *scales,
                         void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (dims->d != 128) return ABATTN_ERR_SHAPE;
    if (rows_per_block < 1 || rows_per_block > 128 || (rows_per_block & (rows_per_block - 1)))
        return ABATTN_ERR_PARAM;
    if (X == nullptr || codes == nullptr || scales == nullptr) return ABATTN_ERR_NULL;
    if (!aligned16(X) || !aligned16(codes)) return ABATTN_ERR_ALIGN;
    if ((rc = check_device())) return rc;
    const int64_t batches = dims->B * dims->H;
    if (batches > 65535) return ABATTN_ERR_SHAPE;
    const dim3 grid(unsigned(cdiv(dims->N, QZ_THREADS)), unsigned(batches));
    quant_e4m3_kernel<<<grid, QZ_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16 *>(X), dims->N, rows_per_block, cdiv(dims->N, rows_per_block),
        static_cast<uint8_t *>(codes), scales);
    return launch_status();
}

int abattn_forward_e4m3(const void *Q8, const float *q_scales, const void *K8, const float *k_scales,
                        const void *V, const abattn_dims *dims, const abattn_params *p, const int32_t *counts,
                        const int32_t *idx, const float *pi_sel, int64_t cap, void *O, float *lse, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, false))) return rc;
    if (dims->d != 128 || dims->N % 4 != 0) return ABATTN_ERR_SHAPE;
    if (Q8 == nullptr || q_scales == nullptr || K8 == nullptr || k_scales == nullptr || V == nullptr ||
        O == nullptr || counts == nullptr || idx == nullptr || pi_sel == nullptr)
        return ABATTN_ERR_NULL;
    if (!aligned16(Q8) || !aligned16(K8) || !aligned16(V) || !aligned16(O)) return ABATTN_ERR_ALIGN;
    if (cap < 1 || cap > cdiv(dims->N, p->kv_block)) return ABATTN_ERR_SHAPE;
    return run_forward_e4m3(Q8, q_scales, K8, k_scales, V, dims, p->kv_block, p->scale, counts, idx, pi_sel, cap,
                            O, lse, static_cast<cudaStream_t>(stream));
}

int abattn_dense_forward(const void *Q, const void *K, const void *V, const abattn_dims *dims, float scale,
                         void *O, float *lse, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if (!(scale >= 0.f) || isinf(scale)) return ABATTN_ERR_PARAM;
    if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr) return ABATTN_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return ABATTN_ERR_ALIGN;
    return run_forward(true, Q, K, V, dims, 128, scale, nullptr, nullptr, nullptr, 1, O, lse,
                       static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ====================================================================== allocation-free plan
// A variant of abattn_plan whose scratch (mean keys, centroids, weights,
// scores and score statistics) lives in a fixed array compiled into this
// library, for callers that may not allocate device memory themselves.
namespace {

// 32 MiB per device, held until exit; the size is the header's, so the C
// limit and the documented one cannot drift apart
constexpr size_t kNoAllocScratchBytes = size_t(ABATTN_NOALLOC_SCRATCH_BYTES);

static __device__ __align__(256) unsigned char g_plan_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_plan_scratch on the current device.  The name of the
// array is only a host-side stand-in; the address comes from
// cudaGetSymbolAddress, looked up once per device with that device current
// and kept for the life of the process (a cudaDeviceReset after the first
// call would leave it stale, which the header rules out).
int scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return ABATTN_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_plan_scratch);
        if (e != cudaSuccess) return cuda_status(e);
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return ABATTN_OK;
}

}  // namespace

extern "C" int abattn_plan_noalloc(const void *Q, const void *K, const abattn_dims *dims, const abattn_params *p,
                                   int32_t *counts, int32_t *idx, float *pi_sel, int64_t cap, void *stream) {
    int rc = check_dims(dims);
    if (rc) return rc;
    if ((rc = check_params(p, true))) return rc;
    if (carve(nullptr, dims, p).bytes > kNoAllocScratchBytes) return ABATTN_ERR_WORKSPACE;
    if (Q == nullptr || K == nullptr || counts == nullptr || idx == nullptr || pi_sel == nullptr)
        return ABATTN_ERR_NULL;
    if ((rc = check_device())) return rc;
    void *scratch = nullptr;
    if ((rc = scratch_address(&scratch))) return rc;
    // Every byte of the scratch that the plan reads is written earlier in the
    // same call, so nothing has to be cleared between calls.
    return abattn_plan(Q, K, dims, p, counts, idx, pi_sel, cap, scratch, kNoAllocScratchBytes, stream);
}
