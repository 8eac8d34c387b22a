/*
 * abattn.h -- C ABI of the B200 (sm_100a) AB-Attention hot path.
 *
 * AB-Attention is training-free dynamic block-sparse softmax attention for
 * video diffusion transformers, described on two pages:
 *  [P1] "AB-Attention: Video Difuzyon Transformer'larini Hizlandirmak Icin
 *       Dogru Blok Dikkat Mekanizmasi" (edumints blog), section "AB-Attention
 *       ve Uc Temel Yeniligi" (the three innovations: IBCS, SIP, kernel).
 *  [P2] "AB-Attention yusarri' tawlid al-video hatta 2,23x ..." (hamidun
 *       news, Arabic), section "three techniques in AB-Attention": the IBCS,
 *       SIP and fine-grained-kernel paragraphs; the last one also says the
 *       sampling plan is rebuilt once every four denoising steps while the
 *       attention runs every step, hence the plan / forward split below.
 *  [P3], [P4] "Nunchux AI VC-Attention speeds up video DiT inference 3.58x"
 *       (dothoosh news, Persian) and "Nunchux AI ra mat VC-Attention"
 *       (aihot, Vietnamese): 8-bit (E4M3) attention on B200, the source of
 *       the optional E4M3 forward below; a different method, whose
 *       quantisation is not part of AB-Attention.
 *
 * Conventions for every entry point
 *  - Tensors are device pointers, caller-allocated and caller-owned; the
 *    library never allocates device memory and never synchronises, except
 *    abattn_check().  Q, K, V and O are bf16, contiguous [B][H][N][d] (row
 *    (b, h, n) at ((b*H + h)*N + n)*d), 16-byte aligned.
 *  - Rows of the plan are q-blocks r = (b*H + h)*nQB + qb, nQB = ceil(N/128);
 *    the last q-block of each head may be ragged (N - 128*(nQB-1) queries).
 *  - KV block j of a head covers keys [j*kv_block, min(N, (j+1)*kv_block));
 *    nKVB = ceil(N / kv_block).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *    enqueued asynchronously; errors found on the host are returned before
 *    anything is launched.  Errors found on the device (a bounded wait that
 *    ran out, a plan row that overflowed its capacity, an index out of range)
 *    set a device error word that abattn_check() reports and clears.
 *  - Return value: ABATTN_OK (0) or a negative ABATTN_ERR_* code.
 */
#ifndef ABATTN_H
#define ABATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ABATTN_OK 0
#define ABATTN_ERR_NULL (-1)          /* a required pointer is NULL */
#define ABATTN_ERR_SHAPE (-2)         /* B, H, N, d or a capacity out of range */
#define ABATTN_ERR_PARAM (-3)         /* q_block, kv_block, clusters, iters, budget, mode, scale */
#define ABATTN_ERR_ALIGN (-4)         /* a pointer is not 16-byte aligned */
#define ABATTN_ERR_WORKSPACE (-5)     /* workspace NULL or smaller than required */
#define ABATTN_ERR_PLAN_OVERFLOW (-6) /* device: a row selected more blocks than cap */
#define ABATTN_ERR_TIMEOUT (-7)       /* device: a bounded wait ran out; kernel returned early */
#define ABATTN_ERR_BOUNDS (-8)        /* device: a plan index outside [0, nKVB) was skipped */
#define ABATTN_ERR_CUDA (-9)          /* a CUDA runtime / driver call failed */
#define ABATTN_ERR_DEVICE (-10)       /* no sm_100 device, or a driver entry point missing */

#define ABATTN_MODE_SIP 0  /* water-filled pi, Poisson sampling, HT weights */
#define ABATTN_MODE_TOPK 1 /* top-k truncation baseline, weight 1 */

typedef struct {
    int64_t B, H, N, d; /* d must be 64 or 128; 1 <= N; B*H*nQB < 2^31 */
} abattn_dims;

typedef struct {
    int32_t q_block;      /* queries per q-block: must be 128 ([P2] IBCS paragraph) */
    int32_t kv_block;     /* tokens per KV block: 4, 8, 16, 32, 64 or 128 ([P2] kernel paragraph: 4) */
    int32_t n_clusters;   /* k-means clusters per q-block, 1..8 ([P2] IBCS paragraph: 8) */
    int32_t kmeans_iters; /* Lloyd iterations, 0..64 (pages silent; 10 used) */
    float budget;         /* (0, 1]: expected selected blocks per row = budget * nKVB */
    int32_t mode;         /* ABATTN_MODE_SIP or ABATTN_MODE_TOPK */
    uint64_t seed;        /* key of the counter-based uniform */
    float scale;          /* softmax scale; 0 means 1/sqrt(d) */
    int32_t head_offset;  /* global index of these tensors' first head (>= 0): a rank that plans a
                             slice of a layer's heads passes the slice's first head, so its uniforms,
                             counter (.., qb, head_offset + h, b), and hence its plan equal those rows
                             of the whole layer's plan; 0 for a whole layer */
} abattn_params;

/* Library identification string (static storage). */
const char *abattn_version(void);

/* Message for a status code (static storage). */
const char *abattn_strerror(int code);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns ABATTN_OK, ABATTN_ERR_PLAN_OVERFLOW, ABATTN_ERR_TIMEOUT,
 * ABATTN_ERR_BOUNDS or ABATTN_ERR_CUDA. */
int abattn_check(void *stream);

/* Per-row capacity of a plan for N tokens:
 * cap = min(nKVB, ceil(budget*nKVB + 8*sqrt(budget*nKVB) + 32)), an
 * 8-sigma margin over the expected Poisson-sampling count. */
int abattn_plan_capacity(const abattn_dims *dims, const abattn_params *p, int64_t *cap);

/* Workspace bytes needed by abattn_plan (mean keys, centroids, weights,
 * scores and score statistics, each 256-byte aligned). */
int abattn_plan_workspace_size(const abattn_dims *dims, const abattn_params *p, size_t *bytes);

/* Workspace bytes needed by abattn_score (per-centroid softmax statistics). */
int abattn_score_workspace_size(const abattn_dims *dims, const abattn_params *p, size_t *bytes);

/* Mean keys ([P2] IBCS paragraph: blocks are scored through their mean key).
 * K bf16 [B][H][N][d] -> Kbar fp32 [B][H][nKVB][d]; a ragged last block is
 * averaged over its true key count. */
int abattn_meanpool(const void *K, const abattn_dims *dims, int32_t kv_block, float *Kbar,
                    void *stream);

/* Intra-block clustering ([P2] IBCS paragraph: 8 clusters per 128-query
 * block, weight = share of the block's queries, no token reordering).
 * Lloyd's k-means in fp32: centroid c starts at query floor(c*M/nc);
 * nearest centroid by squared distance, ties to the lower index; an empty
 * cluster keeps its centroid; weights from the last assignment.
 * Q bf16 [B][H][N][d] -> C fp32 [rows][nc][d], w fp32 [rows][nc],
 * labels int32 [rows][128] (nullable; -1 past a ragged block's end). */
int abattn_kmeans(const void *Q, const abattn_dims *dims, const abattn_params *p, float *C,
                  float *w, int32_t *labels, void *stream);

/* Block scores ([P2] IBCS paragraph: weighted attention of the centroids to
 * the mean keys).  s_j = sum_c w_c * softmax_j(scale * C_c . Kbar_j), fp32
 * arithmetic, two passes (per-centroid max / normaliser, then the weighted
 * sum).  C, w as produced by abattn_kmeans, Kbar by abattn_meanpool ->
 * S fp32 [rows][nKVB].  ws: abattn_score_workspace_size bytes. */
int abattn_score(const float *C, const float *w, const float *Kbar, const abattn_dims *dims,
                 const abattn_params *p, float *S, void *ws, size_t ws_bytes, void *stream);

/* Planner from scores ([P1] SIP bullet, [P2] SIP paragraph).
 * SIP: pi_j = min(1, lambda*s_j) with sum_j pi_j = budget*nKVB (capping
 * iteration, sums in fp64, pi rounded to fp32); block j is taken iff
 * u_j < pi_j in fp32, u_j = (top 24 bits of the high (even j) or low (odd
 * j) 32-bit half of word (j/2)%4 of Philox4x64-10(counter (j/8, qb, h, b),
 * key (seed, 0))) times 2^-24.
 * TOPK: the floor(budget*nKVB + 0.5) highest scores, ties to the lower
 * index, weight 1.
 * Outputs per row, indices ascending: counts int32 [rows], idx int32
 * [rows][cap], pi_sel fp32 [rows][cap]; slots past counts are untouched.
 * pi_out fp32 [rows][nKVB] (nullable) receives pi (SIP only).
 * A row with more than cap selections stores cap of them, sets
 * counts = cap and raises ABATTN_ERR_PLAN_OVERFLOW in the error word. */
int abattn_plan_from_scores(const float *S, const abattn_dims *dims, const abattn_params *p,
                            int32_t *counts, int32_t *idx, float *pi_sel, int64_t cap,
                            float *pi_out, void *stream);

/* Sampling and compaction only, from given inclusion probabilities
 * pi fp32 [rows][nKVB] (same draw and layout as abattn_plan_from_scores). */
int abattn_plan_from_pi(const float *pi, const abattn_dims *dims, const abattn_params *p,
                        int32_t *counts, int32_t *idx, float *pi_sel, int64_t cap, void *stream);

/* The whole selector + planner: meanpool -> kmeans -> score ->
 * plan_from_scores.  ws: abattn_plan_workspace_size bytes. */
int abattn_plan(const void *Q, const void *K, const abattn_dims *dims, const abattn_params *p,
                int32_t *counts, int32_t *idx, float *pi_sel, int64_t cap, void *ws,
                size_t ws_bytes, void *stream);

/* Gathered block-sparse forward ([P2] SIP paragraph: each selected block
 * weighted by 1/pi, realised as a logit shift inside an ordinary softmax;
 * [P2] kernel paragraph: small KV blocks gathered by index into full
 * tensor-core tiles, tokens never reordered).  For each query i of row r:
 *   O_i = softmax over the selected keys t of (scale q_i.k_t + ln(1/pi_j(t))) . V
 * bf16 tensor-core products, fp32 accumulation and softmax.  Only
 * p->kv_block and p->scale are read from p.  Plan arrays as produced by
 * the planner.  O bf16 [B][H][N][d]; lse fp32 [B][H][N] (nullable) gets the
 * natural-log normaliser.  A row with no selected block gets O = 0,
 * lse = -inf. */
int abattn_forward(const void *Q, const void *K, const void *V, const abattn_dims *dims,
                   const abattn_params *p, const int32_t *counts, const int32_t *idx,
                   const float *pi_sel, int64_t cap, void *O, float *lse, void *stream);

/* E4M3 block quantisation for the 8-bit forward ([P3], [P4], B200 results:
 * 8-bit attention on Blackwell).  X bf16 [B][H][N][d] with d = 128 ->
 * codes [B][H][N][d] (one byte each) and scales fp32 [B][H][ceil(N / rpb)].
 * Each block of rows_per_block consecutive rows (a power of two from 1 to
 * 128; the last block of a head may be short) gets scale = amax / 448, amax
 * the largest |x| in the block (1 for a block of zeros), and each element the
 * E4M3 code of fp32(x * fp32(448 / amax)), rounded to nearest even and
 * saturated at +-448 (E4M3: 1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits).  Use 128 rows per block for Q (one scale per query block) and
 * p->kv_block for K (one scale per KV block).  Errors: ABATTN_ERR_SHAPE for
 * d != 128, ABATTN_ERR_PARAM for another block size; nothing is launched
 * after a host-side error. */
int abattn_quantize_e4m3(const void *X, const abattn_dims *dims, int rows_per_block, void *codes,
                         float *scales, void *stream);

/* The gathered block-sparse forward with QK^T in E4M3: as abattn_forward,
 * with Q and K given as abattn_quantize_e4m3 codes and scales (Q with 128
 * rows per block, K with p->kv_block), so that each logit is
 *   scale * q_scale[query block] * k_scale[KV block] * (Q8 . K8)
 *     + ln(1/pi_j)
 * from E4M3 tensor-core products with fp32 accumulation; P and V stay bf16,
 * as in abattn_forward.  Requires d = 128 and N % 4 == 0 (ABATTN_ERR_SHAPE
 * otherwise).  O bf16 [B][H][N][d]; lse fp32 [B][H][N] (nullable). */
int abattn_forward_e4m3(const void *Q8, const float *q_scales, const void *K8, const float *k_scales,
                        const void *V, const abattn_dims *dims, const abattn_params *p,
                        const int32_t *counts, const int32_t *idx, const float *pi_sel, int64_t cap,
                        void *O, float *lse, void *stream);

/* Dense softmax attention ([P1] bottleneck section: 3D full attention), the
 * full-budget reference, same kernel design over all keys.  scale 0 means
 * 1/sqrt(d). */
int abattn_dense_forward(const void *Q, const void *K, const void *V, const abattn_dims *dims,
                         float scale, void *O, float *lse, void *stream);

/* Allocation-free variant of abattn_plan.  The paper has no counterpart:
 * this is a convenience of this library.  Some callers cannot allocate
 * device memory, for instance a host whose runtime owns all device memory
 * through its own pool and forbids other allocations, or code that must not
 * allocate while it runs.  This entry point needs no workspace argument:
 * its scratch is an array of ABATTN_NOALLOC_SCRATCH_BYTES compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  Inputs and outputs are the caller's, as for abattn_plan, and the
 * results are the same.
 *  - Problems whose plan scratch (abattn_plan_workspace_size) exceeds
 *    ABATTN_NOALLOC_SCRATCH_BYTES are rejected with ABATTN_ERR_WORKSPACE
 *    before anything is launched.
 *  - The first call on a device looks up the scratch array's device address
 *    (cudaGetSymbolAddress) with that device current and keeps it for the
 *    life of the process; make that first call before any stream capture,
 *    and do not reset the device (cudaDeviceReset) after it.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents (nothing in it needs clearing: every value read is written
 *    earlier in the same call).  Calls that overlap on the GPU, e.g. on two
 *    streams at once, race on the array and must be serialised by the caller.
 *  - Never calls cudaMalloc, cudaFree or any allocating routine. */
#define ABATTN_NOALLOC_SCRATCH_BYTES (32u << 20)
int abattn_plan_noalloc(const void *Q, const void *K, const abattn_dims *dims, const abattn_params *p,
                        int32_t *counts, int32_t *idx, float *pi_sel, int64_t cap, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* ABATTN_H */
