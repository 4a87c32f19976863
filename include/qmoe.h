/*
 * qmoe.h -- C ABI of libqmoe.so: affine-quantized GEMV and Mixture-of-Experts
 * decode / prefill kernels for NVIDIA B200 (sm_100a).
 *
 * What is computed, and where the pages say so:
 *   - Weights are "MLX affine 4-bit, group 64"; the router is 8-bit; the
 *     routed and shared experts are 4-bit (TurboFieldfare article, jeff.news,
 *     section "성능과 제약" -- performance and constraints).
 *     Reading of the format: element (n, k) of a row-major [rows][cols] matrix
 *     is  w = scale[n][k/64] * q + bias[n][k/64]  with q the unsigned code in
 *     bits [bits*(k%p), bits*(k%p)+bits) of word k/p of row n, p = 32/bits
 *     (least-significant field first); scale and bias are fp16.
 *   - Each layer's router runs on resident weights, picks the top-8 experts,
 *     and the routed experts' output is added to a resident shared expert's
 *     output; prefill runs in chunks of at most 128 tokens so one fetched
 *     expert serves many rows (same article, section "내부 구조가 진짜 흥미로운
 *     부분" -- internal structure).  Router weights are fp32-softmaxed and the
 *     top_k largest logits are kept (ties: lower expert index first), listed
 *     in descending order, renormalised to sum to one.  Experts are SwiGLU:
 *     r = down( silu(gate x) * (up x) ),  silu(z) = z / (1 + e^-z).
 *   - Quantized GEMV is one of the operations such a runtime hand-controls
 *     (same article, section "기술 맥락" -- technical context).
 *
 * Conventions for every entry point:
 *   - fp16 tensors are passed as uint16_t bit patterns; all tensor pointers
 *     are DEVICE pointers owned by the caller, row-major and densely packed.
 *     The three arrays of a qmoe_qmatrix must be 16-byte aligned; other
 *     fp16/fp32/int32 arrays naturally aligned (2/4/4 bytes).  Violations
 *     return QMOE_ERR_ALIGNMENT.
 *   - Weight operands (qmoe_qmatrix, qmoe_moe_layer) are read-only model
 *     parameters.  Kernels start streaming them before the previous kernel on
 *     the stream has finished (programmatic dependent launch), so a weight
 *     buffer must not be written by the kernel enqueued immediately before a
 *     call on the same stream: synchronise after writing weights, or turn the
 *     overlap off with qmoe_set_dependent_launch(0).  Activations, routing
 *     inputs and outputs are ordered as usual.
 *   - `stream` is a cudaStream_t (NULL: the legacy default stream).  Calls are
 *     asynchronous: they validate on the host, enqueue kernels and return.
 *     The library never allocates, frees or synchronises inside a compute
 *     call, with one stated exception: moe_cache_layer synchronises its
 *     stream once to read the router's choice on the host (its cache owns
 *     device slots allocated by qmoe_cache_create).  The current CUDA device
 *     must be the one that owns the pointers.
 *   - `status_dev` (optional, may be NULL) is a device int32 word that kernels
 *     OR device-detected problems into (QMOE_DEV_* flags).  With NULL the
 *     library's own per-device word is used.  qmoe_check_status() reads and
 *     clears it.  Kernels never trap: a bad expert id is skipped (its
 *     contribution is zero) and flagged; a pipeline wait that exceeds its
 *     time limit abandons the work and flags QMOE_DEV_TIMEOUT.
 *   - Host-side validation happens before any launch; on error nothing is
 *     enqueued.  A CUDA launch failure returns QMOE_ERR_CUDA.
 */
#ifndef QMOE_H
#define QMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qmoe_status {
    QMOE_OK = 0,
    QMOE_ERR_INVALID_ARG = -1,   /* NULL pointer, size out of range, shape mismatch */
    QMOE_ERR_ALIGNMENT = -2,     /* pointer not aligned as stated above */
    QMOE_ERR_UNSUPPORTED = -3,   /* valid request outside what the kernels implement */
    QMOE_ERR_CUDA = -4,          /* a CUDA runtime call failed */
    QMOE_ERR_DEVICE_STATUS = -5, /* qmoe_check_status: a kernel flagged bad input */
    QMOE_ERR_TIMEOUT = -6,       /* qmoe_check_status: a kernel wait timed out */
    QMOE_ERR_WORKSPACE = -7      /* workspace missing or smaller than required */
} qmoe_status;

/* flags OR-ed into the device status word */
#define QMOE_DEV_BAD_EXPERT 0x1  /* an expert id outside [0, num_experts) was skipped */
#define QMOE_DEV_TIMEOUT 0x2     /* a pipeline wait gave up; outputs are invalid */

/* One affine-quantized matrix (or a stack of equally-shaped matrices).
 *   packed: uint32 [rows][cols*bits/32]   (16-byte aligned)
 *   scales: fp16   [rows][cols/group]
 *   biases: fp16   [rows][cols/group]
 * bits is 4 or 8, group must be 64, cols a multiple of 64, rows a multiple
 * of 8.  For a stack (the routed experts) the matrices follow each other
 * with no gap: matrix e starts at packed + e*rows*cols*bits/32 and at
 * scales/biases + e*rows*cols/64. */
typedef struct qmoe_qmatrix {
    const uint32_t *packed;
    const uint16_t *scales;
    const uint16_t *biases;
    int32_t rows;
    int32_t cols;
    int32_t bits;
    int32_t group;
} qmoe_qmatrix;

/* One MoE layer: num_experts routed SwiGLU experts stacked in gate/up/down
 * (gate, up: rows = inter, cols = hidden; down: rows = hidden, cols = inter;
 * 4-bit), plus the always-resident shared expert of the same shapes.
 * The router is a separate qmoe_qmatrix (rows = num_experts, cols = hidden,
 * 8-bit) handed to moe_router_topk. */
typedef struct qmoe_moe_layer {
    qmoe_qmatrix gate, up, down;          /* routed experts, stacked */
    qmoe_qmatrix sh_gate, sh_up, sh_down; /* shared expert */
    int32_t num_experts;
    int32_t hidden;
    int32_t inter;
} qmoe_moe_layer;

/* ---------------------------------------------------------------------------
 * Dense affine qGEMV, batch 1..32 (decode projection; quantized GEMV of the
 * "기술 맥락" section, format of the "성능과 제약" section).
 *   y[b][n] = sum_k w[n][k] * x[b][k]     fp32 accumulate, fp16 output
 *   W: bits 4 or 8; x: fp16 [batch][W->cols]; y: fp16 [batch][W->rows].
 * batch 1..32: up to 8 rows of x per kernel launch (tensor-core N = 8); a
 * larger batch (e.g. the 16-32 draft tokens a speculative-decoding step
 * verifies) runs one launch per 8 rows, the later ones reading a matrix
 * that fits L2 from L2.  Where 8 rows of x beside one 16-row weight tile
 * overflow shared memory (long 8-bit rows, e.g. cols 8192), each launch
 * takes as many rows as fit.
 * Errors: INVALID_ARG (NULL, batch outside 1..32, shape), ALIGNMENT,
 * UNSUPPORTED (group != 64, cols % 64, rows % 8, or rows too long for one
 * row of x plus one 16-row tile in shared memory: cols above 18624 at 4 bits,
 * 10944 at 8 bits; qgemv_affine_ws takes such rows from batch 9 on), CUDA.
 * ------------------------------------------------------------------------- */
qmoe_status qgemv_affine(const qmoe_qmatrix *W, const uint16_t *x, int32_t batch,
                         uint16_t *y, int32_t *status_dev, void *stream);

/* ---------------------------------------------------------------------------
 * The same product for batch 9..32 in ONE pass over the weights (the
 * verification step of speculative decoding multiplies every projection by
 * the 16-32 draft tokens at once; uzu page, discuss.pytorch.kr, section "uzu의
 * 추측 디코딩 구조").  The K range is split into S slices whose x fits on chip; CTAs
 * of different slices write fp32 partial tiles to `workspace` and the last
 * one to finish a tile adds them in slice order (results do not depend on
 * the order in which CTAs finish; they differ from qgemv_affine's only by
 * fp32 rounding).
 * qgemv_affine_workspace_bytes(rows, cols, bits, batch): bytes of workspace a
 *   call of that shape needs; 0 when it needs none (batch <= 8, one slice,
 *   or a shape the one-pass kernel does not take: then qgemv_affine_ws runs
 *   qgemv_affine's path).  The one-pass kernel takes rows of whole 128-byte
 *   code chunks (cols % 256 == 0 at 4 bits, % 128 at 8 bits), slices of a
 *   multiple of 512 inputs, x and scales / biases 16-byte aligned (otherwise
 *   it runs qgemv_affine's path even where a workspace was asked for).
 * workspace: device memory, 16-byte aligned, at least that many bytes,
 *   zero-filled once before its first use.  Its first 64 KB hold per-tile
 *   arrival counters that every call returns to zero, the rest fp32 partial
 *   tiles, so one workspace serves calls of any shape in turn; it must not
 *   be used by two calls that can run at the same time.  May be NULL when
 *   the size is 0.
 * Errors: as qgemv_affine; INVALID_ARG also for a missing or short workspace,
 * ALIGNMENT for a workspace not 16-byte aligned.
 * ------------------------------------------------------------------------- */
size_t qgemv_affine_workspace_bytes(int32_t rows, int32_t cols, int32_t bits, int32_t batch);
qmoe_status qgemv_affine_ws(const qmoe_qmatrix *W, const uint16_t *x, int32_t batch, uint16_t *y,
                            void *workspace, size_t workspace_bytes, int32_t *status_dev,
                            void *stream);

/* ---------------------------------------------------------------------------
 * Format variants of the dense qGEMV (uzu page, discuss.pytorch.kr, section
 * "uzu의 모델 변환과 Mirai 양자화 형식": Mirai-M is 4-bit asymmetric with a
 * 4-bit zero point and a bf16 scale, group 64; Mirai-L is 8-bit symmetric;
 * both quantise after a random Hadamard transform of block size 32).
 *   QMOE_FMT_ZP4_BF16:  w = s * (q - z), q 4-bit unsigned codes (packed as
 *                       qmoe_qmatrix, 8 per word), z the zero point 0..15
 *   QMOE_FMT_SYM8_BF16: w = s * q, q 8-bit two's-complement codes (4 per word)
 *   params: uint32 [rows][cols/64], 16-byte aligned: bits 0..15 the bf16
 *           scale s, bits 16..23 the zero point z (0 for SYM8)
 *   rht_signs: NULL, or uint32 [cols/32] (4-byte aligned): the weights were
 *           quantised in a rotated basis and the product is
 *             y[b] = W (R x[b]),  R = blockdiag(H_32 D / sqrt(32)),
 *           H_32[i][j] = (-1)^popcount(i & j), D[i][i] = -1 where bit i % 32
 *           of rht_signs[i / 32] is set.  x must then be 16-byte aligned; the
 *           rotation runs in fp32 inside the kernel and R x enters the product
 *           as an fp16 (hi, lo) pair (about 22 significant bits).
 * batch 1..32 (as qgemv_affine); cols a multiple of 64, rows of 8;
 * y fp16 [batch][rows].  Errors as qgemv_affine (INVALID_ARG also for an
 * unknown format; with rht_signs the x pair halves the room, and rows of
 * more than 15872 cols at 4 bits or 9984 at 8 bits are UNSUPPORTED).
 * ------------------------------------------------------------------------- */
#define QMOE_FMT_ZP4_BF16 1
#define QMOE_FMT_SYM8_BF16 2

typedef struct qmoe_qmatrix_fmt {
    const uint32_t *packed;
    const uint32_t *params;
    const uint32_t *rht_signs;
    int32_t rows;
    int32_t cols;
    int32_t group;
    int32_t format;
} qmoe_qmatrix_fmt;

qmoe_status qgemv_fmt(const qmoe_qmatrix_fmt *W, const uint16_t *x, int32_t batch, uint16_t *y,
                      int32_t *status_dev, void *stream);

/* The format variants for batch 9..32 in ONE pass over the weights, with the
 * same workspace contract as qgemv_affine_workspace_bytes / qgemv_affine_ws
 * (uzu page, "uzu의 추측 디코딩 구조": the 16-32 draft tokens of a
 * verification step multiply every projection at once).  rotated != 0: the
 * call will pass rht_signs (the rotated x is kept as an fp16 (hi, lo) pair,
 * which halves the inputs of a slice).  Shapes the one-pass kernel does not
 * take, and batch <= 8, run qgemv_fmt's path. */
size_t qgemv_fmt_workspace_bytes(int32_t rows, int32_t cols, int32_t format, int32_t rotated,
                                 int32_t batch);
qmoe_status qgemv_fmt_ws(const qmoe_qmatrix_fmt *W, const uint16_t *x, int32_t batch, uint16_t *y,
                         void *workspace, size_t workspace_bytes, int32_t *status_dev,
                         void *stream);

/* ---------------------------------------------------------------------------
 * Router + softmax + top-k + renormalisation ("내부 구조" section: the router
 * runs on resident weights and picks the top-8 experts).
 *   logits[t][e] = sum_k w_router[e][k] x[t][k]    (fp32)
 *   idx[t][0..top_k): the top_k largest logits, descending, ties -> lower e
 *   weights[t][j] = softmax(logits[t])[idx[t][j]] / sum_j' softmax(...)[idx[t][j']]
 * router: rows = num_experts (a multiple of 8, at most 128), bits 4 or 8.
 * x: fp16 [tokens][router->cols], tokens 1..65536; top_k 1..min(16, rows).
 * idx: int32 [tokens][top_k]; weights: fp32 [tokens][top_k];
 * logits: fp32 [tokens][rows] or NULL.
 * Selection uses exactly the fp32 logits written to `logits`.
 * ------------------------------------------------------------------------- */
qmoe_status moe_router_topk(const qmoe_qmatrix *router, const uint16_t *x, int32_t tokens,
                            int32_t top_k, int32_t *idx, float *weights, float *logits,
                            int32_t *status_dev, void *stream);

/* ---------------------------------------------------------------------------
 * Decode MoE layer for one token ("내부 구조" section: routed experts computed
 * from the router's top-8 ids, added to the shared expert's output):
 *   y = shared(x) + sum_j weights[j] * expert_{idx[j]}(x)
 *   expert(x) = down( silu(gate x) * (up x) ), all intermediates fp32.
 * x: fp16 [hidden]; idx: int32 [top_k] (device memory, e.g. written by
 * moe_router_topk); weights: fp32 [top_k]; y: fp16 [hidden]; top_k 1..16.
 * Shapes: hidden and inter multiples of 64; hidden a multiple of 16.
 * workspace: device memory of moe_expert_workspace_bytes() bytes, 16-byte
 * aligned, ZERO-FILLED before its first use (e.g. cudaMemsetAsync).  Every
 * successful call leaves it zero-filled again, so it can be reused by later
 * calls on the same stream (also inside CUDA graphs); calls that overlap in
 * time need separate workspaces.  After a QMOE_DEV_TIMEOUT re-zero it.
 * An idx entry outside [0, num_experts) contributes zero and raises
 * QMOE_DEV_BAD_EXPERT.
 * moe_expert_qmlp == moe_expert_gateup followed by moe_expert_down on the
 * same workspace; the two halves are exported for measurement.
 * ------------------------------------------------------------------------- */
size_t moe_expert_workspace_bytes(const qmoe_moe_layer *L, int32_t top_k);

qmoe_status moe_expert_qmlp(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                            const float *weights, int32_t top_k, uint16_t *y, void *workspace,
                            size_t workspace_bytes, int32_t *status_dev, void *stream);

/* ---------------------------------------------------------------------------
 * Expert-parallel share of the same layer: with the experts split over
 * `world` ranks (rank r holds experts r*E/world .. (r+1)*E/world - 1) and the
 * router replicated, rank `rank` computes only the routed slots whose expert
 * it holds, plus the shared expert on rank 0.  L->num_experts is the global
 * E; L->gate, up and down stack only the E/world experts this rank holds
 * (local expert i is global expert rank*E/world + i):
 *   y_partial = [rank == 0] shared(x) + sum_{j: idx[j] held here} weights[j] expert_{idx[j]}(x)
 * in fp32, so that the sum over ranks (one all-reduce of [hidden] fp32) is
 * the layer output before its rounding to fp16 (qmoe_f32_to_f16).  Only the
 * weights of the held experts are read.  A rank that holds none of the
 * chosen experts (and is not rank 0) gets zeros.  An invalid id belongs to
 * no rank.  world divides num_experts; rank in 0..world-1.  y_partial: fp32
 * [hidden], 4-byte aligned.  Workspace and errors as moe_expert_qmlp.
 * (Page: the routed experts of a token are independent products added
 * together, TurboFieldfare article, section "내부 구조가 진짜 흥미로운 부분".)
 * ------------------------------------------------------------------------- */
qmoe_status moe_expert_qmlp_ep(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                               const float *weights, int32_t top_k, int32_t rank, int32_t world,
                               float *y_partial, void *workspace, size_t workspace_bytes,
                               int32_t *status_dev, void *stream);

/* fp32 [n] -> fp16 [n], round to nearest even, on `stream`. */
qmoe_status qmoe_f32_to_f16(const float *src, uint16_t *dst, int64_t n, void *stream);

/* moe_expert_qmlp for callers that cannot allocate device memory.  The pages
 * have no counterpart: this exists for callers with no way to obtain a
 * workspace -- a plugin or embedded runtime handed only a stream and tensor
 * pointers, a framework whose memory pool may not be touched from the calling
 * thread, a real-time path that must not enter an allocator.  It computes
 * exactly what moe_expert_qmlp computes, using a scratch buffer built into
 * the library: a 1 MiB __device__ array that every GPU loading the library
 * holds until the process exits.  Requests whose workspace
 * (moe_expert_workspace_bytes) exceeds 1 MiB return QMOE_ERR_WORKSPACE.
 * It allocates and frees nothing.  Every call looks up the array's device
 * address in the current device's context (nothing is cached, so a new
 * context after a device reset is picked up); `stream` must belong to the
 * current device.  The first call on a device also loads the array's module
 * there, so make that first call before any stream capture.  A call checks
 * all of its arguments before it enqueues anything: a rejected call leaves
 * the stream and the buffer untouched.  An accepted call clears the buffer's
 * counters on `stream` before its kernels run.  Every call shares the one
 * buffer, so calls that overlap on the GPU (for instance on two streams)
 * race. */
qmoe_status moe_expert_qmlp_noalloc(const qmoe_moe_layer *L, const uint16_t *x,
                                    const int32_t *idx, const float *weights, int32_t top_k,
                                    uint16_t *y, int32_t *status_dev, void *stream);

/* h_j = silu(gate_e x) * (up_e x) for the top_k routed experts e = idx[j] and
 * the shared expert (slot top_k), fp32, kept in the workspace. */
qmoe_status moe_expert_gateup(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                              int32_t top_k, void *workspace, size_t workspace_bytes,
                              int32_t *status_dev, void *stream);

/* y = down_shared h_shared + sum_j weights[j] * down_{idx[j]} h_j, fp16, from
 * the h left in the workspace by moe_expert_gateup. */
qmoe_status moe_expert_down(const qmoe_moe_layer *L, const int32_t *idx, const float *weights,
                            int32_t top_k, uint16_t *y, void *workspace, size_t workspace_bytes,
                            int32_t *status_dev, void *stream);

/* ---------------------------------------------------------------------------
 * The decode loop over a stack of MoE layers for one token per layer, fused
 * into one persistent launch ("내부 구조" section: the router picks the top-8
 * experts of each layer, the shared expert's output is added to the routed
 * output, and generation repeats this routed-layer loop token by token).
 *
 * The layers are first repacked once (like the pages' install-time repack)
 * into the kernel's streaming layout: every work item's codes, scales and
 * biases become one contiguous block, so each item is a single large copy.
 * The packed layer holds exactly the bytes of the row-major one (router +
 * all experts + shared expert), permuted.
 *   moe_decode_pack_bytes(L)            bytes of one packed layer
 *   moe_decode_pack_layer(L, router, packed, bytes, stream)
 *       L: the layer in the row-major format; router: rows = num_experts
 *       (<= 128, a multiple of 8), cols = hidden, 8-bit; hidden % 256 == 0,
 *       inter % 64 == 0.  packed: device memory, 16-byte aligned.
 *
 * For each layer l < n_layers (packed_layers: host array of device pointers):
 *   logits = router_l x[l];  idx[l], weights[l] = top_k of softmax(logits)
 *   y[l] = shared_l(x[l]) + sum_j weights[l][j] * expert_{l, idx[l][j]}(x[l])
 * with the arithmetic of moe_router_topk followed by moe_expert_qmlp (fp32
 * accumulation of exact products).  Layer l+1 starts after layer l has
 * finished, as it would if it consumed y[l]; the weights of later layers
 * that do not depend on the routing are streamed ahead of time.  The parts
 * of a layer output computed on different SM clusters are added with fp32
 * atomics, so the last bits of y may differ from call to call (the routing,
 * idx, weights and logits do not).
 * x, y: fp16 [n_layers][hidden], x 16-byte aligned (it is read 16 bytes at a
 * time); idx: int32 [n_layers][top_k], weights: fp32 [n_layers][top_k],
 * logits: fp32 [n_layers][num_experts]; idx, weights and logits may be
 * NULL.  top_k 1..16.
 * workspace: moe_decode_workspace_bytes() bytes (control words and two fp32
 * [hidden] layer accumulators), 16-byte aligned, ZERO-FILLED before first
 * use; each successful call leaves it zero-filled again (after a call whose
 * status word reports a timeout, zero it again).  Calls sharing a workspace
 * must not overlap in time.  Stacks of more than 32 layers are processed 32
 * layers per launch.  The launch is cooperative, in clusters of 8 CTAs (one
 * CTA per SM, as many clusters as fit at once: 15 on a 148-SM B200); it fails
 * with QMOE_ERR_CUDA if the GPU is busy with other work that prevents
 * co-residency.
 * ------------------------------------------------------------------------- */
size_t moe_decode_pack_bytes(const qmoe_moe_layer *L);

qmoe_status moe_decode_pack_layer(const qmoe_moe_layer *L, const qmoe_qmatrix *router,
                                  void *packed, size_t packed_bytes, void *stream);

size_t moe_decode_workspace_bytes(int32_t num_experts, int32_t hidden, int32_t inter,
                                  int32_t top_k);

qmoe_status moe_decode_layers(const void *const *packed_layers, int32_t n_layers,
                              int32_t num_experts, int32_t hidden, int32_t inter,
                              const uint16_t *x, int32_t top_k, uint16_t *y, int32_t *idx,
                              float *weights, float *logits, void *workspace,
                              size_t workspace_bytes, int32_t *status_dev, void *stream);

/* moe_decode_layers from HOST buffers: x_host -> x_dev (cudaMemcpyAsync), the
 * fused decode, y_dev -> y_host, all enqueued on `stream` in that order (the
 * call returns at once; synchronise the stream before reading y_host).
 * x_host, y_host: fp16 [n_layers][hidden] in host memory (pinned memory lets
 * the copies run asynchronously); x_dev (16-byte aligned), y_dev: device
 * staging buffers of the same size owned by the caller -- the library still
 * allocates nothing.  Checks as moe_decode_layers, made before any copy. */
qmoe_status moe_decode_layers_host(const void *const *packed_layers, int32_t n_layers,
                                   int32_t num_experts, int32_t hidden, int32_t inter,
                                   const uint16_t *x_host, uint16_t *y_host, int32_t top_k,
                                   uint16_t *x_dev, uint16_t *y_dev, void *workspace,
                                   size_t workspace_bytes, int32_t *status_dev, void *stream);

/* ---------------------------------------------------------------------------
 * Host-memory expert streaming through a per-layer LFU cache (TurboFieldfare
 * article, "내부 구조" section: the CPU takes the router's top-8 ids, plans
 * the misses against the layer's 16-slot LFU cache and fills the missed
 * experts into device-visible memory before the routed experts run).
 *
 * Plan, per token (readings; the page names the policy only): the token's
 * hits first -- the slot's use count grows by one and the slot is pinned for
 * this token -- then its misses in id order: the lowest-index empty slot,
 * else the unpinned slot with the smallest count (ties: lowest index); a
 * loaded expert starts at count 1; an evicted expert's count is forgotten.
 *
 * qmoe_lfu_*: the plan alone, host memory only (no GPU needed).
 *   qmoe_lfu_plan returns the number of misses (listed in order as
 *   miss_expert[i] -> miss_slot[i]) and fills slot_of[j] for ids[j]; -1 if
 *   k > nslots, k > 16 or the ids repeat (the state is then unchanged).
 *
 * qmoe_cache_create: `host` holds the layer's routed experts (gate, up, down
 * stacked over num_experts) in PINNED HOST memory; `slots` the same three
 * stacks over nslots = slots->num_experts in device memory, plus the resident
 * shared expert (device).  The cache starts empty.  Allocates its own small
 * pinned and device buffers and an event; qmoe_cache_destroy frees them.
 *
 * moe_cache_layer: one decode token through the layer:
 *   router (resident, device) -> the host reads the top_k ids (this call
 *   SYNCHRONISES `stream` once; every other entry point never does) -> plan
 *   -> each missed expert's nine arrays host -> device, the misses spread
 *   over four copy streams (the first is `copy_stream` when given, the
 *   others the cache's own) -> meanwhile the shared expert runs on `stream`
 *   (it needs no copy; its output is kept in fp32) -> the routed experts
 *   wait for the copies -> y = shared(x) + sum_j weights[j] *
 *   expert_{idx[j]}(x) from the slots, rounded once (the arithmetic of
 *   moe_expert_qmlp; same zero-filled workspace).  idx_out / weights_out
 *   (device, optional) receive the router's choice.  Returns
 *   QMOE_ERR_DEVICE_STATUS if the router produced an id outside [0, E)
 *   (the cache unchanged).  If a copy or launch fails after the plan, the
 *   cache forgets every slot (all empty) so that no later token trusts a
 *   slot whose copy may not have landed.
 * qmoe_cache_stats: cumulative hits, misses, bytes copied; the expert held by
 * each slot (-1: empty).
 * ------------------------------------------------------------------------- */
typedef struct qmoe_lfu qmoe_lfu;
typedef struct qmoe_expert_cache qmoe_expert_cache;

qmoe_status qmoe_lfu_create(int32_t nslots, qmoe_lfu **out);
void qmoe_lfu_destroy(qmoe_lfu *h);
int32_t qmoe_lfu_plan(qmoe_lfu *h, const int32_t *ids, int32_t k, int32_t *slot_of,
                      int32_t *miss_expert, int32_t *miss_slot);
qmoe_status qmoe_lfu_slots(const qmoe_lfu *h, int32_t *expert, int64_t *count);

qmoe_status qmoe_cache_create(const qmoe_moe_layer *host, const qmoe_moe_layer *slots,
                              qmoe_expert_cache **out);
void qmoe_cache_destroy(qmoe_expert_cache *c);
qmoe_status moe_cache_layer(qmoe_expert_cache *c, const qmoe_qmatrix *router, const uint16_t *x,
                            int32_t top_k, uint16_t *y, int32_t *idx_out, float *weights_out,
                            void *workspace, size_t workspace_bytes, int32_t *status_dev,
                            void *stream, void *copy_stream);
qmoe_status qmoe_cache_stats(const qmoe_expert_cache *c, int64_t *hits, int64_t *misses,
                             int64_t *bytes_copied, int32_t *slot_expert);

/* ---------------------------------------------------------------------------
 * Prefill grouping ("내부 구조" section: a chunk's tokens are gathered per
 * expert so one fetched expert serves many rows).
 *   counts[e]  = number of (token, slot) pairs with idx == e
 *   offsets[0..num_experts] = exclusive prefix sum of counts
 *   pairs[offsets[e] .. offsets[e+1]) = flat indices t*top_k + j with
 *                                       idx[t][j] == e, ascending
 * idx: int32 [tokens][top_k], tokens 1..128, top_k 1..16, num_experts 1..256.
 * An id outside [0, num_experts) raises QMOE_DEV_BAD_EXPERT and is dropped.
 * ------------------------------------------------------------------------- */
qmoe_status moe_group_tokens(const int32_t *idx, int32_t tokens, int32_t top_k,
                             int32_t num_experts, int32_t *counts, int32_t *offsets,
                             int32_t *pairs, int32_t *status_dev, void *stream);

/* ---------------------------------------------------------------------------
 * Prefill chunk through the MoE layer as a grouped qGEMM (same formula as
 * moe_expert_qmlp, row by row):
 *   y[t] = shared(x[t]) + sum_j weights[t][j] * expert_{idx[t][j]}(x[t])
 * x: fp16 [tokens][hidden], 16-byte aligned, tokens 1..128; idx: int32 [tokens][top_k];
 * weights: fp32 [tokens][top_k]; y: fp16 [tokens][hidden], 4-byte aligned.
 * workspace: moe_prefill_workspace_bytes() bytes, 16-byte aligned; no
 * initial contents are required.
 * Weights are streamed per 8-token tile of each expert: an expert with at
 * most 8 tokens in the chunk is read once, a heavier one once per tile (the
 * repeats served by L2).  Returns QMOE_ERR_UNSUPPORTED unless hidden is a
 * multiple of 256 and at most 4,352 and inter is at most 2,176 (two
 * activation tiles and two weight sub-blocks must fit shared memory).
 * ------------------------------------------------------------------------- */
size_t moe_prefill_workspace_bytes(const qmoe_moe_layer *L, int32_t tokens, int32_t top_k);

qmoe_status moe_prefill_qgemm(const qmoe_moe_layer *L, const uint16_t *x, int32_t tokens,
                              const int32_t *idx, const float *weights, int32_t top_k,
                              uint16_t *y, void *workspace, size_t workspace_bytes,
                              int32_t *status_dev, void *stream);

/* ---------------------------------------------------------------------------
 * Format helpers (the packing reading of the "성능과 제약" section).
 * codes: uint8 [rows][cols] (values >= 2^bits are masked); packed: uint32
 * [rows][cols*bits/32].  cols must be a multiple of 32/bits.
 * ------------------------------------------------------------------------- */
qmoe_status qmoe_pack_codes(const uint8_t *codes, int32_t rows, int32_t cols, int32_t bits,
                            uint32_t *packed, void *stream);
qmoe_status qmoe_unpack_codes(const uint32_t *packed, int32_t rows, int32_t cols, int32_t bits,
                              uint8_t *codes, void *stream);

/* Synchronises `stream`, reads and clears the status word (NULL: the
 * library's word on the current device).  Returns QMOE_OK, QMOE_ERR_TIMEOUT
 * (if QMOE_DEV_TIMEOUT was set), QMOE_ERR_DEVICE_STATUS (other flags) or
 * QMOE_ERR_CUDA.  If flags_out is not NULL it receives the raw flags. */
qmoe_status qmoe_check_status(int32_t *status_dev, void *stream, int32_t *flags_out);

/* Static, human-readable name of a status code. */
const char *qmoe_status_string(qmoe_status s);

/* Enable (1, the default) or disable (0) programmatic dependent launch for
 * all later calls in this process.  Returns the previous setting. */
int32_t qmoe_set_dependent_launch(int32_t enable);

/* Time limit of every wait inside moe_decode_layers (a wait that does not
 * complete in time flags QMOE_DEV_TIMEOUT, stops the whole launch and lets it
 * return), in nanoseconds; 0 restores the default of 2 s.  Applies to later
 * calls in this process; returns the previous setting. */
uint64_t qmoe_set_decode_wait_limit_ns(uint64_t ns);

/* Experts of a prefill chunk (and the shared expert) with at least
 * `min_tokens` tokens run on the tensor-core (tcgen05) kernels, the others on
 * the streaming kernels; 0 (the default) sends every expert to the streaming
 * kernels, which are the faster choice on skewed (Zipf) routing; 16 is the
 * threshold the tests use when they switch the tensor-core path on.  Shapes
 * the tensor-core kernels do not take stay on the streaming kernels.
 * Applies to later moe_prefill_qgemm calls in this process; returns the
 * previous setting. */
int32_t qmoe_set_prefill_tensor_min(int32_t min_tokens);

/* Library version, major*10000 + minor*100 + patch. */
int32_t qmoe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QMOE_H */
