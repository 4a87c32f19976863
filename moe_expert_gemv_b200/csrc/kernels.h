// kernels.h -- internal launch interface between the C-ABI layer (api.cu) and
// the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qmoe.h"

namespace qmoe {

struct LaunchCfg {
    cudaStream_t stream;
    int num_sms;
    bool pdl;   // launch as a programmatic dependent of the previous kernel
};

// ------------------------------------------------------------ dense qGEMV --
// weight formats of the dense qGEMV
enum QgemvFormat {
    QG_AFFINE = 0,   // w = s*q + b, fp16 scale and bias per group
    QG_ZP4 = 1,      // w = s*(q - z), bf16 scale, 4-bit zero point: params word s | z << 16
    QG_SYM8 = 2,     // w = s*q, two's-complement 8-bit codes, bf16 scale in params
};

struct QgemvArgs {
    const uint32_t *packed;
    const __half *scales, *biases;   // QG_AFFINE
    const uint32_t *params;          // QG_ZP4 / QG_SYM8: [N][K/64]
    const uint32_t *signs;           // block-32 Hadamard rotation of x, or null
    int N, K, bits, fmt;
    const __half *x;   // [B][K]
    int B;
    __half *y;         // [B][N]
    int32_t *status;
};
cudaError_t launch_qgemv(const QgemvArgs &a, const LaunchCfg &c);
// batch up to kMaxQgemvBatch: one launch per slice of 8 rows of x / y (the
// slices after the first read a matrix that fits L2 from L2)
constexpr int kMaxQgemvBatch = 32;
cudaError_t launch_qgemv_batched(const QgemvArgs &a, const LaunchCfg &c);
// One pass over the weights for batch 9..32 (qgemm_small.cu): the workspace
// (a 64 KB region of arrival counters, then fp32 partial tiles; zero-filled
// before first use, reusable across shapes) a
// call needs, 0 if the shape runs without one; the launch falls back to
// launch_qgemv_batched where the shape or alignment rule it out.  *used_ws
// reports whether the workspace was used.
size_t qgemm_small_workspace_bytes(int N, int K, int bits, int B, bool rot = false);
cudaError_t launch_qgemm_small(const QgemvArgs &a, void *ws, size_t ws_bytes, const LaunchCfg &c,
                               bool *used_ws);

// Tensor map over the 4/8-bit codes of a row-major [rows][Kw words] matrix
// (Kw % 32 == 0) as a 3-D tensor [Kw/32 chunks][rows][32 words]: one copy
// brings `box_chunks` 128-byte chunks (0: all, i.e. whole rows) of
// `box_rows` rows, 128-byte swizzled (16-byte unit u of row r, chunk c of
// the box at byte c*box_rows*128 + r*128 + 16*(u ^ (r & 7)) of a 1024-byte
// aligned destination).  False when the driver entry point is unavailable
// or refuses the shape.
bool encode_codes_map(CUtensorMap *m, const uint32_t *packed, long rows, int Kw, int box_rows,
                      int box_chunks = 0);
// 2-D map of a row-major 16-bit array [rows][cols] (no swizzle), boxes of
// box_cols x box_rows; false if the address, the row stride or the box width
// is not a multiple of 16 bytes.
bool encode_u16_map_2d(CUtensorMap *m, const void *base, long rows, int cols, int box_cols,
                       int box_rows);
// the same for a row-major 32-bit array (the parameter words of the formats)
bool encode_u32_map_2d(CUtensorMap *m, const void *base, long rows, int cols, int box_cols,
                       int box_rows);

// scale and folded-bias factor of one parameter word of the bf16 formats:
// ZP4 w = s(q - z) -> (s, -s z); SYM8 w = s(q' - 128) with q' = q + 128 -> (s, -128 s)
template <int FMT>
__device__ __forceinline__ void fmt_scale_bias(uint32_t p, float &s, float &b)
{
    s = __uint_as_float(p << 16);
    b = FMT == QG_ZP4 ? -s * (float)((p >> 16) & 0xFFu) : -128.f * s;
}

// ------------------------------------------------------------------ router --
struct RouterArgs {
    const uint32_t *packed;
    const __half *scales, *biases;
    int E, K, bits;
    const __half *x;   // [T][K]
    int T, top_k;
    int32_t *idx;      // [T][top_k]
    float *weights;    // [T][top_k]
    float *logits;     // [T][E] or null
    int32_t *status;
};
cudaError_t launch_router(const RouterArgs &a, const LaunchCfg &c);

// ------------------------------------------------------- decode experts --
struct QMat {
    const uint32_t *packed;
    const __half *scales, *biases;
};

struct ExpertWorkspace {
    float *h;          // [top_k + 1][inter]   (slot top_k: shared expert)
    float *part;       // [top_k + 1][hidden]
    int32_t *counters; // [hidden / 16]
};
size_t expert_workspace_layout(int hidden, int inter, int top_k, void *base, ExpertWorkspace *ws);
// The argument checks of moe_expert_qmlp (shapes, formats, top_k, pointers,
// alignment, device), run before anything is enqueued.
qmoe_status validate_expert_qmlp(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                                 const float *weights, int32_t top_k, const uint16_t *y,
                                 const int32_t *status_dev);

struct ExpertArgs {
    QMat gate, up, down, sh_gate, sh_up, sh_down;
    int E, H, I, top_k;
    const __half *x;        // [H]
    const int32_t *idx;     // [top_k]
    const float *weights;   // [top_k]
    __half *y;              // [H]
    ExpertWorkspace ws;
    int32_t *status;
    // expert parallelism: this rank computes the routed slots whose expert
    // e has e / (E / ep_world) == ep_rank, and the shared expert on rank 0;
    // gate/up/down stack only its experts, from expert ep_first on; with
    // y_part set, the sum of its slots goes there in fp32 instead of y
    int ep_rank = 0, ep_world = 1, ep_first = 0;
    float *y_part = nullptr;   // [H]
    // an explicit choice of slots instead (bit 0 the shared expert, bit j + 1
    // routed slot j), and an fp32 [H] vector added to the sum of those slots
    uint32_t slot_mask = 0;
    const float *y_add = nullptr;
};
cudaError_t launch_expert_gateup(const ExpertArgs &a, const LaunchCfg &c);
// moe_expert_qmlp restricted to the slots of slot_mask (see ExpertArgs),
// the sum written to y_part (fp32) when given, else y_add + sum to y (fp16)
qmoe_status expert_qmlp_slots(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                              const float *weights, int32_t top_k, uint32_t slot_mask,
                              float *y_part, const float *y_add, uint16_t *y, void *workspace,
                              size_t workspace_bytes, int32_t *status_dev, void *stream);
cudaError_t launch_expert_down(const ExpertArgs &a, const LaunchCfg &c);
cudaError_t launch_f32_to_f16(const float *src, __half *dst, long n, cudaStream_t s);

// ------------------------------------------------ fused multi-layer decode --
constexpr int kDecodeMaxLayers = 32;

struct DecodePackArgs {   // one MoE layer in the row-major (MLX) format
    QMat router, gate, up, down, sh_gate, sh_up, sh_down;
    int E, H, I;
};
size_t decode_pack_bytes(int E, int H, int I);
cudaError_t launch_decode_pack(const DecodePackArgs &a, void *dst, cudaStream_t s);

struct DecodeWorkspace {
    unsigned *ctl;   // control words: layer arrivals, abort, exit (zero between launches)
    float *y_acc;    // [2][H] fp32 layer outputs being summed (zero between launches)
};
size_t decode_workspace_layout(int E, int H, int I, int top_k, void *base, DecodeWorkspace *ws);

struct DecodeArgs {
    int L, E, H, I, top_k;
    int NS;               // ring stages (set by launch_decode)
    unsigned long long wait_ns = 2000000000ull;   // limit of every wait of the kernel (ns)
    const __half *x;      // [L][H]
    __half *y;            // [L][H]
    int32_t *idx;         // [L][top_k] or null
    float *weights;       // [L][top_k] or null
    float *logits;        // [L][E] or null
    DecodeWorkspace ws;
    int32_t *status;
    const void *layer[kDecodeMaxLayers];   // packed layers (decode_pack layout)
};
cudaError_t launch_decode(const DecodeArgs &a, const LaunchCfg &c);

// ---------------------------------------------------------------- prefill --
struct PrefillWorkspace {
    int32_t *counts;    // [E]
    int32_t *offsets;   // [E + 1]
    int32_t *pairs;     // [T * top_k]
    int32_t *inv;       // [T * top_k] position of each (token, slot) pair
    int32_t *tiles;     // 8-position token tiles of all slots: (slot << 4) | tile
    int32_t *unit_ctr;  // [4] gate/up and down work counters, number of tiles
    uint4 *xfrag;       // per position: x of its token in mma fragment order (+64 B pad)
    float *xsum;        // per position: group sums of x
    uint4 *hfrag;       // per position: h (hi, lo) fragments (+64 B pad)
    float *hsum;        // per position: group sums of h hi / lo
    float *r;           // [T * top_k + T][H] unweighted expert outputs per position
    // the tensor-core path of the heavy slots (prefill_tc.cu); activation rows
    // keep the k order (0,4,1,5,2,6,3,7) inside every 8 inputs
    int32_t *heavy;     // [E + 1] heavy slots, most tokens first (count in unit_ctr[3])
    __half *xg;         // [npos][H] x of each position's token
    __half *xb_hi;      // [npos][64] group sums of x, fp16 (hi, lo) pair, zero-padded
    __half *xb_lo;
    __half *hb_hi;      // [npos][I] h, fp16 (hi, lo) pair
    __half *hb_lo;
    __half *hs_hi;      // [npos][64] group sums of h (hi + lo), as a pair, zero-padded
    __half *hs_lo;
    float *tcpart;      // [kTcMaxCtas][128 rows][128 positions][gate, up] partial sums of
                        // the first half of K (each tensor-core CTA its own block)
};
size_t prefill_workspace_layout(int E, int hidden, int inter, int T, int top_k, void *base,
                                PrefillWorkspace *ws);
constexpr int kTcMaxCtas = 160;                         // tensor-core prefill CTAs at most
constexpr size_t kTcPartBytes = (size_t)128 * 128 * 2 * 4;   // one CTA's partial-sum block

struct GroupArgs {
    const int32_t *idx;
    int T, top_k, E;
    int32_t *counts, *offsets, *pairs;
    int32_t *status;
};
cudaError_t launch_group(const GroupArgs &a, const LaunchCfg &c);

struct PrefillArgs {
    QMat gate, up, down, sh_gate, sh_up, sh_down;
    int E, H, I, T, top_k;
    const __half *x;       // [T][H]
    const int32_t *idx;    // [T][top_k]
    const float *weights;  // [T][top_k]
    __half *y;             // [T][H]
    PrefillWorkspace ws;
    int32_t *status;
    int tc_min = 1 << 30;  // slots with at least this many tokens take the tensor-core path
};
cudaError_t launch_prefill(const PrefillArgs &a, const LaunchCfg &c);
// the heavy slots on tcgen05 (prefill_tc.cu): gate/up + SwiGLU, or down
cudaError_t launch_prefill_tc(const PrefillArgs &a, const LaunchCfg &c, bool down);
bool prefill_tc_supported(int hidden, int inter);
constexpr int kTcMinTokens = 16;
// the shared-memory ring of the grouped kernels holds at least two units
bool prefill_shape_supported(int hidden, int inter);

// ------------------------------------------------------------ pack helpers --
cudaError_t launch_pack(const uint8_t *codes, int rows, int cols, int bits, uint32_t *packed,
                        cudaStream_t s);
cudaError_t launch_unpack(const uint32_t *packed, int rows, int cols, int bits, uint8_t *codes,
                          cudaStream_t s);

// ---------------------------------------------------------------- helpers --
template <class Kern, class... Args>
cudaError_t launch_ex(Kern kernel, dim3 grid, dim3 block, size_t smem, const LaunchCfg &c,
                      int cluster_x, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute attrs[2];
    int n = 0;
    if (c.pdl) {
        attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_x > 1) {
        attrs[n].id = cudaLaunchAttributeClusterDimension;
        attrs[n].val.clusterDim.x = cluster_x;
        attrs[n].val.clusterDim.y = 1;
        attrs[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Opt a kernel into more than 48 KB of dynamic shared memory (once per
// device and kernel; cheap to repeat).
template <class Kern>
cudaError_t set_smem(Kern kernel, size_t bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace qmoe
