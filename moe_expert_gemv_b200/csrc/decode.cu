// decode.cu -- persistent fused MoE decode over a stack of layers: for every
// layer, router GEMV -> top-k -> gathered routed SwiGLU experts + resident
// shared expert -> weighted combine, in ONE launch.
//
// TurboFieldfare article (jeff.news), section "내부 구조가 진짜 흥미로운 부분"
// (internal structure): per layer the router runs from resident weights and
// picks the top-8 experts, the shared-expert branch runs beside the routed
// experts and the two outputs are added; generation repeats this routed-layer
// loop token by token.  Format: MLX affine 4-bit experts, 8-bit router, group
// 64 (section "성능과 제약").
//
// B200 design.  One CTA per SM (cooperative launch): 16 consumer warps in 8
// pairs, a static producer warp and a routed producer warp.  The weights of a
// decode step are one long HBM stream and the kernel keeps it going:
//   * static producer: tiles whose address is known in advance (router, the
//     shared expert) in a small ring that runs up to a layer ahead;
//   * routed producer: the routed experts' tiles, issued as soon as the
//     layer's top-k is known, in a deep ring.
// Every item is ONE ~13 KB cp.async.bulk copy: the layer's weights are
// repacked once (moe_decode_pack_layer) so that each item's codes, scales and
// biases are contiguous in HBM, with the 16-byte chunks of each row permuted
// so that the fragment loads from shared memory are free of bank conflicts
// (bulk copies move far fewer bytes per operation when they are small, so
// per-row copies of the row-major format could not keep HBM busy).  A pair of
// warps takes one item and splits its K loop (or its two 16-row tiles).
// Cross-CTA dependencies are arrival counters in the workspace, each waited
// on only where the data is needed:
//   lcount   router items done           -> every CTA computes the top-k;
//   ready[s] gate/up items of slot s done -> down items of slot s may start;
//   done     down tiles combined          -> the next layer may start (its
//            input would be this layer's output in a real model).
// Every wait is bounded; a timeout flags QMOE_DEV_TIMEOUT, raises a shared
// abort word and lets the kernel drain its copies and return.
//
// Items (every one ~12.7 KB of packed weights + scales + biases):
//   R  : 8 router rows x half of K (8-bit).  The 16-row mma tile holds the 8
//        rows twice, over the two quarters of K; the two quarters use x of
//        different groups as batch columns 0 and 1.
//   GU : 4 gate rows + 4 up rows of one expert x full K; the tile holds the
//        8 rows over the two halves of K (same column trick), so one thread
//        ends with gate and up partials of the same index and applies SwiGLU
//        in registers.  h is written as an fp16 (hi, lo) pair in the
//        fragment order of the down projection.
//   DN : 32 rows of one expert's down projection x full K (two 16-row mma
//        tiles, one per warp of the pair); h (hi, lo) are batch columns 0
//        and 1.  The expert partials of a 32-row tile are combined in slot
//        order by the warp that finishes the tile last (arrival counter,
//        reset by that warp).
// The shared expert's gate/up items need only x, so they run before the
// router's result is known.
#include "common.cuh"
#include "kernels.h"

namespace qmoe {

namespace {

constexpr int DC_PAIRS = 8;
constexpr int DC_CW = 2 * DC_PAIRS;           // consumer warps
constexpr int DC_CT = DC_CW * 32;             // consumer threads
constexpr int DC_THREADS = DC_CT + 64;        // + static and routed producer warps
constexpr int DC_NS_STATIC = 3;
constexpr int DC_MAX_ROUTED = 16;
constexpr int DC_GU_ROWS = 4;                 // gate (and up) rows per GU item
constexpr int DC_DN_ROWS = 32;                // down rows per DN item
constexpr int DC_R_ROWS = 8;                  // router rows per R item
constexpr int BAR_ALL = 1;                    // named barrier of all consumer threads
constexpr int BAR_PAIR0 = 2;                  // named barriers 2..9: one per pair

// control words of the workspace
enum { C_LCOUNT = 0, C_DONE, C_EXIT, C_ABORT, C_READY };

// ------------------------------------------------------- packed layout --
// One packed layer (all byte counts are multiples of 16):
//   R blocks   (E/8 row blocks x 2 halves of K), each
//              codes [8 rows][H/2 bytes] (8-bit half rows, 16-byte chunk c of
//              row r stored at c ^ 4(r & 1)) + (scale, bias) half2 [8][GH/2]
//   then for each expert e = 0..E (e == E: the shared expert)
//   GU blocks  (I/4 of them), each codes [8 rows][H/2 bytes] (rows 0..3 gate
//              rows 4o..4o+3, rows 4..7 the same up rows; chunk c of row r at
//              c ^ 2(r & 3)) + (scale, bias) half2 [8][GH]
//   DN blocks  (H/32 of them), each codes [32 rows][I/2 bytes] (row-major) +
//              (scale, bias) half2 [32][GI]
struct PackDims {
    int E, H, I, GH, GI;
    size_t r_bytes, r_codes, gu_bytes, gu_codes, dn_bytes, dn_codes, exp_bytes, nR, total;
};

__host__ __device__ inline PackDims pack_dims(int E, int H, int I)
{
    PackDims p;
    p.E = E;
    p.H = H;
    p.I = I;
    p.GH = H / kGroup;
    p.GI = I / kGroup;
    p.r_codes = (size_t)DC_R_ROWS * (H / 2);
    p.r_bytes = p.r_codes + (size_t)DC_R_ROWS * (p.GH / 2) * 4;
    p.gu_codes = (size_t)2 * DC_GU_ROWS * (H / 2);
    p.gu_bytes = p.gu_codes + (size_t)2 * DC_GU_ROWS * p.GH * 4;
    p.dn_codes = (size_t)DC_DN_ROWS * (I / 2);
    p.dn_bytes = p.dn_codes + (size_t)DC_DN_ROWS * p.GI * 4;
    p.exp_bytes = (size_t)(I / DC_GU_ROWS) * p.gu_bytes + (size_t)(H / DC_DN_ROWS) * p.dn_bytes;
    p.nR = (size_t)(E / DC_R_ROWS) * 2;
    p.total = p.nR * p.r_bytes + (size_t)(E + 1) * p.exp_bytes;
    return p;
}

__host__ __device__ inline size_t pack_r_off(const PackDims &p, int item)
{
    return (size_t)item * p.r_bytes;
}
__host__ __device__ inline size_t pack_gu_off(const PackDims &p, int e, int oct)
{
    return p.nR * p.r_bytes + (size_t)e * p.exp_bytes + (size_t)oct * p.gu_bytes;
}
__host__ __device__ inline size_t pack_dn_off(const PackDims &p, int e, int tile)
{
    return p.nR * p.r_bytes + (size_t)e * p.exp_bytes + (size_t)(p.I / DC_GU_ROWS) * p.gu_bytes +
           (size_t)tile * p.dn_bytes;
}

struct DcLayout {
    int GH, GI, nslot;
    size_t stage;
    size_t xs4_off, xs8_off, xsum_off, xraw_off, xch_off, pfrag_off, phsum_off, topk_off, bar_off,
        ring_off, total;
    int NS_r;
};

__host__ __device__ inline DcLayout dc_layout(int E, int H, int I, int top_k, int NS_r)
{
    DcLayout L;
    const PackDims p = pack_dims(E, H, I);
    L.GH = p.GH;
    L.GI = p.GI;
    L.nslot = top_k + 1;
    size_t st = p.r_bytes > p.gu_bytes ? p.r_bytes : p.gu_bytes;
    st = st > p.dn_bytes ? st : p.dn_bytes;
    L.stage = (st + 127) & ~(size_t)127;
    size_t off = 0;
    L.xs4_off = off;
    off += (size_t)L.GH * 2 * 4 * 16;
    L.xs8_off = off;
    off += (size_t)L.GH * 2 * 4 * 16;
    L.xsum_off = off;
    off += (size_t)L.GH * 8 * 4;
    L.xraw_off = off;
    off += ((size_t)H * 2 + 15) & ~(size_t)15;
    L.xch_off = off;
    off += (size_t)DC_PAIRS * 2 * 32 * 4;
    L.pfrag_off = off;   // per pair: h fragments of one slot
    off += (size_t)DC_PAIRS * L.GI * 2 * 2 * 4 * 16;
    L.phsum_off = off;   // per pair: their group sums
    off += (size_t)DC_PAIRS * L.GI * 2 * 4;
    L.topk_off = off;   // idx[32], wt[32], queue words[16]
    off += 32 * 4 + 32 * 4 + 16 * 4;
    L.bar_off = off;
    off += (2 * (DC_NS_STATIC + DC_MAX_ROUTED) + 2) * 8;
    off = (off + 127) & ~(size_t)127;
    L.ring_off = off;
    L.NS_r = NS_r;
    off += (size_t)(DC_NS_STATIC + NS_r) * L.stage;
    L.total = off;
    return L;
}

// ------------------------------------------------------------ item lists --
// Items of each phase are dealt round-robin to the CTAs, starting at a CTA
// that rotates from phase to phase so the remainders spread evenly.
struct PhaseCounts {
    int nR, nGUs, nGUr, nDNs, nDNr, per_layer;
};

__device__ inline PhaseCounts phase_counts(const DecodeArgs &a)
{
    PhaseCounts c;
    c.nR = (a.E / DC_R_ROWS) * 2;
    c.nGUs = a.I / DC_GU_ROWS;
    c.nGUr = a.top_k * c.nGUs;
    c.nDNs = a.H / DC_DN_ROWS;
    c.nDNr = a.top_k * c.nDNs;
    c.per_layer = c.nR + c.nGUs + c.nGUr + c.nDNs + c.nDNr;
    return c;
}

// first item index of this CTA within a phase whose dealing starts at CTA `rot`
__device__ __forceinline__ int first_item(int rot, int G)
{
    int f = (int)blockIdx.x - rot;
    f %= G;
    return f < 0 ? f + G : f;
}

// ------------------------------------------------------------- counters --
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded spin until *p >= target.  False on timeout or abort.
__device__ __forceinline__ bool spin_until(const DecodeArgs &a, const unsigned *p, unsigned target)
{
    if (ld_acquire_u32(p) >= target)
        return true;
    unsigned *abort = a.ws.ctl + C_ABORT;
    const unsigned long long t0 = global_timer_ns();
    unsigned polls = 0;
    while (ld_acquire_u32(p) < target) {
        __nanosleep(64);   // keep the polled line from drowning the arrivals
        if ((++polls & 63u) == 0u) {
            if (ld_acquire_u32(abort) != 0u)
                return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicExch(abort, 1u);
                flag_status(a.status, QMOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
    return true;
}

// -------------------------------------------------------------- compute --
// One 64-input group of a 16-row 4-bit tile: returns 2^-20 * (sum q x) per C
// element, in the subnormal encoding (class-0 k-blocks into c, class-1 into
// d, recombined as 16c + d).
__device__ __forceinline__ void mma_group4s(float (&r)[4], uint2 wa, uint2 wb, uint4 x0, uint4 x1)
{
    uint32_t pa[8], pb[8];
    dequant4s_word(wa.x, pa);
    dequant4s_word(wa.y, pa + 4);
    dequant4s_word(wb.x, pb);
    dequant4s_word(wb.y, pb + 4);
    float c[4] = {0.f, 0.f, 0.f, 0.f}, d[4] = {0.f, 0.f, 0.f, 0.f};
    mma_16816(c, pa[0], pb[0], pa[2], pb[2], x0.x, x0.y);
    mma_16816(d, pa[1], pb[1], pa[3], pb[3], x1.x, x1.y);
    mma_16816(c, pa[4], pb[4], pa[6], pb[6], x0.z, x0.w);
    mma_16816(d, pa[5], pb[5], pa[7], pb[7], x1.z, x1.w);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        r[i] = fmaf(16.f, c[i], d[i]);
}

// 8-bit: returns 2^-24 * (sum q x).
__device__ __forceinline__ void mma_group8s(float (&c)[4], uint4 wa, uint4 wb, uint4 x0, uint4 x1)
{
    uint32_t pa[8], pb[8];
    dequant8s_word(wa.x, pa);
    dequant8s_word(wb.x, pb);
    dequant8s_word(wa.y, pa + 2);
    dequant8s_word(wb.y, pb + 2);
    dequant8s_word(wa.z, pa + 4);
    dequant8s_word(wb.z, pb + 4);
    dequant8s_word(wa.w, pa + 6);
    dequant8s_word(wb.w, pb + 6);
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    mma_16816(c, pa[0], pb[0], pa[1], pb[1], x0.x, x0.y);
    mma_16816(d, pa[2], pb[2], pa[3], pb[3], x0.z, x0.w);
    mma_16816(c, pa[4], pb[4], pa[5], pb[5], x1.x, x1.y);
    mma_16816(d, pa[6], pb[6], pa[7], pb[7], x1.z, x1.w);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] += d[i];
}

// sum over the 4 lanes of a quad (same gid)
__device__ __forceinline__ float quad_sum(float v)
{
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
}

__device__ __forceinline__ float2 sb_at(const uint32_t *sb, int i)
{
    return __half22float2(u32_as_h2(sb[i]));   // (scale, bias)
}

// R item (packed), steps [j0, j1) of Q = GH/4: 8 router rows over one half
// of K.  The partial logit of row gid is valid in lanes with tig == 0.
__device__ __forceinline__ float r_item(const unsigned char *stage, const PackDims &P,
                                        const uint4 *xs8, const float *xsum, int kh, int j0,
                                        int j1, bool with_bias, int gid, int tig)
{
    const uint32_t *row = reinterpret_cast<const uint32_t *>(stage) + gid * (P.H / 8);
    const int Gh = P.GH / 2, Q = P.GH / 4, g0 = kh * Gh;
    const uint32_t *sb = reinterpret_cast<const uint32_t *>(stage + P.r_codes) + gid * Gh;
    const int sw = 4 * (gid & 1);
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 2
    for (int j = j0; j < j1; ++j) {
        const uint4 wa = *reinterpret_cast<const uint4 *>(row + 4 * ((4 * j + tig) ^ sw));
        const uint4 wb = *reinterpret_cast<const uint4 *>(row + 4 * ((4 * (j + Q) + tig) ^ sw));
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
        if (gid < 2) {
            const int g = g0 + j + gid * Q;
            x0 = xs8[(g * 2 + 0) * 4 + tig];
            x1 = xs8[(g * 2 + 1) * 4 + tig];
        }
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        mma_group8s(c, wa, wb, x0, x1);
        acc0 = fmaf(sb_at(sb, j).x, c[0], acc0);
        acc1 = fmaf(sb_at(sb, j + Q).x, c[3], acc1);
    }
    float bias = 0.f;
    if (with_bias)
        for (int jj = tig; jj < Gh; jj += 4)
            bias = fmaf(sb_at(sb, jj).y, xsum[(g0 + jj) * 8], bias);
    return (acc0 + acc1) * kSub24 + quad_sum(bias);
}

// GU item (packed), steps [j0, j1) of GH/2: smem rows 0..3 gate, 4..7 up, over
// the two halves of K.  Result of smem row gid in lanes with tig == 0.
__device__ __forceinline__ float gu_item(const unsigned char *stage, const PackDims &P,
                                         const uint4 *xs4, const float *xsum, int j0, int j1,
                                         bool with_bias, int gid, int tig)
{
    const uint32_t *row = reinterpret_cast<const uint32_t *>(stage) + gid * (P.H / 8);
    const uint32_t *sb = reinterpret_cast<const uint32_t *>(stage + P.gu_codes) + gid * P.GH;
    const int half = P.GH / 2;
    const int sw = 2 * (gid & 3), t1 = tig >> 1, t0 = 2 * (tig & 1);
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 2
    for (int j = j0; j < j1; ++j) {
        const uint2 wa = *reinterpret_cast<const uint2 *>(row + 4 * ((2 * j + t1) ^ sw) + t0);
        const uint2 wb = *reinterpret_cast<const uint2 *>(row + 4 * ((2 * (j + half) + t1) ^ sw) + t0);
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
        if (gid < 2) {
            const int g = j + gid * half;
            x0 = xs4[(g * 2 + 0) * 4 + tig];
            x1 = xs4[(g * 2 + 1) * 4 + tig];
        }
        float c[4];
        mma_group4s(c, wa, wb, x0, x1);
        acc0 = fmaf(sb_at(sb, j).x, c[0], acc0);
        acc1 = fmaf(sb_at(sb, j + half).x, c[3], acc1);
    }
    float bias = 0.f;
    if (with_bias)
        for (int g = tig; g < P.GH; g += 4)
            bias = fmaf(sb_at(sb, g).y, xsum[g * 8], bias);
    return (acc0 + acc1) * kSub20 + quad_sum(bias);
}

// DN item (packed), 16-row tile mt of the 32: h (hi, lo) as batch columns 0 and
// 1.  Rows mt*16 + gid and mt*16 + gid + 8 in lanes tig == 0.
__device__ __forceinline__ void dn_tile(const unsigned char *stage, const PackDims &P,
                                        const uint4 *frag, const float *hs, int mt, int gid,
                                        int tig, float &r_lo, float &r_hi)
{
    const int Iw = P.I / 8;
    const int rl = mt * 16 + gid;
    const uint32_t *row = reinterpret_cast<const uint32_t *>(stage) + rl * Iw + 2 * tig;
    const uint32_t *sbl = reinterpret_cast<const uint32_t *>(stage + P.dn_codes) + rl * P.GI;
    const uint32_t *sbh = sbl + 8 * P.GI;
    float acc_l = 0.f, acc_h = 0.f;
#pragma unroll 2
    for (int g = 0; g < P.GI; ++g) {
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
        if (gid < 2) {
            x0 = frag[((g * 2 + 0) * 2 + gid) * 4 + tig];
            x1 = frag[((g * 2 + 1) * 2 + gid) * 4 + tig];
        }
        const uint2 wa = *reinterpret_cast<const uint2 *>(row + g * 8);
        const uint2 wb = *reinterpret_cast<const uint2 *>(row + 8 * Iw + g * 8);
        float c[4];
        mma_group4s(c, wa, wb, x0, x1);
        acc_l = fmaf(sb_at(sbl, g).x, c[0] + c[1], acc_l);
        acc_h = fmaf(sb_at(sbh, g).x, c[2] + c[3], acc_h);
    }
    float bl = 0.f, bh = 0.f;
    for (int g = tig; g < P.GI; g += 4) {
        const float X = hs[g * 2] + hs[g * 2 + 1];
        bl = fmaf(sb_at(sbl, g).y, X, bl);
        bh = fmaf(sb_at(sbh, g).y, X, bh);
    }
    r_lo = acc_l * kSub20 + quad_sum(bl);
    r_hi = acc_h * kSub20 + quad_sum(bh);
}

// position of intermediate index k in the down projection's B fragments
// (slot-relative, in halves): [g][hh][col][tig][8], order of xperm_s4
__device__ __forceinline__ int hfrag_half_index(int k, int col)
{
    const int g = k >> 6, kk = k & 63, tig = kk >> 4, p = kk & 15;
    const int i = ((p & 1) << 3) | ((p & 8) >> 1) | (p & 2) | ((p & 4) >> 2);   // inverse of xperm_s4
    const int hh = i >> 3, e = i & 7;
    return ((((g * 2 + hh) * 2 + col) * 4 + tig) * 8) + e;
}

// ------------------------------------------------------------ producers --
struct Ring {
    unsigned char *base;
    uint64_t *full, *empty;
    int ns;
    int seq;
};

__device__ __forceinline__ unsigned char *ring_acquire(Ring &r, const DecodeArgs &a,
                                                       const DcLayout &L, uint64_t **bar, bool *ok)
{
    const int st = r.seq % r.ns, use = r.seq / r.ns;
    if (use > 0 && !mbar_wait(&r.empty[st], (use - 1) & 1, a.status))
        *ok = false;
    *bar = &r.full[st];
    ++r.seq;
    return r.base + (size_t)st * L.stage;
}

__device__ __forceinline__ void ring_drain(Ring &r, const DecodeArgs &a)
{
    for (int s = 0; s < r.ns && s < r.seq; ++s) {
        const int last = r.seq - 1 - ((r.seq - 1 - s) % r.ns);   // last seq that used stage s
        mbar_wait(&r.full[s], (last / r.ns) & 1, a.status);
    }
}

__device__ __forceinline__ void issue_block(const unsigned char *src, uint32_t bytes,
                                            unsigned char *stage, uint64_t *bar, uint64_t pol)
{
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s(stage, src, bytes, bar, pol);
}

__device__ __forceinline__ int clamp_expert(int e, int E) { return (e >= 0 && e < E) ? e : 0; }

// ------------------------------------------------------------------ kernel --
__global__ void __launch_bounds__(DC_THREADS, 1) moe_decode_kernel(const __grid_constant__ DecodeArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const DcLayout L = dc_layout(a.E, a.H, a.I, a.top_k, a.NS_r);
    const PackDims P = pack_dims(a.E, a.H, a.I);
    uint4 *xs4 = reinterpret_cast<uint4 *>(smem + L.xs4_off);
    uint4 *xs8 = reinterpret_cast<uint4 *>(smem + L.xs8_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    uint4 *xraw = reinterpret_cast<uint4 *>(smem + L.xraw_off);
    float *xch = reinterpret_cast<float *>(smem + L.xch_off);
    uint4 *pfrag = reinterpret_cast<uint4 *>(smem + L.pfrag_off);
    float *phsum = reinterpret_cast<float *>(smem + L.phsum_off);
    int *s_idx = reinterpret_cast<int *>(smem + L.topk_off);
    float *s_wt = reinterpret_cast<float *>(smem + L.topk_off + 32 * 4);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    Ring rs, rr;
    rs.base = smem + L.ring_off;
    rs.full = bars;
    rs.empty = bars + DC_NS_STATIC;
    rs.ns = DC_NS_STATIC;
    rs.seq = 0;
    rr.base = rs.base + (size_t)DC_NS_STATIC * L.stage;
    rr.full = bars + 2 * DC_NS_STATIC;
    rr.empty = rr.full + DC_MAX_ROUTED;
    rr.ns = L.NS_r;
    rr.seq = 0;
    uint64_t *topk_bar = bars + 2 * (DC_NS_STATIC + DC_MAX_ROUTED);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const PhaseCounts pc = phase_counts(a);
    unsigned *ctl = a.ws.ctl;

    if (threadIdx.x == 0) {
        for (int s = 0; s < DC_NS_STATIC; ++s) {
            mbar_init(&rs.full[s], 1);
            mbar_init(&rs.empty[s], 2);   // both warps of the consuming pair
        }
        for (int s = 0; s < L.NS_r; ++s) {
            mbar_init(&rr.full[s], 1);
            mbar_init(&rr.empty[s], 2);
        }
        mbar_init(topk_bar, 1);
        mbar_init_fence();
    }
    __syncthreads();
    // the workspace counters may still be in use by the previous launch on
    // this stream until it has completed
    pdl_wait();

    if (warp == DC_CW) {
        // ------------------------------------------------ static producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            bool ok = true;
            for (int l = 0; l < a.L && ok; ++l) {
                const unsigned char *lp = static_cast<const unsigned char *>(a.layer[l]);
                const int base = l * pc.per_layer;
                for (int i = first_item(base % G, G); i < pc.nR && ok; i += G) {
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rs, a, L, &bar, &ok);
                    if (ok)
                        issue_block(lp + pack_r_off(P, i), (uint32_t)P.r_bytes, st, bar, pol);
                }
                const int rot_gus = (base + pc.nR) % G;
                for (int i = first_item(rot_gus, G); i < pc.nGUs && ok; i += G) {
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rs, a, L, &bar, &ok);
                    if (ok)
                        issue_block(lp + pack_gu_off(P, a.E, i), (uint32_t)P.gu_bytes, st, bar, pol);
                }
                const int rot_dns = (base + pc.nR + pc.nGUs + pc.nGUr) % G;
                for (int i = first_item(rot_dns, G); i < pc.nDNs && ok; i += G) {
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rs, a, L, &bar, &ok);
                    if (ok)
                        issue_block(lp + pack_dn_off(P, a.E, i), (uint32_t)P.dn_bytes, st, bar, pol);
                }
            }
            ring_drain(rs, a);
        }
        return;
    }
    if (warp == DC_CW + 1) {
        // ------------------------------------------------ routed producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            bool ok = true;
            for (int l = 0; l < a.L && ok; ++l) {
                const unsigned char *lp = static_cast<const unsigned char *>(a.layer[l]);
                const int base = l * pc.per_layer;
                if (!mbar_wait(topk_bar, l & 1, a.status))
                    break;
                const int rot_gur = (base + pc.nR + pc.nGUs) % G;
                for (int i = first_item(rot_gur, G); i < pc.nGUr && ok; i += G) {
                    const int j = i / pc.nGUs, oct = i % pc.nGUs;
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rr, a, L, &bar, &ok);
                    if (ok)
                        issue_block(lp + pack_gu_off(P, clamp_expert(s_idx[j], a.E), oct),
                                    (uint32_t)P.gu_bytes, st, bar, pol);
                }
                const int rot_dnr = (base + pc.nR + pc.nGUs + pc.nGUr + pc.nDNs) % G;
                for (int i = first_item(rot_dnr, G); i < pc.nDNr && ok; i += G) {
                    const int j = i / pc.nDNs, tile = i % pc.nDNs;
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rr, a, L, &bar, &ok);
                    if (ok)
                        issue_block(lp + pack_dn_off(P, clamp_expert(s_idx[j], a.E), tile),
                                    (uint32_t)P.dn_bytes, st, bar, pol);
                }
            }
            ring_drain(rr, a);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int ctid = threadIdx.x;
    const int pair = warp >> 1, hw = warp & 1;     // pair index, half of the pair
    const int ptid = hw * 32 + lane;                // thread index within the pair
    const int gid = lane >> 2, tig = lane & 3;
    const int H = a.H, E = a.E, K = a.top_k;
    float *my_xch = xch + pair * 2 * 32;
    uint4 *my_frag = pfrag + (size_t)pair * L.GI * 2 * 2 * 4;
    float *my_hsum = phsum + pair * L.GI * 2;
    int *s_q = reinterpret_cast<int *>(smem + L.topk_off + 64 * 4);   // [0] counter, [1+p] hand-off
    bool failed = false;
    int xb = 0;   // exchange-buffer parity of this pair

    auto pair_sync = [&]() { named_bar_sync(BAR_PAIR0 + pair, 64); };
    // the next item index of the running phase, the same in both warps of the pair
    auto grab = [&]() -> int {
        if (ptid == 0)
            s_q[1 + pair] = atomicAdd(s_q, 1);
        pair_sync();
        const int k = s_q[1 + pair];
        pair_sync();
        return k;
    };
    auto wait_full = [&](Ring &R, int seq) -> int {
        const int st = seq % R.ns;
        if (!failed && !mbar_wait(&R.full[st], (seq / R.ns) & 1, a.status))
            failed = true;
        return st;
    };
    auto release = [&](Ring &R, int st) {
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&R.empty[st]);
    };
    // warp 1 hands its partial to warp 0
    auto exchange = [&](float v) -> float {
        if (hw == 1)
            my_xch[xb * 32 + lane] = v;
        pair_sync();
        const float t = hw == 0 ? v + my_xch[xb * 32 + lane] : 0.f;
        xb ^= 1;
        return t;
    };
    auto publish_ready = [&](unsigned *cnt) {   // after this warp's global writes
        __threadfence();
        __syncwarp();
        if (lane == 0)
            atomicAdd(cnt, 1u);
    };

    auto do_r = [&](int item, int seq, int l) {
        const int st = wait_full(rs, seq);
        const int Q = L.GH / 4, hq = (Q + 1) / 2;
        float v = 0.f;
        if (!failed)
            v = r_item(rs.base + (size_t)st * L.stage, P, xs8, xsum, item & 1, hw * hq, hw ? Q : hq,
                       hw == 0, gid, tig);
        release(rs, st);
        v = exchange(v);
        if (hw == 0) {
            if (tig == 0)
                a.ws.logits_part[(item & 1) * E + (item >> 1) * DC_R_ROWS + gid] = v;
            publish_ready(ctl + C_LCOUNT);
        }
    };
    auto do_gu = [&](Ring &R, int seq, int slot, int oct) {
        const int st = wait_full(R, seq);
        const int half = L.GH / 2, hq = (half + 1) / 2;
        float v = 0.f;
        if (!failed)
            v = gu_item(R.base + (size_t)st * L.stage, P, xs4, xsum, hw * hq, hw ? half : hq, hw == 0,
                        gid, tig);
        release(R, st);
        v = exchange(v);
        if (hw == 0) {
            // rows 0..3 gate, 4..7 up (lane + 16)
            const float u = __shfl_down_sync(0xffffffffu, v, 16);
            if (gid < DC_GU_ROWS && tig == 0) {
                const float h = v / (1.f + expf(-v)) * u;
                const __half hh = __float2half_rn(h);
                const __half hl = __float2half_rn(h - __half2float(hh));
                __half *hf =
                    reinterpret_cast<__half *>(a.ws.hfrag) + (size_t)slot * L.GI * 2 * 2 * 4 * 8;
                const int kidx = oct * DC_GU_ROWS + gid;
                hf[hfrag_half_index(kidx, 0)] = hh;
                hf[hfrag_half_index(kidx, 1)] = hl;
            }
            publish_ready(ctl + C_READY + slot);
        }
    };
    auto do_dn = [&](Ring &R, int seq, int slot, int tile, int l) {
        const int st = wait_full(R, seq);
        // h of the slot must be complete (all its gate/up items, every CTA)
        if (ptid == 0 && !spin_until(a, ctl + C_READY + slot, (unsigned)((l + 1) * pc.nGUs)))
            failed = true;
        pair_sync();
        const int nf = L.GI * 2 * 2 * 4;
        const uint4 *src = a.ws.hfrag + (size_t)slot * nf;
        for (int t0 = 0; t0 < nf; t0 += 4 * 64) {   // 4 loads in flight per thread
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (t0 + ptid + u * 64 < nf)
                    v[u] = __ldcg(src + t0 + ptid + u * 64);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (t0 + ptid + u * 64 < nf)
                    my_frag[t0 + ptid + u * 64] = v[u];
        }
        pair_sync();
        for (int t = ptid; t < L.GI * 2; t += 64) {
            const int g = t >> 1, col = t & 1;
            float sum = 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int tg = 0; tg < 4; ++tg) {
                    const uint4 w = my_frag[((g * 2 + hh) * 2 + col) * 4 + tg];
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = __half22float2(u32_as_h2(ws[q]));
                        sum += f.x + f.y;
                    }
                }
            my_hsum[t] = sum;
        }
        pair_sync();
        float r_lo = 0.f, r_hi = 0.f;
        if (!failed)
            dn_tile(R.base + (size_t)st * L.stage, P, my_frag, my_hsum, hw, gid, tig, r_lo, r_hi);
        release(R, st);
        const int r0 = tile * DC_DN_ROWS + hw * 16;
        if (tig == 0) {
            float *p = a.ws.part + (size_t)slot * H + r0;
            p[gid] = r_lo;
            p[gid + 8] = r_hi;
        }
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0)
            old = atomicAdd(a.ws.counters + tile, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == 2 * (K + 1) - 1) {   // last of the 2 (K + 1) halves of this tile
            __threadfence();
            const int row = tile * DC_DN_ROWS + lane;
            float y = __ldcg(a.ws.part + (size_t)K * H + row);
            for (int jj = 0; jj < K; ++jj)
                y = fmaf(s_wt[jj], __ldcg(a.ws.part + (size_t)jj * H + row), y);
            a.y[(size_t)l * H + row] = __float2half_rn(y);
            if (lane == 0)
                a.ws.counters[tile] = 0;
            publish_ready(ctl + C_DONE);
        }
        pair_sync();   // both warps are done with the fragments before the pair reuses them
    };
    // items of this CTA in a phase list: the i-th has index first + i*G
    auto count = [&](int first, int n) { return first < n ? (n - first + G - 1) / G : 0; };

    for (int l = 0; l < a.L; ++l) {
        const int base = l * pc.per_layer;
        // --- this layer starts once the previous one has produced its output
        if (l > 0) {
            if (ctid == 0 && !spin_until(a, ctl + C_DONE, (unsigned)(l * pc.nDNs)))
                failed = true;
            named_bar_sync(BAR_ALL, DC_CT);
        }
        // --- x of this layer: one round of 16-byte loads, then both fragment orders
        {
            const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + (size_t)l * H);
            const int n = H / 8;
            for (int t = ctid; t < n; t += DC_CT)
                xraw[t] = xg[t];
            if (ctid == 0)
                s_q[0] = 0;
            named_bar_sync(BAR_ALL, DC_CT);
            const __half *xh = reinterpret_cast<const __half *>(xraw);
            stage_x<kPermS4>(xs4, xsum, L.GH, 1, 1,
                             [&](int, int, int k) { return __half2float(xh[k]); }, ctid, DC_CT);
            stage_x<8>(xs8, nullptr, L.GH, 1, 1,
                       [&](int, int, int k) { return __half2float(xh[k]); }, ctid, DC_CT);
            named_bar_sync(BAR_ALL, DC_CT);
        }

        // --- router items, then the shared expert's gate/up items (static
        //     ring), dealt dynamically to the pairs: the router items go first
        const int fR = first_item(base % G, G), nRc = count(fR, pc.nR);
        const int fGs = first_item((base + pc.nR) % G, G), nGs = count(fGs, pc.nGUs);
        {
            const int seq0 = rs.seq;
            for (int k = grab(); k < nRc + nGs; k = grab()) {
                if (k < nRc)
                    do_r(fR + k * G, seq0 + k, l);
                else
                    do_gu(rs, seq0 + k, K, fGs + (k - nRc) * G);
            }
            rs.seq = seq0 + nRc + nGs;
        }
        named_bar_sync(BAR_ALL, DC_CT);

        // --- top-k, in every CTA, once all router items are published
        if (warp == 0) {
            if (lane == 0 && !spin_until(a, ctl + C_LCOUNT, (unsigned)((l + 1) * pc.nR)))
                failed = true;
            __syncwarp();
            float v[4];
            unsigned key[4];
            bool taken[4];
            // all eight loads first (a store in between would order them)
            float p0[4], p1[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = lane + 32 * q;
                taken[q] = e >= E;
                p0[q] = taken[q] ? 0.f : __ldcg(a.ws.logits_part + e);
                p1[q] = taken[q] ? 0.f : __ldcg(a.ws.logits_part + E + e);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[q] = p0[q] + p1[q];
                const unsigned u = __float_as_uint(v[q]);   // order-preserving key
                key[q] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
            }
            if (a.logits && blockIdx.x == 0)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (!taken[q])
                        a.logits[(size_t)l * E + lane + 32 * q] = v[q];
            float my_v = 0.f;
            int my_i = 0;
            for (int j = 0; j < K; ++j) {
                unsigned bk = 0u;
                int be = 0x7fffffff;
                float bv = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (!taken[q] && key[q] > bk) {   // strict: the lower index wins ties
                        bk = key[q];
                        be = lane + 32 * q;
                        bv = v[q];
                    }
                const unsigned mk = __reduce_max_sync(0xffffffffu, bk);
                const int win = (int)__reduce_min_sync(0xffffffffu,
                                                       (unsigned)(bk == mk ? be : 0x7fffffff));
                const float wv = __shfl_sync(0xffffffffu, bv, win & 31);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (win == lane + 32 * q)
                        taken[q] = true;
                if (lane == j) {
                    my_v = wv;
                    my_i = win;
                }
            }
            const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
            const float ex = lane < K ? expf(my_v - vmax) : 0.f;
            float sum = ex;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                sum += __shfl_xor_sync(0xffffffffu, sum, off);
            if (lane < K) {
                s_idx[lane] = my_i;
                s_wt[lane] = ex / sum;
                if (blockIdx.x == 0) {
                    if (a.idx)
                        a.idx[(size_t)l * K + lane] = my_i;
                    if (a.weights)
                        a.weights[(size_t)l * K + lane] = ex / sum;
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(topk_bar);   // the routed producer may go
                s_q[0] = 0;
            }
        }
        named_bar_sync(BAR_ALL, DC_CT);

        // --- experts: routed gate/up (routed ring), shared down (static ring),
        //     routed down (routed ring), one dynamic list in that order
        {
            const int fGr = first_item((base + pc.nR + pc.nGUs) % G, G), nGr = count(fGr, pc.nGUr);
            const int fDs = first_item((base + pc.nR + pc.nGUs + pc.nGUr) % G, G),
                      nDs = count(fDs, pc.nDNs);
            const int fDr = first_item((base + pc.nR + pc.nGUs + pc.nGUr + pc.nDNs) % G, G),
                      nDr = count(fDr, pc.nDNr);
            const int s0 = rs.seq, r0 = rr.seq;
            const int total = nGr + nDs + nDr;
            for (int k = grab(); k < total; k = grab()) {
                int m = k;
                if (m < nGr) {
                    const int i = fGr + m * G;
                    do_gu(rr, r0 + m, i / pc.nGUs, i % pc.nGUs);
                    continue;
                }
                m -= nGr;
                if (m < nDs) {
                    do_dn(rs, s0 + m, K, fDs + m * G, l);
                    continue;
                }
                m -= nDs;
                const int i = fDr + m * G;
                do_dn(rr, r0 + nGr + m, i / pc.nDNs, i % pc.nDNs, l);
            }
            rs.seq = s0 + nDs;
            rr.seq = r0 + nGr + nDr;
        }
    }

    // the last CTA to finish resets the control words for the next launch;
    // every other CTA has stopped reading them by then
    named_bar_sync(BAR_ALL, DC_CT);
    if (ctid == 0) {
        __threadfence();
        const unsigned old = atomicAdd(ctl + C_EXIT, 1u);
        if (old == (unsigned)G - 1) {
            atomicExch(ctl + C_LCOUNT, 0u);
            atomicExch(ctl + C_DONE, 0u);
            atomicExch(ctl + C_ABORT, 0u);
            for (int s = 0; s < L.nslot; ++s)
                atomicExch(ctl + C_READY + s, 0u);
            atomicExch(ctl + C_EXIT, 0u);
        }
    }
}

// ------------------------------------------------------------- packing --
// One thread per 16-byte chunk of the packed layer; gathers from the
// row-major format.  (scale, bias) pairs are stored as half2 words.
__global__ void decode_pack_kernel(DecodePackArgs a, uint4 *dst)
{
    const PackDims P = pack_dims(a.E, a.H, a.I);
    const size_t n16 = P.total / 16;
    const size_t rb_bytes = (size_t)a.H / 2;   // bytes of an 8-bit half row / a 4-bit row
    for (size_t q = blockIdx.x * (size_t)blockDim.x + threadIdx.x; q < n16;
         q += (size_t)gridDim.x * blockDim.x) {
        const size_t off = q * 16;
        uint4 out;
        uint32_t sbw[4];
        bool codes = true;
        const unsigned char *src = nullptr;
        if (off < P.nR * P.r_bytes) {
            const int item = (int)(off / P.r_bytes);
            const size_t w = off % P.r_bytes;
            const int rb = item >> 1, kh = item & 1;
            if (w < P.r_codes) {
                const int r = (int)(w / rb_bytes);
                const int c = (int)((w % rb_bytes) / 16) ^ (4 * (r & 1));
                src = reinterpret_cast<const unsigned char *>(a.router.packed) +
                      (size_t)(rb * DC_R_ROWS + r) * a.H + (size_t)kh * rb_bytes + 16 * (size_t)c;
            } else {
                codes = false;
                const int Gh = P.GH / 2;
                for (int t = 0; t < 4; ++t) {
                    const int en = (int)((w - P.r_codes) / 4) + t;
                    const int r = en / Gh, jj = en % Gh;
                    const size_t i = (size_t)(rb * DC_R_ROWS + r) * P.GH + (size_t)kh * Gh + jj;
                    sbw[t] = h2_as_u32(__halves2half2(a.router.scales[i], a.router.biases[i]));
                }
            }
        } else {
            const size_t eoff = off - P.nR * P.r_bytes;
            const int e = (int)(eoff / P.exp_bytes);
            const size_t w = eoff % P.exp_bytes;
            const bool sh = e == a.E;
            const size_t gu_all = (size_t)(a.I / DC_GU_ROWS) * P.gu_bytes;
            if (w < gu_all) {
                const int oct = (int)(w / P.gu_bytes);
                const size_t ww = w % P.gu_bytes;
                if (ww < P.gu_codes) {
                    const int r = (int)(ww / rb_bytes);
                    const int c = (int)((ww % rb_bytes) / 16) ^ (2 * (r & 3));
                    const QMat &m = r < DC_GU_ROWS ? (sh ? a.sh_gate : a.gate) : (sh ? a.sh_up : a.up);
                    const size_t row = (size_t)(sh ? 0 : e) * a.I + (size_t)oct * DC_GU_ROWS + (r & 3);
                    src = reinterpret_cast<const unsigned char *>(m.packed) + row * rb_bytes + 16 * (size_t)c;
                } else {
                    codes = false;
                    for (int t = 0; t < 4; ++t) {
                        const int en = (int)((ww - P.gu_codes) / 4) + t;
                        const int r = en / P.GH, g = en % P.GH;
                        const QMat &m = r < DC_GU_ROWS ? (sh ? a.sh_gate : a.gate) : (sh ? a.sh_up : a.up);
                        const size_t row = (size_t)(sh ? 0 : e) * a.I + (size_t)oct * DC_GU_ROWS + (r & 3);
                        const size_t i = row * P.GH + g;
                        sbw[t] = h2_as_u32(__halves2half2(m.scales[i], m.biases[i]));
                    }
                }
            } else {
                const size_t w2 = w - gu_all;
                const int tile = (int)(w2 / P.dn_bytes);
                const size_t ww = w2 % P.dn_bytes;
                const QMat &m = sh ? a.sh_down : a.down;
                const size_t row0 = (size_t)(sh ? 0 : e) * a.H + (size_t)tile * DC_DN_ROWS;
                if (ww < P.dn_codes) {
                    src = reinterpret_cast<const unsigned char *>(m.packed) + row0 * (a.I / 2) + ww;
                } else {
                    codes = false;
                    for (int t = 0; t < 4; ++t) {
                        const int en = (int)((ww - P.dn_codes) / 4) + t;
                        const int r = en / P.GI, g = en % P.GI;
                        const size_t i = (row0 + r) * P.GI + g;
                        sbw[t] = h2_as_u32(__halves2half2(m.scales[i], m.biases[i]));
                    }
                }
            }
        }
        if (codes)
            out = *reinterpret_cast<const uint4 *>(src);
        else
            out = make_uint4(sbw[0], sbw[1], sbw[2], sbw[3]);
        dst[q] = out;
    }
}

}  // namespace

size_t decode_pack_bytes(int E, int H, int I) { return pack_dims(E, H, I).total; }

cudaError_t launch_decode_pack(const DecodePackArgs &a, void *dst, cudaStream_t s)
{
    decode_pack_kernel<<<1024, 256, 0, s>>>(a, static_cast<uint4 *>(dst));
    return cudaGetLastError();
}

size_t decode_workspace_layout(int E, int H, int I, int top_k, void *base, DecodeWorkspace *ws)
{
    const int nslot = top_k + 1;
    const int GI = I / kGroup;
    size_t off = 0;
    const size_t ctl_off = off;                    // control words
    off = align_up(off + (size_t)(C_READY + nslot) * 4, 256);
    const size_t cnt_off = off;
    off = align_up(off + (size_t)(H / DC_DN_ROWS) * 4, 256);
    const size_t lp_off = off;
    off = align_up(off + (size_t)2 * E * 4, 256);
    const size_t hf_off = off;
    off = align_up(off + (size_t)nslot * GI * 2 * 2 * 4 * 16, 256);
    const size_t part_off = off;
    off = align_up(off + (size_t)nslot * H * 4, 256);
    if (base && ws) {
        unsigned char *b = static_cast<unsigned char *>(base);
        ws->ctl = reinterpret_cast<unsigned *>(b + ctl_off);
        ws->counters = reinterpret_cast<int *>(b + cnt_off);
        ws->logits_part = reinterpret_cast<float *>(b + lp_off);
        ws->hfrag = reinterpret_cast<uint4 *>(b + hf_off);
        ws->part = reinterpret_cast<float *>(b + part_off);
    }
    return off;
}

cudaError_t launch_decode(const DecodeArgs &a0, const LaunchCfg &c)
{
    const DcLayout L0 = dc_layout(a0.E, a0.H, a0.I, a0.top_k, 0);
    const size_t budget = 227 * 1024;
    if (L0.total + 4 * L0.stage > budget)
        return cudaErrorInvalidValue;
    int NS_r = (int)((budget - L0.total) / L0.stage);
    NS_r = NS_r > DC_MAX_ROUTED ? DC_MAX_ROUTED : NS_r;
    DecodeArgs a = a0;
    a.NS_r = NS_r;
    const DcLayout L = dc_layout(a.E, a.H, a.I, a.top_k, NS_r);
    cudaError_t e = set_smem(moe_decode_kernel, L.total);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c.num_sms);
    cfg.blockDim = dim3(DC_THREADS);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = c.stream;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeCooperative;
    attrs[0].val.cooperative = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, moe_decode_kernel, a);
}

}  // namespace qmoe
