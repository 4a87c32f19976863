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
// Tiles are ~13 KB cp.async.bulk copies completing on mbarriers.  A pair of
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

// matrices of one layer, in DecodeLayerPtrs order
enum { M_ROUTER = 0, M_GATE, M_UP, M_DOWN, M_SHG, M_SHU, M_SHD };
// control words of the workspace
enum { C_LCOUNT = 0, C_DONE, C_EXIT, C_ABORT, C_READY };

struct DcLayout {
    int GH, GI, nslot;
    int S_r, S_gu, S_dn;      // smem row strides in words
    size_t stage;
    size_t xs4_off, xs8_off, xsum_off, xraw_off, xch_off, pfrag_off, phsum_off, topk_off, bar_off,
        ring_off, total;
    int NS_r;
};

__host__ __device__ inline DcLayout dc_layout(int H, int I, int top_k, int NS_r)
{
    DcLayout L;
    L.GH = H / kGroup;
    L.GI = I / kGroup;
    L.nslot = top_k + 1;
    // R: half rows of an 8-bit matrix = H/8 words; GU: 4-bit rows = H/8 words;
    // DN: 4-bit rows = I/8 words
    L.S_r = tile_stride_words(H / 2, 8);
    L.S_gu = tile_stride_words(H, 4);
    L.S_dn = tile_stride_words(I, 4);
    const size_t r_bytes = (size_t)DC_R_ROWS * L.S_r * 4 + 2 * (size_t)DC_R_ROWS * L.GH * 2;
    const size_t gu_bytes = (size_t)2 * DC_GU_ROWS * L.S_gu * 4 + 2 * (size_t)2 * DC_GU_ROWS * L.GH * 2;
    const size_t dn_bytes = (size_t)DC_DN_ROWS * L.S_dn * 4 + 2 * (size_t)DC_DN_ROWS * L.GI * 2;
    size_t st = r_bytes > gu_bytes ? r_bytes : gu_bytes;
    st = st > dn_bytes ? st : dn_bytes;
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
    L.topk_off = off;
    off += 32 * 4 + 32 * 4;
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

// Publish: everything this thread (and, through a preceding CTA/warp barrier,
// its peers) wrote before is visible to whoever sees the increment.
__device__ __forceinline__ void publish_add(unsigned *p)
{
    __threadfence();
    atomicAdd(p, 1u);
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
        if ((++polls & 255u) == 0u) {
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
// One 64-input group of a 16-row tile: c += A(codes) * B(x).  The four
// k-blocks go to two independent accumulators so the mma dependency chain is
// two deep instead of four.
__device__ __forceinline__ void mma_group4(float (&c)[4], uint2 wa, uint2 wb, uint4 x0, uint4 x1)
{
    uint32_t pa[8], pb[8];
    dequant4_word(wa.x, pa);
    dequant4_word(wa.y, pa + 4);
    dequant4_word(wb.x, pb);
    dequant4_word(wb.y, pb + 4);
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    mma_16816(c, pa[0], pb[0], pa[1], pb[1], x0.x, x0.y);
    mma_16816(d, pa[2], pb[2], pa[3], pb[3], x0.z, x0.w);
    mma_16816(c, pa[4], pb[4], pa[5], pb[5], x1.x, x1.y);
    mma_16816(d, pa[6], pb[6], pa[7], pb[7], x1.z, x1.w);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] += d[i];
}

__device__ __forceinline__ void mma_group8(float (&c)[4], uint4 wa, uint4 wb, uint4 x0, uint4 x1)
{
    uint32_t pa[8], pb[8];
    dequant8_word(wa.x, pa);
    dequant8_word(wb.x, pb);
    dequant8_word(wa.y, pa + 2);
    dequant8_word(wb.y, pb + 2);
    dequant8_word(wa.z, pa + 4);
    dequant8_word(wb.z, pb + 4);
    dequant8_word(wa.w, pa + 6);
    dequant8_word(wb.w, pb + 6);
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

// R item, steps [j0, j1) of Q = GH/4: router rows rb*8 .. rb*8+7 over groups
// [kh*GH/2, (kh+1)*GH/2).  `with_bias` adds the bias term of all the item's
// groups.  The partial logit of row gid is valid in lanes with tig == 0.
__device__ __forceinline__ float r_item(const unsigned char *stage, const DcLayout &L,
                                        const uint4 *xs8, const float *xsum, int kh, int j0,
                                        int j1, bool with_bias, int gid, int tig)
{
    const uint32_t *tile = reinterpret_cast<const uint32_t *>(stage);
    const __half *sc = reinterpret_cast<const __half *>(stage + (size_t)DC_R_ROWS * L.S_r * 4);
    const __half *bi = sc + DC_R_ROWS * L.GH;
    const int Q = L.GH / 4;            // groups per quarter of K
    const int g0 = kh * 2 * Q;         // first group of this half
    float acc0 = 0.f, acc1 = 0.f;
    const uint32_t *row = tile + gid * L.S_r;
#pragma unroll 2
    for (int j = j0; j < j1; ++j) {
        const uint4 wa = *reinterpret_cast<const uint4 *>(row + j * 16 + 4 * tig);
        const uint4 wb = *reinterpret_cast<const uint4 *>(row + (j + Q) * 16 + 4 * tig);
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
        if (gid < 2) {
            const int g = g0 + j + gid * Q;
            x0 = xs8[(g * 2 + 0) * 4 + tig];
            x1 = xs8[(g * 2 + 1) * 4 + tig];
        }
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        mma_group8(c, wa, wb, x0, x1);
        acc0 = fmaf(__half2float(sc[gid * L.GH + g0 + j]), c[0], acc0);
        acc1 = fmaf(__half2float(sc[gid * L.GH + g0 + Q + j]), c[3], acc1);
    }
    float bias = 0.f;
    if (with_bias)
        for (int g = g0 + tig; g < g0 + 2 * Q; g += 4)
            bias = fmaf(__half2float(bi[gid * L.GH + g]), xsum[g * 8], bias);
    return acc0 + acc1 + quad_sum(bias);
}

// GU item, steps [j0, j1) of GH/2: smem rows 0..3 gate rows r..r+3, rows 4..7
// up rows r..r+3, over the two halves of K.  Result of smem row gid in lanes
// with tig == 0.
__device__ __forceinline__ float gu_item(const unsigned char *stage, const DcLayout &L,
                                         const uint4 *xs4, const float *xsum, int j0, int j1,
                                         bool with_bias, int gid, int tig)
{
    const uint32_t *tile = reinterpret_cast<const uint32_t *>(stage);
    const __half *sc = reinterpret_cast<const __half *>(stage + (size_t)2 * DC_GU_ROWS * L.S_gu * 4);
    const __half *bi = sc + 2 * DC_GU_ROWS * L.GH;
    const int half = L.GH / 2;
    float acc0 = 0.f, acc1 = 0.f;
    const uint32_t *row = tile + gid * L.S_gu;
#pragma unroll 2
    for (int j = j0; j < j1; ++j) {
        const uint2 wa = *reinterpret_cast<const uint2 *>(row + j * 8 + 2 * tig);
        const uint2 wb = *reinterpret_cast<const uint2 *>(row + (j + half) * 8 + 2 * tig);
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
        if (gid < 2) {
            const int g = j + gid * half;
            x0 = xs4[(g * 2 + 0) * 4 + tig];
            x1 = xs4[(g * 2 + 1) * 4 + tig];
        }
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        mma_group4(c, wa, wb, x0, x1);
        acc0 = fmaf(__half2float(sc[gid * L.GH + j]), c[0], acc0);
        acc1 = fmaf(__half2float(sc[gid * L.GH + j + half]), c[3], acc1);
    }
    float bias = 0.f;
    if (with_bias)
        for (int g = tig; g < L.GH; g += 4)
            bias = fmaf(__half2float(bi[gid * L.GH + g]), xsum[g * 8], bias);
    return acc0 + acc1 + quad_sum(bias);
}

// DN item, one 16-row tile mt of the 32: full K of I; h of the slot as batch
// columns hi / lo.  Rows mt*16 + gid and mt*16 + gid + 8 in lanes tig == 0.
__device__ __forceinline__ void dn_tile(const unsigned char *stage, const DcLayout &L,
                                        const uint4 *frag, const float *hs, int mt, int gid,
                                        int tig, float &r_lo, float &r_hi)
{
    const uint32_t *tile = reinterpret_cast<const uint32_t *>(stage);
    const __half *sc = reinterpret_cast<const __half *>(stage + (size_t)DC_DN_ROWS * L.S_dn * 4);
    const __half *bi = sc + DC_DN_ROWS * L.GI;
    const int rl = mt * 16 + gid, rh = rl + 8;
    float acc_l = 0.f, acc_h = 0.f;
    const uint32_t *row = tile + rl * L.S_dn + 2 * tig;
#pragma unroll 2
    for (int g = 0; g < L.GI; ++g) {
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
        if (gid < 2) {
            x0 = frag[((g * 2 + 0) * 2 + gid) * 4 + tig];
            x1 = frag[((g * 2 + 1) * 2 + gid) * 4 + tig];
        }
        const uint2 wa = *reinterpret_cast<const uint2 *>(row + g * 8);
        const uint2 wb = *reinterpret_cast<const uint2 *>(row + 8 * L.S_dn + g * 8);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        mma_group4(c, wa, wb, x0, x1);
        acc_l = fmaf(__half2float(sc[rl * L.GI + g]), c[0] + c[1], acc_l);
        acc_h = fmaf(__half2float(sc[rh * L.GI + g]), c[2] + c[3], acc_h);
    }
    float bl = 0.f, bh = 0.f;
    for (int g = tig; g < L.GI; g += 4) {
        const float X = hs[g * 2] + hs[g * 2 + 1];
        bl = fmaf(__half2float(bi[rl * L.GI + g]), X, bl);
        bh = fmaf(__half2float(bi[rh * L.GI + g]), X, bh);
    }
    r_lo = acc_l + quad_sum(bl);
    r_hi = acc_h + quad_sum(bh);
}

// position of intermediate index k in the down projection's B fragments
// (slot-relative, in halves): [g][hh][col][tig][8]
__device__ __forceinline__ int hfrag_half_index(int k, int col)
{
    const int g = k >> 6, kk = k & 63, tig = kk >> 4, p = kk & 15;
    const int q = p & 7;
    const int i = (p & 8) + 2 * (q & 3) + (q >> 2);   // inverse of xperm(4, .)
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

__device__ void issue_r(const DecodeArgs &a, const DcLayout &L, const DecodeLayerPtrs &lp, int item,
                        unsigned char *stage, uint64_t *bar, uint64_t pol)
{
    const int rb = item >> 1, kh = item & 1;
    const uint32_t half_bytes = (uint32_t)a.H / 2;               // 8-bit half row
    const uint32_t sb = (uint32_t)(DC_R_ROWS * L.GH * 2);
    mbar_arrive_expect_tx(bar, DC_R_ROWS * half_bytes + 2 * sb);
    const unsigned char *P = reinterpret_cast<const unsigned char *>(lp.P[M_ROUTER]);
    for (int r = 0; r < DC_R_ROWS; ++r)
        bulk_g2s(stage + (size_t)r * L.S_r * 4,
                 P + (size_t)(rb * DC_R_ROWS + r) * a.H + (size_t)kh * half_bytes, half_bytes, bar, pol);
    unsigned char *sc = stage + (size_t)DC_R_ROWS * L.S_r * 4;
    bulk_g2s(sc, lp.S[M_ROUTER] + (size_t)rb * DC_R_ROWS * L.GH, sb, bar, pol);
    bulk_g2s(sc + sb, lp.B[M_ROUTER] + (size_t)rb * DC_R_ROWS * L.GH, sb, bar, pol);
}

// GU item `oct` (rows oct*4 .. +3) of expert e (e < 0: shared expert)
__device__ void issue_gu(const DecodeArgs &a, const DcLayout &L, const DecodeLayerPtrs &lp, int e,
                         int oct, unsigned char *stage, uint64_t *bar, uint64_t pol)
{
    const int mg = e < 0 ? M_SHG : M_GATE, mu = e < 0 ? M_SHU : M_UP;
    const size_t r0 = (size_t)(e < 0 ? 0 : e) * a.I + (size_t)oct * DC_GU_ROWS;
    const uint32_t row_bytes = (uint32_t)a.H / 2;
    const uint32_t sb = (uint32_t)(DC_GU_ROWS * L.GH * 2);
    mbar_arrive_expect_tx(bar, 2 * DC_GU_ROWS * row_bytes + 4 * sb);
    const unsigned char *Pg = reinterpret_cast<const unsigned char *>(lp.P[mg]);
    const unsigned char *Pu = reinterpret_cast<const unsigned char *>(lp.P[mu]);
    for (int r = 0; r < DC_GU_ROWS; ++r) {
        bulk_g2s(stage + (size_t)r * L.S_gu * 4, Pg + (r0 + r) * row_bytes, row_bytes, bar, pol);
        bulk_g2s(stage + (size_t)(r + DC_GU_ROWS) * L.S_gu * 4, Pu + (r0 + r) * row_bytes, row_bytes,
                 bar, pol);
    }
    unsigned char *sc = stage + (size_t)2 * DC_GU_ROWS * L.S_gu * 4;
    unsigned char *bi = sc + 2 * sb;
    bulk_g2s(sc, lp.S[mg] + r0 * L.GH, sb, bar, pol);
    bulk_g2s(sc + sb, lp.S[mu] + r0 * L.GH, sb, bar, pol);
    bulk_g2s(bi, lp.B[mg] + r0 * L.GH, sb, bar, pol);
    bulk_g2s(bi + sb, lp.B[mu] + r0 * L.GH, sb, bar, pol);
}

// DN item `tile` (rows tile*32 .. +31) of expert e (e < 0: shared expert)
__device__ void issue_dn(const DecodeArgs &a, const DcLayout &L, const DecodeLayerPtrs &lp, int e,
                         int tile, unsigned char *stage, uint64_t *bar, uint64_t pol)
{
    const int md = e < 0 ? M_SHD : M_DOWN;
    const size_t r0 = (size_t)(e < 0 ? 0 : e) * a.H + (size_t)tile * DC_DN_ROWS;
    const uint32_t row_bytes = (uint32_t)a.I / 2;
    const uint32_t sb = (uint32_t)(DC_DN_ROWS * L.GI * 2);
    mbar_arrive_expect_tx(bar, DC_DN_ROWS * row_bytes + 2 * sb);
    const unsigned char *P = reinterpret_cast<const unsigned char *>(lp.P[md]);
    if ((uint32_t)L.S_dn * 4 == row_bytes) {
        bulk_g2s(stage, P + r0 * row_bytes, DC_DN_ROWS * row_bytes, bar, pol);
    } else {
        for (int r = 0; r < DC_DN_ROWS; ++r)
            bulk_g2s(stage + (size_t)r * L.S_dn * 4, P + (r0 + r) * row_bytes, row_bytes, bar, pol);
    }
    unsigned char *sc = stage + (size_t)DC_DN_ROWS * L.S_dn * 4;
    bulk_g2s(sc, lp.S[md] + r0 * L.GI, sb, bar, pol);
    bulk_g2s(sc + sb, lp.B[md] + r0 * L.GI, sb, bar, pol);
}

__device__ __forceinline__ int clamp_expert(int e, int E) { return (e >= 0 && e < E) ? e : 0; }

// ------------------------------------------------------------------ kernel --
__global__ void __launch_bounds__(DC_THREADS, 1) moe_decode_kernel(const __grid_constant__ DecodeArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const DcLayout L = dc_layout(a.H, a.I, a.top_k, a.NS_r);
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
                const DecodeLayerPtrs &lp = a.layer[l];
                const int base = l * pc.per_layer;
                for (int i = first_item(base % G, G); i < pc.nR && ok; i += G) {
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rs, a, L, &bar, &ok);
                    if (ok)
                        issue_r(a, L, lp, i, st, bar, pol);
                }
                const int rot_gus = (base + pc.nR) % G;
                for (int i = first_item(rot_gus, G); i < pc.nGUs && ok; i += G) {
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rs, a, L, &bar, &ok);
                    if (ok)
                        issue_gu(a, L, lp, -1, i, st, bar, pol);
                }
                const int rot_dns = (base + pc.nR + pc.nGUs + pc.nGUr) % G;
                for (int i = first_item(rot_dns, G); i < pc.nDNs && ok; i += G) {
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rs, a, L, &bar, &ok);
                    if (ok)
                        issue_dn(a, L, lp, -1, i, st, bar, pol);
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
                const DecodeLayerPtrs &lp = a.layer[l];
                const int base = l * pc.per_layer;
                if (!mbar_wait(topk_bar, l & 1, a.status))
                    break;
                const int rot_gur = (base + pc.nR + pc.nGUs) % G;
                for (int i = first_item(rot_gur, G); i < pc.nGUr && ok; i += G) {
                    const int j = i / pc.nGUs, oct = i % pc.nGUs;
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rr, a, L, &bar, &ok);
                    if (ok)
                        issue_gu(a, L, lp, clamp_expert(s_idx[j], a.E), oct, st, bar, pol);
                }
                const int rot_dnr = (base + pc.nR + pc.nGUs + pc.nGUr + pc.nDNs) % G;
                for (int i = first_item(rot_dnr, G); i < pc.nDNr && ok; i += G) {
                    const int j = i / pc.nDNs, tile = i % pc.nDNs;
                    uint64_t *bar;
                    unsigned char *st = ring_acquire(rr, a, L, &bar, &ok);
                    if (ok)
                        issue_dn(a, L, lp, clamp_expert(s_idx[j], a.E), tile, st, bar, pol);
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
    bool failed = false;
    int kp = 0;   // running item counter, dealt round-robin to the pairs

    // the item goes to pair kp % 8; both of its warps wait for the tile
    auto take = [&](Ring &R, int &st) -> bool {
        st = R.seq % R.ns;
        const int use = R.seq / R.ns;
        ++R.seq;
        if ((kp++) % DC_PAIRS != pair)
            return false;
        if (!failed && !mbar_wait(&R.full[st], use & 1, a.status))
            failed = true;
        return true;
    };
    auto release = [&](Ring &R, int st) {
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&R.empty[st]);
    };
    auto pair_sync = [&]() { named_bar_sync(BAR_PAIR0 + pair, 64); };

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
            named_bar_sync(BAR_ALL, DC_CT);
            const __half *xh = reinterpret_cast<const __half *>(xraw);
            stage_x<4>(xs4, xsum, L.GH, 1, 1, [&](int, int, int k) { return __half2float(xh[k]); },
                       ctid, DC_CT);
            stage_x<8>(xs8, nullptr, L.GH, 1, 1,
                       [&](int, int, int k) { return __half2float(xh[k]); }, ctid, DC_CT);
            named_bar_sync(BAR_ALL, DC_CT);
        }

        // --- router items and the shared expert's gate/up items (static ring)
        for (int i = first_item(base % G, G); i < pc.nR; i += G) {
            int st;
            if (!take(rs, st))
                continue;
            const int Q = L.GH / 4, hq = (Q + 1) / 2;
            float v = 0.f;
            if (!failed)
                v = r_item(rs.base + (size_t)st * L.stage, L, xs8, xsum, i & 1, hw * hq,
                           hw ? Q : hq, hw == 0, gid, tig);
            release(rs, st);
            const int xb = (kp >> 3) & 1;
            if (hw == 1)
                my_xch[xb * 32 + lane] = v;
            pair_sync();
            if (hw == 0) {
                v += my_xch[xb * 32 + lane];
                if (tig == 0)
                    a.ws.logits_part[(i & 1) * E + (i >> 1) * DC_R_ROWS + gid] = v;
                __threadfence();
                __syncwarp();
                if (lane == 0)
                    publish_add(ctl + C_LCOUNT);
            }
        }
        auto gu_epilogue = [&](int slot, int oct, float v) {
            // warp 0 of the pair: rows 0..3 gate, 4..7 up (lane + 16)
            const float u = __shfl_down_sync(0xffffffffu, v, 16);
            if (gid < DC_GU_ROWS && tig == 0) {
                const float h = v / (1.f + expf(-v)) * u;
                const __half hh = __float2half_rn(h);
                const __half hl = __float2half_rn(h - __half2float(hh));
                __half *hf = reinterpret_cast<__half *>(a.ws.hfrag) + (size_t)slot * L.GI * 2 * 2 * 4 * 8;
                const int kidx = oct * DC_GU_ROWS + gid;
                hf[hfrag_half_index(kidx, 0)] = hh;
                hf[hfrag_half_index(kidx, 1)] = hl;
            }
            __threadfence();
            __syncwarp();
            if (lane == 0)
                publish_add(ctl + C_READY + slot);
        };
        auto do_gu = [&](Ring &R, int st, int slot, int oct) {
            const int half = L.GH / 2, hq = (half + 1) / 2;
            float v = 0.f;
            if (!failed)
                v = gu_item(R.base + (size_t)st * L.stage, L, xs4, xsum, hw * hq, hw ? half : hq,
                            hw == 0, gid, tig);
            release(R, st);
            const int xb = (kp >> 3) & 1;
            if (hw == 1)
                my_xch[xb * 32 + lane] = v;
            pair_sync();
            if (hw == 0)
                gu_epilogue(slot, oct, v + my_xch[xb * 32 + lane]);
        };
        {
            const int rot_gus = (base + pc.nR) % G;
            for (int i = first_item(rot_gus, G); i < pc.nGUs; i += G) {
                int st;
                if (take(rs, st))
                    do_gu(rs, st, K, i);
            }
        }

        // --- top-k, in every CTA, once all router items are published
        if (ctid == 0 && !spin_until(a, ctl + C_LCOUNT, (unsigned)((l + 1) * pc.nR)))
            failed = true;
        named_bar_sync(BAR_ALL, DC_CT);
        if (warp == 0) {
            float v[4];
            unsigned key[4];
            bool taken[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = lane + 32 * q;
                taken[q] = e >= E;
                v[q] = taken[q] ? 0.f
                                : __ldcg(a.ws.logits_part + e) + __ldcg(a.ws.logits_part + E + e);
                if (!taken[q] && a.logits && blockIdx.x == 0)
                    a.logits[(size_t)l * E + e] = v[q];
                const unsigned u = __float_as_uint(v[q]);   // order-preserving key
                key[q] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
            }
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
            if (lane == 0)
                mbar_arrive(topk_bar);   // the routed producer may go
        }
        named_bar_sync(BAR_ALL, DC_CT);

        // --- routed gate/up items (routed ring)
        {
            const int rot_gur = (base + pc.nR + pc.nGUs) % G;
            for (int i = first_item(rot_gur, G); i < pc.nGUr; i += G) {
                int st;
                if (take(rr, st))
                    do_gu(rr, st, i / pc.nGUs, i % pc.nGUs);
            }
        }

        // --- down items: shared (static ring), then routed; combine
        {
            const int rot_dns = (base + pc.nR + pc.nGUs + pc.nGUr) % G;
            const int rot_dnr = (base + pc.nR + pc.nGUs + pc.nGUr + pc.nDNs) % G;
            int is = first_item(rot_dns, G), ir = first_item(rot_dnr, G);
            while (is < pc.nDNs || ir < pc.nDNr) {
                const bool from_static = is < pc.nDNs;
                const int i = from_static ? is : ir;
                Ring &R = from_static ? rs : rr;
                if (from_static)
                    is += G;
                else
                    ir += G;
                int st;
                if (!take(R, st))
                    continue;
                const int slot = from_static ? K : i / pc.nDNs;
                const int tile = from_static ? i : i % pc.nDNs;
                // h of the slot must be complete (all its gate/up items)
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
                    dn_tile(R.base + (size_t)st * L.stage, L, my_frag, my_hsum, hw, gid, tig, r_lo,
                            r_hi);
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
                    __syncwarp();
                    if (lane == 0) {
                        a.ws.counters[tile] = 0;
                        publish_add(ctl + C_DONE);
                    }
                }
            }
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

}  // namespace

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
    const DcLayout L0 = dc_layout(a0.H, a0.I, a0.top_k, 0);
    const size_t budget = 227 * 1024;
    if (L0.total + 4 * L0.stage > budget)
        return cudaErrorInvalidValue;
    int NS_r = (int)((budget - L0.total) / L0.stage);
    NS_r = NS_r > DC_MAX_ROUTED ? DC_MAX_ROUTED : NS_r;
    DecodeArgs a = a0;
    a.NS_r = NS_r;
    const DcLayout L = dc_layout(a.H, a.I, a.top_k, NS_r);
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
