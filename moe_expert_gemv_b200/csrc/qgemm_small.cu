// qgemm_small.cu -- dense affine-quantized product for a batch of 9..32 rows
// of x in ONE pass over the weights: the small-M verification product of a
// speculative-decoding step (the uzu page, discuss.pytorch.kr, section "uzu의
// 추측 디코딩 구조": a draft model proposes 16-32 tokens and the main model
// checks them in one forward pass, so every projection multiplies 16-32
// rows of activations at once).  Format: MLX affine 4-bit (8-bit) group 64
// (TurboFieldfare article, jeff.news, section "성능과 제약").
//
//   y[b][n] = sum_g s[n][g] * (sum_{k in g} q[n][k] x[b][k]) + b[n][g] * X[b][g]
//
// B200 design.  x of 32 tokens x 4096 inputs is 256 KB of fp16, more than a
// CTA's shared memory next to a weight ring, so the K range is split into S
// slices (S = 1, 2, 4, 8: the smallest whose x slice fits 64 KB).  CTA c
// always works on slice c % S: it stages only that part of x, once, and
// streams TM-row x K/S weight tiles (codes by one 3-D swizzled tensor copy of
// ~32 KB, scales and biases by two 2-D tensor copies) through a ring of
// shared-memory stages fed by a producer warp.  Sixteen consumer warps take
// (16-row m-tile, block of groups) pairs; each dequantises a group's codes
// ONCE into mma fragments (the code bits as exact fp16 subnormals) and runs
// them against every 8-column n-tile of the batch, so the weights cost the
// same instructions at batch 32 as at batch 8.  The warps of an m-tile are
// reduced through shared memory; with S > 1 each CTA writes its fp32 partial
// tile to a workspace and the CTA that finishes a tile last (a per-tile
// arrival counter) adds the S partials in slice order and writes y, so the
// result does not depend on which CTA arrives last.  No CTA ever waits for
// another one.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace qmoe {
namespace {

constexpr int SM_CW = 16;                  // consumer warps
constexpr int SM_CT = SM_CW * 32;
constexpr int SM_THREADS = SM_CT + 32;     // + one producer warp
constexpr int SM_MAX_STAGES = 6;
constexpr int SM_MAX_NT = 4;               // 8-column n-tiles: batch <= 32
constexpr size_t SM_X_BUDGET = 64 * 1024;  // shared memory for the x slice
// Workspace: arrival counters in a fixed region at its start, the partial
// tiles after it.  Every call returns its counters to zero and writes
// partials only past the region, so calls of any shape can share one
// workspace (zero-filled once).
constexpr size_t SM_CTR_BYTES = 64 * 1024;
constexpr int SM_MAX_TILES = (int)(SM_CTR_BYTES / 4);
constexpr int SM_MAX_CTA_TILES = 1024;     // tiles one CTA may take (flags in shared memory)

struct SmArgs {
    const __half *x;
    const uint32_t *signs;   // rotation signs [K / 32] (formats with the rotation)
    __half *y;
    unsigned *ctr;      // [tiles] arrival counters, zero between calls
    float4 *part;       // [tiles][S][MT * NT * 32] partial tiles (S > 1)
    int32_t *status;
    int N, K, B, S, KS, TM;
};

struct SmLayout {
    int GS;
    size_t xs_off, xslo_off, xsum_off, red_off, last_off, bar_off, stage_off;
    size_t codes_bytes, sb_bytes, stage_bytes, total;
};

__host__ __device__ inline SmLayout sm_layout(int KS, int bits, int B, int TM, int NS,
                                              bool rot = false)
{
    SmLayout L;
    L.GS = KS / kGroup;
    size_t off = 0;
    L.xs_off = off;   // x fragments: uint4 per (group, half, column, quad lane)
    off += (size_t)L.GS * 2 * B * 4 * 16;
    L.xslo_off = off;   // the lo parts of a rotated x, same layout
    if (rot)
        off += (size_t)L.GS * 2 * B * 4 * 16;
    L.xsum_off = off;   // group sums: [GS][32]
    off += (size_t)L.GS * 32 * 4;
    L.red_off = off;   // one float4 per (warp, n-tile, lane)
    off += (size_t)SM_CW * SM_MAX_NT * 32 * 16;
    L.last_off = off;   // per tile of this CTA: it arrived last
    off += (size_t)SM_MAX_CTA_TILES * 4;
    L.bar_off = off;
    off += 2 * SM_MAX_STAGES * 8;
    off = (off + 1023) & ~(size_t)1023;
    L.stage_off = off;
    L.codes_bytes = (size_t)TM * KS * bits / 8;
    L.sb_bytes = (size_t)TM * L.GS * 2;
    L.stage_bytes = (L.codes_bytes + 2 * L.sb_bytes + 1023) & ~(size_t)1023;
    off += (size_t)NS * L.stage_bytes;
    L.total = off + 1024;   // slack to align the dynamic window to 1024 bytes
    return L;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int c0, int c1,
                                            uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// (XOR80: two's-complement bytes q -> q + 128 = byte ^ 0x80, the symmetric
// 8-bit format)
template <int BITS, bool XOR80 = false>
__device__ __forceinline__ void dequant_frags(const void *fa, const void *fb, uint32_t (&pa)[8],
                                              uint32_t (&pb)[8])
{
    if (BITS == 4) {
        const uint2 wa = *reinterpret_cast<const uint2 *>(fa);
        const uint2 wb = *reinterpret_cast<const uint2 *>(fb);
        dequant4s_word(wa.x, pa);
        dequant4s_word(wa.y, pa + 4);
        dequant4s_word(wb.x, pb);
        dequant4s_word(wb.y, pb + 4);
    } else {
        uint4 wa = *reinterpret_cast<const uint4 *>(fa);
        uint4 wb = *reinterpret_cast<const uint4 *>(fb);
        if (XOR80) {
            wa.x ^= 0x80808080u;
            wa.y ^= 0x80808080u;
            wa.z ^= 0x80808080u;
            wa.w ^= 0x80808080u;
            wb.x ^= 0x80808080u;
            wb.y ^= 0x80808080u;
            wb.z ^= 0x80808080u;
            wb.w ^= 0x80808080u;
        }
        dequant8s_word(wa.x, pa);
        dequant8s_word(wa.y, pa + 2);
        dequant8s_word(wa.z, pa + 4);
        dequant8s_word(wa.w, pa + 6);
        dequant8s_word(wb.x, pb);
        dequant8s_word(wb.y, pb + 2);
        dequant8s_word(wb.z, pb + 4);
        dequant8s_word(wb.w, pb + 6);
    }
}

// One output unit (m-tile mt, n-tile nt, lane) of tile t: the lane's four
// accumulator elements are rows (gid, gid + 8) x columns (2 tig, 2 tig + 1).
__device__ __forceinline__ void store_unit(const SmArgs &a, int t, int mt, int nt, int lane, float4 v)
{
    const int gid = lane >> 2, tig = lane & 3;
    const int r_lo = t * a.TM + mt * 16 + gid, r_hi = r_lo + 8;
    const int c0 = nt * 8 + 2 * tig, c1 = c0 + 1;
    if (c0 < a.B) {
        if (r_lo < a.N)
            a.y[(size_t)c0 * a.N + r_lo] = __float2half_rn(v.x);
        if (r_hi < a.N)
            a.y[(size_t)c0 * a.N + r_hi] = __float2half_rn(v.z);
    }
    if (c1 < a.B) {
        if (r_lo < a.N)
            a.y[(size_t)c1 * a.N + r_lo] = __float2half_rn(v.y);
        if (r_hi < a.N)
            a.y[(size_t)c1 * a.N + r_hi] = __float2half_rn(v.w);
    }
}

// FMT: QG_AFFINE (fp16 scale + bias arrays: two 2-D copies per tile), or
// QG_ZP4 / QG_SYM8 (one bf16-scale parameter word per group: one 2-D copy
// into the same bytes); ROT: x rotated by the block-32 Hadamard transform and
// kept as an fp16 (hi, lo) pair, both parts through the same dequantised codes
template <int BITS, int NT, int FMT, bool ROT>
__global__ void __launch_bounds__(SM_THREADS, 1)
    qgemm_small_kernel(SmArgs a, int NS, const __grid_constant__ CUtensorMap codes_map,
                       const __grid_constant__ CUtensorMap scales_map,
                       const __grid_constant__ CUtensorMap biases_map)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const SmLayout L = sm_layout(a.KS, BITS, a.B, a.TM, NS, ROT);
    uint4 *xs = reinterpret_cast<uint4 *>(smem + L.xs_off);
    uint4 *xs_lo = reinterpret_cast<uint4 *>(smem + L.xslo_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    float4 *red = reinterpret_cast<float4 *>(smem + L.red_off);
    int *s_last = reinterpret_cast<int *>(smem + L.last_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + SM_MAX_STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = a.S, q = (int)blockIdx.x % S, per = (int)gridDim.x / S;
    const int n_tiles = (a.N + a.TM - 1) / a.TM;
    const int MT = a.TM / 16;             // 16-row m-tiles per tile
    const int U = MT * NT * 32;           // output units (float4) per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], SM_CW);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == SM_CW) {
        // ---------------- producer: weights are parameters, so they may be
        // streamed before the previous kernel of the stream has finished.
        if (lane == 0) {
            prefetch_tensormap(&codes_map);
            prefetch_tensormap(&scales_map);
            if (FMT == QG_AFFINE)
                prefetch_tensormap(&biases_map);
            const uint64_t pol = l2_evict_first_policy();
            const int cps = a.KS * BITS / 32 / 32;   // 128-byte chunks per slice row
            int k = 0;
            int last_use[SM_MAX_STAGES];
            for (int s = 0; s < SM_MAX_STAGES; ++s)
                last_use[s] = -1;
            for (int t = (int)blockIdx.x / S; t < n_tiles; t += per, ++k) {
                const int st = k % NS, use = k / NS;
                if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, a.status))
                    break;
                unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
                // tensor copies deliver whole boxes (rows past N zero-filled)
                mbar_arrive_expect_tx(&full[st], (uint32_t)(L.codes_bytes + 2 * L.sb_bytes));
                tma_load_3d(stage, &codes_map, 0, t * a.TM, q * cps, &full[st], pol);
                // affine: scales then biases; formats: the parameter words
                // (4 bytes per group, the same bytes)
                tma_load_2d(stage + L.codes_bytes, &scales_map, q * L.GS, t * a.TM, &full[st], pol);
                if (FMT == QG_AFFINE)
                    tma_load_2d(stage + L.codes_bytes + L.sb_bytes, &biases_map, q * L.GS, t * a.TM,
                                &full[st], pol);
                last_use[st] = use;
            }
            // no copy may still be landing when the CTA exits
            for (int s = 0; s < NS; ++s)
                if (last_use[s] >= 0)
                    mbar_wait(&full[s], last_use[s] & 1, a.status);
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    pdl_wait();
    pdl_trigger();
    const int ctid = threadIdx.x;
    constexpr int KIND = BITS == 4 ? kPermS4 : 8;
    constexpr float kCodeScale = BITS == 4 ? kCode4 : kCode8;
    // this slice of x: columns 0..B-1 staged, sums of columns B..31 zero
    if (ROT)
        stage_x_groups<KIND, true>(xs, xsum, L.GS, a.B, a.x + (size_t)q * a.KS, a.K, ctid, SM_CT, 32,
                                   a.signs + (size_t)q * (a.KS / 32), xs_lo);
    else
        stage_x_groups<KIND>(xs, xsum, L.GS, a.B, a.x + (size_t)q * a.KS, a.K, ctid, SM_CT, 32);
    for (int t = ctid; t < L.GS * 32; t += SM_CT)
        if ((t & 31) >= a.B)
            xsum[t] = 0.f;
    named_bar_sync(1, SM_CT);

    const int mt = warp % MT, nblk = SM_CW / MT, gpw = L.GS / nblk;
    const int g0 = (warp / MT) * gpw;
    const int gid = lane >> 2, tig = lane & 3;
    const int r_lo = mt * 16 + gid, r_hi = r_lo + 8;
    const int chunk_bytes = a.TM * 128;
    bool failed = false;
    int k = 0;
    for (int t = (int)blockIdx.x / S; t < n_tiles; t += per, ++k) {
        const int st = k % NS, use = k / NS;
        if (!failed && !mbar_wait(&full[st], use & 1, a.status))
            failed = true;
        // the lanes of a warp decide together: the mma below is warp-collective
        failed = __any_sync(0xffffffffu, failed);
        // code products and folded biases in one accumulator; the power-of-two
        // code scale rides on the group scale (exact)
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[nt][i] = 0.f;
        if (!failed) {
            const unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
            const __half *sc = reinterpret_cast<const __half *>(stage + L.codes_bytes);
            const __half *bi = reinterpret_cast<const __half *>(stage + L.codes_bytes + L.sb_bytes);
            const uint32_t *prm = reinterpret_cast<const uint32_t *>(stage + L.codes_bytes);
            for (int g = g0; g < g0 + gpw; ++g) {
                uint32_t pa[8], pb[8];
                dequant_frags<BITS, FMT == QG_SYM8>(swz128_frag<BITS>(stage, chunk_bytes, r_lo, g, tig),
                                                    swz128_frag<BITS>(stage, chunk_bytes, r_hi, g, tig),
                                                    pa, pb);
                float s_lo, s_hi, b_lo, b_hi;
                if (FMT == QG_AFFINE) {
                    s_lo = __half2float(sc[r_lo * L.GS + g]);
                    s_hi = __half2float(sc[r_hi * L.GS + g]);
                    b_lo = __half2float(bi[r_lo * L.GS + g]);
                    b_hi = __half2float(bi[r_hi * L.GS + g]);
                } else {
                    fmt_scale_bias<FMT>(prm[r_lo * L.GS + g], s_lo, b_lo);
                    fmt_scale_bias<FMT>(prm[r_hi * L.GS + g], s_hi, b_hi);
                }
                s_lo *= kCodeScale;
                s_hi *= kCodeScale;
                // one chain per n-tile (the first product into a fresh
                // accumulator), the n-tiles interleaved; columns past the
                // batch repeat column B - 1 (never stored), so the x loads
                // need no zero fill
                float c[NT][4];
                uint4 x0[NT], x1[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int n = min(nt * 8 + gid, a.B - 1);
                    x0[nt] = xs[((g * 2 + 0) * a.B + n) * 4 + tig];
                    x1[nt] = xs[((g * 2 + 1) * a.B + n) * 4 + tig];
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (BITS == 4) {
                        mma_16816_z(c[nt], pa[0], pb[0], pa[2], pb[2], x0[nt].x, x0[nt].y);
                        mma_16816(c[nt], pa[1], pb[1], pa[3], pb[3], x1[nt].x, x1[nt].y);
                    } else {
                        mma_16816_z(c[nt], pa[0], pb[0], pa[1], pb[1], x0[nt].x, x0[nt].y);
                        mma_16816(c[nt], pa[2], pb[2], pa[3], pb[3], x0[nt].z, x0[nt].w);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (BITS == 4) {
                        mma_16816(c[nt], pa[4], pb[4], pa[6], pb[6], x0[nt].z, x0[nt].w);
                        mma_16816(c[nt], pa[5], pb[5], pa[7], pb[7], x1[nt].z, x1[nt].w);
                    } else {
                        mma_16816(c[nt], pa[4], pb[4], pa[5], pb[5], x1[nt].x, x1[nt].y);
                        mma_16816(c[nt], pa[6], pb[6], pa[7], pb[7], x1[nt].z, x1[nt].w);
                    }
                }
                if (ROT) {   // the lo part of the rotated x through the same codes
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int n = min(nt * 8 + gid, a.B - 1);
                        const uint4 l0 = xs_lo[((g * 2 + 0) * a.B + n) * 4 + tig];
                        const uint4 l1 = xs_lo[((g * 2 + 1) * a.B + n) * 4 + tig];
                        if (BITS == 4) {
                            mma_16816(c[nt], pa[0], pb[0], pa[2], pb[2], l0.x, l0.y);
                            mma_16816(c[nt], pa[1], pb[1], pa[3], pb[3], l1.x, l1.y);
                            mma_16816(c[nt], pa[4], pb[4], pa[6], pb[6], l0.z, l0.w);
                            mma_16816(c[nt], pa[5], pb[5], pa[7], pb[7], l1.z, l1.w);
                        } else {
                            mma_16816(c[nt], pa[0], pb[0], pa[1], pb[1], l0.x, l0.y);
                            mma_16816(c[nt], pa[2], pb[2], pa[3], pb[3], l0.z, l0.w);
                            mma_16816(c[nt], pa[4], pb[4], pa[5], pb[5], l1.x, l1.y);
                            mma_16816(c[nt], pa[6], pb[6], pa[7], pb[7], l1.z, l1.w);
                        }
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float *r = c[nt];
                    const float2 X = *reinterpret_cast<const float2 *>(xsum + g * 32 + nt * 8 + 2 * tig);
                    acc[nt][0] = fmaf(b_lo, X.x, fmaf(s_lo, r[0], acc[nt][0]));
                    acc[nt][1] = fmaf(b_lo, X.y, fmaf(s_lo, r[1], acc[nt][1]));
                    acc[nt][2] = fmaf(b_hi, X.x, fmaf(s_hi, r[2], acc[nt][2]));
                    acc[nt][3] = fmaf(b_hi, X.y, fmaf(s_hi, r[3], acc[nt][3]));
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[st]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            red[(warp * SM_MAX_NT + nt) * 32 + lane] =
                make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
        named_bar_sync(1, SM_CT);
        // reduce the group blocks of each m-tile: one output unit per thread
        float4 own = make_float4(0.f, 0.f, 0.f, 0.f);
        const int o_lane = ctid & 31, o_nt = (ctid >> 5) % NT, o_mt = (ctid >> 5) / NT;
        if (ctid < U) {
            for (int b = 0; b < nblk; ++b) {
                const float4 p = red[((b * MT + o_mt) * SM_MAX_NT + o_nt) * 32 + o_lane];
                own.x += p.x;
                own.y += p.y;
                own.z += p.z;
                own.w += p.w;
            }
            if (S == 1)
                store_unit(a, t, o_mt, o_nt, o_lane, own);
            else
                a.part[((size_t)t * S + q) * U + ctid] = own;
        }
        named_bar_sync(1, SM_CT);   // red may be rewritten from here on
    }
    if (S == 1)
        return;
    // Every partial tile of this CTA is written: one fence, then each tile's
    // counter; the CTA that arrives last at a tile adds its S partials (in
    // slice order, whichever CTA that is) and resets the counter.  Nothing
    // here waits for another CTA.
    __threadfence();
    named_bar_sync(1, SM_CT);
    const int first = (int)blockIdx.x / S;
    for (int j = ctid; j < k; j += SM_CT) {
        const int t = first + j * per;
        const unsigned old = atomicAdd(a.ctr + t, 1u);
        const int last = old == (unsigned)(S - 1);
        if (last)
            a.ctr[t] = 0u;   // every slice has arrived: ready for the next call
        s_last[j] = last;
    }
    named_bar_sync(1, SM_CT);
    __threadfence();
    const int o_lane = ctid & 31, o_nt = (ctid >> 5) % NT, o_mt = (ctid >> 5) / NT;
    for (int j = 0; j < k; ++j) {
        if (!s_last[j] || ctid >= U)
            continue;
        const int t = first + j * per;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sl = 0; sl < S; ++sl) {
            const float4 p = __ldcg(a.part + ((size_t)t * S + sl) * U + ctid);
            v.x += p.x;
            v.y += p.y;
            v.z += p.z;
            v.w += p.w;
        }
        store_unit(a, t, o_mt, o_nt, o_lane, v);
    }
}

// ------------------------------------------------------------------ plan --
struct SmPlan {
    bool ok;
    int S, KS, TM, NT, NS;
    size_t smem, ws_bytes, part_bytes;
};

SmPlan plan_small(int N, int K, int bits, int B, bool rot = false)
{
    SmPlan p;
    memset(&p, 0, sizeof(p));
    if (B < 9 || B > 32 || (bits != 4 && bits != 8) || N <= 0 || K % kGroup)
        return p;
    const int Kw = K * bits / 32;
    if (Kw % 32)   // rows of whole 128-byte chunks (swizzled tensor copies)
        return p;
    for (int S = 1; S <= 8; S *= 2) {
        if (K % S)
            continue;
        const int KS = K / S, GS = KS / kGroup;
        if ((Kw / 32) % S)   // whole 128-byte chunks per slice
            continue;
        if ((size_t)KS * B * 2 * (rot ? 2 : 1) > SM_X_BUDGET)
            continue;
        // ~32 KB of codes per tile; 16, 32 or 64 rows
        int TM = (int)(32768 / ((size_t)KS * bits / 8));
        TM = TM >= 64 ? 64 : TM >= 32 ? 32 : 16;
        const int nblk = SM_CW / (TM / 16);
        if (GS % nblk || GS / nblk < 1 || GS > 256 || GS % 8 || KS * bits / 32 / 32 > 256)
            continue;
        const SmLayout L0 = sm_layout(KS, bits, B, TM, 0, rot);
        const size_t budget = 227 * 1024;
        if (L0.total + 2 * L0.stage_bytes > budget)
            continue;
        int NS = (int)((budget - L0.total) / L0.stage_bytes);
        NS = NS > SM_MAX_STAGES ? SM_MAX_STAGES : NS;
        p.S = S;
        p.KS = KS;
        p.TM = TM;
        p.NT = (B + 7) / 8;
        p.NS = NS;
        p.smem = sm_layout(KS, bits, B, TM, NS, rot).total;
        const size_t tiles = (size_t)(N + TM - 1) / TM;
        if (tiles > (size_t)SM_MAX_TILES)
            return p;
        p.ok = true;
        if (S > 1) {
            p.part_bytes = tiles * S * (TM / 16) * p.NT * 32 * 16;
            p.ws_bytes = SM_CTR_BYTES + p.part_bytes;
        }
        return p;
    }
    return p;
}

template <int BITS, int NT, int FMT, bool ROT>
cudaError_t launch_small_t(const SmArgs &a, const SmPlan &p, const LaunchCfg &c, const CUtensorMap &mc,
                           const CUtensorMap &ms, const CUtensorMap &mb)
{
    cudaError_t e;
    if ((e = set_smem(qgemm_small_kernel<BITS, NT, FMT, ROT>, p.smem)) != cudaSuccess)
        return e;
    const int grid = (c.num_sms / p.S) * p.S;
    return launch_ex(qgemm_small_kernel<BITS, NT, FMT, ROT>, dim3(grid), dim3(SM_THREADS), p.smem, c,
                     1, a, p.NS, mc, ms, mb);
}

template <int FMT, bool ROT>
cudaError_t launch_small_nt(int bits, const SmArgs &a, const SmPlan &p, const LaunchCfg &c,
                            const CUtensorMap &mc, const CUtensorMap &ms, const CUtensorMap &mb)
{
    switch (bits * 10 + p.NT) {
    case 42: return launch_small_t<4, 2, FMT, ROT>(a, p, c, mc, ms, mb);
    case 43: return launch_small_t<4, 3, FMT, ROT>(a, p, c, mc, ms, mb);
    case 44: return launch_small_t<4, 4, FMT, ROT>(a, p, c, mc, ms, mb);
    case 82: return launch_small_t<8, 2, FMT, ROT>(a, p, c, mc, ms, mb);
    case 83: return launch_small_t<8, 3, FMT, ROT>(a, p, c, mc, ms, mb);
    case 84: return launch_small_t<8, 4, FMT, ROT>(a, p, c, mc, ms, mb);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

size_t qgemm_small_workspace_bytes(int N, int K, int bits, int B, bool rot)
{
    const SmPlan p = plan_small(N, K, bits, B, rot);
    return p.ok ? p.ws_bytes : 0;
}

// The one-pass product when the shape allows it; otherwise (or with an
// unaligned scale / bias array) one qGEMV launch per 8 rows of x.
cudaError_t launch_qgemm_small(const QgemvArgs &a, void *ws, size_t ws_bytes, const LaunchCfg &c,
                               bool *used_ws)
{
    *used_ws = false;
    const bool rot = a.signs != nullptr;
    const SmPlan p = plan_small(a.N, a.K, a.bits, a.B, rot);
    // x is read with 16-byte loads; scales and biases (or the parameter words)
    // by 2-D tensor copies
    const uintptr_t sb_addr = a.fmt == QG_AFFINE
                                  ? (reinterpret_cast<uintptr_t>(a.scales) |
                                     reinterpret_cast<uintptr_t>(a.biases))
                                  : reinterpret_cast<uintptr_t>(a.params);
    const int sb_row_bytes = a.K / kGroup * (a.fmt == QG_AFFINE ? 2 : 4);
    const bool align_ok = ((reinterpret_cast<uintptr_t>(a.x) | sb_addr) & 15u) == 0 &&
                          sb_row_bytes % 16 == 0;
    if (!p.ok || !align_ok)
        return launch_qgemv_batched(a, c);
    const int per = c.num_sms / p.S, n_tiles = (a.N + p.TM - 1) / p.TM;
    if (per < 1 || (n_tiles + per - 1) / per > SM_MAX_CTA_TILES)
        return launch_qgemv_batched(a, c);
    if (p.S > 1 && (!ws || ws_bytes < p.ws_bytes || (reinterpret_cast<uintptr_t>(ws) & 15u)))
        return cudaErrorInvalidValue;
    CUtensorMap mc, ms, mb;
    memset(&mc, 0, sizeof(mc));
    memset(&ms, 0, sizeof(ms));
    memset(&mb, 0, sizeof(mb));
    const int Kw = a.K * a.bits / 32;
    const int G = a.K / kGroup;
    bool maps = encode_codes_map(&mc, a.packed, a.N, Kw, p.TM, p.KS * a.bits / 32 / 32);
    if (a.fmt == QG_AFFINE)
        maps = maps && encode_u16_map_2d(&ms, a.scales, a.N, G, p.KS / kGroup, p.TM) &&
               encode_u16_map_2d(&mb, a.biases, a.N, G, p.KS / kGroup, p.TM);
    else
        maps = maps && encode_u32_map_2d(&ms, a.params, a.N, G, p.KS / kGroup, p.TM);
    if (!maps)
        return launch_qgemv_batched(a, c);
    SmArgs s;
    s.x = a.x;
    s.signs = a.signs;
    s.y = a.y;
    s.status = a.status;
    s.N = a.N;
    s.K = a.K;
    s.B = a.B;
    s.S = p.S;
    s.KS = p.KS;
    s.TM = p.TM;
    s.ctr = p.S > 1 ? static_cast<unsigned *>(ws) : nullptr;
    s.part = p.S > 1 ? reinterpret_cast<float4 *>(static_cast<unsigned char *>(ws) + SM_CTR_BYTES) : nullptr;
    *used_ws = p.S > 1;
    switch (a.fmt) {
    case QG_AFFINE:
        return launch_small_nt<QG_AFFINE, false>(a.bits, s, p, c, mc, ms, mb);
    case QG_ZP4:
        return rot ? launch_small_nt<QG_ZP4, true>(4, s, p, c, mc, ms, mb)
                   : launch_small_nt<QG_ZP4, false>(4, s, p, c, mc, ms, mb);
    case QG_SYM8:
        return rot ? launch_small_nt<QG_SYM8, true>(8, s, p, c, mc, ms, mb)
                   : launch_small_nt<QG_SYM8, false>(8, s, p, c, mc, ms, mb);
    }
    return cudaErrorInvalidValue;
}

}  // namespace qmoe
