// prefill.cu -- a prefill chunk (<= 128 tokens) through the MoE layer as a
// grouped affine-4-bit qGEMM.
//
// TurboFieldfare article (jeff.news), section "내부 구조가 진짜 흥미로운 부분"
// (internal structure): prompt prefill runs in chunks of at most 128 tokens so
// that one fetched expert is applied to every row of the chunk routed to it;
// the shared expert's output is added to the routed output.  Same arithmetic
// per token as the decode layer:
//   y[t] = shared(x_t) + sum_j wt[t][j] * down_e( silu(gate_e x_t) * (up_e x_t) ).
//
// Pipeline (all launches chained with programmatic dependent launch):
//   1. group   : (token, slot) pairs listed per expert (misc.cu);
//   2. prep    : x of every token in mma fragment order + group sums; the
//                position of every pair; per-expert 8-token tile offsets;
//   3. gate/up : one warp per (expert, 8 gate + 8 up rows, 8 tokens): the
//                expert's weight tile is read from memory by the warps of its
//                token tiles (from L2 after the first), codes enter the
//                tensor cores as exact fp16 integers, per-group fp32 scale;
//                SwiGLU in registers; h written as fp16 (hi, lo) fragments;
//   4. hsum    : per-group sums of h (bias folding of the down projection);
//   5. down    : one warp per (expert, 16 rows, 8 tokens), hi and lo passes;
//                unweighted expert outputs r[pair position][H] in fp32;
//   6. combine : y[t] = r_shared[t] + sum_j wt[t][j] r[pos(t, j)], in slot
//                order, rounded once to fp16.
// Units of steps 3 and 5 are taken from an atomic counter (heavy experts have
// many token tiles, light ones one), so warps stay busy whatever the skew.
#include "common.cuh"
#include "kernels.h"

namespace qmoe {

namespace {

constexpr int PF_WARPS = 8;   // warps per CTA in the unit kernels

struct PfDims {
    int E, H, I, T, K;        // K = top_k
    int GH, GI, npos;         // npos = T*K + T (shared expert positions last)
};

__host__ __device__ inline PfDims pf_dims(int E, int H, int I, int T, int K)
{
    PfDims d;
    d.E = E;
    d.H = H;
    d.I = I;
    d.T = T;
    d.K = K;
    d.GH = H / kGroup;
    d.GI = I / kGroup;
    d.npos = T * K + T;
    return d;
}

// number of positions (tokens) of expert slot s (s == E: the shared expert)
__device__ __forceinline__ int slot_count(const PrefillArgs &a, int s)
{
    return s < a.E ? a.ws.counts[s] : a.T;
}
__device__ __forceinline__ int slot_offset(const PrefillArgs &a, int s)
{
    return s < a.E ? a.ws.offsets[s] : a.T * a.top_k;
}
// token of position p
__device__ __forceinline__ int pos_token(const PrefillArgs &a, int p)
{
    const int tk = a.T * a.top_k;
    return p < tk ? a.ws.pairs[p] / a.top_k : p - tk;
}

// ------------------------------------------------------------------ prep --
// grid: T CTAs of 128 threads.  CTA t: fragments and group sums of x_t;
// CTA 0 also the per-slot tile offsets, pair positions, unit counters.
__global__ void __launch_bounds__(128) prefill_prep_kernel(PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const int t = blockIdx.x;
    const __half *x = a.x + (size_t)t * d.H;
    uint4 *xf = a.ws.xfrag + (size_t)t * d.GH * 2 * 4;
    float *xs = a.ws.xsum + (size_t)t * d.GH * 8;
    stage_x<4>(xf, xs, d.GH, 1, 1, [&](int, int, int k) { return __half2float(x[k]); },
               threadIdx.x, 128);
    if (t == 0) {
        if (threadIdx.x == 0) {
            int acc = 0;
            for (int s = 0; s <= d.E; ++s) {
                a.ws.tile_off[s] = acc;
                acc += (slot_count(a, s) + 7) / 8;
            }
            a.ws.tile_off[d.E + 1] = acc;
            a.ws.unit_ctr[0] = 0;
            a.ws.unit_ctr[1] = 0;
        }
        // positions of the valid pairs (ids out of range were dropped by the
        // grouping, so only offsets[E] positions hold a pair)
        const int nvalid = a.ws.offsets[d.E];
        for (int p = threadIdx.x; p < nvalid; p += blockDim.x)
            a.ws.inv[a.ws.pairs[p]] = p;
    }
}

// slot s of 8-token tile index `tile` (global over slots): binary search
__device__ __forceinline__ int tile_slot(const PrefillArgs &a, int tile)
{
    int lo = 0, hi = a.E;   // tile_off[lo] <= tile < tile_off[hi + 1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.ws.tile_off[mid] <= tile)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// ------------------------------------------------------------- gate / up --
// unit = (token tile, octet o): 8 gate rows o*8.. and the same 8 up rows of
// the tile's expert, over the tile's <= 8 tokens.
__global__ void __launch_bounds__(PF_WARPS * 32) prefill_gateup_kernel(PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const int octs = d.I / 8;
    const int ntiles = a.ws.tile_off[d.E + 1];
    const int nunits = ntiles * octs;
    const int Hw = d.H / 8;
    while (true) {
        int u = 0;
        if (lane == 0)
            u = atomicAdd(a.ws.unit_ctr + 0, 1);
        u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= nunits)
            break;
        // consecutive units share the weight tile: octet-major over tiles of a slot
        const int s_tile = u / octs, o = u % octs;
        const int s = tile_slot(a, s_tile);
        const int c = s_tile - a.ws.tile_off[s];        // token tile within the slot
        const int cnt = slot_count(a, s), off = slot_offset(a, s);
        const QMat gm = s < d.E ? a.gate : a.sh_gate;
        const QMat um = s < d.E ? a.up : a.sh_up;
        const size_t r0 = (size_t)(s < d.E ? s : 0) * d.I + (size_t)o * 8 + gid;
        const uint32_t *ga = gm.packed + r0 * Hw + 2 * tig;
        const uint32_t *ua = um.packed + r0 * Hw + 2 * tig;
        const __half *gs = gm.scales + r0 * d.GH, *gb = gm.biases + r0 * d.GH;
        const __half *us = um.scales + r0 * d.GH, *ub = um.biases + r0 * d.GH;
        // B column n = gid <-> token of position off + c*8 + gid
        const int pn = c * 8 + gid;
        const bool nvalid = pn < cnt;
        const int tok_n = nvalid ? pos_token(a, off + pn) : 0;
        const uint4 *xf = a.ws.xfrag + (size_t)tok_n * d.GH * 2 * 4;
        // C columns 2tig, 2tig+1 <-> their tokens (for the x group sums)
        const int pc0 = c * 8 + 2 * tig, pc1 = pc0 + 1;
        const float *xs0 = a.ws.xsum + (size_t)(pc0 < cnt ? pos_token(a, off + pc0) : 0) * d.GH * 8;
        const float *xs1 = a.ws.xsum + (size_t)(pc1 < cnt ? pos_token(a, off + pc1) : 0) * d.GH * 8;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
        for (int g = 0; g < d.GH; ++g) {
            const uint2 wa = *reinterpret_cast<const uint2 *>(ga + g * 8);
            const uint2 wb = *reinterpret_cast<const uint2 *>(ua + g * 8);
            uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
            if (nvalid) {
                x0 = __ldcg(xf + (g * 2 + 0) * 4 + tig);
                x1 = __ldcg(xf + (g * 2 + 1) * 4 + tig);
            }
            uint32_t pa[8], pb[8];
            dequant4_word(wa.x, pa);
            dequant4_word(wa.y, pa + 4);
            dequant4_word(wb.x, pb);
            dequant4_word(wb.y, pb + 4);
            float cc[4] = {0.f, 0.f, 0.f, 0.f};
            mma_16816(cc, pa[0], pb[0], pa[1], pb[1], x0.x, x0.y);
            mma_16816(cc, pa[2], pb[2], pa[3], pb[3], x0.z, x0.w);
            mma_16816(cc, pa[4], pb[4], pa[5], pb[5], x1.x, x1.y);
            mma_16816(cc, pa[6], pb[6], pa[7], pb[7], x1.z, x1.w);
            const float sg = __half2float(gs[g]), bg = __half2float(gb[g]);
            const float su = __half2float(us[g]), bu = __half2float(ub[g]);
            const float X0 = xs0[g * 8], X1 = xs1[g * 8];
            acc[0] = fmaf(sg, cc[0], fmaf(bg, X0, acc[0]));   // gate row, token col 2tig
            acc[1] = fmaf(sg, cc[1], fmaf(bg, X1, acc[1]));   // gate row, token col 2tig+1
            acc[2] = fmaf(su, cc[2], fmaf(bu, X0, acc[2]));   // up row
            acc[3] = fmaf(su, cc[3], fmaf(bu, X1, acc[3]));
        }
        // h for intermediate index o*8 + gid, tokens of columns 2tig, 2tig+1
        const int kidx = o * 8 + gid;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int pq = c * 8 + 2 * tig + q;
            if (pq < cnt) {
                const float gv = acc[q], uv = acc[2 + q];
                const float h = gv / (1.f + expf(-gv)) * uv;
                const __half hh = __float2half_rn(h);
                const __half hl = __float2half_rn(h - __half2float(hh));
                __half *hf = reinterpret_cast<__half *>(a.ws.hfrag + (size_t)(off + pq) * d.GI * 2 * 2 * 4);
                // fragment order of the down projection: [g][hh][col][tig][8],
                // columns: 0 = hi, 1 = lo
                const int gg = kidx >> 6, kk = kidx & 63, tg = kk >> 4, p = kk & 15;
                const int qq = p & 7;
                const int i = (p & 8) + 2 * (qq & 3) + (qq >> 2);   // inverse of xperm(4, .)
                const int base = (((gg * 2 + (i >> 3)) * 2) * 4 + tg) * 8 + (i & 7);
                hf[base] = hh;
                hf[base + 4 * 8] = hl;   // column 1 is 4 uint4 (32 halves) further
            }
        }
    }
}

// ------------------------------------------------------------------ hsum --
// per position and group of I: sums of the hi and lo halves
__global__ void __launch_bounds__(256) prefill_hsum_kernel(PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const int n = d.npos * d.GI * 2;
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
        const int col = t & 1, pg = t >> 1;   // pg = pos * GI + g
        const uint4 *f = a.ws.hfrag + (size_t)pg * 2 * 2 * 4;
        float s = 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int tg = 0; tg < 4; ++tg) {
                const uint4 w = f[(hh * 2 + col) * 4 + tg];
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 v = __half22float2(u32_as_h2(ws[q]));
                    s += v.x + v.y;
                }
            }
        a.ws.hsum[t] = s;
    }
}

// ------------------------------------------------------------------ down --
// unit = (token tile, 16-row tile of H): rows of the tile's expert's down
// projection over the tile's <= 8 positions; two passes (h hi, h lo).
__global__ void __launch_bounds__(PF_WARPS * 32) prefill_down_kernel(PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const int rtiles = d.H / 16;
    const int ntiles = a.ws.tile_off[d.E + 1];
    const int nunits = ntiles * rtiles;
    const int Iw = d.I / 8;
    while (true) {
        int u = 0;
        if (lane == 0)
            u = atomicAdd(a.ws.unit_ctr + 1, 1);
        u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= nunits)
            break;
        const int s_tile = u / rtiles, rt = u % rtiles;
        const int s = tile_slot(a, s_tile);
        const int c = s_tile - a.ws.tile_off[s];
        const int cnt = slot_count(a, s), off = slot_offset(a, s);
        const QMat dm = s < d.E ? a.down : a.sh_down;
        const size_t rl = (size_t)(s < d.E ? s : 0) * d.H + (size_t)rt * 16 + gid;
        const uint32_t *wa_p = dm.packed + rl * Iw + 2 * tig;
        const uint32_t *wb_p = wa_p + 8 * Iw;
        const __half *sl = dm.scales + rl * d.GI, *sh = sl + 8 * d.GI;
        const __half *bl = dm.biases + rl * d.GI, *bh = bl + 8 * d.GI;
        const int pn = c * 8 + gid;
        const bool nvalid = pn < cnt;
        const uint4 *hf = a.ws.hfrag + (size_t)(off + (nvalid ? pn : 0)) * d.GI * 2 * 2 * 4;
        const int pc0 = c * 8 + 2 * tig, pc1 = pc0 + 1;
        const float *hs0 = a.ws.hsum + (size_t)(off + (pc0 < cnt ? pc0 : 0)) * d.GI * 2;
        const float *hs1 = a.ws.hsum + (size_t)(off + (pc1 < cnt ? pc1 : 0)) * d.GI * 2;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
        for (int g = 0; g < d.GI; ++g) {
            const uint2 wa = *reinterpret_cast<const uint2 *>(wa_p + g * 8);
            const uint2 wb = *reinterpret_cast<const uint2 *>(wb_p + g * 8);
            uint4 h0 = make_uint4(0, 0, 0, 0), h1 = h0, l0 = h0, l1 = h0;
            if (nvalid) {
                h0 = __ldcg(hf + ((g * 2 + 0) * 2 + 0) * 4 + tig);
                h1 = __ldcg(hf + ((g * 2 + 1) * 2 + 0) * 4 + tig);
                l0 = __ldcg(hf + ((g * 2 + 0) * 2 + 1) * 4 + tig);
                l1 = __ldcg(hf + ((g * 2 + 1) * 2 + 1) * 4 + tig);
            }
            uint32_t pa[8], pb[8];
            dequant4_word(wa.x, pa);
            dequant4_word(wa.y, pa + 4);
            dequant4_word(wb.x, pb);
            dequant4_word(wb.y, pb + 4);
            float cc[4] = {0.f, 0.f, 0.f, 0.f};
            mma_16816(cc, pa[0], pb[0], pa[1], pb[1], h0.x, h0.y);
            mma_16816(cc, pa[2], pb[2], pa[3], pb[3], h0.z, h0.w);
            mma_16816(cc, pa[4], pb[4], pa[5], pb[5], h1.x, h1.y);
            mma_16816(cc, pa[6], pb[6], pa[7], pb[7], h1.z, h1.w);
            mma_16816(cc, pa[0], pb[0], pa[1], pb[1], l0.x, l0.y);
            mma_16816(cc, pa[2], pb[2], pa[3], pb[3], l0.z, l0.w);
            mma_16816(cc, pa[4], pb[4], pa[5], pb[5], l1.x, l1.y);
            mma_16816(cc, pa[6], pb[6], pa[7], pb[7], l1.z, l1.w);
            const float s_l = __half2float(sl[g]), b_l = __half2float(bl[g]);
            const float s_h = __half2float(sh[g]), b_h = __half2float(bh[g]);
            const float X0 = __ldcg(hs0 + g * 2) + __ldcg(hs0 + g * 2 + 1);
            const float X1 = __ldcg(hs1 + g * 2) + __ldcg(hs1 + g * 2 + 1);
            acc[0] = fmaf(s_l, cc[0], fmaf(b_l, X0, acc[0]));
            acc[1] = fmaf(s_l, cc[1], fmaf(b_l, X1, acc[1]));
            acc[2] = fmaf(s_h, cc[2], fmaf(b_h, X0, acc[2]));
            acc[3] = fmaf(s_h, cc[3], fmaf(b_h, X1, acc[3]));
        }
        const int row = rt * 16 + gid;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int pq = c * 8 + 2 * tig + q;
            if (pq < cnt) {
                float *r = a.ws.r + (size_t)(off + pq) * d.H;
                r[row] = acc[q];
                r[row + 8] = acc[2 + q];
            }
        }
    }
}

// --------------------------------------------------------------- combine --
__global__ void __launch_bounds__(256) prefill_combine_kernel(PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const int n = d.T * d.H;
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
        const int tok = t / d.H, col = t % d.H;
        float y = __ldcg(a.ws.r + (size_t)(d.T * d.K + tok) * d.H + col);
        for (int j = 0; j < d.K; ++j) {
            const int e = a.idx[tok * d.K + j];
            if (e < 0 || e >= d.E)
                continue;   // flagged by the grouping kernel, contributes nothing
            const int p = a.ws.inv[tok * d.K + j];
            y = fmaf(a.weights[tok * d.K + j], __ldcg(a.ws.r + (size_t)p * d.H + col), y);
        }
        a.y[t] = __float2half_rn(y);
    }
}

}  // namespace

size_t prefill_workspace_layout(int E, int H, int I, int T, int top_k, void *base,
                                PrefillWorkspace *ws)
{
    const PfDims d = pf_dims(E, H, I, T, top_k);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    const size_t counts_off = take((size_t)E * 4);
    const size_t offsets_off = take((size_t)(E + 1) * 4);
    const size_t pairs_off = take((size_t)T * top_k * 4);
    const size_t inv_off = take((size_t)T * top_k * 4);
    const size_t tile_off = take((size_t)(E + 2) * 4);
    const size_t ctr_off = take(2 * 4);
    const size_t xfrag_off = take((size_t)T * d.GH * 2 * 4 * 16);
    const size_t xsum_off = take((size_t)T * d.GH * 8 * 4);
    const size_t hfrag_off = take((size_t)d.npos * d.GI * 2 * 2 * 4 * 16);
    const size_t hsum_off = take((size_t)d.npos * d.GI * 2 * 4);
    const size_t r_off = take((size_t)d.npos * H * 4);
    if (base && ws) {
        unsigned char *b = static_cast<unsigned char *>(base);
        ws->counts = reinterpret_cast<int32_t *>(b + counts_off);
        ws->offsets = reinterpret_cast<int32_t *>(b + offsets_off);
        ws->pairs = reinterpret_cast<int32_t *>(b + pairs_off);
        ws->inv = reinterpret_cast<int32_t *>(b + inv_off);
        ws->tile_off = reinterpret_cast<int32_t *>(b + tile_off);
        ws->unit_ctr = reinterpret_cast<int32_t *>(b + ctr_off);
        ws->xfrag = reinterpret_cast<uint4 *>(b + xfrag_off);
        ws->xsum = reinterpret_cast<float *>(b + xsum_off);
        ws->hfrag = reinterpret_cast<uint4 *>(b + hfrag_off);
        ws->hsum = reinterpret_cast<float *>(b + hsum_off);
        ws->r = reinterpret_cast<float *>(b + r_off);
    }
    return off;
}

cudaError_t launch_prefill(const PrefillArgs &a, const LaunchCfg &c)
{
    cudaError_t e;
    GroupArgs g;
    g.idx = a.idx;
    g.T = a.T;
    g.top_k = a.top_k;
    g.E = a.E;
    g.counts = a.ws.counts;
    g.offsets = a.ws.offsets;
    g.pairs = a.ws.pairs;
    g.status = a.status;
    if ((e = launch_group(g, c)) != cudaSuccess)
        return e;
    if ((e = launch_ex(prefill_prep_kernel, dim3(a.T), dim3(128), 0, c, 1, a)) != cudaSuccess)
        return e;
    const int grid = c.num_sms * 4;
    if ((e = launch_ex(prefill_gateup_kernel, dim3(grid), dim3(PF_WARPS * 32), 0, c, 1, a)) !=
        cudaSuccess)
        return e;
    if ((e = launch_ex(prefill_hsum_kernel, dim3(c.num_sms), dim3(256), 0, c, 1, a)) != cudaSuccess)
        return e;
    if ((e = launch_ex(prefill_down_kernel, dim3(grid), dim3(PF_WARPS * 32), 0, c, 1, a)) !=
        cudaSuccess)
        return e;
    return launch_ex(prefill_combine_kernel, dim3(c.num_sms * 2), dim3(256), 0, c, 1, a);
}

}  // namespace qmoe
