// qgemv.cu -- dense affine-quantized GEMV, batch 1..8 (decode projection).
//
// y[b][n] = sum_g s[n][g] * (sum_{k in g} q[n][k] x[b][k]) + b[n][g] * X[b][g],
// X[b][g] = sum_{k in g} x[b][k]  -- the bias term folded out of the inner
// product; equal to sum_k (s q + b) x exactly in real arithmetic.
//
// Quantized GEMV is one of the hand-controlled operations of the runtime in
// the TurboFieldfare article (jeff.news, section "기술 맥락" -- technical
// context); the format is the article's "MLX affine 4-bit, group 64"
// (section "성능과 제약").
//
// Design (B200): persistent CTAs, one per SM.  A producer warp streams 16-row
// weight tiles (codes + scales + biases) into a ring of shared-memory stages
// tracked by mbarriers: when the row length is a multiple of 128 bytes the
// codes of a tile arrive in ONE 3-D TMA tensor copy with 128-byte swizzling
// (a 32 KB tile at K = 4096, so the copy engine runs at full rate); otherwise
// each row is a 1-D bulk copy into a padded row.  Sixteen consumer warps form
// tile groups of 4 (of 8 for a batch of 8); tile k goes to group k % groups,
// and each warp of a group takes a contiguous block of the tile's 64-wide
// groups, places the codes in registers as exact fp16 values (the code bits
// as subnormals) and runs mma.sync m16n8k16 with the batch as the N=8
// dimension; scale and bias are applied per group in fp32; the group's
// partial sums meet at its own named barrier and are written as fp16.  x is
// staged once per CTA, one thread per (row, group).
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace qmoe {

// ---------------------------------------------------- host: tensor map --
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled_fn()
{
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            (void)cudaGetLastError();
    }
    return fn;
}

namespace {

constexpr int QG_CW = 16;                     // consumer warps
constexpr int QG_CT = QG_CW * 32;             // consumer threads
constexpr int QG_THREADS = QG_CT + 32;        // + one producer warp
constexpr int QG_MAX_STAGES = 8;

struct QgLayout {
    int G, S;
    size_t xs_off, xslo_off, xsum_off, red_off, bar_off, stage_off;
    size_t codes_bytes, sb_bytes, stage_bytes, total;
};

// Offsets from a 1024-byte aligned base (the swizzled TMA destination must be
// 1024-byte aligned); `total` includes the slack to align the dynamic
// shared-memory window.
__host__ __device__ inline QgLayout qg_layout(int K, int bits, int ncol, int NS, bool swz,
                                               bool rot = false)
{
    QgLayout L;
    L.G = K / kGroup;
    L.S = swz ? K * bits / 32 : tile_stride_words(K, bits);
    size_t off = 0;
    L.xs_off = off;
    off += (size_t)L.G * 2 * ncol * 4 * 16;
    L.xslo_off = off;   // lo parts of a rotated x
    if (rot)
        off += (size_t)L.G * 2 * ncol * 4 * 16;
    L.xsum_off = off;
    off += (size_t)L.G * 8 * 4;
    off = (off + 15) & ~(size_t)15;
    L.red_off = off;
    off += 2 * QG_CW * 32 * 16;
    L.bar_off = off;
    off += 2 * QG_MAX_STAGES * 8 + QG_MAX_STAGES * 4 + 16;   // full, empty, armed sequence, zeros
    off = (off + 1023) & ~(size_t)1023;
    L.stage_off = off;
    L.codes_bytes = (size_t)16 * L.S * 4;
    L.sb_bytes = (size_t)16 * L.G * 2;
    L.stage_bytes = (L.codes_bytes + 2 * L.sb_bytes + 1023) & ~(size_t)1023;
    off += (size_t)NS * L.stage_bytes;
    L.total = off + 1024;
    return L;
}

// ONE: a batch of one token (only MMA column 0 is kept, so the per-group
// scale and bias steps of the other columns are left out).  GW: consumer
// warps per tile group (4; 8 for a full batch of 8, measured faster there)
template <int BITS, bool SWZ, int FMT, bool ROT, bool ONE, int GW>
__global__ void __launch_bounds__(QG_THREADS, 1)
    qgemv_kernel(QgemvArgs a, int NS, const __grid_constant__ CUtensorMap codes_map,
                 const __grid_constant__ CUtensorMap sb0_map,
                 const __grid_constant__ CUtensorMap sb1_map, int sbT)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const QgLayout L = qg_layout(a.K, BITS, a.B, NS, SWZ, ROT);
    uint4 *xs = reinterpret_cast<uint4 *>(smem + L.xs_off);
    uint4 *xs_lo = reinterpret_cast<uint4 *>(smem + L.xslo_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    float4 *red = reinterpret_cast<float4 *>(smem + L.red_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + QG_MAX_STAGES;
    // the tile sequence each stage has been armed for (written by the
    // producer before the copy): a tile group waits for its own sequence
    // there first, so running more than one use of a stage ahead of another
    // group never lets it take an older phase of the full barrier for its own
    volatile int *s_arm = reinterpret_cast<volatile int *>(empty + QG_MAX_STAGES);
    // 16 zero bytes: the x fragment of the MMA columns past the batch
    uint4 *xzero = reinterpret_cast<uint4 *>(smem + L.bar_off + 2 * QG_MAX_STAGES * 8 + QG_MAX_STAGES * 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = (a.N + 15) / 16;
    const int Kw = a.K * BITS / 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], GW);   // the warps of the consuming tile group
            s_arm[s] = -1;
        }
        *xzero = make_uint4(0, 0, 0, 0);
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == QG_CW) {
        // ---------------- producer: weights are parameters, so they may be
        // streamed before the previous kernel of the stream has finished.
        if (lane == 0) {
            if (SWZ)
                prefetch_tensormap(&codes_map);
            const uint64_t pol = l2_evict_first_policy();
            int k = 0;
            int last_use[QG_MAX_STAGES];
            for (int s = 0; s < QG_MAX_STAGES; ++s)
                last_use[s] = -1;
            for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++k) {
                const int st = k % NS, use = k / NS;
                if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, a.status))
                    break;
                s_arm[st] = k;
                const int r0 = item * 16;
                const int rows = min(16, a.N - r0);
                const uint32_t row_bytes = (uint32_t)Kw * 4;
                // (a transposed tensor copy delivers all 16 rows, past N zero-filled)
                const uint32_t sb = (uint32_t)(((SWZ && sbT) ? 16 : rows) * L.G * 2);
                unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
                if (SWZ) {
                    // the tensor copy always delivers the whole 16-row box
                    // (rows past N arrive zero-filled)
                    mbar_arrive_expect_tx(&full[st], (uint32_t)L.codes_bytes + 2 * sb);
                    tma_load_3d(stage, &codes_map, 0, r0, 0, &full[st], pol);
                } else {
                    mbar_arrive_expect_tx(&full[st], rows * row_bytes + 2 * sb);
                    for (int r = 0; r < rows; ++r)
                        bulk_g2s(stage + (size_t)r * L.S * 4, a.packed + (size_t)(r0 + r) * Kw,
                                 row_bytes, &full[st], pol);
                }
                if (SWZ && sbT) {
                    // transposed: [G / 8][16 rows][8 halves] (or [G / 4][16][4
                    // words]), so the 8 rows of a fragment read 16 bytes apart
                    tma_load_3d(stage + L.codes_bytes, &sb0_map, 0, r0, 0, &full[st], pol);
                    if (FMT == QG_AFFINE)
                        tma_load_3d(stage + L.codes_bytes + L.sb_bytes, &sb1_map, 0, r0, 0,
                                    &full[st], pol);
                } else if (FMT == QG_AFFINE) {
                    bulk_g2s(stage + L.codes_bytes, a.scales + (size_t)r0 * L.G, sb, &full[st], pol);
                    bulk_g2s(stage + L.codes_bytes + L.sb_bytes, a.biases + (size_t)r0 * L.G, sb,
                             &full[st], pol);
                } else {   // one parameter word per group: the same bytes as scale + bias
                    bulk_g2s(stage + L.codes_bytes, a.params + (size_t)r0 * L.G, 2 * sb, &full[st],
                             pol);
                }
                last_use[st] = use;
            }
            // no copy may still be landing when the CTA exits
            for (int s = 0; s < NS; ++s)
                if (last_use[s] >= 0)
                    mbar_wait(&full[s], last_use[s] & 1, a.status);
        }
        return;
    }

    // -------------------- consumers
    pdl_wait();
    pdl_trigger();
    const int ctid = threadIdx.x;
    constexpr int KIND = BITS == 4 ? kPermS4 : 8;
    constexpr float kCodeScale = BITS == 4 ? kCode4 : kCode8;   // undoes the subnormal codes
    if (ROT)
        stage_x_groups<KIND, true>(xs, xsum, L.G, a.B, a.x, a.K, ctid, QG_CT, 8, a.signs, xs_lo);
    else if ((reinterpret_cast<uintptr_t>(a.x) & 15u) == 0)
        stage_x_groups<KIND>(xs, xsum, L.G, a.B, a.x, a.K, ctid, QG_CT);
    else
        stage_x<KIND>(xs, xsum, L.G, a.B, 1,
                      [&](int, int n, int k) { return __half2float(a.x[(size_t)n * a.K + k]); },
                      ctid, QG_CT);
    named_bar_sync(1, QG_CT);

    // tiles go to groups of GW warps (tile k to group k % NG); a warp
    // takes a contiguous quarter of the tile's groups, so that with G % 64 ==
    // 0 the scales and biases of a row come as one 8-byte load per 4 groups,
    // and the group's partial sums meet at a barrier of its own
    constexpr int NG = QG_CW / GW;   // tile groups
    const int grp = warp / GW, wq = warp % GW;
    const int gpw = (L.G + GW - 1) / GW;
    const int g0 = min(L.G, wq * gpw), g1 = min(L.G, g0 + gpw);
    const bool vec_sb = (L.G & 63) == 0;
    const int gid = lane >> 2, tig = lane & 3;
    bool failed = false;
    int kk = 0;   // tiles this group has done (alternates its partial-sum buffers)
    for (int k = grp; blockIdx.x + k * gridDim.x < n_items; k += NG, ++kk) {
        const int item = blockIdx.x + k * gridDim.x;
        const int st = k % NS, use = k / NS;
        if (!failed && !(wait_armed(s_arm + st, k, a.status) && mbar_wait(&full[st], use & 1, a.status)))
            failed = true;
        // the lanes of a warp decide together: the mma below is warp-collective
        failed = __any_sync(0xffffffffu, failed);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (!failed) {
            const unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
            const uint32_t *tile = reinterpret_cast<const uint32_t *>(stage);
            const __half *sc = reinterpret_cast<const __half *>(stage + L.codes_bytes);
            const __half *bi = reinterpret_cast<const __half *>(stage + L.codes_bytes + L.sb_bytes);
            // code products and folded biases accumulate apart; the subnormal
            // factor is applied once at the end
            float aq[4] = {0.f, 0.f, 0.f, 0.f}, ab[4] = {0.f, 0.f, 0.f, 0.f};
            // one group from its fragment addresses (rows gid, gid+8)
            // branch-free: the MMA columns past the batch read a zero block
            const bool live = gid < a.B;
            const uint4 *xq = live ? xs + gid * 4 + tig : xzero;
            const uint4 *xql = live ? xs_lo + gid * 4 + tig : xzero;
            const int xst = live ? 2 * a.B * 4 : 0, x1o = live ? a.B * 4 : 0;
            auto group = [&](int g, const void *fa, const void *fb, float s_lo, float s_hi,
                             float b_lo, float b_hi) {
                const uint4 x0 = xq[g * xst], x1 = xq[g * xst + x1o];
                uint4 l0 = make_uint4(0, 0, 0, 0), l1 = l0;
                if (ROT) {
                    l0 = xql[g * xst];
                    l1 = xql[g * xst + x1o];
                }
                float r[4];
                if (BITS == 4 && ROT)
                    mma_group_s4_hilo(r, *reinterpret_cast<const uint2 *>(fa),
                                      *reinterpret_cast<const uint2 *>(fb), x0, x1, l0, l1);
                else if (BITS == 4)
                    mma_group_s4_1(r, *reinterpret_cast<const uint2 *>(fa),
                                   *reinterpret_cast<const uint2 *>(fb), x0, x1);
                else if (FMT == QG_SYM8) {
                    // two's-complement byte q -> q + 128 = byte ^ 0x80; the
                    // -128 s offset joins the folded bias
                    uint4 wa = *reinterpret_cast<const uint4 *>(fa);
                    uint4 wb = *reinterpret_cast<const uint4 *>(fb);
                    wa.x ^= 0x80808080u;
                    wa.y ^= 0x80808080u;
                    wa.z ^= 0x80808080u;
                    wa.w ^= 0x80808080u;
                    wb.x ^= 0x80808080u;
                    wb.y ^= 0x80808080u;
                    wb.z ^= 0x80808080u;
                    wb.w ^= 0x80808080u;
                    if (ROT)
                        mma_group_s8_hilo(r, wa, wb, x0, x1, l0, l1);
                    else
                        mma_group_s8_1(r, wa, wb, x0, x1);
                } else
                    mma_group_s8_1(r, *reinterpret_cast<const uint4 *>(fa),
                                   *reinterpret_cast<const uint4 *>(fb), x0, x1);
                if (ONE) {
                    const float X = xsum[g * 8];
                    aq[0] = fmaf(s_lo, r[0], aq[0]);
                    aq[2] = fmaf(s_hi, r[2], aq[2]);
                    ab[0] = fmaf(b_lo, X, ab[0]);
                    ab[2] = fmaf(b_hi, X, ab[2]);
                } else {
                    const float2 X = *reinterpret_cast<const float2 *>(xsum + g * 8 + 2 * tig);
                    aq[0] = fmaf(s_lo, r[0], aq[0]);
                    aq[1] = fmaf(s_lo, r[1], aq[1]);
                    aq[2] = fmaf(s_hi, r[2], aq[2]);
                    aq[3] = fmaf(s_hi, r[3], aq[3]);
                    ab[0] = fmaf(b_lo, X.x, ab[0]);
                    ab[1] = fmaf(b_lo, X.y, ab[1]);
                    ab[2] = fmaf(b_hi, X.x, ab[2]);
                    ab[3] = fmaf(b_hi, X.y, ab[3]);
                }
            };
            // fragment address of row r, group g
            auto frag = [&](int r, int g) -> const void * {
                if (SWZ)
                    return swz128_frag<BITS>(stage, 2048, r, g, tig);
                return BITS == 4 ? (const void *)(tile + r * L.S + g * 8 + 2 * tig)
                                 : (const void *)(tile + r * L.S + g * 16 + 4 * tig);
            };
            if (vec_sb) {
                // 4 groups per step (g0 % 4 == 0): fragment offsets of row gid
                // precomputed; row gid+8 is 16 rows of bytes further
                constexpr int GPC = BITS == 4 ? 4 : 2;   // groups per 128-byte chunk
                int off[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int jc = j % GPC;
                    off[j] = SWZ ? gid * 128 + (j / GPC) * 2048 +
                                       (BITS == 4 ? ((((2 * jc + (tig >> 1)) ^ gid) << 4) + (tig & 1) * 8)
                                                  : (((4 * jc + tig) ^ gid) << 4))
                                 : (gid * L.S + j * (BITS == 4 ? 8 : 16) + tig * (BITS == 4 ? 2 : 4)) * 4;
                }
                const int row8 = SWZ ? 8 * 128 : 8 * L.S * 4;
                for (int gb = g0; gb < g1; gb += 4) {
                    const unsigned char *base =
                        stage + (SWZ ? (gb / GPC) * 2048 : gb * (BITS == 4 ? 32 : 64));
                    if (FMT == QG_AFFINE) {
                        // row r, groups gb..gb+3: row-major [16][G], or
                        // transposed [G/8][16][8]
                        const int olo = sbT ? ((gb >> 3) * 16 + gid) * 8 + (gb & 7) : gid * L.G + gb;
                        const int ohi = sbT ? olo + 8 * 8 : (gid + 8) * L.G + gb;
                        const uint2 slo = *reinterpret_cast<const uint2 *>(sc + olo);
                        const uint2 shi = *reinterpret_cast<const uint2 *>(sc + ohi);
                        const uint2 blo = *reinterpret_cast<const uint2 *>(bi + olo);
                        const uint2 bhi = *reinterpret_cast<const uint2 *>(bi + ohi);
                        const uint32_t sl[2] = {slo.x, slo.y}, sh[2] = {shi.x, shi.y};
                        const uint32_t bl[2] = {blo.x, blo.y}, bh[2] = {bhi.x, bhi.y};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 fsl = __half22float2(u32_as_h2(sl[j >> 1]));
                            const float2 fsh = __half22float2(u32_as_h2(sh[j >> 1]));
                            const float2 fbl = __half22float2(u32_as_h2(bl[j >> 1]));
                            const float2 fbh = __half22float2(u32_as_h2(bh[j >> 1]));
                            group(gb + j, base + off[j], base + off[j] + row8,
                                  (j & 1) ? fsl.y : fsl.x, (j & 1) ? fsh.y : fsh.x,
                                  (j & 1) ? fbl.y : fbl.x, (j & 1) ? fbh.y : fbh.x);
                        }
                    } else {
                        const uint32_t *prm = reinterpret_cast<const uint32_t *>(sc);
                        // row-major [16][G] words, or transposed [G/4][16][4]
                        const int olo = sbT ? ((gb >> 2) * 16 + gid) * 4 : gid * L.G + gb;
                        const int ohi = sbT ? olo + 8 * 4 : (gid + 8) * L.G + gb;
                        const uint4 plo = *reinterpret_cast<const uint4 *>(prm + olo);
                        const uint4 phi = *reinterpret_cast<const uint4 *>(prm + ohi);
                        const uint32_t pl[4] = {plo.x, plo.y, plo.z, plo.w};
                        const uint32_t ph[4] = {phi.x, phi.y, phi.z, phi.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float s_lo, s_hi, b_lo, b_hi;
                            fmt_scale_bias<FMT>(pl[j], s_lo, b_lo);
                            fmt_scale_bias<FMT>(ph[j], s_hi, b_hi);
                            group(gb + j, base + off[j], base + off[j] + row8, s_lo, s_hi, b_lo, b_hi);
                        }
                    }
                }
            } else if (FMT == QG_AFFINE) {
                for (int g = g0; g < g1; ++g)
                    group(g, frag(gid, g), frag(gid + 8, g), __half2float(sc[gid * L.G + g]),
                          __half2float(sc[(gid + 8) * L.G + g]), __half2float(bi[gid * L.G + g]),
                          __half2float(bi[(gid + 8) * L.G + g]));
            } else {
                const uint32_t *prm = reinterpret_cast<const uint32_t *>(sc);
                for (int g = g0; g < g1; ++g) {
                    float s_lo, s_hi, b_lo, b_hi;
                    fmt_scale_bias<FMT>(prm[gid * L.G + g], s_lo, b_lo);
                    fmt_scale_bias<FMT>(prm[(gid + 8) * L.G + g], s_hi, b_hi);
                    group(g, frag(gid, g), frag(gid + 8, g), s_lo, s_hi, b_lo, b_hi);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                acc[i] = fmaf(aq[i], kCodeScale, ab[i]);
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[st]);
        float4 *gred = red + (size_t)((grp * 2 + (kk & 1)) * GW) * 32;
        gred[wq * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        named_bar_sync(2 + grp, GW * 32);
        if (wq == kk % GW) {
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            for (int w = 0; w < GW; ++w) {
                const float4 p = gred[w * 32 + lane];
                v[0] += p.x;
                v[1] += p.y;
                v[2] += p.z;
                v[3] += p.w;
            }
            const int r_lo = item * 16 + gid, r_hi = r_lo + 8;
            const int c0 = 2 * tig, c1 = c0 + 1;
            if (c0 < a.B) {
                if (r_lo < a.N)
                    a.y[(size_t)c0 * a.N + r_lo] = __float2half_rn(v[0]);
                if (r_hi < a.N)
                    a.y[(size_t)c0 * a.N + r_hi] = __float2half_rn(v[2]);
            }
            if (c1 < a.B) {
                if (r_lo < a.N)
                    a.y[(size_t)c1 * a.N + r_lo] = __float2half_rn(v[1]);
                if (r_hi < a.N)
                    a.y[(size_t)c1 * a.N + r_hi] = __float2half_rn(v[3]);
            }
        }
    }
}

// 3-D map of a per-group parameter array [rows][G] of elem-byte entries seen
// as [G / n16][rows][n16] (n16 entries = 16 bytes): one copy delivers a
// 16-row tile transposed, [G / n16][16][n16]
bool encode_param_map_t(CUtensorMap *m, const void *base, long rows, int G, int elem)
{
    EncodeTiledFn fn = encode_tiled_fn();
    const int n16 = 16 / elem;
    if (!fn || (reinterpret_cast<uintptr_t>(base) & 15u) || G % n16 || G / n16 > 256 ||
        ((size_t)G * elem) % 16)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)n16, (cuuint64_t)rows, (cuuint64_t)(G / n16)};
    const cuuint64_t strides[2] = {(cuuint64_t)G * elem, 16};
    const cuuint32_t box[3] = {(cuuint32_t)n16, 16, (cuuint32_t)(G / n16)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 3,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BITS, bool SWZ, int FMT, bool ROT>
cudaError_t launch_qgemv_t(const QgemvArgs &a, const LaunchCfg &c, const CUtensorMap &m)
{
    const size_t budget = 227 * 1024;
    const QgLayout L0 = qg_layout(a.K, BITS, a.B, 0, SWZ, ROT);
    // one stage still works (copy and compute then alternate); it is only
    // needed by the largest rotated 8-bit rows at batch 8
    if (L0.total + L0.stage_bytes > budget)
        return cudaErrorInvalidValue;
    int NS = (int)((budget - L0.total) / L0.stage_bytes);
    NS = NS > QG_MAX_STAGES ? QG_MAX_STAGES : NS;
    const QgLayout L = qg_layout(a.K, BITS, a.B, NS, SWZ, ROT);
    const int n_items = (a.N + 15) / 16;
    const int grid = n_items < c.num_sms ? n_items : c.num_sms;
    cudaError_t e;
    if ((e = set_smem(qgemv_kernel<BITS, SWZ, FMT, ROT, false, 4>, L.total)) != cudaSuccess ||
        (e = set_smem(qgemv_kernel<BITS, SWZ, FMT, ROT, false, 8>, L.total)) != cudaSuccess ||
        (e = set_smem(qgemv_kernel<BITS, SWZ, FMT, ROT, true, 4>, L.total)) != cudaSuccess)
        return e;
    // scales and biases (or the parameter words) transposed by tensor copies
    // where the rows take the swizzled tile path and G % 64 == 0
    const int G = a.K / kGroup;
    CUtensorMap m0, m1;
    memset(&m0, 0, sizeof(m0));
    memset(&m1, 0, sizeof(m1));
    int sbT = 0;
    if (SWZ && G % 64 == 0) {
        if (FMT == QG_AFFINE)
            sbT = encode_param_map_t(&m0, a.scales, a.N, G, 2) &&
                  encode_param_map_t(&m1, a.biases, a.N, G, 2);
        else
            sbT = encode_param_map_t(&m0, a.params, a.N, G, 4);
    }
    if (a.B == 1)
        return launch_ex(qgemv_kernel<BITS, SWZ, FMT, ROT, true, 4>, dim3(grid), dim3(QG_THREADS),
                         L.total, c, 1, a, NS, m, m0, m1, sbT);
    if (a.B == 8)
        return launch_ex(qgemv_kernel<BITS, SWZ, FMT, ROT, false, 8>, dim3(grid), dim3(QG_THREADS),
                         L.total, c, 1, a, NS, m, m0, m1, sbT);
    return launch_ex(qgemv_kernel<BITS, SWZ, FMT, ROT, false, 4>, dim3(grid), dim3(QG_THREADS), L.total, c, 1,
                     a, NS, m, m0, m1, sbT);
}

template <bool SWZ>
cudaError_t launch_qgemv_fmt(const QgemvArgs &a, const LaunchCfg &c, const CUtensorMap &m)
{
    const bool rot = a.signs != nullptr;
    switch (a.fmt) {
    case QG_AFFINE:
        return a.bits == 4 ? launch_qgemv_t<4, SWZ, QG_AFFINE, false>(a, c, m)
                           : launch_qgemv_t<8, SWZ, QG_AFFINE, false>(a, c, m);
    case QG_ZP4:
        return rot ? launch_qgemv_t<4, SWZ, QG_ZP4, true>(a, c, m)
                   : launch_qgemv_t<4, SWZ, QG_ZP4, false>(a, c, m);
    case QG_SYM8:
        return rot ? launch_qgemv_t<8, SWZ, QG_SYM8, true>(a, c, m)
                   : launch_qgemv_t<8, SWZ, QG_SYM8, false>(a, c, m);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool encode_codes_map(CUtensorMap *m, const uint32_t *packed, long rows, int Kw, int box_rows,
                      int box_chunks)
{
    EncodeTiledFn fn = encode_tiled_fn();
    if (box_chunks <= 0)
        box_chunks = Kw / 32;
    if (!fn || Kw % 32 != 0 || box_chunks > 256 || box_chunks > Kw / 32 || box_rows < 1 ||
        box_rows > 256)
        return false;
    const cuuint64_t dims[3] = {32, (cuuint64_t)rows, (cuuint64_t)(Kw / 32)};
    const cuuint64_t strides[2] = {(cuuint64_t)Kw * 4, 128};
    const cuuint32_t box[3] = {32, (cuuint32_t)box_rows, (cuuint32_t)box_chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t *>(packed), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

bool encode_u16_map_2d(CUtensorMap *m, const void *base, long rows, int cols, int box_cols,
                       int box_rows)
{
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn || (reinterpret_cast<uintptr_t>(base) & 15u) || (cols * 2) % 16 || (box_cols * 2) % 16 ||
        box_cols < 1 || box_cols > 256 || box_cols > cols || box_rows < 1 || box_rows > 256)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_u32_map_2d(CUtensorMap *m, const void *base, long rows, int cols, int box_cols,
                       int box_rows)
{
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn || (reinterpret_cast<uintptr_t>(base) & 15u) || (cols * 4) % 16 || (box_cols * 4) % 16 ||
        box_cols < 1 || box_cols > 256 || box_cols > cols || box_rows < 1 || box_rows > 256)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_qgemv(const QgemvArgs &a, const LaunchCfg &c)
{
    const int Kw = a.K * a.bits / 32;
    CUtensorMap m;
    memset(&m, 0, sizeof(m));
    const bool swz = encode_codes_map(&m, a.packed, a.N, Kw, 16) &&
                     qg_layout(a.K, a.bits, a.B, 1, true, a.signs != nullptr).total <= 227 * 1024;
    return swz ? launch_qgemv_fmt<true>(a, c, m) : launch_qgemv_fmt<false>(a, c, m);
}

// does a slice of b rows of x fit on chip beside one stage of 16 weight rows
// (either tile layout launch_qgemv may pick)?
static bool slice_fits(const QgemvArgs &a, int b)
{
    const bool rot = a.signs != nullptr;
    const size_t budget = 227 * 1024;
    const bool swz_ok = (a.K * a.bits / 32) % 32 == 0 &&
                        qg_layout(a.K, a.bits, b, 1, true, rot).total <= budget;
    return swz_ok || qg_layout(a.K, a.bits, b, 1, false, rot).total <= budget;
}

cudaError_t launch_qgemv_batched(const QgemvArgs &a, const LaunchCfg &c)
{
    // rows of x per launch: 8, fewer where long 8-bit rows leave no room
    int step = a.B < 8 ? a.B : 8;
    while (step > 1 && !slice_fits(a, step))
        --step;
    for (int b0 = 0; b0 < a.B; b0 += step) {
        QgemvArgs s = a;
        s.x = a.x + (size_t)b0 * a.K;
        s.y = a.y + (size_t)b0 * a.N;
        s.B = a.B - b0 < step ? a.B - b0 : step;
        const cudaError_t e = launch_qgemv(s, c);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace qmoe
