// prefill_tc.cu -- the heavy experts of a prefill chunk on the 5th-generation
// tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// TurboFieldfare article (jeff.news), section "내부 구조가 진짜 흥미로운 부분"
// (internal structure): a prompt is prefilled in chunks of at most 128
// tokens so that one fetched expert serves every row of the chunk routed to
// it.  Under skewed routing a few experts (and always the shared expert) get
// tens of tokens each; for them the product is a real matrix product and runs
// here.  Experts with fewer tokens stay on the streaming kernels of
// prefill.cu.
//
// A unit is (heavy slot, 128 consecutive weight rows): D[128][N] =
// W[rows, K] X[N tokens, K]^T, the weights as the M operand and the slot's
// tokens (N <= 128, padded to a multiple of 16) as N.  Per 64-input group:
//   * a TMA copy brings the group's 4-bit codes of the 128 rows (4 KB);
//   * 8 dequantisation warps turn them into w' = s*(q - 8) as an EXACT pair
//     of fp16 values: hi = fp16(w') (one HMUL2) and lo = w' - hi (one HFMA2,
//     exact because w' has at most 15 significant bits), written in the
//     128-byte-swizzled K-major layout the tensor core reads.  The centred
//     codes keep the running sums small: the tensor core's additions lose
//     bits in proportion to the accumulator's magnitude, and 0..15 codes
//     would add a 7.5 s sum(x) drift to every partial sum;
//   * one thread issues tcgen05.mma kind::f16: the hi x hi products into
//     one fp32 accumulator in tensor memory, the small cross products
//     (about 2^-11 of the others) into a second one; the epilogue adds the
//     two in fp32.  Chained into the same accumulator, part of the cross
//     products' bits were lost inside the tensor-core additions.
// The bias is one more K-block: A = b' = b + 8 s per (row, group) as an fp16
// (hi, lo) pair, B = the group sums of the activations as an fp16 (hi, lo)
// pair, so that
//   D = sum_g s_g sum_k (q - 8) x + sum_g (b_g + 8 s_g) X_g
//     = sum_g s_g sum_k q x + sum_g b_g X_g   (= the affine product)
// to fp32 accumulation.  A single fp16 or bf16 dequantised tile (s*q + b
// rounded once) would cost up to 2e-2 of relative error on these
// cancellation-heavy outputs; the exact pair keeps the products exact.
//   gate/up: two accumulators (gate and up rows of the same indices), B = x
//            (exact fp16); the epilogue reads both from tensor memory and
//            writes h = silu(g) * u as an fp16 (hi, lo) pair per position,
//            plus the pair's group sums;
//   down:    B = h hi and h lo; products w_hi h_hi + w_lo h_hi + w_hi h_lo
//            (the w_lo h_lo term is below fp32 rounding); the epilogue writes
//            the unweighted expert output r[position][H] in fp32, which the
//            chunk's combine kernel weights and adds per token.
// Activations reach shared memory by TMA from this GPU's own memory only (no
// multicast).  The k order inside every 8 inputs is (0,4,1,5,2,6,3,7) on
// both operands -- the order in which a code word unpacks -- which leaves
// the dot products unchanged.
//
// Roles: warp 0 TMA producer, warp 1 MMA issuer (and tensor-memory owner),
// warps 2..9 dequantisation and epilogue.  Every wait is bounded; on a
// timeout the CTA raises its abort word, every role stops, in-flight copies
// and MMAs are drained and the tensor memory is freed before exit.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace qmoe {

namespace {

constexpr int TC_M = 128;                              // weight rows per unit
constexpr int TC_DQ = 8;                               // dequantisation / epilogue warps
constexpr int TC_THREADS = (2 + TC_DQ) * 32;
constexpr int TC_NC = 6;                               // code stages, 4 KB each
constexpr int TC_NA = 3;                               // A stages: hi + lo tiles
constexpr int TC_NB = 2;                               // B stages: two tiles
constexpr int TC_TILE = 16384;                         // one 128 x 64 fp16 tile
constexpr int TC_CODES = TC_M * 32;                    // codes of one group, 128 rows
constexpr uint32_t TC_TMEM_COLS = 512;                 // all of an SM's tensor memory
constexpr uint32_t TC_LO_COL = 256;                    // first column of the cross products
constexpr int TC_BAR_EPI = 1;                          // named barrier of the epilogue warps
constexpr int TC_SC_STRIDE = 66;                       // scale row stride in halves (33 words: odd)

// barriers
enum {
    B_FULL_C = 0,
    B_EMPTY_C = B_FULL_C + TC_NC,
    B_FULL_A = B_EMPTY_C + TC_NC,
    B_EMPTY_A = B_FULL_A + TC_NA,
    B_FULL_B = B_EMPTY_A + TC_NA,
    B_EMPTY_B = B_FULL_B + TC_NB,
    B_ACC_FULL = B_EMPTY_B + TC_NB,
    B_ACC_EMPTY,
    B_DRAIN,
    B_COUNT
};

struct TcLayout {
    size_t a_off, b_off, c_off, sc_off, hsp_off, bar_off, misc_off, total;
};

__host__ __device__ inline TcLayout tc_layout()
{
    TcLayout L;
    size_t off = 0;
    L.a_off = off;
    off += (size_t)TC_NA * 2 * TC_TILE;
    L.b_off = off;
    off += (size_t)TC_NB * 2 * TC_TILE;
    L.c_off = off;
    off += (size_t)TC_NC * TC_CODES;
    L.sc_off = off;
    off += (size_t)2 * TC_M * TC_SC_STRIDE * 2;
    L.hsp_off = off;
    off += (size_t)4 * TC_M * 4;
    L.bar_off = off;
    off += (size_t)B_COUNT * 8;
    L.misc_off = off;
    off += 16;   // tensor-memory address, abort word
    L.total = off + 1024;   // alignment slack of the dynamic base
    return L;
}

// ------------------------------------------------------------ tcgen05 PTX --
// shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (the canonical layout a 128-byte swizzled TMA box leaves)
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;                  // leading byte offset (unused here)
    d |= (uint64_t)(1024 >> 4) << 32;        // stride byte offset
    d |= (uint64_t)1 << 46;                  // descriptor version
    d |= (uint64_t)2 << 61;                  // 128-byte swizzle
    return d;
}

// instruction descriptor: fp16 A and B (K-major), fp32 D, M = 128, N = n
__device__ __forceinline__ uint32_t tc_idesc(int n)
{
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TC_M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// 32 lanes x 16 consecutive fp32 columns of tensor memory
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

// 2-D tiled TMA load (no multicast) completing on `bar`
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, int c0, int c1,
                                            uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_last_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// ---------------------------------------------------------------- waits --
// bounded wait that gives up at once after another thread of the CTA did
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, int32_t *status,
                                        volatile int *abort_word)
{
    if (*abort_word)
        return false;
    if (mbar_wait(bar, parity, status))
        return true;
    *abort_word = 1;
    return false;
}

// -------------------------------------------------------------- schedule --
// unit u = (heavy slot list entry u / RB, row block u % RB); slots sorted by
// decreasing token count, so the largest units are spread first
struct TcUnit {
    int slot, p0, n, npad, rb;
};

__device__ __forceinline__ TcUnit tc_unit(const PrefillArgs &a, int RB, int u)
{
    TcUnit t;
    t.slot = a.ws.heavy[u / RB];
    t.rb = u % RB;
    t.p0 = t.slot < a.E ? a.ws.offsets[t.slot] : a.T * a.top_k;
    t.n = t.slot < a.E ? a.ws.counts[t.slot] : a.T;
    t.npad = (t.n + 15) & ~15;
    return t;
}

// position in a row of the activation buffers of input k: within every 8
// inputs the order (0,4,1,5,2,6,3,7)
__device__ __forceinline__ int perm_col(int k)
{
    const int j = k & 7;
    return (k & ~7) | ((j & 3) << 1) | (j >> 2);
}

struct TcMaps {
    CUtensorMap codes[2];      // routed matrix codes (gate, up) or (down, -)
    CUtensorMap sh_codes[2];   // the shared expert's
    CUtensorMap act[2];        // B of the main k-blocks: x (gate/up) or h hi, h lo (down)
    CUtensorMap sums[2];       // B of the bias block: group sums hi, lo
};

// =================================================================== kernel --
// DOWN = false: gate/up + SwiGLU (rows = I, K = H); true: down (rows = H, K = I)
template <bool DOWN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ TcMaps maps)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const TcLayout L = tc_layout();
    unsigned char *a_ring = smem + L.a_off;
    unsigned char *b_ring = smem + L.b_off;
    unsigned char *c_ring = smem + L.c_off;
    __half *sc = reinterpret_cast<__half *>(smem + L.sc_off);   // [mat][row][TC_SC_STRIDE]
    float *hsp = reinterpret_cast<float *>(smem + L.hsp_off);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint32_t *tmem_word = reinterpret_cast<uint32_t *>(smem + L.misc_off);
    volatile int *abort_word = reinterpret_cast<volatile int *>(smem + L.misc_off + 4);

    constexpr int NM = DOWN ? 1 : 2;                 // matrices per unit
    // gate/up units run their K in NKH halves with fresh accumulators; the
    // epilogue adds the halves in fp32 (partial sums through tcpart), so no
    // tensor-memory accumulator chains more than half the k-blocks
    constexpr int NKH = DOWN ? 1 : 2;
    const int rows = DOWN ? a.H : a.I;               // rows of one expert's matrix
    const int K = DOWN ? a.I : a.H;
    const int GK = K / kGroup;                       // main k-blocks
    // end of K part kh's k-blocks; the last part also takes the bias block (kb == GK)
    auto kb_end = [&](int kh) { return kh + 1 == NKH ? GK + 1 : (kh + 1) * GK / NKH; };
    const int RB = (rows + TC_M - 1) / TC_M;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < TC_NC; ++i) {
            mbar_init(&bar[B_FULL_C + i], 1);
            mbar_init(&bar[B_EMPTY_C + i], TC_DQ);
        }
        for (int i = 0; i < TC_NA; ++i) {
            mbar_init(&bar[B_FULL_A + i], TC_DQ);
            mbar_init(&bar[B_EMPTY_A + i], 1);
        }
        for (int i = 0; i < TC_NB; ++i) {
            mbar_init(&bar[B_FULL_B + i], 1);
            mbar_init(&bar[B_EMPTY_B + i], 1);
        }
        mbar_init(&bar[B_ACC_FULL], 1);
        mbar_init(&bar[B_ACC_EMPTY], TC_DQ);
        mbar_init(&bar[B_DRAIN], 1);
        *abort_word = 0;
        mbar_init_fence();
    }
    if (warp == 1) {   // tensor memory for the accumulators (this warp frees it)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_word)),
                     "r"(TC_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_word;
    // the heavy-slot list and the activations come from earlier kernels
    pdl_wait();
    pdl_trigger();
    const int nunits = a.ws.unit_ctr[3] * RB;

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0 && nunits > 0) {
            const uint64_t pol_w = l2_evict_first_policy();
            const uint64_t pol_a = l2_evict_last_policy();
            for (int m = 0; m < NM; ++m) {
                prefetch_tensormap(&maps.codes[m]);
                prefetch_tensormap(&maps.sh_codes[m]);
            }
            int cs = 0, bs = 0;   // code / B stage sequence numbers
            int lastc[TC_NC], lastb[TC_NB];
            for (int i = 0; i < TC_NC; ++i)
                lastc[i] = -1;
            for (int i = 0; i < TC_NB; ++i)
                lastb[i] = -1;
            bool ok = true;
            for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
                const TcUnit t = tc_unit(a, RB, u);
                const bool sh = t.slot == a.E;
                const int row0 = (sh ? 0 : t.slot * rows) + t.rb * TC_M;
                const uint32_t btile = (uint32_t)t.npad * 128;
                for (int kh = 0; kh < NKH && ok; ++kh)
                for (int kb = kh * GK / NKH; kb < kb_end(kh) && ok; ++kb) {
                    if (kb < GK) {
                        for (int m = 0; m < NM && ok; ++m) {
                            const int s = cs % TC_NC;
                            if (cs >= TC_NC &&
                                !tc_wait(&bar[B_EMPTY_C + s], ((cs / TC_NC) - 1) & 1, a.status, abort_word)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(&bar[B_FULL_C + s], TC_CODES);
                            tma_load_2d(c_ring + (size_t)s * TC_CODES, sh ? &maps.sh_codes[m] : &maps.codes[m],
                                        kb * 8, row0, &bar[B_FULL_C + s], pol_w);
                            lastc[s] = cs / TC_NC;
                            ++cs;
                        }
                    }
                    if (!ok)
                        break;
                    // B of this k-block: one tile (x), or two (h hi / lo, or the
                    // group sums hi / lo of the bias block)
                    const int s = bs % TC_NB;
                    if (bs >= TC_NB &&
                        !tc_wait(&bar[B_EMPTY_B + s], ((bs / TC_NB) - 1) & 1, a.status, abort_word)) {
                        ok = false;
                        break;
                    }
                    const bool bias = kb == GK;
                    const int ntile = (bias || DOWN) ? 2 : 1;
                    mbar_arrive_expect_tx(&bar[B_FULL_B + s], btile * ntile);
                    for (int ti = 0; ti < ntile; ++ti) {
                        const CUtensorMap *mp = bias ? &maps.sums[ti] : &maps.act[ti];
                        unsigned char *dst = b_ring + ((size_t)s * 2 + ti) * TC_TILE;
                        for (int r = 0; r < t.npad; r += 16)
                            tma_load_2d(dst + (size_t)r * 128, mp, bias ? 0 : kb * kGroup, t.p0 + r,
                                        &bar[B_FULL_B + s], pol_a);
                    }
                    lastb[s] = bs / TC_NB;
                    ++bs;
                }
            }
            // no copy may still be landing when the CTA exits
            for (int i = 0; i < TC_NC; ++i)
                if (lastc[i] >= 0)
                    mbar_wait(&bar[B_FULL_C + i], lastc[i] & 1, a.status);
            for (int i = 0; i < TC_NB; ++i)
                if (lastb[i] >= 0)
                    mbar_wait(&bar[B_FULL_B + i], lastb[i] & 1, a.status);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0 && nunits > 0) {
            int as = 0, bs = 0, nu = 0;
            bool ok = true, issued = false;
            for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x)
            for (int kh = 0; kh < NKH && ok; ++kh, ++nu) {
                const TcUnit t = tc_unit(a, RB, u);
                const uint32_t idesc = tc_idesc(t.npad);
                const int kb0 = kh * GK / NKH;
                // the epilogue has read the previous accumulators
                if (nu > 0 && !tc_wait(&bar[B_ACC_EMPTY], (nu - 1) & 1, a.status, abort_word)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = kb0; kb < kb_end(kh) && ok; ++kb) {
                    const bool bias = kb == GK;
                    const int sb = bs % TC_NB;
                    if (!tc_wait(&bar[B_FULL_B + sb], (bs / TC_NB) & 1, a.status, abort_word)) {
                        ok = false;
                        break;
                    }
                    const uint32_t b0 = smem_u32(b_ring + (size_t)sb * 2 * TC_TILE);
                    const uint32_t b1 = b0 + TC_TILE;
                    for (int m = 0; m < NM; ++m) {
                        const int sa = as % TC_NA;
                        if (!tc_wait(&bar[B_FULL_A + sa], (as / TC_NA) & 1, a.status, abort_word)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t ahi = smem_u32(a_ring + (size_t)sa * 2 * TC_TILE);
                        const uint32_t alo = ahi + TC_TILE;
                        // hi x hi products in d; the small cross products
                        // (lo x hi, hi x lo) in their own accumulator dl
                        const uint32_t d = tmem + (uint32_t)(m * 128);
                        const uint32_t dl = d + TC_LO_COL;
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint32_t ko = 32u * ks;
                            const uint32_t acc0 = (kb > kb0 || ks > 0) ? 1u : 0u;
                            if (bias) {
                                tc_mma(d, tc_desc(ahi + ko), tc_desc(b0 + ko), idesc, 1u);
                                tc_mma(dl, tc_desc(alo + ko), tc_desc(b0 + ko), idesc, 1u);
                                tc_mma(dl, tc_desc(ahi + ko), tc_desc(b1 + ko), idesc, 1u);
                            } else {
                                tc_mma(d, tc_desc(ahi + ko), tc_desc(b0 + ko), idesc, acc0);
                                tc_mma(dl, tc_desc(alo + ko), tc_desc(b0 + ko), idesc, acc0);
                                if (DOWN)
                                    tc_mma(dl, tc_desc(ahi + ko), tc_desc(b1 + ko), idesc, 1u);
                            }
                        }
                        issued = true;
                        tc_commit(&bar[B_EMPTY_A + sa]);   // the A stage is free once these finish
                        ++as;
                    }
                    if (!ok)
                        break;
                    tc_commit(&bar[B_EMPTY_B + sb]);
                    ++bs;
                }
                if (ok)
                    tc_commit(&bar[B_ACC_FULL]);   // the accumulators of this K part are complete
            }
            // every MMA issued has finished before the tensor memory is freed
            if (issued) {
                tc_commit(&bar[B_DRAIN]);
                mbar_wait(&bar[B_DRAIN], 0, a.status);
            }
        }
    } else {
        // ================================================= dequantise + epilogue
        const int dt = threadIdx.x - 64;           // 0 .. 255
        const int r = dt & (TC_M - 1);            // weight row of the unit
        const int hw = dt >> 7;                   // half of the row's 8 code words
        const int dw = warp - 2;                  // 0 .. 7
        const int q = warp & 3;                   // tensor-memory lane quarter
        const int chalf = dw >> 2;                // column half of the epilogue
        int cs = 0, as = 0, nu = 0;
        bool dead = false;   // this warp saw a failed wait (uniform within the warp)
        for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
            // the 8 warps leave together once any of them failed, and only
            // then may this unit's scales overwrite the previous unit's
            if (bar_any(TC_BAR_EPI + 1, TC_DQ * 32, dead || *abort_word != 0))
                break;
            const TcUnit t = tc_unit(a, RB, u);
            const bool sh = t.slot == a.E;
            const int erow = t.rb * TC_M + r;       // row within the expert's matrix
            const bool rvalid = erow < rows;
            const size_t grow = (size_t)(sh ? 0 : t.slot) * rows + erow;
            // scales of this thread's row (half of the groups)
            for (int m = 0; m < NM; ++m) {
                const QMat &W = DOWN ? (sh ? a.sh_down : a.down)
                                     : (m == 0 ? (sh ? a.sh_gate : a.gate) : (sh ? a.sh_up : a.up));
                for (int g = hw; g < GK; g += 2) {
                    const __half sv = rvalid ? W.scales[grow * GK + g] : __float2half(0.f);
                    sc[((size_t)m * TC_M + r) * TC_SC_STRIDE + g] = sv;
                }
            }
            named_bar_sync(TC_BAR_EPI + 1, TC_DQ * 32);
            for (int kh = 0; kh < NKH; ++kh, ++nu) {
            for (int kb = kh * GK / NKH; kb < kb_end(kh) && !dead; ++kb) {
                for (int m = 0; m < NM && !dead; ++m) {
                    const int sa = as % TC_NA;
                    if (as >= TC_NA &&
                        !__all_sync(0xffffffffu, tc_wait(&bar[B_EMPTY_A + sa], ((as / TC_NA) - 1) & 1,
                                                         a.status, abort_word))) {
                        dead = true;
                        break;
                    }
                    unsigned char *ahi = a_ring + (size_t)sa * 2 * TC_TILE;
                    unsigned char *rowhi = ahi + (size_t)r * 128;
                    unsigned char *rowlo = rowhi + TC_TILE;
                    if (kb < GK) {
                        const int s = cs % TC_NC;
                        if (!__all_sync(0xffffffffu, tc_wait(&bar[B_FULL_C + s], (cs / TC_NC) & 1,
                                                             a.status, abort_word))) {
                            dead = true;
                            break;
                        }
                        const uint4 wv =
                            *reinterpret_cast<const uint4 *>(c_ring + (size_t)s * TC_CODES + r * 32 + hw * 16);
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive(&bar[B_EMPTY_C + s]);
                        ++cs;
                        const __half2 s2 = __half2half2(sc[((size_t)m * TC_M + r) * TC_SC_STRIDE + kb]);
                        const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            uint32_t qv[4], hi[4], lo[4];
                            dequant4c_word(words[w], qv);   // q - 8: (c0,c4)(c1,c5)(c2,c6)(c3,c7)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const __half2 h = __hmul2(s2, u32_as_h2(qv[i]));
                                hi[i] = h2_as_u32(h);
                                lo[i] = h2_as_u32(__hfma2(s2, u32_as_h2(qv[i]), __hneg2(h)));
                            }
                            const int chunk = hw * 4 + w;
                            const int off = ((chunk ^ (r & 7)) << 4);
                            *reinterpret_cast<uint4 *>(rowhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                            *reinterpret_cast<uint4 *>(rowlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                        }
                    } else {
                        // bias block: A = b' = b + 8 s per (row, group) for the K / 64
                        // groups (zeros after) as an fp16 (hi, lo) pair -- the 8 s
                        // the centred codes q - 8 left out
                        const QMat &W = DOWN ? (sh ? a.sh_down : a.down)
                                             : (m == 0 ? (sh ? a.sh_gate : a.gate) : (sh ? a.sh_up : a.up));
                        const __half *srow = sc + ((size_t)m * TC_M + r) * TC_SC_STRIDE;
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            const int chunk = hw * 4 + c4;
                            uint32_t vh[4], vl[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                // memory order of the chunk: groups 8c + (0,4,1,5,2,6,3,7)
                                const int g0 = chunk * 8 + i, g1 = chunk * 8 + i + 4;
                                const float f0 = (rvalid && g0 < GK)
                                                     ? __half2float(W.biases[grow * GK + g0]) +
                                                           8.f * __half2float(srow[g0])
                                                     : 0.f;
                                const float f1 = (rvalid && g1 < GK)
                                                     ? __half2float(W.biases[grow * GK + g1]) +
                                                           8.f * __half2float(srow[g1])
                                                     : 0.f;
                                const __half h0 = __float2half_rn(f0), h1 = __float2half_rn(f1);
                                vh[i] = h2_as_u32(__halves2half2(h0, h1));
                                vl[i] = h2_as_u32(__halves2half2(__float2half_rn(f0 - __half2float(h0)),
                                                                 __float2half_rn(f1 - __half2float(h1))));
                            }
                            const int off = ((chunk ^ (r & 7)) << 4);
                            *reinterpret_cast<uint4 *>(rowhi + off) = make_uint4(vh[0], vh[1], vh[2], vh[3]);
                            *reinterpret_cast<uint4 *>(rowlo + off) = make_uint4(vl[0], vl[1], vl[2], vl[3]);
                        }
                    }
                    // generic-proxy writes -> visible to the tensor core
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&bar[B_FULL_A + sa]);
                    ++as;
                }
            }
            // ---------------- epilogue: accumulators -> global
            const bool acc_ok =
                !dead && __all_sync(0xffffffffu, tc_wait(&bar[B_ACC_FULL], nu & 1, a.status, abort_word));
            if (!acc_ok)
                dead = true;
            tc_fence_after();
            const int myrow = t.rb * TC_M + 32 * q + lane;
            // this thread's (gate, up) partial sums of the earlier K parts:
            // row 32 q + lane, the thread's own columns, written and read
            // back by the same thread
            float2 *part = reinterpret_cast<float2 *>(a.ws.tcpart) +
                           (size_t)blockIdx.x * (kTcPartBytes / 8) + (size_t)(32 * q + lane) * 128;
            if (acc_ok) {
                for (int c0 = 16 * chalf; c0 < t.npad; c0 += 32) {
                    float dv[16], uv[16];
                    const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0;
                    float lv[16];
                    tc_ld16(ta, dv);
                    tc_ld16(ta + TC_LO_COL, lv);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        dv[i] += lv[i];
                    if (!DOWN) {
                        tc_ld16(ta + 128, uv);
                        tc_ld16(ta + 128 + TC_LO_COL, lv);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            uv[i] += lv[i];
                        if (kh > 0) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float2 pv = part[c0 + i];
                                dv[i] += pv.x;
                                uv[i] += pv.y;
                            }
                        }
                        if (kh + 1 < NKH) {   // not the last K part: keep the sums
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                part[c0 + i] = make_float2(dv[i], uv[i]);
                            continue;
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int n = c0 + i;
                        if (n >= t.n)
                            continue;   // padding column (the same for every lane)
                        const int pos = t.p0 + n;
                        if (DOWN) {
                            if (myrow < a.H)
                                __stcg(a.ws.r + (size_t)pos * a.H + myrow, dv[i]);
                        } else {
                            float h = 0.f;
                            if (myrow < a.I)
                                h = dv[i] / (1.f + expf(-dv[i])) * uv[i];
                            const __half hh = __float2half_rn(h);
                            const __half hl = __float2half_rn(h - __half2float(hh));
                            if (myrow < a.I) {
                                const size_t o = (size_t)pos * a.I + perm_col(myrow);
                                a.ws.hb_hi[o] = hh;
                                a.ws.hb_lo[o] = hl;
                            }
                            // sum of the pair over the warp's 32 rows (half a group)
                            float sm = __half2float(hh) + __half2float(hl);
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1)
                                sm += __shfl_xor_sync(0xffffffffu, sm, o);
                            if (lane == 0)
                                hsp[q * TC_M + n] = sm;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&bar[B_ACC_EMPTY]);
            if (!DOWN && kh + 1 == NKH) {
                // group sums of h: rows 0..63 of the unit are group 2 rb, 64..127
                // group 2 rb + 1; every warp's partials are in before they are read
                const bool all_ok = !bar_any(TC_BAR_EPI, TC_DQ * 32, !acc_ok);
                if (all_ok)
                    for (int i = dt; i < 2 * t.n; i += TC_DQ * 32) {
                        const int n = i >> 1, gsel = i & 1;
                        const int g = 2 * t.rb + gsel;
                        if (g * kGroup >= a.I)
                            continue;
                        const float sm = hsp[(2 * gsel) * TC_M + n] + hsp[(2 * gsel + 1) * TC_M + n];
                        const __half sh_ = __float2half_rn(sm);
                        const size_t o = (size_t)(t.p0 + n) * 64 + perm_col(g);
                        a.ws.hs_hi[o] = sh_;
                        a.ws.hs_lo[o] = __float2half_rn(sm - __half2float(sh_));
                    }
                named_bar_sync(TC_BAR_EPI, TC_DQ * 32);   // hsp is free for the next unit
            }
            }   // K parts
        }
    }

    // ---- exit: every role is done; the accumulators' owner frees them
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TC_TMEM_COLS)
                     : "memory");
}

// ------------------------------------------------------------ host side --
typedef CUresult (*EncodeTiledFnTc)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                    const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                    const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnTc tc_encode_fn()
{
    static EncodeTiledFnTc fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFnTc>(p);
        else
            (void)cudaGetLastError();
    }
    return fn;
}

// codes [rows][Kw] uint32, box 8 words (one group) x 128 rows, no swizzle
bool tc_codes_map(CUtensorMap *m, const uint32_t *packed, long rows, int Kw)
{
    EncodeTiledFnTc fn = tc_encode_fn();
    if (!fn || (reinterpret_cast<uintptr_t>(packed) & 15u) || (Kw * 4) % 16 || Kw < 8)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)Kw, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)Kw * 4};
    const cuuint32_t box[2] = {8, (cuuint32_t)TC_M};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(packed), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp16 [rows][cols], box 64 x 16 rows, 128-byte swizzle (the K-major layout
// the tensor core reads)
bool tc_act_map(CUtensorMap *m, const void *base, long rows, int cols)
{
    EncodeTiledFnTc fn = tc_encode_fn();
    if (!fn || (reinterpret_cast<uintptr_t>(base) & 15u) || (cols * 2) % 16 || cols < 64)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, 16};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(int H, int I)
{
    return H % 64 == 0 && I % 64 == 0 && H / kGroup <= 64 && I / kGroup <= 64 &&
           tc_encode_fn() != nullptr;
}

cudaError_t launch_prefill_tc(const PrefillArgs &a, const LaunchCfg &c, bool down)
{
    const int npos = a.T * a.top_k + a.T;
    TcMaps mp;
    memset(&mp, 0, sizeof(mp));
    bool ok = true;
    if (!down) {
        const int Kw = a.H / 8;
        ok = ok && tc_codes_map(&mp.codes[0], a.gate.packed, (long)a.E * a.I, Kw);
        ok = ok && tc_codes_map(&mp.codes[1], a.up.packed, (long)a.E * a.I, Kw);
        ok = ok && tc_codes_map(&mp.sh_codes[0], a.sh_gate.packed, a.I, Kw);
        ok = ok && tc_codes_map(&mp.sh_codes[1], a.sh_up.packed, a.I, Kw);
        ok = ok && tc_act_map(&mp.act[0], a.ws.xg, npos, a.H);
        mp.act[1] = mp.act[0];
        ok = ok && tc_act_map(&mp.sums[0], a.ws.xb_hi, npos, 64);
        ok = ok && tc_act_map(&mp.sums[1], a.ws.xb_lo, npos, 64);
    } else {
        const int Kw = a.I / 8;
        ok = ok && tc_codes_map(&mp.codes[0], a.down.packed, (long)a.E * a.H, Kw);
        mp.codes[1] = mp.codes[0];
        ok = ok && tc_codes_map(&mp.sh_codes[0], a.sh_down.packed, a.H, Kw);
        mp.sh_codes[1] = mp.sh_codes[0];
        ok = ok && tc_act_map(&mp.act[0], a.ws.hb_hi, npos, a.I);
        ok = ok && tc_act_map(&mp.act[1], a.ws.hb_lo, npos, a.I);
        ok = ok && tc_act_map(&mp.sums[0], a.ws.hs_hi, npos, 64);
        ok = ok && tc_act_map(&mp.sums[1], a.ws.hs_lo, npos, 64);
    }
    if (!ok)
        return cudaErrorInvalidValue;
    const size_t smem = tc_layout().total;
    const int grid = c.num_sms < kTcMaxCtas ? c.num_sms : kTcMaxCtas;   // tcpart blocks
    cudaError_t e;
    if (down) {
        if ((e = set_smem(prefill_tc_kernel<true>, smem)) != cudaSuccess)
            return e;
        return launch_ex(prefill_tc_kernel<true>, dim3(grid), dim3(TC_THREADS), smem, c, 1, a, mp);
    }
    if ((e = set_smem(prefill_tc_kernel<false>, smem)) != cudaSuccess)
        return e;
    return launch_ex(prefill_tc_kernel<false>, dim3(grid), dim3(TC_THREADS), smem, c, 1, a, mp);
}

}  // namespace qmoe
