// common.cuh -- device building blocks shared by the qmoe kernels (sm_100a).
//
// * mbarrier + cp.async.bulk (TMA bulk copy) helpers with bounded waits;
// * programmatic-dependent-launch controls (griddepcontrol);
// * register dequantisation of packed 4-bit / 8-bit affine codes into exact
//   fp16 integers laid out as mma.sync m16n8k16 A fragments;
// * the x-fragment staging permutation that matches those A fragments.
//
// Storage format (TurboFieldfare article, jeff.news, section "성능과 제약" --
// MLX affine 4-bit, group 64; 8-bit router): element k of a row sits in word
// k / (32/bits) at bit offset bits*(k % (32/bits)); w = scale*q + bias with an
// fp16 scale and bias per group of 64 inputs.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "qmoe.h"

namespace qmoe {

constexpr int kGroup = 64;
// A pipeline wait that has not completed after this long gives up, records
// QMOE_DEV_TIMEOUT and lets the kernel return (no kernel ever spins forever).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// ----------------------------------------------------------------- basics --
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void flag_status(int32_t *status, int32_t flag)
{
    atomicOr(reinterpret_cast<int *>(status), flag);
}

// ------------------------------------------------------------- mbarriers --
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Make mbarrier initialisation visible to the async (TMA) proxy and the rest
// of the CTA; follow with a CTA barrier.
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// try_wait with a suspend-time hint: the waiting thread is parked (it issues
// nothing) until the phase completes or the hint expires, so waiting warps do
// not take issue slots from the warps doing the math.
constexpr uint32_t kSuspendHintNs = 100000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns
// false (and flags QMOE_DEV_TIMEOUT) if it does not within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int32_t *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            flag_status(status, QMOE_DEV_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait until a ring stage has been armed for sequence `sq` (a word
// the producer writes before each copy).  Returns false (and flags
// QMOE_DEV_TIMEOUT) if it is not within kWaitLimitNs.
__device__ __forceinline__ bool wait_armed(const volatile int *arm, int sq, int32_t *status)
{
    if (*arm == sq)
        return true;
    const unsigned long long t0 = global_timer_ns();
    while (*arm != sq) {
        __nanosleep(20);
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            flag_status(status, QMOE_DEV_TIMEOUT);
            return false;
        }
    }
    return true;
}

// ------------------------------------------------------ TMA bulk copies --
// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`
// (transaction bytes).  Both addresses 16-byte aligned, bytes % 16 == 0.
// Streams weights, so it carries an L2 evict-first policy.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void bulk_g2s(void *smem_dst, const void *gsrc, uint32_t bytes,
                                         uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 3-D tiled TMA tensor copy global -> this CTA's shared memory (no multicast),
// completing on `bar`; `tmap` is the address of a __grid_constant__ tensor map
// kernel parameter.  Coordinates are element indices, innermost first.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *tmap, int c0, int c1,
                                            int c2, uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)),
        "l"(policy)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const void *tmap)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// --------------------------------------------------- dependent launches --
// Wait until the preceding kernel of the stream has completed and its memory
// is visible (no-op when the kernel was not launched as a dependent).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next kernel of the stream to start launching.
__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------- named barriers --
__device__ __forceinline__ void named_bar_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// named barrier of n threads that also ORs a predicate over them: every
// participant gets the same answer (used to leave loops together)
__device__ __forceinline__ bool bar_any(int id, int n, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------------------ mma --
// D = A(16x16 f16, row) * B(16x8 f16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// the same product into a fresh accumulator: d = A B
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic)
{
    uint32_t d;
    // d = (a & mask) | magic
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));
    return d;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// ------------------------------------------------- register dequant --
// The codes are exact small integers, so they enter the tensor core as exact
// fp16 values; scale and bias are applied per group in fp32 afterwards.
//
// 4-bit: one word holds codes c0..c7 (nibble i = code i).  Placing a nibble in
// the low mantissa bits of fp16 1024.0 (0x6400) gives 1024 + q exactly, and a
// nibble in mantissa bits 4..7 gives 1024 + 16q; both map back to q exactly
// with one fp16 subtract / fused multiply-add.  Output pairs (low, high half):
//   p[0] = (c0, c4)  p[1] = (c1, c5)  p[2] = (c2, c6)  p[3] = (c3, c7)
__device__ __forceinline__ void dequant4_word(uint32_t w, uint32_t *p)
{
    const uint32_t magic = 0x64006400u;
    const __half2 k1024 = __floats2half2_rn(1024.f, 1024.f);
    const __half2 k1_16 = __floats2half2_rn(0.0625f, 0.0625f);
    const __half2 km64 = __floats2half2_rn(-64.f, -64.f);
    const uint32_t ws = w >> 8;
    p[0] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(w, 0x000F000Fu, magic)), k1024));
    p[1] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(w, 0x00F000F0u, magic)), k1_16, km64));
    p[2] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(ws, 0x000F000Fu, magic)), k1024));
    p[3] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(ws, 0x00F000F0u, magic)), k1_16, km64));
}

// The same pairs centred, q - 8 (exact: 1024 + q - 1032, (1024 + 16q)/16 - 72).
__device__ __forceinline__ void dequant4c_word(uint32_t w, uint32_t *p)
{
    const uint32_t magic = 0x64006400u;
    const __half2 k1032 = __floats2half2_rn(1032.f, 1032.f);
    const __half2 k1_16 = __floats2half2_rn(0.0625f, 0.0625f);
    const __half2 km72 = __floats2half2_rn(-72.f, -72.f);
    const uint32_t ws = w >> 8;
    p[0] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(w, 0x000F000Fu, magic)), k1032));
    p[1] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(w, 0x00F000F0u, magic)), k1_16, km72));
    p[2] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(ws, 0x000F000Fu, magic)), k1032));
    p[3] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(ws, 0x00F000F0u, magic)), k1_16, km72));
}

// 8-bit: one word holds codes c0..c3 (byte i = code i).
//   p[0] = (c0, c2)  p[1] = (c1, c3)
__device__ __forceinline__ void dequant8_word(uint32_t w, uint32_t *p)
{
    const uint32_t magic = 0x64006400u;
    const __half2 k1024 = __floats2half2_rn(1024.f, 1024.f);
    p[0] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(w, 0x00FF00FFu, magic)), k1024));
    p[1] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(w >> 8, 0x00FF00FFu, magic)), k1024));
}

// Cheaper dequantisation for the streaming kernels: the code itself becomes
// the fp16 bit pattern (no exponent bits), i.e. an fp16 subnormal, placed
// high in the mantissa: a nibble in bits 4..7 (16q * 2^-24 = q * 2^-20), a
// byte in bits 2..9 (b * 2^-22).  Measured on B200 (mma.sync m16n8k16, f16 x
// f16 -> f32, error relative to sum |a b|): codes as normal fp16 integers
// ~1e-7, a byte in bits 2..9 1.6e-7, a nibble in bits 6..9 1.0-1.5e-7, in
// bits 4..7 2.9-4.6e-7, in bits 0..3 up to 1.6e-5 (the low subnormals lose
// bits inside the tensor core).  Bits 4..7 cost one shift fewer than 6..9
// (one nibble pair is already in place: 3 shifts + 4 ANDs per word) and stay
// far inside the error budget.  Pairs (both halves of a register):
//   p[0] = (c0, c4)   p[1] = (c1, c5)   p[2] = (c2, c6)   p[3] = (c3, c7)
// all in units of 2^-20; callers scale results by kCode4 = 2^20.
__device__ __forceinline__ void dequant4s_word(uint32_t w, uint32_t *p)
{
    p[0] = (w << 4) & 0x00F000F0u;
    p[1] = w & 0x00F000F0u;
    p[2] = (w >> 4) & 0x00F000F0u;
    p[3] = (w >> 8) & 0x00F000F0u;
}
// 8-bit: bytes as subnormals b * 2^-22: p[0] = (c0, c2), p[1] = (c1, c3).
__device__ __forceinline__ void dequant8s_word(uint32_t w, uint32_t *p)
{
    p[0] = (w << 2) & 0x03FC03FCu;
    p[1] = (w >> 6) & 0x03FC03FCu;
}
constexpr float kCode4 = 1048576.f;   // 2^20: undoes dequant4s_word
constexpr float kCode8 = 4194304.f;   // 2^22: undoes dequant8s_word

// x order matching dequant4s_word, k-blocks (c0,c4)(c2,c6) | (c8,c12)(c10,c14)
// | (c1,c5)(c3,c7) | (c9,c13)(c11,c15): class-0 codes in the first 8 slots.
__host__ __device__ __forceinline__ int xperm_s4(int i)
{
    const int hi = (i & 4) << 1;           // +8 for i = 4..7 and 12..15
    const int odd = (i >> 3) & 1;          // class 1 for i >= 8
    const int j = i & 3;                   // (0,4)(2,6) pattern
    return hi + odd + ((j >> 1) << 1) + ((j & 1) << 2);
}

// Order in which a thread (quad index tig) needs the 16 x values
// x[64g + 16 tig + perm[i]] of group g so that its two 16-byte x fragments
// line up with the A fragments produced above (k-slot order of m16n8k16).
// `kind`: 4 (dequant4_word), 8 (dequant8_word / dequant8s_word), or
// kPermS4 (dequant4s_word).
constexpr int kPermS4 = 5;
__host__ __device__ __forceinline__ int xperm(int kind, int i)
{
    // 4-bit: pairs (0,4)(1,5)(2,6)(3,7)(8,12)(9,13)(10,14)(11,15)
    // 8-bit: pairs (0,2)(1,3)(4,6)(5,7)(8,10)(9,11)(12,14)(13,15)
    if (kind == kPermS4)
        return xperm_s4(i);
    const int hi = i & 8;
    const int j = i & 7;
    if (kind == 4)
        return hi + (j >> 1) + ((j & 1) << 2);
    return hi + ((j >> 2) << 2) + ((j >> 1) & 1) + ((j & 1) << 1);
}

// Accumulate one group (64 inputs) of a 16-row tile held in shared memory
// into acc (C fragment of m16n8k16: rows gid / gid+8, columns 2tig, 2tig+1).
//   tile: row r of the codes at tile + r*stride (words)
//   sc, bi: fp16 [16][G] scales / biases of the tile's rows
//   xs: x fragments, uint4 [G][2][ncol][4]; columns >= ncol read as zero
//   xsum: fp32 [G][8] sum of x over each group, per column (bias folding:
//         sum_k (s q_k + b) x_k = s * sum_k q_k x_k + b * sum_k x_k)
//   frag(r): address of this lane's codes of row r (r = gid or gid + 8) in
//         group g: 8 bytes (words 2tig, 2tig+1 of the group) for 4-bit,
//         16 bytes (words 4tig..4tig+3) for 8-bit
template <int BITS, class Frag>
__device__ __forceinline__ void tile_group_f(Frag frag, const __half *sc, const __half *bi, int G,
                                             const uint4 *xs, const float *xsum, int ncol, int g,
                                             int gid, int tig, float (&acc)[4])
{
    uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
    if (gid < ncol) {
        x0 = xs[((g * 2 + 0) * ncol + gid) * 4 + tig];
        x1 = xs[((g * 2 + 1) * ncol + gid) * 4 + tig];
    }
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    if (BITS == 4) {
        const uint2 wa = *reinterpret_cast<const uint2 *>(frag(gid));
        const uint2 wb = *reinterpret_cast<const uint2 *>(frag(gid + 8));
        uint32_t pa[8], pb[8];
        dequant4_word(wa.x, pa);
        dequant4_word(wa.y, pa + 4);
        dequant4_word(wb.x, pb);
        dequant4_word(wb.y, pb + 4);
        mma_16816(c, pa[0], pb[0], pa[1], pb[1], x0.x, x0.y);
        mma_16816(c, pa[2], pb[2], pa[3], pb[3], x0.z, x0.w);
        mma_16816(c, pa[4], pb[4], pa[5], pb[5], x1.x, x1.y);
        mma_16816(c, pa[6], pb[6], pa[7], pb[7], x1.z, x1.w);
    } else {
        const uint4 wa = *reinterpret_cast<const uint4 *>(frag(gid));
        const uint4 wb = *reinterpret_cast<const uint4 *>(frag(gid + 8));
        uint32_t pa[2], pb[2];
        dequant8_word(wa.x, pa);
        dequant8_word(wb.x, pb);
        mma_16816(c, pa[0], pb[0], pa[1], pb[1], x0.x, x0.y);
        dequant8_word(wa.y, pa);
        dequant8_word(wb.y, pb);
        mma_16816(c, pa[0], pb[0], pa[1], pb[1], x0.z, x0.w);
        dequant8_word(wa.z, pa);
        dequant8_word(wb.z, pb);
        mma_16816(c, pa[0], pb[0], pa[1], pb[1], x1.x, x1.y);
        dequant8_word(wa.w, pa);
        dequant8_word(wb.w, pb);
        mma_16816(c, pa[0], pb[0], pa[1], pb[1], x1.z, x1.w);
    }
    const float s_lo = __half2float(sc[gid * G + g]);
    const float s_hi = __half2float(sc[(gid + 8) * G + g]);
    const float b_lo = __half2float(bi[gid * G + g]);
    const float b_hi = __half2float(bi[(gid + 8) * G + g]);
    const float2 X = *reinterpret_cast<const float2 *>(xsum + g * 8 + 2 * tig);
    acc[0] = fmaf(s_lo, c[0], fmaf(b_lo, X.x, acc[0]));
    acc[1] = fmaf(s_lo, c[1], fmaf(b_lo, X.y, acc[1]));
    acc[2] = fmaf(s_hi, c[2], fmaf(b_hi, X.x, acc[2]));
    acc[3] = fmaf(s_hi, c[3], fmaf(b_hi, X.y, acc[3]));
}

// Row-padded tile: row r of the codes at tile + r*stride (words).
template <int BITS>
__device__ __forceinline__ void tile_group(const uint32_t *tile, int stride, const __half *sc,
                                           const __half *bi, int G, const uint4 *xs,
                                           const float *xsum, int ncol, int g, int gid, int tig,
                                           float (&acc)[4])
{
    const int col = BITS == 4 ? g * 8 + 2 * tig : g * 16 + 4 * tig;
    tile_group_f<BITS>([&](int r) { return tile + r * stride + col; }, sc, bi, G, xs, xsum, ncol,
                       g, gid, tig, acc);
}

// Tile as written by a 3-D TMA tensor copy with 128-byte swizzling (box = 32
// words x R rows x C chunks of 128 bytes, chunk-major, chunk_bytes = R*128):
// the 16-byte unit u of row r, chunk c sits at byte
// c*chunk_bytes + r*128 + 16*(u ^ (r & 7)).  The eight rows of a fragment land
// on eight different bank quads, so the fragment loads are conflict-free
// without row padding.
template <int BITS>
__device__ __forceinline__ const void *swz128_frag(const unsigned char *tile, int chunk_bytes, int r,
                                                   int g, int tig)
{
    if (BITS == 4) {
        const int u = (2 * (g & 3) + (tig >> 1)) ^ (r & 7);
        return tile + (g >> 2) * chunk_bytes + r * 128 + u * 16 + (tig & 1) * 8;
    }
    const int u = (4 * (g & 1) + tig) ^ (r & 7);
    return tile + (g >> 1) * chunk_bytes + r * 128 + u * 16;
}

// Subnormal-code group product of a 16-row tile (rows gid, gid+8 from wa, wb;
// x fragments in the order of xperm(kPermS4, .) for 4-bit, xperm(8, .) for
// 8-bit): returns sum_k q x per C element, scaled by 2^-20 (4-bit) or 2^-22
// (8-bit).  The four products of the group are added in one accumulator
// chain, the first into a fresh accumulator: fewer instructions than two
// chains joined by fp32 adds (measured faster in every caller, which all keep
// enough independent groups in flight to hide the longer chain).
__device__ __forceinline__ void mma_group_s4_1(float (&r)[4], uint2 wa, uint2 wb, uint4 x0, uint4 x1)
{
    uint32_t pa[8], pb[8];
    dequant4s_word(wa.x, pa);
    dequant4s_word(wa.y, pa + 4);
    dequant4s_word(wb.x, pb);
    dequant4s_word(wb.y, pb + 4);
    mma_16816_z(r, pa[0], pb[0], pa[2], pb[2], x0.x, x0.y);
    mma_16816(r, pa[1], pb[1], pa[3], pb[3], x1.x, x1.y);
    mma_16816(r, pa[4], pb[4], pa[6], pb[6], x0.z, x0.w);
    mma_16816(r, pa[5], pb[5], pa[7], pb[7], x1.z, x1.w);
}
__device__ __forceinline__ void mma_group_s8_1(float (&r)[4], uint4 wa, uint4 wb, uint4 x0, uint4 x1)
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
    mma_16816_z(r, pa[0], pb[0], pa[1], pb[1], x0.x, x0.y);
    mma_16816(r, pa[2], pb[2], pa[3], pb[3], x0.z, x0.w);
    mma_16816(r, pa[4], pb[4], pa[5], pb[5], x1.x, x1.y);
    mma_16816(r, pa[6], pb[6], pa[7], pb[7], x1.z, x1.w);
}
// The same products with an activation held as an fp16 (hi, lo) pair: the
// codes are dequantised once and the result is that of mma_group_s4_1 /
// mma_group_s8_1 applied to hi + lo.  The lo products (about 2^-11 of the hi
// ones) accumulate in their own registers and meet the hi sums only in an
// fp32 add: a B200 probe of mma.sync measured twice the error (relative to
// sum |a b|) when they were chained into the hi accumulator instead.
__device__ __forceinline__ void mma_group_s4_hilo(float (&r)[4], uint2 wa, uint2 wb, uint4 h0,
                                                  uint4 h1, uint4 l0, uint4 l1)
{
    uint32_t pa[8], pb[8];
    dequant4s_word(wa.x, pa);
    dequant4s_word(wa.y, pa + 4);
    dequant4s_word(wb.x, pb);
    dequant4s_word(wb.y, pb + 4);
    float c[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
    float cl[4] = {0.f, 0.f, 0.f, 0.f}, el[4] = {0.f, 0.f, 0.f, 0.f};
    mma_16816(c, pa[0], pb[0], pa[2], pb[2], h0.x, h0.y);
    mma_16816(e, pa[1], pb[1], pa[3], pb[3], h1.x, h1.y);
    mma_16816(c, pa[4], pb[4], pa[6], pb[6], h0.z, h0.w);
    mma_16816(e, pa[5], pb[5], pa[7], pb[7], h1.z, h1.w);
    mma_16816(cl, pa[0], pb[0], pa[2], pb[2], l0.x, l0.y);
    mma_16816(el, pa[1], pb[1], pa[3], pb[3], l1.x, l1.y);
    mma_16816(cl, pa[4], pb[4], pa[6], pb[6], l0.z, l0.w);
    mma_16816(el, pa[5], pb[5], pa[7], pb[7], l1.z, l1.w);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        r[i] = (c[i] + e[i]) + (cl[i] + el[i]);
}
__device__ __forceinline__ void mma_group_s8_hilo(float (&r)[4], uint4 wa, uint4 wb, uint4 h0,
                                                  uint4 h1, uint4 l0, uint4 l1)
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
    float c[4] = {0.f, 0.f, 0.f, 0.f}, d[4] = {0.f, 0.f, 0.f, 0.f};
    float cl[4] = {0.f, 0.f, 0.f, 0.f}, dl[4] = {0.f, 0.f, 0.f, 0.f};
    mma_16816(c, pa[0], pb[0], pa[1], pb[1], h0.x, h0.y);
    mma_16816(d, pa[2], pb[2], pa[3], pb[3], h0.z, h0.w);
    mma_16816(c, pa[4], pb[4], pa[5], pb[5], h1.x, h1.y);
    mma_16816(d, pa[6], pb[6], pa[7], pb[7], h1.z, h1.w);
    mma_16816(cl, pa[0], pb[0], pa[1], pb[1], l0.x, l0.y);
    mma_16816(dl, pa[2], pb[2], pa[3], pb[3], l0.z, l0.w);
    mma_16816(cl, pa[4], pb[4], pa[5], pb[5], l1.x, l1.y);
    mma_16816(dl, pa[6], pb[6], pa[7], pb[7], l1.z, l1.w);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        r[i] = (c[i] + d[i]) + (cl[i] + dl[i]);
}

// Smem row stride (in 32-bit words) for a tile of `cols` inputs so that the
// fragment loads of tile_group are free of bank conflicts: the stride must be
// 8 or 24 (mod 32) words for 4-bit (8-byte loads by 16 lanes) and 16 (mod 32)
// for 8-bit (16-byte loads by 8 lanes).
__host__ __device__ __forceinline__ int tile_stride_words(int cols, int bits)
{
    int w = cols * bits / 32;
    if (bits == 4) {
        while ((w & 31) != 8 && (w & 31) != 24)
            w += 8;
    } else {
        while ((w & 31) != 16)
            w += 16;
    }
    return w;
}

// Stage `nvec` independent inputs, each [ncol][G*64] (read through
// `load(v, n, k)` returning the fp32 value of an fp16 number), into the
// fragment layout used by tile_group, plus per-group column sums.  Vector v
// uses xs + v*G*2*ncol*4 and xsum + v*G*8.  The 8 fragment slots of one
// (group, column) sit in 8 consecutive lanes; each lane loads its 8 values at
// once and the group sum is reduced with shuffles, so no thread walks a group
// serially.  All `nthreads` threads (a multiple of 32) starting at `tid` must
// take part.  With xsum == nullptr only the fragments are written.
template <int BITS, class Load>
__device__ __forceinline__ void stage_x(uint4 *xs, float *xsum, int G, int ncol, int nvec, Load load,
                                        int tid, int nthreads)
{
    const int per_vec = G * ncol * 8;
    const int total = nvec * per_vec;
    for (int base = 0; base < total; base += nthreads) {
        const int t = base + tid;
        float part = 0.f;
        int v = 0, g = 0, n = 0;
        if (t < total) {
            v = t / per_vec;
            const int r = t - v * per_vec;
            const int gn = r >> 3;
            const int h = (r >> 2) & 1, tig = r & 3;
            g = gn / ncol;
            n = gn - g * ncol;
            const int kbase = g * kGroup + 16 * tig;
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                f[i] = load(v, n, kbase + xperm(BITS, 8 * h + i));
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __half2 hh = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
                w[i] = h2_as_u32(hh);
                const float2 back = __half22float2(hh);
                part += back.x + back.y;
            }
            xs[(size_t)v * G * 2 * ncol * 4 + ((g * 2 + h) * ncol + n) * 4 + tig] =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        part += __shfl_xor_sync(0xffffffffu, part, 4);
        if (xsum && t < total && (t & 7) == 0)
            xsum[(size_t)v * G * 8 + g * 8 + n] = part;
    }
    // columns ncol..7 of the sums are zero
    if (xsum)
        for (int t = tid; t < nvec * G * 8; t += nthreads)
            if ((t & 7) >= ncol)
                xsum[t] = 0.f;
}

// Stage x [ncol][G*64] (fp16, global, 16-byte aligned rows) into the fragment
// layout of tile_group / mma_group_s*, one thread per (column, group): the
// thread reads the group's 128 bytes with eight 16-byte loads, writes its
// eight permuted 16-byte fragment slots and the group sum.  KIND as xperm.
// All `nthreads` threads starting at `tid` take part.  The sum of (column n,
// group g) goes to xsum[g * sum_stride + n]; with sum_stride 8 (the
// tile_group layout) columns ncol..7 of the sums are zeroed.
// With ROT, each 32-input block is first rotated: x' = H_32 (D x) / sqrt(32)
// (Sylvester Hadamard, D = diag(+-1) from bit i of signs[k / 32], set = -1),
// computed in fp32 by the thread that owns the block, and kept as an fp16
// pair: hi = fp16(x') in xs, lo = fp16(x' - hi) in xs_lo (same layout); the
// sums are those of hi + lo.  (fp16 x' alone would add up to 2^-12 relative
// error per input, far more than the products of the exact codes.)
template <int KIND, bool ROT = false>
__device__ __forceinline__ void stage_x_groups(uint4 *xs, float *xsum, int G, int ncol,
                                               const __half *x, int K, int tid, int nthreads,
                                               int sum_stride = 8,
                                               const uint32_t *signs = nullptr,
                                               uint4 *xs_lo = nullptr)
{
    for (int t = tid; t < ncol * G; t += nthreads) {
        const int n = t / G, g = t - n * G;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)n * K + (size_t)g * kGroup);
        float sum = 0.f;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {   // the group's two 32-input blocks
            uint4 raw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                raw[i] = __ldg(src + 4 * blk + i);
            if (ROT) {
                float v[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 f = __half22float2(reinterpret_cast<const __half2 *>(raw)[i]);
                    v[2 * i] = f.x;
                    v[2 * i + 1] = f.y;
                }
                const uint32_t sg = __ldg(signs + 2 * g + blk);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if ((sg >> i) & 1u)
                        v[i] = -v[i];
#pragma unroll
                for (int h = 1; h < 32; h <<= 1)   // Walsh-Hadamard butterflies
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if ((i & h) == 0) {
                            const float a = v[i], b = v[i + h];
                            v[i] = a + b;
                            v[i + h] = a - b;
                        }
                const float inv = 0.17677669529663687f;   // 1 / sqrt(32)
                uint4 rlo[4];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float a = v[2 * i] * inv, b = v[2 * i + 1] * inv;
                    const __half2 hh = __floats2half2_rn(a, b);
                    const float2 back = __half22float2(hh);
                    reinterpret_cast<__half2 *>(raw)[i] = hh;
                    reinterpret_cast<__half2 *>(rlo)[i] = __floats2half2_rn(a - back.x, b - back.y);
                }
                const __half *lv = reinterpret_cast<const __half *>(rlo);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 f = __half22float2(reinterpret_cast<const __half2 *>(rlo)[i]);
                    sum += f.x + f.y;
                }
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int tl = 0; tl < 2; ++tl) {
                        uint32_t w[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const __half lo = lv[16 * tl + xperm(KIND, 8 * h + 2 * i)];
                            const __half hi = lv[16 * tl + xperm(KIND, 8 * h + 2 * i + 1)];
                            w[i] = h2_as_u32(__halves2half2(lo, hi));
                        }
                        xs_lo[((g * 2 + h) * ncol + n) * 4 + 2 * blk + tl] =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
            }
            const __half *hv = reinterpret_cast<const __half *>(raw);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float2 f = __half22float2(reinterpret_cast<const __half2 *>(raw)[i]);
                sum += f.x + f.y;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int tl = 0; tl < 2; ++tl) {   // fragment slots tig = 2 blk + tl
                    uint32_t w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __half lo = hv[16 * tl + xperm(KIND, 8 * h + 2 * i)];
                        const __half hi = hv[16 * tl + xperm(KIND, 8 * h + 2 * i + 1)];
                        w[i] = h2_as_u32(__halves2half2(lo, hi));
                    }
                    xs[((g * 2 + h) * ncol + n) * 4 + 2 * blk + tl] = make_uint4(w[0], w[1], w[2], w[3]);
                }
        }
        xsum[g * sum_stride + n] = sum;
    }
    if (sum_stride == 8)
        for (int t = tid; t < G * 8; t += nthreads)
            if ((t & 7) >= ncol)
                xsum[t] = 0.f;
}

// Position i (0..15) of the x order xperm(kPermS4, .) that holds input p of a
// 16-input block: the inverse permutation of xperm_s4.
__host__ __device__ __forceinline__ int xperm_s4_inv(int p)
{
    return ((p & 1) << 3) | (((p >> 3) & 1) << 2) | (((p >> 1) & 1) << 1) | ((p >> 2) & 1);
}

}  // namespace qmoe
