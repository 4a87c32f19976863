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
// B200 design.  A decode layer is a chain (x -> router -> top-k -> gate/up ->
// h -> down -> y -> next layer) over ~30 MB of weights, so the kernel is built
// to pay as few grid-wide hand-offs per layer as possible:
//
//   * Clusters of 8 CTAs (one CTA per SM).  Each CTA of a cluster holds E/8
//     router rows in shared memory (loaded during the previous layer) and
//     computes their logits; the logits meet in every CTA of the cluster
//     through distributed shared memory (st.async stores that complete their
//     bytes on the receiver's mbarrier), so each CTA takes the top-k itself
//     without a grid-wide exchange.
//   * Work is cut into units of (expert, 64 consecutive intermediate
//     indices).  A unit belongs to ONE cluster: CTA r of the cluster computes
//     the gate/up rows 8r..8r+7 of the unit and SwiGLU, sends its eight h
//     values (as fp16 hi/lo pairs) to the other 7 CTAs of the cluster by
//     st.async (their bytes complete the receiver's mbarrier of the unit);
//     each CTA then multiplies its own H/8 rows of the down projection by the
//     unit's 64 h values.  The gate/up -> down dependency never leaves the
//     cluster.
//   * Each CTA adds its weighted down rows of all its units in shared memory
//     and then into an fp32 layer accumulator with one vector reduction per
//     four rows; the thread that issued it then increments a grid-wide
//     arrival counter with release semantics, so no CTA-wide barrier or fence
//     sits between the last work item and the arrival.  When the counter
//     shows every reduction of the layer, the layer's output is complete and
//     the next layer starts (its input would be this layer's output in a
//     real model).
//   * One producer thread streams the CTA's weights as ~12.7 KB bulk copies
//     (every copy is one contiguous block of the packed layer) through a
//     shared-memory ring, in the order the consumers use them: the shared
//     expert's units need no routing and are fetched a layer ahead; the
//     routed units are fetched expert by expert as the top-k rounds of the
//     first exchange warp publish them.
//   * 16 consumer warps in 4 groups; work item k of a layer goes to group
//     k % 4 (gate/up items: the 4 warps split K; down items: the 4 warps
//     split the rows).  Consumers hand partial sums over through shared
//     memory and an mbarrier and move on: an exchange warp adds the router
//     partials and sends the CTA's logits to the cluster, and adds each
//     unit's gate/up partials, applies SwiGLU and sends the h values (four
//     8-byte st.async stores and one 4-byte one per destination CTA; no
//     release fence or remote arrive is needed, the bytes themselves complete
//     the receiver's barrier), so no consumer group waits on that traffic.
//
// The fp32 atomics make the last bits of a layer output depend on the order
// in which clusters finish; routing, h and every per-CTA sum do not.
// Every wait is bounded; a timeout flags QMOE_DEV_TIMEOUT, raises an abort
// word that stops every other wait, and lets the kernel drain its copies and
// return.
#include "common.cuh"
#include "kernels.h"

namespace qmoe {

namespace {

constexpr int DC_CLUSTER = 8;                 // CTAs per cluster
constexpr int DC_GROUPS = 4;                  // consumer groups
constexpr int DC_GW = 4;                      // warps per group
constexpr int DC_CW = DC_GROUPS * DC_GW;      // consumer warps
constexpr int DC_CT = DC_CW * 32;             // consumer threads
constexpr int DC_PW = DC_CW;                  // producer warp
constexpr int DC_XW = DC_CW + 1;              // first exchange warp
constexpr int DC_XN = 3;                      // exchange warps (20 warps in all: 96 registers)
constexpr int DC_THREADS = DC_CT + 32 * (1 + DC_XN);   // + producer and exchange warps
constexpr int DC_MAX_UNITS = 16;              // units per cluster and layer
constexpr int DC_MAX_STAGES = 16;
constexpr int BAR_ALL = 1;                    // named barrier of all consumer threads

// control words of the workspace
enum { C_ARRIVE = 0, C_ABORT, C_EXIT, C_WORDS };

// ------------------------------------------------------- packed layout --
// One packed layer (every block a multiple of 128 bytes):
//   router blocks, one per cluster rank r: codes [Rr][H] (8-bit, rows
//     Rr*r .. Rr*r+Rr-1 of the router, Rr = E/8; 16-byte chunk c of row i
//     stored at chunk swz(c, i)) + (scale, bias) half2 [Rr][H/64]
//   then for each expert e = 0..E (e == E: the shared expert), for each
//   group g of 64 intermediate indices, for each rank r, three copies of
//   4.5 H bytes each:
//     gate half: codes [8][H/2] (gate rows 64g+8r .. +7, chunk c of row i at
//                swz(c, i)) + (scale, bias) half2 [8][H/64]
//     up half:   the same rows of the up projection
//     down:      codes [H/8][32 bytes] (rows H/8*r .. +H/8-1 of the down
//                projection, inputs 64g .. 64g+63) + (scale, bias) half2 [H/8]
__host__ __device__ __forceinline__ int swz_chunk(int c, int r) { return (c & ~7) | ((c ^ r) & 7); }

struct PackDims {
    int E, H, I, GH, GI, Rr, Hc;
    size_t rb_codes, rb_bytes, router_bytes, st_codes, st_bytes, unit_bytes, exp_bytes, total;
};

__host__ __device__ inline PackDims pack_dims(int E, int H, int I)
{
    PackDims p;
    p.E = E;
    p.H = H;
    p.I = I;
    p.GH = H / kGroup;
    p.GI = I / kGroup;
    p.Rr = E / DC_CLUSTER;
    p.Hc = H / DC_CLUSTER;
    p.rb_codes = (size_t)p.Rr * H;
    p.rb_bytes = p.rb_codes + (size_t)p.Rr * p.GH * 4;
    p.router_bytes = (size_t)DC_CLUSTER * p.rb_bytes;
    p.st_codes = (size_t)4 * H;               // 8 rows x H/2 bytes = H/8 rows x 32 bytes
    p.st_bytes = p.st_codes + (size_t)H / 2;  // + 8 x H/64 or H/8 (scale, bias) words
    p.unit_bytes = (size_t)DC_CLUSTER * 3 * p.st_bytes;
    p.exp_bytes = (size_t)p.GI * p.unit_bytes;
    p.total = p.router_bytes + (size_t)(E + 1) * p.exp_bytes;
    return p;
}

__host__ __device__ inline size_t pack_router_off(const PackDims &p, int rank)
{
    return (size_t)rank * p.rb_bytes;
}
// kind: 0 gate half, 1 up half, 2 down
__host__ __device__ inline size_t pack_copy_off(const PackDims &p, int e, int g, int rank, int kind)
{
    return p.router_bytes + (size_t)e * p.exp_bytes + (size_t)g * p.unit_bytes +
           (size_t)(rank * 3 + kind) * p.st_bytes;
}

// ------------------------------------------------------- unit schedule --
// Units of a layer: routed units v = 0 .. top_k*GI-1 (slot v / GI, group
// v % GI), then shared units v = top_k*GI .. (top_k+1)*GI-1.  Cluster c owns
// v = c, c + NC, c + 2 NC, ...  Its units get local slots: the shared ones
// first (s = 0 .. ns-1), then the routed ones (s = ns .. nu-1).
struct Units {
    int nu, ns, nr;
};

__host__ __device__ inline Units cluster_units(int c, int NC, int top_k, int GI)
{
    Units u;
    const int Ur = top_k * GI, U = Ur + GI;
    u.nu = U > c ? (U - c + NC - 1) / NC : 0;
    u.nr = Ur > c ? (Ur - c + NC - 1) / NC : 0;
    u.ns = u.nu - u.nr;
    return u;
}

// expert-relative (slot j, group g) of local unit slot s; j == top_k: shared
__device__ __forceinline__ void unit_of(int s, const Units &u, int c, int NC, int top_k, int GI,
                                        int *j, int *g)
{
    const int m = s < u.ns ? u.nr + s : s - u.ns;
    const int v = c + m * NC;
    *j = v / GI;   // top_k for the shared units
    *g = v - *j * GI;
}

// ------------------------------------------------------- shared memory --
struct DcLayout {
    size_t router_off, xs4_off, xs8_off, xsum_off, logit_off, topk_off, unit_off, hfrag_off,
        hsum_off, ypart_off, red_off, gupart_off, bar_off, arm_off, ring_off, total;
};

// barriers (indices into the barrier array after the ring's full/empty pairs)
enum {
    DB_RFULL = 0,        // router rows of the layer landed
    DB_REMPTY,           // router rows consumed
    DB_TOPK,             // top-k of the layer in s_idx / s_wt
    DB_LOGIT,            // the cluster's logits (one arrival per CTA)
    DB_RED,              // router partials of every consumer warp
    DB_H,                // + unit: the unit's h from every CTA of the cluster
    DB_GU = DB_H + DC_MAX_UNITS,   // + unit: gate/up partials of the unit's warps
    DB_ROUND = DB_GU + DC_MAX_UNITS,   // + j: the j-th expert of the top-k is known
    DB_COUNT = DB_ROUND + 16
};

__host__ __device__ inline size_t dc_take(size_t *off, size_t n, size_t align)
{
    *off = (*off + align - 1) & ~(align - 1);
    const size_t o = *off;
    *off += n;
    return o;
}

__host__ __device__ inline DcLayout dc_layout(const PackDims &p, int NS)
{
    DcLayout L;
    size_t off = 0;
    L.router_off = dc_take(&off, p.rb_bytes, 128);
    L.xs4_off = dc_take(&off, (size_t)p.GH * 2 * 4 * 16, 16);
    L.xs8_off = dc_take(&off, (size_t)p.GH * 2 * 4 * 16, 16);
    L.xsum_off = dc_take(&off, (size_t)p.GH * 8 * 4, 16);
    L.logit_off = dc_take(&off, (size_t)p.E * 4, 16);
    L.topk_off = dc_take(&off, 32 * 4 * 2, 16);
    L.unit_off = dc_take(&off, (size_t)2 * DC_MAX_UNITS * 4, 16);   // (slot j, group g) per unit
    L.hfrag_off = dc_take(&off, (size_t)DC_MAX_UNITS * 256, 16);
    L.hsum_off = dc_take(&off, (size_t)DC_MAX_UNITS * DC_CLUSTER * 4, 16);
    L.ypart_off = dc_take(&off, (size_t)DC_GROUPS * p.Hc * 4, 16);
    L.red_off = dc_take(&off, (size_t)DC_CW * 16 * 4, 16);   // router partials
    // gate/up partials [unit][warp of the group][gate 8 | up 8]
    L.gupart_off = dc_take(&off, (size_t)DC_MAX_UNITS * DC_GW * 16 * 4, 16);
    L.bar_off = dc_take(&off, (size_t)(2 * DC_MAX_STAGES + DB_COUNT) * 8, 8);
    L.arm_off = dc_take(&off, (size_t)DC_MAX_STAGES * 4, 16);   // sequence each slot holds
    L.ring_off = dc_take(&off, (size_t)NS * p.st_bytes, 128);
    L.total = off;
    return L;
}

// -------------------------------------------------------- cluster PTX --
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_index()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// every thread of every CTA of the cluster
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_rank(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v2u32(uint32_t addr, uint32_t a, uint32_t b)
{
    asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b)
                 : "memory");
}
// stores into a CTA of the cluster that complete `bytes` of the transaction
// count of an mbarrier in that CTA (the receiver's wait then sees the data):
// no release fence and no separate remote arrive on the sender's side
__device__ __forceinline__ void st_async_v4(uint32_t addr, float4 v, uint32_t mbar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
                 "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)), "r"(__float_as_uint(v.z)),
                 "r"(__float_as_uint(v.w)), "r"(mbar)
                 : "memory");
}
__device__ __forceinline__ void st_async_b32(uint32_t addr, uint32_t v, uint32_t mbar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(addr), "r"(v),
                 "r"(mbar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t addr, uint32_t a, uint32_t b, uint32_t mbar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(addr),
                 "r"(a), "r"(b), "r"(mbar)
                 : "memory");
}
// fire-and-forget vector add (no value returned, so the thread does not wait)
__device__ __forceinline__ void red_add_v4(float4 *p, float4 v)
{
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}
// increment with release semantics at GPU scope: this thread's earlier
// writes (and reductions) are visible to whoever acquires the new value
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// bulk copy without a cache hint (router rows: read by every cluster, so
// they should stay in L2 for the others)
__device__ __forceinline__ void bulk_g2s_plain(void *smem_dst, const void *gsrc, uint32_t bytes,
                                               uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// bring `bytes` (a multiple of 16, 16-byte aligned) into L2
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ---------------------------------------------------- bounded waiting --
// All waits give up after a.wait_ns (flagging QMOE_DEV_TIMEOUT and raising
// the abort word) or as soon as another CTA raised the abort word.
__device__ __noinline__ bool wait_slow(const DecodeArgs &a, uint64_t *bar, uint32_t parity,
                                       bool cluster_scope)
{
    unsigned *abort = a.ws.ctl + C_ABORT;
    const unsigned long long t0 = global_timer_ns();
    for (unsigned n = 1;; ++n) {
        if (cluster_scope ? mbar_try_wait_acq_cluster(bar, parity) : mbar_try_wait(bar, parity))
            return true;
        if ((n & 15u) == 0u) {
            if (ld_acquire_u32(abort) != 0u)
                return false;
            if (global_timer_ns() - t0 > a.wait_ns) {
                atomicExch(abort, 1u);
                flag_status(a.status, QMOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar(const DecodeArgs &a, uint64_t *bar, uint32_t parity)
{
    return mbar_try_wait(bar, parity) || wait_slow(a, bar, parity, false);
}
__device__ __forceinline__ bool wait_bar_cluster(const DecodeArgs &a, uint64_t *bar,
                                                 uint32_t parity)
{
    return mbar_try_wait_acq_cluster(bar, parity) || wait_slow(a, bar, parity, true);
}

// Bounded spin until *p >= target (global counter of the grid).
__device__ __noinline__ bool spin_until(const DecodeArgs &a, const unsigned *p, unsigned target)
{
    unsigned *abort = a.ws.ctl + C_ABORT;
    const unsigned long long t0 = global_timer_ns();
    unsigned polls = 0;
    while (ld_acquire_u32(p) < target) {
        __nanosleep(32);   // keep the polled line from crowding out the arrivals
        if ((++polls & 31u) == 0u) {
            if (ld_acquire_u32(abort) != 0u)
                return false;
            if (global_timer_ns() - t0 > a.wait_ns) {
                atomicExch(abort, 1u);
                flag_status(a.status, QMOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
    return true;
}

// Bounded wait until a ring slot has been armed for sequence `sq`.
__device__ __noinline__ bool wait_arm_slow(const DecodeArgs &a, const volatile int *arm, int sq)
{
    unsigned *abort = a.ws.ctl + C_ABORT;
    const unsigned long long t0 = global_timer_ns();
    for (unsigned n = 1;; ++n) {
        if (*arm == sq)
            return true;
        __nanosleep(20);
        if ((n & 63u) == 0u) {
            if (ld_acquire_u32(abort) != 0u)
                return false;
            if (global_timer_ns() - t0 > a.wait_ns) {
                atomicExch(abort, 1u);
                flag_status(a.status, QMOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_arm(const DecodeArgs &a, const volatile int *arm, int sq)
{
    return *arm == sq || wait_arm_slow(a, arm, sq);
}

// ------------------------------------------------------------ helpers --
__device__ __forceinline__ float2 sb_word(const unsigned char *p)
{
    return __half22float2(*reinterpret_cast<const __half2 *>(p));   // (scale, bias)
}

// The h of a unit (64 intermediate indices k, fp16 hi and lo columns) sits in
// hfrag[unit] as the down projection's B fragments [hh][col][tig][8], in the x
// order of mma_group_s4_1: index k = 16 tig + xperm_s4(8 hh + e) at slot
// ((hh * 2 + col) * 4 + tig) * 8 + e.

// ------------------------------------------------------------------ kernel --
__global__ void __cluster_dims__(DC_CLUSTER, 1, 1) __launch_bounds__(DC_THREADS, 1)
    moe_decode_kernel(const __grid_constant__ DecodeArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const PackDims P = pack_dims(a.E, a.H, a.I);
    const DcLayout L = dc_layout(P, a.NS);
    unsigned char *rbuf = smem + L.router_off;
    uint4 *xs4 = reinterpret_cast<uint4 *>(smem + L.xs4_off);
    uint4 *xs8 = reinterpret_cast<uint4 *>(smem + L.xs8_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    // 16 zero bytes (group 0's unused sum columns 4..7), read by lanes whose
    // B fragment column is not x
    const uint4 *xzero = reinterpret_cast<const uint4 *>(xsum + 4);
    float *s_logit = reinterpret_cast<float *>(smem + L.logit_off);
    int *s_idx = reinterpret_cast<int *>(smem + L.topk_off);
    float *s_wt = reinterpret_cast<float *>(smem + L.topk_off + 32 * 4);
    int *s_uj = reinterpret_cast<int *>(smem + L.unit_off);   // unit -> expert slot j (K: shared)
    int *s_ug = s_uj + DC_MAX_UNITS;                          // unit -> group of 64 indices
    __half *hfrag = reinterpret_cast<__half *>(smem + L.hfrag_off);   // [unit][128]
    float *hsum = reinterpret_cast<float *>(smem + L.hsum_off);       // [unit][8]
    float *ypart = reinterpret_cast<float *>(smem + L.ypart_off);     // [group][Hc]
    float *red = reinterpret_cast<float *>(smem + L.red_off);         // [warp][16]
    float *gupart = reinterpret_cast<float *>(smem + L.gupart_off);   // [unit][wq][16]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *full = bars, *empty = bars + DC_MAX_STAGES;
    // ring sequence number each slot has been armed for (written by the
    // producer before the copy): a consumer first sees its own sequence
    // there, so it never takes an older phase of the slot's full barrier for
    // its own when it runs more than one use of the slot ahead
    volatile int *s_arm = reinterpret_cast<volatile int *>(smem + L.arm_off);
    uint64_t *db = bars + 2 * DC_MAX_STAGES;
    uint64_t *rfull = db + DB_RFULL, *rempty = db + DB_REMPTY, *topk_bar = db + DB_TOPK,
             *logit_bar = db + DB_LOGIT, *red_bar = db + DB_RED, *hbar = db + DB_H,
             *gubar = db + DB_GU, *round_bar = db + DB_ROUND;
    unsigned char *ring = smem + L.ring_off;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank();
    const int cl = (int)cluster_index(), NC = (int)cluster_count();
    const int G = (int)gridDim.x;
    const int K = a.top_k, NS = a.NS;
    const Units U = cluster_units(cl, NC, K, P.GI);
    unsigned *ctl = a.ws.ctl;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], DC_GW);   // one arrival per warp of the consuming group
            s_arm[s] = -1;
        }
        mbar_init(rfull, 1);
        mbar_init(rempty, 1);
        mbar_init(topk_bar, 1);
        mbar_init(logit_bar, 1);   // the exchange warp's expect; the bytes by st.async
        mbar_init(red_bar, DC_CW);
        for (int s = 0; s < DC_MAX_UNITS; ++s) {
            mbar_init(&hbar[s], 1);   // the local exchange warp; the others' bytes by st.async
            mbar_init(&gubar[s], DC_GW);
        }
        for (int j = 0; j < 16; ++j)
            mbar_init(&round_bar[j], 1);
        mbar_init_fence();
    }
    // columns 1..7 of the x group sums stay zero (one input column)
    for (int t = threadIdx.x; t < P.GH * 8; t += blockDim.x)
        xsum[t] = 0.f;
    // the cluster's units are the same in every layer
    if (threadIdx.x < U.nu) {
        int j, g;
        unit_of(threadIdx.x, U, cl, NC, K, P.GI, &j, &g);
        s_uj[threadIdx.x] = j;
        s_ug[threadIdx.x] = g;
    }
    // every CTA of the cluster has initialised its barriers before anyone
    // signals one remotely
    cluster_sync_all();
    // the workspace may still be in use by the previous launch on the stream
    pdl_wait();

    if (warp == DC_PW) {
        // ====================================================== producer
        const uint64_t pol = l2_evict_first_policy();
        bool ok = true;
        int seq = 0;
        auto issue_to = [&](const unsigned char *src, int st, int use, int sq) {
            if (use > 0 && ok && !wait_bar(a, &empty[st], (use - 1) & 1))
                ok = false;
            if (ok) {
                s_arm[st] = sq;
                mbar_arrive_expect_tx(&full[st], (uint32_t)P.st_bytes);
                bulk_g2s(ring + (size_t)st * P.st_bytes, src, (uint32_t)P.st_bytes, &full[st], pol);
            }
        };
        auto issue = [&](const unsigned char *src) {   // the next copy of the ring
            issue_to(src, seq % NS, seq / NS, seq);
            ++seq;
        };
        // A unit's gate and up halves are adjacent in the packed layer: one
        // copy fills both of their (adjacent) ring slots unless the pair
        // wraps around the ring.  Fewer, larger copies keep more bytes in
        // flight per copy the SM's bulk-copy engine holds at once.  The
        // second slot's full barrier is completed by a plain arrival (its
        // data is counted on the first).
        auto issue_pair = [&](const unsigned char *src) {
            const int st = seq % NS;
            if (st + 1 == NS) {
                issue(src);
                issue(src + P.st_bytes);
                return;
            }
            const int use = seq / NS;
            if (use > 0 && ok &&
                !(wait_bar(a, &empty[st], (use - 1) & 1) && wait_bar(a, &empty[st + 1], (use - 1) & 1)))
                ok = false;
            if (ok) {
                s_arm[st] = seq;
                s_arm[st + 1] = seq + 1;
                mbar_arrive_expect_tx(&full[st], (uint32_t)(2 * P.st_bytes));
                bulk_g2s(ring + (size_t)st * P.st_bytes, src, (uint32_t)(2 * P.st_bytes), &full[st], pol);
                mbar_arrive(&full[st + 1]);
            }
            seq += 2;
        };
        if (lane == 0) {   // the first layer's router rows
            mbar_arrive_expect_tx(rfull, (uint32_t)P.rb_bytes);
            bulk_g2s_plain(rbuf, static_cast<const unsigned char *>(a.layer[0]) +
                                     pack_router_off(P, rank),
                           (uint32_t)P.rb_bytes, rfull);
        }
        for (int l = 0; l < a.L; ++l) {
            const unsigned char *lp = static_cast<const unsigned char *>(a.layer[l]);
            if (lane == 0 && ok) {
                for (int s = 0; s < U.ns; ++s)     // shared gate/up
                    issue_pair(lp + pack_copy_off(P, a.E, s_ug[s], rank, 0));
                for (int s = 0; s < U.ns; ++s)     // shared down
                    issue(lp + pack_copy_off(P, a.E, s_ug[s], rank, 2));
                // the next layer's input into L2 (where a real model's previous
                // layer output would be), and its router rows once this
                // layer's are consumed
                if (l + 1 < a.L && rank == 0)
                    prefetch_l2(a.x + (size_t)(l + 1) * a.H, (uint32_t)(a.H * 2));
                if (l + 1 < a.L && ok) {
                    if (!wait_bar(a, rempty, l & 1)) {
                        ok = false;
                    } else {
                        mbar_arrive_expect_tx(rfull, (uint32_t)P.rb_bytes);
                        bulk_g2s_plain(rbuf, static_cast<const unsigned char *>(a.layer[l + 1]) +
                                                 pack_router_off(P, rank),
                                       (uint32_t)P.rb_bytes, rfull);
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            // ---- routed gate/up copies, expert by expert as the exchange
            // warp's top-k rounds finish (units come in slot order), then the
            // routed down copies once the whole top-k is known
            if (lane == 0 && ok) {
                int nxt = U.ns;
                for (int jj = 0; jj < K && nxt < U.nu && ok; ++jj) {
                    if (s_uj[nxt] != jj)
                        continue;   // no unit of this cluster belongs to the jj-th expert
                    if (!wait_bar(a, &round_bar[jj], l & 1)) {
                        ok = false;
                        break;
                    }
                    const int e = s_idx[jj];
                    for (; nxt < U.nu && s_uj[nxt] == jj; ++nxt)
                        issue_pair(lp + pack_copy_off(P, e, s_ug[nxt], rank, 0));
                }
                if (ok && !wait_bar(a, topk_bar, l & 1))
                    ok = false;
            }
            if (lane == 0 && ok)   // the routed down copies
                for (int s = U.ns; s < U.nu; ++s)
                    issue(lp + pack_copy_off(P, s_idx[s_uj[s]], s_ug[s], rank, 2));
            ok = __shfl_sync(0xffffffffu, ok, 0);
            __syncwarp();
        }
        // drain: every copy issued has landed before the CTA may exit
        if (lane == 0) {
            for (int st = 0; st < NS && st < seq; ++st) {
                const int last = seq - 1 - ((seq - 1 - st) % NS);   // last seq that used slot st
                wait_bar(a, &full[st], (last / NS) & 1);
            }
        }
        __syncwarp();
    } else if (warp >= DC_XW) {
        // ====================================================== exchange
        // Finishes what the consumer warps hand over, so that they never wait
        // on distributed-shared-memory traffic: the CTA's logits (first
        // exchange warp) and, unit by unit, SwiGLU and the unit's h, sent to
        // every CTA of the cluster (unit s by exchange warp s % DC_XN: a
        // send takes about a microsecond, so several run at once).
        const int xw = warp - DC_XW;
        const int Rr = P.Rr;
        bool ok = true;
        for (int l = 0; l < a.L && ok; ++l) {
            if (xw == 0) {
                // the other CTAs' logits of this layer (Rr from each) complete
                // the phase; this CTA's own are written in place by this warp
                if (lane == 0)
                    mbar_arrive_expect_tx(logit_bar, (uint32_t)((DC_CLUSTER - 1) * Rr * 4));
                ok = __all_sync(0xffffffffu, wait_bar(a, red_bar, l & 1));
                if (!ok)
                    break;
                if (lane == 0)
                    mbar_arrive(rempty);   // the router rows are consumed
                {
                    // row lane & 15, half of the consumer warps each
                    const int row = lane & 15, w0 = (lane >> 4) * (DC_CW / 2);
                    float v = 0.f;
#pragma unroll
                    for (int w = 0; w < DC_CW / 2; ++w)
                        v += red[(w0 + w) * 16 + row];
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    if (lane < Rr)
                        s_logit[Rr * rank + lane] = v;
                }
                __syncwarp();
                if (lane < DC_CLUSTER && lane != (int)rank) {
                    const float *mine = s_logit + Rr * rank;
                    const uint32_t tb = mapa_rank(smem_u32(mine), lane);
                    const uint32_t tbar = mapa_rank(smem_u32(logit_bar), lane);
                    if ((Rr & 3) == 0) {
                        for (int i = 0; i < Rr; i += 4)
                            st_async_v4(tb + 4 * i, *reinterpret_cast<const float4 *>(mine + i), tbar);
                    } else {
                        for (int i = 0; i < Rr; ++i)
                            st_async_b32(tb + 4 * i, __float_as_uint(mine[i]), tbar);
                    }
                }
            }
            // ---- top-k of this layer (exchange warp 0): each round's
            // winner is published at once (round_bar) so that the producer
            // streams its units while the later rounds run
            if (xw == 0) {
                ok = __all_sync(0xffffffffu, ok && wait_bar_cluster(a, logit_bar, l & 1));
                if (!ok)
                    break;
                float v[4];
                unsigned key[4];
                bool taken[4];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int e = lane + 32 * qq;
                    taken[qq] = e >= a.E;
                    v[qq] = taken[qq] ? 0.f : s_logit[e];
                    const unsigned u = __float_as_uint(v[qq]);   // order-preserving key
                    key[qq] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
                }
                const bool out0 = blockIdx.x == 0;
                if (a.logits && out0)
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        if (!taken[qq])
                            a.logits[(size_t)l * a.E + lane + 32 * qq] = v[qq];
                // each lane sorts its 4 candidates (key descending, lower
                // index first on equal keys); the warp then pops the largest
                // head K times
                unsigned hk[4];
                int hi[4];
                float hv[4];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    hk[qq] = taken[qq] ? 0u : key[qq];
                    hi[qq] = taken[qq] ? 0x7fffffff : lane + 32 * qq;
                    hv[qq] = v[qq];
                }
                auto cx = [&](int x, int y) {   // order (x, y)
                    const bool sw = hk[y] > hk[x] || (hk[y] == hk[x] && hi[y] < hi[x]);
                    if (sw) {
                        const unsigned tk = hk[x];
                        const int ti = hi[x];
                        const float tv = hv[x];
                        hk[x] = hk[y], hi[x] = hi[y], hv[x] = hv[y];
                        hk[y] = tk, hi[y] = ti, hv[y] = tv;
                    }
                };
                cx(0, 1), cx(2, 3), cx(0, 2), cx(1, 3), cx(1, 2);
                float my_v = 0.f;
                int my_i = 0;
                for (int jj = 0; jj < K; ++jj) {
                    const unsigned mk = __reduce_max_sync(0xffffffffu, hk[0]);
                    // one lane holds the maximum unless keys tie: then the
                    // lowest index among the tied heads wins
                    const unsigned tied = __ballot_sync(0xffffffffu, hk[0] == mk);
                    const int wl = __popc(tied) == 1
                                       ? __ffs(tied) - 1
                                       : (int)(__reduce_min_sync(0xffffffffu,
                                                                 (unsigned)(hk[0] == mk ? hi[0] : 0x7fffffff)) &
                                               31u);
                    const int win = __shfl_sync(0xffffffffu, hi[0], wl);
                    const float wv = __shfl_sync(0xffffffffu, hv[0], wl);
                    if (lane == wl) {   // pop the head
                        hk[0] = hk[1], hi[0] = hi[1], hv[0] = hv[1];
                        hk[1] = hk[2], hi[1] = hi[2], hv[1] = hv[2];
                        hk[2] = hk[3], hi[2] = hi[3], hv[2] = hv[3];
                        hk[3] = 0u, hi[3] = 0x7fffffff, hv[3] = 0.f;
                    }
                    if (lane == jj) {
                        my_v = wv;
                        my_i = win;
                    }
                    if (lane == 0) {
                        s_idx[jj] = (win >= 0 && win < a.E) ? win : 0;
                        mbar_arrive(&round_bar[jj]);   // release: s_idx[jj]
                    }
                }
                const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
                const float ex = lane < K ? expf(my_v - vmax) : 0.f;
                float sum = ex;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    sum += __shfl_xor_sync(0xffffffffu, sum, off);
                if (lane < K) {
                    const int ei = (my_i >= 0 && my_i < a.E) ? my_i : 0;
                    s_wt[lane] = ex / sum;
                    if (out0) {
                        if (a.idx)
                            a.idx[(size_t)l * K + lane] = ei;
                        if (a.weights)
                            a.weights[(size_t)l * K + lane] = ex / sum;
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(topk_bar);   // the down copies and items may read s_wt
            }
            for (int s = xw; s < U.nu; s += DC_XN) {
                ok = __all_sync(0xffffffffu, wait_bar(a, &gubar[s], l & 1));
                if (!ok)
                    break;
                float h = 0.f;
                if (lane < 8) {
                    float gs = 0.f, us = 0.f;
#pragma unroll
                    for (int w = 0; w < DC_GW; ++w) {
                        gs += gupart[((size_t)s * DC_GW + w) * 16 + lane];
                        us += gupart[((size_t)s * DC_GW + w) * 16 + 8 + lane];
                    }
                    h = gs / (1.f + expf(-gs)) * us;
                }
                const __half hh = __float2half_rn(h);
                const __half hl = __float2half_rn(h - __half2float(hh));
                float part = __half2float(hh) + __half2float(hl);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                const unsigned bh = __half_as_ushort(hh), bl = __half_as_ushort(hl);
                unsigned vh[8], vl[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    vh[i] = __shfl_sync(0xffffffffu, bh, i);
                    vl[i] = __shfl_sync(0xffffffffu, bl, i);
                }
                if (lane < DC_CLUSTER) {
                    // the CTA's 8 indices k = 8 rank + j sit, per (hh, column),
                    // in 4 consecutive fragment slots: j = hh + (0, 4, 2, 6);
                    // the other CTAs' copies go by st.async (36 bytes each,
                    // counted on their hbar), this CTA's own by plain stores
                    const uint32_t tb = mapa_rank(smem_u32(hfrag + (size_t)s * 128), lane);
                    const uint32_t ts = mapa_rank(smem_u32(hsum + s * DC_CLUSTER + rank), lane);
                    const uint32_t tbar = mapa_rank(smem_u32(&hbar[s]), lane);
                    const bool self = lane == (int)rank;
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int pos_hi = ((hf * 2 + 0) * 4 + (rank >> 1)) * 8 + 4 * (rank & 1);
                        const int pos_lo = ((hf * 2 + 1) * 4 + (rank >> 1)) * 8 + 4 * (rank & 1);
                        const uint32_t h0 = vh[hf] | (vh[hf + 4] << 16), h1 = vh[hf + 2] | (vh[hf + 6] << 16);
                        const uint32_t l0 = vl[hf] | (vl[hf + 4] << 16), l1 = vl[hf + 2] | (vl[hf + 6] << 16);
                        if (self) {
                            st_cluster_v2u32(tb + 2 * pos_hi, h0, h1);
                            st_cluster_v2u32(tb + 2 * pos_lo, l0, l1);
                        } else {
                            st_async_v2(tb + 2 * pos_hi, h0, h1, tbar);
                            st_async_v2(tb + 2 * pos_lo, l0, l1, tbar);
                        }
                    }
                    if (self)
                        st_cluster_f32(ts, part);
                    else
                        st_async_b32(ts, __float_as_uint(part), tbar);
                }
                // this CTA's own part is written: arrive, expecting the other
                // CTAs' bytes of this unit
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_expect_tx(&hbar[s], (uint32_t)((DC_CLUSTER - 1) * 36));
            }
        }
    } else {
        // ====================================================== consumers
        const int ctid = threadIdx.x;
        const int q = warp / DC_GW, wq = warp % DC_GW;   // group, warp within the group
        const int gid = lane >> 2, tig = lane & 3;
        const int H = a.H, GH = P.GH, Hc = P.Hc, Rr = P.Rr;
        const int nitems = 2 * U.nu;
        float *my_ypart = ypart + (size_t)q * Hc;
        bool ok = true;

        for (int t = ctid; t < DC_GROUPS * Hc; t += DC_CT)
            ypart[t] = 0.f;

        // fp32 layer output l -> fp16, this CTA's slice of rows; then zero it
        auto convert_slice = [&](int l) {
            const int per = (H + G - 1) / G;
            const int r0 = (int)blockIdx.x * per;
            const int n = r0 < H ? min(per, H - r0) : 0;
            float *acc = a.ws.y_acc + (size_t)(l & 1) * H;
            for (int t = ctid; t < n; t += DC_CT) {
                const float v = __ldcg(acc + r0 + t);
                a.y[(size_t)l * H + r0 + t] = __float2half_rn(v);
                __stcg(acc + r0 + t, 0.f);
            }
        };

        // ---------------------------------------- one gate/up work item
        // Each warp of the group takes a quarter of K; its partial sums of the
        // unit's 8 gate and 8 up rows go to gupart[slot] and the exchange warp
        // finishes the unit (SwiGLU, h to the cluster), so the group moves on
        // at once.
        auto do_gu = [&](int seq0, int slot) {   // seq0, seq0 + 1: the ring sequences
            const int sa = seq0 % NS, sb = (seq0 + 1) % NS;
            // the lanes of a warp decide together: the mma below is warp-collective
            const bool good = __all_sync(0xffffffffu, ok && wait_arm(a, s_arm + sa, seq0) &&
                                                          wait_bar(a, &full[sa], (seq0 / NS) & 1) &&
                                                          wait_arm(a, s_arm + sb, seq0 + 1) &&
                                                          wait_bar(a, &full[sb], ((seq0 + 1) / NS) & 1));
            float ag = 0.f, au = 0.f, bg = 0.f, bu = 0.f;
            if (good) {
                const unsigned char *A = ring + (size_t)sa * P.st_bytes;
                const unsigned char *B = ring + (size_t)sb * P.st_bytes;
                const unsigned char *rowA = A + (size_t)gid * (H / 2) + 8 * (tig & 1);
                const unsigned char *rowB = B + (size_t)gid * (H / 2) + 8 * (tig & 1);
                const unsigned char *sbA = A + P.st_codes + (size_t)gid * GH * 4;
                const unsigned char *sbB = B + P.st_codes + (size_t)gid * GH * 4;
                const int g0 = wq * GH / DC_GW, g1 = (wq + 1) * GH / DC_GW;
                // branch-free: column 0 of B is x (lanes gid == 0; the other
                // lanes read a zero block), and every lane does the per-group
                // scale and bias steps (only column 0, lanes tig == 0, counts)
                const int th = tig >> 1;
                const uint4 *xq = gid == 0 ? xs4 + tig : xzero;
                const int xst = gid == 0 ? 8 : 0, x1o = gid == 0 ? 4 : 0;
#pragma unroll 2
                for (int g = g0; g < g1; ++g) {
                    const int ch = ((2 * g) | th) ^ gid;   // 16-byte chunk, swizzled by row
                    const uint2 wa = *reinterpret_cast<const uint2 *>(rowA + 16 * ch);
                    const uint2 wb = *reinterpret_cast<const uint2 *>(rowB + 16 * ch);
                    const uint4 x0 = xq[g * xst], x1 = xq[g * xst + x1o];
                    float r[4];
                    mma_group_s4_1(r, wa, wb, x0, x1);
                    const float X = xsum[g * 8];
                    const float2 pa = sb_word(sbA + 4 * g), pb = sb_word(sbB + 4 * g);
                    ag = fmaf(pa.x, r[0], ag);
                    au = fmaf(pb.x, r[2], au);
                    bg = fmaf(pa.y, X, bg);
                    bu = fmaf(pb.y, X, bu);
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty[sa]);
                mbar_arrive(&empty[sb]);
            }
            float *gr = gupart + ((size_t)slot * DC_GW + wq) * 16;
            if (tig == 0) {
                gr[gid] = ag * kCode4 + bg;       // gate row gid
                gr[8 + gid] = au * kCode4 + bu;   // up row gid
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&gubar[slot]);   // release: the partials above
            if (!good)
                ok = false;
        };

        // ---------------------------------------- one down work item
        auto do_dn = [&](int seq, int slot, int j, int l) {   // seq: the ring sequence
            const int st = seq % NS;
            // the lanes of a warp decide together: the mma below is warp-collective
            bool good = __all_sync(0xffffffffu, ok && wait_arm(a, s_arm + st, seq) &&
                                                    wait_bar(a, &full[st], (seq / NS) & 1) &&
                                                    wait_bar_cluster(a, &hbar[slot], l & 1));
            float w = 1.f;
            if (good && j < K) {   // a routed unit: its router weight
                good = __all_sync(0xffffffffu, wait_bar(a, topk_bar, l & 1));
                w = s_wt[j];
            }
            if (good) {
                const unsigned char *S = ring + (size_t)st * P.st_bytes;
                const uint4 *hf = reinterpret_cast<const uint4 *>(hfrag + (size_t)slot * 128);
                uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
                if (gid < 2) {
                    x0 = hf[(0 * 2 + gid) * 4 + tig];
                    x1 = hf[(1 * 2 + gid) * 4 + tig];
                }
                float X = 0.f;
#pragma unroll
                for (int r = 0; r < DC_CLUSTER; ++r)
                    X += hsum[slot * DC_CLUSTER + r];
                const int nmt = Hc / 16;
                for (int mt = wq; mt < nmt; mt += DC_GW) {
                    const int r0 = mt * 16 + gid;
                    const uint2 wa = *reinterpret_cast<const uint2 *>(S + (size_t)r0 * 32 + 8 * tig);
                    const uint2 wb =
                        *reinterpret_cast<const uint2 *>(S + (size_t)(r0 + 8) * 32 + 8 * tig);
                    float r[4];
                    mma_group_s4_1(r, wa, wb, x0, x1);
                    const float2 pa = sb_word(S + P.st_codes + 4 * (size_t)r0);
                    const float2 pb = sb_word(S + P.st_codes + 4 * (size_t)(r0 + 8));
                    const float va = fmaf(pa.x * kCode4, r[0] + r[1], pa.y * X);
                    const float vb = fmaf(pb.x * kCode4, r[2] + r[3], pb.y * X);
                    if (tig == 0) {   // columns 0 and 1 (h hi, lo) of rows r0, r0 + 8
                        my_ypart[r0] = fmaf(w, va, my_ypart[r0]);
                        my_ypart[r0 + 8] = fmaf(w, vb, my_ypart[r0 + 8]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[st]);
            if (!good)
                ok = false;
        };

        // every consumer thread with t < Hc / 4 adds one float4 of the CTA's
        // output rows per layer and then one release increment of the
        // arrival counter: the layer is complete once the counter reaches
        // G * Hc / 4 per layer
        const unsigned nred = (unsigned)(Hc / 4);

        for (int l = 0; l < a.L; ++l) {
            // ---- the previous layer's output is complete in every CTA
            if (l > 0) {
                if (ctid == 0 && !spin_until(a, ctl + C_ARRIVE, (unsigned)l * G * nred))
                    ok = false;
                named_bar_sync(BAR_ALL, DC_CT);
            }
            // ---- x of this layer straight from memory into both fragment
            // orders: thread (g, half, tig) loads x[64 g + 16 tig .. + 15]
            {
                const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + (size_t)l * H);
                for (int t0 = 0; t0 < GH * 8; t0 += DC_CT) {
                    const int t = t0 + ctid;
                    const bool act = t < GH * 8;
                    const int g = t >> 3, hs = (t >> 2) & 1, tg = t & 3;
                    uint4 raw[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
                    if (act) {
                        raw[0] = __ldcg(xg + g * 8 + tg * 2);
                        raw[1] = __ldcg(xg + g * 8 + tg * 2 + 1);
                    }
                    const __half *xv = reinterpret_cast<const __half *>(raw);
                    uint32_t w4[4], w8[4];
                    float sum = 0.f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __half a0 = hs ? xv[xperm(kPermS4, 8 + 2 * i)] : xv[xperm(kPermS4, 2 * i)];
                        const __half a1 =
                            hs ? xv[xperm(kPermS4, 9 + 2 * i)] : xv[xperm(kPermS4, 2 * i + 1)];
                        const __half b0 = hs ? xv[xperm(8, 8 + 2 * i)] : xv[xperm(8, 2 * i)];
                        const __half b1 = hs ? xv[xperm(8, 9 + 2 * i)] : xv[xperm(8, 2 * i + 1)];
                        w4[i] = h2_as_u32(__halves2half2(a0, a1));
                        w8[i] = h2_as_u32(__halves2half2(b0, b1));
                        sum += __half2float(a0) + __half2float(a1);
                    }
                    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                    sum += __shfl_xor_sync(0xffffffffu, sum, 4);
                    if (act) {
                        xs4[(g * 2 + hs) * 4 + tg] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        xs8[(g * 2 + hs) * 4 + tg] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
                        if ((t & 7) == 0)
                            xsum[g * 8] = sum;
                    }
                }
                named_bar_sync(BAR_ALL, DC_CT);
            }
            // ---- router: this CTA's Rr rows, K split over the 16 warps
            {
                const bool good = __all_sync(0xffffffffu, ok && wait_bar(a, rfull, l & 1));
                float acc_lo = 0.f, acc_hi = 0.f, b_lo = 0.f, b_hi = 0.f;
                if (good) {
                    const int ra = gid % Rr, rb = (gid + 8) % Rr;
                    const unsigned char *rowa = rbuf + (size_t)ra * H;
                    const unsigned char *rowb = rbuf + (size_t)rb * H;
                    const unsigned char *sba = rbuf + P.rb_codes + (size_t)ra * GH * 4;
                    const unsigned char *sbb = rbuf + P.rb_codes + (size_t)rb * GH * 4;
                    const int g0 = warp * GH / DC_CW, g1 = (warp + 1) * GH / DC_CW;
                    // branch-free, as in the gate/up items
                    const uint4 *xq = gid == 0 ? xs8 + tig : xzero;
                    const int xst = gid == 0 ? 8 : 0, x1o = gid == 0 ? 4 : 0;
#pragma unroll 2
                    for (int g = g0; g < g1; ++g) {
                        const uint4 wa = *reinterpret_cast<const uint4 *>(
                            rowa + 16 * swz_chunk(4 * g + tig, ra & 7));
                        const uint4 wb = *reinterpret_cast<const uint4 *>(
                            rowb + 16 * swz_chunk(4 * g + tig, rb & 7));
                        const uint4 x0 = xq[g * xst], x1 = xq[g * xst + x1o];
                        float r[4];
                        mma_group_s8_1(r, wa, wb, x0, x1);
                        const float X = xsum[g * 8];
                        const float2 pa = sb_word(sba + 4 * g), pb = sb_word(sbb + 4 * g);
                        acc_lo = fmaf(pa.x, r[0], acc_lo);
                        acc_hi = fmaf(pb.x, r[2], acc_hi);
                        b_lo = fmaf(pa.y, X, b_lo);
                        b_hi = fmaf(pb.y, X, b_hi);
                    }
                }
                if (!good)
                    ok = false;
                // the warp's partials to the exchange warp (which also frees
                // the router rows for the next layer)
                if (tig == 0) {
                    red[warp * 16 + gid] = acc_lo * kCode8 + b_lo;
                    red[warp * 16 + 8 + gid] = acc_hi * kCode8 + b_hi;
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(red_bar);
            }
            // ---- the previous layer's output to fp16 (off the critical path)
            if (l > 0)
                convert_slice(l - 1);
            // ---- the layer's work items, dealt to the groups
            {
                // ring order of a layer: shared gate/up, shared down, routed
                // gate/up, routed down; the items follow it
                const int base = l * 3 * U.nu;
                for (int k = q; k < nitems; k += DC_GROUPS) {
                    if (k < U.ns) {
                        do_gu(base + 2 * k, k);
                    } else if (k < 2 * U.ns) {
                        const int s = k - U.ns;
                        do_dn(base + 2 * U.ns + s, s, s_uj[s], l);
                    } else if (k < 2 * U.ns + U.nr) {
                        const int m = k - 2 * U.ns;
                        do_gu(base + 3 * U.ns + 2 * m, U.ns + m);
                    } else {
                        const int m = k - 2 * U.ns - U.nr;
                        do_dn(base + 3 * U.ns + 2 * U.nr + m, U.ns + m, s_uj[U.ns + m], l);
                    }
                }
            }
            // ---- this CTA's rows of the layer output into the accumulator
            named_bar_sync(BAR_ALL, DC_CT);
            {
                float *acc = a.ws.y_acc + (size_t)(l & 1) * H + (size_t)Hc * rank;
                for (int t = ctid; t < Hc / 4; t += DC_CT) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int g = 0; g < DC_GROUPS; ++g) {
                        const float4 p = reinterpret_cast<const float4 *>(ypart + (size_t)g * Hc)[t];
                        v.x += p.x;
                        v.y += p.y;
                        v.z += p.z;
                        v.w += p.w;
                        reinterpret_cast<float4 *>(ypart + (size_t)g * Hc)[t] =
                            make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    red_add_v4(reinterpret_cast<float4 *>(acc) + t, v);
                    red_release_add(ctl + C_ARRIVE, 1u);   // ordered after the add above
                }
            }
        }
        // ---- the last layer's output
        if (ctid == 0 && !spin_until(a, ctl + C_ARRIVE, (unsigned)a.L * G * nred))
            ok = false;
        named_bar_sync(BAR_ALL, DC_CT);
        convert_slice(a.L - 1);
        (void)ok;
    }

    // no CTA leaves while a CTA of its cluster may still write its shared memory
    __syncthreads();
    cluster_sync_all();
    // the last CTA out resets the control words for the next launch; every
    // other CTA has stopped reading them by then
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned old = atomicAdd(ctl + C_EXIT, 1u);
        if (old == (unsigned)G - 1) {
            atomicExch(ctl + C_ARRIVE, 0u);
            atomicExch(ctl + C_ABORT, 0u);
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
    const int H = a.H, I = a.I;
    for (size_t q = blockIdx.x * (size_t)blockDim.x + threadIdx.x; q < n16;
         q += (size_t)gridDim.x * blockDim.x) {
        const size_t off = q * 16;
        uint32_t sbw[4];
        const unsigned char *src = nullptr;
        if (off < P.router_bytes) {
            const int rank = (int)(off / P.rb_bytes);
            const size_t w = off % P.rb_bytes;
            if (w < P.rb_codes) {
                const int i = (int)(w / H);
                const int c = swz_chunk((int)((w % H) / 16), i & 7);
                src = reinterpret_cast<const unsigned char *>(a.router.packed) +
                      (size_t)(P.Rr * rank + i) * H + 16 * (size_t)c;
            } else {
                for (int t = 0; t < 4; ++t) {
                    const int en = (int)((w - P.rb_codes) / 4) + t;
                    const int i = en / P.GH, g = en % P.GH;
                    const size_t ix = (size_t)(P.Rr * rank + i) * P.GH + g;
                    sbw[t] = h2_as_u32(__halves2half2(a.router.scales[ix], a.router.biases[ix]));
                }
            }
        } else {
            const size_t eo = off - P.router_bytes;
            const int e = (int)(eo / P.exp_bytes);
            const size_t w1 = eo % P.exp_bytes;
            const int g = (int)(w1 / P.unit_bytes);
            const size_t w2 = w1 % P.unit_bytes;
            const int cp = (int)(w2 / P.st_bytes);
            const int rank = cp / 3, kind = cp % 3;
            const size_t w = w2 % P.st_bytes;
            const bool sh = e == a.E;
            const int ex = sh ? 0 : e;
            if (kind < 2) {
                const QMat &m = kind == 0 ? (sh ? a.sh_gate : a.gate) : (sh ? a.sh_up : a.up);
                const size_t row0 = (size_t)ex * I + (size_t)kGroup * g + 8 * rank;
                if (w < P.st_codes) {
                    const int i = (int)(w / (H / 2));
                    const int c = swz_chunk((int)((w % (H / 2)) / 16), i);
                    src = reinterpret_cast<const unsigned char *>(m.packed) + (row0 + i) * (H / 2) +
                          16 * (size_t)c;
                } else {
                    for (int t = 0; t < 4; ++t) {
                        const int en = (int)((w - P.st_codes) / 4) + t;
                        const int i = en / P.GH, gg = en % P.GH;
                        const size_t ix = (row0 + i) * P.GH + gg;
                        sbw[t] = h2_as_u32(__halves2half2(m.scales[ix], m.biases[ix]));
                    }
                }
            } else {
                const QMat &m = sh ? a.sh_down : a.down;
                const size_t row0 = (size_t)ex * H + (size_t)P.Hc * rank;
                if (w < P.st_codes) {
                    const int i = (int)(w / 32);
                    src = reinterpret_cast<const unsigned char *>(m.packed) + (row0 + i) * (I / 2) +
                          32 * (size_t)g + (w % 32);
                } else {
                    for (int t = 0; t < 4; ++t) {
                        const int i = (int)((w - P.st_codes) / 4) + t;
                        const size_t ix = (row0 + i) * P.GI + g;
                        sbw[t] = h2_as_u32(__halves2half2(m.scales[ix], m.biases[ix]));
                    }
                }
            }
        }
        dst[q] = src ? *reinterpret_cast<const uint4 *>(src) : make_uint4(sbw[0], sbw[1], sbw[2], sbw[3]);
    }
}

struct ClusterCache {
    int dev = -1;
    size_t smem = 0;
    int nc = 0;
    bool coop_refused = false;
};
ClusterCache g_cluster_cache[64];

}  // namespace

size_t decode_pack_bytes(int E, int H, int I) { return pack_dims(E, H, I).total; }

cudaError_t launch_decode_pack(const DecodePackArgs &a, void *dst, cudaStream_t s)
{
    decode_pack_kernel<<<1024, 256, 0, s>>>(a, static_cast<uint4 *>(dst));
    return cudaGetLastError();
}

size_t decode_workspace_layout(int E, int H, int I, int top_k, void *base, DecodeWorkspace *ws)
{
    (void)E;
    (void)I;
    (void)top_k;
    size_t off = 0;
    const size_t ctl_off = off;
    off = align_up(off + (size_t)C_WORDS * 4, 256);
    const size_t acc_off = off;
    off = align_up(off + (size_t)2 * H * 4, 256);
    if (base && ws) {
        unsigned char *b = static_cast<unsigned char *>(base);
        ws->ctl = reinterpret_cast<unsigned *>(b + ctl_off);
        ws->y_acc = reinterpret_cast<float *>(b + acc_off);
    }
    return off;
}

cudaError_t launch_decode(const DecodeArgs &a0, const LaunchCfg &c)
{
    const PackDims P = pack_dims(a0.E, a0.H, a0.I);
    const size_t budget = 227 * 1024;
    const DcLayout L0 = dc_layout(P, 0);
    if (L0.total + 2 * P.st_bytes + 128 > budget)
        return cudaErrorInvalidValue;
    int NS = (int)((budget - L0.total - 128) / P.st_bytes);
    NS = NS > DC_MAX_STAGES ? DC_MAX_STAGES : NS;
    DecodeArgs a = a0;
    a.NS = NS;
    const DcLayout L = dc_layout(P, NS);
    cudaError_t e = set_smem(moe_decode_kernel, L.total);
    if (e != cudaSuccess)
        return e;
    // how many 8-CTA clusters fit at once with this much shared memory
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess)
        return e;
    ClusterCache &cc = g_cluster_cache[dev & 63];
    if (cc.dev != dev || cc.smem != L.total) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(DC_CLUSTER * 64);
        q.blockDim = dim3(DC_THREADS);
        q.dynamicSmemBytes = L.total;
        cudaLaunchAttribute qa[1];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = DC_CLUSTER;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        q.attrs = qa;
        q.numAttrs = 1;
        int n = 0;
        if ((e = cudaOccupancyMaxActiveClusters(&n, moe_decode_kernel, &q)) != cudaSuccess)
            return e;
        cc.dev = dev;
        cc.smem = L.total;
        cc.nc = n;
    }
    const int NC = cc.nc;
    if (NC < 1)
        return cudaErrorInvalidValue;
    // every cluster's units of one layer must fit its unit slots
    if (cluster_units(0, NC, a.top_k, P.GI).nu > DC_MAX_UNITS)
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(DC_CLUSTER * NC);
    cfg.blockDim = dim3(DC_THREADS);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = c.stream;
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = DC_CLUSTER;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    attrs[1].id = cudaLaunchAttributeCooperative;
    attrs[1].val.cooperative = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = cc.coop_refused ? 1 : 2;
    e = cudaLaunchKernelEx(&cfg, moe_decode_kernel, a);
    if (e != cudaSuccess && !cc.coop_refused) {
        // a driver that does not take the cooperative attribute together with
        // clusters: launch the same grid (sized by the occupancy query) without
        // it; the grid-wide waits stay bounded either way
        (void)cudaGetLastError();
        cc.coop_refused = true;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, moe_decode_kernel, a);
    }
    return e;
}

}  // namespace qmoe
