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
//     through distributed shared memory, so each CTA takes the top-k itself
//     without a grid-wide exchange.
//   * Work is cut into units of (expert, 64 consecutive intermediate
//     indices).  A unit belongs to ONE cluster: CTA r of the cluster computes
//     the gate/up rows 8r..8r+7 of the unit and SwiGLU, sends its eight h
//     values (as fp16 hi/lo pairs) to the 8 CTAs of the cluster and signals a
//     remote mbarrier; each CTA then multiplies its own H/8 rows of the down
//     projection by the unit's 64 h values.  The gate/up -> down dependency
//     never leaves the cluster.
//   * Each CTA adds its weighted down rows of all its units in shared memory
//     and then into an fp32 layer accumulator with one vector atomic per four
//     rows; one grid-wide arrival counter per layer then says the layer's
//     output is complete, and the next layer starts (its input would be this
//     layer's output in a real model).
//   * One producer thread streams the CTA's weights as ~12.7 KB bulk copies
//     (every copy is one contiguous block of the packed layer) through a
//     shared-memory ring, in the order the consumers use them: the shared
//     expert's units need no routing and are fetched a layer ahead; the
//     routed units are fetched as soon as the top-k is known.  The producer
//     warp itself computes the top-k, since it is the one waiting for it.
//   * 16 consumer warps in 4 groups; work item k of a layer goes to group
//     k % 4 (gate/up items: the 4 warps split K; down items: the 4 warps
//     split the rows).
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
constexpr int DC_THREADS = DC_CT + 32;        // + the producer warp
constexpr int DC_MAX_UNITS = 16;              // units per cluster and layer
constexpr int DC_MAX_STAGES = 16;
constexpr int BAR_ALL = 1;                    // named barrier of all consumer threads
constexpr int BAR_GROUP0 = 2;                 // 2..5: one per consumer group

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
    size_t router_off, xraw_off, xs4_off, xs8_off, xsum_off, logit_off, topk_off, hfrag_off,
        hsum_off, ypart_off, red_off, gured_off, bar_off, ring_off, total;
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
    L.xraw_off = dc_take(&off, (size_t)p.H * 2, 16);
    L.xs4_off = dc_take(&off, (size_t)p.GH * 2 * 4 * 16, 16);
    L.xs8_off = dc_take(&off, (size_t)p.GH * 2 * 4 * 16, 16);
    L.xsum_off = dc_take(&off, (size_t)p.GH * 8 * 4, 16);
    L.logit_off = dc_take(&off, (size_t)p.E * 4, 16);
    L.topk_off = dc_take(&off, 32 * 4 * 2, 16);
    L.hfrag_off = dc_take(&off, (size_t)DC_MAX_UNITS * 256, 16);
    L.hsum_off = dc_take(&off, (size_t)DC_MAX_UNITS * DC_CLUSTER * 4, 16);
    L.ypart_off = dc_take(&off, (size_t)DC_GROUPS * p.Hc * 4, 16);
    L.red_off = dc_take(&off, (size_t)DC_CW * 16 * 4, 16);        // router partials
    L.gured_off = dc_take(&off, (size_t)2 * DC_CW * 16 * 4, 16);  // gate/up partials, 2 buffers
    L.bar_off = dc_take(&off, (size_t)(2 * DC_MAX_STAGES + 4 + DC_MAX_UNITS) * 8, 8);
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
__device__ __forceinline__ void st_cluster_u16(uint32_t addr, unsigned short v)
{
    asm volatile("st.shared::cluster.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
// arrive on an mbarrier of a CTA of the cluster; orders this thread's
// earlier shared::cluster stores before the arrival
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                     bar_cluster_addr)
                 : "memory");
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

// ------------------------------------------------------------ helpers --
__device__ __forceinline__ float2 sb_word(const unsigned char *p)
{
    return __half22float2(*reinterpret_cast<const __half2 *>(p));   // (scale, bias)
}

// position (in halves) of intermediate index k (0..63) of a unit, column col
// (0: hi, 1: lo) in the down projection's B fragments [hh][col][tig][8], in
// the x order of mma_group_s4
__device__ __forceinline__ int hfrag_pos(int k, int col)
{
    const int tig = k >> 4, p = k & 15;
    const int i = xperm_s4_inv(p);
    const int hh = i >> 3, e = i & 7;
    return (((hh * 2 + col) * 4 + tig) * 8) + e;
}

// ------------------------------------------------------------------ kernel --
__global__ void __cluster_dims__(DC_CLUSTER, 1, 1) __launch_bounds__(DC_THREADS, 1)
    moe_decode_kernel(const __grid_constant__ DecodeArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const PackDims P = pack_dims(a.E, a.H, a.I);
    const DcLayout L = dc_layout(P, a.NS);
    unsigned char *rbuf = smem + L.router_off;
    uint4 *xraw = reinterpret_cast<uint4 *>(smem + L.xraw_off);
    uint4 *xs4 = reinterpret_cast<uint4 *>(smem + L.xs4_off);
    uint4 *xs8 = reinterpret_cast<uint4 *>(smem + L.xs8_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    float *s_logit = reinterpret_cast<float *>(smem + L.logit_off);
    int *s_idx = reinterpret_cast<int *>(smem + L.topk_off);
    float *s_wt = reinterpret_cast<float *>(smem + L.topk_off + 32 * 4);
    __half *hfrag = reinterpret_cast<__half *>(smem + L.hfrag_off);   // [unit][128]
    float *hsum = reinterpret_cast<float *>(smem + L.hsum_off);       // [unit][8]
    float *ypart = reinterpret_cast<float *>(smem + L.ypart_off);     // [group][Hc]
    float *red = reinterpret_cast<float *>(smem + L.red_off);
    float *gured = reinterpret_cast<float *>(smem + L.gured_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *full = bars, *empty = bars + DC_MAX_STAGES;
    uint64_t *rfull = bars + 2 * DC_MAX_STAGES, *rempty = rfull + 1, *topk_bar = rfull + 2,
             *logit_bar = rfull + 3, *hbar = rfull + 4;
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
        }
        mbar_init(rfull, 1);
        mbar_init(rempty, 1);
        mbar_init(topk_bar, 1);
        mbar_init(logit_bar, DC_CLUSTER);
        for (int s = 0; s < DC_MAX_UNITS; ++s)
            mbar_init(&hbar[s], DC_CLUSTER);
        mbar_init_fence();
    }
    // every CTA of the cluster has initialised its barriers before anyone
    // signals one remotely
    cluster_sync_all();
    // the workspace may still be in use by the previous launch on the stream
    pdl_wait();

    if (warp == DC_CW) {
        // ====================================================== producer
        const uint64_t pol = l2_evict_first_policy();
        bool ok = true;
        int seq = 0;
        auto issue = [&](const unsigned char *src) {
            const int st = seq % NS, use = seq / NS;
            if (use > 0 && ok && !wait_bar(a, &empty[st], (use - 1) & 1))
                ok = false;
            if (ok) {
                mbar_arrive_expect_tx(&full[st], (uint32_t)P.st_bytes);
                bulk_g2s(ring + (size_t)st * P.st_bytes, src, (uint32_t)P.st_bytes, &full[st], pol);
            }
            ++seq;
        };
        if (lane == 0) {
            mbar_arrive_expect_tx(rfull, (uint32_t)P.rb_bytes);
            bulk_g2s_plain(rbuf, static_cast<const unsigned char *>(a.layer[0]) +
                                     pack_router_off(P, rank),
                           (uint32_t)P.rb_bytes, rfull);
        }
        for (int l = 0; l < a.L; ++l) {
            const unsigned char *lp = static_cast<const unsigned char *>(a.layer[l]);
            if (lane == 0 && ok) {
                int j, g;
                for (int s = 0; s < U.ns; ++s) {   // shared gate/up
                    unit_of(s, U, cl, NC, K, P.GI, &j, &g);
                    issue(lp + pack_copy_off(P, a.E, g, rank, 0));
                    issue(lp + pack_copy_off(P, a.E, g, rank, 1));
                }
                for (int s = 0; s < U.ns; ++s) {   // shared down
                    unit_of(s, U, cl, NC, K, P.GI, &j, &g);
                    issue(lp + pack_copy_off(P, a.E, g, rank, 2));
                }
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
            // ---- top-k of this layer (the whole producer warp)
            if (ok && !wait_bar_cluster(a, logit_bar, l & 1))
                ok = false;
            ok = __all_sync(0xffffffffu, ok);
            {
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
                float my_v = 0.f;
                int my_i = 0;
                for (int jj = 0; jj < K; ++jj) {
                    unsigned bk = 0u;
                    int be = 0x7fffffff;
                    float bv = 0.f;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        if (!taken[qq] && key[qq] > bk) {   // strict: the lower index wins ties
                            bk = key[qq];
                            be = lane + 32 * qq;
                            bv = v[qq];
                        }
                    const unsigned mk = __reduce_max_sync(0xffffffffu, bk);
                    const int win = (int)__reduce_min_sync(0xffffffffu,
                                                           (unsigned)(bk == mk ? be : 0x7fffffff));
                    const float wv = __shfl_sync(0xffffffffu, bv, win & 31);
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        if (win == lane + 32 * qq)
                            taken[qq] = true;
                    if (lane == jj) {
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
                    const int ei = (my_i >= 0 && my_i < a.E) ? my_i : 0;
                    s_idx[lane] = ei;
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
                    mbar_arrive(topk_bar);   // the routed down items may read s_wt
            }
            if (lane == 0 && ok) {
                int j, g;
                for (int s = U.ns; s < U.nu; ++s) {   // routed gate/up
                    unit_of(s, U, cl, NC, K, P.GI, &j, &g);
                    const int e = s_idx[j];
                    issue(lp + pack_copy_off(P, e, g, rank, 0));
                    issue(lp + pack_copy_off(P, e, g, rank, 1));
                }
                for (int s = U.ns; s < U.nu; ++s) {   // routed down
                    unit_of(s, U, cl, NC, K, P.GI, &j, &g);
                    issue(lp + pack_copy_off(P, s_idx[j], g, rank, 2));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            __syncwarp();
        }
        // drain: every copy issued has landed before the CTA may exit
        if (lane == 0) {
            for (int st = 0; st < NS && st < seq; ++st) {
                const int last = seq - 1 - ((seq - 1 - st) % NS);   // last seq that used stage st
                wait_bar(a, &full[st], (last / NS) & 1);
            }
        }
        __syncwarp();
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
        // gate/up partials alternate between two buffers from item to item of a
        // group, so a warp that runs ahead into the next item cannot overwrite
        // what the group's first warp is still reading
        int gu_buf = 0;
        auto do_gu = [&](int seq0, int slot, int l) {
            const int sa = seq0 % NS, sb = (seq0 + 1) % NS;
            // the lanes of a warp decide together: the mma below is warp-collective
            const bool good = __all_sync(0xffffffffu, ok && wait_bar(a, &full[sa], (seq0 / NS) & 1) &&
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
#pragma unroll 2
                for (int g = g0; g < g1; ++g) {
                    const int ch = swz_chunk(2 * g + (tig >> 1), gid);
                    const uint2 wa = *reinterpret_cast<const uint2 *>(rowA + 16 * ch);
                    const uint2 wb = *reinterpret_cast<const uint2 *>(rowB + 16 * ch);
                    uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
                    if (gid == 0) {
                        x0 = xs4[(g * 2 + 0) * 4 + tig];
                        x1 = xs4[(g * 2 + 1) * 4 + tig];
                    }
                    float r[4];
                    mma_group_s4(r, wa, wb, x0, x1);
                    if (tig == 0) {
                        const float X = xsum[g * 8];
                        const float2 pa = sb_word(sbA + 4 * g), pb = sb_word(sbB + 4 * g);
                        ag = fmaf(pa.x, r[0], ag);
                        au = fmaf(pb.x, r[2], au);
                        bg = fmaf(pa.y, X, bg);
                        bu = fmaf(pb.y, X, bu);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&empty[sa]);
                mbar_arrive(&empty[sb]);
            }
            float *gub = gured + (size_t)gu_buf * DC_CW * 16;
            gu_buf ^= 1;
            float *gr = gub + (size_t)warp * 16;
            if (tig == 0) {
                gr[gid] = ag * kCode4 + bg;       // gate row gid
                gr[8 + gid] = au * kCode4 + bu;   // up row gid
            }
            named_bar_sync(BAR_GROUP0 + q, DC_GW * 32);
            if (wq == 0) {
                // SwiGLU of the CTA's 8 intermediate indices, then to every CTA
                // of the cluster as fp16 (hi, lo) fragments + their sum
                const float *g0r = gub + (size_t)(q * DC_GW) * 16;
                float h = 0.f;
                if (lane < 8) {
                    float gs = 0.f, us = 0.f;
#pragma unroll
                    for (int w = 0; w < DC_GW; ++w) {
                        gs += g0r[w * 16 + lane];
                        us += g0r[w * 16 + 8 + lane];
                    }
                    h = gs / (1.f + expf(-gs)) * us;
                }
                const __half hh = __float2half_rn(h);
                const __half hl = __float2half_rn(h - __half2float(hh));
                float part = __half2float(hh) + __half2float(hl);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                const unsigned short bh = __half_as_ushort(hh), bl = __half_as_ushort(hl);
                unsigned short vh[8], vl[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    vh[i] = (unsigned short)__shfl_sync(0xffffffffu, (unsigned)bh, i);
                    vl[i] = (unsigned short)__shfl_sync(0xffffffffu, (unsigned)bl, i);
                }
                part = __shfl_sync(0xffffffffu, part, 0);
                if (lane < DC_CLUSTER) {
                    const uint32_t base = smem_u32(hfrag + (size_t)slot * 128);
                    const uint32_t tbase = mapa_rank(base, lane);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int k = 8 * rank + i;
                        st_cluster_u16(tbase + 2 * hfrag_pos(k, 0), vh[i]);
                        st_cluster_u16(tbase + 2 * hfrag_pos(k, 1), vl[i]);
                    }
                    st_cluster_f32(mapa_rank(smem_u32(hsum + slot * DC_CLUSTER + rank), lane), part);
                    mbar_arrive_remote(mapa_rank(smem_u32(&hbar[slot]), lane));
                }
                (void)l;
            }
            if (!good)
                ok = false;
        };

        // ---------------------------------------- one down work item
        auto do_dn = [&](int seq, int slot, int j, int l) {
            const int st = seq % NS;
            // the lanes of a warp decide together: the mma below is warp-collective
            bool good = __all_sync(0xffffffffu, ok && wait_bar(a, &full[st], (seq / NS) & 1) &&
                                                    wait_bar_cluster(a, &hbar[slot], l & 1));
            float w = 1.f;
            if (good && j < K) {
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
                    mma_group_s4(r, wa, wb, x0, x1);
                    if (tig == 0) {
                        const float2 pa = sb_word(S + P.st_codes + 4 * (size_t)r0);
                        const float2 pb = sb_word(S + P.st_codes + 4 * (size_t)(r0 + 8));
                        const float va = fmaf(pa.x * kCode4, r[0] + r[1], pa.y * X);
                        const float vb = fmaf(pb.x * kCode4, r[2] + r[3], pb.y * X);
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

        for (int l = 0; l < a.L; ++l) {
            // ---- the previous layer's output is complete in every CTA
            if (l > 0) {
                if (ctid == 0 && !spin_until(a, ctl + C_ARRIVE, (unsigned)(l * G)))
                    ok = false;
                named_bar_sync(BAR_ALL, DC_CT);
            }
            // ---- x of this layer: 16-byte loads, then both fragment orders
            {
                const uint4 *xg = reinterpret_cast<const uint4 *>(a.x + (size_t)l * H);
                for (int t = ctid; t < H / 8; t += DC_CT)
                    xraw[t] = __ldcg(xg + t);
                named_bar_sync(BAR_ALL, DC_CT);
                const __half *xh = reinterpret_cast<const __half *>(xraw);
                stage_x<kPermS4>(xs4, xsum, GH, 1, 1,
                                 [&](int, int, int k) { return __half2float(xh[k]); }, ctid, DC_CT);
                stage_x<8>(xs8, nullptr, GH, 1, 1,
                           [&](int, int, int k) { return __half2float(xh[k]); }, ctid, DC_CT);
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
                    for (int g = g0; g < g1; ++g) {
                        const uint4 wa = *reinterpret_cast<const uint4 *>(
                            rowa + 16 * swz_chunk(4 * g + tig, ra & 7));
                        const uint4 wb = *reinterpret_cast<const uint4 *>(
                            rowb + 16 * swz_chunk(4 * g + tig, rb & 7));
                        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0;
                        if (gid == 0) {
                            x0 = xs8[(g * 2 + 0) * 4 + tig];
                            x1 = xs8[(g * 2 + 1) * 4 + tig];
                        }
                        float r[4];
                        mma_group_s8(r, wa, wb, x0, x1);
                        if (tig == 0) {
                            const float X = xsum[g * 8];
                            const float2 pa = sb_word(sba + 4 * g), pb = sb_word(sbb + 4 * g);
                            acc_lo = fmaf(pa.x, r[0], acc_lo);
                            acc_hi = fmaf(pb.x, r[2], acc_hi);
                            b_lo = fmaf(pa.y, X, b_lo);
                            b_hi = fmaf(pb.y, X, b_hi);
                        }
                    }
                }
                if (!good)
                    ok = false;
                if (tig == 0) {
                    red[warp * 16 + gid] = acc_lo * kCode8 + b_lo;
                    red[warp * 16 + 8 + gid] = acc_hi * kCode8 + b_hi;
                }
                named_bar_sync(BAR_ALL, DC_CT);
                if (ctid == 0)
                    mbar_arrive(rempty);   // the producer may load the next layer's rows
                if (warp == 0) {
                    if (lane < 16) {
                        float v = 0.f;
                        for (int w = 0; w < DC_CW; ++w)
                            v += red[w * 16 + lane];
                        if (lane < Rr)
                            s_logit[Rr * rank + lane] = v;
                    }
                    __syncwarp();
                    if (lane < DC_CLUSTER) {   // this CTA's logits to every CTA of the cluster
                        for (int i = 0; i < Rr; ++i) {
                            const uint32_t adr = smem_u32(s_logit + Rr * rank + i);
                            st_cluster_f32(mapa_rank(adr, lane), s_logit[Rr * rank + i]);
                        }
                        mbar_arrive_remote(mapa_rank(smem_u32(logit_bar), lane));
                    }
                }
            }
            // ---- the previous layer's output to fp16 (off the critical path)
            if (l > 0)
                convert_slice(l - 1);
            // ---- the layer's work items, dealt to the groups
            {
                const int base = l * 3 * U.nu;
                for (int k = q; k < nitems; k += DC_GROUPS) {
                    int seq, slot;
                    bool gu;
                    if (k < U.ns) {
                        gu = true, slot = k, seq = base + 2 * k;
                    } else if (k < 2 * U.ns) {
                        gu = false, slot = k - U.ns, seq = base + 2 * U.ns + slot;
                    } else if (k < 2 * U.ns + U.nr) {
                        gu = true, slot = U.ns + (k - 2 * U.ns);
                        seq = base + 3 * U.ns + 2 * (k - 2 * U.ns);
                    } else {
                        gu = false;
                        const int m = k - 2 * U.ns - U.nr;
                        slot = U.ns + m;
                        seq = base + 3 * U.ns + 2 * U.nr + m;
                    }
                    if (gu) {
                        do_gu(seq, slot, l);
                    } else {
                        int j, g;
                        unit_of(slot, U, cl, NC, K, P.GI, &j, &g);
                        do_dn(seq, slot, j, l);
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
                    atomicAdd(reinterpret_cast<float4 *>(acc) + t, v);
                }
            }
            named_bar_sync(BAR_ALL, DC_CT);
            if (ctid == 0) {
                __threadfence();
                atomicAdd(ctl + C_ARRIVE, 1u);
            }
        }
        // ---- the last layer's output
        if (ctid == 0 && !spin_until(a, ctl + C_ARRIVE, (unsigned)(a.L * G)))
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
