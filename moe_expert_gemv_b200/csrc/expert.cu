// expert.cu -- decode-step MoE experts for one token: gathered routed SwiGLU
// experts plus the resident shared expert, combined with the router weights.
//
// TurboFieldfare article (jeff.news), section "내부 구조가 진짜 흥미로운 부분"
// (internal structure): the router's top-8 expert ids select the routed
// experts; the resident shared-expert branch is computed alongside; the
// shared output and the routed output are added.  Experts are SwiGLU:
//   h = silu(gate x) * (up x),  r = down h,  y = r_shared + sum_j wt_j r_{idx_j}.
// Format: MLX affine 4-bit, group 64 (section "성능과 제약").
//
// Two kernels, chained with programmatic dependent launch:
//  gate/up: work item = (expert slot, 8 output rows); the 16-row mma tile
//           holds 8 gate rows over 8 up rows, so each thread ends with gate
//           and up values of the same intermediate index and applies SwiGLU
//           in registers.  Split over 11 consumer warps along K.
//  down:    work item = (expert slot, 16 output rows); one warp per item;
//           h enters the tensor core as an fp16 hi/lo pair (two batch
//           columns) so the fp32 intermediate keeps its precision.  The
//           slot partials of a row tile are combined, in slot order, by
//           whichever warp finishes that tile last (atomic arrival counter
//           that the combining warp resets), so the output is deterministic.
// Weights of the shared expert are streamed before the previous kernel of
// the stream has completed; routed weights follow once the ids are visible.
// Expert parallelism (EP = true, a separate instantiation so the one-GPU
// kernels carry no ownership test): a rank skips the slots whose expert it
// does not hold, before the copy and before the compute, and adds only its
// own slots into an fp32 partial.
#include "common.cuh"
#include "kernels.h"

namespace qmoe {

size_t expert_workspace_layout(int H, int I, int top_k, void *base, ExpertWorkspace *ws)
{
    const int nslot = top_k + 1;
    size_t off = 0;
    const size_t h_off = off;
    off = align_up(off + (size_t)nslot * I * 4, 256);
    const size_t part_off = off;
    off = align_up(off + (size_t)nslot * H * 4, 256);
    const size_t cnt_off = off;
    off = align_up(off + (size_t)(H / 16) * 4, 256);
    if (ws && base) {
        unsigned char *b = static_cast<unsigned char *>(base);
        ws->h = reinterpret_cast<float *>(b + h_off);
        ws->part = reinterpret_cast<float *>(b + part_off);
        ws->counters = reinterpret_cast<int32_t *>(b + cnt_off);
    }
    return off;
}

namespace {

// ------------------------------------------------------------- gate / up --
constexpr int GU_CW = 11;
constexpr int GU_THREADS = (GU_CW + 1) * 32;
constexpr int GU_STAGES = 3;

struct GuLayout {
    int G, S;
    size_t xs_off, xsum_off, red_off, bar_off, stage_off, codes_bytes, sb_bytes, stage_bytes, total;
};

__host__ __device__ inline GuLayout gu_layout(int H)
{
    GuLayout L;
    L.G = H / kGroup;
    L.S = tile_stride_words(H, 4);
    size_t off = 0;
    L.xs_off = off;
    off += (size_t)L.G * 2 * 1 * 4 * 16;
    L.xsum_off = off;
    off += (size_t)L.G * 8 * 4;
    off = (off + 15) & ~(size_t)15;
    L.red_off = off;
    off += 2 * GU_CW * 32 * 16;
    L.bar_off = off;
    off += 2 * GU_STAGES * 8;
    off = (off + 127) & ~(size_t)127;
    L.stage_off = off;
    L.codes_bytes = (size_t)16 * L.S * 4;
    L.sb_bytes = (size_t)16 * L.G * 2;
    L.stage_bytes = L.codes_bytes + 2 * L.sb_bytes;
    off += (size_t)GU_STAGES * L.stage_bytes;
    L.total = off;
    return L;
}

__device__ __forceinline__ int routed_expert(const ExpertArgs &a, int j, bool *valid)
{
    const int e = a.idx[j];
    *valid = (e >= 0 && e < a.E);
    return *valid ? e : 0;
}

// The slots this rank holds, as bits: bit 0 the shared expert (rank 0),
// bit j + 1 routed slot j when its expert e has e / (E / ep_world) ==
// ep_rank (an invalid id belongs to no rank).  One load per id, made once
// per thread after the ids are complete (top_k <= 16).
__device__ __forceinline__ uint32_t owned_slots(const ExpertArgs &a)
{
    if (a.slot_mask) {   // an explicit choice: the routed slots among it with a valid id
        uint32_t m = a.slot_mask & 1u;
        for (int j = 0; j < a.top_k; ++j)
            if ((a.slot_mask >> (j + 1)) & 1u) {
                const int e = __ldcg(a.idx + j);
                if (e >= 0 && e < a.E)
                    m |= 1u << (j + 1);
            }
        return m;
    }
    uint32_t m = a.ep_rank == 0 ? 1u : 0u;
    const int per = a.E / a.ep_world;
    for (int j = 0; j < a.top_k; ++j) {
        const int e = __ldcg(a.idx + j);
        if (e >= 0 && e < a.E && e / per == a.ep_rank)
            m |= 1u << (j + 1);
    }
    return m;
}

template <bool EP>
__global__ void __launch_bounds__(GU_THREADS, 1) expert_gateup_kernel(ExpertArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const GuLayout L = gu_layout(a.H);
    uint4 *xs = reinterpret_cast<uint4 *>(smem + L.xs_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    float4 *red = reinterpret_cast<float4 *>(smem + L.red_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + GU_STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int octs = a.I / 8;
    const int n_items = (a.top_k + 1) * octs;   // slot order 0 = shared, 1.. = routed
    const int Hw = a.H / 8;                      // words per row

    if (threadIdx.x == 0) {
        for (int s = 0; s < GU_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], GU_CW);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == GU_CW) {
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            bool waited = false, bad = false;
            int last_use[GU_STAGES] = {-1, -1, -1};
            int k = 0;
            // before the ids are known: the shared slot only
            uint32_t mine = a.slot_mask ? (a.slot_mask & 1u) : (a.ep_rank == 0 ? 1u : 0u);
            for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
                const int so = item / octs, oct = item % octs;
                QMat g = a.sh_gate, u = a.sh_up;
                size_t mat_off = 0;   // in rows
                if (so > 0 && !waited) {
                    pdl_wait();   // the ids come from the previous kernel
                    waited = true;
                    if (EP)
                        mine = owned_slots(a);
                }
                if (EP && !((mine >> so) & 1u))
                    continue;
                if (so > 0) {
                    bool valid;
                    const int e = routed_expert(a, so - 1, &valid);
                    bad |= !valid;
                    g = a.gate;
                    u = a.up;
                    mat_off = (size_t)(e - a.ep_first) * a.I;   // held slots only: e >= ep_first
                }
                const int st = k % GU_STAGES, use = k / GU_STAGES;
                if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, a.status))
                    break;
                unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
                const uint32_t row_bytes = (uint32_t)Hw * 4;
                const uint32_t sb8 = (uint32_t)(8 * L.G * 2);
                mbar_arrive_expect_tx(&full[st], 16 * row_bytes + 4 * sb8);
                const size_t r0 = mat_off + (size_t)oct * 8;
                for (int r = 0; r < 8; ++r) {
                    bulk_g2s(stage + (size_t)r * L.S * 4, g.packed + (r0 + r) * Hw, row_bytes, &full[st], pol);
                    bulk_g2s(stage + (size_t)(r + 8) * L.S * 4, u.packed + (r0 + r) * Hw, row_bytes,
                             &full[st], pol);
                }
                unsigned char *sc = stage + L.codes_bytes;
                unsigned char *bi = sc + L.sb_bytes;
                bulk_g2s(sc, g.scales + r0 * L.G, sb8, &full[st], pol);
                bulk_g2s(sc + sb8, u.scales + r0 * L.G, sb8, &full[st], pol);
                bulk_g2s(bi, g.biases + r0 * L.G, sb8, &full[st], pol);
                bulk_g2s(bi + sb8, u.biases + r0 * L.G, sb8, &full[st], pol);
                last_use[st] = use;
                ++k;
            }
            if (bad)
                flag_status(a.status, QMOE_DEV_BAD_EXPERT);
            for (int s = 0; s < GU_STAGES; ++s)
                if (last_use[s] >= 0)
                    mbar_wait(&full[s], last_use[s] & 1, a.status);
        }
        return;
    }

    // ---------------- consumers
    pdl_wait();
    pdl_trigger();
    const __half *x = a.x;
    stage_x<4>(xs, xsum, L.G, 1, 1, [&](int, int, int k) { return __half2float(x[k]); },
               threadIdx.x, GU_CW * 32);
    named_bar_sync(1, GU_CW * 32);

    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t mine = EP ? owned_slots(a) : ~0u;   // after the wait above
    bool failed = false;
    int k = -1;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (EP && !((mine >> (item / octs)) & 1u))
            continue;
        ++k;
        const int st = k % GU_STAGES, use = k / GU_STAGES;
        if (!failed && !mbar_wait(&full[st], use & 1, a.status))
            failed = true;
        // the lanes of a warp decide together: the mma below is warp-collective
        failed = __any_sync(0xffffffffu, failed);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (!failed) {
            const unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
            const uint32_t *tile = reinterpret_cast<const uint32_t *>(stage);
            const __half *sc = reinterpret_cast<const __half *>(stage + L.codes_bytes);
            const __half *bi = reinterpret_cast<const __half *>(stage + L.codes_bytes + L.sb_bytes);
            for (int g = warp; g < L.G; g += GU_CW)
                tile_group<4>(tile, L.S, sc, bi, L.G, xs, xsum, 1, g, gid, tig, acc);
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[st]);
        red[((k & 1) * GU_CW + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        named_bar_sync(1, GU_CW * 32);
        if (warp == k % GU_CW && tig == 0) {
            float gv = 0.f, uv = 0.f;
            for (int w = 0; w < GU_CW; ++w) {
                const float4 p = red[((k & 1) * GU_CW + w) * 32 + lane];
                gv += p.x;   // row gid (gate), column 0
                uv += p.z;   // row gid + 8 (up), column 0
            }
            const int so = item / octs, oct = item % octs;
            const int slot = so == 0 ? a.top_k : so - 1;
            bool valid = true;
            if (so > 0)
                routed_expert(a, so - 1, &valid);
            const float h = valid ? gv / (1.f + expf(-gv)) * uv : 0.f;
            a.ws.h[(size_t)slot * a.I + oct * 8 + gid] = h;
        }
    }
}

// ------------------------------------------------------------------ down --
constexpr int DN_CW = 8;
constexpr int DN_THREADS = (DN_CW + 1) * 32;
constexpr int DN_MAX_STAGES = 16;

struct DnLayout {
    int G, S, nslot, NS;
    size_t xs_off, xsum_off, bar_off, stage_off, codes_bytes, sb_bytes, stage_bytes, total;
};

__host__ __device__ inline DnLayout dn_layout(int I, int top_k, int NS)
{
    DnLayout L;
    L.G = I / kGroup;
    L.S = tile_stride_words(I, 4);
    L.nslot = top_k + 1;
    L.NS = NS;
    size_t off = 0;
    L.xs_off = off;
    off += (size_t)L.nslot * L.G * 2 * 2 * 4 * 16;
    L.xsum_off = off;
    off += (size_t)L.nslot * L.G * 8 * 4;
    off = (off + 15) & ~(size_t)15;
    L.bar_off = off;
    off += 2 * DN_MAX_STAGES * 8;
    off = (off + 127) & ~(size_t)127;
    L.stage_off = off;
    L.codes_bytes = (size_t)16 * L.S * 4;
    L.sb_bytes = (size_t)16 * L.G * 2;
    L.stage_bytes = L.codes_bytes + 2 * L.sb_bytes;
    off += (size_t)NS * L.stage_bytes;
    L.total = off;
    return L;
}

template <bool EP>
__global__ void __launch_bounds__(DN_THREADS, 1) expert_down_kernel(ExpertArgs a, int NS)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const DnLayout L = dn_layout(a.I, a.top_k, NS);
    uint4 *xs = reinterpret_cast<uint4 *>(smem + L.xs_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + DN_MAX_STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = a.H / 16;
    const int nslot = a.top_k + 1;
    const int n_items = nslot * tiles;
    const int Iw = a.I / 8;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == DN_CW) {
        if (lane == 0) {
            // The ids were complete before the gate/up kernel that precedes
            // this one let it launch, so they can be read before the wait.
            const uint64_t pol = l2_evict_first_policy();
            int last_use[DN_MAX_STAGES];
            for (int s = 0; s < DN_MAX_STAGES; ++s)
                last_use[s] = -1;
            int k = 0;
            const uint32_t mine = EP ? owned_slots(a) : ~0u;
            for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
                const int so = item / tiles, tile = item % tiles;
                if (EP && !((mine >> so) & 1u))
                    continue;
                QMat d = a.sh_down;
                size_t mat_off = 0;
                if (so > 0) {
                    const int e = __ldcg(a.idx + (so - 1));
                    d = a.down;
                    mat_off = (size_t)((e >= 0 && e < a.E) ? e - a.ep_first : 0) * a.H;
                }
                const int st = k % NS, use = k / NS;
                if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, a.status))
                    break;
                unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
                const uint32_t row_bytes = (uint32_t)Iw * 4;
                const uint32_t sb = (uint32_t)(16 * L.G * 2);
                const size_t r0 = mat_off + (size_t)tile * 16;
                mbar_arrive_expect_tx(&full[st], 16 * row_bytes + 2 * sb);
                if (L.S == Iw) {
                    bulk_g2s(stage, d.packed + r0 * Iw, 16 * row_bytes, &full[st], pol);
                } else {
                    for (int r = 0; r < 16; ++r)
                        bulk_g2s(stage + (size_t)r * L.S * 4, d.packed + (r0 + r) * Iw, row_bytes,
                                 &full[st], pol);
                }
                bulk_g2s(stage + L.codes_bytes, d.scales + r0 * L.G, sb, &full[st], pol);
                bulk_g2s(stage + L.codes_bytes + L.sb_bytes, d.biases + r0 * L.G, sb, &full[st], pol);
                last_use[st] = use;
                ++k;
            }
            for (int s = 0; s < NS; ++s)
                if (last_use[s] >= 0)
                    mbar_wait(&full[s], last_use[s] & 1, a.status);
        }
        return;
    }

    // ---------------- consumers
    pdl_wait();
    pdl_trigger();
    // h of every slot as an fp16 (hi, lo) pair: columns 0 and 1
    const float *hws = a.ws.h;
    const int I = a.I;
    stage_x<4>(xs, xsum, L.G, 2, nslot,
               [&](int v, int n, int k) {
                   const float val = __ldcg(hws + (size_t)v * I + k);
                   const float hi = __half2float(__float2half_rn(val));
                   return n == 0 ? hi : val - hi;
               },
               threadIdx.x, DN_CW * 32);
    named_bar_sync(1, DN_CW * 32);

    // slots of this rank: each tile is complete after that many arrivals
    const uint32_t mine = EP ? owned_slots(a) : ~0u;
    const int n_owned = EP ? __popc(mine) : nslot;
    if (n_owned == 0) {   // nothing to add here: this rank's share is zero
        for (int row = blockIdx.x * DN_CW * 32 + threadIdx.x; row < a.H; row += gridDim.x * DN_CW * 32) {
            const float v = a.y_add ? __ldcg(a.y_add + row) : 0.f;
            if (a.y_part)
                a.y_part[row] = v;
            else if (a.slot_mask)
                a.y[row] = __float2half_rn(v);
        }
        return;
    }
    const int gid = lane >> 2, tig = lane & 3;
    bool failed = false;
    int k = -1;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (EP && !((mine >> (item / tiles)) & 1u))
            continue;
        ++k;
        if (k % DN_CW != warp)
            continue;
        const int st = k % NS, use = k / NS;
        if (!failed && !mbar_wait(&full[st], use & 1, a.status))
            failed = true;
        // the lanes of a warp decide together: the mma below is warp-collective
        failed = __any_sync(0xffffffffu, failed);
        const int so = item / tiles, tile = item % tiles;
        const int slot = so == 0 ? a.top_k : so - 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (!failed) {
            const unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
            const uint32_t *t = reinterpret_cast<const uint32_t *>(stage);
            const __half *sc = reinterpret_cast<const __half *>(stage + L.codes_bytes);
            const __half *bi = reinterpret_cast<const __half *>(stage + L.codes_bytes + L.sb_bytes);
            const uint4 *xsl = xs + (size_t)slot * L.G * 2 * 2 * 4;
            const float *xsuml = xsum + (size_t)slot * L.G * 8;
            for (int g = 0; g < L.G; ++g)
                tile_group<4>(t, L.S, sc, bi, L.G, xsl, xsuml, 2, g, gid, tig, acc);
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[st]);
        const int r0 = tile * 16;
        if (tig == 0) {
            a.ws.part[(size_t)slot * a.H + r0 + gid] = acc[0] + acc[1];
            a.ws.part[(size_t)slot * a.H + r0 + gid + 8] = acc[2] + acc[3];
        }
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0)
            old = atomicAdd(reinterpret_cast<int *>(a.ws.counters + tile), 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == n_owned - 1) {
            __threadfence();
            if (lane < 16) {
                const int row = r0 + lane;
                float v = (mine & 1u) ? __ldcg(a.ws.part + (size_t)a.top_k * a.H + row) : 0.f;
                if (a.y_add)
                    v += __ldcg(a.y_add + row);
                for (int j = 0; j < a.top_k; ++j) {
                    const int e = __ldcg(a.idx + j);
                    if (e >= 0 && e < a.E && ((mine >> (j + 1)) & 1u))
                        v = fmaf(__ldcg(a.weights + j), __ldcg(a.ws.part + (size_t)j * a.H + row), v);
                }
                if (a.y_part)
                    a.y_part[row] = v;
                else
                    a.y[row] = __float2half_rn(v);
            }
            if (lane == 0)
                a.ws.counters[tile] = 0;
        }
    }
}

}  // namespace

cudaError_t launch_expert_gateup(const ExpertArgs &a, const LaunchCfg &c)
{
    const GuLayout L = gu_layout(a.H);
    if (L.total > 227 * 1024)
        return cudaErrorInvalidValue;
    const int n_items = (a.top_k + 1) * (a.I / 8);
    const int grid = n_items < c.num_sms ? n_items : c.num_sms;
    const bool ep = a.ep_world > 1 || a.slot_mask != 0;
    cudaError_t e = ep ? set_smem(expert_gateup_kernel<true>, L.total) : set_smem(expert_gateup_kernel<false>, L.total);
    if (e != cudaSuccess)
        return e;
    return ep ? launch_ex(expert_gateup_kernel<true>, dim3(grid), dim3(GU_THREADS), L.total, c, 1, a)
              : launch_ex(expert_gateup_kernel<false>, dim3(grid), dim3(GU_THREADS), L.total, c, 1, a);
}

cudaError_t launch_expert_down(const ExpertArgs &a, const LaunchCfg &c)
{
    // leave room on each SM for the gate/up kernel it overlaps with
    const size_t budget = 227 * 1024 - gu_layout(a.H).total - 2048;
    const DnLayout L0 = dn_layout(a.I, a.top_k, 0);
    if (L0.total + 2 * L0.stage_bytes > budget)
        return cudaErrorInvalidValue;
    int NS = (int)((budget - L0.total) / L0.stage_bytes);
    NS = NS > DN_MAX_STAGES ? DN_MAX_STAGES : NS;
    const DnLayout L = dn_layout(a.I, a.top_k, NS);
    const int n_items = (a.top_k + 1) * (a.H / 16);
    const int grid = n_items < c.num_sms ? n_items : c.num_sms;
    const bool ep = a.ep_world > 1 || a.slot_mask != 0;
    cudaError_t e = ep ? set_smem(expert_down_kernel<true>, L.total) : set_smem(expert_down_kernel<false>, L.total);
    if (e != cudaSuccess)
        return e;
    return ep ? launch_ex(expert_down_kernel<true>, dim3(grid), dim3(DN_THREADS), L.total, c, 1, a, NS)
              : launch_ex(expert_down_kernel<false>, dim3(grid), dim3(DN_THREADS), L.total, c, 1, a, NS);
}

}  // namespace qmoe
