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
//   1. group   : (token, slot) pairs listed per expert (misc.cu); a pair's
//                index in that list is its position; the shared expert's
//                positions follow, one per token;
//   2. prep    : x of every position in mma fragment order (gathered, so
//                that the 8 positions of a token tile are contiguous) + group
//                sums; the list of 8-position token tiles of every slot;
//   3. gate/up : persistent CTAs; a unit is (token tile, 64 gate + 64 up
//                rows).  A producer warp takes units from a global queue and
//                streams the tile's x (one copy) and the unit's weights in
//                8+8-row sub-blocks into shared-memory rings; each consumer
//                warp owns one sub-block: codes enter the tensor cores as
//                exact fp16 values (subnormal code bits), per-group fp32
//                scale, SwiGLU in registers, h written as fp16 (hi, lo)
//                fragments per position;
//   4. hsum    : per-group sums of h (bias folding of the down projection);
//   5. down    : the same scheme, a unit is (token tile, 256 rows of the
//                hidden size) in 32-row sub-blocks, h hi and lo passes
//                sharing the dequantised codes; unweighted expert outputs
//                r[position][H] in fp32;
//   6. combine : y[t] = r_shared[t] + sum_j wt[t][j] r[pos(t, j)], in slot
//                order, rounded once to fp16.
// Every operand of the inner loops is in shared memory.  A light expert (at
// most 8 tokens: most of them under skewed routing) is streamed from HBM
// exactly once; a heavy one once per token tile, the repeats hitting L2.
// Slots with at least qmoe_set_prefill_tensor_min tokens (0 by default: off)
// skip steps 3 and 5 and run on the tcgen05 kernels of prefill_tc.cu.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace qmoe {

namespace {

constexpr int PF_CW = 8;                      // consumer warps = sub-blocks per unit
constexpr int PF_THREADS = (PF_CW + 1) * 32;  // + one producer warp
constexpr int PF_MAX_STAGES = 12;
constexpr int TILE_T = 8;                     // positions per token tile
constexpr int GU_ROWS = 8;                    // gate rows (and the same up rows) per sub-block
constexpr int DN_ROWS = 32;                   // down rows per sub-block

// how a weight tile reaches shared memory
enum TileMode {
    TILE_CONTIG = 1,   // rows already at a conflict-free stride: one 1-D bulk copy
    TILE_SWZ = 2,      // rows of 128-byte multiples: one swizzled 3-D tensor copy
    TILE_ROWS = 3,     // otherwise: one bulk copy per row into padded rows
};

struct PfDims {
    int E, H, I, T, K;        // K = top_k
    int GH, GI, npos;         // npos = T*K + T (shared expert positions last)
    int xg_stride;            // uint4 per position of the gathered x fragments (+64 B pad)
    int xs_stride;            // floats per position of the x group sums
    int hf_stride;            // uint4 per position of the h fragments (+64 B pad)
    int hs_stride;            // floats per position of the h group sums
    int max_tiles;
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
    d.xg_stride = d.GH * 8 + 4;
    d.xs_stride = (d.GH + 3) & ~3;
    d.hf_stride = d.GI * 16 + 4;
    d.hs_stride = (d.GI * 2 + 3) & ~3;
    d.max_tiles = (T * K + T) / TILE_T + E + 2;
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

// slot s goes to the tensor-core kernels (prefill_tc.cu)
__device__ __forceinline__ bool slot_heavy(const PrefillArgs &a, int s)
{
    return slot_count(a, s) >= a.tc_min;
}

// ------------------------------------------------------------- stage layout --
struct PfStage {
    int rows;           // rows per matrix tile
    int S;              // shared-memory row stride of a tile (words)
    int mode;           // TileMode
    size_t codes;       // bytes of one matrix tile's codes region (1024-aligned)
    size_t sb;          // bytes of one scales (or biases) array of a tile
    size_t bytes;       // one ring stage, 1024-aligned
};

__host__ __device__ inline PfStage pf_stage(int rows, int Kw, int mode, int S, int G, int nmat)
{
    PfStage st;
    st.rows = rows;
    st.S = S;
    st.mode = mode;
    st.codes = ((size_t)rows * (mode == TILE_ROWS ? S : Kw) * 4 + 1023) & ~(size_t)1023;
    st.sb = (size_t)rows * G * 2;
    st.bytes = ((size_t)nmat * (st.codes + 2 * st.sb) + 1023) & ~(size_t)1023;
    return st;
}

// barriers: ring full/empty, activation-buffer full/empty (2 each)
constexpr int PF_BARS = 2 * PF_MAX_STAGES + 4;

struct PfLayout {
    size_t bar_off, unit_off, act_off, act_bytes, stage_off, total;
};

// offsets from a 1024-byte aligned base; total includes the alignment slack
__host__ __device__ inline PfLayout pf_layout(const PfStage &st, size_t act_bytes, int NS)
{
    PfLayout L;
    size_t off = 0;
    L.bar_off = off;
    off += PF_BARS * 8;
    L.unit_off = off;
    off += (4 + PF_MAX_STAGES) * 4;   // unit id per activation buffer, abort word, pad,
                                       // then the sequence number each ring slot holds
    off = (off + 1023) & ~(size_t)1023;
    L.act_off = off;
    L.act_bytes = (act_bytes + 1023) & ~(size_t)1023;
    off += 2 * L.act_bytes;
    L.stage_off = off;
    off += (size_t)NS * st.bytes;
    L.total = off + 1024;
    return L;
}

__host__ __device__ inline size_t gu_act_bytes(const PfDims &d)
{
    return (size_t)TILE_T * d.xg_stride * 16 + (size_t)TILE_T * d.xs_stride * 4;
}
__host__ __device__ inline size_t dn_act_bytes(const PfDims &d)
{
    return (size_t)TILE_T * d.hf_stride * 16 + (size_t)TILE_T * d.hs_stride * 4;
}

// issue the copies of one matrix tile (rows [row0, row0 + st.rows) of a
// row-major [.][Kw] code array) into `dst`
__device__ __forceinline__ void issue_tile(unsigned char *dst, const PfStage &st,
                                           const CUtensorMap *map, const uint32_t *packed,
                                           size_t row0, int Kw, uint64_t *bar, uint64_t pol)
{
    const uint32_t row_bytes = (uint32_t)Kw * 4;
    if (st.mode == TILE_SWZ)
        tma_load_3d(dst, map, 0, (int)row0, 0, bar, pol);
    else if (st.mode == TILE_CONTIG)
        bulk_g2s(dst, packed + row0 * Kw, row_bytes * st.rows, bar, pol);
    else
        for (int r = 0; r < st.rows; ++r)
            bulk_g2s(dst + (size_t)r * st.S * 4, packed + (row0 + r) * Kw, row_bytes, bar, pol);
}

// h of intermediate index kidx at position pos from its gate and up values,
// stored as fp16 (hi, lo) in the fragment order of the down projection:
// [g][k half][column: 0 = hi, 1 = lo][tig][8], k order xperm(kPermS4, .)
__device__ __forceinline__ void write_h(const PrefillArgs &a, const PfDims &d, int pos, int kidx,
                                        float gv, float uv)
{
    const float h = gv / (1.f + expf(-gv)) * uv;
    const __half hh = __float2half_rn(h);
    const __half hl = __float2half_rn(h - __half2float(hh));
    __half *hf = reinterpret_cast<__half *>(a.ws.hfrag + (size_t)pos * d.hf_stride);
    const int gg = kidx >> 6, kk = kidx & 63, tg = kk >> 4;
    const int i = xperm_s4_inv(kk & 15);
    const int base = (((gg * 2 + (i >> 3)) * 2) * 4 + tg) * 8 + (i & 7);
    hf[base] = hh;
    hf[base + 4 * 8] = hl;   // column 1 is 4 uint4 (32 halves) further
}

// bounded wait that gives up at once after another thread of the CTA gave up
__device__ __forceinline__ bool pf_wait(uint64_t *bar, uint32_t parity, int32_t *status,
                                        volatile int *abort_word)
{
    if (*abort_word)
        return false;
    if (mbar_wait(bar, parity, status))
        return true;
    *abort_word = 1;
    return false;
}

// Wait until ring slot `seq_word` has been armed for ring sequence k.  A
// consumer warp may run up to two units ahead of the slowest one, i.e. more
// than a ring's length, while the slot still holds sequence k - NS; a parity
// wait on the full barrier would then see the earlier phase as complete.
__device__ __forceinline__ bool pf_wait_seq(const volatile int *seq_word, int k, int32_t *status,
                                            volatile int *abort_word)
{
    if (*seq_word == k)
        return true;
    const unsigned long long t0 = global_timer_ns();
    while (*seq_word != k) {
        if (*abort_word)
            return false;
        __nanosleep(32);
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            flag_status(status, QMOE_DEV_TIMEOUT);
            *abort_word = 1;
            return false;
        }
    }
    return true;
}

// ------------------------------------------------------------------ prep --
// grid: npos CTAs of 128 threads.  CTA p: x of position p's token, gathered
// in fragment order, and its group sums; CTA 0 also the token-tile list,
// the pair positions and the unit counters.
__global__ void __launch_bounds__(128) prefill_prep_kernel(PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const int p = blockIdx.x;
    const int nvalid = a.ws.offsets[d.E];
    if (p < nvalid || p >= d.T * d.K) {
        const int tok = pos_token(a, p);
        stage_x_groups<kPermS4>(a.ws.xfrag + (size_t)p * d.xg_stride,
                                a.ws.xsum + (size_t)p * d.xs_stride, d.GH, 1,
                                a.x + (size_t)tok * d.H, d.H, threadIdx.x, 128, 1);
        if (a.tc_min <= a.T) {
            // the tensor-core path's rows: x in the k order (0,4,1,5,2,6,3,7)
            // of every 8 inputs, its group sums as an fp16 pair, and zeroed h
            // sums (only the groups that exist are written later)
            const uint4 *src = reinterpret_cast<const uint4 *>(a.x + (size_t)tok * d.H);
            uint4 *dst = reinterpret_cast<uint4 *>(a.ws.xg + (size_t)p * d.H);
            for (int c = threadIdx.x; c < d.H / 8; c += blockDim.x) {
                const uint4 v = __ldg(src + c);
                dst[c] = make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632),
                                    __byte_perm(v.y, v.w, 0x5410), __byte_perm(v.y, v.w, 0x7632));
            }
            if (threadIdx.x < 64) {
                const int g = threadIdx.x;
                float sum = 0.f;
                if (g < d.GH)
                    for (int k = 0; k < kGroup; ++k)
                        sum += __half2float(a.x[(size_t)tok * d.H + g * kGroup + k]);
                const __half hi = __float2half_rn(sum);
                const int col = (g & ~7) | ((g & 3) << 1) | ((g & 7) >> 2);
                a.ws.xb_hi[(size_t)p * 64 + col] = hi;
                a.ws.xb_lo[(size_t)p * 64 + col] = __float2half_rn(sum - __half2float(hi));
                a.ws.hs_hi[(size_t)p * 64 + g] = __float2half(0.f);
                a.ws.hs_lo[(size_t)p * 64 + g] = __float2half(0.f);
            }
        }
    }
    if (p == 0) {
        // token tiles of every slot in slot order: a block-wide exclusive scan
        // of the per-slot tile counts, 128 slots per pass
        __shared__ int s_scan[128];
        __shared__ int s_base;
        if (threadIdx.x == 0)
            s_base = 0;
        for (int s0 = 0; s0 <= d.E; s0 += 128) {
            const int s = s0 + threadIdx.x;
            const int nt = (s <= d.E && !slot_heavy(a, s)) ? (slot_count(a, s) + TILE_T - 1) / TILE_T : 0;
            s_scan[threadIdx.x] = nt;
            __syncthreads();
            for (int o = 1; o < 128; o <<= 1) {   // inclusive Hillis-Steele scan
                const int v = threadIdx.x >= o ? s_scan[threadIdx.x - o] : 0;
                __syncthreads();
                s_scan[threadIdx.x] += v;
                __syncthreads();
            }
            const int first = s_base + s_scan[threadIdx.x] - nt;
            for (int t = 0; t < nt; ++t)
                a.ws.tiles[first + t] = (s << 4) | t;
            __syncthreads();
            if (threadIdx.x == 127)
                s_base += s_scan[127];
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            a.ws.unit_ctr[0] = 0;
            a.ws.unit_ctr[1] = 0;
            a.ws.unit_ctr[2] = s_base;
        }
        // heavy slots, most tokens first (ties: lower slot first)
        int nh = 0;
        for (int s = threadIdx.x; s <= d.E; s += blockDim.x) {
            if (!slot_heavy(a, s))
                continue;
            const int cs = slot_count(a, s);
            int rank = 0;
            for (int s2 = 0; s2 <= d.E; ++s2)
                if (slot_heavy(a, s2)) {
                    const int c2 = slot_count(a, s2);
                    rank += (c2 > cs || (c2 == cs && s2 < s)) ? 1 : 0;
                }
            a.ws.heavy[rank] = s;
            ++nh;
        }
        __shared__ int s_nh;
        if (threadIdx.x == 0)
            s_nh = 0;
        __syncthreads();
        atomicAdd(&s_nh, nh);
        __syncthreads();
        if (threadIdx.x == 0)
            a.ws.unit_ctr[3] = s_nh;
        // positions of the valid pairs (ids out of range were dropped by the
        // grouping, so only offsets[E] positions hold a pair)
        for (int q = threadIdx.x; q < nvalid; q += blockDim.x)
            a.ws.inv[a.ws.pairs[q]] = q;
    }
}

// ------------------------------------------------------ unit kernel frame --
struct UnitTile {
    int s, p0, nv;   // slot, first position, valid positions (<= 8)
};

__device__ __forceinline__ UnitTile unit_tile(const PrefillArgs &a, int i)
{
    const int tl = a.ws.tiles[i];
    UnitTile u;
    u.s = tl >> 4;
    const int t = tl & 15;
    u.p0 = slot_offset(a, u.s) + t * TILE_T;
    u.nv = min(TILE_T, slot_count(a, u.s) - t * TILE_T);
    return u;
}

// Producer of both unit kernels.  Unit u = (chunk u / ntiles, tile
// u % ntiles): tiles of one slot are consecutive, so the CTAs that take them
// read the slot's weights at about the same time (one HBM read, L2 hits).
// For each unit: the tile's activations into activation buffer (q & 1), then
// nsub(chunk) weight sub-blocks into the ring.  A unit id of -1 in an
// activation buffer tells the consumers that the queue is empty.
template <class ActCopy, class SubCopy>
__device__ __forceinline__ void unit_producer(const PrefillArgs &a, int *ctr, int nunits,
                                              int ntiles, int nsub_total, int NS,
                                              const PfStage &st, const PfLayout &L,
                                              unsigned char *smem, uint64_t *full,
                                              uint64_t *empty, uint64_t *afull, uint64_t *aempty,
                                              int *s_unit, volatile int *abort_word,
                                              ActCopy act_copy, SubCopy sub_copy)
{
    volatile int *s_seq = s_unit + 4;
    int last_use[PF_MAX_STAGES], act_last[2] = {-1, -1};
    for (int s = 0; s < PF_MAX_STAGES; ++s)
        last_use[s] = -1;
    int k = 0;
    for (int q = 0;; ++q) {
        const int b = q & 1;
        if (q >= 2 && !pf_wait(&aempty[b], ((q >> 1) - 1) & 1, a.status, abort_word))
            break;
        act_last[b] = -1;   // the buffer's previous copies were consumed
        const int u = atomicAdd(ctr, 1);
        if (u >= nunits) {
            s_unit[b] = -1;
            mbar_arrive(&afull[b]);
            break;
        }
        s_unit[b] = u;
        const int c = u / ntiles;
        const UnitTile ut = unit_tile(a, u - c * ntiles);
        act_copy(ut, smem + L.act_off + b * L.act_bytes, &afull[b]);
        act_last[b] = q >> 1;
        const int nsub = min(PF_CW, nsub_total - c * PF_CW);
        bool ok = true;
        for (int j = 0; j < nsub; ++j, ++k) {
            const int slot = k % NS, use = k / NS;
            if (use > 0 && !pf_wait(&empty[slot], (use - 1) & 1, a.status, abort_word)) {
                ok = false;
                break;
            }
            s_seq[slot] = k;   // published by the arrive that arms the barrier
            sub_copy(ut, c * PF_CW + j, smem + L.stage_off + (size_t)slot * st.bytes, &full[slot]);
            last_use[slot] = use;
        }
        if (!ok)
            break;
    }
    // no copy may still be landing when the CTA exits
    for (int s = 0; s < NS; ++s)
        if (last_use[s] >= 0)
            mbar_wait(&full[s], last_use[s] & 1, a.status);
    for (int b = 0; b < 2; ++b)
        if (act_last[b] >= 0)
            mbar_wait(&afull[b], act_last[b] & 1, a.status);
}

__device__ __forceinline__ void init_bars(uint64_t *full, uint64_t *empty, uint64_t *afull,
                                          uint64_t *aempty, int NS, int *s_unit)
{
    for (int s = 0; s < NS; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);   // one consumer warp per sub-block
    }
    for (int b = 0; b < 2; ++b) {
        mbar_init(&afull[b], 1);
        mbar_init(&aempty[b], PF_CW);
    }
    s_unit[2] = 0;   // abort word
    for (int s = 0; s < PF_MAX_STAGES; ++s)
        s_unit[4 + s] = -1;
    mbar_init_fence();
}

// ------------------------------------------------------------- gate / up --
// Sub-block o of a slot: gate rows 8o .. 8o+7 and the same up rows.  mma A
// rows (gid, gid+8) = (gate row, up row), so each C fragment holds a gate
// and an up value of one intermediate index, tokens 2tig and 2tig+1.
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_gateup_kernel(PrefillArgs a, PfStage st, int NS,
                          const __grid_constant__ CUtensorMap gate_map,
                          const __grid_constant__ CUtensorMap up_map,
                          const __grid_constant__ CUtensorMap sh_gate_map,
                          const __grid_constant__ CUtensorMap sh_up_map)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const PfLayout L = pf_layout(st, gu_act_bytes(d), NS);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + PF_MAX_STAGES, *afull = empty + PF_MAX_STAGES, *aempty = afull + 2;
    int *s_unit = reinterpret_cast<int *>(smem + L.unit_off);
    volatile int *abort_word = s_unit + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0)
        init_bars(full, empty, afull, aempty, NS, s_unit);
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    const int ntiles = a.ws.unit_ctr[2];
    const int nsub_total = d.I / GU_ROWS;
    const int nunits = ntiles * ((nsub_total + PF_CW - 1) / PF_CW);
    const int Kw = d.H / 8;
    const size_t sb_row = (size_t)d.GH;   // fp16 scales per row

    if (warp == PF_CW) {
        if (lane == 0) {
            if (st.mode == TILE_SWZ) {
                prefetch_tensormap(&gate_map);
                prefetch_tensormap(&up_map);
                prefetch_tensormap(&sh_gate_map);
                prefetch_tensormap(&sh_up_map);
            }
            const uint64_t pol = l2_evict_first_policy();
            const uint32_t sub_bytes = (uint32_t)(2 * GU_ROWS * Kw * 4 + 4 * st.sb);
            unit_producer(
                a, a.ws.unit_ctr + 0, nunits, ntiles, nsub_total, NS, st, L, smem, full, empty,
                afull, aempty, s_unit, abort_word,
                [&](const UnitTile &ut, unsigned char *dst, uint64_t *bar) {
                    const uint32_t fb = (uint32_t)ut.nv * d.xg_stride * 16;
                    const uint32_t sbb = (uint32_t)ut.nv * d.xs_stride * 4;
                    mbar_arrive_expect_tx(bar, fb + sbb);
                    bulk_g2s(dst, a.ws.xfrag + (size_t)ut.p0 * d.xg_stride, fb, bar, pol);
                    bulk_g2s(dst + (size_t)TILE_T * d.xg_stride * 16,
                             a.ws.xsum + (size_t)ut.p0 * d.xs_stride, sbb, bar, pol);
                },
                [&](const UnitTile &ut, int o, unsigned char *dst, uint64_t *bar) {
                    const bool sh = ut.s >= d.E;
                    const QMat gm = sh ? a.sh_gate : a.gate, um = sh ? a.sh_up : a.up;
                    const size_t row0 = (size_t)(sh ? 0 : ut.s) * d.I + (size_t)o * GU_ROWS;
                    mbar_arrive_expect_tx(bar, sub_bytes);
                    issue_tile(dst, st, sh ? &sh_gate_map : &gate_map, gm.packed, row0, Kw, bar,
                               pol);
                    issue_tile(dst + st.codes, st, sh ? &sh_up_map : &up_map, um.packed, row0, Kw,
                               bar, pol);
                    unsigned char *sb = dst + 2 * st.codes;
                    bulk_g2s(sb, gm.scales + row0 * sb_row, (uint32_t)st.sb, bar, pol);
                    bulk_g2s(sb + st.sb, gm.biases + row0 * sb_row, (uint32_t)st.sb, bar, pol);
                    bulk_g2s(sb + 2 * st.sb, um.scales + row0 * sb_row, (uint32_t)st.sb, bar, pol);
                    bulk_g2s(sb + 3 * st.sb, um.biases + row0 * sb_row, (uint32_t)st.sb, bar, pol);
                });
        }
        return;
    }

    // -------------------- consumers: warp j takes sub-block j of every unit
    const int gid = lane >> 2, tig = lane & 3;
    int k = 0;
    for (int q = 0;; ++q) {
        const int b = q & 1;
        // every decision below is taken by whole warps (the mma is warp-collective)
        if (!__all_sync(0xffffffffu, pf_wait(&afull[b], (q >> 1) & 1, a.status, abort_word)))
            break;
        const int u = s_unit[b];
        if (u < 0)
            break;
        const int c = u / ntiles;
        const UnitTile ut = unit_tile(a, u - c * ntiles);
        const int nsub = min(PF_CW, nsub_total - c * PF_CW);
        const unsigned char *act = smem + L.act_off + b * L.act_bytes;
        const uint4 *xf = reinterpret_cast<const uint4 *>(act);
        const float *xsm = reinterpret_cast<const float *>(act + (size_t)TILE_T * d.xg_stride * 16);
        if (warp < nsub) {
            const int kk = k + warp, slot = kk % NS;
            if (__all_sync(0xffffffffu, pf_wait_seq(s_unit + 4 + slot, kk, a.status, abort_word) &&
                                            pf_wait(&full[slot], (kk / NS) & 1, a.status, abort_word))) {
                const unsigned char *stage = smem + L.stage_off + (size_t)slot * st.bytes;
                const unsigned char *gt = stage, *utl = stage + st.codes;
                const __half *gs = reinterpret_cast<const __half *>(stage + 2 * st.codes);
                const __half *gb = gs + GU_ROWS * d.GH, *us = gb + GU_ROWS * d.GH,
                             *ub = us + GU_ROWS * d.GH;
                // column gid of the MMA is tile token gid: tokens past ut.nv read
                // whatever the tile row holds, which only reaches their own
                // columns, and those are never stored
                const uint4 *xr = xf + gid * d.xg_stride;
                const float *xs0 = xsm + (2 * tig) * d.xs_stride;
                const float *xs1 = xs0 + d.xs_stride;
                // fragment byte offsets of row gid for the 4 groups of a step of
                // 4 (GH % 4 == 0): step q4 adds q4 * cstride
                int off[4], cstride;
                if (st.mode == TILE_SWZ) {
                    cstride = GU_ROWS * 128;   // one swizzled 128-byte chunk per 4 groups
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        off[j] = gid * 128 + (((2 * j + (tig >> 1)) ^ gid) << 4) + (tig & 1) * 8;
                } else {
                    cstride = 128;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        off[j] = gid * st.S * 4 + j * 32 + tig * 8;
                }
                // code products and folded biases accumulate apart; the
                // subnormal factor kCode4 is applied once at the end
                float aq[4] = {0.f, 0.f, 0.f, 0.f}, ab[4] = {0.f, 0.f, 0.f, 0.f};
                const int nch = d.GH / 4;
                for (int q4 = 0; q4 < nch; ++q4) {
                    const unsigned char *gtc = gt + q4 * cstride, *utc = utl + q4 * cstride;
                    const uint2 sgv = *reinterpret_cast<const uint2 *>(gs + gid * d.GH + 4 * q4);
                    const uint2 bgv = *reinterpret_cast<const uint2 *>(gb + gid * d.GH + 4 * q4);
                    const uint2 suv = *reinterpret_cast<const uint2 *>(us + gid * d.GH + 4 * q4);
                    const uint2 buv = *reinterpret_cast<const uint2 *>(ub + gid * d.GH + 4 * q4);
                    const float4 X0 = *reinterpret_cast<const float4 *>(xs0 + 4 * q4);
                    const float4 X1 = *reinterpret_cast<const float4 *>(xs1 + 4 * q4);
                    const float x0s[4] = {X0.x, X0.y, X0.z, X0.w};
                    const float x1s[4] = {X1.x, X1.y, X1.z, X1.w};
                    const uint32_t sgw[2] = {sgv.x, sgv.y}, bgw[2] = {bgv.x, bgv.y};
                    const uint32_t suw[2] = {suv.x, suv.y}, buw[2] = {buv.x, buv.y};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int g = 4 * q4 + j;
                        const uint4 x0 = xr[(g * 2 + 0) * 4 + tig];
                        const uint4 x1 = xr[(g * 2 + 1) * 4 + tig];
                        float r[4];
                        mma_group_s4_1(r, *reinterpret_cast<const uint2 *>(gtc + off[j]),
                                       *reinterpret_cast<const uint2 *>(utc + off[j]), x0, x1);
                        const float2 fsg = __half22float2(u32_as_h2(sgw[j >> 1]));
                        const float2 fbg = __half22float2(u32_as_h2(bgw[j >> 1]));
                        const float2 fsu = __half22float2(u32_as_h2(suw[j >> 1]));
                        const float2 fbu = __half22float2(u32_as_h2(buw[j >> 1]));
                        const float sg = (j & 1) ? fsg.y : fsg.x, bg = (j & 1) ? fbg.y : fbg.x;
                        const float su = (j & 1) ? fsu.y : fsu.x, bu = (j & 1) ? fbu.y : fbu.x;
                        aq[0] = fmaf(sg, r[0], aq[0]);   // gate, token 2tig
                        aq[1] = fmaf(sg, r[1], aq[1]);   // gate, token 2tig+1
                        aq[2] = fmaf(su, r[2], aq[2]);   // up
                        aq[3] = fmaf(su, r[3], aq[3]);
                        ab[0] = fmaf(bg, x0s[j], ab[0]);
                        ab[1] = fmaf(bg, x1s[j], ab[1]);
                        ab[2] = fmaf(bu, x0s[j], ab[2]);
                        ab[3] = fmaf(bu, x1s[j], ab[3]);
                    }
                }
                float acc[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    acc[i] = fmaf(aq[i], kCode4, ab[i]);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[slot]);
                const int kidx = (c * PF_CW + warp) * GU_ROWS + gid;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq)
                    if (2 * tig + qq < ut.nv)
                        write_h(a, d, ut.p0 + 2 * tig + qq, kidx, acc[qq], acc[2 + qq]);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&aempty[b]);
        k += nsub;
    }
}

// ------------------------------------------------------------------ hsum --
// per position and group of I: sums of the hi and lo halves
__global__ void __launch_bounds__(256) prefill_hsum_kernel(PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const int nvalid = a.ws.offsets[d.E];
    const int n = d.npos * d.GI * 2;
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
        const int col = t & 1, pg = t >> 1;
        const int pos = pg / d.GI, g = pg - pos * d.GI;
        if (pos >= nvalid && pos < d.T * d.K)
            continue;   // no pair holds this position
        const uint4 *f = a.ws.hfrag + (size_t)pos * d.hf_stride + g * 16;
        float s = 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int tg = 0; tg < 4; ++tg) {
                const uint4 w = __ldcg(f + (hh * 2 + col) * 4 + tg);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const float2 v = __half22float2(u32_as_h2(ws[qq]));
                    s += v.x + v.y;
                }
            }
        a.ws.hsum[(size_t)pos * d.hs_stride + g * 2 + col] = s;
    }
}

// ------------------------------------------------------------------ down --
// Sub-block o of a slot: down rows 32o .. 32o+31, two 16-row mma tiles.
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_down_kernel(PrefillArgs a, PfStage st, int NS,
                        const __grid_constant__ CUtensorMap down_map,
                        const __grid_constant__ CUtensorMap sh_down_map)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const PfLayout L = pf_layout(st, dn_act_bytes(d), NS);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + PF_MAX_STAGES, *afull = empty + PF_MAX_STAGES, *aempty = afull + 2;
    int *s_unit = reinterpret_cast<int *>(smem + L.unit_off);
    volatile int *abort_word = s_unit + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0)
        init_bars(full, empty, afull, aempty, NS, s_unit);
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    const int ntiles = a.ws.unit_ctr[2];
    const int nsub_total = d.H / DN_ROWS;
    const int nunits = ntiles * ((nsub_total + PF_CW - 1) / PF_CW);
    const int Kw = d.I / 8;
    const size_t sb_row = (size_t)d.GI;

    if (warp == PF_CW) {
        if (lane == 0) {
            if (st.mode == TILE_SWZ) {
                prefetch_tensormap(&down_map);
                prefetch_tensormap(&sh_down_map);
            }
            const uint64_t pol = l2_evict_first_policy();
            const uint32_t sub_bytes = (uint32_t)(DN_ROWS * Kw * 4 + 2 * st.sb);
            unit_producer(
                a, a.ws.unit_ctr + 1, nunits, ntiles, nsub_total, NS, st, L, smem, full, empty,
                afull, aempty, s_unit, abort_word,
                [&](const UnitTile &ut, unsigned char *dst, uint64_t *bar) {
                    const uint32_t fb = (uint32_t)ut.nv * d.hf_stride * 16;
                    const uint32_t sbb = (uint32_t)ut.nv * d.hs_stride * 4;
                    mbar_arrive_expect_tx(bar, fb + sbb);
                    bulk_g2s(dst, a.ws.hfrag + (size_t)ut.p0 * d.hf_stride, fb, bar, pol);
                    bulk_g2s(dst + (size_t)TILE_T * d.hf_stride * 16,
                             a.ws.hsum + (size_t)ut.p0 * d.hs_stride, sbb, bar, pol);
                },
                [&](const UnitTile &ut, int o, unsigned char *dst, uint64_t *bar) {
                    const bool sh = ut.s >= d.E;
                    const QMat dm = sh ? a.sh_down : a.down;
                    const size_t row0 = (size_t)(sh ? 0 : ut.s) * d.H + (size_t)o * DN_ROWS;
                    mbar_arrive_expect_tx(bar, sub_bytes);
                    issue_tile(dst, st, sh ? &sh_down_map : &down_map, dm.packed, row0, Kw, bar,
                               pol);
                    bulk_g2s(dst + st.codes, dm.scales + row0 * sb_row, (uint32_t)st.sb, bar, pol);
                    bulk_g2s(dst + st.codes + st.sb, dm.biases + row0 * sb_row, (uint32_t)st.sb,
                             bar, pol);
                });
        }
        return;
    }

    const int gid = lane >> 2, tig = lane & 3;
    int k = 0;
    for (int q = 0;; ++q) {
        const int b = q & 1;
        // every decision below is taken by whole warps (the mma is warp-collective)
        if (!__all_sync(0xffffffffu, pf_wait(&afull[b], (q >> 1) & 1, a.status, abort_word)))
            break;
        const int u = s_unit[b];
        if (u < 0)
            break;
        const int c = u / ntiles;
        const UnitTile ut = unit_tile(a, u - c * ntiles);
        const int nsub = min(PF_CW, nsub_total - c * PF_CW);
        const unsigned char *act = smem + L.act_off + b * L.act_bytes;
        const uint4 *hb = reinterpret_cast<const uint4 *>(act);
        const float *hsm = reinterpret_cast<const float *>(act + (size_t)TILE_T * d.hf_stride * 16);
        if (warp < nsub) {
            const int kk = k + warp, slot = kk % NS;
            if (__all_sync(0xffffffffu, pf_wait_seq(s_unit + 4 + slot, kk, a.status, abort_word) &&
                                            pf_wait(&full[slot], (kk / NS) & 1, a.status, abort_word))) {
                const unsigned char *wt = smem + L.stage_off + (size_t)slot * st.bytes;
                const __half *sc = reinterpret_cast<const __half *>(wt + st.codes);
                const __half *bi = sc + DN_ROWS * d.GI;
                // as in the gate/up kernel: columns of tokens past ut.nv are
                // computed from whatever their tile rows hold and never stored
                const uint4 *hr = hb + gid * d.hf_stride;
                const float *hs0 = hsm + (2 * tig) * d.hs_stride;
                const float *hs1 = hs0 + d.hs_stride;
                // rows gid, gid+8, gid+16, gid+24 share (r & 7) = gid
                const bool swz = st.mode == TILE_SWZ;
                int rowoff[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    rowoff[i] = swz ? (gid + 8 * i) * 128 + (tig & 1) * 8
                                    : (gid + 8 * i) * st.S * 4 + tig * 8;
                float aq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                float ab[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int g = 0; g < d.GI; ++g) {
                    const uint4 h0 = hr[((g * 2 + 0) * 2 + 0) * 4 + tig];
                    const uint4 h1 = hr[((g * 2 + 1) * 2 + 0) * 4 + tig];
                    const uint4 l0 = hr[((g * 2 + 0) * 2 + 1) * 4 + tig];
                    const uint4 l1 = hr[((g * 2 + 1) * 2 + 1) * 4 + tig];
                    const float2 S0 = *reinterpret_cast<const float2 *>(hs0 + g * 2);
                    const float2 S1 = *reinterpret_cast<const float2 *>(hs1 + g * 2);
                    const float X0 = S0.x + S0.y, X1 = S1.x + S1.y;
                    const int goff = swz ? (g >> 2) * (DN_ROWS * 128) +
                                               (((2 * (g & 3) + (tig >> 1)) ^ gid) << 4)
                                         : g * 32;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int ra = half * 16 + gid, rb = ra + 8;
                        float r[4];
                        mma_group_s4_hilo(
                            r, *reinterpret_cast<const uint2 *>(wt + rowoff[2 * half] + goff),
                            *reinterpret_cast<const uint2 *>(wt + rowoff[2 * half + 1] + goff), h0,
                            h1, l0, l1);
                        const float sa = __half2float(sc[ra * d.GI + g]);
                        const float ba = __half2float(bi[ra * d.GI + g]);
                        const float sb = __half2float(sc[rb * d.GI + g]);
                        const float bb = __half2float(bi[rb * d.GI + g]);
                        aq[4 * half + 0] = fmaf(sa, r[0], aq[4 * half + 0]);
                        aq[4 * half + 1] = fmaf(sa, r[1], aq[4 * half + 1]);
                        aq[4 * half + 2] = fmaf(sb, r[2], aq[4 * half + 2]);
                        aq[4 * half + 3] = fmaf(sb, r[3], aq[4 * half + 3]);
                        ab[4 * half + 0] = fmaf(ba, X0, ab[4 * half + 0]);
                        ab[4 * half + 1] = fmaf(ba, X1, ab[4 * half + 1]);
                        ab[4 * half + 2] = fmaf(bb, X0, ab[4 * half + 2]);
                        ab[4 * half + 3] = fmaf(bb, X1, ab[4 * half + 3]);
                    }
                }
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    acc[i] = fmaf(aq[i], kCode4, ab[i]);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[slot]);
                const int row0 = (c * PF_CW + warp) * DN_ROWS + gid;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const int pq = 2 * tig + qq;
                    if (pq < ut.nv) {
                        float *r = a.ws.r + (size_t)(ut.p0 + pq) * d.H + row0;
                        r[0] = acc[qq];
                        r[8] = acc[2 + qq];
                        r[16] = acc[4 + qq];
                        r[24] = acc[6 + qq];
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&aempty[b]);
        k += nsub;
    }
}

// --------------------------------------------------------------- combine --
// four consecutive outputs of one token per thread (H % 4 == 0)
__global__ void __launch_bounds__(256) prefill_combine_kernel(PrefillArgs a)
{
    pdl_wait();
    pdl_trigger();
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
    const int H4 = d.H / 4;
    const int n = d.T * H4;
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
        const int tok = t / H4, c4 = t - tok * H4;
        float4 y = __ldcg(reinterpret_cast<const float4 *>(a.ws.r + (size_t)(d.T * d.K + tok) * d.H) +
                          c4);
        for (int j = 0; j < d.K; ++j) {
            const int e = a.idx[tok * d.K + j];
            if (e < 0 || e >= d.E)
                continue;   // flagged by the grouping kernel, contributes nothing
            const int p = a.ws.inv[tok * d.K + j];
            const float w = a.weights[tok * d.K + j];
            const float4 r = __ldcg(reinterpret_cast<const float4 *>(a.ws.r + (size_t)p * d.H) + c4);
            y.x = fmaf(w, r.x, y.x);
            y.y = fmaf(w, r.y, y.y);
            y.z = fmaf(w, r.z, y.z);
            y.w = fmaf(w, r.w, y.w);
        }
        __half2 *out = reinterpret_cast<__half2 *>(a.y + (size_t)tok * d.H) + 2 * c4;
        out[0] = __floats2half2_rn(y.x, y.y);
        out[1] = __floats2half2_rn(y.z, y.w);
    }
}

// tile mode and stride for rows of K 4-bit codes; `map_ok`: tensor maps encoded
PfStage choose_stage(int rows, int K, int nmat, bool map_ok)
{
    const int Kw = K / 8, G = K / kGroup;
    const int m = Kw & 31;
    if (m == 8 || m == 24)
        return pf_stage(rows, Kw, TILE_CONTIG, Kw, G, nmat);
    if (m == 0 && map_ok)
        return pf_stage(rows, Kw, TILE_SWZ, Kw, G, nmat);
    return pf_stage(rows, Kw, TILE_ROWS, tile_stride_words(K, 4), G, nmat);
}

int stages_for(const PfStage &st, size_t act_bytes)
{
    const size_t budget = 227 * 1024;
    const PfLayout L0 = pf_layout(st, act_bytes, 0);
    if (L0.total + 2 * st.bytes > budget)
        return 0;
    const int NS = (int)((budget - L0.total) / st.bytes);
    return NS > PF_MAX_STAGES ? PF_MAX_STAGES : NS;
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
    const size_t tiles_off = take((size_t)d.max_tiles * 4);
    const size_t ctr_off = take(4 * 4);
    const size_t xfrag_off = take((size_t)d.npos * d.xg_stride * 16);
    const size_t xsum_off = take((size_t)d.npos * d.xs_stride * 4);
    const size_t hfrag_off = take((size_t)d.npos * d.hf_stride * 16);
    const size_t hsum_off = take((size_t)d.npos * d.hs_stride * 4);
    const size_t r_off = take((size_t)d.npos * H * 4);
    const size_t heavy_off = take((size_t)(E + 1) * 4);
    const size_t xg_off = take((size_t)d.npos * H * 2);
    const size_t xb_off = take((size_t)d.npos * 64 * 2 * 2);
    const size_t hb_off = take((size_t)d.npos * I * 2 * 2);
    const size_t hs_off = take((size_t)d.npos * 64 * 2 * 2);
    const size_t tcpart_off = take((size_t)kTcMaxCtas * kTcPartBytes);
    if (base && ws) {
        unsigned char *b = static_cast<unsigned char *>(base);
        ws->counts = reinterpret_cast<int32_t *>(b + counts_off);
        ws->offsets = reinterpret_cast<int32_t *>(b + offsets_off);
        ws->pairs = reinterpret_cast<int32_t *>(b + pairs_off);
        ws->inv = reinterpret_cast<int32_t *>(b + inv_off);
        ws->tiles = reinterpret_cast<int32_t *>(b + tiles_off);
        ws->unit_ctr = reinterpret_cast<int32_t *>(b + ctr_off);
        ws->xfrag = reinterpret_cast<uint4 *>(b + xfrag_off);
        ws->xsum = reinterpret_cast<float *>(b + xsum_off);
        ws->hfrag = reinterpret_cast<uint4 *>(b + hfrag_off);
        ws->hsum = reinterpret_cast<float *>(b + hsum_off);
        ws->r = reinterpret_cast<float *>(b + r_off);
        ws->heavy = reinterpret_cast<int32_t *>(b + heavy_off);
        ws->xg = reinterpret_cast<__half *>(b + xg_off);
        ws->xb_hi = reinterpret_cast<__half *>(b + xb_off);
        ws->xb_lo = ws->xb_hi + (size_t)d.npos * 64;
        ws->hb_hi = reinterpret_cast<__half *>(b + hb_off);
        ws->hb_lo = ws->hb_hi + (size_t)d.npos * I;
        ws->hs_hi = reinterpret_cast<__half *>(b + hs_off);
        ws->hs_lo = ws->hs_hi + (size_t)d.npos * 64;
        ws->tcpart = reinterpret_cast<float *>(b + tcpart_off);
    }
    return off;
}

bool prefill_shape_supported(int H, int I)
{
    const PfDims d = pf_dims(1, H, I, 128, 16);
    return H % 256 == 0 && I % GU_ROWS == 0 &&
           stages_for(choose_stage(GU_ROWS, H, 2, false), gu_act_bytes(d)) >= 2 &&
           stages_for(choose_stage(DN_ROWS, I, 1, false), dn_act_bytes(d)) >= 2;
}

cudaError_t launch_prefill(const PrefillArgs &a, const LaunchCfg &c)
{
    cudaError_t e;
    const PfDims d = pf_dims(a.E, a.H, a.I, a.T, a.top_k);
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
    if ((e = launch_ex(prefill_prep_kernel, dim3(d.npos), dim3(128), 0, c, 1, a)) != cudaSuccess)
        return e;

    // gate / up: tensor maps (8-row boxes) over the stacked routed matrices
    // and the shared ones
    CUtensorMap mg, mu, msg, msu;
    memset(&mg, 0, sizeof(mg));
    memset(&mu, 0, sizeof(mu));
    memset(&msg, 0, sizeof(msg));
    memset(&msu, 0, sizeof(msu));
    const int Kw_gu = a.H / 8, Kw_dn = a.I / 8;
    bool ok = (Kw_gu & 31) == 0;
    ok = ok && encode_codes_map(&mg, a.gate.packed, (long)a.E * a.I, Kw_gu, GU_ROWS);
    ok = ok && encode_codes_map(&mu, a.up.packed, (long)a.E * a.I, Kw_gu, GU_ROWS);
    ok = ok && encode_codes_map(&msg, a.sh_gate.packed, a.I, Kw_gu, GU_ROWS);
    ok = ok && encode_codes_map(&msu, a.sh_up.packed, a.I, Kw_gu, GU_ROWS);
    const PfStage sgu = choose_stage(GU_ROWS, a.H, 2, ok);
    const int ns_gu = stages_for(sgu, gu_act_bytes(d));
    if (ns_gu < 2)
        return cudaErrorInvalidValue;
    const size_t smem_gu = pf_layout(sgu, gu_act_bytes(d), ns_gu).total;
    if ((e = set_smem(prefill_gateup_kernel, smem_gu)) != cudaSuccess)
        return e;
    if ((e = launch_ex(prefill_gateup_kernel, dim3(c.num_sms), dim3(PF_THREADS), smem_gu, c, 1, a,
                       sgu, ns_gu, mg, mu, msg, msu)) != cudaSuccess)
        return e;
    const bool tc = a.tc_min <= a.T;
    if (tc && (e = launch_prefill_tc(a, c, false)) != cudaSuccess)
        return e;
    if ((e = launch_ex(prefill_hsum_kernel, dim3(c.num_sms), dim3(256), 0, c, 1, a)) != cudaSuccess)
        return e;

    CUtensorMap md, msd;
    memset(&md, 0, sizeof(md));
    memset(&msd, 0, sizeof(msd));
    bool okd = (Kw_dn & 31) == 0;
    okd = okd && encode_codes_map(&md, a.down.packed, (long)a.E * a.H, Kw_dn, DN_ROWS);
    okd = okd && encode_codes_map(&msd, a.sh_down.packed, a.H, Kw_dn, DN_ROWS);
    const PfStage sdn = choose_stage(DN_ROWS, a.I, 1, okd);
    const int ns_dn = stages_for(sdn, dn_act_bytes(d));
    if (ns_dn < 2)
        return cudaErrorInvalidValue;
    const size_t smem_dn = pf_layout(sdn, dn_act_bytes(d), ns_dn).total;
    if ((e = set_smem(prefill_down_kernel, smem_dn)) != cudaSuccess)
        return e;
    if ((e = launch_ex(prefill_down_kernel, dim3(c.num_sms), dim3(PF_THREADS), smem_dn, c, 1, a,
                       sdn, ns_dn, md, msd)) != cudaSuccess)
        return e;
    if (tc && (e = launch_prefill_tc(a, c, true)) != cudaSuccess)
        return e;
    return launch_ex(prefill_combine_kernel, dim3(c.num_sms * 2), dim3(256), 0, c, 1, a);
}

}  // namespace qmoe
