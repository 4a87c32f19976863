// router.cu -- MoE router: affine-quantized router GEMV -> fp32 logits ->
// top-k (ties: lower expert index first) -> weights renormalised over the
// selected experts.
//
// TurboFieldfare article (jeff.news), section "내부 구조가 진짜 흥미로운 부분"
// (internal structure): each layer's router runs on the GPU from resident
// weights and selects the top-8 experts; section "성능과 제약": the router is
// 8-bit affine, group 64.  Softmax followed by renormalisation over the
// selected experts equals exp(l_j - l_max) / sum_{j' selected} exp(l_j' - l_max).
//
// Design (B200): one thread-block cluster per block of 8 tokens; CTA r of the
// cluster owns router rows [16r, 16r+16).  Each CTA streams its 16-row tile
// with cp.async.bulk (before the previous kernel has finished: the weights
// are parameters), computes its logits with the register-dequant mma.sync
// tile (tokens as the N=8 dimension), and keeps them in shared memory.  After
// a cluster barrier, CTA 0 reads all logits through distributed shared memory
// and one warp per token selects the top-k with warp shuffles.
#include "common.cuh"
#include "kernels.h"

namespace qmoe {
namespace {

constexpr int RT_CW = 8;
constexpr int RT_THREADS = (RT_CW + 1) * 32;
constexpr int RT_TOKENS = 8;   // tokens per cluster (the mma N dimension)

struct RtLayout {
    int G, S;
    size_t xs_off, xsum_off, red_off, lg_off, bar_off, tile_off, codes_bytes, sb_bytes, total;
};

__host__ __device__ inline RtLayout rt_layout(int K, int bits)
{
    RtLayout L;
    L.G = K / kGroup;
    L.S = tile_stride_words(K, bits);
    size_t off = 0;
    L.xs_off = off;
    off += (size_t)L.G * 2 * RT_TOKENS * 4 * 16;
    L.xsum_off = off;
    off += (size_t)L.G * 8 * 4;
    off = (off + 15) & ~(size_t)15;
    L.red_off = off;
    off += RT_CW * 32 * 16;
    L.lg_off = off;
    off += 16 * RT_TOKENS * 4;
    L.bar_off = off;
    off += 16;
    off = (off + 127) & ~(size_t)127;
    L.tile_off = off;
    L.codes_bytes = (size_t)16 * L.S * 4;
    L.sb_bytes = (size_t)16 * L.G * 2;
    off += L.codes_bytes + 2 * L.sb_bytes;
    L.total = off;
    return L;
}

__device__ __forceinline__ float ld_dsmem_f32(const float *local, uint32_t rank)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

template <int BITS>
__global__ void __launch_bounds__(RT_THREADS, 1) router_kernel(RouterArgs a, int CL)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const RtLayout L = rt_layout(a.K, BITS);
    uint4 *xs = reinterpret_cast<uint4 *>(smem + L.xs_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    float4 *red = reinterpret_cast<float4 *>(smem + L.red_off);
    float *lg = reinterpret_cast<float *>(smem + L.lg_off);   // [16 rows][8 tokens]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    unsigned char *tile_base = smem + L.tile_off;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = blockIdx.x % CL;
    const int t0 = (blockIdx.x / CL) * RT_TOKENS;
    const int nt = min(RT_TOKENS, a.T - t0);
    const int r0 = rank * 16;
    const int rows = max(0, min(16, a.E - r0));
    const int Kw = a.K * BITS / 32;

    if (threadIdx.x == 0) {
        mbar_init(full, 1);
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == RT_CW) {
        if (lane == 0 && rows > 0) {
            const uint32_t row_bytes = (uint32_t)Kw * 4;
            const uint32_t sb = (uint32_t)(rows * L.G * 2);
            const uint64_t pol = l2_evict_first_policy();
            mbar_arrive_expect_tx(full, rows * row_bytes + 2 * sb);
            for (int r = 0; r < rows; ++r)
                bulk_g2s(tile_base + (size_t)r * L.S * 4, a.packed + (size_t)(r0 + r) * Kw, row_bytes,
                         full, pol);
            bulk_g2s(tile_base + L.codes_bytes, a.scales + (size_t)r0 * L.G, sb, full, pol);
            bulk_g2s(tile_base + L.codes_bytes + L.sb_bytes, a.biases + (size_t)r0 * L.G, sb, full,
                     pol);
            mbar_wait(full, 0, a.status);   // nothing may land after the CTA exits
        }
    } else {
        pdl_wait();
        pdl_trigger();
        const __half *x = a.x + (size_t)t0 * a.K;
        const int K = a.K;
        stage_x<BITS>(xs, xsum, L.G, nt, 1,
                      [&](int, int n, int k) { return __half2float(x[n * K + k]); }, threadIdx.x,
                      RT_CW * 32);
        named_bar_sync(1, RT_CW * 32);
        const int gid = lane >> 2, tig = lane & 3;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        // the lanes of a warp decide together: the mma below is warp-collective
        if (__all_sync(0xffffffffu, rows > 0 && mbar_wait(full, 0, a.status))) {
            const uint32_t *tile = reinterpret_cast<const uint32_t *>(tile_base);
            const __half *sc = reinterpret_cast<const __half *>(tile_base + L.codes_bytes);
            const __half *bi = reinterpret_cast<const __half *>(tile_base + L.codes_bytes + L.sb_bytes);
            for (int g = warp; g < L.G; g += RT_CW)
                tile_group<BITS>(tile, L.S, sc, bi, L.G, xs, xsum, nt, g, gid, tig, acc);
        }
        red[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        named_bar_sync(1, RT_CW * 32);
        if (warp == 0) {
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            for (int w = 0; w < RT_CW; ++w) {
                const float4 p = red[w * 32 + lane];
                v[0] += p.x;
                v[1] += p.y;
                v[2] += p.z;
                v[3] += p.w;
            }
            const int c0 = 2 * tig;
            lg[gid * RT_TOKENS + c0] = v[0];
            lg[gid * RT_TOKENS + c0 + 1] = v[1];
            lg[(gid + 8) * RT_TOKENS + c0] = v[2];
            lg[(gid + 8) * RT_TOKENS + c0 + 1] = v[3];
            if (a.logits) {
                const int rr[4] = {gid, gid, gid + 8, gid + 8};
                const int cc[4] = {c0, c0 + 1, c0, c0 + 1};
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (rr[i] < rows && cc[i] < nt)
                        a.logits[(size_t)(t0 + cc[i]) * a.E + r0 + rr[i]] = v[i];
            }
        }
    }

    cluster_sync_all();   // every CTA's logits are in its shared memory

    if (rank == 0 && warp < nt) {
        // one warp per token: expert e = lane + 32 q, q < 4 (E <= 128)
        const int t = t0 + warp;
        float v[4];
        bool taken[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = lane + 32 * q;
            taken[q] = e >= a.E;
            v[q] = taken[q] ? 0.f : ld_dsmem_f32(lg + (e & 15) * RT_TOKENS + warp, (uint32_t)(e >> 4));
        }
        float my_v = 0.f;
        int my_i = -1;
        for (int j = 0; j < a.top_k; ++j) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = lane + 32 * q;
                if (!taken[q] && (v[q] > bv || (v[q] == bv && e < bi))) {
                    bv = v[q];
                    bi = e;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                if (ov > bv || (ov == bv && oi < bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            if (bi >= 0 && bi < a.E && (bi & 31) == lane)
                taken[bi >> 5] = true;
            if (lane == j) {
                my_v = bv;
                my_i = bi;
            }
        }
        const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
        float ex = lane < a.top_k ? expf(my_v - vmax) : 0.f;
        float sum = ex;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane < a.top_k) {
            a.idx[(size_t)t * a.top_k + lane] = my_i;
            a.weights[(size_t)t * a.top_k + lane] = ex / sum;
        }
    }

    cluster_sync_all();   // keep shared memory alive until CTA 0 has read it
}

}  // namespace

cudaError_t launch_router(const RouterArgs &a, const LaunchCfg &c)
{
    const RtLayout L = rt_layout(a.K, a.bits);
    if (L.total > 227 * 1024)
        return cudaErrorInvalidValue;
    const int CL = (a.E + 15) / 16;
    const int nblk = (a.T + RT_TOKENS - 1) / RT_TOKENS;
    cudaError_t e;
    if (a.bits == 4) {
        if ((e = set_smem(router_kernel<4>, L.total)) != cudaSuccess)
            return e;
        return launch_ex(router_kernel<4>, dim3(CL * nblk), dim3(RT_THREADS), L.total, c, CL, a, CL);
    }
    if ((e = set_smem(router_kernel<8>, L.total)) != cudaSuccess)
        return e;
    return launch_ex(router_kernel<8>, dim3(CL * nblk), dim3(RT_THREADS), L.total, c, CL, a, CL);
}

}  // namespace qmoe
