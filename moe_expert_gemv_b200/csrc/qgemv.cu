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
// weight tiles (codes + scales + biases) with cp.async.bulk into a ring of
// shared-memory stages tracked by mbarriers; eight consumer warps split the
// tile's 64-wide groups, dequantise codes to exact fp16 integers in registers
// and run mma.sync m16n8k16 with the batch as the N=8 dimension; scale and
// bias are applied per group in fp32; partial tiles are reduced through
// shared memory and written as fp16.
#include "common.cuh"
#include "kernels.h"

namespace qmoe {
namespace {

constexpr int QG_CW = 8;                      // consumer warps
constexpr int QG_THREADS = (QG_CW + 1) * 32;  // + one producer warp
constexpr int QG_MAX_STAGES = 8;

struct QgLayout {
    int G, S;
    size_t xs_off, xsum_off, red_off, bar_off, stage_off;
    size_t codes_bytes, sb_bytes, stage_bytes, total;
};

__host__ __device__ inline QgLayout qg_layout(int K, int bits, int ncol, int NS)
{
    QgLayout L;
    L.G = K / kGroup;
    L.S = tile_stride_words(K, bits);
    size_t off = 0;
    L.xs_off = off;
    off += (size_t)L.G * 2 * ncol * 4 * 16;
    L.xsum_off = off;
    off += (size_t)L.G * 8 * 4;
    off = (off + 15) & ~(size_t)15;
    L.red_off = off;
    off += 2 * QG_CW * 32 * 16;
    L.bar_off = off;
    off += 2 * QG_MAX_STAGES * 8;
    off = (off + 127) & ~(size_t)127;
    L.stage_off = off;
    L.codes_bytes = (size_t)16 * L.S * 4;
    L.sb_bytes = (size_t)16 * L.G * 2;
    L.stage_bytes = L.codes_bytes + 2 * L.sb_bytes;
    off += (size_t)NS * L.stage_bytes;
    L.total = off;
    return L;
}

template <int BITS>
__global__ void __launch_bounds__(QG_THREADS, 1) qgemv_kernel(QgemvArgs a, int NS)
{
    extern __shared__ __align__(128) unsigned char smem[];
    const QgLayout L = qg_layout(a.K, BITS, a.B, NS);
    uint4 *xs = reinterpret_cast<uint4 *>(smem + L.xs_off);
    float *xsum = reinterpret_cast<float *>(smem + L.xsum_off);
    float4 *red = reinterpret_cast<float4 *>(smem + L.red_off);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bar_off);
    uint64_t *empty = full + QG_MAX_STAGES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = (a.N + 15) / 16;
    const int Kw = a.K * BITS / 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], QG_CW);
        }
        mbar_init_fence();
    }
    __syncthreads();

    if (warp == QG_CW) {
        // ---------------- producer: weights are parameters, so they may be
        // streamed before the previous kernel of the stream has finished.
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            int k = 0;
            int last_use[QG_MAX_STAGES];
            for (int s = 0; s < QG_MAX_STAGES; ++s)
                last_use[s] = -1;
            for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++k) {
                const int st = k % NS, use = k / NS;
                if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, a.status))
                    break;
                const int r0 = item * 16;
                const int rows = min(16, a.N - r0);
                const uint32_t row_bytes = (uint32_t)Kw * 4;
                const uint32_t sb = (uint32_t)(rows * L.G * 2);
                unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
                mbar_arrive_expect_tx(&full[st], rows * row_bytes + 2 * sb);
                for (int r = 0; r < rows; ++r)
                    bulk_g2s(stage + (size_t)r * L.S * 4, a.packed + (size_t)(r0 + r) * Kw,
                             row_bytes, &full[st], pol);
                bulk_g2s(stage + L.codes_bytes, a.scales + (size_t)r0 * L.G, sb, &full[st], pol);
                bulk_g2s(stage + L.codes_bytes + L.sb_bytes, a.biases + (size_t)r0 * L.G, sb,
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

    // -------------------- consumers
    pdl_wait();
    pdl_trigger();
    const int ctid = threadIdx.x;
    const __half *x = a.x;
    const int K = a.K;
    stage_x<BITS>(xs, xsum, L.G, a.B, 1,
                  [&](int, int n, int k) { return __half2float(x[n * K + k]); }, ctid, QG_CW * 32);
    named_bar_sync(1, QG_CW * 32);

    const int gid = lane >> 2, tig = lane & 3;
    bool failed = false;
    int k = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++k) {
        const int st = k % NS, use = k / NS;
        if (!failed && !mbar_wait(&full[st], use & 1, a.status))
            failed = true;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (!failed) {
            const unsigned char *stage = smem + L.stage_off + (size_t)st * L.stage_bytes;
            const uint32_t *tile = reinterpret_cast<const uint32_t *>(stage);
            const __half *sc = reinterpret_cast<const __half *>(stage + L.codes_bytes);
            const __half *bi = reinterpret_cast<const __half *>(stage + L.codes_bytes + L.sb_bytes);
            for (int g = warp; g < L.G; g += QG_CW)
                tile_group<BITS>(tile, L.S, sc, bi, L.G, xs, xsum, a.B, g, gid, tig, acc);
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[st]);
        red[((k & 1) * QG_CW + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        named_bar_sync(1, QG_CW * 32);
        if (warp == k % QG_CW) {
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            for (int w = 0; w < QG_CW; ++w) {
                const float4 p = red[((k & 1) * QG_CW + w) * 32 + lane];
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

}  // namespace

cudaError_t launch_qgemv(const QgemvArgs &a, const LaunchCfg &c)
{
    const size_t budget = 227 * 1024;
    const QgLayout L0 = qg_layout(a.K, a.bits, a.B, 0);
    if (L0.total + 2 * L0.stage_bytes > budget)
        return cudaErrorInvalidValue;
    int NS = (int)((budget - L0.total) / L0.stage_bytes);
    NS = NS > QG_MAX_STAGES ? QG_MAX_STAGES : NS;
    const QgLayout L = qg_layout(a.K, a.bits, a.B, NS);
    const int n_items = (a.N + 15) / 16;
    const int grid = n_items < c.num_sms ? n_items : c.num_sms;
    cudaError_t e;
    if (a.bits == 4) {
        if ((e = set_smem(qgemv_kernel<4>, L.total)) != cudaSuccess)
            return e;
        return launch_ex(qgemv_kernel<4>, dim3(grid), dim3(QG_THREADS), L.total, c, 1, a, NS);
    }
    if ((e = set_smem(qgemv_kernel<8>, L.total)) != cudaSuccess)
        return e;
    return launch_ex(qgemv_kernel<8>, dim3(grid), dim3(QG_THREADS), L.total, c, 1, a, NS);
}

}  // namespace qmoe
