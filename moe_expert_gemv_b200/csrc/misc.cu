// misc.cu -- packing helpers and the prefill grouping kernel.
//
// Packing follows the MLX affine layout named in the TurboFieldfare article
// (jeff.news, section "성능과 제약"): code k of a row in word k/(32/bits),
// bits*(k % (32/bits)) from the least significant end.
//
// Grouping: a prefill chunk's (token, slot) pairs listed per expert so that
// one fetched expert serves every row routed to it (same article, section
// "내부 구조가 진짜 흥미로운 부분": prefill in chunks of at most 128 tokens).
#include "common.cuh"
#include "kernels.h"

namespace qmoe {
namespace {

__global__ void pack_kernel(const uint8_t *codes, int rows, int cols, int bits, uint32_t *packed)
{
    const int per = 32 / bits;
    const long long words = (long long)rows * (cols / per);
    const uint32_t mask = (1u << bits) - 1u;
    for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < words;
         w += (long long)gridDim.x * blockDim.x) {
        const uint8_t *c = codes + w * per;
        uint32_t v = 0;
        for (int j = 0; j < per; ++j)
            v |= ((uint32_t)c[j] & mask) << (bits * j);
        packed[w] = v;
    }
}

__global__ void unpack_kernel(const uint32_t *packed, int rows, int cols, int bits, uint8_t *codes)
{
    const int per = 32 / bits;
    const long long words = (long long)rows * (cols / per);
    const uint32_t mask = (1u << bits) - 1u;
    for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < words;
         w += (long long)gridDim.x * blockDim.x) {
        const uint32_t v = packed[w];
        for (int j = 0; j < per; ++j)
            codes[w * per + j] = (uint8_t)((v >> (bits * j)) & mask);
    }
}

// One CTA of 1024 threads; warp w owns pairs [32w, 32w+32) of each 1024-pair
// round.  Stable order comes from: (a) per-warp counts of each expert,
// prefix-summed over warps in pair order, and (b) the rank of a lane among the
// lanes of its warp holding the same expert (__match_any_sync).
constexpr int GR_THREADS = 1024;

__global__ void __launch_bounds__(GR_THREADS) group_kernel(GroupArgs a)
{
    extern __shared__ int gsm[];
    const int n = a.T * a.top_k;
    const int nw = (n + 31) / 32;           // warp chunks in pair order
    int *cnt = gsm;                          // [nw][E]
    int *off = gsm + nw * a.E;               // [E + 1]
    pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i < nw * a.E; i += blockDim.x)
        cnt[i] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    // pass 1: per-chunk counts
    for (int base = 0; base < n; base += GR_THREADS) {
        const int i = base + threadIdx.x;
        const int chunk = i >> 5;
        int e = -1;
        if (i < n) {
            e = a.idx[i];
            if (e < 0 || e >= a.E) {
                flag_status(a.status, QMOE_DEV_BAD_EXPERT);
                e = -1;
            }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (peers & lt) == 0)
            cnt[chunk * a.E + e] = __popc(peers);
    }
    __syncthreads();
    // exclusive prefix over chunks, per expert; totals
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = 0;
        for (int c = 0; c < nw; ++c) {
            const int t = cnt[c * a.E + e];
            cnt[c * a.E + e] = run;
            run += t;
        }
        off[e + 1] = run;
        a.counts[e] = run;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        off[0] = 0;
        for (int e = 0; e < a.E; ++e)
            off[e + 1] += off[e];
    }
    __syncthreads();
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x)
        a.offsets[e] = off[e];
    // pass 2: scatter
    for (int base = 0; base < n; base += GR_THREADS) {
        const int i = base + threadIdx.x;
        const int chunk = i >> 5;
        int e = -1;
        if (i < n) {
            e = a.idx[i];
            if (e < 0 || e >= a.E)
                e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0)
            a.pairs[off[e] + cnt[chunk * a.E + e] + __popc(peers & lt)] = i;
    }
}

}  // namespace

cudaError_t launch_pack(const uint8_t *codes, int rows, int cols, int bits, uint32_t *packed,
                        cudaStream_t s)
{
    const long long words = (long long)rows * (cols * bits / 32);
    const int grid = (int)((words + 255) / 256 < 65535 ? (words + 255) / 256 : 65535);
    pack_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(codes, rows, cols, bits, packed);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const uint32_t *packed, int rows, int cols, int bits, uint8_t *codes,
                          cudaStream_t s)
{
    const long long words = (long long)rows * (cols * bits / 32);
    const int grid = (int)((words + 255) / 256 < 65535 ? (words + 255) / 256 : 65535);
    unpack_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(packed, rows, cols, bits, codes);
    return cudaGetLastError();
}

size_t group_smem_bytes(int n, int E) { return ((size_t)((n + 31) / 32) * E + E + 1) * 4; }

cudaError_t launch_group(const GroupArgs &a, const LaunchCfg &c)
{
    const size_t smem = group_smem_bytes(a.T * a.top_k, a.E);
    cudaError_t e = set_smem(group_kernel, smem);
    if (e != cudaSuccess)
        return e;
    return launch_ex(group_kernel, dim3(1), dim3(GR_THREADS), smem, c, 1, a);
}

// fp32 -> fp16, round to nearest even (the last step of an expert-parallel
// layer: the all-reduced fp32 partials become the fp16 layer output)
namespace {
__global__ void f32_to_f16_kernel(const float *src, __half *dst, long n)
{
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
        dst[i] = __float2half_rn(src[i]);
}
}  // namespace

cudaError_t launch_f32_to_f16(const float *src, __half *dst, long n, cudaStream_t s)
{
    const long blocks = (n + 255) / 256;
    f32_to_f16_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, s>>>(src, dst, n);
    return cudaGetLastError();
}

}  // namespace qmoe
