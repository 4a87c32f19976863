// api.cu -- the C ABI of libqmoe.so (declared in include/qmoe.h): host-side
// validation, per-device state, workspace layout and kernel launches.
//
// The operations and where the pages define them are listed in qmoe.h.  This
// layer allocates nothing and never synchronises inside a compute call; the
// one per-device object it owns is a status word in a __device__ variable.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace qmoe {

__device__ int32_t g_status_word;

namespace {

constexpr int kMaxDevices = 64;

struct DevState {
    bool init = false;
    int num_sms = 0;
    int cc_major = 0;
    int32_t *status = nullptr;
};

DevState g_dev[kMaxDevices];
std::mutex g_mu;
std::atomic<int32_t> g_pdl_enabled{1};
std::atomic<int32_t> g_prefill_tc_min{0};
std::atomic<unsigned long long> g_decode_wait_ns{kWaitLimitNs};

qmoe_status device_state(DevState **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return QMOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DevState &d = g_dev[dev];
    if (!d.init) {
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return QMOE_ERR_CUDA;
        if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) !=
            cudaSuccess)
            return QMOE_ERR_CUDA;
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&d.status), g_status_word) !=
            cudaSuccess)
            return QMOE_ERR_CUDA;
        d.init = true;
    }
    if (d.cc_major != 10)
        return QMOE_ERR_UNSUPPORTED;   // built for sm_100a only
    *out = &d;
    return QMOE_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Validate one (possibly stacked) quantized matrix of `rows` x `cols`.
qmoe_status check_qmatrix(const qmoe_qmatrix *W, int rows, int cols, int bits_required)
{
    if (!W || !W->packed || !W->scales || !W->biases)
        return QMOE_ERR_INVALID_ARG;
    if (W->rows != rows || W->cols != cols || rows <= 0 || cols <= 0)
        return QMOE_ERR_INVALID_ARG;
    if (W->bits != 4 && W->bits != 8)
        return QMOE_ERR_INVALID_ARG;
    if (bits_required && W->bits != bits_required)
        return QMOE_ERR_UNSUPPORTED;
    if (W->group != kGroup || cols % kGroup != 0 || rows % 8 != 0)
        return QMOE_ERR_UNSUPPORTED;
    if (!aligned(W->packed, 16) || !aligned(W->scales, 16) || !aligned(W->biases, 16))
        return QMOE_ERR_ALIGNMENT;
    return QMOE_OK;
}

qmoe_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess)
        return QMOE_OK;
    if (e == cudaErrorInvalidValue)
        return QMOE_ERR_UNSUPPORTED;   // a shape whose tiles do not fit on chip
    return QMOE_ERR_CUDA;
}

QMat qmat(const qmoe_qmatrix &m)
{
    QMat q;
    q.packed = m.packed;
    q.scales = reinterpret_cast<const __half *>(m.scales);
    q.biases = reinterpret_cast<const __half *>(m.biases);
    return q;
}

qmoe_status check_layer(const qmoe_moe_layer *L)
{
    if (!L)
        return QMOE_ERR_INVALID_ARG;
    const int E = L->num_experts, H = L->hidden, I = L->inter;
    if (E < 1 || E > 256 || H < 64 || I < 64)
        return QMOE_ERR_INVALID_ARG;
    if (H % 64 || I % 64)
        return QMOE_ERR_UNSUPPORTED;
    qmoe_status s;
    if ((s = check_qmatrix(&L->gate, I, H, 4)) != QMOE_OK ||
        (s = check_qmatrix(&L->up, I, H, 4)) != QMOE_OK ||
        (s = check_qmatrix(&L->down, H, I, 4)) != QMOE_OK ||
        (s = check_qmatrix(&L->sh_gate, I, H, 4)) != QMOE_OK ||
        (s = check_qmatrix(&L->sh_up, I, H, 4)) != QMOE_OK ||
        (s = check_qmatrix(&L->sh_down, H, I, 4)) != QMOE_OK)
        return s;
    return QMOE_OK;
}

LaunchCfg launch_cfg(const DevState *d, void *stream)
{
    LaunchCfg c;
    c.stream = static_cast<cudaStream_t>(stream);
    c.num_sms = d->num_sms;
    c.pdl = g_pdl_enabled.load() != 0;
    return c;
}

qmoe_status expert_args(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                        const float *weights, int32_t top_k, uint16_t *y, void *workspace,
                        size_t ws_bytes, int32_t *status, ExpertArgs *a)
{
    a->gate = qmat(L->gate);
    a->up = qmat(L->up);
    a->down = qmat(L->down);
    a->sh_gate = qmat(L->sh_gate);
    a->sh_up = qmat(L->sh_up);
    a->sh_down = qmat(L->sh_down);
    a->E = L->num_experts;
    a->H = L->hidden;
    a->I = L->inter;
    a->top_k = top_k;
    a->x = reinterpret_cast<const __half *>(x);
    a->idx = idx;
    a->weights = weights;
    a->y = reinterpret_cast<__half *>(y);
    a->status = status;
    if (!workspace)
        return QMOE_ERR_WORKSPACE;
    if (!aligned(workspace, 16))
        return QMOE_ERR_ALIGNMENT;
    if (ws_bytes < expert_workspace_layout(a->H, a->I, top_k, nullptr, nullptr))
        return QMOE_ERR_WORKSPACE;
    expert_workspace_layout(a->H, a->I, top_k, workspace, &a->ws);
    return QMOE_OK;
}

qmoe_status check_expert_common(const qmoe_moe_layer *L, int32_t top_k)
{
    qmoe_status s = check_layer(L);
    if (s != QMOE_OK)
        return s;
    if (top_k < 1 || top_k > 16 || top_k > L->num_experts)
        return QMOE_ERR_INVALID_ARG;
    if (L->hidden % 16)
        return QMOE_ERR_UNSUPPORTED;
    return QMOE_OK;
}

}  // namespace

// Every check moe_expert_qmlp makes before it enqueues anything: the layer's
// shapes and formats, top_k, the pointers and their alignment, and that the
// current device is one the library was built for.
qmoe_status validate_expert_qmlp(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                                 const float *weights, int32_t top_k, const uint16_t *y,
                                 const int32_t *status_dev)
{
    qmoe_status s = check_expert_common(L, top_k);
    if (s != QMOE_OK)
        return s;
    if (!x || !idx || !weights || !y)
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(idx, 4) || !aligned(weights, 4) || !aligned(y, 2) ||
        (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    return device_state(&d);
}

qmoe_status expert_qmlp_slots(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                              const float *weights, int32_t top_k, uint32_t slot_mask,
                              float *y_part, const float *y_add, uint16_t *y, void *workspace,
                              size_t workspace_bytes, int32_t *status_dev, void *stream)
{
    if (slot_mask == 0 || (slot_mask >> (top_k + 1)) != 0 || (!y_part && !y))
        return QMOE_ERR_INVALID_ARG;
    uint16_t *yy = y ? y : reinterpret_cast<uint16_t *>(y_part);   // alignment checks only
    qmoe_status s = validate_expert_qmlp(L, x, idx, weights, top_k, yy, status_dev);
    if (s != QMOE_OK)
        return s;
    if ((y_part && !aligned(y_part, 4)) || (y_add && !aligned(y_add, 4)))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    ExpertArgs a;
    if ((s = expert_args(L, x, idx, weights, top_k, y, workspace, workspace_bytes,
                         status_dev ? status_dev : d->status, &a)) != QMOE_OK)
        return s;
    a.slot_mask = slot_mask;
    a.y_part = y_part;
    a.y_add = y_add;
    const LaunchCfg c = launch_cfg(d, stream);
    if ((s = cuda_status(launch_expert_gateup(a, c))) != QMOE_OK)
        return s;
    return cuda_status(launch_expert_down(a, c));
}

}  // namespace qmoe

using namespace qmoe;

extern "C" {

qmoe_status qgemv_affine(const qmoe_qmatrix *W, const uint16_t *x, int32_t batch, uint16_t *y,
                         int32_t *status_dev, void *stream)
{
    if (!W || !x || !y)
        return QMOE_ERR_INVALID_ARG;
    if (batch < 1 || batch > kMaxQgemvBatch)
        return QMOE_ERR_INVALID_ARG;
    qmoe_status s = check_qmatrix(W, W->rows, W->cols, 0);
    if (s != QMOE_OK)
        return s;
    if (!aligned(x, 2) || !aligned(y, 2) || (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    QgemvArgs a;
    a.packed = W->packed;
    a.scales = reinterpret_cast<const __half *>(W->scales);
    a.biases = reinterpret_cast<const __half *>(W->biases);
    a.N = W->rows;
    a.K = W->cols;
    a.bits = W->bits;
    a.params = nullptr;
    a.signs = nullptr;
    a.fmt = QG_AFFINE;
    a.x = reinterpret_cast<const __half *>(x);
    a.B = batch;
    a.y = reinterpret_cast<__half *>(y);
    a.status = status_dev ? status_dev : d->status;
    return cuda_status(launch_qgemv_batched(a, launch_cfg(d, stream)));
}

size_t qgemv_affine_workspace_bytes(int32_t rows, int32_t cols, int32_t bits, int32_t batch)
{
    if (rows <= 0 || cols <= 0 || (bits != 4 && bits != 8) || batch < 1 || batch > kMaxQgemvBatch)
        return 0;
    return qgemm_small_workspace_bytes(rows, cols, bits, batch);
}

qmoe_status qgemv_affine_ws(const qmoe_qmatrix *W, const uint16_t *x, int32_t batch, uint16_t *y,
                            void *workspace, size_t workspace_bytes, int32_t *status_dev, void *stream)
{
    if (!W || !x || !y)
        return QMOE_ERR_INVALID_ARG;
    if (batch < 1 || batch > kMaxQgemvBatch)
        return QMOE_ERR_INVALID_ARG;
    qmoe_status s = check_qmatrix(W, W->rows, W->cols, 0);
    if (s != QMOE_OK)
        return s;
    if (!aligned(x, 2) || !aligned(y, 2) || (status_dev && !aligned(status_dev, 4)) ||
        (workspace && !aligned(workspace, 16)))
        return QMOE_ERR_ALIGNMENT;
    const size_t need = qgemm_small_workspace_bytes(W->rows, W->cols, W->bits, batch);
    if (need > 0 && (!workspace || workspace_bytes < need))
        return QMOE_ERR_INVALID_ARG;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    QgemvArgs a;
    a.packed = W->packed;
    a.scales = reinterpret_cast<const __half *>(W->scales);
    a.biases = reinterpret_cast<const __half *>(W->biases);
    a.N = W->rows;
    a.K = W->cols;
    a.bits = W->bits;
    a.params = nullptr;
    a.signs = nullptr;
    a.fmt = QG_AFFINE;
    a.x = reinterpret_cast<const __half *>(x);
    a.B = batch;
    a.y = reinterpret_cast<__half *>(y);
    a.status = status_dev ? status_dev : d->status;
    if (batch <= 8)
        return cuda_status(launch_qgemv_batched(a, launch_cfg(d, stream)));
    bool used = false;
    return cuda_status(launch_qgemm_small(a, workspace, workspace_bytes, launch_cfg(d, stream), &used));
}

// checks shared by qgemv_fmt and qgemv_fmt_ws; fills the launch arguments
static qmoe_status fmt_args(const qmoe_qmatrix_fmt *W, const uint16_t *x, int32_t batch,
                            uint16_t *y, int32_t *status_dev, DevState **d, QgemvArgs *a)
{
    if (!W || !W->packed || !W->params || !x || !y)
        return QMOE_ERR_INVALID_ARG;
    if (batch < 1 || batch > kMaxQgemvBatch || W->rows <= 0 || W->cols <= 0)
        return QMOE_ERR_INVALID_ARG;
    if (W->format != QMOE_FMT_ZP4_BF16 && W->format != QMOE_FMT_SYM8_BF16)
        return QMOE_ERR_INVALID_ARG;
    if (W->group != kGroup || W->cols % kGroup != 0 || W->rows % 8 != 0)
        return QMOE_ERR_UNSUPPORTED;
    if (!aligned(W->packed, 16) || !aligned(W->params, 16) ||
        (W->rht_signs && !aligned(W->rht_signs, 4)))
        return QMOE_ERR_ALIGNMENT;
    if (!aligned(x, W->rht_signs ? 16 : 2) || !aligned(y, 2) ||
        (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    qmoe_status s;
    if ((s = device_state(d)) != QMOE_OK)
        return s;
    a->packed = W->packed;
    a->scales = nullptr;
    a->biases = nullptr;
    a->params = W->params;
    a->signs = W->rht_signs;
    a->N = W->rows;
    a->K = W->cols;
    a->fmt = W->format == QMOE_FMT_ZP4_BF16 ? QG_ZP4 : QG_SYM8;
    a->bits = W->format == QMOE_FMT_ZP4_BF16 ? 4 : 8;
    a->x = reinterpret_cast<const __half *>(x);
    a->B = batch;
    a->y = reinterpret_cast<__half *>(y);
    a->status = status_dev ? status_dev : (*d)->status;
    return QMOE_OK;
}

qmoe_status qgemv_fmt(const qmoe_qmatrix_fmt *W, const uint16_t *x, int32_t batch, uint16_t *y,
                      int32_t *status_dev, void *stream)
{
    DevState *d;
    QgemvArgs a;
    const qmoe_status s = fmt_args(W, x, batch, y, status_dev, &d, &a);
    if (s != QMOE_OK)
        return s;
    return cuda_status(launch_qgemv_batched(a, launch_cfg(d, stream)));
}

size_t qgemv_fmt_workspace_bytes(int32_t rows, int32_t cols, int32_t format, int32_t rotated,
                                 int32_t batch)
{
    if (rows <= 0 || cols <= 0 || batch < 1 || batch > kMaxQgemvBatch ||
        (format != QMOE_FMT_ZP4_BF16 && format != QMOE_FMT_SYM8_BF16))
        return 0;
    return qgemm_small_workspace_bytes(rows, cols, format == QMOE_FMT_ZP4_BF16 ? 4 : 8, batch,
                                       rotated != 0);
}

qmoe_status qgemv_fmt_ws(const qmoe_qmatrix_fmt *W, const uint16_t *x, int32_t batch, uint16_t *y,
                         void *workspace, size_t workspace_bytes, int32_t *status_dev,
                         void *stream)
{
    DevState *d;
    QgemvArgs a;
    qmoe_status s = fmt_args(W, x, batch, y, status_dev, &d, &a);
    if (s != QMOE_OK)
        return s;
    if (workspace && !aligned(workspace, 16))
        return QMOE_ERR_ALIGNMENT;
    const size_t need =
        qgemm_small_workspace_bytes(a.N, a.K, a.bits, batch, W->rht_signs != nullptr);
    if (need > 0 && (!workspace || workspace_bytes < need))
        return QMOE_ERR_INVALID_ARG;
    bool used = false;
    return cuda_status(launch_qgemm_small(a, workspace, workspace_bytes, launch_cfg(d, stream), &used));
}

qmoe_status moe_router_topk(const qmoe_qmatrix *router, const uint16_t *x, int32_t tokens,
                            int32_t top_k, int32_t *idx, float *weights, float *logits,
                            int32_t *status_dev, void *stream)
{
    if (!router || !x || !idx || !weights)
        return QMOE_ERR_INVALID_ARG;
    if (tokens < 1 || tokens > 65536)
        return QMOE_ERR_INVALID_ARG;
    qmoe_status s = check_qmatrix(router, router->rows, router->cols, 0);
    if (s != QMOE_OK)
        return s;
    if (router->rows > 128)
        return QMOE_ERR_UNSUPPORTED;
    if (top_k < 1 || top_k > 16 || top_k > router->rows)
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(idx, 4) || !aligned(weights, 4) ||
        (logits && !aligned(logits, 4)) || (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    RouterArgs a;
    a.packed = router->packed;
    a.scales = reinterpret_cast<const __half *>(router->scales);
    a.biases = reinterpret_cast<const __half *>(router->biases);
    a.E = router->rows;
    a.K = router->cols;
    a.bits = router->bits;
    a.x = reinterpret_cast<const __half *>(x);
    a.T = tokens;
    a.top_k = top_k;
    a.idx = idx;
    a.weights = weights;
    a.logits = logits;
    a.status = status_dev ? status_dev : d->status;
    return cuda_status(launch_router(a, launch_cfg(d, stream)));
}

size_t moe_expert_workspace_bytes(const qmoe_moe_layer *L, int32_t top_k)
{
    if (!L || L->hidden <= 0 || L->inter <= 0 || top_k < 1)
        return 0;
    return expert_workspace_layout(L->hidden, L->inter, top_k, nullptr, nullptr);
}

qmoe_status moe_expert_gateup(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                              int32_t top_k, void *workspace, size_t workspace_bytes,
                              int32_t *status_dev, void *stream)
{
    qmoe_status s = check_expert_common(L, top_k);
    if (s != QMOE_OK)
        return s;
    if (!x || !idx)
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(idx, 4) || (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    ExpertArgs a;
    if ((s = expert_args(L, x, idx, nullptr, top_k, nullptr, workspace, workspace_bytes,
                         status_dev ? status_dev : d->status, &a)) != QMOE_OK)
        return s;
    return cuda_status(launch_expert_gateup(a, launch_cfg(d, stream)));
}

qmoe_status moe_expert_down(const qmoe_moe_layer *L, const int32_t *idx, const float *weights,
                            int32_t top_k, uint16_t *y, void *workspace, size_t workspace_bytes,
                            int32_t *status_dev, void *stream)
{
    qmoe_status s = check_expert_common(L, top_k);
    if (s != QMOE_OK)
        return s;
    if (!idx || !weights || !y)
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(idx, 4) || !aligned(weights, 4) || !aligned(y, 2) ||
        (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    ExpertArgs a;
    if ((s = expert_args(L, nullptr, idx, weights, top_k, y, workspace, workspace_bytes,
                         status_dev ? status_dev : d->status, &a)) != QMOE_OK)
        return s;
    return cuda_status(launch_expert_down(a, launch_cfg(d, stream)));
}

qmoe_status moe_expert_qmlp(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                            const float *weights, int32_t top_k, uint16_t *y, void *workspace,
                            size_t workspace_bytes, int32_t *status_dev, void *stream)
{
    qmoe_status s = qmoe::validate_expert_qmlp(L, x, idx, weights, top_k, y, status_dev);
    if (s != QMOE_OK)
        return s;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    ExpertArgs a;
    if ((s = expert_args(L, x, idx, weights, top_k, y, workspace, workspace_bytes,
                         status_dev ? status_dev : d->status, &a)) != QMOE_OK)
        return s;
    const LaunchCfg c = launch_cfg(d, stream);
    if ((s = cuda_status(launch_expert_gateup(a, c))) != QMOE_OK)
        return s;
    return cuda_status(launch_expert_down(a, c));
}

qmoe_status moe_expert_qmlp_ep(const qmoe_moe_layer *L, const uint16_t *x, const int32_t *idx,
                               const float *weights, int32_t top_k, int32_t rank, int32_t world,
                               float *y_partial, void *workspace, size_t workspace_bytes,
                               int32_t *status_dev, void *stream)
{
    qmoe_status s = check_expert_common(L, top_k);
    if (s != QMOE_OK)
        return s;
    if (!x || !idx || !weights || !y_partial || world < 1 || rank < 0 || rank >= world ||
        L->num_experts % world)
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(idx, 4) || !aligned(weights, 4) || !aligned(y_partial, 4) ||
        (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    ExpertArgs a;
    if ((s = expert_args(L, x, idx, weights, top_k, nullptr, workspace, workspace_bytes,
                         status_dev ? status_dev : d->status, &a)) != QMOE_OK)
        return s;
    a.ep_rank = rank;
    a.ep_world = world;
    a.ep_first = rank * (L->num_experts / world);
    a.y_part = y_partial;
    const LaunchCfg c = launch_cfg(d, stream);
    if ((s = cuda_status(launch_expert_gateup(a, c))) != QMOE_OK)
        return s;
    return cuda_status(launch_expert_down(a, c));
}

qmoe_status qmoe_f32_to_f16(const float *src, uint16_t *dst, int64_t n, void *stream)
{
    if (!src || !dst || n < 0)
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(src, 4) || !aligned(dst, 2))
        return QMOE_ERR_ALIGNMENT;
    if (n == 0)
        return QMOE_OK;
    return cuda_status(launch_f32_to_f16(src, reinterpret_cast<__half *>(dst), (long)n,
                                         static_cast<cudaStream_t>(stream)));
}

size_t moe_decode_pack_bytes(const qmoe_moe_layer *L)
{
    if (!L || L->num_experts < 1 || L->hidden < 256 || L->inter < 64)
        return 0;
    return decode_pack_bytes(L->num_experts, L->hidden, L->inter);
}

qmoe_status moe_decode_pack_layer(const qmoe_moe_layer *L, const qmoe_qmatrix *router, void *packed,
                                  size_t packed_bytes, void *stream)
{
    qmoe_status s = check_layer(L);
    if (s != QMOE_OK)
        return s;
    if ((s = check_qmatrix(router, L->num_experts, L->hidden, 8)) != QMOE_OK)
        return s;
    if (L->num_experts > 128 || L->num_experts % 8 || L->hidden % 256)
        return QMOE_ERR_UNSUPPORTED;
    if (!packed)
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(packed, 16))
        return QMOE_ERR_ALIGNMENT;
    if (packed_bytes < moe_decode_pack_bytes(L))
        return QMOE_ERR_WORKSPACE;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    DecodePackArgs a;
    a.router = qmat(*router);
    a.gate = qmat(L->gate);
    a.up = qmat(L->up);
    a.down = qmat(L->down);
    a.sh_gate = qmat(L->sh_gate);
    a.sh_up = qmat(L->sh_up);
    a.sh_down = qmat(L->sh_down);
    a.E = L->num_experts;
    a.H = L->hidden;
    a.I = L->inter;
    return cuda_status(launch_decode_pack(a, packed, static_cast<cudaStream_t>(stream)));
}

size_t moe_decode_workspace_bytes(int32_t num_experts, int32_t hidden, int32_t inter,
                                  int32_t top_k)
{
    if (num_experts < 1 || hidden <= 0 || inter <= 0 || top_k < 1)
        return 0;
    return decode_workspace_layout(num_experts, hidden, inter, top_k, nullptr, nullptr);
}

// every check of moe_decode_layers, before anything is enqueued
static qmoe_status decode_validate(const void *const *packed_layers, int32_t n_layers,
                                   int32_t num_experts, int32_t hidden, int32_t inter,
                                   const uint16_t *x, int32_t top_k, const uint16_t *y,
                                   const int32_t *idx, const float *weights, const float *logits,
                                   const void *workspace, size_t workspace_bytes,
                                   const int32_t *status_dev)
{
    if (!packed_layers || !x || !y || n_layers < 1)
        return QMOE_ERR_INVALID_ARG;
    if (num_experts < 8 || num_experts > 128 || num_experts % 8 || hidden < 256 ||
        hidden % 256 || inter < 64 || inter % 64)
        return QMOE_ERR_UNSUPPORTED;
    if (top_k < 1 || top_k > 16 || top_k > num_experts)
        return QMOE_ERR_INVALID_ARG;
    for (int l = 0; l < n_layers; ++l) {
        if (!packed_layers[l])
            return QMOE_ERR_INVALID_ARG;
        if (!aligned(packed_layers[l], 16))
            return QMOE_ERR_ALIGNMENT;
    }
    // each layer's x is read with 16-byte loads (hidden % 256 keeps every
    // layer's row 16-byte aligned once the first is)
    if (!aligned(x, 16) || !aligned(y, 2) || (idx && !aligned(idx, 4)) ||
        (weights && !aligned(weights, 4)) || (logits && !aligned(logits, 4)) ||
        (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    if (!workspace)
        return QMOE_ERR_WORKSPACE;
    if (!aligned(workspace, 16))
        return QMOE_ERR_ALIGNMENT;
    if (workspace_bytes < moe_decode_workspace_bytes(num_experts, hidden, inter, top_k))
        return QMOE_ERR_WORKSPACE;
    DevState *d;
    return device_state(&d);
}

qmoe_status moe_decode_layers(const void *const *packed_layers, int32_t n_layers,
                              int32_t num_experts, int32_t hidden, int32_t inter,
                              const uint16_t *x, int32_t top_k, uint16_t *y, int32_t *idx,
                              float *weights, float *logits, void *workspace,
                              size_t workspace_bytes, int32_t *status_dev, void *stream)
{
    qmoe_status s = decode_validate(packed_layers, n_layers, num_experts, hidden, inter, x, top_k,
                                    y, idx, weights, logits, workspace, workspace_bytes,
                                    status_dev);
    if (s != QMOE_OK)
        return s;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    const LaunchCfg c = launch_cfg(d, stream);
    DecodeArgs a;
    a.E = num_experts;
    a.H = hidden;
    a.I = inter;
    a.top_k = top_k;
    a.NS = 0;
    a.wait_ns = g_decode_wait_ns.load();
    a.status = status_dev ? status_dev : d->status;
    decode_workspace_layout(a.E, a.H, a.I, top_k, workspace, &a.ws);
    for (int l0 = 0; l0 < n_layers; l0 += kDecodeMaxLayers) {
        const int n = n_layers - l0 < kDecodeMaxLayers ? n_layers - l0 : kDecodeMaxLayers;
        a.L = n;
        a.x = reinterpret_cast<const __half *>(x) + (size_t)l0 * a.H;
        a.y = reinterpret_cast<__half *>(y) + (size_t)l0 * a.H;
        a.idx = idx ? idx + (size_t)l0 * top_k : nullptr;
        a.weights = weights ? weights + (size_t)l0 * top_k : nullptr;
        a.logits = logits ? logits + (size_t)l0 * a.E : nullptr;
        for (int l = 0; l < n; ++l)
            a.layer[l] = packed_layers[l0 + l];
        if ((s = cuda_status(launch_decode(a, c))) != QMOE_OK)
            return s;
    }
    return QMOE_OK;
}

qmoe_status moe_decode_layers_host(const void *const *packed_layers, int32_t n_layers,
                                   int32_t num_experts, int32_t hidden, int32_t inter,
                                   const uint16_t *x_host, uint16_t *y_host, int32_t top_k,
                                   uint16_t *x_dev, uint16_t *y_dev, void *workspace,
                                   size_t workspace_bytes, int32_t *status_dev, void *stream)
{
    if (!x_host || !y_host)
        return QMOE_ERR_INVALID_ARG;
    // every check of the decode first: a rejected call copies nothing
    qmoe_status s = decode_validate(packed_layers, n_layers, num_experts, hidden, inter, x_dev,
                                    top_k, y_dev, nullptr, nullptr, nullptr, workspace,
                                    workspace_bytes, status_dev);
    if (s != QMOE_OK)
        return s;
    const size_t bytes = (size_t)n_layers * hidden * 2;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return QMOE_ERR_CUDA;
    if ((s = moe_decode_layers(packed_layers, n_layers, num_experts, hidden, inter, x_dev, top_k,
                               y_dev, nullptr, nullptr, nullptr, workspace, workspace_bytes,
                               status_dev, stream)) != QMOE_OK)
        return s;
    if (cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return QMOE_ERR_CUDA;
    return QMOE_OK;
}

qmoe_status moe_group_tokens(const int32_t *idx, int32_t tokens, int32_t top_k,
                             int32_t num_experts, int32_t *counts, int32_t *offsets,
                             int32_t *pairs, int32_t *status_dev, void *stream)
{
    if (!idx || !counts || !offsets || !pairs)
        return QMOE_ERR_INVALID_ARG;
    if (tokens < 1 || tokens > 128 || top_k < 1 || top_k > 16 || num_experts < 1 ||
        num_experts > 256)
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(idx, 4) || !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(pairs, 4) ||
        (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    qmoe_status s;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    GroupArgs a;
    a.idx = idx;
    a.T = tokens;
    a.top_k = top_k;
    a.E = num_experts;
    a.counts = counts;
    a.offsets = offsets;
    a.pairs = pairs;
    a.status = status_dev ? status_dev : d->status;
    return cuda_status(launch_group(a, launch_cfg(d, stream)));
}

size_t moe_prefill_workspace_bytes(const qmoe_moe_layer *L, int32_t tokens, int32_t top_k)
{
    if (!L || tokens < 1 || top_k < 1 || L->num_experts < 1)
        return 0;
    return prefill_workspace_layout(L->num_experts, L->hidden, L->inter, tokens, top_k, nullptr,
                                    nullptr);
}

qmoe_status moe_prefill_qgemm(const qmoe_moe_layer *L, const uint16_t *x, int32_t tokens,
                              const int32_t *idx, const float *weights, int32_t top_k,
                              uint16_t *y, void *workspace, size_t workspace_bytes,
                              int32_t *status_dev, void *stream)
{
    qmoe_status s = check_expert_common(L, top_k);
    if (s != QMOE_OK)
        return s;
    if (!x || !idx || !weights || !y)
        return QMOE_ERR_INVALID_ARG;
    if (tokens < 1 || tokens > 128)
        return QMOE_ERR_INVALID_ARG;
    if (!prefill_shape_supported(L->hidden, L->inter))
        return QMOE_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(idx, 4) || !aligned(weights, 4) || !aligned(y, 4) ||
        (status_dev && !aligned(status_dev, 4)))
        return QMOE_ERR_ALIGNMENT;
    if (!workspace)
        return QMOE_ERR_WORKSPACE;
    if (!aligned(workspace, 16))
        return QMOE_ERR_ALIGNMENT;
    if (workspace_bytes < moe_prefill_workspace_bytes(L, tokens, top_k))
        return QMOE_ERR_WORKSPACE;
    DevState *d;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    PrefillArgs a;
    a.gate = qmat(L->gate);
    a.up = qmat(L->up);
    a.down = qmat(L->down);
    a.sh_gate = qmat(L->sh_gate);
    a.sh_up = qmat(L->sh_up);
    a.sh_down = qmat(L->sh_down);
    a.E = L->num_experts;
    a.H = L->hidden;
    a.I = L->inter;
    a.T = tokens;
    a.top_k = top_k;
    a.x = reinterpret_cast<const __half *>(x);
    a.idx = idx;
    a.weights = weights;
    a.y = reinterpret_cast<__half *>(y);
    a.status = status_dev ? status_dev : d->status;
    prefill_workspace_layout(a.E, a.H, a.I, tokens, top_k, workspace, &a.ws);
    const int tc_min = g_prefill_tc_min.load();
    a.tc_min = (tc_min > 0 && prefill_tc_supported(a.H, a.I)) ? tc_min : (1 << 30);
    return cuda_status(launch_prefill(a, launch_cfg(d, stream)));
}

qmoe_status qmoe_pack_codes(const uint8_t *codes, int32_t rows, int32_t cols, int32_t bits,
                            uint32_t *packed, void *stream)
{
    if (!codes || !packed || rows < 1 || cols < 1 || (bits != 4 && bits != 8))
        return QMOE_ERR_INVALID_ARG;
    if (cols % (32 / bits))
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(packed, 4))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    qmoe_status s;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    return cuda_status(launch_pack(codes, rows, cols, bits, packed, static_cast<cudaStream_t>(stream)));
}

qmoe_status qmoe_unpack_codes(const uint32_t *packed, int32_t rows, int32_t cols, int32_t bits,
                              uint8_t *codes, void *stream)
{
    if (!codes || !packed || rows < 1 || cols < 1 || (bits != 4 && bits != 8))
        return QMOE_ERR_INVALID_ARG;
    if (cols % (32 / bits))
        return QMOE_ERR_INVALID_ARG;
    if (!aligned(packed, 4))
        return QMOE_ERR_ALIGNMENT;
    DevState *d;
    qmoe_status s;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    return cuda_status(
        launch_unpack(packed, rows, cols, bits, codes, static_cast<cudaStream_t>(stream)));
}

qmoe_status qmoe_check_status(int32_t *status_dev, void *stream, int32_t *flags_out)
{
    DevState *d;
    qmoe_status s;
    if ((s = device_state(&d)) != QMOE_OK)
        return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t *word = status_dev ? status_dev : d->status;
    int32_t flags = 0;
    if (cudaMemcpyAsync(&flags, word, sizeof(flags), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return QMOE_ERR_CUDA;
    if (cudaMemsetAsync(word, 0, sizeof(int32_t), st) != cudaSuccess)
        return QMOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return QMOE_ERR_CUDA;
    if (flags_out)
        *flags_out = flags;
    if (flags & QMOE_DEV_TIMEOUT)
        return QMOE_ERR_TIMEOUT;
    if (flags)
        return QMOE_ERR_DEVICE_STATUS;
    return QMOE_OK;
}

const char *qmoe_status_string(qmoe_status s)
{
    switch (s) {
    case QMOE_OK: return "QMOE_OK";
    case QMOE_ERR_INVALID_ARG: return "QMOE_ERR_INVALID_ARG: invalid argument";
    case QMOE_ERR_ALIGNMENT: return "QMOE_ERR_ALIGNMENT: misaligned pointer";
    case QMOE_ERR_UNSUPPORTED: return "QMOE_ERR_UNSUPPORTED: unsupported shape or device";
    case QMOE_ERR_CUDA: return "QMOE_ERR_CUDA: CUDA runtime error";
    case QMOE_ERR_DEVICE_STATUS: return "QMOE_ERR_DEVICE_STATUS: a kernel flagged bad input";
    case QMOE_ERR_TIMEOUT: return "QMOE_ERR_TIMEOUT: a kernel wait timed out";
    case QMOE_ERR_WORKSPACE: return "QMOE_ERR_WORKSPACE: workspace missing or too small";
    }
    return "unknown qmoe_status";
}

int32_t qmoe_set_dependent_launch(int32_t enable)
{
    return g_pdl_enabled.exchange(enable ? 1 : 0);
}

uint64_t qmoe_set_decode_wait_limit_ns(uint64_t ns)
{
    return g_decode_wait_ns.exchange(ns == 0 ? kWaitLimitNs : ns);
}

int32_t qmoe_set_prefill_tensor_min(int32_t min_tokens)
{
    return g_prefill_tc_min.exchange(min_tokens < 0 ? 0 : min_tokens);
}

int32_t qmoe_version(void) { return 100; }

}  // extern "C"
