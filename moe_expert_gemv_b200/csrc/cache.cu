// cache.cu -- host-memory expert streaming through a per-layer LFU cache.
//
// TurboFieldfare article (jeff.news), section "내부 구조가 진짜 흥미로운 부분"
// (internal structure): the router runs on resident weights; the CPU takes
// its top-8 expert ids, plans the misses against the layer's 16-slot LFU
// cache and fills the missed experts (bounded parallel reads from SSD) into
// device-visible memory, while the resident shared expert runs; then the
// routed experts run and the two outputs are added.
//
// On B200 the whole model fits HBM, so this path exists for models that do
// not: the routed experts of a layer live in pinned host memory, the cache is
// `nslots` device slots laid out as a stacked expert array, and a miss is one
// host-to-device copy per array of the expert, spread over four copy
// streams (bounded parallel copies).  Host code
// only (no kernels): the router and the experts run the library's kernels.
//
// Plan (host, per token and layer): hits first -- the slot's count grows by
// one and the slot is pinned for this token -- then the misses in id order:
// the lowest-index empty slot, else the unpinned slot with the smallest count
// (ties: lowest index); a loaded expert starts at count 1.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "kernels.h"
#include "qmoe.h"

namespace qmoe {
namespace {

constexpr int kMaxSlots = 256;
constexpr int kMaxTopK = 16;
constexpr int kCopyStreams = 4;   // misses copied in parallel (bounded, as the pages' reads)

struct Lfu {
    int nslots;
    int32_t expert[kMaxSlots];   // -1: empty
    int64_t count[kMaxSlots];
};

void lfu_reset(Lfu *c, int nslots)
{
    c->nslots = nslots;
    for (int s = 0; s < kMaxSlots; ++s) {
        c->expert[s] = -1;
        c->count[s] = 0;
    }
}

// One token: slot_of[j] for ids[j]; misses as (expert, slot); returns their
// number, or -1 for k > nslots or repeated ids (the cache is then unchanged).
int lfu_plan(Lfu *c, const int32_t *ids, int k, int32_t *slot_of, int32_t *miss_expert,
             int32_t *miss_slot)
{
    if (k < 1 || k > c->nslots || k > kMaxTopK)
        return -1;
    for (int a = 0; a < k; ++a)
        for (int b = 0; b < a; ++b)
            if (ids[a] == ids[b])
                return -1;
    bool pin[kMaxSlots] = {};
    // where each id is cached, if it is
    for (int j = 0; j < k; ++j) {
        slot_of[j] = -1;
        for (int s = 0; s < c->nslots; ++s)
            if (c->expert[s] == ids[j]) {
                slot_of[j] = s;
                break;
            }
        if (slot_of[j] >= 0) {
            c->count[slot_of[j]] += 1;
            pin[slot_of[j]] = true;
        }
    }
    int n = 0;
    for (int j = 0; j < k; ++j) {
        if (slot_of[j] >= 0)
            continue;
        int victim = -1;
        int64_t best = 0;
        for (int s = 0; s < c->nslots; ++s) {
            if (pin[s])
                continue;
            if (c->expert[s] < 0) {   // an empty slot beats any occupied one
                victim = s;
                break;
            }
            if (victim < 0 || c->count[s] < best) {
                victim = s;
                best = c->count[s];
            }
        }
        c->expert[victim] = ids[j];
        c->count[victim] = 1;
        pin[victim] = true;
        slot_of[j] = victim;
        miss_expert[n] = ids[j];
        miss_slot[n] = victim;
        ++n;
    }
    return n;
}

}  // namespace
}  // namespace qmoe

using namespace qmoe;

// ------------------------------------------------------------ the planner --
struct qmoe_lfu {
    Lfu c;
};

extern "C" {

qmoe_status qmoe_lfu_create(int32_t nslots, qmoe_lfu **out)
{
    if (!out || nslots < 1 || nslots > kMaxSlots)
        return QMOE_ERR_INVALID_ARG;
    qmoe_lfu *h = static_cast<qmoe_lfu *>(malloc(sizeof(qmoe_lfu)));
    if (!h)
        return QMOE_ERR_INVALID_ARG;
    lfu_reset(&h->c, nslots);
    *out = h;
    return QMOE_OK;
}

void qmoe_lfu_destroy(qmoe_lfu *h) { free(h); }

int32_t qmoe_lfu_plan(qmoe_lfu *h, const int32_t *ids, int32_t k, int32_t *slot_of,
                      int32_t *miss_expert, int32_t *miss_slot)
{
    if (!h || !ids || !slot_of || !miss_expert || !miss_slot)
        return -1;
    return lfu_plan(&h->c, ids, k, slot_of, miss_expert, miss_slot);
}

qmoe_status qmoe_lfu_slots(const qmoe_lfu *h, int32_t *expert, int64_t *count)
{
    if (!h || !expert)
        return QMOE_ERR_INVALID_ARG;
    for (int s = 0; s < h->c.nslots; ++s) {
        expert[s] = h->c.expert[s];
        if (count)
            count[s] = h->c.count[s];
    }
    return QMOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------- the cache layer --
struct qmoe_expert_cache {
    qmoe_moe_layer host;    // routed experts in pinned host memory (stacked over E)
    qmoe_moe_layer slots;   // nslots device slots (stacked) + the resident shared expert
    qmoe_lfu plan;
    int32_t *ids_host;      // pinned [kMaxTopK]: the router's choice, read by the host
    int32_t *slot_host;     // pinned [kMaxTopK]: the plan, copied to the device
    int32_t *idx_dev;       // device [kMaxTopK]
    float *wt_dev;          // device [kMaxTopK]
    int32_t *slot_dev;      // device [kMaxTopK]
    float *ysh_dev;         // device fp32 [hidden]: the shared expert's output
    cudaStream_t copy[kCopyStreams];   // the cache's own copy streams
    cudaEvent_t copied[kCopyStreams];
    int64_t hits, misses, bytes;
};

namespace {

// bytes of one expert's array in a stacked matrix, and its source/destination
struct ArrayPart {
    const void *src;
    void *dst;
    size_t bytes;
};

int expert_parts(const qmoe_moe_layer &host, const qmoe_moe_layer &slots, int e, int s,
                 ArrayPart *out)
{
    const qmoe_qmatrix *hm[3] = {&host.gate, &host.up, &host.down};
    const qmoe_qmatrix *dm[3] = {&slots.gate, &slots.up, &slots.down};
    int n = 0;
    for (int i = 0; i < 3; ++i) {
        const size_t codes = (size_t)hm[i]->rows * hm[i]->cols * hm[i]->bits / 8;
        const size_t sb = (size_t)hm[i]->rows * (hm[i]->cols / 64) * 2;
        out[n++] = {reinterpret_cast<const unsigned char *>(hm[i]->packed) + e * codes,
                    reinterpret_cast<unsigned char *>(const_cast<uint32_t *>(dm[i]->packed)) +
                        s * codes,
                    codes};
        out[n++] = {reinterpret_cast<const unsigned char *>(hm[i]->scales) + e * sb,
                    reinterpret_cast<unsigned char *>(const_cast<uint16_t *>(dm[i]->scales)) +
                        s * sb,
                    sb};
        out[n++] = {reinterpret_cast<const unsigned char *>(hm[i]->biases) + e * sb,
                    reinterpret_cast<unsigned char *>(const_cast<uint16_t *>(dm[i]->biases)) +
                        s * sb,
                    sb};
    }
    return n;
}

}  // namespace

extern "C" {

qmoe_status qmoe_cache_create(const qmoe_moe_layer *host, const qmoe_moe_layer *slots,
                              qmoe_expert_cache **out)
{
    if (!host || !slots || !out || !host->gate.packed || !host->up.packed || !host->down.packed ||
        !slots->gate.packed || !slots->up.packed || !slots->down.packed || !slots->sh_gate.packed)
        return QMOE_ERR_INVALID_ARG;
    const int E = host->num_experts, ns = slots->num_experts;
    if (E < 1 || ns < 1 || ns > kMaxSlots || host->hidden != slots->hidden ||
        host->inter != slots->inter || host->gate.rows != host->inter ||
        slots->gate.rows != slots->inter)
        return QMOE_ERR_INVALID_ARG;
    qmoe_expert_cache *c = static_cast<qmoe_expert_cache *>(calloc(1, sizeof(qmoe_expert_cache)));
    if (!c)
        return QMOE_ERR_INVALID_ARG;
    c->host = *host;
    c->slots = *slots;
    lfu_reset(&c->plan.c, ns);
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess)
        e = cudaMallocHost(&c->ids_host, kMaxTopK * sizeof(int32_t));
    if (e == cudaSuccess)
        e = cudaMallocHost(&c->slot_host, kMaxTopK * sizeof(int32_t));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->idx_dev, kMaxTopK * sizeof(int32_t));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->wt_dev, kMaxTopK * sizeof(float));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->slot_dev, kMaxTopK * sizeof(int32_t));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->ysh_dev, (size_t)host->hidden * sizeof(float));
    for (int i = 0; i < kCopyStreams && e == cudaSuccess; ++i) {
        e = cudaStreamCreateWithFlags(&c->copy[i], cudaStreamNonBlocking);
        if (e == cudaSuccess)
            e = cudaEventCreateWithFlags(&c->copied[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
        qmoe_cache_destroy(c);
        return QMOE_ERR_CUDA;
    }
    *out = c;
    return QMOE_OK;
}

void qmoe_cache_destroy(qmoe_expert_cache *c)
{
    if (!c)
        return;
    if (c->ids_host)
        cudaFreeHost(c->ids_host);
    if (c->slot_host)
        cudaFreeHost(c->slot_host);
    if (c->idx_dev)
        cudaFree(c->idx_dev);
    if (c->wt_dev)
        cudaFree(c->wt_dev);
    if (c->slot_dev)
        cudaFree(c->slot_dev);
    if (c->ysh_dev)
        cudaFree(c->ysh_dev);
    for (int i = 0; i < kCopyStreams; ++i) {
        if (c->copied[i])
            cudaEventDestroy(c->copied[i]);
        if (c->copy[i])
            cudaStreamDestroy(c->copy[i]);
    }
    free(c);
}

qmoe_status moe_cache_layer(qmoe_expert_cache *c, const qmoe_qmatrix *router, const uint16_t *x,
                            int32_t top_k, uint16_t *y, int32_t *idx_out, float *weights_out,
                            void *workspace, size_t workspace_bytes, int32_t *status_dev,
                            void *stream, void *copy_stream)
{
    if (!c || !router || !x || !y)
        return QMOE_ERR_INVALID_ARG;
    if (top_k < 1 || top_k > kMaxTopK || top_k > c->plan.c.nslots ||
        router->rows != c->host.num_experts)
        return QMOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // copy streams: the caller's (if any) first, then the cache's own
    cudaStream_t cs[kCopyStreams];
    cudaEvent_t ev[kCopyStreams];
    for (int i = 0; i < kCopyStreams; ++i) {
        cs[i] = c->copy[i];
        ev[i] = c->copied[i];
    }
    if (copy_stream)
        cs[0] = static_cast<cudaStream_t>(copy_stream);
    // 1. router on resident weights
    qmoe_status s = moe_router_topk(router, x, 1, top_k, c->idx_dev, c->wt_dev, nullptr,
                                    status_dev, stream);
    if (s != QMOE_OK)
        return s;
    // 2. the host reads the choice (the plan is made on the host)
    if (cudaMemcpyAsync(c->ids_host, c->idx_dev, top_k * sizeof(int32_t),
                        cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return QMOE_ERR_CUDA;
    // 3. plan (the router only emits ids in [0, E); anything else means the
    //    router failed, and the cache is left as it was)
    int32_t ids[kMaxTopK], miss_e[kMaxTopK], miss_s[kMaxTopK];
    for (int j = 0; j < top_k; ++j) {
        ids[j] = c->ids_host[j];
        if (ids[j] < 0 || ids[j] >= c->host.num_experts)
            return QMOE_ERR_DEVICE_STATUS;
    }
    const int nm = lfu_plan(&c->plan.c, ids, top_k, c->slot_host, miss_e, miss_s);
    if (nm < 0)
        return QMOE_ERR_INVALID_ARG;
    // From here the plan already names the new slot contents: if any step
    // fails, forget the whole cache (every slot empty) rather than keep a plan
    // whose copies may not have landed; the next token copies again.
    auto fail = [&](qmoe_status st_) {
        lfu_reset(&c->plan.c, c->plan.c.nslots);
        return st_;
    };
    // 4. the missed experts' arrays, host -> device, one copy each; expert m
    //    on copy stream m % kCopyStreams.  A slot must not be overwritten
    //    while an earlier token's experts read it: the synchronisation above
    //    already ordered everything enqueued on `stream` before this point,
    //    and the copy streams also wait on an event of `stream`.
    const int nstreams = nm < kCopyStreams ? nm : kCopyStreams;
    if (nstreams > 0) {
        if (cudaEventRecord(ev[0], st) != cudaSuccess)
            return fail(QMOE_ERR_CUDA);
        for (int i = 0; i < nstreams; ++i)
            if (cudaStreamWaitEvent(cs[i], ev[0], 0) != cudaSuccess)
                return fail(QMOE_ERR_CUDA);
    }
    for (int m = 0; m < nm; ++m) {
        ArrayPart parts[9];
        const int np = expert_parts(c->host, c->slots, miss_e[m], miss_s[m], parts);
        for (int i = 0; i < np; ++i) {
            if (cudaMemcpyAsync(parts[i].dst, parts[i].src, parts[i].bytes,
                                cudaMemcpyHostToDevice, cs[m % kCopyStreams]) != cudaSuccess)
                return fail(QMOE_ERR_CUDA);
            c->bytes += (int64_t)parts[i].bytes;
        }
    }
    c->hits += top_k - nm;
    c->misses += nm;
    // 5. the shared expert needs no copy: it runs on `stream` while the
    //    missed experts are in flight, its fp32 output kept for the sum
    s = expert_qmlp_slots(&c->slots, x, c->slot_dev, c->wt_dev, top_k, 1u, c->ysh_dev, nullptr,
                          nullptr, workspace, workspace_bytes, status_dev, stream);
    if (s != QMOE_OK)
        return fail(s);
    // 6. the routed experts wait for the copies; the slot ids follow the plan
    for (int i = 0; i < nstreams; ++i)
        if (cudaEventRecord(ev[i], cs[i]) != cudaSuccess ||
            cudaStreamWaitEvent(st, ev[i], 0) != cudaSuccess)
            return fail(QMOE_ERR_CUDA);
    if (cudaMemcpyAsync(c->slot_dev, c->slot_host, top_k * sizeof(int32_t),
                        cudaMemcpyHostToDevice, st) != cudaSuccess)
        return fail(QMOE_ERR_CUDA);
    // 7. y = shared output + sum_j weights[j] * routed expert j, from the slots
    const uint32_t routed = ((1u << top_k) - 1u) << 1;
    s = expert_qmlp_slots(&c->slots, x, c->slot_dev, c->wt_dev, top_k, routed, nullptr,
                          c->ysh_dev, y, workspace, workspace_bytes, status_dev, stream);
    if (s != QMOE_OK)
        return fail(s);
    if (idx_out && cudaMemcpyAsync(idx_out, c->idx_dev, top_k * sizeof(int32_t),
                                   cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return QMOE_ERR_CUDA;
    if (weights_out && cudaMemcpyAsync(weights_out, c->wt_dev, top_k * sizeof(float),
                                       cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return QMOE_ERR_CUDA;
    return QMOE_OK;
}

qmoe_status qmoe_cache_stats(const qmoe_expert_cache *c, int64_t *hits, int64_t *misses,
                             int64_t *bytes_copied, int32_t *slot_expert)
{
    if (!c)
        return QMOE_ERR_INVALID_ARG;
    if (hits)
        *hits = c->hits;
    if (misses)
        *misses = c->misses;
    if (bytes_copied)
        *bytes_copied = c->bytes;
    if (slot_expert)
        for (int s = 0; s < c->plan.c.nslots; ++s)
            slot_expert[s] = c->plan.c.expert[s];
    return QMOE_OK;
}

}  // extern "C"
