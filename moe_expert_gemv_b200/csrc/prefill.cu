// prefill.cu -- 128-token prefill chunk through the MoE layer as a grouped
// qGEMM (placeholder until the grouped kernels land).
#include "common.cuh"
#include "kernels.h"

namespace qmoe {

size_t prefill_workspace_layout(int E, int H, int I, int T, int top_k, void *base,
                                PrefillWorkspace *ws)
{
    const size_t rows = (size_t)T * top_k + T;
    size_t off = 0;
    const size_t counts_off = off;
    off = align_up(off + (size_t)E * 4, 256);
    const size_t offsets_off = off;
    off = align_up(off + (size_t)(E + 1) * 4, 256);
    const size_t pairs_off = off;
    off = align_up(off + (size_t)T * top_k * 4, 256);
    const size_t h_off = off;
    off = align_up(off + rows * I * 4, 256);
    const size_t r_off = off;
    off = align_up(off + rows * H * 4, 256);
    if (base && ws) {
        unsigned char *b = static_cast<unsigned char *>(base);
        ws->counts = reinterpret_cast<int32_t *>(b + counts_off);
        ws->offsets = reinterpret_cast<int32_t *>(b + offsets_off);
        ws->pairs = reinterpret_cast<int32_t *>(b + pairs_off);
        ws->h = reinterpret_cast<float *>(b + h_off);
        ws->r = reinterpret_cast<float *>(b + r_off);
    }
    return off;
}

cudaError_t launch_prefill(const PrefillArgs &, const LaunchCfg &) { return cudaErrorNotSupported; }

}  // namespace qmoe
