// moe_permute_static: the token permutation without a caller-provided
// workspace, for callers that cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory: a plugin running inside
// a host runtime that owns every device allocation and only hands it
// pre-allocated input and output buffers, or a real-time path where
// cudaMalloc (which can synchronise the whole device) is not permitted, or a
// deployment whose device-memory budget is fixed by another allocator.  For
// them this entry point keeps its scratch in a file-scope device array of a
// fixed size instead of asking for a workspace.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "api_range.h"

namespace {

constexpr int kStaticMaxTokens = MOE_STATIC_MAX_TOKENS;
// Chunk histograms [ceil(T/256)][E] and per-pair ranks [T][k] for T = 16384,
// E = 256, k = 8, each section 256-byte aligned: 64 KiB + 512 KiB.
constexpr size_t kStaticScratchBytes = ((kStaticMaxTokens + 255) / 256) * 256 * 4 + (size_t)kStaticMaxTokens * 8 * 4;

// Every GPU that loads this library holds this array until the process exits.
__device__ __align__(256) uint8_t g_permute_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side handle, so the address is looked up
// once per device (with that device current) and cached.
int32_t scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" int32_t moe_permute_static(const moe_config_t* cfg, int32_t T, const int32_t* topk_idx,
                                      const int32_t* counts, int32_t* offsets, int32_t* row_to_pair,
                                      int32_t* pair_to_row, int32_t* err_out, void* stream) {
    moe::ApiRange api_range("moe_permute_static");
    if (!cfg) return MOE_ERR_INVALID_ARG;
    if (cfg->num_experts != 256 || cfg->top_k != 8 || cfg->group_size != 64 || cfg->hidden < 256 ||
        cfg->hidden % 256 != 0 || cfg->inter < 128 || cfg->inter % 128 != 0 ||
        (cfg->has_shared != 0 && cfg->has_shared != 1))
        return MOE_ERR_UNSUPPORTED;
    if (T < 1) return MOE_ERR_INVALID_ARG;
    if (T > kStaticMaxTokens) return MOE_ERR_UNSUPPORTED;   // beyond the fixed scratch array
    if (moe::permute_ws_bytes(T, cfg->num_experts, cfg->top_k) > kStaticScratchBytes) return MOE_ERR_UNSUPPORTED;
    if (!topk_idx || !offsets || !row_to_pair || !pair_to_row) return MOE_ERR_INVALID_ARG;
    if (!aligned4(topk_idx) || !aligned4(counts) || !aligned4(offsets) || !aligned4(row_to_pair) ||
        !aligned4(pair_to_row) || !aligned4(err_out))
        return MOE_ERR_INVALID_ARG;
    void* scratch = nullptr;
    int32_t st = scratch_address(&scratch);
    if (st != MOE_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (err_out && cudaMemsetAsync(err_out, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    moe::PermuteArgs a;
    a.T = T;
    a.E = cfg->num_experts;
    a.topk_idx = topk_idx;
    a.counts = counts;
    a.offsets = offsets;
    a.row_to_pair = row_to_pair;
    a.pair_to_row = pair_to_row;
    a.scratch = static_cast<uint8_t*>(scratch);
    a.err = err_out;
    return moe::launch_permute(a, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
