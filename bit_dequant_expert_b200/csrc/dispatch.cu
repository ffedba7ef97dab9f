// Expert-parallel dispatch: the activation rows of a range of the token
// permutation, copied out in row order, each with its routing weight.  A rank
// that holds a shard of the experts sends every other rank the contiguous
// block of permuted rows whose experts that rank holds.
//
// Lily pages: "Perplexity built an inference engine for one model, one chip",
// second paragraph (each token is sent to eight of 256 experts).
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

// One warp per row: rows_out[i] = x[row_to_pair[row_begin + i] / K] (16-byte
// vectors), w_out[i] = topk_w[row_to_pair[row_begin + i]].  An out-of-range
// pair index zero-fills its row and raises MOE_ERR_BOUNDS.
__global__ void __launch_bounds__(256) k_gather_dispatch(GatherArgs a) {
    const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    griddep_launch_dependents();
    griddep_wait();   // the permutation comes from the previous grid
    if (i >= a.n_rows) return;
    const int p = __ldg(a.row_to_pair + a.row_begin + i);
    const bool ok = p >= 0 && p < a.T * a.K;
    if (!ok && lane == 0) set_error(a.err, MOE_ERR_BOUNDS);
    uint4* dst = reinterpret_cast<uint4*>(a.rows_out + (size_t)i * a.H);
    const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)(ok ? p / a.K : 0) * a.H);
    for (int c = lane; c < a.H / 8; c += 32) dst[c] = ok ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
    if (a.w_out && lane == 0) a.w_out[i] = ok && a.topk_w ? __ldg(a.topk_w + p) : 0.0f;
}

}  // namespace

cudaError_t launch_gather_dispatch(const GatherArgs& a, cudaStream_t st) {
    if (a.n_rows <= 0) return cudaSuccess;
    return launch_pdl(k_gather_dispatch, dim3((a.n_rows + 7) / 8), dim3(256), 0, st, a);
}

}  // namespace moe
