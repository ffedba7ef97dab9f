// Weighted combine of the expert outputs into the layer output (bf16).
//
// Lily pages: "Perplexity built an inference engine for one model, one chip",
// second paragraph (eight routed experts plus one shared expert per token).
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

// y = bf16(y_acc), eight values per thread.
__global__ void __launch_bounds__(256) k_combine_scatter(size_t n8, const float* __restrict__ y_acc,
                                                         uint16_t* __restrict__ y) {
    griddep_launch_dependents();   // the next grid may start its own prologue
    griddep_wait();                // y_acc comes from the expert FFN
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        const float4 a = reinterpret_cast<const float4*>(y_acc)[2 * i];
        const float4 b = reinterpret_cast<const float4*>(y_acc)[2 * i + 1];
        uint4 o;
        o.x = pack_bf16x2(a.x, a.y);
        o.y = pack_bf16x2(a.z, a.w);
        o.z = pack_bf16x2(b.x, b.y);
        o.w = pack_bf16x2(b.z, b.w);
        reinterpret_cast<uint4*>(y)[i] = o;
    }
}

// y[t] = bf16(sum_slot w[t, slot] * rows[pair_to_row[t*K + slot]] + shared[t]),
// fp32 sum in slot order.  One block per token, eight outputs per thread.
template <int K>
__global__ void __launch_bounds__(256) k_combine_pairs(int T, int H, int has_shared, const uint16_t* __restrict__ rows,
                                                       const uint16_t* __restrict__ shared,
                                                       const int32_t* __restrict__ pair_to_row,
                                                       const float* __restrict__ w, uint16_t* __restrict__ y,
                                                       int32_t* err) {
    const int t = blockIdx.x;
    __shared__ int s_row[K];
    __shared__ float s_w[K];
    griddep_launch_dependents();   // the next grid may start its own prologue
    griddep_wait();                // rows come from the expert FFN
    if (threadIdx.x < K) {
        int r = pair_to_row[(size_t)t * K + threadIdx.x];
        if (r < 0 || r >= T * K) {
            set_error(err, MOE_ERR_BOUNDS);
            r = 0;
        }
        s_row[threadIdx.x] = r;
        s_w[threadIdx.x] = w[(size_t)t * K + threadIdx.x];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll
        for (int s = 0; s < K; ++s) {
            const uint4 v = *reinterpret_cast<const uint4*>(rows + (size_t)s_row[s] * H + 8 * c);
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[2 * q] = __fmaf_rn(s_w[s], bf16_lo(vw[q]), acc[2 * q]);
                acc[2 * q + 1] = __fmaf_rn(s_w[s], bf16_hi(vw[q]), acc[2 * q + 1]);
            }
        }
        if (has_shared) {
            const uint4 v = *reinterpret_cast<const uint4*>(shared + (size_t)t * H + 8 * c);
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[2 * q] += bf16_lo(vw[q]);
                acc[2 * q + 1] += bf16_hi(vw[q]);
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(y + (size_t)t * H + 8 * c) = o;
    }
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
    if (a.mode == MOE_MODE_SCATTER) {
        const size_t n8 = (size_t)a.T * a.H / 8;
        const int blocks = (int)std::min<size_t>((n8 + 255) / 256, 148 * 16);
        return launch_pdl(k_combine_scatter, dim3(blocks), dim3(256), 0, st, n8, a.y_acc, a.y);
    }
    return launch_pdl(k_combine_pairs<8>, dim3(a.T), dim3(256), 0, st, a.T, a.H, a.has_shared, a.rows, a.shared,
                      a.pair_to_row, a.w, a.y, a.err);
}

}  // namespace moe
