// Router: fp32 logits in the contract order, top-k selection with
// lowest-index tie-break, renormalised softmax weights and per-expert counts.
//
// Lily pages: "Perplexity built an inference engine for one model, one chip",
// second paragraph (a router picks eight subnetworks out of 256) and third
// paragraph (routing is never handed back to the CPU); "Perplexity open-
// sources Lily", section "The Narrowness Is the Performance Argument"
// (GPU-resident expert routing).
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {

// Logits of a TT-token x TE-expert tile per warp.  Lane s owns the 8-input
// chunks c = s, s+32, ... of H and accumulates them in order with fma (the
// product of two bf16 values is exact in fp32, so fma rounds once per step
// exactly like the contract); the 32 lane partials are then combined by the
// xor butterfly 16, 8, 4, 2, 1.  A block has 8 warps stacked along experts.
template <int TT, int TE>
__device__ __forceinline__ void router_tile(int T, int H, int E, int t0, int e0, const uint16_t* __restrict__ x,
                                            const uint16_t* __restrict__ wr, const float* __restrict__ bias,
                                            int64_t bias_stride, float* __restrict__ logits) {
    const int lane = threadIdx.x & 31;
    if (e0 >= E) return;
    const int nchunk = H / 8;

    float acc[TT][TE];
#pragma unroll
    for (int a = 0; a < TT; ++a)
#pragma unroll
        for (int b = 0; b < TE; ++b) acc[a][b] = 0.0f;

    for (int c = lane; c < nchunk; c += 32) {
        // this chunk of every token, widened to fp32 once and reused for all TE experts
        float xf[TT][8];
#pragma unroll
        for (int a = 0; a < TT; ++a) {
            const int t = t0 + a;
            const uint4 xv = (t < T) ? *reinterpret_cast<const uint4*>(x + (size_t)t * H + 8 * c) : make_uint4(0, 0, 0, 0);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                xf[a][2 * q] = bf16_lo(xw[q]);
                xf[a][2 * q + 1] = bf16_hi(xw[q]);
            }
        }
#pragma unroll
        for (int b = 0; b < TE; ++b) {
            const uint4 wv = *reinterpret_cast<const uint4*>(wr + (size_t)(e0 + b) * H + 8 * c);
            const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
            float wf[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                wf[2 * q] = bf16_lo(ww[q]);
                wf[2 * q + 1] = bf16_hi(ww[q]);
            }
#pragma unroll
            for (int a = 0; a < TT; ++a) {
                float s = acc[a][b];
#pragma unroll
                for (int j = 0; j < 8; ++j) s = __fmaf_rn(xf[a][j], wf[j], s);   // inputs ascending in the chunk
                acc[a][b] = s;
            }
        }
    }
#pragma unroll
    for (int a = 0; a < TT; ++a)
#pragma unroll
        for (int b = 0; b < TE; ++b) {
            float v = acc[a][b];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
            acc[a][b] = v;
        }
#pragma unroll
    for (int i = 0; i < TT * TE; ++i) {
        if ((i & 31) == lane) {
            const int t = t0 + i / TE;
            const int e = e0 + i % TE;
            if (t < T) {
                float v = acc[i / TE][i % TE];
                if (bias) v = __fadd_rn(v, bias[(int64_t)t * bias_stride + e]);
                logits[(size_t)t * E + e] = v;
            }
        }
    }
}

template <int TT, int TE>
__global__ void __launch_bounds__(256) k_router_logits(int T, int H, int E, const uint16_t* __restrict__ x,
                                                       const uint16_t* __restrict__ wr,
                                                       const float* __restrict__ bias, int64_t bias_stride,
                                                       float* __restrict__ logits, int32_t* __restrict__ counts) {
    // the top-k kernel that follows on the stream accumulates the counts
    if (counts && blockIdx.x == 0 && blockIdx.y == 0)
        for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = 0;
    const int warp = threadIdx.x >> 5;
    router_tile<TT, TE>(T, H, E, blockIdx.x * TT, (blockIdx.y * 8 + warp) * TE, x, wr, bias, bias_stride, logits);
}

template <int EPL, int K>
__global__ void __launch_bounds__(256) k_topk(int T, int E, const float* __restrict__ logits,
                                              const float* __restrict__ bias, int64_t bias_stride,
                                              int32_t* __restrict__ idx, float* __restrict__ wout,
                                              int32_t* __restrict__ counts, int32_t* err) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    topk_token<EPL, K>(t, E, logits, bias, bias_stride, idx, wout, counts, err);
}

// A handful of tokens (T <= 8) in one launch: every block computes the logits
// of all tokens for 8 experts (one per warp); the last block to finish (an
// atomic ticket, reset by that block for the next call) selects the top-k of
// every token and writes the counts.
__global__ void __launch_bounds__(256) k_route_small(int T, int H, int E, const uint16_t* __restrict__ x,
                                                     const uint16_t* __restrict__ wr,
                                                     const float* __restrict__ bias, int64_t bias_stride,
                                                     float* __restrict__ logits, int32_t* __restrict__ idx,
                                                     float* __restrict__ wout, int32_t* __restrict__ counts,
                                                     uint32_t* ticket, int32_t* err) {
    __shared__ bool last;
    const int warp = threadIdx.x >> 5;
    router_tile<8, 1>(T, H, E, 0, blockIdx.x * 8 + warp, x, wr, bias, bias_stride, logits);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = 0;
    __syncthreads();
    if (warp < T) topk_token<8, 8>(warp, E, logits, nullptr, 0, idx, wout, counts, err);
    if (threadIdx.x == 0) *ticket = 0u;
}

// A handful of tokens (T <= 8, H <= 2048): one warp per expert, two experts
// per block, so the router matrix streams through 128 SMs.  Each lane issues
// all of its weight chunks at once, before waiting on the previous grid (the
// weights never depend on it); x is staged in shared memory.  The logits of
// (token, expert) follow the same contract order as router_tile.  The last
// block (atomic ticket, reset by that block) selects the top-k and counts.
constexpr int kSmallMaxChunksPerLane = 8;   // H <= 8 * 8 * 32

__global__ void __launch_bounds__(64) k_route_small_wide(int T, int H, int E, const uint16_t* __restrict__ x,
                                                         const uint16_t* __restrict__ wr,
                                                         const float* __restrict__ bias, int64_t bias_stride,
                                                         float* __restrict__ logits, int32_t* __restrict__ idx,
                                                         float* __restrict__ wout, int32_t* __restrict__ counts,
                                                         uint32_t* ticket, int32_t* err) {
    extern __shared__ uint4 xs4[];   // [T][H/8]
    __shared__ bool last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 2 + warp;
    const int nchunk = H / 8;
    uint4 wv[kSmallMaxChunksPerLane];
#pragma unroll
    for (int i = 0; i < kSmallMaxChunksPerLane; ++i) {
        const int c = lane + 32 * i;
        wv[i] = c < nchunk ? ldg_v4(wr + (size_t)e * H + 8 * c) : make_uint4(0, 0, 0, 0);
    }
    griddep_launch_dependents();   // the next grid may start its own prologue
    griddep_wait();                // x may come from the previous grid
    for (int q = threadIdx.x; q < T * nchunk; q += blockDim.x) xs4[q] = reinterpret_cast<const uint4*>(x)[q];
    __syncthreads();
    float acc[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.0f;
#pragma unroll
    for (int i = 0; i < kSmallMaxChunksPerLane; ++i) {
        const int c = lane + 32 * i;
        if (c >= nchunk) break;
        const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
        float wf[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            wf[2 * q] = bf16_lo(ww[q]);
            wf[2 * q + 1] = bf16_hi(ww[q]);
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            if (t < T) {
                const uint4 xv = xs4[t * nchunk + c];
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                float sacc = acc[t];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    sacc = __fmaf_rn(bf16_lo(xw[q]), wf[2 * q], sacc);   // inputs ascending in the chunk
                    sacc = __fmaf_rn(bf16_hi(xw[q]), wf[2 * q + 1], sacc);
                }
                acc[t] = sacc;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        if (t < T) {   // T is the same for the whole warp
            float v = acc[t];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
            if (lane == t) {
                if (bias) v = __fadd_rn(v, bias[(int64_t)t * bias_stride + e]);
                logits[(size_t)t * E + e] = v;
            }
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int q = threadIdx.x; q < E; q += blockDim.x) counts[q] = 0;
    __syncthreads();
    for (int t = warp; t < T; t += 2) topk_token<8, 8>(t, E, logits, nullptr, 0, idx, wout, counts, err);
    if (threadIdx.x == 0) *ticket = 0u;
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t st) {
    if (!a.logits_in && a.T <= 8 && a.E == 256 && a.H <= 8 * kSmallMaxChunksPerLane * 32) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(a.E / 2);
        cfg.blockDim = dim3(64);
        cfg.dynamicSmemBytes = (size_t)a.T * a.H * 2;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, k_route_small_wide, a.T, a.H, a.E, a.x, a.w_router, a.bias, a.bias_stride,
                                  a.logits_ws, a.topk_idx, a.topk_w, a.counts, a.ticket, a.err);
    }
    if (!a.logits_in && a.T <= 8 && a.E == 256) {
        k_route_small<<<a.E / 8, 256, 0, st>>>(a.T, a.H, a.E, a.x, a.w_router, a.bias, a.bias_stride, a.logits_ws,
                                               a.topk_idx, a.topk_w, a.counts, a.ticket, a.err);
        return cudaGetLastError();
    }
    const float* lg = a.logits_in;
    const float* topk_bias = a.bias;
    if (!lg) {
        // 4 tokens x 16 experts per warp, 8 warps over 128 experts: the x chunk of
        // a token is widened once for 16 experts, and the small accumulator tile
        // leaves room for two blocks per SM
        dim3 grid((a.T + 3) / 4, a.E / 128);
        k_router_logits<4, 16><<<grid, 256, 0, st>>>(a.T, a.H, a.E, a.x, a.w_router, a.bias, a.bias_stride,
                                                      a.logits_ws, a.counts);
        lg = a.logits_ws;
        topk_bias = nullptr;
    } else {
        cudaError_t ce = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, st);
        if (ce != cudaSuccess) return ce;
    }
    k_topk<8, 8><<<(a.T + 7) / 8, 256, 0, st>>>(a.T, a.E, lg, topk_bias, a.bias_stride, a.topk_idx, a.topk_w,
                                                a.counts, a.err);
    return cudaGetLastError();
}

}  // namespace moe
