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

namespace moe {

// Logits of a TT-token x TE-expert tile per warp.  Lane s owns the 8-input
// chunks c = s, s+32, ... of H and accumulates them in order with fma (the
// product of two bf16 values is exact in fp32, so fma rounds once per step
// exactly like the contract); the 32 lane partials are then combined by the
// xor butterfly 16, 8, 4, 2, 1.  A block has 8 warps stacked along experts.
template <int TT, int TE>
__global__ void __launch_bounds__(256) k_router_logits(int T, int H, int E, const uint16_t* __restrict__ x,
                                                       const uint16_t* __restrict__ wr,
                                                       const float* __restrict__ bias, int64_t bias_stride,
                                                       float* __restrict__ logits) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int t0 = blockIdx.x * TT;
    const int e0 = (blockIdx.y * 8 + warp) * TE;
    if (e0 >= E) return;
    const int nchunk = H / 8;

    float acc[TT][TE];
#pragma unroll
    for (int a = 0; a < TT; ++a)
#pragma unroll
        for (int b = 0; b < TE; ++b) acc[a][b] = 0.0f;

    for (int c = lane; c < nchunk; c += 32) {
        uint4 xv[TT];
#pragma unroll
        for (int a = 0; a < TT; ++a) {
            const int t = t0 + a;
            xv[a] = (t < T) ? *reinterpret_cast<const uint4*>(x + (size_t)t * H + 8 * c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int b = 0; b < TE; ++b) {
            const uint4 wv = *reinterpret_cast<const uint4*>(wr + (size_t)(e0 + b) * H + 8 * c);
            const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int a = 0; a < TT; ++a) {
                const uint32_t xw[4] = {xv[a].x, xv[a].y, xv[a].z, xv[a].w};
                float s = acc[a][b];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    s = __fmaf_rn(bf16_lo(xw[q]), bf16_lo(ww[q]), s);
                    s = __fmaf_rn(bf16_hi(xw[q]), bf16_hi(ww[q]), s);
                }
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

// Order-preserving map of a finite float to uint32 (larger float -> larger
// key); -0.0 is folded onto +0.0 so the two tie.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f == 0.0f) f = 0.0f;
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// One warp per token.  Lane l holds the logits of experts l, l+32, ...; each
// of the K rounds takes the warp-wide maximum of (value, -index) and retires
// the winner.  Weights are the softmax over the K selected logits, which is
// the E-way softmax restricted to them and renormalised.
template <int EPL, int K>
__global__ void __launch_bounds__(256) k_topk(int T, int E, const float* __restrict__ logits,
                                              const float* __restrict__ bias, int64_t bias_stride,
                                              int32_t* __restrict__ idx, float* __restrict__ wout,
                                              int32_t* __restrict__ counts, int32_t* err) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    float v[EPL];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        float l = logits[(size_t)t * E + e];
        if (bias) l = __fadd_rn(l, bias[(int64_t)t * bias_stride + e]);
        v[i] = l;
        bad |= !isfinite(l);
    }
    if (__any_sync(0xFFFFFFFFu, bad)) {
        if (lane == 0) set_error(err, MOE_ERR_NONFINITE);
        if (lane < K) {
            idx[(size_t)t * K + lane] = lane;
            wout[(size_t)t * K + lane] = 1.0f / K;
            atomicAdd(&counts[lane], 1);
        }
        return;
    }
    uint32_t key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) key[i] = order_key(v[i]);
    uint32_t taken = 0;
    int sel_e[K];
    float sel_v[K];
#pragma unroll
    for (int r = 0; r < K; ++r) {
        unsigned long long best = 0ull;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const unsigned long long kk =
                ((unsigned long long)key[i] << 32) | (uint32_t)(~(uint32_t)(lane + 32 * i));
            if (!((taken >> i) & 1u) && kk > best) best = kk;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xFFFFFFFFu, best, off);
            best = o > best ? o : best;
        }
        const int e = (int)(~(uint32_t)best);
        if ((e & 31) == lane) taken |= 1u << (e >> 5);
        sel_e[r] = e;
        sel_v[r] = key_value((uint32_t)(best >> 32));
    }
    const float m = sel_v[0];
    float ex[K];
    float s = 0.0f;
#pragma unroll
    for (int r = 0; r < K; ++r) {
        ex[r] = expf(sel_v[r] - m);
        s += ex[r];
    }
#pragma unroll
    for (int r = 0; r < K; ++r) {
        if (lane == r) {
            idx[(size_t)t * K + r] = sel_e[r];
            wout[(size_t)t * K + r] = ex[r] / s;
            atomicAdd(&counts[sel_e[r]], 1);
        }
    }
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t st) {
    cudaError_t ce = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.E, st);
    if (ce != cudaSuccess) return ce;
    const float* lg = a.logits_in;
    const float* topk_bias = a.bias;
    if (!lg) {
        if (a.T <= 4) {
            dim3 grid(a.T, a.E / 8);
            k_router_logits<1, 1><<<grid, 256, 0, st>>>(a.T, a.H, a.E, a.x, a.w_router, a.bias, a.bias_stride,
                                                         a.logits_ws);
        } else {
            dim3 grid((a.T + 7) / 8, a.E / 64);
            k_router_logits<8, 8><<<grid, 256, 0, st>>>(a.T, a.H, a.E, a.x, a.w_router, a.bias, a.bias_stride,
                                                         a.logits_ws);
        }
        lg = a.logits_ws;
        topk_bias = nullptr;
    }
    k_topk<8, 8><<<(a.T + 7) / 8, 256, 0, st>>>(a.T, a.E, lg, topk_bias, a.bias_stride, a.topk_idx, a.topk_w,
                                                a.counts, a.err);
    return cudaGetLastError();
}

}  // namespace moe
