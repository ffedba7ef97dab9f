// Top-k selection of one token's router logits (shared by the router kernels
// and the fused decode kernel).
//
// Lily pages: "Perplexity built an inference engine for one model, one chip",
// second paragraph (a router picks eight subnetworks out of 256); the
// selection keeps the largest logits, the lowest expert index first among
// equal ones, and weights them by the softmax restricted to the selected
// logits (the 256-way softmax renormalised over the eight).
#pragma once

#include "common.cuh"

namespace moe {

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

// One warp per token, the logits already in registers: lane l holds the
// logits of experts l, l+32, ... in v.  Each of the K rounds takes the
// warp-wide maximum of the value, then the lowest expert index holding it,
// and retires the winner.  Weights are the softmax over the K selected
// logits, which is the E-way softmax restricted to them and renormalised.
// Lane r < K receives the r-th expert and its weight.  A non-finite logit
// anywhere in the row makes the selection experts 0..K-1 with weight 1/K and
// returns true (warp-uniform).
template <int EPL, int K>
__device__ __forceinline__ bool topk_from_values(const float (&v)[EPL], int& e_out, float& w_out) {
    const int lane = threadIdx.x & 31;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < EPL; ++i) bad |= !isfinite(v[i]);
    if (__any_sync(0xFFFFFFFFu, bad)) {
        e_out = lane;
        w_out = 1.0f / K;
        return true;
    }
    uint32_t key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) key[i] = order_key(v[i]);
    uint32_t taken = 0;
    int sel_e[K];
    float sel_v[K];
#pragma unroll
    for (int r = 0; r < K; ++r) {
        // this lane's best untaken (key, lowest index): its experts ascend with i
        uint32_t bk = 0u;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            if (!((taken >> i) & 1u) && (bi < 0 || key[i] > bk)) {
                bk = key[i];
                bi = i;
            }
        }
        // warp maximum of the key, then the lowest expert index holding it
        const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, bk);
        const uint32_t cand = (bi >= 0 && bk == kmax) ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu;
        const int e = (int)__reduce_min_sync(0xFFFFFFFFu, cand);
        if ((e & 31) == lane) taken |= 1u << (e >> 5);
        sel_e[r] = e;
        sel_v[r] = key_value(kmax);
    }
    const float m = sel_v[0];
    float ex[K];
    float s = 0.0f;
#pragma unroll
    for (int r = 0; r < K; ++r) {
        ex[r] = expf(sel_v[r] - m);
        s += ex[r];
    }
    e_out = 0;
    w_out = 0.0f;
#pragma unroll
    for (int r = 0; r < K; ++r) {
        if (lane == r) {
            e_out = sel_e[r];
            w_out = ex[r] / s;
        }
    }
    return false;
}

// topk_from_values on token t's row of an fp32 [T, E] logits array (read
// through L2), with an optional bias added first.
template <int EPL, int K>
__device__ __forceinline__ bool topk_select(int t, int E, const float* __restrict__ logits,
                                            const float* __restrict__ bias, int64_t bias_stride, int& e_out,
                                            float& w_out) {
    const int lane = threadIdx.x & 31;
    float v[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        float l = __ldcg(logits + (size_t)t * E + e);
        if (bias) l = __fadd_rn(l, bias[(int64_t)t * bias_stride + e]);
        v[i] = l;
    }
    return topk_from_values<EPL, K>(v, e_out, w_out);
}

// topk_select for token t, written to idx / wout [T, K] and counted in counts.
template <int EPL, int K>
__device__ __forceinline__ void topk_token(int t, int E, const float* __restrict__ logits,
                                           const float* __restrict__ bias, int64_t bias_stride,
                                           int32_t* __restrict__ idx, float* __restrict__ wout,
                                           int32_t* __restrict__ counts, int32_t* err) {
    const int lane = threadIdx.x & 31;
    int e;
    float w;
    if (topk_select<EPL, K>(t, E, logits, bias, bias_stride, e, w) && lane == 0) set_error(err, MOE_ERR_NONFINITE);
    if (lane < K) {
        idx[(size_t)t * K + lane] = e;
        wout[(size_t)t * K + lane] = w;
        atomicAdd(&counts[e], 1);
    }
}

}  // namespace moe
