// Router: fp32 logits in the contract order, top-k selection with
// lowest-index tie-break, renormalised softmax weights and per-expert counts.
//
// Lily pages: "Perplexity built an inference engine for one model, one chip",
// second paragraph (a router picks eight subnetworks out of 256) and third
// paragraph (routing is never handed back to the CPU); "Perplexity open-
// sources Lily", section "The Narrowness Is the Performance Argument"
// (GPU-resident expert routing).
#include <cuda.h>

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

// ------------------------------------------------------------------ prefill router, weights resident
//
// Many tokens: each CTA keeps the router rows of 32 experts (32 x H bf16,
// 128 KB at H = 2048) in shared memory and streams 16-token tiles of x
// through a ring of 256-input stages (TMA, one producer thread).  Warp
// (ti, ei) of the 8 consumer warps owns tokens 8 ti .. 8 ti + 7 and experts
// 8 ei .. 8 ei + 7 of the tile; lane s is slice s of the contract order and
// reads its 8-input chunk 32 kc + s of stage kc with one 16-byte load per row
// (a warp's 32 loads cover 512 contiguous bytes: no bank conflicts).  The
// (16-token, 32-expert) steps are dealt to the CTAs in contiguous runs in
// expert-group-major order, so a CTA reloads the resident rows at most once
// or twice, and every token row is read from L2 E / 32 times in all.
//
// The 32 slice partials of the warp's 64 outputs are combined by a
// transposing reduction: at the step with distance d, a lane keeps the half
// of its list selected by its lane bit d and adds the partner's value of the
// same outputs.  Each output's sum is built from the same pairs as the xor
// butterfly 16, 8, 4, 2, 1 (fp32 addition is commutative, so a + b and b + a
// round alike), with 62 adds per lane instead of 320.  Lane l ends up
// holding outputs 2 l and 2 l + 1 of the tile.
namespace {

constexpr int kRwExperts = 32;     // resident experts per CTA
constexpr int kRwTokens = 16;      // tokens per step
constexpr int kRwK = 256;          // inputs per stage (32 chunks of 8)
constexpr int kRwStages = 8;
constexpr int kRwConsumerWarps = 8;
constexpr int kRwThreads = 32 * (kRwConsumerWarps + 1);
constexpr int kRwMaxH = 2048;
constexpr size_t kRwStageBytes = (size_t)kRwTokens * kRwK * 2;

size_t rw_smem_bytes(int H) {
    return (size_t)kRwExperts * H * 2 + kRwStages * kRwStageBytes + 64 * sizeof(uint64_t) + 128;
}

struct RwSmemBars {
    uint64_t x_full[kRwStages];
    uint64_t x_empty[kRwStages];
    uint64_t w_full;
    uint64_t w_empty;
};

__global__ void __launch_bounds__(kRwThreads, 1)
    k_router_wres(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap w_map, int T, int H,
                  int E, const float* __restrict__ bias, int64_t bias_stride, float* __restrict__ logits,
                  int32_t* __restrict__ counts, int32_t* err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint16_t* ws = reinterpret_cast<uint16_t*>(smem_raw);                                 // [H/256][32][256]
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw + (size_t)kRwExperts * H * 2);    // [stages][16][256]
    RwSmemBars& bars = *reinterpret_cast<RwSmemBars*>(smem_raw + (size_t)kRwExperts * H * 2 +
                                                      kRwStages * kRwStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkc = H / kRwK;
    const int ntb = (T + kRwTokens - 1) / kRwTokens;
    const int nsteps = (E / kRwExperts) * ntb;
    const int s_lo = (int)((int64_t)blockIdx.x * nsteps / gridDim.x);
    const int s_hi = (int)((int64_t)(blockIdx.x + 1) * nsteps / gridDim.x);

    // the top-k kernel that follows on the stream accumulates the counts
    if (counts && blockIdx.x == 0)
        for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRwStages; ++i) {
            mbar_init(&bars.x_full[i], 1);
            mbar_init(&bars.x_empty[i], kRwConsumerWarps);
        }
        mbar_init(&bars.w_full, 1);
        mbar_init(&bars.w_empty, kRwConsumerWarps);
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kRwConsumerWarps) {
        // producer: the resident rows at every change of expert group, then x stages
        if (lane == 0) {
            prefetch_tensormap(&x_map);
            prefetch_tensormap(&w_map);
            uint32_t it = 0, nload = 0;
            int group = -1;
            for (int s = s_lo; s < s_hi; ++s) {
                const int g = s / ntb, tb = s - g * ntb;
                if (g != group) {
                    if (nload > 0 && !mbar_wait_bounded(&bars.w_empty, (nload - 1) & 1, err)) break;
                    mbar_arrive_expect_tx(&bars.w_full, (uint32_t)(kRwExperts * H * 2));
                    for (int kc = 0; kc < nkc; ++kc)
                        tma_load_2d(ws + (size_t)kc * kRwExperts * kRwK, &w_map, kc * kRwK, g * kRwExperts,
                                    &bars.w_full);
                    group = g;
                    ++nload;
                }
                bool ok = true;
                for (int kc = 0; kc < nkc; ++kc, ++it) {
                    const uint32_t st = it % kRwStages;
                    if (it >= kRwStages && !mbar_wait_bounded(&bars.x_empty[st], ((it / kRwStages) - 1) & 1, err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars.x_full[st], (uint32_t)kRwStageBytes);
                    tma_load_2d(xs + (size_t)st * kRwTokens * kRwK, &x_map, kc * kRwK, tb * kRwTokens,
                                &bars.x_full[st]);
                }
                if (!ok) break;
            }
        }
        return;
    }

    const int ti = warp >> 2, ei = warp & 3;
    uint32_t it = 0, nload = 0;
    int group = -1;
    for (int s = s_lo; s < s_hi; ++s) {
        const int g = s / ntb, tb = s - g * ntb;
        if (g != group) {
            if (!mbar_wait_bounded(&bars.w_full, nload & 1, err)) return;
            group = g;
            ++nload;
        }
        float acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
        for (int kc = 0; kc < nkc; ++kc, ++it) {
            const uint32_t st = it % kRwStages;
            if (!mbar_wait_bounded(&bars.x_full[st], (it / kRwStages) & 1, err)) return;
            const uint16_t* xrow = xs + (size_t)st * kRwTokens * kRwK + (size_t)(8 * ti) * kRwK + 8 * lane;
            const uint16_t* wrow = ws + (size_t)kc * kRwExperts * kRwK + (size_t)(8 * ei) * kRwK + 8 * lane;
            uint4 xr[8], wr[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) xr[a] = *reinterpret_cast<const uint4*>(xrow + a * kRwK);
#pragma unroll
            for (int b = 0; b < 8; ++b) wr[b] = *reinterpret_cast<const uint4*>(wrow + b * kRwK);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float xl[8], xh[8], wl[8], wh[8];
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    const uint32_t u = q == 0 ? xr[a].x : q == 1 ? xr[a].y : q == 2 ? xr[a].z : xr[a].w;
                    xl[a] = bf16_lo(u);
                    xh[a] = bf16_hi(u);
                }
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    const uint32_t u = q == 0 ? wr[b].x : q == 1 ? wr[b].y : q == 2 ? wr[b].z : wr[b].w;
                    wl[b] = bf16_lo(u);
                    wh[b] = bf16_hi(u);
                }
                // inputs 2q then 2q + 1 of the chunk, in order, for every output
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 8; ++b) acc[8 * a + b] = __fmaf_rn(xl[a], wl[b], acc[8 * a + b]);
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 8; ++b) acc[8 * a + b] = __fmaf_rn(xh[a], wh[b], acc[8 * a + b]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.x_empty[st]);
        }
        // the resident rows are free once the last step of this group is done
        if (s + 1 == s_hi || (s + 1) / ntb != g) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.w_empty);
        }
        // transposing reduction over the 32 slices (distances 16, 8, 4, 2, 1)
#pragma unroll
        for (int d = 16, half = 32; d >= 1; d >>= 1, half >>= 1) {
            const bool up = (lane & d) != 0;
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = up ? acc[i] : acc[i + half];
                const float keep = up ? acc[i + half] : acc[i];
                acc[i] = __fadd_rn(keep, __shfl_xor_sync(0xFFFFFFFFu, send, d));
            }
        }
        const int t = tb * kRwTokens + 8 * ti + (lane >> 2);
        const int e = g * kRwExperts + 8 * ei + 2 * (lane & 3);
        if (t < T) {
            float v0 = acc[0], v1 = acc[1];
            if (bias) {
                v0 = __fadd_rn(v0, bias[(int64_t)t * bias_stride + e]);
                v1 = __fadd_rn(v1, bias[(int64_t)t * bias_stride + e + 1]);
            }
            *reinterpret_cast<float2*>(logits + (size_t)t * E + e) = make_float2(v0, v1);
        }
    }
}

using RwEncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

RwEncodeTiled rw_encode_fn() {
    static RwEncodeTiled fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<RwEncodeTiled>(p);
    }
    return fn;
}

// A [rows, H] bf16 matrix read in boxes of 256 inputs x box_rows rows (rows
// past the end read as zero).
bool rw_make_map(CUtensorMap* m, const uint16_t* base, int rows, int H, int box_rows) {
    RwEncodeTiled enc = rw_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)H * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kRwK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int rw_num_sms() {
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    return sms[dev];
}

bool rw_supported(int T, int H, int E) {
    return T >= 64 && H % kRwK == 0 && H <= kRwMaxH && E % kRwExperts == 0;
}

cudaError_t launch_router_wres(const RouterArgs& a, cudaStream_t st) {
    CUtensorMap x_map, w_map;
    if (!rw_make_map(&x_map, a.x, a.T, a.H, kRwTokens) || !rw_make_map(&w_map, a.w_router, a.E, a.H, kRwExperts))
        return cudaErrorInvalidValue;
    const int nsteps = (a.E / kRwExperts) * ((a.T + kRwTokens - 1) / kRwTokens);
    const int sms = rw_num_sms();
    const int G = sms < nsteps ? sms : nsteps;
    if (G <= 0) return cudaErrorInvalidValue;
    const size_t smem = rw_smem_bytes(a.H);
    cudaError_t ce = cudaFuncSetAttribute(k_router_wres, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (ce != cudaSuccess) return ce;
    k_router_wres<<<G, kRwThreads, smem, st>>>(x_map, w_map, a.T, a.H, a.E, a.bias, a.bias_stride, a.logits_ws,
                                               a.counts, a.err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_logits(const RouterArgs& a, cudaStream_t st) {
    if (rw_supported(a.T, a.H, a.E) && ((uintptr_t)a.x & 15) == 0 && ((uintptr_t)a.w_router & 15) == 0)
        return launch_router_wres(a, st);
    // 4 tokens x 16 experts per warp, 8 warps over 128 experts: the x chunk of
    // a token is widened once for 16 experts, and the small accumulator tile
    // leaves room for two blocks per SM
    dim3 grid((a.T + 3) / 4, a.E / 128);
    k_router_logits<4, 16><<<grid, 256, 0, st>>>(a.T, a.H, a.E, a.x, a.w_router, a.bias, a.bias_stride, a.logits_ws,
                                                  a.counts);
    return cudaGetLastError();
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
        cudaError_t ce = launch_router_logits(a, st);   // bias added there; counts zeroed
        if (ce != cudaSuccess) return ce;
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
