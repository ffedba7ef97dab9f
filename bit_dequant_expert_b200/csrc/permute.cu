// Token permutation: per-expert counts, exclusive scan and the stable
// expert-major order of the (token, slot) pairs, all on the device.
//
// Lily pages: "Perplexity built an inference engine for one model, one chip",
// third paragraph (leaving the routing step on the GPU throughout was worth
// +89% prefill at 512 tokens); "Perplexity's Lily brings fast local AI to
// Apple silicon Macs", section "Where the Engine Gains Speed" (routing kept
// on the GPU during prefill).
//
// Tokens are cut into chunks of 256.  For each chunk a block builds, per
// expert, a 256-bit mask of the chunk's tokens that chose it (a token never
// chooses an expert twice, so one bit per (expert, token) suffices).  The
// rank of a pair among its expert's pairs of the chunk is the popcount of the
// mask below its token, which makes the order stable by token without any
// ordering of atomics.  A one-block scan then turns the chunk histograms into
// per-(chunk, expert) row bases.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

constexpr int kChunk = 256;

// Builds the chunk's masks in shared memory; returns false (and records the
// error) if a routing index is out of range or repeated within a token.
template <int K>
__device__ void build_masks(int T, int E, int chunk, const int32_t* __restrict__ idx, uint32_t* mask,
                            int32_t* err) {
    for (int i = threadIdx.x; i < E * (kChunk / 32); i += blockDim.x) mask[i] = 0u;
    __syncthreads();
    const int t = chunk * kChunk + threadIdx.x;
    if (threadIdx.x < kChunk && t < T) {
        int sel[K];
        bool ok = true;
#pragma unroll
        for (int a = 0; a < K; ++a) {
            sel[a] = idx[(size_t)t * K + a];
            ok &= (sel[a] >= 0 && sel[a] < E);
#pragma unroll
            for (int b = 0; b < a; ++b) ok &= (sel[a] != sel[b]);
        }
        if (!ok) set_error(err, MOE_ERR_BOUNDS);
#pragma unroll
        for (int a = 0; a < K; ++a)
            if (sel[a] >= 0 && sel[a] < E)
                atomicOr(&mask[sel[a] * (kChunk / 32) + (threadIdx.x >> 5)], 1u << (threadIdx.x & 31));
    }
    __syncthreads();
}

__device__ __forceinline__ int mask_rank(const uint32_t* m, int tl) {
    int r = 0;
    for (int w = 0; w < (tl >> 5); ++w) r += __popc(m[w]);
    return r + __popc(m[tl >> 5] & ((1u << (tl & 31)) - 1u));
}

__device__ __forceinline__ int mask_count(const uint32_t* m) {
    int r = 0;
#pragma unroll
    for (int w = 0; w < kChunk / 32; ++w) r += __popc(m[w]);
    return r;
}

// Exclusive block scan of one int per thread (blockDim.x a multiple of 32, <= 1024).
__device__ int block_exclusive_scan(int v, int* total) {
    __shared__ int warp_sums[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nwarp ? warp_sums[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, s, off);
            if (lane >= off) s += o;
        }
        warp_sums[lane] = s;   // inclusive prefix of warp sums
    }
    __syncthreads();
    const int base = warp > 0 ? warp_sums[warp - 1] : 0;
    if (total) *total = warp_sums[nwarp - 1];
    const int out = base + inc - v;
    __syncthreads();
    return out;
}

// Pass 1: chunk histograms hist[chunk][E] and the in-chunk rank of every pair.
template <int K>
__global__ void __launch_bounds__(256) k_perm_hist(int T, int E, const int32_t* __restrict__ idx,
                                                   int32_t* __restrict__ hist, int32_t* __restrict__ rank,
                                                   int32_t* err) {
    extern __shared__ uint32_t mask[];
    const int chunk = blockIdx.x;
    build_masks<K>(T, E, chunk, idx, mask, err);
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        hist[(size_t)chunk * E + e] = mask_count(mask + e * (kChunk / 32));
    const int t = chunk * kChunk + threadIdx.x;
    if (t < T) {
#pragma unroll
        for (int a = 0; a < K; ++a) {
            const int e = idx[(size_t)t * K + a];
            rank[(size_t)t * K + a] = (e >= 0 && e < E) ? mask_rank(mask + e * (kChunk / 32), threadIdx.x) : 0;
        }
    }
}

// Pass 2 (one block, one thread per expert): per-expert totals, check against
// counts, exclusive scan -> offsets, and per-(chunk, expert) row bases.
__global__ void __launch_bounds__(1024) k_perm_scan(int T, int E, int nchunk, int K, int32_t* __restrict__ hist,
                                                    const int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets, int32_t* err) {
    const int e = threadIdx.x;
    int run = 0;
    if (e < E)
        for (int c = 0; c < nchunk; ++c) {
            const int v = hist[(size_t)c * E + e];
            hist[(size_t)c * E + e] = run;
            run += v;
        }
    if (e < E && counts && counts[e] != run) set_error(err, MOE_ERR_BOUNDS);
    int total = 0;
    const int off = block_exclusive_scan(e < E ? run : 0, &total);
    if (e < E) {
        offsets[e] = off;
        for (int c = 0; c < nchunk; ++c) hist[(size_t)c * E + e] += off;
    }
    if (e == 0) {
        offsets[E] = total;
        if (total != T * K) set_error(err, MOE_ERR_BOUNDS);
    }
}

// Pass 3: row of every pair = base[chunk][expert] + rank.
template <int K>
__global__ void __launch_bounds__(256) k_perm_scatter(int T, int E, const int32_t* __restrict__ idx,
                                                      const int32_t* __restrict__ base,
                                                      const int32_t* __restrict__ rank,
                                                      int32_t* __restrict__ row_to_pair,
                                                      int32_t* __restrict__ pair_to_row, int32_t* err) {
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= T * K) return;
    const int t = p / K;
    const int e = idx[p];
    int row = -1;
    if (e >= 0 && e < E) row = base[(size_t)(t / kChunk) * E + e] + rank[p];
    if (row < 0 || row >= T * K) {
        set_error(err, MOE_ERR_BOUNDS);
        pair_to_row[p] = 0;
        return;
    }
    row_to_pair[row] = p;
    pair_to_row[p] = row;
}

// All three passes in one block for T <= 256 (one chunk): the decode and
// small-batch case, one launch.
template <int K>
__global__ void __launch_bounds__(256) k_perm_small(int T, int E, const int32_t* __restrict__ idx,
                                                    const int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ row_to_pair,
                                                    int32_t* __restrict__ pair_to_row, int32_t* err) {
    extern __shared__ uint32_t mask[];
    int* s_off = reinterpret_cast<int*>(mask + E * (kChunk / 32));
    griddep_launch_dependents();   // the next grid may start its own prologue
    griddep_wait();                // idx and counts come from the router
    build_masks<K>(T, E, 0, idx, mask, err);
    // E <= 1024: each thread scans E / blockDim.x experts in order
    const int per = (E + blockDim.x - 1) / blockDim.x;
    int local = 0;
    for (int q = 0; q < per; ++q) {
        const int e = threadIdx.x * per + q;
        if (e < E) local += mask_count(mask + e * (kChunk / 32));
    }
    int total = 0;
    int run = block_exclusive_scan(local, &total);
    for (int q = 0; q < per; ++q) {
        const int e = threadIdx.x * per + q;
        if (e < E) {
            const int c = mask_count(mask + e * (kChunk / 32));
            if (counts && counts[e] != c) set_error(err, MOE_ERR_BOUNDS);
            s_off[e] = run;
            offsets[e] = run;
            run += c;
        }
    }
    if (threadIdx.x == 0) {
        offsets[E] = total;
        if (total != T * K) set_error(err, MOE_ERR_BOUNDS);
    }
    __syncthreads();
    const int t = threadIdx.x;
    if (t < T) {
#pragma unroll
        for (int a = 0; a < K; ++a) {
            const int p = t * K + a;
            const int e = idx[p];
            int row = -1;
            if (e >= 0 && e < E) row = s_off[e] + mask_rank(mask + e * (kChunk / 32), t);
            if (row < 0 || row >= T * K) {
                set_error(err, MOE_ERR_BOUNDS);
                pair_to_row[p] = 0;
                continue;
            }
            row_to_pair[row] = p;
            pair_to_row[p] = row;
        }
    }
}

size_t permute_ws_bytes(int T, int E, int K) {
    const size_t nchunk = (size_t)(T + kChunk - 1) / kChunk;
    return align256(nchunk * E * sizeof(int32_t)) + align256((size_t)T * K * sizeof(int32_t));
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st) {
    const size_t mask_bytes = (size_t)a.E * (kChunk / 32) * sizeof(uint32_t);
    if (a.T <= kChunk) {
        return launch_pdl(k_perm_small<8>, dim3(1), dim3(256), mask_bytes + a.E * sizeof(int), st, a.T, a.E,
                          a.topk_idx, a.counts, a.offsets, a.row_to_pair, a.pair_to_row, a.err);
    }
    const int nchunk = (a.T + kChunk - 1) / kChunk;
    int32_t* hist = reinterpret_cast<int32_t*>(a.scratch);
    int32_t* rank = reinterpret_cast<int32_t*>(a.scratch + align256((size_t)nchunk * a.E * sizeof(int32_t)));
    k_perm_hist<8><<<nchunk, 256, mask_bytes, st>>>(a.T, a.E, a.topk_idx, hist, rank, a.err);
    k_perm_scan<<<1, ((a.E + 31) / 32) * 32, 0, st>>>(a.T, a.E, nchunk, 8, hist, a.counts, a.offsets, a.err);
    const int npairs = a.T * 8;
    k_perm_scatter<8><<<(npairs + 255) / 256, 256, 0, st>>>(a.T, a.E, a.topk_idx, hist, rank, a.row_to_pair,
                                                           a.pair_to_row, a.err);
    return cudaGetLastError();
}

}  // namespace moe
