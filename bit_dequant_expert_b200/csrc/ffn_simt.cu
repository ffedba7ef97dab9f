// Expert FFNs on CUDA cores: 4-bit weights are dequantised in registers
// (fp32 fma of scale * q + bias) and consumed at once, so no expanded weight
// array exists anywhere.  The general-shape path and the reference for the
// tensor-core path's epilogues.
//
// Lily pages: "Perplexity's Lily brings fast local AI to Apple silicon Macs",
// section "Where the Engine Gains Speed" (weights reconstructed inside the
// grouped GEMM, one tile at a time); "Perplexity built an inference engine
// for one model, one chip", second paragraph (eight routed experts plus one
// shared expert that sees every token).
#include "common.cuh"
#include "kernels.h"

namespace moe {

// Row tiles of the grouped problem: expert e's rows offsets[e]..offsets[e+1]-1
// in tiles of R, then the shared expert's T rows (if any) in tiles of R.
// s_pre[e] = first tile of expert e (e = 0..E), s_pre[E+1] = total tiles.
template <int R>
__device__ void build_tile_prefix(int T, int E, int K, int has_shared, const int32_t* __restrict__ offsets,
                                  int* s_pre, int32_t* err) {
    __shared__ int warp_tot[32];
    int tiles = 0;
    const int e = threadIdx.x;
    if (e < E) {
        int lo = offsets[e], hi = offsets[e + 1];
        if (lo < 0 || hi < lo || hi > T * K) {
            set_error(err, MOE_ERR_BOUNDS);
            hi = lo = 0;
        }
        tiles = (hi - lo + R - 1) / R;
    }
    // block inclusive scan (blockDim.x >= E, multiple of 32)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = tiles;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    if (e < E) s_pre[e] = base + inc - tiles;
    if (threadIdx.x == blockDim.x - 1) {
        const int routed = base + inc;
        s_pre[E] = routed;
        s_pre[E + 1] = routed + (has_shared ? (T + R - 1) / R : 0);
    }
    __syncthreads();
}

struct RowTile {
    int e;       // matrix index (E = shared)
    int r0;      // first row (routed: permuted row; shared: token)
    int nr;      // rows in the tile
};

template <int R>
__device__ bool find_tile(int b, int T, int E, const int32_t* __restrict__ offsets, const int* s_pre, RowTile& tl) {
    if (b >= s_pre[E + 1]) return false;
    if (b >= s_pre[E]) {
        const int q = b - s_pre[E];
        tl.e = E;
        tl.r0 = q * R;
        tl.nr = min(R, T - tl.r0);
        return true;
    }
    int lo = 0, hi = E - 1;   // last e with s_pre[e] <= b
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pre[mid] <= b) lo = mid; else hi = mid - 1;
    }
    tl.e = lo;
    tl.r0 = offsets[lo] + (b - s_pre[lo]) * R;
    tl.nr = min(R, offsets[lo + 1] - tl.r0);
    return true;
}

// Token of row i of a tile, validated (-1 for padding rows).
__device__ __forceinline__ int tile_token(const RowTile& tl, int i, int T, int E, int K,
                                          const int32_t* __restrict__ row_to_pair, int32_t* err) {
    if (i >= tl.nr) return -1;
    if (tl.e == E) return tl.r0 + i;
    const int p = row_to_pair[tl.r0 + i];
    if (p < 0 || p >= T * K) {
        set_error(err, MOE_ERR_BOUNDS);
        return 0;
    }
    return p / K;
}

// h[row][j] = bf16(silu(x . Wg[j]) * (x . Wu[j])) for a tile of R rows and
// 32 j per block (8 warps x 4 j).  Lane l takes the u32 code words l, l+32,
// ... of a weight row (8 inputs each, so its x reads are conflict-free
// 16-byte shared loads).
template <int R>
__global__ void __launch_bounds__(256) k_ffn1_simt(FfnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    int* s_pre = reinterpret_cast<int*>(smem);
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + align256((a.E + 2) * sizeof(int)));
    __shared__ int s_tok[R];
    const int H = a.H, I = a.I, E = a.E, K = a.K;
    build_tile_prefix<R>(a.T, E, K, a.has_shared, a.offsets, s_pre, a.err);
    RowTile tl;
    if (!find_tile<R>(blockIdx.x, a.T, E, a.offsets, s_pre, tl)) return;
    if (threadIdx.x < R) s_tok[threadIdx.x] = tile_token(tl, threadIdx.x, a.T, E, K, a.row_to_pair, a.err);
    __syncthreads();
    // stage x rows (zero for padding)
    const int wpr = H / 8;   // uint4 per row
    for (int q = threadIdx.x; q < R * wpr; q += blockDim.x) {
        const int i = q / wpr, c = q % wpr;
        const int t = s_tok[i];
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t >= 0) v = *reinterpret_cast<const uint4*>(a.x + (size_t)t * H + 8 * c);
        *reinterpret_cast<uint4*>(xs + (size_t)i * H + 8 * c) = v;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ngroups = H / a.G;
    const uint32_t* codes = a.gu_codes + (size_t)tl.e * 2 * I * (H / 8);
    const uint32_t* sbp = reinterpret_cast<const uint32_t*>(a.gu_sb) + (size_t)tl.e * 2 * I * ngroups;
    for (int jj = 0; jj < 4; ++jj) {
        const int j = blockIdx.y * 32 + warp * 4 + jj;
        if (j >= I) break;
        float ag[R], au[R];
#pragma unroll
        for (int i = 0; i < R; ++i) ag[i] = au[i] = 0.0f;
        for (int w = lane; w < H / 8; w += 32) {
            const uint32_t cg = ldg_u32(codes + (size_t)j * (H / 8) + w);
            const uint32_t cu = ldg_u32(codes + (size_t)(I + j) * (H / 8) + w);
            const int g = (8 * w) / a.G;
            const uint32_t pg = ldg_u32(sbp + (size_t)j * ngroups + g);
            const uint32_t pu = ldg_u32(sbp + (size_t)(I + j) * ngroups + g);
            const float sg = bf16_lo(pg), bg = bf16_hi(pg), su = bf16_lo(pu), bu = bf16_hi(pu);
            float wg[8], wu[8];
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                wg[n] = __fmaf_rn(sg, float((cg >> (4 * n)) & 15u), bg);
                wu[n] = __fmaf_rn(su, float((cu >> (4 * n)) & 15u), bu);
            }
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)i * H + 8 * w);
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float x0 = bf16_lo(xw[q]), x1 = bf16_hi(xw[q]);
                    ag[i] = __fmaf_rn(wg[2 * q], x0, ag[i]);
                    ag[i] = __fmaf_rn(wg[2 * q + 1], x1, ag[i]);
                    au[i] = __fmaf_rn(wu[2 * q], x0, au[i]);
                    au[i] = __fmaf_rn(wu[2 * q + 1], x1, au[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < R; ++i) {
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                ag[i] += __shfl_xor_sync(0xFFFFFFFFu, ag[i], off);
                au[i] += __shfl_xor_sync(0xFFFFFFFFu, au[i], off);
            }
        }
#pragma unroll
        for (int i = 0; i < R; ++i) {
            if (lane == i && i < tl.nr) {
                const size_t row = (tl.e == E) ? (size_t)a.T * K + tl.r0 + i : (size_t)tl.r0 + i;
                a.h[row * I + j] = f32_to_bf16(silu(ag[i]) * au[i]);
            }
        }
    }
}

// y_row[n] = h_row . Wd[n] for a tile of R rows and 32 outputs n per block,
// then either the weighted scatter-add into y_acc or a bf16 store per row.
template <int R>
__global__ void __launch_bounds__(256) k_ffn2_simt(FfnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    int* s_pre = reinterpret_cast<int*>(smem);
    uint16_t* hs = reinterpret_cast<uint16_t*>(smem + align256((a.E + 2) * sizeof(int)));
    __shared__ int s_tok[R];
    __shared__ float s_w[R];
    const int H = a.H, I = a.I, E = a.E, K = a.K;
    build_tile_prefix<R>(a.T, E, K, a.has_shared, a.offsets, s_pre, a.err);
    RowTile tl;
    if (!find_tile<R>(blockIdx.x, a.T, E, a.offsets, s_pre, tl)) return;
    if (threadIdx.x < R) {
        const int i = threadIdx.x;
        s_tok[i] = tile_token(tl, i, a.T, E, K, a.row_to_pair, a.err);
        float w = 1.0f;
        if (tl.e != E && i < tl.nr) {
            const int p = a.row_to_pair[tl.r0 + i];
            w = (p >= 0 && p < a.T * K) ? a.topk_w[p] : 0.0f;
        }
        s_w[i] = w;
    }
    const size_t hrow0 = (tl.e == E) ? (size_t)a.T * K + tl.r0 : (size_t)tl.r0;
    const int wpr = I / 8;
    for (int q = threadIdx.x; q < R * wpr; q += blockDim.x) {
        const int i = q / wpr, c = q % wpr;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (i < tl.nr) v = *reinterpret_cast<const uint4*>(a.h + (hrow0 + i) * I + 8 * c);
        *reinterpret_cast<uint4*>(hs + (size_t)i * I + 8 * c) = v;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ngroups = I / a.G;
    const uint32_t* codes = a.d_codes + (size_t)tl.e * H * (I / 8);
    const uint32_t* sbp = reinterpret_cast<const uint32_t*>(a.d_sb) + (size_t)tl.e * H * ngroups;
    for (int nn = 0; nn < 4; ++nn) {
        const int n = blockIdx.y * 32 + warp * 4 + nn;
        if (n >= H) break;
        float acc[R];
#pragma unroll
        for (int i = 0; i < R; ++i) acc[i] = 0.0f;
        for (int w = lane; w < I / 8; w += 32) {
            const uint32_t c = ldg_u32(codes + (size_t)n * (I / 8) + w);
            const uint32_t p = ldg_u32(sbp + (size_t)n * ngroups + (8 * w) / a.G);
            const float s = bf16_lo(p), b = bf16_hi(p);
            float wd[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) wd[q] = __fmaf_rn(s, float((c >> (4 * q)) & 15u), b);
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const uint4 hv = *reinterpret_cast<const uint4*>(hs + (size_t)i * I + 8 * w);
                const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[i] = __fmaf_rn(wd[2 * q], bf16_lo(hw[q]), acc[i]);
                    acc[i] = __fmaf_rn(wd[2 * q + 1], bf16_hi(hw[q]), acc[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < R; ++i) {
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], off);
        }
#pragma unroll
        for (int i = 0; i < R; ++i) {
            if (lane == i && i < tl.nr) {
                const int t = s_tok[i];
                if (a.mode == MOE_MODE_SCATTER) {
                    atomicAdd(a.y_acc + (size_t)t * H + n, s_w[i] * acc[i]);
                } else if (tl.e == E) {
                    a.y_shared[(size_t)t * H + n] = f32_to_bf16(acc[i]);
                } else {
                    a.y_rows[(size_t)(tl.r0 + i) * H + n] = f32_to_bf16(acc[i]);
                }
            }
        }
    }
}

template <int R>
static int max_row_tiles(int T, int E, int K, int has_shared) {
    return (T * K + R - 1) / R + E + (has_shared ? (T + R - 1) / R : 0);
}

cudaError_t launch_ffn_simt(const FfnArgs& a, cudaStream_t st) {
    constexpr int R = 8;
    const int ntiles = max_row_tiles<R>(a.T, a.E, a.K, a.has_shared);
    const size_t pre = align256((a.E + 2) * sizeof(int));
    {
        dim3 grid(ntiles, (a.I + 31) / 32);
        const size_t sm = pre + (size_t)R * a.H * sizeof(uint16_t);
        static int done[64] = {0};
        if (sm > 48 * 1024) {
            cudaError_t ce = set_smem_once(k_ffn1_simt<R>, (int)sm, done);
            if (ce != cudaSuccess) return ce;
        }
        k_ffn1_simt<R><<<grid, 256, sm, st>>>(a);
    }
    {
        dim3 grid(ntiles, (a.H + 31) / 32);
        const size_t sm = pre + (size_t)R * a.I * sizeof(uint16_t);
        static int done[64] = {0};
        if (sm > 48 * 1024) {
            cudaError_t ce = set_smem_once(k_ffn2_simt<R>, (int)sm, done);
            if (ce != cudaSuccess) return ce;
        }
        k_ffn2_simt<R><<<grid, 256, sm, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace moe
