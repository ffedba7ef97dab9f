// Gated DeltaNet recurrent scan with the state held in registers for the
// whole call: read once from HBM, updated token by token, written once.
//
// Lily pages: "Perplexity built an inference engine for one model, one chip",
// second paragraph (30 of 40 layers run Gated DeltaNet with a recurrent state
// of fixed size); "Perplexity's Lily brings fast local AI to Apple silicon
// Macs", section "Where the Engine Gains Speed" (a register-resident Gated
// DeltaNet scan).  Per value head, with S the [dv, dk] state:
//   S = a S;  u = S k;  S += beta (v - u) k^T;  o = scale S q   (a = exp(g)).
// Rows of S never mix (row i only sees v[i]), so the rows of a head split
// across CTAs with no exchange: a CTA owns 16 rows of one (sequence, head),
// an 8-lane group one row, a lane 16 of its 128 columns (columns
// 32 m + 4 (lane & 7) + e, m, e in 0..3, so that a warp's state loads are
// whole 128-byte lines).  Dot products over a row reduce across the group's
// 8 lanes with three xor shuffles.
//
// Per chunk of kChunk tokens the CTA stages k and q (fp32), its 16 rows of v,
// the decays and the betas in shared memory; the next chunk's global loads
// are issued before the current chunk's steps and land in registers while
// they run.
#include <cuda_runtime.h>

#include "../../include/gdn_b200.h"
#include "common.cuh"
#include "kernels.h"
#include "api_range.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kD = 128;          // dk = dv
constexpr int kRows = 16;        // state rows per CTA
constexpr int kChunk = 16;       // tokens staged at a time
constexpr int kThreads = 128;
constexpr int kPieces = kChunk * (kD / 8) / kThreads;   // 16-byte pieces of k (and of q) per thread

struct GdnSmem {
    float k[2][kChunk][kD];
    float q[2][kChunk][kD];
    float v[2][kChunk][kRows];
    float a[2][kChunk];
    float beta[2][kChunk];
    float o[kChunk][kRows];
};

// Global loads of one chunk, held in registers until the chunk is staged.
struct ChunkRegs {
    uint4 kq[2 * kPieces];   // k (n < kPieces) and q: 16-byte pieces tid + 128 (n % kPieces)
    uint4 v;                 // threads 0..2 kChunk-1: token tid / 2, rows 8 (tid & 1) .. + 7
    float gb;                // threads 64..64+kChunk-1: g of token tid - 64; 96..: beta of token tid - 96
};

__device__ __forceinline__ void load_chunk(const GdnArgs& a, int b, int h, int hk, int row0, int t0, ChunkRegs& r) {
    const int tid = threadIdx.x;
#pragma unroll
    for (int n = 0; n < 2 * kPieces; ++n) {
        const int idx = tid + kThreads * (n % kPieces);   // token idx / 16, piece idx % 16
        const int t = t0 + (idx >> 4);
        const uint16_t* src = n < kPieces ? a.k : a.q;
        r.kq[n] = t < a.T ? __ldg(reinterpret_cast<const uint4*>(src + ((size_t)(b * a.T + t) * a.Hk + hk) * kD) +
                                  (idx & 15))
                          : make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid < 2 * kChunk) {
        const int t = t0 + (tid >> 1);
        r.v = t < a.T ? __ldg(reinterpret_cast<const uint4*>(a.v + ((size_t)(b * a.T + t) * a.Hv + h) * kD + row0) +
                              (tid & 1))
                      : make_uint4(0u, 0u, 0u, 0u);
    } else if (tid >= 64 && (tid & 31) < kChunk) {
        const int t = t0 + (tid & 31);
        const float* src = tid < 96 ? a.g : a.beta;
        r.gb = t < a.T ? __ldg(src + (size_t)(b * a.T + t) * a.Hv + h) : 0.0f;
    }
}

__device__ __forceinline__ void store_chunk(GdnSmem& sm, int buf, const ChunkRegs& r) {
    const int tid = threadIdx.x;
#pragma unroll
    for (int n = 0; n < 2 * kPieces; ++n) {
        const int idx = tid + kThreads * (n % kPieces);
        float* dst = (n < kPieces ? &sm.k[buf][0][0] : &sm.q[buf][0][0]) + (idx >> 4) * kD + 8 * (idx & 15);
        const uint32_t w[4] = {r.kq[n].x, r.kq[n].y, r.kq[n].z, r.kq[n].w};
        reinterpret_cast<float4*>(dst)[0] = make_float4(bf16_lo(w[0]), bf16_hi(w[0]), bf16_lo(w[1]), bf16_hi(w[1]));
        reinterpret_cast<float4*>(dst)[1] = make_float4(bf16_lo(w[2]), bf16_hi(w[2]), bf16_lo(w[3]), bf16_hi(w[3]));
    }
    if (tid < 2 * kChunk) {
        float* dst = &sm.v[buf][tid >> 1][8 * (tid & 1)];
        const uint32_t w[4] = {r.v.x, r.v.y, r.v.z, r.v.w};
        reinterpret_cast<float4*>(dst)[0] = make_float4(bf16_lo(w[0]), bf16_hi(w[0]), bf16_lo(w[1]), bf16_hi(w[1]));
        reinterpret_cast<float4*>(dst)[1] = make_float4(bf16_lo(w[2]), bf16_hi(w[2]), bf16_lo(w[3]), bf16_hi(w[3]));
    } else if (tid >= 64 && (tid & 31) < kChunk) {
        if (tid < 96) sm.a[buf][tid & 31] = expf(r.gb);
        else sm.beta[buf][tid & 31] = r.gb;
    }
}

__global__ void __launch_bounds__(kThreads, 5) k_gdn_scan(GdnArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    GdnSmem& sm = *reinterpret_cast<GdnSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int blocks_per_head = kD / kRows;
    const int row_blk = blockIdx.x % blocks_per_head;
    const int bh = blockIdx.x / blocks_per_head;
    const int h = bh % a.Hv, b = bh / a.Hv;
    const int hk = h / (a.Hv / a.Hk);
    const int row0 = row_blk * kRows;
    const int lr = 4 * warp + (lane >> 3);        // the group's row within the CTA
    const int c8 = lane & 7;

    griddep_launch_dependents();
    griddep_wait();   // the inputs and the state may come from the previous grid

    // the state: columns 32 m + 4 c8 + e of row row0 + lr
    float S[16];
    const float* s_in = a.state_in + ((size_t)(b * a.Hv + h) * kD + row0 + lr) * kD;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float4 v4 = *reinterpret_cast<const float4*>(s_in + 32 * m + 4 * c8);
        S[4 * m] = v4.x;
        S[4 * m + 1] = v4.y;
        S[4 * m + 2] = v4.z;
        S[4 * m + 3] = v4.w;
    }

    const int nchunks = (a.T + kChunk - 1) / kChunk;
    ChunkRegs regs;
    load_chunk(a, b, h, hk, row0, 0, regs);
    store_chunk(sm, 0, regs);
    __syncthreads();
    for (int c = 0; c < nchunks; ++c) {
        const int buf = c & 1;
        const int t0 = c * kChunk;
        if (c + 1 < nchunks) load_chunk(a, b, h, hk, row0, t0 + kChunk, regs);   // lands during the steps
        const int steps = min(kChunk, a.T - t0);
        // two tokens per trip: a token's output reduction overlaps the next one's update
#pragma unroll 2
        for (int s = 0; s < steps; ++s) {
            const float* kr = &sm.k[buf][s][4 * c8];
            const float* qr = &sm.q[buf][s][4 * c8];
            float kv[16];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 v4 = *reinterpret_cast<const float4*>(kr + 32 * m);
                kv[4 * m] = v4.x;
                kv[4 * m + 1] = v4.y;
                kv[4 * m + 2] = v4.z;
                kv[4 * m + 3] = v4.w;
            }
            // u = (a S) k = a (S k): four partial chains, then the group's 8 lanes
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                p0 = fmaf(S[4 * m], kv[4 * m], p0);
                p1 = fmaf(S[4 * m + 1], kv[4 * m + 1], p1);
                p2 = fmaf(S[4 * m + 2], kv[4 * m + 2], p2);
                p3 = fmaf(S[4 * m + 3], kv[4 * m + 3], p3);
            }
            float u = (p0 + p1) + (p2 + p3);
            u += __shfl_xor_sync(0xFFFFFFFFu, u, 1);
            u += __shfl_xor_sync(0xFFFFFFFFu, u, 2);
            u += __shfl_xor_sync(0xFFFFFFFFu, u, 4);
            const float dec = sm.a[buf][s];
            const float w = sm.beta[buf][s] * (sm.v[buf][s][lr] - dec * u);
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(dec, S[j], w * kv[j]);
            // o = scale S q
            float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 q4 = *reinterpret_cast<const float4*>(qr + 32 * m);
                r0 = fmaf(S[4 * m], q4.x, r0);
                r1 = fmaf(S[4 * m + 1], q4.y, r1);
                r2 = fmaf(S[4 * m + 2], q4.z, r2);
                r3 = fmaf(S[4 * m + 3], q4.w, r3);
            }
            float o = (r0 + r1) + (r2 + r3);
            o += __shfl_xor_sync(0xFFFFFFFFu, o, 1);
            o += __shfl_xor_sync(0xFFFFFFFFu, o, 2);
            o += __shfl_xor_sync(0xFFFFFFFFu, o, 4);
            if (c8 == 0) sm.o[s][lr] = a.scale * o;
        }
        __syncthreads();   // o of the chunk complete; the other buffer no longer read
        if (tid < 2 * steps) {
            const int s = tid >> 1, half = tid & 1;
            const float* src = &sm.o[s][8 * half];
            uint4 w;
            w.x = pack_bf16x2(src[0], src[1]);
            w.y = pack_bf16x2(src[2], src[3]);
            w.z = pack_bf16x2(src[4], src[5]);
            w.w = pack_bf16x2(src[6], src[7]);
            *reinterpret_cast<uint4*>(a.o + ((size_t)(b * a.T + t0 + s) * a.Hv + h) * kD + row0 + 8 * half) = w;
        }
        if (c + 1 < nchunks) store_chunk(sm, buf ^ 1, regs);
        __syncthreads();
    }

    float* s_out = a.state_out + ((size_t)(b * a.Hv + h) * kD + row0 + lr) * kD;
#pragma unroll
    for (int m = 0; m < 4; ++m)
        *reinterpret_cast<float4*>(s_out + 32 * m + 4 * c8) =
            make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
}

// A handful of tokens (T <= kChunk: decode, verification): the call is a
// stream of state rows (8 KB in, 8 KB out per 16 rows) with little
// arithmetic between, so a resident CTA walks over several (sequence, head,
// row block) items and fetches the next item's state (cp.async, 16 bytes a
// copy) and inputs while it runs the current one.
__device__ __forceinline__ void cp_async16(uint32_t dst_saddr, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst_saddr), "l"(src) : "memory");
}

struct GdnSmallSmem {
    GdnSmem base;               // k, q, v, decays, betas (two items), o
    float s[2][kRows][kD];      // the state rows of the current and the next item
};

__global__ void __launch_bounds__(kThreads, 4) k_gdn_scan_small(GdnArgs a, int nitems) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    GdnSmallSmem& ss = *reinterpret_cast<GdnSmallSmem*>(smem_raw);
    GdnSmem& sm = ss.base;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lr = 4 * warp + (lane >> 3);   // the group's row within the item
    const int c8 = lane & 7;                 // columns 32 m + 4 c8 + e
    const int blocks_per_head = kD / kRows;
    griddep_launch_dependents();
    griddep_wait();   // the inputs and the state may come from the previous grid

    struct Item {
        int b, h, hk, row0;
    };
    auto coords = [&](int item) {
        Item it;
        const int bh = item / blocks_per_head;
        it.h = bh % a.Hv;
        it.b = bh / a.Hv;
        it.hk = it.h / (a.Hv / a.Hk);
        it.row0 = (item % blocks_per_head) * kRows;
        return it;
    };
    auto fetch_state = [&](const Item& it, int sb) {
        const float* src = a.state_in + ((size_t)(it.b * a.Hv + it.h) * kD + it.row0) * kD;
        for (int p = tid; p < kRows * kD / 4; p += kThreads) cp_async16(smem_u32(&ss.s[sb][0][0] + 4 * p), src + 4 * p);
        cp_async_commit();
    };

    int item = blockIdx.x;
    if (item >= nitems) return;
    ChunkRegs regs;
    {
        const Item it = coords(item);
        fetch_state(it, 0);
        load_chunk(a, it.b, it.h, it.hk, it.row0, 0, regs);
    }
    for (int n = 0; item < nitems; ++n) {
        const int cur = n & 1;
        const Item it = coords(item);
        store_chunk(sm, cur, regs);
        const int next = item + gridDim.x;
        if (next < nitems) {
            const Item nx = coords(next);
            fetch_state(nx, cur ^ 1);
            load_chunk(a, nx.b, nx.h, nx.hk, nx.row0, 0, regs);   // lands while this item runs
            cp_async_wait<1>();   // this item's state (the older group) has landed
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();

        float S[16];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 v4 = *reinterpret_cast<const float4*>(&ss.s[cur][lr][32 * m + 4 * c8]);
            S[4 * m] = v4.x;
            S[4 * m + 1] = v4.y;
            S[4 * m + 2] = v4.z;
            S[4 * m + 3] = v4.w;
        }
        for (int st = 0; st < a.T; ++st) {
            const float* kr = &sm.k[cur][st][4 * c8];
            const float* qr = &sm.q[cur][st][4 * c8];
            float kv[16];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 v4 = *reinterpret_cast<const float4*>(kr + 32 * m);
                kv[4 * m] = v4.x;
                kv[4 * m + 1] = v4.y;
                kv[4 * m + 2] = v4.z;
                kv[4 * m + 3] = v4.w;
            }
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                p0 = fmaf(S[4 * m], kv[4 * m], p0);
                p1 = fmaf(S[4 * m + 1], kv[4 * m + 1], p1);
                p2 = fmaf(S[4 * m + 2], kv[4 * m + 2], p2);
                p3 = fmaf(S[4 * m + 3], kv[4 * m + 3], p3);
            }
            float u = (p0 + p1) + (p2 + p3);
            u += __shfl_xor_sync(0xFFFFFFFFu, u, 1);
            u += __shfl_xor_sync(0xFFFFFFFFu, u, 2);
            u += __shfl_xor_sync(0xFFFFFFFFu, u, 4);
            const float dec = sm.a[cur][st];
            const float w = sm.beta[cur][st] * (sm.v[cur][st][lr] - dec * u);
#pragma unroll
            for (int j = 0; j < 16; ++j) S[j] = fmaf(dec, S[j], w * kv[j]);
            float r0 = 0.f, r1 = 0.f, r2 = 0.f, r3 = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 q4 = *reinterpret_cast<const float4*>(qr + 32 * m);
                r0 = fmaf(S[4 * m], q4.x, r0);
                r1 = fmaf(S[4 * m + 1], q4.y, r1);
                r2 = fmaf(S[4 * m + 2], q4.z, r2);
                r3 = fmaf(S[4 * m + 3], q4.w, r3);
            }
            float o = (r0 + r1) + (r2 + r3);
            o += __shfl_xor_sync(0xFFFFFFFFu, o, 1);
            o += __shfl_xor_sync(0xFFFFFFFFu, o, 2);
            o += __shfl_xor_sync(0xFFFFFFFFu, o, 4);
            if (c8 == 0) sm.o[st][lr] = a.scale * o;
        }
        float* s_out = a.state_out + ((size_t)(it.b * a.Hv + it.h) * kD + it.row0 + lr) * kD;
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4*>(s_out + 32 * m + 4 * c8) =
                make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
        __syncthreads();   // o of the item complete
        if (tid < 2 * a.T) {
            const int st = tid >> 1, half = tid & 1;
            const float* src = &sm.o[st][8 * half];
            uint4 w4;
            w4.x = pack_bf16x2(src[0], src[1]);
            w4.y = pack_bf16x2(src[2], src[3]);
            w4.z = pack_bf16x2(src[4], src[5]);
            w4.w = pack_bf16x2(src[6], src[7]);
            *reinterpret_cast<uint4*>(a.o + ((size_t)(it.b * a.T + st) * a.Hv + it.h) * kD + it.row0 + 8 * half) = w4;
        }
        __syncthreads();   // this item's buffers are free for the item after next
        item = next;
    }
}

}  // namespace

bool gdn_scan_supported(const GdnArgs& a) {
    return a.B >= 1 && a.T >= 1 && a.Hk >= 1 && a.Hv >= 1 && a.Hv % a.Hk == 0 && a.dk == kD && a.dv == kD &&
           (int64_t)a.B * a.Hv * (kD / kRows) <= 0x7FFFFFFF;
}

cudaError_t launch_gdn_scan(const GdnArgs& a, cudaStream_t st) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess)
        return cudaErrorInvalidDevice;
    const int nitems = a.B * a.Hv * (kD / kRows);
    // the item-walking kernel pays off once every resident CTA gets two items or more
    if (a.T <= kChunk && nitems >= 8 * sms) {
        static int done_s[64] = {0};
        const int smem_s = (int)sizeof(GdnSmallSmem);
        cudaError_t ce = set_smem_once(k_gdn_scan_small, smem_s, done_s);
        if (ce != cudaSuccess) return ce;
        return launch_pdl(k_gdn_scan_small, dim3(4 * sms), dim3(kThreads), (size_t)smem_s, st, a, nitems);
    }
    static int done[64] = {0};
    const int smem = (int)sizeof(GdnSmem);
    cudaError_t ce = set_smem_once(k_gdn_scan, smem, done);
    if (ce != cudaSuccess) return ce;
    const int grid = a.B * a.Hv * (kD / kRows);
    return launch_pdl(k_gdn_scan, dim3(grid), dim3(kThreads), (size_t)smem, st, a);
}

}  // namespace moe

// ------------------------------------------------------------------ C ABI

namespace {
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
}  // namespace

extern "C" int32_t gdn_scan(int32_t B, int32_t T, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, const uint16_t* q,
                            const uint16_t* k, const uint16_t* v, const float* g, const float* beta, float scale,
                            const float* state_in, float* state_out, uint16_t* o, void* stream) {
    moe::ApiRange api_range("gdn_scan");
    if (B < 1 || T < 1 || Hk < 1 || Hv < 1) return MOE_ERR_INVALID_ARG;
    if (!q || !k || !v || !g || !beta || !state_in || !state_out || !o) return MOE_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state_in) || !aligned16(state_out) ||
        !aligned16(o) || !aligned4(g) || !aligned4(beta))
        return MOE_ERR_INVALID_ARG;
    moe::GdnArgs a;
    a.B = B;
    a.T = T;
    a.Hk = Hk;
    a.Hv = Hv;
    a.dk = dk;
    a.dv = dv;
    a.q = q;
    a.k = k;
    a.v = v;
    a.g = g;
    a.beta = beta;
    a.scale = scale;
    a.state_in = state_in;
    a.state_out = state_out;
    a.o = o;
    if (!moe::gdn_scan_supported(a)) return MOE_ERR_UNSUPPORTED;
    return moe::launch_gdn_scan(a, (cudaStream_t)stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
