// Expert FFNs for a handful of tokens (T <= 8, decode): one kernel per call,
// bound by HBM bandwidth.
//
// Lily pages: "Perplexity's Lily brings fast local AI to Apple silicon Macs",
// section "Where the Engine Gains Speed" (decode minimises the bytes moved per
// token; weights reconstructed inside the expert GEMM one tile at a time);
// "Perplexity open-sources Lily", section "The Narrowness Is the Performance
// Argument" (decode has little reuse, so memory traffic dominates).
//
// Design (B200):
//  - Work unit = (active expert, 32-wide block of the intermediate size); at
//    T = 1 the 9 experts x 16 blocks fill 144 of the 148 SMs, one CTA each.
//    A CTA computes gate/up + SwiGLU for its 32 intermediate columns over all
//    of H, keeps those 32 h values in shared memory, and multiplies them by
//    the matching 32 columns of the down matrix for every output row
//    (split-K over the intermediate size), adding w * y into y_acc.  No CTA
//    waits for another's compute; only the first addition into y_acc waits
//    until every CTA has cleared its slice of it (last point below).
//  - A producer warp moves each unit in a few large TMA boxes: gate and up
//    codes of 8 of the 32 rows per box, whole rows (16 KB: two contiguous
//    8 KB runs of HBM; 128B-swizzled so the consumers' 16-byte reads hit
//    distinct banks), and
//    the block's down codes (H rows x 16 B, one box).  The shared expert's
//    units do not depend on routing, so their loads are issued before the
//    kernel waits on the previous grid (programmatic dependent launch).
//  - Consumers (16 warps) turn 4-bit codes into bf16 weights in registers
//    (shift, one mask-or, one bf16x2 subtract and one bf16x2 fma per two
//    weights) laid out as warp-MMA A fragments; tokens are the MMA's N = 8
//    columns.  A code word yields the nibble pairs (j, j+4); x and h are kept
//    in shared memory in the same order inside every 8-element group, so the
//    dot products see matching operands.  Box t feeds row tile t (four
//    warps, one quarter of H each), so work starts with the first box to
//    land.  (scale, bias) words come straight from global memory into
//    registers at the start of a unit.
//  - y_acc is zeroed by the kernel itself: every CTA clears a slice and
//    counts itself in a monotonic counter; the producer warp waits for the
//    full count while the consumers compute, and the first accumulation
//    waits on its signal.  All CTAs are co-resident (one per SM), and every
//    wait is bounded.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxT = 8;
constexpr int kMaxActive = 257;
constexpr int kCodeSlots = 4;
constexpr int kCodePiece = 2 * 8 * 8 * 128;    // (gate, up) x 8 chunks x 8 rows x 128 B
constexpr int kJ = 32;                           // intermediate columns per unit

struct GemvLayout {
    int d_piece;   // H rows x 16 B
    int xs;        // x row stride (bytes)
    int off_code, off_d, off_x, off_red, off_h, off_dsb, off_tab, off_bar, total;
};

__host__ __device__ inline int round_up(int v, int a) { return (v + a - 1) / a * a; }

__host__ __device__ inline GemvLayout gemv_layout(int H) {
    GemvLayout L;
    L.d_piece = H * 16;
    L.xs = 2 * H + 16;
    L.off_code = 0;
    L.off_d = L.off_code + kCodeSlots * kCodePiece;
    L.off_x = round_up(L.off_d + 2 * L.d_piece, 1024);
    L.off_red = round_up(L.off_x + kMaxT * L.xs, 128);
    L.off_h = L.off_red + kConsumerWarps * 32 * 16;
    L.off_dsb = round_up(L.off_h + 2 * kMaxT * kJ * 2, 128);   // [2][H] down (scale, bias) words
    L.off_tab = L.off_dsb + 2 * H * 4;
    // act_e, act_row0, act_cnt [kMaxActive]; row -> pair [64]; pair -> weight [64]; misc [4];
    // selected expert [64] and weight [64] per pair; expert offsets [kMaxActive]
    L.off_bar = round_up(L.off_tab + (3 * kMaxActive + 64 + 64 + 4 + 64 + 64 + kMaxActive) * 4, 128);
    L.total = L.off_bar + 32 * 8;
    return L;
}

// Routing done inside the decode kernel (fused layer): inputs and the outputs
// the separate route and permute calls would have written.
struct GemvRoute {
    const uint16_t* w_router;   // [E, H] bf16
    const float* bias;          // nullable; [T, E] with row stride bias_stride (0: one row for all tokens)
    int64_t bias_stride;
    float* logits;              // [T, E] fp32 scratch
    int32_t* topk_idx;          // [T, K]
    float* topk_w;              // [T, K]
    int32_t* counts;            // [E]
    int32_t* offsets;           // [E + 1]
    int32_t* row_to_pair;       // [T K]
    int32_t* pair_to_row;       // [T K]
};

struct GemvArgs {
    FfnArgs f;
    GemvLayout L;
    unsigned long long* sync;   // monotonic arrival counter (workspace header)
    GemvRoute r;
};

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long atom_add_release_u64(unsigned long long* p, unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.add.release.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    return old;
}

// MMA row g of a gate/up tile <-> row 8t + perm8(g) of the unit's 32: rows read
// by one 8-lane phase then differ in bit 2 of (row & 7), which the 128-byte
// swizzle turns into distinct banks.
__device__ __forceinline__ int perm8(int g) { return (g >> 1) | ((g & 1) << 2); }

// Position of element i of an 8-group in the split order (0,4,1,5,2,6,3,7).
__device__ __forceinline__ int split_pos(int i) { return i < 4 ? 2 * i : 2 * (i - 4) + 1; }

// 8 consecutive bf16 (as 4 pairs) -> the split order.
__device__ __forceinline__ uint4 to_split_order(uint4 v) {
    uint4 r;
    r.x = prmt(v.x, v.z, 0x5410);
    r.y = prmt(v.x, v.z, 0x7632);
    r.z = prmt(v.y, v.w, 0x5410);
    r.w = prmt(v.y, v.w, 0x7632);
    return r;
}

// Two MMAs over one code word per row: rows g / g+8 give words va / vb, the
// (scale, bias) pairs s/b, the B fragment pairs bx (split order).
__device__ __forceinline__ void mma_word(float (&d)[4], uint32_t va, uint32_t vb, uint32_t sA, uint32_t bA,
                                         uint32_t sB, uint32_t bB, uint4 bx) {
    mma_bf16_16816(d, dequant_split(va, sA, bA), dequant_split(vb, sB, bB), dequant_split(va >> 4, sA, bA),
                   dequant_split(vb >> 4, sB, bB), bx.x, bx.y);
    mma_bf16_16816(d, dequant_split(va >> 8, sA, bA), dequant_split(vb >> 8, sB, bB),
                   dequant_split(va >> 12, sA, bA), dequant_split(vb >> 12, sB, bB), bx.z, bx.w);
}

__device__ __forceinline__ uint32_t sb_scale2(uint32_t w) { return prmt(w, w, 0x1010); }
__device__ __forceinline__ uint32_t sb_bias2(uint32_t w) { return prmt(w, w, 0x3232); }

// Adds this CTA to the monotonic counter and waits (bounded) until every CTA
// of the launch is counted: a grid-wide barrier for co-resident CTAs.  Every
// earlier launch added exactly gridDim.x, so the count starts at a multiple
// of it.  Releases this thread's (and, through the preceding CTA barrier,
// the CTA's) writes; acquires everyone's.
__device__ void grid_arrive_wait(unsigned long long* sync, int32_t* err) {
    __threadfence();
    const unsigned long long old = atom_add_release_u64(sync, 1ull);
    const unsigned long long target = old / gridDim.x * gridDim.x + gridDim.x;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u64(sync) < target) {
        if (globaltimer_ns() - t0 > 200000000ull) {
            set_error(err, MOE_ERR_TIMEOUT);
            break;
        }
        __nanosleep(32);
    }
}

// kRoute: the kernel also routes (router logits, top-k, permutation); else it
// reads the permutation written by the route and permute calls.
template <bool kRoute>
__global__ void __launch_bounds__(kThreads, 1)
    k_ffn_gemv(const __grid_constant__ CUtensorMap gu_map, const __grid_constant__ CUtensorMap d_map,
               const GemvArgs ga) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const FfnArgs& a = ga.f;
    const GemvLayout& L = ga.L;
    const int H = a.H, I = a.I, E = a.E, K = a.K, T = a.T;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NJ = I / kJ;          // units per expert
    const int NP = H / 512;         // 128-input steps per warp (a quarter of H)
    const int NCH = H / 256;        // 256-input chunks (128-byte lines) per gate/up row
    const int ngr = H / 64;         // (scale, bias) groups per gate/up row
    const int NB = I / 64;          // (scale, bias) groups per down row

    int* act_e = reinterpret_cast<int*>(smem + L.off_tab);
    int* act_row0 = act_e + kMaxActive;
    int* act_cnt = act_row0 + kMaxActive;
    int* s_r2p = act_cnt + kMaxActive;
    float* s_pw = reinterpret_cast<float*>(s_r2p + 64);
    int* s_misc = reinterpret_cast<int*>(s_pw + 64);
    int* s_sel = s_misc + 4;                                         // [T K] selected expert per pair
    float* s_selw = reinterpret_cast<float*>(s_sel + 64);            // [T K] its weight
    int* s_off = reinterpret_cast<int*>(s_selw + 64);                // [E + 1] expert offsets
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.off_bar);
    uint64_t* code_full = bars;
    uint64_t* code_empty = bars + 4;
    uint64_t* d_full = bars + 8;
    uint64_t* d_empty = bars + 10;
    uint64_t* zero_done = bars + 12;   // every CTA has cleared its slice of y_acc
    uint16_t* hbuf = reinterpret_cast<uint16_t*>(smem + L.off_h);   // [2][kMaxT][kJ], split order
    float4* red = reinterpret_cast<float4*>(smem + L.off_red);
    uint8_t* xs = smem + L.off_x;                                    // [kMaxT][H], split order
    uint32_t* dsb_s = reinterpret_cast<uint32_t*>(smem + L.off_dsb);  // [2][H]

    if (warp == kConsumerWarps && lane == 0) {
        prefetch_tensormap(&gu_map);
        prefetch_tensormap(&d_map);
    }
    if (tid == 0) {
        for (int i = 0; i < kCodeSlots; ++i) {
            mbar_init(&code_full[i], 1);
            mbar_init(&code_empty[i], 4);   // the box's row tile: four warps
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&d_full[i], 1);
            mbar_init(&d_empty[i], kConsumerWarps);
        }
        mbar_init(zero_done, 1);
        fence_mbar_init();
    }
    __syncthreads();

    // Loads of unit k of this CTA (expert e, column block jb); producer lane 0.
    auto issue_unit = [&](int k, int e, int jb) {
        for (int p = 0; p < 4; ++p) {
            const int n = k * 4 + p, cs = n % kCodeSlots;
            if (n >= kCodeSlots) mbar_wait_bounded(&code_empty[cs], ((n / kCodeSlots) - 1) & 1, a.err);
            mbar_arrive_expect_tx(&code_full[cs], 2 * 8 * (H / 2));   // 8 gate + 8 up rows of H/2 bytes
            tma_load_5d(smem + L.off_code + cs * kCodePiece, &gu_map, 0, kJ * jb + 8 * p, 0, 0, e, &code_full[cs]);
        }
        const int ds = k & 1;
        if (k >= 2) mbar_wait_bounded(&d_empty[ds], ((k >> 1) - 1) & 1, a.err);
        mbar_arrive_expect_tx(&d_full[ds], L.d_piece);
        tma_load_4d(smem + L.off_d + ds * L.d_piece, &d_map, 0, 0, e * (H / 256), jb, &d_full[ds]);
    };
    // the shared expert's units come first in the unit order (active index 0)
    const bool early = a.has_shared && (int)blockIdx.x < NJ;
    if (warp == kConsumerWarps && lane == 0 && early) issue_unit(0, E, blockIdx.x);
    // router rows of this CTA (warp w: expert b + w gridDim.x; warps 0 and 1 on 148 SMs),
    // lane l holding chunks l, l+32, ... of the row
    constexpr int kRChunks = 8;   // H <= 2048
    uint4 wv[kRChunks];
    const int r_e = (int)blockIdx.x + warp * (int)gridDim.x;
    const bool r_on = kRoute && warp < kConsumerWarps && r_e < E;
    if (kRoute) {
#pragma unroll
        for (int i = 0; i < kRChunks; ++i) {
            const int c = lane + 32 * i;
            wv[i] = r_on && c < H / 8 ? ldg_v4(ga.r.w_router + (size_t)r_e * H + 8 * c) : make_uint4(0, 0, 0, 0);
        }
    }

    // The next grid may start its prologue; everything below reads what
    // earlier grids on the stream wrote.
    griddep_launch_dependents();
    griddep_wait();

    if (kRoute) {
        if (warp < kConsumerWarps) {
            // ---- x (split order), this CTA's slice of y_acc
            for (int q = tid; q < T * (H / 8); q += kConsumerWarps * 32) {
                const int n = q / (H / 8), c8 = q % (H / 8);
                const uint4 v = *reinterpret_cast<const uint4*>(a.x + (size_t)n * H + 8 * c8);
                *reinterpret_cast<uint4*>(xs + (size_t)n * L.xs + 16 * c8) = to_split_order(v);
            }
            const size_t n4 = (size_t)T * H / 4, per = (n4 + gridDim.x - 1) / gridDim.x;
            const size_t lo = blockIdx.x * per, hi = min(n4, lo + per);
            for (size_t q = lo + tid; q < hi; q += kConsumerWarps * 32)
                reinterpret_cast<float4*>(a.y_acc)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            named_barrier(1, kConsumerWarps * 32);
            // ---- router logits of this CTA's experts: lane l accumulates its chunks in
            // order with fma, the 32 partials meet in the xor butterfly 16..1, then
            // the bias is added
            if (r_on) {
                float acc[kMaxT];
#pragma unroll
                for (int t = 0; t < kMaxT; ++t) acc[t] = 0.0f;
#pragma unroll
                for (int i = 0; i < kRChunks; ++i) {
                    const int c = lane + 32 * i;
                    if (c < H / 8) {
                        const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
                        for (int t = 0; t < kMaxT; ++t) {
                            if (t < T) {
                                // x chunk in split order: (x0,x4) (x1,x5) (x2,x6) (x3,x7)
                                const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)t * L.xs + 16 * c);
                                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                                float sacc = acc[t];
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const float xj = j < 4 ? bf16_lo(xw[j]) : bf16_hi(xw[j - 4]);
                                    const float wj = (j & 1) ? bf16_hi(ww[j >> 1]) : bf16_lo(ww[j >> 1]);
                                    sacc = __fmaf_rn(xj, wj, sacc);
                                }
                                acc[t] = sacc;
                            }
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < kMaxT; ++t) {
                    if (t < T) {   // T is the same for the whole warp
                        float v = acc[t];
#pragma unroll
                        for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
                        if (lane == t) {
                            if (ga.r.bias) v = __fadd_rn(v, ga.r.bias[(int64_t)t * ga.r.bias_stride + r_e]);
                            ga.r.logits[(size_t)t * E + r_e] = v;
                        }
                    }
                }
            }
            named_barrier(1, kConsumerWarps * 32);
            // ---- every CTA's logits and y_acc slice are written
            if (tid == 0) grid_arrive_wait(ga.sync, a.err);
            named_barrier(1, kConsumerWarps * 32);
            // ---- top-k of every token, in every CTA
            if (warp < T) {
                int e_sel;
                float w_sel;
                if (topk_select<8, 8>(warp, E, ga.r.logits, nullptr, 0, e_sel, w_sel) && lane == 0 &&
                    blockIdx.x == 0)
                    set_error(a.err, MOE_ERR_NONFINITE);
                if (lane < K) {
                    s_sel[warp * K + lane] = e_sel;
                    s_selw[warp * K + lane] = w_sel;
                }
            }
            named_barrier(6, kThreads);   // selections ready for the producer
            named_barrier(8, kThreads);   // the producer built the tables
        } else {
            named_barrier(6, kThreads);
            // ---- permutation: rows expert-major, token-ascending.  Pairs p = t K + k
            // come in token order, so a pair's rank among its expert's rows is the
            // number of earlier pairs with the same expert: lanes holding equal
            // experts find each other with match_any, 32 pairs at a time.
            constexpr int EPL = 8;
            const int np = T * K;
            const uint32_t lt = (1u << lane) - 1u;
            for (int q = lane; q < kMaxActive; q += 32) s_off[q] = 0;   // histogram first
            __syncwarp();
            int prow[2];
            for (int h = 0; h < 2; ++h) {
                const int p = 32 * h + lane;
                const int e = p < np ? s_sel[p] : E + lane;   // lanes without a pair match nobody real
                const uint32_t m = __match_any_sync(0xFFFFFFFFu, e);
                prow[h] = (p < np ? s_off[e] : 0) + __popc(m & lt);
                __syncwarp();
                if (p < np && (m & lt) == 0) s_off[e] += __popc(m);   // the group's first lane counts it
                __syncwarp();
            }
            int cnt[EPL], mine = 0, tot = 0;
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const int e = lane * EPL + q;
                cnt[q] = e < E ? s_off[e] : 0;
                tot += cnt[q];
                mine += cnt[q] > 0;
            }
            __syncwarp();
            int incl = tot, incl_act = mine;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                const int oa = __shfl_up_sync(0xFFFFFFFFu, incl_act, off);
                if (lane >= off) {
                    incl += o;
                    incl_act += oa;
                }
            }
            int run = incl - tot;
            const int first = a.has_shared ? 1 : 0;
            int slot = first + incl_act - mine;
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const int e = lane * EPL + q;
                if (e < E) {
                    s_off[e] = run;
                    if (blockIdx.x == 0) {
                        ga.r.offsets[e] = run;
                        ga.r.counts[e] = cnt[q];
                    }
                }
                if (cnt[q] > 0) {
                    act_e[slot] = e;
                    act_row0[slot] = run;
                    act_cnt[slot] = cnt[q];
                    ++slot;
                }
                run += cnt[q];
            }
            if (lane == 31) {
                if (a.has_shared) {
                    act_e[0] = E;
                    act_row0[0] = 0;
                    act_cnt[0] = T;
                }
                s_misc[0] = first + incl_act;
                if (blockIdx.x == 0) ga.r.offsets[E] = incl;
            }
            __syncwarp();
            for (int h = 0; h < 2; ++h) {
                const int p = 32 * h + lane;
                if (p < np) {
                    const int e = s_sel[p];
                    const int row = s_off[e] + prow[h];
                    s_r2p[row] = p;
                    s_pw[p] = s_selw[p];
                    if (blockIdx.x == 0) {
                        ga.r.row_to_pair[row] = p;
                        ga.r.pair_to_row[p] = row;
                        ga.r.topk_idx[p] = e;
                        ga.r.topk_w[p] = s_selw[p];
                    }
                }
            }
            __syncwarp();
            __threadfence_block();
            named_barrier_arrive(8, kThreads);
            const int A = s_misc[0];
            if (lane == 0) {
                int k = 0;
                for (int u = blockIdx.x; u < A * NJ; u += gridDim.x, ++k) {
                    if (k == 0 && early) continue;
                    issue_unit(k, act_e[u / NJ], u % NJ);
                }
            }
            __syncwarp();
        }
    } else if (warp == kConsumerWarps) {
        // ---- active experts (the shared one first, then routed ones with rows)
        constexpr int EPL = 8;   // experts per lane (E <= 256)
        int ofs[EPL + 1];
#pragma unroll
        for (int q = 0; q <= EPL; ++q) {
            const int e = lane * EPL + q;
            ofs[q] = e <= E ? __ldcg(a.offsets + e) : 0;
        }
        int cnt[EPL], lo[EPL], mine = 0;
        bool bad = false;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane * EPL + q;
            const int l0 = ofs[q], h0 = ofs[q + 1];
            const bool ok = e < E && l0 >= 0 && h0 >= l0 && h0 <= T * K && h0 - l0 <= kMaxT;
            bad |= e < E && !ok;
            cnt[q] = ok ? h0 - l0 : 0;
            lo[q] = ok ? l0 : 0;
            mine += cnt[q] > 0;
        }
        if (bad) set_error(a.err, MOE_ERR_BOUNDS);
        int incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += o;
        }
        const int first = a.has_shared ? 1 : 0;
        int slot = first + incl - mine;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            if (cnt[q] > 0) {
                act_e[slot] = lane * EPL + q;
                act_row0[slot] = lo[q];
                act_cnt[slot] = cnt[q];
                ++slot;
            }
        }
        if (lane == 31) {
            if (a.has_shared) {
                act_e[0] = E;
                act_row0[0] = 0;
                act_cnt[0] = T;
            }
            s_misc[0] = first + incl;
        }
        __syncwarp();
        __threadfence_block();
        named_barrier_arrive(6, kThreads);
        // ---- producer: every unit of this CTA, in order.  Units 0 and 1 never
        // wait for a down phase (their down slots are fresh), so they go first;
        // the rest may, and a down phase waits for the y_acc count below.
        const int A = s_misc[0];
        auto issue_from = [&](int k0, int k1) {
            if (lane != 0) return;
            int k = k0;
            for (int u = blockIdx.x + k0 * gridDim.x; u < A * NJ && k < k1; u += gridDim.x, ++k) {
                if (k == 0 && early) continue;
                issue_unit(k, act_e[u / NJ], u % NJ);
            }
        };
        issue_from(0, 2);
        // ---- y_acc: once the consumers cleared this CTA's slice, count the CTA
        // and wait until every CTA of the launch is counted
        named_barrier(7, kThreads);
        if (lane == 0) {
            // every earlier launch added exactly gridDim.x, so the count starts at
            // a multiple of it
            __threadfence();
            const unsigned long long old = atom_add_release_u64(ga.sync, 1ull);
            const unsigned long long target = old / gridDim.x * gridDim.x + gridDim.x;
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_u64(ga.sync) < target) {
                if (globaltimer_ns() - t0 > 200000000ull) {
                    set_error(a.err, MOE_ERR_TIMEOUT);
                    break;
                }
                __nanosleep(64);
            }
            mbar_arrive(zero_done);
        }
        issue_from(2, 1 << 30);
        __syncwarp();
    } else {
        // ---- routing tables, x (split order), this CTA's slice of y_acc
        if (tid < T * K) {
            s_r2p[tid] = __ldcg(a.row_to_pair + tid);
            s_pw[tid] = __ldcg(a.topk_w + tid);
        }
        for (int q = tid; q < T * (H / 8); q += kConsumerWarps * 32) {
            const int n = q / (H / 8), c8 = q % (H / 8);
            const uint4 v = *reinterpret_cast<const uint4*>(a.x + (size_t)n * H + 8 * c8);
            *reinterpret_cast<uint4*>(xs + (size_t)n * L.xs + 16 * c8) = to_split_order(v);
        }
        {
            const size_t n4 = (size_t)T * H / 4, per = (n4 + gridDim.x - 1) / gridDim.x;
            const size_t lo = blockIdx.x * per, hi = min(n4, lo + per);
            for (size_t q = lo + tid; q < hi; q += kConsumerWarps * 32)
                reinterpret_cast<float4*>(a.y_acc)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        named_barrier_arrive(7, kThreads);   // the slice is written
        named_barrier(6, kThreads);          // the active list (producer); x and the tables (consumers)
    }

    if (warp < kConsumerWarps) {
        const int A = s_misc[0];
        const int g = lane >> 2, c = lane & 3;
        const int t = warp & 3, kq = warp >> 2;        // gate/up: row tile, step within each box
        const int jr = 8 * t + perm8(g);               // gate/up row (of the unit's 32) of MMA rows g, g+8
        const int TW = H / 256;                        // 16-row down tiles per warp
        const int nbase = 16 * TW * warp;              // first down row of this warp
        bool zero_seen = kRoute;   // the routing barrier already covered the zeroing
        int k = 0;
        for (int u = blockIdx.x; u < A * NJ; u += gridDim.x, ++k) {
            const int ai = u / NJ, jb = u % NJ;
            const int e = act_e[ai], cnt = act_cnt[ai], row0 = act_row0[ai];
            auto column = [&](int col, float& w) -> int {   // token and weight of the expert's row col
                w = 0.0f;
                if (col >= cnt) return 0;
                if (e == E) {
                    w = 1.0f;
                    return col;
                }
                const int p = s_r2p[row0 + col];
                if (p < 0 || p >= T * K) {
                    set_error(a.err, MOE_ERR_BOUNDS);
                    return 0;
                }
                w = s_pw[p];
                return p / K;
            };
            float wg;
            const int tok_g = column(g, wg);

            // (scale, bias) words: gate/up rows of this lane for its steps, down rows of its tiles
            const uint32_t* gsb = reinterpret_cast<const uint32_t*>(a.gu_sb);
            const size_t grow = (size_t)e * 2 * I + kJ * jb + jr;   // gate row; up row = + I
            uint32_t sbg[4], sbu[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (i < NP) {
                    const int grp = 2 * (kq * NP + i) + (c >> 1);
                    sbg[i] = ldg_u32(gsb + grow * ngr + grp);
                    sbu[i] = ldg_u32(gsb + (grow + I) * ngr + grp);
                }
            }
            // the down rows' (scale, bias) words of this block's group, into shared memory
            uint32_t* dsb = dsb_s + (k & 1) * H;
            {
                const uint32_t* dsbp = reinterpret_cast<const uint32_t*>(a.d_sb) + (size_t)e * H * NB + (jb >> 1);
                for (int n = tid; n < H; n += kConsumerWarps * 32) cp_async4(smem_u32(dsb + n), dsbp + (size_t)n * NB);
                cp_async_commit();
            }

            // ---- gate/up: MMA rows g (gate) and g+8 (up) of tile t; steps kq NP .. kq NP + NP-1
            float part[4][4];
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int q = 0; q < 4; ++q) part[w][q] = 0.0f;
            const uint8_t* xrow = xs + (size_t)tok_g * L.xs;
            const int rr = perm8(g);                   // row within the box
            {
                const int n = k * 4 + t, cs = n % kCodeSlots;
                mbar_wait_bounded(&code_full[cs], (n / kCodeSlots) & 1, a.err);
                const uint8_t* pb = smem + L.off_code + cs * kCodePiece;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (i >= NP) break;
                    const int s = kq * NP + i;
                    const int ch = s >> 1;                 // 256-input chunk = 128-byte line of the row
                    const int phys = ((4 * (s & 1) + c) ^ rr) * 16;
                    const uint4 ca = *reinterpret_cast<const uint4*>(pb + ((0 * NCH + ch) * 8 + rr) * 128 + phys);
                    const uint4 cb = *reinterpret_cast<const uint4*>(pb + ((1 * NCH + ch) * 8 + rr) * 128 + phys);
                    const uint32_t sA = sb_scale2(sbg[i]), bA = sb_bias2(sbg[i]);
                    const uint32_t sB = sb_scale2(sbu[i]), bB = sb_bias2(sbu[i]);
                    const uint8_t* xp = xrow + 2 * (128 * s + 32 * c);
                    mma_word(part[0], ca.x, cb.x, sA, bA, sB, bB, *reinterpret_cast<const uint4*>(xp));
                    mma_word(part[1], ca.y, cb.y, sA, bA, sB, bB, *reinterpret_cast<const uint4*>(xp + 16));
                    mma_word(part[2], ca.z, cb.z, sA, bA, sB, bB, *reinterpret_cast<const uint4*>(xp + 32));
                    mma_word(part[3], ca.w, cb.w, sA, bA, sB, bB, *reinterpret_cast<const uint4*>(xp + 48));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&code_empty[cs]);
            }
            float acc[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = (part[0][q] + part[1][q]) + (part[2][q] + part[3][q]);
            red[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            named_barrier(2 + t, 128);   // the tile's four warps
            uint16_t* hb = hbuf + (size_t)(k & 1) * kMaxT * kJ;
            if (kq == 0) {
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const float4 v = red[(t + 4 * w) * 32 + lane];
                    s4[0] += v.x;
                    s4[1] += v.y;
                    s4[2] += v.z;
                    s4[3] += v.w;
                }
                // rows g (gate j) and g+8 (up j); columns 2c, 2c+1 = the expert's rows
                const int pj = (jr & ~7) | split_pos(jr & 7);
                hb[(2 * c) * kJ + pj] = 2 * c < cnt ? f32_to_bf16(silu(s4[0]) * s4[2]) : (uint16_t)0;
                hb[(2 * c + 1) * kJ + pj] = 2 * c + 1 < cnt ? f32_to_bf16(silu(s4[1]) * s4[3]) : (uint16_t)0;
            }
            cp_async_wait<0>();
            named_barrier(1, kConsumerWarps * 32);   // h and the down (scale, bias) words complete; red[] free

            // ---- down: rows nbase + 16 tt + {g, g+8}, K = the unit's 32 columns
            const int ds = k & 1;
            mbar_wait_bounded(&d_full[ds], (k >> 1) & 1, a.err);
            const uint4 hv = *reinterpret_cast<const uint4*>(hb + g * kJ + 8 * c);
            const uint8_t* dbase = smem + L.off_d + ds * L.d_piece;
            float w0, w1;
            const int tok0 = column(2 * c, w0), tok1 = column(2 * c + 1, w1);
            if (!zero_seen) {
                mbar_wait_bounded(zero_done, 0, a.err);
                zero_seen = true;
            }
            // four tiles' codes and products at a time (independent), then their reductions
            const bool lead = (g & 3) == 0;
            for (int t0 = 0; t0 < TW; t0 += 4) {
            float d[4][4];
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                if (t0 + tt < TW) {
                    const int nl = nbase + 16 * (t0 + tt) + g;
                    const uint32_t va = *reinterpret_cast<const uint32_t*>(dbase + (size_t)nl * 16 + 4 * c);
                    const uint32_t vb = *reinterpret_cast<const uint32_t*>(dbase + (size_t)(nl + 8) * 16 + 4 * c);
                    const uint32_t sa = dsb[nl], sb = dsb[nl + 8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) d[tt][q] = 0.0f;
                    mma_word(d[tt], va, vb, sb_scale2(sa), sb_bias2(sa), sb_scale2(sb), sb_bias2(sb), hv);
                }
            }
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                if (t0 + tt >= TW) break;
                const int nl = nbase + 16 * (t0 + tt) + g;
                // lanes g = 0 and 4 collect rows g..g+3 (and g+8..g+11) of their
                // column from lanes g+1..g+3 and add them with one vector reduction
                float4 q0, q2;
                q0.x = d[tt][0];
                q0.y = __shfl_down_sync(0xFFFFFFFFu, d[tt][0], 4);
                q0.z = __shfl_down_sync(0xFFFFFFFFu, d[tt][0], 8);
                q0.w = __shfl_down_sync(0xFFFFFFFFu, d[tt][0], 12);
                q2.x = d[tt][2];
                q2.y = __shfl_down_sync(0xFFFFFFFFu, d[tt][2], 4);
                q2.z = __shfl_down_sync(0xFFFFFFFFu, d[tt][2], 8);
                q2.w = __shfl_down_sync(0xFFFFFFFFu, d[tt][2], 12);
                if (lead && 2 * c < cnt) {
                    float* y0 = a.y_acc + (size_t)tok0 * H + nl;
                    red_add_v4(y0, w0 * q0.x, w0 * q0.y, w0 * q0.z, w0 * q0.w);
                    red_add_v4(y0 + 8, w0 * q2.x, w0 * q2.y, w0 * q2.z, w0 * q2.w);
                }
                if (cnt > 1) {   // odd columns hold tokens only when the expert has two or more rows
                    float4 q1, q3;
                    q1.x = d[tt][1];
                    q1.y = __shfl_down_sync(0xFFFFFFFFu, d[tt][1], 4);
                    q1.z = __shfl_down_sync(0xFFFFFFFFu, d[tt][1], 8);
                    q1.w = __shfl_down_sync(0xFFFFFFFFu, d[tt][1], 12);
                    q3.x = d[tt][3];
                    q3.y = __shfl_down_sync(0xFFFFFFFFu, d[tt][3], 4);
                    q3.z = __shfl_down_sync(0xFFFFFFFFu, d[tt][3], 8);
                    q3.w = __shfl_down_sync(0xFFFFFFFFu, d[tt][3], 12);
                    if (lead && 2 * c + 1 < cnt) {
                        float* y1 = a.y_acc + (size_t)tok1 * H + nl;
                        red_add_v4(y1, w1 * q1.x, w1 * q1.y, w1 * q1.z, w1 * q1.w);
                        red_add_v4(y1 + 8, w1 * q3.x, w1 * q3.y, w1 * q3.z, w1 * q3.w);
                    }
                }
            }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[ds]);
        }
    }
}

int num_sms_cached() {
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    return sms[dev];
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled gemv_encode_fn() {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    }
    return fn;
}

// Gate/up codes as a 5-D view (32 words of a 256-input chunk, row j of I,
// chunk, gate|up, expert); one box = 8 whole rows of gate and the same 8 of
// up (two contiguous runs of HBM), landing as [gate|up][chunk][row][128 B] so
// a 128-byte line's swizzle phase is its row.
bool make_gu_map(CUtensorMap* m, const FfnArgs& a) {
    EncodeTiled enc = gemv_encode_fn();
    if (!enc) return false;
    const uint64_t row = (uint64_t)a.H / 2;
    const cuuint64_t dims[5] = {32, (cuuint64_t)a.I, (cuuint64_t)(a.H / 256), 2, (cuuint64_t)(a.E + 1)};
    const cuuint64_t strides[4] = {row, 128, (cuuint64_t)a.I * row, (cuuint64_t)2 * a.I * row};
    const cuuint32_t box[5] = {32, 8, (cuuint32_t)(a.H / 256), 2, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 5, const_cast<uint32_t*>(a.gu_codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Down codes as a 4-D view (4 words of a 32-input block, row of a 256-row
// band, band, block); one box = the H rows of one expert and block.
bool make_d_map(CUtensorMap* m, const FfnArgs& a) {
    EncodeTiled enc = gemv_encode_fn();
    if (!enc) return false;
    const uint64_t row = (uint64_t)a.I / 2;
    const cuuint64_t dims[4] = {4, 256, (cuuint64_t)(a.E + 1) * (a.H / 256), (cuuint64_t)(a.I / kJ)};
    const cuuint64_t strides[3] = {row, 256 * row, 16};
    const cuuint32_t box[4] = {4, 256, (cuuint32_t)(a.H / 256), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint32_t*>(a.d_codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool ffn_gemv_supported(const FfnArgs& a) {
    return a.mode == MOE_MODE_SCATTER && a.T >= 1 && a.T <= kMaxT && a.K == 8 && a.G == 64 && a.E <= 256 &&
           (a.H == 512 || a.H == 1024 || a.H == 2048) && a.I % 64 == 0 && a.I >= 64 && a.I <= 8192;
}

namespace {

template <bool kRoute>
cudaError_t launch_gemv(const GemvArgs& ga, cudaStream_t st) {
    CUtensorMap gu_map, d_map;
    if (!make_gu_map(&gu_map, ga.f) || !make_d_map(&d_map, ga.f)) return cudaErrorInvalidValue;
    static int done[64] = {0};
    const int smem = ga.L.total + 1024;
    cudaError_t ce = set_smem_once(k_ffn_gemv<kRoute>, smem, done);
    if (ce != cudaSuccess) return ce;
    const int G = num_sms_cached();
    if (G <= 0) return cudaErrorInvalidDevice;
    if (kRoute && G * kConsumerWarps < ga.f.E) return cudaErrorInvalidConfiguration;
    // one CTA per SM, all resident at once (the in-kernel counts wait for
    // every CTA of the launch)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_ffn_gemv<kRoute>, gu_map, d_map, ga);
}

}  // namespace

cudaError_t launch_ffn_gemv(const FfnArgs& a, unsigned long long* sync, cudaStream_t st) {
    GemvArgs ga = {};
    ga.f = a;
    ga.L = gemv_layout(a.H);
    ga.sync = sync;
    return launch_gemv<false>(ga, st);
}

bool decode_fused_supported(const FfnArgs& a) {
    return ffn_gemv_supported(a) && a.E == 256 && a.H <= 2048;
}

cudaError_t launch_decode_fused(const FfnArgs& a, const DecodeRoute& r, unsigned long long* sync, cudaStream_t st) {
    GemvArgs ga = {};
    ga.f = a;
    ga.L = gemv_layout(a.H);
    ga.sync = sync;
    ga.r.w_router = r.w_router;
    ga.r.bias = r.bias;
    ga.r.bias_stride = r.bias_stride;
    ga.r.logits = r.logits;
    ga.r.topk_idx = r.topk_idx;
    ga.r.topk_w = r.topk_w;
    ga.r.counts = r.counts;
    ga.r.offsets = r.offsets;
    ga.r.row_to_pair = r.row_to_pair;
    ga.r.pair_to_row = r.pair_to_row;
    return launch_gemv<true>(ga, st);
}

}  // namespace moe
