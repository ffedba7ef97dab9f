// Expert FFNs for a handful of tokens (T <= 8, decode): one persistent,
// cooperative kernel per call, bound by HBM bandwidth.
//
// Lily pages: "Perplexity's Lily brings fast local AI to Apple silicon Macs",
// section "Where the Engine Gains Speed" (decode minimises the bytes moved per
// token; weights reconstructed inside the expert GEMM one tile at a time);
// "Perplexity open-sources Lily", section "The Narrowness Is the Performance
// Argument" (decode has little reuse, so memory traffic dominates).
//
// Design (B200):
//  - One CTA per SM.  Warp 16 is a producer: it streams the packed rows of
//    every active expert (codes and (scale, bias) rows, exactly the bytes of
//    the active experts, each once) into a ring of shared-memory stages with
//    1-D bulk async copies completing on mbarriers.  Warps 0..15 consume the
//    ring as four quads.
//  - Consumers turn 4-bit codes into bf16 weights in registers (byte permute,
//    mask, one bf16x2 subtract and one bf16x2 fma per two weights) laid out
//    as warp-MMA A fragments; the tokens are the MMA's N = 8 columns, so up
//    to 8 tokens cost the same as one.  The k order inside a 128-input step
//    is permuted identically on both operands (ldmatrix hands each lane one
//    code word of four consecutive 16-byte chunks), which a dot product does
//    not see.
//  - Phase 1: gate/up rows of 8 outputs (gate j0..j0+7 on MMA rows 0..7, up
//    j0..j0+7 on rows 8..15, so SwiGLU pairs sit in one thread), K split over
//    the quad's four warps and reduced in shared memory; h is stored in bf16.
//  - A bounded grid barrier (every CTA is co-resident: cooperative launch)
//    separates phase 1 from phase 2; the producer keeps prefetching phase-2
//    (down) weights across it.
//  - Phase 2: 64 down rows per stage, 16 per warp, full K; the epilogue adds
//    w * y into y_acc (scatter mode, zeroed in phase 1) or stores bf16 rows.
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxT = 8;
constexpr int kMaxActive = 257;
constexpr int kMaxStages = 8;
constexpr int kSmemBudget = 225 * 1024;

struct GemvLayout {
    int rs1, rs2;        // code-row strides in a stage (bytes), phase 1 / phase 2
    int stage_bytes;     // one ring stage
    int stages;          // ring depth
    int xs;              // padded x row stride (bytes)
    int hs;              // padded h row stride (bytes) of the phase-2 staging
    int off_ring, off_x, off_red, off_tab, off_bar, total;
};

__host__ __device__ inline int round_up(int v, int a) { return (v + a - 1) / a * a; }

__host__ __device__ inline GemvLayout gemv_layout(int H, int I) {
    GemvLayout L;
    L.rs1 = H / 2;
    L.rs2 = I / 2;
    const int p1 = 16 * L.rs1 + 16 * (H / 16);
    const int p2 = 64 * L.rs2 + 64 * (I / 16);
    L.stage_bytes = round_up(p1 > p2 ? p1 : p2, 128);
    L.xs = 2 * H + 16;
    L.hs = 2 * I + 16;
    // phase 1 reads the x tile, phase 2 reuses the same bytes for each quad's h rows
    const int x_need = kMaxT * L.xs, h_need = 4 * kMaxT * L.hs;
    const int x_bytes = round_up(x_need > h_need ? x_need : h_need, 128);
    const int red_bytes = 4 * 4 * 32 * 16;
    // act_e, act_row0, act_cnt, then per (active, i): token, weight
    const int tab_bytes = round_up(kMaxActive * 3 * 4 + kMaxActive * kMaxT * 8 + 64, 128);
    const int bar_bytes = 2 * kMaxStages * 8;
    const int fixed = x_bytes + red_bytes + tab_bytes + bar_bytes + 1024;
    int s = (kSmemBudget - fixed) / L.stage_bytes;
    L.stages = s > kMaxStages ? kMaxStages : s;
    L.off_ring = 0;
    L.off_x = L.stages * L.stage_bytes;
    L.off_red = L.off_x + x_bytes;
    L.off_tab = L.off_red + red_bytes;
    L.off_bar = L.off_tab + tab_bytes;
    L.total = L.off_bar + bar_bytes;
    return L;
}

struct GemvArgs {
    FfnArgs f;
    GemvLayout L;
    unsigned long long* sync;   // grid barrier arrival counter (monotonic)
};

// Per-CTA schedule: phase-1 tiles v = b, b+G, ... < V1, then phase-2 stages.
struct Sched {
    int b, G, V1, V2, n1, n2;
    __device__ void init(int A, int I, int H) {
        b = blockIdx.x;
        G = gridDim.x;
        V1 = A * (I / 8);
        V2 = A * (H / 64);
        n1 = b < V1 ? (V1 - b + G - 1) / G : 0;
        n2 = b < V2 ? (V2 - b + G - 1) / G : 0;
    }
    __device__ int total() const { return n1 + n2; }
    __device__ bool phase1(int l) const { return l < n1; }
    __device__ int unit(int l) const { return l < n1 ? b + l * G : b + (l - n1) * G; }
};

__device__ __forceinline__ uint32_t dup_lo(uint32_t w) { return prmt(w, w, 0x1010); }
__device__ __forceinline__ uint32_t dup_hi(uint32_t w) { return prmt(w, w, 0x3232); }

// 16 x 8 x (128 * nsteps) MMA over a stage's code rows [0, 16) (row stride
// rs bytes, 64 bytes of codes per 128-input step).  Lane (g, c) = (lane/4,
// lane%4) reads the 16-byte chunk c of rows g and g+8, i.e. inputs
// [32c, 32c+32) of the step, which lie in one (scale, bias) group.  Within a
// step, MMA k-step (w, half) takes the inputs 32c + 8w + 4half + {0..3} of
// every c: the two operands are permuted alike, which a dot product does not
// see.  B fragments come from bsrc(S, w): 8 bf16 of the lane's column g at
// inputs 128S + 32c + 8w.  (scale, bias) rows hold `ngroups` u32 each.
template <typename BLoad>
__device__ __forceinline__ void mma_rows16(float (&acc)[4], const uint8_t* codes, int rs, const uint32_t* sb,
                                           int ngroups, int step0, int nsteps, BLoad bsrc) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const uint8_t* rowA = codes + (size_t)g * rs + 16 * c;
    const uint8_t* rowB = rowA + 8 * rs;
    float part[4][4];   // one accumulator chain per code word: four independent MMA chains
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int q = 0; q < 4; ++q) part[w][q] = 0.0f;
    for (int S = step0; S < step0 + nsteps; ++S) {
        const uint4 ca = *reinterpret_cast<const uint4*>(rowA + S * 64);
        const uint4 cb = *reinterpret_cast<const uint4*>(rowB + S * 64);
        const int grp = 2 * S + (c >> 1);
        const uint32_t swA = sb[(size_t)g * ngroups + grp];
        const uint32_t swB = sb[(size_t)(g + 8) * ngroups + grp];
        const uint32_t sA = dup_lo(swA), bA = dup_hi(swA), sB = dup_lo(swB), bB = dup_hi(swB);
        const uint32_t wa[4] = {ca.x, ca.y, ca.z, ca.w};
        const uint32_t wb[4] = {cb.x, cb.y, cb.z, cb.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint4 xv = bsrc(S, w);
            const uint32_t vA = wa[w], vA4 = vA >> 4, vB = wb[w], vB4 = vB >> 4;
            mma_bf16_16816(part[w], dequant_pair<0>(vA, vA4, sA, bA), dequant_pair<0>(vB, vB4, sB, bB),
                           dequant_pair<1>(vA, vA4, sA, bA), dequant_pair<1>(vB, vB4, sB, bB), xv.x, xv.y);
            mma_bf16_16816(part[w], dequant_pair<2>(vA, vA4, sA, bA), dequant_pair<2>(vB, vB4, sB, bB),
                           dequant_pair<3>(vA, vA4, sA, bA), dequant_pair<3>(vB, vB4, sB, bB), xv.z, xv.w);
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] += (part[0][q] + part[1][q]) + (part[2][q] + part[3][q]);
}

__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Bounded grid-wide barrier over all CTAs of a cooperative launch.  The
// counter only ever grows: a launch whose CTAs read `base` at start (a
// multiple of the grid size, since every earlier launch completed) is
// released when the counter reaches base + gridDim.x.
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ void grid_barrier(unsigned long long* counter, unsigned long long target, int32_t* err) {
    __threadfence();
    atomicAdd(counter, 1ull);
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_u64(counter) < target) {
        if (globaltimer_ns() - t0 > 500000000ull) {
            set_error(err, MOE_ERR_TIMEOUT);
            break;
        }
    }
    __threadfence();
}

__global__ void __launch_bounds__(kThreads, 1) k_ffn_gemv(GemvArgs ga) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const FfnArgs& a = ga.f;
    const GemvLayout& L = ga.L;
    const int H = a.H, I = a.I, E = a.E, K = a.K, T = a.T;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    int* act_e = reinterpret_cast<int*>(smem + L.off_tab);
    int* act_row0 = act_e + kMaxActive;
    int* act_cnt = act_row0 + kMaxActive;
    int* act_tok = act_cnt + kMaxActive;                       // [kMaxActive][kMaxT]
    float* act_w = reinterpret_cast<float*>(act_tok + kMaxActive * kMaxT);
    int* s_misc = reinterpret_cast<int*>(act_w + kMaxActive * kMaxT);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.off_bar);
    uint64_t* empty = full + kMaxStages;
    uint8_t* xs = smem + L.off_x;
    float4* red = reinterpret_cast<float4*>(smem + L.off_red);

    if (tid == 0) {
        for (int st = 0; st < L.stages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 4);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // Phase-1 units: v = a * (I/8) + jt over the active experts, the shared
    // expert first (a = 0).  Unit b of this CTA is then known before any
    // routing output is read: the shared expert's tile b, if b < I/8.
    auto issue_phase1 = [&](int slot, int e, int j0) {
        // gate rows j0..j0+7 and up rows I+j0..I+j0+7 are contiguous in memory:
        // two copies of codes, two of (scale, bias)
        uint8_t* st = smem + L.off_ring + (size_t)slot * L.stage_bytes;
        const uint8_t* codes = reinterpret_cast<const uint8_t*>(a.gu_codes) + (size_t)e * 2 * I * (H / 2);
        const uint8_t* sbg = reinterpret_cast<const uint8_t*>(a.gu_sb) + (size_t)e * 2 * I * (H / 16);
        if (lane == 0) {
            mbar_arrive_expect_tx(&full[slot], 16 * (H / 2) + 16 * (H / 16));
            bulk_g2s(st, codes + (size_t)j0 * (H / 2), 8 * (H / 2), &full[slot]);
            bulk_g2s(st + 8 * (H / 2), codes + (size_t)(I + j0) * (H / 2), 8 * (H / 2), &full[slot]);
            bulk_g2s(st + 16 * (H / 2), sbg + (size_t)j0 * (H / 16), 8 * (H / 16), &full[slot]);
            bulk_g2s(st + 16 * (H / 2) + 8 * (H / 16), sbg + (size_t)(I + j0) * (H / 16), 8 * (H / 16), &full[slot]);
        }
        __syncwarp();
    };
    const bool early = a.has_shared && (int)blockIdx.x < I / 8;
    if (warp == kConsumerWarps && early) issue_phase1(0, E, blockIdx.x * 8);
    // Work that needs no routing output: the x tile (tokens on the MMA's 8
    // columns, zero beyond T), zeroing this CTA's slice of y_acc, and the
    // grid-barrier base.
    unsigned long long bar_base = 0;
    int r2p = 0;
    float pw = 0.0f;
    if (tid < T * K) {      // T <= 8: every (row -> pair) entry and routing weight, loaded up front
        r2p = a.row_to_pair[tid];
        pw = a.topk_w[tid];
    }
    if (warp < kConsumerWarps) {
        for (int q = tid; q < kMaxT * (H / 8); q += kConsumerWarps * 32) {
            const int n = q / (H / 8), c8 = q % (H / 8);
            uint4 v = make_uint4(0, 0, 0, 0);
            if (n < T) v = *reinterpret_cast<const uint4*>(a.x + (size_t)n * H + 8 * c8);
            *reinterpret_cast<uint4*>(xs + (size_t)n * L.xs + 16 * c8) = v;
        }
        if (a.mode == MOE_MODE_SCATTER) {
            const size_t n4 = (size_t)T * H / 4, per = (n4 + gridDim.x - 1) / gridDim.x;
            const size_t lo = blockIdx.x * per, hi = min(n4, lo + per);
            for (size_t q = lo + tid; q < hi; q += kConsumerWarps * 32)
                reinterpret_cast<float4*>(a.y_acc)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (tid == 0) bar_base = ld_acquire_u64(ga.sync) / gridDim.x * gridDim.x;
    }

    // ---- active experts (the shared one first, then routed ones with rows),
    // compacted by the producer warp alone so it can start issuing at once;
    // the consumers wait for the list on named barrier 6.
    __shared__ int s_r2p[kMaxT * 8];     // row -> pair (T*K <= 64 entries)
    __shared__ float s_pw[kMaxT * 8];    // pair -> routing weight
    if (warp == kConsumerWarps) {
        constexpr int EPL = 8;           // experts per lane (E <= 256)
        int cnt[EPL], lo[EPL], mine = 0;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const int e = lane * EPL + q;
            cnt[q] = 0;
            lo[q] = 0;
            if (e < E) {
                const int l0 = a.offsets[e], h0 = a.offsets[e + 1];
                if (l0 < 0 || h0 < l0 || h0 > T * K || h0 - l0 > kMaxT) {
                    set_error(a.err, MOE_ERR_BOUNDS);
                } else {
                    cnt[q] = h0 - l0;
                    lo[q] = l0;
                }
            }
            mine += cnt[q] > 0;
        }
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
                act_row0[0] = T * K;
                act_cnt[0] = T;
            }
            s_misc[0] = first + incl;
        }
        __syncwarp();
        __threadfence_block();
        named_barrier_arrive(6, kThreads);
    } else {
        if (tid < T * K) {
            s_r2p[tid] = r2p;
            s_pw[tid] = pw;
        }
        named_barrier(6, kThreads);
    }
    const int A = s_misc[0];
    if (warp < kConsumerWarps) {
        // token and weight of each active expert's rows, from shared memory only
        for (int q = tid; q < A * kMaxT; q += kConsumerWarps * 32) {
            const int ai = q / kMaxT, i = q % kMaxT;
            int tok = -1;
            float w = 0.0f;
            if (i < act_cnt[ai]) {
                if (act_e[ai] == E) {
                    tok = i;
                    w = 1.0f;
                } else {
                    const int p = s_r2p[act_row0[ai] + i];
                    if (p < 0 || p >= T * K) {
                        set_error(a.err, MOE_ERR_BOUNDS);
                        tok = 0;
                    } else {
                        tok = p / K;
                        w = s_pw[p];
                    }
                }
            }
            act_tok[q] = tok;
            act_w[q] = w;
        }
        named_barrier(1, kConsumerWarps * 32);
    }
    Sched sc;
    sc.init(A, I, H);
    const int nst = sc.total();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        for (int l = early ? 1 : 0; l < nst; ++l) {
            const int slot = l % L.stages;
            if (l >= L.stages && !mbar_wait_bounded(&empty[slot], ((l / L.stages) - 1) & 1, a.err)) break;
            const int u = sc.unit(l);
            if (sc.phase1(l)) {
                issue_phase1(slot, act_e[u / (I / 8)], (u % (I / 8)) * 8);
            } else {
                uint8_t* st = smem + L.off_ring + (size_t)slot * L.stage_bytes;
                const int ai = u / (H / 64), n0 = (u % (H / 64)) * 64, e = act_e[ai];
                const uint8_t* codes = reinterpret_cast<const uint8_t*>(a.d_codes) + (size_t)e * H * (I / 2);
                const uint8_t* sbd = reinterpret_cast<const uint8_t*>(a.d_sb) + (size_t)e * H * (I / 16);
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[slot], 64 * (I / 2) + 64 * (I / 16));
                    bulk_g2s(st, codes + (size_t)n0 * (I / 2), 64 * (I / 2), &full[slot]);
                    bulk_g2s(st + 64 * (I / 2), sbd + (size_t)n0 * (I / 16), 64 * (I / 16), &full[slot]);
                }
                __syncwarp();
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int quad = warp >> 2, wq = warp & 3;
    const int g = lane >> 2, c = lane & 3;
    bool grid_synced = false;
    for (int l = quad;; l += 4) {
        const bool done = l >= nst;
        if (!grid_synced && (done || !sc.phase1(l))) {
            // all phase-1 tiles of this CTA are finished once every quad gets here
            named_barrier(1, kConsumerWarps * 32);
            if (tid == 0) grid_barrier(ga.sync, bar_base + gridDim.x, a.err);
            named_barrier(1, kConsumerWarps * 32);
            grid_synced = true;
        }
        if (done) break;
        const int slot = l % L.stages;
        const uint8_t* st = smem + L.off_ring + (size_t)slot * L.stage_bytes;
        const int u = sc.unit(l);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (sc.phase1(l)) {
            const int ai = u / (I / 8), j0 = (u % (I / 8)) * 8;
            const int nsteps = H / 128 / 4;
            const uint8_t* xrow = xs + (size_t)g * L.xs + 64 * c;
            mbar_wait_bounded(&full[slot], (l / L.stages) & 1, a.err);
            mma_rows16(acc, st, L.rs1, reinterpret_cast<const uint32_t*>(st + 16 * L.rs1), H / 64, wq * nsteps,
                       nsteps, [&](int S, int w) {
                           return *reinterpret_cast<const uint4*>(xrow + 2 * (128 * S + 8 * w));
                       });
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            red[(quad * 4 + wq) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            named_barrier(2 + quad, 128);
            if (wq == 0) {
                float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const float4 v = red[(quad * 4 + w) * 32 + lane];
                    t[0] += v.x;
                    t[1] += v.y;
                    t[2] += v.z;
                    t[3] += v.w;
                }
                // rows g (gate j0+g) and g+8 (up j0+g); columns = tokens 2c, 2c+1
                const float h0 = silu(t[0]) * t[2];
                const float h1 = silu(t[1]) * t[3];
                const int cnt = act_cnt[ai];
                for (int i = 0; i < cnt; ++i) {
                    const int tok = act_tok[ai * kMaxT + i];
                    if (tok == 2 * c || tok == 2 * c + 1) {
                        const size_t row = (size_t)act_row0[ai] + i;
                        a.h[row * I + j0 + g] = f32_to_bf16(tok == 2 * c ? h0 : h1);
                    }
                }
            }
            named_barrier(2 + quad, 128);
        } else {
            const int ai = u / (H / 64), n0 = (u % (H / 64)) * 64 + 16 * wq;
            const int cnt = act_cnt[ai];
            // stage this expert's h rows (written by phase 1 on any CTA) for the quad
            uint8_t* hq = xs + (size_t)quad * kMaxT * L.hs;
            named_barrier(2 + quad, 128);                 // previous stage's readers are done
            for (int q = wq * 32 + lane; q < kMaxT * (I / 8); q += 128) {
                const int i = q / (I / 8), c8 = q % (I / 8);
                uint4 v = make_uint4(0, 0, 0, 0);
                if (i < cnt) v = ld_cg_v4(a.h + ((size_t)act_row0[ai] + i) * I + 8 * c8);
                *reinterpret_cast<uint4*>(hq + (size_t)i * L.hs + 16 * c8) = v;
            }
            named_barrier(2 + quad, 128);
            const uint8_t* hrow = hq + (size_t)g * L.hs + 64 * c;
            mbar_wait_bounded(&full[slot], (l / L.stages) & 1, a.err);
            mma_rows16(acc, st + (size_t)16 * wq * L.rs2, L.rs2,
                       reinterpret_cast<const uint32_t*>(st + 64 * L.rs2) + 16 * wq * (I / 64), I / 64, 0, I / 128,
                       [&](int S, int w) {
                           return *reinterpret_cast<const uint4*>(hrow + 2 * (128 * S + 8 * w));
                       });
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            // rows n0+g, n0+g+8; columns = the expert's rows 2c, 2c+1
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = 2 * c + (q & 1);
                const int n = n0 + g + (q >> 1) * 8;
                if (i < cnt) {
                    const int tok = act_tok[ai * kMaxT + i];
                    if (a.mode == MOE_MODE_SCATTER) {
                        atomicAdd(a.y_acc + (size_t)tok * H + n, act_w[ai * kMaxT + i] * acc[q]);
                    } else if (act_e[ai] == E) {
                        a.y_shared[(size_t)tok * H + n] = f32_to_bf16(acc[q]);
                    } else {
                        a.y_rows[((size_t)act_row0[ai] + i) * H + n] = f32_to_bf16(acc[q]);
                    }
                }
            }
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

}  // namespace

bool ffn_gemv_supported(const FfnArgs& a) {
    if (a.T > kMaxT || a.H > 2048 || a.H % 512 != 0 || a.I % 128 != 0 || a.E > 256 || a.K != 8) return false;
    const GemvLayout L = gemv_layout(a.H, a.I);
    return L.stages >= 4 && L.total <= kSmemBudget;
}

cudaError_t launch_ffn_gemv(const FfnArgs& a, unsigned long long* sync, cudaStream_t st) {
    GemvArgs ga;
    ga.f = a;
    ga.L = gemv_layout(a.H, a.I);
    ga.sync = sync;
    static int done[64] = {0};
    cudaError_t ce = set_smem_once(k_ffn_gemv, ga.L.total, done);
    if (ce != cudaSuccess) return ce;
    const int G = num_sms_cached();
    if (G <= 0) return cudaErrorInvalidDevice;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = ga.L.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_ffn_gemv, ga);
}

}  // namespace moe
