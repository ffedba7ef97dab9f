// Expert FFNs for a handful of tokens (T <= 8, decode), and the decode layer's
// router, top-k, permutation and expert FFNs in one launch.  Bound by HBM
// bandwidth and latency.
//
// Lily pages: "Perplexity's Lily brings fast local AI to Apple silicon Macs",
// section "Where the Engine Gains Speed" (decode minimises the bytes moved per
// token; weights reconstructed inside the expert GEMM one tile at a time);
// "Perplexity built an inference engine for one model, one chip", third
// paragraph (routing stays on the GPU); "Perplexity open-sources Lily",
// section "The Narrowness Is the Performance Argument" (decode has little
// reuse, so memory traffic dominates).
//
// Design (B200, one CTA per SM, all CTAs co-resident by a cooperative launch):
//  - Work unit = (active expert, 32-wide block of the intermediate size): its
//    32 gate rows + 32 up rows over all of H, streamed as four TMA boxes
//    (8 gate + the matching 8 up rows, whole rows, 128B-swizzled) with their
//    (scale, bias) rows, then the block's 32 columns of the down matrix for
//    all H rows (split-K over the intermediate size): w * (h . Wd) is added
//    into y_acc with vector reductions.  At T = 1 the 9 experts x 16 blocks are
//    one unit on each of 144 SMs.  Every unit computes all T tokens (the
//    MMA's N = 8 columns); a token's routing weight is zero where it did not
//    pick the expert.  Each warp stages its 16-row down tiles in shared memory
//    so that one vector reduction adds 4 consecutive rows of one token.
//  - Three modes: the T <= 8 tokens of a launch (expert FFN call), the same
//    with routing fused in (decode layer), and a row list (any T): units of
//    the experts that hold 1..8 rows, whose MMA columns are those rows, x rows
//    brought per unit from the gathered rows, the tensor-core kernel taking
//    every other expert.
//  - Group-factored dequantisation: w = s q + b over a group of inputs is
//    s (128 + q) + (b - 128 s), so the MMAs run on the exact bf16 values
//    128 + q (one mask-and-or per two weights) and each group's fp32 partial
//    is scaled afterwards: acc += s * D + (b - 128 s) * sum(activations over
//    the group).  The weights are used exactly (not rounded to bf16).
//  - A counter in the workspace header numbers the launches: every CTA reads
//    it at its start and adds one once it has cleared its slice of y_acc, so
//    each launch adds exactly its grid size.  The first reduction into y_acc
//    waits until the count is complete; the fused layer tags its router
//    logits with the launch number, and every CTA polls the logits until
//    each tag is current (no grid barrier).
//  - The shared expert does not depend on routing: its loads (and the router
//    rows) are issued before the kernel waits on the previous grid
//    (programmatic dependent launch); in the fused layer its unit is computed
//    while the other CTAs' logits are in flight.
// Every wait is bounded (MOE_ERR_TIMEOUT, never a hang).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kWarps = 16;                      // compute warps
constexpr int kThreads = (kWarps + 1) * 32;     // + one producer warp
constexpr int kMaxT = 8;
// Copies of the tagged router logits: every CTA polls all of a token's logits,
// and 148 CTAs reading one 2 KB block at once queue on the L2 slices that hold
// it; CTA b reads copy b mod kLogitCopies.
constexpr int kLogitCopies = 8;
constexpr int kJ = 32;                          // intermediate columns per unit
constexpr int kMaxGuSlots = 6;                  // gate/up box ring (fewer when x needs the room)
constexpr int kDnSlots = 2;                     // down ring: one unit's down columns each
constexpr int kMaxSlots = 1 + 8 * kMaxT;        // active experts: shared + 8 per token
constexpr int kSmemLimit = 232448;              // dynamic shared memory per block (227 KB)
constexpr int kRouterRows = 2;                  // router rows per CTA (experts b and b + grid size)
constexpr int kExtraBars = 9;                   // mbarriers besides the two rings
constexpr int kMaxRows = 8;                     // row-list launches: experts of at most this many rows
// k_decode modes: the T <= 8 tokens of a launch (four-call path), the same
// with the routing fused in, or the rows of the experts that hold few of them
// (the tensor-core path's small experts)
constexpr int kModeTokens = 0, kModeRoute = 1, kModeRows = 2;

struct DecLayout {
    int gu_box;     // gate/up codes box: 16 rows x H/2 bytes
    int gu_sbb;     // gate/up (scale, bias) box slot: 16 rows x H/16 bytes, 1 KB aligned
    int gu_slots;   // gate/up ring depth
    int dn_box;     // one unit's down codes: H rows x 16 bytes
    int sb_tma;     // 1: the down (scale, bias) words arrive as one TMA box of H rows x 16 bytes (I >= 256)
    int dsb_bytes;  // their landing area: H x 16 bytes by TMA, else H words by cp.async
    int xs;         // x row stride (bytes)
    int off_gu, off_gusb, off_dn, off_dsb, off_x, off_sx, off_red, off_hs, off_rt, off_tab, off_bar, total;
};

// Routing state of the CTA (shared memory).
struct DecTab {
    int slot_e[256 + 8];                // expert of each active slot (slot 0 = shared when present)
    float wsel[kMaxSlots + 7][kMaxT];   // routing weight of (slot, token); 0 = not routed there
    int slot_of[256];                   // active slot of each expert
    int off[260];                       // expert offsets (routing outputs; the row list of a row-list launch)
    int sel[8 * kMaxT];                 // selected expert per pair (fused layer)
    float selw[8 * kMaxT];              // its weight
    float hsum[2][4][kMaxT];            // per unit parity and box: sums of the rounded h per token
    uint32_t bitmap[8];                 // selected experts
    int wtot[16];
    int A;                              // active slots
    uint32_t epoch;                     // launch number (+1): the logits' tag
    unsigned long long zero_target;     // counter value at which every CTA has cleared its slice of y_acc
};

__host__ __device__ inline int round_up(int v, int a) { return (v + a - 1) / a * a; }

// Row-list launch: units a CTA can hold the column tables of (token, weight per
// column: 8 bytes x kMaxRows), in the router-row area the other modes use.
__host__ __device__ constexpr int row_units_cap(int H) { return kRouterRows * 2 * H / (8 * kMaxRows); }

DecLayout dec_layout(int H, int I, int T) {
    DecLayout L;
    L.gu_box = 8 * H;
    L.gu_sbb = round_up(H, 1024);
    L.dn_box = 16 * H;
    L.sb_tma = I >= 256 ? 1 : 0;
    L.dsb_bytes = L.sb_tma ? 16 * H : 4 * H;
    L.xs = 2 * H + 16;
    const int fixed = kDnSlots * L.dn_box + L.dsb_bytes + round_up(T * L.xs, 128) + (H / 64) * kMaxT * 4 +
                      kWarps * 32 * 16 + 2 * kMaxT * 32 * 2 + kRouterRows * 2 * H + round_up((int)sizeof(DecTab), 128) +
                      (2 * kMaxGuSlots + 2 * kDnSlots + kExtraBars) * 8 + 6 * 128;
    L.gu_slots = (kSmemLimit - 1024 - fixed) / (L.gu_box + L.gu_sbb);
    if (L.gu_slots > kMaxGuSlots) L.gu_slots = kMaxGuSlots;
    L.off_gu = 0;
    L.off_gusb = L.off_gu + L.gu_slots * L.gu_box;
    L.off_dn = L.off_gusb + L.gu_slots * L.gu_sbb;
    L.off_dsb = L.off_dn + kDnSlots * L.dn_box;
    L.off_x = round_up(L.off_dsb + L.dsb_bytes, 128);
    L.off_sx = round_up(L.off_x + T * L.xs, 128);
    L.off_red = round_up(L.off_sx + (H / 64) * kMaxT * 4, 128);
    L.off_hs = round_up(L.off_red + kWarps * 32 * 16, 128);
    L.off_rt = round_up(L.off_hs + 2 * kMaxT * kJ * 2, 128);
    L.off_tab = round_up(L.off_rt + kRouterRows * 2 * H, 128);
    L.off_bar = round_up(L.off_tab + (int)sizeof(DecTab), 8);
    L.total = L.off_bar + (2 * kMaxGuSlots + 2 * kDnSlots + kExtraBars) * 8;
    return L;
}

// Workspace sections the decode kernels use.
struct DecArgs {
    FfnArgs f;
    DecLayout L;
    unsigned long long* launches;   // CTAs of decode launches so far (workspace header)
    unsigned long long* tlogits;    // [kLogitCopies][kMaxT][E] tagged router logits (fused layer)
    DecodeRoute r;                  // fused layer: router inputs and routing outputs
    int lgI;                        // log2 of the intermediate size
};

// MMA row g <-> box row perm8(g): the rows one half-warp reads then differ in
// bit 1..2 of (row & 7), which the swizzle turns into distinct banks.
__device__ __forceinline__ int perm8(int g) { return 2 * (g & 3) + (g >> 2); }

// bf16x2 (128 + q_j, 128 + q_{j+4}) of nibbles j, j+4 of a code word: exact.
__device__ __forceinline__ uint32_t nib(uint32_t w, int j) { return nibble_pair_split(w >> (4 * j)); }

// 8 consecutive bf16 (4 pairs) -> the split order (0,4)(1,5)(2,6)(3,7).
__device__ __forceinline__ uint4 to_split_order(uint4 v) {
    uint4 r;
    r.x = prmt(v.x, v.z, 0x5410);
    r.y = prmt(v.x, v.z, 0x7632);
    r.z = prmt(v.y, v.w, 0x5410);
    r.w = prmt(v.y, v.w, 0x7632);
    return r;
}

// D = (128 + q) . act over one 64-input group for MMA rows g / g+8 (code words
// ca / cb: two consecutive words each) and token column g (activation pairs
// b0 for the first word, b1 for the second, split order).
__device__ __forceinline__ void group_mma(float (&d)[4], uint2 ca, uint2 cb, uint4 b0, uint4 b1) {
    d[0] = d[1] = d[2] = d[3] = 0.0f;
    mma_bf16_16816(d, nib(ca.x, 0), nib(cb.x, 0), nib(ca.x, 1), nib(cb.x, 1), b0.x, b0.y);
    mma_bf16_16816(d, nib(ca.x, 2), nib(cb.x, 2), nib(ca.x, 3), nib(cb.x, 3), b0.z, b0.w);
    mma_bf16_16816(d, nib(ca.y, 0), nib(cb.y, 0), nib(ca.y, 1), nib(cb.y, 1), b1.x, b1.y);
    mma_bf16_16816(d, nib(ca.y, 2), nib(cb.y, 2), nib(ca.y, 3), nib(cb.y, 3), b1.z, b1.w);
}

// (scale, bias) word -> s and b - 128 s.
__device__ __forceinline__ void sb_factor(uint32_t w, float& s, float& bp) {
    s = __uint_as_float(w << 16);
    bp = fmaf(-128.0f, s, __uint_as_float(w & 0xFFFF0000u));
}

// Down-phase staging of a warp's 16-row tile, [token][row] floats in 16-float
// slots: token t in slot (t odd) * 4 + t / 2, row quads of tokens 4..7 swapped
// in pairs.  The four stores of a lane (rows g, g + 8; tokens 2c, 2c + 1) and
// the 8-lane phases of the float4 reads each touch 32 distinct banks.
__device__ __forceinline__ int stage_word(int t, int r) {
    return 16 * ((t & 1) * 4 + (t >> 1)) + 4 * ((r >> 2) ^ (((t >> 2) & 1) << 1)) + (r & 3);
}

__device__ __forceinline__ uint2 lds64(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

__device__ __forceinline__ unsigned long long tag_word(uint32_t epoch, float v) {
    return ((unsigned long long)__float_as_uint(v) << 32) | epoch;
}

template <int kH, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    k_decode(const __grid_constant__ CUtensorMap gu_map, const __grid_constant__ CUtensorMap gsb_map,
             const __grid_constant__ CUtensorMap dn_map, const __grid_constant__ CUtensorMap dsb_map,
             const DecArgs da) {
    constexpr int kNG = kH / 64;                 // (scale, bias) groups per gate/up row
    constexpr int kNGW = kNG / 4;                // groups per K-quarter warp
    constexpr int kNCH = kH / 256;               // 128-byte lines per gate/up code row
    constexpr int kRB = kH / 16;                 // bytes of one gate/up (scale, bias) row
    constexpr uint32_t kSmask = kRB / 16 - 1;    // its swizzle span, in 16-byte units - 1
    constexpr int kXS = 2 * kH + 16;             // x row stride in shared memory (bytes)
    constexpr int kRChunks = kH / 256;           // router chunks per lane
    constexpr int kTW = kH / 256;                // 16-row down tiles per warp
    constexpr bool kRoute = kMode == kModeRoute;
    constexpr bool kRows = kMode == kModeRows;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const FfnArgs& a = da.f;
    const DecLayout& L = da.L;
    const int I = a.I, E = a.E, T = a.T;
    const int lgI = da.lgI;                      // I is a power of two
    const int G = gridDim.x, b = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int rg = perm8(g);
    const int NJ = I >> 5;                       // units per expert
    const bool sh = !kRows && a.has_shared != 0;   // a row-list launch leaves the shared expert to its caller
    const bool early_unit = sh && b < NJ;        // the first unit is the shared expert's block b
    const int gus = L.gu_slots;

    DecTab& tab = *reinterpret_cast<DecTab*>(smem + L.off_tab);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.off_bar);
    uint64_t* gu_full = bars;
    uint64_t* gu_empty = bars + kMaxGuSlots;
    uint64_t* dn_full = bars + 2 * kMaxGuSlots;
    uint64_t* dn_empty = dn_full + kDnSlots;
    uint64_t* rt_full = dn_empty + kDnSlots;
    uint64_t* zero_done = rt_full + 1;
    uint64_t* list_ready = rt_full + 2;   // the active list is in shared memory (producer lane 0 waits)
    uint64_t* zt_ready = rt_full + 3;     // the launch number is in shared memory (the logits' tag)
    uint64_t* zeroed = rt_full + 4;       // this CTA's slice of y_acc is cleared (producer lane 0 waits)
    uint64_t* dsb_full = rt_full + 5;     // the unit's down (scale, bias) box landed (TMA form)
    uint64_t* dsb_empty = rt_full + 6;    // and was read by every compute warp
    uint64_t* x_full = rt_full + 7;       // row-list launch: the unit's x rows landed
    uint64_t* x_empty = rt_full + 8;      // and were read by every compute warp
    uint8_t* xs = smem + L.off_x;                                    // [T][kH] bf16, split order
    float* sx = reinterpret_cast<float*>(smem + L.off_sx);           // [kNG][kMaxT] group sums of x
    float4* red = reinterpret_cast<float4*>(smem + L.off_red);       // [kWarps][32]
    uint16_t* hs = reinterpret_cast<uint16_t*>(smem + L.off_hs);     // [2][kMaxT][kJ] h of a unit, split order
    uint32_t* dsb = reinterpret_cast<uint32_t*>(smem + L.off_dsb);   // [kH] down (scale, bias) words of a unit
    // row-list launch: token and routing weight of each column of this CTA's units (router-row area)
    int* utok = reinterpret_cast<int*>(smem + L.off_rt);                         // [unit][kMaxRows]
    float* uw = reinterpret_cast<float*>(smem + L.off_rt) + row_units_cap(kH) * kMaxRows;

    if (tid == 0) {
        for (int i = 0; i < gus; ++i) {
            mbar_init(&gu_full[i], 1);
            mbar_init(&gu_empty[i], 4);   // the box's four K-quarter warps
        }
        for (int i = 0; i < kDnSlots; ++i) {
            mbar_init(&dn_full[i], 1);
            mbar_init(&dn_empty[i], kWarps);
        }
        mbar_init(rt_full, 1);
        mbar_init(zero_done, 1);
        mbar_init(list_ready, 1);
        mbar_init(zt_ready, 1);
        mbar_init(zeroed, 1);
        mbar_init(dsb_full, 1);
        mbar_init(dsb_empty, kWarps);
        mbar_init(x_full, 1);
        mbar_init(x_empty, 1);
        fence_mbar_init();
    }
    if (warp == kWarps && lane == 0) {
        prefetch_tensormap(&gu_map);
        prefetch_tensormap(&gsb_map);
        prefetch_tensormap(&dn_map);
        if (L.sb_tma) prefetch_tensormap(&dsb_map);
    }
    __syncthreads();

    // ---- loads (producer lane 0)
    // gate/up boxes of a unit (expert e, column block jb), then its down columns
    int gu_n = 0, gu_cs = 0, gu_ph = 0, dn_n = 0, sb_n = 0, x_n = 0;
    // Producer lane 0: the first reductions into y_acc wait until every CTA has
    // cleared its slice.  release_zero polls the launch counter for that and
    // opens zero_done; it must run before any load waits on a down phase.
    bool released = kRows;   // a row-list launch adds into y_acc as it is
    auto release_zero = [&]() {
        const unsigned long long target = tab.zero_target;
        const uint64_t t0 = globaltimer_ns();
        while (ld_relaxed_u64(da.launches) < target) {
            if (globaltimer_ns() - t0 > 200000000ull) {
                set_error(a.err, MOE_ERR_TIMEOUT);
                break;
            }
            __nanosleep(64);
        }
        __threadfence();
        mbar_arrive(zero_done);
        released = true;
    };
    auto issue_unit = [&](int e, int jb) {
        if (kRows) {
            // the expert's gathered x rows (split order, rows off[e].. of xg) into the one x slot,
            // once the previous unit's gate/up has read it
            if (x_n >= 1) mbar_wait_bounded(x_empty, (x_n - 1) & 1, a.err);
            const int lo = tab.off[e], n = min(max(tab.slot_of[e], 0), kMaxRows);   // slot_of: rows of each expert
            mbar_arrive_expect_tx(x_full, (uint32_t)(n * 2 * kH));
            for (int r = 0; r < n; ++r)
                bulk_load(xs + (size_t)r * kXS, a.xg + (size_t)(lo + r) * kH, 2 * kH, x_full);
            ++x_n;
        }
        for (int p = 0; p < 4; ++p) {
            if (gu_n >= gus) mbar_wait_bounded(&gu_empty[gu_cs], (gu_ph - 1) & 1, a.err);
            mbar_arrive_expect_tx(&gu_full[gu_cs], L.gu_box + kH);
            tma_load_5d(smem + L.off_gu + gu_cs * L.gu_box, &gu_map, 0, kJ * jb + 8 * p, 0, 0, e, &gu_full[gu_cs]);
            tma_load_4d(smem + L.off_gusb + gu_cs * L.gu_sbb, &gsb_map, 0, kJ * jb + 8 * p, 0, e, &gu_full[gu_cs]);
            ++gu_n;
            if (++gu_cs == gus) {
                gu_cs = 0;
                ++gu_ph;
            }
        }
        const int ds = dn_n & 1;
        if (dn_n >= kDnSlots) mbar_wait_bounded(&dn_empty[ds], ((dn_n >> 1) - 1) & 1, a.err);
        mbar_arrive_expect_tx(&dn_full[ds], L.dn_box);
        tma_load_4d(smem + L.off_dn + ds * L.dn_box, &dn_map, 0, 0, e * (kH / 256), jb, &dn_full[ds]);
        ++dn_n;
        if (L.sb_tma) {
            // every row's 16-byte piece holding word jb / 2 of its (scale, bias) row; one slot
            if (sb_n >= 1) {
                if (!released) release_zero();   // the previous unit's down phase may wait on it
                mbar_wait_bounded(dsb_empty, (sb_n - 1) & 1, a.err);
            }
            mbar_arrive_expect_tx(dsb_full, (uint32_t)L.dsb_bytes);
            tma_load_4d(smem + L.off_dsb, &dsb_map, 0, 0, e * (kH / 256), (jb >> 1) >> 2, dsb_full);
            ++sb_n;
        }
    };
    // weights do not depend on earlier grids: the router rows and the shared expert's unit go first
    const int nr = kRoute ? min((E - b + G - 1) / G, kRouterRows) : 0;
    if (warp == kWarps && lane == 0) {
        // the router rows first: every CTA's logits wait on them, and the slowest CTA's decide the top-k
        if (kRoute) {
            mbar_arrive_expect_tx(rt_full, (uint32_t)(nr * 2 * kH));
            for (int r = 0; r < nr; ++r)
                bulk_load(smem + L.off_rt + r * 2 * kH, da.r.w_router + (size_t)(b + r * G) * kH, 2 * kH, rt_full);
        }
        if (early_unit) issue_unit(E, b);
    }
    const int r_e = b + warp * G;
    const bool r_on = kRoute && warp < nr;

    // The next grid may start its prologue; everything below may read what
    // earlier grids on the stream wrote.
    griddep_launch_dependents();
    griddep_wait();

    // ------------------------------------------------------------ unit compute
    // Unit k (active slot s, column block jb) by the 16 compute warps.  Gate/up:
    // warp w takes box p = w & 3 (MMA rows g: gate row perm8(g) of the box, g + 8:
    // the same up row) and K quarter kq = w >> 2.  Down: warp w takes the 16-row
    // tiles w, w + 16, ... of all H rows, K = the unit's 32 columns.
    const int p_box = warp & 3, kq = warp >> 2;
    const int gt_all = g < T ? g : T - 1;        // absent tokens read a present one; their weight is 0
    int* rows_n = tab.slot_of;                   // row-list launch: rows of each expert (a route-mode table otherwise)
    // group sums of x, per column: thread (gr, t)
    auto x_group_sums = [&](int ncols) {
        if (tid < kNG * kMaxT) {
            const int gr = tid >> 3, t = tid & 7;
            float sum = 0.0f;
            if (t < ncols) {
                const uint4* px = reinterpret_cast<const uint4*>(xs + (size_t)t * kXS + 128 * gr);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 v = px[u];
                    sum += (bf16_lo(v.x) + bf16_hi(v.x)) + (bf16_lo(v.y) + bf16_hi(v.y)) +
                           (bf16_lo(v.z) + bf16_hi(v.z)) + (bf16_lo(v.w) + bf16_hi(v.w));
                }
            }
            sx[gr * kMaxT + t] = sum;
        }
    };
    auto code_off = [&](int gr) -> uint32_t {
        return (uint32_t)(((gr >> 2) * 8 + rg) * 128) + (((uint32_t)((2 * (gr & 3)) | (c >> 1)) ^ (uint32_t)rg) << 4) +
               (uint32_t)((c & 1) << 3);
    };
    auto sb_off = [&](int row, int gr) -> uint32_t {
        const uint32_t o = (uint32_t)(row * kRB + 4 * gr);
        return o ^ (((o >> 7) & kSmask) << 4);
    };
    int cu_n = 0, cu_cs = 0, cu_ph = 0;   // consumers' view of the gate/up ring
    bool zero_seen = kRows;   // a row-list launch adds into y_acc as it is
    auto compute_unit = [&](int k, int s, int jb) {
        const int e = tab.slot_e[s];
        // MMA columns holding tokens (row-list launch: the expert's rows); absent columns read a
        // present one, and their weight is 0
        const int ncol = kRows ? rows_n[e] : T;
        const int gt = kRows ? (g < ncol ? g : ncol - 1) : gt_all;
        const uint8_t* xrow = xs + (size_t)gt * kXS + 32 * c;
        if (kRows) {
            mbar_wait_bounded(x_full, k & 1, a.err);
            x_group_sums(ncol);
            named_barrier(1, kWarps * 32);
        }
        // the down (scale, bias) word of every row for this block's group of I (the
        // TMA form lands with the unit's other boxes)
        if (!L.sb_tma) {
            const uint32_t* src = reinterpret_cast<const uint32_t*>(a.d_sb) + (size_t)e * kH * (I >> 6) + (jb >> 1);
            for (int n = tid; n < kH; n += kWarps * 32) cp_async4(smem_u32(dsb + n), src + (size_t)n * (I >> 6));
        }
        cp_async_commit();
        // ---- gate/up
        while (cu_n < 4 * k + p_box) {
            ++cu_n;
            if (++cu_cs == gus) {
                cu_cs = 0;
                cu_ph ^= 1;
            }
        }
        mbar_wait_bounded(&gu_full[cu_cs], cu_ph, a.err);
        const uint8_t* box = smem + L.off_gu + cu_cs * L.gu_box;      // [gate|up][kNCH][8 rows][128 B]
        const uint8_t* sbb = smem + L.off_gusb + cu_cs * L.gu_sbb;    // [gate|up][8 rows][kRB]
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < kNGW; ++i) {
            const int gr = kq * kNGW + i;
            const uint32_t og = code_off(gr);
            const uint2 cg = lds64(box + og), cu = lds64(box + og + kNCH * 8 * 128);
            const uint4 x0 = *reinterpret_cast<const uint4*>(xrow + 128 * gr);
            const uint4 x1 = *reinterpret_cast<const uint4*>(xrow + 128 * gr + 16);
            float d[4];
            group_mma(d, cg, cu, x0, x1);
            float sg, bg, su, bu;
            sb_factor(lds32(sbb + sb_off(rg, gr)), sg, bg);
            sb_factor(lds32(sbb + sb_off(8 + rg, gr)), su, bu);
            const float2 xsum = *reinterpret_cast<const float2*>(sx + gr * kMaxT + 2 * c);
            acc[0] = fmaf(sg, d[0], fmaf(bg, xsum.x, acc[0]));
            acc[1] = fmaf(sg, d[1], fmaf(bg, xsum.y, acc[1]));
            acc[2] = fmaf(su, d[2], fmaf(bu, xsum.x, acc[2]));
            acc[3] = fmaf(su, d[3], fmaf(bu, xsum.y, acc[3]));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&gu_empty[cu_cs]);
        red[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        named_barrier(2 + p_box, 128);   // the box's four warps
        uint16_t* hk = hs + (k & 1) * kMaxT * kJ;
        if (kq == 0) {
            float4 sum = red[p_box * 32 + lane];
#pragma unroll
            for (int q = 1; q < 4; ++q) {
                const float4 v = red[(p_box + 4 * q) * 32 + lane];
                sum.x += v.x;
                sum.y += v.y;
                sum.z += v.z;
                sum.w += v.w;
            }
            // gate (row g) and up (row g + 8) of column 8 p + rg of the block, tokens 2c, 2c+1;
            // h is kept in the split order inside each 8 columns
            const uint16_t h0 = f32_to_bf16(silu(sum.x) * sum.z);
            const uint16_t h1 = f32_to_bf16(silu(sum.y) * sum.w);
            const int pos = 8 * p_box + (rg < 4 ? 2 * rg : 2 * (rg - 4) + 1);
            hk[(2 * c) * kJ + pos] = h0;
            hk[(2 * c + 1) * kJ + pos] = h1;
            // sums of the rounded h over the box's 8 columns, per token
            float v0 = __uint_as_float((uint32_t)h0 << 16), v1 = __uint_as_float((uint32_t)h1 << 16);
#pragma unroll
            for (int off = 4; off <= 16; off <<= 1) {
                v0 += __shfl_xor_sync(0xFFFFFFFFu, v0, off);
                v1 += __shfl_xor_sync(0xFFFFFFFFu, v1, off);
            }
            if (g == 0) {
                tab.hsum[k & 1][p_box][2 * c] = v0;
                tab.hsum[k & 1][p_box][2 * c + 1] = v1;
            }
        }
        cp_async_wait<0>();
        named_barrier(1, kWarps * 32);   // h, its sums and the down (scale, bias) words complete; red[] free
        if (kRows && tid == 0) mbar_arrive(x_empty);   // x and its sums read
        // ---- down: rows 16 t + {g, g + 8} of tile t, K = the block's 32 columns
        const int ds = k & 1;
        mbar_wait_bounded(&dn_full[ds], (k >> 1) & 1, a.err);
        const uint8_t* dbox = smem + L.off_dn + ds * L.dn_box;   // [kH rows][4 words]
        const uint4 hv = *reinterpret_cast<const uint4*>(hk + gt * kJ + 8 * c);
        const int t0c = 2 * c < ncol ? 2 * c : ncol - 1, t1c = 2 * c + 1 < ncol ? 2 * c + 1 : ncol - 1;
        const float hs0 = (tab.hsum[k & 1][0][t0c] + tab.hsum[k & 1][1][t0c]) +
                          (tab.hsum[k & 1][2][t0c] + tab.hsum[k & 1][3][t0c]);
        const float hs1 = (tab.hsum[k & 1][0][t1c] + tab.hsum[k & 1][1][t1c]) +
                          (tab.hsum[k & 1][2][t1c] + tab.hsum[k & 1][3][t1c]);
        const float* wcol = kRows ? uw + k * kMaxRows : tab.wsel[s];
        const float w0 = wcol[2 * c], w1 = wcol[2 * c + 1];
        if (L.sb_tma) mbar_wait_bounded(dsb_full, k & 1, a.err);
        // row n's word: a 16-byte piece per row holding word (jb / 2) % 4 (TMA form), else one word per row
        const uint8_t* sbrow = reinterpret_cast<const uint8_t*>(dsb) + (L.sb_tma ? 4 * ((jb >> 1) & 3) : 0);
        const int sbs = L.sb_tma ? 16 : 4;
        if (!zero_seen) {   // the first reduction into y_acc waits until every CTA cleared its slice
            mbar_wait_bounded(zero_done, 0, a.err);
            zero_seen = true;
        }
        const bool two = ncol > 1;   // odd columns hold tokens
        float* stg = reinterpret_cast<float*>(red) + warp * 128;   // this warp's staging area
        // what this lane reduces: 16-float slot lane / 4 (token rd_t), its float4 lane % 4 (rows rd_row..+3)
        const int rd_s = lane >> 2;
        const int rd_t = rd_s < 4 ? 2 * rd_s : 2 * (rd_s - 4) + 1;
        const int rd_row = 4 * ((lane & 3) ^ (((rd_t >> 2) & 1) << 1));
#pragma unroll
        for (int tt = 0; tt < kTW; ++tt) {
            const int n = 16 * (warp + kWarps * tt) + g;
            const uint32_t ca = lds32(dbox + n * 16 + 4 * c), cb = lds32(dbox + (n + 8) * 16 + 4 * c);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            mma_bf16_16816(d, nib(ca, 0), nib(cb, 0), nib(ca, 1), nib(cb, 1), hv.x, hv.y);
            mma_bf16_16816(d, nib(ca, 2), nib(cb, 2), nib(ca, 3), nib(cb, 3), hv.z, hv.w);
            float sa, ba, sb2, bb2;
            sb_factor(lds32(sbrow + n * sbs), sa, ba);
            sb_factor(lds32(sbrow + (n + 8) * sbs), sb2, bb2);
            // w (s D + (b - 128 s) sum(h)) for rows n (d0, d1) and n + 8 (d2, d3), tokens 2c, 2c+1
            const float v0 = w0 != 0.0f ? w0 * fmaf(sa, d[0], ba * hs0) : 0.0f;
            const float v2 = w0 != 0.0f ? w0 * fmaf(sb2, d[2], bb2 * hs0) : 0.0f;
            const float v1 = (two && w1 != 0.0f) ? w1 * fmaf(sa, d[1], ba * hs1) : 0.0f;
            const float v3 = (two && w1 != 0.0f) ? w1 * fmaf(sb2, d[3], bb2 * hs1) : 0.0f;
            // the tile's [8 tokens][16 rows] through the warp's staging area, then one vector
            // reduction of 4 consecutive rows of one token per lane
            stg[stage_word(2 * c, g)] = v0;
            stg[stage_word(2 * c, g + 8)] = v2;
            stg[stage_word(2 * c + 1, g)] = v1;
            stg[stage_word(2 * c + 1, g + 8)] = v3;
            __syncwarp();
            const float4 r4 = *reinterpret_cast<const float4*>(stg + 16 * (lane >> 2) + 4 * (lane & 3));
            if (rd_t < ncol)
                red_add_v4(a.y_acc + (size_t)(kRows ? utok[k * kMaxRows + rd_t] : rd_t) * kH + 16 * (warp + kWarps * tt) + rd_row,
                           r4.x, r4.y, r4.z, r4.w);
            __syncwarp();   // the next tile overwrites the staging area
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&dn_empty[ds]);
            if (L.sb_tma) mbar_arrive(dsb_empty);
        }
        named_barrier(1, kWarps * 32);   // hs, dsb and the sums free for the next unit
    };

    if (warp < kWarps) {
        // ---------------------------------------------------------- prologue
        // (four-call path) the expert offsets first: the routed loads wait on them
        int lo = 0, hi = 0;
        if (!kRoute && tid < E) {
            lo = __ldcg(a.offsets + tid);
            hi = __ldcg(a.offsets + tid + 1);
        }
        // this CTA's slice of y_acc (a row-list launch adds into it as it is)
        if (!kRows) {
            const size_t n4 = (size_t)T * kH / 4, per = (n4 + G - 1) / G;
            const size_t lo4 = (size_t)b * per, hi4 = min(n4, lo4 + per);
            for (size_t q = lo4 + tid; q < hi4; q += kWarps * 32)
                reinterpret_cast<float4*>(a.y_acc)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // x (split order; a row-list launch loads each unit's rows)
        for (int t = 0; t < (kRows ? 0 : T); ++t) {
            for (int c8 = tid; c8 < kH / 8; c8 += kWarps * 32) {
                const uint4 v = *reinterpret_cast<const uint4*>(a.x + (size_t)t * kH + 8 * c8);
                *reinterpret_cast<uint4*>(xs + (size_t)t * kXS + 16 * c8) = to_split_order(v);
            }
        }
        for (int q = tid; q < (kMaxSlots + 7) * kMaxT; q += kWarps * 32) (&tab.wsel[0][0])[q] = 0.0f;
        if (tid < 8) tab.bitmap[tid] = 0u;
        named_barrier(1, kWarps * 32);
        if (sh && tid < T) tab.wsel[0][tid] = 1.0f;   // the shared expert: every token, weight 1
        if (tid == 0) {
            tab.slot_e[0] = E;
            mbar_arrive(zeroed);   // the slice is cleared; the producer counts this CTA
        }
        if (!kRows) x_group_sums(T);
        const int first = sh ? 1 : 0;
        if (kRoute) {
            // ---- router logits of this CTA's experts in the contract order: lane l
            // accumulates its chunks in order with fma, the 32 partials meet in the xor
            // butterfly 16..1, then the bias is added; tagged with the launch number
            if (r_on) {
                mbar_wait_bounded(zt_ready, 0, a.err);
                const uint32_t ep = tab.epoch;
                mbar_wait_bounded(rt_full, 0, a.err);
                const uint8_t* wrow = smem + L.off_rt + warp * 2 * kH;
                for (int t = 0; t < T; ++t) {
                    float accl = 0.0f;
#pragma unroll
                    for (int i = 0; i < kRChunks; ++i) {
                        const int ch = lane + 32 * i;
                        const uint4 wvi = *reinterpret_cast<const uint4*>(wrow + 16 * ch);
                        const uint32_t ww[4] = {wvi.x, wvi.y, wvi.z, wvi.w};
                        // x chunk in split order: (x0,x4) (x1,x5) (x2,x6) (x3,x7)
                        const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)t * kXS + 16 * ch);
                        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float xj = j < 4 ? bf16_lo(xw[j]) : bf16_hi(xw[j - 4]);
                            const float wj = (j & 1) ? bf16_hi(ww[j >> 1]) : bf16_lo(ww[j >> 1]);
                            accl = __fmaf_rn(xj, wj, accl);
                        }
                    }
#pragma unroll
                    for (int off = 16; off >= 1; off >>= 1) accl = __fadd_rn(accl, __shfl_xor_sync(0xFFFFFFFFu, accl, off));
                    if (lane < kLogitCopies) {   // every lane holds the sum; one copy each
                        if (da.r.bias) accl = __fadd_rn(accl, da.r.bias[(int64_t)t * da.r.bias_stride + r_e]);
                        st_relaxed_u64(da.tlogits + (size_t)lane * kMaxT * E + (size_t)t * E + r_e, tag_word(ep, accl));
                    }
                }
            }
            named_barrier(1, kWarps * 32);   // x group sums ready
            // ---- the shared expert's block while the other CTAs' logits arrive
            if (early_unit) compute_unit(0, 0, b);
            // ---- top-k of every token, in every CTA: poll the tagged logits
            if (warp < T) {
                mbar_wait_bounded(zt_ready, 0, a.err);
                const uint32_t ep = tab.epoch;
                float v[8];
                const uint64_t t0 = globaltimer_ns();
                bool timed_out = false;
                for (;;) {
                    bool ok = true;
                    unsigned long long w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        w[i] = ldcg_u64(da.tlogits + (size_t)(b % kLogitCopies) * kMaxT * E + (size_t)warp * E + lane + 32 * i);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        ok &= (uint32_t)w[i] == ep;
                        v[i] = __uint_as_float((uint32_t)(w[i] >> 32));
                    }
                    if (__all_sync(0xFFFFFFFFu, ok)) break;
                    if (globaltimer_ns() - t0 > 200000000ull) {
                        timed_out = true;
                        break;
                    }
                    __nanosleep(32);
                }
                if (timed_out && lane == 0) set_error(a.err, MOE_ERR_TIMEOUT);
                int e_sel;
                float w_sel;
                if (topk_from_values<8, 8>(v, e_sel, w_sel) && lane == 0 && b == 0) set_error(a.err, MOE_ERR_NONFINITE);
                if (lane < 8) {
                    tab.sel[warp * 8 + lane] = e_sel;
                    tab.selw[warp * 8 + lane] = w_sel;
                }
                if (T == 1) {
                    // one token: its 8 (distinct) experts ranked by index are the routed slots
                    int rank = 0;
#pragma unroll
                    for (int j = 0; j < 8; ++j) rank += __shfl_sync(0xFFFFFFFFu, e_sel, j) < e_sel ? 1 : 0;
                    if (lane < 8) {
                        tab.slot_e[first + rank] = e_sel;
                        tab.slot_of[e_sel] = first + rank;
                        tab.wsel[first + rank][0] = w_sel;
                    }
                    if (lane == 0) {
                        tab.A = first + 8;
                        if (sh) tab.slot_e[0] = E;
                    }
                }
            }
            if (T == 1) {
                named_barrier(1, kWarps * 32);           // the active list and its weights
                if (tid == 0) mbar_arrive(list_ready);   // are ready for the producer
            } else {
                named_barrier(1, kWarps * 32);
                // ---- active experts: the shared one, then the selected ones by index
                if (tid < T * 8) atomicOr(&tab.bitmap[tab.sel[tid] >> 5], 1u << (tab.sel[tid] & 31));
                named_barrier(1, kWarps * 32);
                if (tid < E) {
                    const int wdx = tid >> 5;
                    int below = __popc(tab.bitmap[wdx] & ((1u << (tid & 31)) - 1u));
                    for (int q = 0; q < wdx; ++q) below += __popc(tab.bitmap[q]);
                    if ((tab.bitmap[wdx] >> (tid & 31)) & 1u) {
                        tab.slot_e[first + below] = tid;
                        tab.slot_of[tid] = first + below;
                    }
                }
                if (tid == 0) {
                    int tot = 0;
                    for (int q = 0; q < 8; ++q) tot += __popc(tab.bitmap[q]);
                    tab.A = first + tot;
                    if (sh) tab.slot_e[0] = E;
                }
                named_barrier(1, kWarps * 32);
                if (tid == 0) mbar_arrive(list_ready);   // the active list is ready for the producer
                if (tid < T * 8) tab.wsel[tab.slot_of[tab.sel[tid]]][tid >> 3] = tab.selw[tid];
                named_barrier(1, kWarps * 32);           // and the weights for every compute warp
            }
            // ---- the routing outputs, by the last CTA (the four calls' results)
            if (b == G - 1) {
                const int np = T * 8;
                int cnt = 0;
                if (tid < E)
                    for (int p = 0; p < np; ++p) cnt += tab.sel[p] == tid;
                // exclusive scan of the counts over the E experts (warps 0..7)
                int inc = cnt;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int o = __shfl_up_sync(0xFFFFFFFFu, inc, off);
                    if (lane >= off) inc += o;
                }
                if (lane == 31) tab.wtot[warp] = inc;
                named_barrier(1, kWarps * 32);
                int base = 0;
                for (int q = 0; q < warp; ++q) base += tab.wtot[q];
                if (tid < E) {
                    tab.off[tid] = base + inc - cnt;
                    da.r.offsets[tid] = base + inc - cnt;
                    da.r.counts[tid] = cnt;
                }
                if (tid == 0) da.r.offsets[E] = np;
                named_barrier(1, kWarps * 32);
                if (tid < np) {
                    const int e = tab.sel[tid];
                    int rank = 0;
                    for (int q = 0; q < tid; ++q) rank += tab.sel[q] == e;
                    const int row = tab.off[e] + rank;
                    da.r.row_to_pair[row] = tid;
                    da.r.pair_to_row[tid] = row;
                    da.r.topk_idx[tid] = e;
                    da.r.topk_w[tid] = tab.selw[tid];
                }
            }
        } else {
            // ---- active experts from the permutation tables (offsets, rows -> pairs)
            bool act = false;
            if (tid < E) {
                const bool ok = lo >= 0 && hi >= lo && hi <= T * a.K && hi - lo <= T;
                if (!ok) {
                    set_error(a.err, MOE_ERR_BOUNDS);
                    lo = hi = 0;
                }
                act = hi > lo && (!kRows || hi - lo <= kMaxRows);
                if (kRows) {
                    tab.off[tid] = lo;
                    rows_n[tid] = hi - lo;
                }
            }
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, act);
            if (lane == 0) tab.wtot[warp] = __popc(bal);
            named_barrier(1, kWarps * 32);
            int s_mine = 0;
            if (act) {
                int below = __popc(bal & ((1u << lane) - 1u));
                for (int q = 0; q < warp; ++q) below += tab.wtot[q];
                s_mine = first + below;
                tab.slot_e[s_mine] = tid;
            }
            if (tid == 0) {
                int tot = 0;
                for (int q = 0; q < kWarps; ++q) tot += (q * 32 < E) ? tab.wtot[q] : 0;
                tab.A = first + tot;
                if (sh) tab.slot_e[0] = E;
            }
            named_barrier(1, kWarps * 32);
            if (tid == 0) mbar_arrive(list_ready);   // the active list is ready for the producer
            if (kRows) {
                // token and routing weight of each column of this CTA's units
                const int nk = min(b < tab.A * NJ ? (tab.A * NJ - 1 - b) / G + 1 : 0, row_units_cap(kH));
                for (int q = tid; q < nk * kMaxRows; q += kWarps * 32) {
                    const int kk = q / kMaxRows, cc = q % kMaxRows;
                    const int ee = tab.slot_e[(b + kk * G) >> (lgI - 5)];
                    int tk = 0;
                    float ww = 0.0f;
                    if (cc < rows_n[ee]) {
                        const int pr = __ldcg(a.row_to_pair + tab.off[ee] + cc);
                        if (pr < 0 || pr >= T * a.K) {
                            set_error(a.err, MOE_ERR_BOUNDS);
                        } else {
                            tk = pr / a.K;
                            ww = __ldcg(a.topk_w + pr);
                        }
                    }
                    utok[q] = tk;
                    uw[q] = ww;
                }
            }
            // routing weights of each (slot, token)
            if (!kRows && act) {
                for (int r = lo; r < hi; ++r) {
                    const int p = __ldcg(a.row_to_pair + r);
                    if (p < 0 || p >= T * a.K) {
                        set_error(a.err, MOE_ERR_BOUNDS);
                        continue;
                    }
                    tab.wsel[s_mine][p >> 3] = __ldcg(a.topk_w + p);
                }
            }
            named_barrier(1, kWarps * 32);
        }

        // ---------------------------------------------------------- units
        const int A = tab.A;
        int k = 0, u = b, s = b >> (lgI - 5), jb = b & (NJ - 1);
        const int dsl = G >> (lgI - 5), dj = G & (NJ - 1);   // advance of (slot, block) per unit
        const int kcap = kRows ? row_units_cap(kH) : 1 << 30;   // units whose column tables fit
        for (; u < A * NJ && k < kcap; u += G, ++k) {
            if (!(kRoute && k == 0 && early_unit)) compute_unit(k, s, jb);   // else done above
            s += dsl;
            jb += dj;
            if (jb >= NJ) {
                jb -= NJ;
                ++s;
            }
        }
    } else {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            if (!kRows) {   // a row-list launch neither clears y_acc nor counts itself
                // the launch number, and the count at which every CTA has cleared its slice of y_acc
                const unsigned long long v = ld_relaxed_u64(da.launches);
                tab.epoch = (uint32_t)((v / (unsigned long long)G) % 0xFFFFFFFFull) + 1u;
                tab.zero_target = (v / (unsigned long long)G + 1ull) * (unsigned long long)G;
                mbar_arrive(zt_ready);
                // count this CTA once its slice is cleared (the consumers' stores, seen through
                // the mbarrier, are ordered before the count by the fence)
                mbar_wait_bounded(zeroed, 0, a.err);
                __threadfence();
                red_add_relaxed_u64(da.launches, 1ull);
            }
            // the fused layer's shared-expert unit reduces into y_acc before the active
            // list exists; otherwise units 0 and 1 go first (their loads never wait on a
            // reduction), then the release, then the rest
            if (kRoute && early_unit) release_zero();
            mbar_wait_bounded(list_ready, 0, a.err);
            const int A = tab.A;
            int u = b, s = b >> (lgI - 5), jb = b & (NJ - 1), k = 0;
            const int dsl = G >> (lgI - 5), dj = G & (NJ - 1);
            const int kcap = kRows ? row_units_cap(kH) : 1 << 30;
            for (; u < A * NJ && k < kcap; u += G, ++k) {
                if (!released && k == 2) release_zero();
                if (!(u == b && early_unit)) issue_unit(tab.slot_e[s], jb);
                s += dsl;
                jb += dj;
                if (jb >= NJ) {
                    jb -= NJ;
                    ++s;
                }
            }
            if (!released) release_zero();
        }
        __syncwarp();
    }
}

// ------------------------------------------------------------------ host side

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

EncodeTiled dec_encode_fn() {
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

CUtensorMapSwizzle swizzle_for(int row_bytes) {
    return row_bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                            : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

// Gate/up codes as a 5-D view (32 words of a 256-input line, row j of I,
// line, gate|up, expert); one box = 8 whole rows of gate and the same 8 of
// up, landing as [gate|up][line][row][128 B].
bool make_gu_map(CUtensorMap* m, const FfnArgs& a) {
    EncodeTiled enc = dec_encode_fn();
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

// Gate/up (scale, bias) words as a 4-D view (H/64 words, row j of I,
// gate|up, expert); one box = the 8 gate and 8 up rows of a codes box,
// [gate|up][row][H/16 B], swizzled over the row's width.
bool make_gsb_map(CUtensorMap* m, const FfnArgs& a) {
    EncodeTiled enc = dec_encode_fn();
    if (!enc) return false;
    const uint64_t row = (uint64_t)a.H / 16;
    const cuuint64_t dims[4] = {(cuuint64_t)(a.H / 64), (cuuint64_t)a.I, 2, (cuuint64_t)(a.E + 1)};
    const cuuint64_t strides[3] = {row, (cuuint64_t)a.I * row, (cuuint64_t)2 * a.I * row};
    const cuuint32_t box[4] = {(cuuint32_t)(a.H / 64), 8, 2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint16_t*>(a.gu_sb), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for((int)row), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Down codes as a 4-D view (4 words of a 32-input column block, row of a
// 256-row band, band of all experts' [H, I] matrices, block); one box = the
// H rows of one expert and block: [row][16 B].
bool make_dn_map(CUtensorMap* m, const FfnArgs& a) {
    EncodeTiled enc = dec_encode_fn();
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

// Down (scale, bias) words as a 4-D view (4 words = one 16-byte piece of a
// row's I/64 words, row of a 256-row band, band of all experts' rows, piece);
// one box = the H rows of one expert, the piece holding a unit's word.
bool make_dsb_map(CUtensorMap* m, const FfnArgs& a) {
    EncodeTiled enc = dec_encode_fn();
    if (!enc) return false;
    const uint64_t row = (uint64_t)a.I / 16;   // bytes of one row's words
    const cuuint64_t dims[4] = {4, 256, (cuuint64_t)(a.E + 1) * (a.H / 256), (cuuint64_t)(a.I / 256)};
    const cuuint64_t strides[3] = {row, 256 * row, 16};
    const cuuint32_t box[4] = {4, 256, (cuuint32_t)(a.H / 256), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint16_t*>(a.d_sb), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kH, int kMode>
cudaError_t launch_dec_h(const DecArgs& da, const CUtensorMap& gu_map, const CUtensorMap& gsb_map,
                         const CUtensorMap& dn_map, const CUtensorMap& dsb_map, cudaStream_t st) {
    static int done[64] = {0};
    const int smem = da.L.total + 1024;
    cudaError_t ce = set_smem_once(k_decode<kH, kMode>, smem, done);
    if (ce != cudaSuccess) return ce;
    const int G = num_sms_cached();
    if (G <= 0) return cudaErrorInvalidDevice;
    // every 16-row down tile needs a CTA, and every router row one of the CTAs' row slots
    if (G < kH / 16 || (kMode == kModeRoute && G * kRouterRows < da.f.E)) return cudaErrorInvalidConfiguration;
    // One CTA per SM.  CTAs read words other CTAs of the launch write, so they
    // must all be resident at once: a cooperative launch fails rather than
    // starting when they cannot be.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k_decode<kH, kMode>, gu_map, gsb_map, dn_map, dsb_map, da);
}

template <int kMode>
cudaError_t launch_dec(const DecArgs& da, cudaStream_t st) {
    CUtensorMap gu_map, gsb_map, dn_map, dsb_map;
    if (!make_gu_map(&gu_map, da.f) || !make_gsb_map(&gsb_map, da.f) || !make_dn_map(&dn_map, da.f))
        return cudaErrorInvalidValue;
    if (da.L.sb_tma) {
        if (!make_dsb_map(&dsb_map, da.f)) return cudaErrorInvalidValue;
    } else {
        dsb_map = dn_map;   // not read
    }
    switch (da.f.H) {
        case 512: return launch_dec_h<512, kMode>(da, gu_map, gsb_map, dn_map, dsb_map, st);
        case 1024: return launch_dec_h<1024, kMode>(da, gu_map, gsb_map, dn_map, dsb_map, st);
        case 2048: return launch_dec_h<2048, kMode>(da, gu_map, gsb_map, dn_map, dsb_map, st);
        default: return cudaErrorInvalidValue;
    }
}

int ilog2(int v) {
    int r = 0;
    while ((1 << (r + 1)) <= v) ++r;
    return r;
}

DecArgs dec_args(const FfnArgs& a, const DecodeWs& w) {
    DecArgs da = {};
    da.f = a;
    da.L = dec_layout(a.H, a.I, a.T);
    da.launches = w.launches;
    da.tlogits = w.tlogits;
    da.lgI = ilog2(a.I);
    return da;
}

}  // namespace

bool ffn_decode_supported(const FfnArgs& a) {
    // I a power of two from 128 to 2048 (its index arithmetic is shifts)
    if (!(a.mode == MOE_MODE_SCATTER && a.T >= 1 && a.T <= kMaxT && a.K == 8 && a.G == 64 && a.E <= 256 &&
          (a.H == 512 || a.H == 1024 || a.H == 2048) && a.I >= 128 && a.I <= 2048 && (a.I & (a.I - 1)) == 0))
        return false;
    // a whole unit's four gate/up boxes fit in the ring
    return dec_layout(a.H, a.I, a.T).gu_slots >= 4;
}

size_t decode_ws_bytes(int T, int E, int I) {
    (void)T;
    (void)I;
    return align256((size_t)kLogitCopies * kMaxT * E * 8);
}

DecodeWs decode_ws_carve(uint8_t* base, int T, int E, int I, unsigned long long* launches) {
    (void)T;
    (void)E;
    (void)I;
    DecodeWs w;
    w.launches = launches;
    w.tlogits = reinterpret_cast<unsigned long long*>(base);
    return w;
}

cudaError_t launch_ffn_decode(const FfnArgs& a, const DecodeWs& w, cudaStream_t st) {
    DecArgs da = dec_args(a, w);
    return launch_dec<kModeTokens>(da, st);
}

bool decode_layer_supported(const FfnArgs& a) { return ffn_decode_supported(a) && a.E == 256; }

bool ffn_rows_supported(const FfnArgs& a) {
    if (!(a.mode == MOE_MODE_SCATTER && a.T >= 1 && a.K >= 1 && a.K <= 8 && a.G == 64 && a.E <= 256 &&
          (a.H == 512 || a.H == 1024 || a.H == 2048) && a.I >= 128 && a.I <= 2048 && (a.I & (a.I - 1)) == 0))
        return false;
    const int G = num_sms_cached();
    // a whole unit's four gate/up boxes fit in the ring beside the x slot of kMaxRows rows, and
    // every CTA's units (at most all E experts' blocks) have room for their column tables
    return G >= a.H / 16 && dec_layout(a.H, a.I, kMaxT).gu_slots >= 4 &&
           (a.E * (a.I / kJ) + G - 1) / G <= row_units_cap(a.H);
}

cudaError_t launch_ffn_rows(const FfnArgs& a, cudaStream_t st) {
    DecodeWs w = {};   // no launch counter, no logits: y_acc is not cleared, nothing is polled
    DecArgs da = dec_args(a, w);
    da.L = dec_layout(a.H, a.I, kMaxT);
    return launch_dec<kModeRows>(da, st);
}

cudaError_t launch_decode_layer(const FfnArgs& a, const DecodeRoute& r, const DecodeWs& w, cudaStream_t st) {
    DecArgs da = dec_args(a, w);
    da.r = r;
    return launch_dec<kModeRoute>(da, st);
}

}  // namespace moe
