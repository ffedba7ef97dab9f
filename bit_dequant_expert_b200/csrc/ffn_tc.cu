// Expert FFNs for prefill: grouped GEMMs on the 5th-generation tensor cores
// with the 4-bit dequantisation fused into the main loop.
//
// Lily pages: "Perplexity's Lily brings fast local AI to Apple silicon Macs",
// section "Where the Engine Gains Speed" (weights reconstructed inside the
// grouped GEMM, one tile at a time; expert GEMMs take about 90% of prefill);
// "Perplexity built an inference engine for one model, one chip", third
// paragraph (folding the dequantisation into the matrix multiplication so an
// expanded array never touches memory: +77.4% prefill at 512 tokens).
//
// One persistent kernel, launched once for gate/up (+SwiGLU) and once for
// down (+weighted combine).  A tile is 128 weight rows (MMA M) x up to nt
// token rows (MMA N) of one expert; K runs in 128-input stages (two (scale,
// bias) groups), three stages in flight.  nt is 128, or 80 when the experts
// hold few rows each (T k <= 96 E): one thread's stream of tcgen05.mma
// instructions runs at about one per 66 ns for any N up to 256, so narrow
// tiles are bound by the issue rate, and then the two 64-input halves of
// every stage go to two issuing threads with an accumulator each.  Roles:
//   warp 0       TMA of the codes (128 rows x 256 inputs per 16 KB box, two
//                stages, 128B-swizzled) and of each tile's (scale, bias) rows;
//   warps 2-3    one 3-D TMA box per stage of the B operand: the tile's token
//                rows (x gathered into expert order for gate/up, h for down),
//                two 64-input halves, 128B-swizzled and K-major as the MMA
//                reads them; alternate stages each; for down also each
//                tile's per-column token and routing weight;
//   warps 4-11   dequantise codes to bf16 (scale * q + bias; a code word
//                gives the nibble pairs (j, j+4), and x and h are stored in
//                that order inside every 8 inputs) and write them as the A
//                operand straight into tensor memory (tcgen05.st); warps
//                4-7 the first 64 inputs of a stage, 8-11 the other 64;
//   warps 1, 16  one thread each issues the tcgen05.mma (K = 16 each) of a
//                stage (warp 1 all 8 when nt = 128; 4 each, one 64-input
//                half, when nt = 80) into the tile's accumulator(s), double-
//                buffered, and commits to mbarriers;
//   warps 12-15  epilogue from TMEM (the sum of the two K-half accumulators
//                when split): SwiGLU (gate and up rows interleaved on
//                adjacent TMEM lanes) -> h in bf16, or bf16 rows (paired
//                32-bit stores) / w * y added into y_acc (fp32 red).
// Every wait is bounded (error word MOE_ERR_TIMEOUT, never a hang).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kThreads = 544;
// Token rows per tile (MMA N, max), chosen per launch: 128 with one MMA
// issuer and two accumulator buffers, or 80 with the K halves of every chunk
// on two issuers (four accumulators: two K halves, double-buffered); either
// way the accumulators end below column kACol0 and the A stages fill the
// rest of the 512 TMEM columns.
constexpr int kNTWide = 128;
constexpr int kNTSplit = 80;
static_assert(kNTSplit % 16 == 0, "MMA N is a multiple of 16");
constexpr int kBK = 128;                 // inputs per chunk = two (scale, bias) groups
constexpr int kStages = 3;              // B ring and TMEM A stages (128 inputs each)
constexpr int kCStages = 4;             // codes ring
constexpr int kCodesStage = 128 * 128;  // 128 rows x 256 nibbles (four chunks), 128B-swizzled
constexpr int kBRows = 128;              // rows of the larger B box (tiles of more than 64 rows)
constexpr int kBStage = kBRows * 2 * 128;   // two 64-input halves of up to 128 rows x 64 bf16
constexpr int kACol0 = 4 * kNTSplit;     // TMEM: the accumulators, then the A stages
static_assert(2 * kNTWide <= kACol0, "TMEM budget");
constexpr int kAStageCols = kBK / 2;     // bf16 pairs per 32-bit column
constexpr int kTmemCols = 512;
constexpr int kTabs = 4;                 // column tables in flight (down epilogue)
constexpr int kStageStride = 36;         // floats per staged column (32 rows + 4: conflict-free float4 reads)
constexpr int kSbBytes = 16384;          // one tile's (scale, bias) words: 128 rows x up to 32 groups
static_assert(kACol0 + kStages * kAStageCols <= kTmemCols, "TMEM budget");

struct Smem {
    uint8_t b[kStages][kBStage];                 // offset 0, 1024-aligned
    uint8_t codes[kCStages][kCodesStage];
    uint32_t sbs[2][kSbBytes / 4];               // per-tile (scale, bias) rows, double-buffered
    uint64_t full[kStages], a_full[2][kStages], mma_done[kStages], cfull[kCStages], cempty[kCStages];
    uint64_t acc_full[2], acc_empty[2], tab_full[kTabs], tab_empty[kTabs], sb_full[2], sb_empty[2];
    int tok[kTabs][kNTWide];
    float w[kTabs][kNTWide];
    int pre[260];
    int off[260];                                // offsets[0..E], cached
    float stage[4][16 * kStageStride];           // scatter epilogue: a warp's 16 columns x 32 rows
    uint32_t tmem_base;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory per block");

struct TcArgs {
    FfnArgs f;
    int gateup;      // 1: gate/up + SwiGLU; 0: down + combine
    int nt;          // token rows per tile: kNTSplit (ksplit) or kNTWide
    int ksplit;      // 1: the K halves of every chunk on two MMA issuers
};

struct Tile {
    int e, r0, nr, npad, mb;   // expert (E = shared), first row, rows, rows padded to 16, M block
    size_t hrow0;              // first h row of the tile
};

__device__ __forceinline__ int tiles_per_block_row(const FfnArgs& a, int gateup) {
    return gateup ? a.I / 64 : a.H / 128;
}

// Prefix of tiles per expert: pre[e] first tile of expert e, pre[E] first
// shared tile, pre[E+1] total.  blockDim.x >= E.  Experts of 1..kSkipRows
// rows get no tiles (another launch takes them).
template <int kSkipRows>
__device__ void tile_prefix(const FfnArgs& a, int gateup, int nt, int* pre, int* off) {
    __shared__ int warp_tot[32];
    const int MB = tiles_per_block_row(a, gateup);
    const int e = threadIdx.x;
    int tiles = 0;
    if (e < a.E) {
        int lo = a.offsets[e], hi = a.offsets[e + 1];
        if (lo < 0 || hi < lo || hi > a.T * a.K) {
            set_error(a.err, MOE_ERR_BOUNDS);
            lo = hi = 0;
        }
        tiles = (hi - lo + nt - 1) / nt * MB;
        if (kSkipRows > 0 && hi - lo <= kSkipRows) tiles = 0;
        off[e] = lo;
        if (e == a.E - 1) off[a.E] = hi;
    }
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
    if (e < a.E) pre[e] = base + inc - tiles;
    if (threadIdx.x == blockDim.x - 1) {
        const int routed = base + inc;
        pre[a.E] = routed;
        pre[a.E + 1] = routed + (a.has_shared ? (a.T + nt - 1) / nt * MB : 0);
    }
    __syncthreads();
}

__device__ __forceinline__ Tile decode_tile(const FfnArgs& a, int gateup, int nt, const int* pre, const int* off,
                                            int t) {
    const int MB = tiles_per_block_row(a, gateup);
    Tile tl;
    int e;
    if (t >= pre[a.E]) {
        e = a.E;
    } else {
        int lo = 0, hi = a.E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pre[mid] <= t) lo = mid; else hi = mid - 1;
        }
        e = lo;
    }
    const int local = t - pre[e];
    const int tb = local / MB;
    tl.e = e;
    tl.mb = local % MB;
    if (e == a.E) {
        tl.r0 = tb * nt;
        tl.nr = min(nt, a.T - tl.r0);
        tl.hrow0 = (size_t)a.T * a.K + tl.r0;
    } else {
        tl.r0 = off[e] + tb * nt;
        tl.nr = min(nt, (e + 1 < a.E ? off[e + 1] : off[a.E]) - tl.r0);
        tl.hrow0 = tl.r0;
    }
    tl.npad = (tl.nr + 15) & ~15;
    return tl;
}

// First weight row (within the packed matrices) of the tile's two 64-row
// halves (gate/up) or of its 128 rows (down).
__device__ __forceinline__ int wrow_gate(const FfnArgs& a, const Tile& tl) { return tl.e * 2 * a.I + 64 * tl.mb; }
__device__ __forceinline__ int wrow_up(const FfnArgs& a, const Tile& tl) { return tl.e * 2 * a.I + a.I + 64 * tl.mb; }
__device__ __forceinline__ int wrow_down(const FfnArgs& a, const Tile& tl) { return tl.e * a.H + 128 * tl.mb; }

template <int kSkipRows>
__global__ void __launch_bounds__(kThreads, 1)
    k_ffn_tc(const __grid_constant__ CUtensorMap codes_map, const __grid_constant__ CUtensorMap b_map64,
             const __grid_constant__ CUtensorMap b_map128, const __grid_constant__ CUtensorMap sb_map,
             const TcArgs ta) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the 128B-swizzled B stages need a 1024-byte aligned base
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const FfnArgs& a = ta.f;
    const int gateup = ta.gateup;
    const int nt = ta.nt, ksplit = ta.ksplit;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = gateup ? a.H : a.I;            // reduction length of this GEMM
    const int KC = K / kBK;                      // chunks per tile
    const int ngroups = K / 64;
    // codes come in stages of cw u32 words (8 cw inputs) per row: 256 inputs,
    // or all of K when K is shorter; a stage feeds 1 << cps_sh chunks
    const int cw = K >= 256 ? 32 : K / 8;
    const int cps_sh = cw == 32 ? 1 : 0;         // a stage feeds 1 << cps_sh chunks
    const int cps_mask = (1 << cps_sh) - 1;
    // (scale, bias) rows go through shared memory by TMA when a row's words
    // span whole 16-byte units; otherwise (tiny K) each thread reads its own
    const bool sb_tma = (ngroups & 3) == 0;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.a_full[0][s], 4);
            mbar_init(&sm.a_full[1][s], 4);
            mbar_init(&sm.mma_done[s], ksplit ? 2 : 1);
        }
        for (int s = 0; s < kCStages; ++s) {
            mbar_init(&sm.cfull[s], 1);
            mbar_init(&sm.cempty[s], 8);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], ksplit ? 2 : 1);
            mbar_init(&sm.acc_empty[b], 4);
        }
        for (int b = 0; b < kTabs; ++b) {
            mbar_init(&sm.tab_full[b], 2);
            mbar_init(&sm.tab_empty[b], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.sb_full[b], 1);
            mbar_init(&sm.sb_empty[b], 8);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    // y_acc is accumulated by the down launch; the gate/up launch (which runs
    // before it on the stream) zeroes it.
    if (gateup && a.mode == MOE_MODE_SCATTER) {
        const size_t n4 = (size_t)a.T * a.H / 4, per = (n4 + gridDim.x - 1) / gridDim.x;
        const size_t lo = blockIdx.x * per, hi = min(n4, lo + per);
        for (size_t q = lo + tid; q < hi; q += kThreads)
            reinterpret_cast<float4*>(a.y_acc)[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tile_prefix<kSkipRows>(a, gateup, nt, sm.pre, sm.off);   // contains __syncthreads
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int ntiles = sm.pre[a.E + 1];

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // (scale, bias) rows once per tile, codes once per stage of 1 << cps_sh chunks;
        // a stage is refilled once its chunks were dequantised.
        uint32_t it = 0, lt = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
            const Tile tl = decode_tile(a, gateup, nt, sm.pre, sm.off, t);
            if (sb_tma && lane == 0) {
                const int buf = lt & 1;
                if (lt >= 2) mbar_wait_bounded(&sm.sb_empty[buf], ((lt >> 1) - 1) & 1, a.err);
                mbar_arrive_expect_tx(&sm.sb_full[buf], 128 * ngroups * 4);
                if (gateup) {
                    tma_load_2d(sm.sbs[buf], &sb_map, 0, wrow_gate(a, tl), &sm.sb_full[buf]);
                    tma_load_2d(sm.sbs[buf] + 64 * ngroups, &sb_map, 0, wrow_up(a, tl), &sm.sb_full[buf]);
                } else {
                    tma_load_2d(sm.sbs[buf], &sb_map, 0, wrow_down(a, tl), &sm.sb_full[buf]);
                }
            }
            for (int kc = 0; kc < KC; ++kc, ++it) {
                if (lane == 0) {
                    if ((kc & cps_mask) == 0) {
                        const uint32_t cit = it >> cps_sh;    // tiles hold whole codes stages
                        const int cs = cit & (kCStages - 1);
                        if (cit >= kCStages) mbar_wait_bounded(&sm.cempty[cs], ((cit / kCStages) - 1) & 1, a.err);
                        mbar_arrive_expect_tx(&sm.cfull[cs], 128 * cw * 4);
                        if (gateup) {
                            tma_load_2d(sm.codes[cs], &codes_map, kc * 16, wrow_gate(a, tl), &sm.cfull[cs]);
                            tma_load_2d(sm.codes[cs] + 64 * cw * 4, &codes_map, kc * 16, wrow_up(a, tl), &sm.cfull[cs]);
                        } else {
                            tma_load_2d(sm.codes[cs], &codes_map, kc * 16, wrow_down(a, tl), &sm.cfull[cs]);
                        }
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 1 || warp == 16) {
        // ------------------------------------------------------------ MMA issuers
        // One thread of warp 1 issues the MMAs of the first 64 inputs of every
        // chunk into K-half accumulator 0 of the tile's buffer, one of warp 16
        // those of the other 64 into accumulator 1: a thread's tcgen05.mma
        // stream runs at about one instruction per 66 ns whatever N is, so two
        // streams raise the rate for the narrow token tiles; the epilogue adds
        // the two accumulators.
        const int h = warp == 1 ? 0 : 1;
        // one issuer (warp 1) for the whole chunk when the K halves are not split
        if (lane == 0 && (ksplit || h == 0)) {
            uint32_t lt = 0, par = 0;
            int s = 0;   // ring stage and its phase, advanced per chunk
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
                const Tile tl = decode_tile(a, gateup, nt, sm.pre, sm.off, t);
                const int ab = lt & 1;
                if (lt >= 2) mbar_wait_bounded(&sm.acc_empty[ab], ((lt >> 1) - 1) & 1, a.err);
                tc_fence_after();
                const uint32_t idesc = idesc_bf16_f32(128, tl.npad);
                const uint32_t d_tmem = tmem + (ksplit ? (2 * ab + h) * nt : ab * nt);
                for (int kc = 0; kc < KC; ++kc) {
                    if (ksplit) {
                        mbar_wait_bounded(&sm.a_full[h][s], par, a.err);
                    } else {
                        mbar_wait_bounded(&sm.a_full[0][s], par, a.err);
                        mbar_wait_bounded(&sm.a_full[1][s], par, a.err);
                    }
                    mbar_wait_bounded(&sm.full[s], par, a.err);
                    tc_fence_after();
                    // B stage: two 64-input halves of R token rows each (R = 64 or 128)
                    const int R = tl.npad > 64 ? 128 : 64;
                    const uint64_t bdesc0 = smem_desc_sw128(smem_u32(sm.b[s]));
                    const uint64_t bdesc1 = smem_desc_sw128(smem_u32(sm.b[s] + R * 128));
                    const uint32_t a_tmem = tmem + kACol0 + s * kAStageCols;
                    // straight-line issue: a branch between two tcgen05.mma costs about
                    // as much as the instruction itself
                    if (ksplit) {
                        const uint64_t bd = h ? bdesc1 : bdesc0;
                        const uint32_t at = a_tmem + 32 * h;
#pragma unroll
                        for (int j = 0; j < 4; ++j) tc_mma_ts(d_tmem, at + 8 * j, bd + 2 * j, idesc, (kc | j) != 0);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            tc_mma_ts(d_tmem, a_tmem + 8 * j, (j < 4 ? bdesc0 : bdesc1) + 2 * (j & 3), idesc,
                                      (kc | j) != 0);
                    }
                    tc_commit(&sm.mma_done[s]);
                    if (++s == kStages) {
                        s = 0;
                        par ^= 1u;
                    }
                }
                tc_commit(&sm.acc_full[ab]);
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ B producers (+ down column tables)
        // A single thread can keep only one TMA box in flight at a time, so the
        // B boxes are issued by two warps, alternate chunks each.
        const int bt = tid - 64;
        const uint32_t par = warp - 2;
        uint32_t it = 0, lt = 0, bph = 0;
        int bst = 0;   // ring stage of chunk it and its phase
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
            const Tile tl = decode_tile(a, gateup, nt, sm.pre, sm.off, t);
            if (!gateup) {
                const int slot = lt % kTabs;
                if (lt >= kTabs) mbar_wait_bounded(&sm.tab_empty[slot], ((lt / kTabs) - 1) & 1, a.err);
#pragma unroll
                for (int h = 0; h < kNTWide / 64; ++h) {   // 64 builder threads, nt columns
                    const int c = bt + 64 * h;
                    if (c >= nt) break;
                    int tok = 0;
                    float w = 0.0f;
                    if (c < tl.nr) {
                        if (tl.e == a.E) {
                            tok = tl.r0 + c;
                            w = 1.0f;
                        } else {
                            const int p = a.row_to_pair[tl.r0 + c];
                            if (p >= 0 && p < a.T * a.K) {
                                tok = p / a.K;
                                w = a.topk_w[p];
                            } else {
                                set_error(a.err, MOE_ERR_BOUNDS);
                            }
                        }
                    }
                    sm.tok[slot][c] = tok;
                    sm.w[slot][c] = w;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.tab_full[slot]);
            }
            // one 3-D box per chunk: R token rows x two 64-input halves
            const int R = tl.npad > 64 ? 128 : 64;
            for (int kc = 0; kc < KC; ++kc, ++it) {
                const int s = bst;
                const uint32_t ph = bph;
                if (++bst == kStages) {
                    bst = 0;
                    bph ^= 1u;
                }
                if ((it & 1u) != par) continue;
                if (lane == 0) {
                    if (it >= kStages) mbar_wait_bounded(&sm.mma_done[s], ph ^ 1u, a.err);
                    mbar_arrive_expect_tx(&sm.full[s], R * 2 * 128);
                    tma_load_3d(sm.b[s], R == 128 ? &b_map128 : &b_map64, 0, (int)tl.hrow0, 2 * kc, &sm.full[s]);
                }
                __syncwarp();
            }
        }
    } else if (warp < 12) {
        // ------------------------------------------------------------ dequantisers
        const int q = warp & 3;              // TMEM lane quadrant
        const int khalf = (warp - 4) >> 2;   // which 64 inputs (group) of the chunk
        const int L = 32 * q + lane;         // A row == TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16) + kACol0 + 32 * khalf;
        const uint32_t* sbase = reinterpret_cast<const uint32_t*>(gateup ? a.gu_sb : a.d_sb);
        // codes of row L inside a stage: gate/up interleave gate and up rows on
        // adjacent lanes (even: gate, odd: up), so SwiGLU pairs are lane pairs
        // row of lane L inside a codes stage; rows are cw words wide and, when
        // 128 bytes wide, 128B-swizzled (16-byte unit u of row r sits at u ^ (r & 7))
        const int crow = gateup ? ((L & 1) * 64 + (L >> 1)) : L;
        // 16-byte unit u of row crow in codes stage cs (128B-swizzled when the rows are
        // 128 bytes wide: unit u of row r sits at u ^ (r & 7))
        auto codes_at = [&](int cs, int u) -> uint4 {
            const int phys = cw == 32 ? (u ^ (crow & 7)) : u;
            return *reinterpret_cast<const uint4*>(sm.codes[cs] + crow * cw * 4 + phys * 16);
        };
        uint32_t it = 0, lt = 0, dph = 0;
        int dst = 0;   // ring stage of chunk it and its phase
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
            const Tile tl = decode_tile(a, gateup, nt, sm.pre, sm.off, t);
            const int wrow = gateup ? ((L & 1) ? wrow_up(a, tl) : wrow_gate(a, tl)) + (L >> 1) : wrow_down(a, tl) + L;
            const uint32_t* sbrow = sbase + (size_t)wrow * ngroups;
            const int buf = lt & 1;
            // this row's (scale, bias) words in shared memory: gate rows 0..63, up rows 64..127
            const int srow = gateup ? ((L & 1) * 64 + (L >> 1)) : L;
            const uint32_t* sbs_row = sm.sbs[buf] + (size_t)srow * ngroups;
            if (sb_tma) mbar_wait_bounded(&sm.sb_full[buf], (lt >> 1) & 1, a.err);
            auto dequant16 = [&](uint4 cw, uint32_t sbw, uint32_t* v) {
                const uint32_t s2 = prmt(sbw, sbw, 0x1010), b2 = prmt(sbw, sbw, 0x3232);
                const uint32_t wds[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint32_t w0 = wds[m], w4 = w0 >> 4;
                    // nibble pairs (j, j+4) of the word: the split order of every 8 inputs,
                    // which the activation rows (xg, h) are stored in as well
                    v[4 * m + 0] = dequant_split(w0, s2, b2);
                    v[4 * m + 1] = dequant_split(w4, s2, b2);
                    v[4 * m + 2] = dequant_split(w0 >> 8, s2, b2);
                    v[4 * m + 3] = dequant_split(w0 >> 12, s2, b2);
                }
            };
            // one chunk per round: this warp's 64 inputs (one group) of 32 rows
            for (int kc = 0; kc < KC; ++kc, ++it) {
                const int s = dst;
                const uint32_t ph = dph;
                if (++dst == kStages) {
                    dst = 0;
                    dph ^= 1u;
                }
                const int grp = 2 * kc + khalf;
                // 128-byte (scale, bias) rows are 128B-swizzled: word g of row r at unit (g/4) ^ (r&7)
                const uint32_t sbw = !sb_tma ? ldg_u32(sbrow + grp)
                                     : ngroups == 32 ? sbs_row[(((grp >> 2) ^ (srow & 7)) << 2) | (grp & 3)]
                                                     : sbs_row[grp];
                const uint32_t cit = it >> cps_sh;    // tiles hold whole codes stages
                const int cs = cit & (kCStages - 1);
                mbar_wait_bounded(&sm.cfull[cs], (cit / kCStages) & 1, a.err);
                const int u0 = (kc & cps_mask) * 4 + khalf * 2;
                const uint4 cw0 = codes_at(cs, u0);
                const uint4 cw1 = codes_at(cs, u0 + 1);
                if (((kc + 1) & cps_mask) == 0) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.cempty[cs]);
                }
                uint32_t v0[16], v1[16];
                dequant16(cw0, sbw, v0);
                dequant16(cw1, sbw, v1);
                // the tensor-memory A stage is free once the MMAs of its previous use completed
                if (it >= kStages) mbar_wait_bounded(&sm.mma_done[s], ph ^ 1u, a.err);
                tc_fence_after();
                tmem_st16(lane_addr + s * kAStageCols, v0);
                tmem_st16(lane_addr + s * kAStageCols + 16, v1);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.a_full[khalf][s]);
            }
            if (sb_tma) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sb_empty[buf]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        uint32_t lt = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
            const Tile tl = decode_tile(a, gateup, nt, sm.pre, sm.off, t);
            const int slot = lt % kTabs;
            if (!gateup) mbar_wait_bounded(&sm.tab_full[slot], (lt / kTabs) & 1, a.err);
            const int ab = lt & 1;
            mbar_wait_bounded(&sm.acc_full[ab], (lt >> 1) & 1, a.err);
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (ksplit ? 2 : 1) * ab * nt;
            for (int c0 = 0; c0 < tl.npad; c0 += 16) {
                // the sum of the two K-half accumulators (the warp is converged for
                // the warp-wide tensor-memory loads)
                uint32_t v[16];
                __syncwarp();
                tmem_ld16(taddr + c0, v);
                if (ksplit) {
                    uint32_t v1[16];
                    tmem_ld16(taddr + nt + c0, v1);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) + __uint_as_float(v1[c]));
                } else {
                    tmem_ld_wait();
                }
                if (gateup) {
                    // lanes 2i / 2i+1 hold gate / up of row j = 64 mb + 16 q + i; the
                    // even lane finishes the even columns, the odd lane the odd ones
                    const int j = 64 * tl.mb + 16 * q + (lane >> 1);
                    const int odd = lane & 1;
#pragma unroll
                    for (int c = 0; c < 16; c += 2) {
                        const float m0 = __uint_as_float(v[c]), m1 = __uint_as_float(v[c + 1]);
                        // even lane sends column c+1, odd lane sends column c
                        const float recv = __shfl_xor_sync(0xFFFFFFFFu, odd ? m0 : m1, 1);
                        const float gate = odd ? recv : m0;       // column c + odd
                        const float up = odd ? m1 : recv;
                        const int col = c0 + c + odd;
                        if (col < tl.nr) {
                            const float hval = __fdividef(gate, 1.0f + __expf(-gate)) * up;
                            // h is kept in the split order inside every 8 columns (the down
                            // GEMM's dequantised weights come in that order)
                            const int js = (j & ~7) | ((j & 4) ? 2 * (j & 3) + 1 : 2 * (j & 3));
                            a.h[(tl.hrow0 + col) * a.I + js] = f32_to_bf16(hval);
                        }
                    }
                } else if (a.mode != MOE_MODE_SCATTER) {
                    // bf16 rows: lanes 2i / 2i+1 swap one column so that each writes two
                    // adjacent outputs (n, n+1) of one token row with a 32-bit store
                    const int n = 128 * tl.mb + 32 * q + lane;
                    const int odd = lane & 1;
                    uint16_t* dst = tl.e == a.E ? a.y_shared : a.y_rows;
#pragma unroll
                    for (int c = 0; c < 16; c += 2) {
                        const float y0 = __uint_as_float(v[c]), y1 = __uint_as_float(v[c + 1]);
                        const float recv = __shfl_xor_sync(0xFFFFFFFFu, odd ? y0 : y1, 1);
                        const int col = c0 + c + odd;
                        const uint32_t pk = odd ? pack_bf16x2(recv, y1) : pack_bf16x2(y0, recv);
                        if (col < tl.nr)
                            *reinterpret_cast<uint32_t*>(dst + (size_t)(tl.r0 + col) * a.H + (n & ~1)) = pk;
                    }
                } else {
                    // fp32 y_acc: w * y added into the token's row.  The warp's 32 rows x 16
                    // columns go through shared memory so that each lane adds 4 consecutive
                    // outputs of one token with one vector reduction
                    float* stg = sm.stage[q];
                    const int n0 = 128 * tl.mb + 32 * q;
#pragma unroll
                    for (int c = 0; c < 16; ++c) stg[c * kStageStride + lane] = sm.w[slot][c0 + c] * __uint_as_float(v[c]);
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c = (lane >> 3) + 4 * i, r4 = lane & 7;   // column, row quad
                        const int col = c0 + c;
                        if (col < tl.nr) {
                            const float4 f = *reinterpret_cast<const float4*>(stg + c * kStageStride + 4 * r4);
                            red_add_v4(a.y_acc + (size_t)sm.tok[slot][col] * a.H + n0 + 4 * r4, f.x, f.y, f.z, f.w);
                        }
                    }
                    __syncwarp();   // the next chunk overwrites the staging area
                }
            }
            if (!gateup) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.tab_empty[slot]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
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

// Packed codes of n_mat stacked [N, K] matrices as a 2-D tensor of u32 words
// (K/8 per row), read in boxes of 8 words x box_rows rows.
bool make_codes_map(CUtensorMap* m, const uint32_t* codes, int rows, int K, int box_rows) {
    EncodeTiled enc = encode_fn();
    if (!enc) return false;
    const int cw = K >= 256 ? 32 : K / 8;      // words per row per box, as the kernel reads them
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 8), (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    const cuuint32_t box[2] = {(cuuint32_t)cw, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, cw == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [rows, cols] activations as a 3-D view (64 columns of a 64-column
// block, row, block), read in boxes of box_rows rows x two blocks (128
// columns), each block 128B-swizzled: the K-major layout the MMA reads.
bool make_act_map(CUtensorMap* m, const uint16_t* base, int rows, int cols, int box_rows) {
    EncodeTiled enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
    const cuuint64_t strides[2] = {(cuuint64_t)cols * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (scale, bias) words of stacked [N, K] matrices: rows of K/64 u32, read
// in boxes of all K/64 words x box_rows rows.
bool make_sb_map(CUtensorMap* m, const uint16_t* sb, int rows, int K, int box_rows) {
    EncodeTiled enc = encode_fn();
    if (!enc) return false;
    const int ng = K / 64;
    const cuuint64_t dims[2] = {(cuuint64_t)ng, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ng * 4};
    const cuuint32_t box[2] = {(cuuint32_t)ng, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    // 128-byte rows land 128B-swizzled, so the 32 rows one load instruction
    // touches spread over the banks
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint16_t*>(sb), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, ng == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    return sms[dev];
}

// xg[r] = x[token of row r]: routed rows in expert order (row_to_pair), then
// the shared expert's rows (tokens 0..T-1), each 8 inputs in the split order.
// One warp per row, 16-byte moves.
__global__ void __launch_bounds__(256) k_gather_rows(FfnArgs a) {
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    const int rows = (a.K + 1) * a.T;
    if (row >= rows) return;
    int tok;
    if (row >= a.T * a.K) {
        tok = row - a.T * a.K;
    } else {
        const int p = a.row_to_pair[row];
        tok = (p >= 0 && p < a.T * a.K) ? p / a.K : 0;
        if (p < 0 || p >= a.T * a.K) set_error(a.err, MOE_ERR_BOUNDS);
    }
    const uint4* __restrict__ src = reinterpret_cast<const uint4*>(a.x + (size_t)tok * a.H);
    uint4* __restrict__ dst = reinterpret_cast<uint4*>(a.xg + (size_t)row * a.H);
    // each 8 inputs in the split order (0,4,1,5,2,6,3,7) of the dequantised weights; a lane
    // issues up to kPer loads before its stores (one round covers H = 2048)
    constexpr int kPer = 8;
    const int n8 = a.H / 8;
    for (int c0 = lane; c0 < n8; c0 += 32 * kPer) {
        uint4 v[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i)
            if (c0 + 32 * i < n8) v[i] = __ldg(src + c0 + 32 * i);
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            if (c0 + 32 * i < n8) {
                uint4 r;
                r.x = prmt(v[i].x, v[i].z, 0x5410);
                r.y = prmt(v[i].x, v[i].z, 0x7632);
                r.z = prmt(v[i].y, v[i].w, 0x5410);
                r.w = prmt(v[i].y, v[i].w, 0x7632);
                dst[c0 + 32 * i] = r;
            }
        }
    }
}

}  // namespace

bool ffn_tc_supported(const FfnArgs& a) {
    // a codes stage (256 inputs, or all of K when K is 128) holds whole chunks
    // of 128 inputs and every tile whole stages: K is 128 or a multiple of 256
    // for both GEMMs; one tile's (scale, bias) rows must fit their buffer
    auto k_ok = [](int k) { return k == 128 || (k >= 256 && k % 256 == 0); };
    return a.E <= 256 && a.K >= 1 && a.K <= 8 && a.G == 64 && k_ok(a.H) && k_ok(a.I) && 128 * (a.H / 64) * 4 <= kSbBytes &&
           128 * (a.I / 64) * 4 <= kSbBytes;
}

cudaError_t launch_ffn_tc(const FfnArgs& a, int skip_rows, cudaStream_t st) {
    const int nmat = a.E + 1;
    CUtensorMap gu_map, d_map, x_map, h_map, x_map128, h_map128;
    if (!make_codes_map(&gu_map, a.gu_codes, nmat * 2 * a.I, a.H, 64)) return cudaErrorInvalidValue;
    if (!make_codes_map(&d_map, a.d_codes, nmat * a.H, a.I, 128)) return cudaErrorInvalidValue;
    if (!make_act_map(&x_map, a.xg, (a.K + 1) * a.T, a.H, 64)) return cudaErrorInvalidValue;
    if (!make_act_map(&h_map, a.h, (a.K + 1) * a.T, a.I, 64)) return cudaErrorInvalidValue;
    if (!make_act_map(&x_map128, a.xg, (a.K + 1) * a.T, a.H, 128)) return cudaErrorInvalidValue;
    if (!make_act_map(&h_map128, a.h, (a.K + 1) * a.T, a.I, 128)) return cudaErrorInvalidValue;
    // (scale, bias) maps only when a row's words fill whole 16-byte units
    CUtensorMap gsb_map = gu_map, dsb_map = d_map;
    if ((a.H / 64) % 4 == 0 && !make_sb_map(&gsb_map, a.gu_sb, nmat * 2 * a.I, a.H, 64)) return cudaErrorInvalidValue;
    if ((a.I / 64) % 4 == 0 && !make_sb_map(&dsb_map, a.d_sb, nmat * a.H, a.I, 128)) return cudaErrorInvalidValue;
    const int grows = (a.K + 1) * a.T;
    k_gather_rows<<<(grows + 7) / 8, 256, 0, st>>>(a);
    const int smem = (int)sizeof(Smem) + 1024;
    static int done[64] = {0};
    // experts of at most 8 rows left to the decode kernel's row-list launch, or none
    auto kern = skip_rows == 8 ? k_ffn_tc<8> : k_ffn_tc<0>;
    if (skip_rows != 0 && skip_rows != 8) return cudaErrorInvalidValue;
    static int done8[64] = {0};
    cudaError_t ce = set_smem_once(kern, smem, skip_rows == 8 ? done8 : done);
    if (ce != cudaSuccess) return ce;
    const int G = num_sms();
    if (G <= 0) return cudaErrorInvalidDevice;
    TcArgs ta;
    ta.f = a;
    ta.gateup = 1;
    // narrow tiles on two MMA issuers when the experts hold few rows each
    // (a tcgen05.mma stream costs about the same per instruction for any N)
    ta.ksplit = (int64_t)a.T * a.K <= (int64_t)96 * a.E ? 1 : 0;
    ta.nt = ta.ksplit ? kNTSplit : kNTWide;
    kern<<<G, kThreads, smem, st>>>(gu_map, x_map, x_map128, gsb_map, ta);
    ce = cudaGetLastError();
    if (ce != cudaSuccess) return ce;
    ta.gateup = 0;
    kern<<<G, kThreads, smem, st>>>(d_map, h_map, h_map128, dsb_map, ta);
    return cudaGetLastError();
}

}  // namespace moe
