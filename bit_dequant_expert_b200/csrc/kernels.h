// Host-side launchers of the moe_b200 kernels (internal interface).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

namespace moe {

struct RouterArgs {
    int T, H, E;
    const uint16_t* x;
    const uint16_t* w_router;
    const float* logits_in;
    const float* bias;
    int64_t bias_stride;
    int32_t* topk_idx;
    float* topk_w;
    int32_t* counts;
    float* logits_ws;   // [T, E] scratch
    uint32_t* ticket;   // last-block ticket of the small-T router (workspace header, zero between calls)
    int32_t* err;
};

struct PermuteArgs {
    int T, E;
    const int32_t* topk_idx;
    const int32_t* counts;
    int32_t* offsets;
    int32_t* row_to_pair;
    int32_t* pair_to_row;
    uint8_t* scratch;   // permute_ws_bytes(T, E, K)
    int32_t* err;
};

struct FfnArgs {
    int T, H, I, E, K, G, has_shared, mode;
    const uint16_t* x;
    const uint32_t* gu_codes;
    const uint16_t* gu_sb;
    const uint32_t* d_codes;
    const uint16_t* d_sb;
    const int32_t* offsets;
    const int32_t* row_to_pair;
    const float* topk_w;
    uint16_t* h;          // [(K+1) T, I] bf16 scratch: routed rows, then shared rows
    uint16_t* xg;         // [(K+1) T, H] bf16 scratch: x rows in the same row order (tensor-core path)
    float* y_acc;         // scatter mode
    uint16_t* y_rows;     // pairs mode
    uint16_t* y_shared;   // pairs mode
    int32_t* err;
};

struct CombineArgs {
    int T, H, has_shared, mode;
    const float* y_acc;
    const uint16_t* rows;
    const uint16_t* shared;
    const int32_t* pair_to_row;
    const float* w;
    uint16_t* y;
    int32_t* err;
};

// Rows [row_begin, row_begin + n_rows) of the permutation, gathered for an
// expert-parallel dispatch.
struct GatherArgs {
    int T, H, K, row_begin, n_rows;
    const uint16_t* x;
    const int32_t* row_to_pair;
    const float* topk_w;
    uint16_t* rows_out;
    float* w_out;
    int32_t* err;
};

cudaError_t launch_gather_dispatch(const GatherArgs& a, cudaStream_t st);

// Gated DeltaNet recurrent scan (gdn_scan in the C ABI).
struct GdnArgs {
    int B, T, Hk, Hv, dk, dv;
    const uint16_t* q;        // [B, T, Hk, dk] bf16
    const uint16_t* k;        // [B, T, Hk, dk] bf16
    const uint16_t* v;        // [B, T, Hv, dv] bf16
    const float* g;           // [B, T, Hv] log of the decay
    const float* beta;        // [B, T, Hv]
    float scale;
    const float* state_in;    // [B, Hv, dv, dk]
    float* state_out;         // [B, Hv, dv, dk] (may equal state_in)
    uint16_t* o;              // [B, T, Hv, dv] bf16
};

bool gdn_scan_supported(const GdnArgs& a);
cudaError_t launch_gdn_scan(const GdnArgs& a, cudaStream_t st);
cudaError_t launch_router(const RouterArgs& a, cudaStream_t st);
// The logits alone (+ bias) into a.logits_ws; zeroes a.counts when non-null.
cudaError_t launch_router_logits(const RouterArgs& a, cudaStream_t st);
size_t permute_ws_bytes(int T, int E, int K);
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t st);
cudaError_t launch_ffn_simt(const FfnArgs& a, cudaStream_t st);
// Experts of 1..skip_rows rows get no tiles (0: every expert is computed).
cudaError_t launch_ffn_tc(const FfnArgs& a, int skip_rows, cudaStream_t st);

// Workspace sections of the decode kernels (T <= 8): the launch counter in
// the workspace header and the tagged router logits (several copies).
struct DecodeWs {
    unsigned long long* launches;
    unsigned long long* tlogits;
};
size_t decode_ws_bytes(int T, int E, int I);
DecodeWs decode_ws_carve(uint8_t* base, int T, int E, int I, unsigned long long* launches);

// Expert FFNs for T <= 8 (scatter mode): one launch, y_acc overwritten.
bool ffn_decode_supported(const FfnArgs& a);
cudaError_t launch_ffn_decode(const FfnArgs& a, const DecodeWs& w, cudaStream_t st);

// The experts of 1..8 rows of a launch of any T (scatter mode), one unit per
// (expert, 32 columns of I) as in the decode kernel, each MMA column a row of
// the expert: x rows from xg (the gathered rows the tensor-core path reads),
// w * y added into y_acc as it stands (the tensor-core launch with skip_rows 8
// clears it and adds the other experts).
bool ffn_rows_supported(const FfnArgs& a);
cudaError_t launch_ffn_rows(const FfnArgs& a, cudaStream_t st);

// The decode layer's router logits, top-k, permutation and expert FFNs in one
// kernel (the routing outputs written as the route and permute calls would,
// y_acc as the FFN call would), then the combine.
struct DecodeRoute {
    const uint16_t* w_router;
    const float* bias;
    int64_t bias_stride;
    int32_t* topk_idx;
    float* topk_w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* row_to_pair;
    int32_t* pair_to_row;
};
bool decode_layer_supported(const FfnArgs& a);
cudaError_t launch_decode_layer(const FfnArgs& a, const DecodeRoute& r, const DecodeWs& w, cudaStream_t st);
bool ffn_tc_supported(const FfnArgs& a);
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st);

}  // namespace moe
