// C ABI of moe_b200: argument validation, workspace carving and kernel
// launches on the caller's stream.  See include/moe_b200.h for the contract.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "api_range.h"

using namespace moe;

namespace {

constexpr int kMaxTokens = 65536;

// Any expert count up to 256 and k up to 8: an expert-parallel rank runs the
// expert FFN over its own shard of the experts, with each dispatched row as
// one pair (k = 1).  The router and the permutation stay at 256 experts, top 8.
bool config_ok(const moe_config_t* c) {
    return c && c->hidden >= 256 && c->hidden % 256 == 0 && c->hidden <= 16384 && c->inter >= 128 &&
           c->inter % 128 == 0 && c->inter <= 8192 && c->num_experts >= 1 && c->num_experts <= 256 &&
           c->top_k >= 1 && c->top_k <= 8 && c->top_k <= c->num_experts && c->group_size == 64 &&
           (c->has_shared == 0 || c->has_shared == 1);
}

bool routing_shape_ok(const moe_config_t* c) { return c->num_experts == 256 && c->top_k == 8; }

struct WsLayout {
    size_t logits, perm, h, xg, dec, total;
};

WsLayout layout(const moe_config_t* c, int T) {
    WsLayout L;
    size_t off = sizeof(WsHeader);
    L.logits = off;
    off += align256((size_t)T * c->num_experts * sizeof(float));
    L.perm = off;
    off += permute_ws_bytes(T, c->num_experts, c->top_k);
    L.h = off;
    off += align256((size_t)(c->top_k + 1) * T * c->inter * sizeof(uint16_t));
    L.xg = off;
    off += align256((size_t)(c->top_k + 1) * T * c->hidden * sizeof(uint16_t));
    L.dec = off;
    off += decode_ws_bytes(T, c->num_experts, c->inter);
    L.total = off;
    return L;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int32_t check_common(const moe_config_t* cfg, int32_t T, const void* ws, size_t ws_bytes) {
    if (!cfg) return MOE_ERR_INVALID_ARG;
    if (!config_ok(cfg)) return MOE_ERR_UNSUPPORTED;
    if (T < 1) return MOE_ERR_INVALID_ARG;
    if (T > kMaxTokens) return MOE_ERR_UNSUPPORTED;
    if (ws) {
        if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
        if (ws_bytes < layout(cfg, T).total) return MOE_ERR_WORKSPACE;
    }
    return MOE_OK;
}

int32_t* err_word(void* ws) { return reinterpret_cast<int32_t*>(ws); }

int32_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// The decode kernel's row-list launch takes the experts of at most 8 rows off
// the tensor-core kernel.  Measured on one B200 (expert FFN, L2 flushed): at
// H 2048 / I 512, T = 16 119 -> 107 us and T = 300 273 -> 261 us, but the
// Zipf-skewed T = 512 layer 168 -> 175 us (its time is in the experts of many
// rows) and T = 33 at H 512 42 -> 46 us (units too small to amortise the
// per-unit handoffs).  So: the largest hidden size, at most 12 rows per expert
// on average.
bool split_small_experts(const FfnArgs& a) {
    return a.H >= 2048 && ffn_rows_supported(a) && (int64_t)a.T * a.K <= (int64_t)12 * a.E;
}

// Implementation chosen for MOE_PATH_AUTO: the memory-bound decode kernel for
// a handful of tokens, else the tensor-core kernel where its shape rules
// hold, else the CUDA-core path.
int32_t resolve_path(const FfnArgs& a) {
    if (ffn_decode_supported(a)) return MOE_PATH_GEMV;
    if (ffn_tc_supported(a)) return split_small_experts(a) ? MOE_PATH_TC_GEMV : MOE_PATH_TC;
    return MOE_PATH_SIMT;
}

DecodeWs decode_ws(void* ws, const moe_config_t* cfg, int32_t T) {
    return decode_ws_carve(static_cast<uint8_t*>(ws) + layout(cfg, T).dec, T, cfg->num_experts, cfg->inter,
                           &reinterpret_cast<WsHeader*>(ws)->decode_launches);
}

FfnArgs shape_only(const moe_config_t* cfg, int32_t T) {
    FfnArgs a = {};
    a.T = T;
    a.H = cfg->hidden;
    a.I = cfg->inter;
    a.E = cfg->num_experts;
    a.K = cfg->top_k;
    a.G = cfg->group_size;
    a.has_shared = cfg->has_shared;
    return a;
}

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_config_t* cfg, int32_t max_tokens) {
    if (!config_ok(cfg) || max_tokens < 1 || max_tokens > kMaxTokens) return 0;
    return layout(cfg, max_tokens).total;
}

int32_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    moe::ApiRange api_range("moe_workspace_init");
    if (!ws || ws_bytes < sizeof(WsHeader) || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
    // all of it: the decode kernels' tagged words must not match a restarted launch count
    return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

int32_t moe_route(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint16_t* w_router,
                  const float* logits_in, const float* logit_bias, int64_t logit_bias_row_stride,
                  int32_t* topk_idx, float* topk_w, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
    moe::ApiRange api_range("moe_route");
    if (!ws) return MOE_ERR_WORKSPACE;
    int32_t st = check_common(cfg, T, ws, ws_bytes);
    if (st) return st;
    if (!routing_shape_ok(cfg)) return MOE_ERR_UNSUPPORTED;
    if (!topk_idx || !topk_w || !counts) return MOE_ERR_INVALID_ARG;
    if (!logits_in && (!x || !w_router)) return MOE_ERR_INVALID_ARG;
    if (logit_bias_row_stride < 0) return MOE_ERR_INVALID_ARG;
    if ((x && !aligned(x, 16)) || (w_router && !aligned(w_router, 16)) || !aligned(logits_in, 4) ||
        !aligned(logit_bias, 4) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) || !aligned(counts, 4))
        return MOE_ERR_INVALID_ARG;
    RouterArgs a;
    a.T = T;
    a.H = cfg->hidden;
    a.E = cfg->num_experts;
    a.x = x;
    a.w_router = w_router;
    a.logits_in = logits_in;
    a.bias = logit_bias;
    a.bias_stride = logit_bias_row_stride;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.counts = counts;
    a.logits_ws = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + layout(cfg, T).logits);
    a.ticket = &reinterpret_cast<WsHeader*>(ws)->route_ticket;
    a.err = err_word(ws);
    return cuda_status(launch_router(a, (cudaStream_t)stream));
}

int32_t moe_router_logits(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint16_t* w_router,
                          const float* logit_bias, int64_t logit_bias_row_stride, float* logits, void* ws,
                          size_t ws_bytes, void* stream) {
    moe::ApiRange api_range("moe_router_logits");
    if (!ws) return MOE_ERR_WORKSPACE;
    int32_t st = check_common(cfg, T, ws, ws_bytes);
    if (st) return st;
    if (!routing_shape_ok(cfg)) return MOE_ERR_UNSUPPORTED;
    if (!x || !w_router || !logits) return MOE_ERR_INVALID_ARG;
    if (logit_bias_row_stride < 0) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(logit_bias, 4) || !aligned(logits, 8))
        return MOE_ERR_INVALID_ARG;
    RouterArgs a = {};
    a.T = T;
    a.H = cfg->hidden;
    a.E = cfg->num_experts;
    a.x = x;
    a.w_router = w_router;
    a.bias = logit_bias;
    a.bias_stride = logit_bias_row_stride;
    a.logits_ws = logits;
    a.err = err_word(ws);
    return cuda_status(launch_router_logits(a, (cudaStream_t)stream));
}

int32_t moe_permute(const moe_config_t* cfg, int32_t T, const int32_t* topk_idx, const int32_t* counts,
                    int32_t* offsets, int32_t* row_to_pair, int32_t* pair_to_row, void* ws, size_t ws_bytes,
                    void* stream) {
    moe::ApiRange api_range("moe_permute");
    if (!ws) return MOE_ERR_WORKSPACE;
    int32_t st = check_common(cfg, T, ws, ws_bytes);
    if (st) return st;
    if (!routing_shape_ok(cfg)) return MOE_ERR_UNSUPPORTED;
    if (!topk_idx || !offsets || !row_to_pair || !pair_to_row) return MOE_ERR_INVALID_ARG;
    if (!aligned(topk_idx, 4) || !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(row_to_pair, 4) ||
        !aligned(pair_to_row, 4))
        return MOE_ERR_INVALID_ARG;
    PermuteArgs a;
    a.T = T;
    a.E = cfg->num_experts;
    a.topk_idx = topk_idx;
    a.counts = counts;
    a.offsets = offsets;
    a.row_to_pair = row_to_pair;
    a.pair_to_row = pair_to_row;
    a.scratch = static_cast<uint8_t*>(ws) + layout(cfg, T).perm;
    a.err = err_word(ws);
    return cuda_status(launch_permute(a, (cudaStream_t)stream));
}

int32_t moe_expert_ffn_path(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint32_t* gu_codes,
                            const uint16_t* gu_sb, const uint32_t* d_codes, const uint16_t* d_sb,
                            const int32_t* offsets, const int32_t* row_to_pair, const float* topk_w,
                            int32_t mode, void* out0, void* out1, void* ws, size_t ws_bytes, int32_t path,
                            void* stream) {
    moe::ApiRange api_range("moe_expert_ffn_path");
    if (!ws) return MOE_ERR_WORKSPACE;
    int32_t st = check_common(cfg, T, ws, ws_bytes);
    if (st) return st;
    if (mode != MOE_MODE_SCATTER && mode != MOE_MODE_PAIRS) return MOE_ERR_INVALID_ARG;
    if (!x || !gu_codes || !gu_sb || !d_codes || !d_sb || !offsets || !row_to_pair || !topk_w || !out0)
        return MOE_ERR_INVALID_ARG;
    if (mode == MOE_MODE_PAIRS && cfg->has_shared && !out1) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(gu_codes, 256) || !aligned(gu_sb, 256) || !aligned(d_codes, 256) ||
        !aligned(d_sb, 256) || !aligned(out0, 16) || !aligned(out1, 16) || !aligned(offsets, 4) ||
        !aligned(row_to_pair, 4) || !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    FfnArgs a;
    a.T = T;
    a.H = cfg->hidden;
    a.I = cfg->inter;
    a.E = cfg->num_experts;
    a.K = cfg->top_k;
    a.G = cfg->group_size;
    a.has_shared = cfg->has_shared;
    a.mode = mode;
    a.x = x;
    a.gu_codes = gu_codes;
    a.gu_sb = gu_sb;
    a.d_codes = d_codes;
    a.d_sb = d_sb;
    a.offsets = offsets;
    a.row_to_pair = row_to_pair;
    a.topk_w = topk_w;
    a.h = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + layout(cfg, T).h);
    a.xg = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + layout(cfg, T).xg);
    a.y_acc = mode == MOE_MODE_SCATTER ? static_cast<float*>(out0) : nullptr;
    a.y_rows = mode == MOE_MODE_PAIRS ? static_cast<uint16_t*>(out0) : nullptr;
    a.y_shared = mode == MOE_MODE_PAIRS ? static_cast<uint16_t*>(out1) : nullptr;
    a.err = err_word(ws);
    cudaStream_t s = (cudaStream_t)stream;
    if (path == MOE_PATH_AUTO) path = resolve_path(a);
    switch (path) {
        case MOE_PATH_SIMT:
            if (mode == MOE_MODE_SCATTER) {
                cudaError_t ce = cudaMemsetAsync(a.y_acc, 0, sizeof(float) * (size_t)T * a.H, s);
                if (ce != cudaSuccess) return MOE_ERR_CUDA;
            }
            return cuda_status(launch_ffn_simt(a, s));
        case MOE_PATH_GEMV:
            if (!ffn_decode_supported(a)) return MOE_ERR_UNSUPPORTED;
            return cuda_status(launch_ffn_decode(a, decode_ws(ws, cfg, T), s));
        case MOE_PATH_TC:
            if (!ffn_tc_supported(a)) return MOE_ERR_UNSUPPORTED;
            return cuda_status(launch_ffn_tc(a, 0, s));
        case MOE_PATH_TC_GEMV: {
            if (!ffn_tc_supported(a) || !ffn_rows_supported(a)) return MOE_ERR_UNSUPPORTED;
            const int32_t st = cuda_status(launch_ffn_tc(a, 8, s));
            return st != MOE_OK ? st : cuda_status(launch_ffn_rows(a, s));
        }
        default:
            return MOE_ERR_UNSUPPORTED;
    }
}

int32_t moe_expert_ffn(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint32_t* gu_codes,
                       const uint16_t* gu_sb, const uint32_t* d_codes, const uint16_t* d_sb, const int32_t* offsets,
                       const int32_t* row_to_pair, const float* topk_w, int32_t mode, void* out0, void* out1,
                       void* ws, size_t ws_bytes, void* stream) {
    return moe_expert_ffn_path(cfg, T, x, gu_codes, gu_sb, d_codes, d_sb, offsets, row_to_pair, topk_w, mode, out0,
                               out1, ws, ws_bytes, MOE_PATH_AUTO, stream);
}

int32_t moe_combine(const moe_config_t* cfg, int32_t T, int32_t mode, const void* in0, const void* in1,
                    const int32_t* pair_to_row, const float* topk_w, uint16_t* y, void* stream) {
    moe::ApiRange api_range("moe_combine");
    int32_t st = check_common(cfg, T, nullptr, 0);
    if (st) return st;
    if (mode != MOE_MODE_SCATTER && mode != MOE_MODE_PAIRS) return MOE_ERR_INVALID_ARG;
    if (!in0 || !y) return MOE_ERR_INVALID_ARG;
    if (mode == MOE_MODE_PAIRS && (!pair_to_row || !topk_w || (cfg->has_shared && !in1)))
        return MOE_ERR_INVALID_ARG;
    if (mode == MOE_MODE_PAIRS && cfg->top_k != 8) return MOE_ERR_UNSUPPORTED;
    if (!aligned(in0, 16) || !aligned(in1, 16) || !aligned(y, 16) || !aligned(pair_to_row, 4) ||
        !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    CombineArgs a;
    a.T = T;
    a.H = cfg->hidden;
    a.has_shared = cfg->has_shared;
    a.mode = mode;
    a.y_acc = static_cast<const float*>(in0);
    a.rows = static_cast<const uint16_t*>(in0);
    a.shared = static_cast<const uint16_t*>(in1);
    a.pair_to_row = pair_to_row;
    a.w = topk_w;
    a.y = y;
    a.err = nullptr;   // no workspace here: out-of-range rows are clamped, the permute already reported them
    return cuda_status(launch_combine(a, (cudaStream_t)stream));
}

int32_t moe_gather_rows(const moe_config_t* cfg, int32_t T, const uint16_t* x, const int32_t* row_to_pair,
                        const float* topk_w, int32_t row_begin, int32_t n_rows, uint16_t* rows_out, float* w_out,
                        void* ws, size_t ws_bytes, void* stream) {
    moe::ApiRange api_range("moe_gather_rows");
    if (!ws) return MOE_ERR_WORKSPACE;
    int32_t st = check_common(cfg, T, ws, ws_bytes);
    if (st) return st;
    if (row_begin < 0 || n_rows < 0 || (int64_t)row_begin + n_rows > (int64_t)T * cfg->top_k)
        return MOE_ERR_INVALID_ARG;
    if (n_rows == 0) return MOE_OK;
    if (!x || !row_to_pair || !rows_out) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(rows_out, 16) || !aligned(row_to_pair, 4) || !aligned(topk_w, 4) ||
        !aligned(w_out, 4))
        return MOE_ERR_INVALID_ARG;
    GatherArgs a;
    a.T = T;
    a.H = cfg->hidden;
    a.K = cfg->top_k;
    a.row_begin = row_begin;
    a.n_rows = n_rows;
    a.x = x;
    a.row_to_pair = row_to_pair;
    a.topk_w = topk_w;
    a.rows_out = rows_out;
    a.w_out = w_out;
    a.err = err_word(ws);
    return cuda_status(launch_gather_dispatch(a, (cudaStream_t)stream));
}

int32_t moe_get_device_error(const void* ws, void* stream) {
    if (!ws) return MOE_ERR_WORKSPACE;
    int32_t v = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    return v;
}

int32_t moe_decode_layer(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint16_t* w_router,
                         const float* logit_bias, int64_t logit_bias_row_stride, const uint32_t* gu_codes,
                         const uint16_t* gu_sb, const uint32_t* d_codes, const uint16_t* d_sb, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* offsets, int32_t* row_to_pair,
                         int32_t* pair_to_row, float* y_acc, uint16_t* y, void* ws, size_t ws_bytes,
                         void* stream) {
    moe::ApiRange api_range("moe_decode_layer");
    if (!ws) return MOE_ERR_WORKSPACE;
    int32_t st = check_common(cfg, T, ws, ws_bytes);
    if (st) return st;
    if (!routing_shape_ok(cfg)) return MOE_ERR_UNSUPPORTED;
    if (!x || !w_router || !gu_codes || !gu_sb || !d_codes || !d_sb || !topk_idx || !topk_w || !counts ||
        !offsets || !row_to_pair || !pair_to_row || !y_acc || !y)
        return MOE_ERR_INVALID_ARG;
    if (logit_bias_row_stride < 0) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(logit_bias, 4) || !aligned(gu_codes, 256) ||
        !aligned(gu_sb, 256) || !aligned(d_codes, 256) || !aligned(d_sb, 256) || !aligned(topk_idx, 4) ||
        !aligned(topk_w, 4) || !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(row_to_pair, 4) ||
        !aligned(pair_to_row, 4) || !aligned(y_acc, 16) || !aligned(y, 16))
        return MOE_ERR_INVALID_ARG;
    FfnArgs a = shape_only(cfg, T);
    a.mode = MOE_MODE_SCATTER;
    if (!decode_layer_supported(a)) return MOE_ERR_UNSUPPORTED;
    a.x = x;
    a.gu_codes = gu_codes;
    a.gu_sb = gu_sb;
    a.d_codes = d_codes;
    a.d_sb = d_sb;
    a.y_acc = y_acc;
    a.err = err_word(ws);
    DecodeRoute r;
    r.w_router = w_router;
    r.bias = logit_bias;
    r.bias_stride = logit_bias_row_stride;
    r.topk_idx = topk_idx;
    r.topk_w = topk_w;
    r.counts = counts;
    r.offsets = offsets;
    r.row_to_pair = row_to_pair;
    r.pair_to_row = pair_to_row;
    cudaStream_t s = (cudaStream_t)stream;
    st = cuda_status(launch_decode_layer(a, r, decode_ws(ws, cfg, T), s));
    if (st) return st;
    CombineArgs c = {};
    c.T = T;
    c.H = cfg->hidden;
    c.has_shared = cfg->has_shared;
    c.mode = MOE_MODE_SCATTER;
    c.y_acc = y_acc;
    c.y = y;
    c.err = err_word(ws);
    return cuda_status(launch_combine(c, s));
}

int32_t moe_launch_count(const moe_config_t* cfg, int32_t T, int32_t mode, int32_t path) {
    if (!config_ok(cfg) || T < 1 || T > kMaxTokens) return -1;
    if (mode != MOE_MODE_SCATTER && mode != MOE_MODE_PAIRS) return -1;
    const int route = T <= 8 ? 1 : 2;
    const int permute = T <= 256 ? 1 : 3;
    FfnArgs a = shape_only(cfg, T);
    a.mode = mode;
    if (path == MOE_PATH_AUTO) path = resolve_path(a);
    int ffn;
    switch (path) {
        case MOE_PATH_SIMT: ffn = 2; break;
        case MOE_PATH_GEMV: if (!ffn_decode_supported(a)) return -1; ffn = 1; break;
        case MOE_PATH_TC: if (!ffn_tc_supported(a)) return -1; ffn = 3; break;
        case MOE_PATH_TC_GEMV: if (!ffn_tc_supported(a) || !ffn_rows_supported(a)) return -1; ffn = 4; break;
        default: return -1;
    }
    return route + permute + ffn + 1;
}

const char* moe_status_string(int32_t s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_NONFINITE: return "MOE_ERR_NONFINITE";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
        case MOE_ERR_BOUNDS: return "MOE_ERR_BOUNDS";
        default: return "MOE_ERR_UNKNOWN";
    }
}

}  // extern "C"
