/*
 * moe_b200: one mixture-of-experts layer with groupwise-affine 4-bit expert
 * weights, for NVIDIA B200 (sm_100a).  C ABI.
 *
 * The layer (the Lily pages: "Perplexity's Lily brings fast local AI to Apple
 * silicon Macs", sections "A 35B Model Built for Local Memory" and "Where the
 * Engine Gains Speed"; "Perplexity built an inference engine for one model,
 * one chip", second and third paragraphs):
 *   a router scores E = 256 experts per token, keeps the top k = 8 and
 *   renormalises their softmax weights; one shared expert sees every token;
 *   every expert is a SwiGLU FFN whose weights are 4-bit codes with a bf16
 *   (scale, bias) per group of G = 64 inputs, reconstructed inside the
 *   expert GEMM tile by tile; the outputs are combined with the routing
 *   weights.  Routing never returns to the host.
 *
 * The layer is four calls on one CUDA stream:
 *   moe_route -> moe_permute -> moe_expert_ffn -> moe_combine.
 *
 * Conventions for every call:
 *  - All pointers are DEVICE pointers unless stated otherwise; the caller
 *    owns every buffer.  The library allocates nothing, frees nothing and
 *    keeps no global state.  Tensors are row-major and contiguous.  bf16
 *    values travel as uint16_t bit patterns.
 *  - Alignment: every pointer 16-byte aligned; the packed weight arrays
 *    (codes and scale/bias) and the workspace 256-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    are asynchronous and never synchronise the host, except
 *    moe_get_device_error.
 *  - Host-side problems (null pointer, unsupported shape, small workspace)
 *    return an error before anything is launched.  Device-side problems
 *    (non-finite logit, routing index out of range, an expired bounded
 *    wait) set a sticky error word in the workspace and the kernels carry
 *    on with safe values; moe_get_device_error reads it.
 *  - Concurrent calls must use distinct workspaces.
 *  - The decode kernels (moe_decode_layer, and moe_expert_ffn for T <= 8 on
 *    the automatic or GEMV path) run one CTA per SM, read words that other
 *    CTAs of the same launch write, and are launched as cooperative grids:
 *    the launch fails (MOE_ERR_CUDA) rather than starting when the CTAs
 *    cannot all be resident.  Issue decode calls of concurrent layers on
 *    one stream (or order their streams with events).
 *
 * Supported shapes: hidden % 256 == 0, inter % 128 == 0, group_size == 64,
 * has_shared in {0, 1}, 1 <= T <= 65536.  The router, the permutation and
 * moe_decode_layer need num_experts == 256 and top_k == 8.  moe_expert_ffn,
 * moe_gather_rows and the scatter combine also take any 1 <= num_experts <=
 * 256 and 1 <= top_k <= min(8, num_experts): an expert-parallel rank runs
 * its shard of the experts over dispatched rows with top_k == 1.  Anything
 * else returns MOE_ERR_UNSUPPORTED.
 *
 * Packed weights of an [N, K] matrix (N outputs, K inputs), matrices of all
 * experts stacked, shared expert last (index num_experts):
 *   codes [n_mat][N][K/8] uint32: nibble j (bits 4j..4j+3) of word m holds the
 *         unsigned code q of input 8m + j;
 *   sb    [n_mat][N][K/G][2] bf16: (scale, bias) of the group of G inputs;
 *   weight(n, k) = scale * q + bias.
 * gate_up matrices are [2I, H] (gate rows 0..I-1, up rows I..2I-1); down
 * matrices are [H, I].
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, T < 1, bad mode */
    MOE_ERR_UNSUPPORTED = 2, /* shape outside the supported set */
    MOE_ERR_WORKSPACE = 3,   /* workspace too small or misaligned */
    MOE_ERR_CUDA = 4,        /* a CUDA runtime call failed */
    MOE_ERR_NONFINITE = 5,   /* device: NaN or Inf among a token's logits */
    MOE_ERR_TIMEOUT = 6,     /* device: a bounded wait expired */
    MOE_ERR_BOUNDS = 7       /* device: routing index out of range or repeated */
} moe_status_t;

typedef struct {
    int32_t hidden;      /* H */
    int32_t inter;       /* I, expert intermediate size */
    int32_t num_experts; /* E routed experts */
    int32_t top_k;       /* k */
    int32_t group_size;  /* G inputs per (scale, bias) pair */
    int32_t has_shared;  /* 1: matrix index E is the always-on shared expert */
} moe_config_t;

/* Output modes of moe_expert_ffn / moe_combine. */
#define MOE_MODE_SCATTER 0 /* out0 = y_acc fp32 [T, H]: weighted sum accumulated in place */
#define MOE_MODE_PAIRS 1   /* out0 = y_rows bf16 [T*k, H] per routed row, out1 = y_shared bf16 [T, H] */

/* Expert-FFN implementations for moe_expert_ffn_path (0 chooses by shape). */
#define MOE_PATH_AUTO 0
#define MOE_PATH_SIMT 1    /* CUDA-core dequant + dot products, any T */
#define MOE_PATH_GEMV 2    /* memory-bound split-K GEMV, few rows per expert */
#define MOE_PATH_TC 3      /* TMA; dequant in registers into tensor memory (A); tcgen05 MMA */
#define MOE_PATH_TC_GEMV 4 /* scatter mode: MOE_PATH_TC for experts of more than 8 rows, then
                             the split-K GEMV kernel over the rows of the others (T unrestricted);
                             MOE_PATH_AUTO takes it when hidden >= 2048 and
                             T * top_k <= 12 * num_experts */

/* Bytes of workspace that the calls need for up to max_tokens tokens; 0 if
 * the configuration is unsupported.  Caller allocates it (256-byte aligned)
 * and zero-fills it once, or calls moe_workspace_init. */
size_t moe_workspace_size(const moe_config_t* cfg, int32_t max_tokens);

/* Zero-fills all ws_bytes of the workspace (async on stream): the sticky
 * error word, the decode kernels' launch counter and their tagged words. */
int32_t moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * Router (the pages: "a router picks eight subnetworks out of 256"; "GPU-
 * resident expert routing").
 *   x          bf16 [T, H] activations.
 *   w_router   bf16 [E, H] router weights.
 *   logits_in  nullable fp32 [T, E]: when given, used instead of x . w_router^T
 *              (x and w_router may then be NULL).
 *   logit_bias nullable fp32, row t at logit_bias + t * logit_bias_row_stride
 *              (stride 0: one [E] row for every token); added once.
 * Logits are fp32 in a fixed order (the contract order): slice s in 0..31
 * owns the 8-input chunks c = s, s+32, ...; acc[s] = fma(x, w, acc[s]) over
 * its chunks in order, inputs ascending within a chunk; then an xor
 * butterfly over the slices (offsets 16, 8, 4, 2, 1); then + bias.
 * Outputs:
 *   topk_idx  int32 [T, k]: the k largest logits, ordered by (logit desc,
 *             expert asc); -0.0 == +0.0.
 *   topk_w    fp32  [T, k]: softmax of the selected logits (== the 256-way
 *             softmax restricted to them and renormalised).
 *   counts    int32 [E]: tokens routed to each expert.
 * A token with a non-finite logit sets MOE_ERR_NONFINITE and is routed to
 * experts 0..k-1 with weight 1/k.
 */
int32_t moe_route(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint16_t* w_router,
                  const float* logits_in, const float* logit_bias, int64_t logit_bias_row_stride,
                  int32_t* topk_idx, float* topk_w, int32_t* counts, void* ws, size_t ws_bytes,
                  void* stream);

/*
 * The router logits alone: logits fp32 [T, E] (device, caller-owned, 8-byte
 * aligned) = x . w_router^T in the contract order above, + logit_bias when
 * given; the same values moe_route selects from.  x, w_router, logit_bias and
 * the stride as for moe_route; the workspace carries the error word (a
 * bounded wait that expires sets MOE_ERR_TIMEOUT there).  Returns
 * MOE_ERR_INVALID_ARG for a null or misaligned pointer or a negative stride,
 * else as moe_route.
 */
int32_t moe_router_logits(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint16_t* w_router,
                          const float* logit_bias, int64_t logit_bias_row_stride, float* logits, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * Token permutation: stable expert-major order of the T*k (token, slot)
 * pairs, pair p = t*k + slot.
 *   counts      nullable int32 [E] from moe_route; when given it is checked
 *               against topk_idx (mismatch sets MOE_ERR_BOUNDS).
 *   offsets     int32 [E+1]: exclusive scan of the counts, offsets[E] = T*k.
 *   row_to_pair int32 [T*k]: rows offsets[e]..offsets[e+1]-1 hold expert e's
 *               pairs in increasing token order.
 *   pair_to_row int32 [T*k]: inverse of row_to_pair.
 * An index outside 0..E-1 or an expert repeated within a token sets
 * MOE_ERR_BOUNDS.
 */
int32_t moe_permute(const moe_config_t* cfg, int32_t T, const int32_t* topk_idx, const int32_t* counts,
                    int32_t* offsets, int32_t* row_to_pair, int32_t* pair_to_row, void* ws,
                    size_t ws_bytes, void* stream);

/*
 * Expert FFNs (the pages: "reconstructs weights inside the grouped GEMM, one
 * tile at a time"; "one shared expert sees everything"): for every row r of
 * expert e with token t,
 *   h = silu(x_t . Wg_e^T) * (x_t . Wu_e^T)  (h rounded to bf16),
 *   y_r = h . Wd_e^T,
 * plus the shared expert on every token when cfg->has_shared.  Weights are
 * dequantised to bf16 on chip; accumulation is fp32.
 *   gu_codes/gu_sb  packed gate_up matrices, E (+1 shared) of [2I, H].
 *   d_codes/d_sb    packed down matrices, E (+1 shared) of [H, I].
 *   offsets, row_to_pair from moe_permute; topk_w from moe_route.
 *   mode MOE_MODE_SCATTER: out0 = y_acc fp32 [T, H] is overwritten with
 *        sum_slot w * y_row (+ y_shared); out1 unused.
 *   mode MOE_MODE_PAIRS: out0 = bf16 [T*k, H] row outputs (row order),
 *        out1 = bf16 [T, H] shared-expert outputs (unused without shared).
 */
int32_t moe_expert_ffn(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint32_t* gu_codes,
                       const uint16_t* gu_sb, const uint32_t* d_codes, const uint16_t* d_sb,
                       const int32_t* offsets, const int32_t* row_to_pair, const float* topk_w,
                       int32_t mode, void* out0, void* out1, void* ws, size_t ws_bytes, void* stream);

/* moe_expert_ffn with an explicit implementation (MOE_PATH_*). */
int32_t moe_expert_ffn_path(const moe_config_t* cfg, int32_t T, const uint16_t* x,
                            const uint32_t* gu_codes, const uint16_t* gu_sb, const uint32_t* d_codes,
                            const uint16_t* d_sb, const int32_t* offsets, const int32_t* row_to_pair,
                            const float* topk_w, int32_t mode, void* out0, void* out1, void* ws,
                            size_t ws_bytes, int32_t path, void* stream);

/*
 * Combine into the layer output y bf16 [T, H].
 *   MOE_MODE_SCATTER: in0 = y_acc fp32 [T, H]; y = bf16(y_acc).
 *   MOE_MODE_PAIRS:   in0 = row outputs bf16 [T*k, H], in1 = shared outputs
 *                     bf16 [T, H] (ignored without shared);
 *                     y[t] = bf16(sum_slot w[t,slot] * in0[pair_to_row[t*k+slot]]
 *                                 + in1[t]), summed in fp32 in slot order.
 */
int32_t moe_combine(const moe_config_t* cfg, int32_t T, int32_t mode, const void* in0, const void* in1,
                    const int32_t* pair_to_row, const float* topk_w, uint16_t* y, void* stream);

/*
 * moe_decode_layer: the whole layer for a handful of tokens in two launches
 * (decode-step integration).  Computes exactly what moe_route (x, w_router,
 * optional logit bias; logits computed by the router, not given) ->
 * moe_permute -> moe_expert_ffn (MOE_MODE_SCATTER) -> moe_combine compute,
 * and writes every intermediate those calls write: topk_idx, topk_w, counts,
 * offsets, row_to_pair, pair_to_row, y_acc fp32 [T, H] and y bf16 [T, H].
 * Lily pages: "Perplexity built an inference engine for one model, one
 * chip", third paragraph (the routing decision stays on the GPU with the
 * expert work; the decode step as few kernels as possible).
 * The first kernel computes the router logits over all CTAs and publishes
 * each tagged with the launch's number; every CTA polls (bounded) until it
 * holds all of a token's logits, selects the top-k, builds the list of
 * active experts and runs its share of the decode expert FFN, and the last
 * CTA writes the routing outputs; the second kernel converts y_acc.
 * Supported: 1 <= T <= 8, hidden 512, 1024 or 2048, E == 256, k == 8;
 * otherwise MOE_ERR_UNSUPPORTED before any launch (use the four calls).
 * Same pointer rules as the four calls; the workspace must hold T tokens.
 */
int32_t moe_decode_layer(const moe_config_t* cfg, int32_t T, const uint16_t* x, const uint16_t* w_router,
                         const float* logit_bias, int64_t logit_bias_row_stride, const uint32_t* gu_codes,
                         const uint16_t* gu_sb, const uint32_t* d_codes, const uint16_t* d_sb, int32_t* topk_idx,
                         float* topk_w, int32_t* counts, int32_t* offsets, int32_t* row_to_pair,
                         int32_t* pair_to_row, float* y_acc, uint16_t* y, void* ws, size_t ws_bytes,
                         void* stream);

/*
 * moe_gather_rows: the dispatch step of expert parallelism.  A rank holding
 * the experts [e0, e1) receives from every rank the permuted rows
 * offsets[e0] .. offsets[e1]-1 of that rank's permutation; this call copies
 * such a block out of the activations, in row order.
 *   x            bf16 [T, H] activations; row_to_pair int32 [T*k] from
 *                moe_permute; topk_w nullable fp32 [T*k] from moe_route.
 *   row_begin, n_rows  the block [row_begin, row_begin + n_rows) of rows,
 *                inside [0, T*k) (else MOE_ERR_INVALID_ARG); n_rows 0 does
 *                nothing.
 *   rows_out     bf16 [n_rows, H]: rows_out[i] = x[row_to_pair[row_begin+i] / k].
 *   w_out        nullable fp32 [n_rows]: w_out[i] = topk_w[row_to_pair[row_begin+i]]
 *                (0 when topk_w is NULL).
 * A pair index outside [0, T*k) zero-fills its row and sets MOE_ERR_BOUNDS.
 * The workspace is only read for its error word (size checked for T).
 */
int32_t moe_gather_rows(const moe_config_t* cfg, int32_t T, const uint16_t* x, const int32_t* row_to_pair,
                        const float* topk_w, int32_t row_begin, int32_t n_rows, uint16_t* rows_out, float* w_out,
                        void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream` and returns the workspace's sticky device error
 * (MOE_OK if none), or MOE_ERR_CUDA if the synchronisation failed. */
int32_t moe_get_device_error(const void* ws, void* stream);

/*
 * moe_permute_static: moe_permute for callers that cannot allocate device
 * memory.  The Lily pages have no counterpart to this call; it exists for
 * callers with no way to obtain scratch memory: a plugin inside a host
 * runtime that owns every device allocation and hands it only pre-allocated
 * input and output buffers, a real-time path where cudaMalloc (which can
 * synchronise the device) is not allowed, or a deployment whose device
 * memory is budgeted by another allocator.
 *
 * Same inputs, outputs and results as moe_permute, without a workspace: the
 * scratch (chunk histograms and ranks) lives in a fixed device array inside
 * the library, MOE_STATIC_MAX_TOKENS tokens' worth (576 KiB), which every GPU
 * that loads the library holds until the process exits.  The call allocates
 * and frees nothing.
 *   err_out  nullable device int32: zeroed by the call, then receives the
 *            call's device error (MOE_ERR_BOUNDS) if any.
 * T > MOE_STATIC_MAX_TOKENS returns MOE_ERR_UNSUPPORTED before any launch.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls share the one array, which keeps the previous call's
 * contents: calls that overlap on the GPU (other streams, other host threads
 * on the same device) race on it and must be serialised by the caller.
 */
#define MOE_STATIC_MAX_TOKENS 16384
int32_t moe_permute_static(const moe_config_t* cfg, int32_t T, const int32_t* topk_idx, const int32_t* counts,
                           int32_t* offsets, int32_t* row_to_pair, int32_t* pair_to_row, int32_t* err_out,
                           void* stream);

/* Number of kernels the four calls launch for one layer of T tokens with the
 * router computing the logits (memsets excluded); -1 if unsupported. */
int32_t moe_launch_count(const moe_config_t* cfg, int32_t T, int32_t mode, int32_t path);

/* Human-readable name of a status code (static string). */
const char* moe_status_string(int32_t status);

/*
 * moe_wait_selftest: failure-detection self-test.  The Lily pages have no
 * counterpart; it exists so that a caller (a test, a health check) can make
 * one of the library's bounded device waits expire on purpose and confirm
 * that the expiry is reported and that the context stays usable.  It
 * computes nothing.
 *   kind 0     one thread waits on a shared-memory mbarrier that nothing
 *              arrives on (the pipeline wait of the FFN kernels); ctas must
 *              be 1 and skip_cta -1.  Always ends in MOE_ERR_TIMEOUT.
 *   kind 1     ctas CTAs (1..148) meet at a grid barrier on a 64-bit counter
 *              (the decode kernels' barrier); the arrival of CTA skip_cta is
 *              suppressed, so the others' waits expire (MOE_ERR_TIMEOUT);
 *              skip_cta = -1 suppresses none and the barrier completes with
 *              no error.
 *   limit_ns   how long each wait lasts before it gives up: 1e3..1e9 ns.
 *   ws         a workspace (256-byte aligned, at least 256 bytes): the
 *              timeout goes to its sticky error word, read it with
 *              moe_get_device_error.  The call also clears and uses 8
 *              reserved bytes of the workspace header for the counter;
 *              nothing else in the workspace is touched.
 * Asynchronous on stream.  Returns MOE_ERR_WORKSPACE for a null or
 * misaligned ws, MOE_ERR_INVALID_ARG for any other bad argument (nothing is
 * launched), MOE_ERR_CUDA if the launch fails, else MOE_OK.
 */
int32_t moe_wait_selftest(int32_t kind, int32_t ctas, int32_t skip_cta, uint64_t limit_ns, void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
