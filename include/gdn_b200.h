/*
 * gdn_b200: the Gated DeltaNet recurrent scan, for NVIDIA B200 (sm_100a).
 * C ABI, in the same library as moe_b200 (libmoe_b200.so), with its status
 * codes (moe_status_t).
 *
 * The Lily pages ("Perplexity built an inference engine for one model, one
 * chip", second paragraph; "Perplexity's Lily brings fast local AI to Apple
 * silicon Macs", section "Where the Engine Gains Speed"): 30 of the model's
 * 40 layers run Gated DeltaNet, which keeps everything before a token in a
 * recurrent state of fixed size, and the engine scans that state with the
 * state held in registers.  The pages give no formula; this call computes
 * the gated delta rule, per sequence b and value head h, with S the
 * [dv, dk] state and, for each new token t in order,
 *     a = exp(g[t]);  S = a S;  u = S k[t];  S = S + beta[t] (v[t] - u) k[t]^T;
 *     o[t] = scale * S q[t]
 * (S_t = a_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T).  Value head h
 * reads query/key head h / (Hv / Hk).  q and k enter as given: any
 * normalisation happens before the call.
 *
 * Arguments (all DEVICE pointers, row-major, contiguous; the caller owns
 * every buffer; bf16 travels as uint16_t bits):
 *   B, T       sequences and new tokens per sequence (both >= 1).
 *   Hk, Hv     query/key heads and value heads, Hv a multiple of Hk.
 *   dk, dv     head sizes: 128 and 128 (anything else: MOE_ERR_UNSUPPORTED).
 *   q, k       bf16 [B, T, Hk, dk];  v bf16 [B, T, Hv, dv].
 *   g          fp32 [B, T, Hv]: log of the decay (<= 0 keeps |S| bounded).
 *   beta       fp32 [B, T, Hv]: write strength.
 *   scale      fp32 output scale (typically dk^-1/2).
 *   state_in   fp32 [B, Hv, dv, dk]: the state before the first token.
 *   state_out  fp32 [B, Hv, dv, dk]: the state after the last token; may be
 *              the same buffer as state_in (updated in place).
 *   o          bf16 [B, T, Hv, dv].
 * Arithmetic is fp32; each CTA reads its rows of the state once, keeps them
 * in registers over all T tokens and writes them once.  Pointers 16-byte
 * aligned (g and beta 4-byte).  Asynchronous on `stream`; it reads what
 * earlier work on the stream wrote (programmatic dependent launch).
 * Returns MOE_ERR_INVALID_ARG for a null or misaligned pointer or a count
 * below 1, MOE_ERR_UNSUPPORTED for other head sizes, MOE_ERR_CUDA if the
 * launch fails, else MOE_OK.
 */
#ifndef GDN_B200_H
#define GDN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int32_t gdn_scan(int32_t B, int32_t T, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, const uint16_t* q,
                 const uint16_t* k, const uint16_t* v, const float* g, const float* beta, float scale,
                 const float* state_in, float* state_out, uint16_t* o, void* stream);

#ifdef __cplusplus
}
#endif

#endif
