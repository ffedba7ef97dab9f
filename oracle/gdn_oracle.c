/*
 * CPU oracle of the Gated DeltaNet recurrent scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code with
 * the CUDA path and must never be used as a fallback for it.
 *
 * Sources (the Lily pages):
 *  - "Perplexity built an inference engine for one model, one chip"
 *    (aiinsiders.net), second paragraph: 30 of the model's 40 layers run
 *    Gated DeltaNet, which folds everything before a token into a recurrent
 *    state of fixed size instead of a growing cache.
 *  - "Perplexity's Lily brings fast local AI to Apple silicon Macs"
 *    (artiverse.ca), section "Where the Engine Gains Speed": the scan over
 *    that state is kept in registers (a +5.6% prefill gain).
 *
 * The pages give no formula.  Readings taken where they are silent:
 *  D1 the gated delta rule, per sequence b and value head h, with the state
 *     S a [dv, dk] matrix: for each new token t in order,
 *         a   = exp(g[t])                      (the gate: a decay in (0, 1])
 *         S   = a * S                          (forget)
 *         u   = S k[t]                         (what the state recalls for k)
 *         S   = S + beta[t] * (v[t] - u) k[t]^T  (write the correction)
 *         o[t] = scale * S q[t]                (read with the query)
 *     i.e. S_t = a_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T and
 *     o_t = scale S_t q_t;
 *  D2 value head h reads key head h / (Hv / Hk) (query and key heads shared
 *     by groups of value heads); q, k and v enter as given (bf16): any
 *     normalisation of q and k happens before the scan;
 *  D3 g and beta are per (token, value head) fp32; the state enters and
 *     leaves as fp32 [B, Hv, dv, dk] (row i of S is output channel i);
 *  D4 arithmetic in fp64 here.
 * Layouts: q, k [B, T, Hk, dk]; v [B, T, Hv, dv]; g, beta [B, T, Hv];
 * S0, S_out [B, Hv, dv, dk]; o [B, T, Hv, dv].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1

static double bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

int gdn_oracle_scan(int64_t B, int64_t T, int64_t Hk, int64_t Hv, int64_t dk, int64_t dv, const uint16_t* q,
                    const uint16_t* k, const uint16_t* v, const float* g, const float* beta, double scale,
                    const float* S0, double* o, double* S_out) {
    if (B < 1 || T < 0 || Hk < 1 || Hv < 1 || Hv % Hk || dk < 1 || dv < 1) return ORACLE_ERR_ARG;
    const int64_t group = Hv / Hk;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < Hv; ++h) {
            const int64_t hk = h / group;
            double* S = S_out + (b * Hv + h) * dv * dk;
            const float* S_in = S0 + (b * Hv + h) * dv * dk;
            for (int64_t i = 0; i < dv * dk; ++i) S[i] = (double)S_in[i];
            double* kt = (double*)malloc(sizeof(double) * (size_t)dk);
            double* qt = (double*)malloc(sizeof(double) * (size_t)dk);
            for (int64_t t = 0; t < T; ++t) {
                const int64_t tk = (b * T + t) * Hk + hk, tv = (b * T + t) * Hv + h;
                for (int64_t j = 0; j < dk; ++j) {
                    kt[j] = bf16_value(k[tk * dk + j]);
                    qt[j] = bf16_value(q[tk * dk + j]);
                }
                const double a = exp((double)g[tv]);
                const double bt = (double)beta[tv];
                for (int64_t i = 0; i < dv; ++i) {
                    double* row = S + i * dk;
                    double u = 0.0;
                    for (int64_t j = 0; j < dk; ++j) {
                        row[j] = a * row[j];
                        u += row[j] * kt[j];
                    }
                    const double w = bt * (bf16_value(v[tv * dv + i]) - u);
                    double r = 0.0;
                    for (int64_t j = 0; j < dk; ++j) {
                        row[j] = row[j] + w * kt[j];
                        r += row[j] * qt[j];
                    }
                    o[tv * dv + i] = scale * r;
                }
            }
            free(kt);
            free(qt);
        }
    return ORACLE_OK;
}
