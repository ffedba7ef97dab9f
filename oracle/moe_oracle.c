/*
 * CPU oracle of one MoE expert layer (routing, 4-bit dequant, SwiGLU experts,
 * shared expert, weighted combine).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code with
 * the CUDA path and must never be used as a fallback for it.
 *
 * Sources (the Lily pages):
 *  - "Perplexity's Lily brings fast local AI to Apple silicon Macs"
 *    (artiverse.ca), section "A 35B Model Built for Local Memory": 256
 *    experts, eight selected per token; groupwise affine 4-bit weights.
 *  - Same page, section "Where the Engine Gains Speed": weights are
 *    reconstructed inside the grouped GEMM, routing stays on the GPU.
 *  - "Perplexity built an inference engine for one model, one chip"
 *    (aiinsiders.net), second paragraph: a router picks eight of 256
 *    subnetworks and one shared expert sees every token.
 *
 * The pages give no formulas.  Readings taken where they are silent:
 *  R1 router logits l[t,e] = sum_h x[t,h] * Wr[e,h] (+ bias), accumulated in
 *     fp32 in one fixed order (the "contract order", below), because the
 *     routing decision must be reproduced bit for bit;
 *  R2 selection = first k of the sort by (logit descending, expert ascending);
 *     -0.0 and +0.0 tie; non-finite logits are rejected;
 *  R3 weights = softmax over all E logits, restricted to the k selected and
 *     renormalised to sum to one (fp64);
 *  R4 dequant w = scale * q + bias with (scale, bias) bf16 per group of G
 *     consecutive inputs of an output row, q the unsigned nibble; nibble j of
 *     u32 word m holds input 8m + j (little-endian nibbles);
 *  R5 expert = SwiGLU: g = x Wg^T, u = x Wu^T (gate rows 0..I-1, up rows
 *     I..2I-1 of the gate_up matrix), h = silu(g) * u, y = h Wd^T (fp64);
 *  R6 shared expert: same shape and format, weight 1, no gate;
 *     y = sum_k w_k y_{idx_k} + y_shared (fp64).
 *
 * Contract order of R1 (H a multiple of 256): the inputs are cut into chunks
 * of 8 consecutive h; slice s in 0..31 owns chunks c = s, s+32, s+64, ...
 * acc[s] starts at +0.0f and takes acc[s] = fmaf(x, w, acc[s]) over its
 * chunks in increasing c, and within a chunk over h = 8c..8c+7.  The 32
 * slices are then combined by an xor butterfly: for off = 16, 8, 4, 2, 1,
 * acc[s] = acc[s] + acc[s ^ off] for all s at once; the logit is acc[0],
 * plus bias[t * stride + e] in one fp32 addition when a bias is given.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NONFINITE 5
#define ORACLE_ERR_BOUNDS 7

static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ---------------------------------------------------------------- R4 ---- */

/* The 4-bit code of input k of a row whose packed words start at row_words. */
int moe_oracle_code(const uint32_t* row_words, int64_t k) {
    uint32_t word = row_words[k / 8];
    int j = (int)(k % 8);
    return (int)((word >> (4 * j)) & 0xFu);
}

/* Dequantised weight (n, k) of an [N, K] matrix stored as codes [N][K/8] and
 * (scale, bias) pairs [N][K/G][2]. */
double moe_oracle_dequant_one(const uint32_t* codes, const uint16_t* sb, int64_t K, int64_t G,
                              int64_t n, int64_t k) {
    const uint32_t* row = codes + n * (K / 8);
    const uint16_t* pair = sb + (n * (K / G) + k / G) * 2;
    double scale = bf16_to_double(pair[0]);
    double bias = bf16_to_double(pair[1]);
    return scale * (double)moe_oracle_code(row, k) + bias;
}

void moe_oracle_dequant_matrix(const uint32_t* codes, const uint16_t* sb, int64_t N, int64_t K,
                               int64_t G, double* W) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) W[n * K + k] = moe_oracle_dequant_one(codes, sb, K, G, n, k);
}

/* ---------------------------------------------------------------- R1 ---- */

static float logit_contract_order(const uint16_t* xr, const uint16_t* wr, int64_t H) {
    float acc[32];
    int64_t nchunks = H / 8;
    for (int s = 0; s < 32; ++s) {
        acc[s] = 0.0f;
        for (int64_t c = s; c < nchunks; c += 32)
            for (int j = 0; j < 8; ++j) {
                int64_t h = 8 * c + j;
                acc[s] = fmaf(bf16_to_float(xr[h]), bf16_to_float(wr[h]), acc[s]);
            }
    }
    for (int off = 16; off >= 1; off /= 2) {
        float nxt[32];
        for (int s = 0; s < 32; ++s) nxt[s] = acc[s] + acc[s ^ off];
        memcpy(acc, nxt, sizeof(acc));
    }
    return acc[0];
}

/* logits[t][e] for tokens tok[0..n-1] (tok == NULL: tokens 0..n-1). */
int moe_oracle_router_logits(int64_t n, const int32_t* tok, int64_t H, int64_t E,
                             const uint16_t* x, const uint16_t* wr, const float* bias,
                             int64_t bias_stride, float* logits) {
    if (H % 256 != 0) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
        int64_t t = tok ? tok[i] : i;
        for (int64_t e = 0; e < E; ++e) {
            float l = logit_contract_order(x + t * H, wr + e * H, H);
            if (bias) l = l + bias[t * bias_stride + e];
            logits[i * E + e] = l;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------ R2 + R3 ---- */

/* Top-k of each row of logits [n][E] -> idx [n][k] (in selection order) and
 * renormalised weights w [n][k] (fp64). */
int moe_oracle_select(int64_t n, int64_t E, int64_t k, const float* logits, int32_t* idx, double* w) {
    if (k < 1 || k > E) return ORACLE_ERR_ARG;
    int status = ORACLE_OK;
    char* taken = (char*)malloc((size_t)E);
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    for (int64_t t = 0; t < n; ++t) {
        const float* l = logits + t * E;
        for (int64_t e = 0; e < E; ++e)
            if (!isfinite(l[e])) status = ORACLE_ERR_NONFINITE;
        if (status != ORACLE_OK) break;
        /* R2: repeatedly take the largest logit not yet taken, lowest index on ties. */
        memset(taken, 0, (size_t)E);
        for (int64_t s = 0; s < k; ++s) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: earlier index wins ties */
            }
            taken[best] = 1;
            idx[t * k + s] = (int32_t)best;
        }
        /* R3: softmax over all E logits, then renormalise over the selected. */
        double m = -INFINITY;
        for (int64_t e = 0; e < E; ++e) m = fmax(m, (double)l[e]);
        double z = 0.0;
        for (int64_t e = 0; e < E; ++e) {
            p[e] = exp((double)l[e] - m);
            z += p[e];
        }
        for (int64_t e = 0; e < E; ++e) p[e] /= z;
        double sel = 0.0;
        for (int64_t s = 0; s < k; ++s) sel += p[idx[t * k + s]];
        for (int64_t s = 0; s < k; ++s) w[t * k + s] = p[idx[t * k + s]] / sel;
    }
    free(taken);
    free(p);
    return status;
}

/* ------------------------------------------------------------- counts ---- */

/* counts[e], offsets[e] (exclusive scan, offsets[E] = T*k), and the stable
 * expert-major permutation: the pairs of expert e take rows offsets[e]...
 * in increasing token order.  Pair p = t*k + slot. */
int moe_oracle_permute(int64_t T, int64_t E, int64_t k, const int32_t* idx, int32_t* counts,
                       int32_t* offsets, int32_t* row_to_pair, int32_t* pair_to_row) {
    for (int64_t t = 0; t < T; ++t)
        for (int64_t a = 0; a < k; ++a) {
            int32_t e = idx[t * k + a];
            if (e < 0 || e >= E) return ORACLE_ERR_BOUNDS;
            for (int64_t b = 0; b < a; ++b)
                if (idx[t * k + b] == e) return ORACLE_ERR_BOUNDS;
        }
    for (int64_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < T * k; ++p) counts[idx[p]] += 1;
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t next = 0;
    for (int64_t e = 0; e < E; ++e)
        for (int64_t t = 0; t < T; ++t)
            for (int64_t a = 0; a < k; ++a)
                if (idx[t * k + a] == e) {
                    row_to_pair[next] = (int32_t)(t * k + a);
                    pair_to_row[t * k + a] = next;
                    ++next;
                }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ R5 ---- */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* One expert on nrows token rows.  Wgu [2I][H] and Wd [H][I] already
 * dequantised.  h_out [nrows][I] may be NULL. */
static void expert_apply(int64_t H, int64_t I, const double* Wgu, const double* Wd, int64_t nrows,
                         const double* xr, double* h_out, double* y_out) {
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    for (int64_t r = 0; r < nrows; ++r) {
        const double* xv = xr + r * H;
        for (int64_t j = 0; j < I; ++j) {
            double g = 0.0, u = 0.0;
            for (int64_t q = 0; q < H; ++q) g += xv[q] * Wgu[j * H + q];
            for (int64_t q = 0; q < H; ++q) u += xv[q] * Wgu[(I + j) * H + q];
            h[j] = silu(g) * u;
            if (h_out) h_out[r * I + j] = h[j];
        }
        for (int64_t o = 0; o < H; ++o) {
            double y = 0.0;
            for (int64_t j = 0; j < I; ++j) y += h[j] * Wd[o * I + j];
            y_out[r * H + o] = y;
        }
    }
    free(h);
}

/* Expert `e` of the packed weight arrays applied to bf16 rows x [nrows][H]. */
void moe_oracle_expert_rows(int64_t H, int64_t I, int64_t G, int64_t e, const uint32_t* gu_codes,
                            const uint16_t* gu_sb, const uint32_t* d_codes, const uint16_t* d_sb,
                            int64_t nrows, const uint16_t* x, double* h_out, double* y_out) {
    double* Wgu = (double*)malloc(sizeof(double) * (size_t)(2 * I * H));
    double* Wd = (double*)malloc(sizeof(double) * (size_t)(H * I));
    double* xr = (double*)malloc(sizeof(double) * (size_t)(nrows * H));
    moe_oracle_dequant_matrix(gu_codes + e * (2 * I) * (H / 8), gu_sb + e * (2 * I) * (H / G) * 2,
                              2 * I, H, G, Wgu);
    moe_oracle_dequant_matrix(d_codes + e * H * (I / 8), d_sb + e * H * (I / G) * 2, H, I, G, Wd);
    for (int64_t i = 0; i < nrows * H; ++i) xr[i] = bf16_to_double(x[i]);
    expert_apply(H, I, Wgu, Wd, nrows, xr, h_out, y_out);
    free(Wgu);
    free(Wd);
    free(xr);
}

/* ------------------------------------------------------------------ R6 ---- */

/* The layer output y [n][H] (fp64) for tokens tok[0..n-1] of a T-token batch.
 * logits_in (nullable, [T][E]) replaces the router product; bias is added in
 * either case.  idx_out [n][k] and w_out [n][k] are optional. */
int moe_oracle_layer(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, int64_t G,
                     int has_shared, const uint16_t* x, const uint16_t* wr, const float* logits_in,
                     const float* bias, int64_t bias_stride, const uint32_t* gu_codes,
                     const uint16_t* gu_sb, const uint32_t* d_codes, const uint16_t* d_sb,
                     int64_t n, const int32_t* tok, double* y, int32_t* idx_out, double* w_out) {
    if (H % 256 != 0 || H % G != 0 || I % G != 0 || G % 8 != 0) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < n; ++i)
        if (tok[i] < 0 || tok[i] >= T) return ORACLE_ERR_ARG;
    float* logits = (float*)malloc(sizeof(float) * (size_t)(n * E));
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n * k));
    double* w = (double*)malloc(sizeof(double) * (size_t)(n * k));
    int status = ORACLE_OK;
    if (logits_in) {
        for (int64_t i = 0; i < n; ++i)
            for (int64_t e = 0; e < E; ++e) {
                float l = logits_in[(int64_t)tok[i] * E + e];
                if (bias) l = l + bias[(int64_t)tok[i] * bias_stride + e];
                logits[i * E + e] = l;
            }
    } else {
        status = moe_oracle_router_logits(n, tok, H, E, x, wr, bias, bias_stride, logits);
    }
    if (status == ORACLE_OK) status = moe_oracle_select(n, E, k, logits, idx, w);
    if (status != ORACLE_OK) {
        free(logits);
        free(idx);
        free(w);
        return status;
    }
    /* per (token, slot) expert outputs; slot k is the shared expert */
    int64_t nslot = k + 1;
    double* ys = (double*)calloc((size_t)(n * nslot * H), sizeof(double));
    int64_t nexp = E + (has_shared ? 1 : 0);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t e = 0; e < nexp; ++e) {
        int64_t cnt = 0;
        for (int64_t i = 0; i < n; ++i) {
            if (e == E) { ++cnt; continue; }
            for (int64_t s = 0; s < k; ++s) cnt += (idx[i * k + s] == e);
        }
        if (cnt == 0) continue;
        uint16_t* xr = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(cnt * H));
        int64_t* dst = (int64_t*)malloc(sizeof(int64_t) * (size_t)cnt);
        int64_t r = 0;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t s = 0; s < nslot; ++s) {
                int hit = (e == E) ? (s == k) : (s < k && idx[i * k + s] == e);
                if (!hit) continue;
                memcpy(xr + r * H, x + (int64_t)tok[i] * H, sizeof(uint16_t) * (size_t)H);
                dst[r++] = i * nslot + s;
            }
        double* yr = (double*)malloc(sizeof(double) * (size_t)(cnt * H));
        moe_oracle_expert_rows(H, I, G, e, gu_codes, gu_sb, d_codes, d_sb, cnt, xr, NULL, yr);
        for (int64_t q = 0; q < cnt; ++q) memcpy(ys + dst[q] * H, yr + q * H, sizeof(double) * (size_t)H);
        free(xr);
        free(dst);
        free(yr);
    }
    for (int64_t i = 0; i < n; ++i)
        for (int64_t o = 0; o < H; ++o) {
            double acc = 0.0;
            for (int64_t s = 0; s < k; ++s) acc += w[i * k + s] * ys[(i * nslot + s) * H + o];
            if (has_shared) acc += ys[(i * nslot + k) * H + o];
            y[i * H + o] = acc;
        }
    if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * (size_t)(n * k));
    if (w_out) memcpy(w_out, w, sizeof(double) * (size_t)(n * k));
    free(ys);
    free(logits);
    free(idx);
    free(w);
    return ORACLE_OK;
}
