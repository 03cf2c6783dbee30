/*
 * oracle.c -- plain fp64 CPU reference for the DM0.5 action-expert (suffix)
 * attention.  TEST INFRASTRUCTURE: only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file.  The product path (the
 * CUDA library) never calls it and shares no code, header, table or helper
 * with it.
 *
 * What it computes (page "TensorRT+Triton+FlexAttention: OpenDM VLA
 * 快速推理加速栈深度剖析", section 2.2 "Triton 大 Kernel"): the action-expert
 * (suffix) attention reads the prefix KV cache and the suffix's own K/V at
 * once, applies the prefix-visibility mask, takes a softmax over the scaled
 * logits and forms the value-weighted sum.  The suffix path's shape table in
 * the same section fixes head_dim 256 and 8 query heads over 4 KV heads
 * (GQA).  The prefix cache is padded to a length bucket (same page, section 3;
 * page "DM05 推理指南", section "Fast Backend 约束"), hence a valid length.
 *
 * Readings taken where the pages are silent (each one is listed with its
 * reason in the design notes):
 *   - every suffix key is visible to every suffix query (bidirectional);
 *   - prefix key j of sample b is visible iff j < clamp(valid_len[b], 0, P)
 *     and (no mask given or mask[b, j] != 0); the same for every head/query;
 *   - query head h reads KV head h / (Hq / Hkv) (contiguous groups);
 *   - logits are scaled by 1 / sqrt(D); no soft-cap, no extra scalar;
 *   - LSE is the natural-log log-sum-exp of the scaled logits.
 *
 * Arithmetic: every bf16 input is widened exactly to double; all sums,
 * exponentials and logarithms are in double with the host libm (exp, log).
 * The softmax is the plain two-pass form: max, then sum of exponentials.
 * There is no blocking, no online rescaling and no reordering beyond that.
 *
 * Parity status: pinned (see tests/test_oracle.py): float64 library
 * scaled-dot-product attention on tiny shapes, closed forms (all-equal
 * logits, constant V, one visible key), invariants (masked rows ignored,
 * prefix permutation), and an arbitrary-precision brute force.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact widening of a bf16 bit pattern: bf16 is the upper half of an IEEE
 * binary32, so shifting the 16 bits up gives the same value as a float. */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int clamp_valid_len(const int32_t *valid_len, int b, int P)
{
    if (valid_len == NULL) return P;
    int v = valid_len[b];
    if (v < 0) return 0;
    if (v > P) return P;
    return v;
}

/* Key index space of one sample: [0, P) are the prefix positions, [P, P+S)
 * the suffix positions.  Returns 1 if key x is visible to every query of
 * sample b. */
static int key_visible(int x, int P, int vl, const uint8_t *mask_row)
{
    if (x >= P) return 1; /* suffix keys: always visible */
    if (x >= vl) return 0; /* bucket padding */
    if (mask_row != NULL && mask_row[x] == 0) return 0;
    return 1;
}

/* One (b, h, i) row restricted to keys x in [key_lo, key_hi) of the index
 * space above.  Writes D outputs and the LSE.  If no key in the range is
 * visible, writes O = 0 and LSE = -inf. */
static void attend_row(const uint16_t *q_row, const uint16_t *kp, const uint16_t *vp,
                       const uint16_t *ks, const uint16_t *vs, const uint8_t *mask_row,
                       int vl, int P, int S, int D, int key_lo, int key_hi,
                       double *logit_buf, double *o_row, double *lse_out)
{
    const double scale = 1.0 / sqrt((double)D);
    int n = 0;
    double m = -INFINITY;
    /* pass 1: logits of the visible keys and their maximum */
    for (int x = key_lo; x < key_hi; ++x) {
        if (!key_visible(x, P, vl, mask_row)) continue;
        const uint16_t *k_row = (x < P) ? kp + (size_t)x * D : ks + (size_t)(x - P) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(k_row[d]);
        double l = scale * dot;
        logit_buf[x - key_lo] = l;
        if (l > m) m = l;
        ++n;
    }
    for (int d = 0; d < D; ++d) o_row[d] = 0.0;
    if (n == 0) {
        *lse_out = -INFINITY;
        return;
    }
    /* pass 2: normaliser Z = sum exp(l - m), LSE = m + ln Z */
    double z = 0.0;
    for (int x = key_lo; x < key_hi; ++x) {
        if (!key_visible(x, P, vl, mask_row)) continue;
        z += exp(logit_buf[x - key_lo] - m);
    }
    double lse = m + log(z);
    /* pass 3: O = sum over visible keys of softmax weight times the V row */
    for (int x = key_lo; x < key_hi; ++x) {
        if (!key_visible(x, P, vl, mask_row)) continue;
        double w = exp(logit_buf[x - key_lo] - lse);
        const uint16_t *v_row = (x < P) ? vp + (size_t)x * D : vs + (size_t)(x - P) * D;
        for (int d = 0; d < D; ++d) o_row[d] += w * bf16_bits_to_double(v_row[d]);
    }
    *lse_out = lse;
}

static int check_shape(int B, int Hq, int Hkv, int P, int S, int D)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || P < 0 || S < 1 || D < 1) return -2;
    if (Hq % Hkv != 0) return -2;
    return 0;
}

/*
 * Attention of the query rows r in [row_lo, row_hi) (flat index
 * r = (b*Hq + h)*S + i) over the keys x in [key_lo, key_hi) of the index
 * space [0, P+S) (prefix positions, then suffix positions).  With the full
 * ranges this is the whole result; rows outside [row_lo, row_hi) are not
 * written.  Layouts (row-major, bf16 passed as uint16 bit patterns):
 *   q [B,Hq,S,D], k_prefix/v_prefix [B,Hkv,P,D], k_suffix/v_suffix [B,Hkv,S,D],
 *   prefix_valid_len int32 [B] or NULL, prefix_mask uint8 [B,P] or NULL,
 *   out double [B,Hq,S,D], lse double [B,Hq,S].
 * nthreads > 1 spreads the rows over OpenMP threads.
 * Returns 0, -1 for a NULL pointer, -2 for a bad shape, -7 for no memory.
 */
int oracle_suffix_attn_rows(const uint16_t *q, const uint16_t *k_prefix, const uint16_t *v_prefix,
                            const int32_t *prefix_valid_len, const uint8_t *prefix_mask,
                            const uint16_t *k_suffix, const uint16_t *v_suffix,
                            double *out, double *lse,
                            int B, int Hq, int Hkv, int P, int S, int D,
                            int key_lo, int key_hi, long row_lo, long row_hi, int nthreads)
{
    if (!q || !k_suffix || !v_suffix || !out || !lse) return -1;
    if (P > 0 && (!k_prefix || !v_prefix)) return -1;
    int rc = check_shape(B, Hq, Hkv, P, S, D);
    if (rc) return rc;
    if (key_lo < 0) key_lo = 0;
    if (key_hi > P + S) key_hi = P + S;
    if (key_hi < key_lo) key_hi = key_lo;
    const long n_rows = (long)B * Hq * S;
    if (row_lo < 0) row_lo = 0;
    if (row_hi > n_rows) row_hi = n_rows;
    const int G = Hq / Hkv;
    const int n_keys = key_hi - key_lo;
    int failed = 0;
    if (nthreads < 1) nthreads = 1;

#pragma omp parallel num_threads(nthreads) reduction(| : failed)
    {
        double *logit_buf = (double *)malloc(sizeof(double) * (size_t)(n_keys > 0 ? n_keys : 1));
        if (!logit_buf) {
            failed = 1;
        } else {
#pragma omp for schedule(static)
            for (long row = row_lo; row < row_hi; ++row) {
                const int b = (int)(row / ((long)Hq * S));
                const int h = (int)((row / S) % Hq);
                const int kv = h / G;
                const int vl = clamp_valid_len(prefix_valid_len, b, P);
                const uint8_t *mask_row = prefix_mask ? prefix_mask + (size_t)b * P : NULL;
                const size_t kv_off_p = ((size_t)b * Hkv + kv) * (size_t)P * D;
                const size_t kv_off_s = ((size_t)b * Hkv + kv) * (size_t)S * D;
                attend_row(q + (size_t)row * D,
                           P > 0 ? k_prefix + kv_off_p : NULL,
                           P > 0 ? v_prefix + kv_off_p : NULL,
                           k_suffix + kv_off_s, v_suffix + kv_off_s, mask_row,
                           vl, P, S, D, key_lo, key_hi, logit_buf,
                           out + (size_t)row * D, lse + row);
            }
            free(logit_buf);
        }
    }
    return failed ? -7 : 0;
}

/* Every query row over the keys x in [key_lo, key_hi). */
int oracle_suffix_attn_range(const uint16_t *q, const uint16_t *k_prefix, const uint16_t *v_prefix,
                             const int32_t *prefix_valid_len, const uint8_t *prefix_mask,
                             const uint16_t *k_suffix, const uint16_t *v_suffix,
                             double *out, double *lse,
                             int B, int Hq, int Hkv, int P, int S, int D,
                             int key_lo, int key_hi, int nthreads)
{
    return oracle_suffix_attn_rows(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask,
                                   k_suffix, v_suffix, out, lse, B, Hq, Hkv, P, S, D,
                                   key_lo, key_hi, 0, (long)B * Hq * S, nthreads);
}

/* The full attention: every visible prefix key and every suffix key. */
int oracle_suffix_attn(const uint16_t *q, const uint16_t *k_prefix, const uint16_t *v_prefix,
                       const int32_t *prefix_valid_len, const uint8_t *prefix_mask,
                       const uint16_t *k_suffix, const uint16_t *v_suffix,
                       double *out, double *lse,
                       int B, int Hq, int Hkv, int P, int S, int D, int nthreads)
{
    return oracle_suffix_attn_range(q, k_prefix, v_prefix, prefix_valid_len, prefix_mask,
                                    k_suffix, v_suffix, out, lse, B, Hq, Hkv, P, S, D,
                                    0, P + S, nthreads);
}

/*
 * Combination of n_parts partial results over disjoint key sets into the
 * result over their union (the log-sum-exp identity):
 *   LSE = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - LSE) * O_s,
 * where O_s is the softmax-weighted sum over part s alone (weights summing to
 * one within the part) and lse_s its log-sum-exp.  A part with lse_s = -inf
 * (no visible key) contributes nothing.  Inputs are [n_parts][rows][D] and
 * [n_parts][rows]; outputs [rows][D] and [rows].
 */
int oracle_merge_parts(const double *o_parts, const double *lse_parts, int n_parts,
                       long rows, int D, double *out, double *lse)
{
    if (!o_parts || !lse_parts || !out || !lse) return -1;
    if (n_parts < 1 || rows < 0 || D < 1) return -2;
    for (long r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int s = 0; s < n_parts; ++s) {
            double l = lse_parts[(size_t)s * rows + r];
            if (l > m) m = l;
        }
        for (int d = 0; d < D; ++d) out[r * D + d] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double z = 0.0;
        for (int s = 0; s < n_parts; ++s) z += exp(lse_parts[(size_t)s * rows + r] - m);
        double total = m + log(z);
        for (int s = 0; s < n_parts; ++s) {
            double l = lse_parts[(size_t)s * rows + r];
            if (l == -INFINITY) continue;
            double w = exp(l - total);
            const double *o = o_parts + ((size_t)s * rows + r) * D;
            for (int d = 0; d < D; ++d) out[r * D + d] += w * o[d];
        }
        lse[r] = total;
    }
    return 0;
}

/*
 * Prefix-prefill attention under the prefix-causal mask (page
 * "TensorRT+Triton+FlexAttention: OpenDM VLA 快速推理加速栈深度剖析", section
 * 2.3: the prefix stage runs its attention through flex_attention with a
 * custom causal mask mapping built by _make_prefix_causal_mask_mapping).
 * The queries are the P prefix positions themselves and the keys/values the
 * prefix K/V of the same call (the tensors that later form the prefix KV
 * cache the suffix attention reads).
 *
 * Readings where the page is silent (listed in the design notes):
 *   - "causal" is the standard rule: prefix query i sees prefix key j iff
 *     j <= i; positions at or past clamp(valid_len[b], 0, P) are bucket
 *     padding and are never keys;
 *   - the query rows i >= valid length are padding: they are not computed
 *     (their out / lse entries are left as they were);
 *   - a row with no visible key (valid length 0 cannot reach a computed row)
 *     cannot occur among the computed rows, since key 0 <= i is in range;
 *   - GQA, scale 1/sqrt(D) and the natural-log LSE as in the suffix call.
 *
 * Layouts: q [B,Hq,P,D], k/v [B,Hkv,P,D] bf16 bit patterns, valid_len int32
 * [B] or NULL (every position in range), out double [B,Hq,P,D], lse double
 * [B,Hq,P].  Each row takes the same three passes as attend_row: the logits
 * and their maximum, the normaliser, the weighted sum of the value rows.
 * Returns 0, -1 for a NULL pointer, -2 for a bad shape, -7 for no memory.
 */
int oracle_prefix_causal_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              const int32_t *valid_len, double *out, double *lse,
                              int B, int Hq, int Hkv, int P, int D, int nthreads)
{
    if (!q || !k || !v || !out || !lse) return -1;
    if (B < 1 || Hq < 1 || Hkv < 1 || P < 1 || D < 1 || Hq % Hkv != 0) return -2;
    const int G = Hq / Hkv;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    const long n_rows = (long)B * Hq * P;
    int failed = 0;
    if (nthreads < 1) nthreads = 1;

#pragma omp parallel num_threads(nthreads) reduction(| : failed)
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)P);
        if (!logit) {
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long row = 0; row < n_rows; ++row) {
                const int b = (int)(row / ((long)Hq * P));
                const int h = (int)((row / P) % Hq);
                const int i = (int)(row % P);
                const int vl = clamp_valid_len(valid_len, b, P);
                if (i >= vl) continue; /* padding query: not computed */
                const size_t kv_off = ((size_t)b * Hkv + h / G) * (size_t)P * D;
                const uint16_t *q_row = q + (size_t)row * D;
                /* visible keys: j <= i (and j < vl, implied since i < vl) */
                const int n = i + 1;
                double m = -INFINITY;
                for (int j = 0; j < n; ++j) {
                    const uint16_t *k_row = k + kv_off + (size_t)j * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(k_row[d]);
                    logit[j] = inv_sqrt_d * dot;
                    if (logit[j] > m) m = logit[j];
                }
                double z = 0.0;
                for (int j = 0; j < n; ++j) z += exp(logit[j] - m);
                const double l = m + log(z);
                double *o_row = out + (size_t)row * D;
                for (int d = 0; d < D; ++d) o_row[d] = 0.0;
                for (int j = 0; j < n; ++j) {
                    const double w = exp(logit[j] - l);
                    const uint16_t *v_row = v + kv_off + (size_t)j * D;
                    for (int d = 0; d < D; ++d) o_row[d] += w * bf16_bits_to_double(v_row[d]);
                }
                lse[row] = l;
            }
            free(logit);
        }
    }
    return failed ? -7 : 0;
}

/*
 * Suffix attention prologue: QKV projection, QK-Norm and RoPE in one step
 * (page "TensorRT+Triton+FlexAttention: OpenDM VLA 快速推理加速栈深度剖析",
 * section 2.2, lists "QKV projection + QK-Norm + RoPE done at once" among
 * the fused steps; the action expert's shape table gives hidden 1024,
 * head_dim 256 and 8 / 4 heads).  It produces the suffix queries and keys
 * and values in the layout the suffix attention reads.
 *
 * Readings where the page is silent (listed in the design notes):
 *   - one weight matrix w [(Hq + 2 Hkv) * D, H] (rows: the Hq query heads,
 *     then the Hkv key heads, then the Hkv value heads), no bias;
 *   - QK-Norm is an RMS norm over each head's D features with a learned
 *     per-feature weight shared by all heads of its kind (qw for queries, kw
 *     for keys): y_d = x_d / sqrt(mean_d x_d^2 + eps) * w_d; values are not
 *     normalised;
 *   - RoPE rotates the normalised query and key features in the
 *     "rotate-half" pairing (d, d + D/2) by the angle pos * theta^(-2d/D),
 *     pos the token's position (an input per token);
 *   - everything in double from bf16 inputs widened exactly.
 *
 * Layouts: x [B*S, H] bf16 bits (token t = b*S + i), w [(Hq+2Hkv)*D, H] bf16
 * bits, qw / kw [D] bf16 bits, pos int32 [B*S]; outputs double
 * q [B,Hq,S,D], k [B,Hkv,S,D], v [B,Hkv,S,D].
 * Returns 0, -1 for a NULL pointer, -2 for a bad shape, -7 for no memory.
 */
int oracle_qkv_prologue(const uint16_t *x, const uint16_t *w, const uint16_t *qw, const uint16_t *kw,
                        const int32_t *pos, double eps, double theta, double *q, double *k, double *v,
                        int B, int S, int H, int Hq, int Hkv, int D, int nthreads)
{
    if (!x || !w || !qw || !kw || !pos || !q || !k || !v) return -1;
    if (B < 1 || S < 1 || H < 1 || Hq < 1 || Hkv < 1 || D < 2 || D % 2 != 0) return -2;
    const int n_heads = Hq + 2 * Hkv;
    const long n_items = (long)B * S * n_heads; /* (token, head) pairs */
    int failed = 0;
    if (nthreads < 1) nthreads = 1;

#pragma omp parallel num_threads(nthreads) reduction(| : failed)
    {
        double *feat = (double *)malloc(sizeof(double) * (size_t)D);
        if (!feat) {
            failed = 1;
        } else {
#pragma omp for schedule(static)
            for (long it = 0; it < n_items; ++it) {
                const long t = it / n_heads;           /* token b*S + i */
                const int hd = (int)(it % n_heads);    /* head in projection order */
                const int b = (int)(t / S), i = (int)(t % S);
                /* projection: feature f of this head = <w row, x_t> */
                for (int d = 0; d < D; ++d) {
                    const uint16_t *w_row = w + ((size_t)hd * D + d) * (size_t)H;
                    const uint16_t *x_row = x + (size_t)t * H;
                    double acc = 0.0;
                    for (int c = 0; c < H; ++c) acc += bf16_bits_to_double(w_row[c]) * bf16_bits_to_double(x_row[c]);
                    feat[d] = acc;
                }
                double *dst;
                if (hd >= Hq + Hkv) { /* value head: projection only */
                    dst = v + (((size_t)b * Hkv + (hd - Hq - Hkv)) * S + i) * (size_t)D;
                    for (int d = 0; d < D; ++d) dst[d] = feat[d];
                    continue;
                }
                const int is_q = hd < Hq;
                const uint16_t *nw = is_q ? qw : kw;
                dst = is_q ? q + (((size_t)b * Hq + hd) * S + i) * (size_t)D
                           : k + (((size_t)b * Hkv + (hd - Hq)) * S + i) * (size_t)D;
                /* QK-Norm: RMS over the head's features, then the weight */
                double ms = 0.0;
                for (int d = 0; d < D; ++d) ms += feat[d] * feat[d];
                const double inv_rms = 1.0 / sqrt(ms / (double)D + eps);
                for (int d = 0; d < D; ++d) feat[d] = feat[d] * inv_rms * bf16_bits_to_double(nw[d]);
                /* RoPE, rotate-half pairing: (d, d + D/2) turned by pos * theta^(-2d/D) */
                const int half = D / 2;
                const double p = (double)pos[t];
                for (int d = 0; d < half; ++d) {
                    const double ang = p * pow(theta, -2.0 * (double)d / (double)D);
                    const double c = cos(ang), s = sin(ang);
                    const double a = feat[d], e = feat[d + half];
                    dst[d] = a * c - e * s;
                    dst[d + half] = a * s + e * c;
                }
            }
            free(feat);
        }
    }
    return failed ? -7 : 0;
}

/*
 * Post-attention block of an action-expert layer (page "TensorRT+Triton+
 * FlexAttention: OpenDM VLA 快速推理加速栈深度剖析", section 2.2: after the
 * three attention stages the suffix path chains the time modulation Adarms,
 * the GEGLU gate-up and the MLP down; the action expert's shape table gives
 * hidden 1024 and intermediate 4096).
 *
 * Readings where the page is silent (listed in the design notes), for token
 * t = b * S + i of sample b:
 *   a_t   = the attention output of the token, its Hq heads' D features
 *           concatenated (head-major) into Hq * D values;
 *   h1    = h_t + Wo a_t                          (output projection, residual)
 *   u     = h1 / sqrt(mean(h1^2) + eps) * (1 + scale_b) + shift_b   (Adarms:
 *           an RMS norm whose weight and bias come from the time embedding,
 *           one (scale, shift, gate) triple per sample)
 *   m     = gelu_tanh(Wg u) * (Wu u)              (GEGLU, gate and up rows of Wgu)
 *   out_t = h1 + gate_b * (Wd m)                  (MLP down, gated residual)
 * with gelu_tanh(z) = z / 2 * (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).
 *
 * Layouts: attn [B,Hq,S,D] bf16 bits; h [B*S, Hd] bf16 bits; scale, shift,
 * gate [B, Hd] bf16 bits; wo [Hd, Hq*D], wgu [2*F, Hd] (gate rows then up
 * rows), wd [Hd, F] bf16 bits; out double [B*S, Hd].
 * Returns 0, -1 for a NULL pointer, -2 for a bad shape, -7 for no memory.
 */
int oracle_post_attention(const uint16_t *attn, const uint16_t *h, const uint16_t *scale, const uint16_t *shift,
                          const uint16_t *gate, const uint16_t *wo, const uint16_t *wgu, const uint16_t *wd,
                          double eps, double *out, int B, int S, int Hq, int D, int Hd, int F, int nthreads)
{
    if (!attn || !h || !scale || !shift || !gate || !wo || !wgu || !wd || !out) return -1;
    if (B < 1 || S < 1 || Hq < 1 || D < 1 || Hd < 1 || F < 1) return -2;
    const long T = (long)B * S;
    const int A = Hq * D;
    int failed = 0;
    if (nthreads < 1) nthreads = 1;

#pragma omp parallel num_threads(nthreads) reduction(| : failed)
    {
        double *av = (double *)malloc(sizeof(double) * (size_t)A);
        double *h1 = (double *)malloc(sizeof(double) * (size_t)Hd);
        double *u = (double *)malloc(sizeof(double) * (size_t)Hd);
        double *m = (double *)malloc(sizeof(double) * (size_t)F);
        if (!av || !h1 || !u || !m) {
            failed = 1;
        } else {
#pragma omp for schedule(static)
            for (long t = 0; t < T; ++t) {
                const int b = (int)(t / S), i = (int)(t % S);
                /* the token's attention output, heads concatenated */
                for (int hh = 0; hh < Hq; ++hh)
                    for (int d = 0; d < D; ++d)
                        av[hh * D + d] = bf16_bits_to_double(attn[(((size_t)b * Hq + hh) * S + i) * D + d]);
                /* output projection and residual */
                for (int o = 0; o < Hd; ++o) {
                    double acc = 0.0;
                    for (int c = 0; c < A; ++c) acc += bf16_bits_to_double(wo[(size_t)o * A + c]) * av[c];
                    h1[o] = bf16_bits_to_double(h[(size_t)t * Hd + o]) + acc;
                }
                /* Adarms: RMS norm with the time modulation as weight and bias */
                double ms = 0.0;
                for (int o = 0; o < Hd; ++o) ms += h1[o] * h1[o];
                const double inv_rms = 1.0 / sqrt(ms / (double)Hd + eps);
                for (int o = 0; o < Hd; ++o)
                    u[o] = h1[o] * inv_rms * (1.0 + bf16_bits_to_double(scale[(size_t)b * Hd + o])) +
                           bf16_bits_to_double(shift[(size_t)b * Hd + o]);
                /* GEGLU: gelu(gate projection) times up projection */
                for (int f = 0; f < F; ++f) {
                    double g = 0.0, up = 0.0;
                    for (int c = 0; c < Hd; ++c) {
                        g += bf16_bits_to_double(wgu[(size_t)f * Hd + c]) * u[c];
                        up += bf16_bits_to_double(wgu[((size_t)F + f) * Hd + c]) * u[c];
                    }
                    const double z = g;
                    const double gelu = 0.5 * z * (1.0 + tanh(sqrt(2.0 / M_PI) * (z + 0.044715 * z * z * z)));
                    m[f] = gelu * up;
                }
                /* MLP down and the gated residual */
                for (int o = 0; o < Hd; ++o) {
                    double acc = 0.0;
                    for (int f = 0; f < F; ++f) acc += bf16_bits_to_double(wd[(size_t)o * F + f]) * m[f];
                    out[(size_t)t * Hd + o] = h1[o] + bf16_bits_to_double(gate[(size_t)b * Hd + o]) * acc;
                }
            }
        }
        free(av);
        free(h1);
        free(u);
        free(m);
    }
    return failed ? -7 : 0;
}

/* Number of OpenMP threads the oracle can use (1 when compiled without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
