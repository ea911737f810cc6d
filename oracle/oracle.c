/*
 * fp64 CPU oracle for the attention core of a hybrid sliding-window /
 * full-attention GQA decoder layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * statement of what the GPU path computes.  It is linked by nothing in the
 * product: only the tests, the package's smoke entry and the benchmark's
 * CPU-baseline leg load it.  It shares no source, header, table or helper
 * with the CUDA library.
 *
 * What it follows (page / section):
 *  - "Step-3.7-Flash-oQ3e" explainer (m.lqnn.cn), section 2.2: two masks,
 *    a plain causal one for full-attention layers and a sliding-window
 *    causal one for sliding layers, whose KV cache keeps only the last 512
 *    tokens.  Reading taken: query i sees key j iff i-W < j <= i (W keys,
 *    self included); W = infinity on full layers.
 *  - same page, section 2.3: rope_theta is per layer, partial_rotary_factors
 *    rotate only part of the head dims on full layers, and every head has
 *    its own sigmoid output gate.  Readings taken: the first rotary_dim dims
 *    are rotated, pairs (k, k + rotary_dim/2) ("rotate-half"), frequency
 *    theta^(-2k/rotary_dim); the gate is one logit per (token, q-head) and
 *    multiplies the normalised attention output.
 *  - "Step-3.7-Flash" spec card (llm-atlas), config dump:
 *    num_attention_groups = 8 for 64 q-heads, att_impl_type GQA.  Reading
 *    taken: contiguous groups, kv head = h / (Hq / Hkv).
 *  - "Muse-Glimmer-30B-6bit" explainer (discosf.com), GQA and RoPE
 *    sections: 16:1 GQA, layer_rope_theta = 0 on full layers means no
 *    rotary position encoding (identity), and the KV-cache footprint
 *    arithmetic (128K context, 2 KV heads, 52 layers, about 6.5 GiB).
 *  - The pages say only "attention"; the oracle is the plain definition of
 *    masked softmax attention: s_j = scale * <q_i, k_j>, weights
 *    exp(s_j - max) / sum, output sum_j w_j v_j.  Scale reading: 1/sqrt(D).
 *
 * Every function is fp64 over the exact bf16 input values; no intermediate
 * rounding.  OpenMP parallelises over independent output rows only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t window;        /* >= 1: sliding window of W keys; -1: full causal */
    double rope_theta;     /* 0 => no rotary position encoding */
    int32_t rotary_dim;    /* even, 0..head_dim */
    double softmax_scale;  /* <= 0 => 1/sqrt(head_dim) */
    const double* inv_freq;  /* rotary_dim/2 angular frequencies, or NULL for theta^(-2k/r) */
} oracle_layer;

enum { ORACLE_OK = 0, ORACLE_BAD_ARG = 1, ORACLE_NO_MEM = 2 };

/* bf16 -> double by placing the 16 stored bits above 16 zero bits of an
 * IEEE binary32 value (bf16 is the upper half of binary32). */
static double bf16_bits_to_f64(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int layer_ok(const oracle_layer* L) {
    if (!L) return 0;
    if (L->num_q_heads <= 0 || L->num_kv_heads <= 0 || L->head_dim <= 0) return 0;
    if (L->num_q_heads % L->num_kv_heads != 0) return 0;
    if (L->window == 0 || L->window < -1) return 0;
    if (L->rotary_dim < 0 || L->rotary_dim > L->head_dim || (L->rotary_dim & 1)) return 0;
    if (L->rope_theta < 0.0) return 0;
    if (L->inv_freq)
        for (int32_t k = 0; k < L->rotary_dim / 2; ++k)
            if (!(L->inv_freq[k] >= 0.0) || isinf(L->inv_freq[k])) return 0;
    return 1;
}

static double layer_scale(const oracle_layer* L) {
    return L->softmax_scale > 0.0 ? L->softmax_scale : 1.0 / sqrt((double)L->head_dim);
}

/* Rotary position encoding of one head vector, in place, at position p.
 * Explainer section 2.3 (per-layer theta, partial rotary) and the Muse
 * RoPE section (theta = 0 means no rotation).  For k < r/2 the pair
 * (x_k, x_{k+r/2}) is turned by the angle p * theta^(-2k/r). */
void oracle_rope_vec(double* x, int32_t D, int32_t r, double theta, double p) {
    if (theta == 0.0 || r == 0) return;
    int32_t half = r / 2;
    for (int32_t k = 0; k < half; ++k) {
        double freq = pow(theta, -2.0 * (double)k / (double)r);
        double phi = p * freq;
        double c = cos(phi), s = sin(phi);
        double a = x[k], b = x[k + half];
        x[k] = a * c - b * s;
        x[k + half] = b * c + a * s;
    }
    (void)D;
}

/* The same rotation with the frequency of pair k taken from a table
 * (inv_freq[k], k < r/2) instead of theta^(-2k/r).  The Step explainer's
 * section 2.3 gives the full layers a YaRN rope scaling (rope_type llama3,
 * factor 2.0) whose remaining parameters it does not state, so the caller
 * supplies the scaled frequencies; with inv_freq[k] = theta^(-2k/r) this is
 * oracle_rope_vec. */
void oracle_rope_vec_table(double* x, int32_t r, const double* inv_freq, double p) {
    if (r == 0) return;
    int32_t half = r / 2;
    for (int32_t k = 0; k < half; ++k) {
        double phi = p * inv_freq[k];
        double c = cos(phi), s = sin(phi);
        double a = x[k], b = x[k + half];
        x[k] = a * c - b * s;
        x[k + half] = b * c + a * s;
    }
}

/* A layer's rotation: its frequency table if it has one, else theta. */
static void layer_rope(const oracle_layer* L, double* x, double p) {
    if (L->inv_freq)
        oracle_rope_vec_table(x, L->rotary_dim, L->inv_freq, p);
    else
        oracle_rope_vec(x, L->head_dim, L->rotary_dim, L->rope_theta, p);
}

/* RoPE with a frequency table over a bf16 tensor x[T, H, D] (token t at
 * position pos[t]); output out[T, H, D] in fp64. */
int oracle_rope_table(const uint16_t* x, int64_t T, int32_t H, int32_t D, const int64_t* pos,
                      const double* inv_freq, int32_t r, double* out) {
    if (!x || !pos || !out || !inv_freq || T < 0 || H <= 0 || D <= 0 || r < 0 || r > D || (r & 1))
        return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t h = 0; h < H; ++h) {
            double* y = out + (t * H + h) * (int64_t)D;
            const uint16_t* xs = x + (t * H + h) * (int64_t)D;
            for (int32_t d = 0; d < D; ++d) y[d] = bf16_bits_to_f64(xs[d]);
            oracle_rope_vec_table(y, r, inv_freq, (double)pos[t]);
        }
    }
    return ORACLE_OK;
}

/* RoPE over a bf16 tensor x[T, H, D] whose token t sits at position pos[t].
 * Output out[T, H, D] in fp64. */
int oracle_rope(const uint16_t* x, int64_t T, int32_t H, int32_t D, const int64_t* pos,
                double theta, int32_t r, double* out) {
    if (!x || !pos || !out || T < 0 || H <= 0 || D <= 0 || r < 0 || r > D || (r & 1))
        return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t h = 0; h < H; ++h) {
            double* y = out + (t * H + h) * (int64_t)D;
            const uint16_t* xs = x + (t * H + h) * (int64_t)D;
            for (int32_t d = 0; d < D; ++d) y[d] = bf16_bits_to_f64(xs[d]);
            oracle_rope_vec(y, D, r, theta, (double)pos[t]);
        }
    }
    return ORACLE_OK;
}

/* Whether key position j is visible to query position i (section 2.2 of the
 * Step explainer, reading i-W < j <= i; W = -1 is the plain causal mask). */
static int visible(int64_t i, int64_t j, int32_t W) {
    if (j > i) return 0;
    if (W < 0) return 1;
    return j > i - (int64_t)W;
}

static double sigmoid(double g) { return 1.0 / (1.0 + exp(-g)); }

/* One output row of masked softmax attention.  keys[n][D] are already
 * rotated, vals[n][D]; the row attends to all n given keys.  gate_logit
 * NULL => ungated.  Plain two-pass softmax: max, then normalised weights. */
static void attend_row(const double* q, const double* keys, const double* vals, int64_t n,
                       int32_t D, double scale, const float* gate_logit, double* out,
                       double* scratch /* n */) {
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        double s = 0.0;
        for (int32_t d = 0; d < D; ++d) s += q[d] * keys[j * D + d];
        s *= scale;
        scratch[j] = s;
        if (s > m) m = s;
    }
    double denom = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        scratch[j] = exp(scratch[j] - m);
        denom += scratch[j];
    }
    for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double w = scratch[j] / denom;
        for (int32_t d = 0; d < D; ++d) out[d] += w * vals[j * D + d];
    }
    if (gate_logit) {
        double g = sigmoid((double)*gate_logit);
        for (int32_t d = 0; d < D; ++d) out[d] *= g;
    }
}

/* Prefill attention at positions 0..S-1 on un-rotated bf16 q[B,S,Hq,D],
 * k[B,S,Hkv,D], v[B,S,Hkv,D]; gate[B,S,Hq] fp32 or NULL.
 * rows: n_rows (b, i, h) triples, or NULL for every row.  out: [n_rows, D]
 * when rows is given, else [B,S,Hq,D].  Keys are rotated once per
 * (b, kv-head) into an fp64 copy, then each requested row is computed from
 * the definition over its visible keys. */
int oracle_prefill(const oracle_layer* L, int32_t B, int32_t S, const uint16_t* q,
                   const uint16_t* k, const uint16_t* v, const float* gate, int64_t n_rows,
                   const int64_t* rows, double* out, int32_t n_threads) {
    if (!layer_ok(L) || B < 0 || S < 0 || !q || !k || !v || !out) return ORACLE_BAD_ARG;
    const int32_t Hq = L->num_q_heads, Hkv = L->num_kv_heads, D = L->head_dim;
    const int32_t G = Hq / Hkv;
    const double scale = layer_scale(L);
    const int64_t total = rows ? n_rows : (int64_t)B * S * Hq;
    if (rows) {
        for (int64_t t = 0; t < n_rows; ++t) {
            int64_t b = rows[3 * t], i = rows[3 * t + 1], h = rows[3 * t + 2];
            if (b < 0 || b >= B || i < 0 || i >= S || h < 0 || h >= Hq) return ORACLE_BAD_ARG;
        }
    }
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    double* krot = (double*)malloc(sizeof(double) * (size_t)S * D + 8);
    double* vd = (double*)malloc(sizeof(double) * (size_t)S * D + 8);
    if (!krot || !vd) { free(krot); free(vd); return ORACLE_NO_MEM; }

    for (int32_t b = 0; b < B; ++b) {
        for (int32_t kvh = 0; kvh < Hkv; ++kvh) {
            /* does any requested row use this (b, kv-head)? */
            int used = 0;
            for (int64_t t = 0; t < total && !used; ++t) {
                int64_t rb = rows ? rows[3 * t] : t / ((int64_t)S * Hq);
                int64_t rh = rows ? rows[3 * t + 2] : t % Hq;
                if (rb == b && rh / G == kvh) used = 1;
            }
            if (!used) continue;
#pragma omp parallel for schedule(static)
            for (int64_t j = 0; j < S; ++j) {
                const uint16_t* ks = k + (((int64_t)b * S + j) * Hkv + kvh) * D;
                const uint16_t* vs = v + (((int64_t)b * S + j) * Hkv + kvh) * D;
                for (int32_t d = 0; d < D; ++d) {
                    krot[j * D + d] = bf16_bits_to_f64(ks[d]);
                    vd[j * D + d] = bf16_bits_to_f64(vs[d]);
                }
                layer_rope(L, krot + j * D, (double)j);
            }
            int err = 0;
#pragma omp parallel
            {
                double* qv = (double*)malloc(sizeof(double) * D);
                double* sc = (double*)malloc(sizeof(double) * (size_t)S + 8);
                if (!qv || !sc) {
#pragma omp atomic write
                    err = 1;
                } else {
#pragma omp for schedule(dynamic, 16)
                    for (int64_t t = 0; t < total; ++t) {
                        int64_t rb, ri, rh;
                        if (rows) { rb = rows[3 * t]; ri = rows[3 * t + 1]; rh = rows[3 * t + 2]; }
                        else { rb = t / ((int64_t)S * Hq); ri = (t / Hq) % S; rh = t % Hq; }
                        if (rb != b || rh / G != kvh) continue;
                        const uint16_t* qs = q + ((rb * S + ri) * Hq + rh) * D;
                        for (int32_t d = 0; d < D; ++d) qv[d] = bf16_bits_to_f64(qs[d]);
                        layer_rope(L, qv, (double)ri);
                        /* the visible keys of row ri form the interval [j0, ri] */
                        int64_t j0 = (L->window > 0 && ri - (int64_t)L->window + 1 > 0)
                                         ? ri - (int64_t)L->window + 1 : 0;
                        int64_t n = ri - j0 + 1;
                        const float* g = gate ? gate + (rb * S + ri) * Hq + rh : NULL;
                        attend_row(qv, krot + j0 * D, vd + j0 * D, n, D, scale, g, out + t * D, sc);
                    }
                }
                free(qv);
                free(sc);
            }
            if (err) { free(krot); free(vd); return ORACLE_NO_MEM; }
        }
    }
    free(krot);
    free(vd);
    return ORACLE_OK;
}

/* Materialised variant for tiny inputs: for every (b, h) build the full
 * S x S score matrix with -inf outside the mask, softmax each row over all
 * S columns, then multiply by V.  weights (optional) receives the
 * [B, Hq, S, S] probability matrices. */
int oracle_prefill_materialised(const oracle_layer* L, int32_t B, int32_t S, const uint16_t* q,
                                const uint16_t* k, const uint16_t* v, const float* gate,
                                double* out, double* weights) {
    if (!layer_ok(L) || B < 0 || S < 0 || !q || !k || !v || !out) return ORACLE_BAD_ARG;
    const int32_t Hq = L->num_q_heads, Hkv = L->num_kv_heads, D = L->head_dim;
    const int32_t G = Hq / Hkv;
    const double scale = layer_scale(L);
    double* Qr = (double*)malloc(sizeof(double) * (size_t)S * D + 8);
    double* Kr = (double*)malloc(sizeof(double) * (size_t)S * D + 8);
    double* P = (double*)malloc(sizeof(double) * (size_t)S * S + 8);
    if (!Qr || !Kr || !P) { free(Qr); free(Kr); free(P); return ORACLE_NO_MEM; }
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t h = 0; h < Hq; ++h) {
            int32_t kvh = h / G;
            for (int32_t i = 0; i < S; ++i) {
                for (int32_t d = 0; d < D; ++d) {
                    Qr[(int64_t)i * D + d] = bf16_bits_to_f64(q[(((int64_t)b * S + i) * Hq + h) * D + d]);
                    Kr[(int64_t)i * D + d] = bf16_bits_to_f64(k[(((int64_t)b * S + i) * Hkv + kvh) * D + d]);
                }
                layer_rope(L, Qr + (int64_t)i * D, (double)i);
                layer_rope(L, Kr + (int64_t)i * D, (double)i);
            }
            /* scores with the mask as -inf */
            for (int32_t i = 0; i < S; ++i)
                for (int32_t j = 0; j < S; ++j) {
                    double s = 0.0;
                    for (int32_t d = 0; d < D; ++d) s += Qr[(int64_t)i * D + d] * Kr[(int64_t)j * D + d];
                    P[(int64_t)i * S + j] = visible(i, j, L->window) ? s * scale : -INFINITY;
                }
            /* row softmax over all S columns */
            for (int32_t i = 0; i < S; ++i) {
                double m = -INFINITY, z = 0.0;
                for (int32_t j = 0; j < S; ++j) if (P[(int64_t)i * S + j] > m) m = P[(int64_t)i * S + j];
                for (int32_t j = 0; j < S; ++j) {
                    double e = exp(P[(int64_t)i * S + j] - m);
                    P[(int64_t)i * S + j] = e;
                    z += e;
                }
                for (int32_t j = 0; j < S; ++j) P[(int64_t)i * S + j] /= z;
            }
            if (weights) memcpy(weights + ((int64_t)b * Hq + h) * S * S, P, sizeof(double) * (size_t)S * S);
            /* out = P @ V, then the gate */
            for (int32_t i = 0; i < S; ++i) {
                double* o = out + (((int64_t)b * S + i) * Hq + h) * D;
                for (int32_t d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int32_t j = 0; j < S; ++j)
                        acc += P[(int64_t)i * S + j] *
                               bf16_bits_to_f64(v[(((int64_t)b * S + j) * Hkv + kvh) * D + d]);
                    o[d] = acc;
                }
                if (gate) {
                    double g = sigmoid((double)gate[((int64_t)b * S + i) * Hq + h]);
                    for (int32_t d = 0; d < D; ++d) o[d] *= g;
                }
            }
        }
    }
    free(Qr);
    free(Kr);
    free(P);
    return ORACLE_OK;
}

/* Decode: one query per sequence at position L_b - 1, where L_b =
 * seq_lens[b] counts the current token.  q_rot[B,Hq,D] is the query after
 * RoPE (fp64).  The cache k_cache/v_cache [B,Hkv,C,D] bf16 holds rotated
 * keys and raw values.  On a sliding layer the cache is a ring of W slots
 * (slot = position mod W) and the visible keys are exactly the min(L_b, W)
 * filled slots; on a full layer slots 0..L_b-1 (Step explainer section 2.2:
 * each sliding layer keeps only the last W tokens).  k_new/v_new [B,Hkv,D]
 * (fp64, optional) replace the current token's slot, so the append step can
 * be checked without rounding the new key to bf16.
 * rows: n_rows (b, h) pairs or NULL for all; out [n_rows or B*Hq, D]. */
int oracle_decode(const oracle_layer* L, int32_t B, const double* q_rot, const float* gate,
                  const uint16_t* k_cache, const uint16_t* v_cache, int32_t C,
                  const int32_t* seq_lens, const double* k_new, const double* v_new,
                  int64_t n_rows, const int64_t* rows, double* out, int32_t n_threads) {
    if (!layer_ok(L) || B < 0 || !q_rot || !k_cache || !v_cache || !seq_lens || !out || C <= 0)
        return ORACLE_BAD_ARG;
    const int32_t Hq = L->num_q_heads, Hkv = L->num_kv_heads, D = L->head_dim;
    const int32_t G = Hq / Hkv;
    const double scale = layer_scale(L);
    for (int32_t b = 0; b < B; ++b) {
        if (seq_lens[b] < 1) return ORACLE_BAD_ARG;
        if (L->window < 0 && seq_lens[b] > C) return ORACLE_BAD_ARG;
        if (L->window > 0 && C != L->window) return ORACLE_BAD_ARG;
    }
    const int64_t total = rows ? n_rows : (int64_t)B * Hq;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    int err = 0;
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t kvh = 0; kvh < Hkv; ++kvh) {
            int used = 0;
            for (int64_t t = 0; t < total && !used; ++t) {
                int64_t rb = rows ? rows[2 * t] : t / Hq, rh = rows ? rows[2 * t + 1] : t % Hq;
                if (rb == b && rh / G == kvh) used = 1;
            }
            if (!used) continue;
            int64_t Lb = seq_lens[b];
            int64_t n = (L->window > 0 && Lb > L->window) ? L->window : Lb;
            int64_t cur_slot = (L->window > 0) ? (Lb - 1) % L->window : Lb - 1;
            double* kd = (double*)malloc(sizeof(double) * (size_t)n * D + 8);
            double* vd = (double*)malloc(sizeof(double) * (size_t)n * D + 8);
            if (!kd || !vd) { free(kd); free(vd); return ORACLE_NO_MEM; }
#pragma omp parallel for schedule(static)
            for (int64_t j = 0; j < n; ++j) {
                const uint16_t* ks = k_cache + (((int64_t)b * Hkv + kvh) * C + j) * D;
                const uint16_t* vs = v_cache + (((int64_t)b * Hkv + kvh) * C + j) * D;
                for (int32_t d = 0; d < D; ++d) {
                    kd[j * D + d] = bf16_bits_to_f64(ks[d]);
                    vd[j * D + d] = bf16_bits_to_f64(vs[d]);
                }
                if (j == cur_slot) {
                    if (k_new) for (int32_t d = 0; d < D; ++d) kd[j * D + d] = k_new[((int64_t)b * Hkv + kvh) * D + d];
                    if (v_new) for (int32_t d = 0; d < D; ++d) vd[j * D + d] = v_new[((int64_t)b * Hkv + kvh) * D + d];
                }
            }
#pragma omp parallel
            {
                double* sc = (double*)malloc(sizeof(double) * (size_t)n + 8);
                if (!sc) {
#pragma omp atomic write
                    err = 1;
                } else {
#pragma omp for schedule(dynamic, 1)
                    for (int64_t t = 0; t < total; ++t) {
                        int64_t rb = rows ? rows[2 * t] : t / Hq, rh = rows ? rows[2 * t + 1] : t % Hq;
                        if (rb != b || rh / G != kvh) continue;
                        const float* g = gate ? gate + rb * Hq + rh : NULL;
                        attend_row(q_rot + (rb * Hq + rh) * D, kd, vd, n, D, scale, g, out + t * D, sc);
                    }
                }
                free(sc);
            }
            free(kd);
            free(vd);
            if (err) return ORACLE_NO_MEM;
        }
    }
    return ORACLE_OK;
}

/* Same as oracle_decode but with an fp64 cache [B,Hkv,C,D]; for tiny
 * self-checks where the cache holds exact rotated keys. */
int oracle_decode_f64(const oracle_layer* L, int32_t B, const double* q_rot, const float* gate,
                      const double* k_cache, const double* v_cache, int32_t C,
                      const int32_t* seq_lens, double* out) {
    if (!layer_ok(L) || B < 0 || !q_rot || !k_cache || !v_cache || !seq_lens || !out || C <= 0)
        return ORACLE_BAD_ARG;
    const int32_t Hq = L->num_q_heads, Hkv = L->num_kv_heads, D = L->head_dim;
    const int32_t G = Hq / Hkv;
    const double scale = layer_scale(L);
    for (int32_t b = 0; b < B; ++b) {
        int64_t Lb = seq_lens[b];
        if (Lb < 1) return ORACLE_BAD_ARG;
        if (L->window < 0 && Lb > C) return ORACLE_BAD_ARG;
        if (L->window > 0 && C != L->window) return ORACLE_BAD_ARG;
        int64_t n = (L->window > 0 && Lb > L->window) ? L->window : Lb;
        double* sc = (double*)malloc(sizeof(double) * (size_t)n + 8);
        if (!sc) return ORACLE_NO_MEM;
        for (int32_t h = 0; h < Hq; ++h) {
            int32_t kvh = h / G;
            const double* kd = k_cache + ((int64_t)b * Hkv + kvh) * C * D;
            const double* vd = v_cache + ((int64_t)b * Hkv + kvh) * C * D;
            const float* g = gate ? gate + (int64_t)b * Hq + h : NULL;
            attend_row(q_rot + ((int64_t)b * Hq + h) * D, kd, vd, n, D, scale, g,
                       out + ((int64_t)b * Hq + h) * D, sc);
        }
        free(sc);
    }
    return ORACLE_OK;
}

/* Multi-query decode: T consecutive new tokens per sequence -- the Step spec
 * card's architecture notes list three extra multi-token-prediction (MTP)
 * layers that speed up decoding; the tokens they propose are checked by one
 * attention call -- at positions
 * L0 .. L0 + T - 1, where L0 = seq_lens[b] - T.  The cache holds only the
 * L0 earlier tokens (rotated keys, raw values): on a sliding layer a ring of
 * W slots with position p in slot p mod W, so the last min(L0, W) positions
 * are there (Step explainer section 2.2); on a full layer slots 0 .. L0 - 1.
 * The new tokens' rotated keys and raw values come separately, k_new/v_new
 * [B,T,Hkv,D] bf16 in position order.  Query t (position p = L0 + t) attends
 * to the keys at positions j with p - W < j <= p (W = -1: 0 <= j <= p) --
 * the band of every other query -- taking position j from the cache when
 * j < L0, else new token j - L0.
 * q_rot [B,T,Hq,D] fp64 (after RoPE); gate [B,T,Hq] or NULL;
 * rows: n_rows (b, t, h) triples or NULL for all; out [n_rows or B*T*Hq, D]. */
int oracle_decode_mq(const oracle_layer* L, int32_t B, int32_t T, const double* q_rot, const float* gate,
                     const uint16_t* k_cache, const uint16_t* v_cache, int32_t C, const int32_t* seq_lens,
                     const uint16_t* k_new, const uint16_t* v_new, int64_t n_rows, const int64_t* rows,
                     double* out, int32_t n_threads) {
    if (!layer_ok(L) || B < 0 || T < 1 || !q_rot || !k_cache || !v_cache || !seq_lens || !k_new || !v_new ||
        !out || C <= 0 || (rows && n_rows < 0))
        return ORACLE_BAD_ARG;
    const int32_t Hq = L->num_q_heads, Hkv = L->num_kv_heads, D = L->head_dim;
    const int32_t G = Hq / Hkv, W = L->window;
    const double scale = layer_scale(L);
    for (int32_t b = 0; b < B; ++b) {
        int64_t L0 = (int64_t)seq_lens[b] - T;
        if (L0 < 0) return ORACLE_BAD_ARG;
        if (W < 0 && L0 > C) return ORACLE_BAD_ARG;
        if (W > 0 && C != W) return ORACLE_BAD_ARG;
    }
    const int64_t total = rows ? n_rows : (int64_t)B * T * Hq;
    for (int64_t r = 0; rows && r < total; ++r)
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= T ||
            rows[3 * r + 2] < 0 || rows[3 * r + 2] >= Hq)
            return ORACLE_BAD_ARG;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    int err = 0;
#pragma omp parallel
    {
        double* kd = NULL;
        double* vd = NULL;
        double* sc = NULL;
        int64_t cap = 0;
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < total; ++r) {
            const int64_t b = rows ? rows[3 * r] : r / ((int64_t)T * Hq);
            const int64_t t = rows ? rows[3 * r + 1] : (r / Hq) % T;
            const int64_t h = rows ? rows[3 * r + 2] : r % Hq;
            const int64_t kvh = h / G;
            const int64_t L0 = (int64_t)seq_lens[b] - T, p = L0 + t;
            int64_t lo = 0;
            for (; lo <= p && !visible(p, lo, W); ++lo) {
            }
            const int64_t n = p - lo + 1;
            if (n > cap) {
                free(kd); free(vd); free(sc);
                kd = (double*)malloc(sizeof(double) * (size_t)n * D);
                vd = (double*)malloc(sizeof(double) * (size_t)n * D);
                sc = (double*)malloc(sizeof(double) * (size_t)n);
                cap = (kd && vd && sc) ? n : 0;
            }
            if (!cap) {
#pragma omp atomic write
                err = 1;
                continue;
            }
            for (int64_t j = lo; j <= p; ++j) {
                const uint16_t *ks, *vs;
                if (j < L0) {
                    const int64_t slot = W > 0 ? j % W : j;
                    ks = k_cache + ((b * Hkv + kvh) * C + slot) * D;
                    vs = v_cache + ((b * Hkv + kvh) * C + slot) * D;
                } else {
                    ks = k_new + ((b * T + (j - L0)) * Hkv + kvh) * D;
                    vs = v_new + ((b * T + (j - L0)) * Hkv + kvh) * D;
                }
                for (int32_t d = 0; d < D; ++d) {
                    kd[(j - lo) * D + d] = bf16_bits_to_f64(ks[d]);
                    vd[(j - lo) * D + d] = bf16_bits_to_f64(vs[d]);
                }
            }
            const float* g = gate ? gate + (b * T + t) * Hq + h : NULL;
            attend_row(q_rot + ((b * T + t) * Hq + h) * D, kd, vd, n, D, scale, g, out + r * D, sc);
        }
        free(kd); free(vd); free(sc);
    }
    return err ? ORACLE_NO_MEM : ORACLE_OK;
}

/* KV-cache footprint in bytes: tokens x kv-heads x head_dim x (K and V) x
 * bytes per element, summed over layers (Muse explainer, GQA section). */
int64_t oracle_kv_cache_bytes(int64_t tokens, int32_t kv_heads, int32_t head_dim,
                              int32_t bytes_per_elem, int32_t layers) {
    return tokens * (int64_t)kv_heads * head_dim * 2 * bytes_per_elem * layers;
}

/* Visible key count for a query at position i under window W (W = -1:
 * full), from the mask definition; used by the uniform-score checks. */
int64_t oracle_visible_count(int64_t i, int32_t W) {
    int64_t c = 0;
    for (int64_t j = 0; j <= i; ++j) c += visible(i, j, W);
    return c;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
