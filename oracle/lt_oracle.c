/*
 * lt_oracle.c -- plain fp64 CPU oracle for kernelised (linear) attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file or the library built from it; only the test suite, the
 * package's smoke check and the benchmark's CPU-baseline leg use it.  It
 * shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (sources, by page and section):
 *   - "lineartile 1.0.0" (PyPI page), section "How It Works": the feature map
 *     phi(x) = ELU(x) + 1 and the reordered non-causal product
 *     phi(Q) (phi(K)^T V), i.e. compute phi(K)^T V first.
 *   - same page, section "Reference": the method is the linear attention of
 *     "Transformers are RNNs" (Katharopoulos et al., 2020): causal output
 *         O_i = phi(Q_i) S_i / (phi(Q_i) . z_i + eps),
 *         S_i = sum_{j<=i} phi(K_j)^T V_j,   z_i = sum_{j<=i} phi(K_j),
 *     which can be evaluated either as a masked quadratic form or as a
 *     recurrence over a fixed-size state (the "RNN view").
 *   - same page, section "Features": variable sequence length (packed
 *     sequences, no padding), grouped-query attention, KV-cache reuse
 *     (for linear attention the cache is the fixed-size (S, z) state).
 *   - "Why Stream Wins at Ultra-Long Context", section 4.2: the forward
 *     linear recurrence h_t = h_{t-1} a_t + b_t, here with a_t = 1 and
 *     b_t = phi(K_t)^T V_t.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   ELU alpha = 1; no 1/sqrt(d) score scale inside the method; eps is added
 *   to the denominator only; the causal sum is inclusive (j <= i); the
 *   non-causal mode returns the same normalised form with the sum over all
 *   j; query head h uses KV head floor(h * H_kv / H_q); token-major layouts
 *   [B][N][H][d] (dense) and [N_total][H][d] (packed, cu_seqlens).
 *
 * Every input is widened exactly to double before any arithmetic: bf16 and
 * fp32 values are exactly representable in fp64, so the oracle sees the very
 * values the GPU sees.  All arithmetic is fp64.
 *
 * Backward pass (the gradient of the forward above with respect to Q, K, V
 * for an upstream gradient dO): the "lineartile 1.0.0" page lists one
 * ("Project Structure": core/kernels/backward.py, tests/test_backward) but
 * prints no formula; "Why Stream Wins at Ultra-Long Context", section 4.2,
 * gives the reverse recurrence of a linear scan's backward pass.  Two
 * independent forms below: the quadratic definition differentiated term by
 * term, and a forward recurrence (for dQ) plus a reverse recurrence (for dK,
 * dV) over the state.
 *
 * Pins (tests in tests/test_oracle_pins.py): a hand-worked 2x2 example,
 * agreement of the two independent forms, associativity of the non-causal
 * product, closed forms (constant keys -> prefix mean of V), invariants
 * (denominator > 0, implied weights sum to 1 - eps/den), GQA == explicit KV
 * replication, packed == independent per-sequence calls, decode chaining ==
 * quadratic causal form.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* element type codes for the raw input buffers */
#define ORC_F32 0
#define ORC_BF16 1
#define ORC_F64 2
#define ORC_F16 3

/* IEEE binary16 bits -> double, exactly: sign, 5-bit exponent (bias 15),
 * 10-bit fraction; exponent 0 holds the subnormals, 31 infinities and NaN. */
static double half_to_double(uint16_t h) {
    const int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double x;
    if (e == 0) x = ldexp((double)m, -24);
    else if (e == 31) x = m ? NAN : INFINITY;
    else x = ldexp(1024.0 + m, e - 25);
    return sign ? -x : x;
}

/* Read element idx of a raw buffer of the given type, widened to double. */
static double load_elem(const void *p, int64_t idx, int type) {
    if (type == ORC_F64) return ((const double *)p)[idx];
    if (type == ORC_F32) return (double)((const float *)p)[idx];
    if (type == ORC_F16) return half_to_double(((const uint16_t *)p)[idx]);
    /* bf16: the 16 stored bits are the high half of an IEEE binary32 */
    uint32_t bits = (uint32_t)((const uint16_t *)p)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* The feature map.  Kind 0, the method's: phi(x) = ELU(x) + 1 with alpha =
 * 1, i.e. x + 1 for x > 0 and exp(x) for x <= 0.  The "lineartile 1.0.0"
 * page's "Features" list lets the map be replaced; the other maps the CUDA
 * library offers are kind 1, ReLU: max(x, 0), and kind 2, exp(x).  The kind
 * in force is set by lt_oracle_set_phi (default 0); the backward forms
 * support kind 0 only. */
static int g_phi_kind = 0;

int lt_oracle_set_phi(int kind) {
    if (kind < 0 || kind > 2) return 1;
    g_phi_kind = kind;
    return 0;
}

static double phi_elu1(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

double lt_oracle_phi(double x) {
    if (g_phi_kind == 1) return x > 0.0 ? x : 0.0;
    if (g_phi_kind == 2) return exp(x);
    return phi_elu1(x);
}

int lt_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sequence geometry: start token (in the packed/dense token index space of
 * one batch row) and length.  Dense mode: every sequence has N tokens and
 * lives in its own batch row; packed mode: one batch row, offsets from
 * cu_seqlens. */
static void seq_range(int s, int N, const int32_t *cu, int64_t *base_tok, int64_t *len) {
    if (cu) {
        *base_tok = cu[s];
        *len = (int64_t)cu[s + 1] - cu[s];
    } else {
        *base_tok = (int64_t)s * N;
        *len = N;
    }
}

/* Flat offset of element c of row (token t, head h) in a token-major tensor
 * whose rows have H heads of width w.  t is the global token index
 * (b*N + n in dense mode, the packed index in packed mode). */
static int64_t off(int64_t t, int h, int H, int w, int c) {
    return ((t * H + h) * (int64_t)w) + c;
}

static int check_args(int B, int Hq, int Hkv, int N, int d, int dv, double eps) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || dv <= 0) return 1;
    if (Hq % Hkv != 0) return 1;
    if (!(eps >= 0.0)) return 1;
    return 0;
}

/*
 * Form 1: the masked quadratic form, straight from the definition.
 * For each sequence, query head h (KV head g = h*Hkv/Hq) and query i:
 *     a_ij = phi(Q_i) . phi(K_j)       for j <= i (all j when causal == 0)
 *     O_i  = (sum_j a_ij V_j) / (sum_j a_ij + eps)
 * O(n^2) per sequence: use only for small n.
 */
int lt_oracle_fwd_quadratic(const void *q, const void *k, const void *v, int in_type,
                            double *out, int B, int Hq, int Hkv, int N, int d, int dv,
                            int causal, double eps, const int32_t *cu_seqlens) {
    if (check_args(B, Hq, Hkv, N, d, dv, eps)) return 1;
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < B; ++s) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            int64_t t0, n;
            seq_range(s, N, cu_seqlens, &t0, &n);
            double *pq = malloc(sizeof(double) * d);
            double *pk = malloc(sizeof(double) * d);
            double *num = malloc(sizeof(double) * dv);
            for (int64_t i = 0; i < n; ++i) {
                for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
                for (int c = 0; c < dv; ++c) num[c] = 0.0;
                double den = 0.0;
                const int64_t jend = causal ? i + 1 : n;
                for (int64_t j = 0; j < jend; ++j) {
                    for (int c = 0; c < d; ++c) pk[c] = lt_oracle_phi(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
                    double a = 0.0;
                    for (int c = 0; c < d; ++c) a += pq[c] * pk[c];
                    for (int c = 0; c < dv; ++c) num[c] += a * load_elem(v, off(t0 + j, g, Hkv, dv, c), in_type);
                    den += a;
                }
                for (int c = 0; c < dv; ++c) out[off(t0 + i, h, Hq, dv, c)] = num[c] / (den + eps);
            }
            free(pq);
            free(pk);
            free(num);
        }
    }
    return 0;
}

/*
 * Form 2: the recurrence over the fixed-size state (the RNN view).
 *     S <- S0 (d x dv), z <- z0 (d)          (zero unless a state is given)
 *     for i = 0..n-1:  S += phi(K_i)^T V_i;  z += phi(K_i);
 *                      O_i = phi(Q_i) S / (phi(Q_i) . z + eps)
 * Non-causal: run the state update over the whole sequence first, then
 * evaluate every O_i with the final (S, z).
 * With S0/z0 the sequence continues from that state: the "RNN view" of the
 * "Reference" section and the KV-cache reuse of "Features" (the cache is
 * the state), so splitting a sequence and carrying (S, z) across the split
 * reproduces the unsplit output.  S0, S_out: [B][Hkv][d][dv]; z0, z_out:
 * [B][Hkv][d] (one state per sequence and KV head); any may be NULL.
 * S_out/z_out receive the state after the sequence's last token.
 */
static int recurrent_impl(const void *q, const void *k, const void *v, int in_type,
                          double *out, int B, int Hq, int Hkv, int N, int d, int dv,
                          int causal, double eps, const int32_t *cu_seqlens,
                          const double *S0, const double *z0, double *S_out, double *z_out) {
    if (check_args(B, Hq, Hkv, N, d, dv, eps)) return 1;
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < B; ++s) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            int64_t t0, n;
            seq_range(s, N, cu_seqlens, &t0, &n);
            double *S = calloc((size_t)d * dv, sizeof(double));
            double *z = calloc((size_t)d, sizeof(double));
            double *pq = malloc(sizeof(double) * d);
            double *pk = malloc(sizeof(double) * d);
            double *vv = malloc(sizeof(double) * dv);
            const int64_t sg = (int64_t)s * Hkv + g;  /* this (sequence, KV head) state */
            if (S0) memcpy(S, S0 + sg * d * dv, sizeof(double) * d * dv);
            if (z0) memcpy(z, z0 + sg * d, sizeof(double) * d);
            if (!causal) {
                for (int64_t i = 0; i < n; ++i) {
                    for (int c = 0; c < d; ++c) pk[c] = lt_oracle_phi(load_elem(k, off(t0 + i, g, Hkv, d, c), in_type));
                    for (int c = 0; c < dv; ++c) vv[c] = load_elem(v, off(t0 + i, g, Hkv, dv, c), in_type);
                    for (int a = 0; a < d; ++a) {
                        for (int c = 0; c < dv; ++c) S[a * dv + c] += pk[a] * vv[c];
                        z[a] += pk[a];
                    }
                }
            }
            for (int64_t i = 0; i < n; ++i) {
                if (causal) {
                    for (int c = 0; c < d; ++c) pk[c] = lt_oracle_phi(load_elem(k, off(t0 + i, g, Hkv, d, c), in_type));
                    for (int c = 0; c < dv; ++c) vv[c] = load_elem(v, off(t0 + i, g, Hkv, dv, c), in_type);
                    for (int a = 0; a < d; ++a) {
                        for (int c = 0; c < dv; ++c) S[a * dv + c] += pk[a] * vv[c];
                        z[a] += pk[a];
                    }
                }
                for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
                double den = eps;
                for (int a = 0; a < d; ++a) den += pq[a] * z[a];
                for (int c = 0; c < dv; ++c) {
                    double num = 0.0;
                    for (int a = 0; a < d; ++a) num += pq[a] * S[a * dv + c];
                    out[off(t0 + i, h, Hq, dv, c)] = num / den;
                }
            }
            if (h % G == 0) {  /* one query head per group writes the group's state */
                if (S_out) memcpy(S_out + sg * d * dv, S, sizeof(double) * d * dv);
                if (z_out) memcpy(z_out + sg * d, z, sizeof(double) * d);
            }
            free(S);
            free(z);
            free(pq);
            free(pk);
            free(vv);
        }
    }
    return 0;
}

int lt_oracle_fwd_recurrent(const void *q, const void *k, const void *v, int in_type,
                            double *out, int B, int Hq, int Hkv, int N, int d, int dv,
                            int causal, double eps, const int32_t *cu_seqlens) {
    return recurrent_impl(q, k, v, in_type, out, B, Hq, Hkv, N, d, dv, causal, eps, cu_seqlens,
                          NULL, NULL, NULL, NULL);
}

/* The forward pass continued from a given state and returning the final
 * state (either may be NULL): form 2 with S0/z0 and S_out/z_out. */
int lt_oracle_fwd_state(const void *q, const void *k, const void *v, int in_type,
                        double *out, int B, int Hq, int Hkv, int N, int d, int dv,
                        int causal, double eps, const int32_t *cu_seqlens,
                        const double *S0, const double *z0, double *S_out, double *z_out) {
    return recurrent_impl(q, k, v, in_type, out, B, Hq, Hkv, N, d, dv, causal, eps, cu_seqlens,
                          S0, z0, S_out, z_out);
}

/*
 * Selected output rows by the quadratic definition, for checking outputs of
 * very long sequences without evaluating every row.  rows holds nrows
 * triples (sequence s, position i within the sequence, query head h);
 * out_rows receives nrows x dv values.  Cost per row: O(i * (d + dv)).
 */
int lt_oracle_fwd_rows(const void *q, const void *k, const void *v, int in_type,
                       int B, int Hq, int Hkv, int N, int d, int dv, int causal, double eps,
                       const int32_t *cu_seqlens, const int64_t *rows, int nrows, double *out_rows) {
    if (check_args(B, Hq, Hkv, N, d, dv, eps)) return 1;
    const int G = Hq / Hkv;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < nrows; ++r) {
        const int s = (int)rows[3 * r + 0];
        const int64_t i = rows[3 * r + 1];
        const int h = (int)rows[3 * r + 2];
        int64_t t0, n;
        if (s < 0 || s >= B || h < 0 || h >= Hq) { bad = 1; continue; }
        seq_range(s, N, cu_seqlens, &t0, &n);
        if (i < 0 || i >= n) { bad = 1; continue; }
        const int g = h / G;
        double *pq = malloc(sizeof(double) * d);
        double *num = calloc((size_t)dv, sizeof(double));
        for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
        double den = 0.0;
        const int64_t jend = causal ? i + 1 : n;
        for (int64_t j = 0; j < jend; ++j) {
            double a = 0.0;
            for (int c = 0; c < d; ++c) a += pq[c] * lt_oracle_phi(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
            for (int c = 0; c < dv; ++c) num[c] += a * load_elem(v, off(t0 + j, g, Hkv, dv, c), in_type);
            den += a;
        }
        for (int c = 0; c < dv; ++c) out_rows[(int64_t)r * dv + c] = num[c] / (den + eps);
        free(pq);
        free(num);
    }
    return bad;
}

/*
 * The unnormalised non-causal product of the "How It Works" section,
 * evaluated in either association order:
 *   order 0:  (phi(Q) phi(K)^T) V      -- scores first, O(n^2)
 *   order 1:  phi(Q) (phi(K)^T V)      -- key/value product first, O(n)
 * Mathematically identical; used to pin associativity.  Dense or packed.
 */
int lt_oracle_noncausal_numerator(const void *q, const void *k, const void *v, int in_type,
                                  double *out, int B, int Hq, int Hkv, int N, int d, int dv,
                                  const int32_t *cu_seqlens, int order) {
    if (check_args(B, Hq, Hkv, N, d, dv, 0.0)) return 1;
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < B; ++s) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            int64_t t0, n;
            seq_range(s, N, cu_seqlens, &t0, &n);
            double *pq = malloc(sizeof(double) * d);
            double *pk = malloc(sizeof(double) * d);
            double *KV = calloc((size_t)d * dv, sizeof(double));
            if (order == 1) {
                for (int64_t j = 0; j < n; ++j) {
                    for (int c = 0; c < d; ++c) pk[c] = lt_oracle_phi(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
                    for (int a = 0; a < d; ++a)
                        for (int c = 0; c < dv; ++c)
                            KV[a * dv + c] += pk[a] * load_elem(v, off(t0 + j, g, Hkv, dv, c), in_type);
                }
            }
            for (int64_t i = 0; i < n; ++i) {
                for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
                for (int c = 0; c < dv; ++c) {
                    double acc = 0.0;
                    if (order == 1) {
                        for (int a = 0; a < d; ++a) acc += pq[a] * KV[a * dv + c];
                    }
                    out[off(t0 + i, h, Hq, dv, c)] = acc;
                }
                if (order == 0) {
                    for (int64_t j = 0; j < n; ++j) {
                        double a = 0.0;
                        for (int c = 0; c < d; ++c) a += pq[c] * lt_oracle_phi(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
                        for (int c = 0; c < dv; ++c)
                            out[off(t0 + i, h, Hq, dv, c)] += a * load_elem(v, off(t0 + j, g, Hkv, dv, c), in_type);
                    }
                }
            }
            free(pq);
            free(pk);
            free(KV);
        }
    }
    return 0;
}

/*
 * One recurrent decode step (the fixed-size state standing in for a KV
 * cache).  For each batch row b and KV head g:
 *     S[b][g] += phi(k)^T v,  z[b][g] += phi(k)        (update first: j <= i)
 * then for every query head h of the group:
 *     out[b][h] = phi(q[b][h]) S[b][g] / (phi(q[b][h]) . z[b][g] + eps)
 * q [B][Hq][d], k [B][Hkv][d], v [B][Hkv][dv] (raw, in_type);
 * S [B][Hkv][d][dv], z [B][Hkv][d] fp64 in/out; out [B][Hq][dv] fp64.
 */
int lt_oracle_decode_step(const void *q, const void *k, const void *v, int in_type,
                          double *S, double *z, double *out, int B, int Hq, int Hkv, int d,
                          int dv, double eps) {
    if (check_args(B, Hq, Hkv, 1, d, dv, eps)) return 1;
    const int G = Hq / Hkv;
    for (int b = 0; b < B; ++b) {
        for (int g = 0; g < Hkv; ++g) {
            double *Sg = S + ((int64_t)b * Hkv + g) * d * dv;
            double *zg = z + ((int64_t)b * Hkv + g) * d;
            for (int a = 0; a < d; ++a) {
                const double pk = lt_oracle_phi(load_elem(k, ((int64_t)b * Hkv + g) * d + a, in_type));
                for (int c = 0; c < dv; ++c)
                    Sg[a * dv + c] += pk * load_elem(v, ((int64_t)b * Hkv + g) * dv + c, in_type);
                zg[a] += pk;
            }
        }
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            const double *Sg = S + ((int64_t)b * Hkv + g) * d * dv;
            const double *zg = z + ((int64_t)b * Hkv + g) * d;
            double den = eps;
            for (int a = 0; a < d; ++a)
                den += lt_oracle_phi(load_elem(q, ((int64_t)b * Hq + h) * d + a, in_type)) * zg[a];
            for (int c = 0; c < dv; ++c) {
                double num = 0.0;
                for (int a = 0; a < d; ++a)
                    num += lt_oracle_phi(load_elem(q, ((int64_t)b * Hq + h) * d + a, in_type)) * Sg[a * dv + c];
                out[((int64_t)b * Hq + h) * dv + c] = num / den;
            }
        }
    }
    return 0;
}

/* phi'(x): 1 for x > 0, e^x for x <= 0 (both give 1 at x = 0). */
static double phi_prime(double x) { return x > 0.0 ? 1.0 : exp(x); }

/*
 * Backward pass, form 1: the quadratic definition differentiated.  With
 * a_ij = phi(Q_i).phi(K_j) over the kept pairs (j <= i causal, all j
 * otherwise), den_i = sum_j a_ij + eps and O_i = sum_j a_ij V_j / den_i, an
 * upstream gradient dO gives
 *     g_i = dO_i / den_i,   h_i = -(dO_i . O_i) / den_i,
 *     da_ij = g_i . V_j + h_i,
 *     dphi(Q_i) = sum_j da_ij phi(K_j),   dphi(K_j) = sum_i da_ij phi(Q_i),
 *     dV_j = sum_i a_ij g_i,
 *     dQ = dphi(Q) * phi'(Q),   dK = dphi(K) * phi'(K)   (elementwise).
 * A KV head's dK, dV sum the contributions of every query head of its group.
 * dq [.][Hq][d], dk [.][Hkv][d], dv [.][Hkv][dv] fp64 (overwritten).
 */
int lt_oracle_bwd_quadratic(const void *q, const void *k, const void *v, const void *dout,
                            int in_type, double *dq, double *dk, double *dv, int B, int Hq,
                            int Hkv, int N, int d, int dvw, int causal, double eps,
                            const int32_t *cu_seqlens) {
    if (check_args(B, Hq, Hkv, N, d, dvw, eps) || g_phi_kind != 0) return 1;
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < B; ++s) {
        for (int g = 0; g < Hkv; ++g) {
            int64_t t0, n;
            seq_range(s, N, cu_seqlens, &t0, &n);
            double *pq = malloc(sizeof(double) * d), *pk = malloc(sizeof(double) * d);
            double *o = malloc(sizeof(double) * dvw), *gi = malloc(sizeof(double) * dvw);
            for (int64_t j = 0; j < n; ++j) {
                for (int c = 0; c < d; ++c) dk[off(t0 + j, g, Hkv, d, c)] = 0.0;
                for (int c = 0; c < dvw; ++c) dv[off(t0 + j, g, Hkv, dvw, c)] = 0.0;
            }
            for (int h = g * G; h < (g + 1) * G; ++h) {
                for (int64_t i = 0; i < n; ++i) {
                    for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
                    const int64_t jend = causal ? i + 1 : n;
                    /* the forward row: den_i and O_i */
                    double den = eps;
                    for (int c = 0; c < dvw; ++c) o[c] = 0.0;
                    for (int64_t j = 0; j < jend; ++j) {
                        double a = 0.0;
                        for (int c = 0; c < d; ++c) a += pq[c] * lt_oracle_phi(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
                        den += a;
                        for (int c = 0; c < dvw; ++c) o[c] += a * load_elem(v, off(t0 + j, g, Hkv, dvw, c), in_type);
                    }
                    double go = 0.0;
                    for (int c = 0; c < dvw; ++c) {
                        o[c] /= den;
                        gi[c] = load_elem(dout, off(t0 + i, h, Hq, dvw, c), in_type) / den;
                        go += load_elem(dout, off(t0 + i, h, Hq, dvw, c), in_type) * o[c];
                    }
                    const double hi = -go / den;
                    /* the gradient terms of every kept pair (i, j) */
                    for (int c = 0; c < d; ++c) dq[off(t0 + i, h, Hq, d, c)] = 0.0;
                    for (int64_t j = 0; j < jend; ++j) {
                        double a = 0.0, gv = 0.0;
                        for (int c = 0; c < d; ++c) {
                            pk[c] = lt_oracle_phi(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
                            a += pq[c] * pk[c];
                        }
                        for (int c = 0; c < dvw; ++c) gv += gi[c] * load_elem(v, off(t0 + j, g, Hkv, dvw, c), in_type);
                        const double da = gv + hi;
                        for (int c = 0; c < d; ++c) {
                            dq[off(t0 + i, h, Hq, d, c)] += da * pk[c];
                            dk[off(t0 + j, g, Hkv, d, c)] += da * pq[c];
                        }
                        for (int c = 0; c < dvw; ++c) dv[off(t0 + j, g, Hkv, dvw, c)] += a * gi[c];
                    }
                    for (int c = 0; c < d; ++c)
                        dq[off(t0 + i, h, Hq, d, c)] *= phi_prime(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
                }
            }
            for (int64_t j = 0; j < n; ++j)
                for (int c = 0; c < d; ++c)
                    dk[off(t0 + j, g, Hkv, d, c)] *= phi_prime(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
            free(pq); free(pk); free(o); free(gi);
        }
    }
    return 0;
}

/*
 * Backward pass, form 2: recurrences over the state.  Per query head:
 *   forward, i = 0..n-1 (causal; non-causal uses the final sums for every i):
 *     S += phi(K_i)^T V_i,  z += phi(K_i)   (the forward pass's state)
 *     O_i, den_i from phi(Q_i), S, z;  g_i, h_i as in form 1
 *     dphi(Q_i) = S g_i + z h_i
 *   reverse, j = n-1..0 (the backward recurrence of a linear scan):
 *     R += phi(Q_j) g_j^T,  r += phi(Q_j) h_j     (sums over i >= j)
 *     dphi(K_j) = R V_j + r,   dV_j = R^T phi(K_j)
 *   (non-causal: R, r summed over the whole sequence before any j).
 * Same outputs as form 1.
 */
int lt_oracle_bwd_recurrent(const void *q, const void *k, const void *v, const void *dout,
                            int in_type, double *dq, double *dk, double *dv, int B, int Hq,
                            int Hkv, int N, int d, int dvw, int causal, double eps,
                            const int32_t *cu_seqlens) {
    if (check_args(B, Hq, Hkv, N, d, dvw, eps) || g_phi_kind != 0) return 1;
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < B; ++s) {
        for (int g = 0; g < Hkv; ++g) {
            int64_t t0, n;
            seq_range(s, N, cu_seqlens, &t0, &n);
            double *S = malloc(sizeof(double) * d * dvw), *z = malloc(sizeof(double) * d);
            double *R = malloc(sizeof(double) * d * dvw), *r = malloc(sizeof(double) * d);
            double *pq = malloc(sizeof(double) * d), *pk = malloc(sizeof(double) * d);
            double *vv = malloc(sizeof(double) * dvw), *o = malloc(sizeof(double) * dvw);
            double *gs = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * dvw);
            double *hs = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
            for (int64_t j = 0; j < n; ++j) {
                for (int c = 0; c < d; ++c) dk[off(t0 + j, g, Hkv, d, c)] = 0.0;
                for (int c = 0; c < dvw; ++c) dv[off(t0 + j, g, Hkv, dvw, c)] = 0.0;
            }
            for (int h = g * G; h < (g + 1) * G; ++h) {
                /* forward recurrence: O_i, den_i, g_i, h_i and dphi(Q_i) */
                memset(S, 0, sizeof(double) * d * dvw);
                memset(z, 0, sizeof(double) * d);
                for (int pass = causal ? 1 : 0; pass < 2; ++pass) {
                    for (int64_t i = 0; i < n; ++i) {
                        if (pass == 0 || causal) {
                            for (int c = 0; c < d; ++c) pk[c] = lt_oracle_phi(load_elem(k, off(t0 + i, g, Hkv, d, c), in_type));
                            for (int c = 0; c < dvw; ++c) vv[c] = load_elem(v, off(t0 + i, g, Hkv, dvw, c), in_type);
                            for (int a = 0; a < d; ++a) {
                                for (int c = 0; c < dvw; ++c) S[a * dvw + c] += pk[a] * vv[c];
                                z[a] += pk[a];
                            }
                        }
                        if (pass == 0) continue;  /* non-causal: the sums first */
                        for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
                        double den = eps;
                        for (int a = 0; a < d; ++a) den += pq[a] * z[a];
                        double go = 0.0;
                        for (int c = 0; c < dvw; ++c) {
                            double num = 0.0;
                            for (int a = 0; a < d; ++a) num += pq[a] * S[a * dvw + c];
                            o[c] = num / den;
                            const double d_o = load_elem(dout, off(t0 + i, h, Hq, dvw, c), in_type);
                            gs[i * dvw + c] = d_o / den;
                            go += d_o * o[c];
                        }
                        hs[i] = -go / den;
                        for (int a = 0; a < d; ++a) {
                            double acc = z[a] * hs[i];
                            for (int c = 0; c < dvw; ++c) acc += S[a * dvw + c] * gs[i * dvw + c];
                            dq[off(t0 + i, h, Hq, d, a)] =
                                acc * phi_prime(load_elem(q, off(t0 + i, h, Hq, d, a), in_type));
                        }
                    }
                }
                /* reverse recurrence: dphi(K_j) and dV_j */
                memset(R, 0, sizeof(double) * d * dvw);
                memset(r, 0, sizeof(double) * d);
                for (int pass = causal ? 1 : 0; pass < 2; ++pass) {
                    for (int64_t j = n - 1; j >= 0; --j) {
                        if (pass == 0 || causal) {
                            for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + j, h, Hq, d, c), in_type));
                            for (int a = 0; a < d; ++a) {
                                for (int c = 0; c < dvw; ++c) R[a * dvw + c] += pq[a] * gs[j * dvw + c];
                                r[a] += pq[a] * hs[j];
                            }
                        }
                        if (pass == 0) continue;
                        for (int c = 0; c < d; ++c) pk[c] = lt_oracle_phi(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
                        for (int c = 0; c < dvw; ++c) vv[c] = load_elem(v, off(t0 + j, g, Hkv, dvw, c), in_type);
                        for (int a = 0; a < d; ++a) {
                            double acc = r[a];
                            for (int c = 0; c < dvw; ++c) acc += R[a * dvw + c] * vv[c];
                            dk[off(t0 + j, g, Hkv, d, a)] += acc;
                        }
                        for (int c = 0; c < dvw; ++c) {
                            double acc = 0.0;
                            for (int a = 0; a < d; ++a) acc += R[a * dvw + c] * pk[a];
                            dv[off(t0 + j, g, Hkv, dvw, c)] += acc;
                        }
                    }
                }
            }
            for (int64_t j = 0; j < n; ++j)
                for (int c = 0; c < d; ++c)
                    dk[off(t0 + j, g, Hkv, d, c)] *= phi_prime(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
            free(S); free(z); free(R); free(r); free(pq); free(pk); free(vv); free(o); free(gs); free(hs);
        }
    }
    return 0;
}

/*
 * Sliding-window causal attention ("lineartile 1.0.0", "Features": sliding
 * window attention).  Read plainly for linear attention: row i attends to
 * the w most recent keys, i - w < j <= i, i.e. the state S_i - S_{i-w}:
 *     O_i = phi(Q_i) (S_i - S_{i-w}) / (phi(Q_i) . (z_i - z_{i-w}) + eps)
 * with S_m = z_m = 0 for m < 0.  w >= 1; w >= n is the causal form.
 *
 * Form 1 (quadratic): the masked definition with the window.
 */
int lt_oracle_fwd_window_quadratic(const void *q, const void *k, const void *v, int in_type,
                                   double *out, int B, int Hq, int Hkv, int N, int d, int dv,
                                   int window, double eps, const int32_t *cu_seqlens) {
    if (check_args(B, Hq, Hkv, N, d, dv, eps) || window < 1) return 1;
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < B; ++s) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            int64_t t0, n;
            seq_range(s, N, cu_seqlens, &t0, &n);
            double *pq = malloc(sizeof(double) * d), *num = malloc(sizeof(double) * dv);
            for (int64_t i = 0; i < n; ++i) {
                for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
                for (int c = 0; c < dv; ++c) num[c] = 0.0;
                double den = 0.0;
                const int64_t jbeg = i - window + 1 > 0 ? i - window + 1 : 0;
                for (int64_t j = jbeg; j <= i; ++j) {
                    double a = 0.0;
                    for (int c = 0; c < d; ++c) a += pq[c] * lt_oracle_phi(load_elem(k, off(t0 + j, g, Hkv, d, c), in_type));
                    for (int c = 0; c < dv; ++c) num[c] += a * load_elem(v, off(t0 + j, g, Hkv, dv, c), in_type);
                    den += a;
                }
                for (int c = 0; c < dv; ++c) out[off(t0 + i, h, Hq, dv, c)] = num[c] / (den + eps);
            }
            free(pq);
            free(num);
        }
    }
    return 0;
}

/*
 * Form 2 (recurrences): the prefix state S, z and a second state S', z'
 * that follows w tokens behind (token i - w is added to it at step i), so
 * that S - S' is the window's state:
 *     S += phi(K_i)^T V_i, z += phi(K_i);   if i >= w: S' += phi(K_{i-w})^T V_{i-w}, ...
 *     O_i = phi(Q_i)(S - S') / (phi(Q_i).(z - z') + eps).
 */
int lt_oracle_fwd_window_recurrent(const void *q, const void *k, const void *v, int in_type,
                                   double *out, int B, int Hq, int Hkv, int N, int d, int dv,
                                   int window, double eps, const int32_t *cu_seqlens) {
    if (check_args(B, Hq, Hkv, N, d, dv, eps) || window < 1) return 1;
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int s = 0; s < B; ++s) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            int64_t t0, n;
            seq_range(s, N, cu_seqlens, &t0, &n);
            double *S = calloc((size_t)d * dv, sizeof(double)), *z = calloc((size_t)d, sizeof(double));
            double *Sl = calloc((size_t)d * dv, sizeof(double)), *zl = calloc((size_t)d, sizeof(double));
            double *pq = malloc(sizeof(double) * d), *pk = malloc(sizeof(double) * d);
            double *vv = malloc(sizeof(double) * dv);
            for (int64_t i = 0; i < n; ++i) {
                for (int lag = 0; lag < 2; ++lag) {
                    const int64_t t = lag ? i - window : i;
                    if (t < 0) continue;
                    double *St = lag ? Sl : S, *zt = lag ? zl : z;
                    for (int c = 0; c < d; ++c) pk[c] = lt_oracle_phi(load_elem(k, off(t0 + t, g, Hkv, d, c), in_type));
                    for (int c = 0; c < dv; ++c) vv[c] = load_elem(v, off(t0 + t, g, Hkv, dv, c), in_type);
                    for (int a = 0; a < d; ++a) {
                        for (int c = 0; c < dv; ++c) St[a * dv + c] += pk[a] * vv[c];
                        zt[a] += pk[a];
                    }
                }
                for (int c = 0; c < d; ++c) pq[c] = lt_oracle_phi(load_elem(q, off(t0 + i, h, Hq, d, c), in_type));
                double den = eps;
                for (int a = 0; a < d; ++a) den += pq[a] * (z[a] - zl[a]);
                for (int c = 0; c < dv; ++c) {
                    double num = 0.0;
                    for (int a = 0; a < d; ++a) num += pq[a] * (S[a * dv + c] - Sl[a * dv + c]);
                    out[off(t0 + i, h, Hq, dv, c)] = num / den;
                }
            }
            free(S); free(z); free(Sl); free(zl); free(pq); free(pk); free(vv);
        }
    }
    return 0;
}
