/*
 * oracle.c -- plain, slow, sequential fp64 CPU oracle for the Mamba hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) includes, links, loads or calls this file.  Only the tests,
 * the package's smoke check and the benchmark's CPU-baseline leg use it.  It
 * shares no header, helper, table or constant with the CUDA code.
 *
 * What it computes (all arithmetic in double; inputs are the already-rounded
 * I/O values widened to double, intermediates are never rounded):
 *
 *   causal conv1d   xc[t] = bias + sum_{k=0}^{W-1} w[k] * x[t-(W-1)+k]
 *                   (x at t < 0 comes from the incoming conv_state, whose W
 *                   entries are the last W raw inputs, oldest first; zeros for
 *                   a fresh sequence)
 *   SiLU            silu(v) = v / (1 + exp(-v))
 *   softplus        softplus(v) = log(1 + exp(v))   (no threshold)
 *   Delta           delta = softplus(dt + dt_bias)  (or dt + dt_bias when the
 *                   softplus flag is off)
 *   scan            h[n] <- exp(delta*A[n]) * h[n] + delta * B[n] * u
 *                   y     = sum_n C[n] * h[n] + D * u
 *   gate            out   = y * silu(z)             (no gate when z is absent)
 *
 * Sources: the operator list "causal-conv1d, selective-scan, silu,
 * element-mul" of "feat(llama.cu): 适配 mamba 模型" (InfiniLM-Rust PR #48),
 * section 2.1; the state caches read and updated by capturing the conv and scan
 * operators, same page section 3.1; and the argument list
 * (state, x, dt, A, B, C, D, z, dt_bias, dt_softplus, out) of the
 * selective_state_update call in "[XPU] Add tuned Mamba SSU configs for Intel
 * Arc Pro B70" (vLLM PR #50534 report), section 关键源码片段.  The pages do not
 * print the equations; the ones above are the method's definition (discrete
 * A = exp(delta*A), Euler step delta*B*x) and every place where the pages are
 * silent is taken at its plainest reading, listed in the design notes.
 *
 * Layouts (all dense, row-major, last index fastest):
 *   scan:  x, dt, z, out (B, D, L);  A (D, N);  Bm, Cm (B, G, N, L);
 *          D, dt_bias, conv_bias (D);  conv_w (D, W);  conv_state (B, D, W);
 *          h (B, D, N).   Channel d reads group g = d / (D / G).
 *   scan, Mamba-2 layout:  x, z, out (B, H, P, L);  dt (B, H, L);  A (H);
 *          Bm, Cm (B, G, N, L);  D, dt_bias (H);  h (B, H, P, N).
 *          Head h reads group g = h / (H / G).
 *   ssu:   state (B, H, P, N);  x, z, out (B, H, P);  dt (B, H, P);
 *          A (H, P, N);  Bm, Cm (B, G, N);  D, dt_bias (H, P);
 *          conv_w (H*P, W); conv_bias (H*P); conv_state (B, H*P, W).
 *          Head h reads group g = h / (H / G).
 *
 * Return value: 0 on success, -1 on an argument the oracle cannot take.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double o_silu(double v) { return v / (1.0 + exp(-v)); }

/* log(1 + exp(v)), written so that exp never overflows; same function. */
static double o_softplus(double v) {
    if (v > 0.0) return v + log1p(exp(-v));
    return log1p(exp(v));
}

double oracle_silu(double v) { return o_silu(v); }
double oracle_softplus(double v) { return o_softplus(v); }

/* ---------------------------------------------------------------------------
 * Causal conv1d over one channel.  xin holds the W-1 history values followed by
 * the L current values, so xc[t] = bias + sum_k w[k] * xin[t + k].
 * ------------------------------------------------------------------------- */
static void o_conv_channel(int64_t L, int64_t W, const double* hist_w /* W entries or NULL */,
                           const double* x, const double* w, double bias, int silu,
                           double* out, double* hist_out /* W entries or NULL */) {
    double* xin = (double*)malloc(sizeof(double) * (size_t)(L + W));
    int64_t k, t;
    /* history: the last W-1 of the incoming W raw values (oldest first) */
    for (k = 0; k < W - 1; ++k) xin[k] = hist_w ? hist_w[k + 1] : 0.0;
    for (t = 0; t < L; ++t) xin[W - 1 + t] = x[t];
    for (t = 0; t < L; ++t) {
        double acc = bias;
        for (k = 0; k < W; ++k) acc += w[k] * xin[t + k];
        out[t] = silu ? o_silu(acc) : acc;
    }
    if (hist_out) {
        /* last W raw inputs of (incoming state ++ x), oldest first */
        double* all = (double*)malloc(sizeof(double) * (size_t)(L + W));
        for (k = 0; k < W; ++k) all[k] = hist_w ? hist_w[k] : 0.0;
        for (t = 0; t < L; ++t) all[W + t] = x[t];
        for (k = 0; k < W; ++k) hist_out[k] = all[L + k];
        free(all);
    }
    free(xin);
}

int oracle_conv1d(int64_t B, int64_t D, int64_t L, int64_t W,
                  const double* x, const double* weight, const double* bias,
                  const double* conv_state_in, int silu,
                  double* out, double* conv_state_out) {
    int64_t b, d;
    if (B < 0 || D < 0 || L < 0 || W < 1) return -1;
    for (b = 0; b < B; ++b) {
        for (d = 0; d < D; ++d) {
            const int64_t row = (b * D + d);
            o_conv_channel(L, W, conv_state_in ? conv_state_in + row * W : NULL,
                           x + row * L, weight + d * W, bias ? bias[d] : 0.0, silu,
                           out + row * L, conv_state_out ? conv_state_out + row * W : NULL);
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Prefill: per (b, d), sequentially over t, conv -> SiLU -> Delta -> scan ->
 * gate.  conv_w == NULL means no conv and no SiLU: u = x.
 * ------------------------------------------------------------------------- */
int oracle_scan(int64_t B, int64_t D, int64_t L, int64_t N, int64_t G, int64_t W,
                const double* x, const double* dt, const double* A,
                const double* Bm, const double* Cm,
                const double* Dv, const double* z, const double* dt_bias, int dt_softplus,
                const double* conv_w, const double* conv_b, const double* conv_state_in,
                const double* h0,
                double* out, double* h_final, double* conv_state_out) {
    int64_t b, d, t, n;
    if (B < 0 || D < 0 || L < 0 || N < 1 || G < 1 || D % G != 0) return -1;
    if (conv_w && W < 1) return -1;
    double* u = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* h = (double*)malloc(sizeof(double) * (size_t)N);
    for (b = 0; b < B; ++b) {
        for (d = 0; d < D; ++d) {
            const int64_t row = b * D + d;
            const int64_t g = d / (D / G);
            const double* Brow = Bm + (b * G + g) * N * L;
            const double* Crow = Cm + (b * G + g) * N * L;
            /* a1 + a2: causal conv1d then SiLU (or the raw input) */
            if (conv_w) {
                o_conv_channel(L, W, conv_state_in ? conv_state_in + row * W : NULL,
                               x + row * L, conv_w + d * W, conv_b ? conv_b[d] : 0.0, 1, u,
                               conv_state_out ? conv_state_out + row * W : NULL);
            } else {
                for (t = 0; t < L; ++t) u[t] = x[row * L + t];
            }
            for (n = 0; n < N; ++n) h[n] = h0 ? h0[row * N + n] : 0.0;
            for (t = 0; t < L; ++t) {
                /* a3: Delta */
                double v = dt[row * L + t] + (dt_bias ? dt_bias[d] : 0.0);
                double delta = dt_softplus ? o_softplus(v) : v;
                /* a4: recurrence and readout */
                double y = 0.0;
                for (n = 0; n < N; ++n) {
                    double a = exp(delta * A[d * N + n]);
                    h[n] = a * h[n] + delta * Brow[n * L + t] * u[t];
                    y += Crow[n * L + t] * h[n];
                }
                y += (Dv ? Dv[d] : 0.0) * u[t];
                /* a5: gate */
                if (z) y *= o_silu(z[row * L + t]);
                out[row * L + t] = y;
            }
            if (h_final)
                for (n = 0; n < N; ++n) h_final[row * N + n] = h[n];
        }
    }
    free(u);
    free(h);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Single-token state update, general (B, H, P, N) form.  Every row
 * (b, h, p) is one recurrence over N state entries; A is given per element
 * and dt per row (callers broadcast a per-head scalar).  With conv_w, x is the
 * raw channel input: the conv state of channel c = h*P + p is rolled left by
 * one, x is appended, u = silu(sum_k w[c,k] * cs[k] + bias[c]).
 * ------------------------------------------------------------------------- */
int oracle_ssu(int64_t B, int64_t H, int64_t P, int64_t N, int64_t G, int64_t W,
               double* state, const double* x, const double* dt, const double* A,
               const double* Bm, const double* Cm,
               const double* Dv, const double* z, const double* dt_bias, int dt_softplus,
               const double* conv_w, const double* conv_b, double* conv_state,
               double* out) {
    int64_t b, hh, p, n, k;
    if (B < 0 || H < 1 || P < 1 || N < 1 || G < 1 || H % G != 0) return -1;
    if (conv_w && (W < 1 || !conv_state)) return -1;
    for (b = 0; b < B; ++b) {
        for (hh = 0; hh < H; ++hh) {
            const int64_t g = hh / (H / G);
            const double* Bv = Bm + (b * G + g) * N;
            const double* Cv = Cm + (b * G + g) * N;
            for (p = 0; p < P; ++p) {
                const int64_t row = (b * H + hh) * P + p; /* (b, h, p) */
                const int64_t hp = hh * P + p;            /* (h, p) */
                double u = x[row];
                if (conv_w) {
                    double* cs = conv_state + (b * H * P + hp) * W;
                    for (k = 0; k < W - 1; ++k) cs[k] = cs[k + 1];
                    cs[W - 1] = x[row];
                    double acc = conv_b ? conv_b[hp] : 0.0;
                    for (k = 0; k < W; ++k) acc += conv_w[hp * W + k] * cs[k];
                    u = o_silu(acc);
                }
                double v = dt[row] + (dt_bias ? dt_bias[hp] : 0.0);
                double delta = dt_softplus ? o_softplus(v) : v;
                double y = 0.0;
                double* s = state + row * N;
                for (n = 0; n < N; ++n) {
                    double a = exp(delta * A[hp * N + n]);
                    s[n] = a * s[n] + delta * Bv[n] * u;
                    y += Cv[n] * s[n];
                }
                y += (Dv ? Dv[hp] : 0.0) * u;
                if (z) y *= o_silu(z[row]);
                out[row] = y;
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Mamba-2 layout with its own notation: scalar A per head, dt per head,
 * D and dt_bias per head, no conv.  Written separately from oracle_ssu so that
 * the two layouts can be checked against each other.
 * ------------------------------------------------------------------------- */
int oracle_ssu_mamba2(int64_t B, int64_t H, int64_t P, int64_t N, int64_t G,
                      double* state, const double* x, const double* dt_head /* (B,H) */,
                      const double* A_head /* (H) */, const double* Bm, const double* Cm,
                      const double* D_head /* (H) or NULL */, const double* z,
                      const double* dt_bias_head /* (H) or NULL */, int dt_softplus,
                      double* out) {
    int64_t b, hh, p, n;
    if (B < 0 || H < 1 || P < 1 || N < 1 || G < 1 || H % G != 0) return -1;
    const int64_t heads_per_group = H / G;
    for (b = 0; b < B; ++b) {
        for (hh = 0; hh < H; ++hh) {
            double v = dt_head[b * H + hh] + (dt_bias_head ? dt_bias_head[hh] : 0.0);
            double delta = dt_softplus ? o_softplus(v) : v;
            double dA = exp(delta * A_head[hh]);
            const double* Bv = Bm + (b * G + hh / heads_per_group) * N;
            const double* Cv = Cm + (b * G + hh / heads_per_group) * N;
            for (p = 0; p < P; ++p) {
                const int64_t row = (b * H + hh) * P + p;
                double xv = x[row];
                double* s = state + row * N;
                double y = 0.0;
                for (n = 0; n < N; ++n) {
                    s[n] = dA * s[n] + delta * Bv[n] * xv;
                    y += Cv[n] * s[n];
                }
                if (D_head) y += D_head[hh] * xv;
                if (z) y *= o_silu(z[row]);
                out[row] = y;
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Prefill in the Mamba-2 layout: per batch entry and head, sequentially over
 * t, one Delta and one decay per head and step, then every (p, n) state entry
 * of the head takes the same update as in the scan above with u = x (no conv):
 *   delta   = softplus(dt[b,h,t] + dt_bias[h])
 *   s[p,n]  = exp(delta * A[h]) * s[p,n] + delta * B[b,g,n,t] * x[b,h,p,t]
 *   out     = (sum_n C[b,g,n,t] * s[p,n] + D[h] * x[b,h,p,t]) * silu(z[b,h,p,t])
 * with g = h / (H / G).  The per-head scalar A and the group sharing are the
 * Mamba-2 shape (batch, nheads, headdim, dstate, ngroups) of "[XPU] Add tuned
 * Mamba SSU configs for Intel Arc Pro B70", section 实现拆解.  h0 (B,H,P,N) or
 * NULL (zeros); the state after the last step goes to h_final (B,H,P,N).
 * ------------------------------------------------------------------------- */
int oracle_scan_mamba2(int64_t B, int64_t H, int64_t P, int64_t N, int64_t G, int64_t L,
                       const double* x, const double* dt, const double* A_head, const double* Bm,
                       const double* Cm, const double* D_head, const double* z,
                       const double* dt_bias_head, int dt_softplus, const double* h0,
                       double* out, double* h_final) {
    int64_t b, hh, p, n, t;
    if (B < 0 || H < 1 || P < 1 || N < 1 || G < 1 || L < 0 || H % G != 0) return -1;
    const int64_t per_group = H / G;
    for (b = 0; b < B; ++b) {
        for (hh = 0; hh < H; ++hh) {
            double* S = h_final + (b * H + hh) * P * N;  /* the head's P x N state */
            for (p = 0; p < P; ++p)
                for (n = 0; n < N; ++n)
                    S[p * N + n] = h0 ? h0[((b * H + hh) * P + p) * N + n] : 0.0;
            const int64_t grp = hh / per_group;
            const double* Bg = Bm + (b * G + grp) * N * L;
            const double* Cg = Cm + (b * G + grp) * N * L;
            for (t = 0; t < L; ++t) {
                double v = dt[(b * H + hh) * L + t] + (dt_bias_head ? dt_bias_head[hh] : 0.0);
                double delta = dt_softplus ? o_softplus(v) : v;
                double decay = exp(delta * A_head[hh]);
                for (p = 0; p < P; ++p) {
                    const int64_t at = ((b * H + hh) * P + p) * L + t;
                    double xv = x[at];
                    double acc = 0.0;
                    for (n = 0; n < N; ++n) {
                        S[p * N + n] = decay * S[p * N + n] + delta * Bg[n * L + t] * xv;
                        acc += Cg[n * L + t] * S[p * N + n];
                    }
                    if (D_head) acc += D_head[hh] * xv;
                    if (z) acc *= o_silu(z[at]);
                    out[at] = acc;
                }
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Rounding of a state cache to its storage dtype, for comparisons of several
 * consecutive decode steps against a GPU cache kept in fp32, fp16 or bf16:
 * after each step the stored state is the updated value rounded to nearest,
 * ties to even (the readout of that step has already used the unrounded
 * value).  dtype: 0 = keep fp64, 1 = fp32, 2 = fp16, 3 = bf16.
 *
 * fp16 keeps 11 significant bits for |v| >= 2^-14 and a fixed quantum of
 * 2^-24 below (subnormals); bf16 keeps 8 significant bits for |v| >= 2^-126
 * and a quantum of 2^-133 below.  Values past the largest finite value round
 * to infinity (65504 for fp16; bf16 shares fp32's exponent range).
 * ------------------------------------------------------------------------- */
static double o_round_bits(double v, int sig_bits, int min_exp, double max_finite, double max_half_ulp) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e = ilogb(v);                      /* 2^e <= |v| < 2^(e+1) */
    if (e < min_exp) e = min_exp;          /* subnormal range: fixed quantum */
    const double q = ldexp(1.0, e - (sig_bits - 1));
    const double r = nearbyint(v / q) * q; /* default rounding mode: to nearest even */
    if (fabs(r) > max_finite) {
        /* values at or beyond max + half an ulp overflow */
        return fabs(v) >= max_finite + max_half_ulp ? copysign(INFINITY, v) : copysign(max_finite, v);
    }
    return r;
}

int oracle_round_cache(double* v, int64_t n, int dtype) {
    int64_t i;
    if (n < 0 || dtype < 0 || dtype > 3) return -1;
    for (i = 0; i < n; ++i) {
        if (dtype == 1) {
            v[i] = (double)(float)v[i];
        } else if (dtype == 2) {
            v[i] = o_round_bits(v[i], 11, -14, 65504.0, 16.0);
        } else if (dtype == 3) {
            v[i] = o_round_bits(v[i], 8, -126, 3.3895313892515355e38, ldexp(1.0, 127 - 8));
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Sequence pieces.  A prefill over a sequence cut into consecutive pieces
 * equals the prefills of the pieces, each started from the state that the
 * earlier pieces leave (the scan is a first-order linear recurrence in h).
 * Started from a zero state, piece j ends in h_end(j); the state entering
 * piece j+1 is
 *     h_in(j+1)[b,d,n] = exp(A[d,n] * S(j)[b,d]) * h_in(j)[b,d,n] + h_end(j)[b,d,n]
 * where S(j)[b,d] is the sum over the piece's steps of delta (softplus(dt +
 * dt_bias), or dt + dt_bias without the softplus): the product of the piece's
 * per-step decays exp(delta*A) is exp(A * sum delta).  Pages: the long-context
 * claim of "feat(llama.cu): 适配 mamba 模型" section 6.1 (the scan is linear in
 * the sequence length); the decomposition itself is the recurrence's algebra.
 *
 *   oracle_delta_sum   S[b,d] = sum_t delta(dt[b,d,t] + dt_bias[d])   dt (B, D, L)
 *   oracle_carry_fold  state[b,d,n] <- exp(A[d,n] * S[b,d]) * state[b,d,n] + h_end[b,d,n]
 *                      A (D, N); S (B, D); h_end, state (B, D, N)
 * ------------------------------------------------------------------------- */
int oracle_delta_sum(int64_t B, int64_t D, int64_t L, const double* dt, const double* dt_bias,
                     int dt_softplus, double* out) {
    int64_t b, d, t;
    if (B < 0 || D < 0 || L < 0 || !dt || !out) return -1;
    for (b = 0; b < B; ++b) {
        for (d = 0; d < D; ++d) {
            double sum = 0.0;
            for (t = 0; t < L; ++t) {
                const double v = dt[(b * D + d) * L + t] + (dt_bias ? dt_bias[d] : 0.0);
                sum += dt_softplus ? o_softplus(v) : v;
            }
            out[b * D + d] = sum;
        }
    }
    return 0;
}

int oracle_carry_fold(int64_t B, int64_t D, int64_t N, const double* A, const double* S,
                      const double* h_end, double* state) {
    int64_t b, d, n;
    if (B < 0 || D < 0 || N < 0 || !A || !S || !h_end || !state) return -1;
    for (b = 0; b < B; ++b)
        for (d = 0; d < D; ++d)
            for (n = 0; n < N; ++n) {
                const int64_t i = (b * D + d) * N + n;
                state[i] = exp(A[d * N + n] * S[b * D + d]) * state[i] + h_end[i];
            }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Double-gated short causal conv: the convolution of the "double-gated LIV
 * convolution blocks" that "LFM2.5-1.2B-Thinking性能优化CUDA核心编程技巧"
 * (section 2.1) names next to the GQA blocks.  The page prints no equation;
 * the reading taken here is the plainest one the name supports: two
 * input-dependent multiplicative gates around a depthwise causal conv, one
 * before it (Bg) and one after it (Cg), with no activation:
 *
 *   v[t]   = Bg[t] * x[t]
 *   c[t]   = bias + sum_{k=0}^{W-1} w[k] * v[t-(W-1)+k]
 *   out[t] = Cg[t] * c[t]
 *
 * v at t < 0 comes from the incoming conv_state, whose W entries are the last
 * W gated inputs v, oldest first (zeros for a fresh sequence); conv_state_out
 * holds the last W entries of (incoming state ++ v).
 *
 * Layouts: x, Bg, Cg, out (B, D, L); weight (D, W); bias (D);
 * conv_state (B, D, W).
 * ------------------------------------------------------------------------- */
int oracle_gated_conv1d(int64_t B, int64_t D, int64_t L, int64_t W,
                        const double* x, const double* Bg, const double* Cg,
                        const double* weight, const double* bias, const double* conv_state_in,
                        double* out, double* conv_state_out) {
    int64_t b, d, t;
    if (B < 0 || D < 0 || L < 0 || W < 1 || !x || !Bg || !Cg || !weight || !out) return -1;
    double* v = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* c = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (b = 0; b < B; ++b) {
        for (d = 0; d < D; ++d) {
            const int64_t row = b * D + d;
            /* the input gate */
            for (t = 0; t < L; ++t) v[t] = Bg[row * L + t] * x[row * L + t];
            /* the causal conv of the gated input, no activation */
            o_conv_channel(L, W, conv_state_in ? conv_state_in + row * W : NULL, v, weight + d * W,
                           bias ? bias[d] : 0.0, 0, c, conv_state_out ? conv_state_out + row * W : NULL);
            /* the output gate */
            for (t = 0; t < L; ++t) out[row * L + t] = Cg[row * L + t] * c[t];
        }
    }
    free(v);
    free(c);
    return 0;
}
