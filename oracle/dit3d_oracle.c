/*
 * dit3d_oracle.c -- plain fp64 CPU oracle for the DiT attention-block hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or load
 * this file; it exists so that tests, the smoke check and the benchmark's CPU
 * baseline leg can compare the CUDA kernels against an obviously correct
 * restatement of the formulas. It shares no code, header or table with the
 * CUDA library.
 *
 * Every function works in double precision on double inputs, loops over the
 * data in the order the formula is written, and parallelises only over
 * independent output rows (OpenMP), which does not change any result.
 *
 * Sources (web pages on video Diffusion Transformers):
 *  - "DiT, Flow Matching e 3D Attention: A Engenharia de Video com IA",
 *    section "A ruptura da U-Net": adaLN-Zero, x' = x + alpha*SelfAttn(gamma*LN(x)+beta),
 *    with alpha initialised to zero so the block is the identity.
 *  - same page, section "3D-RoPE e atencao espaco-temporal": d_head = d_t+d_h+d_w,
 *    q_rot = R3D(t,y,x) q, k_rot = R3D(t,y,x) k,
 *    Attention = softmax(q_rot k_rot^T / sqrt(d_head)) V.
 *  - "Por que e absurdamente dificil gerar um filme inteiro usando IA",
 *    section "Matematica por tras": Attention(Q,K,V) = softmax(QK^T/sqrt(d)) V.
 * Readings where the pages are silent (frequency law, pair layout, token order,
 * LayerNorm epsilon) are stated at each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* The number of threads the OpenMP loops below run on (1 without OpenMP), and a way
 * to set it, so that a timing of the oracle can state the host cores it used. No
 * arithmetic of the method. */
int oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Token j of a sequence laid out row-major over the patch grid (t slowest, w
 * fastest): recover its (t, h, w) patch coordinates. Reading: the pages give
 * only N = (T/p_t)(H/p_h)(W/p_w); the row-major order is this library's choice. */
static void token_coords(int64_t j, int32_t grid_h, int32_t grid_w, int64_t* t, int64_t* h,
                         int64_t* w) {
  *w = j % grid_w;
  *h = (j / grid_w) % grid_h;
  *t = j / ((int64_t)grid_w * grid_h);
}

/* Index of the sequence that holds global token `row` (cu_seqlens is the
 * exclusive prefix sum of the sequence lengths, n_seq + 1 entries). */
static int32_t seq_of_row(const int32_t* cu_seqlens, int32_t n_seq, int64_t row) {
  for (int32_t s = 0; s < n_seq; ++s)
    if (row >= cu_seqlens[s] && row < cu_seqlens[s + 1]) return s;
  return -1;
}

/*
 * adaLN modulation (page 2, "A ruptura da U-Net"): u = LN(x) * (s0 + gamma_g) + beta_g.
 * LN is over the D features of one token, without learned affine, with the
 * biased (divide by D) variance and eps inside the square root. s0 = 0 is the
 * page's form gamma*LN(x)+beta; s0 = 1 is the common (1+gamma) parameterisation.
 * The parameter group of row r is g = r / rows_per_group (one group per sample,
 * or one per latent frame).
 */
void oracle_adaln_modulate(const double* x, const double* gamma, const double* beta, double* out,
                           int64_t rows, int32_t D, int64_t rows_per_group, double eps,
                           double scale_offset) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const double* xr = x + r * D;
    const int64_t g = r / rows_per_group;
    double mean = 0.0;
    for (int32_t c = 0; c < D; ++c) mean += xr[c];
    mean /= D;
    double var = 0.0;
    for (int32_t c = 0; c < D; ++c) var += (xr[c] - mean) * (xr[c] - mean);
    var /= D;
    const double inv_std = 1.0 / sqrt(var + eps);
    for (int32_t c = 0; c < D; ++c) {
      const double xhat = (xr[c] - mean) * inv_std;
      out[r * D + c] = xhat * (scale_offset + gamma[g * D + c]) + beta[g * D + c];
    }
  }
}

/*
 * Gated residual (page 2, "A ruptura da U-Net"): out = x + alpha_g * y, with
 * alpha a D-vector per parameter group (a scalar gate is its broadcast).
 */
void oracle_gated_residual(const double* x, const double* y, const double* alpha, double* out,
                           int64_t rows, int32_t D, int64_t rows_per_group) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t g = r / rows_per_group;
    for (int32_t c = 0; c < D; ++c) out[r * D + c] = x[r * D + c] + alpha[g * D + c] * y[r * D + c];
  }
}

/*
 * One explicit Euler step of the rectified-flow ODE dx/dt = u (page 2, "Flow
 * Matching e Rectified Flow": straight path x_t = (1-t) x_0 + t x_1 whose velocity
 * is x_1 - x_0; Euler sampler) with per-frame local times (page 3, Flowception,
 * "Metodologia": frame i has its own time t_i, so its step is dt_i = t_i' - t_i):
 *   out[r, c] = x[r, c] + dt[r / rows_per_group] * u[r, c].
 */
void oracle_flow_euler_step(const double* x, const double* u, const double* dt, double* out,
                            int64_t rows, int32_t D, int64_t rows_per_group) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const double h = dt[r / rows_per_group];
    for (int32_t c = 0; c < D; ++c) out[r * D + c] = x[r * D + c] + h * u[r * D + c];
  }
}

/*
 * Linear layer of the block (page 1, "Matematica por tras": Y = X W, cost
 * O(n d m); page 2, "A ruptura da U-Net": the attention output projection and the
 * MLP inside the adaLN-Zero residuals):
 *   y[m, n] = sum_k x[m, k] w[n, k] + bias[n]          (w in [out, in] layout)
 *   y       = gelu(y) if act == 1, with the tanh form
 *             gelu(y) = y/2 (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3)))
 *   out     = y, or res + alpha[g, n] * y (g = m / rows_per_group) when res is given.
 * Readings (the pages name only "MLP" and the gates): GELU in its tanh form, a
 * bias per output column, the gate applied after the activation.
 * bias, res, alpha may be NULL (no bias; plain output).
 */
void oracle_linear(const double* x, const double* w, const double* bias, double* out,
                   int64_t M, int32_t N, int32_t K, int32_t act, const double* res,
                   const double* alpha, int64_t rows_per_group) {
  const double c = sqrt(2.0 / 3.14159265358979323846);
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int32_t n = 0; n < N; ++n) {
      double y = 0.0;
      for (int32_t k = 0; k < K; ++k) y += x[m * K + k] * w[(int64_t)n * K + k];
      if (bias) y += bias[n];
      if (act == 1) y = 0.5 * y * (1.0 + tanh(c * (y + 0.044715 * y * y * y)));
      if (res) y = res[m * N + n] + alpha[(m / rows_per_group) * N + n] * y;
      out[m * N + n] = y;
    }
  }
}

/*
 * FP8 E4M3 quantisation (page 2, "Engenharia de inferencia e paralelismo de contexto:
 * Ulysses, Ring Attention e FP8": activations quantised to FP8 E4M3/E5M2). E4M3 as
 * the OCP format defines it: 1 sign, 4 exponent (bias 7) and 3 mantissa bits, no
 * infinities, normal numbers 2^-6 .. 448 = 1.75 * 2^8, subnormals k * 2^-9. Values are
 * rounded to nearest, ties to even, and saturated at +-448 (the reading taken for
 * values beyond the range: clamp, as a per-tensor scale is meant to avoid them).
 * out[i] = e4m3(x[i] * inv_scale), returned as its real value.
 */
static double e4m3_round(double x) {
  if (x != x) return x;
  const double a = fabs(x);
  double q;
  if (a >= 448.0) {
    q = 448.0;
  } else if (a < 0.015625) {  /* below 2^-6: subnormal spacing 2^-9 */
    q = nearbyint(a * 512.0) / 512.0;
  } else {
    int e;
    frexp(a, &e);                     /* a = f * 2^e, f in [0.5, 1): 2^(e-1) <= a < 2^e */
    const double quantum = ldexp(1.0, e - 1 - 3);
    q = nearbyint(a / quantum) * quantum;
    if (q > 448.0) q = 448.0;
  }
  return x < 0 ? -q : q;
}

void oracle_quantize_e4m3(const double* x, double* out, int64_t n, double inv_scale) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_round(x[i] * inv_scale);
}

/* Round to the nearest bf16 value (8 significant bits, ties to even). */
void oracle_round_bf16(const double* x, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) {
    const double a = fabs(x[i]);
    if (a == 0.0 || x[i] != x[i]) { out[i] = x[i]; continue; }
    int e;
    frexp(a, &e);
    const double quantum = ldexp(1.0, e - 8);
    const double q = nearbyint(a / quantum) * quantum;
    out[i] = x[i] < 0 ? -q : q;
  }
}

/*
 * 3D rotary position embedding (page 2, "3D-RoPE e atencao espaco-temporal").
 * The head dimension is cut into three contiguous bands [t | h | w] of widths
 * d_t, d_h, d_w (each even, summing to d). Within band a, the pair
 * (v[o_a + 2i], v[o_a + 2i + 1]) is rotated by the angle pos_a * theta_{a,i},
 * theta_{a,i} = base^(-2i / d_a), with the rotation [[cos, -sin], [sin, cos]].
 * Readings (the pages give only the band split): the frequency law, base,
 * interleaved pair layout and band order above. Positions are the token's patch
 * coordinates counted from 0 at the start of its own sequence, plus the offsets
 * (t0, h0, w0). The same rotation is applied to every head.
 * in/out: [rows, H, d]; cu_seqlens: n_seq + 1 host entries.
 */
void oracle_rope3d(const double* in, double* out, int64_t rows, int32_t H, int32_t d,
                   const int32_t* cu_seqlens, int32_t n_seq, int32_t grid_h, int32_t grid_w,
                   int32_t d_t, int32_t d_h, int32_t d_w, double base, int32_t t0, int32_t h0,
                   int32_t w0) {
  const int32_t band_width[3] = {d_t, d_h, d_w};
  const int32_t band_offset[3] = {0, d_t, d_t + d_h};
  (void)d;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const int32_t s = seq_of_row(cu_seqlens, n_seq, r);
    const int64_t j = r - cu_seqlens[s];
    int64_t t, h, w;
    token_coords(j, grid_h, grid_w, &t, &h, &w);
    const double pos[3] = {(double)(t + t0), (double)(h + h0), (double)(w + w0)};
    for (int32_t head = 0; head < H; ++head) {
      const double* v = in + (r * H + head) * d;
      double* o = out + (r * H + head) * d;
      for (int32_t a = 0; a < 3; ++a) {
        for (int32_t i = 0; i < band_width[a] / 2; ++i) {
          const double theta = pow(base, -2.0 * i / band_width[a]);
          const double phi = pos[a] * theta;
          const int32_t c = band_offset[a] + 2 * i;
          const double x0 = v[c], x1 = v[c + 1];
          o[c] = x0 * cos(phi) - x1 * sin(phi);
          o[c + 1] = x0 * sin(phi) + x1 * cos(phi);
        }
      }
    }
  }
}

/*
 * Full (non-causal) attention per sequence and head (page 1, "Matematica por
 * tras"; page 2, "3D-RoPE e atencao espaco-temporal"):
 *   s_j = scale * <q_i, k_j> over the keys j of the query's own sequence,
 *   p_j = exp(s_j - max s), l = sum p, o_i = sum_j p_j v_j / l, lse = max s + ln l.
 * Packed sequences (cu_seqlens) never attend to one another. q, k and v are the
 * already-rotated vectors when 3D-RoPE is in use.
 * q, k, v: [rows, H, d]. Only the query rows listed in `qrows` (n_q entries;
 * NULL means every row, in order) are computed: o is [n_q, H, d], lse [n_q, H]
 * (lse may be NULL). Rows are independent, so a listed row's result is exact.
 */
void oracle_attn_fwd(const double* q, const double* k, const double* v, double* o, double* lse,
                     int64_t rows, int32_t H, int32_t d, const int32_t* cu_seqlens, int32_t n_seq,
                     double scale, const int64_t* qrows, int64_t n_q) {
  if (qrows == NULL) n_q = rows;
#pragma omp parallel
  {
    double* s = NULL;
    int64_t s_cap = 0;
#pragma omp for schedule(dynamic, 1)
    for (int64_t idx = 0; idx < n_q * H; ++idx) {
      const int64_t qi = idx / H;
      const int32_t head = (int32_t)(idx % H);
      const int64_t row = qrows ? qrows[qi] : qi;
      const int32_t sq = seq_of_row(cu_seqlens, n_seq, row);
      const int64_t k0 = cu_seqlens[sq], k1 = cu_seqlens[sq + 1];
      if (k1 - k0 > s_cap) {
        free(s);
        s_cap = k1 - k0;
        s = (double*)malloc(sizeof(double) * s_cap);
      }
      const double* qv = q + (row * H + head) * d;
      double m = -INFINITY;
      for (int64_t j = k0; j < k1; ++j) {
        const double* kv = k + (j * H + head) * d;
        double dot = 0.0;
        for (int32_t c = 0; c < d; ++c) dot += qv[c] * kv[c];
        s[j - k0] = scale * dot;
        if (s[j - k0] > m) m = s[j - k0];
      }
      double l = 0.0;
      for (int64_t j = k0; j < k1; ++j) {
        s[j - k0] = exp(s[j - k0] - m);
        l += s[j - k0];
      }
      double* ov = o + (qi * H + head) * d;
      for (int32_t c = 0; c < d; ++c) ov[c] = 0.0;
      for (int64_t j = k0; j < k1; ++j) {
        const double* vv = v + (j * H + head) * d;
        for (int32_t c = 0; c < d; ++c) ov[c] += s[j - k0] * vv[c];
      }
      for (int32_t c = 0; c < d; ++c) ov[c] /= l;
      if (lse) lse[qi * H + head] = m + log(l);
    }
    free(s);
  }
}
