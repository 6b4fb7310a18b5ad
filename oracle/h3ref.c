/* Oracle, second implementation: the MiniMax-H3-Image dense DiT block in plain C.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
 * baseline leg may load this library. It shares no code with the CUDA library
 * or with the numpy oracle beside it; the two oracles are written
 * independently and checked against each other.
 *
 * Arithmetic type REAL: double by default, float when built with
 * -DH3REF_REAL_FLOAT (the block computed in plain fp32 from bf16-valued
 * weights, nothing rounded in between). Every loop follows the definition in
 * the order it is written: no blocking, no fusion, no reordering.
 *
 * Sources (page titles and sections):
 *   [card] MiniMax-H3-Image model card, "Model Architecture": one packed
 *          sequence of text and image tokens through a single-stream
 *          transformer; hidden 5376, 56 heads, FFN 14336; "3D multimodal
 *          RoPE"; timestep layers in FP32.
 *   [apx]  apxml "MiniMax H3 Image", "Architecture Diagram": per block
 *          RMSNorm + timestep scale/shift -> joint attention -> "+" ->
 *          RMSNorm + timestep scale/shift -> GELU MLP -> "+";
 *          "Specifications": RoPE, RMS normalization, GELU.
 *   [vllm] "H3-Image Day-0 Support: 4K in 0.87s with Vera Rubin",
 *          "Faster DiT": the AdaLN conditioning is computed once and reused.
 * Where the pages are silent the same readings as the numpy oracle apply:
 * 256-channel [cos | sin] timestep sinusoid with frequencies 10000^(-i/128)
 * at argument t_scale * t; AdaLN chunks shift1, scale1, gate1, shift2,
 * scale2, gate2 from W_ada SiLU(c) + b_ada; RMSNorm without gain; (1 + scale)
 * and + shift; no biases in the block linears; an ungated GELU FFN; RoPE
 * sections per (frame, row, col) axis, each a rotate-half rotation of its own
 * 2 s_a channels by pos_a * theta^(-j / s_a); text tokens at (0, 0, 0);
 * unmasked attention scaled by 1 / sqrt(head_dim).
 *
 * Weights are nn.Linear [out, in] arrays of float (bf16 weights widen to
 * float exactly); activations are REAL. All pointers are host memory owned by
 * the caller. Functions that allocate return 0, or -1 when memory runs out.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef H3REF_REAL_FLOAT
typedef float REAL;
#define R_EXP expf
#define R_SQRT sqrtf
#define R_ERF erff
#define R_TANH tanhf
#define R_COS cosf
#define R_SIN sinf
#define R_POW powf
#else
typedef double REAL;
#define R_EXP exp
#define R_SQRT sqrt
#define R_ERF erf
#define R_TANH tanh
#define R_COS cos
#define R_SIN sin
#define R_POW pow
#endif

typedef struct {
  int hidden, heads, head_dim, ffn;
  int sections[3]; /* rotation pairs per (frame, row, col) axis; sum = head_dim / 2 */
  int gelu_tanh;   /* 0: x Phi(x) with erf; 1: the tanh approximation */
  double theta;    /* RoPE base */
  double eps;      /* RMSNorm epsilon */
} h3ref_cfg;

int h3ref_real_bytes(void) { return (int)sizeof(REAL); }

static REAL silu(REAL x) { return x / ((REAL)1 + R_EXP(-x)); }

/* [apx] "Specifications": GELU, read as x Phi(x). */
static REAL gelu(REAL x, int use_tanh) {
  if (use_tanh) {
    const REAL c = (REAL)0.7978845608028654; /* sqrt(2 / pi) */
    return (REAL)0.5 * x * ((REAL)1 + R_TANH(c * (x + (REAL)0.044715 * x * x * x)));
  }
  return (REAL)0.5 * x * ((REAL)1 + R_ERF(x / (REAL)1.4142135623730951));
}

/* y[r][o] = sum_k x[r][k] w[o][k], for rows r < n: an nn.Linear without bias. */
static void linear(const REAL *x, int n, int in, const float *w, int out, REAL *y) {
  for (int r = 0; r < n; ++r)
    for (int o = 0; o < out; ++o) {
      REAL acc = 0;
      for (int k = 0; k < in; ++k) acc += x[(size_t)r * in + k] * (REAL)w[(size_t)o * in + k];
      y[(size_t)r * out + o] = acc;
    }
}

/* (frame, row, col) per token of [text; image 0; image 1; ...]: text at
 * (0, 0, 0), image g row-major over its height x width at its frame.
 * grids: n_grids triples (frame, height, width). pos: [n][3]. */
void h3ref_token_positions(int n_txt, const int *grids, int n_grids, int *pos) {
  int i = 0;
  for (; i < n_txt; ++i) pos[3 * i] = pos[3 * i + 1] = pos[3 * i + 2] = 0;
  for (int g = 0; g < n_grids; ++g) {
    const int frame = grids[3 * g], h = grids[3 * g + 1], w = grids[3 * g + 2];
    for (int r = 0; r < h; ++r)
      for (int c = 0; c < w; ++c, ++i) {
        pos[3 * i] = frame;
        pos[3 * i + 1] = r;
        pos[3 * i + 2] = c;
      }
  }
}

/* Step a1 ([card]: timestep layers in FP32): e = [cos(t_scale t w_i) |
 * sin(t_scale t w_i)], w_i = 10000^(-i / (dim/2)); c = W_t2 SiLU(W_t1 e +
 * b_t1) + b_t2 with W_t1 [hidden, dim], W_t2 [hidden, hidden]. */
int h3ref_timestep_condition(double t, int dim, double t_scale, int hidden, const float *w_t1,
                             const float *b_t1, const float *w_t2, const float *b_t2, REAL *c) {
  const int half = dim / 2;
  REAL *e = (REAL *)malloc(sizeof(REAL) * (size_t)dim);
  REAL *h = (REAL *)malloc(sizeof(REAL) * (size_t)hidden);
  if (!e || !h) {
    free(e);
    free(h);
    return -1;
  }
  for (int i = 0; i < half; ++i) {
    const REAL freq = R_POW((REAL)10000, -(REAL)i / (REAL)half);
    const REAL arg = (REAL)t_scale * (REAL)t * freq;
    e[i] = R_COS(arg);
    e[half + i] = R_SIN(arg);
  }
  for (int o = 0; o < hidden; ++o) {
    REAL acc = (REAL)b_t1[o];
    for (int k = 0; k < dim; ++k) acc += (REAL)w_t1[(size_t)o * dim + k] * e[k];
    h[o] = silu(acc);
  }
  for (int o = 0; o < hidden; ++o) {
    REAL acc = (REAL)b_t2[o];
    for (int k = 0; k < hidden; ++k) acc += (REAL)w_t2[(size_t)o * hidden + k] * h[k];
    c[o] = acc;
  }
  free(e);
  free(h);
  return 0;
}

/* Step a2 ([vllm] "Faster DiT": computed once per step): mod = W_ada SiLU(c)
 * + b_ada, W_ada [6 hidden, hidden]; mod is [6][hidden] in the chunk order
 * shift1, scale1, gate1, shift2, scale2, gate2. */
int h3ref_adaln(int hidden, const REAL *c, const float *w_ada, const float *b_ada, REAL *mod) {
  REAL *s = (REAL *)malloc(sizeof(REAL) * (size_t)hidden);
  if (!s) return -1;
  for (int k = 0; k < hidden; ++k) s[k] = silu(c[k]);
  for (int o = 0; o < 6 * hidden; ++o) {
    REAL acc = (REAL)b_ada[o];
    for (int k = 0; k < hidden; ++k) acc += (REAL)w_ada[(size_t)o * hidden + k] * s[k];
    mod[o] = acc;
  }
  free(s);
  return 0;
}

/* Steps a3 / a7 ([apx] diagram: RMSNorm, then timestep scale/shift):
 * out = x / sqrt(mean(x^2) + eps) * (1 + scale) + shift, per row. */
static void norm_modulate(const REAL *x, int n, int d, const REAL *shift, const REAL *scale,
                          double eps, REAL *out) {
  for (int r = 0; r < n; ++r) {
    const REAL *xr = x + (size_t)r * d;
    REAL ss = 0;
    for (int j = 0; j < d; ++j) ss += xr[j] * xr[j];
    const REAL inv = (REAL)1 / R_SQRT(ss / (REAL)d + (REAL)eps);
    for (int j = 0; j < d; ++j) out[(size_t)r * d + j] = xr[j] * inv * ((REAL)1 + scale[j]) + shift[j];
  }
}

/* [card] "3D multimodal RoPE": rotate every head of x [n][heads][head_dim] in
 * place. Axis a owns channels [o_a, o_a + 2 s_a); its pair j is
 * (o_a + j, o_a + s_a + j) and turns by pos_a * theta^(-j / s_a). */
static void rope(REAL *x, int n, const h3ref_cfg *cfg, const int *pos) {
  const int dh = cfg->head_dim;
  for (int i = 0; i < n; ++i)
    for (int h = 0; h < cfg->heads; ++h) {
      REAL *v = x + ((size_t)i * cfg->heads + h) * dh;
      int o = 0;
      for (int a = 0; a < 3; ++a) {
        const int s = cfg->sections[a];
        for (int j = 0; j < s; ++j) {
          const REAL ang = (REAL)pos[3 * i + a] * R_POW((REAL)cfg->theta, -(REAL)j / (REAL)s);
          const REAL cs = R_COS(ang), sn = R_SIN(ang);
          const REAL x1 = v[o + j], x2 = v[o + s + j];
          v[o + j] = x1 * cs - x2 * sn;
          v[o + s + j] = x2 * cs + x1 * sn;
        }
        o += 2 * s;
      }
    }
}

/* Step a5 ([card]: one packed sequence; bidirectional): for every head and
 * query i, o_i = sum_j softmax_j(q_i . k_j / sqrt(d)) v_j over all n keys.
 * q, k, v, o: [n][heads][head_dim]. p: scratch of n. */
static void attention(const REAL *q, const REAL *k, const REAL *v, int n, int heads, int dh,
                      REAL *p, REAL *o) {
  const REAL scale = (REAL)1 / R_SQRT((REAL)dh);
  for (int h = 0; h < heads; ++h)
    for (int i = 0; i < n; ++i) {
      const REAL *qi = q + ((size_t)i * heads + h) * dh;
      REAL mx = -INFINITY;
      for (int j = 0; j < n; ++j) {
        const REAL *kj = k + ((size_t)j * heads + h) * dh;
        REAL s = 0;
        for (int c = 0; c < dh; ++c) s += qi[c] * kj[c];
        p[j] = s * scale;
        if (p[j] > mx) mx = p[j];
      }
      REAL sum = 0;
      for (int j = 0; j < n; ++j) {
        p[j] = R_EXP(p[j] - mx);
        sum += p[j];
      }
      REAL *oi = o + ((size_t)i * heads + h) * dh;
      for (int c = 0; c < dh; ++c) oi[c] = 0;
      for (int j = 0; j < n; ++j) {
        const REAL *vj = v + ((size_t)j * heads + h) * dh;
        const REAL w = p[j] / sum;
        for (int c = 0; c < dh; ++c) oi[c] += w * vj[c];
      }
    }
}

/* Steps a3..a9: one block on the packed sequence x [n][hidden] ([apx] order):
 *   xm = RMSNorm(x)(1 + scale1) + shift1
 *   Q, K, V = xm W_q^T, xm W_k^T, xm W_v^T (rows of w_qkv: Q heads | K | V);
 *   Q, K <- RoPE(pos)
 *   x1 = x + gate1 * (Attention(Q, K, V) W_o^T)
 *   y  = x1 + gate2 * (GELU((RMSNorm(x1)(1 + scale2) + shift2) W_1^T) W_2^T)
 * mod: [6][hidden]; pos: [n][3]; y: [n][hidden] (may not alias x). */
int h3ref_block_forward(const h3ref_cfg *cfg, int n, const REAL *x, const REAL *mod,
                        const float *w_qkv, const float *w_o, const float *w_ff1,
                        const float *w_ff2, const int *pos, REAL *y) {
  const int D = cfg->hidden, H = cfg->heads, dh = cfg->head_dim, F = cfg->ffn;
  const int I = H * dh;
  const REAL *sh1 = mod, *sc1 = mod + D, *g1 = mod + 2 * D;
  const REAL *sh2 = mod + 3 * D, *sc2 = mod + 4 * D, *g2 = mod + 5 * D;
  if (2 * (cfg->sections[0] + cfg->sections[1] + cfg->sections[2]) != dh) return -1;
  REAL *xm = (REAL *)malloc(sizeof(REAL) * (size_t)n * D);
  REAL *q = (REAL *)malloc(sizeof(REAL) * (size_t)n * I);
  REAL *k = (REAL *)malloc(sizeof(REAL) * (size_t)n * I);
  REAL *v = (REAL *)malloc(sizeof(REAL) * (size_t)n * I);
  REAL *att = (REAL *)malloc(sizeof(REAL) * (size_t)n * I);
  REAL *t = (REAL *)malloc(sizeof(REAL) * (size_t)n * (D > F ? D : F));
  REAL *x1 = (REAL *)malloc(sizeof(REAL) * (size_t)n * D);
  REAL *p = (REAL *)malloc(sizeof(REAL) * (size_t)(n > 0 ? n : 1));
  int rc = -1;
  if (!xm || !q || !k || !v || !att || !t || !x1 || !p) goto done;

  norm_modulate(x, n, D, sh1, sc1, cfg->eps, xm);
  linear(xm, n, D, w_qkv, I, q);
  linear(xm, n, D, w_qkv + (size_t)I * D, I, k);
  linear(xm, n, D, w_qkv + (size_t)2 * I * D, I, v);
  rope(q, n, cfg, pos);
  rope(k, n, cfg, pos);
  attention(q, k, v, n, H, dh, p, att);
  linear(att, n, I, w_o, D, t);
  for (size_t i = 0; i < (size_t)n * D; ++i) x1[i] = x[i] + g1[i % D] * t[i];

  norm_modulate(x1, n, D, sh2, sc2, cfg->eps, xm);
  REAL *u = q; /* [n][F] needs its own buffer when F > I */
  if (F > I) {
    free(q);
    q = u = (REAL *)malloc(sizeof(REAL) * (size_t)n * F);
    if (!u) goto done;
  }
  linear(xm, n, D, w_ff1, F, u);
  for (size_t i = 0; i < (size_t)n * F; ++i) u[i] = gelu(u[i], cfg->gelu_tanh);
  linear(u, n, F, w_ff2, D, t);
  for (size_t i = 0; i < (size_t)n * D; ++i) y[i] = x1[i] + g2[i % D] * t[i];
  rc = 0;
done:
  free(xm);
  free(q);
  free(k);
  free(v);
  free(att);
  free(t);
  free(x1);
  free(p);
  return rc;
}
