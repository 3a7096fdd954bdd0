/*
 * had_oracle.c -- plain, slow CPU reference ("the oracle") for binarized-QK
 * top-N attention, as "Hamming Attention Distillation: Binarizing Keys and
 * Queries for Efficient Long-Context Transformers" (HAD) and "BinaryAttention:
 * One-Bit QK-Attention for Vision and Diffusion Transformers" define it.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline use it.  It shares no code, header, table or helper with the CUDA
 * library in binarized_qk_sparse_b200/.
 *
 * Every step is the plain definition written out with loops, in the order the
 * method states it, with fp64 for every floating-point accumulation:
 *   1. mu[c]   = mean over the valid tokens of X[:, c]     (BinaryAttention §2.2, scaled binarization eq.)
 *   2. bit     = X < mu  (bit 1 <=> sign(X - mu) = -1)     (BinaryAttention §2.2; HAD abstract: {-1,+1} keys/queries)
 *   3. s       = d - 2 * popcount(q XOR k)                  (BinaryAttention §2.1 distance view, §2.2 XNOR+popcount)
 *   4. l       = fmaf(s, c, b_ij), c = alpha_q*alpha_k/sqrt(d) (BinaryAttention §2.3 eq. softmax(QK^T/sqrt(d) + B))
 *   5. kept    = first K_eff keys of the full sort by (l desc, j asc)  (HAD summary "main points": top-N per query)
 *   6. p       = softmax over the kept keys, fp64                (BinaryAttention §2.3 eq.)
 *   7. O       = sum_j p_j V_j (float mode), or
 *      O       = dequant(sum_j A_q V_q) with A_q = floor(255 p + 0.5), V_q per-channel int8
 *                                                            (BinaryAttention §2.4 mixed quantization)
 * Readings where the pages are silent (all listed in the design notes):
 *   - mu is a per-(batch, head, channel) mean over the valid tokens of that
 *     sequence, summed in fp64 in token order, divided by L, rounded once to fp32.
 *   - sign(0) is +1: bit = (x < mu); bit j of word w is channel 32w + j.
 *   - alpha is one positive scalar per head; NULL means 1.
 *   - top-N selects on the final logit (scale and bias included); ties go to
 *     the lower key index; N == 0 or N >= L keeps every valid key.
 *   - relative-position bias: token t >= prefix is patch (y, x) with
 *     t = prefix + y*gw + x; b_ij = table[h][(y_i - y_j) + gh - 1][(x_i - x_j) + gw - 1];
 *     b = 0 when i or j is a prefix (cls) token or when there is no table.
 *   - dense bias matrix (BinaryAttention §2.3, one learnable bias per query-key
 *     pair), selected by gh == gw == 0 (prefix 0): b_ij = table[h][i][j] of an
 *     [H][n][n] table.
 *   - keys j >= L are never kept; output rows i >= L are 0; bits of tokens
 *     i >= L are 0; the V scales use valid tokens only.
 *   - V scale s_c = absmax_c / 127 in fp32 (1 when absmax is 0);
 *     V_q = clamp(rint(V / s_c), -127, 127), fp32 division, half-to-even.
 *   - A_q = floor(255 p + 0.5) from the normalized fp64 p.
 *   - 4-bit V (mode 2; BinaryAttention's conclusion names lower-bit V as future
 *     work without defining it): the int8 scheme with 4 bits, s_c = absmax_c / 7,
 *     V_q = clamp(rint(V / s_c), -7, 7); O = sum_j A_q V_q * s_c / 255 as in mode 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define HADO_OK 0
#define HADO_ERR_ARG 1
#define HADO_ERR_NOMEM 2

static int valid_len(const int32_t* seqlens, int b, int n) {
  return seqlens ? (int)seqlens[b] : n;
}

int hado_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void hado_set_num_threads(int t) {
#ifdef _OPENMP
  if (t > 0) omp_set_num_threads(t);
#else
  (void)t;
#endif
}

/* Step 1: mu[b][h][c] = (float)( (sum_{i<L} (double)X[b][h][i][c]) / L ), token order. */
int hado_channel_mean(const float* X, int B, int H, int n, int d, const int32_t* seqlens, float* mu) {
  if (!X || !mu || B <= 0 || H <= 0 || n <= 0 || d <= 0) return HADO_ERR_ARG;
  for (int b = 0; b < B; ++b) {
    int L = valid_len(seqlens, b, n);
    if (L < 1 || L > n) return HADO_ERR_ARG;
  }
  /* (b, h) pairs are independent; each channel's sum keeps token order. */
#pragma omp parallel for schedule(static)
  for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
    int b = (int)(bh / H);
    int L = valid_len(seqlens, b, n);
    const float* Xh = X + (size_t)bh * (size_t)n * d;
    for (int c = 0; c < d; ++c) {
      double sum = 0.0;
      for (int i = 0; i < L; ++i) sum += (double)Xh[(size_t)i * d + c];
      mu[(size_t)bh * d + c] = (float)(sum / (double)L);
    }
  }
  return HADO_OK;
}

/* The projection that precedes the path, with its binarization (the step the
 * attention's inputs come from; BinaryAttention's Table 8 counts the Q/K/V
 * quantization of this step against the kernel).  X is [B][n][Dm] tokens,
 * W is [3*H*d][Dm] (output channel o = t*H*d + h*d + c of tensor t in {Q, K, V},
 * the row layout of a linear layer's weight).  Per the plain definition:
 *   P[t][b][h][i][c] = sum_k X[b][i][k] * W[o][k]          (fp64, k in order)
 *   mu_t[b][h][c]    = mean over the valid tokens of P[t]   (fp64 sum in token
 *                      order, divided by L, rounded once to fp32; t in {Q, K})
 *   bits_t           = P[t] < mu_t, packed as in hado_sign_pack (tokens past L: 0)
 * Q, K, V receive P in fp64 [B][H][n][d] (rows past L included). */
int hado_qkv_project(const float* X, const float* W, int B, int n, int Dm, int H, int d, const int32_t* seqlens,
                     double* Q, double* K, double* V, float* mu_q, float* mu_k, uint32_t* qbits, uint32_t* kbits) {
  if (!X || !W || !Q || !K || !V || !mu_q || !mu_k || !qbits || !kbits || B <= 0 || n <= 0 || Dm <= 0 || H <= 0 ||
      d <= 0 || d % 32 != 0)
    return HADO_ERR_ARG;
  for (int b = 0; b < B; ++b) {
    int L = valid_len(seqlens, b, n);
    if (L < 1 || L > n) return HADO_ERR_ARG;
  }
  double* outs[3] = {Q, K, V};
  const int64_t hd = (int64_t)H * d;
#pragma omp parallel for schedule(static)
  for (int64_t bi = 0; bi < (int64_t)B * n; ++bi) {
    int b = (int)(bi / n), i = (int)(bi % n);
    const float* x = X + (size_t)bi * Dm;
    for (int t = 0; t < 3; ++t)
      for (int h = 0; h < H; ++h)
        for (int c = 0; c < d; ++c) {
          const float* w = W + (size_t)(t * hd + (int64_t)h * d + c) * Dm;
          double acc = 0.0;
          for (int k = 0; k < Dm; ++k) acc += (double)x[k] * (double)w[k];
          outs[t][(((size_t)b * H + h) * n + i) * d + c] = acc;
        }
  }
  const int Wd = d / 32;
  for (int t = 0; t < 2; ++t) {
    const double* P = outs[t];
    float* mu = t == 0 ? mu_q : mu_k;
    uint32_t* bits = t == 0 ? qbits : kbits;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
      int L = valid_len(seqlens, (int)(bh / H), n);
      const double* Ph = P + (size_t)bh * n * d;
      for (int c = 0; c < d; ++c) {
        double sum = 0.0;
        for (int i = 0; i < L; ++i) sum += Ph[(size_t)i * d + c];
        mu[(size_t)bh * d + c] = (float)(sum / (double)L);
      }
      for (int i = 0; i < n; ++i)
        for (int w = 0; w < Wd; ++w) {
          uint32_t word = 0;
          if (i < L)
            for (int j = 0; j < 32; ++j) {
              int c = 32 * w + j;
              if (Ph[(size_t)i * d + c] < (double)mu[(size_t)bh * d + c]) word |= (uint32_t)1 << j;
            }
          bits[((size_t)bh * n + i) * Wd + w] = word;
        }
    }
  }
  return HADO_OK;
}

/* Step 2: sign and pack.  bits[b][h][i][w], bit j of word w <=> channel 32w+j is
 * negative after centering (x < mu).  Tokens i >= L get all-zero words. */
int hado_sign_pack(const float* X, const float* mu, int B, int H, int n, int d, const int32_t* seqlens,
                   uint32_t* bits) {
  if (!X || !mu || !bits || B <= 0 || H <= 0 || n <= 0 || d <= 0 || d % 32 != 0) return HADO_ERR_ARG;
  int W = d / 32;
#pragma omp parallel for schedule(static)
  for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
    int L = valid_len(seqlens, (int)(bh / H), n);
    const float* Xh = X + (size_t)bh * (size_t)n * d;
    const float* m = mu + (size_t)bh * d;
    uint32_t* out = bits + (size_t)bh * (size_t)n * W;
    for (int i = 0; i < n; ++i) {
      for (int w = 0; w < W; ++w) {
        uint32_t word = 0;
        if (i < L) {
          for (int j = 0; j < 32; ++j) {
            int c = 32 * w + j;
            if (Xh[(size_t)i * d + c] < m[c]) word |= (uint32_t)1 << j;
          }
        }
        out[(size_t)i * W + w] = word;
      }
    }
  }
  return HADO_OK;
}

static int popcount32(uint32_t x) {
  int c = 0;
  while (x) {
    c += (int)(x & 1u);
    x >>= 1;
  }
  return c;
}

/* Step 3: binary score s = d - 2 * Hamming(q, k) over the d packed bits. */
static int binary_score(const uint32_t* q, const uint32_t* k, int d) {
  int W = d / 32, ham = 0;
  for (int w = 0; w < W; ++w) ham += popcount32(q[w] ^ k[w]);
  return d - 2 * ham;
}

/* Integer score matrix for parity of the score step.  S[b][h][i][j] = s for
 * i, j < L; 0 elsewhere. */
int hado_binary_scores(const uint32_t* qbits, const uint32_t* kbits, int B, int H, int n, int d,
                       const int32_t* seqlens, int32_t* S) {
  if (!qbits || !kbits || !S || d % 32 != 0) return HADO_ERR_ARG;
  int W = d / 32;
  for (int b = 0; b < B; ++b) {
    int L = valid_len(seqlens, b, n);
    for (int h = 0; h < H; ++h) {
      size_t bh = (size_t)b * H + h;
      for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) {
          int32_t v = 0;
          if (i < L && j < L) v = binary_score(qbits + (bh * n + i) * W, kbits + (bh * n + j) * W, d);
          S[(bh * n + i) * (size_t)n + j] = v;
        }
    }
  }
  return HADO_OK;
}

/* Per-channel symmetric int8 quantization of V (BinaryAttention §2.4, V bullet). */
/* Per-channel symmetric quantization of V to the integers [-qmax, qmax] with
 * scale absmax / qmax: qmax = 127 is the int8 V of BinaryAttention §2.4 (V
 * bullet), qmax = 7 the 4-bit V of mode 2. */
static int v_quant_q(const float* V, int B, int H, int n, int d, const int32_t* seqlens, float qmax, int8_t* Vq,
                     float* scale) {
  if (!V || !Vq || !scale) return HADO_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
    int L = valid_len(seqlens, (int)(bh / H), n);
    const float* Vh = V + (size_t)bh * (size_t)n * d;
    for (int c = 0; c < d; ++c) {
      float amax = 0.0f;
      for (int i = 0; i < L; ++i) {
        float a = fabsf(Vh[(size_t)i * d + c]);
        if (a > amax) amax = a;
      }
      float s = (amax > 0.0f) ? amax / qmax : 1.0f;
      scale[(size_t)bh * d + c] = s;
      for (int i = 0; i < n; ++i) {
        int8_t qv = 0;
        if (i < L) {
          float r = rintf(Vh[(size_t)i * d + c] / s);
          if (r > qmax) r = qmax;
          if (r < -qmax) r = -qmax;
          qv = (int8_t)r;
        }
        Vq[((size_t)bh * n + i) * (size_t)d + c] = qv;
      }
    }
  }
  return HADO_OK;
}

int hado_v_quant(const float* V, int B, int H, int n, int d, const int32_t* seqlens, int8_t* Vq, float* scale) {
  return v_quant_q(V, B, H, n, d, seqlens, 127.0f, Vq, scale);
}

/* 4-bit V (mode 2): integers in [-7, 7], scale absmax / 7. */
int hado_v_quant4(const float* V, int B, int H, int n, int d, const int32_t* seqlens, int8_t* Vq, float* scale) {
  return v_quant_q(V, B, H, n, d, seqlens, 7.0f, Vq, scale);
}

/* Bias b_ij for head h (readings stated in the header): the relative-position
 * table, or with gh == gw == 0 the dense matrix [H][n][n]. */
static float rel_bias(const float* table, int H, int h, int gh, int gw, int prefix, int n, int i, int j) {
  (void)H;
  if (table && gh == 0 && gw == 0) return table[((size_t)h * n + i) * n + j];
  if (!table || i < prefix || j < prefix) return 0.0f;
  int ti = i - prefix, tj = j - prefix;
  int yi = ti / gw, xi = ti % gw, yj = tj / gw, xj = tj % gw;
  int th = 2 * gh - 1, tw = 2 * gw - 1;
  int r = (yi - yj) + gh - 1, c = (xi - xj) + gw - 1;
  return table[((size_t)h * th + r) * tw + c];
}

/* The logit scale c = fp32(alpha_q * alpha_k / sqrt(d)). */
static float logit_scale(const float* alpha_q, const float* alpha_k, int h, int d) {
  double aq = alpha_q ? (double)alpha_q[h] : 1.0;
  double ak = alpha_k ? (double)alpha_k[h] : 1.0;
  return (float)(aq * ak / sqrt((double)d));
}

typedef struct {
  float l;
  int j;
} keyed;

/* Total order of the top-N selection: larger logit first, then lower key index. */
static int by_logit_desc_index_asc(const void* pa, const void* pb) {
  const keyed* a = (const keyed*)pa;
  const keyed* b = (const keyed*)pb;
  if (a->l > b->l) return -1;
  if (a->l < b->l) return 1;
  return (a->j < b->j) ? -1 : (a->j > b->j ? 1 : 0);
}

static int by_int_asc(const void* pa, const void* pb) {
  int a = *(const int*)pa, b = *(const int*)pb;
  return (a > b) - (a < b);
}

/* Logit matrix l[b][h][i][j] for i, j < L (NAN elsewhere) from packed bits. */
int hado_logits(const uint32_t* qbits, const uint32_t* kbits, int B, int H, int n, int d, const int32_t* seqlens,
                const float* table, int gh, int gw, int prefix, const float* alpha_q, const float* alpha_k,
                float* out) {
  if (!qbits || !kbits || !out || d % 32 != 0) return HADO_ERR_ARG;
  int W = d / 32;
  for (int b = 0; b < B; ++b) {
    int L = valid_len(seqlens, b, n);
    for (int h = 0; h < H; ++h) {
      size_t bh = (size_t)b * H + h;
      float c = logit_scale(alpha_q, alpha_k, h, d);
      for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) {
          float v = NAN;
          if (i < L && j < L) {
            int s = binary_score(qbits + (bh * n + i) * W, kbits + (bh * n + j) * W, d);
            v = fmaf((float)s, c, rel_bias(table, H, h, gh, gw, prefix, n, i, j));
          }
          out[(bh * n + i) * (size_t)n + j] = v;
        }
    }
  }
  return HADO_OK;
}

/*
 * The whole forward pass.  mode 0 = float A.V, mode 1 = uint8 A x int8 V, mode 2 = uint8 A x 4-bit V.
 * rows: optional list of flat row ids ((b*H + h)*n + i); NULL = all B*H*n rows.
 * Outputs (row-major over the selected rows):
 *   O   [nrows][d]  fp64 (required)
 *   idx [nrows][N]  kept key indices ascending, -1 padded (optional; needs N > 0)
 *   Aq  [nrows][n]  uint8 codes floor(255 p + 0.5), 0 off the kept set (optional)
 *   P   [nrows][n]  fp64 probabilities, 0 off the kept set (optional)
 * Intermediates (optional, full size): mu_q/mu_k [B][H][d], qbits/kbits
 * [B][H][n][d/32], Vq [B][H][n][d], vscale [B][H][d].
 */
int hado_attention(const float* Q, const float* K, const float* V, int B, int H, int n, int d,
                   const int32_t* seqlens, const float* table, int gh, int gw, int prefix, const float* alpha_q,
                   const float* alpha_k, int N, int mode, const int64_t* rows, int64_t nrows, double* O,
                   int32_t* idx, uint8_t* Aq, double* P, float* mu_q_out, float* mu_k_out, uint32_t* qbits_out,
                   uint32_t* kbits_out, int8_t* Vq_out, float* vscale_out) {
  if (!Q || !K || !V || !O || B <= 0 || H <= 0 || n <= 0 || d <= 0 || d % 32 != 0 || N < 0) return HADO_ERR_ARG;
  if (mode != 0 && mode != 1 && mode != 2) return HADO_ERR_ARG;
  if (table && !(gh == 0 && gw == 0 && prefix == 0) &&
      (gh <= 0 || gw <= 0 || prefix < 0 || (int64_t)gh * gw + prefix != n))
    return HADO_ERR_ARG;
  for (int h = 0; h < H; ++h) {
    if (alpha_q && !(alpha_q[h] > 0.0f)) return HADO_ERR_ARG;
    if (alpha_k && !(alpha_k[h] > 0.0f)) return HADO_ERR_ARG;
  }
  for (int b = 0; b < B; ++b) {
    int L = valid_len(seqlens, b, n);
    if (L < 1 || L > n) return HADO_ERR_ARG;
  }
  int W = d / 32;
  size_t nbh = (size_t)B * H;
  float* mu_q = (float*)malloc(nbh * d * sizeof(float));
  float* mu_k = (float*)malloc(nbh * d * sizeof(float));
  uint32_t* qb = (uint32_t*)malloc(nbh * n * W * sizeof(uint32_t));
  uint32_t* kb = (uint32_t*)malloc(nbh * n * W * sizeof(uint32_t));
  int8_t* Vq = (int8_t*)malloc(nbh * n * d);
  float* vs = (float*)malloc(nbh * d * sizeof(float));
  if (!mu_q || !mu_k || !qb || !kb || !Vq || !vs) {
    free(mu_q); free(mu_k); free(qb); free(kb); free(Vq); free(vs);
    return HADO_ERR_NOMEM;
  }
  hado_channel_mean(Q, B, H, n, d, seqlens, mu_q);
  hado_channel_mean(K, B, H, n, d, seqlens, mu_k);
  hado_sign_pack(Q, mu_q, B, H, n, d, seqlens, qb);
  hado_sign_pack(K, mu_k, B, H, n, d, seqlens, kb);
  if (mode == 2) hado_v_quant4(V, B, H, n, d, seqlens, Vq, vs);
  else hado_v_quant(V, B, H, n, d, seqlens, Vq, vs);

  int64_t total = rows ? nrows : (int64_t)nbh * n;
  int failed = 0;
#pragma omp parallel for schedule(dynamic, 8)
  for (int64_t r = 0; r < total; ++r) {
    int64_t flat = rows ? rows[r] : r;
    int i = (int)(flat % n);
    int64_t bh = flat / n;
    int h = (int)(bh % H), b = (int)(bh / H);
    int L = valid_len(seqlens, b, n);
    double* o = O + (size_t)r * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (idx)
      for (int t = 0; t < N; ++t) idx[(size_t)r * N + t] = -1;
    if (Aq)
      for (int j = 0; j < n; ++j) Aq[(size_t)r * n + j] = 0;
    if (P)
      for (int j = 0; j < n; ++j) P[(size_t)r * n + j] = 0.0;
    if (i >= L) continue;

    keyed* key = (keyed*)malloc((size_t)L * sizeof(keyed));
    double* e = (double*)malloc((size_t)L * sizeof(double));
    int* kept = (int*)malloc((size_t)L * sizeof(int));
    if (!key || !e || !kept) {
      free(key); free(e); free(kept);
#pragma omp atomic write
      failed = 1;
      continue;
    }
    /* Steps 3-4: score and logit for every valid key. */
    float c = logit_scale(alpha_q, alpha_k, h, d);
    const uint32_t* q = qb + ((size_t)bh * n + i) * W;
    for (int j = 0; j < L; ++j) {
      int s = binary_score(q, kb + ((size_t)bh * n + j) * W, d);
      key[j].l = fmaf((float)s, c, rel_bias(table, H, h, gh, gw, prefix, n, i, j));
      key[j].j = j;
    }
    /* Step 5: the kept set is the first K_eff keys of the full sort. */
    int keff = (N == 0 || N >= L) ? L : N;
    qsort(key, (size_t)L, sizeof(keyed), by_logit_desc_index_asc);
    for (int t = 0; t < keff; ++t) kept[t] = key[t].j;
    /* Step 6: softmax over the kept keys in fp64. */
    double m = -INFINITY;
    for (int t = 0; t < keff; ++t)
      if ((double)key[t].l > m) m = (double)key[t].l;
    double denom = 0.0;
    for (int t = 0; t < keff; ++t) {
      e[t] = exp((double)key[t].l - m);
      denom += e[t];
    }
    /* Step 7: A.V. */
    const float* Vh = V + (size_t)bh * n * d;
    const int8_t* Vqh = Vq + (size_t)bh * n * d;
    const float* sh = vs + (size_t)bh * d;
    if (mode == 0) {
      for (int t = 0; t < keff; ++t) {
        double p = e[t] / denom;
        int j = kept[t];
        for (int cc = 0; cc < d; ++cc) o[cc] += p * (double)Vh[(size_t)j * d + cc];
      }
    } else {
      int64_t* acc = (int64_t*)calloc((size_t)d, sizeof(int64_t));
      if (!acc) {
#pragma omp atomic write
        failed = 1;
      } else {
        for (int t = 0; t < keff; ++t) {
          double p = e[t] / denom;
          int64_t a = (int64_t)floor(255.0 * p + 0.5);
          int j = kept[t];
          for (int cc = 0; cc < d; ++cc) acc[cc] += a * (int64_t)Vqh[(size_t)j * d + cc];
        }
        for (int cc = 0; cc < d; ++cc) o[cc] = (double)acc[cc] * (double)sh[cc] / 255.0;
        free(acc);
      }
    }
    if (Aq || P) {
      for (int t = 0; t < keff; ++t) {
        double p = e[t] / denom;
        if (Aq) Aq[(size_t)r * n + kept[t]] = (uint8_t)floor(255.0 * p + 0.5);
        if (P) P[(size_t)r * n + kept[t]] = p;
      }
    }
    if (idx && N > 0) {
      int cnt = keff < N ? keff : N;
      qsort(kept, (size_t)keff, sizeof(int), by_int_asc);
      for (int t = 0; t < cnt; ++t) idx[(size_t)r * N + t] = kept[t];
    }
    free(key);
    free(e);
    free(kept);
  }

  if (mu_q_out) memcpy(mu_q_out, mu_q, nbh * d * sizeof(float));
  if (mu_k_out) memcpy(mu_k_out, mu_k, nbh * d * sizeof(float));
  if (qbits_out) memcpy(qbits_out, qb, nbh * n * W * sizeof(uint32_t));
  if (kbits_out) memcpy(kbits_out, kb, nbh * n * W * sizeof(uint32_t));
  if (Vq_out) memcpy(Vq_out, Vq, nbh * n * d);
  if (vscale_out) memcpy(vscale_out, vs, nbh * d * sizeof(float));
  free(mu_q); free(mu_k); free(qb); free(kb); free(Vq); free(vs);
  return failed ? HADO_ERR_NOMEM : HADO_OK;
}

/*
 * Dense standard attention on the unbinarized inputs, for the library's
 * comparison mode: l = (q . k) / sqrt(d) + b_ij with q, k taken as given (the
 * caller rounds them to bf16 first when the device inputs are bf16), fp64
 * throughout, then top-N by (l desc, j asc) and softmax.  O fp64.
 */
int hado_dense_attention(const float* Q, const float* K, const float* V, int B, int H, int n, int d,
                         const int32_t* seqlens, const float* table, int gh, int gw, int prefix, int N,
                         const int64_t* rows, int64_t nrows, double* O) {
  if (!Q || !K || !V || !O || B <= 0 || H <= 0 || n <= 0 || d <= 0 || N < 0) return HADO_ERR_ARG;
  if (table && !(gh == 0 && gw == 0 && prefix == 0) &&
      (gh <= 0 || gw <= 0 || prefix < 0 || (int64_t)gh * gw + prefix != n))
    return HADO_ERR_ARG;
  for (int b = 0; b < B; ++b) {
    int L = valid_len(seqlens, b, n);
    if (L < 1 || L > n) return HADO_ERR_ARG;
  }
  int64_t total = rows ? nrows : (int64_t)B * H * n;
  int failed = 0;
#pragma omp parallel for schedule(dynamic, 8)
  for (int64_t r = 0; r < total; ++r) {
    int64_t flat = rows ? rows[r] : r;
    int i = (int)(flat % n);
    int64_t bh = flat / n;
    int h = (int)(bh % H), b = (int)(bh / H);
    int L = valid_len(seqlens, b, n);
    double* o = O + (size_t)r * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (i >= L) continue;
    double* l = (double*)malloc((size_t)L * sizeof(double));
    int* order = (int*)malloc((size_t)L * sizeof(int));
    if (!l || !order) {
      free(l); free(order);
#pragma omp atomic write
      failed = 1;
      continue;
    }
    const float* q = Q + ((size_t)bh * n + i) * d;
    for (int j = 0; j < L; ++j) {
      const float* k = K + ((size_t)bh * n + j) * d;
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += (double)q[c] * (double)k[c];
      l[j] = dot / sqrt((double)d) + (double)rel_bias(table, H, h, gh, gw, prefix, n, i, j);
      order[j] = j;
    }
    int keff = (N == 0 || N >= L) ? L : N;
    /* selection by repeated maximum (ties to the lower index), plain O(L*keff) */
    for (int t = 0; t < keff; ++t) {
      int best = t;
      for (int u = t + 1; u < L; ++u) {
        if (l[order[u]] > l[order[best]] || (l[order[u]] == l[order[best]] && order[u] < order[best])) best = u;
      }
      int tmp = order[t];
      order[t] = order[best];
      order[best] = tmp;
    }
    double m = -INFINITY;
    for (int t = 0; t < keff; ++t)
      if (l[order[t]] > m) m = l[order[t]];
    double denom = 0.0;
    for (int t = 0; t < keff; ++t) denom += exp(l[order[t]] - m);
    const float* Vh = V + (size_t)bh * n * d;
    for (int t = 0; t < keff; ++t) {
      int j = order[t];
      double p = exp(l[j] - m) / denom;
      for (int c = 0; c < d; ++c) o[c] += p * (double)Vh[(size_t)j * d + c];
    }
    free(l);
    free(order);
  }
  return failed ? HADO_ERR_NOMEM : HADO_OK;
}
