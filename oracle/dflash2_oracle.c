/*
 * CPU oracle for the DFlash 2 drafter block step.  TEST INFRASTRUCTURE ONLY:
 * tests, the package's smoke check and the benchmark's CPU-baseline leg use it;
 * the product path never links, loads or calls it.  It shares no code, header
 * or constant table with the CUDA path.
 *
 * Plain, slow, obviously correct: every step is written out in double
 * precision straight from its definition, one request at a time, with OpenMP
 * only over independent output rows of a matrix product.  bf16 and fp16
 * operands are widened exactly; Q4_K weights are decoded exactly
 * (d*sc*q - dmin*m from fp16 d/dmin and small integers).  The oracle never
 * rounds activations; the one place it rounds is the KV cache, which is a
 * 16-bit store by definition (aiqre.com model page, "Memory": 20 KiB per
 * token at 16-bit).
 *
 * Sources (web pages on the DFlash 2 drafter):
 *  - FastFlowLM model card, "Draft" row: 5 Qwen3-style layers, hidden 5120,
 *    FFN 17408, 32 query / 8 key-value heads of 128, sliding window 2048,
 *    block of 8, two-tap dynamic convolutions, candidate selector (top 16,
 *    rank 256), shared embedding table and output head.
 *  - same card, "Weights" row: Q4_K matrices; norms, dynamic-convolution
 *    tensors, selector projection and two 248320 x 256 codebooks in BF16.
 *  - same card, "Taps" row: features of target layers 5, 19, 33, 47, 61,
 *    fused by the draft's fc layer.
 *  - same card, "How it is used": 7 tokens proposed in one pass, one coherent
 *    path through the top-16 candidates per position, the target keeps the
 *    longest agreeing prefix plus one token of its own.
 *  - MLX sidecar card ("Contents"): the drafter reads the residual stream at
 *    five tapped layers and proposes a whole block in one forward.
 * Where the pages leave a formula open, the reading taken is stated at the
 * function that implements it (dynamic convolution, selector score, RoPE,
 * norm epsilon, tie-breaks).
 *
 * Parity pins: see tests/test_oracle_*.py.  Every exported function below is
 * pinned by at least one closed form, invariant, brute-force enumeration or
 * library routine there.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_MAX_LAYERS 8

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_TOKEN (-2)
#define ORC_ERR_PAGE (-3)
#define ORC_ERR_NOMEM (-4)

typedef struct {
  int32_t layers, hidden, ffn, n_q, n_kv, head_dim, window, vocab, n_taps, block, topk, rank,
      page_size, wfmt; /* fc and layer matrices: 0 = Q4_K, 1 = bf16, 2 = MLX 4-bit g64, 3 = Q8_0 */
  double rope_theta, rms_eps;
} orc_dims;

typedef struct {
  const void *wq, *wk, *wv, *wo, *wg, *wu, *wd;
  const uint16_t *ln1, *ln2, *qn, *kn, *dc_w, *dc_s0, *dc_s1;
} orc_layer;

typedef struct {
  const void *fc;
  const uint16_t *fc_norm;
  orc_layer layer[ORC_MAX_LAYERS];
  const uint16_t *final_norm, *embed, *lm_head, *sel_proj, *cb_a, *cb_b;
} orc_weights;

/* Optional per-request traces; any pointer may be NULL. */
typedef struct {
  double *hidden;     /* [layers+1][block][hidden]: after embedding, then after each layer */
  double *ctx;        /* [block][hidden]: fc output after its RMSNorm (rows < n_new) */
  double *final_h;    /* [block-1][hidden]: final-normed rows 1..block-1 */
  int32_t *cand;      /* [block-1][topk] */
  double *cand_logit; /* [block-1][topk] */
  double *z;          /* [block-1][rank] */
  double *q0;         /* [block][n_q*head_dim]: layer 0 block queries after q-norm and RoPE */
  double *k0;         /* [block][n_kv*head_dim]: layer 0 block keys after k-norm and RoPE */
} orc_trace;

/* ------------------------------------------------------------------ */
/* number formats                                                       */

double orc_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

double orc_fp16(uint16_t h) {
  int sign = (h >> 15) & 1, ex = (h >> 10) & 31, man = h & 1023;
  double v;
  if (ex == 0)
    v = ldexp((double)man, -24);
  else if (ex == 31)
    v = man ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + man), ex - 25);
  return sign ? -v : v;
}

/* Round to the nearest bf16, ties to even (8 significant bits). */
uint16_t orc_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
  int e;
  double m = frexp(fabs(x), &e);
  double v = ldexp(nearbyint(ldexp(m, 8)), e - 8);
  float f = (float)(signbit(x) ? -v : v);
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

/* One 144-byte Q4_K super-block -> 256 weights.
 * Layout: d (fp16), dmin (fp16), eight 6-bit scales packed little-endian in 6
 * bytes, eight 6-bit mins likewise, 128 bytes of 4-bit codes (element e at byte
 * 16 + e/2, low nibble first).  Weight e = d*sc[e/32]*q[e] - dmin*m[e/32].
 * The card fixes the Q4_K family (FastFlowLM card, "Weights" row); the
 * super-block of 256 with 6-bit sub-scales and sub-mins is the Q4_K format. */
static void q4k_block(const uint8_t *b, double *out) {
  double d = orc_fp16((uint16_t)(b[0] | (b[1] << 8)));
  double dmin = orc_fp16((uint16_t)(b[2] | (b[3] << 8)));
  uint64_t scp = 0, mp = 0;
  for (int i = 0; i < 6; ++i) {
    scp |= (uint64_t)b[4 + i] << (8 * i);
    mp |= (uint64_t)b[10 + i] << (8 * i);
  }
  for (int e = 0; e < 256; ++e) {
    int j = e / 32;
    int sc = (int)((scp >> (6 * j)) & 63), m = (int)((mp >> (6 * j)) & 63);
    int byte = b[16 + e / 2];
    int q = (e & 1) ? (byte >> 4) : (byte & 15);
    out[e] = d * sc * q - dmin * m;
  }
}

void orc_q4k_dequant(const uint8_t *blocks, int64_t nblocks, double *out) {
  for (int64_t i = 0; i < nblocks; ++i) q4k_block(blocks + 144 * i, out + 256 * i);
}

/* MLX-style 4-bit group-64 (MLX sidecar card, "Contents": 4-bit weights in groups of 64): each
 * group of 64 consecutive weights of a row is stored as 32 bytes of 4-bit codes (element e at byte
 * e/2, low nibble first; the uint32-packed order of MLX read little-endian) followed by its scale
 * and bias in bf16 (36 bytes per group); weight e = scale * q_e + bias. */
void orc_mlx4_dequant(const uint8_t *groups, int64_t ngroups, double *out) {
  for (int64_t g = 0; g < ngroups; ++g) {
    const uint8_t *b = groups + 36 * g;
    const double sc = orc_bf16((uint16_t)(b[32] | (b[33] << 8)));
    const double bi = orc_bf16((uint16_t)(b[34] | (b[35] << 8)));
    for (int e = 0; e < 64; ++e) {
      const int q = (e & 1) ? (b[e / 2] >> 4) : (b[e / 2] & 15);
      out[64 * g + e] = sc * q + bi;
    }
  }
}

/* Q8_0 (Mindket listing, "Good to know": Q8_0 files): blocks of 32 weights, an fp16 scale d then
 * 32 signed 8-bit codes (34 bytes); weight e = d * q_e. */
void orc_q8_0_dequant(const uint8_t *blocks, int64_t nblocks, double *out) {
  for (int64_t i = 0; i < nblocks; ++i) {
    const uint8_t *b = blocks + 34 * i;
    const double d = orc_fp16((uint16_t)(b[0] | (b[1] << 8)));
    for (int e = 0; e < 32; ++e) out[32 * i + e] = d * (double)(int8_t)b[2 + e];
  }
}

/* Row n of a [N, K] matrix stored as Q4_K (fmt 0), bf16 (fmt 1), MLX 4-bit group-64 (fmt 2) or
 * Q8_0 (fmt 3). */
static void weight_row(int fmt, const void *W, int K, int64_t n, double *row) {
  if (fmt == 0) {
    orc_q4k_dequant((const uint8_t *)W + (int64_t)n * (K / 256) * 144, K / 256, row);
  } else if (fmt == 2) {
    orc_mlx4_dequant((const uint8_t *)W + (int64_t)n * (K / 64) * 36, K / 64, row);
  } else if (fmt == 3) {
    orc_q8_0_dequant((const uint8_t *)W + (int64_t)n * (K / 32) * 34, K / 32, row);
  } else {
    const uint16_t *r = (const uint16_t *)W + (int64_t)n * K;
    for (int k = 0; k < K; ++k) row[k] = orc_bf16(r[k]);
  }
}

/* Y[m][n] = sum_k W[n][k] * X[m][k] for m < M, n < N. */
void orc_matmul(int fmt, const void *W, int N, int K, const double *X, int M, double *Y) {
#pragma omp parallel
  {
    double *row = (double *)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(static)
    for (int n = 0; n < N; ++n) {
      weight_row(fmt, W, K, n, row);
      for (int m = 0; m < M; ++m) {
        const double *x = X + (int64_t)m * K;
        double s = 0.0;
        for (int k = 0; k < K; ++k) s += row[k] * x[k];
        Y[(int64_t)m * N + n] = s;
      }
    }
    free(row);
  }
}

/* ------------------------------------------------------------------ */
/* elementwise pieces                                                   */

/* RMSNorm of a Qwen3-style layer (FastFlowLM card, "Draft" row):
 * y = x / sqrt(mean(x^2) + eps) * w. */
void orc_rmsnorm(const double *x, int n, const uint16_t *w, double eps, double *y) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double r = 1.0 / sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) y[i] = x[i] * r * orc_bf16(w[i]);
}

/* Rotary embedding, Qwen3 convention ("Qwen3-style", FastFlowLM card): the
 * head vector is split into halves (i, i + hd/2) that rotate by pos*theta^(-2i/hd). */
void orc_rope(double *v, int hd, int64_t pos, double theta) {
  int half = hd / 2;
  for (int i = 0; i < half; ++i) {
    double inv = pow(theta, -2.0 * i / hd);
    double a = (double)pos * inv, c = cos(a), s = sin(a);
    double x0 = v[i], x1 = v[i + half];
    v[i] = x0 * c - x1 * s;
    v[i + half] = x1 * c + x0 * s;
  }
}

static double silu(double x) { return x / (1.0 + exp(-x)); }

/* Two-tap dynamic convolution along the block (FastFlowLM card, "Draft" row;
 * Mindket listing, "For newcomers and experts": it sits inside the backbone and
 * keeps draft quality from falling along the block).  The pages give no
 * formula; the reading fixed here:
 *   g_t = W_dc x_t, W_dc in R^{2(H/4) x H}; gate value c/4 is shared by 4 channels
 *   y_t[c] = (s0[c] + tanh g_t[c/4]) * x_t[c] + (s1[c] + tanh g_t[H/4 + c/4]) * x_{t-1}[c]
 * causal along block positions, x_{-1} = 0.  x, y: [Bk][H]. */
void orc_dynconv(int Bk, int H, const double *x, const uint16_t *dc_w, const uint16_t *s0,
                 const uint16_t *s1, double *y) {
  int G = H / 4;
  double *g = (double *)malloc(sizeof(double) * (size_t)Bk * 2 * G);
  orc_matmul(1, dc_w, 2 * G, H, x, Bk, g);
  for (int t = 0; t < Bk; ++t)
    for (int c = 0; c < H; ++c) {
      double a0 = orc_bf16(s0[c]) + tanh(g[(int64_t)t * 2 * G + c / 4]);
      double a1 = orc_bf16(s1[c]) + tanh(g[(int64_t)t * 2 * G + G + c / 4]);
      double prev = t > 0 ? x[(int64_t)(t - 1) * H + c] : 0.0;
      y[(int64_t)t * H + c] = a0 * x[(int64_t)t * H + c] + a1 * prev;
    }
  free(g);
}

/* ------------------------------------------------------------------ */
/* attention                                                            */

static const uint16_t *cache_row(const uint16_t *cache, const orc_dims *c, int32_t page, int head,
                                 int slot) {
  return cache + (((int64_t)page * c->n_kv + head) * c->page_size + slot) * c->head_dim;
}

/* Sliding-window GQA attention of the block rows (FastFlowLM card, "Draft" row:
 * 32 query / 8 key-value heads of 128, sliding window 2048).  Block row t sits
 * at position p = Lb + t.  It sees cache keys j with max(0, p - W + 1) <= j < Lb
 * (the window, read from the 16-bit paged cache) and all block keys kb/vb of
 * this step (bidirectional inside the block, positions Lb..Lb+Bk-1).
 * Scores q.k / sqrt(hd), softmax, weighted sum of values.  Query head h reads
 * key-value head h / (n_q / n_kv).
 * q, o: [Bk][n_q*hd]; kb, vb: [Bk][n_kv*hd]; caches: [pages][n_kv][page][hd]. */
int orc_attention(const orc_dims *c, int Bk, const double *q, const double *kb, const double *vb,
                  const uint16_t *kcache, const uint16_t *vcache, const int32_t *page_table,
                  int max_pages, int64_t Lb, double *o) {
  int hd = c->head_dim, nq = c->n_q, nkv = c->n_kv, grp = nq / nkv;
  int64_t maxkeys = (int64_t)c->window + Bk;
  double *s = (double *)malloc(sizeof(double) * (size_t)maxkeys);
  int err = ORC_OK;
  double scale = 1.0 / sqrt((double)hd);
  for (int t = 0; t < Bk && err == ORC_OK; ++t) {
    int64_t p = Lb + t;
    int64_t j0 = p - c->window + 1;
    if (j0 < 0) j0 = 0;
    for (int h = 0; h < nq && err == ORC_OK; ++h) {
      int kvh = h / grp;
      const double *qv = q + ((int64_t)t * nq + h) * hd;
      int64_t n = 0;
      for (int64_t j = j0; j < Lb; ++j) {
        int64_t lp = j / c->page_size;
        if (lp >= max_pages || page_table[lp] < 0) { err = ORC_ERR_PAGE; break; }
        const uint16_t *kr = cache_row(kcache, c, page_table[lp], kvh, (int)(j % c->page_size));
        double d = 0.0;
        for (int i = 0; i < hd; ++i) d += qv[i] * orc_bf16(kr[i]);
        s[n++] = d * scale;
      }
      if (err != ORC_OK) break;
      for (int u = 0; u < Bk; ++u) {
        const double *kr = kb + ((int64_t)u * nkv + kvh) * hd;
        double d = 0.0;
        for (int i = 0; i < hd; ++i) d += qv[i] * kr[i];
        s[n++] = d * scale;
      }
      double mx = s[0];
      for (int64_t i = 1; i < n; ++i) mx = s[i] > mx ? s[i] : mx;
      double den = 0.0;
      for (int64_t i = 0; i < n; ++i) { s[i] = exp(s[i] - mx); den += s[i]; }
      double *ov = o + ((int64_t)t * nq + h) * hd;
      for (int i = 0; i < hd; ++i) ov[i] = 0.0;
      int64_t idx = 0;
      for (int64_t j = j0; j < Lb; ++j, ++idx) {
        const uint16_t *vr = cache_row(vcache, c, page_table[j / c->page_size], kvh,
                                       (int)(j % c->page_size));
        double wgt = s[idx] / den;
        for (int i = 0; i < hd; ++i) ov[i] += wgt * orc_bf16(vr[i]);
      }
      for (int u = 0; u < Bk; ++u, ++idx) {
        const double *vr = vb + ((int64_t)u * nkv + kvh) * hd;
        double wgt = s[idx] / den;
        for (int i = 0; i < hd; ++i) ov[i] += wgt * vr[i];
      }
    }
  }
  free(s);
  return err;
}

/* ------------------------------------------------------------------ */
/* candidates, selector, acceptance                                     */

/* (a, ia) ranks before (b, ib): larger value first, smaller id on equal values. */
static int better(double a, int32_t ia, double b, int32_t ib) { return a > b || (a == b && ia < ib); }

/* The K best of n logits (FastFlowLM card: top 16 candidates per position),
 * ordered by logit descending, then token id ascending. */
void orc_topk(const double *logits, int n, int K, int32_t *ids, double *vals) {
  int have = 0;
  for (int i = 0; i < n; ++i) {
    double v = logits[i];
    if (have == K && !better(v, i, vals[K - 1], ids[K - 1])) continue;
    int pos = have < K ? have++ : K - 1;
    while (pos > 0 && better(v, i, vals[pos - 1], ids[pos - 1])) {
      vals[pos] = vals[pos - 1];
      ids[pos] = ids[pos - 1];
      --pos;
    }
    vals[pos] = v;
    ids[pos] = i;
  }
}

/* Max-sum path over D positions x K candidates (the selector "picks one
 * coherent path through its top 16 candidates", FastFlowLM card).
 *   delta_0(j) = unary[0][j] + trans[0][0][j]           (one source: the block's first token)
 *   delta_t(j) = unary[t][j] + max_i (delta_{t-1}(i) + trans[t][i][j])
 * Ties: the smaller candidate index wins, both in the max over i and in the
 * final argmax.  Outputs the chosen index per position and delta_t along it.
 * unary: [D][K]; trans: [D][K][K] (row i = source, column j = destination). */
void orc_viterbi(int D, int K, const double *unary, const double *trans, int32_t *idx,
                 double *scores) {
  double *delta = (double *)malloc(sizeof(double) * (size_t)D * K);
  int32_t *bp = (int32_t *)malloc(sizeof(int32_t) * (size_t)D * K);
  for (int j = 0; j < K; ++j) {
    delta[j] = unary[j] + trans[j];
    bp[j] = 0;
  }
  for (int t = 1; t < D; ++t)
    for (int j = 0; j < K; ++j) {
      double best = 0.0;
      int bi = -1;
      for (int i = 0; i < K; ++i) {
        double s = delta[(t - 1) * K + i] + trans[((int64_t)t * K + i) * K + j];
        if (bi < 0 || s > best) { best = s; bi = i; }
      }
      delta[t * K + j] = unary[t * K + j] + best;
      bp[t * K + j] = bi;
    }
  int j = 0;
  for (int i = 1; i < K; ++i)
    if (delta[(D - 1) * K + i] > delta[(D - 1) * K + j]) j = i;
  for (int t = D - 1; t >= 0; --t) {
    idx[t] = j;
    scores[t] = delta[t * K + j];
    j = bp[t * K + j];
  }
  free(delta);
  free(bp);
}

/* Selector transition scores and path (FastFlowLM card: selector with top 16 and
 * rank 256; "Weights" row: a selector projection and two 248320 x 256 codebooks).
 * The pages give no score formula; the reading fixed here is a rank-R bilinear
 * transition through the position's projected state:
 *   tau_t(a -> b) = sum_r A[a][r] * z_t[r] * Bc[b][r],  z_t = W_s h~_t
 * with A = first codebook (source token), Bc = second codebook (destination),
 * unary score = the candidate's raw logit (a per-position log-softmax shift
 * does not move the argmax path).  Sources at position 0 are the block's first
 * token x0, at position t > 0 the candidates of position t-1.
 * cand: [D][K]; z: [D][R]; trans: [D][K][K] (row = source index, column = destination). */
void orc_selector_trans(int D, int K, int R, const int32_t *cand, const double *z, int32_t x0,
                        const uint16_t *cb_a, const uint16_t *cb_b, double *trans) {
  memset(trans, 0, sizeof(double) * (size_t)D * K * K);
  for (int t = 0; t < D; ++t) {
    int nsrc = t == 0 ? 1 : K;
    for (int i = 0; i < nsrc; ++i) {
      int32_t a = t == 0 ? x0 : cand[(t - 1) * K + i];
      for (int j = 0; j < K; ++j) {
        int32_t b = cand[t * K + j];
        double s = 0.0;
        for (int r = 0; r < R; ++r)
          s += orc_bf16(cb_a[(int64_t)a * R + r]) * z[(int64_t)t * R + r] *
               orc_bf16(cb_b[(int64_t)b * R + r]);
        trans[((int64_t)t * K + i) * K + j] = s;
      }
    }
  }
}

/* The path itself: Viterbi over the candidates with tau as transitions and the
 * raw logits as unary scores.  path: token ids [D]; scores: [D]. */
void orc_selector(int D, int K, int R, const int32_t *cand, const double *cand_logit,
                  const double *z, int32_t x0, const uint16_t *cb_a, const uint16_t *cb_b,
                  int32_t *path, double *scores) {
  double *trans = (double *)malloc(sizeof(double) * (size_t)D * K * K);
  int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)D);
  orc_selector_trans(D, K, R, cand, z, x0, cb_a, cb_b, trans);
  orc_viterbi(D, K, cand_logit, trans, idx, scores);
  for (int t = 0; t < D; ++t) path[t] = cand[t * K + idx[t]];
  free(trans);
  free(idx);
}

/* Greedy acceptance (FastFlowLM card, "How it is used"; drafted tokens are
 * compared with the target's most likely token, "FastFlowLM measurements").
 * target[b][i] is the target's argmax for block position i+1.  accepted[b] =
 * longest n <= D with draft[b][i] == target[b][i] for all i < n; emitted =
 * draft[0..n-1] then target[n], padded with -1 to the block length. */
void orc_accept(int B, int Bk, const int32_t *draft, const int32_t *target, int32_t *accepted,
                int32_t *emitted) {
  int D = Bk - 1;
  for (int b = 0; b < B; ++b) {
    int n = 0;
    while (n < D && draft[b * D + n] == target[b * Bk + n]) ++n;
    accepted[b] = n;
    for (int i = 0; i < Bk; ++i)
      emitted[b * Bk + i] = i < n ? draft[b * D + i] : (i == n ? target[b * Bk + n] : -1);
  }
}

/* The next round's draft inputs from an acceptance (FastFlowLM card, "How it is used": the
 * target keeps the longest agreeing prefix plus one token of its own, and drafting continues
 * from there).  The accepted tokens and the target's own token are the tokens whose target
 * features the next round fuses as context rows, so n_new_next[b] = accepted[b] + 1; the next
 * block starts from the target's token: block_tokens_next[b][0] = target[b][accepted[b]],
 * positions 1..Bk-1 hold the caller's mask id. */
void orc_accept_chain(int B, int Bk, int32_t mask_id, const int32_t *draft, const int32_t *target,
                      int32_t *accepted, int32_t *emitted, int32_t *n_new_next,
                      int32_t *block_tokens_next) {
  orc_accept(B, Bk, draft, target, accepted, emitted);
  for (int b = 0; b < B; ++b) {
    n_new_next[b] = accepted[b] + 1;
    block_tokens_next[b * Bk] = target[b * Bk + accepted[b]];
    for (int i = 1; i < Bk; ++i) block_tokens_next[b * Bk + i] = mask_id;
  }
}

/* Sampled decoding: exact rejection sampling of the drafted path (MLX sidecar card, "Contents":
 * lossless acceptance for sampled decoding; Mindket listing, "For newcomers and experts").  The
 * pages name the rule, not its arithmetic; the reading fixed here is the standard speculative-
 * sampling rule with the draft's own distribution q_i at block position i:
 *   accept drafted token d_i with probability min(1, p_i(d_i) / q_i(d_i)), in order, stopping at the
 *   first rejection; at a rejection at i emit a token drawn from max(0, p_i - q_i) (normalised); if
 *   every drafted token is accepted emit a token drawn from p_D (the target's distribution after the
 *   block).  The selector picks its path deterministically, so by default q_i is the point mass on
 *   d_i (q = NULL): accept with probability p_i(d_i), resample from p_i without d_i.
 * Decisions are exact, so every implementation takes the same ones:
 *   accept iff u_acc[i] * q_i(d_i) < p_i(d_i), the product of the two fp32 inputs formed exactly
 *     (in double: 24 + 24 significant bits); fp32 inputs below the normal range count as zero;
 *   the residual r(x) = max(0, p(x) - q(x)) in fp32, then r_int(x) = floor(r(x) * 2^32) (exact),
 *     T = sum of r_int (64-bit integer), threshold t = floor(u_s * T / 2^32) with the 32-bit uniform
 *     integer u_s, and the emitted token is the smallest x whose running sum of r_int exceeds t
 *     (T = 0, a residual that is empty in fp32, falls back to p itself).
 * p: fp32 [B][Bk][V], row i = the target's probabilities for block position i+1 (row D after the
 * drafted tokens); q: fp32 [B][D][V] or NULL; u_acc: fp32 [B][D] in [0,1); u_s: uint32 [B].
 * accepted [B], emitted [B][Bk] (the accepted tokens, the sampled token, then -1).  A drafted id
 * outside [0, V) has probability 0 under the target: it is rejected (no table is indexed by it). */
/* fp32 values below the normal range (|v| < 2^-126) count as zero, inputs and the residual alike:
 * the decisions then do not depend on how an implementation treats subnormal numbers. */
static float flush32(float v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  return (u & 0x7F800000u) == 0 ? 0.0f : v;
}

/* Residual mass of token x in fp32: p - q (q given), p without the drafted token (point-mass
 * draft), or p itself (dtok < 0: the bonus position, or the fallback of an empty residual). */
static float residual(const float *p, const float *q, int32_t dtok, int x) {
  if (dtok < 0) return flush32(p[x]);
  if (q) return flush32(flush32(p[x]) - flush32(q[x]));
  return x == dtok ? flush32(flush32(p[x]) - 1.0f) : flush32(p[x]);
}

static uint64_t fixed32(float r) { return r > 0.0f ? (uint64_t)floor((double)r * 4294967296.0) : 0; }

/* The smallest x whose running sum of floor(max(0, r) * 2^32) exceeds floor(us * T / 2^32). */
static int32_t sample_residual(const float *p, const float *q, int32_t dtok, int V, uint32_t us) {
  uint64_t T = 0;
  for (int x = 0; x < V; ++x) T += fixed32(residual(p, q, dtok, x));
  if (T == 0) {  /* empty residual: sample p itself */
    dtok = -1;
    for (int x = 0; x < V; ++x) T += fixed32(flush32(p[x]));
    if (T == 0) return 0;
  }
  const uint64_t t = (uint64_t)(((unsigned __int128)us * T) >> 32);
  uint64_t run = 0;
  for (int x = 0; x < V; ++x) {
    run += fixed32(residual(p, q, dtok, x));
    if (run > t) return x;
  }
  return V - 1;
}

void orc_accept_sampled(int B, int Bk, int V, const int32_t *draft, const float *p, const float *q,
                        const float *u_acc, const uint32_t *u_s, int32_t *accepted, int32_t *emitted) {
  const int D = Bk - 1;
  for (int b = 0; b < B; ++b) {
    int n = 0;
    while (n < D) {
      const int32_t d = draft[b * D + n];
      if (d < 0 || d >= V) break; /* a token outside the vocabulary has target probability 0 */
      const float *pr = p + ((int64_t)b * Bk + n) * V;
      const double qd = q ? (double)flush32(q[((int64_t)b * D + n) * V + d]) : 1.0;
      if ((double)flush32(u_acc[b * D + n]) * qd < (double)flush32(pr[d])) ++n;
      else break;
    }
    accepted[b] = n;
    const float *pr = p + ((int64_t)b * Bk + n) * V;
    const float *qr = q && n < D ? q + ((int64_t)b * D + n) * V : NULL;
    const int32_t tok = sample_residual(pr, qr, n < D ? draft[b * D + n] : -1, V, u_s[b]);
    for (int i = 0; i < Bk; ++i) emitted[b * Bk + i] = i < n ? draft[b * D + i] : (i == n ? tok : -1);
  }
}

/* LM head + top-K from given bf16 rows (the shared output head, FastFlowLM card).
 * hn: [rows][H] bf16; ids, vals: [rows][K]. */
void orc_lmhead_topk(int rows, int H, int V, int K, const uint16_t *hn, const uint16_t *lm_head,
                     int32_t *ids, double *vals) {
  double *x = (double *)malloc(sizeof(double) * (size_t)rows * H);
  double *lg = (double *)malloc(sizeof(double) * (size_t)rows * V);
  for (int64_t i = 0; i < (int64_t)rows * H; ++i) x[i] = orc_bf16(hn[i]);
  orc_matmul(1, lm_head, V, H, x, rows, lg);
  for (int r = 0; r < rows; ++r) orc_topk(lg + (int64_t)r * V, V, K, ids + r * K, vals + r * K);
  free(x);
  free(lg);
}

/* Logits of given token ids for given bf16 rows: out[r][i] = lm_head[ids[r][i]] . hn[r]. */
void orc_logits_at(int rows, int H, int K, const uint16_t *hn, const uint16_t *lm_head,
                   const int32_t *ids, double *out) {
  for (int r = 0; r < rows; ++r)
    for (int i = 0; i < K; ++i) {
      const uint16_t *w = lm_head + (int64_t)ids[r * K + i] * H;
      double s = 0.0;
      for (int k = 0; k < H; ++k) s += orc_bf16(w[k]) * orc_bf16(hn[(int64_t)r * H + k]);
      out[r * K + i] = s;
    }
}

/* ------------------------------------------------------------------ */
/* the block step, one request                                          */

static double *dalloc(int64_t n) { return (double *)calloc((size_t)(n > 0 ? n : 1), sizeof(double)); }

/* One request's block step.
 * taps: [Bk][n_taps*H] bf16 (rows < n_new valid), tap-major in increasing target
 *   layer (FastFlowLM card, "Taps" row), fused by fc then its RMSNorm into the
 *   context rows (reading: the context rows give each layer's cached K/V).
 * btok: [Bk] block tokens (position 0 = last emitted token; 1..Bk-1 = mask ids).
 * seq_len: cached tokens before the step; advanced by n_new.
 * kc/vc: per-layer paged caches [pages][n_kv][page][hd] bf16, updated in place.
 * path/scores: [Bk-1]. */
int orc_draft_request(const orc_dims *c, const orc_weights *w, const uint16_t *taps, int n_new,
                      const int32_t *btok, uint16_t *const *kc, uint16_t *const *vc,
                      const int32_t *page_table, int max_pages, int32_t *seq_len, int32_t *path,
                      float *scores, const orc_trace *tr) {
  const int H = c->hidden, F = c->ffn, T = c->n_taps, nq = c->n_q, nkv = c->n_kv, hd = c->head_dim;
  const int HQ = nq * hd, HKV = nkv * hd, Bk = c->block, D = Bk - 1, V = c->vocab, R = c->rank,
            K = c->topk, fmt = c->wfmt;
  const double eps = c->rms_eps;
  if (c->layers < 1 || c->layers > ORC_MAX_LAYERS || Bk < 2 || n_new < 0 || n_new > Bk ||
      H % 4 || nq % nkv || hd % 2 || K < 1)
    return ORC_ERR_ARG;
  for (int t = 0; t < Bk; ++t)
    if (btok[t] < 0 || btok[t] >= V) return ORC_ERR_TOKEN;
  const int64_t L0 = *seq_len, Lb = L0 + n_new;
  int err = ORC_OK;

  double *xt = dalloc((int64_t)Bk * T * H), *ctx = dalloc((int64_t)Bk * H), *pre = dalloc((int64_t)Bk * H);
  double *h = dalloc((int64_t)Bk * H), *x = dalloc((int64_t)Bk * H), *y = dalloc((int64_t)Bk * H);
  double *q = dalloc((int64_t)Bk * HQ), *kb = dalloc((int64_t)Bk * HKV), *vb = dalloc((int64_t)Bk * HKV);
  double *kx = dalloc((int64_t)Bk * HKV), *vx = dalloc((int64_t)Bk * HKV), *o = dalloc((int64_t)Bk * HQ);
  double *tmp = dalloc((int64_t)Bk * H), *gt = dalloc((int64_t)Bk * F), *ut = dalloc((int64_t)Bk * F);
  double *hn = dalloc((int64_t)D * H), *lg = dalloc(V), *z = dalloc((int64_t)D * R);
  double *cl = dalloc((int64_t)D * K), *sc = dalloc(D), *nrm = dalloc(H);
  int32_t *cand = (int32_t *)calloc((size_t)D * K, sizeof(int32_t));

  /* context rows: fc over the concatenated taps, then the fc RMSNorm */
  for (int64_t i = 0; i < (int64_t)n_new * T * H; ++i) xt[i] = orc_bf16(taps[i]);
  orc_matmul(fmt, w->fc, H, T * H, xt, n_new, pre);
  for (int i = 0; i < n_new; ++i) orc_rmsnorm(pre + (int64_t)i * H, H, w->fc_norm, eps, ctx + (int64_t)i * H);
  if (tr && tr->ctx) memcpy(tr->ctx, ctx, sizeof(double) * (size_t)n_new * H);

  /* block rows: the target's (shared) embedding table */
  for (int t = 0; t < Bk; ++t)
    for (int k = 0; k < H; ++k) h[(int64_t)t * H + k] = orc_bf16(w->embed[(int64_t)btok[t] * H + k]);
  if (tr && tr->hidden) memcpy(tr->hidden, h, sizeof(double) * (size_t)Bk * H);

  for (int l = 0; l < c->layers && err == ORC_OK; ++l) {
    const orc_layer *L = &w->layer[l];
    for (int t = 0; t < Bk; ++t) orc_rmsnorm(h + (int64_t)t * H, H, L->ln1, eps, x + (int64_t)t * H);
    orc_dynconv(Bk, H, x, L->dc_w, L->dc_s0, L->dc_s1, y);
    orc_matmul(fmt, L->wq, HQ, H, y, Bk, q);
    orc_matmul(fmt, L->wk, HKV, H, y, Bk, kb);
    orc_matmul(fmt, L->wv, HKV, H, y, Bk, vb);
    orc_matmul(fmt, L->wk, HKV, H, ctx, n_new, kx);
    orc_matmul(fmt, L->wv, HKV, H, ctx, n_new, vx);
    /* per-head q/k RMSNorm, then RoPE at absolute positions */
    for (int t = 0; t < Bk; ++t) {
      for (int hh = 0; hh < nq; ++hh) {
        double *v = q + ((int64_t)t * nq + hh) * hd;
        orc_rmsnorm(v, hd, L->qn, eps, nrm);
        memcpy(v, nrm, sizeof(double) * hd);
        orc_rope(v, hd, Lb + t, c->rope_theta);
      }
      for (int hh = 0; hh < nkv; ++hh) {
        double *v = kb + ((int64_t)t * nkv + hh) * hd;
        orc_rmsnorm(v, hd, L->kn, eps, nrm);
        memcpy(v, nrm, sizeof(double) * hd);
        orc_rope(v, hd, Lb + t, c->rope_theta);
      }
    }
    if (l == 0 && tr) {
      if (tr->q0) memcpy(tr->q0, q, sizeof(double) * (size_t)Bk * HQ);
      if (tr->k0) memcpy(tr->k0, kb, sizeof(double) * (size_t)Bk * HKV);
    }
    /* context rows: K/V of this layer appended to its cache at L0..Lb-1 */
    for (int i = 0; i < n_new && err == ORC_OK; ++i) {
      int64_t pos = L0 + i, lp = pos / c->page_size;
      if (lp >= max_pages || page_table[lp] < 0) { err = ORC_ERR_PAGE; break; }
      for (int hh = 0; hh < nkv; ++hh) {
        double *v = kx + ((int64_t)i * nkv + hh) * hd;
        orc_rmsnorm(v, hd, L->kn, eps, nrm);
        memcpy(v, nrm, sizeof(double) * hd);
        orc_rope(v, hd, pos, c->rope_theta);
        int64_t off = (((int64_t)page_table[lp] * nkv + hh) * c->page_size + pos % c->page_size) * hd;
        for (int d = 0; d < hd; ++d) {
          kc[l][off + d] = orc_to_bf16(v[d]);
          vc[l][off + d] = orc_to_bf16(vx[((int64_t)i * nkv + hh) * hd + d]);
        }
      }
    }
    if (err != ORC_OK) break;
    err = orc_attention(c, Bk, q, kb, vb, kc[l], vc[l], page_table, max_pages, Lb, o);
    if (err != ORC_OK) break;
    orc_matmul(fmt, L->wo, H, HQ, o, Bk, tmp);
    for (int64_t i = 0; i < (int64_t)Bk * H; ++i) h[i] += tmp[i];
    /* SwiGLU MLP on the second norm */
    for (int t = 0; t < Bk; ++t) orc_rmsnorm(h + (int64_t)t * H, H, L->ln2, eps, x + (int64_t)t * H);
    orc_matmul(fmt, L->wg, F, H, x, Bk, gt);
    orc_matmul(fmt, L->wu, F, H, x, Bk, ut);
    for (int64_t i = 0; i < (int64_t)Bk * F; ++i) gt[i] = silu(gt[i]) * ut[i];
    orc_matmul(fmt, L->wd, H, F, gt, Bk, tmp);
    for (int64_t i = 0; i < (int64_t)Bk * H; ++i) h[i] += tmp[i];
    if (tr && tr->hidden) memcpy(tr->hidden + (int64_t)(l + 1) * Bk * H, h, sizeof(double) * (size_t)Bk * H);
  }

  if (err == ORC_OK) {
    /* drafted rows 1..D: final norm, shared LM head, top-K, selector path */
    for (int t = 1; t < Bk; ++t)
      orc_rmsnorm(h + (int64_t)t * H, H, w->final_norm, eps, hn + (int64_t)(t - 1) * H);
    for (int t = 0; t < D; ++t) {
      orc_matmul(1, w->lm_head, V, H, hn + (int64_t)t * H, 1, lg);
      orc_topk(lg, V, K, cand + t * K, cl + t * K);
    }
    orc_matmul(1, w->sel_proj, R, H, hn, D, z);
    orc_selector(D, K, R, cand, cl, z, btok[0], w->cb_a, w->cb_b, path, sc);
    for (int t = 0; t < D; ++t) scores[t] = (float)sc[t];
    *seq_len = (int32_t)Lb;
    if (tr) {
      if (tr->final_h) memcpy(tr->final_h, hn, sizeof(double) * (size_t)D * H);
      if (tr->cand) memcpy(tr->cand, cand, sizeof(int32_t) * (size_t)D * K);
      if (tr->cand_logit) memcpy(tr->cand_logit, cl, sizeof(double) * (size_t)D * K);
      if (tr->z) memcpy(tr->z, z, sizeof(double) * (size_t)D * R);
    }
  }
  free(xt); free(ctx); free(pre); free(h); free(x); free(y); free(q); free(kb); free(vb);
  free(kx); free(vx); free(o); free(tmp); free(gt); free(ut); free(hn); free(lg); free(z);
  free(cl); free(sc); free(nrm); free(cand);
  return err;
}

int orc_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    {
#ifdef _OPENMP
      extern int omp_get_num_threads(void);
      n = omp_get_num_threads();
#endif
    }
  }
  return n;
}
