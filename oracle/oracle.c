/*
 * oracle.c -- plain CPU reference of the Qwen2-style decoder forward.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h).  Each function writes out the
 * plain definition of its operator, with no blocking, fusion or reordering:
 * sums run in index order in IEEE double, and each operator rounds its result
 * once to the storage type.  Citations name the page and the section that the
 * definition follows; where the pages are silent the comment says which
 * reading is taken.
 */
#include "oracle.h"

/* The accumulator of the linear and of attention's probability-weighted sum
 * of V: double.  Building with -DORACLE_FP32_ACCUMULATION makes it float --
 * not an oracle, but a copy of it with the rounding behaviour of fp32
 * accumulation, used only to measure how far that alone moves the model's
 * logits (oracle/drift.py), from which the free-running tolerances are
 * derived. */
#ifdef ORACLE_FP32_ACCUMULATION
typedef float oracle_acc_t;
#else
typedef double oracle_acc_t;
#endif

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* storage types                                                             */
/* ------------------------------------------------------------------------ */

double oracle_bf16_to_double(uint16_t h) {
  uint32_t bits = (uint32_t)h << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Direct double -> bf16 rounding to nearest, ties to even (no intermediate
 * float rounding).  bf16 keeps 8 significant bits and float's exponent range:
 * for |x| in [2^(e-1), 2^e) the spacing is 2^(e-8), never finer than the
 * subnormal spacing 2^-133. */
uint16_t oracle_bf16_from_double(double x) {
  if (isnan(x)) return (uint16_t)(signbit(x) ? 0xFFC0u : 0x7FC0u);
  uint16_t sign = (uint16_t)(signbit(x) ? 0x8000u : 0u);
  double ax = fabs(x);
  if (ax == 0.0) return sign;
  if (isinf(ax)) return (uint16_t)(sign | 0x7F80u);
  int e;
  frexp(ax, &e);
  int q = e - 8;
  if (q < -133) q = -133;
  double r = rint(ldexp(ax, -q)); /* default rounding mode: nearest, ties to even */
  double v = ldexp(r, q);        /* at most 8 significant bits */
  float f = (float)v;            /* exact, or +inf when v >= 2^128 */
  uint32_t bits;
  memcpy(&bits, &f, sizeof bits);
  return (uint16_t)(sign | (uint16_t)(bits >> 16));
}

static size_t esize(int dt) { return dt == ORACLE_F32 ? 4u : 2u; }
static int dtype_ok(int dt) { return dt == ORACLE_F32 || dt == ORACLE_BF16; }

static double ld(const void* p, size_t i, int dt) {
  if (dt == ORACLE_F32) return (double)((const float*)p)[i];
  return oracle_bf16_to_double(((const uint16_t*)p)[i]);
}

static void st(void* p, size_t i, double v, int dt) {
  if (dt == ORACLE_F32)
    ((float*)p)[i] = (float)v;
  else
    ((uint16_t*)p)[i] = oracle_bf16_from_double(v);
}

int oracle_round(void* out, const double* in, size_t n, int dtype) {
  if (!dtype_ok(dtype)) return ORACLE_EINVAL;
  for (size_t i = 0; i < n; ++i) st(out, i, in[i], dtype);
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* operators (LLAISYS final report, section 3.2, third layer: CUDA operators) */
/* ------------------------------------------------------------------------ */

/* add: c = a + b, elementwise (the residual add). */
int oracle_add(void* c, const void* a, const void* b, size_t n, int dtype) {
  if (!dtype_ok(dtype)) return ORACLE_EINVAL;
  for (size_t i = 0; i < n; ++i) st(c, i, ld(a, i, dtype) + ld(b, i, dtype), dtype);
  return ORACLE_OK;
}

/* Does (v, i) beat the current best (bv, bi)?  The largest value wins; among
 * equal values the lowest index.  NaN is read as larger than every number
 * (first NaN wins), as numpy's argmax does.  The report only says each rank
 * takes a local argmax and the host picks the global best (section 4.3,
 * item 4); the tie rule is this build's reading. */
static int beats(double v, size_t i, double bv, size_t bi) {
  int vn = isnan(v), bn = isnan(bv);
  if (vn || bn) {
    if (vn && bn) return i < bi;
    return vn;
  }
  if (v > bv) return 1;
  if (v < bv) return 0;
  return i < bi;
}

int oracle_argmax(int64_t* idx, void* val, const void* x, size_t rows, size_t n, int dtype) {
  if (!dtype_ok(dtype) || (rows > 0 && n == 0)) return ORACLE_EINVAL;
  for (size_t r = 0; r < rows; ++r) {
    size_t bi = 0;
    double bv = ld(x, r * n, dtype);
    for (size_t i = 1; i < n; ++i) {
      double v = ld(x, r * n + i, dtype);
      if (beats(v, i, bv, bi)) {
        bv = v;
        bi = i;
      }
    }
    idx[r] = (int64_t)bi;
    if (val) st(val, r, bv, dtype);
  }
  return ORACLE_OK;
}

/* embedding: out[t] = table[ids[t]].  An id outside [0, vocab) gives a zero
 * row and the call reports ORACLE_ERANGE. */
int oracle_embedding(void* out, const int64_t* ids, const void* table, size_t ntok, size_t vocab,
                     size_t d, int dtype) {
  if (!dtype_ok(dtype)) return ORACLE_EINVAL;
  size_t es = esize(dtype);
  int rc = ORACLE_OK;
  for (size_t t = 0; t < ntok; ++t) {
    char* dst = (char*)out + t * d * es;
    if (ids[t] < 0 || (uint64_t)ids[t] >= vocab) {
      memset(dst, 0, d * es);
      rc = ORACLE_ERANGE;
      continue;
    }
    memcpy(dst, (const char*)table + (size_t)ids[t] * d * es, d * es);
  }
  return rc;
}

/* linear: Y = X W^T (+ b), W stored [out, in] as in the HF checkpoints; the
 * bias is optional (report section 3.2: the no-bias linear path and the
 * Python wrapper's "bias is None"). */
int oracle_linear(void* y, const void* x, const void* w, const void* b, size_t M, size_t N,
                  size_t K, int dtype, int out_dtype) {
  if (!dtype_ok(dtype) || !dtype_ok(out_dtype)) return ORACLE_EINVAL;
  double* xs = (double*)malloc((K ? K : 1) * sizeof(double));
  if (!xs) return ORACLE_ENOMEM;
  for (size_t m = 0; m < M; ++m) {
    for (size_t k = 0; k < K; ++k) xs[k] = ld(x, m * K + k, dtype);
    for (size_t n = 0; n < N; ++n) {
      oracle_acc_t acc = 0.0;
      if (dtype == ORACLE_BF16) {
        const uint16_t* wr = (const uint16_t*)w + n * K;
        for (size_t k = 0; k < K; ++k) acc += (oracle_acc_t)xs[k] * (oracle_acc_t)oracle_bf16_to_double(wr[k]);
      } else {
        const float* wr = (const float*)w + n * K;
        for (size_t k = 0; k < K; ++k) acc += (oracle_acc_t)xs[k] * (oracle_acc_t)wr[k];
      }
      if (b) acc += ld(b, n, dtype);
      st(y, m * N + n, acc, out_dtype);
    }
  }
  free(xs);
  return ORACLE_OK;
}

/* rms_norm: y = w * x / sqrt(mean(x^2) + eps), eps inside the square root,
 * one rounding at the output. */
int oracle_rms_norm(void* y, const void* x, const void* w, size_t M, size_t d, double eps,
                    int dtype) {
  if (!dtype_ok(dtype) || d == 0) return ORACLE_EINVAL;
  for (size_t m = 0; m < M; ++m) {
    double ss = 0.0;
    for (size_t i = 0; i < d; ++i) {
      double v = ld(x, m * d + i, dtype);
      ss += v * v;
    }
    double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (size_t i = 0; i < d; ++i)
      st(y, m * d + i, ld(x, m * d + i, dtype) * inv * ld(w, i, dtype), dtype);
  }
  return ORACLE_OK;
}

/* rope: rotary position embedding.  The pages name the operator but print no
 * formula; the reading taken is the one of the HF Qwen2 model that the report
 * matches token for token: pairs (j, j + hd/2), angle pos * theta^(-2j/hd). */
int oracle_rope(void* y, const void* x, const int64_t* pos, size_t ntok, size_t nhead, size_t hd,
                double theta, int dtype) {
  if (!dtype_ok(dtype) || hd == 0 || hd % 2 != 0) return ORACLE_EINVAL;
  size_t half = hd / 2;
  for (size_t t = 0; t < ntok; ++t) {
    if (pos[t] < 0) return ORACLE_ERANGE;
    for (size_t h = 0; h < nhead; ++h) {
      size_t base = (t * nhead + h) * hd;
      for (size_t j = 0; j < half; ++j) {
        double freq = pow(theta, -(2.0 * (double)j) / (double)hd);
        double phi = (double)pos[t] * freq;
        double c = cos(phi), s = sin(phi);
        double a = ld(x, base + j, dtype);
        double b = ld(x, base + j + half, dtype);
        st(y, base + j, a * c - b * s, dtype);
        st(y, base + j + half, b * c + a * s, dtype);
      }
    }
  }
  return ORACLE_OK;
}

/* self_attention, after the attention sketch of the Day-0 adaptation
 * tutorial (step 5): scores = q k^T * scale, causal mask, numerically stable
 * softmax (subtract the row maximum), probabilities times V.  The causal
 * offset for a KV cache: query row i sits at position total_len - seqlen + i.
 * GQA: q head h reads kv head floor(h / (nh / nkv)). */
int oracle_self_attention(void* out, const void* q, const void* k, const void* v, size_t seqlen,
                          size_t total_len, size_t nh, size_t nkv, size_t hd, double scale,
                          int dtype) {
  if (!dtype_ok(dtype) || nkv == 0 || nh % nkv != 0 || seqlen > total_len || hd == 0)
    return ORACLE_EINVAL;
  if (seqlen == 0) return ORACLE_OK;
  size_t group = nh / nkv;
  double* s = (double*)malloc(total_len * sizeof(double));
  double* p = (double*)malloc(total_len * sizeof(double));
  if (!s || !p) {
    free(s);
    free(p);
    return ORACLE_ENOMEM;
  }
  int rc = ORACLE_OK;
  for (size_t i = 0; i < seqlen; ++i) {
    size_t last = total_len - seqlen + i; /* keys 0..last are visible */
    for (size_t h = 0; h < nh; ++h) {
      size_t g = h / group;
      size_t qb = (i * nh + h) * hd;
      double mx = -INFINITY;
      for (size_t j = 0; j <= last; ++j) {
        size_t kb = (j * nkv + g) * hd;
        double dot = 0.0;
        for (size_t d = 0; d < hd; ++d) dot += ld(q, qb + d, dtype) * ld(k, kb + d, dtype);
        s[j] = dot * scale;
        if (s[j] > mx) mx = s[j];
      }
      double z = 0.0;
      for (size_t j = 0; j <= last; ++j) {
        p[j] = exp(s[j] - mx);
        z += p[j];
      }
      double mass = 0.0;
      for (size_t j = 0; j <= last; ++j) {
        p[j] /= z;
        mass += p[j];
      }
      if (!(fabs(mass - 1.0) <= 1e-12)) rc = ORACLE_ECHECK;
      for (size_t d = 0; d < hd; ++d) {
        oracle_acc_t acc = 0.0;
        for (size_t j = 0; j <= last; ++j) acc += (oracle_acc_t)p[j] * (oracle_acc_t)ld(v, (j * nkv + g) * hd + d, dtype);
        st(out, qb + d, acc, dtype);
      }
    }
  }
  free(s);
  free(p);
  return rc;
}

/* swiglu: out = up * silu(gate) = up * gate / (1 + e^-gate). */
int oracle_swiglu(void* out, const void* gate, const void* up, size_t n, int dtype) {
  if (!dtype_ok(dtype)) return ORACLE_EINVAL;
  for (size_t i = 0; i < n; ++i) {
    double g = ld(gate, i, dtype);
    st(out, i, ld(up, i, dtype) * (g / (1.0 + exp(-g))), dtype);
  }
  return ORACLE_OK;
}

/* rearrange: strided copy, out[idx . out_strides] = in[idx . in_strides]. */
int oracle_rearrange(void* out, const void* in, int ndim, const int64_t* shape,
                     const int64_t* out_strides, const int64_t* in_strides, size_t elem_size) {
  if (ndim < 0 || elem_size == 0) return ORACLE_EINVAL;
  int64_t idx[64];
  if (ndim > 64) return ORACLE_EINVAL;
  for (int d = 0; d < ndim; ++d) {
    if (shape[d] < 0) return ORACLE_EINVAL;
    if (shape[d] == 0) return ORACLE_OK;
    idx[d] = 0;
  }
  for (;;) {
    int64_t oo = 0, io = 0;
    for (int d = 0; d < ndim; ++d) {
      oo += idx[d] * out_strides[d];
      io += idx[d] * in_strides[d];
    }
    memcpy((char*)out + oo * (int64_t)elem_size, (const char*)in + io * (int64_t)elem_size,
           elem_size);
    int d = ndim - 1;
    while (d >= 0) {
      if (++idx[d] < shape[d]) break;
      idx[d] = 0;
      --d;
    }
    if (d < 0) break;
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* the model (report section 3.2, fourth layer: model inference integration) */
/* ------------------------------------------------------------------------ */

struct oracle_model {
  oracle_meta m;
  const void* glob[3];       /* embed, lm_head, final_norm */
  const void** layer_w;      /* [n_layers][ORACLE_W_COUNT] */
  void* kc;                  /* [n_layers][max_batch][max_seq][nkv][hd] */
  void* vc;
  int* len;                  /* [max_batch] */
};

static size_t weight_numel(const oracle_meta* m, int kind) {
  size_t H = (size_t)m->hidden, I = (size_t)m->intermediate, V = (size_t)m->vocab;
  size_t qd = (size_t)m->n_heads * m->head_dim, kd = (size_t)m->n_kv_heads * m->head_dim;
  switch (kind) {
    case ORACLE_W_EMBED:
    case ORACLE_W_LM_HEAD: return V * H;
    case ORACLE_W_FINAL_NORM:
    case ORACLE_W_IN_NORM:
    case ORACLE_W_POST_NORM: return H;
    case ORACLE_W_Q: return qd * H;
    case ORACLE_W_QB: return qd;
    case ORACLE_W_K:
    case ORACLE_W_V: return kd * H;
    case ORACLE_W_KB:
    case ORACLE_W_VB: return kd;
    case ORACLE_W_O: return H * qd;
    case ORACLE_W_GATE:
    case ORACLE_W_UP: return I * H;
    case ORACLE_W_DOWN: return H * I;
    default: return 0;
  }
}

oracle_model* oracle_model_create(const oracle_meta* meta) {
  const oracle_meta* m = meta;
  if (!m || !dtype_ok(m->dtype) || m->n_layers < 0 || m->hidden <= 0 || m->n_heads <= 0 ||
      m->n_kv_heads <= 0 || m->n_heads % m->n_kv_heads != 0 || m->head_dim <= 0 ||
      m->head_dim % 2 != 0 || m->intermediate <= 0 || m->vocab <= 0 || m->max_seq <= 0 ||
      m->max_batch <= 0)
    return NULL;
  oracle_model* om = (oracle_model*)calloc(1, sizeof *om);
  if (!om) return NULL;
  om->m = *m;
  size_t L = (size_t)(m->n_layers ? m->n_layers : 1);
  size_t kvn = (size_t)m->n_layers * m->max_batch * m->max_seq * m->n_kv_heads * m->head_dim;
  om->layer_w = (const void**)calloc(L * ORACLE_W_COUNT, sizeof(void*));
  om->kc = calloc(kvn ? kvn : 1, esize(m->dtype));
  om->vc = calloc(kvn ? kvn : 1, esize(m->dtype));
  om->len = (int*)calloc((size_t)m->max_batch, sizeof(int));
  if (!om->layer_w || !om->kc || !om->vc || !om->len) {
    oracle_model_destroy(om);
    return NULL;
  }
  return om;
}

void oracle_model_destroy(oracle_model* om) {
  if (!om) return;
  free(om->layer_w);
  free(om->kc);
  free(om->vc);
  free(om->len);
  free(om);
}

int oracle_model_set_weight(oracle_model* om, int kind, int layer, const void* data,
                            size_t nbytes) {
  if (!om || kind < 0 || kind >= ORACLE_W_COUNT || !data) return ORACLE_EINVAL;
  if (nbytes != weight_numel(&om->m, kind) * esize(om->m.dtype)) return ORACLE_EINVAL;
  if (kind <= ORACLE_W_FINAL_NORM) {
    om->glob[kind] = data;
  } else {
    if (layer < 0 || layer >= om->m.n_layers) return ORACLE_EINVAL;
    om->layer_w[(size_t)layer * ORACLE_W_COUNT + kind] = data;
  }
  return ORACLE_OK;
}

static size_t kv_offset(const oracle_model* om, int layer, int seq) {
  const oracle_meta* m = &om->m;
  return (((size_t)layer * m->max_batch + seq) * m->max_seq) * m->n_kv_heads * m->head_dim;
}

int oracle_model_kv(oracle_model* om, int layer, int seq, void** k, void** v) {
  if (!om || layer < 0 || layer >= om->m.n_layers || seq < 0 || seq >= om->m.max_batch)
    return ORACLE_EINVAL;
  size_t off = kv_offset(om, layer, seq) * esize(om->m.dtype);
  *k = (char*)om->kc + off;
  *v = (char*)om->vc + off;
  return ORACLE_OK;
}

int oracle_model_set_len(oracle_model* om, int seq, int len) {
  if (!om || seq < 0 || seq >= om->m.max_batch || len < 0 || len > om->m.max_seq)
    return ORACLE_EINVAL;
  om->len[seq] = len;
  return ORACLE_OK;
}

int oracle_model_get_len(const oracle_model* om, int seq) {
  if (!om || seq < 0 || seq >= om->m.max_batch) return ORACLE_EINVAL;
  return om->len[seq];
}

static int weights_ready(const oracle_model* om, int need_ends) {
  if (need_ends)
    for (int i = 0; i < 3; ++i)
      if (!om->glob[i]) return 0;
  for (int l = 0; l < om->m.n_layers; ++l)
    for (int k = ORACLE_W_IN_NORM; k < ORACLE_W_COUNT; ++k)
      if (!om->layer_w[(size_t)l * ORACLE_W_COUNT + k]) return 0;
  return 1;
}

/* One decoder layer on x [T, H] (in place) for tokens at positions
 * pos0 .. pos0+T-1 of sequence seq.  Order of the Qwen2 layer: RMSNorm,
 * q/k/v linears with bias, RoPE on q and k, KV write-back into the cache,
 * causal GQA attention over the cache, o linear, residual add, RMSNorm,
 * gate/up linears, SwiGLU, down linear, residual add. */
static int decoder_layer(oracle_model* om, int l, int seq, void* x, int T, int pos0) {
  const oracle_meta* m = &om->m;
  int dt = m->dtype;
  size_t es = esize(dt);
  size_t H = (size_t)m->hidden, I = (size_t)m->intermediate;
  size_t nh = (size_t)m->n_heads, nkv = (size_t)m->n_kv_heads, hd = (size_t)m->head_dim;
  size_t qd = nh * hd, kd = nkv * hd;
  const void** w = om->layer_w + (size_t)l * ORACLE_W_COUNT;
  size_t t = (size_t)T;
  int rc = ORACLE_OK;

  char* h = (char*)malloc(t * H * es);
  char* q = (char*)malloc(t * qd * es);
  char* k = (char*)malloc(t * kd * es);
  char* v = (char*)malloc(t * kd * es);
  char* a = (char*)malloc(t * qd * es);
  char* o = (char*)malloc(t * H * es);
  char* g = (char*)malloc(t * I * es);
  char* u = (char*)malloc(t * I * es);
  int64_t* pos = (int64_t*)malloc(t * sizeof(int64_t));
  if (!h || !q || !k || !v || !a || !o || !g || !u || !pos) {
    rc = ORACLE_ENOMEM;
    goto done;
  }
  for (size_t i = 0; i < t; ++i) pos[i] = (int64_t)pos0 + (int64_t)i;

  oracle_rms_norm(h, x, w[ORACLE_W_IN_NORM], t, H, m->eps, dt);
  oracle_linear(q, h, w[ORACLE_W_Q], w[ORACLE_W_QB], t, qd, H, dt, dt);
  oracle_linear(k, h, w[ORACLE_W_K], w[ORACLE_W_KB], t, kd, H, dt, dt);
  oracle_linear(v, h, w[ORACLE_W_V], w[ORACLE_W_VB], t, kd, H, dt, dt);
  oracle_rope(q, q, pos, t, nh, hd, m->theta, dt);
  oracle_rope(k, k, pos, t, nkv, hd, m->theta, dt);

  /* KV write-back through rearrange: rows pos0.. of the [max_seq, nkv, hd] cache. */
  {
    void *kc, *vc;
    oracle_model_kv(om, l, seq, &kc, &vc);
    int64_t shape[3] = {(int64_t)t, (int64_t)nkv, (int64_t)hd};
    int64_t strides[3] = {(int64_t)kd, (int64_t)hd, 1};
    oracle_rearrange((char*)kc + (size_t)pos0 * kd * es, k, 3, shape, strides, strides, es);
    oracle_rearrange((char*)vc + (size_t)pos0 * kd * es, v, 3, shape, strides, strides, es);
    int arc = oracle_self_attention(a, q, kc, vc, t, (size_t)pos0 + t, nh, nkv, hd,
                                    1.0 / sqrt((double)hd), dt);
    if (arc != ORACLE_OK) {
      rc = arc;
      goto done;
    }
  }

  oracle_linear(o, a, w[ORACLE_W_O], NULL, t, H, qd, dt, dt);
  oracle_add(x, x, o, t * H, dt);
  oracle_rms_norm(h, x, w[ORACLE_W_POST_NORM], t, H, m->eps, dt);
  oracle_linear(g, h, w[ORACLE_W_GATE], NULL, t, I, H, dt, dt);
  oracle_linear(u, h, w[ORACLE_W_UP], NULL, t, I, H, dt, dt);
  oracle_swiglu(g, g, u, t * I, dt);
  oracle_linear(o, g, w[ORACLE_W_DOWN], NULL, t, H, I, dt, dt);
  oracle_add(x, x, o, t * H, dt);

done:
  free(h);
  free(q);
  free(k);
  free(v);
  free(a);
  free(o);
  free(g);
  free(u);
  free(pos);
  return rc;
}

static int run_layers(oracle_model* om, int seq, void* x, int T) {
  int pos0 = om->len[seq];
  for (int l = 0; l < om->m.n_layers; ++l) {
    int rc = decoder_layer(om, l, seq, x, T, pos0);
    if (rc != ORACLE_OK) return rc;
  }
  om->len[seq] = pos0 + T;
  return ORACLE_OK;
}

int oracle_model_forward(oracle_model* om, int seq, const int64_t* ids, int T, float* logits_last,
                         float* logits_all, int64_t* next) {
  if (!om || seq < 0 || seq >= om->m.max_batch || T <= 0 || !ids) return ORACLE_EINVAL;
  if (!weights_ready(om, 1)) return ORACLE_EINVAL;
  if (om->len[seq] + T > om->m.max_seq) return ORACLE_ERANGE;
  const oracle_meta* m = &om->m;
  int dt = m->dtype;
  size_t es = esize(dt), H = (size_t)m->hidden, V = (size_t)m->vocab, t = (size_t)T;
  char* x = (char*)malloc(t * H * es);
  char* h = (char*)malloc(t * H * es);
  float* lg = (float*)malloc(V * sizeof(float));
  int rc = ORACLE_OK;
  if (!x || !h || !lg) {
    rc = ORACLE_ENOMEM;
    goto done;
  }
  rc = oracle_embedding(x, ids, om->glob[ORACLE_W_EMBED], t, V, H, dt);
  if (rc != ORACLE_OK) goto done;
  rc = run_layers(om, seq, x, T);
  if (rc != ORACLE_OK) goto done;
  /* final RMSNorm, untied lm_head (fp32 logits), greedy argmax */
  oracle_rms_norm(h, x, om->glob[ORACLE_W_FINAL_NORM], t, H, m->eps, dt);
  if (logits_all)
    oracle_linear(logits_all, h, om->glob[ORACLE_W_LM_HEAD], NULL, t, V, H, dt, ORACLE_F32);
  oracle_linear(lg, h + (t - 1) * H * es, om->glob[ORACLE_W_LM_HEAD], NULL, 1, V, H, dt,
                ORACLE_F32);
  if (logits_last) memcpy(logits_last, lg, V * sizeof(float));
  if (next) oracle_argmax(next, NULL, lg, 1, V, ORACLE_F32);
done:
  free(x);
  free(h);
  free(lg);
  return rc;
}

int oracle_model_forward_hidden(oracle_model* om, int seq, const void* x_in, int T, void* x_out) {
  if (!om || seq < 0 || seq >= om->m.max_batch || T <= 0 || !x_in || !x_out)
    return ORACLE_EINVAL;
  if (!weights_ready(om, 0)) return ORACLE_EINVAL;
  if (om->len[seq] + T > om->m.max_seq) return ORACLE_ERANGE;
  size_t bytes = (size_t)T * om->m.hidden * esize(om->m.dtype);
  memmove(x_out, x_in, bytes);
  return run_layers(om, seq, x_out, T);
}
