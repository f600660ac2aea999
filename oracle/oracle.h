/*
 * oracle.h -- plain, slow, single-threaded CPU reference of the Qwen2-style
 * decoder forward (prefill + greedy decode).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library under
 * qwen2_decode_step_b200/ includes, links or calls this code; only the tests,
 * the smoke check and the benchmark's CPU-baseline leg use it.  It shares no
 * code, header, table or constant generator with the CUDA path.
 *
 * Numerics, after the precision policy of the LLAISYS final report
 * (section 3.3, item 3: "low-precision storage, float compute, low-precision
 * write-back"): every op reads its operands exactly (a bf16 value widens
 * exactly), computes in IEEE double, and rounds its result once to the storage
 * type with round-to-nearest-even.  Logits are kept in fp32.
 *
 * Operator list: LLAISYS final report, section 3.2, "third layer: CUDA
 * operators" (add, argmax, embedding, linear, rms_norm, rope, self_attention,
 * swiglu, rearrange).  Model flow: same report, section 3.2, "fourth layer:
 * model inference integration" (weights, buffers and KV cache, bias-free
 * linears, KV write-back through rearrange).
 *
 * All functions return 0 on success and a negative code on a bad argument.
 * Pointers are host pointers; nothing here allocates on behalf of the caller
 * except the model object.
 */
#ifndef QWEN2_ORACLE_H
#define QWEN2_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

enum {
  ORACLE_OK = 0,
  ORACLE_EINVAL = -1,
  ORACLE_ERANGE = -2,   /* a token id or position out of range */
  ORACLE_ENOMEM = -3,
  ORACLE_ECHECK = -4    /* an internal invariant failed (softmax mass != 1) */
};

/* Storage-type conversion (round to nearest, ties to even). */
uint16_t oracle_bf16_from_double(double x);
double oracle_bf16_to_double(uint16_t h);
/* Round n doubles into the storage type (used by the tests). */
int oracle_round(void* out, const double* in, size_t n, int dtype);

/* ---- the operators ---- */
int oracle_add(void* c, const void* a, const void* b, size_t n, int dtype);
/* Per row: the lowest index of the maximum (a NaN counts as larger than any
 * number; the first NaN wins), and the value there (same dtype as x). */
int oracle_argmax(int64_t* idx, void* val, const void* x, size_t rows, size_t n, int dtype);
int oracle_embedding(void* out, const int64_t* ids, const void* table, size_t ntok,
                     size_t vocab, size_t d, int dtype);
/* Y[m,n] = sum_k X[m,k] W[n,k] (+ b[n]); W is [N,K]; b may be NULL.
 * X, W, b in dtype; Y in out_dtype. */
int oracle_linear(void* y, const void* x, const void* w, const void* b, size_t M, size_t N,
                  size_t K, int dtype, int out_dtype);
int oracle_rms_norm(void* y, const void* x, const void* w, size_t M, size_t d, double eps,
                    int dtype);
/* x [ntok, nhead, hd]; half-split pairs (j, j + hd/2) rotated by pos*theta^(-2j/hd). */
int oracle_rope(void* y, const void* x, const int64_t* pos, size_t ntok, size_t nhead,
                size_t hd, double theta, int dtype);
/* q [seqlen, nh, hd]; k, v [total_len, nkv, hd]; out [seqlen, nh, hd].
 * Query row i sits at absolute position total_len - seqlen + i and sees keys
 * j <= that position; q head h reads kv head h / (nh / nkv). */
int oracle_self_attention(void* out, const void* q, const void* k, const void* v,
                          size_t seqlen, size_t total_len, size_t nh, size_t nkv, size_t hd,
                          double scale, int dtype);
/* out = up * gate / (1 + exp(-gate)) */
int oracle_swiglu(void* out, const void* gate, const void* up, size_t n, int dtype);
/* out[sum idx_i*out_strides_i] = in[sum idx_i*in_strides_i]; strides in elements. */
int oracle_rearrange(void* out, const void* in, int ndim, const int64_t* shape,
                     const int64_t* out_strides, const int64_t* in_strides, size_t elem_size);

/* ---- the model ---- */
typedef struct oracle_meta {
  int dtype;
  int n_layers, hidden, n_heads, n_kv_heads, head_dim, intermediate, vocab;
  double eps, theta;
  int max_seq, max_batch;
} oracle_meta;

enum {
  ORACLE_W_EMBED = 0, ORACLE_W_LM_HEAD, ORACLE_W_FINAL_NORM,
  ORACLE_W_IN_NORM, ORACLE_W_Q, ORACLE_W_QB, ORACLE_W_K, ORACLE_W_KB, ORACLE_W_V, ORACLE_W_VB,
  ORACLE_W_O, ORACLE_W_POST_NORM, ORACLE_W_GATE, ORACLE_W_UP, ORACLE_W_DOWN,
  ORACLE_W_COUNT
};

typedef struct oracle_model oracle_model;

oracle_model* oracle_model_create(const oracle_meta* meta);
void oracle_model_destroy(oracle_model* m);
/* Borrows `data` (the caller keeps it alive); nbytes must equal the tensor's size. */
int oracle_model_set_weight(oracle_model* m, int kind, int layer, const void* data, size_t nbytes);
/* The cache of (layer, seq): K and V, each [max_seq, n_kv_heads, head_dim] in dtype. */
int oracle_model_kv(oracle_model* m, int layer, int seq, void** k, void** v);
int oracle_model_set_len(oracle_model* m, int seq, int len);
int oracle_model_get_len(const oracle_model* m, int seq);
/* Run T tokens of sequence `seq` (a prefill chunk, or T = 1 for a decode step)
 * at positions len .. len+T-1, append their K/V, advance len.  Writes the fp32
 * logits of the last token (logits_last, [vocab], may be NULL), of every token
 * (logits_all, [T, vocab], may be NULL), and the greedy next token. */
int oracle_model_forward(oracle_model* m, int seq, const int64_t* ids, int T,
                         float* logits_last, float* logits_all, int64_t* next);
/* Same decoder layers on a given hidden input x_in [T, hidden] (no embedding,
 * no final norm / lm_head); x_out [T, hidden] is the residual stream after the
 * last layer.  Used for the one-layer workload. */
int oracle_model_forward_hidden(oracle_model* m, int seq, const void* x_in, int T, void* x_out);

#ifdef __cplusplus
}
#endif
#endif
