/*
 * q2.h -- C ABI of the B200 (sm_100a) Qwen2-style decoder library.
 *
 * The library runs the forward pass of a Qwen2-style decoder as a prefill
 * followed by greedy decode steps, on one GPU, in hand-written CUDA kernels.
 * It follows the operator and model contract of the LLAISYS training-camp
 * final report (section 3.2: "third layer: CUDA operators" names add, argmax,
 * embedding, linear, rms_norm, rope, self_attention, swiglu and rearrange;
 * "fourth layer: model inference integration" puts weights, intermediate
 * buffers and the KV cache on the GPU, fixes the bias-free linear path, takes
 * a missing bias as "None", and writes the KV cache back with rearrange).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every function returns a q2_status.  Nothing aborts and no C++ exception
 *   crosses this boundary.  On failure q2_last_error() describes the cause
 *   (a thread-local string, valid until the next call on the same thread).
 * - Tensor arguments are DEVICE pointers owned by the caller unless a
 *   function says otherwise (the *_host variants take host pointers).  They
 *   are dense, row-major and contiguous unless strides are passed.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *   stream).  Calls are asynchronous on that stream unless they say they
 *   synchronise.  The stream must belong to the current device (for model
 *   calls: the model's device).
 * - `dtype` is the storage type of the floating-point tensors of the call:
 *   Q2_F32 (float) or Q2_BF16 (bfloat16).  Arithmetic is fp32 throughout
 *   ("low-precision storage, float compute, low-precision write-back",
 *   report section 3.3, item 3); each operator rounds its output once, to
 *   nearest even.
 * - Sizes are element counts unless named *_bytes.
 * - Argument checks that need no device access happen before any launch and
 *   leave outputs untouched.  Errors that only the GPU can see (a token id
 *   outside the vocabulary; a bounded wait inside a kernel that ran out) are
 *   recorded in a device-side flag and reported by q2_check_device_error() /
 *   q2_model_check_error().
 */
#ifndef Q2_H
#define Q2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum q2_status {
  Q2_OK = 0,
  Q2_ERR_INVALID_ARG = 1, /* a NULL pointer, a zero/negative size, a bad enum value */
  Q2_ERR_DTYPE = 2,       /* unsupported dtype for this call */
  Q2_ERR_SHAPE = 3,       /* sizes inconsistent with each other or with the model */
  Q2_ERR_CAPACITY = 4,    /* a sequence would pass max_seq, or a batch passes max_batch */
  Q2_ERR_INDEX = 5,       /* a kernel saw a token id outside [0, vocab) */
  Q2_ERR_CUDA = 6,        /* a CUDA runtime call failed (message in q2_last_error) */
  Q2_ERR_OOM = 7,         /* device allocation failed */
  Q2_ERR_STATE = 8,       /* call not valid in the object's current state */
  Q2_ERR_TIMEOUT = 9      /* a bounded device-side wait ran out: a pipeline or grid-phase
                             dependency never arrived; results since the last check are
                             undefined (reported by the check functions) */
} q2_status;

typedef enum q2_dtype { Q2_F32 = 0, Q2_BF16 = 1 } q2_dtype;

/* Thread-local description of the last failure on this thread ("" if none). */
const char* q2_last_error(void);
/* Library version string, e.g. "q2 0.1 sm_100a". */
const char* q2_version(void);

/* Synchronises `stream`, then reports what the per-operator kernels on the
 * current device recorded since the last check, and clears the record:
 * Q2_ERR_TIMEOUT if a bounded wait inside a kernel ran out (the tcgen05 GEMM
 * behind q2_linear), else Q2_ERR_INDEX if a kernel saw a token id outside
 * the vocabulary, else Q2_OK. */
q2_status q2_check_device_error(void* stream);

/* Test hook: ORs `bits` (1: out-of-range id, 2: wait ran out) into the
 * operators' device error word of the current device, as a kernel would.
 * Synchronises. */
q2_status q2_test_raise_device_error(int bits, void* stream);

/* Test hook: the host-side work plans of the tensor-core kernels for a
 * machine of `sms` SMs (no device is touched).
 * q2_test_attn_plan: the tcgen05 prefill attention of `rows` query rows at
 * positions pos0.. with nh query heads (128-row items of one head, each
 * head's longest first): out[0] items run whole, out[1] key ranges ts per
 * later item, out[2] CTAs launched, out[3] items, out[4] range slots the
 * scratch holds, out[5] item counters it holds.  Q2_ERR_INVALID_ARG for
 * NULL out, rows, nh or sms of 0, or sizes past 2^30.
 * q2_test_gemm_tile: the token tile width (64, 128, 192 or 256) the tcgen05
 * GEMM takes for M tokens x N features, in *bn. */
q2_status q2_test_attn_plan(size_t rows, size_t pos0, size_t nh, int sms, int* out);
q2_status q2_test_gemm_tile(size_t M, size_t N, int sms, int* bn);

/* ======================================================================== */
/* Operators (report section 3.2, third layer).  Device pointers, caller-   */
/* owned; asynchronous on `stream`.                                          */
/* ======================================================================== */

/* add: c[i] = a[i] + b[i], i < n (the residual add).  c may alias a or b. */
q2_status q2_add(void* c, const void* a, const void* b, size_t n, int dtype, void* stream);

/* argmax over each row of vals [rows, n]: max_idx[r] (int64) = the lowest
 * index of the row maximum (a NaN counts as larger than any number; the
 * first NaN wins); max_val[r] = that value in `dtype` (max_val may be NULL).
 * Two passes: per-block partial maxima, then a per-row reduction of the
 * partials.  The partials live in stream-ordered scratch memory that the
 * call allocates and frees on `stream`. */
q2_status q2_argmax(int64_t* max_idx, void* max_val, const void* vals, size_t rows, size_t n,
                    int dtype, void* stream);

/* q2_argmax without any device allocation (the pages have no counterpart:
 * an addition of this library).  Same arguments and results as q2_argmax,
 * for callers that must not have a library allocate device memory at the
 * moment they call it -- a host that hands all device memory to its own pool
 * and passes only its inputs and outputs, a latency-critical loop that must
 * not wait on the allocator, or code recording into a CUDA graph under a
 * capture mode that refuses allocation calls.  The pass-1 partials live in
 * a fixed 192 KiB array in the library's device memory (every GPU that
 * loads the library holds one until the process exits); the call makes no
 * cudaMalloc/cudaFree or other allocating call.
 * Limits: rows <= 16384 (rows x partials <= 16384 entries); larger inputs
 * return Q2_ERR_CAPACITY before any launch.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture.
 * Sharing: all calls on a device use the same array and it keeps the last
 * call's partials.  Nothing in it needs to start at zero (pass 1 writes every
 * partial that pass 2 reads), but calls whose kernels overlap on the GPU
 * (different streams, no ordering between them) race on it: order them. */
q2_status q2_argmax_noalloc(int64_t* max_idx, void* max_val, const void* vals, size_t rows,
                            size_t n, int dtype, void* stream);

/* embedding: out[t, :] = weight[ids[t], :] for t < ntok; weight [vocab, d],
 * out [ntok, d].  An id outside [0, vocab) writes a zero row and sets the
 * device error flag (see q2_check_device_error). */
q2_status q2_embedding(void* out, const int64_t* ids, const void* weight, size_t ntok,
                       size_t vocab, size_t d, int dtype, void* stream);

/* linear: out[m, n] = sum_k in[m, k] * weight[n, k] + bias[n]; in [M, K],
 * weight [N, K] (the [out_features, in_features] layout of the checkpoints),
 * bias [N] or NULL (no bias), out [M, N].  fp32 accumulation; bf16 inputs
 * with M large enough run on the tcgen05 tensor cores. */
q2_status q2_linear(void* out, const void* in, const void* weight, const void* bias, size_t M,
                    size_t N, size_t K, int dtype, void* stream);

/* Test hook for the tcgen05 GEMM (bf16 operands): y = x[M, K] . w[N, K]^T
 * (+ bias[N]) with an epilogue: 0 plain (out [M, ldo], out_dtype bf16 or
 * fp32), 1 SwiGLU over interleaved gate/up rows (out[m, j] = silu(bf16(y[m,
 * 2j])) * bf16(y[m, 2j+1]), bf16), 2 residual add in place (out[m, n] =
 * bf16(out[m, n] + bf16(y[m, n])), bf16).  Requires M >= 1, K % 8 == 0 and
 * 16-byte aligned x and w.  allow_split != 0 lets a product with fewer tiles
 * than SMs split K (through a temporary fp32 workspace the call allocates and
 * frees).  Synchronises; returns Q2_ERR_CUDA if a pipeline wait in the kernel
 * ran out. */
q2_status q2_test_tc_gemm(void* out, size_t ldo, int out_dtype, int epilogue, const void* x,
                          const void* w, const void* bias, size_t M, size_t N, size_t K,
                          int allow_split, void* stream);

/* rms_norm: out[m, :] = weight * in[m, :] / sqrt(mean(in[m, :]^2) + eps);
 * in, out [M, d]; weight [d].  out may alias in. */
q2_status q2_rms_norm(void* out, const void* in, const void* weight, size_t M, size_t d,
                      float eps, int dtype, void* stream);

/* Fused residual add + RMSNorm: residual[m, :] += y[m, :] (rounded to dtype;
 * skipped when y is NULL), then h[m, :] = rms_norm(residual[m, :]).  */
q2_status q2_add_rms_norm(void* residual, const void* y, void* h, const void* weight, size_t M,
                          size_t d, float eps, int dtype, void* stream);

/* rope: rotary position embedding of in [ntok, nhead, hd] at positions
 * pos[t] (int64, >= 0).  For j < hd/2 the pair (x[j], x[j + hd/2]) is
 * rotated by the angle pos * theta^(-2j/hd) (the half-split pairing of the
 * HF Qwen2 model the report matched token for token).  Angles and their
 * cosines/sines are computed in double, the rotation in fp32.  hd even;
 * out may alias in. */
q2_status q2_rope(void* out, const void* in, const int64_t* pos, size_t ntok, size_t nhead,
                  size_t hd, float theta, int dtype, void* stream);

/* self_attention: causal GQA attention of q [seqlen, nh, hd] against
 * k, v [total_len, nkv, hd] (seqlen <= total_len; the last seqlen positions
 * are the queries' own).  Query row i sees keys j <= total_len - seqlen + i;
 * q head h reads kv head h / (nh / nkv).  out [seqlen, nh, hd] =
 * softmax(q k^T * scale) v, scores and softmax in fp32 (online, split over
 * the keys; the split partials live in stream-ordered scratch memory that
 * the call allocates and frees on `stream`).  hd in {32, 64, 128};
 * nh / nkv <= 8. */
q2_status q2_self_attention(void* out, const void* q, const void* k, const void* v, size_t seqlen,
                            size_t total_len, size_t nh, size_t nkv, size_t hd, float scale,
                            int dtype, void* stream);

/* swiglu: out[i] = up[i] * gate[i] / (1 + exp(-gate[i])), i < n. */
q2_status q2_swiglu(void* out, const void* gate, const void* up, size_t n, int dtype,
                    void* stream);

/* rearrange: strided copy.  For every index tuple idx < shape (ndim <= 8):
 * out[sum idx[d]*out_strides[d]] = in[sum idx[d]*in_strides[d]], strides in
 * elements of elem_size bytes (1, 2, 4, 8 or 16).  shape, out_strides and
 * in_strides are HOST arrays.  Dense same-order layouts take a plain
 * device-to-device copy.  Overlapping in/out is not supported. */
q2_status q2_rearrange(void* out, const void* in, int ndim, const int64_t* shape,
                       const int64_t* out_strides, const int64_t* in_strides, size_t elem_size,
                       void* stream);

/* ======================================================================== */
/* Model (report section 3.2, fourth layer; section 3.3, item 4: no per-     */
/* token allocation or handle creation -- everything is created once).       */
/* ======================================================================== */

typedef struct q2_meta {
  int dtype;              /* Q2_F32 or Q2_BF16: weights, activations, KV cache */
  int n_layers;           /* L */
  int hidden;             /* H */
  int n_heads;            /* nh (query heads) */
  int n_kv_heads;         /* nkv; nh % nkv == 0, nh / nkv <= 8 */
  int head_dim;           /* hd in {32, 64, 128} */
  int intermediate;       /* I (MLP) */
  int vocab;              /* V */
  float eps;              /* RMSNorm epsilon */
  float theta;            /* RoPE base */
  int max_seq;            /* KV capacity per sequence (positions) */
  int max_batch;          /* sequences (decode batch) */
  int max_prefill_tokens; /* prefill chunk size; 0 = default 4096 */
} q2_meta;

typedef struct q2_model q2_model;

typedef enum q2_wkind {
  Q2_W_EMBED = 0,      /* [V, H] */
  Q2_W_LM_HEAD = 1,    /* [V, H] (untied) */
  Q2_W_FINAL_NORM = 2, /* [H] */
  Q2_W_IN_NORM = 3,    /* [H], per layer */
  Q2_W_Q = 4,          /* [nh*hd, H] */
  Q2_W_Q_BIAS = 5,     /* [nh*hd] */
  Q2_W_K = 6,          /* [nkv*hd, H] */
  Q2_W_K_BIAS = 7,     /* [nkv*hd] */
  Q2_W_V = 8,          /* [nkv*hd, H] */
  Q2_W_V_BIAS = 9,     /* [nkv*hd] */
  Q2_W_O = 10,         /* [H, nh*hd] (no bias) */
  Q2_W_POST_NORM = 11, /* [H] */
  Q2_W_GATE = 12,      /* [I, H] (no bias) */
  Q2_W_UP = 13,        /* [I, H] (no bias) */
  Q2_W_DOWN = 14       /* [H, I] (no bias) */
} q2_wkind;

/* Creates a model on `device` (which becomes current): allocates the
 * weights, the KV cache [L][max_batch][nkv][max_seq][hd] for K and for V,
 * and every activation buffer once.  Sequence lengths start at 0. */
q2_status q2_model_create(const q2_meta* meta, int device, q2_model** out);

/* Frees everything the model owns (including captured CUDA graphs).
 * Call with no work of the model in flight. */
q2_status q2_model_destroy(q2_model* model);

/* Copies one weight tensor (device pointer, dtype of the model, layout as
 * listed in q2_wkind) into library-owned storage, possibly repacked (q/k/v
 * fused, gate/up interleaved).  `layer` is ignored for the three global
 * kinds.  The caller may free `src` once the copy has completed on
 * `stream`.  Q2_ERR_SHAPE if nbytes does not match the tensor's size. */
q2_status q2_model_load_weight(q2_model* model, int kind, int layer, const void* src,
                               size_t nbytes, void* stream);

/* Prefill: for b < batch, appends lens_host[b] tokens (a HOST array) to
 * sequence b at its current length; ids [sum lens] (device, int64) holds
 * the sequences' tokens one after another.  Long prompts run in chunks of
 * max_prefill_tokens.  next [batch] (device, int64) receives the greedy next
 * token after each sequence's last token; logits [batch, V] (device, fp32,
 * may be NULL) their logits.  A sequence with lens_host[b] == 0 is skipped
 * (its next/logits rows are left untouched).  Q2_ERR_CAPACITY if a sequence
 * would pass max_seq. */
q2_status q2_model_prefill(q2_model* model, const int64_t* ids, int batch, const int32_t* lens_host,
                           int64_t* next, float* logits, void* stream);

/* One greedy decode step for sequences 0..batch-1: token ids[b] (device,
 * int64) is appended at sequence b's current position; next [batch]
 * (device, int64) = argmax of the fp32 logits; logits [batch, V] (device,
 * fp32) may be NULL.  Runs as one captured CUDA graph per (batch, logits?)
 * pair; the first call with a new pair captures it.  Q2_ERR_CAPACITY if any
 * of the sequences is full. */
q2_status q2_model_decode_step(q2_model* model, const int64_t* ids, int batch, int64_t* next,
                               float* logits, void* stream);

/* q2_model_decode_step with HOST ids and next: copies ids in, runs the
 * step, copies next out and synchronises `stream` before returning.  For
 * best speed ids/next should be pinned host memory. */
q2_status q2_model_decode_step_host(q2_model* model, const int64_t* ids_host, int batch,
                                    int64_t* next_host, void* stream);

/* One decode step of the decoder layers alone on hidden inputs: x_in [batch,
 * H] (device, dtype) is the input of layer 0 for sequences 0..batch-1;
 * x_out [batch, H] receives the residual stream after the last layer (no
 * final norm, no lm_head).  Appends K/V and advances lengths like a decode
 * step. */
q2_status q2_model_forward_hidden(q2_model* model, const void* x_in, int batch, void* x_out,
                                  void* stream);

/* The decoder layers alone over T positions of sequence `seq` (a prefill
 * on hidden states): x_in [T, H] (device, dtype) is the input of layer 0 at
 * positions len .. len+T-1; x_out [T, H] receives the residual stream after
 * the last layer.  Appends K/V and advances the length like q2_model_prefill
 * (chunked by max_prefill_tokens).  With forward_hidden and q2_model_head it
 * lets a caller feed every layer a given input (layer-wise teacher forcing,
 * the per-layer bisection of the Day-0 adaptation tutorial, step 6). */
q2_status q2_model_prefill_hidden(q2_model* model, int seq, const void* x_in, int T, void* x_out,
                                  void* stream);

/* The model's head on given hidden states: x [rows, H] (device, dtype,
 * rows <= max_batch) -> final RMSNorm -> lm_head -> fp32 logits [rows, V]
 * (device, may be NULL) and greedy next [rows] (device, int64).  No KV or
 * length change. */
q2_status q2_model_head(q2_model* model, const void* x, int rows, int64_t* next, float* logits,
                        void* stream);

/* Resets sequence `seq` (or every sequence when seq == -1) to length 0. */
q2_status q2_model_reset_kv(q2_model* model, int seq);

/* Sets the current length of sequence `seq` (0 <= len <= max_seq), e.g.
 * after filling its cache directly through q2_model_kv_cache. */
q2_status q2_model_set_seq_len(q2_model* model, int seq, int len);
q2_status q2_model_get_seq_len(const q2_model* model, int seq, int* len);

/* Device pointers to the KV cache of (layer, seq): k and v each point at an
 * [nkv][max_seq][hd] block in the model's dtype (position p of kv head g is
 * at element (g * max_seq + p) * hd).  The model keeps ownership. */
q2_status q2_model_kv_cache(q2_model* model, int layer, int seq, void** k, void** v);

/* Synchronises `stream`, then reports what the model's kernels recorded since
 * the last check, and clears the record: Q2_ERR_TIMEOUT if a bounded
 * device-side wait ran out (every wait in the decode kernels, the persistent
 * and streaming steps and the tcgen05 GEMM gives up after a deadline instead
 * of hanging; the results since the last check are then undefined), else
 * Q2_ERR_INDEX if a kernel saw a token id outside the vocabulary, else Q2_OK. */
q2_status q2_model_check_error(q2_model* model, void* stream);

/* Test hook: ORs `bits` (1: out-of-range id, 2: wait ran out) into the model's
 * device error word, as a kernel would.  Synchronises. */
q2_status q2_test_model_raise_error(q2_model* model, int bits, void* stream);

/* Profiling hook of the batch-1 streaming step: runs one step on ids_dev[0]
 * (eager launch, not a graph) with per-CTA timestamps of the global timer and
 * copies them to `out` (host, n >= (5 * n_layers + 1) * grid * 4 words): for
 * phase p and CTA c, out[(p * grid + c) * 4 + k] with k = 0 phase entered,
 * 1 previous phase seen complete, 2 phase work done, 3 arrival; `grid` gets
 * the CTA count.  The model's lengths are restored afterwards (the K/V rows
 * of the traced position are written).  Synchronises. */
q2_status q2_test_trace_stream_step(q2_model* model, const int64_t* ids_dev, unsigned long long* out,
                                    size_t n, int* grid, void* stream);

/* Test hook for the waits of the batch-1 streaming step: with phase >= 0 the
 * grid counter of that phase (phases of layer l are 5l .. 5l+4: q/k/v,
 * attention, o, gate/up, down; 5 * n_layers is the lm_head) needs one more
 * arrival than the grid makes, so every CTA's wait on it runs out, and every
 * wait is bounded by `deadline_ns` instead of 200 ms; the step then carries
 * on and q2_model_check_error reports Q2_ERR_TIMEOUT.  phase = -1 restores
 * the defaults.  Drops the captured decode graphs.  Not for production use. */
q2_status q2_test_set_wait_fault(q2_model* model, int phase, unsigned long long deadline_ns);

/* Turns CUDA-graph capture of decode steps on (default) or off (eager
 * launches, for debugging and per-kernel timing). */
q2_status q2_model_set_graphs(q2_model* model, int enable);

/* Decode-step implementation for bf16 models at batch <= 4:
 * Q2_PATH_AUTO (default: the streaming step at batch 1, the persistent kernel
 * for 2 <= batch <= 4, where the shapes allow),
 * Q2_PATH_PERSISTENT (one cooperative launch per step: every CTA streams its
 * share of all weights through one TMA ring while the phases of the step run
 * between grid-wide counters), Q2_PATH_KERNELS (five fused kernels per layer
 * chained by programmatic dependent launch), Q2_PATH_GENERIC (one kernel per
 * operator), Q2_PATH_STREAM (batch 1 only: one cooperative launch per step
 * whose producer warps stream the weights of every phase ahead of the
 * phases, while the consumer warps run the phases between grid-wide
 * counters).  Larger batches and fp32 models always take the generic path.
 * Q2_ERR_STATE if the requested path is not available for this model. */
typedef enum q2_path {
  Q2_PATH_AUTO = 0,
  Q2_PATH_PERSISTENT = 1,
  Q2_PATH_KERNELS = 2,
  Q2_PATH_GENERIC = 3,
  Q2_PATH_STREAM = 4
} q2_path;
q2_status q2_model_set_decode_path(q2_model* model, int path);

/* Kernel classes of a decode step, for q2_model_time_kernels. */
typedef enum q2_kclass {
  Q2_K_EMBED = 0,   /* embedding gather */
  Q2_K_NORM = 1,    /* residual add + RMSNorm (stand-alone launches) */
  Q2_K_QKV = 2,     /* q/k/v linear (+ fused epilogues) */
  Q2_K_ROPE_KV = 3, /* RoPE + KV-cache write-back (stand-alone launches) */
  Q2_K_ATTN = 4,    /* attention over the cache (split pass + combine) */
  Q2_K_O = 5,       /* o linear */
  Q2_K_GATE_UP = 6, /* gate/up linear (+ fused epilogues) */
  Q2_K_SWIGLU = 7,  /* SwiGLU (stand-alone launches) */
  Q2_K_DOWN = 8,    /* down linear */
  Q2_K_LM_HEAD = 9, /* final norm + lm_head linear */
  Q2_K_ARGMAX = 10, /* argmax over the vocabulary */
  Q2_K_OTHER = 11,  /* length bookkeeping */
  Q2_K_STEP = 12,   /* the whole step as one persistent kernel */
  Q2_K_COUNT = 13
} q2_kclass;

/* Per-kernel device timing of decode steps.  Captures (once per batch size)
 * a copy of the decode-step graph with CUDA event-record nodes around every
 * kernel class instance, replays it `steps` times on ids [batch] (device)
 * -- each replay a real decode step that appends K/V -- then restores every
 * sequence length to its value before the call.  Writes, per class,
 * mean_ms[c] = mean device time of one instance (ms, event to event: the
 * event nodes serialise the step, so launch/drain gaps are included) and
 * per_step[c] = instances per step; *kernels_per_step = the number of
 * kernel launches in one uninstrumented step.  Synchronises `stream`. */
q2_status q2_model_time_kernels(q2_model* model, const int64_t* ids, int batch, int steps,
                                float* mean_ms, int* per_step, int* kernels_per_step,
                                void* stream);

#ifdef __cplusplus
}
#endif
#endif /* Q2_H */
