// model.cu -- the Qwen2-style decoder runtime behind q2_model_*: weights, KV
// cache and every activation buffer allocated once at create time (LLAISYS
// final report, section 3.3, item 4: per-token buffer allocation and
// per-call handle creation were the cost that dominated), prefill in
// chunks, and a decode step captured once per batch size as a CUDA graph
// whose kernels chain with programmatic dependent launch.
//
// Layer order (the Qwen2 decoder the report runs on the GPU, section 3.2,
// fourth layer): RMSNorm -> q/k/v linear (+bias) -> RoPE -> KV write-back ->
// causal GQA attention -> o linear -> residual add + RMSNorm -> gate/up
// linear -> SwiGLU -> down linear -> residual add (+ next RMSNorm).  Final:
// RMSNorm -> lm_head (fp32 logits) -> argmax.
#include <math.h>

#include <algorithm>
#include <map>
#include <vector>

#include "common.cuh"
#include "decode.h"
#include "kernels.h"
#include "gemm_tc.h"
#include "pdecode.h"
#include "sdecode.h"
#include <cstdlib>
#include "tma.h"

using namespace q2;

// Packed weight layouts (the library repacks on load):
//  wqkv [nh*hd + 2*nkv*hd, H]: head slots (q heads, then k heads, then v
//       heads); inside a slot, row 2j holds original row j and row 2j+1
//       original row j + hd/2, so the two members of a RoPE pair are adjacent
//       rows (one fused-epilogue stage sees both).  bqkv the same way.
//  wgu  [2I, H]: row 2i = gate row i, row 2i+1 = up row i.
struct LayerW {
  void* in_norm;
  void* wqkv;
  void* bqkv;
  void* wo;    // [H, nh*hd]
  void* post_norm;
  void* wgu;
  void* wd;    // [H, I]
};

// Event pairs around kernel-class instances, for q2_model_time_kernels.
struct KTiming {
  std::vector<cudaEvent_t> ev;  // 2 per mark: begin, end
  std::vector<int> cls;
  size_t used = 0;
  cudaGraphExec_t exec = nullptr;
  int kernels = 0;
};

struct q2_model {
  q2_meta m{};
  int device = 0;
  int dt = Q2_BF16;
  size_t es = 2;
  int qd = 0, kd = 0, qkvd = 0, chunk = 0, tmax = 0;

  void* wbuf = nullptr;
  void* embed = nullptr;
  void* lm_head = nullptr;
  void* final_norm = nullptr;
  std::vector<LayerW> layers;

  void* kc = nullptr;  // [L][Bmax][nkv][max_seq][hd]
  void* vc = nullptr;
  long long kv_seq_stride = 0, kv_layer_stride = 0;
  int* d_len = nullptr;
  std::vector<int> h_len;

  void *x = nullptr, *h = nullptr, *qkv = nullptr, *qb = nullptr, *att = nullptr, *o = nullptr,
       *gu = nullptr, *s = nullptr;
  float* logits = nullptr;
  int64_t* d_ids = nullptr;
  int64_t* d_next = nullptr;
  float2* rope = nullptr;  // [max_seq][hd/2] (cos, sin)
  void* attn_scratch = nullptr;
  void* attn_tc_ws = nullptr;  // the tensor-core prefill attention's work split (zeroed at creation)
  float* am_val = nullptr;
  int64_t* am_idx = nullptr;
  int* d_err = nullptr;
  unsigned* d_counters = nullptr;  // [max_batch * nkv] attention + [1] lm_head (zero between launches)
  float* lm_val = nullptr;         // lm_head per-CTA argmax partials [num_sms][kDecodeMaxBatch]
  int64_t* lm_idx = nullptr;
  void* abuf = nullptr;
  bool fused = false;              // bf16 and the fused decode kernels support the shapes
  bool persistent = false;         // ... and the persistent decode kernel does too
  bool streaming = false;          // ... and the batch-1 streaming step does too
  int sd_ring = 0;                 // streaming step: weight ring slots (Q2_SDECODE_RING overrides)
  int sd_l2_ahead = 0;             // streaming step: slots pulled into L2 ahead of the ring
  unsigned long long wait_ns = 200ull * 1000 * 1000;  // bound of every device-side wait
  uint64_t* sd_ll = nullptr;       // streaming step: tagged exchange words
  unsigned* sd_epoch = nullptr;    // streaming step: step counter (never reset)
  int stall_phase = -1;            // test hook: a phase counter that never completes
  int path = Q2_PATH_AUTO;
  // Weight stages each CTA of the persistent step pulls into L2 ahead of its
  // shared-memory ring (Q2_PDECODE_L2_AHEAD overrides; 0 turns it off).
  int l2_ahead = 16;
  PLayer* d_layers = nullptr;      // device copy of the per-layer weight pointers
  unsigned* d_sync = nullptr;      // persistent step phase counters
  unsigned long long* d_trace = nullptr;  // persistent step phase timestamps [5L + 1][4]
  float* tc_ws = nullptr;                 // split-K partial sums of the tcgen05 GEMM
  size_t tc_ws_bytes = 0;
  CUtensorMap kmap{}, vmap{};      // the K and V caches as 2-D [rows, hd] tensors

  cudaStream_t cap = nullptr;
  bool use_graphs = true;
  std::map<int, cudaGraphExec_t> graphs;
  KTiming* tm = nullptr;  // set while capturing an instrumented step
  std::map<int, KTiming*> timed;
};

namespace {

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Begin / end of one kernel-class instance (no-ops unless an instrumented
// step is being captured).
void tbeg(q2_model* M, int cls, cudaStream_t st) {
  KTiming* t = M->tm;
  if (!t) return;
  while (t->ev.size() < 2 * t->used + 2) {
    cudaEvent_t e;
    cudaEventCreate(&e);
    t->ev.push_back(e);
  }
  t->cls.resize(t->used + 1);
  t->cls[t->used] = cls;
  cudaEventRecordWithFlags(t->ev[2 * t->used], st, cudaEventRecordExternal);
}
void tend(q2_model* M, cudaStream_t st) {
  KTiming* t = M->tm;
  if (!t) return;
  cudaEventRecordWithFlags(t->ev[2 * t->used + 1], st, cudaEventRecordExternal);
  t->used++;
}
#define TIMED(cls, expr)         \
  do {                           \
    tbeg(M, (cls), st);          \
    q2_status _ts = (expr);      \
    if (_ts != Q2_OK) return _ts; \
    tend(M, st);                 \
  } while (0)

// -------------------------------------------------- RoPE + KV write-back
// One thread per (token, head, pair j) over the nh q heads, nkv k heads and
// nkv v heads of the fused qkv row.  q is rotated in place; k is rotated and
// written to the cache; v is copied to the cache.  Decode: token t is the
// next position of sequence t.  Prefill: token t is position pos0 + t of
// sequence `seq`.
template <typename T>
__global__ void rope_kv_kernel(const T* qkv, int qkvd, T* qb, int qd, int T_, int nh, int nkv, int hd,
                               const float2* rope, T* kc, T* vc, long long kv_seq_stride, int max_seq,
                               const int* lens, int decode, int seq, int pos0) {
  pdl_launch_dependents();
  pdl_wait();
  const int half = hd >> 1;
  const int heads = nh + 2 * nkv;
  const long long total = (long long)T_ * heads * half;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(i % half);
    const int hh = (int)((i / half) % heads);
    const int t = (int)(i / ((long long)half * heads));
    const int sq = decode ? t : seq;
    const int pos = decode ? lens[t] : pos0 + t;
    const T* row = qkv + (size_t)t * qkvd + (size_t)hh * hd;  // packed: pair j at 2j, 2j+1
    const float a = to_f(row[2 * j]), b = to_f(row[2 * j + 1]);
    if (hh < nh + nkv) {
      const float2 cs = rope[(size_t)pos * half + j];
      const T ra = from_f<T>(a * cs.x - b * cs.y);
      const T rb = from_f<T>(b * cs.x + a * cs.y);
      T* dst = hh < nh ? qb + (size_t)t * qd + (size_t)hh * hd
                       : kc + (size_t)sq * kv_seq_stride + ((size_t)(hh - nh) * max_seq + pos) * hd;
      dst[j] = ra;
      dst[j + half] = rb;
    } else {
      T* dst = vc + (size_t)sq * kv_seq_stride + ((size_t)(hh - nh - nkv) * max_seq + pos) * hd;
      dst[j] = row[2 * j];
      dst[j + half] = row[2 * j + 1];
    }
  }
}

__global__ void inc_lens_kernel(int* lens, int B) {
  pdl_launch_dependents();
  pdl_wait();
  int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) lens[b] += 1;
}

__global__ void set_len_kernel(int* lens, int seq, int v) {
  pdl_wait();
  lens[seq] = v;
}

q2_status launch_rope_kv(q2_model* M, int l, int T, const int* lens, int decode, int seq, int pos0,
                         cudaStream_t st, bool pdl) {
  const q2_meta& m = M->m;
  long long work = (long long)T * (m.n_heads + 2 * m.n_kv_heads) * (m.head_dim / 2);
  int blocks = (int)((work + 255) / 256);
  if (blocks > num_sms() * 8) blocks = num_sms() * 8;
  if (blocks < 1) blocks = 1;
  size_t loff = (size_t)l * M->kv_layer_stride;
  if (M->dt == Q2_F32)
    Q2_LAUNCH(rope_kv_kernel<float>, dim3(blocks), dim3(256), 0, st, pdl, (const float*)M->qkv,
              M->qkvd, (float*)M->qb, M->qd, T, m.n_heads, m.n_kv_heads, m.head_dim,
              (const float2*)M->rope, (float*)M->kc + loff, (float*)M->vc + loff, M->kv_seq_stride,
              m.max_seq, lens, decode, seq, pos0);
  else
    Q2_LAUNCH(rope_kv_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, pdl,
              (const __nv_bfloat16*)M->qkv, M->qkvd, (__nv_bfloat16*)M->qb, M->qd, T, m.n_heads,
              m.n_kv_heads, m.head_dim, (const float2*)M->rope, (__nv_bfloat16*)M->kc + loff,
              (__nv_bfloat16*)M->vc + loff, M->kv_seq_stride, m.max_seq, lens, decode, seq, pos0);
  return Q2_OK;
}

int decode_splits(const q2_model* M, int rows) {
  return attn_splits(rows, M->m.n_kv_heads, M->m.max_seq);
}

// The decoder layers on x [T, H].  decode != 0: row t is the next token of
// sequence t; else rows are positions pos0.. of sequence `seq`.  On return,
// x holds the residual stream after the last layer.  bf16 with T >= 64 runs
// the linears on the tcgen05 GEMM with fused epilogues (gate/up + SwiGLU,
// o and down + the residual add in place); otherwise one kernel per operator.
q2_status run_layers(q2_model* M, int T, int decode, int seq, int pos0, cudaStream_t st, bool pdl) {
  const q2_meta& m = M->m;
  const int H = m.hidden, I = m.intermediate, dt = M->dt;
  const bool tc = dt == Q2_BF16 && tc_linear_supported(T, H, I, M->x, M->s, M->layers[0].wd) &&
                  tc_linear_supported(T, H, M->qd, M->x, M->att, M->layers[0].wo) &&
                  tc_linear_supported(T, 2 * I, H, M->s, M->h, M->layers[0].wgu);
  for (int l = 0; l < m.n_layers; ++l) {
    const LayerW& w = M->layers[l];
    if (l == 0)
      TIMED(Q2_K_NORM, launch_add_rms_norm(M->x, nullptr, M->h, w.in_norm, T, H, m.eps, dt, st, pdl));
    if (tc)
      TIMED(Q2_K_QKV, tc_gemm(M->qkv, M->qkvd, Q2_BF16, TC_EPI_PLAIN, M->h, w.wqkv, w.bqkv, T, M->qkvd, H,
                              st, M->d_err, M->tc_ws, M->tc_ws_bytes));
    else
      TIMED(Q2_K_QKV, launch_linear(M->qkv, M->h, w.wqkv, w.bqkv, T, M->qkvd, H, dt, dt, st, pdl));
    TIMED(Q2_K_ROPE_KV, launch_rope_kv(M, l, T, M->d_len, decode, seq, pos0, st, pdl));

    AttnRows a = {};
    a.q = M->qb;
    a.q_row_stride = M->qd;
    size_t loff = (size_t)l * M->kv_layer_stride * M->es;
    a.k = (const char*)M->kc + loff;
    a.v = (const char*)M->vc + loff;
    a.kv_seq_stride = M->kv_seq_stride;
    a.kv_tok_stride = m.head_dim;
    a.kv_head_stride = (long long)m.max_seq * m.head_dim;
    a.out = M->att;
    a.out_row_stride = M->qd;
    a.rows = T;
    a.nh = m.n_heads;
    a.nkv = m.n_kv_heads;
    a.hd = m.head_dim;
    a.scale = 1.0f / sqrtf((float)m.head_dim);
    if (decode && M->fused && dt == Q2_BF16 &&
        dattn_mma_supported(m.n_heads, m.n_kv_heads, m.head_dim, decode_splits(M, T))) {
      // decode rows over the cache: the tensor-core attention
      DAttn d = {};
      d.q = M->qb;
      d.q_stride = M->qd;
      d.out = M->att;
      d.nsplit = decode_splits(M, T);
      d.part_o = (float*)M->attn_scratch;
      d.part_ml = d.part_o + (size_t)T * m.n_heads * d.nsplit * m.head_dim;
      d.counters = M->d_counters;
      d.lens = M->d_len;
      d.B = T;
      d.nh = m.n_heads;
      d.nkv = m.n_kv_heads;
      d.hd = m.head_dim;
      d.max_seq = m.max_seq;
      d.Bmax = m.max_batch;
      d.layer = l;
      d.scale = 1.0f / sqrtf((float)m.head_dim);
      d.err = M->d_err;
      TIMED(Q2_K_ATTN, launch_dattn_mma(d, M->kmap, M->vmap, st));
    } else {
      int nsplit;
      if (decode) {
        a.base = 1;
        a.row_step = 0;
        a.lens = M->d_len;
        a.seq_is_row = 1;
        a.fixed_seq = 0;
        nsplit = decode_splits(M, T);
      } else {
        a.base = pos0 + 1;
        a.row_step = 1;
        a.lens = nullptr;
        a.seq_is_row = 0;
        a.fixed_seq = seq;
        nsplit = attn_splits(T, m.n_kv_heads, pos0 + T);
      }
      TIMED(Q2_K_ATTN, launch_attention(a, nsplit, M->attn_scratch, dt, st, pdl, M->d_err, M->attn_tc_ws));
    }

    if (tc) {
      TIMED(Q2_K_O, tc_gemm(M->x, H, Q2_BF16, TC_EPI_RESID, M->att, w.wo, nullptr, T, H, M->qd, st, M->d_err, M->tc_ws,
                              M->tc_ws_bytes));
      TIMED(Q2_K_NORM, launch_add_rms_norm(M->x, nullptr, M->h, w.post_norm, T, H, m.eps, dt, st, pdl));
      TIMED(Q2_K_GATE_UP, tc_gemm(M->s, I, Q2_BF16, TC_EPI_SWIGLU, M->h, w.wgu, nullptr, T, 2 * I, H, st,
                                    M->d_err, M->tc_ws, M->tc_ws_bytes));
      TIMED(Q2_K_DOWN, tc_gemm(M->x, H, Q2_BF16, TC_EPI_RESID, M->s, w.wd, nullptr, T, H, I, st, M->d_err, M->tc_ws,
                                 M->tc_ws_bytes));
      if (l + 1 < m.n_layers)
        TIMED(Q2_K_NORM, launch_add_rms_norm(M->x, nullptr, M->h, M->layers[l + 1].in_norm, T, H, m.eps,
                                             dt, st, pdl));
    } else {
      TIMED(Q2_K_O, launch_linear(M->o, M->att, w.wo, nullptr, T, H, M->qd, dt, dt, st, pdl));
      TIMED(Q2_K_NORM, launch_add_rms_norm(M->x, M->o, M->h, w.post_norm, T, H, m.eps, dt, st, pdl));
      TIMED(Q2_K_GATE_UP, launch_linear(M->gu, M->h, w.wgu, nullptr, T, 2 * I, H, dt, dt, st, pdl));
      TIMED(Q2_K_SWIGLU, launch_swiglu_interleaved(M->s, M->gu, T, I, dt, st, pdl));
      TIMED(Q2_K_DOWN, launch_linear(M->o, M->s, w.wd, nullptr, T, H, I, dt, dt, st, pdl));
      // the residual add of the down projection (fused with the next RMSNorm)
      TIMED(Q2_K_NORM, launch_add_rms_norm(M->x, M->o, l + 1 < m.n_layers ? M->h : nullptr,
                                           l + 1 < m.n_layers ? M->layers[l + 1].in_norm : nullptr, T,
                                           H, m.eps, dt, st, pdl));
    }
  }
  return Q2_OK;
}

// Final residual add + RMSNorm of `rows` rows starting at row r0, lm_head
// into logits rows lrow.., argmax into next rows lrow...
q2_status run_head(q2_model* M, int r0, int rows, int lrow, cudaStream_t st, bool pdl,
                   bool add_o = true) {
  const q2_meta& m = M->m;
  const int H = m.hidden, V = m.vocab, dt = M->dt;
  char* x = (char*)M->x + (size_t)r0 * H * M->es;
  char* o = add_o ? (char*)M->o + (size_t)r0 * H * M->es : nullptr;
  char* h = (char*)M->h + (size_t)r0 * H * M->es;
  TIMED(Q2_K_NORM, launch_add_rms_norm(x, o, h, M->final_norm, rows, H, m.eps, dt, st, pdl));
  float* lg = M->logits + (size_t)lrow * V;
  TIMED(Q2_K_LM_HEAD, launch_linear(lg, h, M->lm_head, nullptr, rows, V, H, dt, Q2_F32, st, pdl));
  int parts = argmax_parts(rows, V);
  TIMED(Q2_K_ARGMAX, launch_argmax(M->d_next + lrow, nullptr, lg, rows, V, Q2_F32, M->am_val,
                                   M->am_idx, parts, st, pdl));
  return Q2_OK;
}

// ---- the fused bf16 decode path (batch <= kDecodeMaxBatch): five kernels
// per layer, norms/RoPE/KV append/SwiGLU/residual adds in the linears'
// prologues and epilogues, split attention with its combine folded in.
bool use_stream(const q2_model* M, int B) {
  // AUTO: the streaming step at batch 1.
  return M->streaming && B == 1 && (M->path == Q2_PATH_STREAM || M->path == Q2_PATH_AUTO);
}
bool use_persistent(const q2_model* M, int B) {
  // AUTO: the persistent step where it is measured faster than the per-layer
  // kernels (2 <= B <= 4 on B200).
  return !use_stream(M, B) && M->persistent && B >= 1 && B <= kPMaxBatch &&
         (M->path == Q2_PATH_PERSISTENT || (M->path == Q2_PATH_AUTO && B >= 2));
}
bool use_fused(const q2_model* M, int B) {
  return M->fused && B >= 1 && B <= kDecodeMaxBatch && M->path != Q2_PATH_GENERIC;
}

// The whole step (or the layers alone) as one persistent cooperative launch.
q2_status persistent_step(q2_model* M, int B, bool head, bool embed_in, cudaStream_t st,
                          bool trace = false) {
  const q2_meta& m = M->m;
  PDecode p = {};
  p.layers = M->d_layers;
  p.L = m.n_layers;
  p.H = m.hidden;
  p.I = m.intermediate;
  p.V = m.vocab;
  p.nh = m.n_heads;
  p.nkv = m.n_kv_heads;
  p.hd = m.head_dim;
  p.qkvd = M->qkvd;
  p.qd = M->qd;
  p.max_seq = m.max_seq;
  p.Bmax = m.max_batch;
  p.B = B;
  p.nsplit = decode_splits(M, B);
  p.eps = m.eps;
  p.scale = 1.0f / sqrtf((float)m.head_dim);
  p.l2_ahead = M->l2_ahead;
  p.embed_in = embed_in ? 1 : 0;
  p.run_head = head ? 1 : 0;
  p.embed = M->embed;
  p.lm_head = M->lm_head;
  p.final_norm = M->final_norm;
  p.ids = M->d_ids;
  p.x = M->x;
  p.qb = M->qb;
  p.s = M->s;
  p.kc = M->kc;
  p.vc = M->vc;
  p.kv_layer_stride = M->kv_layer_stride;
  p.kv_seq_stride = M->kv_seq_stride;
  p.rope = M->rope;
  p.lens = M->d_len;
  p.part_o = (float*)M->attn_scratch;
  p.part_ml = p.part_o + (size_t)B * m.n_heads * p.nsplit * m.head_dim;
  p.logits = M->logits;
  p.am_val = M->lm_val;
  p.am_idx = M->lm_idx;
  p.next = M->d_next;
  p.att = M->att;
  p.sync = M->d_sync;
  p.trace = trace ? M->d_trace : nullptr;
  p.err = M->d_err;
  Q2_CUDA_TRY(cudaMemsetAsync(M->d_sync, 0, pdecode_sync_words(m.n_layers) * sizeof(unsigned), st));
  if (trace)
    Q2_CUDA_TRY(cudaMemsetAsync(M->d_trace, 0, (5 * (size_t)m.n_layers + 1) * 4 * sizeof(unsigned long long), st));
  TIMED(Q2_K_STEP, launch_pdecode(p, M->kmap, M->vmap, st));
  return Q2_OK;
}

// The batch-1 step (or the layers alone) as one streaming cooperative launch.
q2_status stream_step(q2_model* M, bool head, bool embed_in, cudaStream_t st, bool trace = false,
                      unsigned long long* ctrace = nullptr) {
  const q2_meta& m = M->m;
  SDecode p = {};
  p.layers = M->d_layers;
  p.L = m.n_layers;
  p.H = m.hidden;
  p.I = m.intermediate;
  p.V = m.vocab;
  p.nh = m.n_heads;
  p.nkv = m.n_kv_heads;
  p.hd = m.head_dim;
  p.qkvd = M->qkvd;
  p.qd = M->qd;
  p.max_seq = m.max_seq;
  p.Bmax = m.max_batch;
  p.nsplit = decode_splits(M, 1);
  p.eps = m.eps;
  p.scale = 1.0f / sqrtf((float)m.head_dim);
  p.embed_in = embed_in ? 1 : 0;
  p.run_head = head ? 1 : 0;
  p.embed = M->embed;
  p.lm_head = M->lm_head;
  p.final_norm = M->final_norm;
  p.ids = M->d_ids;
  p.x = M->x;
  p.kc = M->kc;
  p.vc = M->vc;
  p.kv_layer_stride = M->kv_layer_stride;
  p.rope = M->rope;
  p.lens = M->d_len;
  p.ll = sdecode_ll_carve(M->sd_ll, m.hidden, m.intermediate, m.n_heads, m.n_kv_heads, m.head_dim, num_sms());
  p.epoch = M->sd_epoch;
  p.logits = M->logits;
  p.next = M->d_next;
  p.sync = M->d_sync;
  p.trace = trace ? M->d_trace : nullptr;
  p.ctrace = ctrace;
  p.err = M->d_err;
  p.ring = M->sd_ring;
  p.l2_ahead = M->sd_l2_ahead;
  p.deadline_ns = M->wait_ns;
  p.stall_phase = M->stall_phase;
  Q2_CUDA_TRY(cudaMemsetAsync(M->d_sync, 0, sdecode_sync_words() * sizeof(unsigned), st));
  if (trace)
    Q2_CUDA_TRY(cudaMemsetAsync(M->d_trace, 0, (5 * (size_t)m.n_layers + 1) * 4 * sizeof(unsigned long long), st));
  TIMED(Q2_K_STEP, launch_sdecode(p, M->kmap, M->vmap, st));
  return Q2_OK;
}

q2_status fused_layers(q2_model* M, int B, cudaStream_t st) {
  const q2_meta& m = M->m;
  const int H = m.hidden, I = m.intermediate;
  const int nsplit = decode_splits(M, B);
  for (int l = 0; l < m.n_layers; ++l) {
    const LayerW& w = M->layers[l];
    const size_t loff = (size_t)l * M->kv_layer_stride * M->es;
    DGemv q = {};
    q.w = w.wqkv;
    q.N = M->qkvd;
    q.K = H;
    q.M = B;
    q.x = M->x;
    q.norm_w = w.in_norm;
    q.eps = m.eps;
    q.bias = w.bqkv;
    q.out = M->qb;
    q.out_stride = M->qd;
    q.kc = (char*)M->kc + loff;
    q.vc = (char*)M->vc + loff;
    q.kv_seq_stride = M->kv_seq_stride;
    q.max_seq = m.max_seq;
    q.rope = M->rope;
    q.lens = M->d_len;
    q.nh = m.n_heads;
    q.nkv = m.n_kv_heads;
    q.hd = m.head_dim;
    q.err = M->d_err;
    TIMED(Q2_K_QKV, launch_dgemv(EPI_QKV, q, st));

    DAttn a = {};
    a.q = M->qb;
    a.q_stride = M->qd;
    a.out = M->att;
    a.part_o = (float*)M->attn_scratch;
    a.part_ml = a.part_o + (size_t)B * m.n_heads * nsplit * m.head_dim;
    a.counters = M->d_counters;
    a.lens = M->d_len;
    a.B = B;
    a.nh = m.n_heads;
    a.nkv = m.n_kv_heads;
    a.hd = m.head_dim;
    a.nsplit = nsplit;
    a.max_seq = m.max_seq;
    a.Bmax = m.max_batch;
    a.layer = l;
    a.scale = 1.0f / sqrtf((float)m.head_dim);
    a.err = M->d_err;
    if (dattn_mma_supported(a.nh, a.nkv, a.hd, a.nsplit))
      TIMED(Q2_K_ATTN, launch_dattn_mma(a, M->kmap, M->vmap, st));
    else
      TIMED(Q2_K_ATTN, launch_dattn(a, M->kmap, M->vmap, st));

    DGemv o = {};
    o.w = w.wo;
    o.N = H;
    o.K = M->qd;
    o.M = B;
    o.x = M->att;
    o.out = M->x;
    o.out_stride = H;
    o.err = M->d_err;
    TIMED(Q2_K_O, launch_dgemv(EPI_RESID, o, st));

    DGemv gu = {};
    gu.w = w.wgu;
    gu.N = 2 * I;
    gu.K = H;
    gu.M = B;
    gu.x = M->x;
    gu.norm_w = w.post_norm;
    gu.eps = m.eps;
    gu.out = M->s;
    gu.out_stride = I;
    gu.err = M->d_err;
    TIMED(Q2_K_GATE_UP, launch_dgemv(EPI_SWIGLU, gu, st));

    DGemv dn = {};
    dn.w = w.wd;
    dn.N = H;
    dn.K = I;
    dn.M = B;
    dn.x = M->s;
    dn.out = M->x;
    dn.out_stride = H;
    dn.err = M->d_err;
    TIMED(Q2_K_DOWN, launch_dgemv(EPI_RESID, dn, st));
  }
  return Q2_OK;
}

q2_status fused_head(q2_model* M, int B, cudaStream_t st) {
  const q2_meta& m = M->m;
  DGemv h = {};
  h.w = M->lm_head;
  h.N = m.vocab;
  h.K = m.hidden;
  h.M = B;
  h.x = M->x;
  h.norm_w = M->final_norm;
  h.eps = m.eps;
  h.logits = M->logits;
  h.am_val = M->lm_val;
  h.am_idx = M->lm_idx;
  h.counter = M->d_counters + (size_t)m.max_batch * m.n_kv_heads;
  h.next = M->d_next;
  h.lens_inc = M->d_len;
  h.err = M->d_err;
  TIMED(Q2_K_LM_HEAD, launch_dgemv(EPI_LOGITS, h, st));
  return Q2_OK;
}

q2_status decode_body_fused(q2_model* M, int B, cudaStream_t st) {
  const q2_meta& m = M->m;
  TIMED(Q2_K_EMBED,
        launch_embedding(M->x, M->d_ids, M->embed, B, m.vocab, m.hidden, M->dt, M->d_err, st, true));
  Q2_TRY(fused_layers(M, B, st));
  return fused_head(M, B, st);
}

q2_status decode_body(q2_model* M, int B, cudaStream_t st) {
  if (use_stream(M, B)) return stream_step(M, true, true, st);
  if (use_persistent(M, B)) return persistent_step(M, B, true, true, st);
  if (use_fused(M, B)) return decode_body_fused(M, B, st);
  const bool pdl = true;
  const q2_meta& m = M->m;
  TIMED(Q2_K_EMBED,
        launch_embedding(M->x, M->d_ids, M->embed, B, m.vocab, m.hidden, M->dt, M->d_err, st, pdl));
  Q2_TRY(run_layers(M, B, 1, 0, 0, st, pdl));
  Q2_TRY(run_head(M, 0, B, 0, st, pdl, false));
  tbeg(M, Q2_K_OTHER, st);
  Q2_LAUNCH(inc_lens_kernel, dim3(1), dim3(64 * ((B + 63) / 64)), 0, st, pdl, M->d_len, B);
  tend(M, st);
  return Q2_OK;
}

q2_status check_stream_device(q2_model* M, cudaStream_t st) {
  if (!st) return Q2_OK;
  int dev = -1;
  cudaError_t e = cudaStreamGetDevice(st, &dev);
  if (e == cudaSuccess && dev != M->device) {
    set_error("stream belongs to another device than the model");
    return Q2_ERR_INVALID_ARG;
  }
  return Q2_OK;
}

q2_status check_decode_capacity(q2_model* M, int B) {
  for (int b = 0; b < B; ++b)
    if (M->h_len[b] >= M->m.max_seq) {
      set_error("decode_step: a sequence is full (max_seq)");
      return Q2_ERR_CAPACITY;
    }
  return Q2_OK;
}

// Runs one decode step on the ids already in d_ids: the captured graph for
// this batch size (captured on first use), or eager launches.
q2_status decode_launch(q2_model* M, int B, cudaStream_t st) {
  if (M->use_graphs) {
    auto it = M->graphs.find(B);
    if (it == M->graphs.end()) {
      cudaGraph_t graph = nullptr;
      Q2_CUDA_TRY(cudaStreamBeginCapture(M->cap, cudaStreamCaptureModeThreadLocal));
      q2_status s = decode_body(M, B, M->cap);
      cudaError_t e = cudaStreamEndCapture(M->cap, &graph);
      if (s != Q2_OK) {
        if (graph) cudaGraphDestroy(graph);
        return s;
      }
      if (e != cudaSuccess) {
        set_error(std::string("decode graph capture: ") + cudaGetErrorString(e));
        return Q2_ERR_CUDA;
      }
      cudaGraphExec_t exec = nullptr;
      e = cudaGraphInstantiate(&exec, graph, 0);
      cudaGraphDestroy(graph);
      if (e != cudaSuccess) {
        set_error(std::string("decode graph instantiate: ") + cudaGetErrorString(e));
        return Q2_ERR_CUDA;
      }
      it = M->graphs.emplace(B, exec).first;
    }
    Q2_CUDA_TRY(cudaGraphLaunch(it->second, st));
  } else {
    Q2_TRY(decode_body(M, B, st));
  }
  for (int b = 0; b < B; ++b) M->h_len[b] += 1;
  return Q2_OK;
}

}  // namespace

// ===================================================================== ABI
extern "C" {

q2_status q2_model_create(const q2_meta* meta, int device, q2_model** out) {
  clear_error();
  Q2_CHECK_ARG(meta && out, Q2_ERR_INVALID_ARG, "model_create: NULL argument");
  const q2_meta& m = *meta;
  Q2_CHECK_ARG(m.dtype == Q2_F32 || m.dtype == Q2_BF16, Q2_ERR_DTYPE, "model_create: bad dtype");
  Q2_CHECK_ARG(m.n_layers > 0 && m.hidden > 0 && m.n_heads > 0 && m.n_kv_heads > 0 &&
                   m.intermediate > 0 && m.vocab > 0 && m.max_seq > 0 && m.max_batch > 0 &&
                   m.max_prefill_tokens >= 0,
               Q2_ERR_SHAPE, "model_create: sizes must be positive");
  Q2_CHECK_ARG(m.head_dim == 32 || m.head_dim == 64 || m.head_dim == 128, Q2_ERR_SHAPE,
               "model_create: head_dim must be 32, 64 or 128");
  Q2_CHECK_ARG(m.n_heads % m.n_kv_heads == 0 && m.n_heads / m.n_kv_heads <= 8, Q2_ERR_SHAPE,
               "model_create: need n_heads % n_kv_heads == 0 and a group of at most 8");
  Q2_CHECK_ARG(m.hidden % 8 == 0 && m.intermediate % 8 == 0, Q2_ERR_SHAPE,
               "model_create: hidden and intermediate must be multiples of 8");
  Q2_CHECK_ARG(m.max_batch <= 1024 && m.max_seq <= (1 << 24), Q2_ERR_SHAPE,
               "model_create: max_batch <= 1024 and max_seq <= 2^24");
  int ndev = 0;
  Q2_CUDA_TRY(cudaGetDeviceCount(&ndev));
  Q2_CHECK_ARG(device >= 0 && device < ndev, Q2_ERR_INVALID_ARG, "model_create: no such device");
  Q2_CUDA_TRY(cudaSetDevice(device));

  q2_model* M = new q2_model();
  M->m = m;
  M->device = device;
  M->dt = m.dtype;
  M->es = dtype_size(m.dtype);
  M->qd = m.n_heads * m.head_dim;
  M->kd = m.n_kv_heads * m.head_dim;
  M->qkvd = M->qd + 2 * M->kd;
  M->chunk = m.max_prefill_tokens > 0 ? m.max_prefill_tokens : 4096;
  M->tmax = M->chunk > m.max_batch ? M->chunk : m.max_batch;
  M->h_len.assign(m.max_batch, 0);
  M->layers.resize(m.n_layers);

  auto fail = [&](q2_status s) {
    q2_model_destroy(M);
    return s;
  };

  // ---- weights: one allocation, 256-byte aligned pieces
  const size_t es = M->es, H = m.hidden, I = m.intermediate, V = m.vocab;
  std::vector<std::pair<void**, size_t>> wl;
  wl.push_back({&M->embed, V * H * es});
  wl.push_back({&M->lm_head, V * H * es});
  wl.push_back({&M->final_norm, H * es});
  for (auto& L : M->layers) {
    wl.push_back({&L.in_norm, H * es});
    wl.push_back({&L.wqkv, (size_t)M->qkvd * H * es});
    wl.push_back({&L.bqkv, (size_t)M->qkvd * es});
    wl.push_back({&L.wo, H * M->qd * es});
    wl.push_back({&L.post_norm, H * es});
    wl.push_back({&L.wgu, 2 * I * H * es});
    wl.push_back({&L.wd, H * I * es});
  }
  size_t wbytes = 0;
  for (auto& p : wl) wbytes += align_up(p.second, 256);
  if (cudaMalloc(&M->wbuf, wbytes) != cudaSuccess) {
    set_error("model_create: cannot allocate weights");
    return fail(Q2_ERR_OOM);
  }
  cudaMemset(M->wbuf, 0, wbytes);
  {
    char* p = (char*)M->wbuf;
    for (auto& q : wl) {
      *q.first = p;
      p += align_up(q.second, 256);
    }
  }

  // ---- KV cache
  M->kv_seq_stride = (long long)m.n_kv_heads * m.max_seq * m.head_dim;
  M->kv_layer_stride = M->kv_seq_stride * m.max_batch;
  size_t kvbytes = (size_t)M->kv_layer_stride * m.n_layers * es;
  if (cudaMalloc(&M->kc, kvbytes) != cudaSuccess || cudaMalloc(&M->vc, kvbytes) != cudaSuccess) {
    set_error("model_create: cannot allocate the KV cache");
    return fail(Q2_ERR_OOM);
  }
  cudaMemset(M->kc, 0, kvbytes);
  cudaMemset(M->vc, 0, kvbytes);

  // ---- activations and scratch
  size_t T = M->tmax;
  size_t scratch = 0;
  for (int r = 1; r <= M->tmax; ++r) {
    size_t b = attn_scratch_bytes(r, m.n_heads, m.head_dim, attn_splits(r, m.n_kv_heads, m.max_seq));
    if (b > scratch) scratch = b;
  }
  // The fused decode attention always writes split partials (even with one split).
  for (int r = 1; r <= m.max_batch && r <= kDecodeMaxBatch; ++r) {
    const size_t n = (size_t)r * m.n_heads * attn_splits(r, m.n_kv_heads, m.max_seq);
    const size_t b = n * m.head_dim * sizeof(float) + 2 * n * sizeof(float) + 256;
    if (b > scratch) scratch = b;
  }
  size_t am = 0;
  for (int r = 1; r <= m.max_batch; ++r) {
    size_t b = (size_t)r * argmax_parts(r, V);
    if (b > am) am = b;
  }
  std::vector<std::pair<void**, size_t>> al;
  al.push_back({&M->x, T * H * es});
  al.push_back({&M->h, T * H * es});
  al.push_back({&M->qkv, T * M->qkvd * es});
  al.push_back({&M->qb, T * M->qd * es});
  al.push_back({&M->att, T * M->qd * es});
  al.push_back({&M->o, T * H * es});
  al.push_back({&M->gu, T * 2 * I * es});
  al.push_back({&M->s, T * I * es});
  al.push_back({(void**)&M->logits, (size_t)m.max_batch * V * sizeof(float)});
  al.push_back({(void**)&M->d_ids, T * sizeof(int64_t)});
  al.push_back({(void**)&M->d_next, (size_t)m.max_batch * sizeof(int64_t)});
  al.push_back({(void**)&M->rope, (size_t)m.max_seq * (m.head_dim / 2) * sizeof(float2)});
  al.push_back({&M->attn_scratch, scratch});
  if (M->dt == Q2_BF16 && m.head_dim == 128) al.push_back({&M->attn_tc_ws, attn_tc_ws_bytes()});
  al.push_back({(void**)&M->am_val, am * sizeof(float)});
  al.push_back({(void**)&M->am_idx, am * sizeof(int64_t)});
  al.push_back({(void**)&M->d_len, (size_t)m.max_batch * sizeof(int)});
  al.push_back({(void**)&M->d_err, sizeof(int)});
  al.push_back({(void**)&M->d_counters, ((size_t)m.max_batch * m.n_kv_heads + 16) * sizeof(unsigned)});
  al.push_back({(void**)&M->lm_val, (size_t)num_sms() * kDecodeMaxBatch * sizeof(float)});
  al.push_back({(void**)&M->lm_idx, (size_t)num_sms() * kDecodeMaxBatch * sizeof(int64_t)});
  const size_t sync_words = std::max(pdecode_sync_words(m.n_layers), sdecode_sync_words());
  al.push_back({(void**)&M->d_sync, sync_words * sizeof(unsigned)});
  if (M->dt == Q2_BF16 && m.head_dim % 2 == 0 && m.n_heads % m.n_kv_heads == 0) {
    al.push_back({(void**)&M->sd_ll, sdecode_ll_words(m.hidden, m.intermediate, m.n_heads, m.n_kv_heads,
                                                      m.head_dim, num_sms()) * sizeof(uint64_t)});
    al.push_back({(void**)&M->sd_epoch, sizeof(unsigned)});
  }
  al.push_back({(void**)&M->d_layers, (size_t)m.n_layers * sizeof(PLayer)});
  al.push_back({(void**)&M->d_trace, (5 * (size_t)m.n_layers + 1) * 4 * sizeof(unsigned long long)});
  if (M->dt == Q2_BF16) {
    // Split-K partial sums of the tcgen05 GEMM: a product is split only while
    // it has fewer tiles than SMs, so splits x tokens x features stays near
    // SMs x 256 x 128 x 4 bytes (~20 MB); calls that need more split less.
    M->tc_ws_bytes = (size_t)40 << 20;
    al.push_back({(void**)&M->tc_ws, M->tc_ws_bytes});
  }
  size_t abytes = 0;
  for (auto& p : al) abytes += align_up(p.second ? p.second : 1, 256);
  if (cudaMalloc(&M->abuf, abytes) != cudaSuccess) {
    set_error("model_create: cannot allocate activation buffers");
    return fail(Q2_ERR_OOM);
  }
  cudaMemset(M->abuf, 0, abytes);
  {
    char* p = (char*)M->abuf;
    for (auto& q : al) {
      *q.first = p;
      p += align_up(q.second ? q.second : 1, 256);
    }
  }
  if (!scratch) M->attn_scratch = nullptr;

  // ---- RoPE table: angle pos * theta^(-2j/hd) and its cos/sin in double,
  // stored as fp32 pairs.
  {
    const int half = m.head_dim / 2;
    std::vector<float2> tab((size_t)m.max_seq * half);
    for (int j = 0; j < half; ++j) {
      double inv = pow((double)m.theta, -(2.0 * j) / (double)m.head_dim);
      for (int p = 0; p < m.max_seq; ++p) {
        double a = (double)p * inv;
        tab[(size_t)p * half + j] = make_float2((float)cos(a), (float)sin(a));
      }
    }
    if (cudaMemcpy(M->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) !=
        cudaSuccess) {
      set_error("model_create: cannot upload the RoPE table");
      return fail(Q2_ERR_CUDA);
    }
  }
  // ---- the fused bf16 decode path: K/V caches as 2-D [rows, hd] tensors for TMA
  if (m.dtype == Q2_BF16 && dattn_supported(m.n_heads, m.n_kv_heads, m.head_dim) &&
      dgemv_supported(EPI_QKV, M->qkvd, m.hidden) && dgemv_supported(EPI_RESID, m.hidden, M->qd) &&
      dgemv_supported(EPI_SWIGLU, 2 * m.intermediate, m.hidden) &&
      dgemv_supported(EPI_RESID, m.hidden, m.intermediate) &&
      dgemv_supported(EPI_LOGITS, m.vocab, m.hidden)) {
    const uint64_t rows = (uint64_t)m.n_layers * m.max_batch * m.n_kv_heads * m.max_seq;
    const uint64_t pitch = (uint64_t)m.head_dim * 2;
    q2_status ks = make_tmap_2d_bf16(&M->kmap, M->kc, rows, m.head_dim, pitch, 64, 64, 128);
    q2_status vs = ks == Q2_OK ? make_tmap_2d_bf16(&M->vmap, M->vc, rows, m.head_dim, pitch, 64, 64, 128)
                               : ks;
    M->fused = (vs == Q2_OK) && rows < (1ull << 31);
    M->persistent = M->fused && pdecode_supported(m.hidden, m.intermediate, m.vocab, m.n_heads,
                                                  m.n_kv_heads, m.head_dim, M->qkvd, M->qd);
    M->streaming = M->fused && sdecode_supported(m.hidden, m.intermediate, m.vocab, m.n_heads,
                                                 m.n_kv_heads, m.head_dim, M->qkvd, M->qd);
    M->sd_ring = std::min(6, sdecode_max_ring(m.n_layers));
    M->streaming = M->streaming && M->sd_ring >= 2 && M->sd_ll != nullptr;
    // Tuning knobs of the persistent and streaming steps (for measurements).
    if (const char* env = getenv("Q2_PDECODE_L2_AHEAD")) {
      const int v = atoi(env);
      if (v >= 0 && v <= 256) M->l2_ahead = v;
    }
    if (const char* env = getenv("Q2_SDECODE_RING")) {
      const int v = atoi(env);
      if (v >= 2 && v <= 16) M->sd_ring = v;
    }
    if (const char* env = getenv("Q2_SDECODE_L2_AHEAD")) {
      const int v = atoi(env);
      if (v >= 0 && v <= 256) M->sd_l2_ahead = v;
    }
    clear_error();
  }
  {
    std::vector<PLayer> pl(m.n_layers);
    for (int l = 0; l < m.n_layers; ++l) {
      const LayerW& w = M->layers[l];
      pl[l] = PLayer{w.in_norm, w.wqkv, w.bqkv, w.wo, w.post_norm, w.wgu, w.wd};
    }
    if (cudaMemcpy(M->d_layers, pl.data(), pl.size() * sizeof(PLayer), cudaMemcpyHostToDevice) !=
        cudaSuccess) {
      set_error("model_create: cannot upload the layer table");
      return fail(Q2_ERR_CUDA);
    }
  }
  if (cudaStreamCreateWithFlags(&M->cap, cudaStreamNonBlocking) != cudaSuccess) {
    set_error("model_create: cannot create a stream");
    return fail(Q2_ERR_CUDA);
  }
  if (cudaDeviceSynchronize() != cudaSuccess) {
    set_error(std::string("model_create: ") + cudaGetErrorString(cudaGetLastError()));
    return fail(Q2_ERR_CUDA);
  }
  *out = M;
  return Q2_OK;
}

q2_status q2_model_destroy(q2_model* M) {
  clear_error();
  if (!M) return Q2_OK;
  DeviceGuard g(M->device);
  for (auto& kv : M->graphs) cudaGraphExecDestroy(kv.second);
  M->graphs.clear();
  for (auto& kv : M->timed) {
    if (kv.second->exec) cudaGraphExecDestroy(kv.second->exec);
    for (cudaEvent_t e : kv.second->ev) cudaEventDestroy(e);
    delete kv.second;
  }
  M->timed.clear();
  if (M->cap) cudaStreamDestroy(M->cap);
  cudaFree(M->wbuf);
  cudaFree(M->kc);
  cudaFree(M->vc);
  cudaFree(M->abuf);
  delete M;
  return Q2_OK;
}

q2_status q2_model_load_weight(q2_model* M, int kind, int layer, const void* src, size_t nbytes,
                               void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && src, Q2_ERR_INVALID_ARG, "load_weight: NULL argument");
  const q2_meta& m = M->m;
  const size_t es = M->es, H = m.hidden, I = m.intermediate, V = m.vocab;
  bool per_layer = kind >= Q2_W_IN_NORM && kind <= Q2_W_DOWN;
  Q2_CHECK_ARG(kind >= Q2_W_EMBED && kind <= Q2_W_DOWN, Q2_ERR_INVALID_ARG, "load_weight: bad kind");
  Q2_CHECK_ARG(!per_layer || (layer >= 0 && layer < m.n_layers), Q2_ERR_INVALID_ARG,
               "load_weight: bad layer");
  LayerW* L = per_layer ? &M->layers[layer] : nullptr;
  char* dst = nullptr;
  size_t want = 0;
  switch (kind) {
    case Q2_W_EMBED: dst = (char*)M->embed; want = V * H; break;
    case Q2_W_LM_HEAD: dst = (char*)M->lm_head; want = V * H; break;
    case Q2_W_FINAL_NORM: dst = (char*)M->final_norm; want = H; break;
    case Q2_W_IN_NORM: dst = (char*)L->in_norm; want = H; break;
    case Q2_W_Q: dst = (char*)L->wqkv; want = (size_t)M->qd * H; break;
    case Q2_W_K: dst = (char*)L->wqkv + (size_t)M->qd * H * es; want = (size_t)M->kd * H; break;
    case Q2_W_V: dst = (char*)L->wqkv + (size_t)(M->qd + M->kd) * H * es; want = (size_t)M->kd * H; break;
    case Q2_W_Q_BIAS: dst = (char*)L->bqkv; want = M->qd; break;
    case Q2_W_K_BIAS: dst = (char*)L->bqkv + (size_t)M->qd * es; want = M->kd; break;
    case Q2_W_V_BIAS: dst = (char*)L->bqkv + (size_t)(M->qd + M->kd) * es; want = M->kd; break;
    case Q2_W_O: dst = (char*)L->wo; want = H * M->qd; break;
    case Q2_W_POST_NORM: dst = (char*)L->post_norm; want = H; break;
    case Q2_W_GATE: dst = (char*)L->wgu; want = I * H; break;
    case Q2_W_UP: dst = (char*)L->wgu + I * H * es; want = I * H; break;
    case Q2_W_DOWN: dst = (char*)L->wd; want = H * I; break;
  }
  Q2_CHECK_ARG(nbytes == want * es, Q2_ERR_SHAPE, "load_weight: nbytes does not match the tensor size");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  const char* sp = static_cast<const char*>(src);
  const size_t hd = m.head_dim, half = hd / 2;
  switch (kind) {
    case Q2_W_Q:
    case Q2_W_K:
    case Q2_W_V:
    case Q2_W_Q_BIAS:
    case Q2_W_K_BIAS:
    case Q2_W_V_BIAS: {
      // Head slot by head slot: original rows j < hd/2 go to packed rows 2j,
      // rows j + hd/2 to packed rows 2j + 1 (a row of a bias is one element).
      const bool bias = kind == Q2_W_Q_BIAS || kind == Q2_W_K_BIAS || kind == Q2_W_V_BIAS;
      const size_t row = bias ? es : H * es;
      const int heads = (kind == Q2_W_Q || kind == Q2_W_Q_BIAS) ? m.n_heads : m.n_kv_heads;
      for (int hh = 0; hh < heads; ++hh) {
        char* d = dst + (size_t)hh * hd * row;
        const char* s0 = sp + (size_t)hh * hd * row;
        Q2_CUDA_TRY(cudaMemcpy2DAsync(d, 2 * row, s0, row, row, half, cudaMemcpyDeviceToDevice, st));
        Q2_CUDA_TRY(cudaMemcpy2DAsync(d + row, 2 * row, s0 + half * row, row, row, half,
                                      cudaMemcpyDeviceToDevice, st));
      }
      return Q2_OK;
    }
    case Q2_W_GATE:
    case Q2_W_UP: {
      // Interleaved rows: gate row i -> packed row 2i, up row i -> 2i + 1.
      char* d = (char*)L->wgu + (kind == Q2_W_UP ? H * es : 0);
      Q2_CUDA_TRY(cudaMemcpy2DAsync(d, 2 * H * es, sp, H * es, H * es, I, cudaMemcpyDeviceToDevice, st));
      return Q2_OK;
    }
    default:
      Q2_CUDA_TRY(cudaMemcpyAsync(dst, src, nbytes, cudaMemcpyDeviceToDevice, st));
      return Q2_OK;
  }
}

q2_status q2_model_decode_step(q2_model* M, const int64_t* ids, int B, int64_t* next, float* logits,
                               void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && ids && next, Q2_ERR_INVALID_ARG, "decode_step: NULL argument");
  Q2_CHECK_ARG(B >= 1 && B <= M->m.max_batch, Q2_ERR_CAPACITY, "decode_step: batch outside [1, max_batch]");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  Q2_TRY(check_decode_capacity(M, B));
  Q2_CUDA_TRY(cudaMemcpyAsync(M->d_ids, ids, B * sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
  Q2_TRY(decode_launch(M, B, st));
  Q2_CUDA_TRY(cudaMemcpyAsync(next, M->d_next, B * sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
  if (logits)
    Q2_CUDA_TRY(cudaMemcpyAsync(logits, M->logits, (size_t)B * M->m.vocab * sizeof(float),
                                cudaMemcpyDeviceToDevice, st));
  return Q2_OK;
}

q2_status q2_model_decode_step_host(q2_model* M, const int64_t* ids_host, int B, int64_t* next_host,
                                    void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && ids_host && next_host, Q2_ERR_INVALID_ARG, "decode_step_host: NULL argument");
  Q2_CHECK_ARG(B >= 1 && B <= M->m.max_batch, Q2_ERR_CAPACITY, "decode_step_host: batch outside [1, max_batch]");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  Q2_TRY(check_decode_capacity(M, B));
  Q2_CUDA_TRY(cudaMemcpyAsync(M->d_ids, ids_host, B * sizeof(int64_t), cudaMemcpyHostToDevice, st));
  Q2_TRY(decode_launch(M, B, st));
  Q2_CUDA_TRY(cudaMemcpyAsync(next_host, M->d_next, B * sizeof(int64_t), cudaMemcpyDeviceToHost, st));
  Q2_CUDA_TRY(cudaStreamSynchronize(st));
  return Q2_OK;
}

q2_status q2_model_forward_hidden(q2_model* M, const void* x_in, int B, void* x_out, void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && x_in && x_out, Q2_ERR_INVALID_ARG, "forward_hidden: NULL argument");
  Q2_CHECK_ARG(B >= 1 && B <= M->m.max_batch, Q2_ERR_CAPACITY, "forward_hidden: batch outside [1, max_batch]");
  for (int b = 0; b < B; ++b)
    Q2_CHECK_ARG(M->h_len[b] < M->m.max_seq, Q2_ERR_CAPACITY, "forward_hidden: a sequence is full");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  const size_t bytes = (size_t)B * M->m.hidden * M->es;
  Q2_CUDA_TRY(cudaMemcpyAsync(M->x, x_in, bytes, cudaMemcpyDeviceToDevice, st));
  if (use_stream(M, B) || use_persistent(M, B)) {
    if (use_stream(M, B))
      Q2_TRY(stream_step(M, false, false, st));  // advances the length itself
    else
      Q2_TRY(persistent_step(M, B, false, false, st));  // advances the lengths itself
    Q2_CUDA_TRY(cudaMemcpyAsync(x_out, M->x, bytes, cudaMemcpyDeviceToDevice, st));
    for (int b = 0; b < B; ++b) M->h_len[b] += 1;
    return Q2_OK;
  }
  if (use_fused(M, B)) {
    Q2_TRY(fused_layers(M, B, st));  // the residual stream ends in x
  } else {
    Q2_TRY(run_layers(M, B, 1, 0, 0, st, false));
  }
  Q2_CUDA_TRY(cudaMemcpyAsync(x_out, M->x, bytes, cudaMemcpyDeviceToDevice, st));
  Q2_LAUNCH(inc_lens_kernel, dim3(1), dim3(64 * ((B + 63) / 64)), 0, st, false, M->d_len, B);
  for (int b = 0; b < B; ++b) M->h_len[b] += 1;
  return Q2_OK;
}

q2_status q2_model_prefill(q2_model* M, const int64_t* ids, int batch, const int32_t* lens,
                           int64_t* next, float* logits, void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && ids && lens && next, Q2_ERR_INVALID_ARG, "prefill: NULL argument");
  Q2_CHECK_ARG(batch >= 1 && batch <= M->m.max_batch, Q2_ERR_CAPACITY, "prefill: batch outside [1, max_batch]");
  for (int b = 0; b < batch; ++b) {
    Q2_CHECK_ARG(lens[b] >= 0, Q2_ERR_INVALID_ARG, "prefill: negative length");
    Q2_CHECK_ARG((long long)M->h_len[b] + lens[b] <= M->m.max_seq, Q2_ERR_CAPACITY,
                 "prefill: a sequence would pass max_seq");
  }
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  const q2_meta& m = M->m;
  const bool pdl = true;
  size_t off = 0;
  for (int b = 0; b < batch; ++b) {
    const int n = lens[b];
    for (int c = 0; c < n; c += M->chunk) {
      const int T = n - c < M->chunk ? n - c : M->chunk;
      const int pos0 = M->h_len[b];
      Q2_CUDA_TRY(cudaMemcpyAsync(M->d_ids, ids + off + c, T * sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
      Q2_TRY(launch_embedding(M->x, M->d_ids, M->embed, T, m.vocab, m.hidden, M->dt, M->d_err, st, pdl));
      Q2_TRY(run_layers(M, T, 0, b, pos0, st, pdl));
      M->h_len[b] = pos0 + T;
      Q2_LAUNCH(set_len_kernel, dim3(1), dim3(1), 0, st, pdl, M->d_len, b, pos0 + T);
      if (c + T == n) {
        Q2_TRY(run_head(M, T - 1, 1, b, st, pdl, false));
        Q2_CUDA_TRY(cudaMemcpyAsync(next + b, M->d_next + b, sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
        if (logits)
          Q2_CUDA_TRY(cudaMemcpyAsync(logits + (size_t)b * m.vocab, M->logits + (size_t)b * m.vocab,
                                      (size_t)m.vocab * sizeof(float), cudaMemcpyDeviceToDevice, st));
      }
    }
    off += n;
  }
  return Q2_OK;
}

q2_status q2_model_reset_kv(q2_model* M, int seq) {
  clear_error();
  Q2_CHECK_ARG(M, Q2_ERR_INVALID_ARG, "reset_kv: NULL model");
  Q2_CHECK_ARG(seq >= -1 && seq < M->m.max_batch, Q2_ERR_INVALID_ARG, "reset_kv: bad sequence");
  DeviceGuard g(M->device);
  Q2_CUDA_TRY(cudaDeviceSynchronize());
  if (seq == -1) {
    std::fill(M->h_len.begin(), M->h_len.end(), 0);
    Q2_CUDA_TRY(cudaMemset(M->d_len, 0, M->m.max_batch * sizeof(int)));
  } else {
    M->h_len[seq] = 0;
    Q2_CUDA_TRY(cudaMemset(M->d_len + seq, 0, sizeof(int)));
  }
  return Q2_OK;
}

q2_status q2_model_set_seq_len(q2_model* M, int seq, int len) {
  clear_error();
  Q2_CHECK_ARG(M, Q2_ERR_INVALID_ARG, "set_seq_len: NULL model");
  Q2_CHECK_ARG(seq >= 0 && seq < M->m.max_batch, Q2_ERR_INVALID_ARG, "set_seq_len: bad sequence");
  Q2_CHECK_ARG(len >= 0 && len <= M->m.max_seq, Q2_ERR_CAPACITY, "set_seq_len: length outside [0, max_seq]");
  DeviceGuard g(M->device);
  Q2_CUDA_TRY(cudaDeviceSynchronize());
  M->h_len[seq] = len;
  Q2_CUDA_TRY(cudaMemcpy(M->d_len + seq, &len, sizeof(int), cudaMemcpyHostToDevice));
  return Q2_OK;
}

q2_status q2_model_get_seq_len(const q2_model* M, int seq, int* len) {
  clear_error();
  Q2_CHECK_ARG(M && len, Q2_ERR_INVALID_ARG, "get_seq_len: NULL argument");
  Q2_CHECK_ARG(seq >= 0 && seq < M->m.max_batch, Q2_ERR_INVALID_ARG, "get_seq_len: bad sequence");
  *len = M->h_len[seq];
  return Q2_OK;
}

q2_status q2_model_kv_cache(q2_model* M, int layer, int seq, void** k, void** v) {
  clear_error();
  Q2_CHECK_ARG(M && k && v, Q2_ERR_INVALID_ARG, "kv_cache: NULL argument");
  Q2_CHECK_ARG(layer >= 0 && layer < M->m.n_layers && seq >= 0 && seq < M->m.max_batch,
               Q2_ERR_INVALID_ARG, "kv_cache: bad layer or sequence");
  size_t off = ((size_t)layer * M->kv_layer_stride + (size_t)seq * M->kv_seq_stride) * M->es;
  *k = (char*)M->kc + off;
  *v = (char*)M->vc + off;
  return Q2_OK;
}

q2_status q2_model_check_error(q2_model* M, void* stream) {
  clear_error();
  Q2_CHECK_ARG(M, Q2_ERR_INVALID_ARG, "check_error: NULL model");
  DeviceGuard g(M->device);
  Q2_CUDA_TRY(cudaStreamSynchronize(as_stream(stream)));
  int v = 0;
  Q2_CUDA_TRY(cudaMemcpy(&v, M->d_err, sizeof v, cudaMemcpyDeviceToHost));
  if (v) {
    int zero = 0;
    Q2_CUDA_TRY(cudaMemcpy(M->d_err, &zero, sizeof zero, cudaMemcpyHostToDevice));
    return device_error_status(v, "model_check_error");
  }
  return Q2_OK;
}

q2_status q2_test_model_raise_error(q2_model* M, int bits, void* stream) {
  clear_error();
  Q2_CHECK_ARG(M, Q2_ERR_INVALID_ARG, "test_model_raise_error: NULL model");
  Q2_CHECK_ARG(bits > 0 && bits <= (kErrIndex | kErrTimeout), Q2_ERR_INVALID_ARG,
               "test_model_raise_error: bits must be 1, 2 or 3");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  int cur = 0;
  Q2_CUDA_TRY(cudaMemcpyAsync(&cur, M->d_err, sizeof cur, cudaMemcpyDeviceToHost, st));
  Q2_CUDA_TRY(cudaStreamSynchronize(st));
  cur |= bits;
  Q2_CUDA_TRY(cudaMemcpyAsync(M->d_err, &cur, sizeof cur, cudaMemcpyHostToDevice, st));
  Q2_CUDA_TRY(cudaStreamSynchronize(st));
  return Q2_OK;
}

q2_status q2_test_trace_stream_step(q2_model* M, const int64_t* ids, unsigned long long* out, size_t n,
                                    int* grid, void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && ids && out && grid, Q2_ERR_INVALID_ARG, "trace_stream_step: NULL argument");
  Q2_CHECK_ARG(M->streaming, Q2_ERR_STATE, "trace_stream_step: the streaming step does not support this model");
  Q2_CHECK_ARG(M->h_len[0] < M->m.max_seq, Q2_ERR_CAPACITY, "trace_stream_step: the sequence is full");
  const size_t words = (5 * (size_t)M->m.n_layers + 1) * num_sms() * 4;
  Q2_CHECK_ARG(n >= words, Q2_ERR_SHAPE, "trace_stream_step: output too small");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  unsigned long long* d = nullptr;
  Q2_CUDA_TRY(cudaMalloc(&d, words * sizeof(unsigned long long)));
  Q2_CUDA_TRY(cudaMemsetAsync(d, 0, words * sizeof(unsigned long long), st));
  const int saved = M->h_len[0];
  Q2_CUDA_TRY(cudaMemcpyAsync(M->d_ids, ids, sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
  q2_status s = stream_step(M, true, true, st, false, d);
  if (s == Q2_OK) s = cudaMemcpyAsync(out, d, words * sizeof(unsigned long long), cudaMemcpyDeviceToHost, st) == cudaSuccess ? Q2_OK : Q2_ERR_CUDA;
  if (s == Q2_OK) s = cudaStreamSynchronize(st) == cudaSuccess ? Q2_OK : Q2_ERR_CUDA;
  cudaFree(d);
  // the traced step leaves the model where it was
  if (s == Q2_OK) s = cudaMemcpy(M->d_len, &saved, sizeof(int), cudaMemcpyHostToDevice) == cudaSuccess ? Q2_OK : Q2_ERR_CUDA;
  *grid = num_sms();
  if (s != Q2_OK && q2_last_error()[0] == 0) set_error("trace_stream_step: a CUDA call failed");
  return s;
}

q2_status q2_test_set_wait_fault(q2_model* M, int phase, unsigned long long deadline_ns) {
  clear_error();
  Q2_CHECK_ARG(M, Q2_ERR_INVALID_ARG, "test_set_wait_fault: NULL model");
  Q2_CHECK_ARG(phase >= -1 && phase <= 5 * M->m.n_layers, Q2_ERR_INVALID_ARG,
               "test_set_wait_fault: phase outside [-1, 5 * n_layers]");
  Q2_CHECK_ARG(deadline_ns >= 1000, Q2_ERR_INVALID_ARG, "test_set_wait_fault: deadline below 1 us");
  DeviceGuard g(M->device);
  cudaDeviceSynchronize();
  // captured steps hold the old settings: drop them
  for (auto& kv : M->graphs) cudaGraphExecDestroy(kv.second);
  M->graphs.clear();
  M->stall_phase = phase;
  M->wait_ns = phase < 0 ? 200ull * 1000 * 1000 : deadline_ns;
  return Q2_OK;
}

q2_status q2_model_set_graphs(q2_model* M, int enable) {
  clear_error();
  Q2_CHECK_ARG(M, Q2_ERR_INVALID_ARG, "set_graphs: NULL model");
  M->use_graphs = enable != 0;
  return Q2_OK;
}

q2_status q2_model_time_kernels(q2_model* M, const int64_t* ids, int B, int steps, float* mean_ms,
                                int* per_step, int* kernels_per_step, void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && ids && mean_ms && per_step && kernels_per_step, Q2_ERR_INVALID_ARG,
               "time_kernels: NULL argument");
  Q2_CHECK_ARG(B >= 1 && B <= M->m.max_batch, Q2_ERR_CAPACITY, "time_kernels: batch outside [1, max_batch]");
  Q2_CHECK_ARG(steps >= 1, Q2_ERR_INVALID_ARG, "time_kernels: steps must be positive");
  for (int b = 0; b < B; ++b)
    Q2_CHECK_ARG(M->h_len[b] + steps <= M->m.max_seq, Q2_ERR_CAPACITY,
                 "time_kernels: a sequence would pass max_seq");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  if (use_stream(M, B) || use_persistent(M, B)) {
    // One kernel per step: per-phase critical-path times from the kernel's
    // own global-timer stamps (latest end of a phase minus the latest end of
    // the phase before), and the whole launch by CUDA events.
    const int L = M->m.n_layers, nph = 5 * L + 1;
    std::vector<int> saved(M->h_len.begin(), M->h_len.begin() + B);
    std::vector<double> sum(Q2_K_COUNT, 0.0);
    std::vector<int> cnt(Q2_K_COUNT, 0);
    std::vector<unsigned long long> tr((size_t)nph * 4);
    const int cls[6] = {Q2_K_QKV, Q2_K_ATTN, Q2_K_O, Q2_K_GATE_UP, Q2_K_DOWN, Q2_K_LM_HEAD};
    cudaEvent_t e0, e1;
    Q2_CUDA_TRY(cudaEventCreate(&e0));
    Q2_CUDA_TRY(cudaEventCreate(&e1));
    for (int r = 0; r < steps; ++r) {
      Q2_CUDA_TRY(cudaMemcpyAsync(M->d_ids, ids, B * sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
      Q2_CUDA_TRY(cudaEventRecord(e0, st));
      if (use_stream(M, B))
        Q2_TRY(stream_step(M, true, true, st, true));
      else
        Q2_TRY(persistent_step(M, B, true, true, st, true));
      Q2_CUDA_TRY(cudaEventRecord(e1, st));
      Q2_CUDA_TRY(cudaStreamSynchronize(st));
      float ms = 0.f;
      Q2_CUDA_TRY(cudaEventElapsedTime(&ms, e0, e1));
      sum[Q2_K_STEP] += ms;
      Q2_CUDA_TRY(cudaMemcpy(tr.data(), M->d_trace, tr.size() * sizeof(unsigned long long),
                             cudaMemcpyDeviceToHost));
      for (int ph = 0; ph < nph; ++ph) {
        const unsigned long long end = tr[ph * 4 + 0];
        const unsigned long long prev = ph == 0 ? tr[1] : tr[(ph - 1) * 4 + 0];
        const int kind = ph == 5 * L ? 5 : ph % 5;
        sum[cls[kind]] += (double)(end - prev) * 1e-6;  // ns -> ms
      }
      Q2_CUDA_TRY(cudaMemcpy(M->d_len, saved.data(), B * sizeof(int), cudaMemcpyHostToDevice));
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cnt[Q2_K_QKV] = cnt[Q2_K_ATTN] = cnt[Q2_K_O] = cnt[Q2_K_GATE_UP] = cnt[Q2_K_DOWN] = L;
    cnt[Q2_K_LM_HEAD] = 1;
    cnt[Q2_K_STEP] = 1;
    for (int c = 0; c < Q2_K_COUNT; ++c) {
      per_step[c] = cnt[c];
      mean_ms[c] = cnt[c] ? (float)(sum[c] / ((double)cnt[c] * steps)) : 0.f;
    }
    *kernels_per_step = 1;
    return Q2_OK;
  }
  KTiming* t = nullptr;
  auto it = M->timed.find(B);
  if (it == M->timed.end()) {
    t = new KTiming();
    M->tm = t;
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamBeginCapture(M->cap, cudaStreamCaptureModeThreadLocal);
    q2_status s = e == cudaSuccess ? decode_body(M, B, M->cap) : Q2_ERR_CUDA;
    if (e == cudaSuccess) e = cudaStreamEndCapture(M->cap, &graph);
    M->tm = nullptr;
    if (s == Q2_OK && e == cudaSuccess) {
      size_t n = 0;
      cudaGraphGetNodes(graph, nullptr, &n);
      std::vector<cudaGraphNode_t> nodes(n);
      cudaGraphGetNodes(graph, nodes.data(), &n);
      for (auto nd : nodes) {
        cudaGraphNodeType ty;
        if (cudaGraphNodeGetType(nd, &ty) == cudaSuccess && ty == cudaGraphNodeTypeKernel) t->kernels++;
      }
      e = cudaGraphInstantiate(&t->exec, graph, 0);
    }
    if (graph) cudaGraphDestroy(graph);
    if (s != Q2_OK || e != cudaSuccess) {
      for (cudaEvent_t ev : t->ev) cudaEventDestroy(ev);
      delete t;
      if (s == Q2_OK) set_error(std::string("time_kernels: capture: ") + cudaGetErrorString(e));
      return s != Q2_OK ? s : Q2_ERR_CUDA;
    }
    M->timed[B] = t;
  } else {
    t = it->second;
  }
  std::vector<int> saved(M->h_len.begin(), M->h_len.begin() + B);
  std::vector<double> sum(Q2_K_COUNT, 0.0);
  std::vector<int> cnt(Q2_K_COUNT, 0);
  for (size_t i = 0; i < t->used; ++i) cnt[t->cls[i]]++;
  Q2_CUDA_TRY(cudaMemcpyAsync(M->d_ids, ids, B * sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
  for (int r = 0; r < steps; ++r) {
    Q2_CUDA_TRY(cudaGraphLaunch(t->exec, st));
    Q2_CUDA_TRY(cudaStreamSynchronize(st));
    for (size_t i = 0; i < t->used; ++i) {
      float ms = 0.f;
      Q2_CUDA_TRY(cudaEventElapsedTime(&ms, t->ev[2 * i], t->ev[2 * i + 1]));
      sum[t->cls[i]] += ms;
    }
  }
  Q2_CUDA_TRY(cudaMemcpy(M->d_len, saved.data(), B * sizeof(int), cudaMemcpyHostToDevice));
  for (int c = 0; c < Q2_K_COUNT; ++c) {
    per_step[c] = cnt[c];
    mean_ms[c] = cnt[c] ? (float)(sum[c] / ((double)cnt[c] * steps)) : 0.f;
  }
  *kernels_per_step = t->kernels;
  return Q2_OK;
}

q2_status q2_model_prefill_hidden(q2_model* M, int seq, const void* x_in, int T, void* x_out,
                                  void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && x_in && x_out, Q2_ERR_INVALID_ARG, "prefill_hidden: NULL argument");
  Q2_CHECK_ARG(seq >= 0 && seq < M->m.max_batch, Q2_ERR_INVALID_ARG, "prefill_hidden: bad sequence");
  Q2_CHECK_ARG(T >= 1, Q2_ERR_INVALID_ARG, "prefill_hidden: T must be positive");
  Q2_CHECK_ARG((long long)M->h_len[seq] + T <= M->m.max_seq, Q2_ERR_CAPACITY,
               "prefill_hidden: the sequence would pass max_seq");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  const size_t row = (size_t)M->m.hidden * M->es;
  for (int c = 0; c < T; c += M->chunk) {
    const int Tc = T - c < M->chunk ? T - c : M->chunk;
    const int pos0 = M->h_len[seq];
    Q2_CUDA_TRY(cudaMemcpyAsync(M->x, (const char*)x_in + c * row, Tc * row, cudaMemcpyDeviceToDevice, st));
    Q2_TRY(run_layers(M, Tc, 0, seq, pos0, st, true));
    Q2_CUDA_TRY(cudaMemcpyAsync((char*)x_out + c * row, M->x, Tc * row, cudaMemcpyDeviceToDevice, st));
    M->h_len[seq] = pos0 + Tc;
    Q2_LAUNCH(set_len_kernel, dim3(1), dim3(1), 0, st, true, M->d_len, seq, pos0 + Tc);
  }
  return Q2_OK;
}

q2_status q2_model_head(q2_model* M, const void* x, int rows, int64_t* next, float* logits,
                        void* stream) {
  clear_error();
  Q2_CHECK_ARG(M && x && next, Q2_ERR_INVALID_ARG, "head: NULL argument");
  Q2_CHECK_ARG(rows >= 1 && rows <= M->m.max_batch, Q2_ERR_CAPACITY, "head: rows outside [1, max_batch]");
  DeviceGuard g(M->device);
  cudaStream_t st = as_stream(stream);
  Q2_TRY(check_stream_device(M, st));
  Q2_CUDA_TRY(cudaMemcpyAsync(M->x, x, (size_t)rows * M->m.hidden * M->es, cudaMemcpyDeviceToDevice, st));
  Q2_TRY(run_head(M, 0, rows, 0, st, true, false));
  Q2_CUDA_TRY(cudaMemcpyAsync(next, M->d_next, rows * sizeof(int64_t), cudaMemcpyDeviceToDevice, st));
  if (logits)
    Q2_CUDA_TRY(cudaMemcpyAsync(logits, M->logits, (size_t)rows * M->m.vocab * sizeof(float),
                                cudaMemcpyDeviceToDevice, st));
  return Q2_OK;
}

q2_status q2_model_set_decode_path(q2_model* M, int path) {
  clear_error();
  Q2_CHECK_ARG(M, Q2_ERR_INVALID_ARG, "set_decode_path: NULL model");
  Q2_CHECK_ARG(path >= Q2_PATH_AUTO && path <= Q2_PATH_STREAM, Q2_ERR_INVALID_ARG,
               "set_decode_path: bad path");
  Q2_CHECK_ARG(path != Q2_PATH_STREAM || M->streaming, Q2_ERR_STATE,
               "set_decode_path: the streaming step does not support this model");
  Q2_CHECK_ARG(path != Q2_PATH_PERSISTENT || M->persistent, Q2_ERR_STATE,
               "set_decode_path: the persistent kernel does not support this model");
  Q2_CHECK_ARG(path != Q2_PATH_KERNELS || M->fused, Q2_ERR_STATE,
               "set_decode_path: the fused kernels do not support this model");
  if (path != M->path) {
    DeviceGuard g(M->device);
    cudaDeviceSynchronize();
    for (auto& kv : M->graphs) cudaGraphExecDestroy(kv.second);
    M->graphs.clear();
    for (auto& kv : M->timed) {
      if (kv.second->exec) cudaGraphExecDestroy(kv.second->exec);
      for (cudaEvent_t e : kv.second->ev) cudaEventDestroy(e);
      delete kv.second;
    }
    M->timed.clear();
  }
  M->path = path;
  return Q2_OK;
}

}  // extern "C"
