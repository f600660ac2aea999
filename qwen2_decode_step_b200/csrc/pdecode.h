// pdecode.h -- the persistent bf16 decode step (batch <= 4): one cooperative
// launch, one CTA per SM, runs a whole decode step (or the decoder layers
// alone).
//
// Each CTA has a producer warp, kPConsumers consumer warps and an epilogue
// warp.  The producer streams this CTA's row groups of every weight matrix of
// the step -- layer by layer q/k/v, o, gate/up, down, then the lm_head --
// through one TMA ring (one bulk copy per weight row), running ahead across
// phase boundaries as far as the ring allows and pulling later stages into
// L2.  The consumers split each stage's columns and run the dot products on
// the tensor cores (mma.sync), posting per-warp partial sums; the epilogue
// warp finishes each row group (bias + RoPE + KV append, SwiGLU, residual
// add, logits + argmax).  The phases run in order, separated by grid-wide
// counters:
//   QKV(l)  RMSNorm prologue (layer 0: embedding gather), q/k/v rows
//   ATTN(l) split attention over the cache, splits merged by the last CTA
//   O(l)    o rows, residual add
//   GU(l)   RMSNorm prologue; gate/up row pairs, SwiGLU
//   DOWN(l) down rows, residual add
//   HEAD    final RMSNorm; lm_head rows, fp32 logits, argmax (the last arrival
//           reduces the CTAs' partials), lengths advanced
// Every wait is bounded (a deadline on the global timer); a wait that runs
// out sets bit 1 of the error word and the step carries on, so a broken
// dependency can never hang the GPU.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/q2.h"

namespace q2 {

struct PLayer {
  const void* in_norm;
  const void* wqkv;  // packed (RoPE partner rows adjacent)
  const void* bqkv;
  const void* wo;
  const void* post_norm;
  const void* wgu;   // packed (gate/up rows interleaved)
  const void* wd;
};

struct PDecode {
  const PLayer* layers;  // device array [L]
  int L, H, I, V, nh, nkv, hd, qkvd, qd;
  int max_seq, Bmax, B, nsplit;
  float eps, scale;
  int embed_in;          // 1: layer 0 reads ids through the embedding table; 0: x holds the input
  int run_head;          // 1: final norm + lm_head + argmax; 0: stop after the layers
  const void* embed;
  const void* lm_head;
  const void* final_norm;
  const int64_t* ids;    // [B]
  void* x;               // residual stream [Bmax][H] (bf16)
  void* qb;              // [Bmax][qd]
  void* s;               // [Bmax][I]
  void* kc;              // K / V cache [L][Bmax][nkv][max_seq][hd]
  void* vc;
  long long kv_layer_stride, kv_seq_stride;
  const float2* rope;    // [max_seq][hd/2]
  int* lens;             // [Bmax]
  float* part_o;         // [B][nh][nsplit][hd]
  float* part_ml;        // [B][nh][nsplit][2]
  float* logits;         // [B][V]
  float* am_val;         // [grid][4]
  int64_t* am_idx;
  int64_t* next;         // [B]
  void* att;             // [B][qd] merged attention output (bf16)
  unsigned* sync;        // [pdecode_sync_words(L)] phase and merge counters, zero at launch
  unsigned long long* trace;  // optional [5L + 1][4] phase timestamps (see q2_model_time_kernels)
  int* err;              // bit 0: id outside the vocabulary; bit 1: a wait ran out
  int l2_ahead;          // weight stages the producer pulls into L2 ahead of its ring
};

constexpr int kPConsumers = 8;
constexpr int kPMaxBatch = 4;

bool pdecode_supported(int H, int I, int V, int nh, int nkv, int hd, int qkvd, int qd);
size_t pdecode_sync_words(int L);  // phase counters + per (sequence, kv head) merge tickets
q2_status launch_pdecode(const PDecode& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                         cudaStream_t st);

}  // namespace q2
