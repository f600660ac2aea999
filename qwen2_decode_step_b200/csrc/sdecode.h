// sdecode.h -- the batch-1 streaming decode step: one cooperative launch, one
// CTA per SM, runs a whole greedy decode step of one sequence (or the decoder
// layers alone).
//
// At batch 1 every linear is a matrix-vector product, so the step is bound by
// reading the weights once (3.09 GB for the Qwen2-1.5B shape).  What keeps a
// step from that bound is not the streaming itself but the fixed cost of each
// dependency: the layer is a chain of five all-to-all steps (q/k/v, attention,
// o, gate/up, down), each needing the whole output of the one before.  The
// kernel therefore decouples the two:
//
//  * a producer warp per CTA streams this CTA's rows of every weight matrix
//    of the step -- layer by layer q/k/v, o, gate/up, down, then the lm_head
//    -- through a ring of shared-memory slots (one bulk copy per slot of
//    whole rows).  It waits only for free slots, never for a phase, so the
//    weights of the next phases are already landing while the grid waits at a
//    phase boundary or runs attention;
//  * eight consumer warps run the phases in order, separated by grid-wide
//    counters.  Each warp keeps the phase's input vector in registers (for
//    the RMSNorm phases it normalises the whole vector itself: no block-level
//    reduction), takes whole rows of a slot (rows of K = hidden) or a column
//    slice of a row (the down rows), and parks the row results in shared
//    memory; the phase's epilogue (bias + RoPE + KV append, residual add,
//    SwiGLU, logits + argmax) runs once at the phase end from there.
//
// Phases (l = layer):
//   QKV(l)  RMSNorm (layer 0: embedding gather) -> q/k/v rows, bias, RoPE,
//           q out, K/V appended to the cache
//   ATTN(l) split attention over the cache (K/V tiles by TMA), the splits of a
//           kv head merged by the last of its CTAs
//   O(l)    o rows, residual add
//   GU(l)   RMSNorm -> gate/up row pairs, SwiGLU
//   DOWN(l) down rows (each split over the warps by columns), residual add
//   HEAD    final RMSNorm -> lm_head rows, fp32 logits, argmax (the last
//           arrival reduces the CTAs' partials and advances the length)
// Every wait is bounded by a deadline on the global timer; a wait that runs
// out sets bit 1 (value 2) of the error word and the step carries on (its
// results are then undefined), so a broken dependency cannot hang the GPU.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/q2.h"
#include "pdecode.h"  // PLayer

namespace q2 {

struct SDecode {
  const PLayer* layers;  // device array [L]
  int L, H, I, V, nh, nkv, hd, qkvd, qd;
  int max_seq, Bmax, nsplit;
  float eps, scale;
  int embed_in;          // 1: layer 0 reads the id's embedding row; 0: x holds the input
  int run_head;          // 1: final norm + lm_head + argmax; 0: stop after the layers
  const void* embed;
  const void* lm_head;
  const void* final_norm;
  const int64_t* ids;    // [1]
  void* x;               // residual stream [H] (bf16), sequence 0
  void* qb;              // [qd] rotated q
  void* att;             // [qd] merged attention output
  void* s;               // [I] SwiGLU output
  void* kc;              // K / V cache [L][Bmax][nkv][max_seq][hd]
  void* vc;
  long long kv_layer_stride;
  const float2* rope;    // [max_seq][hd/2]
  int* lens;             // [Bmax]; sequence 0's length = the new token's position
  float* part_o;         // [nh][nsplit][hd]
  float* part_ml;        // [nh][nsplit][2]
  float* logits;         // [V]
  float* am_val;         // [grid]
  int64_t* am_idx;       // [grid]
  int64_t* next;         // [1]
  unsigned* sync;        // [sdecode_sync_words(L, nkv)], zero at launch
  unsigned long long* trace;  // optional [5L + 1][4] phase timestamps
  unsigned long long* ctrace;  // optional [5L + 1][grid][4] per-CTA timestamps: phase entered,
                               // previous phase seen complete, stages consumed, arrival
  int* err;              // bit 0 (1): id outside the vocabulary; bit 1 (2): a wait ran out
  int ring;              // weight ring slots
  int l2_ahead;          // weight slots the producer pulls into L2 ahead of the ring (0: none)
  unsigned long long deadline_ns;  // bound of every wait
  int stall_phase;       // test hook: the counter of this phase needs one arrival more than
                         // the grid makes, so its waits run out (-1: none)
};

bool sdecode_supported(int H, int I, int V, int nh, int nkv, int hd, int qkvd, int qd);
// phase counters, per (layer, kv head) merge tickets, and one word a wait
// that ran out sets so the launch's other grid waits give up at once
size_t sdecode_sync_words(int L, int nkv);
int sdecode_default_ring();
q2_status launch_sdecode(const SDecode& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                         cudaStream_t st);

}  // namespace q2
