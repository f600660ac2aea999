// sdecode.h -- the batch-1 streaming decode step: one cooperative launch, one
// CTA per SM, runs a whole greedy decode step of one sequence (or the decoder
// layers alone).
//
// At batch 1 every linear is a matrix-vector product, so the step is bound by
// reading the weights once (3.09 GB for the Qwen2-1.5B shape).  What keeps a
// step from that bound is not the streaming itself but the fixed cost of each
// dependency: the layer is a chain of five all-to-all steps (q/k/v, attention,
// o, gate/up, down), each needing the whole output of the one before.  The
// kernel attacks both sides:
//
//  * a producer warp per CTA streams this CTA's rows of every weight matrix
//    of the step -- layer by layer q/k/v, o, gate/up, down, then the lm_head
//    -- through a ring of shared-memory slots (one bulk copy per slot of
//    whole rows).  It waits only for free slots, never for a phase, so the
//    weights of the next phases are already landing while the consumers wait
//    for a phase's input or run attention;
//  * the phases exchange their outputs as tagged words: every 8-byte word
//    holds 4 bytes of data and a 4-byte tag naming the step and the phase
//    that wrote it, stored with one 8-byte store.  A reader polls the words
//    it needs until each carries the tag it expects -- one store-to-load hop,
//    with no fence, no grid barrier and no counter.  (Each phase needs the
//    whole output of the previous one, so no CTA can get more than one phase
//    ahead of another; that ordering is what makes every buffer reuse safe.)
//  * eight consumer warps run the phases.  Each warp keeps the phase's input
//    vector in registers (for the RMSNorm phases it normalises the whole
//    vector itself), takes whole rows of a slot (rows of K = hidden) or a
//    column slice of a row (the down rows), and parks the row results in
//    shared memory; the phase's epilogue (bias + RoPE + KV append, residual
//    add, SwiGLU, logits + argmax) runs once at the phase end from there.
//
// Phases (l = layer):
//   QKV(l)  RMSNorm (layer 0: embedding row) -> q/k/v rows, bias, RoPE; q and
//           the new K/V row published, K/V appended to the cache
//   ATTN(l) split attention over the cache, one tile of 64 keys per CTA while
//           the splits fit (K/V tiles by TMA a layer ahead, the tile holding the
//           new position patched with the published row); each split publishes
//           its partial, and CTA G - 1 - h merges query head h's partials and
//           publishes its output
//   O(l)    o rows, residual add (x published)
//   GU(l)   RMSNorm -> gate/up row pairs, SwiGLU (s published)
//   DOWN(l) down rows (each split over the warps by columns), residual add
//   HEAD    final RMSNorm -> lm_head rows, fp32 logits, per-CTA argmax; CTA 0
//           reduces the partials, writes the token and advances the length
//           and the step counter
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

// The tagged exchange buffers (8-byte words), carved from one allocation.
struct SDecodeLL {
  uint64_t* x;     // [H / 2]        residual stream, bf16 pairs (2i, 2i + 1)
  uint64_t* q;     // [nh * hd / 2]  rotated q, head h word j = (q[j], q[j + hd/2])
  uint64_t* kv;    // [2 * nkv * hd / 2] the new K row pairs, then the new V row pairs (same pairing)
  uint64_t* att;   // [nh * hd / 2]  attention output, bf16 pairs (2i, 2i + 1)
  uint64_t* s;     // [I / 2]        SwiGLU output, bf16 pairs
  uint64_t* part;  // [nkv][split max][nh / nkv][hd + 2] fp32 split partials (o, then max, sum)
  uint64_t* am;    // [grid][2]      per-CTA argmax (value bits, index)
};
size_t sdecode_ll_words(int H, int I, int nh, int nkv, int hd, int grid);
SDecodeLL sdecode_ll_carve(uint64_t* base, int H, int I, int nh, int nkv, int hd, int grid);

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
  void* x;               // residual stream [H] (bf16), sequence 0: the input when embed_in = 0,
                         // the output of the layers at the end
  void* kc;              // K / V cache [L][Bmax][nkv][max_seq][hd]
  void* vc;
  long long kv_layer_stride;
  const float2* rope;    // [max_seq][hd/2]
  int* lens;             // [Bmax]; sequence 0's length = the new token's position
  SDecodeLL ll;          // tagged exchange buffers
  unsigned* epoch;       // step counter (tags are unique per step and phase); advanced by CTA 0
  float* logits;         // [V]
  int64_t* next;         // [1]
  unsigned* sync;        // [sdecode_sync_words()], zero at launch: [0] a wait of this launch gave up
  unsigned long long* trace;   // optional [5L + 1][4] phase timestamps
  unsigned long long* ctrace;  // optional [5L + 1][grid][4] per-CTA timestamps: phase entered,
                               // input complete, phase work done, outputs published
  int* err;              // bit 0 (1): id outside the vocabulary; bit 1 (2): a wait ran out
  int ring;              // weight ring slots
  int l2_ahead;          // weight slots the producer pulls into L2 ahead of the ring (0: none)
  unsigned long long deadline_ns;  // bound of every wait
  int stall_phase;       // test hook: the output of this phase never carries the tag its
                         // readers wait for, so their waits run out (-1: none)
};

bool sdecode_supported(int H, int I, int V, int nh, int nkv, int hd, int qkvd, int qd);
constexpr int kSDecodeSplitMax = 64;
size_t sdecode_sync_words();
// The deepest weight ring whose shared-memory plan fits for L layers (0: none).
int sdecode_max_ring(int L);
q2_status launch_sdecode(const SDecode& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                         cudaStream_t st);

}  // namespace q2
