// decode.h -- the fused bf16 decode-step kernels (batch <= 4).
//
// Decode GEMV ("dgemv"): every CTA streams a contiguous slice of weight rows
// through a shared-memory ring filled by TMA bulk copies; the first stages
// are issued before griddepcontrol.wait, so a kernel's weight fetch overlaps
// the tail of the kernel before it.  Fused prologue/epilogues:
//   EPI_QKV    RMSNorm prologue; bias, RoPE, q out, K/V appended to the cache
//   EPI_RESID  plain activation; residual add into the residual stream
//   EPI_SWIGLU RMSNorm prologue; SwiGLU of the interleaved gate/up rows
//   EPI_LOGITS RMSNorm prologue; fp32 logits, argmax (last CTA reduces),
//              sequence lengths advanced
// Decode attention ("dattn"): split over the keys, K/V tiles by TMA tensor
// loads (128-byte swizzle), online softmax in fp32, the split partials
// merged by the last CTA of each (sequence, kv head).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/q2.h"

namespace q2 {

enum DEpi { EPI_QKV = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_LOGITS = 3 };
constexpr int kDecodeMaxBatch = 4;

struct DGemv {
  const void* w;   // [N, K] bf16, packed (QKV: RoPE partner rows adjacent; SWIGLU: gate/up interleaved)
  int N, K, M;     // rows, reduction length, tokens (M <= kDecodeMaxBatch)
  const void* x;   // [M, K]: the activation, or the residual stream when norm_w != null
  const void* norm_w;
  float eps;
  const void* bias;  // EPI_QKV: packed bias [N]
  void* out;         // QKV: q [M, out_stride]; RESID: residual stream; SWIGLU: s [M, out_stride]
  int out_stride;
  void* kc;          // EPI_QKV: this layer's K / V cache ([Bmax][nkv][max_seq][hd])
  void* vc;
  long long kv_seq_stride;
  int max_seq;
  const float2* rope;  // [max_seq][hd/2] (cos, sin)
  const int* lens;     // current length of each sequence (its next position)
  int nh, nkv, hd;
  float* logits;       // EPI_LOGITS: [M, N] fp32
  float* am_val;       // EPI_LOGITS: per-CTA partials [grid][kDecodeMaxBatch]
  int64_t* am_idx;
  unsigned* counter;   // EPI_LOGITS: last-CTA ticket (zero between launches)
  int64_t* next;       // EPI_LOGITS: [M]
  int* lens_inc;       // EPI_LOGITS: lengths advanced by one (may be null)
  int* err;            // bit 1: a bounded wait gave up
};

bool dgemv_supported(int epi, int N, int K);
int dgemv_grid(int epi, int N, int K);
q2_status launch_dgemv(int epi, const DGemv& a, cudaStream_t st);

struct DAttn {
  const void* q;      // [B][q_stride] bf16; q heads [nh][hd] at the start of each row
  int q_stride;
  void* out;          // [B][nh*hd] bf16
  float* part_o;      // [B][nh][nsplit][hd]
  float* part_ml;     // [B][nh][nsplit][2]
  unsigned* counters; // [B][nkv], zero between launches
  const int* lens;    // length before this step's token (the new K/V sit at position lens[b])
  int B, nh, nkv, hd, nsplit, max_seq, Bmax, layer;
  float scale;
  int* err;
};

bool dattn_supported(int nh, int nkv, int hd);
q2_status launch_dattn(const DAttn& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       cudaStream_t st);
// The same attention with the dot products on the tensor cores (mma.sync):
// head dim 128, up to 8 query heads per kv head, any batch, nsplit <= 64.
bool dattn_mma_supported(int nh, int nkv, int hd, int nsplit);
q2_status launch_dattn_mma(const DAttn& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                           cudaStream_t st);

}  // namespace q2
