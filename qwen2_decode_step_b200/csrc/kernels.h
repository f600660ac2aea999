// kernels.h -- internal launchers shared by the C-ABI entry points and the
// model runtime.  Every launcher enqueues on `st` and returns a status; none
// synchronises.  `pdl` requests programmatic dependent launch (the kernel
// then waits for its predecessor with griddepcontrol.wait before touching
// any activation).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/q2.h"

namespace q2 {

size_t dtype_size(int dtype);

q2_status launch_add(void* c, const void* a, const void* b, size_t n, int dtype, cudaStream_t st);
q2_status launch_swiglu(void* out, const void* gate, const void* up, size_t n, int dtype,
                        cudaStream_t st);
// out[t, i] = silu(gate_up[t, 2i]) * gate_up[t, 2i+1]; rows of stride 2I.
q2_status launch_swiglu_interleaved(void* out, const void* gate_up, int T, int I, int dtype,
                                    cudaStream_t st, bool pdl);
q2_status launch_embedding(void* out, const int64_t* ids, const void* table, size_t ntok,
                           size_t vocab, size_t d, int dtype, int* err_flag, cudaStream_t st,
                           bool pdl);
// residual += y (rounded; y may be NULL), h = rms_norm(residual) * w.  h may be NULL
// (then only the add happens).
q2_status launch_add_rms_norm(void* residual, const void* y, void* h, const void* w, size_t M,
                              size_t d, float eps, int dtype, cudaStream_t st, bool pdl);
q2_status launch_rms_norm(void* out, const void* in, const void* w, size_t M, size_t d, float eps,
                          int dtype, cudaStream_t st);
q2_status launch_rope(void* out, const void* in, const int64_t* pos, size_t ntok, size_t nhead,
                      size_t hd, float theta, int dtype, cudaStream_t st);
q2_status launch_rearrange(void* out, const void* in, int ndim, const int64_t* shape,
                           const int64_t* out_strides, const int64_t* in_strides, size_t elem_size,
                           cudaStream_t st);
// Two-pass argmax.  part_val/part_idx hold rows * parts partials (parts from
// argmax_parts()).
int argmax_parts(size_t rows, size_t n);
q2_status launch_argmax(int64_t* idx, void* val, const void* x, size_t rows, size_t n, int dtype,
                        float* part_val, int64_t* part_idx, int parts, cudaStream_t st, bool pdl);

// ------------------------------------------------------------------ linear
// out[M, N] (out_dtype) = in[M, K] . W[N, K]^T + b (dtype).
q2_status launch_linear(void* out, const void* in, const void* w, const void* b, int M, int N,
                        int K, int dtype, int out_dtype, cudaStream_t st, bool pdl);

// --------------------------------------------------------------- attention
struct AttnRows {
  const void* q;
  long long q_row_stride;  // elements between query rows
  const void* k;
  const void* v;
  long long kv_seq_stride;   // elements between sequences
  long long kv_tok_stride;   // elements between positions
  long long kv_head_stride;  // elements between kv heads
  void* out;
  long long out_row_stride;
  int rows, nh, nkv, hd;
  // visible keys of query row r: base + row_step * r + (lens ? lens[seq(r)] : 0),
  // with seq(r) = seq_is_row ? r : fixed_seq.
  int base, row_step;
  const int* lens;
  int seq_is_row, fixed_seq;
  float scale;
};
// Split count for a given problem (decode: enough CTAs for the machine).
int attn_splits(int rows, int nkv, int max_keys);
size_t attn_scratch_bytes(int rows, int nh, int hd, int nsplit);
// tc_ws: the tensor-core path's work-split scratch (attn_tc_ws_bytes(), its
// first 4 KB zero before the first call; the path leaves it zero), or null
// (then every item runs whole).
q2_status launch_attention(const AttnRows& a, int nsplit, void* scratch, int dtype,
                           cudaStream_t st, bool pdl, int* err = nullptr, void* tc_ws = nullptr);
// Rows of one sequence (prefill), bf16, head dim 128: flash-attention on the
// tensor cores (launch_attention takes it by itself when it applies).
bool attn_prefill_mma_supported(const AttnRows& a, int dtype);
q2_status launch_attn_prefill_mma(const AttnRows& a, cudaStream_t st, bool pdl);
// The same on the sm_100a tensor cores (tcgen05, TMEM accumulators): K/V
// head-major or token-major, head dim 128, bf16.  A bounded wait that runs
// out sets value 2 in *err.  launch_attention takes it when it applies.
bool attn_tc_supported(const AttnRows& a, int dtype);
int prefill_attn_impl();
size_t attn_tc_ws_bytes();
// Its work plan (host only; `sms` the machine's SM count): of the
// ceil(rows / 128) * nh items (128 query rows of one head), the first
// *n_whole run whole, one CTA each, and each later item as *ts key ranges;
// with !split_ok (no scratch) every item runs whole.  The scratch holds
// attn_tc_slot_capacity(sms) ranges and attn_tc_counter_capacity() items.
void attn_tc_plan(int rows, int pos0, int nh, int sms, bool split_ok, int* n_whole, int* ts);
int attn_tc_slot_capacity(int sms);
int attn_tc_counter_capacity();
q2_status launch_attn_tc(const AttnRows& a, void* ws, int* err, cudaStream_t st);

}  // namespace q2
