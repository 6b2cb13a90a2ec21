// launch.h -- internal launchers behind the C ABI (gdn_api.cu). Each enqueues its kernels
// on `stream` and returns cudaGetLastError(); arguments are validated by the caller.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr int kF32 = 0;   // GDN_F32
constexpr int kBF16 = 1;  // GDN_BF16

cudaError_t launch_conv1d_silu(int dtype, const void* x, void* y, const void* w,
                               const int32_t* cu, int32_t n_seq, int64_t T, int32_t Cc,
                               const void* conv_state_in, void* conv_state_out,
                               cudaStream_t stream);

// state_dtype: kF32, or kBF16 for bf16 state storage (fp32 arithmetic)
cudaError_t launch_decode_step(int dtype, const void* x, const void* conv_w, void* conv_state,
                               const float* g, const float* beta, void* state, int state_dtype,
                               void* o, int32_t B, int32_t Hk, int32_t Hv, int32_t d, float scale,
                               cudaStream_t stream);
// n_tok (1..8) tokens per sequence; x [B, n_tok, Cc], g/beta [B, n_tok, Hv], o [B, n_tok, Hv, d]
cudaError_t launch_decode_tokens(int dtype, const void* x, const void* conv_w, void* conv_state,
                                 const float* g, const float* beta, void* state, int state_dtype,
                                 void* o, int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv, int32_t d,
                                 float scale, cudaStream_t stream);

// States at block boundaries (prefix caching): after every block_tokens tokens of a sequence
// (block_tokens a positive multiple of 64; 0 = none), its state goes to row
// block_rows[n] + m - 1 of block_states [n_block_rows, Hv, dv, dk] (the state dtype of the
// call) for the m-th boundary; rows outside [0, n_block_rows) are skipped.
struct BlockStates {
  int32_t block_tokens = 0;
  void* states = nullptr;
  const int32_t* rows = nullptr;
  int64_t n_rows = 0;
};

// Token-by-token fp32 recurrence (SIMT): the fp32-activation prefill path. States (initial,
// final, block) are stored as state_dtype (kF32, or kBF16 storage with fp32 math).
cudaError_t launch_prefill_recurrent(int dtype, const void* q, const void* k, const void* v,
                                     const float* g, const float* beta, void* o, int64_t T,
                                     int32_t Hk, int32_t Hv, int32_t d, int64_t qk_stride,
                                     int64_t v_stride, const int32_t* cu, int32_t n_seq,
                                     const void* init, void* final_state, int state_dtype,
                                     float scale, int32_t l2norm, BlockStates blocks,
                                     cudaStream_t stream);

// Chunked WY/UT prefill on tcgen05 (bf16 activations, dk = dv = 128, at most
// kPrefillTcMaxG value heads per key head). Needs
// prefill_chunk_tc_workspace(...) bytes of workspace.
constexpr int kPrefillTcMaxG = 8;
size_t prefill_chunk_tc_workspace(int64_t T, int32_t n_seq, int32_t Hv);
// The workspace's first int: 0, or the code of a bounded wait that gave up in the last call.
const char* prefill_chunk_tc_error_string(int code);
int prefill_chunk_tc_launches(int64_t T, int32_t n_seq, int32_t Hv, int num_sms);
cudaError_t launch_prefill_chunk_tc(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, void* o, int64_t T, int32_t Hk, int32_t Hv,
                                    int64_t qk_stride, int64_t v_stride, const int32_t* cu,
                                    int32_t n_seq, const void* init, void* fin, int state_dtype,
                                    float scale, BlockStates blocks, void* workspace,
                                    cudaStream_t stream);

// Workspace bytes the prefill path chosen for these arguments needs (0 for the
// token-recurrent path, which takes no workspace); SIZE_MAX for unsupported shapes.
size_t prefill_workspace_need(gdn_dtype_t dt, int64_t T, int32_t n_seq, int32_t Hk, int32_t Hv,
                              int32_t dk, int32_t dv, int32_t qk_l2norm);

// Records the calling thread's gdn_last_error() text and returns s.
gdn_status_t set_error(gdn_status_t s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));

}  // namespace gdn
