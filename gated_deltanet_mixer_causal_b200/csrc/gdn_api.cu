// gdn_api.cu -- the extern "C" boundary of libgdn.so (declared in include/gdn.h).
//
// Every entry point validates its arguments on the host before launching anything,
// returns a status code, never prints and never throws. Work is enqueued on the caller's
// stream; the library allocates no device memory.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "gdn.h"
#include "launch.h"

namespace {

thread_local char g_last_error[256] = "";

gdn_status_t fail(gdn_status_t s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
gdn_status_t fail(gdn_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

gdn_status_t ok() {
  g_last_error[0] = '\0';
  return GDN_OK;
}

gdn_status_t cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(GDN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// [a, a + na) and [b, b + nb) share a byte (null or empty ranges never overlap).
bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + nb && y < x + na;
}

size_t elt_size(gdn_dtype_t dt) { return dt == GDN_F32 ? 4 : 2; }

bool valid_dtype(gdn_dtype_t dt) { return dt == GDN_F32 || dt == GDN_BF16; }

bool supported_head_dim(int32_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// bf16 activations with 128-wide heads (and at most 8 value heads per key head) run the
// chunked tensor-core prefill; everything else runs the token-by-token fp32 kernel.
// TMA coordinates are 32-bit: the tensor-core prefill addresses tokens and workspace rows
// (chunk slot x value head x 128) with int32, which bounds the tokens of one call.
bool tc_rows_fit(int64_t T, int32_t n_seq, int32_t Hv) {
  const int64_t slots = (T + 63) / 64 + (n_seq < 1 ? 1 : n_seq);
  return T <= 0x7fffffffLL && slots * Hv * 128 <= 0x7fffffffLL;
}

// The tensor-core prefill folds the q/k L2 norm into its factors; inputs used as given
// (qk_l2norm = 0) take the token-recurrent path.
bool use_tensor_core_prefill(gdn_dtype_t dt, int32_t d, int32_t Hk, int32_t Hv, int32_t qk_l2norm = 1) {
  return dt == GDN_BF16 && d == 128 && Hv / Hk <= gdn::kPrefillTcMaxG && qk_l2norm != 0;
}

}  // namespace

namespace gdn {

size_t prefill_workspace_need(gdn_dtype_t dt, int64_t T, int32_t n_seq, int32_t Hk, int32_t Hv,
                              int32_t dk, int32_t dv, int32_t qk_l2norm) {
  if (!valid_dtype(dt) || T < 0 || Hk <= 0 || Hv <= 0 || Hv % Hk != 0 || dk != dv ||
      !supported_head_dim(dk))
    return SIZE_MAX;
  if (n_seq < 1) n_seq = 1;
  if (!use_tensor_core_prefill(dt, dk, Hk, Hv, qk_l2norm)) return 0;
  return tc_rows_fit(T, n_seq, Hv) ? prefill_chunk_tc_workspace(T, n_seq, Hv) : SIZE_MAX;
}

gdn_status_t set_error(gdn_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

}  // namespace gdn

extern "C" {

const char* gdn_status_string(gdn_status_t s) {
  switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
  }
  return "GDN_ERR_UNKNOWN";
}

const char* gdn_last_error(void) { return g_last_error; }

const char* gdn_version(void) { return "0.1.0"; }

gdn_status_t gdn_conv1d_silu(const void* x, void* y, gdn_dtype_t dt, const void* w,
                             const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Cc,
                             const void* conv_state_in, void* conv_state_out,
                             gdn_stream_t stream) {
  if (!valid_dtype(dt)) return fail(GDN_ERR_UNSUPPORTED, "conv1d_silu: unknown dtype %d", (int)dt);
  if (T < 0) return fail(GDN_ERR_INVALID_ARG, "conv1d_silu: T = %lld < 0", (long long)T);
  if (Cc <= 0 || Cc % 8 != 0)
    return fail(GDN_ERR_INVALID_ARG, "conv1d_silu: Cc = %d must be a positive multiple of 8", Cc);
  if (cu_seqlens == nullptr) n_seq = 1;
  if (n_seq < 1 || n_seq > 65535)
    return fail(GDN_ERR_INVALID_ARG, "conv1d_silu: n_seq = %d outside [1, 65535]", n_seq);
  if (T > 0 && (x == nullptr || y == nullptr || w == nullptr))
    return fail(GDN_ERR_INVALID_ARG, "conv1d_silu: x, y and w must be non-null");
  if (!aligned16(x) || !aligned16(y) || !aligned16(w) || !aligned16(conv_state_in) ||
      !aligned16(conv_state_out))
    return fail(GDN_ERR_INVALID_ARG, "conv1d_silu: pointers must be 16-byte aligned");
  const size_t es = elt_size(dt);
  const size_t xb = (size_t)T * Cc * es, sb = (size_t)n_seq * 3 * Cc * es;
  if (overlap(x, xb, y, xb)) return fail(GDN_ERR_INVALID_ARG, "conv1d_silu: y overlaps x");
  if (overlap(conv_state_in, sb, conv_state_out, sb))
    return fail(GDN_ERR_INVALID_ARG, "conv1d_silu: conv_state_out overlaps conv_state_in");
  if (overlap(y, xb, conv_state_out, sb) || overlap(y, xb, conv_state_in, sb) ||
      overlap(x, xb, conv_state_out, sb))
    return fail(GDN_ERR_INVALID_ARG, "conv1d_silu: conv states overlap x or y");
  return cuda_status(gdn::launch_conv1d_silu((int)dt, x, y, w, cu_seqlens, n_seq, T, Cc,
                                             conv_state_in, conv_state_out, (cudaStream_t)stream),
                     "conv1d_silu launch");
}

size_t gdn_chunk_prefill_workspace_size(int64_t T, int32_t n_seq, int32_t Hk, int32_t Hv,
                                        int32_t dk, int32_t dv, gdn_dtype_t dt) {
  return gdn::prefill_workspace_need(dt, T, n_seq, Hk, Hv, dk, dv, 1);
}

int32_t gdn_chunk_prefill_path(gdn_dtype_t dt, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                               int32_t qk_l2norm) {
  if (!valid_dtype(dt) || Hk <= 0 || Hv <= 0 || Hv % Hk != 0 || dk != dv || !supported_head_dim(dk))
    return -1;
  return use_tensor_core_prefill(dt, dk, Hk, Hv, qk_l2norm) ? GDN_PATH_CHUNKED_TC : GDN_PATH_RECURRENT;
}

int32_t gdn_chunk_prefill_launches(int64_t T, int32_t n_seq, int32_t Hk, int32_t Hv, int32_t dk,
                                   int32_t dv, gdn_dtype_t dt, int32_t qk_l2norm, int32_t num_sms) {
  if (gdn_chunk_prefill_path(dt, Hk, Hv, dk, dv, qk_l2norm) < 0 || T < 0 || n_seq < 1 || num_sms < 1) return -1;
  if (!use_tensor_core_prefill(dt, dk, Hk, Hv, qk_l2norm)) return 1;
  if (!tc_rows_fit(T, n_seq, Hv)) return -1;
  return gdn::prefill_chunk_tc_launches(T, n_seq, Hv, num_sms);
}

gdn_status_t gdn_chunk_prefill_ex(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, void* o, gdn_dtype_t dt, int64_t T,
                                  int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int64_t qk_stride,
                                  int64_t v_stride, const int32_t* cu_seqlens, int32_t n_seq,
                                  const void* initial_state, void* final_state,
                                  gdn_dtype_t state_dt, float scale, int32_t qk_l2norm,
                                  int32_t block_tokens, void* block_states,
                                  const int32_t* block_rows, int64_t n_block_rows, void* workspace,
                                  size_t workspace_bytes, gdn_stream_t stream) {
  if (!valid_dtype(dt)) return fail(GDN_ERR_UNSUPPORTED, "chunk_prefill: unknown dtype %d", (int)dt);
  if (!valid_dtype(state_dt))
    return fail(GDN_ERR_UNSUPPORTED, "chunk_prefill: unknown state dtype %d", (int)state_dt);
  if (T < 0) return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: T = %lld < 0", (long long)T);
  if (Hk <= 0 || Hv <= 0) return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: Hk, Hv must be > 0");
  if (Hv % Hk != 0) return fail(GDN_ERR_UNSUPPORTED, "chunk_prefill: Hv %% Hk != 0 (%d, %d)", Hv, Hk);
  if (dk != dv || !supported_head_dim(dk))
    return fail(GDN_ERR_UNSUPPORTED, "chunk_prefill: head dims dk=%d dv=%d (need dk = dv in {16,32,64,128})", dk, dv);
  if (cu_seqlens == nullptr) n_seq = 1;
  if (n_seq < 1) return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: n_seq = %d < 1", n_seq);
  if (qk_stride == 0) qk_stride = (int64_t)Hk * dk;
  if (v_stride == 0) v_stride = (int64_t)Hv * dv;
  if (qk_stride < (int64_t)Hk * dk || v_stride < (int64_t)Hv * dv || qk_stride % 8 != 0 ||
      v_stride % 8 != 0)
    return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: strides (%lld, %lld) must cover a token row and be multiples of 8",
                (long long)qk_stride, (long long)v_stride);
  if (T > 0 && (!q || !k || !v || !g || !beta || !o))
    return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: q, k, v, g, beta, o must be non-null");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) ||
      !aligned16(o) || !aligned16(initial_state) || !aligned16(final_state))
    return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: pointers must be 16-byte aligned");
  const size_t es = elt_size(dt);
  const size_t ob = (size_t)T * Hv * dv * es;
  const size_t qkb = T > 0 ? ((size_t)(T - 1) * qk_stride + (size_t)Hk * dk) * es : 0;
  const size_t vb = T > 0 ? ((size_t)(T - 1) * v_stride + (size_t)Hv * dv) * es : 0;
  const size_t sts = elt_size(state_dt);
  const size_t gb = (size_t)T * Hv * 4, stb = (size_t)n_seq * Hv * dv * dk * sts;
  if (overlap(o, ob, q, qkb) || overlap(o, ob, k, qkb) || overlap(o, ob, v, vb) ||
      overlap(o, ob, g, gb) || overlap(o, ob, beta, gb) || overlap(o, ob, initial_state, stb) ||
      overlap(o, ob, final_state, stb))
    return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: o overlaps an input or a state");
  if (final_state != initial_state && overlap(initial_state, stb, final_state, stb))
    return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: final_state partially overlaps initial_state");
  gdn::BlockStates blocks;
  if (block_tokens < 0 || block_tokens % 64 != 0)
    return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: block_tokens = %d must be 0 or a positive multiple of 64",
                block_tokens);
  if (block_tokens > 0) {
    if (!block_states || !block_rows || n_block_rows < 1)
      return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: block states need block_states, block_rows and n_block_rows >= 1");
    if (!aligned16(block_states))
      return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: block_states must be 16-byte aligned");
    const size_t bsb = (size_t)n_block_rows * Hv * dv * dk * sts;
    if (overlap(block_states, bsb, q, qkb) || overlap(block_states, bsb, k, qkb) ||
        overlap(block_states, bsb, v, vb) || overlap(block_states, bsb, g, gb) ||
        overlap(block_states, bsb, beta, gb) || overlap(block_states, bsb, o, ob) ||
        overlap(block_states, bsb, initial_state, stb) || overlap(block_states, bsb, final_state, stb) ||
        overlap(block_states, bsb, block_rows, (size_t)n_seq * 4))
      return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: block_states overlaps another buffer");
    blocks.block_tokens = block_tokens;
    blocks.states = block_states;
    blocks.rows = block_rows;
    blocks.n_rows = n_block_rows;
  }
  const bool tensor_core = use_tensor_core_prefill(dt, dk, Hk, Hv, qk_l2norm);
  if (tensor_core && !tc_rows_fit(T, n_seq, Hv))
    return fail(GDN_ERR_UNSUPPORTED, "chunk_prefill: %lld tokens of %d value heads exceed the 32-bit "
                "TMA coordinates of one call; split the batch", (long long)T, Hv);
  const size_t need = tensor_core ? gdn::prefill_chunk_tc_workspace(T, n_seq, Hv) : 0;
  if (workspace_bytes < need || (need > 0 && workspace == nullptr))
    return fail(GDN_ERR_WORKSPACE, "chunk_prefill: workspace %zu bytes < %zu needed", workspace_bytes, need);
  if (T == 0 && final_state == nullptr) return ok();
  if (tensor_core) {
    if (!aligned16(workspace) || ((uintptr_t)workspace & 255u) != 0)
      return fail(GDN_ERR_INVALID_ARG, "chunk_prefill: workspace must be 256-byte aligned");
    return cuda_status(gdn::launch_prefill_chunk_tc(q, k, v, g, beta, o, T, Hk, Hv, qk_stride, v_stride,
                                                    cu_seqlens, n_seq, initial_state, final_state,
                                                    (int)state_dt, scale, blocks, workspace,
                                                    (cudaStream_t)stream),
                       "chunk_prefill (tensor-core) launch");
  }
  if (workspace != nullptr && workspace_bytes >= sizeof(int)) {   // no wait can fail here
    const cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e, "chunk_prefill: clearing the status word");
  }
  return cuda_status(gdn::launch_prefill_recurrent((int)dt, q, k, v, g, beta, o, T, Hk, Hv, dk,
                                                   qk_stride, v_stride, cu_seqlens, n_seq,
                                                   initial_state, final_state, (int)state_dt, scale,
                                                   qk_l2norm, blocks, (cudaStream_t)stream),
                     "chunk_prefill launch");
}

gdn_status_t gdn_prefill_status(const void* workspace, gdn_stream_t stream) {
  if (workspace == nullptr) return fail(GDN_ERR_INVALID_ARG, "prefill_status: workspace is NULL");
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost,
                                  (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "prefill_status");
  if (word == 0) return ok();
  return fail(GDN_ERR_TIMEOUT, "prefill_status: a bounded device-side wait gave up (%s, code %d); "
              "the outputs of that call are invalid", gdn::prefill_chunk_tc_error_string(word), word);
}

gdn_status_t gdn_chunk_prefill(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, void* o, gdn_dtype_t dt, int64_t T,
                               int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, int64_t qk_stride,
                               int64_t v_stride, const int32_t* cu_seqlens, int32_t n_seq,
                               const float* initial_state, float* final_state, float scale,
                               int32_t qk_l2norm, void* workspace, size_t workspace_bytes,
                               gdn_stream_t stream) {
  return gdn_chunk_prefill_ex(q, k, v, g, beta, o, dt, T, Hk, Hv, dk, dv, qk_stride, v_stride,
                              cu_seqlens, n_seq, initial_state, final_state, GDN_F32, scale,
                              qk_l2norm, 0, nullptr, nullptr, 0, workspace, workspace_bytes, stream);
}

gdn_status_t gdn_decode_step_ex(const void* x, const void* conv_w, void* conv_state, const float* g,
                                const float* beta, void* state, gdn_dtype_t state_dt, void* o,
                                gdn_dtype_t dt, int32_t B, int32_t Hk, int32_t Hv, int32_t dk,
                                int32_t dv, float scale, gdn_stream_t stream) {
  if (!valid_dtype(dt)) return fail(GDN_ERR_UNSUPPORTED, "decode_step: unknown dtype %d", (int)dt);
  if (!valid_dtype(state_dt)) return fail(GDN_ERR_UNSUPPORTED, "decode_step: unknown state dtype %d", (int)state_dt);
  if (B < 0) return fail(GDN_ERR_INVALID_ARG, "decode_step: B = %d < 0", B);
  if (Hk <= 0 || Hv <= 0) return fail(GDN_ERR_INVALID_ARG, "decode_step: Hk, Hv must be > 0");
  if (Hv % Hk != 0) return fail(GDN_ERR_UNSUPPORTED, "decode_step: Hv %% Hk != 0 (%d, %d)", Hv, Hk);
  if (dk != dv || !supported_head_dim(dk))
    return fail(GDN_ERR_UNSUPPORTED, "decode_step: head dims dk=%d dv=%d (need dk = dv in {16,32,64,128})", dk, dv);
  if ((int64_t)B * Hk > 0x7fffffffLL) return fail(GDN_ERR_INVALID_ARG, "decode_step: B * Hk too large");
  if (B == 0) return ok();
  if (!x || !conv_w || !conv_state || !g || !beta || !state || !o)
    return fail(GDN_ERR_INVALID_ARG, "decode_step: all pointers must be non-null");
  if (!aligned16(x) || !aligned16(conv_w) || !aligned16(conv_state) || !aligned16(g) ||
      !aligned16(beta) || !aligned16(state) || !aligned16(o))
    return fail(GDN_ERR_INVALID_ARG, "decode_step: pointers must be 16-byte aligned");
  const size_t es = elt_size(dt);
  const int64_t Cc = 2LL * Hk * dk + (int64_t)Hv * dv;
  const size_t xb = (size_t)B * Cc * es, csb = (size_t)B * 3 * Cc * es;
  const size_t stb = (size_t)B * Hv * dv * dk * elt_size(state_dt), ob = (size_t)B * Hv * dv * es;
  const size_t gb = (size_t)B * Hv * 4, wb = (size_t)Cc * 4 * es;
  const void* ro[4] = {x, conv_w, g, beta};
  const size_t rob[4] = {xb, wb, gb, gb};
  for (int i = 0; i < 4; ++i)
    if (overlap(ro[i], rob[i], conv_state, csb) || overlap(ro[i], rob[i], state, stb) ||
        overlap(ro[i], rob[i], o, ob))
      return fail(GDN_ERR_INVALID_ARG, "decode_step: an output overlaps an input");
  if (overlap(conv_state, csb, state, stb) || overlap(conv_state, csb, o, ob) ||
      overlap(state, stb, o, ob))
    return fail(GDN_ERR_INVALID_ARG, "decode_step: conv_state, state and o must not overlap");
  return cuda_status(gdn::launch_decode_step((int)dt, x, conv_w, conv_state, g, beta, state,
                                             (int)state_dt, o, B, Hk, Hv, dk, scale,
                                             (cudaStream_t)stream),
                     "decode_step launch");
}

gdn_status_t gdn_decode_step(const void* x, const void* conv_w, void* conv_state, const float* g,
                             const float* beta, float* state, void* o, gdn_dtype_t dt, int32_t B,
                             int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, float scale,
                             gdn_stream_t stream) {
  return gdn_decode_step_ex(x, conv_w, conv_state, g, beta, state, GDN_F32, o, dt, B, Hk, Hv, dk,
                            dv, scale, stream);
}

gdn_status_t gdn_decode_tokens_ex(const void* x, const void* conv_w, void* conv_state, const float* g,
                                  const float* beta, void* state, gdn_dtype_t state_dt, void* o,
                                  gdn_dtype_t dt, int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv,
                                  int32_t dk, int32_t dv, float scale, gdn_stream_t stream) {
  if (!valid_dtype(dt)) return fail(GDN_ERR_UNSUPPORTED, "decode_tokens: unknown dtype %d", (int)dt);
  if (!valid_dtype(state_dt)) return fail(GDN_ERR_UNSUPPORTED, "decode_tokens: unknown state dtype %d", (int)state_dt);
  if (B < 0) return fail(GDN_ERR_INVALID_ARG, "decode_tokens: B = %d < 0", B);
  if (n_tok < 1 || n_tok > 8) return fail(GDN_ERR_INVALID_ARG, "decode_tokens: n_tok = %d outside [1, 8]", n_tok);
  if (Hk <= 0 || Hv <= 0) return fail(GDN_ERR_INVALID_ARG, "decode_tokens: Hk, Hv must be > 0");
  if (Hv % Hk != 0) return fail(GDN_ERR_UNSUPPORTED, "decode_tokens: Hv %% Hk != 0 (%d, %d)", Hv, Hk);
  if (dk != dv || !supported_head_dim(dk))
    return fail(GDN_ERR_UNSUPPORTED, "decode_tokens: head dims dk=%d dv=%d (need dk = dv in {16,32,64,128})", dk, dv);
  const int64_t G = Hv / Hk;
  if ((int64_t)n_tok * ((2 + G) * dk + G * dk + 1) * 4 > 227 * 1024)
    return fail(GDN_ERR_UNSUPPORTED, "decode_tokens: %d tokens of %lld value heads per key head exceed shared memory",
                n_tok, (long long)G);
  if ((int64_t)B * Hk > 0x7fffffffLL) return fail(GDN_ERR_INVALID_ARG, "decode_tokens: B * Hk too large");
  if (B == 0) return ok();
  if (!x || !conv_w || !conv_state || !g || !beta || !state || !o)
    return fail(GDN_ERR_INVALID_ARG, "decode_tokens: all pointers must be non-null");
  if (!aligned16(x) || !aligned16(conv_w) || !aligned16(conv_state) || !aligned16(g) ||
      !aligned16(beta) || !aligned16(state) || !aligned16(o))
    return fail(GDN_ERR_INVALID_ARG, "decode_tokens: pointers must be 16-byte aligned");
  const size_t es = elt_size(dt);
  const int64_t Cc = 2LL * Hk * dk + (int64_t)Hv * dv;
  const size_t xb = (size_t)B * n_tok * Cc * es, csb = (size_t)B * 3 * Cc * es;
  const size_t stb = (size_t)B * Hv * dv * dk * elt_size(state_dt), ob = (size_t)B * n_tok * Hv * dv * es;
  const size_t gb = (size_t)B * n_tok * Hv * 4, wb = (size_t)Cc * 4 * es;
  const void* ro[4] = {x, conv_w, g, beta};
  const size_t rob[4] = {xb, wb, gb, gb};
  for (int i = 0; i < 4; ++i)
    if (overlap(ro[i], rob[i], conv_state, csb) || overlap(ro[i], rob[i], state, stb) ||
        overlap(ro[i], rob[i], o, ob))
      return fail(GDN_ERR_INVALID_ARG, "decode_tokens: an output overlaps an input");
  if (overlap(conv_state, csb, state, stb) || overlap(conv_state, csb, o, ob) ||
      overlap(state, stb, o, ob))
    return fail(GDN_ERR_INVALID_ARG, "decode_tokens: conv_state, state and o must not overlap");
  return cuda_status(gdn::launch_decode_tokens((int)dt, x, conv_w, conv_state, g, beta, state,
                                               (int)state_dt, o, B, n_tok, Hk, Hv, dk, scale,
                                               (cudaStream_t)stream),
                     "decode_tokens launch");
}

gdn_status_t gdn_decode_tokens(const void* x, const void* conv_w, void* conv_state, const float* g,
                               const float* beta, float* state, void* o, gdn_dtype_t dt, int32_t B,
                               int32_t n_tok, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                               float scale, gdn_stream_t stream) {
  return gdn_decode_tokens_ex(x, conv_w, conv_state, g, beta, state, GDN_F32, o, dt, B, n_tok, Hk,
                              Hv, dk, dv, scale, stream);
}

}  // extern "C"
