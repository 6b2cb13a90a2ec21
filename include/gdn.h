/*
 * gdn.h -- C ABI of libgdn.so, the B200 (sm_100a) Gated DeltaNet token mixer.
 *
 * The mixer (from "Inside Qwen3.5: a hybrid linear + full attention LLM",
 * romaanj.github.io/study/models/hybrid-attention, sections 2, 4, 5 and the config
 * footnote; the ungated rule is in "Hybrid Mamba-Transformer MoE", sotaaz.com,
 * section "Gated DeltaNet"):
 *
 *   y      = SiLU(depthwise causal conv, width 4, of x)           over q|k|v channels
 *   q, k  <- q / sqrt(|q|^2 + 1e-6), k / sqrt(|k|^2 + 1e-6)      per token and key head
 *   S_t    = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  alpha_t = exp(g_t)
 *   o_t    = scale * S_t q_t
 *
 * One recurrent state S (dv x dk, fp32, row index = value dimension) exists per sequence
 * and value head; the _ex calls (prefill and decode) can store it in bf16 instead. Value
 * head h reads key head h / (Hv / Hk).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers: device pointers unless stated; 16-byte aligned; tensors row-major and dense
 *   unless a stride argument says otherwise. The caller owns every buffer, including the
 *   workspace; the library allocates no device memory and keeps no state between calls,
 *   except gdn_chunk_prefill_noalloc's static scratch and, per device, three streams and a
 *   set of events that a long single-sequence prefill forks onto and joins back from
 *   (created on first use, kept for the life of the process).
 * Streams: every call is asynchronous on `stream` (NULL = the legacy default stream) and
 *   returns once its kernels are enqueued. Inputs must stay valid until they complete.
 * Errors: arguments are validated before anything is launched; an invalid call returns a
 *   status and launches nothing. Nothing is printed and no exception crosses the ABI.
 *   gdn_last_error() gives a short reason for the calling thread's last failure.
 *   A launch failure returns GDN_ERR_CUDA (and leaves the outputs undefined).
 * Channel order of the conv input/output and of the decode input x:
 *   [ q: Hk*dk | k: Hk*dk | v: Hv*dv ]  (Cc = 2*Hk*dk + Hv*dv).
 * Supported shapes: dk = dv in {16, 32, 64, 128}; Hv a multiple of Hk; conv width 4.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the same handle type); NULL is the legacy default stream. */
typedef struct CUstream_st* gdn_stream_t;

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, aliasing, bad cu_seqlens */
  GDN_ERR_UNSUPPORTED = 2,   /* valid but not built: head size, dtype, Hv % Hk != 0, or a
                                size beyond a path's limits */
  GDN_ERR_WORKSPACE = 3,     /* workspace too small (see the *_workspace_size query) */
  GDN_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  GDN_ERR_TIMEOUT = 5        /* a bounded device-side wait gave up (gdn_prefill_status) */
} gdn_status_t;

typedef enum {
  GDN_F32 = 0,               /* fp32 activations; fp32 state */
  GDN_BF16 = 1               /* bf16 activations, fp32 math and state (as a state_dt of
                                the _ex calls: bf16 state storage, fp32 math) */
} gdn_dtype_t;

/* Static string naming a status code. Never NULL. */
const char* gdn_status_string(gdn_status_t status);

/* Reason for the calling thread's most recent non-OK status ("" if none). The pointer is
 * valid until that thread's next call into the library. */
const char* gdn_last_error(void);

/* Library version, "major.minor.patch". */
const char* gdn_version(void);

/*
 * gdn_conv1d_silu -- width-4 depthwise causal conv followed by SiLU (prefill).
 *
 * Defined by the Qwen3.5 page, section 5 (the short kernel-4 causal convolution that
 * gives the recurrence local mixing) and its config footnote (conv kernel 4); SiLU
 * z / (1 + e^-z) follows the conv on every channel.
 *
 *   y[t, c] = SiLU( sum_{j=0..3} w[c, j] * x[t - 3 + j, c] )
 *
 * x, y            [T, Cc], dtype dt. y must not overlap x.
 * w               [Cc, 4], dtype dt; w[c, 3] multiplies the current token (PyTorch
 *                 cross-correlation order), no bias.
 * cu_seqlens      device int32 [n_seq + 1], cu[0] = 0, cu[n_seq] = T, non-decreasing;
 *                 every sequence restarts its window. NULL means one sequence of length T
 *                 (n_seq is then ignored and taken as 1).
 * conv_state_in   [n_seq, 3, Cc] dtype dt, the three inputs preceding each sequence
 *                 (oldest first), or NULL for zeros.
 * conv_state_out  [n_seq, 3, Cc] dtype dt, receives the last three inputs of each
 *                 sequence (reaching into conv_state_in for sequences shorter than 3),
 *                 or NULL. Must not overlap conv_state_in.
 * Returns GDN_OK, GDN_ERR_INVALID_ARG (T < 0, Cc <= 0 or Cc % 8 != 0, bad pointers),
 * GDN_ERR_UNSUPPORTED (dtype), GDN_ERR_CUDA. T = 0 is valid and launches only what
 * conv_state_out needs.
 */
gdn_status_t gdn_conv1d_silu(const void* x, void* y, gdn_dtype_t dt, const void* w,
                             const int32_t* cu_seqlens, int32_t n_seq, int64_t T, int32_t Cc,
                             const void* conv_state_in, void* conv_state_out,
                             gdn_stream_t stream);

/*
 * gdn_chunk_prefill_workspace_size -- bytes of device workspace gdn_chunk_prefill needs
 * for these sizes (0 is a valid answer); an upper bound, since calls with qk_l2norm = 0
 * need none. Returns SIZE_MAX for unsupported shapes, including bf16 heads of 128 whose
 * chunk rows (about T / 64 x Hv x 128) pass 2^31 - 1: the tensor-core path addresses them
 * with 32-bit TMA coordinates, so such a batch is split into several calls.
 */
size_t gdn_chunk_prefill_workspace_size(int64_t T, int32_t n_seq, int32_t Hk, int32_t Hv,
                                        int32_t dk, int32_t dv, gdn_dtype_t dt);

/*
 * gdn_chunk_prefill_path -- which kernels gdn_chunk_prefill (and _ex, _noalloc) runs for
 * these arguments, so that a caller can see a slow path before taking it:
 *   GDN_PATH_CHUNKED_TC (1)  the chunked WY/UT form on tcgen05 tensor cores: bf16
 *                            activations, dk = dv = 128, Hv / Hk <= 8, qk_l2norm = 1;
 *   GDN_PATH_RECURRENT  (0)  the token-by-token fp32 SIMT kernel: every other supported
 *                            shape (fp32 activations, heads of 16/32/64, qk_l2norm = 0).
 *                            It is exact to fp32 rounding but about 25x slower on long
 *                            bf16 sequences of 128-wide heads;
 *   -1                       unsupported arguments (the prefill returns an error).
 * The same path serves every length, sequence count and state dtype.
 */
enum { GDN_PATH_RECURRENT = 0, GDN_PATH_CHUNKED_TC = 1 };
int32_t gdn_chunk_prefill_path(gdn_dtype_t dt, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                               int32_t qk_l2norm);

/*
 * gdn_chunk_prefill_launches -- how many kernels of this library one gdn_chunk_prefill call
 * with these arguments enqueues on a GPU of num_sms SMs (host-only: no CUDA call is made):
 * 1 on the token-recurrent path; on the tensor-core path the plan, then one intra-chunk and
 * one chain launch, or, for one long sequence run in pieces, one chain launch per piece and
 * the intra-chunk launches of its schedule. Returns -1 for arguments the prefill rejects.
 */
int32_t gdn_chunk_prefill_launches(int64_t T, int32_t n_seq, int32_t Hk, int32_t Hv, int32_t dk,
                                   int32_t dv, gdn_dtype_t dt, int32_t qk_l2norm, int32_t num_sms);

/*
 * gdn_chunk_prefill -- the gated delta rule over packed sequences (prefill).
 *
 * Defined by the Qwen3.5 page, section 5: S <- alpha S + beta (v - S k) k^T read as
 * decay then delta write (equivalently S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) +
 * beta_t v_t k_t^T), the L2 norm on q and k, alpha and beta per token and per head;
 * section 2 for the read-out o = S q. The kernels evaluate it chunk by chunk (the
 * WY/UT form of the same recurrence); results equal the token-by-token recurrence up to
 * rounding. On the tensor-core path a single sequence of 32768 tokens or more is run in
 * eight pieces: the call forks onto library streams (the intra-chunk work of later
 * pieces beside the state pass of the current one) and joins back into `stream` with
 * events, so the call stays ordered with the rest of `stream`.
 *
 * q, k        token t, key head j at q + t*qk_stride + j*dk (elements), dtype dt.
 * v           token t, value head h at v + t*v_stride + h*dv, dtype dt.
 *             qk_stride = 0 means Hk*dk, v_stride = 0 means Hv*dv (dense). Strides let
 *             q/k/v be views into gdn_conv1d_silu's output (stride Cc, no copy).
 * g           [T, Hv] fp32 log-decay (alpha = exp(g), g <= 0 expected, not checked).
 * beta        [T, Hv] fp32 write strength.
 * o           [T, Hv, dv] dtype dt, written. Must not overlap any input.
 * cu_seqlens  device int32 [n_seq + 1] as for gdn_conv1d_silu, or NULL (one sequence).
 * initial_state  fp32 [n_seq, Hv, dv, dk] or NULL (zeros).
 * final_state    fp32 [n_seq, Hv, dv, dk] or NULL (not written). May equal
 *                initial_state (updated in place); must not partially overlap it.
 * scale       multiplies o (1.0 for the plain o = S q).
 * qk_l2norm   1: normalise q and k as above; 0: use them as given.
 * workspace   device memory of at least gdn_chunk_prefill_workspace_size(...) bytes,
 *             256-byte aligned, or NULL when that size is 0. Contents on entry are
 *             ignored; the caller must not use it concurrently with the call.
 * Returns GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_ERR_CUDA.
 */
gdn_status_t gdn_chunk_prefill(const void* q, const void* k, const void* v,
                               const float* g, const float* beta, void* o,
                               gdn_dtype_t dt, int64_t T, int32_t Hk, int32_t Hv,
                               int32_t dk, int32_t dv, int64_t qk_stride, int64_t v_stride,
                               const int32_t* cu_seqlens, int32_t n_seq,
                               const float* initial_state, float* final_state,
                               float scale, int32_t qk_l2norm,
                               void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_prefill_status -- whether the last gdn_chunk_prefill / gdn_chunk_prefill_ex that used
 * this workspace completed its device-side waits. The tensor-core kernels bound every wait
 * (for a TMA load or an MMA) and, when one gives up, record a code in the workspace's first
 * int and return early instead of hanging; the call itself has already returned GDN_OK.
 * This waits for the work queued on `stream`, reads that word and returns GDN_OK, or
 * GDN_ERR_TIMEOUT (the outputs of that call are invalid; gdn_last_error() names the kernel
 * and the wait), GDN_ERR_INVALID_ARG for a NULL workspace, GDN_ERR_CUDA if the read fails.
 * gdn_prefill_noalloc_status is the same for gdn_chunk_prefill_noalloc's static scratch on
 * the current device.
 */
gdn_status_t gdn_prefill_status(const void* workspace, gdn_stream_t stream);
gdn_status_t gdn_prefill_noalloc_status(gdn_stream_t stream);

/*
 * gdn_chunk_prefill_ex -- gdn_chunk_prefill with a selectable state storage dtype, that can
 * also store each sequence's state at block boundaries for prefix caching (a block's cached
 * state lets a later request that shares the prefix resume from it; the state after token t
 * is the S_t of the Qwen3.5 page, section 5).
 *
 * initial_state, final_state  [n_seq, Hv, dv, dk] of state_dt (as in gdn_chunk_prefill).
 * state_dt      GDN_F32, or GDN_BF16: states stored in bf16 (the storage a server that keeps
 *               bf16 decode states uses, see gdn_decode_step_ex). Each element is widened to
 *               fp32 on load; the recurrence runs in fp32 as for GDN_F32; the final and block
 *               states are rounded to bf16 (nearest, ties to even) once, when stored.
 * block_tokens  0: no block states (the other three block arguments are ignored); else a
 *               positive multiple of 64 (the chunk length, so boundaries fall on chunk ends).
 * block_states  [n_block_rows, Hv, dv, dk] of state_dt, 16-byte aligned: after the first
 *               m * block_tokens tokens of sequence n (m >= 1, m * block_tokens <= its
 *               length) its state is written to row block_rows[n] + m - 1. A sequence whose
 *               length is a multiple of block_tokens also gets its final state there.
 * block_rows    int32 [n_seq] device array: the first row of each sequence. Rows outside
 *               [0, n_block_rows) are skipped, not an error.
 * Other arguments and return codes as gdn_chunk_prefill; GDN_ERR_UNSUPPORTED also for an
 * unknown state_dt; GDN_ERR_INVALID_ARG also for a bad block_tokens, missing block buffers
 * or block_states overlapping another buffer.
 */
gdn_status_t gdn_chunk_prefill_ex(const void* q, const void* k, const void* v,
                                  const float* g, const float* beta, void* o,
                                  gdn_dtype_t dt, int64_t T, int32_t Hk, int32_t Hv,
                                  int32_t dk, int32_t dv, int64_t qk_stride, int64_t v_stride,
                                  const int32_t* cu_seqlens, int32_t n_seq,
                                  const void* initial_state, void* final_state,
                                  gdn_dtype_t state_dt, float scale, int32_t qk_l2norm,
                                  int32_t block_tokens, void* block_states,
                                  const int32_t* block_rows, int64_t n_block_rows,
                                  void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_chunk_prefill_noalloc -- gdn_chunk_prefill for callers that cannot allocate.
 *
 * The pages have no counterpart to this call; it is a convenience of this library.
 * Some callers cannot allocate device memory: a plugin inside a host application that
 * owns all GPU memory through its own pool and gives plugins no allocation hook, or a
 * latency-critical loop where cudaMalloc (and the synchronisation it may imply) is not
 * acceptable. This variant takes the same arguments as gdn_chunk_prefill minus the
 * workspace, and uses a scratch array that the library reserves statically on every GPU
 * that loads it (64 MiB, held until the process exits). It allocates nothing and calls
 * no allocating routine.
 *
 * Limit: the call is refused with GDN_ERR_WORKSPACE, launching nothing, when the path it
 * takes (gdn_chunk_prefill_path) needs more than 64 MiB of scratch for these sizes. The
 * tensor-core path needs gdn_chunk_prefill_workspace_size(...) bytes: with 48 value heads
 * of 128 in one sequence that allows 1,472 tokens per call (2,240 with 32 value heads); use
 * gdn_chunk_prefill with a caller workspace beyond that. The token-recurrent path needs
 * no scratch and is never refused.
 * Set-up: the first call on each device looks up the scratch array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call before any
 * stream capture. The array is shared by every call: its first word (the status word of
 * gdn_prefill_noalloc_status) is cleared by every call, the kernels rewrite everything
 * else they read from it, but calls whose execution overlaps on the GPU (different
 * streams, or different host threads on one device) race on it -- order them on one
 * stream or synchronise between them.
 * Returns the same codes as gdn_chunk_prefill.
 */
gdn_status_t gdn_chunk_prefill_noalloc(const void* q, const void* k, const void* v,
                                       const float* g, const float* beta, void* o,
                                       gdn_dtype_t dt, int64_t T, int32_t Hk, int32_t Hv,
                                       int32_t dk, int32_t dv, int64_t qk_stride,
                                       int64_t v_stride, const int32_t* cu_seqlens,
                                       int32_t n_seq, const float* initial_state,
                                       float* final_state, float scale, int32_t qk_l2norm,
                                       gdn_stream_t stream);

/*
 * gdn_decode_step -- one token for each of B sequences, state updated in place.
 *
 * Defined by the Qwen3.5 page, section 8 (decode becomes a state-update workload:
 * fixed-size fp32 state read, modified and written every token) with the update of
 * section 5 and the conv of the config footnote. Per sequence b:
 *   z_c = w[c,0] cs[b,0,c] + w[c,1] cs[b,1,c] + w[c,2] cs[b,2,c] + w[c,3] x[b,c]; y = SiLU(z)
 *   cs[b] <- [cs[b,1], cs[b,2], x[b]]             (taps shift by one, in place)
 *   q, k, v from y (channel order above), q and k L2-normalised
 *   S[b,h] <- alpha S[b,h] (I - beta k k^T) + beta v k^T;  o[b,h] = scale * S[b,h] q
 *
 * x           [B, Cc] dtype dt, this step's pre-conv q|k|v.
 * conv_w      [Cc, 4] dtype dt.
 * conv_state  [B, 3, Cc] dtype dt, read and updated in place.
 * g, beta     [B, Hv] fp32.
 * state       [B, Hv, dv, dk] fp32, read and updated in place.
 * o           [B, Hv, dv] dtype dt.
 * Returns GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA. B = 0 is a no-op.
 */
gdn_status_t gdn_decode_step(const void* x, const void* conv_w, void* conv_state,
                             const float* g, const float* beta, float* state, void* o,
                             gdn_dtype_t dt, int32_t B, int32_t Hk, int32_t Hv,
                             int32_t dk, int32_t dv, float scale, gdn_stream_t stream);

/*
 * gdn_decode_tokens -- n_tok consecutive tokens (1 <= n_tok <= 8) for each of B sequences,
 * conv taps and states updated in place: a multi-token decode or speculative verify step.
 *
 * Defined as n_tok applications of gdn_decode_step's update (Qwen3.5 page, section 5 and the
 * conv of the config footnote), token t of every sequence before token t + 1: the result
 * equals n_tok calls of gdn_decode_step, and a prefill of B sequences of n_tok tokens from
 * the same states. Each state is read and written once per call (Qwen3.5 page, section 8:
 * decode is bound by moving the fixed-size state).
 *
 * x           [B, n_tok, Cc] dtype dt, the tokens' pre-conv q|k|v in order.
 * conv_w      [Cc, 4] dtype dt.
 * conv_state  [B, 3, Cc] dtype dt, read and updated in place (advances by n_tok taps).
 * g, beta     [B, n_tok, Hv] fp32.
 * state       [B, Hv, dv, dk] fp32, read and updated in place.
 * o           [B, n_tok, Hv, dv] dtype dt.
 * All tokens are committed: a caller that rejects speculative tokens keeps a copy of the
 * states from before the call. Returns GDN_OK, GDN_ERR_INVALID_ARG (n_tok outside [1, 8],
 * null, misaligned or overlapping buffers), GDN_ERR_UNSUPPORTED (as gdn_decode_step, or a
 * head group whose n_tok tokens exceed one CTA's shared memory), GDN_ERR_CUDA. B = 0 is a
 * no-op.
 */
gdn_status_t gdn_decode_tokens(const void* x, const void* conv_w, void* conv_state,
                               const float* g, const float* beta, float* state, void* o,
                               gdn_dtype_t dt, int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv,
                               int32_t dk, int32_t dv, float scale, gdn_stream_t stream);

/*
 * gdn_decode_step_ex, gdn_decode_tokens_ex -- gdn_decode_step and gdn_decode_tokens with the
 * recurrent state stored as state_dt: GDN_F32 (the calls above), or GDN_BF16, which halves
 * the bytes that dominate decode (Qwen3.5 page, section 8: decode moves the fixed-size state
 * every token). With GDN_BF16 each state element is widened to fp32 on load, the update is
 * computed in fp32 as for GDN_F32, and the result is rounded to bf16 (nearest, ties to even)
 * once per call when it is stored: gdn_decode_tokens_ex rounds after all n_tok tokens.
 *
 * state       [B, Hv, dv, dk] of state_dt, 16-byte aligned, read and updated in place.
 * Every other argument, and the return codes, as in gdn_decode_step / gdn_decode_tokens
 * (GDN_ERR_UNSUPPORTED also for an unknown state_dt).
 */
gdn_status_t gdn_decode_step_ex(const void* x, const void* conv_w, void* conv_state,
                                const float* g, const float* beta, void* state,
                                gdn_dtype_t state_dt, void* o, gdn_dtype_t dt, int32_t B,
                                int32_t Hk, int32_t Hv, int32_t dk, int32_t dv, float scale,
                                gdn_stream_t stream);
gdn_status_t gdn_decode_tokens_ex(const void* x, const void* conv_w, void* conv_state,
                                  const float* g, const float* beta, void* state,
                                  gdn_dtype_t state_dt, void* o, gdn_dtype_t dt, int32_t B,
                                  int32_t n_tok, int32_t Hk, int32_t Hv, int32_t dk, int32_t dv,
                                  float scale, gdn_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* GDN_H_ */
