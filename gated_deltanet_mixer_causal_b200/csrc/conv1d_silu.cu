// conv1d_silu.cu -- width-4 depthwise causal conv + SiLU over packed sequences.
//
// y[t, c] = SiLU(sum_j w[c, j] x[t - 3 + j, c]), restarting at every sequence start from
// the carried taps or zeros (Qwen3.5 page, section 5 and config footnote: conv kernel 4).
//
// HBM-bound: each thread owns 8 channels (one 16-byte bf16 vector) and a run of
// kRunTokens tokens, sliding a 3-token window in registers, so every input is read once
// (plus a 3-token halo per run, which hits L2) and every output written once. A warp
// covers 32 consecutive vectors of one token row: 512 contiguous bytes per access.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kVec = 8;          // channels per thread
constexpr int kThreads = 128;    // threads per CTA (128 vectors = 1024 channels)
constexpr int kRunTokens = 32;   // tokens per thread
constexpr int kPrefetch = 4;     // tokens loaded ahead of use

// Index of the sequence holding token t: the n with cu[n] <= t < cu[n+1] (clamped).
__device__ __forceinline__ int32_t find_seq(const int32_t* cu, int32_t n_seq, int64_t t) {
  int32_t lo = 0, hi = n_seq - 1;
  while (lo < hi) {
    int32_t mid = (lo + hi + 1) >> 1;
    if ((int64_t)cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <typename T>
__device__ __forceinline__ void load_tap(const T* state_in, int32_t n, int32_t j, int32_t Cc,
                                         int32_t c0, float (&v)[kVec]) {
  if (state_in == nullptr || j < 0 || j > 2) {   // j outside [0, 2] only for malformed cu
#pragma unroll
    for (int i = 0; i < kVec; ++i) v[i] = 0.f;
  } else {
    VecIO<T, kVec>::load(state_in + ((int64_t)n * 3 + j) * Cc + c0, v);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
conv1d_silu_kernel(const T* __restrict__ x, T* __restrict__ y, const T* __restrict__ w,
                   const int32_t* __restrict__ cu, int32_t n_seq, int64_t T_tok, int32_t Cc,
                   const T* __restrict__ state_in, T* __restrict__ state_out) {
  const int32_t n_vec = Cc / kVec;
  const int32_t cv = blockIdx.y * kThreads + threadIdx.x;
  if (cv >= n_vec) return;
  const int32_t c0 = cv * kVec;
  const int64_t t0 = (int64_t)blockIdx.x * kRunTokens;
  int64_t t1 = t0 + kRunTokens;
  if (t1 > T_tok) t1 = T_tok;

  float wt[4][kVec];
  {
    float wr[4 * kVec];
    VecIO<T, 4 * kVec>::load(w + (int64_t)c0 * 4, wr);   // [8 channels][4 taps]
#pragma unroll
    for (int i = 0; i < kVec; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) wt[j][i] = wr[i * 4 + j];
  }

  int32_t n = (cu == nullptr) ? 0 : find_seq(cu, n_seq, t0);
  int64_t bos, eos;
  seq_bounds(cu, n, T_tok, bos, eos);

  // window[0] = x[t-3], window[1] = x[t-2], window[2] = x[t-1]
  float win[3][kVec];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int64_t s = t0 - 3 + j;
    if (s >= bos) VecIO<T, kVec>::load(x + s * Cc + c0, win[j]);
    else load_tap(state_in, n, (int32_t)(3 + (s - bos)), Cc, c0, win[j]);
  }

  for (int64_t tb = t0; tb < t1; tb += kPrefetch) {
    float xin[kPrefetch][kVec];
#pragma unroll
    for (int p = 0; p < kPrefetch; ++p)
      if (tb + p < t1) VecIO<T, kVec>::load(x + (tb + p) * Cc + c0, xin[p]);
#pragma unroll
    for (int p = 0; p < kPrefetch; ++p) {
      const int64_t t = tb + p;
      if (t >= t1) break;
      if (t >= eos) {                       // entered the next non-empty sequence
        while (n + 1 < n_seq && (int64_t)cu[n + 1] <= t) ++n;
        seq_bounds(cu, n, T_tok, bos, eos);
#pragma unroll
        for (int j = 0; j < 3; ++j) load_tap(state_in, n, j, Cc, c0, win[j]);
      }
      float out[kVec];
#pragma unroll
      for (int i = 0; i < kVec; ++i) {
        float z = wt[0][i] * win[0][i];
        z = fmaf(wt[1][i], win[1][i], z);
        z = fmaf(wt[2][i], win[2][i], z);
        z = fmaf(wt[3][i], xin[p][i], z);
        out[i] = silu(z);
      }
      VecIO<T, kVec>::store(y + t * Cc + c0, out);
#pragma unroll
      for (int i = 0; i < kVec; ++i) {
        win[0][i] = win[1][i]; win[1][i] = win[2][i]; win[2][i] = xin[p][i];
      }
      if (state_out != nullptr && t == eos - 1) {
#pragma unroll
        for (int j = 0; j < 3; ++j)
          VecIO<T, kVec>::store(state_out + ((int64_t)n * 3 + j) * Cc + c0, win[j]);
      }
    }
  }
}

// conv_state_out for sequences with no tokens: the carried taps pass through (or zeros).
template <typename T>
__global__ void conv_state_empty_kernel(const int32_t* __restrict__ cu, int32_t n_seq,
                                        int64_t T_tok, int32_t Cc, const T* __restrict__ state_in,
                                        T* __restrict__ state_out) {
  const int32_t n = blockIdx.y;
  int64_t bos, eos;
  seq_bounds(cu, n, T_tok, bos, eos);
  if (eos > bos) return;
  const int64_t per_seq = 3LL * Cc;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < per_seq;
       e += (int64_t)gridDim.x * blockDim.x) {
    state_out[n * per_seq + e] = state_in ? state_in[n * per_seq + e] : from_f<T>(0.f);
  }
}

template <typename T>
cudaError_t launch_typed(const void* x, void* y, const void* w, const int32_t* cu, int32_t n_seq,
                         int64_t T_tok, int32_t Cc, const void* sin, void* sout, cudaStream_t st) {
  if (T_tok > 0) {
    // x: token runs (consecutive CTAs share halo rows in L2), y: channel blocks
    dim3 grid((unsigned)((T_tok + kRunTokens - 1) / kRunTokens),
              (unsigned)((Cc / kVec + kThreads - 1) / kThreads));
    conv1d_silu_kernel<T><<<grid, kThreads, 0, st>>>(
        (const T*)x, (T*)y, (const T*)w, cu, n_seq, T_tok, Cc, (const T*)sin, (T*)sout);
  }
  if (sout != nullptr) {
    dim3 grid((unsigned)((3LL * Cc + 255) / 256), (unsigned)n_seq);
    conv_state_empty_kernel<T><<<grid, 256, 0, st>>>(cu, n_seq, T_tok, Cc, (const T*)sin, (T*)sout);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv1d_silu(int dtype, const void* x, void* y, const void* w,
                               const int32_t* cu, int32_t n_seq, int64_t T, int32_t Cc,
                               const void* sin, void* sout, cudaStream_t stream) {
  if (dtype == kF32) return launch_typed<float>(x, y, w, cu, n_seq, T, Cc, sin, sout, stream);
  return launch_typed<bf16>(x, y, w, cu, n_seq, T, Cc, sin, sout, stream);
}

}  // namespace gdn
