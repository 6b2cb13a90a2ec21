// conv1d_silu.cu -- width-4 depthwise causal conv + SiLU over packed sequences.
//
// y[t, c] = SiLU(sum_j w[c, j] x[t - 3 + j, c]), restarting at every sequence start from
// the carried taps or zeros (Qwen3.5 page, section 5 and config footnote: conv kernel 4).
//
// HBM-bound: every input is read once and every output written once. A CTA owns a tile of
// kTileTokens tokens x kTileVecs * 8 channels: it copies the tile plus a 3-token halo into
// shared memory with 16-byte cp.async (zero-filled outside [0, T)), so many bytes are in
// flight per SM without holding them in registers; then each thread slides a 3-token
// window over 16 consecutive tokens of 8 channels and writes 16-byte vectors, consecutive
// threads covering consecutive channels (1 KB contiguous per token row for bf16). Runs
// that lie inside one sequence with their three predecessors take a fully unrolled path
// (no per-token boundary tests, the window in renamed registers); the general path
// handles sequence starts, carried taps and ragged ends.
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

// Tiles of 32 tokens x 512 channels, 128 threads, five CTAs per SM (96 registers, 36 KB
// of shared memory each): one CTA's loads overlap the others' compute and stores. Measured
// on the 27B layer at T = 65536 against the alternatives (tokens x threads x CTAs per SM):
// 64 x 256 x 2 0.561 ms, 64 x 256 x 3 0.526, 32 x 128 x 4 0.500, 16 x 64 x 8 0.490,
// 32 x 128 x 5 0.467 (5.7 TB/s).
constexpr int kVec = 8;            // channels per thread
constexpr int kTileTokens = 32;
constexpr int kTileVecs = 64;      // 8-channel vectors per tile (512 channels)
constexpr int kThreads = 128;
constexpr int kMinBlocks = 5;
constexpr int kTokPerThread = kTileTokens * kTileVecs / kThreads;   // 16
constexpr int kRows = kTileTokens + 3;

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

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(valid ? 16 : 0)
               : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
conv1d_silu_kernel(const T* __restrict__ x, T* __restrict__ y, const T* __restrict__ w,
                   const int32_t* __restrict__ cu, int32_t n_seq, int64_t T_tok, int32_t Cc,
                   const T* __restrict__ state_in, T* __restrict__ state_out) {
  constexpr int kRowElems = kTileVecs * kVec;
  constexpr int kChunksPerRow = kRowElems * (int)sizeof(T) / 16;
  constexpr int kElemsPerChunk = 16 / (int)sizeof(T);
  extern __shared__ __align__(16) uint8_t smem_raw[];
  T* tile = reinterpret_cast<T*>(smem_raw);   // [kRows][kRowElems], row 0 = token t0 - 3

  const int64_t t0 = (int64_t)blockIdx.x * kTileTokens;
  const int32_t cbase = blockIdx.y * kRowElems;
  const int tid = threadIdx.x;

  for (int idx = tid; idx < kRows * kChunksPerRow; idx += kThreads) {
    const int row = idx / kChunksPerRow, ch = idx % kChunksPerRow;
    const int64_t t = t0 - 3 + row;
    const int32_t c = cbase + ch * kElemsPerChunk;
    const bool valid = t >= 0 && t < T_tok && c < Cc;
    const T* src = valid ? x + t * Cc + c : x;
    cp_async16(tile + row * kRowElems + ch * kElemsPerChunk, src, valid);
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  const int cv = tid % kTileVecs, tg = tid / kTileVecs;
  const int32_t c0 = cbase + cv * kVec;
  if (c0 >= Cc) return;
  const int64_t ta = t0 + (int64_t)tg * kTokPerThread;
  if (ta >= T_tok) return;
  int64_t tb = ta + kTokPerThread;
  if (tb > T_tok) tb = T_tok;

  float wt[4][kVec];
  {
    float wr[4 * kVec];
    VecIO<T, 4 * kVec>::load(w + (int64_t)c0 * 4, wr);   // [8 channels][4 taps]
#pragma unroll
    for (int i = 0; i < kVec; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) wt[j][i] = wr[i * 4 + j];
  }

  int32_t n = (cu == nullptr) ? 0 : find_seq(cu, n_seq, ta);
  int64_t bos, eos;
  seq_bounds(cu, n, T_tok, bos, eos);
  auto row_of = [&](int64_t t) { return tile + (int)(t - t0 + 3) * kRowElems + cv * kVec; };

  if (ta - 3 >= bos && tb == ta + kTokPerThread && tb <= eos) {
    // the run and its three predecessors lie in one sequence (every run of a long sequence
    // but its first): fully unrolled, the sliding window lives in renamed registers
    float w0[kVec], w1[kVec], w2[kVec];
    VecIO<T, kVec>::load(row_of(ta - 3), w0);
    VecIO<T, kVec>::load(row_of(ta - 2), w1);
    VecIO<T, kVec>::load(row_of(ta - 1), w2);
    T* yp = y + ta * Cc + c0;
#pragma unroll
    for (int k = 0; k < kTokPerThread; ++k) {
      float xin[kVec], out[kVec];
      VecIO<T, kVec>::load(row_of(ta + k), xin);
#pragma unroll
      for (int i = 0; i < kVec; ++i) {
        float z = wt[0][i] * w0[i];
        z = fmaf(wt[1][i], w1[i], z);
        z = fmaf(wt[2][i], w2[i], z);
        z = fmaf(wt[3][i], xin[i], z);
        out[i] = silu(z);
      }
      VecIO<T, kVec>::store(yp + (int64_t)k * Cc, out);
#pragma unroll
      for (int i = 0; i < kVec; ++i) { w0[i] = w1[i]; w1[i] = w2[i]; w2[i] = xin[i]; }
    }
    if (state_out != nullptr && tb == eos) {   // the run ends the sequence: carry its taps
      VecIO<T, kVec>::store(state_out + ((int64_t)n * 3 + 0) * Cc + c0, w0);
      VecIO<T, kVec>::store(state_out + ((int64_t)n * 3 + 1) * Cc + c0, w1);
      VecIO<T, kVec>::store(state_out + ((int64_t)n * 3 + 2) * Cc + c0, w2);
    }
    return;
  }

  // window[0] = x[t-3], window[1] = x[t-2], window[2] = x[t-1]
  float win[3][kVec];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int64_t s = ta - 3 + j;
    if (s >= bos) VecIO<T, kVec>::load(row_of(s), win[j]);
    else load_tap(state_in, n, (int32_t)(3 + (s - bos)), Cc, c0, win[j]);
  }

  for (int64_t t = ta; t < tb; ++t) {
    if (t >= eos) {                       // entered the next non-empty sequence
      while (n + 1 < n_seq && (int64_t)cu[n + 1] <= t) ++n;
      seq_bounds(cu, n, T_tok, bos, eos);
#pragma unroll
      for (int j = 0; j < 3; ++j) load_tap(state_in, n, j, Cc, c0, win[j]);
    }
    float xin[kVec], out[kVec];
    VecIO<T, kVec>::load(row_of(t), xin);
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      float z = wt[0][i] * win[0][i];
      z = fmaf(wt[1][i], win[1][i], z);
      z = fmaf(wt[2][i], win[2][i], z);
      z = fmaf(wt[3][i], xin[i], z);
      out[i] = silu(z);
    }
    VecIO<T, kVec>::store(y + t * Cc + c0, out);
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      win[0][i] = win[1][i]; win[1][i] = win[2][i]; win[2][i] = xin[i];
    }
    if (state_out != nullptr && t == eos - 1) {
#pragma unroll
      for (int j = 0; j < 3; ++j)
        VecIO<T, kVec>::store(state_out + ((int64_t)n * 3 + j) * Cc + c0, win[j]);
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
    const int smem = kRows * kTileVecs * kVec * (int)sizeof(T);
    static uint64_t attrs_set = 0;   // devices with the shared-memory attribute set
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (smem > 48 * 1024 && (dev >= 64 || !(attrs_set >> dev & 1))) {
      e = cudaFuncSetAttribute(conv1d_silu_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      if (dev < 64) attrs_set |= 1ull << dev;
    }
    // x: token tiles (consecutive CTAs share halo rows in L2), y: channel tiles
    dim3 grid((unsigned)((T_tok + kTileTokens - 1) / kTileTokens),
              (unsigned)((Cc + kTileVecs * kVec - 1) / (kTileVecs * kVec)));
    conv1d_silu_kernel<T><<<grid, kThreads, smem, st>>>(
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
