// decode_step.cu -- one token for each of B sequences, conv taps and states in place (states
// stored in fp32, or in bf16 with fp32 arithmetic).
//
// Workload (Qwen3.5 page, section 8): decode is a state-update stream -- every token reads,
// modifies and writes each fixed-size fp32 state. It is HBM-bound: per (sequence, value
// head) the 128 x 128 state (64 KB) is read once and written once; nothing else is large.
//
// One CTA owns one (sequence b, key head hk): the conv channels of that key head's q and k
// and of its G = Hv/Hk value heads. Owning the channels makes the in-place tap shift
// race-free without a second kernel. After the conv, SiLU and the q/k L2 norm (in shared
// memory), each warp streams whole state rows (value index i): an fp32 row is 128 floats,
// one float4 per lane, so a warp access is 512 contiguous bytes; a bf16 row (256 bytes) is
// read by half a warp with 16-byte loads, two rows per access. Per row, with s the old row:
//   sk = s.k, sq = s.q                  (one two-value warp reduction)
//   u  = beta (v_i - alpha sk)          (delta write strength for this row)
//   s' = alpha s + u k                  (decay, then the write along k)
//   o_i = scale (alpha sq + u (k.q))    (= s'.q without a second pass)
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowUnroll = 4;      // rows per warp iteration (loads in flight)
constexpr float kEps = 1e-6f;

// VEC consecutive state values of one row, streamed (evict-first): fp32 storage, or bf16
// storage widened to fp32 for the arithmetic and rounded once on the store.
template <typename S, int VEC> struct RowIO;
template <> struct RowIO<float, 4> {
  static __device__ __forceinline__ void load(const float* p, float (&s)[4]) {
    float4 v = __ldcs(reinterpret_cast<const float4*>(p));
    s[0] = v.x; s[1] = v.y; s[2] = v.z; s[3] = v.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&s)[4]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(s[0], s[1], s[2], s[3]));
  }
};
template <> struct RowIO<float, 2> {
  static __device__ __forceinline__ void load(const float* p, float (&s)[2]) {
    float2 v = __ldcs(reinterpret_cast<const float2*>(p));
    s[0] = v.x; s[1] = v.y;
  }
  static __device__ __forceinline__ void store(float* p, const float (&s)[2]) {
    __stcs(reinterpret_cast<float2*>(p), make_float2(s[0], s[1]));
  }
};
template <> struct RowIO<float, 1> {
  static __device__ __forceinline__ void load(const float* p, float (&s)[1]) { s[0] = __ldcs(p); }
  static __device__ __forceinline__ void store(float* p, const float (&s)[1]) { __stcs(p, s[0]); }
};
template <> struct RowIO<bf16, 8> {
  static __device__ __forceinline__ void load(const bf16* p, float (&s)[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      s[2 * i] = f.x; s[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store(bf16* p, const float (&s)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 f = __floats2bfloat162_rn(s[2 * i], s[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&f);
    }
    __stcs(reinterpret_cast<uint4*>(p), make_uint4(w[0], w[1], w[2], w[3]));
  }
};
template <> struct RowIO<bf16, 2> {
  static __device__ __forceinline__ void load(const bf16* p, float (&s)[2]) {
    const unsigned int u = __ldcs(reinterpret_cast<const unsigned int*>(p));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
    s[0] = a.x; s[1] = a.y;
  }
  static __device__ __forceinline__ void store(bf16* p, const float (&s)[2]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(s[0], s[1]);
    __stcs(reinterpret_cast<unsigned int*>(p), *reinterpret_cast<unsigned int*>(&a));
  }
};
template <> struct RowIO<bf16, 1> {
  static __device__ __forceinline__ void load(const bf16* p, float (&s)[1]) { s[0] = __bfloat162float(p[0]); }
  static __device__ __forceinline__ void store(bf16* p, const float (&s)[1]) { p[0] = __float2bfloat16_rn(s[0]); }
};

// Lanes per state row: a row of 128 bf16 values (256 bytes) is read by 16 lanes with 16-byte
// loads, two rows per warp access, so a warp instruction still moves 512 bytes and each
// row's dot products reduce over 16 lanes (4 shuffle rounds); every other case uses the
// whole warp per row.
template <typename S, int D> struct RowShape {
  static constexpr int VEC = (sizeof(S) == 2 && D == 128) ? 8 : (D >= 32 ? D / 32 : 1);
  static constexpr int LPR = (sizeof(S) == 2 && D == 128) ? 16 : 32;
};

template <typename T, int D, typename S>
__global__ void __launch_bounds__(kThreads, 3)   // three CTAs per SM: 24 warps of loads in flight
decode_step_kernel(const T* __restrict__ x, const T* __restrict__ conv_w, T* __restrict__ conv_state,
                   const float* __restrict__ g, const float* __restrict__ beta,
                   S* __restrict__ state, T* __restrict__ o, int32_t Hk, int32_t Hv,
                   float scale) {
  constexpr int VEC = RowShape<S, D>::VEC;
  constexpr int LPR = RowShape<S, D>::LPR;   // lanes per row
  constexpr int RPW = 32 / LPR;              // rows per warp access
  const int G = Hv / Hk;
  const int32_t Cc = 2 * Hk * D + Hv * D;
  const int64_t b = blockIdx.x / Hk;
  const int hk = blockIdx.x % Hk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  extern __shared__ float smem[];
  float* ys = smem;                       // [(2 + G) * D]: q | k | v of the G heads
  float* os = smem + (2 + G) * D;         // [G * D] outputs
  float2* ab = reinterpret_cast<float2*>(os + G * D);   // [G] (e^g, beta) of each value head

  // 1. conv + SiLU over this CTA's channels; shift the taps in place.
  const int n_local = (2 + G) * D;
  for (int lv = threadIdx.x; lv < n_local / 8; lv += kThreads) {
    const int lc = lv * 8;
    int gc;
    if (lc < D) gc = hk * D + lc;
    else if (lc < 2 * D) gc = Hk * D + hk * D + (lc - D);
    else gc = 2 * Hk * D + hk * G * D + (lc - 2 * D);
    float xv[8], t0[8], t1[8], t2[8], wr[32];
    VecIO<T, 8>::load(x + b * Cc + gc, xv);
    T* cs = conv_state + b * 3 * Cc + gc;
    VecIO<T, 8>::load(cs, t0);
    VecIO<T, 8>::load(cs + Cc, t1);
    VecIO<T, 8>::load(cs + 2 * Cc, t2);
    VecIO<T, 32>::load(conv_w + (int64_t)gc * 4, wr);
    float yv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float z = wr[i * 4 + 0] * t0[i];
      z = fmaf(wr[i * 4 + 1], t1[i], z);
      z = fmaf(wr[i * 4 + 2], t2[i], z);
      z = fmaf(wr[i * 4 + 3], xv[i], z);
      yv[i] = silu(z);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) ys[lc + i] = yv[i];
    VecIO<T, 8>::store(cs, t1);
    VecIO<T, 8>::store(cs + Cc, t2);
    VecIO<T, 8>::store(cs + 2 * Cc, xv);
  }
  if (threadIdx.x < G) {   // once per CTA rather than once per row lane
    const int64_t gi = b * Hv + (int64_t)hk * G + threadIdx.x;
    ab[threadIdx.x] = make_float2(expf(g[gi]), beta[gi]);
  }
  __syncthreads();

  // 2. L2-normalised q and k, per warp, in registers (VEC columns per lane; with LPR = 16
  //    lanes l and l + 16 hold the same columns).
  const int col = (lane % LPR) * VEC;
  const bool active = col < D;
  float qh[VEC], kh[VEC];
  float qq = 0.f, kk = 0.f, kq = 0.f;
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    qh[j] = active ? ys[col + j] : 0.f;
    kh[j] = active ? ys[D + col + j] : 0.f;
    qq = fmaf(qh[j], qh[j], qq);
    kk = fmaf(kh[j], kh[j], kk);
    kq = fmaf(kh[j], qh[j], kq);
  }
#pragma unroll
  for (int m = LPR / 2; m >= 1; m >>= 1) {
    qq += __shfl_xor_sync(0xffffffffu, qq, m);
    kk += __shfl_xor_sync(0xffffffffu, kk, m);
    kq += __shfl_xor_sync(0xffffffffu, kq, m);
  }
  const float iq = 1.0f / sqrtf(qq + kEps), ik = 1.0f / sqrtf(kk + kEps);
#pragma unroll
  for (int j = 0; j < VEC; ++j) { qh[j] *= iq; kh[j] *= ik; }
  const float kqh = kq * iq * ik;

  // 3. stream the G * D state rows of this CTA: a warp takes kRowUnroll x RPW rows per
  //    iteration (row r0 + u * RPW + lane / LPR in slot u).
  const int rows = G * D;
  const int sub = lane / LPR;
  for (int r0 = warp * kRowUnroll * RPW; r0 < rows; r0 += kWarps * kRowUnroll * RPW) {
    float s[kRowUnroll][VEC];
    // the CTA's G value heads are consecutive, so its rows are one contiguous block
    S* rows_base = state + (b * Hv + (int64_t)hk * G) * D * D + col;
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int r = r0 + u * RPW + sub;
      if (r < rows && active) RowIO<S, VEC>::load(rows_base + (int64_t)r * D, s[u]);
      else {
#pragma unroll
        for (int j = 0; j < VEC; ++j) s[u][j] = 0.f;
      }
    }
    float sk[kRowUnroll], sq[kRowUnroll];
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      float a = 0.f, c = 0.f;
#pragma unroll
      for (int j = 0; j < VEC; ++j) { a = fmaf(s[u][j], kh[j], a); c = fmaf(s[u][j], qh[j], c); }
      sk[u] = a; sq[u] = c;
    }
#pragma unroll
    for (int m = LPR / 2; m >= 1; m >>= 1)
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) {
        sk[u] += __shfl_xor_sync(0xffffffffu, sk[u], m);
        sq[u] += __shfl_xor_sync(0xffffffffu, sq[u], m);
      }
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int r = r0 + u * RPW + sub;
      if (r >= rows) continue;
      const float2 sc = ab[r / D];
      const float alpha = sc.x, bt = sc.y;
      const float uu = bt * (ys[2 * D + r] - alpha * sk[u]);
#pragma unroll
      for (int j = 0; j < VEC; ++j) s[u][j] = fmaf(alpha, s[u][j], uu * kh[j]);
      if (active) RowIO<S, VEC>::store(rows_base + (int64_t)r * D, s[u]);
      if (lane % LPR == 0) os[r] = scale * fmaf(alpha, sq[u], uu * kqh);
    }
  }
  __syncthreads();

  // 4. outputs of the G heads are contiguous: o[b, hk*G .. hk*G+G-1, :]
  T* ob = o + (b * Hv + (int64_t)hk * G) * D;
  for (int e = threadIdx.x; e < rows; e += kThreads) ob[e] = from_f<T>(os[e]);
}

template <typename T, int D, typename S>
cudaError_t launch_typed(const void* x, const void* w, void* cs, const float* g, const float* beta,
                         void* state, void* o, int32_t B, int32_t Hk, int32_t Hv, float scale,
                         cudaStream_t st) {
  const int G = Hv / Hk;
  const size_t smem = sizeof(float) * (size_t)((2 + G) * D + G * D + 2 * G);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_step_kernel<T, D, S>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)((int64_t)B * Hk));
  decode_step_kernel<T, D, S><<<grid, kThreads, smem, st>>>(
      (const T*)x, (const T*)w, (T*)cs, g, beta, (S*)state, (T*)o, Hk, Hv, scale);
  return cudaGetLastError();
}

template <typename T, typename S>
cudaError_t launch_d(const void* x, const void* w, void* cs, const float* g, const float* beta,
                     void* state, void* o, int32_t B, int32_t Hk, int32_t Hv, int32_t d,
                     float scale, cudaStream_t st) {
  switch (d) {
    case 16: return launch_typed<T, 16, S>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    case 32: return launch_typed<T, 32, S>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    case 64: return launch_typed<T, 64, S>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    default: return launch_typed<T, 128, S>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
  }
}

}  // namespace

cudaError_t launch_decode_step(int dtype, const void* x, const void* conv_w, void* conv_state,
                               const float* g, const float* beta, void* state, int state_dtype,
                               void* o, int32_t B, int32_t Hk, int32_t Hv, int32_t d, float scale,
                               cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  if (dtype == kF32) {
    if (state_dtype == kF32)
      return launch_d<float, float>(x, conv_w, conv_state, g, beta, state, o, B, Hk, Hv, d, scale, stream);
    return launch_d<float, bf16>(x, conv_w, conv_state, g, beta, state, o, B, Hk, Hv, d, scale, stream);
  }
  if (state_dtype == kF32)
    return launch_d<bf16, float>(x, conv_w, conv_state, g, beta, state, o, B, Hk, Hv, d, scale, stream);
  return launch_d<bf16, bf16>(x, conv_w, conv_state, g, beta, state, o, B, Hk, Hv, d, scale, stream);
}

}  // namespace gdn
