// decode_tokens.cu -- n_tok (1..8) consecutive tokens for each of B sequences, conv taps and
// fp32 states in place: a multi-token decode / speculative verify step.
//
// Same update as the single-token step (Qwen3.5 page, section 5: decay, then the delta
// write along k; section 8: decode is a state-update stream), applied n_tok times. The
// update of state row i (value index) only reads that row, so each row is loaded once, run
// through all n_tok tokens in registers and stored once: the 64 KB state of a (sequence,
// value head) crosses HBM once per call instead of once per token.
//
// One CTA owns one (sequence b, key head hk), as in the single-token kernel:
//  1. conv + SiLU of the call's tokens over this key head's channels: the three carried taps
//     and the n_tok new inputs form one window; the taps advance by n_tok, in place;
//  2. q_t, k_t L2-normalised per token in shared memory, read per token by the row loop;
//  3. each warp streams whole state rows: per token t, with s the current row,
//       sk = s.k_t, sq = s.q_t;  u = beta_t (v_t,i - alpha_t sk);  s <- alpha_t s + u k_t
//       o_t,i = scale (alpha_t sq + u (k_t.q_t))
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowUnroll = 4;      // rows per warp iteration, all of one value head
constexpr int kMaxTok = 8;
constexpr float kEps = 1e-6f;

template <int VEC> struct Row;
template <> struct Row<4> {
  static __device__ __forceinline__ void load(const float* p, float (&s)[4]) {
    const float4 v = __ldcs(reinterpret_cast<const float4*>(p));
    s[0] = v.x; s[1] = v.y; s[2] = v.z; s[3] = v.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&s)[4]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(s[0], s[1], s[2], s[3]));
  }
};
template <> struct Row<2> {
  static __device__ __forceinline__ void load(const float* p, float (&s)[2]) {
    const float2 v = __ldcs(reinterpret_cast<const float2*>(p));
    s[0] = v.x; s[1] = v.y;
  }
  static __device__ __forceinline__ void store(float* p, const float (&s)[2]) {
    __stcs(reinterpret_cast<float2*>(p), make_float2(s[0], s[1]));
  }
};
template <> struct Row<1> {
  static __device__ __forceinline__ void load(const float* p, float (&s)[1]) { s[0] = __ldcs(p); }
  static __device__ __forceinline__ void store(float* p, const float (&s)[1]) { __stcs(p, s[0]); }
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 3)
decode_tokens_kernel(const T* __restrict__ x, const T* __restrict__ conv_w, T* __restrict__ conv_state,
                     const float* __restrict__ g, const float* __restrict__ beta,
                     float* __restrict__ state, T* __restrict__ o, int32_t Hk, int32_t Hv,
                     int32_t n_tok, float scale) {
  constexpr int VEC = D >= 32 ? D / 32 : 1;
  const int G = Hv / Hk;
  const int32_t Cc = 2 * Hk * D + Hv * D;
  const int64_t b = blockIdx.x / Hk;
  const int hk = blockIdx.x % Hk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_local = (2 + G) * D;        // q | k | v of the G heads

  extern __shared__ float smem[];
  float* ys = smem;                       // [n_tok][n_local]
  float* os = smem + n_tok * n_local;     // [n_tok][G * D], then k_t.q_t [n_tok]

  // 1. conv + SiLU of every token over this CTA's channels; the taps advance by n_tok.
  for (int lv = threadIdx.x; lv < n_local / 4; lv += kThreads) {
    const int lc = lv * 4;
    int gc;
    if (lc < D) gc = hk * D + lc;
    else if (lc < 2 * D) gc = Hk * D + hk * D + (lc - D);
    else gc = 2 * Hk * D + hk * G * D + (lc - 2 * D);
    float win[3 + kMaxTok][4], wr[16];
    T* cs = conv_state + b * 3 * Cc + gc;
#pragma unroll
    for (int j = 0; j < 3; ++j) VecIO<T, 4>::load(cs + j * Cc, win[j]);
#pragma unroll
    for (int t = 0; t < kMaxTok; ++t) {
      if (t < n_tok) {
        VecIO<T, 4>::load(x + (b * n_tok + t) * Cc + gc, win[3 + t]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) win[3 + t][i] = 0.f;
      }
    }
    VecIO<T, 16>::load(conv_w + (int64_t)gc * 4, wr);
#pragma unroll
    for (int t = 0; t < kMaxTok; ++t) {
      if (t < n_tok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float z = wr[i * 4 + 0] * win[t][i];
          z = fmaf(wr[i * 4 + 1], win[t + 1][i], z);
          z = fmaf(wr[i * 4 + 2], win[t + 2][i], z);
          z = fmaf(wr[i * 4 + 3], win[t + 3][i], z);
          ys[t * n_local + lc + i] = silu(z);
        }
      }
    }
    // new taps: the last three entries of the window, win[n_tok .. n_tok + 2]; those that
    // are new inputs are read again by address (cache hits) rather than picked out of
    // registers by a runtime index
    float nt[3][4];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int e = n_tok + j;
      if (e >= 3) {
        VecIO<T, 4>::load(x + (b * n_tok + (e - 3)) * Cc + gc, nt[j]);
      } else {   // e is 1 or 2 (n_tok < 3): an old tap
#pragma unroll
        for (int i = 0; i < 4; ++i) nt[j][i] = e == 1 ? win[1][i] : win[2][i];
      }
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) VecIO<T, 4>::store(cs + j * Cc, nt[j]);
  }
  __syncthreads();

  // 2. q_t and k_t L2-normalised in place (warp t takes token t), k_t.q_t beside them.
  float* kqs = os + n_tok * G * D;        // [n_tok]
  const bool active = lane * VEC < D;
  if (warp < n_tok) {
    float* yt = ys + warp * n_local;
    float qv[VEC], kv[VEC];
    float qq = 0.f, kk = 0.f, kq = 0.f;
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      qv[j] = active ? yt[lane * VEC + j] : 0.f;
      kv[j] = active ? yt[D + lane * VEC + j] : 0.f;
      qq = fmaf(qv[j], qv[j], qq);
      kk = fmaf(kv[j], kv[j], kk);
      kq = fmaf(kv[j], qv[j], kq);
    }
    qq = warp_sum(qq); kk = warp_sum(kk); kq = warp_sum(kq);
    const float iq = 1.0f / sqrtf(qq + kEps), ik = 1.0f / sqrtf(kk + kEps);
    if (active) {
#pragma unroll
      for (int j = 0; j < VEC; ++j) { yt[lane * VEC + j] = qv[j] * iq; yt[D + lane * VEC + j] = kv[j] * ik; }
    }
    if (lane == 0) kqs[warp] = kq * iq * ik;
  }
  __syncthreads();

  // 3. stream the G * D state rows of this CTA, each through every token.
  const int rows = G * D;
  for (int r0 = warp * kRowUnroll; r0 < rows; r0 += kWarps * kRowUnroll) {
    const int h = hk * G + r0 / D;          // kRowUnroll divides D: one value head per group
    float s[kRowUnroll][VEC];
    float* ptr[kRowUnroll];
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int r = r0 + u;
      ptr[u] = state + ((b * Hv + h) * (int64_t)D + r % D) * D + lane * VEC;
      if (r < rows && active) Row<VEC>::load(ptr[u], s[u]);
      else {
#pragma unroll
        for (int j = 0; j < VEC; ++j) s[u][j] = 0.f;
      }
    }
#pragma unroll
    for (int t = 0; t < kMaxTok; ++t) {
      if (t >= n_tok) break;
      float qh[VEC], kh[VEC];
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        qh[j] = active ? ys[t * n_local + lane * VEC + j] : 0.f;
        kh[j] = active ? ys[t * n_local + D + lane * VEC + j] : 0.f;
      }
      const float kqh = kqs[t];
      float sk[kRowUnroll], sq[kRowUnroll];
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) {
        float a = 0.f, c = 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j) { a = fmaf(s[u][j], kh[j], a); c = fmaf(s[u][j], qh[j], c); }
        sk[u] = a; sq[u] = c;
      }
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
          sk[u] += __shfl_xor_sync(0xffffffffu, sk[u], m);
          sq[u] += __shfl_xor_sync(0xffffffffu, sq[u], m);
        }
      const float alpha = expf(g[(b * n_tok + t) * Hv + h]);
      const float bt = beta[(b * n_tok + t) * Hv + h];
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) {
        const int r = r0 + u;
        const float uu = r < rows ? bt * (ys[t * n_local + 2 * D + r] - alpha * sk[u]) : 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j) s[u][j] = fmaf(alpha, s[u][j], uu * kh[j]);
        if (lane == 0 && r < rows) os[t * rows + r] = scale * fmaf(alpha, sq[u], uu * kqh);
      }
    }
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u)
      if (r0 + u < rows && active) Row<VEC>::store(ptr[u], s[u]);
  }
  __syncthreads();

  // 4. outputs: o[b, t, hk*G .. hk*G+G-1, :] is contiguous per token
  for (int t = 0; t < n_tok; ++t) {
    T* ob = o + ((b * n_tok + t) * Hv + (int64_t)hk * G) * D;
    for (int e = threadIdx.x; e < rows; e += kThreads) ob[e] = from_f<T>(os[t * rows + e]);
  }
}

template <typename T, int D>
cudaError_t launch_typed(const void* x, const void* w, void* cs, const float* g, const float* beta,
                         float* state, void* o, int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv,
                         float scale, cudaStream_t st) {
  const int G = Hv / Hk;
  const size_t smem = sizeof(float) * (size_t)n_tok * ((2 + G) * D + G * D + 1);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_tokens_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)((int64_t)B * Hk));
  decode_tokens_kernel<T, D><<<grid, kThreads, smem, st>>>(
      (const T*)x, (const T*)w, (T*)cs, g, beta, state, (T*)o, Hk, Hv, n_tok, scale);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_d(const void* x, const void* w, void* cs, const float* g, const float* beta,
                     float* state, void* o, int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv,
                     int32_t d, float scale, cudaStream_t st) {
  switch (d) {
    case 16: return launch_typed<T, 16>(x, w, cs, g, beta, state, o, B, n_tok, Hk, Hv, scale, st);
    case 32: return launch_typed<T, 32>(x, w, cs, g, beta, state, o, B, n_tok, Hk, Hv, scale, st);
    case 64: return launch_typed<T, 64>(x, w, cs, g, beta, state, o, B, n_tok, Hk, Hv, scale, st);
    default: return launch_typed<T, 128>(x, w, cs, g, beta, state, o, B, n_tok, Hk, Hv, scale, st);
  }
}

}  // namespace

cudaError_t launch_decode_tokens(int dtype, const void* x, const void* conv_w, void* conv_state,
                                 const float* g, const float* beta, float* state, void* o,
                                 int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv, int32_t d,
                                 float scale, cudaStream_t stream) {
  if (dtype == kF32)
    return launch_d<float>(x, conv_w, conv_state, g, beta, state, o, B, n_tok, Hk, Hv, d, scale, stream);
  return launch_d<bf16>(x, conv_w, conv_state, g, beta, state, o, B, n_tok, Hk, Hv, d, scale, stream);
}

}  // namespace gdn
