// decode_tokens.cu -- n_tok (1..8) consecutive tokens for each of B sequences, conv taps and
// states in place (fp32, or bf16 storage with fp32 arithmetic): a multi-token decode /
// speculative verify step.
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
//  3. the warps stream the state rows (D / 16 lanes per row): per token t, with s the row,
//       sk = s.k_t, sq = s.q_t;  u = beta_t (v_t,i - alpha_t sk);  s <- alpha_t s + u k_t
//       o_t,i = scale (alpha_t sq + u (k_t.q_t))
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kEps = 1e-6f;

// Four consecutive state values, streamed (evict-first): fp32 storage, or bf16 storage
// widened to fp32 for the arithmetic and rounded once on the store.
template <typename S> struct Quad;
template <> struct Quad<float> {
  static __device__ __forceinline__ float4 load(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
  static __device__ __forceinline__ void store(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }
};
template <> struct Quad<bf16> {
  static __device__ __forceinline__ float4 load(const bf16* p) {
    const uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
  static __device__ __forceinline__ void store(bf16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    __stcs(reinterpret_cast<uint2*>(p), make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b)));
  }
};

template <typename T, int D, typename S, int NT>
__global__ void __launch_bounds__(kThreads, 3)
decode_tokens_kernel(const T* __restrict__ x, const T* __restrict__ conv_w, T* __restrict__ conv_state,
                     const float* __restrict__ g, const float* __restrict__ beta,
                     S* __restrict__ state, T* __restrict__ o, int32_t Hk, int32_t Hv, float scale) {
  constexpr int n_tok = NT;
  constexpr int VEC = D >= 32 ? D / 32 : 1;
  const int G = Hv / Hk;
  const int32_t Cc = 2 * Hk * D + Hv * D;
  const int64_t b = blockIdx.x / Hk;
  const int hk = blockIdx.x % Hk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_local = (2 + G) * D;        // q | k | v of the G heads

  extern __shared__ float smem[];
  float* ys = smem;                       // [n_tok][n_local]
  float* os = smem + n_tok * n_local;     // [n_tok][G * D], then k_t.q_t [n_tok], then
                                          // (alpha_t, beta_t) per value head [G][n_tok]

  // 1. conv + SiLU of every token over this CTA's channels; the taps advance by n_tok.
  for (int lv = threadIdx.x; lv < n_local / 4; lv += kThreads) {
    const int lc = lv * 4;
    int gc;
    if (lc < D) gc = hk * D + lc;
    else if (lc < 2 * D) gc = Hk * D + hk * D + (lc - D);
    else gc = 2 * Hk * D + hk * G * D + (lc - 2 * D);
    float win[3 + NT][4], wr[16];
    T* cs = conv_state + b * 3 * Cc + gc;
#pragma unroll
    for (int j = 0; j < 3; ++j) VecIO<T, 4>::load(cs + j * Cc, win[j]);
#pragma unroll
    for (int t = 0; t < NT; ++t) VecIO<T, 4>::load(x + (b * n_tok + t) * Cc + gc, win[3 + t]);
    VecIO<T, 16>::load(conv_w + (int64_t)gc * 4, wr);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      {
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
  // the decay and write strength of each (value head, token), once per CTA
  float2* ab = reinterpret_cast<float2*>(kqs + ((n_tok + 1) & ~1));   // 8-byte aligned
  for (int i = threadIdx.x; i < G * n_tok; i += kThreads) {
    const int hh = i / n_tok, t = i % n_tok;
    const int64_t gi = (b * n_tok + t) * Hv + hk * G + hh;
    ab[i] = make_float2(expf(g[gi]), beta[gi]);
  }
  __syncthreads();

  // 3. stream the G * D state rows of this CTA, each through every token. A row is split
  //    over L = D / 16 lanes of 16 columns each, so its dot products need log2(L) shuffle
  //    rounds; a warp takes 32 / L consecutive rows per pass. Lane seg of a row holds the
  //    float4 columns j * 4L + 4 seg (j < 4): for each of its four loads the row's lanes
  //    cover one contiguous 16L-float span, so every access is a full line.
  //    The next pass's rows are loaded before this pass's tokens run (software pipelining),
  //    so each warp keeps a pass of loads in flight while it computes.
  constexpr int SEG = 16;
  constexpr int L = D / SEG;
  constexpr int RPW = 32 / L;
  const int rows = G * D;
  const int seg = lane % L;
  auto row_ptr = [&](int r) {
    const int rr = r < rows ? r : 0;
    return state + ((b * Hv + hk * G + rr / D) * (int64_t)D + rr % D) * D + seg * 4;
  };
  auto load_row = [&](int r, float (&dst)[SEG]) {
    S* p = row_ptr(r);
#pragma unroll
    for (int j = 0; j < SEG; j += 4) {
      const float4 v = r < rows ? Quad<S>::load(p + j * L) : make_float4(0.f, 0.f, 0.f, 0.f);
      dst[j] = v.x; dst[j + 1] = v.y; dst[j + 2] = v.z; dst[j + 3] = v.w;
    }
  };
  float s_next[SEG];
  load_row(warp * RPW + lane / L, s_next);
  for (int r0 = warp * RPW; r0 < rows; r0 += kWarps * RPW) {
    const int r = r0 + lane / L;
    const bool live = r < rows;
    const float2* abh = ab + ((live ? r : 0) / D) * n_tok;   // this row's value head
    S* ptr = row_ptr(r);
    float s[SEG];
#pragma unroll
    for (int j = 0; j < SEG; ++j) s[j] = s_next[j];
    if (r0 + kWarps * RPW < rows) load_row(r + kWarps * RPW, s_next);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const float* qt = ys + t * n_local + seg * 4;
      const float* kt = qt + D;
      float kv[SEG], a = 0.f, c = 0.f;
#pragma unroll
      for (int j = 0; j < SEG; j += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(kt + j * L);
        const float4 q4 = *reinterpret_cast<const float4*>(qt + j * L);
        kv[j] = k4.x; kv[j + 1] = k4.y; kv[j + 2] = k4.z; kv[j + 3] = k4.w;
        a = fmaf(s[j], k4.x, a); a = fmaf(s[j + 1], k4.y, a); a = fmaf(s[j + 2], k4.z, a); a = fmaf(s[j + 3], k4.w, a);
        c = fmaf(s[j], q4.x, c); c = fmaf(s[j + 1], q4.y, c); c = fmaf(s[j + 2], q4.z, c); c = fmaf(s[j + 3], q4.w, c);
      }
#pragma unroll
      for (int m = L / 2; m >= 1; m >>= 1) {   // within the row's L lanes
        a += __shfl_xor_sync(0xffffffffu, a, m);
        c += __shfl_xor_sync(0xffffffffu, c, m);
      }
      if (live) {
        const float2 sc = abh[t];
        const float alpha = sc.x, bt = sc.y;
        const float uu = bt * (ys[t * n_local + 2 * D + r] - alpha * a);
#pragma unroll
        for (int j = 0; j < SEG; ++j) s[j] = fmaf(alpha, s[j], uu * kv[j]);
        if (seg == 0) os[t * rows + r] = scale * fmaf(alpha, c, uu * kqs[t]);
      }
    }
    if (live) {
#pragma unroll
      for (int j = 0; j < SEG; j += 4)
        Quad<S>::store(ptr + j * L, make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]));
    }
  }
  __syncthreads();

  // 4. outputs: o[b, t, hk*G .. hk*G+G-1, :] is contiguous per token
  for (int t = 0; t < n_tok; ++t) {
    T* ob = o + ((b * n_tok + t) * Hv + (int64_t)hk * G) * D;
    for (int e = threadIdx.x; e < rows; e += kThreads) ob[e] = from_f<T>(os[t * rows + e]);
  }
}

template <typename T, int D, typename S, int NT>
cudaError_t launch_nt(const void* x, const void* w, void* cs, const float* g, const float* beta,
                      void* state, void* o, int32_t B, int32_t Hk, int32_t Hv, float scale, cudaStream_t st) {
  const int G = Hv / Hk;
  // ys, os, k_t.q_t (padded to an even count), (alpha, beta) per value head and token
  const size_t smem = sizeof(float) * ((size_t)NT * ((2 + G) * D + G * D) + ((NT + 1) & ~1) + 2 * (size_t)G * NT);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_tokens_kernel<T, D, S, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)((int64_t)B * Hk));
  decode_tokens_kernel<T, D, S, NT><<<grid, kThreads, smem, st>>>(
      (const T*)x, (const T*)w, (T*)cs, g, beta, (S*)state, (T*)o, Hk, Hv, scale);
  return cudaGetLastError();
}

// the token count is a template parameter, so the per-token loops are unrolled
template <typename T, int D, typename S>
cudaError_t launch_typed(const void* x, const void* w, void* cs, const float* g, const float* beta,
                         void* state, void* o, int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv,
                         float scale, cudaStream_t st) {
  switch (n_tok) {
    case 1: return launch_nt<T, D, S, 1>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    case 2: return launch_nt<T, D, S, 2>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    case 3: return launch_nt<T, D, S, 3>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    case 4: return launch_nt<T, D, S, 4>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    case 5: return launch_nt<T, D, S, 5>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    case 6: return launch_nt<T, D, S, 6>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    case 7: return launch_nt<T, D, S, 7>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
    default: return launch_nt<T, D, S, 8>(x, w, cs, g, beta, state, o, B, Hk, Hv, scale, st);
  }
}

template <typename T, typename S>
cudaError_t launch_d(const void* x, const void* w, void* cs, const float* g, const float* beta,
                     void* state, void* o, int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv,
                     int32_t d, float scale, cudaStream_t st) {
  switch (d) {
    case 16: return launch_typed<T, 16, S>(x, w, cs, g, beta, state, o, B, n_tok, Hk, Hv, scale, st);
    case 32: return launch_typed<T, 32, S>(x, w, cs, g, beta, state, o, B, n_tok, Hk, Hv, scale, st);
    case 64: return launch_typed<T, 64, S>(x, w, cs, g, beta, state, o, B, n_tok, Hk, Hv, scale, st);
    default: return launch_typed<T, 128, S>(x, w, cs, g, beta, state, o, B, n_tok, Hk, Hv, scale, st);
  }
}

}  // namespace

cudaError_t launch_decode_tokens(int dtype, const void* x, const void* conv_w, void* conv_state,
                                 const float* g, const float* beta, void* state, int state_dtype,
                                 void* o, int32_t B, int32_t n_tok, int32_t Hk, int32_t Hv, int32_t d,
                                 float scale, cudaStream_t stream) {
  if (dtype == kF32) {
    if (state_dtype == kF32)
      return launch_d<float, float>(x, conv_w, conv_state, g, beta, state, o, B, n_tok, Hk, Hv, d, scale, stream);
    return launch_d<float, bf16>(x, conv_w, conv_state, g, beta, state, o, B, n_tok, Hk, Hv, d, scale, stream);
  }
  if (state_dtype == kF32)
    return launch_d<bf16, float>(x, conv_w, conv_state, g, beta, state, o, B, n_tok, Hk, Hv, d, scale, stream);
  return launch_d<bf16, bf16>(x, conv_w, conv_state, g, beta, state, o, B, n_tok, Hk, Hv, d, scale, stream);
}

}  // namespace gdn
