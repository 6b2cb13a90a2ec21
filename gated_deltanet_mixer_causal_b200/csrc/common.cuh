// common.cuh -- small device helpers shared by the libgdn kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

typedef __nv_bfloat16 bf16;

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// (a, b) as a bf16 pair hi (nearest, ties to even) and the bf16 pair lo of what hi left out,
// so hi + lo carries about 16 significant bits: one paired conversion for each, the
// widening of hi back to fp32 by bit operations.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  hi = *reinterpret_cast<uint32_t*>(&h);
  __nv_bfloat162 l = __floats2bfloat162_rn(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xFFFF0000u));
  lo = *reinterpret_cast<uint32_t*>(&l);
}

// The same split without the conversion unit (integer and fp32 ALU only): hi is x rounded
// to the nearest bf16 by adding half a bf16 unit in the last place to the bit pattern (half-way
// cases go away from zero), lo = x - hi (exact in fp32) truncated to bf16, so
// |x - hi - lo| < 2^-15 |x|.
__device__ __forceinline__ void split_bf16x2_alu(float a, float b, uint32_t& hi, uint32_t& lo) {
  const uint32_t ha = (__float_as_uint(a) + 0x8000u) & 0xFFFF0000u;
  const uint32_t hb = (__float_as_uint(b) + 0x8000u) & 0xFFFF0000u;
  hi = __byte_perm(ha, hb, 0x7632);
  lo = __byte_perm(__float_as_uint(a - __uint_as_float(ha)), __float_as_uint(b - __uint_as_float(hb)), 0x7632);
}

// Recurrent-state elements in HBM: fp32, or bf16 storage (widened to fp32 on load, rounded
// to nearest-even once on store).
__device__ __forceinline__ float state_load(const void* p, int64_t i, bool bf) {
  return bf ? __bfloat162float(static_cast<const bf16*>(p)[i]) : static_cast<const float*>(p)[i];
}
__device__ __forceinline__ void state_store(void* p, int64_t i, float v, bool bf) {
  if (bf) static_cast<bf16*>(p)[i] = __float2bfloat16_rn(v);
  else static_cast<float*>(p)[i] = v;
}

// N contiguous elements starting at p (p aligned to N * sizeof(T)), widened to fp32.
template <typename T, int N> struct VecIO;

template <int N> struct VecIO<float, N> {
  static __device__ __forceinline__ void load(const float* p, float (&o)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 4) {
        float4 v = *reinterpret_cast<const float4*>(p + i);
        o[i] = v.x; o[i + 1] = v.y; o[i + 2] = v.z; o[i + 3] = v.w;
      }
    } else if constexpr (N == 2) {
      float2 v = *reinterpret_cast<const float2*>(p);
      o[0] = v.x; o[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) o[i] = p[i];
    }
  }
  static __device__ __forceinline__ void store(float* p, const float (&o)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 4)
        *reinterpret_cast<float4*>(p + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
    } else if constexpr (N == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(o[0], o[1]);
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) p[i] = o[i];
    }
  }
};

template <int N> struct VecIO<bf16, N> {
  static __device__ __forceinline__ void load(const bf16* p, float (&o)[N]) {
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 8) {
        uint4 u = *reinterpret_cast<const uint4*>(p + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
          o[i + 2 * j] = f.x; o[i + 2 * j + 1] = f.y;
        }
      }
    } else if constexpr (N == 4) {
      uint2 u = *reinterpret_cast<const uint2*>(p);
      float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
      o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    } else if constexpr (N == 2) {
      float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
      o[0] = a.x; o[1] = a.y;
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) o[i] = __bfloat162float(p[i]);
    }
  }
  static __device__ __forceinline__ void store(bf16* p, const float (&o)[N]) {
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 8) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __nv_bfloat162 h = __floats2bfloat162_rn(o[i + 2 * j], o[i + 2 * j + 1]);
          w[j] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p + i) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else if constexpr (N == 4) {
      __nv_bfloat162 a = __floats2bfloat162_rn(o[0], o[1]);
      __nv_bfloat162 b = __floats2bfloat162_rn(o[2], o[3]);
      *reinterpret_cast<uint2*>(p) =
          make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
    } else if constexpr (N == 2) {
      *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(o[0], o[1]);
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) p[i] = __float2bfloat16_rn(o[i]);
    }
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

// z * sigmoid(z); the fast reciprocal (about 2 ulp) is ample for bf16 and the 1e-4 fp32 gate.
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// Sequence bounds with every value clamped into [0, T], so that a malformed cu_seqlens
// can give wrong answers but never an out-of-range access.
__device__ __forceinline__ void seq_bounds(const int32_t* cu, int32_t n, int64_t T, int64_t& bos,
                                           int64_t& eos) {
  if (cu == nullptr) { bos = 0; eos = T; return; }
  int64_t a = cu[n], b = cu[n + 1];
  a = a < 0 ? 0 : (a > T ? T : a);
  b = b < a ? a : (b > T ? T : b);
  bos = a; eos = b;
}

}  // namespace gdn
