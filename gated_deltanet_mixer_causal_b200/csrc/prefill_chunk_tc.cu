// prefill_chunk_tc.cu -- chunked gated delta rule on tcgen05 tensor cores (bf16, d = 128).
//
// The recurrence (Qwen3.5 page, section 5: decay, then the delta write along k) is
// evaluated 64 tokens at a time in its WY / UT form. Within a chunk starting from state
// S0, with G_r the in-chunk cumulative log-decay and unit keys k_r (L2 norm folded in):
//
//   A_ri = beta_r e^{G_r - G_i} k_r.k_i  (i < r),   Tm = (I + A)^{-1}
//   U    = Tm diag(beta) V - Tm diag(beta e^G) K S0^T          (the chunk's delta writes)
//   O    = diag(e^G) Q S0^T + (M o Q K^T) U,   M_ri = e^{G_r - G_i} (i <= r)
//   S    = e^{G_L} S0 + U^T diag(e^{G_L - G}) K
//
// Three kernels:
//  1. plan  : chunk offsets of every packed sequence (chunks never straddle sequences).
//  2. intra : one CTA per (chunk, key head): TMA loads q, k; tcgen05 computes K K^T and
//             Q K^T in TMEM; per value head the decay-masked A and M o QK^T, the unit lower
//             triangular inverse Tm (fp32, 16x16 diagonal blocks by warps, then block
//             products), and writes P = Tm diag(beta), Pk = Tm diag(beta e^G / |k|) and
//             Mqk = M o QK^T / (|q||k|) (bf16) plus row scales to the workspace.
//  3. chain : one CTA per (sequence, value head, 64-wide slice of dv): walks the chunks in
//             order with the fp32 state slice in registers (its bf16 copy in shared memory
//             feeds the MMAs), five tcgen05 GEMMs per chunk:
//               W = Pk K,  U = P V - W S0^T,  O1 = Q S0^T,  O2 = Mqk U,  dS^T = K^T U'
//             and writes o = scale (e^{G_r}/|q_r| O1 + O2). Inputs for chunk c+1 stream in
//             by TMA while chunk c computes.
// Operands are staged in shared memory in the 128-byte-swizzled layouts TMA writes; K-major
// and MN-major descriptors read the same q/k/v tiles. Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = 64;        // chunk length
constexpr int D = 128;       // head dim (dk = dv)
constexpr int DT = 64;       // dv slice per chain CTA
constexpr int NT = D / DT;   // slices per head
constexpr float kEps = 1e-6f;
constexpr int kMatBytes = C * C * 2;   // one 64x64 bf16 matrix

// error codes recorded in the workspace's error word
constexpr int kErrIntraTma = 11, kErrIntraMma = 12, kErrChainTma = 21, kErrChainMma = 22;

// ------------------------------------------------------------------ workspace layout

struct Ws {
  size_t err, prefix, mats, vecs, last, total;
};

__host__ __device__ inline int64_t max_slots(int64_t T, int32_t n_seq) { return (T + C - 1) / C + n_seq; }

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ __device__ inline Ws ws_layout(int64_t T, int32_t n_seq, int32_t Hv) {
  Ws w;
  const size_t slots = (size_t)max_slots(T, n_seq);
  w.err = 0;
  w.prefix = 256;
  w.mats = align256(w.prefix + (size_t)(n_seq + 1) * 4);
  w.vecs = align256(w.mats + slots * Hv * 3 * kMatBytes);
  w.last = align256(w.vecs + slots * Hv * 2 * C * 4);
  w.total = align256(w.last + slots * Hv * 4);
  return w;
}

// --------------------------------------------------------------------------- plan

__global__ void __launch_bounds__(1024) chunk_plan_kernel(const int32_t* __restrict__ cu,
                                                          int32_t n_seq, int64_t T,
                                                          int32_t* __restrict__ prefix,
                                                          int* __restrict__ err) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) { carry = 0; *err = 0; }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int base = 0; base < n_seq; base += blockDim.x) {
    const int n = base + threadIdx.x;
    int cnt = 0;
    if (n < n_seq) {
      int64_t b, e;
      seq_bounds(cu, n, T, b, e);
      cnt = (int)((e - b + C - 1) / C);
    }
    int x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
      int s = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_tot[lane] = s;
    }
    __syncthreads();
    const int incl = carry + x + (w > 0 ? warp_tot[w - 1] : 0);
    if (n < n_seq) prefix[n] = incl - cnt;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) prefix[n_seq] = carry;
}

// Largest n in [0, n_seq) with prefix[n] <= slot.
__device__ __forceinline__ int32_t slot_to_seq(const int32_t* prefix, int32_t n_seq, int32_t slot) {
  int32_t lo = 0, hi = n_seq - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= slot) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------ MMA descriptors

// K-major operand: [rows][128-byte swizzled row] atoms of 64 columns, atoms atom_bytes
// apart; kk-th K step of 16 elements.
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int kk, uint32_t atom_bytes) {
  return smem_desc(base + (uint32_t)(kk >> 2) * atom_bytes + (uint32_t)(kk & 3) * 32u, 16u, 1024u);
}
// MN-major operand: rows are the K index (128 bytes = 64 MN elements each), MN atoms
// atom_bytes apart; kk-th K step = 16 rows.
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int kk, uint32_t atom_bytes) {
  return smem_desc(base + (uint32_t)kk * 2048u, atom_bytes, 1024u);
}

// Row r (0..63) of an M = 64 accumulator lives in TMEM lane 32 * (r / 16) + r % 16.
__device__ __forceinline__ uint32_t tmem_quadrant(uint32_t tmem, int warp) {
  return tmem + ((uint32_t)(warp * 32) << 16);
}

// ------------------------------------------------------------------------ intra

// shared memory of the intra kernel (offsets from a 1024-aligned base)
constexpr int kIQ = 0;                          // q tile: 2 atoms x 8 KB
constexpr int kIK = 16384;                      // k tile: 2 atoms x 8 KB
constexpr int kIA = 32768;                      // A   fp32 [64][65]
constexpr int kIT = kIA + 64 * 65 * 4;          // Tm  fp32 [64][65]
constexpr int kITmp = kIT + 64 * 65 * 4;        // block-product scratch fp32 [3][16][17]
constexpr int kIVec = kITmp + 3 * 16 * 17 * 4;  // rq, rk, G, beta  [4][64] fp32
constexpr int kIBar = kIVec + 4 * 64 * 4;       // 2 mbarriers + tmem address
constexpr int kIntraSmem = kIBar + 64 + 1024;   // + alignment slack

__global__ void __launch_bounds__(128)
chunk_intra_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const float* __restrict__ g, const float* __restrict__ beta,
                   const int32_t* __restrict__ cu, int32_t n_seq, int64_t T, int32_t Hk, int32_t Hv,
                   uint8_t* __restrict__ ws) {
  const Ws L = ws_layout(T, n_seq, Hv);
  int* err = reinterpret_cast<int*>(ws + L.err);
  const int32_t* prefix = reinterpret_cast<const int32_t*>(ws + L.prefix);
  const int32_t slot = blockIdx.x, hk = blockIdx.y;
  if (slot >= prefix[n_seq]) return;
  const int32_t n = slot_to_seq(prefix, n_seq, slot);
  int64_t bos, eos;
  seq_bounds(cu, n, T, bos, eos);
  const int64_t t0 = bos + (int64_t)(slot - prefix[n]) * C;
  const int len = (int)(eos - t0 < C ? eos - t0 : C);
  const int G = Hv / Hk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float(*A)[65] = reinterpret_cast<float(*)[65]>(sm + kIA);
  float(*Tm)[65] = reinterpret_cast<float(*)[65]>(sm + kIT);
  float(*tmp)[16][17] = reinterpret_cast<float(*)[16][17]>(sm + kITmp);
  float* rq = reinterpret_cast<float*>(sm + kIVec);
  float* rk = rq + 64;
  float* sG = rq + 128;
  float* sb = rq + 192;
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + kIBar);
  uint64_t* bar_mma = bar_tma + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 2);

  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(tmem_slot, 128); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_tma, 4 * 8192);
    for (int hh = 0; hh < 2; ++hh) {
      tma_load_2d(sm + kIQ + hh * 8192, &map_q, hk * D + hh * 64, (int32_t)t0, bar_tma);
      tma_load_2d(sm + kIK + hh * 8192, &map_k, hk * D + hh * 64, (int32_t)t0, bar_tma);
    }
  }
  bool ok = mbar_wait(bar_tma, 0, err, kErrIntraTma);
  if (__syncthreads_or(!ok)) goto teardown;

  {  // inverse L2 norms of the chunk's q and k rows (0 for rows past the sequence end)
    const int r = tid & 63;
    const uint8_t* tile = sm + (tid < 64 ? kIQ : kIK);
    float ss = 0.f;
    for (int hh = 0; hh < 2; ++hh)
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint4 u = *reinterpret_cast<const uint4*>(tile + hh * 8192 + sw128_off(r, c8 * 8));
        const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[j]));
          ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
        }
      }
    const float inv = r < len ? 1.0f / sqrtf(ss + kEps) : 0.f;
    (tid < 64 ? rq : rk)[r] = inv;
  }

  if (tid == 0) {   // K K^T -> TMEM cols [0, 64), Q K^T -> cols [64, 128); M = N = 64, K = 128
    tc_fence_after();
    const uint32_t q0 = smem_u32(sm + kIQ), k0 = smem_u32(sm + kIK);
    const uint32_t id = idesc_bf16(64, 64, 0, 0);
    for (int kk = 0; kk < 8; ++kk) mma_bf16(tmem, desc_k(k0, kk, 8192), desc_k(k0, kk, 8192), id, kk > 0);
    for (int kk = 0; kk < 8; ++kk) mma_bf16(tmem + 64, desc_k(q0, kk, 8192), desc_k(k0, kk, 8192), id, kk > 0);
    mma_commit(bar_mma);
  }
  ok = mbar_wait(bar_mma, 0, err, kErrIntraMma);
  if (__syncthreads_or(!ok)) goto teardown;
  tc_fence_after();

  for (int j = 0; j < G; ++j) {
    const int h = hk * G + j;
    if (tid < 64) {
      const bool v = tid < len;
      sG[tid] = v ? g[(t0 + tid) * Hv + h] : 0.f;
      sb[tid] = v ? beta[(t0 + tid) * Hv + h] : 0.f;
    }
    __syncthreads();
    if (warp == 0) {   // inclusive cumulative log-decay over the chunk (2 values per lane)
      float a0 = sG[2 * lane], a1 = sG[2 * lane + 1];
      float s = a0 + a1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      const float excl = s - (a0 + a1);
      sG[2 * lane] = excl + a0;
      sG[2 * lane + 1] = excl + a0 + a1;
    }
    __syncthreads();

    // rows of A (from K K^T) and of Mqk (from Q K^T): lane l < 16 of warp w owns row 16w+l
    {
      const int r = warp * 16 + lane;
      const bool own = lane < 16;
      const float Gr = own ? sG[r] : 0.f, br = own ? sb[r] : 0.f;
      const float rkr = own ? rk[r] : 0.f, rqr = own ? rq[r] : 0.f;
      uint8_t* mq = ws + L.mats + ((size_t)(slot * Hv + h) * 3 + 2) * kMatBytes;
      for (int cb = 0; cb < 2; ++cb) {
        float kkv[32], qkv[32];
        tmem_ld32(tmem_quadrant(tmem, warp) + cb * 32, kkv);
        tmem_ld32(tmem_quadrant(tmem, warp) + 64 + cb * 32, qkv);
        if (own) {
          float mrow[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int i = cb * 32 + e;
            const float dec = (i <= r) ? expf(Gr - sG[i]) : 0.f;
            A[r][i] = (i < r) ? br * dec * rkr * rk[i] * kkv[e] : 0.f;
            mrow[e] = dec * rqr * rk[i] * qkv[e];
          }
          VecIO<bf16, 32>::store(reinterpret_cast<bf16*>(mq) + r * C + cb * 32, mrow);
        }
      }
    }
    __syncthreads();

    // Tm = (I + A)^{-1}: diagonal 16x16 blocks by forward substitution, one warp each
    {
      const int b0 = warp * 16;
      const int jc = lane & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float s = (r == jc) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < r; ++i) s = fmaf(-A[b0 + r][b0 + i], x[i], s);
        x[r] = s;
      }
      if (lane < 16) {
#pragma unroll
        for (int r = 0; r < 16; ++r) Tm[b0 + r][b0 + jc] = x[r];
      }
      // blocks above the diagonal are zero
      for (int e = lane; e < 16 * 64; e += 32) {
        const int r = e >> 6, c = e & 63;
        if (c >= b0 + 16) Tm[b0 + r][c] = 0.f;
      }
    }
    __syncthreads();
    // off-diagonal blocks: Tm_ba = -Tm_bb sum_{c=a}^{b-1} A_bc Tm_ca, by block distance
    for (int dist = 1; dist < 4; ++dist) {
      const int npair = 4 - dist;
      for (int e = tid; e < npair * 256; e += 128) {
        const int p = e >> 8, r = (e >> 4) & 15, col = e & 15;
        const int bb = p + dist, aa = p;
        float s = 0.f;
        for (int cblk = aa; cblk < bb; ++cblk)
#pragma unroll
          for (int k = 0; k < 16; ++k) s = fmaf(A[16 * bb + r][16 * cblk + k], Tm[16 * cblk + k][16 * aa + col], s);
        tmp[p][r][col] = s;
      }
      __syncthreads();
      for (int e = tid; e < npair * 256; e += 128) {
        const int p = e >> 8, r = (e >> 4) & 15, col = e & 15;
        const int bb = p + dist, aa = p;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) s = fmaf(Tm[16 * bb + r][16 * bb + k], tmp[p][k][col], s);
        Tm[16 * bb + r][16 * aa + col] = -s;
      }
      __syncthreads();
    }

    // P = Tm diag(beta), Pk = Tm diag(beta e^G |k|^-1), row scales
    {
      uint8_t* base = ws + L.mats + (size_t)(slot * Hv + h) * 3 * kMatBytes;
      for (int e = tid; e < 64 * 8; e += 128) {     // (row, 8-column group)
        const int r = e >> 3, c0 = (e & 7) * 8;
        float pv[8], pk[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int i = c0 + q;
          const float t = Tm[r][i] * sb[i];
          pv[q] = t;
          pk[q] = t * expf(sG[i]) * rk[i];
        }
        VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(base) + r * C + c0, pv);
        VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(base + kMatBytes) + r * C + c0, pk);
      }
      float* vec = reinterpret_cast<float*>(ws + L.vecs) + (size_t)(slot * Hv + h) * 2 * C;
      const float Gl = sG[C - 1];
      if (tid < 64) vec[tid] = expf(sG[tid]) * rq[tid];
      else vec[tid] = expf(Gl - sG[tid - 64]) * rk[tid - 64];
      if (tid == 0) reinterpret_cast<float*>(ws + L.last)[slot * Hv + h] = expf(Gl);
    }
    __syncthreads();
  }

teardown:
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// ------------------------------------------------------------------------ chain

// shared memory of the chain kernel (offsets from a 1024-aligned base)
constexpr int kStage = 65536;                 // one chunk's TMA inputs
constexpr int kSK = 0, kSQ = 16384, kSV = 32768, kSP = 40960, kSPk = 49152, kSM = 57344;
constexpr int kCW = 2 * kStage;               // -W as bf16, K-major [64][128]: 16 KB
constexpr int kCS = kCW + 16384;              // S0^T bf16, MN-major [128][64]: 16 KB
constexpr int kCU = kCS + 16384;              // U   bf16 [64][64]: 8 KB
constexpr int kCU2 = kCU + 8192;              // U'  bf16 [64][64]: 8 KB
constexpr int kCVec = kCU2 + 8192;            // o_scale, u_scale fp32 [2][64]
constexpr int kCBar = kCVec + 512;            // 3 mbarriers + tmem address
constexpr int kChainSmem = kCBar + 64 + 1024;

// TMEM columns
constexpr uint32_t kTW = 0, kTU = 128, kTO1 = 192, kTO2 = 256, kTdS = 320;

__global__ void __launch_bounds__(128, 1)
chunk_chain_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_ws,
                   const int32_t* __restrict__ cu, int32_t n_seq, int64_t T, int32_t Hk, int32_t Hv,
                   const uint8_t* __restrict__ ws_ro, int* err_word, const float* init, float* fin,
                   bf16* __restrict__ o, float scale) {
  const Ws L = ws_layout(T, n_seq, Hv);
  const int32_t* prefix = reinterpret_cast<const int32_t*>(ws_ro + L.prefix);
  const int tile = blockIdx.x % NT;
  const int h = (blockIdx.x / NT) % Hv;
  const int32_t n = blockIdx.x / (NT * Hv);
  const int hk = h / (Hv / Hk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t bos, eos;
  seq_bounds(cu, n, T, bos, eos);
  const int nc = (int)((eos - bos + C - 1) / C);
  const int32_t slot0 = prefix[n];

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_os = reinterpret_cast<float*>(sm + kCVec);
  float* s_us = s_os + 64;
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + kCBar);   // [2]
  uint64_t* bar_mma = bar_tma + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 3);

  if (tid == 0) {
    mbar_init(&bar_tma[0], 1);
    mbar_init(&bar_tma[1], 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    if (nc > 0) {
      tma_prefetch_desc(&map_q); tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v); tma_prefetch_desc(&map_ws);
    }
  }
  if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }

  // state slice: thread t holds column t of S for rows tile*DT .. +DT (i.e. row t of S^T)
  float s[DT];
  const int64_t sbase = ((int64_t)n * Hv + h) * D * D + (int64_t)tile * DT * D;
#pragma unroll
  for (int j = 0; j < DT; ++j) s[j] = init ? init[sbase + (int64_t)j * D + tid] : 0.f;
  {
    uint8_t* st = sm + kCS;
#pragma unroll
    for (int c8 = 0; c8 < DT / 8; ++c8) {
      float v8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v8[q] = s[c8 * 8 + q];
      VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(st + sw128_off(tid, c8 * 8)), v8);
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto issue_loads = [&](int c, int b) {
    const int64_t t0 = bos + (int64_t)c * C;
    const int32_t slot = slot0 + c;
    uint8_t* stg = sm + b * kStage;
    mbar_arrive_expect_tx(&bar_tma[b], kStage);
    for (int hh = 0; hh < 2; ++hh) {
      tma_load_2d(stg + kSK + hh * 8192, &map_k, hk * D + hh * 64, (int32_t)t0, &bar_tma[b]);
      tma_load_2d(stg + kSQ + hh * 8192, &map_q, hk * D + hh * 64, (int32_t)t0, &bar_tma[b]);
    }
    tma_load_2d(stg + kSV, &map_v, h * D + tile * DT, (int32_t)t0, &bar_tma[b]);
    const int32_t row = (int32_t)(((int64_t)slot * Hv + h) * 3 * C);
    tma_load_2d(stg + kSP, &map_ws, 0, row, &bar_tma[b]);
    tma_load_2d(stg + kSPk, &map_ws, 0, row + C, &bar_tma[b]);
    tma_load_2d(stg + kSM, &map_ws, 0, row + 2 * C, &bar_tma[b]);
  };

  if (tid == 0 && nc > 0) issue_loads(0, 0);
  uint32_t ph_tma[2] = {0u, 0u}, ph_mma = 0u;
  bool ok = true;
  const float* vecs = reinterpret_cast<const float*>(ws_ro + L.vecs);
  const float* lastv = reinterpret_cast<const float*>(ws_ro + L.last);

  for (int c = 0; c < nc; ++c) {
    const int b = c & 1;
    const int64_t t0 = bos + (int64_t)c * C;
    const int len = (int)(eos - t0 < C ? eos - t0 : C);
    const int32_t slot = slot0 + c;
    if (tid == 0 && c + 1 < nc) issue_loads(c + 1, b ^ 1);
    {
      const float* v = vecs + (size_t)(slot * Hv + h) * 2 * C;
      if (tid < 64) s_os[tid] = v[tid]; else s_us[tid - 64] = v[tid];
    }
    const float decay_last = lastv[slot * Hv + h];
    ok = mbar_wait(&bar_tma[b], ph_tma[b], err_word, kErrChainTma);
    ph_tma[b] ^= 1u;
    if (__syncthreads_or(!ok)) break;

    uint8_t* stg = sm + b * kStage;
    const uint32_t aK = smem_u32(stg + kSK), aQ = smem_u32(stg + kSQ), aV = smem_u32(stg + kSV);
    const uint32_t aP = smem_u32(stg + kSP), aPk = smem_u32(stg + kSPk), aM = smem_u32(stg + kSM);
    const uint32_t aW = smem_u32(sm + kCW), aS = smem_u32(sm + kCS);
    const uint32_t aU = smem_u32(sm + kCU), aU2 = smem_u32(sm + kCU2);

    // round 1: W = Pk K (64 x 128), U = P V (64 x 64)
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kTW, desc_k(aPk, kk, 0), desc_mn(aK, kk, 8192), idesc_bf16(64, 128, 0, 1), kk > 0);
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kTU, desc_k(aP, kk, 0), desc_mn(aV, kk, 8192), idesc_bf16(64, DT, 0, 1), kk > 0);
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, ph_mma, err_word, kErrChainMma);
    ph_mma ^= 1u;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    {  // W -> bf16, K-major [64 rows][128]
      const int r = warp * 16 + lane;
      for (int cb = 0; cb < 4; ++cb) {
        float v[32];
        tmem_ld32(tmem_quadrant(tmem, warp) + kTW + cb * 32, v);
        if (lane < 16) {
          uint8_t* atom = sm + kCW + (cb >> 1) * 8192;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float v8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v8[q] = v[c8 * 8 + q];
            VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(atom + sw128_off(r, (cb & 1) * 32 + c8 * 8)), v8);
          }
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // round 2: U += (-W) S0^T, O1 = Q S0^T   (K = 128)
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kTU, desc_k(aW, kk, 8192), desc_mn(aS, kk, 0), idesc_bf16(64, DT, 0, 1, 1), true);
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kTO1, desc_k(aQ, kk, 8192), desc_mn(aS, kk, 0), idesc_bf16(64, DT, 0, 1), kk > 0);
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, ph_mma, err_word, kErrChainMma);
    ph_mma ^= 1u;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    {  // U and U' = diag(e^{G_L - G} / |k|) U as bf16 [64 tokens][64]
      const int r = warp * 16 + lane;
      const float us = lane < 16 ? s_us[r] : 0.f;
      for (int cb = 0; cb < DT / 32; ++cb) {
        float v[32];
        tmem_ld32(tmem_quadrant(tmem, warp) + kTU + cb * 32, v);
        if (lane < 16) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float v8[8], w8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) { v8[q] = v[c8 * 8 + q]; w8[q] = us * v8[q]; }
            const uint32_t off = sw128_off(r, cb * 32 + c8 * 8);
            VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(sm + kCU + off), v8);
            VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(sm + kCU2 + off), w8);
          }
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // round 3: O2 = Mqk U (K = 64), dS^T = K^T U' (M = 128, K = 64)
    if (tid == 0) {
      tc_fence_after();
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kTO2, desc_k(aM, kk, 0), desc_mn(aU, kk, 0), idesc_bf16(64, DT, 0, 1), kk > 0);
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kTdS, desc_mn(aK, kk, 8192), desc_mn(aU2, kk, 0), idesc_bf16(128, DT, 1, 1), kk > 0);
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, ph_mma, err_word, kErrChainMma);
    ph_mma ^= 1u;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    {  // state: S^T row tid <- e^{G_L} S^T + dS^T; refresh the bf16 copy
      for (int cb = 0; cb < DT / 32; ++cb) {
        float v[32];
        tmem_ld32(tmem_quadrant(tmem, warp) + kTdS + cb * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[cb * 32 + e] = fmaf(decay_last, s[cb * 32 + e], v[e]);
      }
#pragma unroll
      for (int c8 = 0; c8 < DT / 8; ++c8) {
        float v8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v8[q] = s[c8 * 8 + q];
        VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(sm + kCS + sw128_off(tid, c8 * 8)), v8);
      }
    }
    {  // outputs: o_r = scale (e^{G_r}/|q_r| O1_r + O2_r)
      const int r = warp * 16 + lane;
      const float os = lane < 16 ? s_os[r] : 0.f;
      for (int cb = 0; cb < DT / 32; ++cb) {
        float v1[32], v2[32];
        tmem_ld32(tmem_quadrant(tmem, warp) + kTO1 + cb * 32, v1);
        tmem_ld32(tmem_quadrant(tmem, warp) + kTO2 + cb * 32, v2);
        if (lane < 16 && r < len) {
          bf16* dst = o + ((t0 + r) * Hv + h) * (int64_t)D + tile * DT + cb * 32;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float v8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v8[q] = scale * fmaf(os, v1[c8 * 8 + q], v2[c8 * 8 + q]);
            VecIO<bf16, 8>::store(dst + c8 * 8, v8);
          }
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (ok && fin != nullptr) {
#pragma unroll
    for (int j = 0; j < DT; ++j) fin[sbase + (int64_t)j * D + tid] = s[j];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 2D map over `rows` rows of `cols` elements with a row pitch of `pitch` elements;
// 64 x 64 boxes, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_chunk_tc_workspace(int64_t T, int32_t n_seq, int32_t Hv) {
  return ws_layout(T, n_seq, Hv).total;
}

cudaError_t launch_prefill_chunk_tc(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, void* o, int64_t T, int32_t Hk, int32_t Hv,
                                    int64_t qk_stride, int64_t v_stride, const int32_t* cu,
                                    int32_t n_seq, const float* init, float* fin, float scale,
                                    void* workspace, cudaStream_t stream) {
  static uint64_t attrs_set = 0;   // one bit per device that has the smem attributes
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attrs_set >> dev & 1)) {
    e = cudaFuncSetAttribute(chunk_intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kIntraSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chunk_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kChainSmem);
    if (e != cudaSuccess) return e;
    if (dev < 64) attrs_set |= 1ull << dev;
  }
  const Ws L = ws_layout(T, n_seq, Hv);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t slots = max_slots(T, n_seq);
  // with no tokens every sequence is empty: the chain kernel only copies the states and
  // never touches the maps, which are left zeroed
  CUtensorMap mq{}, mk{}, mv{}, mw{};
  if (T > 0 && (!make_map(&mq, q, (uint64_t)Hk * D, (uint64_t)T, (uint64_t)qk_stride) ||
                !make_map(&mk, k, (uint64_t)Hk * D, (uint64_t)T, (uint64_t)qk_stride) ||
                !make_map(&mv, v, (uint64_t)Hv * D, (uint64_t)T, (uint64_t)v_stride) ||
                !make_map(&mw, ws + L.mats, 64, (uint64_t)slots * Hv * 3 * C, 64)))
    return cudaErrorInvalidValue;
  chunk_plan_kernel<<<1, 1024, 0, stream>>>(cu, n_seq, T, reinterpret_cast<int32_t*>(ws + L.prefix),
                                            reinterpret_cast<int*>(ws + L.err));
  if (T > 0) {
    dim3 gi((unsigned)slots, (unsigned)Hk);
    chunk_intra_kernel<<<gi, 128, kIntraSmem, stream>>>(mq, mk, g, beta, cu, n_seq, T, Hk, Hv, ws);
  }
  dim3 gc((unsigned)((int64_t)n_seq * Hv * NT));
  chunk_chain_kernel<<<gc, 128, kChainSmem, stream>>>(mq, mk, mv, mw, cu, n_seq, T, Hk, Hv, ws,
                                                      reinterpret_cast<int*>(ws + L.err), init, fin,
                                                      static_cast<bf16*>(o), scale);
  return cudaGetLastError();
}

}  // namespace gdn
