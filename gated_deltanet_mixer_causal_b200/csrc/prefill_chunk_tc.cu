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
//  2. intra : persistent CTAs over the (chunk, key head) items, everything that does not
//             depend on the state: [K; Q] K^T on tcgen05 (M = 128); per value head the
//             decay-masked A and Mqk = M o QK^T / (|q||k|), the unit lower triangular
//             inverse Tm (16-row blocks: fp32 substitution on the diagonal, tf32 warp MMAs
//             off it), then [P; Pk] V and [P; Pk] K on tcgen05 with P = Tm diag(beta),
//             Pk = Tm diag(beta e^G / |k|), giving U~ = P V and W = Pk K. Writes -W, U~ and
//             its low bf16 half, Mqk (bf16) and the row scales to the workspace.
//  3. chain : one CTA per (sequence, value head, 64-wide slice of dv) walks the chunks in
//             order with the fp32 state slice in registers and its bf16 copy in shared
//             memory; per chunk only the state-dependent GEMMs remain:
//               [-W; Q] S0^T  (U = U~ - W S0^T in rows 0..63, Q S0^T in rows 64..127)
//               dS^T = K^T [U' | U'lo],   O2 = Mqk U
//             rA is split along K over two issuing warps, dS^T and O2 come from the second;
//             a producer warp issues the TMA loads and seeds A with U~.
// A single sequence of 512 chunks or more runs as eight pieces (ranges of chunks): the intra
// kernel of every piece on two low-priority side streams in turn, the chain of piece i on a
// high-priority stream once piece i's intra work is done, beside the intra work of the later
// pieces; events alone order the streams and the state passes between chain pieces in fp32.
// Operands are staged in shared memory in the 128-byte-swizzled layouts TMA writes; K-major
// and MN-major descriptors read the same tiles, and stacking two 64-row tiles 8 KB apart
// makes one M = 128 operand. Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <mutex>

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
  size_t err, ctr, prefix, order, wu, ul, mq, vecs, carry, total;
};

// Per (chunk, value head): wu = [-W (64 x 128) ; U~ (64 x 128)] bf16 rows of 128 elements,
// ul = U~ - bf16(U~) (64 x 128 bf16: U~ is carried as a hi + lo pair, because a chunk that
// rewrites one key many times turns U~ into differences of values whose bf16 roundings would
// add up in the state), mq = Mqk (64 x 64) bf16, vecs = row scales: [0, 64) e^{G_r}/|q_r|,
// [64, 128) e^{G_L - G_r}/|k_r|, [128] e^{G_L}; 132 floats = 528 bytes (a multiple of 16).
constexpr int kWuBytes = 2 * C * D * 2;
constexpr int kUlBytes = C * D * 2;   // U~ - bf16(U~): the low half of a hi + lo bf16 pair
constexpr int kVecFloats = 132;
constexpr int kVecBytes = kVecFloats * 4;

__host__ __device__ inline int64_t max_slots(int64_t T, int32_t n_seq) { return (T + C - 1) / C + n_seq; }

// A long single sequence is prefilled in pieces: the intra-chunk kernel of the next pieces
// runs beside the chain kernel of the current one, which occupies only 2 Hv of the SMs.
// kTargetPieces pieces of at least kMinPieceChunks chunks: a chain piece costs ~15 us to
// start, so shorter pieces lose more than the overlap gains (measured on the 27B layer: 8
// pieces take the 65536-token prefill from 3.38 to 3.07 ms and the 32768-token one from 1.72
// to 1.66 ms, while 16384 tokens gain nothing and 8192 tokens lose 14 %). The workspace then
// also holds the fp32 state handed from one chain piece to the next.
constexpr int64_t kMinPieceChunks = 64;
constexpr int64_t kTargetPieces = 8;
constexpr int kMaxPieces = 64;
__host__ __device__ inline int64_t piece_chunks(int64_t n_chunks) {
  const int64_t per = (n_chunks + kTargetPieces - 1) / kTargetPieces;
  return per > kMinPieceChunks ? per : kMinPieceChunks;
}
__host__ __device__ inline bool piece_layout(int64_t T, int32_t n_seq) {
  return n_seq == 1 && T >= kTargetPieces * kMinPieceChunks * C;
}

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ __device__ inline Ws ws_layout(int64_t T, int32_t n_seq, int32_t Hv) {
  Ws w;
  const size_t slots = (size_t)max_slots(T, n_seq);
  w.err = 0;
  w.ctr = 64;      // [kMaxPieces] item counters of the intra-chunk kernel, one per piece
  w.prefix = 512;
  w.order = w.prefix + (size_t)(n_seq + 1) * 4;   // [n_seq] sequences, longest first
  w.wu = align256(w.order + (size_t)n_seq * 4);
  w.ul = align256(w.wu + slots * Hv * kWuBytes);
  w.mq = align256(w.ul + slots * Hv * kUlBytes);
  w.vecs = align256(w.mq + slots * Hv * kMatBytes);
  w.carry = align256(w.vecs + slots * Hv * kVecBytes);
  w.total = align256(w.carry + (piece_layout(T, n_seq) ? (size_t)Hv * D * D * 4 : 0));
  return w;
}

// --------------------------------------------------------------------------- plan

// Sequences ranked by chunk count (longest first, ties by index) for batches of up to this
// many; larger batches keep their own order.
constexpr int32_t kOrderMaxSeq = 1024;

__global__ void __launch_bounds__(1024) chunk_plan_kernel(const int32_t* __restrict__ cu,
                                                          int32_t n_seq, int64_t T,
                                                          int32_t* __restrict__ prefix,
                                                          int32_t* __restrict__ order,
                                                          int* __restrict__ err, int* __restrict__ ctr) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) { carry = 0; *err = 0; }
  if (threadIdx.x < kMaxPieces) ctr[threadIdx.x] = 0;
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
  // the chain kernel takes its sequences in this order, so that the longest chains start in
  // the first wave of CTAs instead of lengthening the last
  __syncthreads();
  for (int32_t n = threadIdx.x; n < n_seq; n += blockDim.x) {
    if (n_seq > kOrderMaxSeq) { order[n] = n; continue; }
    const int32_t len = prefix[n + 1] - prefix[n];
    int32_t rank = 0;
    for (int32_t m = 0; m < n_seq; ++m) {
      const int32_t lm = prefix[m + 1] - prefix[m];
      rank += (lm > len || (lm == len && m < n)) ? 1 : 0;
    }
    order[rank] = n;
  }
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

// TMEM address of lane 32 * quadrant (a warp reads the 32 lanes of its quadrant, warp % 4).
__device__ __forceinline__ uint32_t tmem_quadrant(uint32_t tmem, int warp) {
  return tmem + ((uint32_t)(warp * 32) << 16);
}

// Barrier `id` (1..15) over `threads` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Barrier over `threads` threads that also returns whether any of them passed `pred`.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r) : "r"((uint32_t)pred), "r"(id), "r"(threads) : "memory");
  return r != 0;
}

// ------------------------------------------------------------------------ intra

// Warp-level MMAs (m16n8k8, tf32 inputs, fp32 accumulate) for the 16 x 16 block products of the
// triangular inverse off its diagonal. The inverse is rounded to bf16 right after (as the
// factors P, Pk of the tcgen05 products), which dominates tf32's 10-bit operand rounding: a
// split hi + lo tf32 form (fp32-accurate) changes the errors of the whole prefill by under 1 %
// on the near-collinear, repeated-key and no-decay inputs, so the plain form is used.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// c (one 16x8 half, columns 8 nh .. 8 nh + 7, of a 16x16 block) += X[xr.., xc..] Y[yr.., yc..]
// for fp32 matrices with row pitches px, py.
__device__ __forceinline__ void block_mma16h(float (&c)[4], const float* Xs, int px, int xr, int xc,
                                             const float* Ys, int py, int yr, int yc, int nh, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    const int k0 = 8 * ks + t;
    const uint32_t a[4] = {to_tf32(Xs[(xr + g) * px + xc + k0]), to_tf32(Xs[(xr + g + 8) * px + xc + k0]),
                           to_tf32(Xs[(xr + g) * px + xc + k0 + 4]), to_tf32(Xs[(xr + g + 8) * px + xc + k0 + 4])};
    const uint32_t bb[2] = {to_tf32(Ys[(yr + k0) * py + yc + 8 * nh + g]),
                            to_tf32(Ys[(yr + k0 + 4) * py + yc + 8 * nh + g])};
    mma_tf32_16x8x8(c, a, bb);
  }
}
// Both halves of a 16 x 16 block product.
__device__ __forceinline__ void block_mma16(float (&c)[2][4], const float* Xs, int px, int xr, int xc,
                                            const float* Ys, int py, int yr, int yc, int lane) {
  block_mma16h(c[0], Xs, px, xr, xc, Ys, py, yr, yc, 0, lane);
  block_mma16h(c[1], Xs, px, xr, xc, Ys, py, yr, yc, 1, lane);
}

// Stores sign * (one m16n8 accumulator fragment) into columns co .. co + 7 of a 16-row block
// of an fp32 matrix with row pitch p.
__device__ __forceinline__ void frag_store(float* M, int p, int co, const float (&c)[4], int lane, float sign) {
  const int g = lane >> 2, t = lane & 3;
  float* row0 = M + g * p + co + 2 * t;
  float* row8 = row0 + 8 * p;
  row0[0] = sign * c[0]; row0[1] = sign * c[1];
  row8[0] = sign * c[2]; row8[1] = sign * c[3];
}

// shared memory of the intra kernel (offsets from a 1024-aligned base)
constexpr int kMaxG = kPrefillTcMaxG;           // value heads per key head on this path
constexpr int kIKQ = 0;                         // [K0 | Q0 | K1 | Q1]: [K; Q] is one 128-row operand
constexpr int kIV = 32768;                      // V tile of one value head: 2 atoms; once [K; Q] K^T
                                                // is done the Q atoms hold a second V tile
constexpr int kIPP = 49152;                     // [P | Pk] bf16, K-major
constexpr int kLd = 72;                         // fp32 row pitch of Tm (= 8 mod 32: conflict-free
                                                // tf32 B-fragment loads)
constexpr int kLdA = 68;                        // fp32 row pitch of A (= 4 mod 32: conflict-free
                                                // 16-byte row stores and tf32 A-fragment loads)
constexpr int kIA = 65536;                      // A fp32 [64][kLdA] (region sized [64][kLd])
constexpr int kIT = kIA + 64 * kLd * 4;         // Tm  fp32 [64][kLd]
constexpr int kITmp = kIT + 64 * kLd * 4;       // per-warp block scratch fp32 [4][16][kLd16]
constexpr int kLd16 = 24;
constexpr int kIVec = kITmp + 4 * 16 * kLd16 * 4;   // rq, rk, G, colP, colPk, colInv [6][64]
constexpr int kIGB = kIVec + 6 * 64 * 4;        // g, beta of every value head [2][kMaxG][64]
constexpr int kIBar = kIGB + 2 * kMaxG * 64 * 4;    // 4 mbarriers + tmem address
constexpr int kIntraSmem = kIBar + 128 + 1024;  // + alignment slack
// TMEM columns: [KK^T; QK^T] (N = 64); [P; Pk] V (N = 128); [P; Pk] K in two N = 64 halves,
// the first beside the other two, the second into the columns of [P; Pk] V that the U~
// epilogue has read first
constexpr uint32_t kTKQ = 0, kTWa = 64, kTU = 128, kTWb = 128;

__global__ void __launch_bounds__(128, 2)   // two CTAs per SM (shared and tensor memory allow two)
chunk_intra_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_wu,
                   const __grid_constant__ CUtensorMap map_mq, const __grid_constant__ CUtensorMap map_ul,
                   const float* __restrict__ g,
                   const float* __restrict__ beta, const int32_t* __restrict__ cu, int32_t n_seq,
                   int64_t T, int32_t Hk, int32_t Hv, uint8_t* __restrict__ ws, int32_t slot_lo,
                   int32_t slot_hi, int piece) {
  const Ws L = ws_layout(T, n_seq, Hv);
  int* err = reinterpret_cast<int*>(ws + L.err);
  int* ctr = reinterpret_cast<int*>(ws + L.ctr) + piece;
  const int32_t* prefix = reinterpret_cast<const int32_t*>(ws + L.prefix);
  // items = (slot, key head) pairs of the slots [slot_lo, slot_hi) (item = slot * Hk + key head)
  const int32_t n_slots = prefix[n_seq];
  const int32_t item_lo = (slot_lo < n_slots ? slot_lo : n_slots) * Hk;
  const int32_t n_items = (slot_hi < n_slots ? slot_hi : n_slots) * Hk;
  const int G = Hv / Hk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (item_lo + (int32_t)blockIdx.x >= n_items) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* Am = reinterpret_cast<float*>(sm + kIA);
  float* Tm = reinterpret_cast<float*>(sm + kIT);
  float* scratch = reinterpret_cast<float*>(sm + kITmp) + warp * 16 * kLd16;
  float* rq = reinterpret_cast<float*>(sm + kIVec);
  float* rk = rq + 64;
  float* colP = rq + 192;
  float* colPk = rq + 256;
  float* colInv = rq + 320;
  float* gAll = reinterpret_cast<float*>(sm + kIGB);
  float* bAll = gAll + kMaxG * 64;
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + kIBar);   // K landed
  uint64_t* bar_mma = bar_tma + 1;
  uint64_t* bar_v = bar_tma + 2;   // [2] V tile of a value head landed in buffer j % 2
  uint64_t* bar_drain = bar_tma + 4;   // on an early exit: every MMA of this CTA has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 5);
  int32_t* next_item = reinterpret_cast<int32_t*>(bar_tma + 6);   // taken by thread 0 per item
  uint64_t* bar_mma2 = bar_tma + 7;   // the second half of [P; Pk] K has completed
  uint64_t* bar_q = bar_tma + 8;      // Q landed
  // loads issued into each barrier (thread 0 only): an early exit waits for the last of each
  uint32_t n_k = 0, n_q = 0, n_v0 = 0, n_v1 = 0;   // n_k: thread 64's

  // The CTA is persistent: its first item is item_lo + blockIdx.x, and each further one is
  // taken from the piece's counter while the current one starts (so CTAs that become
  // resident late, beside another kernel, take fewer). Each item's inputs are fetched as soon
  // as the previous item's last reader of their buffers has completed: Q and the first V tile
  // during its last value heads, K once its last [P; Pk] K is done, g and beta during its
  // last head.
  struct Item { int32_t slot, hk; int64_t t0; int len; };
  auto item_at = [&](int32_t it, Item& x) {
    if (it >= n_items) return false;
    x.slot = it / Hk;
    x.hk = it - x.slot * Hk;
    const int32_t n = slot_to_seq(prefix, n_seq, x.slot);
    int64_t bos, eos;
    seq_bounds(cu, n, T, bos, eos);
    x.t0 = bos + (int64_t)(x.slot - prefix[n]) * C;
    x.len = (int)(eos - x.t0 < C ? eos - x.t0 : C);
    return true;
  };
  // V tiles are double-buffered: buffer 0 at kIV, buffer 1 in the Q atoms (free once the
  // [K; Q] K^T MMA has read them); head j + 2 loads while head j + 1 is computed
  auto v_tile = [&](int b) { return sm + (b == 0 ? kIV : kIKQ + 8192); };
  auto load_v = [&](const Item& x, int j) {   // value head hk * G + j into buffer j % 2
    uint8_t* dst = v_tile(j & 1);
    const uint32_t atom = (j & 1) ? 16384u : 8192u;
    if (j & 1) ++n_v1; else ++n_v0;
    mbar_arrive_expect_tx(&bar_v[j & 1], 16384);
    for (int hh = 0; hh < 2; ++hh)
      tma_load_2d(dst + hh * atom, &map_v, (x.hk * G + j) * D + hh * 64, (int32_t)x.t0, &bar_v[j & 1]);
  };
  // K of item x (thread 64, as soon as the last MMA reading K has completed), Q (thread 0,
  // once the last V tile in the Q atoms has been read)
  auto load_k = [&](const Item& x) {
    ++n_k;
    mbar_arrive_expect_tx(bar_tma, 16384);
    for (int hh = 0; hh < 2; ++hh)
      tma_load_2d(sm + kIKQ + hh * 16384, &map_k, x.hk * D + hh * 64, (int32_t)x.t0, bar_tma);
  };
  auto load_q = [&](const Item& x) {
    ++n_q;
    mbar_arrive_expect_tx(bar_q, 16384);
    for (int hh = 0; hh < 2; ++hh)
      tma_load_2d(sm + kIKQ + hh * 16384 + 8192, &map_q, x.hk * D + hh * 64, (int32_t)x.t0, bar_q);
  };
  // the last value heads whose V tiles use buffer 1 (the Q atoms) and buffer 0: once their
  // [P; Pk] V has completed, the next item's Q and first V tile are loaded into them
  const int j_q = (G & 1) ? G - 2 : G - 1, j_v = (G & 1) ? G - 1 : G - 2;
  // g, beta of the G value heads of item x, this thread's share (rows past the sequence: 0)
  constexpr int kGB = kMaxG * 64 / 128;
  float gr[kGB], br[kGB];
  auto fetch_gb = [&](const Item& x) {
#pragma unroll
    for (int i = 0; i < kGB; ++i) {
      const int e = tid + i * 128, j = e >> 6, r = e & 63;
      const bool v = j < G && r < x.len;
      gr[i] = v ? g[(x.t0 + r) * Hv + x.hk * G + j] : 0.f;
      br[i] = v ? beta[(x.t0 + r) * Hv + x.hk * G + j] : 0.f;
    }
  };
  auto store_gb = [&]() {
#pragma unroll
    for (int i = 0; i < kGB; ++i) {
      const int e = tid + i * 128;
      if ((e >> 6) < G) { gAll[e] = gr[i]; bAll[e] = br[i]; }
    }
  };

  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    mbar_init(&bar_v[0], 1);
    mbar_init(&bar_v[1], 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_mma2, 1);
    mbar_init(bar_q, 1);
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(tmem_slot, 256); tmem_relinquish(); }
  Item cur;
  item_at(item_lo + (int32_t)blockIdx.x, cur);
  fetch_gb(cur);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) { load_q(cur); load_v(cur, 0); }
  if (tid == 64) load_k(cur);
  store_gb();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tq = tmem_quadrant(tmem, warp);   // lanes 32 w .. 32 w + 31: rows of M = 128 results
  uint32_t ph_mma = 0u, ph_mma2 = 0u, ph_kq = 0u;
  uint32_t vbase0 = 0u, vbase1 = 0u;   // completed loads of V buffers 0 and 1 before this item
  bool ok = true;
  __syncthreads();

  for (;;) {
  const int32_t slot = cur.slot, hk = cur.hk;
  const int len = cur.len;
  if (tid == 0) *next_item = item_lo + (int32_t)gridDim.x + atomicAdd(ctr, 1);   // read after a barrier
  Item nxt;
  bool has_next = false;
  if (warp < G) {   // inclusive cumulative log-decay of every value head, in place (2 values per lane)
    for (int j = warp; j < G; j += 4) {
      const float a0 = gAll[j * 64 + 2 * lane], a1 = gAll[j * 64 + 2 * lane + 1];
      float s = a0 + a1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      const float excl = s - (a0 + a1);
      gAll[j * 64 + 2 * lane] = excl + a0;
      gAll[j * 64 + 2 * lane + 1] = excl + a0 + a1;
    }
  }
  ok = mbar_wait(bar_tma, ph_kq, err, kErrIntraTma) && mbar_wait(bar_q, ph_kq, err, kErrIntraTma);
  ph_kq ^= 1u;
  if (__syncthreads_or(!ok)) { ok = false; goto teardown; }
  has_next = item_at(*next_item, nxt);   // thread 0 wrote it before the barrier above

  // [K; Q] K^T -> rows 0..63: K K^T, rows 64..127: Q K^T  (M = 128, N = 64, K = 128), issued
  // first so that it runs while the threads take the norms of the same tiles
  if (tid == 0) {
    tc_fence_after();
    const uint64_t kq = smem_desc(smem_u32(sm + kIKQ), 16u, 1024u);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t off = (uint64_t)((kk >> 2) * (16384 >> 4) + (kk & 3) * 2);
      mma_bf16(tmem + kTKQ, kq + off, kq + off, idesc_bf16(128, 64, 0, 0), kk > 0);
    }
    mma_commit(bar_mma);
  }
  {  // inverse L2 norms of the chunk's q and k rows (0 for rows past the sequence end)
    const int r = tid & 63;
    const uint8_t* tile = sm + kIKQ + (tid < 64 ? 8192 : 0);
    float ss = 0.f;
    for (int hh = 0; hh < 2; ++hh)
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint4 u = *reinterpret_cast<const uint4*>(tile + hh * 16384 + sw128_off(r, c8 * 8));
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

  ok = mbar_wait(bar_mma, ph_mma, err, kErrIntraMma);
  ph_mma ^= 1u;
  if (__syncthreads_or(!ok)) { ok = false; goto teardown; }
  tc_fence_after();
  if (tid == 0) {   // into the Q atoms, which the MMA and the norms have finished reading
    if (G > 1) load_v(cur, 1);
    else if (has_next) load_q(nxt);
  }

  for (int j = 0; j < G; ++j) {
    const int h = hk * G + j;
    // the next item's g, beta into registers while the last head runs (stored to shared
    // memory once this item is done with its own)
    if (j == G - 1 && has_next) fetch_gb(nxt);
    const float* sG = gAll + j * 64;   // cumulative log-decay of this head
    const float* sb = bAll + j * 64;
    if (tid < 64) {   // column factors of P = Tm diag(beta), Pk = Tm diag(beta e^G / |k|), A, Mqk
      colP[tid] = sb[tid];
      colPk[tid] = sb[tid] * __expf(sG[tid]) * rk[tid];
      colInv[tid] = -sG[C - 1] < 60.f ? __expf(-sG[tid]) * rk[tid] : 0.f;
    }
    __syncthreads();
    // each warp pair waits only for its own staging tiles of the previous head to be read out:
    // warps 0, 1 for U~ (in the A and Tm regions, stored by thread 0), warps 2, 3 for -W
    // (in [P | Pk], stored by thread 64)
    if (tid == 0 || tid == 64) tma_store_wait_read();
    if (warp < 2) named_bar_sync(1, 64);
    else named_bar_sync(2, 64);

    // thread t < 64: row t of A from K K^T; t >= 64: row t-64 of Mqk, staged (swizzled) in
    // the [P | Pk] region, which is free until the solve is done, and stored by TMA.
    // e^{G_r - G_i} = e^{G_r} e^{-G_i} with the column factors e^{-G_i}/|k_i| in shared
    // memory; when the chunk's cumulative decay could leave the fp32 range the difference
    // form is used instead (one exp per element).
    uint8_t* mq_stage = sm + kIPP;
    {
      const int r = tid & 63;
      const float Gr = sG[r];
      const bool factored = -sG[C - 1] < 60.f;     // G is non-increasing: G_63 is the minimum
      const float f = tid < 64 ? sb[r] * rk[r] : rq[r];
      const float fr = factored ? f * __expf(Gr) : f;
      uint32_t raw[2][32];
      tmem_ld32_async(tq + kTKQ, raw[0]);
      tmem_ld32_async(tq + kTKQ + 32, raw[1]);
      tmem_wait_ld(raw[0], raw[1]);
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        float v[32], ci[32];
        if (factored) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 c4 = *reinterpret_cast<const float4*>(colInv + cb * 32 + e);
            ci[e] = c4.x; ci[e + 1] = c4.y; ci[e + 2] = c4.z; ci[e + 3] = c4.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ci[e] = __expf(Gr - sG[cb * 32 + e]) * rk[cb * 32 + e];
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int i = cb * 32 + e;
          const bool keep = tid < 64 ? (i < r) : (i <= r);
          v[e] = keep ? fr * ci[e] * __uint_as_float(raw[cb][e]) : 0.f;
        }
        if (tid < 64) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(Am + r * kLdA + cb * 32 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        } else {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float v8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v8[q] = v[c8 * 8 + q];
            VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(mq_stage + sw128_off(r, cb * 32 + c8 * 8)), v8);
          }
        }
      }
      if (tid >= 64) fence_async_smem();
    }
    // Tm = (I + A)^{-1}. Diagonal 16x16 blocks by the warp that wrote their rows of A (warp w,
    // w < 2: blocks 2w and 2w + 1, one per half warp), by fp32 forward substitution: lane
    // col of its half solves column col of (I + L) X = I (L the block of A, strictly lower):
    // x_i = delta_ij - sum_{k<i} L_ik x_k, accumulating each x_k into every later row as soon
    // as it is known (a 15-step dependent chain; the L loads are half-warp broadcasts, the two
    // halves on different banks). The column stays in registers until it is complete, so no
    // store to Tm sits between the loads of L.
    if (warp < 2) {
      __syncwarp();
      const int b0 = (2 * warp + (lane >> 4)) * 16, col = lane & 15;
      float acc[16], x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        x[k] = k == col ? 1.f : (k < col ? 0.f : -acc[k]);
#pragma unroll
        for (int i = k + 1; i < 16; ++i) acc[i] = fmaf(Am[(b0 + i) * kLdA + b0 + k], x[k], acc[i]);   // L(i, k)
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) Tm[(b0 + k) * kLd + b0 + col] = x[k];
      // the same warp closes its 32 x 32 diagonal block: Tm_ba = -Tm_bb A_ba Tm_aa for
      // a = 2w, b = 2w + 1 (tf32 warp MMAs), from blocks only this warp has written
      __syncwarp();
      const int aa = 2 * warp, bb = aa + 1;
      float c[2][4] = {};
      block_mma16(c, Am, kLdA, 16 * bb, 16 * aa, Tm, kLd, 16 * aa, 16 * aa, lane);
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) frag_store(scratch, kLd16, 8 * nh, c[nh], lane, 1.f);
      __syncwarp();
      float d[2][4] = {};
      block_mma16(d, Tm, kLd, 16 * bb, 16 * bb, scratch, kLd16, 0, 0, lane);
#pragma unroll
      for (int nh = 0; nh < 2; ++nh)
        frag_store(Tm + 16 * bb * kLd + 16 * aa, kLd, 8 * nh, d[nh], lane, -1.f);
    }
    __syncthreads();
    if (tid == 0) {
      tma_store_2d(&map_mq, 0, (int32_t)(((int64_t)slot * Hv + h) * C), mq_stage);
      tma_store_commit();
    }
    // the lower-left 32 x 32 block: with X = A[32:64, 0:32] Tm[0:32, 0:32],
    // Tm[32:64, 0:32] = -Tm[32:64, 32:64] X, i.e. per 16-column block a:
    //   Tm_2a = -Tm_22 X_2a,  Tm_3a = -(Tm_32 X_2a + Tm_33 X_3a),  X_ba = sum_{c=a}^{1} A_bc Tm_ca.
    // Warp w takes column block a = w / 2 and 8-column half w % 2 of both results (a half of
    // a result needs only the same half of X), so the round needs no barrier inside it.
    {
      const int aa = warp >> 1, nh = warp & 1;
      float x2[4] = {}, x3[4] = {};
      for (int cblk = aa; cblk < 2; ++cblk) {
        block_mma16h(x2, Am, kLdA, 32, 16 * cblk, Tm, kLd, 16 * cblk, 16 * aa, nh, lane);
        block_mma16h(x3, Am, kLdA, 48, 16 * cblk, Tm, kLd, 16 * cblk, 16 * aa, nh, lane);
      }
      frag_store(scratch, kLd16, 0, x2, lane, 1.f);   // X_2a half in columns 0..7
      frag_store(scratch, kLd16, 8, x3, lane, 1.f);   // X_3a half in columns 8..15
      __syncwarp();
      float t2[4] = {}, t3[4] = {};
      block_mma16h(t2, Tm, kLd, 32, 32, scratch, kLd16, 0, 0, 0, lane);
      block_mma16h(t3, Tm, kLd, 48, 32, scratch, kLd16, 0, 0, 0, lane);
      block_mma16h(t3, Tm, kLd, 48, 48, scratch, kLd16, 0, 8, 0, lane);
      frag_store(Tm + 32 * kLd + 16 * aa, kLd, 8 * nh, t2, lane, -1.f);
      frag_store(Tm + 48 * kLd + 16 * aa, kLd, 8 * nh, t3, lane, -1.f);
    }
    if (tid == 0) tma_store_wait_read();   // Mqk left its staging tile ([P | Pk])
    __syncthreads();

    // [P | Pk] as bf16 K-major operands: warps 0, 1 form P, warps 2, 3 Pk. A lane takes 4
    // columns (chunk c) of a row per step, a warp 8 rows x 4 chunks with the 8 rows on
    // consecutive lanes; the 8-byte swizzled stores of a half warp hit 16 different words.
    // Row scales out.
    {
      const int m = warp >> 1, wm = warp & 1, rl = lane & 7, cl = lane >> 3;
      const float* fv = m == 0 ? colP : colPk;
      float4 f[4];   // column factors of this lane's chunks cg * 4 + cl
#pragma unroll
      for (int cg = 0; cg < 4; ++cg) f[cg] = *reinterpret_cast<const float4*>(fv + 16 * cg + 4 * cl);
      uint8_t* tile = sm + kIPP + m * 8192;
#pragma unroll
      for (int rb = 0; rb < 4; ++rb) {
        const int r = (wm * 4 + rb) * 8 + rl;
        // Tm is block lower triangular; its blocks above the diagonal are never written
        // (the staging tiles reuse that memory), so they are masked here
        const int live_end = (r & ~15) + 16;
#pragma unroll
        for (int cg = 0; cg < 4; ++cg) {
          const int c = cg * 4 + cl;
          const float4 t = 4 * c < live_end ? *reinterpret_cast<const float4*>(Tm + r * kLd + 4 * c)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
          uint2 pk;
          __nv_bfloat162 lo = __floats2bfloat162_rn(t.x * f[cg].x, t.y * f[cg].y);
          __nv_bfloat162 hi = __floats2bfloat162_rn(t.z * f[cg].z, t.w * f[cg].w);
          pk.x = *reinterpret_cast<uint32_t*>(&lo);
          pk.y = *reinterpret_cast<uint32_t*>(&hi);
          *reinterpret_cast<uint2*>(tile + sw128_off(r, 4 * c)) = pk;
        }
      }
      float* vec = reinterpret_cast<float*>(ws + L.vecs) + (size_t)(slot * Hv + h) * kVecFloats;
      const float Gl = sG[C - 1];
      if (tid < 64) vec[tid] = __expf(sG[tid]) * rq[tid];
      else vec[tid] = __expf(Gl - sG[tid - 64]) * rk[tid - 64];
      if (tid < kVecFloats - 128) vec[128 + tid] = tid == 0 ? __expf(Gl) : 0.f;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    const uint64_t dpp = smem_desc(smem_u32(sm + kIPP), 16u, 1024u);
    // K as the MN-major B operand of [P; Pk] K (N = dk, K = the chunk's rows), half h at atom h
    const uint64_t dk = smem_desc(smem_u32(sm + kIKQ), 16384u, 1024u);
    if (tid == 0) {   // [P; Pk] V: rows 0..63 = U~ (M = 128, N = 128, K = 64), and beside it
                      // [P; Pk] K atom 0: rows 64..127 = W columns 0..63 (N = 64)
      if (mbar_wait(&bar_v[j & 1], ((j & 1 ? vbase1 : vbase0) + (uint32_t)(j >> 1)) & 1u, err, kErrIntraTma)) {
        tc_fence_after();
        const uint64_t dv = smem_desc(smem_u32(v_tile(j & 1)), (j & 1) ? 16384u : 8192u, 1024u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kTU, dpp + 2 * kk, dv + 128 * kk, idesc_bf16(128, 128, 0, 1), kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + kTWa, dpp + 2 * kk, dk + 128 * kk, idesc_bf16(128, 64, 0, 1), kk > 0);
        mma_commit(bar_mma);
      }
    }
    ok = mbar_wait(bar_mma, ph_mma, err, kErrIntraMma);
    ph_mma ^= 1u;
    if (__syncthreads_or(!ok)) { ok = false; goto teardown; }
    tc_fence_after();
    if (tid == 0) {   // this V buffer is free
      if (j + 2 < G) load_v(cur, j + 2);
      else if (has_next && j == j_q) load_q(nxt);
      else if (has_next && j == j_v) load_v(nxt, 0);
    }
    uint8_t* stage_u = sm + kIA;   // U~: 2 swizzled atoms of [64][64] in the free A region
    uint8_t* stage_ul = sm + kIT;  // U~ - bf16(U~), in the Tm region (read for the last time
                                   // by the [P | Pk] build)
    uint8_t* stage_w = sm + kIPP;  // -W, in [P | Pk] once the last MMA reading it has completed
    const int32_t wrow = (int32_t)(((int64_t)slot * Hv + h) * 2 * C);   // [-W; U~] rows
    const int32_t lrow = (int32_t)(((int64_t)slot * Hv + h) * C);       // U~lo rows
    if (warp < 2) {
      // U~ (rows 0..63) -> bf16 hi + lo tiles. Once its first 64 columns are in registers,
      // thread 0 issues [P; Pk] K atom 1 into them, behind the rest of this epilogue.
#pragma unroll
      for (int cp = 0; cp < 4; cp += 2) {
        uint32_t raw[2][32];
        tmem_ld32_async(tq + kTU + cp * 32, raw[0]);
        tmem_ld32_async(tq + kTU + cp * 32 + 32, raw[1]);
        tmem_wait_ld(raw[0], raw[1]);
        if (cp == 0) {
          tc_fence_before();
          named_bar_sync(1, 64);
          if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(tmem + kTWb, dpp + 2 * kk, dk + (16384 >> 4) + 128 * kk, idesc_bf16(128, 64, 0, 1), kk > 0);
            mma_commit(bar_mma2);
          }
        }
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          const int cb = cp + hb;
          uint8_t* atom = stage_u + (cb >> 1) * 8192;
          uint8_t* atom_l = stage_ul + (cb >> 1) * 8192;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              split_bf16x2(__uint_as_float(raw[hb][c8 * 8 + 2 * q]), __uint_as_float(raw[hb][c8 * 8 + 2 * q + 1]),
                           hi[q], lo[q]);
            const uint32_t off = sw128_off(tid, (cb & 1) * 32 + c8 * 8);
            *reinterpret_cast<uint4*>(atom + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(atom_l + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
        // this pass's atom of U~ and U~lo leaves at once (64 columns each)
        fence_async_smem();
        named_bar_sync(1, 64);
        if (tid == 0) {
          tma_store_2d(&map_wu, cp * 32, wrow + C, stage_u + (cp >> 1) * 8192);
          tma_store_2d(&map_ul, cp * 32, lrow, stage_ul + (cp >> 1) * 8192);
          tma_store_commit();
        }
      }
    } else {
      // -W (rows 64..127): columns 0..63 are converted while [P; Pk] K atom 1 runs, and
      // both halves are written once it has completed
      const int r = tid - 64;
      auto neg_pack = [](const uint32_t (&x)[2][32], uint32_t (&p)[32]) {
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const __nv_bfloat162 t = __floats2bfloat162_rn(-__uint_as_float(x[q >> 4][(2 * q) & 31]),
                                                         -__uint_as_float(x[q >> 4][(2 * q + 1) & 31]));
          p[q] = *reinterpret_cast<const uint32_t*>(&t);
        }
      };
      auto store_atom = [&](const uint32_t (&p)[32], uint8_t* atom) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8)
          *reinterpret_cast<uint4*>(atom + sw128_off(r, c8 * 8)) =
              make_uint4(p[4 * c8], p[4 * c8 + 1], p[4 * c8 + 2], p[4 * c8 + 3]);
      };
      uint32_t wp[32];
      {
        uint32_t raw[2][32];
        tmem_ld32_async(tq + kTWa, raw[0]);
        tmem_ld32_async(tq + kTWa + 32, raw[1]);
        tmem_wait_ld(raw[0], raw[1]);
        neg_pack(raw, wp);
      }
      ok = mbar_wait(bar_mma2, ph_mma2, err, kErrIntraMma);
      // the last MMA reading K has completed: the next item's K
      if (tid == 64 && ok && j == G - 1 && has_next) load_k(nxt);
      tc_fence_after();
      if (ok) {
        store_atom(wp, stage_w);
        uint32_t raw[2][32];
        tmem_ld32_async(tq + kTWb, raw[0]);
        tmem_ld32_async(tq + kTWb + 32, raw[1]);
        tmem_wait_ld(raw[0], raw[1]);
        neg_pack(raw, wp);
        store_atom(wp, stage_w + 8192);
      }
      fence_async_smem();
      if (named_bar_or(2, 64, !ok)) ok = false;
      if (tid == 64 && ok) {   // read out before the next head's Mqk rewrites [P | Pk]
        tma_store_2d(&map_wu, 0, wrow, stage_w);
        tma_store_2d(&map_wu, 64, wrow, stage_w + 8192);
        tma_store_commit();
      }
    }
    ph_mma2 ^= 1u;
    tc_fence_before();
    if (__syncthreads_or(!ok)) { ok = false; goto teardown; }
    tc_fence_before();
  }
  vbase0 += (uint32_t)(G + 1) / 2;
  vbase1 += (uint32_t)G / 2;
  if (!has_next) break;
  store_gb();   // this item's last reader of g, beta was its last head's row scales
  cur = nxt;
  __syncthreads();
  }

teardown:
  if (tid == 0) {
    if (!ok) {   // a wait gave up: let this CTA's loads and MMAs in flight finish (bounded)
      if (n_q) mbar_wait(bar_q, (n_q - 1) & 1u, nullptr, 0);
      if (n_v0) mbar_wait(&bar_v[0], (n_v0 - 1) & 1u, nullptr, 0);
      if (n_v1) mbar_wait(&bar_v[1], (n_v1 - 1) & 1u, nullptr, 0);
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0u, nullptr, 0);
    }
    tma_store_wait_all();
  }
  if (tid == 64) {   // its -W stores and, after a wait gave up, its K load in flight
    if (!ok && n_k) mbar_wait(bar_tma, (n_k - 1) & 1u, nullptr, 0);
    tma_store_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------------ chain

// shared memory of the chain kernel (offsets from a 1024-aligned base). A stage holds one
// chunk in two parts with their own loads and releases, so that the data the serial path
// needs first is requested as early as possible:
//   part A (read by the seed and rA; released as soon as rA has completed):
//     WQ : [-W atom0 | Q atom0 | -W atom1 | Q atom1]: [-W; Q] is one K-major 128-row operand
//     U~ and U~lo (this slice)
//   part B (read by dS, O2 and the epilogues; released once the chunk's output is out):
//     K : 2 atoms, then Mqk: [K atom1; Mqk] is O2's 128-row A operand, whose top half only
//         lands in rows nobody reads; then the chunk's row scales
constexpr int kSWQ = 0, kSU = 32768, kSUl = 40960;          // part A: 48 KB
constexpr int kSB = 49152;                                  // part B
constexpr int kSK = kSB, kSM = kSB + 16384, kSVec = kSB + 24576;
constexpr int kStage = 74752;                 // one chunk (1024-aligned)
constexpr int kStageTxA = 32768 + 8192 + 8192;              // bytes the part A loads deliver
constexpr int kStageTxB = 16384 + 8192 + kVecBytes;         // and part B
constexpr int kCS = 2 * kStage;               // S0^T bf16, MN-major [128][64]: 16 KB
constexpr int kCU = kCS + 16384;              // U   bf16 [64][64]: 8 KB (for O2)
constexpr int kCUp = kCU + 8192;              // U' = diag(e^{G_L - G_r}/|k_r|) U as a bf16 hi + lo
constexpr int kCUpl = kCUp + 8192;            //   pair [64][64] each (for dS): 16 KB
constexpr int kCI = kCUpl + 8192;             // [I; 0] bf16 K-major [128][64]: 16 KB (seeds A with U~)
constexpr int kCO = kCI + 16384;              // o staging, 2 x [64 tokens][64] bf16: 16 KB
constexpr int kCBar = kCO + 16384;            // mbarriers + tmem address
constexpr int kChainSmem = kCBar + 256 + 1024;
// warps 0..7 compute, 8 and 9 issue MMAs, 10 issues the TMA loads
constexpr int kComputeWarps = 8;
constexpr int kChainThreads = (kComputeWarps + 3) * 32;
constexpr int kOBarrier = 1;                  // named barrier of the four output warps
constexpr int kStateInitBf16 = 1, kStateFinBf16 = 2, kStateBlocksBf16 = 4;   // chain state_flags

// TMEM columns (M = 128 accumulators, lane = row). A = [-W; Q] S0^T is accumulated in two
// K halves (lo: dk 0..63, hi: dk 64..127) by the two issuers, each double-buffered; the lo
// half starts from [I; 0] U~, so its rows 0..63 plus the hi half's are U itself. dS^T =
// K^T [U' | U'lo] is one N = 128 accumulator whose column halves the state epilogue sums (an
// N = 128 MMA takes about as long as an N = 64 one, so this halves the MMAs on the serial
// path); O2 = [K atom1; Mqk] U (rows 64..127 used), double-buffered:
// chunk c's O2 is issued once chunk c's loads have landed, and those were requested only after
// chunk c - 2's output warps had read the same buffer.
constexpr uint32_t kTAlo = 0, kTAhi = 128, kTdS = 256, kTO2 = 384;

// Wait until at most one committed bulk store group of this thread still reads shared memory.
__device__ __forceinline__ void tma_store_wait_read_le1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// One chain CTA: sequence n, value head h, dv rows [tile*64, tile*64 + 64). Per chunk c:
//   issuers : rA(c) = [-W; Q] S0^T in two K halves (dk rows 0..63 after the state warps of
//             quadrants 0, 1 are done, 64..127 after quadrants 2, 3), the lo half on top of
//             [I; 0] U~ (issued as soon as the stage lands, off the serial path);
//             dS^T = K^T [U' | U'lo] once all of U' is written (U' is carried as a bf16
//             hi + lo pair on the state path, where a chunk that rewrites one key
//             telescopes U's rows), then O2 = [K atom1; Mqk] U behind it (second issuer)
//   compute : U = rows 0..63 of rA -> U' (hi + lo) -> "U' ready", U (bf16) -> "U ready"
//             (quadrants 0, 1)
//             S^T <- e^{G_L} S^T + dS^T, bf16 copy (all 8 warps)               -> "S ready"
//             o = scale (e^{G_r}/|q_r| rows 64..127 of rA + O2) (quadrants 2, 3): a full
//             chunk is staged in shared memory and leaves by one TMA store     -> "stage free"
//   producer: chunk c+2's loads into stage c % 2 once it is free; chunk c+1's seed of A-lo
//             once its stage has landed
// The serial path is rA -> U -> dS -> S -> rA(c+1); no thread on it issues anything else.
__global__ void __launch_bounds__(kChainThreads, 1)
chunk_chain_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_wu, const __grid_constant__ CUtensorMap map_mq,
                   const __grid_constant__ CUtensorMap map_ul, const __grid_constant__ CUtensorMap map_o,
                   const int32_t* __restrict__ cu, int32_t n_seq, int64_t T, int32_t Hk, int32_t Hv,
                   const uint8_t* __restrict__ ws_ro, int* err_word, const void* init, void* fin,
                   int state_flags, bf16* __restrict__ o, float scale, BlockStates blocks,
                   int32_t c_begin, int32_t c_end) {
  const Ws L = ws_layout(T, n_seq, Hv);
  const int32_t* prefix = reinterpret_cast<const int32_t*>(ws_ro + L.prefix);
  const int tile = blockIdx.x % NT;
  const int h = (blockIdx.x / NT) % Hv;
  const int32_t n = reinterpret_cast<const int32_t*>(ws_ro + L.order)[blockIdx.x / (NT * Hv)];
  const int hk = h / (Hv / Hk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // storage of the initial, final and block states: fp32, or bf16 (kStateInitBf16 ...)
  const bool init_bf = (state_flags & kStateInitBf16) != 0, fin_bf = (state_flags & kStateFinBf16) != 0;
  const bool sbf = (state_flags & kStateBlocksBf16) != 0;
  int64_t bos, eos;
  seq_bounds(cu, n, T, bos, eos);
  // this launch's chunks of the sequence: [c_begin, c_end) clamped to its length; bos and the
  // first slot move to the first of them, cfirst keeps its index for the block states
  const int nc_all = (int)((eos - bos + C - 1) / C);
  const int cfirst = c_begin < nc_all ? c_begin : nc_all;
  const int clast = c_end < nc_all ? c_end : nc_all;
  const int nc = clast > cfirst ? clast - cfirst : 0;
  bos += (int64_t)cfirst * C;
  const int32_t slot0 = prefix[n] + cfirst;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kCBar);
  uint64_t* bar_tma = bars;        // [2] part A of stage b landed
  uint64_t* bar_tmb = bars + 2;    // [2] part B landed
  uint64_t* bar_free_a = bars + 4; // [2] part A no longer read (rA has completed)
  uint64_t* bar_free = bars + 6;   // [2] part B no longer read (8 compute warps)
  uint64_t* bar_A0 = bars + 8;
  uint64_t* bar_A1 = bars + 9;
  uint64_t* bar_B = bars + 10;     // dS^T complete
  uint64_t* bar_O = bars + 12;
  uint64_t* bar_U0 = bars + 13;    // U rows 0..31 written (the 2 warps of quadrant 0)
  uint64_t* bar_U1 = bars + 14;    // rows 32..63 (quadrant 1)
  uint64_t* bar_Up0 = bars + 23;   // U' (hi + lo) rows 0..31 written, before U itself
  uint64_t* bar_Up1 = bars + 24;   // rows 32..63
  uint64_t* bar_S0 = bars + 15;    // state bf16 rows 0..63 written (quadrants 0, 1: 4 warps)
  uint64_t* bar_S1 = bars + 16;    // rows 64..127 (quadrants 2, 3)
  uint64_t* bar_drain = bars + 17; // [3] on an early exit: each issuing thread's MMAs have completed
  uint64_t* bar_seed = bars + 20;  // [2] A-lo buffer b holds [I; 0] (U~ + U~lo) of its next chunk
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 22);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_tma[i], 1);
      mbar_init(&bar_tmb[i], 1);
      mbar_init(&bar_free_a[i], 1);
      mbar_init(&bar_free[i], kComputeWarps);
    }
    for (int i = 8; i < 13; ++i) mbar_init(&bars[i], 1);
    mbar_init(bar_U0, 2);
    mbar_init(bar_U1, 2);
    mbar_init(bar_Up0, 2);
    mbar_init(bar_Up1, 2);
    mbar_init(bar_S0, 4);
    mbar_init(bar_S1, 4);
    for (int i = 0; i < 3; ++i) mbar_init(&bar_drain[i], 1);
    mbar_init(&bar_seed[0], 1);
    mbar_init(&bar_seed[1], 1);
    fence_mbar_init();
  }
  // [I; 0]: rows 0..63 the identity, rows 64..127 zero (K-major, 128-byte swizzle)
  for (int e = tid; e < 128 * 8; e += kChainThreads) {
    const int r = e >> 3, c8 = e & 7;
    uint4 z = make_uint4(0u, 0u, 0u, 0u);
    if (r < 64 && (r >> 3) == c8) {
      const uint32_t one = 0x3F80u << (16 * (r & 1));   // bf16 1.0 in the low or high half
      const int w = (r & 7) >> 1;
      if (w == 0) z.x = one; else if (w == 1) z.y = one; else if (w == 2) z.z = one; else z.w = one;
    }
    *reinterpret_cast<uint4*>(sm + kCI + sw128_off(r, c8 * 8)) = z;
  }
  fence_async_smem();
  if (warp == 0) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp >= kComputeWarps) {
    // ---------------------------------------------------------------- issuers / producer
    // the producer is one lane; each issuer is a whole warp, one elected lane of which issues
    if (nc == 0 || (warp == kComputeWarps + 2 && lane != 0)) goto done;
    const uint32_t st0 = smem_u32(sm);
    auto soff = [](int b) { return (uint64_t)(b * (kStage >> 4)); };
    const uint64_t dS = smem_desc(smem_u32(sm + kCS), 8192u, 1024u);
    const uint64_t dU = smem_desc(smem_u32(sm + kCU), 8192u, 1024u);
    // [U' | U'lo] as one MN-major B operand of N = 128 (its two 64-column atoms 8 KB apart)
    const uint64_t dUp = smem_desc(smem_u32(sm + kCUp), 8192u, 1024u);
    const uint64_t dI = smem_desc(smem_u32(sm + kCI), 16u, 1024u);
    constexpr uint32_t kIA = idesc_bf16(128, DT, 0, 1);     // K-major A, MN-major B
    constexpr uint32_t kIB = idesc_bf16(128, 2 * DT, 1, 1); // MN-major A and B, N = 128 (dS^T)
    const uint64_t dUt = smem_desc(st0 + kSU, 8192u, 1024u);    // U~ as an MN-major B operand
    const uint64_t dUtl = smem_desc(st0 + kSUl, 8192u, 1024u);  // and its low half
    if (warp == kComputeWarps + 2) {
      // TMA producer. Once a chunk's stage has landed and its A-lo buffer's previous chunk is
      // done, it also seeds that buffer with [I; 0] (U~ + U~lo) (rows 0..63 = U~, rows
      // 64..127 = 0), off the issuers' serial path.
      tma_prefetch_desc(&map_q);
      auto issue_a = [&](int c, int b) {   // part A of chunk c into stage b
        const int32_t slot = slot0 + c;
        const int64_t t0 = bos + (int64_t)c * C;
        uint8_t* stg = sm + b * kStage;
        const int32_t wrow = (int32_t)(((int64_t)slot * Hv + h) * 2 * C);
        mbar_arrive_expect_tx(&bar_tma[b], kStageTxA);
        for (int hh = 0; hh < 2; ++hh) {
          tma_load_2d(stg + kSWQ + hh * 16384, &map_wu, hh * 64, wrow, &bar_tma[b]);
          tma_load_2d(stg + kSWQ + hh * 16384 + 8192, &map_q, hk * D + hh * 64, (int32_t)t0, &bar_tma[b]);
        }
        tma_load_2d(stg + kSU, &map_wu, tile * DT, wrow + C, &bar_tma[b]);
        tma_load_2d(stg + kSUl, &map_ul, tile * DT, (int32_t)(((int64_t)slot * Hv + h) * C), &bar_tma[b]);
      };
      auto issue_b = [&](int c, int b) {   // part B of chunk c into stage b
        const int32_t slot = slot0 + c;
        const int64_t t0 = bos + (int64_t)c * C;
        uint8_t* stg = sm + b * kStage;
        mbar_arrive_expect_tx(&bar_tmb[b], kStageTxB);
        for (int hh = 0; hh < 2; ++hh)
          tma_load_2d(stg + kSK + hh * 8192, &map_k, hk * D + hh * 64, (int32_t)t0, &bar_tmb[b]);
        tma_load_2d(stg + kSM, &map_mq, 0, (int32_t)(((int64_t)slot * Hv + h) * C), &bar_tmb[b]);
        bulk_load(stg + kSVec, ws_ro + L.vecs + ((size_t)slot * Hv + h) * kVecBytes, kVecBytes, &bar_tmb[b]);
      };
      auto seed = [&](int c) {   // chunk c's part A has landed and its A-lo buffer is free
        const int b = c & 1;
        const uint32_t ta = tmem + kTAlo + 64 * b;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16(ta, dI + 2 * kk, dUt + soff(b) + 128 * kk, kIA, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_bf16(ta, dI + 2 * kk, dUtl + soff(b) + 128 * kk, kIA, true);
        mma_commit(&bar_seed[b]);
      };
      int issued_a = nc > 1 ? 2 : 1, issued_b = issued_a;
      for (int c = 0; c < issued_a; ++c) { issue_a(c, c); issue_b(c, c); }
      bool good = mbar_wait(&bar_tma[0], 0u, err_word, kErrChainTma);
      if (good) seed(0);
      for (int c = 0; good && c < nc; ++c) {
        const uint32_t ph = (uint32_t)(c >> 1) & 1u;
        // chunk c + 1's seed: its part A; its A-lo buffer was last read by chunk c - 1
        if (c + 1 < nc) {
          if (!(good = mbar_wait(&bar_tma[(c + 1) & 1], (uint32_t)((c + 1) >> 1) & 1u, err_word, kErrChainTma))) break;
          if (c >= 1 && !(good = mbar_wait(&bar_free[(c - 1) & 1], (uint32_t)((c - 1) >> 1) & 1u, err_word,
                                           kErrChainTma))) break;
          seed(c + 1);
        }
        if (c + 2 < nc) {   // chunk c + 2 into stage c % 2: part A once rA(c) is done, B after c
          if (!(good = mbar_wait(&bar_free_a[c & 1], ph, err_word, kErrChainTma))) break;
          issue_a(c + 2, c & 1);
          issued_a = c + 3;
          if (!(good = mbar_wait(&bar_free[c & 1], ph, err_word, kErrChainTma))) break;
          issue_b(c + 2, c & 1);
          issued_b = c + 3;
        }
      }
      if (!good) {   // gave up: let the loads in flight land (bounded) before exiting
        for (int b = 0; b < 2; ++b) {   // the last chunk loaded into each part of stage b
          if (b < issued_a) {
            const int last = (issued_a - 1) - (((issued_a - 1) - b) & 1);
            mbar_wait(&bar_tma[b], (uint32_t)(last >> 1) & 1u, nullptr, 0);
          }
          if (b < issued_b) {
            const int last = (issued_b - 1) - (((issued_b - 1) - b) & 1);
            mbar_wait(&bar_tmb[b], (uint32_t)(last >> 1) & 1u, nullptr, 0);
          }
        }
      }
      mma_commit(&bar_drain[2]);   // every seed MMA has completed before TMEM is released
      mbar_wait(&bar_drain[2], 0u, nullptr, 0);
      goto done;
    }
    const int part = warp - kComputeWarps;   // 0: lo halves, 1: hi halves and O2
    uint64_t* bar_Sp = part ? bar_S1 : bar_S0;
    const uint64_t dWQ = smem_desc(st0 + kSWQ, 16u, 1024u) + (uint64_t)(part * (16384 >> 4));
    const uint64_t dK = smem_desc(st0 + kSK, 8192u, 1024u);
    const uint64_t dUM = smem_desc(st0 + kSK + 8192, 16u, 1024u);   // [K atom1; Mqk]
    auto issue_rA = [&](int b) {
      const uint32_t ta = tmem + (part ? kTAhi : kTAlo) + 64 * b;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_warp(ta, dWQ + soff(b) + 2 * kk, dS + 128 * (4 * part + kk), kIA, part == 0 || kk > 0);
      mma_commit_warp(part ? bar_A1 : bar_A0);
    };
    // rA(0): chunk 0 landed (and, for the lo half, was seeded) and this half of the initial
    // state is in shared memory
    // (every wait's outcome is made warp-uniform: the warp issues together or leaves together)
    if (__any_sync(0xffffffffu, !mbar_spin(&bar_tma[0], 0u, err_word, kErrChainTma) ||
                                    (part == 0 && !mbar_spin(&bar_seed[0], 0u, err_word, kErrChainMma)) ||
                                    !mbar_spin(bar_Sp, 0u, err_word, kErrChainMma))) goto done;
    tc_fence_after();
    issue_rA(0);
    for (int c = 0; c < nc; ++c) {
      const int b = c & 1;
      if (part == 1) {   // once all of U' is written: dS^T; once U is: O2 behind it in the queue
        if (__any_sync(0xffffffffu, !mbar_spin(bar_Up1, (uint32_t)c & 1u, err_word, kErrChainMma) ||
                                        !mbar_spin(bar_Up0, (uint32_t)c & 1u, err_word, kErrChainMma) ||
                                        !mbar_spin(&bar_tmb[b], (uint32_t)(c >> 1) & 1u, err_word, kErrChainTma))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // dS^T = K^T [U' | U'lo]: N = 128, the two halves summed later
          mma_bf16_warp(tmem + kTdS, dK + soff(b) + 128 * kk, dUp + 128 * kk, kIB, kk > 0);
        mma_commit_warp(bar_B);
        if (__any_sync(0xffffffffu, !mbar_spin(bar_U1, (uint32_t)c & 1u, err_word, kErrChainMma) ||
                                        !mbar_spin(bar_U0, (uint32_t)c & 1u, err_word, kErrChainMma))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // rows 64..127 of [K atom1; Mqk] U
          mma_bf16_warp(tmem + kTO2 + 64 * b, dUM + soff(b) + 2 * kk, dU + 128 * kk, kIA, kk > 0);
        mma_commit_warp(bar_O);
      }
      if (c + 1 < nc) {
        if (__any_sync(0xffffffffu,
                       !mbar_spin(&bar_tma[b ^ 1], (uint32_t)((c + 1) >> 1) & 1u, err_word, kErrChainTma) ||
                       (part == 0 && !mbar_spin(&bar_seed[b ^ 1], (uint32_t)((c + 1) >> 1) & 1u, err_word,
                                                kErrChainMma)) ||
                       !mbar_spin(bar_Sp, (uint32_t)(c + 1) & 1u, err_word, kErrChainMma))) break;
        tc_fence_after();
        issue_rA(b ^ 1);
      }
    }
    // every MMA this warp issued has completed before the tensor memory is released
    mma_commit_warp(&bar_drain[part]);
    mbar_wait(&bar_drain[part], 0u, nullptr, 0);
    goto done;
  }

  {
    // ------------------------------------------------------------------- compute warps
    const int quad = warp & 3, half = warp >> 2;     // TMEM lanes 32 quad.., column half
    const int lrow = quad * 32 + lane;               // this thread's accumulator row (lane)
    const uint32_t tq = tmem_quadrant(tmem, quad);
    uint64_t* bar_Sq = quad < 2 ? bar_S0 : bar_S1;

    // state slice: thread (lrow, half) holds S[tile*64 + half*32 + j][lrow], j < 32
    constexpr int SJ = DT / 2;
    float s[SJ];
    const int64_t sbase = ((int64_t)n * Hv + h) * D * D + (int64_t)(tile * DT + half * SJ) * D + lrow;
#pragma unroll
    for (int j = 0; j < SJ; ++j) s[j] = init ? state_load(init, sbase + (int64_t)j * D, init_bf) : 0.f;
    auto store_state_bf16 = [&]() {
#pragma unroll
      for (int c8 = 0; c8 < SJ / 8; ++c8) {
        float v8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v8[q] = s[c8 * 8 + q];
        VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(sm + kCS + sw128_off(lrow, half * SJ + c8 * 8)), v8);
      }
    };
    auto warp_arrive = [&](uint64_t* bar) {   // one arrival per warp after all its lanes
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    store_state_bf16();
    fence_async_smem();
    warp_arrive(bar_Sq);

    uint32_t phA = 0u, phB = 0u;
    for (int c = 0; c < nc; ++c) {
      const int b = c & 1;
      const int64_t t0 = bos + (int64_t)c * C;
      const int len = (int)(eos - t0 < C ? eos - t0 : C);
      const float* vec = reinterpret_cast<const float*>(sm + b * kStage + kSVec);
      if (!(ok = mbar_wait(&bar_tmb[b], (uint32_t)(c >> 1) & 1u, err_word, kErrChainTma))) break;

      // U = U~ + (-W S0^T): rows 0..63 (quadrants 0, 1) -> U and U' in bf16
      if (!(ok = mbar_wait(bar_A0, phA, err_word, kErrChainMma) && mbar_wait(bar_A1, phA, err_word, kErrChainMma))) break;
      phA ^= 1u;
      if (warp == 0 && lane == 0) mbar_arrive(&bar_free_a[b]);   // rA(c) and its seed are done
      tc_fence_after();
      float os = 0.f;
      if (quad < 2) {
        // U is free: its last reader, O2 of chunk c - 1, was issued before rA_hi(c) by the
        // same thread, and that thread's commit of rA_hi(c) tracks every MMA it issued before
        const int r = lrow;
        const float us = vec[64 + r];
        uint32_t a0[32], a1[32];
        tmem_ld32_async(tq + kTAlo + 64 * b + half * 32, a0);
        tmem_ld32_async(tq + kTAhi + 64 * b + half * 32, a1);
        tmem_wait_ld(a0, a1);
#pragma unroll
        // U' (a hi + lo bf16 pair) first: dS^T, on the serial path, needs only U'; then U in
        // bf16 for O2
        uint32_t u[4][4];
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float x0 = __uint_as_float(a0[c8 * 8 + 2 * q]) + __uint_as_float(a1[c8 * 8 + 2 * q]);
            const float x1 = __uint_as_float(a0[c8 * 8 + 2 * q + 1]) + __uint_as_float(a1[c8 * 8 + 2 * q + 1]);
            __nv_bfloat162 ub = __floats2bfloat162_rn(x0, x1);
            u[c8][q] = *reinterpret_cast<uint32_t*>(&ub);
            split_bf16x2_alu(us * x0, us * x1, hi[q], lo[q]);
          }
          const uint32_t off = sw128_off(r, half * 32 + c8 * 8);
          *reinterpret_cast<uint4*>(sm + kCUp + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sm + kCUpl + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        fence_async_smem();
        tc_fence_before();
        warp_arrive(quad == 0 ? bar_Up0 : bar_Up1);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8)
          *reinterpret_cast<uint4*>(sm + kCU + sw128_off(r, half * 32 + c8 * 8)) =
              make_uint4(u[c8][0], u[c8][1], u[c8][2], u[c8][3]);
        fence_async_smem();
        tc_fence_before();
        warp_arrive(quad == 0 ? bar_U0 : bar_U1);
      } else {
        os = vec[lrow - 64];
      }

      // state update: S^T <- e^{G_L} S^T + dS^T (both K halves)
      if (!(ok = mbar_wait(bar_B, phB, err_word, kErrChainMma))) break;
      phB ^= 1u;
      tc_fence_after();
      {
        const float decay_last = vec[128];
        uint32_t d0[32], d1[32];
        tmem_ld32_async(tq + kTdS + half * 32, d0);        // K^T U'
        tmem_ld32_async(tq + kTdS + DT + half * 32, d1);   // K^T U'lo
        tmem_wait_ld(d0, d1);
#pragma unroll
        for (int e = 0; e < SJ; ++e)
          s[e] = fmaf(decay_last, s[e], __uint_as_float(d0[e]) + __uint_as_float(d1[e]));
        store_state_bf16();
      }
      fence_async_smem();
      tc_fence_before();
      warp_arrive(bar_Sq);
      // the state after a full chunk that ends a block of the sequence (prefix caching)
      if (blocks.block_tokens > 0 && len == C && ((int64_t)(cfirst + c + 1) * C) % blocks.block_tokens == 0) {
        const int64_t brow = (int64_t)blocks.rows[n] + (int64_t)(cfirst + c + 1) * C / blocks.block_tokens - 1;
        if (brow >= 0 && brow < blocks.n_rows) {
          const int64_t dst = ((brow * Hv + h) * D + tile * DT + half * SJ) * (int64_t)D + lrow;
#pragma unroll
          for (int j = 0; j < SJ; ++j) state_store(blocks.states, dst + (int64_t)j * D, s[j], sbf);
        }
      }

      // chunk c's output (quadrants 2, 3): o_r = scale (e^{G_r}/|q_r| O1_r + O2_r)
      if (quad >= 2) {
        const bool got = mbar_wait(bar_O, (uint32_t)c & 1u, err_word, kErrChainMma);
        // all four output warps leave together if any wait gave up; this barrier also
        // orders this chunk's staging writes after the read of the store from two chunks ago
        if (named_bar_or(kOBarrier, 128, !got)) { ok = false; break; }
        tc_fence_after();
        const int r = lrow - 64;
        uint32_t a0[32], a1[32];
        tmem_ld32_async(tq + kTAlo + 64 * b + half * 32, a0);
        tmem_ld32_async(tq + kTAhi + 64 * b + half * 32, a1);
        tmem_wait_ld(a0, a1);
        float o1[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) o1[e] = os * (__uint_as_float(a0[e]) + __uint_as_float(a1[e]));
        uint32_t o2[32];
        tmem_ld32_async(tq + kTO2 + 64 * b + half * 32, o2);
        tmem_wait_ld(o2);
        if (len == C) {   // a full chunk: stage the 64 x 64 tile, one TMA store
          uint8_t* ost = sm + kCO + b * 8192;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float v8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v8[q] = scale * (o1[c8 * 8 + q] + __uint_as_float(o2[c8 * 8 + q]));
            VecIO<bf16, 8>::store(reinterpret_cast<bf16*>(ost + sw128_off(r, half * 32 + c8 * 8)), v8);
          }
          fence_async_smem();
          named_bar_sync(kOBarrier, 128);
          if (warp == 2 && lane == 0) {
            tma_store_2d(&map_o, h * D + tile * DT, (int32_t)t0, ost);
            tma_store_commit();
            tma_store_wait_read_le1();   // the other staging buffer may be written next chunk
          }
        } else if (r < len) {   // the ragged end of a sequence: rows past it belong to the next
          bf16* dst = o + ((t0 + r) * Hv + h) * (int64_t)D + tile * DT + half * 32;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float v8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v8[q] = scale * (o1[c8 * 8 + q] + __uint_as_float(o2[c8 * 8 + q]));
            VecIO<bf16, 8>::store(dst + c8 * 8, v8);
          }
        }
        tc_fence_before();
      }
      warp_arrive(&bar_free[b]);
    }
    if (warp == 2 && lane == 0) tma_store_wait_all();
    if (ok && fin != nullptr) {
#pragma unroll
      for (int j = 0; j < SJ; ++j) state_store(fin, sbase + (int64_t)j * D, s[j], fin_bf);
    }
  }

done:
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

const char* prefill_chunk_tc_error_string(int code) {
  switch (code) {
    case kErrIntraTma: return "intra-chunk kernel: a TMA load did not land";
    case kErrIntraMma: return "intra-chunk kernel: an MMA did not complete";
    case kErrChainTma: return "chain kernel: a TMA load did not land";
    case kErrChainMma: return "chain kernel: an MMA or a warp handoff did not complete";
    default: return "unknown wait";
  }
}

size_t prefill_chunk_tc_workspace(int64_t T, int32_t n_seq, int32_t Hv) {
  return ws_layout(T, n_seq, Hv).total;
}

// How many leading chunks of a long sequence get their intra-chunk work done up front, on the
// whole GPU, before the first chain piece starts; the intra-chunk work of the other chunks then
// runs on the SMs the chain leaves free, up to the end of a piece per launch. A persistent
// intra-chunk grid holds its SMs until its items run out, so a chain piece that becomes ready
// beside one gets only the SMs that free up whole; restricting the later grids to the chain's
// free SMs keeps every chain piece at full width. The split (a multiple of 16 chunks, at least
// the first piece) minimises a model of the call: chain pieces back to back, each starting once the intra-chunk
// work of its chunks is done, with costs measured on B200 (intra-chunk work per chunk and value
// head: 3.60 SM-us on the whole GPU, 4.15 SM-us beside the chain; chain: 2.07 us per chunk).
// Only the schedule depends on these figures, never the results.
constexpr double kIntraSmUsAlone = 3.60, kIntraSmUsBeside = 4.15, kChainUsPerChunk = 2.07;
int64_t upfront_chunks(int64_t n_chunks, int64_t per, int pieces, int32_t Hv, int num_sms, int chain_ctas) {
  const int free_sms = num_sms - chain_ctas;
  auto piece_end = [&](int i) { return (i + 1) * per < n_chunks ? (i + 1) * per : n_chunks; };
  int64_t best = n_chunks;
  double best_t = -1.0;
  for (int64_t x = (per + 15) / 16 * 16; x <= n_chunks; x += 16) {   // x >= per: chain 0 needs
                                                                     // only the up-front launch
    const double t_e = kIntraSmUsAlone * Hv * (double)x / num_sms;
    double t_intra = t_e, t = t_e;
    int64_t done = x;   // chunks whose intra-chunk work is done by t_intra
    for (int i = 0; i < pieces; ++i) {
      const int64_t c0 = i * per, c1 = piece_end(i);
      if (c1 > done) {   // the launch that completes this piece's chunks
        t_intra += kIntraSmUsBeside * Hv * (double)(c1 - done) / free_sms;
        done = c1;
        t = t > t_intra ? t : t_intra;
      }
      t += kChainUsPerChunk * (double)(c1 - c0);
    }
    if (best_t < 0.0 || t < best_t) { best = x; best_t = t; }
  }
  return best;
}

// Per device: the streams a prefill in pieces forks onto (one for the up-front intra-chunk
// work and one for the rest, at the lowest priority; one for the chains at the highest) and
// the events that order them, created on first use and kept for the life of the process.
// Calls on one device take the mutex while they enqueue.
struct PieceStreams {
  std::mutex mu;
  cudaStream_t side[2] = {nullptr, nullptr}, chain = nullptr;
  cudaEvent_t ev[kMaxPieces + 3] = {};   // plan, up-front work, one per piece, chain start, join
};

PieceStreams* piece_streams(int dev) {
  static PieceStreams slots[64];
  static std::mutex init_mu;
  if (dev < 0 || dev >= 64) return nullptr;
  PieceStreams* p = &slots[dev];
  std::lock_guard<std::mutex> lock(init_mu);
  if (p->chain != nullptr) return p;
  int lo = 0, hi = 0;   // numerically lowest = highest priority
  if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return nullptr;
  for (int i = 0; i < 2; ++i)
    if (p->side[i] == nullptr && cudaStreamCreateWithPriority(&p->side[i], cudaStreamNonBlocking, lo) != cudaSuccess)
      return nullptr;
  for (int i = 0; i < kMaxPieces + 3; ++i)
    if (p->ev[i] == nullptr && cudaEventCreateWithFlags(&p->ev[i], cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
  cudaStream_t chain = nullptr;
  if (cudaStreamCreateWithPriority(&chain, cudaStreamNonBlocking, hi) != cudaSuccess) return nullptr;
  p->chain = chain;   // set last: a non-null chain stream means the set is complete
  return p;
}

// Kernels launch_prefill_chunk_tc enqueues for these sizes on a GPU of num_sms SMs: the plan,
// then one intra-chunk and one chain launch, or in pieces one chain launch per piece and one
// intra-chunk launch for the up-front chunks plus one per piece that ends past them.
int prefill_chunk_tc_launches(int64_t T, int32_t n_seq, int32_t Hv, int num_sms) {
  if (!piece_layout(T, n_seq) || (int64_t)Hv * NT > num_sms - 16) return T > 0 ? 3 : 2;
  const int64_t n_chunks = (T + C - 1) / C;
  const int64_t per = piece_chunks(n_chunks);
  const int pieces = (int)((n_chunks + per - 1) / per);
  const int64_t x = upfront_chunks(n_chunks, per, pieces, Hv, num_sms, (int)(Hv * NT));
  int n = 2 + pieces;
  for (int i = 0; i < pieces; ++i)
    if (((i + 1) * per < n_chunks ? (i + 1) * per : n_chunks) > x) ++n;
  return n;
}

cudaError_t launch_prefill_chunk_tc(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, void* o, int64_t T, int32_t Hk, int32_t Hv,
                                    int64_t qk_stride, int64_t v_stride, const int32_t* cu,
                                    int32_t n_seq, const void* init, void* fin, int state_dtype,
                                    float scale, BlockStates blocks, void* workspace,
                                    cudaStream_t stream) {
  static uint64_t attrs_set = 0;   // one bit per device that has the smem attributes
  static int sm_count[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int num_sms = dev < 64 ? sm_count[dev] : 0;
  if (num_sms == 0) {
    e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev < 64) sm_count[dev] = num_sms;
  }
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
  CUtensorMap mq{}, mk{}, mv{}, mwu{}, mmq{}, mul{}, mo{};
  if (T > 0 && (!make_map(&mq, q, (uint64_t)Hk * D, (uint64_t)T, (uint64_t)qk_stride) ||
                !make_map(&mk, k, (uint64_t)Hk * D, (uint64_t)T, (uint64_t)qk_stride) ||
                !make_map(&mv, v, (uint64_t)Hv * D, (uint64_t)T, (uint64_t)v_stride) ||
                !make_map(&mwu, ws + L.wu, D, (uint64_t)slots * Hv * 2 * C, D) ||
                !make_map(&mmq, ws + L.mq, C, (uint64_t)slots * Hv * C, C) ||
                !make_map(&mul, ws + L.ul, D, (uint64_t)slots * Hv * C, D) ||
                !make_map(&mo, o, (uint64_t)Hv * D, (uint64_t)T, (uint64_t)Hv * D)))
    return cudaErrorInvalidValue;
  chunk_plan_kernel<<<1, 1024, 0, stream>>>(cu, n_seq, T, reinterpret_cast<int32_t*>(ws + L.prefix),
                                            reinterpret_cast<int32_t*>(ws + L.order),
                                            reinterpret_cast<int*>(ws + L.err),
                                            reinterpret_cast<int*>(ws + L.ctr));
  const int user_bf = state_dtype == kBF16 ? 1 : 0;
  const int flags = user_bf * (kStateInitBf16 | kStateFinBf16 | kStateBlocksBf16);
  const int64_t n_chunks = (T + C - 1) / C;
  // persistent intra-chunk grid: two CTAs per SM (shared and tensor memory allow two)
  auto intra_grid = [&](int64_t n_slots) {
    const int64_t items = n_slots * Hk;
    return (unsigned)(items < 2 * (int64_t)num_sms ? items : 2 * (int64_t)num_sms);
  };
  dim3 gc((unsigned)((int64_t)n_seq * Hv * NT));
  if (!piece_layout(T, n_seq) || (int64_t)Hv * NT > num_sms - 16) {
    // one pass: every chunk's intra-chunk work, then the chains
    if (T > 0)
      chunk_intra_kernel<<<intra_grid(slots), 128, kIntraSmem, stream>>>(
          mq, mk, mv, mwu, mmq, mul, g, beta, cu, n_seq, T, Hk, Hv, ws, 0, (int32_t)slots, 0);
    chunk_chain_kernel<<<gc, kChainThreads, kChainSmem, stream>>>(
        mq, mk, mwu, mmq, mul, mo, cu, n_seq, T, Hk, Hv, ws, reinterpret_cast<int*>(ws + L.err), init, fin,
        flags, static_cast<bf16*>(o), scale, blocks, 0, INT32_MAX);
    return cudaGetLastError();
  }
  // One long sequence in pieces of piece_chunks() chunks. The intra-chunk work of the first x
  // chunks (upfront_chunks) runs first as one launch on the whole GPU; then the chain pieces
  // run back to back on a high-priority stream, piece i once the intra-chunk work of its
  // chunks is done, beside the intra-chunk work of the rest on a low-priority stream, one
  // launch up to the end of each piece, each with a persistent grid sized to the SMs the chain
  // leaves free (the chain takes 2 Hv SMs). The state goes from one chain piece to the next
  // through the workspace in fp32. Only events order the streams: no kernel waits for another.
  const int64_t per = piece_chunks(n_chunks);
  const int pieces = (int)((n_chunks + per - 1) / per);   // at most kTargetPieces + 1 <= kMaxPieces
  const int chain_ctas = (int)gc.x;
  const int64_t x = upfront_chunks(n_chunks, per, pieces, Hv, num_sms, chain_ctas);
  PieceStreams* ps = piece_streams(dev);
  if (ps == nullptr) return cudaErrorInitializationError;
  std::lock_guard<std::mutex> lock(ps->mu);   // the events are reused by every call on this device
  void* carry = ws + L.carry;
  cudaEvent_t* ev = ps->ev;
  // slot s of a single sequence is its chunk s; the padding slot goes with the last chunk
  auto slot_end = [&](int64_t c) { return (int32_t)(c == n_chunks ? slots : c); };
  if ((e = cudaEventRecord(ev[0], stream)) != cudaSuccess) return e;   // the plan is done
  if ((e = cudaStreamWaitEvent(ps->side[0], ev[0], 0)) != cudaSuccess) return e;
  chunk_intra_kernel<<<intra_grid(slot_end(x)), 128, kIntraSmem, ps->side[0]>>>(
      mq, mk, mv, mwu, mmq, mul, g, beta, cu, n_seq, T, Hk, Hv, ws, 0, slot_end(x), 0);
  if ((e = cudaEventRecord(ev[1], ps->side[0])) != cudaSuccess) return e;   // chunks 0 .. x-1
  if ((e = cudaStreamWaitEvent(ps->chain, ev[1], 0)) != cudaSuccess) return e;
  auto chain_piece = [&](int i, cudaEvent_t started) {
    const int64_t c0 = i * per, c1 = (i + 1) * per < n_chunks ? (i + 1) * per : n_chunks;
    const bool first = i == 0, last = i == pieces - 1;
    const int f = (first ? user_bf * kStateInitBf16 : 0) | (last ? user_bf * kStateFinBf16 : 0) |
                  user_bf * kStateBlocksBf16;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = gc;
    cfg.blockDim = dim3(kChainThreads);
    cfg.dynamicSmemBytes = kChainSmem;
    cfg.stream = ps->chain;
    cudaLaunchAttribute attr[1];
    if (started != nullptr) {   // fires once the piece's CTAs have all begun (at worst at its end)
      attr[0].id = cudaLaunchAttributeLaunchCompletionEvent;
      attr[0].val.launchCompletionEvent.event = started;
      attr[0].val.launchCompletionEvent.flags = 0;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, chunk_chain_kernel, mq, mk, mwu, mmq, mul, mo, cu, n_seq, T, Hk, Hv,
                              (const uint8_t*)ws, reinterpret_cast<int*>(ws + L.err), first ? init : carry,
                              last ? fin : carry, f, static_cast<bf16*>(o), scale, blocks, (int32_t)c0,
                              (int32_t)(last ? INT32_MAX : c1));
  };
  // chain piece 0 first: the intra-chunk work beside the chains starts only once its CTAs have
  // all begun, so that they take whole SMs before the intra-chunk grid spreads over the GPU
  // (x >= the first piece: chain piece 0 waits for nothing on that stream, so no cycle)
  if ((e = chain_piece(0, ev[kMaxPieces + 1])) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(ps->side[1], ev[0], 0)) != cudaSuccess) return e;   // the plan
  if ((e = cudaStreamWaitEvent(ps->side[1], ev[kMaxPieces + 1], 0)) != cudaSuccess) return e;
  const int64_t free_ctas = 2 * (int64_t)(num_sms - chain_ctas);
  int64_t done = x;
  for (int i = 0; i < pieces; ++i) {   // the rest, up to the end of each piece
    const int64_t c1 = (i + 1) * per < n_chunks ? (i + 1) * per : n_chunks;
    if (c1 <= done) continue;
    const unsigned grid = intra_grid(slot_end(c1) - done);
    chunk_intra_kernel<<<(unsigned)(grid < free_ctas ? grid : free_ctas), 128, kIntraSmem, ps->side[1]>>>(
        mq, mk, mv, mwu, mmq, mul, g, beta, cu, n_seq, T, Hk, Hv, ws, (int32_t)done, slot_end(c1), 1 + i);
    if ((e = cudaEventRecord(ev[2 + i], ps->side[1])) != cudaSuccess) return e;
    done = c1;
  }
  for (int i = 1; i < pieces; ++i) {   // after the records above: each wait is on this call's
    const int64_t c1 = (i + 1) * per < n_chunks ? (i + 1) * per : n_chunks;
    if (c1 > x && (e = cudaStreamWaitEvent(ps->chain, ev[2 + i], 0)) != cudaSuccess) return e;
    if ((e = chain_piece(i, nullptr)) != cudaSuccess) return e;
  }
  if ((e = cudaEventRecord(ev[kMaxPieces + 2], ps->chain)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(stream, ev[kMaxPieces + 2], 0)) != cudaSuccess) return e;   // join
  return cudaGetLastError();
}

}  // namespace gdn
