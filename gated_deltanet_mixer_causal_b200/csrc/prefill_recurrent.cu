// prefill_recurrent.cu -- the gated delta rule token by token in fp32 on CUDA cores.
//
// This is the fp32-activation prefill: it evaluates S_t = alpha_t S_{t-1}(I - beta_t k k^T)
// + beta_t v k^T, o_t = scale S_t q_t in exactly the page's order (Qwen3.5 page, section
// 5), so fp32 inputs meet a 1e-4 relative gate against the fp64 recurrence.
//
// Rows of S evolve independently (the update multiplies S from the right), so a sequence's
// state splits over CTAs by value rows: a CTA holds kWarps x kRows rows of one
// (sequence, value head) in registers for the whole sequence, one warp per kRows rows,
// dk/32 columns per lane. Per token every warp reads q_t, k_t (its key head), v_t, g_t,
// beta_t, and performs one warp reduction of 3 + 2 kRows values:
//   |q|^2, |k|^2, k.q and, per row, s.k and s.q (un-normalised; scaled after),
// then u = beta (v_i - alpha s.k^), s <- alpha s + u k^, o_i = scale (alpha s.q^ + u k^.q^).
// Optionally the rows are also stored after every block_tokens tokens (block states). States
// in HBM are fp32 or bf16 storage (the arithmetic is fp32 either way).
#include "common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kWarps = 4;
constexpr int kRows = 4;           // rows per warp
constexpr float kEps = 1e-6f;

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
prefill_recurrent_kernel(const T* __restrict__ q, const T* __restrict__ k,
                         const T* __restrict__ v, const float* __restrict__ g,
                         const float* __restrict__ beta, T* __restrict__ o, int64_t T_tok,
                         int32_t Hk, int32_t Hv, int64_t qk_stride, int64_t v_stride,
                         const int32_t* __restrict__ cu, const void* init, void* fin,
                         int32_t state_bf16, float scale, int32_t l2norm, BlockStates blocks) {
  constexpr int VEC = D >= 32 ? D / 32 : 1;
  constexpr int kRowsPerCta = kWarps * kRows;
  constexpr int kRowBlocks = (D + kRowsPerCta - 1) / kRowsPerCta;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rb = blockIdx.x % kRowBlocks;
  const int h = (blockIdx.x / kRowBlocks) % Hv;
  const int32_t n = blockIdx.x / (kRowBlocks * Hv);
  const int hk = h / (Hv / Hk);
  const int row0 = rb * kRowsPerCta + warp * kRows;
  const bool active = lane * VEC < D;
  const bool sbf = state_bf16 != 0;

  int64_t bos, eos;
  seq_bounds(cu, n, T_tok, bos, eos);

  float s[kRows][VEC];
  const int64_t sbase = ((int64_t)n * Hv + h) * D * D;
#pragma unroll
  for (int r = 0; r < kRows; ++r)
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      const int row = row0 + r, col = lane * VEC + j;
      s[r][j] = (init != nullptr && row < D && active) ? state_load(init, sbase + (int64_t)row * D + col, sbf) : 0.f;
    }

  for (int64_t t = bos; t < eos; ++t) {
    float qv[VEC], kv[VEC];
    if (active) {
      VecIO<T, VEC>::load(q + t * qk_stride + (int64_t)hk * D + lane * VEC, qv);
      VecIO<T, VEC>::load(k + t * qk_stride + (int64_t)hk * D + lane * VEC, kv);
    } else {
#pragma unroll
      for (int j = 0; j < VEC; ++j) { qv[j] = 0.f; kv[j] = 0.f; }
    }
    float vr[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      vr[r] = (row0 + r < D) ? to_f<T>(v[t * v_stride + (int64_t)h * D + row0 + r]) : 0.f;
    const float alpha = expf(g[t * Hv + h]);
    const float bt = beta[t * Hv + h];

    float red[3 + 2 * kRows];
    red[0] = red[1] = red[2] = 0.f;
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      red[0] = fmaf(qv[j], qv[j], red[0]);
      red[1] = fmaf(kv[j], kv[j], red[1]);
      red[2] = fmaf(kv[j], qv[j], red[2]);
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      float a = 0.f, c = 0.f;
#pragma unroll
      for (int j = 0; j < VEC; ++j) { a = fmaf(s[r][j], kv[j], a); c = fmaf(s[r][j], qv[j], c); }
      red[3 + 2 * r] = a; red[4 + 2 * r] = c;
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
      for (int e = 0; e < 3 + 2 * kRows; ++e) red[e] += __shfl_xor_sync(0xffffffffu, red[e], m);

    const float iq = l2norm ? 1.0f / sqrtf(red[0] + kEps) : 1.0f;
    const float ik = l2norm ? 1.0f / sqrtf(red[1] + kEps) : 1.0f;
    const float kqh = red[2] * iq * ik;
    float kh[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) kh[j] = kv[j] * ik;
    float outv[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const float sk = red[3 + 2 * r] * ik, sq = red[4 + 2 * r] * iq;
      const float u = bt * (vr[r] - alpha * sk);
#pragma unroll
      for (int j = 0; j < VEC; ++j) s[r][j] = fmaf(alpha, s[r][j], u * kh[j]);
      outv[r] = scale * fmaf(alpha, sq, u * kqh);
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (lane == r && row0 + r < D) o[(t * Hv + h) * (int64_t)D + row0 + r] = from_f<T>(outv[r]);
    const int64_t done = t - bos + 1;   // tokens of the sequence consumed so far
    if (blocks.block_tokens > 0 && done % blocks.block_tokens == 0) {
      const int64_t brow = (int64_t)blocks.rows[n] + done / blocks.block_tokens - 1;
      if (brow >= 0 && brow < blocks.n_rows) {
        const int64_t dst = (brow * Hv + h) * D * D;
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
          for (int j = 0; j < VEC; ++j) {
            const int row = row0 + r, col = lane * VEC + j;
            if (row < D && active) state_store(blocks.states, dst + (int64_t)row * D + col, s[r][j], sbf);
          }
      }
    }
  }

  if (fin != nullptr) {
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        const int row = row0 + r, col = lane * VEC + j;
        if (row < D && active) state_store(fin, sbase + (int64_t)row * D + col, s[r][j], sbf);
      }
  }
}

template <typename T, int D>
cudaError_t launch_typed(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, void* o, int64_t n_tok, int32_t Hk, int32_t Hv,
                         int64_t qks, int64_t vs, const int32_t* cu, int32_t n_seq,
                         const void* init, void* fin, int32_t sbf, float scale, int32_t l2,
                         BlockStates bl, cudaStream_t st) {
  constexpr int kRowBlocks = (D + kWarps * kRows - 1) / (kWarps * kRows);
  dim3 grid((unsigned)((int64_t)n_seq * Hv * kRowBlocks));
  prefill_recurrent_kernel<T, D><<<grid, kWarps * 32, 0, st>>>(
      (const T*)q, (const T*)k, (const T*)v, g, beta, (T*)o, n_tok, Hk, Hv, qks, vs, cu, init, fin,
      sbf, scale, l2, bl);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_d(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, void* o, int64_t n_tok, int32_t Hk, int32_t Hv, int32_t d,
                     int64_t qks, int64_t vs, const int32_t* cu, int32_t n_seq, const void* init,
                     void* fin, int32_t sbf, float scale, int32_t l2, BlockStates bl, cudaStream_t st) {
  switch (d) {
    case 16: return launch_typed<T, 16>(q, k, v, g, beta, o, n_tok, Hk, Hv, qks, vs, cu, n_seq, init, fin, sbf, scale, l2, bl, st);
    case 32: return launch_typed<T, 32>(q, k, v, g, beta, o, n_tok, Hk, Hv, qks, vs, cu, n_seq, init, fin, sbf, scale, l2, bl, st);
    case 64: return launch_typed<T, 64>(q, k, v, g, beta, o, n_tok, Hk, Hv, qks, vs, cu, n_seq, init, fin, sbf, scale, l2, bl, st);
    default: return launch_typed<T, 128>(q, k, v, g, beta, o, n_tok, Hk, Hv, qks, vs, cu, n_seq, init, fin, sbf, scale, l2, bl, st);
  }
}

}  // namespace

cudaError_t launch_prefill_recurrent(int dtype, const void* q, const void* k, const void* v,
                                     const float* g, const float* beta, void* o, int64_t T,
                                     int32_t Hk, int32_t Hv, int32_t d, int64_t qk_stride,
                                     int64_t v_stride, const int32_t* cu, int32_t n_seq,
                                     const void* init, void* fin, int state_dtype, float scale,
                                     int32_t l2norm, BlockStates blocks, cudaStream_t stream) {
  const int32_t sbf = state_dtype == kBF16 ? 1 : 0;
  if (dtype == kF32)
    return launch_d<float>(q, k, v, g, beta, o, T, Hk, Hv, d, qk_stride, v_stride, cu, n_seq,
                           init, fin, sbf, scale, l2norm, blocks, stream);
  return launch_d<bf16>(q, k, v, g, beta, o, T, Hk, Hv, d, qk_stride, v_stride, cu, n_seq, init,
                        fin, sbf, scale, l2norm, blocks, stream);
}

}  // namespace gdn
