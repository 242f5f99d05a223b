// Stage 1 for fp32 weights on CUDA cores (no tf32: the fp32 path promises 1e-4
// on final logits, which tf32's 10-bit mantissa would not keep).
// out[m, v] = sum_k W[v, k] h[m, k] with W's rows ldw elements apart: the base
// logits (W = W_lm; Domino study notes, gsyq.cn, §二.1(1)) and the hidden-state
// half of the bottleneck pre-activation (W = W1[:, 0:d]; yhxrc.cn article, §四).
//
// 64 (vocabulary) x 32 (positions) output tile per 256-thread block, k-tiles of
// 32 staged in shared memory; each thread owns 8 outputs of one vocabulary row.
#include <cstdint>

#include "domino_internal.h"

namespace domino {
namespace {

constexpr int TV = 64, TM = 32, TK = 32;

__global__ void __launch_bounds__(256) lm_head_f32_kernel(const float* __restrict__ w, const float* __restrict__ h,
                                                          float* __restrict__ out, int V, int M, int Kd, int ldw) {
  __shared__ float ws[TK][TV + 1];
  __shared__ float hs[TK][TM + 1];
  const int v0 = blockIdx.x * TV, m0 = blockIdx.y * TM;
  const int tv = threadIdx.x % TV, tm = threadIdx.x / TV;  // tm in [0, 4)
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < Kd; k0 += TK) {
    for (int q = threadIdx.x; q < TV * TK; q += 256) {
      const int r = q / TK, c = q % TK;
      ws[c][r] = (v0 + r < V && k0 + c < Kd) ? w[static_cast<size_t>(v0 + r) * ldw + k0 + c] : 0.f;
    }
    for (int q = threadIdx.x; q < TM * TK; q += 256) {
      const int r = q / TK, c = q % TK;
      hs[c][r] = (m0 + r < M && k0 + c < Kd) ? h[static_cast<size_t>(m0 + r) * Kd + k0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < TK; ++c) {
      const float wv = ws[c][tv];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = fmaf(wv, hs[c][tm + 4 * j], acc[j]);
    }
    __syncthreads();
  }
  const int v = v0 + tv;
  if (v < V) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int m = m0 + tm + 4 * j;
      if (m < M) out[static_cast<size_t>(m) * V + v] = acc[j];
    }
  }
}

}  // namespace

cudaError_t launch_lm_head_f32(const float* w, const float* hidden, float* out, int V, int M, int Kd, int ldw,
                               cudaStream_t stream) {
  const dim3 grid((V + TV - 1) / TV, (M + TM - 1) / TM);
  lm_head_f32_kernel<<<grid, 256, 0, stream>>>(w, hidden, out, V, M, Kd, ldw);
  return cudaGetLastError();
}

}  // namespace domino
