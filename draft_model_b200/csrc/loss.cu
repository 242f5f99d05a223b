// Base-anchored curriculum loss of Domino's training forward (sm_100a).
//
// Domino study notes (gsyq.cn), §二.2(2) Base-Anchored 渐进式课程损失: the base
// logits and the final corrected logits are supervised jointly,
//     L = (1 - lambda) L_final + lambda L_base,
// and every block position's loss carries an exponentially decaying weight.
// Per position the loss is the cross-entropy -log softmax(L)[y]; the decay
// weight of position i+1 is gamma^i; L_final and L_base are weighted means over
// positions and means over the batch.
//
// Two launches over rows of fp32 logits (R = B K rows per tensor, V columns):
//   row_lse_partial_kernel  one CTA per (row, vocabulary chunk): coalesced pass
//                      with an online (max, sum of exp) per thread, merged across
//                      the CTA; the chunk holding the label also records its logit;
//   ce_combine_kernel  one CTA: log-sum-exp of every row from its chunks, the
//                      row's cross-entropy, and the weighted loss, summed in fp64
//                      in a fixed order (deterministic).
// HBM-bound: both logit tensors are read once (2 R V 4 bytes).
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "domino_internal.h"

namespace domino {
namespace {

constexpr int CE_THREADS = 256;
constexpr int COMBINE_THREADS = 1024;

struct MS {
  float m, s;  // running max and sum of exp(x - m)
};

__device__ __forceinline__ MS ms_merge(MS a, MS b) {
  const float m = fmaxf(a.m, b.m);
  if (m == -INFINITY) return {m, 0.f};
  return {m, a.s * __expf(a.m - m) + b.s * __expf(b.m - m)};
}

__device__ __forceinline__ void ms_push(MS& a, float x) {
  if (x > a.m) {
    a.s = a.s * __expf(a.m - x) + 1.f;
    a.m = x;
  } else {
    a.s += __expf(x - a.m);
  }
}

// Row log-sum-exp partials.  Rows r in [0, B (K0 + K1)): the B K0 rows of X0
// (request b, position i at row b K0 + i), then the B K1 rows of X1.  CTA
// (chunk c, row r) merges (max, sum exp(y - max)) of y = scale * x over the
// row's c-th vocabulary chunk into part[r chunks + c]; the chunk holding
// idx[b Kidx + i] (for i < Kidx, when idx is given) records that raw logit in
// picked[r].  Out-of-range indices are clamped and flagged.
__global__ void __launch_bounds__(CE_THREADS) row_lse_partial_kernel(const float* __restrict__ X0, int K0,
                                                                     const float* __restrict__ X1, int K1, int B,
                                                                     int V, float scale, int chunks,
                                                                     const int32_t* __restrict__ idx, int Kidx,
                                                                     float2* __restrict__ part,
                                                                     float* __restrict__ picked, Control* ctl) {
  const int r = blockIdx.y, c = blockIdx.x;
  const int R0 = B * K0;
  const bool first = r < R0;
  const int rr = first ? r : r - R0;
  const int Kr = first ? K0 : K1;
  const int b = rr / Kr, i = rr % Kr;
  const float* row = (first ? X0 : X1) + static_cast<size_t>(rr) * V;
  const int lo = static_cast<int>(static_cast<long long>(V) * c / chunks);
  const int hi = static_cast<int>(static_cast<long long>(V) * (c + 1) / chunks);
  MS a{-INFINITY, 0.f};
  int v = lo + static_cast<int>(threadIdx.x);
  // eight independent loads in flight per thread (about 56 KB per SM with seven CTAs)
  for (; v + 7 * CE_THREADS < hi; v += 8 * CE_THREADS) {
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = __ldcs(row + v + u * CE_THREADS);
#pragma unroll
    for (int u = 0; u < 8; ++u) ms_push(a, x[u] * scale);
  }
  for (; v < hi; v += CE_THREADS) ms_push(a, __ldcs(row + v) * scale);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const MS o2{__shfl_xor_sync(0xFFFFFFFFu, a.m, o), __shfl_xor_sync(0xFFFFFFFFu, a.s, o)};
    a = ms_merge(a, o2);
  }
  __shared__ MS warp_ms[CE_THREADS / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) warp_ms[warp] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    MS t = warp_ms[0];
    for (int w = 1; w < CE_THREADS / 32; ++w) t = ms_merge(t, warp_ms[w]);
    part[static_cast<size_t>(r) * chunks + c] = make_float2(t.m, t.s);
    if (idx && i < Kidx) {
      int y = idx[static_cast<size_t>(b) * Kidx + i];
      if (y < 0 || y >= V) {
        if (c == 0 && first) raise_error(ctl, ERRBIT_BAD_TOKEN);
        y = min(max(y, 0), V - 1);
      }
      if (y >= lo && y < hi) picked[r] = row[y];
    }
  }
}

__global__ void __launch_bounds__(COMBINE_THREADS) ce_combine_kernel(const float2* __restrict__ part,
                                                                     const float* __restrict__ picked, int R, int K,
                                                                     int chunks, float lambda, float gamma,
                                                                     float* __restrict__ ce_out,
                                                                     float* __restrict__ loss_out) {
  __shared__ double red[COMBINE_THREADS];
  double acc = 0.0;
  for (int rr = threadIdx.x; rr < R; rr += COMBINE_THREADS) {
    double ce[2];
    for (int t = 0; t < 2; ++t) {
      const int r = t * R + rr;
      const float2* p = part + static_cast<size_t>(r) * chunks;
      float M = -INFINITY;
      for (int c = 0; c < chunks; ++c) M = fmaxf(M, p[c].x);
      double S = 0.0;
      for (int c = 0; c < chunks; ++c)
        if (p[c].x != -INFINITY) S += static_cast<double>(p[c].y * expf(p[c].x - M));
      ce[t] = static_cast<double>(M) + log(S) - static_cast<double>(picked[r]);
      if (ce_out) ce_out[static_cast<size_t>(rr) * 2 + t] = static_cast<float>(ce[t]);
    }
    const double w = pow(static_cast<double>(gamma), static_cast<double>(rr % K));
    acc += w * ((1.0 - lambda) * ce[0] + static_cast<double>(lambda) * ce[1]);
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = COMBINE_THREADS / 2; s > 0; s >>= 1) {
    if (static_cast<int>(threadIdx.x) < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    double wsum = 0.0;
    for (int i = 0; i < K; ++i) wsum += pow(static_cast<double>(gamma), static_cast<double>(i));
    *loss_out = static_cast<float>(red[0] / (static_cast<double>(R / K) * wsum));
  }
}

}  // namespace

int lse_chunks(int rows, int V) {
  // about 1024 CTAs over the rows, chunks of at least 2048 logits, at most 64
  int c = (1024 + rows - 1) / rows;
  const int cap = V / 2048 > 0 ? V / 2048 : 1;
  if (c > cap) c = cap;
  if (c > 64) c = 64;
  return c < 1 ? 1 : c;
}

size_t loss_scratch_bytes(int B, int K, int V) {
  const size_t rows = 2ull * B * K;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  return al(rows * lse_chunks(static_cast<int>(rows), V) * sizeof(float2)) + al(rows * sizeof(float));
}

cudaError_t launch_row_lse_partial(const float* X0, int K0, const float* X1, int K1, int B, int V, float scale,
                                   int chunks, const int32_t* idx, int Kidx, float2* part, float* picked, Control* ctl,
                                   cudaStream_t stream) {
  row_lse_partial_kernel<<<dim3(chunks, B * (K0 + K1)), CE_THREADS, 0, stream>>>(X0, K0, X1, K1, B, V, scale, chunks,
                                                                                 idx, Kidx, part, picked, ctl);
  return cudaGetLastError();
}

cudaError_t launch_curriculum_loss(const float* final_logits, const float* base_logits, const int32_t* labels, int B,
                                   int K, int V, float lambda, float gamma, void* scratch, float* ce_out,
                                   float* loss_out, Control* ctl, cudaStream_t stream) {
  const int R = B * K;
  const int chunks = lse_chunks(2 * R, V);
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  float2* part = static_cast<float2*>(scratch);
  float* picked = reinterpret_cast<float*>(static_cast<char*>(scratch) + al(2ull * R * chunks * sizeof(float2)));
  row_lse_partial_kernel<<<dim3(chunks, 2 * R), CE_THREADS, 0, stream>>>(final_logits, K, base_logits, K, B, V, 1.f,
                                                                         chunks, labels, K, part, picked, ctl);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ce_combine_kernel<<<1, COMBINE_THREADS, 0, stream>>>(part, picked, R, K, chunks, lambda, gamma, ce_out, loss_out);
  return cudaGetLastError();
}

}  // namespace domino
