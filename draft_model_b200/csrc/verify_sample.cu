// Stochastic verification at T > 0 (speculative sampling) of a draft block.
//
// The pages report Domino's acceptance at temperature 1 (Domino study notes,
// gsyq.cn, §三.2(1)) without a verification mechanism; this is the standard
// lossless rule on the draft distributions p_i = softmax(L_i / T) and the target
// distributions q_i = softmax(Lq_i / T): accept t_i with probability
// min(1, q_i(t_i) / p_i(t_i)); at the first rejection emit a sample of
// norm(max(0, q_i - p_i)); after K acceptances a bonus sample of q_{K+1}.
// Randomness: Philox4x32-10 with key = seed on streams the draft's Gumbel picks
// never use (counter word 3): acceptance uniforms (0, i-1, b, 2) word 0;
// resampling Gumbel noise (j >> 2, i-1, b, 1) word j & 3, drawn by Gumbel-max.
//
// Launches (rows = B (2K + 1): the K draft rows, then the K + 1 target rows):
//   row_lse_partial_kernel (loss.cu)  chunked log-sum-exp of every row at scale
//                          1/T and the logits of the drafted tokens;
//   accept_kernel          one warp per request: the K acceptance tests in parallel;
//   resample_kernel        CTA per (vocabulary chunk, request): Gumbel-max over
//                          the residual (or the bonus row), 64-bit atomicMax;
//   finish_kernel          warp per request: tau and the emitted token (a draw
//                          from q when the residual had no positive fp32 entry).
// HBM-bound: the draft and target rows are read once, plus one row pair again.
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "domino_internal.h"

namespace domino {
namespace {

constexpr uint32_t kStreamResample = 1u;
constexpr uint32_t kStreamAccept = 2u;

__device__ __forceinline__ float philox_uniform(uint64_t seed, uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                uint32_t word) {
  const Philox4 r = philox4x32_10(c0, c1, c2, c3, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  const uint32_t w = word == 0u ? r.x[0] : word == 1u ? r.x[1] : word == 2u ? r.x[2] : r.x[3];
  return (static_cast<float>(w >> 9) * 2.0f + 1.0f) * 5.9604644775390625e-8f;  // (2 (w >> 9) + 1) 2^-24, exact
}

// log-sum-exp of row r from its chunk partials (fp32 terms, fp64 sum)
__device__ __forceinline__ double row_lse(const float2* part, int r, int chunks) {
  const float2* p = part + static_cast<size_t>(r) * chunks;
  float M = -INFINITY;
  for (int c = 0; c < chunks; ++c) M = fmaxf(M, p[c].x);
  double S = 0.0;
  for (int c = 0; c < chunks; ++c)
    if (p[c].x != -INFINITY) S += static_cast<double>(p[c].y * expf(p[c].x - M));
  return static_cast<double>(M) + log(S);
}

// One warp per request, lane i = position i + 1 (K <= 32): every lane takes its
// acceptance test, the first rejecting lane ends the block.
__global__ void __launch_bounds__(32) accept_kernel(const float2* __restrict__ part, const float* __restrict__ picked,
                                                    int B, int K, int chunks, float scale, uint64_t seed,
                                                    int32_t* __restrict__ pos_out, double* __restrict__ lse_p_out,
                                                    double* __restrict__ lse_q_out) {
  const int b = blockIdx.x, lane = threadIdx.x;
  const int R0 = B * K;
  double lp = 0.0, lq = 0.0;
  bool reject = false;
  if (lane < K) {
    const int rp = b * K + lane, rq = R0 + b * (K + 1) + lane;
    lp = row_lse(part, rp, chunks);
    lq = row_lse(part, rq, chunks);
    const double logp = static_cast<double>(picked[rp]) * scale - lp;
    const double logq = static_cast<double>(picked[rq]) * scale - lq;
    const float u = philox_uniform(seed, 0u, static_cast<uint32_t>(lane), static_cast<uint32_t>(b), kStreamAccept, 0u);
    reject = !(static_cast<double>(u) < exp(logq - logp));   // u < 1, so min(1, .) is implied
  }
  const uint32_t rejects = __ballot_sync(0xFFFFFFFFu, reject);
  const int pos = rejects ? __ffs(rejects) - 1 : K;
  const int src = pos < K ? pos : 0;
  const double lp_pos = __shfl_sync(0xFFFFFFFFu, lp, src);
  const double lq_pos = __shfl_sync(0xFFFFFFFFu, lq, src);
  if (lane == 0) {
    pos_out[b] = pos;
    lse_p_out[b] = pos < K ? lp_pos : 0.0;
    lse_q_out[b] = pos < K ? lq_pos : row_lse(part, R0 + b * (K + 1) + K, chunks);
  }
}

__global__ void __launch_bounds__(256) resample_kernel(const float* __restrict__ draft_logits,
                                                       const float* __restrict__ target_logits, int B, int K, int V,
                                                       float scale, int chunks, uint64_t seed,
                                                       const int32_t* __restrict__ pos_in,
                                                       const double* __restrict__ lse_p_in,
                                                       const double* __restrict__ lse_q_in,
                                                       unsigned long long* __restrict__ best) {
  const int b = blockIdx.y, c = blockIdx.x;
  const int pos = pos_in[b];
  const bool bonus = pos >= K;
  const float lse_p = static_cast<float>(lse_p_in[b]), lse_q = static_cast<float>(lse_q_in[b]);
  const float* rq = target_logits + (static_cast<size_t>(b) * (K + 1) + pos) * V;
  const float* rp = bonus ? nullptr : draft_logits + (static_cast<size_t>(b) * K + pos) * V;
  const int lo = static_cast<int>(static_cast<long long>(V) * c / chunks);
  const int hi = static_cast<int>(static_cast<long long>(V) * (c + 1) / chunks);
  unsigned long long key = 0ull;
  for (int j = lo + static_cast<int>(threadIdx.x); j < hi; j += blockDim.x) {
    const float lq = rq[j] * scale - lse_q;      // log q_j
    float score;
    if (bonus) {
      score = lq;
    } else {
      const float d = expf(lq) - expf(rp[j] * scale - lse_p);   // q_j - p_j
      score = d > 0.f ? logf(d) : -INFINITY;
    }
    if (score == -INFINITY) continue;
    const float u = philox_uniform(seed, static_cast<uint32_t>(j) >> 2, static_cast<uint32_t>(pos),
                                   static_cast<uint32_t>(b), kStreamResample, static_cast<uint32_t>(j) & 3u);
    const unsigned long long k = argmax_key(score - logf(-logf(u)), static_cast<uint32_t>(j));
    key = k > key ? k : key;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, key, o);
    key = other > key ? other : key;
  }
  __shared__ unsigned long long wkey[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) wkey[warp] = key;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long k = wkey[0];
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) k = wkey[w] > k ? wkey[w] : k;
    if (k) atomicMax(&best[b], k);
  }
}

// One warp per request: tau and the emitted token.  A rejection whose residual
// max(0, q - p) had no positive entry in fp32 (p and q agree to working
// precision except at the drafted token, whose probability lies below it) left
// no key; the token is then drawn from q at that position with the same noise
// (Gumbel-max over log q), which keeps the emitted token's law q.
__global__ void __launch_bounds__(32) finish_kernel(const float* __restrict__ target_logits, int K, int V, float scale,
                                                    uint64_t seed, const unsigned long long* __restrict__ best,
                                                    const int32_t* __restrict__ pos_in,
                                                    const double* __restrict__ lse_q_in,
                                                    int32_t* __restrict__ tau_out, int32_t* __restrict__ token_out) {
  const int b = blockIdx.x, lane = threadIdx.x;
  const int pos = pos_in[b];
  unsigned long long key = best[b];
  if (key == 0ull) {   // warp-uniform
    const float lse_q = static_cast<float>(lse_q_in[b]);
    const float* rq = target_logits + (static_cast<size_t>(b) * (K + 1) + pos) * V;
    for (int j = lane; j < V; j += 32) {
      const float u = philox_uniform(seed, static_cast<uint32_t>(j) >> 2, static_cast<uint32_t>(pos),
                                     static_cast<uint32_t>(b), kStreamResample, static_cast<uint32_t>(j) & 3u);
      const unsigned long long k = argmax_key(rq[j] * scale - lse_q - logf(-logf(u)), static_cast<uint32_t>(j));
      key = k > key ? k : key;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, key, o);
      key = other > key ? other : key;
    }
  }
  if (lane == 0) {
    tau_out[b] = pos;
    token_out[b] = static_cast<int32_t>(argmax_key_index(key));
  }
}

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t verify_sample_scratch_bytes(int B, int K, int V) {
  const size_t rows = static_cast<size_t>(B) * (2 * K + 1);
  const int chunks = lse_chunks(static_cast<int>(rows), V);
  return al256(rows * chunks * sizeof(float2)) + al256(rows * 4) + al256(static_cast<size_t>(B) * 4) +
         2 * al256(static_cast<size_t>(B) * 8) + al256(static_cast<size_t>(B) * 8);
}

cudaError_t launch_verify_sample(const float* draft_logits, const float* target_logits, const int32_t* draft, int B,
                                 int K, int V, float temperature, uint64_t seed, void* scratch, int32_t* tau_out,
                                 int32_t* token_out, Control* ctl, cudaStream_t stream) {
  const size_t rows = static_cast<size_t>(B) * (2 * K + 1);
  const int chunks = lse_chunks(static_cast<int>(rows), V);
  char* p = static_cast<char*>(scratch);
  float2* part = reinterpret_cast<float2*>(p);
  p += al256(rows * chunks * sizeof(float2));
  float* picked = reinterpret_cast<float*>(p);
  p += al256(rows * 4);
  int32_t* pos = reinterpret_cast<int32_t*>(p);
  p += al256(static_cast<size_t>(B) * 4);
  double* lse_p = reinterpret_cast<double*>(p);
  p += al256(static_cast<size_t>(B) * 8);
  double* lse_q = reinterpret_cast<double*>(p);
  p += al256(static_cast<size_t>(B) * 8);
  unsigned long long* best = reinterpret_cast<unsigned long long*>(p);
  const float scale = 1.0f / temperature;
  cudaError_t e = cudaMemsetAsync(best, 0, static_cast<size_t>(B) * 8, stream);
  if (e != cudaSuccess) return e;
  e = launch_row_lse_partial(draft_logits, K, target_logits, K + 1, B, V, scale, chunks, draft, K, part, picked, ctl,
                             stream);
  if (e != cudaSuccess) return e;
  accept_kernel<<<B, 32, 0, stream>>>(part, picked, B, K, chunks, scale, seed, pos, lse_p, lse_q);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int rchunks = lse_chunks(B, V);
  resample_kernel<<<dim3(rchunks, B), 256, 0, stream>>>(draft_logits, target_logits, B, K, V, scale, rchunks, seed, pos,
                                                        lse_p, lse_q, best);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  finish_kernel<<<B, 32, 0, stream>>>(target_logits, K, V, scale, seed, best, pos, lse_q, tau_out, token_out);
  return cudaGetLastError();
}

}  // namespace domino
