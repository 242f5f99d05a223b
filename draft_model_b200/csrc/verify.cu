// Stage 3: greedy verification.  tau_b = number of leading block positions where
// the draft token equals the target's (Domino study notes, gsyq.cn, §一.1 接受长度τ;
// digest page "大三本科生一作…", §4 简单批量验证).
//
// One warp per request: lane i compares position i, a ballot collects the
// mismatches, and the index of the lowest mismatch is tau (K when none).
#include <cstdint>

#include "domino_internal.h"

namespace domino {
namespace {

__global__ void __launch_bounds__(256) verify_kernel(const int32_t* __restrict__ draft,
                                                     const int32_t* __restrict__ target, int B, int K,
                                                     int32_t* __restrict__ tau) {
  const int b = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const bool miss = lane < K && draft[static_cast<size_t>(b) * K + lane] != target[static_cast<size_t>(b) * K + lane];
  const unsigned m = __ballot_sync(0xFFFFFFFFu, miss);
  if (lane == 0) tau[b] = m ? __ffs(static_cast<int>(m)) - 1 : K;
}

}  // namespace

cudaError_t launch_verify(const int32_t* draft, const int32_t* target, int B, int K, int32_t* tau,
                          cudaStream_t stream) {
  verify_kernel<<<(B + 7) / 8, 256, 0, stream>>>(draft, target, B, K, tau);
  return cudaGetLastError();
}

}  // namespace domino
