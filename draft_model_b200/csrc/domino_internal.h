// Internal declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace domino {

struct Control;

// Bytes per slot of the correction loop's weight ring.
constexpr uint32_t kLoopSlotBytes = 16384;
// Largest grid the correction loop is planned for (one CTA per SM).
constexpr int kLoopMaxGrid = 192;
// int64 words between consecutive entries of the bottleneck accumulator (each
// entry in its own 32-byte sector, so concurrent reductions do not share one).
constexpr int kUaccStride = 4;
// Bytes of the bottleneck accumulator: 2 buffers x 8 requests x rank entries.
constexpr size_t uacc_bytes(int rank) { return 2ull * 8 * rank * kUaccStride * 8; }

// Launch arguments of the persistent correction-loop kernel (one request group).
struct LoopArgs {
  // weights
  const void* embed;
  const void* w_ih;
  const void* w_hh;
  const float* b_ih;
  const float* b_hh;
  const void* w1;
  const void* w2;
  // inputs (already offset to the group's first request)
  const void* hidden;   // [nb, K, d]
  const float* base;    // [nb, K, V]
  const float* hp;      // [nb, K, r]  W1[:, 0:d] h terms (stage-1 output)
  const int32_t* anchor;
  const int32_t* forced;  // or null
  const int32_t* target;  // or null
  // outputs (offset to the group)
  int32_t* draft;
  float* logits;        // or null
  int32_t* tau;         // or null
  // scratch
  Control* ctl;
  float* S_glob;                 // [2][NB][H]
  long long* u_acc;              // [2][8][r] x kUaccStride: W1 [h ; S] in 2^-32 fixed point
  unsigned long long* best;      // [K][NB]
  uint64_t seed;
  uint64_t budget_ns;
  float temperature;
  int32_t V, d, E, H, r, K;
  int32_t b0;       // global index of the group's first request (Philox counter)
  int32_t nb;       // requests in this group (<= NB)
  int32_t mode;     // 0 greedy, 1 Gumbel
  int32_t wbytes;   // 2 (bf16) or 4 (f32)
  int32_t selftest; // 1: run only the unreachable-barrier self-test
  // segment plan
  int32_t segE3, nsegE3, segH3, nsegH3;
  int32_t max_ih, max_hh;  // ring items of W_ih / W_hh per CTA per step, at most
  int32_t nslot;
  int32_t vmax;     // largest vocabulary slice of any CTA (rounded up to 4)
  int32_t vsplit[kLoopMaxGrid + 1];  // CTA c owns W2 rows [vsplit[c], vsplit[c+1])
  // shared-memory carve-up (byte offsets)
  uint32_t off_bars, off_S, off_x, off_base, off_part, off_hp, off_bias, off_w1s, off_sown, off_u, off_tok, off_wbest,
      off_flags, off_items;
};

// Fills the segment plan and shared-memory offsets; returns the dynamic shared
// memory size, or 0 if the shapes do not fit.
size_t loop_plan(LoopArgs& a, int NB, int grid, size_t smem_cap);
int loop_group_size(int B);
int loop_threads(int NB);
cudaError_t launch_correct_loop(LoopArgs a, int NB, int grid, size_t smem, cudaStream_t stream);

// LM head (stage 1).
// out [M, V] = hidden . W_lm^T (skipped if out is null); out2 [M, rows2] =
// hidden . W1[:, 0:Kd]^T with W1 rows w1_stride elements apart (skipped if null).
// sk_part / sk_flag: stream-K scratch (partial tiles [kLoopMaxGrid][BN][128] fp32
// and [kLoopMaxGrid] flags, zero between launches), or null for whole tiles only.
cudaError_t launch_lm_head_tc(const void* w_lm, const void* hidden, float* out, int V, int M, int Kd,
                              const void* w1, int rows2, int w1_stride, float* out2, float* sk_part,
                              uint32_t* sk_flag, Control* ctl, uint64_t budget_ns, int num_sms,
                              cudaStream_t stream);
// Bytes of stream-K partial tiles for M block positions.
inline size_t lm_head_sk_bytes(int M) {
  const int bn = ((M + 15) / 16 * 16) > 256 ? 256 : (M + 15) / 16 * 16;
  return static_cast<size_t>(kLoopMaxGrid) * bn * 128 * 4;
}
cudaError_t launch_lm_head_f32(const float* w, const float* hidden, float* out, int V, int M, int Kd, int ldw,
                               cudaStream_t stream);

// Verification (stage 3).
cudaError_t launch_verify(const int32_t* draft, const int32_t* target, int B, int K, int32_t* tau,
                          cudaStream_t stream);

}  // namespace domino
