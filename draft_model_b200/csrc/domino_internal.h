// Internal declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
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
  const float* gate_table;  // [V, 3H] token->gate table W_ih E + b_ih, or null (then W_ih is streamed)
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

// Stage 2 for larger batches on the tensor cores (bf16 weights), loop_tc.cu.
constexpr int kLoopTcMinBatch = 4;     // batches from this size take the tensor-core path
constexpr int kLoopTcMaxSplits = 8;    // split-K partial buffers of the gate and bottleneck GEMMs
constexpr int kLoopTcReqPerLaunch = 128;  // requests per W2 GEMM launch (one 256-column tile)
constexpr int kLoopTcLaunchesPerStep = 5; // gate GEMM, GRU, bottleneck GEMM, SiLU, pick (+ W2 per chunk)
struct LoopTcArgs {
  const void* embed; const void* w_ih; const void* w_hh; const float* b_ih; const float* b_hh;
  const void* w1; const void* w2;
  const float* base;       // [B, K, V]
  const float* hp;         // [B, K, r]
  const int32_t* anchor; const int32_t* forced; const int32_t* target;
  int32_t* draft; float* logits; int32_t* tau;
  // scratch
  __nv_bfloat16* X;        // [B, E]   embeddings of the fed tokens
  float* S;                // [B, H]   GRU state
  __nv_bfloat16* S2;       // [B, 2*Hp] bf16 hi | lo halves of S, each padded to Hp columns
  float* gi_part;          // [kLoopTcMaxSplits, B, 3H]
  float* gh_part;          // [kLoopTcMaxSplits, B, 3H]
  float* u_part;           // [kLoopTcMaxSplits, B, r]
  __nv_bfloat16* U2;       // [2B, r]  interleaved bf16 hi / lo rows of u
  unsigned long long* best;  // [K, B]
  int32_t* fed;            // [B]     token fed to the GRU after the current position
  const float* gate_table; // [V, 3H] token->gate table E W_ih^T + b_ih, or null
  Control* ctl;
  uint64_t budget_ns, seed;
  float temperature;
  int mode, B, K, V, d, E, H, r, num_sms;
};
cudaError_t run_loop_tc(const LoopTcArgs& args, cudaStream_t stream);
cudaError_t launch_add_row_bias(float* table, const float* bias, size_t rows, int cols, int num_sms,
                                cudaStream_t stream);
// Shapes the tensor-core path accepts (16-byte aligned tensor-map strides, < 2^16 vocabulary tiles).
bool loop_tc_supported(int E, int H, int d, int r, int V);
// H rounded up to whole 64-wide k-blocks: each bf16 half of S2 has this many columns.
inline int loop_tc_padded_h(int H) { return (H + 63) / 64 * 64; }
// Workspace bytes of the tensor-core path's scratch for batch B.
inline size_t loop_tc_scratch_bytes(int B, int E, int H, int r) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t Hp = static_cast<size_t>(loop_tc_padded_h(H));
  return al(static_cast<size_t>(B) * E * 2) + al(static_cast<size_t>(B) * H * 4) + al(static_cast<size_t>(B) * 2 * Hp * 2) +
         2 * al(static_cast<size_t>(kLoopTcMaxSplits) * B * 3 * H * 4) +
         al(static_cast<size_t>(kLoopTcMaxSplits) * B * r * 4) + al(static_cast<size_t>(2) * B * r * 2) +
         al(static_cast<size_t>(B) * 4);
}

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
// Base-anchored curriculum loss over fp32 logit rows (loss.cu).
int lse_chunks(int rows, int V);
cudaError_t launch_row_lse_partial(const float* X0, int K0, const float* X1, int K1, int B, int V, float scale,
                                   int chunks, const int32_t* idx, int Kidx, float2* part, float* picked, Control* ctl,
                                   cudaStream_t stream);
size_t loss_scratch_bytes(int B, int K, int V);
cudaError_t launch_curriculum_loss(const float* final_logits, const float* base_logits, const int32_t* labels, int B,
                                   int K, int V, float lambda, float gamma, void* scratch, float* ce_out,
                                   float* loss_out, Control* ctl, cudaStream_t stream);

// Stochastic verification at T > 0 (verify_sample.cu).
size_t verify_sample_scratch_bytes(int B, int K, int V);
cudaError_t launch_verify_sample(const float* draft_logits, const float* target_logits, const int32_t* draft, int B,
                                 int K, int V, float temperature, uint64_t seed, void* scratch, int32_t* tau_out,
                                 int32_t* token_out, Control* ctl, cudaStream_t stream);

cudaError_t launch_verify(const int32_t* draft, const int32_t* target, int B, int K, int32_t* tau,
                          cudaStream_t stream);

}  // namespace domino
