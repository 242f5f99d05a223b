// Allocation-free variant of stage 2 (domino_correct_loop_noalloc).
//
// Some callers cannot hand the library a workspace: engines that reserve all
// device memory in their own arena at start-up and forbid any other
// allocation, plugins running inside such an engine, and deployments that must
// not allocate after initialisation because cudaMalloc may synchronise the
// device and has no latency bound.  This entry point needs no workspace and
// allocates nothing: its scratch (control block, W1_h h terms, GRU state,
// bottleneck accumulator, argmax keys) lives in one file-scope device array of fixed
// size, which every GPU that loads the library holds until the process exits.
//
// In host code the array's name is only a host-side stand-in, so the device
// address is looked up once per device with cudaGetSymbolAddress (the first
// call on a device does this, with that device current) and passed to the
// kernels.  All calls share the array and it keeps the last call's contents:
// each call clears the control block first, and every other piece is written
// before it is read.  Calls whose work overlaps on the GPU (other streams, other
// host threads on the same device) race on the array.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "domino.h"
#include "domino_internal.h"

namespace {

constexpr int kMaxB = 8;       // requests per call
constexpr int kMaxK = 32;      // block positions
constexpr int kMaxR = 256;     // bottleneck rank
constexpr int kMaxH = 4096;    // GRU state width
constexpr size_t kCtlBytes = 256;
constexpr size_t kHpBytes = static_cast<size_t>(kMaxB) * kMaxK * kMaxR * 4;   // W1_h h terms [B,K,r]
constexpr size_t kSBytes = 2ull * 8 * kMaxH * 4;                               // GRU state [2][8][H]
constexpr size_t kUBytes = domino::uacc_bytes(kMaxR);                           // bottleneck accumulator
constexpr size_t kBestBytes = static_cast<size_t>(kMaxK) * 8 * 8;              // argmax keys [K][8]
constexpr size_t kScratchBytes = kCtlBytes + kHpBytes + kSBytes + kUBytes + kBestBytes;  // 657,664 bytes

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr uint64_t kBudgetNs = 2000000000ull;  // bound of every device wait in this variant
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

domino_status to_status(cudaError_t e) {
  if (e == cudaSuccess) return DOMINO_OK;
  (void)cudaGetLastError();
  if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorLaunchOutOfResources) return DOMINO_ERR_LAUNCH;
  return DOMINO_ERR_CUDA;
}

}  // namespace

extern "C" domino_status domino_correct_loop_noalloc(const domino_weights* w, const void* hidden, const float* base,
                                                     const int32_t* anchor, int32_t B, int32_t K, int32_t mode,
                                                     float temperature, uint64_t seed, const int32_t* forced,
                                                     const int32_t* target, int32_t* draft_out, float* logits_out,
                                                     int32_t* tau_out, void* stream) {
  // ---- arguments (same rules as domino_correct_loop) and the scratch limits
  if (!w || (w->dtype != DOMINO_BF16 && w->dtype != DOMINO_F32)) return DOMINO_ERR_INVALID_ARG;
  if (w->vocab < 1 || w->d_model < 8 || w->embed_dim < 8 || w->gru_hidden < 8 || w->rank < 8) return DOMINO_ERR_INVALID_ARG;
  if (w->d_model % 8 || w->embed_dim % 8 || w->gru_hidden % 8 || w->rank % 8) return DOMINO_ERR_INVALID_ARG;
  if (B < 1 || K < 1 || K > 32) return DOMINO_ERR_INVALID_ARG;
  if (mode != DOMINO_GREEDY && mode != DOMINO_GUMBEL) return DOMINO_ERR_INVALID_ARG;
  if (mode == DOMINO_GUMBEL && !(temperature > 0.f && temperature < 3.4e38f)) return DOMINO_ERR_INVALID_ARG;
  const void* req[] = {w->embed, w->w_ih, w->w_hh, w->w1, w->w2, hidden, base, anchor, draft_out};
  for (const void* p : req)
    if (!p || !a16(p)) return DOMINO_ERR_INVALID_ARG;
  if ((w->b_ih && !a16(w->b_ih)) || (w->b_hh && !a16(w->b_hh)) || (forced && !a16(forced)) ||
      (logits_out && !a16(logits_out)))
    return DOMINO_ERR_INVALID_ARG;
  if (target && (!a16(target) || !tau_out || !a16(tau_out))) return DOMINO_ERR_INVALID_ARG;
  if (w->rank > (w->dtype == DOMINO_BF16 ? 256 : 128)) return DOMINO_ERR_UNSUPPORTED;
  if (B > kMaxB || K > kMaxK || w->rank > kMaxR || w->gru_hidden > kMaxH) return DOMINO_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) return to_status(e);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return DOMINO_ERR_CUDA;

  char* s = static_cast<char*>(scratch);
  domino::Control* ctl = reinterpret_cast<domino::Control*>(s);
  float* hp = reinterpret_cast<float*>(s + kCtlBytes);
  float* S = reinterpret_cast<float*>(s + kCtlBytes + kHpBytes);
  long long* uacc = reinterpret_cast<long long*>(s + kCtlBytes + kHpBytes + kSBytes);
  unsigned long long* best = reinterpret_cast<unsigned long long*>(s + kCtlBytes + kHpBytes + kSBytes + kUBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // error word and barrier counters must start at zero
  e = cudaMemsetAsync(ctl, 0, kCtlBytes, st);
  if (e != cudaSuccess) return to_status(e);

  // W1_h h_i terms for every position (hidden-state half of the bottleneck)
  const int M = B * K;
  const int w1_stride = w->d_model + w->gru_hidden;
  if (w->dtype == DOMINO_BF16)
    e = domino::launch_lm_head_tc(nullptr, hidden, nullptr, w->vocab, M, w->d_model, w->w1, w->rank, w1_stride, hp,
                                  nullptr, nullptr, ctl, kBudgetNs, sms, st);
  else
    e = domino::launch_lm_head_f32(static_cast<const float*>(w->w1), static_cast<const float*>(hidden), hp, w->rank, M,
                                   w->d_model, w1_stride, st);
  if (e != cudaSuccess) return to_status(e);

  // the correction loop, request groups of up to 8
  const size_t wb = w->dtype == DOMINO_BF16 ? 2 : 4;
  const int NB = domino::loop_group_size(B);
  domino::LoopArgs a;
  std::memset(&a, 0, sizeof(a));
  a.embed = w->embed;
  a.w_ih = w->w_ih;
  a.w_hh = w->w_hh;
  a.b_ih = w->b_ih;
  a.b_hh = w->b_hh;
  a.w1 = w->w1;
  a.w2 = w->w2;
  a.ctl = ctl;
  a.S_glob = S;
  a.u_acc = uacc;
  a.best = best;
  a.seed = seed;
  a.budget_ns = kBudgetNs;
  a.temperature = temperature;
  a.V = w->vocab;
  a.d = w->d_model;
  a.E = w->embed_dim;
  a.H = w->gru_hidden;
  a.r = w->rank;
  a.K = K;
  a.mode = mode;
  a.wbytes = static_cast<int>(wb);
  const size_t smem = domino::loop_plan(a, NB, sms, 227 * 1024);
  if (smem == 0) return DOMINO_ERR_UNSUPPORTED;
  for (int g0 = 0; g0 < B; g0 += NB) {
    const int nb = B - g0 < NB ? B - g0 : NB;
    domino::LoopArgs g = a;
    g.b0 = g0;
    g.nb = nb;
    g.hidden = static_cast<const char*>(hidden) + static_cast<size_t>(g0) * K * w->d_model * wb;
    g.base = base + static_cast<size_t>(g0) * K * w->vocab;
    g.hp = hp + static_cast<size_t>(g0) * K * w->rank;
    g.anchor = anchor + g0;
    g.forced = forced ? forced + static_cast<size_t>(g0) * K : nullptr;
    g.target = target ? target + static_cast<size_t>(g0) * K : nullptr;
    g.draft = draft_out + static_cast<size_t>(g0) * K;
    g.logits = logits_out ? logits_out + static_cast<size_t>(g0) * K * w->vocab : nullptr;
    g.tau = tau_out ? tau_out + g0 : nullptr;
    e = domino::launch_correct_loop(g, NB, sms, smem, st);
    if (e != cudaSuccess) return to_status(e);
  }

  // wait for the call and report what the device flagged
  uint32_t err = 0;
  e = cudaMemcpyAsync(&err, &ctl->err, sizeof(err), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return to_status(e);
  if (err & domino::ERRBIT_TIMEOUT) return DOMINO_ERR_TIMEOUT;
  if (err & domino::ERRBIT_BAD_TOKEN) return DOMINO_ERR_BAD_TOKEN;
  return DOMINO_OK;
}
