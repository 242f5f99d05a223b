// C ABI of the Domino draft-block library (declared in include/domino.h).
//
// Host side only: argument validation, workspace carve-up and the launch
// sequence.  Every step of the path runs in the kernels of this library.
#include <atomic>
#include <cmath>
#include <cstring>

#include "domino.h"
#include "common.cuh"
#include "domino_internal.h"

using domino::Control;

namespace {

std::atomic<uint64_t> g_budget_ns{2000000000ull};

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// The control region (zeroed by domino_workspace_init and after device errors)
// holds the control block and the stream-K ready flags of the LM head.
constexpr size_t kCtlRegion = 1024;
static_assert(sizeof(Control) + domino::kLoopMaxGrid * 4 <= kCtlRegion, "control region");

struct Layout {
  size_t ctl, skflag, base, hp, S, u, best, skp, tc, end;  // device workspace
  size_t h_hidden, h_anchor, h_forced, h_target, h_draft, h_tau, h_end;  // host-variant staging
};

bool weights_ok(const domino_weights* w) {
  if (!w) return false;
  if (w->dtype != DOMINO_BF16 && w->dtype != DOMINO_F32) return false;
  if (w->vocab < 1 || w->d_model < 8 || w->embed_dim < 8 || w->gru_hidden < 8 || w->rank < 8) return false;
  if (w->d_model % 8 || w->embed_dim % 8 || w->gru_hidden % 8 || w->rank % 8) return false;
  return true;
}

bool weight_ptrs_ok(const domino_weights* w, bool need_lm, bool need_loop) {
  if (need_lm && (!w->w_lm || !aligned16(w->w_lm))) return false;
  if (need_loop) {
    const void* req[] = {w->embed, w->w_ih, w->w_hh, w->w1, w->w2};
    for (const void* p : req)
      if (!p || !aligned16(p)) return false;
    if (w->b_ih && !aligned16(w->b_ih)) return false;
    if (w->b_hh && !aligned16(w->b_hh)) return false;
  }
  return true;
}

Layout layout_of(const domino_weights* w, int B, int K) {
  Layout L{};
  const size_t wb = w->dtype == DOMINO_BF16 ? 2 : 4;
  size_t o = 0;
  L.ctl = o;
  L.skflag = o + sizeof(Control);
  o += kCtlRegion;
  L.base = o; o += align_up(static_cast<size_t>(B) * K * w->vocab * 4);
  L.hp = o; o += align_up(static_cast<size_t>(B) * K * w->rank * 4);
  L.S = o; o += align_up(2ull * 8 * w->gru_hidden * 4);
  L.u = o; o += align_up(domino::uacc_bytes(w->rank));
  L.best = o; o += align_up(static_cast<size_t>(K) * (B > 8 ? B : 8) * 8);
  L.skp = o; o += align_up(domino::lm_head_sk_bytes(B * K));
  L.tc = o; o += align_up(domino::loop_tc_scratch_bytes(B, w->embed_dim, w->gru_hidden, w->rank));
  L.end = o;
  L.h_hidden = o; o += align_up(static_cast<size_t>(B) * K * w->d_model * wb);
  L.h_anchor = o; o += align_up(static_cast<size_t>(B) * 4);
  L.h_forced = o; o += align_up(static_cast<size_t>(B) * K * 4);
  L.h_target = o; o += align_up(static_cast<size_t>(B) * K * 4);
  L.h_draft = o; o += align_up(static_cast<size_t>(B) * K * 4);
  L.h_tau = o; o += align_up(static_cast<size_t>(B) * 4);
  L.h_end = o;
  return L;
}

domino_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return DOMINO_OK;
  (void)cudaGetLastError();
  if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorLaunchOutOfResources) return DOMINO_ERR_LAUNCH;
  return DOMINO_ERR_CUDA;
}

domino_status check_workspace(void* ws, size_t bytes, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || bytes < need) return DOMINO_ERR_WORKSPACE;
  return DOMINO_OK;
}

// Stage 1: base logits (base != null) and/or the hidden-state half of the
// bottleneck pre-activation hp[m, k] = W1[k, 0:d] h[m] (hp != null).
domino_status run_lm_head(const domino_weights* w, const void* hidden, int B, int K, float* base, float* hp,
                          char* ws, const Layout& L, cudaStream_t st) {
  Control* ctl = reinterpret_cast<Control*>(ws + L.ctl);
  const int M = B * K;
  const int w1_stride = w->d_model + w->gru_hidden;
  cudaError_t e = cudaSuccess;
  if (w->dtype == DOMINO_BF16) {
    const int sms = num_sms();
    if (sms <= 0) return DOMINO_ERR_CUDA;
    e = domino::launch_lm_head_tc(w->w_lm, hidden, base, w->vocab, M, w->d_model, w->w1, w->rank, w1_stride, hp,
                                  reinterpret_cast<float*>(ws + L.skp), reinterpret_cast<uint32_t*>(ws + L.skflag),
                                  ctl, g_budget_ns.load(), sms, st);
  } else {
    const float* h = static_cast<const float*>(hidden);
    if (base) e = domino::launch_lm_head_f32(static_cast<const float*>(w->w_lm), h, base, w->vocab, M, w->d_model,
                                             w->d_model, st);
    if (e == cudaSuccess && hp)
      e = domino::launch_lm_head_f32(static_cast<const float*>(w->w1), h, hp, w->rank, M, w->d_model, w1_stride, st);
  }
  return from_cuda(e);
}

// Stage 2 takes the per-step tensor-core path for bf16 batches from
// kLoopTcMinBatch requests on shapes it supports, else the persistent loop.
bool use_loop_tc(const domino_weights* w, int B) {
  return w->dtype == DOMINO_BF16 && B >= domino::kLoopTcMinBatch &&
         domino::loop_tc_supported(w->embed_dim, w->gru_hidden, w->d_model, w->rank, w->vocab);
}

domino_status run_loop(const domino_weights* w, const void* hidden, const float* base, const int32_t* anchor, int B,
                       int K, int mode, float temperature, uint64_t seed, const int32_t* forced,
                       const int32_t* target, int32_t* draft, float* logits, int32_t* tau, char* ws, const Layout& L,
                       cudaStream_t st) {
  const int sms = num_sms();
  if (sms <= 0) return DOMINO_ERR_CUDA;
  const size_t wb = w->dtype == DOMINO_BF16 ? 2 : 4;
  if (use_loop_tc(w, B)) {
    // larger batches: per-step tensor-core GEMMs over the whole batch
    domino::LoopTcArgs t;
    std::memset(&t, 0, sizeof(t));
    t.embed = w->embed; t.w_ih = w->w_ih; t.w_hh = w->w_hh; t.b_ih = w->b_ih; t.b_hh = w->b_hh;
    t.w1 = w->w1; t.w2 = w->w2;
    t.base = base;
    t.hp = reinterpret_cast<const float*>(ws + L.hp);
    t.anchor = anchor; t.forced = forced; t.target = target;
    t.draft = draft; t.logits = logits; t.tau = tau;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    const int E = w->embed_dim, H = w->gru_hidden, r = w->rank;
    char* p = ws + L.tc;
    t.X = reinterpret_cast<__nv_bfloat16*>(p); p += al(static_cast<size_t>(B) * E * 2);
    t.S = reinterpret_cast<float*>(p); p += al(static_cast<size_t>(B) * H * 4);
    t.S2 = reinterpret_cast<__nv_bfloat16*>(p); p += al(static_cast<size_t>(B) * 2 * domino::loop_tc_padded_h(H) * 2);
    t.gi_part = reinterpret_cast<float*>(p); p += al(static_cast<size_t>(domino::kLoopTcMaxSplits) * B * 3 * H * 4);
    t.gh_part = reinterpret_cast<float*>(p); p += al(static_cast<size_t>(domino::kLoopTcMaxSplits) * B * 3 * H * 4);
    t.u_part = reinterpret_cast<float*>(p); p += al(static_cast<size_t>(domino::kLoopTcMaxSplits) * B * r * 4);
    t.U2 = reinterpret_cast<__nv_bfloat16*>(p); p += al(static_cast<size_t>(2) * B * r * 2);
    t.fed = reinterpret_cast<int32_t*>(p);
    t.gate_table = w->gate_table;
    t.best = reinterpret_cast<unsigned long long*>(ws + L.best);
    t.ctl = reinterpret_cast<Control*>(ws + L.ctl);
    t.budget_ns = g_budget_ns.load();
    t.seed = seed;
    t.temperature = temperature;
    t.mode = mode;
    t.B = B; t.K = K; t.V = w->vocab; t.d = w->d_model; t.E = E; t.H = H; t.r = r; t.num_sms = sms;
    return from_cuda(domino::run_loop_tc(t, st));
  }
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
  a.gate_table = w->gate_table;
  a.ctl = reinterpret_cast<Control*>(ws + L.ctl);
  a.S_glob = reinterpret_cast<float*>(ws + L.S);
  a.u_acc = reinterpret_cast<long long*>(ws + L.u);
  const float* hp = reinterpret_cast<const float*>(ws + L.hp);
  a.best = reinterpret_cast<unsigned long long*>(ws + L.best);
  a.seed = seed;
  a.budget_ns = g_budget_ns.load();
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
    g.draft = draft + static_cast<size_t>(g0) * K;
    g.logits = logits ? logits + static_cast<size_t>(g0) * K * w->vocab : nullptr;
    g.tau = tau ? tau + g0 : nullptr;
    const domino_status s = from_cuda(domino::launch_correct_loop(g, NB, sms, smem, st));
    if (s != DOMINO_OK) return s;
  }
  return DOMINO_OK;
}

domino_status validate_block(const domino_weights* w, const void* hidden, const int32_t* anchor, int B, int K,
                             int mode, float temperature, const int32_t* forced, const int32_t* target,
                             const void* draft_out, const void* logits_out, const void* tau_out) {
  if (!weights_ok(w)) return DOMINO_ERR_INVALID_ARG;
  if (B < 1 || K < 1 || K > 32) return DOMINO_ERR_INVALID_ARG;
  if (mode != DOMINO_GREEDY && mode != DOMINO_GUMBEL) return DOMINO_ERR_INVALID_ARG;
  if (mode == DOMINO_GUMBEL && !(temperature > 0.f && std::isfinite(temperature))) return DOMINO_ERR_INVALID_ARG;
  if (!hidden || !aligned16(hidden) || !anchor || !aligned16(anchor)) return DOMINO_ERR_INVALID_ARG;
  if (!draft_out || !aligned16(draft_out)) return DOMINO_ERR_INVALID_ARG;
  if (forced && !aligned16(forced)) return DOMINO_ERR_INVALID_ARG;
  if (target && (!aligned16(target) || !tau_out || !aligned16(tau_out))) return DOMINO_ERR_INVALID_ARG;
  if (logits_out && !aligned16(logits_out)) return DOMINO_ERR_INVALID_ARG;
  const int rmax = w->dtype == DOMINO_BF16 ? 256 : 128;
  if (w->rank > rmax) return DOMINO_ERR_UNSUPPORTED;
  return DOMINO_OK;
}

}  // namespace

extern "C" {

size_t domino_workspace_bytes(const domino_weights* w, int32_t B, int32_t K) {
  if (!weights_ok(w) || B < 1 || K < 1 || K > 32) return 0;
  return layout_of(w, B, K).end;
}

size_t domino_workspace_bytes_host(const domino_weights* w, int32_t B, int32_t K) {
  if (!weights_ok(w) || B < 1 || K < 1 || K > 32) return 0;
  return layout_of(w, B, K).h_end;
}

int32_t domino_launches_per_block(const domino_weights* w, int32_t B, int32_t K) {
  if (!weights_ok(w) || B < 1 || K < 1 || K > 32) return -1;
  if (use_loop_tc(w, B)) {
    const int chunks = (B + domino::kLoopTcReqPerLaunch - 1) / domino::kLoopTcReqPerLaunch;
    // with a token->gate table the first position needs no gate GEMM (W_hh S = 0)
    return 1 /* LM head */ + 1 /* anchor tokens */ + K * (domino::kLoopTcLaunchesPerStep + chunks) -
           (w->gate_table ? 1 : 0);
  }
  const int NB = domino::loop_group_size(B);
  return 1 /* LM head */ + (B + NB - 1) / NB;
}

domino_status domino_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || workspace_bytes < kCtlRegion)
    return DOMINO_ERR_WORKSPACE;
  return from_cuda(cudaMemsetAsync(workspace, 0, kCtlRegion, static_cast<cudaStream_t>(stream)));
}

domino_status domino_lm_head(const domino_weights* w, const void* hidden, int32_t B, int32_t K, float* base_out,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (!weights_ok(w) || !weight_ptrs_ok(w, true, false)) return DOMINO_ERR_INVALID_ARG;
  if (B < 1 || K < 1 || K > 32 || !hidden || !aligned16(hidden) || !base_out || !aligned16(base_out))
    return DOMINO_ERR_INVALID_ARG;
  const Layout L = layout_of(w, B, K);
  const domino_status ws = check_workspace(workspace, workspace_bytes, L.end);
  if (ws != DOMINO_OK) return ws;
  return run_lm_head(w, hidden, B, K, base_out, nullptr, static_cast<char*>(workspace), L,
                     static_cast<cudaStream_t>(stream));
}

domino_status domino_correct_loop(const domino_weights* w, const void* hidden, const float* base,
                                  const int32_t* anchor, int32_t B, int32_t K, int32_t mode, float temperature,
                                  uint64_t seed, const int32_t* forced, const int32_t* target, int32_t* draft_out,
                                  float* logits_out, int32_t* tau_out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  domino_status s = validate_block(w, hidden, anchor, B, K, mode, temperature, forced, target, draft_out,
                                   logits_out, tau_out);
  if (s != DOMINO_OK) return s;
  if (!weight_ptrs_ok(w, false, true) || !base || !aligned16(base)) return DOMINO_ERR_INVALID_ARG;
  const Layout L = layout_of(w, B, K);
  s = check_workspace(workspace, workspace_bytes, L.end);
  if (s != DOMINO_OK) return s;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = run_lm_head(w, hidden, B, K, nullptr, reinterpret_cast<float*>(ws + L.hp), ws, L, st);
  if (s != DOMINO_OK) return s;
  return run_loop(w, hidden, base, anchor, B, K, mode, temperature, seed, forced, target, draft_out, logits_out,
                  tau_out, ws, L, st);
}

domino_status domino_draft_block_events(const domino_weights* w, const void* hidden, const int32_t* anchor, int32_t B,
                                        int32_t K, int32_t mode, float temperature, uint64_t seed,
                                        const int32_t* forced, const int32_t* target, int32_t* draft_out,
                                        float* logits_out, int32_t* tau_out, void* workspace, size_t workspace_bytes,
                                        void* stream, void* const* events) {
  domino_status s = validate_block(w, hidden, anchor, B, K, mode, temperature, forced, target, draft_out,
                                   logits_out, tau_out);
  if (s != DOMINO_OK) return s;
  if (!weight_ptrs_ok(w, true, true)) return DOMINO_ERR_INVALID_ARG;
  const Layout L = layout_of(w, B, K);
  s = check_workspace(workspace, workspace_bytes, L.end);
  if (s != DOMINO_OK) return s;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto mark = [&](int k) -> domino_status {
    if (!events || !events[k]) return DOMINO_OK;
    return from_cuda(cudaEventRecord(static_cast<cudaEvent_t>(events[k]), st));
  };
  if ((s = mark(0)) != DOMINO_OK) return s;
  float* base = reinterpret_cast<float*>(ws + L.base);
  s = run_lm_head(w, hidden, B, K, base, reinterpret_cast<float*>(ws + L.hp), ws, L, st);
  if (s != DOMINO_OK) return s;
  if ((s = mark(1)) != DOMINO_OK) return s;
  s = run_loop(w, hidden, base, anchor, B, K, mode, temperature, seed, forced, target, draft_out, logits_out, tau_out,
               ws, L, st);
  if (s != DOMINO_OK) return s;
  return mark(2);
}

domino_status domino_draft_block(const domino_weights* w, const void* hidden, const int32_t* anchor, int32_t B,
                                 int32_t K, int32_t mode, float temperature, uint64_t seed, const int32_t* forced,
                                 const int32_t* target, int32_t* draft_out, float* logits_out, int32_t* tau_out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return domino_draft_block_events(w, hidden, anchor, B, K, mode, temperature, seed, forced, target, draft_out,
                                   logits_out, tau_out, workspace, workspace_bytes, stream, nullptr);
}

// ---------------------------------------------------------------- token -> gate table

size_t domino_gate_table_bytes(const domino_weights* w) {
  if (!weights_ok(w)) return 0;
  return static_cast<size_t>(w->vocab) * 3 * w->gru_hidden * 4;
}

domino_status domino_build_gate_table(const domino_weights* w, float* table_out, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!weights_ok(w) || !table_out || !aligned16(table_out)) return DOMINO_ERR_INVALID_ARG;
  if (!w->embed || !aligned16(w->embed) || !w->w_ih || !aligned16(w->w_ih)) return DOMINO_ERR_INVALID_ARG;
  if (w->b_ih && !aligned16(w->b_ih)) return DOMINO_ERR_INVALID_ARG;
  domino_status s = check_workspace(workspace, workspace_bytes, kCtlRegion);
  if (s != DOMINO_OK) return s;
  const int sms = num_sms();
  if (sms <= 0) return DOMINO_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G3 = 3 * w->gru_hidden;
  cudaError_t e;
  // G[t, :] = W_ih E[t, :] for every token: the LM-head GEMM with the embedding
  // rows as its positions and W_ih as its row operand (output [V, 3H])
  if (w->dtype == DOMINO_BF16)
    e = domino::launch_lm_head_tc(w->w_ih, w->embed, table_out, G3, w->vocab, w->embed_dim, nullptr, 0, 0, nullptr,
                                  nullptr, nullptr, static_cast<Control*>(workspace), g_budget_ns.load(), sms, st);
  else
    e = domino::launch_lm_head_f32(static_cast<const float*>(w->w_ih), static_cast<const float*>(w->embed), table_out,
                                   G3, w->vocab, w->embed_dim, w->embed_dim, st);
  if (e == cudaSuccess && w->b_ih) e = domino::launch_add_row_bias(table_out, w->b_ih, w->vocab, G3, sms, st);
  return from_cuda(e);
}

// ---------------------------------------------------------------- training forward

size_t domino_curriculum_loss_workspace_bytes(int32_t B, int32_t K, int32_t V) {
  if (B < 1 || K < 1 || K > 32 || V < 1) return 0;
  return kCtlRegion + align_up(domino::loss_scratch_bytes(B, K, V));
}

domino_status domino_curriculum_loss(const float* final_logits, const float* base_logits, const int32_t* labels,
                                     int32_t B, int32_t K, int32_t V, float lambda, float gamma, float* ce_out,
                                     float* loss_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 1 || K < 1 || K > 32 || V < 1 || static_cast<long long>(B) * K > 65535 / 2) return DOMINO_ERR_INVALID_ARG;
  if (!final_logits || !base_logits || !labels || !loss_out) return DOMINO_ERR_INVALID_ARG;
  if (!aligned16(final_logits) || !aligned16(base_logits) || !aligned16(labels) || !aligned16(loss_out) ||
      (ce_out && !aligned16(ce_out)))
    return DOMINO_ERR_INVALID_ARG;
  if (!(lambda >= 0.f && lambda <= 1.f) || !(gamma > 0.f && std::isfinite(gamma))) return DOMINO_ERR_INVALID_ARG;
  domino_status s = check_workspace(workspace, workspace_bytes, domino_curriculum_loss_workspace_bytes(B, K, V));
  if (s != DOMINO_OK) return s;
  char* ws = static_cast<char*>(workspace);
  return from_cuda(domino::launch_curriculum_loss(final_logits, base_logits, labels, B, K, V, lambda, gamma,
                                                  ws + kCtlRegion, ce_out, loss_out, reinterpret_cast<Control*>(ws),
                                                  static_cast<cudaStream_t>(stream)));
}

size_t domino_draft_loss_workspace_bytes(const domino_weights* w, int32_t B, int32_t K) {
  if (!weights_ok(w) || B < 1 || K < 1 || K > 32) return 0;
  const size_t rows = static_cast<size_t>(B) * K;
  return layout_of(w, B, K).end + align_up(rows * w->vocab * 4) + align_up(rows * 4) +
         align_up(domino::loss_scratch_bytes(B, K, w->vocab));
}

domino_status domino_draft_loss(const domino_weights* w, const void* hidden, const int32_t* anchor,
                                const int32_t* labels, int32_t B, int32_t K, float lambda, float gamma,
                                float* ce_out, float* loss_out, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (!labels || !loss_out || !aligned16(loss_out) || (ce_out && !aligned16(ce_out))) return DOMINO_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * K > 65535 / 2) return DOMINO_ERR_INVALID_ARG;
  if (!(lambda >= 0.f && lambda <= 1.f) || !(gamma > 0.f && std::isfinite(gamma))) return DOMINO_ERR_INVALID_ARG;
  const Layout L = layout_of(w, B, K);
  const size_t rows = static_cast<size_t>(B) * K;
  domino_status s = check_workspace(workspace, workspace_bytes, domino_draft_loss_workspace_bytes(w, B, K));
  if (s != DOMINO_OK) return s;
  char* ws = static_cast<char*>(workspace);
  float* final_logits = reinterpret_cast<float*>(ws + L.end);
  int32_t* picks = reinterpret_cast<int32_t*>(ws + L.end + align_up(rows * w->vocab * 4));
  void* scratch = ws + L.end + align_up(rows * w->vocab * 4) + align_up(rows * 4);
  s = validate_block(w, hidden, anchor, B, K, DOMINO_GREEDY, 1.f, labels, nullptr, picks, final_logits, nullptr);
  if (s != DOMINO_OK) return s;
  if (!weight_ptrs_ok(w, true, true)) return DOMINO_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* base = reinterpret_cast<float*>(ws + L.base);
  // teacher forcing: the labels are the GRU's inputs after each position
  s = run_lm_head(w, hidden, B, K, base, reinterpret_cast<float*>(ws + L.hp), ws, L, st);
  if (s != DOMINO_OK) return s;
  s = run_loop(w, hidden, base, anchor, B, K, DOMINO_GREEDY, 1.f, 0, labels, nullptr, picks, final_logits, nullptr,
               ws, L, st);
  if (s != DOMINO_OK) return s;
  return from_cuda(domino::launch_curriculum_loss(final_logits, base, labels, B, K, w->vocab, lambda, gamma, scratch,
                                                  ce_out, loss_out, reinterpret_cast<Control*>(ws + L.ctl), st));
}

size_t domino_verify_sample_workspace_bytes(int32_t B, int32_t K, int32_t V) {
  if (B < 1 || K < 1 || K > 32 || V < 1) return 0;
  return kCtlRegion + align_up(domino::verify_sample_scratch_bytes(B, K, V));
}

domino_status domino_verify_sample(const float* draft_logits, const float* target_logits, const int32_t* draft,
                                   int32_t B, int32_t K, int32_t V, float temperature, uint64_t seed,
                                   int32_t* tau_out, int32_t* token_out, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (B < 1 || K < 1 || K > 32 || V < 1 || static_cast<long long>(B) * (2 * K + 1) > 65535) return DOMINO_ERR_INVALID_ARG;
  if (!draft_logits || !target_logits || !draft || !tau_out || !token_out) return DOMINO_ERR_INVALID_ARG;
  if (!aligned16(draft_logits) || !aligned16(target_logits) || !aligned16(draft) || !aligned16(tau_out) ||
      !aligned16(token_out))
    return DOMINO_ERR_INVALID_ARG;
  if (!(temperature > 0.f && std::isfinite(temperature))) return DOMINO_ERR_INVALID_ARG;
  domino_status s = check_workspace(workspace, workspace_bytes, domino_verify_sample_workspace_bytes(B, K, V));
  if (s != DOMINO_OK) return s;
  char* ws = static_cast<char*>(workspace);
  return from_cuda(domino::launch_verify_sample(draft_logits, target_logits, draft, B, K, V, temperature, seed,
                                                ws + kCtlRegion, tau_out, token_out, reinterpret_cast<Control*>(ws),
                                                static_cast<cudaStream_t>(stream)));
}

domino_status domino_verify(const int32_t* draft, const int32_t* target, int32_t B, int32_t K, int32_t* tau_out,
                            void* stream) {
  if (!draft || !target || !tau_out || B < 1 || K < 1 || K > 32) return DOMINO_ERR_INVALID_ARG;
  if (!aligned16(draft) || !aligned16(target) || !aligned16(tau_out)) return DOMINO_ERR_INVALID_ARG;
  return from_cuda(domino::launch_verify(draft, target, B, K, tau_out, static_cast<cudaStream_t>(stream)));
}

domino_status domino_draft_block_host(const domino_weights* w, const void* hidden_host, const int32_t* anchor_host,
                                      int32_t B, int32_t K, int32_t mode, float temperature, uint64_t seed,
                                      const int32_t* forced_host, const int32_t* target_host,
                                      int32_t* draft_out_host, int32_t* tau_out_host, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!weights_ok(w) || B < 1 || K < 1 || K > 32) return DOMINO_ERR_INVALID_ARG;
  if (!hidden_host || !anchor_host || !draft_out_host || (target_host && !tau_out_host)) return DOMINO_ERR_INVALID_ARG;
  const Layout L = layout_of(w, B, K);
  domino_status s = check_workspace(workspace, workspace_bytes, L.h_end);
  if (s != DOMINO_OK) return s;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t wb = w->dtype == DOMINO_BF16 ? 2 : 4;
  const size_t tok = static_cast<size_t>(B) * K * 4;
  cudaError_t e = cudaMemcpyAsync(ws + L.h_hidden, hidden_host, static_cast<size_t>(B) * K * w->d_model * wb,
                                  cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(ws + L.h_anchor, anchor_host, static_cast<size_t>(B) * 4, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && forced_host) e = cudaMemcpyAsync(ws + L.h_forced, forced_host, tok, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && target_host) e = cudaMemcpyAsync(ws + L.h_target, target_host, tok, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return from_cuda(e);
  int32_t* d_draft = reinterpret_cast<int32_t*>(ws + L.h_draft);
  int32_t* d_tau = reinterpret_cast<int32_t*>(ws + L.h_tau);
  s = domino_draft_block(w, ws + L.h_hidden, reinterpret_cast<const int32_t*>(ws + L.h_anchor), B, K, mode,
                         temperature, seed, forced_host ? reinterpret_cast<const int32_t*>(ws + L.h_forced) : nullptr,
                         target_host ? reinterpret_cast<const int32_t*>(ws + L.h_target) : nullptr, d_draft, nullptr,
                         target_host ? d_tau : nullptr, workspace, L.end, stream);
  if (s != DOMINO_OK) return s;
  e = cudaMemcpyAsync(draft_out_host, d_draft, tok, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess && target_host)
    e = cudaMemcpyAsync(tau_out_host, d_tau, static_cast<size_t>(B) * 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return from_cuda(e);
}

domino_status domino_poll(void* workspace, void* stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return DOMINO_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t err = 0;
  cudaError_t e = cudaMemcpyAsync(&err, workspace, sizeof(err), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return from_cuda(e);
  if (err == 0) return DOMINO_OK;
  e = cudaMemsetAsync(workspace, 0, kCtlRegion, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return from_cuda(e);
  if (err & domino::ERRBIT_TIMEOUT) return DOMINO_ERR_TIMEOUT;
  return DOMINO_ERR_BAD_TOKEN;
}

void domino_set_wait_budget_ns(uint64_t ns) { g_budget_ns.store(ns ? ns : 1); }

domino_status domino_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint64_t budget_ns, void* stream) {
  const domino_status s = check_workspace(workspace, workspace_bytes, kCtlRegion);
  if (s != DOMINO_OK) return s;
  const int sms = num_sms();
  if (sms <= 0) return DOMINO_ERR_CUDA;
  domino::LoopArgs a;
  std::memset(&a, 0, sizeof(a));
  a.ctl = static_cast<Control*>(workspace);
  a.budget_ns = budget_ns;
  a.selftest = 1;
  a.wbytes = 2;
  a.nslot = 0;
  const domino_status ls =
      from_cuda(domino::launch_correct_loop(a, 1, sms, 1024, static_cast<cudaStream_t>(stream)));
  if (ls != DOMINO_OK) return ls;
  return domino_poll(workspace, stream);
}

const char* domino_status_str(domino_status s) {
  switch (s) {
    case DOMINO_OK: return "DOMINO_OK";
    case DOMINO_ERR_INVALID_ARG: return "DOMINO_ERR_INVALID_ARG";
    case DOMINO_ERR_UNSUPPORTED: return "DOMINO_ERR_UNSUPPORTED";
    case DOMINO_ERR_LAUNCH: return "DOMINO_ERR_LAUNCH";
    case DOMINO_ERR_CUDA: return "DOMINO_ERR_CUDA";
    case DOMINO_ERR_TIMEOUT: return "DOMINO_ERR_TIMEOUT";
    case DOMINO_ERR_BAD_TOKEN: return "DOMINO_ERR_BAD_TOKEN";
    case DOMINO_ERR_WORKSPACE: return "DOMINO_ERR_WORKSPACE";
  }
  return "DOMINO_ERR_UNKNOWN";
}

}  // extern "C"
