// Stage 2 of the Domino draft block: the sequential correction loop, as one
// persistent, cooperatively launched kernel per request group (<= 8 requests).
//
// Method (Domino study notes, gsyq.cn, §二.1(2); yhxrc.cn article, §四): for block
// positions i = 1..K
//     x      = E[t_{i-1}]                      (t_0 = anchor token)
//     S      = GRU(x, S)                       (S_0 = 0; gates r, z, n)   -> S_{i-1}
//     u      = SiLU(W1 [h_i ; S_{i-1}])        (rank r)
//     L_i    = L_i^base + W2 u
//     t_i    = argmax_j L_i[j]   or  argmax_j (L_i[j]/T + g_ij)   (Gumbel-max)
// and finally tau = leading agreement of t with the target tokens.
//
// B200 mapping.  One CTA per SM (148), all co-resident.  Each CTA statically owns
//   * GRU hidden units [j0, j1): the three gate rows of W_ih and W_hh,
//   * bottleneck rows [k0, k1) of W1,
//   * a contiguous vocabulary range [v0, v1) of W2 (balanced so every CTA streams
//     about the same number of weight bytes per step).
// A producer warp streams exactly those weight bytes, step after step, through a
// shared-memory ring with 1-D bulk copies (TMA engine, no tensor map).  The
// weights never depend on data, so the producer runs ahead across the grid
// barriers and HBM stays busy while consumers wait for data dependencies.
// Four consumer warps compute from the ring; item n is always handled by warp
// n % 4 and lands in slot n % NSLOT (NSLOT a multiple of 4), so a slot is only
// ever waited on by the warp that consumed its previous occupant.
// Per step three bounded grid barriers: after the GRU (S_i complete), after the
// bottleneck (u complete), after the vocabulary pass (argmax keys merged with a
// 64-bit atomicMax).  W1 [h_i ; S] is split as W1_h h_i + W1_s S; the W1_h h_i
// terms of the CTA's own rows are computed once for all positions up front.
// Delta L and L_i never touch HBM unless final logits are requested.
#include <cstdint>

#include "common.cuh"
#include "domino_internal.h"

namespace domino {

namespace {

constexpr int NCW = 4;                       // consumer warps
constexpr int NTHREADS = (NCW + 1) * 32;     // + one producer warp
constexpr int CONS_THREADS = NCW * 32;
constexpr uint32_t BAR_CONS = 1;             // named barrier id among consumer warps

struct Partition {
  int j0, j1;  // GRU units
  int k0, k1;  // bottleneck rows
  int v0, v1;  // vocabulary rows of W2
};

__device__ __host__ __forceinline__ long long vend_raw(const LoopArgs& a, int c, int G) {
  if (c < 0) return 0;
  if (c >= G - 1) return a.V;
  const long long unitB = 3ll * (a.E + a.H) * a.wbytes;
  const long long w1B = 1ll * a.H * a.wbytes;
  const long long rowB = 1ll * a.r * a.wbytes;
  const long long total = 1ll * a.H * unitB + 1ll * a.r * w1B + 1ll * a.V * rowB;
  const long long target = total * (c + 1) / G;
  const long long used = 1ll * ((c + 1) * a.H / G) * unitB + 1ll * ((c + 1) * a.r / G) * w1B;
  long long v = (target - used) / rowB;
  if (v < 0) v = 0;
  if (v > a.V) v = a.V;
  return v;
}

__device__ __forceinline__ Partition partition_of(const LoopArgs& a, int c, int G) {
  Partition p;
  p.j0 = c * a.H / G;
  p.j1 = (c + 1) * a.H / G;
  p.k0 = c * a.r / G;
  p.k1 = (c + 1) * a.r / G;
  long long lo = 0;
  for (int cc = 0; cc < c; ++cc) lo = max(lo, vend_raw(a, cc, G));
  const long long hi = max(lo, vend_raw(a, c, G));
  p.v0 = static_cast<int>(lo);
  p.v1 = static_cast<int>(hi);
  return p;
}

struct Seg {
  int n;      // number of segments
  int len;    // nominal segment length (elements, multiple of 8)
};
__device__ __forceinline__ int seg_len(const Seg& s, int total, int idx) {
  const int lo = idx * s.len;
  return min(total, lo + s.len) - lo;
}

struct Shared {
  uint64_t* full;
  uint64_t* empty;
  uint8_t* ring;
  float* S;        // [NB][H]   S_{i-1} (whole vector, all requests)
  uint8_t* x;      // [NB][E]   embedding of the fed token, storage type
  float* u;        // [NB][r]
  float* part;     // [max_part][32] per-item partial sums
  float* hp;       // [kmax][NB][K] W1_h h terms of this CTA's rows
  int* tok;        // [NB][K] picks (CTA 0 verifies from here)
  uint64_t* wbest; // [NCW][NB]
  int* flags;      // [0] abort
  int* fed;        // [NB] token fed to the GRU at the next step
};

template <int NB>
__device__ __forceinline__ Shared carve(uint8_t* base, const LoopArgs& a) {
  Shared s;
  s.ring = base;
  s.full = reinterpret_cast<uint64_t*>(base + a.off_bars);
  s.empty = s.full + a.nslot;
  s.S = reinterpret_cast<float*>(base + a.off_S);
  s.x = base + a.off_x;
  s.u = reinterpret_cast<float*>(base + a.off_u);
  s.part = reinterpret_cast<float*>(base + a.off_part);
  s.hp = reinterpret_cast<float*>(base + a.off_hp);
  s.tok = reinterpret_cast<int*>(base + a.off_tok);
  s.wbest = reinterpret_cast<uint64_t*>(base + a.off_wbest);
  s.flags = reinterpret_cast<int*>(base + a.off_flags);
  s.fed = s.flags + 4;
  return s;
}

__device__ __forceinline__ bool aborted(const Shared& s) {
  return *reinterpret_cast<volatile int*>(&s.flags[0]) != 0;
}
__device__ __forceinline__ void set_abort(const Shared& s) {
  *reinterpret_cast<volatile int*>(&s.flags[0]) = 1;
}

// Consumer-wide grid barrier: named barrier, one thread arrives and waits,
// named barrier.  Keeps control flow uniform even after an abort.
__device__ __forceinline__ void consumer_grid_sync(const LoopArgs& a, const Shared& s, uint32_t nblocks) {
  named_barrier(BAR_CONS, CONS_THREADS);
  if (threadIdx.x == 0 && !aborted(s)) {
    if (!grid_barrier_one_thread(a.ctl, nblocks, a.budget_ns)) set_abort(s);
  }
  named_barrier(BAR_CONS, CONS_THREADS);
}

// ---------------------------------------------------------------- per-step item schedule
struct Sched {
  Partition p;
  Seg e3, h3, h1;
  int nA, nB, nC, per_step;
};
__device__ __forceinline__ Sched make_sched(const LoopArgs& a, int c, int G) {
  Sched s;
  s.p = partition_of(a, c, G);
  s.e3 = Seg{a.nsegE3, a.segE3};
  s.h3 = Seg{a.nsegH3, a.segH3};
  s.h1 = Seg{a.nsegH1, a.segH1};
  s.nA = (s.p.j1 - s.p.j0) * (s.e3.n + s.h3.n);
  s.nB = (s.p.k1 - s.p.k0) * s.h1.n;
  s.nC = (s.p.v1 - s.p.v0 + 31) / 32;
  s.per_step = s.nA + s.nB + s.nC;
  return s;
}

// ---------------------------------------------------------------- producer
template <typename W>
__device__ void producer(const LoopArgs& a, const Shared& sh, const Sched& sc) {
  if ((threadIdx.x & 31) != 0) return;
  const W* w_ih = static_cast<const W*>(a.w_ih);
  const W* w_hh = static_cast<const W*>(a.w_hh);
  const W* w1 = static_cast<const W*>(a.w1);
  const W* w2 = static_cast<const W*>(a.w2);
  const uint64_t pol = policy_evict_first();
  const int nslot = a.nslot;
  const uint32_t slot_bytes = kLoopSlotBytes;
  int n = 0;
  bool ok = true;
  auto acquire = [&](int item) -> uint8_t* {
    const int slot = item % nslot;
    if (item >= nslot) {
      const uint32_t par = ((item / nslot) - 1) & 1;
      // wait for the consumer to release the slot; give up on abort
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&sh.empty[slot], par)) {
        if (aborted(sh)) return nullptr;
        if (globaltimer_ns() - t0 > a.budget_ns) {
          raise_error(a.ctl, ERRBIT_TIMEOUT);
          set_abort(sh);
          return nullptr;
        }
      }
    }
    return sh.ring + static_cast<size_t>(slot) * slot_bytes;
  };
  for (int step = 0; step < a.K && ok; ++step) {
    // phase A: GRU gate-row triples, input side then recurrent side
    for (int j = sc.p.j0; j < sc.p.j1 && ok; ++j) {
      for (int side = 0; side < 2 && ok; ++side) {
        const W* m = side == 0 ? w_ih : w_hh;
        const int ncol = side == 0 ? a.E : a.H;
        const Seg sg = side == 0 ? sc.e3 : sc.h3;
        for (int s = 0; s < sg.n; ++s, ++n) {
          uint8_t* dst = acquire(n);
          if (!dst) { ok = false; break; }
          const int c0 = s * sg.len, len = seg_len(sg, ncol, s);
          const uint32_t rowb = static_cast<uint32_t>(len) * sizeof(W);
          mbar_arrive_expect_tx(&sh.full[n % nslot], 3u * rowb);
          for (int g = 0; g < 3; ++g)
            bulk_g2s(dst + g * rowb, m + (static_cast<size_t>(g) * a.H + j) * ncol + c0, rowb, &sh.full[n % nslot], pol);
        }
      }
    }
    // phase B: recurrent block of W1 rows
    for (int k = sc.p.k0; k < sc.p.k1 && ok; ++k) {
      for (int s = 0; s < sc.h1.n; ++s, ++n) {
        uint8_t* dst = acquire(n);
        if (!dst) { ok = false; break; }
        const int c0 = s * sc.h1.len, len = seg_len(sc.h1, a.H, s);
        const uint32_t rowb = static_cast<uint32_t>(len) * sizeof(W);
        mbar_arrive_expect_tx(&sh.full[n % nslot], rowb);
        bulk_g2s(dst, w1 + static_cast<size_t>(k) * (a.d + a.H) + a.d + c0, rowb, &sh.full[n % nslot], pol);
      }
    }
    // phase C: W2 row chunks of 32 rows
    for (int v = sc.p.v0; v < sc.p.v1 && ok; v += 32, ++n) {
      uint8_t* dst = acquire(n);
      if (!dst) { ok = false; break; }
      const int rows = min(32, sc.p.v1 - v);
      const uint32_t bytes = static_cast<uint32_t>(rows) * a.r * sizeof(W);
      mbar_arrive_expect_tx(&sh.full[n % nslot], bytes);
      bulk_g2s(dst, w2 + static_cast<size_t>(v) * a.r, bytes, &sh.full[n % nslot], pol);
    }
  }
  // drain: every issued copy must land before the CTA may exit
  const int first = max(0, n - nslot);
  for (int item = first; item < n; ++item) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&sh.full[item % nslot], (item / nslot) & 1)) {
      if (globaltimer_ns() - t0 > a.budget_ns) {
        raise_error(a.ctl, ERRBIT_TIMEOUT);
        break;
      }
    }
  }
}

// ---------------------------------------------------------------- consumer helpers
template <typename W>
__device__ __forceinline__ void load_vec8(const uint8_t* base, int idx, float* out) {
  widen8(reinterpret_cast<const W*>(base) + idx, out);
}

// wait for item n (bound to this warp); returns the slot pointer or null on abort
__device__ __forceinline__ const uint8_t* consume_begin(const LoopArgs& a, const Shared& sh, int n) {
  if (aborted(sh)) return nullptr;
  const int slot = n % a.nslot;
  if (!mbar_wait(&sh.full[slot], (n / a.nslot) & 1, a.ctl, a.budget_ns)) {
    set_abort(sh);
    return nullptr;
  }
  return sh.ring + static_cast<size_t>(slot) * kLoopSlotBytes;
}
__device__ __forceinline__ void consume_end(const LoopArgs& a, const Shared& sh, int n) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&sh.empty[n % a.nslot]);
}

template <typename W, int NB>
__device__ void consumer(const LoopArgs& a, const Shared& sh, const Sched& sc) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const bool cta0 = blockIdx.x == 0;
  const int nb = a.nb;
  const int K = a.K;
  const W* embed = static_cast<const W*>(a.embed);
  const W* hidden = static_cast<const W*>(a.hidden);
  const W* w1 = static_cast<const W*>(a.w1);
  const int kmine = sc.p.k1 - sc.p.k0;

  // ---- prologue: zero argmax keys, W1_h h_i for own rows, S = 0, first GRU input
  if (cta0)
    for (int q = tid; q < K * NB; q += CONS_THREADS) a.best[q] = 0ull;
  for (int q = warp; q < kmine * nb * K; q += NCW) {
    const int kl = q / (nb * K), rem = q % (nb * K), b = rem / K, p = rem % K;
    const W* wrow = w1 + static_cast<size_t>(sc.p.k0 + kl) * (a.d + a.H);
    const W* hrow = hidden + (static_cast<size_t>(b) * K + p) * a.d;
    float acc = 0.f;
    for (int g = lane; g < a.d / 8; g += 32) {
      float wv[8], hv[8];
      widen8(wrow + g * 8, wv);
      widen8(hrow + g * 8, hv);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(wv[e], hv[e], acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) sh.hp[(kl * NB + b) * K + p] = acc;
  }
  for (int q = tid; q < NB * a.H; q += CONS_THREADS) sh.S[q] = 0.f;
  if (tid < NB) {
    int t = tid < nb ? a.anchor[tid] : 0;
    if (t < 0 || t >= a.V) {
      if (cta0) raise_error(a.ctl, ERRBIT_BAD_TOKEN);
      t = min(max(t, 0), a.V - 1);
    }
    sh.fed[tid] = t;
  }
  named_barrier(BAR_CONS, CONS_THREADS);
  const int xg = a.E / 8;  // 8-element groups per embedding row
  for (int q = tid; q < NB * xg; q += CONS_THREADS) {
    const int b = q / xg, g = q % xg;
    const uint4 v = *reinterpret_cast<const uint4*>(embed + static_cast<size_t>(sh.fed[b]) * a.E + g * 8);
    // storage widths: bf16 -> 16 B per group; f32 -> 32 B per group
    if (sizeof(W) == 2) {
      reinterpret_cast<uint4*>(sh.x)[q] = v;
    } else {
      const uint4 v2 = *reinterpret_cast<const uint4*>(embed + static_cast<size_t>(sh.fed[b]) * a.E + g * 8 + 4);
      reinterpret_cast<uint4*>(sh.x)[2 * q] = v;
      reinterpret_cast<uint4*>(sh.x)[2 * q + 1] = v2;
    }
  }
  named_barrier(BAR_CONS, CONS_THREADS);

  int n_base = 0;  // global item index of the first item of the current phase

  for (int i = 0; i < K; ++i) {
    // ================= phase A: GRU partial dot products
    for (int q = 0; q < sc.nA; ++q) {
      const int n = n_base + q;
      if (n % NCW != warp) continue;
      const uint8_t* slot = consume_begin(a, sh, n);
      if (slot) {
        const int per_unit = sc.e3.n + sc.h3.n;
        const int s_all = q % per_unit;
        const bool side_hh = s_all >= sc.e3.n;
        const int s = side_hh ? s_all - sc.e3.n : s_all;
        const Seg sg = side_hh ? sc.h3 : sc.e3;
        const int ncol = side_hh ? a.H : a.E;
        const int c0 = s * sg.len, len = seg_len(sg, ncol, s);
        float acc[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) acc[t] = 0.f;
        for (int g = lane; g < len / 8; g += 32) {
          float w0[8], w1v[8], w2v[8];
          load_vec8<W>(slot, g * 8, w0);
          load_vec8<W>(slot, len + g * 8, w1v);
          load_vec8<W>(slot, 2 * len + g * 8, w2v);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            float xv[8];
            if (side_hh) {
              const float* sp = sh.S + b * a.H + c0 + g * 8;
              const float4 p0 = *reinterpret_cast<const float4*>(sp);
              const float4 p1 = *reinterpret_cast<const float4*>(sp + 4);
              xv[0] = p0.x; xv[1] = p0.y; xv[2] = p0.z; xv[3] = p0.w;
              xv[4] = p1.x; xv[5] = p1.y; xv[6] = p1.z; xv[7] = p1.w;
            } else {
              load_vec8<W>(sh.x, b * a.E + c0 + g * 8, xv);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              acc[0 * NB + b] = fmaf(w0[e], xv[e], acc[0 * NB + b]);
              acc[1 * NB + b] = fmaf(w1v[e], xv[e], acc[1 * NB + b]);
              acc[2 * NB + b] = fmaf(w2v[e], xv[e], acc[2 * NB + b]);
            }
          }
        }
        const float tot = warp_reduce_scatter32(acc);
        sh.part[q * 32 + lane] = tot;
      }
      consume_end(a, sh, n);
    }
    n_base += sc.nA;
    named_barrier(BAR_CONS, CONS_THREADS);

    // GRU epilogue for own units: S_i[b][j]
    float* S_new = a.S_glob + static_cast<size_t>((i + 1) & 1) * NB * a.H;
    if (!aborted(sh)) {
      const int per_unit = sc.e3.n + sc.h3.n;
      for (int q = tid; q < (sc.p.j1 - sc.p.j0) * NB; q += CONS_THREADS) {
        const int jl = q / NB, b = q % NB;
        const int j = sc.p.j0 + jl;
        float gi[3] = {0.f, 0.f, 0.f}, gh[3] = {0.f, 0.f, 0.f};
        for (int s = 0; s < sc.e3.n; ++s)
          for (int g = 0; g < 3; ++g) gi[g] += sh.part[(jl * per_unit + s) * 32 + g * NB + b];
        for (int s = 0; s < sc.h3.n; ++s)
          for (int g = 0; g < 3; ++g) gh[g] += sh.part[(jl * per_unit + sc.e3.n + s) * 32 + g * NB + b];
        for (int g = 0; g < 3; ++g) {
          gi[g] += a.b_ih ? a.b_ih[g * a.H + j] : 0.f;
          gh[g] += a.b_hh ? a.b_hh[g * a.H + j] : 0.f;
        }
        const float r = 1.f / (1.f + expf(-(gi[0] + gh[0])));
        const float z = 1.f / (1.f + expf(-(gi[1] + gh[1])));
        const float nn = tanhf(gi[2] + r * gh[2]);
        const float s_old = sh.S[b * a.H + j];
        S_new[b * a.H + j] = (1.f - z) * nn + z * s_old;
      }
    }
    consumer_grid_sync(a, sh, G);  // ---- barrier 1: S_i complete

    // S_i -> shared (L1 bypassed: other SMs wrote it)
    if (!aborted(sh)) {
      for (int q = tid; q < NB * a.H / 4; q += CONS_THREADS)
        reinterpret_cast<float4*>(sh.S)[q] = __ldcg(reinterpret_cast<const float4*>(S_new) + q);
    }
    named_barrier(BAR_CONS, CONS_THREADS);

    // ================= phase B: u rows of this CTA
    for (int q = 0; q < sc.nB; ++q) {
      const int n = n_base + q;
      if (n % NCW != warp) continue;
      const uint8_t* slot = consume_begin(a, sh, n);
      if (slot) {
        const int s = q % sc.h1.n;
        const int c0 = s * sc.h1.len, len = seg_len(sc.h1, a.H, s);
        float acc[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) acc[t] = 0.f;
        for (int g = lane; g < len / 8; g += 32) {
          float wv[8];
          load_vec8<W>(slot, g * 8, wv);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const float* sp = sh.S + b * a.H + c0 + g * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[b] = fmaf(wv[e], sp[e], acc[b]);
          }
        }
        const float tot = warp_reduce_scatter32(acc);
        sh.part[q * 32 + lane] = tot;
      }
      consume_end(a, sh, n);
    }
    n_base += sc.nB;
    named_barrier(BAR_CONS, CONS_THREADS);
    if (!aborted(sh)) {
      for (int q = tid; q < kmine * nb; q += CONS_THREADS) {
        const int kl = q / nb, b = q % nb;
        float pre = sh.hp[(kl * NB + b) * K + i];
        for (int s = 0; s < sc.h1.n; ++s) pre += sh.part[(kl * sc.h1.n + s) * 32 + b];
        const float silu = pre / (1.f + expf(-pre));
        a.u_glob[b * a.r + sc.p.k0 + kl] = silu;
      }
    }
    consumer_grid_sync(a, sh, G);  // ---- barrier 2: u complete

    // u -> registers: lane holds u[b][8*lane .. 8*lane+8)
    float ureg[NB][8];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) ureg[b][e] = 0.f;
    if (!aborted(sh) && lane * 8 < a.r) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b < nb) {
          const float4 p0 = __ldcg(reinterpret_cast<const float4*>(a.u_glob + b * a.r + lane * 8));
          const float4 p1 = __ldcg(reinterpret_cast<const float4*>(a.u_glob + b * a.r + lane * 8 + 4));
          ureg[b][0] = p0.x; ureg[b][1] = p0.y; ureg[b][2] = p0.z; ureg[b][3] = p0.w;
          ureg[b][4] = p1.x; ureg[b][5] = p1.y; ureg[b][6] = p1.z; ureg[b][7] = p1.w;
        }
      }
    }

    // ================= phase C: W2 chunks, residual, pick
    constexpr int RPI = 32 / NB;           // rows per reduce-scatter round
    const int my_b = lane % NB;            // request whose sums this lane ends up with
    float best_s = -INFINITY;
    int best_v = 0x7FFFFFFF;
    const bool greedy = a.mode == 0;
    for (int q = 0; q < sc.nC; ++q) {
      const int n = n_base + q;
      if (n % NCW != warp) continue;
      const int vstart = sc.p.v0 + q * 32;
      const int rows = min(32, sc.p.v1 - vstart);
      // prefetch base logits for the (row, request) pairs this lane finalises
      float bpre[NB];
#pragma unroll
      for (int it = 0; it < NB; ++it) {
        const int rl = it * RPI + lane / NB;
        bpre[it] = (rl < rows && my_b < nb)
                       ? __ldg(a.base + (static_cast<size_t>(my_b) * K + i) * a.V + vstart + rl)
                       : 0.f;
      }
      const uint8_t* slot = consume_begin(a, sh, n);
      if (slot) {
#pragma unroll
        for (int it = 0; it < NB; ++it) {
          float acc[32];
#pragma unroll
          for (int t = 0; t < 32; ++t) acc[t] = 0.f;
          if (lane * 8 < a.r) {
#pragma unroll
            for (int rho = 0; rho < RPI; ++rho) {
              const int rl = it * RPI + rho;
              if (rl < rows) {
                float wv[8];
                load_vec8<W>(slot, rl * a.r + lane * 8, wv);
#pragma unroll
                for (int b = 0; b < NB; ++b)
#pragma unroll
                  for (int e = 0; e < 8; ++e) acc[rho * NB + b] = fmaf(wv[e], ureg[b][e], acc[rho * NB + b]);
              }
            }
          }
          const float dl = warp_reduce_scatter32(acc);
          const int rl = it * RPI + lane / NB;
          if (rl < rows && my_b < nb) {
            const int v = vstart + rl;
            const float L = bpre[it] + dl;
            if (a.logits) a.logits[(static_cast<size_t>(my_b) * K + i) * a.V + v] = L;
            float score = L;
            if (!greedy) score = __fdiv_rn(L, a.temperature) + gumbel_noise(a.seed, a.b0 + my_b, i, v);
            if (score > best_s) { best_s = score; best_v = v; }
          }
        }
      }
      consume_end(a, sh, n);
    }
    n_base += sc.nC;
    // merge lanes that hold the same request, then warps, then CTAs
#pragma unroll
    for (int off = 16; off >= NB; off >>= 1) {
      const float os = __shfl_xor_sync(0xFFFFFFFFu, best_s, off);
      const int ov = __shfl_xor_sync(0xFFFFFFFFu, best_v, off);
      if (os > best_s || (os == best_s && ov < best_v)) { best_s = os; best_v = ov; }
    }
    if (lane < NB) sh.wbest[warp * NB + lane] = best_v == 0x7FFFFFFF ? 0ull : argmax_key(best_s, best_v);
    named_barrier(BAR_CONS, CONS_THREADS);
    if (tid < nb && !aborted(sh)) {
      uint64_t k = 0;
      for (int w = 0; w < NCW; ++w) k = max(k, sh.wbest[w * NB + tid]);
      if (k != 0ull) atomicMax(reinterpret_cast<unsigned long long*>(&a.best[i * NB + tid]), static_cast<unsigned long long>(k));
    }
    consumer_grid_sync(a, sh, G);  // ---- barrier 3: picks merged

    // picks, next GRU input
    if (tid < nb) {
      const int b = tid;
      const uint64_t key = __ldcg(reinterpret_cast<const unsigned long long*>(&a.best[i * NB + b]));
      const int t = static_cast<int>(argmax_key_index(key));
      sh.tok[b * K + i] = t;
      if (cta0 && a.draft) a.draft[static_cast<size_t>(b) * K + i] = t;
      int f = a.forced ? a.forced[static_cast<size_t>(b) * K + i] : t;
      if (f < 0 || f >= a.V) {
        if (cta0) raise_error(a.ctl, ERRBIT_BAD_TOKEN);
        f = min(max(f, 0), a.V - 1);
      }
      sh.fed[b] = f;
    }
    named_barrier(BAR_CONS, CONS_THREADS);
    if (i + 1 < K && !aborted(sh)) {
      for (int q = tid; q < nb * xg; q += CONS_THREADS) {
        const int b = q / xg, g = q % xg;
        const uint4 v = *reinterpret_cast<const uint4*>(embed + static_cast<size_t>(sh.fed[b]) * a.E + g * 8);
        if (sizeof(W) == 2) {
          reinterpret_cast<uint4*>(sh.x)[q] = v;
        } else {
          const uint4 v2 = *reinterpret_cast<const uint4*>(embed + static_cast<size_t>(sh.fed[b]) * a.E + g * 8 + 4);
          reinterpret_cast<uint4*>(sh.x)[2 * q] = v;
          reinterpret_cast<uint4*>(sh.x)[2 * q + 1] = v2;
        }
      }
    }
    named_barrier(BAR_CONS, CONS_THREADS);
  }

  // verification (fused tail): CTA 0 has every pick in shared memory
  if (cta0 && a.target && a.tau && !aborted(sh)) {
    for (int b = tid; b < nb; b += CONS_THREADS) {
      int t = 0;
      while (t < K && sh.tok[b * K + t] == a.target[static_cast<size_t>(b) * K + t]) ++t;
      a.tau[b] = t;
    }
  }
}

template <typename W, int NB>
__global__ void __launch_bounds__(NTHREADS, 1) correct_loop_kernel(const LoopArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Shared sh = carve<NB>(smem, a);
  const int G = gridDim.x;
  if (a.selftest) {
    // one barrier episode that can never complete: exercises the bounded wait
    if (threadIdx.x == 0) grid_barrier_one_thread(a.ctl, static_cast<uint32_t>(G) + 1u, a.budget_ns);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.nslot; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    sh.flags[0] = 0;
    sh.flags[1] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const Sched sc = make_sched(a, blockIdx.x, G);
  if (threadIdx.x >= CONS_THREADS) {
    producer<W>(a, sh, sc);
  } else {
    consumer<W, NB>(a, sh, sc);
  }
}

template <typename W, int NB>
cudaError_t launch_one(const LoopArgs& a, int grid, size_t smem, cudaStream_t stream) {
  auto kern = correct_loop_kernel<W, NB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NTHREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  void* params[] = {const_cast<LoopArgs*>(&a)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), dim3(grid), dim3(NTHREADS), params, smem, stream);
}

}  // namespace

// Shared-memory layout and segment plan for a request group of NB requests.
size_t loop_plan(LoopArgs& a, int NB, int grid, size_t smem_cap) {
  const int wb = a.wbytes;
  // segments: triples of rows fit one slot; single rows fit one slot
  auto plan = [](int total, int maxlen, int& nseg, int& len) {
    maxlen = maxlen / 8 * 8;
    nseg = (total + maxlen - 1) / maxlen;
    len = ((total + nseg - 1) / nseg + 7) / 8 * 8;
  };
  plan(a.E, kLoopSlotBytes / (3 * wb), a.nsegE3, a.segE3);
  plan(a.H, kLoopSlotBytes / (3 * wb), a.nsegH3, a.segH3);
  plan(a.H, kLoopSlotBytes / wb, a.nsegH1, a.segH1);
  const int umax = (a.H + grid - 1) / grid;
  const int kmax = (a.r + grid - 1) / grid;
  a.max_part = umax * (a.nsegE3 + a.nsegH3);
  a.max_part = a.max_part > kmax * a.nsegH1 ? a.max_part : kmax * a.nsegH1;
  size_t off = 0;
  auto take = [&](size_t bytes, size_t align) {
    off = (off + align - 1) / align * align;
    const size_t at = off;
    off += bytes;
    return static_cast<uint32_t>(at);
  };
  // everything except the ring first, then as many slots as fit (multiple of NCW)
  size_t fixed = 0;
  {
    size_t o = 0;
    auto t2 = [&](size_t bytes, size_t align) { o = (o + align - 1) / align * align; o += bytes; };
    t2(2 * 8 * 64, 8);
    t2(static_cast<size_t>(NB) * a.H * 4, 16);
    t2(static_cast<size_t>(NB) * a.E * wb, 16);
    t2(static_cast<size_t>(NB) * a.r * 4, 16);
    t2(static_cast<size_t>(a.max_part) * 32 * 4, 16);
    t2(static_cast<size_t>(kmax) * NB * a.K * 4, 16);
    t2(static_cast<size_t>(NB) * a.K * 4, 16);
    t2(static_cast<size_t>(NCW) * NB * 8, 8);
    t2(64, 16);
    fixed = o + 1024;
  }
  if (fixed >= smem_cap) return 0;
  int nslot = static_cast<int>((smem_cap - fixed) / kLoopSlotBytes) / NCW * NCW;
  if (nslot > 16) nslot = 16;
  if (nslot < NCW) return 0;
  a.nslot = nslot;
  off = 0;
  take(static_cast<size_t>(nslot) * kLoopSlotBytes, 1024);
  a.off_bars = take(2 * 8 * nslot, 8);
  a.off_S = take(static_cast<size_t>(NB) * a.H * 4, 16);
  a.off_x = take(static_cast<size_t>(NB) * a.E * wb, 16);
  a.off_u = take(static_cast<size_t>(NB) * a.r * 4, 16);
  a.off_part = take(static_cast<size_t>(a.max_part) * 32 * 4, 16);
  a.off_hp = take(static_cast<size_t>(kmax) * NB * a.K * 4, 16);
  a.off_tok = take(static_cast<size_t>(NB) * a.K * 4, 16);
  a.off_wbest = take(static_cast<size_t>(NCW) * NB * 8, 8);
  a.off_flags = take(64, 16);
  return off;
}

int loop_group_size(int B) {
  if (B >= 8) return 8;
  if (B >= 4) return 4;
  if (B >= 2) return 2;
  return 1;
}

cudaError_t launch_correct_loop(LoopArgs a, int NB, int grid, size_t smem, cudaStream_t stream) {
  if (a.wbytes == 2) {
    switch (NB) {
      case 1: return launch_one<__nv_bfloat16, 1>(a, grid, smem, stream);
      case 2: return launch_one<__nv_bfloat16, 2>(a, grid, smem, stream);
      case 4: return launch_one<__nv_bfloat16, 4>(a, grid, smem, stream);
      default: return launch_one<__nv_bfloat16, 8>(a, grid, smem, stream);
    }
  }
  switch (NB) {
    case 1: return launch_one<float, 1>(a, grid, smem, stream);
    case 2: return launch_one<float, 2>(a, grid, smem, stream);
    case 4: return launch_one<float, 4>(a, grid, smem, stream);
    default: return launch_one<float, 8>(a, grid, smem, stream);
  }
}

int loop_threads() { return NTHREADS; }

}  // namespace domino
