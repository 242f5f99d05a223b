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
//   * GRU hidden units [j0, j1): the three gate rows of W_ih and W_hh and the
//     matching columns of W1's state block (kept in shared memory),
//   * bottleneck rows [k0, k1) (their W1_h h_i terms come from stage 1),
//   * a contiguous vocabulary range [v0, v1) of W2 (balanced so every CTA streams
//     about the same number of weight bytes per step).
// A producer warp streams exactly those weight bytes, step after step, through a
// shared-memory ring with 1-D bulk copies (TMA engine, no tensor map) and bulk
// L2 prefetches a fixed distance ahead of the ring.  The weights never depend on
// data, so HBM keeps streaming while consumers wait on grid barriers.  Consumer
// warps compute from the ring; item n is always handled by warp n % NCW and lands
// in slot n % NSLOT (NSLOT a multiple of NCW), so a slot is only ever waited on
// by the warp that consumed its previous occupant.
//
// Per step i, with two grid barriers:
//   A  W_ih x_i partial dots (ring) -> GRU epilogue for own units (the W_hh S
//      half was computed at the end of step i-1) -> each CTA's share of
//      W1 [h_i ; S] (own state columns + own rows' h terms) added into a
//      fixed-point int64 accumulator with red.add (exact, so order-free and
//      deterministic)
//   ---- barrier: S_i and the bottleneck pre-activation complete
//   C  u = SiLU(acc); W2 row chunks (ring) + base logits (staged in shared memory
//      with cp.async during A) -> per-lane argmax -> 64-bit atomicMax per request
//   ---- barrier arrive; meanwhile W_hh S_i partial dots for step i+1 (ring);
//        barrier wait -> picks, next embedding rows
// Delta L and L_i never touch HBM unless final logits are requested.
// With a token->gate table (LoopArgs::gate_table, G = W_ih E + b_ih built once per
// weight set) the W_ih items are dropped from the ring, the GRU epilogue reads
// the fed token's row of G, and no embedding rows are gathered.
#include <cstdint>

#include "common.cuh"
#include "domino_internal.h"

namespace domino {

namespace {

constexpr uint32_t BAR_CONS = 1;             // named barrier id among consumer warps
constexpr int L2_AHEAD = 32;                 // items prefetched into L2 ahead of the ring's next item
constexpr int VCHUNK = 32;                   // W2 rows per ring item
constexpr float kFixScale = 4294967296.0f;   // 2^32: fixed-point scale of the bottleneck accumulator

// Logistic function with the hardware exponential and divide: these sit on the
// per-step critical path (relative error ~1e-6, far inside the parity bounds).
__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
// tanh(x) = 2 sigmoid(2x) - 1
__device__ __forceinline__ float tanh_fast(float x) { return fmaf(2.f, sigmoid_fast(2.f * x), -1.f); }

// Consumer warps per CTA for a request group of NB: enough warps per scheduler to
// hide FMA / shuffle / shared-memory latency, within the register file and the
// shared memory left beside the larger groups' per-request state.
template <int NB> struct Warps { static constexpr int NCW = NB == 1 ? 12 : (NB <= 4 ? 8 : 4); };
constexpr int ncw_of(int NB) { return NB == 1 ? 12 : (NB <= 4 ? 8 : 4); }

struct Partition {
  int j0, j1;  // GRU units
  int k0, k1;  // bottleneck rows
  int v0, v1;  // vocabulary rows of W2
};

// Byte-balanced cut point of the vocabulary after CTA c (raw, before the
// running maximum that makes the split monotone).
__host__ __forceinline__ long long vend_raw(const LoopArgs& a, int c, int G) {
  if (c < 0) return 0;
  if (c >= G - 1) return a.V;
  const long long unitB = 3ll * (a.E + a.H) * a.wbytes;
  const long long rowB = 1ll * a.r * a.wbytes;
  const long long total = 1ll * a.H * unitB + 1ll * a.V * rowB;
  const long long target = total * (c + 1) / G;
  const long long used = 1ll * ((c + 1) * a.H / G) * unitB;
  long long v = (target - used) / rowB;
  if (v < 0) v = 0;
  if (v > a.V) v = a.V;
  return v;
}

// Units and bottleneck rows split evenly; the vocabulary split (computed once
// on the host into a.vsplit) balances the weight bytes every CTA streams.
__device__ __host__ __forceinline__ Partition partition_of(const LoopArgs& a, int c, int G) {
  Partition p;
  p.j0 = c * a.H / G;
  p.j1 = (c + 1) * a.H / G;
  p.k0 = c * a.r / G;
  p.k1 = (c + 1) * a.r / G;
  p.v0 = a.vsplit[c];
  p.v1 = a.vsplit[c + 1];
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
  float* base;     // [NB][vmax] this CTA's slice of the step's base logits
  float* part_ih;  // [max_ih][32] partial sums of the W_ih items
  float* part_hh;  // [max_hh][32] partial sums of the W_hh items
  float* hp;       // [kmax][NB][K] W1_h h terms of this CTA's rows
  float* bias;     // [umax][6] b_ih r,z,n then b_hh r,z,n of this CTA's units
  float* w1s;      // [umax][r] W1 state-block columns of this CTA's units
  float* s_own;    // [umax][NB] new state of this CTA's units
  float* u;        // [NB][r] bottleneck output u = SiLU(W1 [h_i ; S_{i-1}])
  int* tok;        // [NB][K] picks (CTA 0 verifies from here)
  uint64_t* wbest; // [NCW][NB]
  int* flags;      // [0] abort
  int* fed;        // [NB] token fed to the GRU at the next step
  uint8_t* items;  // [per_step] ring item table (producer)
};

__device__ __forceinline__ Shared carve(uint8_t* base, const LoopArgs& a) {
  Shared s;
  s.ring = base;
  s.full = reinterpret_cast<uint64_t*>(base + a.off_bars);
  s.empty = s.full + a.nslot;
  s.S = reinterpret_cast<float*>(base + a.off_S);
  s.x = base + a.off_x;
  s.base = reinterpret_cast<float*>(base + a.off_base);
  s.part_ih = reinterpret_cast<float*>(base + a.off_part);
  s.part_hh = s.part_ih + static_cast<size_t>(a.max_ih) * 32;
  s.hp = reinterpret_cast<float*>(base + a.off_hp);
  s.bias = reinterpret_cast<float*>(base + a.off_bias);
  s.w1s = reinterpret_cast<float*>(base + a.off_w1s);
  s.s_own = reinterpret_cast<float*>(base + a.off_sown);
  s.u = reinterpret_cast<float*>(base + a.off_u);
  s.tok = reinterpret_cast<int*>(base + a.off_tok);
  s.wbest = reinterpret_cast<uint64_t*>(base + a.off_wbest);
  s.flags = reinterpret_cast<int*>(base + a.off_flags);
  s.fed = s.flags + 4;
  s.items = base + a.off_items;
  return s;
}

__device__ __forceinline__ bool aborted(const Shared& s) {
  return *reinterpret_cast<volatile int*>(&s.flags[0]) != 0;
}
__device__ __forceinline__ void set_abort(const Shared& s) {
  *reinterpret_cast<volatile int*>(&s.flags[0]) = 1;
}

// Split grid barrier number k for the consumer warps.  arrive: after every
// consumer has finished its writes, one thread publishes the CTA's arrival.
// wait: one thread polls until all CTAs arrived, then every consumer proceeds.
// Control flow stays uniform after an abort (the waits are skipped).
template <int CONS_THREADS>
__device__ __forceinline__ void grid_arrive(const LoopArgs& a, const Shared& s) {
  named_barrier(BAR_CONS, CONS_THREADS);
  if (threadIdx.x == 0 && !aborted(s)) grid_barrier_arrive(a.ctl);
}
template <int CONS_THREADS>
__device__ __forceinline__ void grid_wait(const LoopArgs& a, const Shared& s, uint32_t k) {
  if (threadIdx.x == 0 && !aborted(s)) {
    if (!grid_barrier_wait(a.ctl, gridDim.x * (k + 1), a.budget_ns)) set_abort(s);
  }
  named_barrier(BAR_CONS, CONS_THREADS);
}

// ---------------------------------------------------------------- per-step item schedule
// Step i's ring items: [W_ih triples of own units] [W2 chunks] [W_hh triples of
// own units, for step i+1; absent in the last step].
struct Sched {
  Partition p;
  Seg e3, h3;
  int nIH, nC, nHH, per_step;
};
__device__ __forceinline__ Sched make_sched(const LoopArgs& a, int c, int G) {
  Sched s;
  s.p = partition_of(a, c, G);
  s.e3 = Seg{a.nsegE3, a.segE3};
  s.h3 = Seg{a.nsegH3, a.segH3};
  s.nIH = a.gate_table ? 0 : (s.p.j1 - s.p.j0) * s.e3.n;   // a token->gate table replaces the W_ih items
  s.nHH = (s.p.j1 - s.p.j0) * s.h3.n;
  s.nC = (s.p.v1 - s.p.v0 + VCHUNK - 1) / VCHUNK;
  s.per_step = s.nIH + s.nC + s.nHH;
  return s;
}

// Source ranges of per-step item q: `ncopy` copies of `bytes` each.
struct Item {
  const uint8_t* src[3];
  uint32_t bytes;
  int ncopy;
};
__device__ __forceinline__ Item item_of(const LoopArgs& a, const Sched& sc, int q) {
  Item it;
  const int wb = a.wbytes;
  if (q < sc.nIH || q >= sc.nIH + sc.nC) {
    const bool hh = q >= sc.nIH;
    const int qq = hh ? q - sc.nIH - sc.nC : q;
    const Seg sg = hh ? sc.h3 : sc.e3;
    const int j = sc.p.j0 + qq / sg.n, s = qq % sg.n;
    const int ncol = hh ? a.H : a.E;
    const uint8_t* m = static_cast<const uint8_t*>(hh ? a.w_hh : a.w_ih);
    const int c0 = s * sg.len, len = seg_len(sg, ncol, s);
    it.bytes = static_cast<uint32_t>(len) * wb;
    it.ncopy = 3;
    for (int g = 0; g < 3; ++g) it.src[g] = m + ((static_cast<size_t>(g) * a.H + j) * ncol + c0) * wb;
    return it;
  }
  const int v = sc.p.v0 + (q - sc.nIH) * VCHUNK;
  const int rows = min(VCHUNK, sc.p.v1 - v);
  it.bytes = static_cast<uint32_t>(rows) * a.r * wb;
  it.ncopy = 1;
  it.src[0] = static_cast<const uint8_t*>(a.w2) + static_cast<size_t>(v) * a.r * wb;
  it.src[1] = it.src[2] = nullptr;
  return it;
}

// Walks the item sequence: q over the step's table, W_hh items skipped in the last step.
struct Cursor {
  int step, q;
  __device__ __forceinline__ void next(const Sched& sc, int K) {
    ++q;
    if (step == K - 1 && q == sc.nIH + sc.nC) q = sc.per_step;
    if (q >= sc.per_step) {
      q = 0;
      ++step;
    }
  }
};

// ---------------------------------------------------------------- producer
__device__ void producer(const LoopArgs& a, const Shared& sh, const Sched& sc) {
  if ((threadIdx.x & 31) != 0) return;
  if (sc.per_step == 0) return;
  Item* table = reinterpret_cast<Item*>(sh.items);
  for (int q = 0; q < sc.per_step; ++q) table[q] = item_of(a, sc, q);
  const uint64_t pol = policy_evict_first();
  const int nslot = a.nslot;
  Cursor cur{0, 0}, ahead{0, 0};
  // warm L2 with the first items
  for (int p = 0; p < L2_AHEAD && ahead.step < a.K; ++p) {
    const Item& it = table[ahead.q];
    for (int c = 0; c < it.ncopy; ++c) bulk_prefetch_l2(it.src[c], it.bytes);
    ahead.next(sc, a.K);
  }
  int n = 0, n_ahead = L2_AHEAD, slot = 0;
  uint32_t phase = 0;
  // one more L2 prefetch, at most L2_AHEAD items beyond the ring's next item
  auto prefetch_one = [&]() {
    if (ahead.step < a.K && n_ahead < n + L2_AHEAD) {
      const Item& ah = table[ahead.q];
      for (int c = 0; c < ah.ncopy; ++c) bulk_prefetch_l2(ah.src[c], ah.bytes);
      ahead.next(sc, a.K);
      ++n_ahead;
    }
  };
  for (; cur.step < a.K; ++n, cur.next(sc, a.K)) {
    if (n >= nslot) {
      const uint64_t t0 = globaltimer_ns();
      bool ok = true;
      while (!mbar_try_wait(&sh.empty[slot], phase ^ 1u)) {
        prefetch_one();             // keep HBM busy while the consumers are held up
        if (aborted(sh)) { ok = false; break; }
        if (globaltimer_ns() - t0 > a.budget_ns) {
          raise_error(a.ctl, ERRBIT_TIMEOUT);
          set_abort(sh);
          ok = false;
          break;
        }
      }
      if (!ok) break;
    }
    prefetch_one();
    const Item& it = table[cur.q];
    uint8_t* dst = sh.ring + static_cast<size_t>(slot) * kLoopSlotBytes;
    mbar_arrive_expect_tx(&sh.full[slot], it.bytes * it.ncopy);
    for (int c = 0; c < it.ncopy; ++c) bulk_g2s(dst + c * it.bytes, it.src[c], it.bytes, &sh.full[slot], pol);
    if (++slot == nslot) { slot = 0; phase ^= 1u; }
  }
  // drain: every issued copy must land before the CTA may exit
  for (int item = max(0, n - nslot); item < n; ++item) {
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

// Eight storage elements loaded raw from shared memory, widened later (keeps
// several rows' loads in flight before the arithmetic that consumes them).
template <typename W> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void load(const uint8_t* base, int idx) {
    v = *reinterpret_cast<const uint4*>(base + static_cast<size_t>(idx) * 2);
  }
  __device__ __forceinline__ void widen(float* out) const {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      out[2 * k] = __uint_as_float(w[k] << 16);
      out[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const uint8_t* base, int idx) {
    const float4* p = reinterpret_cast<const float4*>(base + static_cast<size_t>(idx) * 4);
    a = p[0];
    b = p[1];
  }
  __device__ __forceinline__ void widen(float* out) const {
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  }
};

template <typename W, int CONS_THREADS>
__device__ __forceinline__ void gather_rows(const LoopArgs& a, const Shared& sh, int nrows) {
  const W* embed = static_cast<const W*>(a.embed);
  const int xg = a.E / 8;  // 8-element groups per embedding row
  for (int q = threadIdx.x; q < nrows * xg; q += CONS_THREADS) {
    const int b = q / xg, g = q % xg;
    const W* src = embed + static_cast<size_t>(sh.fed[b]) * a.E + g * 8;
    if (sizeof(W) == 2) {
      reinterpret_cast<uint4*>(sh.x)[q] = __ldg(reinterpret_cast<const uint4*>(src));
    } else {
      reinterpret_cast<uint4*>(sh.x)[2 * q] = __ldg(reinterpret_cast<const uint4*>(src));
      reinterpret_cast<uint4*>(sh.x)[2 * q + 1] = __ldg(reinterpret_cast<const uint4*>(src) + 1);
    }
  }
}

// Three gate-row dot products of one ring item (3 rows x len columns starting at
// column c0) against NB vectors: the fed embeddings (ih) or the state (hh).
// Lane l ends with slot l of [gate][request] (the warp's reduce-scatter).
template <typename W, int NB, bool HH>
__device__ __forceinline__ float gate_triple(const LoopArgs& a, const Shared& sh, const uint8_t* slot, int c0,
                                             int len) {
  const int lane = threadIdx.x & 31;
  float acc[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) acc[t] = 0.f;
  for (int g = lane; g < len / 8; g += 32) {
    Raw8<W> r0, r1, r2;
    r0.load(slot, g * 8);
    r1.load(slot, len + g * 8);
    r2.load(slot, 2 * len + g * 8);
    float w0[8], w1v[8], w2v[8];
    r0.widen(w0);
    r1.widen(w1v);
    r2.widen(w2v);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float xv[8];
      if (HH) {
        const float* sp = sh.S + b * a.H + c0 + g * 8;
        const float4 p0 = *reinterpret_cast<const float4*>(sp);
        const float4 p1 = *reinterpret_cast<const float4*>(sp + 4);
        xv[0] = p0.x; xv[1] = p0.y; xv[2] = p0.z; xv[3] = p0.w;
        xv[4] = p1.x; xv[5] = p1.y; xv[6] = p1.z; xv[7] = p1.w;
      } else {
        Raw8<W> rx;
        rx.load(sh.x, b * a.E + c0 + g * 8);
        rx.widen(xv);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc[0 * NB + b] = fmaf(w0[e], xv[e], acc[0 * NB + b]);
        acc[1 * NB + b] = fmaf(w1v[e], xv[e], acc[1 * NB + b]);
        acc[2 * NB + b] = fmaf(w2v[e], xv[e], acc[2 * NB + b]);
      }
    }
  }
  return warp_reduce_scatter32(acc);
}

__device__ __forceinline__ long long* uacc_at(const LoopArgs& a, int buf, int b, int k) {
  return a.u_acc + ((static_cast<size_t>(buf) * 8 + b) * a.r + k) * kUaccStride;
}

template <typename W, int NB, int NCW>
__device__ void consumer(const LoopArgs& a, const Shared& sh, const Sched& sc) {
  constexpr int CONS_THREADS = NCW * 32;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool cta0 = blockIdx.x == 0;
  const int G = gridDim.x;
  const int nb = a.nb;
  const int K = a.K;
  const int kmine = sc.p.k1 - sc.p.k0;
  const int umine = sc.p.j1 - sc.p.j0;
  const int vrows = sc.p.v1 - sc.p.v0;
  const W* w1 = static_cast<const W*>(a.w1);
  uint32_t nbar = 0;

  // ---- prologue: zero argmax keys and this CTA's share of both accumulators,
  // stage biases, W1 state columns and W1_h h terms, S = 0, first GRU input
  if (cta0)
    for (int q = tid; q < K * NB; q += CONS_THREADS) a.best[q] = 0ull;
  for (int q = blockIdx.x * CONS_THREADS + tid; q < 2 * NB * a.r; q += G * CONS_THREADS)
    *uacc_at(a, q / (NB * a.r), (q / a.r) % NB, q % a.r) = 0ll;
  for (int q = tid; q < umine * 6; q += CONS_THREADS) {
    const int jl = q / 6, g = q % 6;
    const float* bsrc = g < 3 ? a.b_ih : a.b_hh;
    sh.bias[q] = bsrc ? bsrc[(g % 3) * a.H + sc.p.j0 + jl] : 0.f;
  }
  for (int q = tid; q < umine * a.r; q += CONS_THREADS) {
    const int jl = q / a.r, k = q % a.r;
    const W wv = w1[static_cast<size_t>(k) * (a.d + a.H) + a.d + sc.p.j0 + jl];
    sh.w1s[jl * a.r + k] = static_cast<float>(wv);
  }
  for (int q = tid; q < kmine * nb * K; q += CONS_THREADS) {
    const int kl = q / (nb * K), rem = q % (nb * K), b = rem / K, p = rem % K;
    sh.hp[(kl * NB + b) * K + p] = a.hp[(static_cast<size_t>(b) * K + p) * a.r + sc.p.k0 + kl];
  }
  for (int q = tid; q < NB * a.H; q += CONS_THREADS) sh.S[q] = 0.f;
  for (int q = tid; q < sc.nHH * 32; q += CONS_THREADS) sh.part_hh[q] = 0.f;   // W_hh S_0 = 0
  if (tid < NB) {
    int t = tid < nb ? a.anchor[tid] : 0;
    if (t < 0 || t >= a.V) {
      if (cta0) raise_error(a.ctl, ERRBIT_BAD_TOKEN);
      t = min(max(t, 0), a.V - 1);
    }
    sh.fed[tid] = t;
  }
  named_barrier(BAR_CONS, CONS_THREADS);
  if (!a.gate_table) gather_rows<W, CONS_THREADS>(a, sh, NB);
  grid_arrive<CONS_THREADS>(a, sh);         // zeroed keys and accumulators visible to all
  grid_wait<CONS_THREADS>(a, sh, nbar++);

  int n = 0;  // global ring item index of the next item
  for (int i = 0; i < K; ++i) {
    const int buf = i & 1;
    // base-logit slice of this step -> shared memory, overlapped with the GRU
    if (!aborted(sh)) {
      for (int q = tid; q < nb * vrows; q += CONS_THREADS) {
        const int b = q / vrows, v = q % vrows;
        cp_async4(sh.base + b * a.vmax + v, a.base + (static_cast<size_t>(b) * K + i) * a.V + sc.p.v0 + v);
      }
    }
    cp_async_commit();

    // ================= A: W_ih x partial dots
    for (int q = 0; q < sc.nIH; ++q) {
      const int nn = n + q;
      if (nn % NCW != warp) continue;
      const uint8_t* slot = consume_begin(a, sh, nn);
      if (slot) {
        const int s = q % sc.e3.n;
        const float tot = gate_triple<W, NB, false>(a, sh, slot, s * sc.e3.len, seg_len(sc.e3, a.E, s));
        sh.part_ih[q * 32 + lane] = tot;
      }
      consume_end(a, sh, nn);
    }
    n += sc.nIH;
    named_barrier(BAR_CONS, CONS_THREADS);

    // GRU epilogue for own units: S_i[b][j]
    float* S_new = a.S_glob + static_cast<size_t>((i + 1) & 1) * NB * a.H;
    if (!aborted(sh)) {
      for (int q = tid; q < umine * NB; q += CONS_THREADS) {
        const int jl = q / NB, b = q % NB;
        const int j = sc.p.j0 + jl;
        float gi[3], gh[3];
        for (int g = 0; g < 3; ++g) {
          gi[g] = sh.bias[jl * 6 + g];
          gh[g] = sh.bias[jl * 6 + 3 + g];
        }
        if (a.gate_table) {
          // the fed token's row of G = W_ih E + b_ih (sh.fed is always a valid token)
          const float* trow = a.gate_table + static_cast<size_t>(sh.fed[b]) * 3 * a.H;
          for (int g = 0; g < 3; ++g) gi[g] = trow[g * a.H + j];
        } else {
          for (int s = 0; s < sc.e3.n; ++s)
            for (int g = 0; g < 3; ++g) gi[g] += sh.part_ih[(jl * sc.e3.n + s) * 32 + g * NB + b];
        }
        for (int s = 0; s < sc.h3.n; ++s)
          for (int g = 0; g < 3; ++g) gh[g] += sh.part_hh[(jl * sc.h3.n + s) * 32 + g * NB + b];
        const float r = sigmoid_fast(gi[0] + gh[0]);
        const float z = sigmoid_fast(gi[1] + gh[1]);
        const float nn = tanh_fast(gi[2] + r * gh[2]);
        const float s_old = sh.S[b * a.H + j];
        const float s_new = (1.f - z) * nn + z * s_old;
        S_new[b * a.H + j] = s_new;
        sh.s_own[jl * NB + b] = s_new;
      }
    }
    named_barrier(BAR_CONS, CONS_THREADS);
    // this CTA's share of the bottleneck pre-activation, in 2^-32 fixed point
    if (!aborted(sh)) {
      for (int q = tid; q < a.r * nb; q += CONS_THREADS) {
        const int k = q % a.r, b = q / a.r;
        const bool own_row = k >= sc.p.k0 && k < sc.p.k1;
        if (umine == 0 && !own_row) continue;
        float p = 0.f;
        for (int jl = 0; jl < umine; ++jl) p = fmaf(sh.w1s[jl * a.r + k], sh.s_own[jl * NB + b], p);
        if (own_row) p += sh.hp[((k - sc.p.k0) * NB + b) * K + i];
        const long long fx = __float2ll_rn(p * kFixScale);
        asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(uacc_at(a, buf, b, k)), "l"(fx) : "memory");
      }
    }
    grid_arrive<CONS_THREADS>(a, sh);
    grid_wait<CONS_THREADS>(a, sh, nbar++);   // ---- S_i and the pre-activation complete

    // S_i -> shared (L1 bypassed: other SMs wrote it); clear this CTA's share of
    // the other accumulator for step i+1 (all reads of it ended before this barrier)
    if (!aborted(sh)) {
      for (int q = tid; q < NB * a.H / 4; q += CONS_THREADS)
        reinterpret_cast<float4*>(sh.S)[q] = __ldcg(reinterpret_cast<const float4*>(S_new) + q);
      for (int q = blockIdx.x * CONS_THREADS + tid; q < NB * a.r; q += G * CONS_THREADS)
        *uacc_at(a, buf ^ 1, q / a.r, q % a.r) = 0ll;
    }
    // u = SiLU(pre-activation): read once per CTA (one thread per entry) into
    // shared memory, then every warp takes its registers from there
    if (!aborted(sh)) {
      for (int q = tid; q < nb * a.r; q += CONS_THREADS) {
        const int b = q / a.r, k = q % a.r;
        const long long fx = __ldcg(uacc_at(a, buf, b, k));
        const float pre = static_cast<float>(static_cast<double>(fx) * (1.0 / 4294967296.0));
        sh.u[b * a.r + k] = pre * sigmoid_fast(pre);
      }
    }
    cp_async_wait_all();
    named_barrier(BAR_CONS, CONS_THREADS);
    float ureg[NB][8];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const bool have = b < nb && lane * 8 < a.r;
      const float4 p0 = have ? *reinterpret_cast<const float4*>(sh.u + b * a.r + lane * 8) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 p1 = have ? *reinterpret_cast<const float4*>(sh.u + b * a.r + lane * 8 + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      ureg[b][0] = p0.x; ureg[b][1] = p0.y; ureg[b][2] = p0.z; ureg[b][3] = p0.w;
      ureg[b][4] = p1.x; ureg[b][5] = p1.y; ureg[b][6] = p1.z; ureg[b][7] = p1.w;
    }

    // ================= C: W2 chunks, residual, pick
    constexpr int RPI = 32 / NB;           // rows per reduce-scatter round
    const int my_b = lane % NB;            // request whose sums this lane ends up with
    float best_s = -INFINITY;
    int best_v = 0x7FFFFFFF;
    const bool greedy = a.mode == 0;
    for (int q = 0; q < sc.nC; ++q) {
      const int nn = n + q;
      if (nn % NCW != warp) continue;
      const int vl0 = q * VCHUNK;          // chunk start, relative to v0
      const int rows = min(VCHUNK, vrows - vl0);
      const uint8_t* slot = consume_begin(a, sh, nn);
      if (slot) {
#pragma unroll
        for (int it = 0; it < NB; ++it) {
          float acc[32];
#pragma unroll
          for (int t = 0; t < 32; ++t) acc[t] = 0.f;
          if (lane * 8 < a.r) {
            constexpr int BATCH = RPI < 8 ? RPI : 8;
#pragma unroll
            for (int rb = 0; rb < RPI; rb += BATCH) {
              Raw8<W> raw[BATCH];
#pragma unroll
              for (int q2 = 0; q2 < BATCH; ++q2) raw[q2].load(slot, (it * RPI + rb + q2) * a.r + lane * 8);
#pragma unroll
              for (int q2 = 0; q2 < BATCH; ++q2) {
                const int rho = rb + q2;
                // rows past the chunk end read stale slot bytes: replace them by zero
                const bool keep = (it * RPI + rho) < rows;
                float wv[8];
                raw[q2].widen(wv);
#pragma unroll
                for (int e = 0; e < 8; ++e) wv[e] = keep ? wv[e] : 0.f;
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
            const int v = sc.p.v0 + vl0 + rl;
            const float L = sh.base[my_b * a.vmax + vl0 + rl] + dl;
            if (a.logits) a.logits[(static_cast<size_t>(my_b) * K + i) * a.V + v] = L;
            float score = L;
            if (!greedy) score = __fdiv_rn(L, a.temperature) + gumbel_noise(a.seed, a.b0 + my_b, i, v);
            if (score > best_s) { best_s = score; best_v = v; }
          }
        }
      }
      consume_end(a, sh, nn);
    }
    n += sc.nC;
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
      if (k != 0ull) {
        atomicMax(reinterpret_cast<unsigned long long*>(&a.best[i * NB + tid]), static_cast<unsigned long long>(k));
        // this CTA's candidate may win: bring its embedding row to L2 for the next gather
        if (i + 1 < K && !a.forced)
          bulk_prefetch_l2(static_cast<const uint8_t*>(a.embed) +
                               static_cast<size_t>(argmax_key_index(k)) * a.E * a.wbytes,
                           static_cast<uint32_t>(a.E) * a.wbytes);
      }
    }
    grid_arrive<CONS_THREADS>(a, sh);

    // ================= W_hh S_i partial dots for step i+1, overlapping the barrier
    if (i + 1 < K) {
      for (int q = 0; q < sc.nHH; ++q) {
        const int nn = n + q;
        if (nn % NCW != warp) continue;
        const uint8_t* slot = consume_begin(a, sh, nn);
        if (slot) {
          const int s = q % sc.h3.n;
          const float tot = gate_triple<W, NB, true>(a, sh, slot, s * sc.h3.len, seg_len(sc.h3, a.H, s));
          sh.part_hh[q * 32 + lane] = tot;
        }
        consume_end(a, sh, nn);
      }
      n += sc.nHH;
    }
    grid_wait<CONS_THREADS>(a, sh, nbar++);   // ---- picks merged

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
    if (i + 1 < K && !aborted(sh) && !a.gate_table) gather_rows<W, CONS_THREADS>(a, sh, nb);
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
  if (tid == 0) grid_exit(a.ctl, gridDim.x);
}

template <typename W, int NB, int NCW>
__global__ void __launch_bounds__((NCW + 1) * 32, 1) correct_loop_kernel(const LoopArgs a) {
  constexpr int CONS_THREADS = NCW * 32;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int G = gridDim.x;
  if (a.selftest) {
    // one barrier episode that can never complete: exercises the bounded wait
    if (threadIdx.x == 0) {
      grid_barrier_arrive(a.ctl);
      grid_barrier_wait(a.ctl, static_cast<uint32_t>(G) + 1u, a.budget_ns);
      grid_exit(a.ctl, G);
    }
    return;
  }
  Shared sh = carve(smem, a);
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.nslot; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    sh.flags[0] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const Sched sc = make_sched(a, blockIdx.x, G);
  if (threadIdx.x >= CONS_THREADS) {
    producer(a, sh, sc);
  } else {
    consumer<W, NB, NCW>(a, sh, sc);
  }
}

template <typename W, int NB>
cudaError_t launch_one(const LoopArgs& a, int grid, size_t smem, cudaStream_t stream) {
  constexpr int NCW = Warps<NB>::NCW;
  constexpr int NTHREADS = (NCW + 1) * 32;
  auto kern = correct_loop_kernel<W, NB, NCW>;
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

// Shared-memory layout, vocabulary split and segment plan for a request group of NB.
size_t loop_plan(LoopArgs& a, int NB, int grid, size_t smem_cap) {
  const int wb = a.wbytes;
  const int NCW = ncw_of(NB);
  // segments: a triple of gate rows fits one slot
  auto plan = [](int total, int maxlen, int& nseg, int& len) {
    maxlen = maxlen / 8 * 8;
    nseg = (total + maxlen - 1) / maxlen;
    len = ((total + nseg - 1) / nseg + 7) / 8 * 8;
  };
  plan(a.E, kLoopSlotBytes / (3 * wb), a.nsegE3, a.segE3);
  plan(a.H, kLoopSlotBytes / (3 * wb), a.nsegH3, a.segH3);
  const int umax = (a.H + grid - 1) / grid;
  const int kmax = (a.r + grid - 1) / grid;
  a.max_ih = umax * a.nsegE3;
  a.max_hh = umax * a.nsegH3;
  if (grid > kLoopMaxGrid) return 0;
  // vocabulary split: running maximum of the byte-balanced cut points
  long long lo = 0;
  a.vsplit[0] = 0;
  for (int c = 0; c < grid; ++c) {
    const long long raw = vend_raw(a, c, grid);
    lo = lo > raw ? lo : raw;
    a.vsplit[c + 1] = static_cast<int32_t>(lo);
  }
  a.vsplit[grid] = a.V;
  int vmax = 0, items_max = 0;
  for (int c = 0; c < grid; ++c) {
    const Partition p = partition_of(a, c, grid);
    vmax = vmax > p.v1 - p.v0 ? vmax : p.v1 - p.v0;
    const int n = (p.j1 - p.j0) * (a.nsegE3 + a.nsegH3) + (p.v1 - p.v0 + VCHUNK - 1) / VCHUNK;
    items_max = items_max > n ? items_max : n;
  }
  a.vmax = (vmax + 3) / 4 * 4;
  struct Piece { uint32_t* off; size_t bytes; size_t align; };
  const Piece pieces[] = {
      {&a.off_S, static_cast<size_t>(NB) * a.H * 4, 16},
      {&a.off_x, static_cast<size_t>(NB) * a.E * wb, 16},
      {&a.off_base, static_cast<size_t>(NB) * a.vmax * 4, 16},
      {&a.off_part, static_cast<size_t>(a.max_ih + a.max_hh) * 32 * 4, 16},
      {&a.off_hp, static_cast<size_t>(kmax) * NB * a.K * 4, 16},
      {&a.off_bias, static_cast<size_t>(umax) * 6 * 4, 16},
      {&a.off_w1s, static_cast<size_t>(umax) * a.r * 4, 16},
      {&a.off_sown, static_cast<size_t>(umax) * NB * 4, 16},
      {&a.off_u, static_cast<size_t>(NB) * a.r * 4, 16},
      {&a.off_tok, static_cast<size_t>(NB) * a.K * 4, 16},
      {&a.off_wbest, static_cast<size_t>(NCW) * NB * 8, 8},
      {&a.off_flags, 64, 16},
      {&a.off_items, static_cast<size_t>(items_max) * sizeof(Item), 16},
  };
  size_t fixed = 2 * 8 * 16 + 16;  // barriers of up to 16 slots
  for (const Piece& p : pieces) fixed = (fixed + p.align - 1) / p.align * p.align + p.bytes;
  fixed += 1024;
  if (fixed >= smem_cap) return 0;
  int nslot = static_cast<int>((smem_cap - fixed) / kLoopSlotBytes);
  if (nslot > 16) nslot = 16;
  nslot = nslot / NCW * NCW;
  if (nslot < NCW) return 0;
  a.nslot = nslot;
  size_t off = static_cast<size_t>(nslot) * kLoopSlotBytes;
  a.off_bars = static_cast<uint32_t>(off);
  off += 2 * 8 * nslot;
  for (const Piece& p : pieces) {
    off = (off + p.align - 1) / p.align * p.align;
    *p.off = static_cast<uint32_t>(off);
    off += p.bytes;
  }
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

int loop_threads(int NB) { return (ncw_of(NB) + 1) * 32; }

}  // namespace domino
