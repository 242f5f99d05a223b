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
// shared-memory ring with 1-D bulk copies (TMA engine, no tensor map), and
// issues bulk L2 prefetches a fixed distance ahead of the ring.  The weights
// never depend on data, so HBM keeps streaming while consumers wait on grid
// barriers.  Four consumer warps compute from the ring; item n is always handled
// by warp n % 4 and lands in slot n % NSLOT (NSLOT a multiple of 4), so a slot is
// only ever waited on by the warp that consumed its previous occupant.
// Per step three bounded grid barriers: after the GRU (S_i complete), after the
// bottleneck (u complete), after the vocabulary pass (argmax keys merged with a
// 64-bit atomicMax).  W1 [h_i ; S] is split as W1_h h_i + W1_s S; the W1_h h_i
// terms come precomputed from stage 1.  The CTA's slice of the base logits for
// step i is copied into shared memory with cp.async while the GRU runs.
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
constexpr int L2_AHEAD = 16;                 // items prefetched into L2 ahead of the ring
constexpr int VCHUNK = 32;                   // W2 rows per ring item

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
  float* part;     // [max_part][32] per-item partial sums
  float* hp;       // [kmax][NB][K] W1_h h terms of this CTA's rows
  float* bias;     // [umax][6] b_ih r,z,n then b_hh r,z,n of this CTA's units
  int* tok;        // [NB][K] picks (CTA 0 verifies from here)
  uint64_t* wbest; // [NCW][NB]
  int* flags;      // [0] abort
  int* fed;        // [NB] token fed to the GRU at the next step
  uint8_t* items;  // [max_items] per-step ring item table (producer)
};

__device__ __forceinline__ Shared carve(uint8_t* base, const LoopArgs& a) {
  Shared s;
  s.ring = base;
  s.full = reinterpret_cast<uint64_t*>(base + a.off_bars);
  s.empty = s.full + a.nslot;
  s.S = reinterpret_cast<float*>(base + a.off_S);
  s.x = base + a.off_x;
  s.base = reinterpret_cast<float*>(base + a.off_base);
  s.part = reinterpret_cast<float*>(base + a.off_part);
  s.hp = reinterpret_cast<float*>(base + a.off_hp);
  s.bias = reinterpret_cast<float*>(base + a.off_bias);
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

// Consumer-wide grid barrier number k: named barrier, one thread arrives and
// waits, named barrier.  Keeps control flow uniform even after an abort.
__device__ __forceinline__ void consumer_grid_sync(const LoopArgs& a, const Shared& s, uint32_t k) {
  named_barrier(BAR_CONS, CONS_THREADS);
  if (threadIdx.x == 0 && !aborted(s)) {
    if (!grid_barrier_one_thread(a.ctl, gridDim.x * (k + 1), a.budget_ns)) set_abort(s);
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
  s.nC = (s.p.v1 - s.p.v0 + VCHUNK - 1) / VCHUNK;
  s.per_step = s.nA + s.nB + s.nC;
  return s;
}

// Source ranges of ring item n: `ncopy` copies of `bytes` each (3 gate rows of
// one unit, one W1 row segment, or one W2 row chunk).
struct Item {
  const uint8_t* src[3];
  uint32_t bytes;
  int ncopy;
};
__device__ __forceinline__ Item item_of(const LoopArgs& a, const Sched& sc, int n) {
  Item it;
  int q = n % sc.per_step;
  const int wb = a.wbytes;
  if (q < sc.nA) {
    const int per_unit = sc.e3.n + sc.h3.n;
    const int j = sc.p.j0 + q / per_unit;
    const int s_all = q % per_unit;
    const bool hh = s_all >= sc.e3.n;
    const int s = hh ? s_all - sc.e3.n : s_all;
    const Seg sg = hh ? sc.h3 : sc.e3;
    const int ncol = hh ? a.H : a.E;
    const uint8_t* m = static_cast<const uint8_t*>(hh ? a.w_hh : a.w_ih);
    const int c0 = s * sg.len, len = seg_len(sg, ncol, s);
    it.bytes = static_cast<uint32_t>(len) * wb;
    it.ncopy = 3;
    for (int g = 0; g < 3; ++g) it.src[g] = m + ((static_cast<size_t>(g) * a.H + j) * ncol + c0) * wb;
    return it;
  }
  q -= sc.nA;
  if (q < sc.nB) {
    const int k = sc.p.k0 + q / sc.h1.n, s = q % sc.h1.n;
    const int c0 = s * sc.h1.len, len = seg_len(sc.h1, a.H, s);
    it.bytes = static_cast<uint32_t>(len) * wb;
    it.ncopy = 1;
    it.src[0] = static_cast<const uint8_t*>(a.w1) + (static_cast<size_t>(k) * (a.d + a.H) + a.d + c0) * wb;
    it.src[1] = it.src[2] = nullptr;
    return it;
  }
  q -= sc.nB;
  const int v = sc.p.v0 + q * VCHUNK;
  const int rows = min(VCHUNK, sc.p.v1 - v);
  it.bytes = static_cast<uint32_t>(rows) * a.r * wb;
  it.ncopy = 1;
  it.src[0] = static_cast<const uint8_t*>(a.w2) + static_cast<size_t>(v) * a.r * wb;
  it.src[1] = it.src[2] = nullptr;
  return it;
}

// ---------------------------------------------------------------- producer
// The per-step item sequence is identical for every step, so the producer
// decodes it once into shared memory and then only walks the table.
__device__ void producer(const LoopArgs& a, const Shared& sh, const Sched& sc) {
  if ((threadIdx.x & 31) != 0) return;
  Item* table = reinterpret_cast<Item*>(sh.items);
  for (int q = 0; q < sc.per_step; ++q) table[q] = item_of(a, sc, q);
  const uint64_t pol = policy_evict_first();
  const int nslot = a.nslot;
  const int total = a.K * sc.per_step;
  // warm L2 with the first items
  int ahead_q = 0;
  for (int p = 0; p < L2_AHEAD && p < total; ++p) {
    const Item& it = table[ahead_q];
    for (int c = 0; c < it.ncopy; ++c) bulk_prefetch_l2(it.src[c], it.bytes);
    if (++ahead_q == sc.per_step) ahead_q = 0;
  }
  int n = 0, q = 0, slot = 0;
  uint32_t phase = 0;
  for (; n < total; ++n) {
    if (n >= nslot) {
      const uint64_t t0 = globaltimer_ns();
      bool ok = true;
      while (!mbar_try_wait(&sh.empty[slot], phase ^ 1u)) {
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
    if (n + L2_AHEAD < total) {
      const Item& ah = table[ahead_q];
      for (int c = 0; c < ah.ncopy; ++c) bulk_prefetch_l2(ah.src[c], ah.bytes);
      if (++ahead_q == sc.per_step) ahead_q = 0;
    }
    const Item& it = table[q];
    uint8_t* dst = sh.ring + static_cast<size_t>(slot) * kLoopSlotBytes;
    mbar_arrive_expect_tx(&sh.full[slot], it.bytes * it.ncopy);
    for (int c = 0; c < it.ncopy; ++c) bulk_g2s(dst + c * it.bytes, it.src[c], it.bytes, &sh.full[slot], pol);
    if (++q == sc.per_step) q = 0;
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

template <typename W>
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

template <typename W, int NB>
__device__ void consumer(const LoopArgs& a, const Shared& sh, const Sched& sc) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const bool cta0 = blockIdx.x == 0;
  const int nb = a.nb;
  const int K = a.K;
  const int kmine = sc.p.k1 - sc.p.k0;
  const int umine = sc.p.j1 - sc.p.j0;
  const int vrows = sc.p.v1 - sc.p.v0;
  uint32_t nbar = 0;

  // ---- prologue: argmax keys, biases, precomputed W1_h h terms, S = 0, first GRU input
  if (cta0)
    for (int q = tid; q < K * NB; q += CONS_THREADS) a.best[q] = 0ull;
  for (int q = tid; q < umine * 6; q += CONS_THREADS) {
    const int jl = q / 6, g = q % 6;
    const float* bsrc = g < 3 ? a.b_ih : a.b_hh;
    sh.bias[q] = bsrc ? bsrc[(g % 3) * a.H + sc.p.j0 + jl] : 0.f;
  }
  for (int q = tid; q < kmine * nb * K; q += CONS_THREADS) {
    const int kl = q / (nb * K), rem = q % (nb * K), b = rem / K, p = rem % K;
    sh.hp[(kl * NB + b) * K + p] = a.hp[(static_cast<size_t>(b) * K + p) * a.r + sc.p.k0 + kl];
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
  gather_rows<W>(a, sh, NB);
  named_barrier(BAR_CONS, CONS_THREADS);

  int n_base = 0;  // global item index of the first item of the current phase

  for (int i = 0; i < K; ++i) {
    // base-logit slice of this step -> shared memory, overlapped with the GRU
    if (!aborted(sh)) {
      for (int q = tid; q < nb * vrows; q += CONS_THREADS) {
        const int b = q / vrows, v = q % vrows;
        cp_async4(sh.base + b * a.vmax + v, a.base + (static_cast<size_t>(b) * K + i) * a.V + sc.p.v0 + v);
      }
    }
    cp_async_commit();

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
      for (int q = tid; q < umine * NB; q += CONS_THREADS) {
        const int jl = q / NB, b = q % NB;
        const int j = sc.p.j0 + jl;
        float gi[3], gh[3];
        for (int g = 0; g < 3; ++g) {
          gi[g] = sh.bias[jl * 6 + g];
          gh[g] = sh.bias[jl * 6 + 3 + g];
        }
        for (int s = 0; s < sc.e3.n; ++s)
          for (int g = 0; g < 3; ++g) gi[g] += sh.part[(jl * per_unit + s) * 32 + g * NB + b];
        for (int s = 0; s < sc.h3.n; ++s)
          for (int g = 0; g < 3; ++g) gh[g] += sh.part[(jl * per_unit + sc.e3.n + s) * 32 + g * NB + b];
        const float r = 1.f / (1.f + expf(-(gi[0] + gh[0])));
        const float z = 1.f / (1.f + expf(-(gi[1] + gh[1])));
        const float nn = tanhf(gi[2] + r * gh[2]);
        const float s_old = sh.S[b * a.H + j];
        S_new[b * a.H + j] = (1.f - z) * nn + z * s_old;
      }
    }
    consumer_grid_sync(a, sh, nbar++);  // ---- barrier 1: S_i complete

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
    consumer_grid_sync(a, sh, nbar++);  // ---- barrier 2: u complete

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
    cp_async_wait_all();
    named_barrier(BAR_CONS, CONS_THREADS);

    // ================= phase C: W2 chunks, residual, pick
    constexpr int RPI = 32 / NB;           // rows per reduce-scatter round
    const int my_b = lane % NB;            // request whose sums this lane ends up with
    float best_s = -INFINITY;
    int best_v = 0x7FFFFFFF;
    const bool greedy = a.mode == 0;
    for (int q = 0; q < sc.nC; ++q) {
      const int n = n_base + q;
      if (n % NCW != warp) continue;
      const int vl0 = q * VCHUNK;          // chunk start, relative to v0
      const int rows = min(VCHUNK, vrows - vl0);
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
            const int v = sc.p.v0 + vl0 + rl;
            const float L = sh.base[my_b * a.vmax + vl0 + rl] + dl;
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
    consumer_grid_sync(a, sh, nbar++);  // ---- barrier 3: picks merged

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
    if (i + 1 < K && !aborted(sh)) gather_rows<W>(a, sh, nb);
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

template <typename W, int NB>
__global__ void __launch_bounds__(NTHREADS, 1) correct_loop_kernel(const LoopArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int G = gridDim.x;
  if (a.selftest) {
    // one barrier episode that can never complete: exercises the bounded wait
    if (threadIdx.x == 0) {
      grid_barrier_one_thread(a.ctl, static_cast<uint32_t>(G) + 1u, a.budget_ns);
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
    const int n = (p.j1 - p.j0) * (a.nsegE3 + a.nsegH3) + (p.k1 - p.k0) * a.nsegH1 + (p.v1 - p.v0 + VCHUNK - 1) / VCHUNK;
    items_max = items_max > n ? items_max : n;
  }
  a.vmax = (vmax + 3) / 4 * 4;
  struct Piece { uint32_t* off; size_t bytes; size_t align; };
  const Piece pieces[] = {
      {&a.off_S, static_cast<size_t>(NB) * a.H * 4, 16},
      {&a.off_x, static_cast<size_t>(NB) * a.E * wb, 16},
      {&a.off_base, static_cast<size_t>(NB) * a.vmax * 4, 16},
      {&a.off_part, static_cast<size_t>(a.max_part) * 32 * 4, 16},
      {&a.off_hp, static_cast<size_t>(kmax) * NB * a.K * 4, 16},
      {&a.off_bias, static_cast<size_t>(umax) * 6 * 4, 16},
      {&a.off_tok, static_cast<size_t>(NB) * a.K * 4, 16},
      {&a.off_wbest, static_cast<size_t>(NCW) * NB * 8, 8},
      {&a.off_flags, 64, 16},
      {&a.off_items, static_cast<size_t>(items_max) * sizeof(Item), 16},
  };
  size_t fixed = 2 * 8 * 16 + 16;  // barriers of up to 16 slots
  for (const Piece& p : pieces) fixed = (fixed + p.align - 1) / p.align * p.align + p.bytes;
  fixed += 1024;
  if (fixed >= smem_cap) return 0;
  int nslot = static_cast<int>((smem_cap - fixed) / kLoopSlotBytes) / NCW * NCW;
  if (nslot > 16) nslot = 16;
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

int loop_threads() { return NTHREADS; }

}  // namespace domino
