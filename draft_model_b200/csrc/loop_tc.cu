// Stage 2 for larger batches on the tcgen05 tensor cores (sm_100a).
//
// Same method as correct_loop.cu (Domino study notes, gsyq.cn, §二.1(2);
// yhxrc.cn article, §四), but with B requests the per-step products are dense
// contractions, so each step runs as a short chain of launches over the batch:
//   1. gate GEMMs     gi = W_ih X   and   gh = W_hh S       (tcgen05, split-K partials)
//                     X = embeddings of the fed tokens (bf16, exact); S is kept as
//                     bf16 hi + lo halves along K (each half padded to a whole
//                     number of 64-wide k-blocks), so W_hh S keeps ~16 bits
//   2. GRU            S' = GRU(sum of gi partials + b_ih, sum of gh partials + b_hh, S)
//   3. bottleneck     W1_s S' on the tensor cores (same hi / lo operand, split-K)
//   4. SiLU           u = SiLU(P + W1_s S') with P = W1_h h_i from stage 1, stored as
//                     interleaved bf16 hi / lo rows so W2 u keeps ~16 bits
//   5. W2 GEMM        L = L_base + W2 u fused with the pick (greedy or Gumbel): the
//                     epilogue streams L_base through a per-thread cp.async ring,
//                     keeps each thread's best (score, tile) per request in
//                     registers across its tiles, and reduces lanes, warps and
//                     CTAs once at the end (redux.sync, then 64-bit atomicMax)
//   6. pick           t_i, draft_out, the next fed token and its embedding row
// Every accumulation is fp32; results are deterministic (split-K partials are
// summed in a fixed order; the argmax merge is order-free).
#include <cstdint>
#include <cstring>
#include <utility>

#include "common.cuh"
#include "domino_internal.h"
#include "tc_common.cuh"

namespace domino {
namespace {

using namespace tc;
constexpr int EPI_WARPS = 16;                // four warps per TMEM lane quarter
constexpr int NTH = 64 + 32 * EPI_WARPS;     // producer, MMA issuer, epilogue
constexpr int MAXREQ_TILE = kLoopTcReqPerLaunch;   // requests per W2 tile (2 columns each)
constexpr int MAX_ACC = 8;                   // TMEM accumulator buffers (as many as fit in 512 columns)
constexpr int NSLOT = 4;                     // L_base staging ring depth (items of 8 requests)
constexpr uint32_t SLOT_BYTES = EPI_WARPS * 8 * 32 * 4;   // 16 KB: [warp][request][lane] fp32
constexpr int MAX_MY_GROUPS = 4;             // 16-column groups one epilogue warp owns per tile

// Epilogue variants: split-K partial output, or the W2 product fused with the
// residual and the pick (greedy or Gumbel-max; optionally storing L_i).
enum Epi : int { EPI_PARTIAL = 0, EPI_GREEDY = 1, EPI_GREEDY_LOGITS = 2, EPI_GUMBEL = 3, EPI_GUMBEL_LOGITS = 4 };

// One GEMM D[m][v] = sum_k A[v][k] B[m][k] (A: nrows x K, B: M x K; both bf16, K-major).
struct Prob {
  int nrows, M;
  int num_vt, num_mt, num_kb, splits;
  int a_kwrap;            // A's k coordinate is taken modulo a_kwrap (0: none)
  float* out;             // EPI_PARTIAL: out[split * split_stride + m * nrows + v]
  size_t split_stride;
};

struct GArgs {
  Prob p[2];
  int nprob;
  int units0, units;      // work units (tile, split) of problem 0 and in total
  int BN, stages, nacc, tmem_cols;
  Control* ctl;
  uint64_t budget_ns;
  // W2 epilogues: 2 columns (u hi, u lo) per request
  const float* base;      // [B, K, V], offset to the chunk's first request
  float* logits;          // [B, K, V], offset likewise (logits variants)
  unsigned long long* best;  // [chunk requests] keys of this step
  int K, step, V, nreq;   // nreq: requests of this chunk (<= MAXREQ_TILE, one m-tile)
  int req0;               // global index of the chunk's first request (Philox counter)
  float temperature;
  uint64_t seed;
};

__device__ __forceinline__ void unit_decode(const GArgs& a, int u, int& pi, int& vt, int& mt, int& kb0, int& kb1,
                                            int& split) {
  pi = u < a.units0 ? 0 : 1;
  const int uu = pi == 0 ? u : u - a.units0;
  const Prob& p = a.p[pi];
  split = uu % p.splits;
  const int tile = uu / p.splits;
  vt = tile / p.num_mt;
  mt = tile % p.num_mt;
  kb0 = static_cast<int>(static_cast<long long>(p.num_kb) * split / p.splits);
  kb1 = static_cast<int>(static_cast<long long>(p.num_kb) * (split + 1) / p.splits);
}

// Which (tile, 16-column group) items an epilogue warp owns.  The four warps of
// a lane quarter (slot qs) split a tile's G groups as j = qs, qs+4, ... when
// G >= 4; with fewer groups they take different tiles instead (the CTA's k-th
// tile goes to the slots with k % TS == qs / G), so the epilogue of several
// tiles runs at once.  Either way a warp's groups are the same in every tile.
struct EpiPlan {
  int TS, k0, ngroups, j0, jstep;
  __device__ EpiPlan(int G, int qs) {
    if (G >= 4) {
      TS = 1; k0 = 0; j0 = qs; jstep = 4;
      ngroups = G > qs ? (G - qs + 3) >> 2 : 0;
    } else {
      TS = 4 / G; k0 = qs / G; j0 = qs % G; jstep = 4;
      ngroups = (qs < G * TS) ? 1 : 0;
    }
  }
  __device__ bool owns(int k) const { return ngroups > 0 && (k % TS) == k0; }
};

template <int EPI>
__global__ void __launch_bounds__(NTH, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1, const GArgs a) {
  constexpr bool PICK = EPI != EPI_PARTIAL;
  constexpr bool GUMBEL = EPI == EPI_GUMBEL || EPI == EPI_GUMBEL_LOGITS;
  constexpr bool LOGITS = EPI == EPI_GREEDY_LOGITS || EPI == EPI_GUMBEL_LOGITS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t b_bytes = static_cast<uint32_t>(a.BN) * BK * 2;
  const uint32_t stage_bytes = A_STAGE_BYTES + b_bytes;
  float* ring = reinterpret_cast<float*>(smem + static_cast<size_t>(a.stages) * stage_bytes);
  uint8_t* ctrl = reinterpret_cast<uint8_t*>(ring) + (PICK ? NSLOT * SLOT_BYTES : 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + a.stages;
  uint64_t* tfull = empty + a.stages;   // [nacc]
  uint64_t* tempty = tfull + MAX_ACC;   // [nacc]
  uint64_t* mma_done = tempty + MAX_ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  unsigned long long* sbest = reinterpret_cast<unsigned long long*>(tmem_slot + 4);  // [MAXREQ_TILE] (8-byte aligned)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < a.nacc; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA0);
    prefetch_tmap(&tmB0);
    if (a.nprob > 1) {
      prefetch_tmap(&tmA1);
      prefetch_tmap(&tmB1);
    }
  }
  if (PICK)
    for (int q = threadIdx.x; q < MAXREQ_TILE; q += NTH) sbest[q] = 0ull;
  if (warp == 1) tmem_alloc(tmem_slot, a.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the setup above overlaps the previous kernel of the step chain; every global
  // access below comes after it has completed
  griddep_launch_dependents();
  griddep_wait();

  auto bounded_wait = [&](uint64_t* bar, uint32_t par) -> bool {
    if (mbar_try_wait(bar, par)) return true;   // fast path: no timer read
    if (*abort_flag) return false;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, par)) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > a.budget_ns) {
        raise_error(a.ctl, ERRBIT_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
    return true;
  };

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int it = 0, s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < a.units && ok; u += gridDim.x) {
        int pi, vt, mt, kb0, kb1, split;
        unit_decode(a, u, pi, vt, mt, kb0, kb1, split);
        const CUtensorMap* tA = pi == 0 ? &tmA0 : &tmA1;
        const CUtensorMap* tB = pi == 0 ? &tmB0 : &tmB1;
        const int wrap = a.p[pi].a_kwrap;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          if (it >= a.stages && !bounded_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
          uint8_t* sa = smem + static_cast<size_t>(s) * stage_bytes;
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          const int kc = kb * BK;
          tma_load_2d(sa, tA, wrap ? kc % wrap : kc, vt * BM, &full[s]);
          tma_load_2d(sa + A_STAGE_BYTES, tB, kc, mt * a.BN, &full[s]);
          if (++s == a.stages) { s = 0; ph ^= 1u; }
        }
      }
      for (int j = max(0, it - a.stages); j < it; ++j) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[j % a.stages], (j / a.stages) & 1)) {
          if (globaltimer_ns() - t0 > a.budget_ns) { raise_error(a.ctl, ERRBIT_TIMEOUT); break; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(a.BN);
      int it = 0, local = 0, s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < a.units && ok; u += gridDim.x, ++local) {
        int pi, vt, mt, kb0, kb1, split;
        unit_decode(a, u, pi, vt, mt, kb0, kb1, split);
        const int acc = local % a.nacc;
        if (local >= a.nacc && !bounded_wait(&tempty[acc], ((local / a.nacc) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.BN);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          if (!bounded_wait(&full[s], ph)) { ok = false; break; }
          tc_fence_after();
          // descriptors advance by (bytes >> 4) in their start-address field
          const uint64_t da = smem_desc_sw128(smem_u32(smem + static_cast<size_t>(s) * stage_bytes));
          const uint64_t db = da + (A_STAGE_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_bf16(d_tmem, da + ((kk * 32) >> 4), db + ((kk * 32) >> 4), idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
          if (++s == a.stages) { s = 0; ph ^= 1u; }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      tc_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(mma_done, 0)) {
        if (globaltimer_ns() - t0 > a.budget_ns) { raise_error(a.ctl, ERRBIT_TIMEOUT); break; }
      }
    }
  } else {
    // ---------------- epilogue: warps 2..17; TMEM lane quarter = warp % 4
    const int ew = warp - 2;
    const int q = warp & 3;
    const int qs = ew >> 2;
    const int row = q * 32 + lane;
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const EpiPlan plan(a.BN >> 4, qs);
    if (!PICK) {
      int k = 0;
      for (int u = blockIdx.x; u < a.units; u += gridDim.x, ++k) {
        const int acc = k % a.nacc;
        if (lane == 0) bounded_wait(&tfull[acc], (k / a.nacc) & 1);
        __syncwarp();
        if (*abort_flag) break;
        tc_fence_after();
        if (plan.owns(k)) {
          int pi, vt, mt, kb0, kb1, split;
          unit_decode(a, u, pi, vt, mt, kb0, kb1, split);
          const Prob& p = a.p[pi];
          const int v = vt * BM + row;
          float* dst = p.out + static_cast<size_t>(split) * p.split_stride;
          for (int g = 0; g < plan.ngroups; ++g) {
            const int c0 = (plan.j0 + plan.jstep * g) * 16;
            float vals[16];
            tmem_ld16(tlane + static_cast<uint32_t>(acc * a.BN + c0), vals);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int m = mt * a.BN + c0 + c;
              if (v < p.nrows && m < p.M) dst[static_cast<size_t>(m) * p.nrows + v] = vals[c];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      }
    } else {
      // Each thread owns one vocabulary row per tile and keeps, for every request
      // of its groups, the best (score, tile) seen so far in registers: a later
      // tile has larger indices, so a strict > keeps the lowest index on ties.
      // The 32 rows of a warp are reduced once, after the last tile.
      // (tile indices are kept as 16-bit halves, two per register)
      uint32_t bkey[MAX_MY_GROUPS * 8], btile[MAX_MY_GROUPS * 4];
#pragma unroll
      for (int x = 0; x < MAX_MY_GROUPS * 8; ++x) bkey[x] = 0u;
#pragma unroll
      for (int x = 0; x < MAX_MY_GROUPS * 4; ++x) btile[x] = 0u;
      // L_base values reach shared memory through a per-thread cp.async ring:
      // the item NSLOT - 1 ahead (in this warp's own item order, across tiles)
      // is requested before the current one is consumed.
      float* my_ring = ring + ew * 8 * 32 + lane;    // + slot * (SLOT_BYTES / 4) + c * 32
      const size_t req_stride = static_cast<size_t>(a.K) * a.V;
      int ik = plan.k0, ig = 0, issued = 0;
      const int nlocal = a.units > static_cast<int>(blockIdx.x)
                             ? (a.units - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x)
                             : 0;
      auto issue = [&]() {
        if (plan.ngroups > 0 && ik < nlocal) {
          const int j = plan.j0 + plan.jstep * ig;
          const int v = (static_cast<int>(blockIdx.x) + ik * static_cast<int>(gridDim.x)) * BM + row;
          float* dst = my_ring + (issued % NSLOT) * (SLOT_BYTES / 4);
          if (v < a.V) {
            const float* src = a.base + static_cast<size_t>(a.step) * a.V + v + static_cast<size_t>(8 * j) * req_stride;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              if (8 * j + c < a.nreq) cp_async4(dst + c * 32, src + c * req_stride);
          }
          if (++ig == plan.ngroups) { ig = 0; ik += plan.TS; }
        }
        cp_async_commit();
        ++issued;
      };
#pragma unroll 1
      for (int p = 0; p < NSLOT - 1; ++p) issue();
      int n = 0;
      for (int k = 0; k < nlocal; ++k) {
        const int acc = k % a.nacc;
        if (lane == 0) bounded_wait(&tfull[acc], (k / a.nacc) & 1);
        __syncwarp();
        if (*abort_flag) break;
        tc_fence_after();
        if (plan.owns(k)) {
          const int vt = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);   // unit == vocabulary tile
          const int v = vt * BM + row;
          const bool vok = v < a.V;
#pragma unroll
          for (int g = 0; g < MAX_MY_GROUPS; ++g) {
            if (g < plan.ngroups) {
              issue();
              cp_async_wait_group<NSLOT - 1>();
              const int j = plan.j0 + plan.jstep * g;
              float vals[16];
              tmem_ld16(tlane + static_cast<uint32_t>(acc * a.BN + 16 * j), vals);
              const float* src = my_ring + (n % NSLOT) * (SLOT_BYTES / 4);
              ++n;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const int bl = 8 * j + c;   // request within the chunk
                const bool ok = vok && bl < a.nreq;
                const float L = vals[2 * c] + vals[2 * c + 1] + src[c * 32];
                if (LOGITS && ok) __stcs(a.logits + static_cast<size_t>(bl) * req_stride + static_cast<size_t>(a.step) * a.V + v, L);
                float score = L;
                if (GUMBEL && ok) score = __fdiv_rn(L, a.temperature) + gumbel_noise(a.seed, a.req0 + bl, a.step, v);
                const uint32_t okey = ok ? orderable_u32(score) : 0u;
                if (okey > bkey[g * 8 + c]) {
                  bkey[g * 8 + c] = okey;
                  uint32_t& bt = btile[g * 4 + (c >> 1)];
                  bt = (c & 1) ? ((bt & 0x0000FFFFu) | (static_cast<uint32_t>(vt) << 16))
                               : ((bt & 0xFFFF0000u) | static_cast<uint32_t>(vt));
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      }
      cp_async_wait_all();
      // lanes -> one key per request and warp -> CTA keys in shared memory
      if (!*abort_flag) {
#pragma unroll
        for (int g = 0; g < MAX_MY_GROUPS; ++g) {
          if (g < plan.ngroups) {
            const int j = plan.j0 + plan.jstep * g;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int bl = 8 * j + c;
              const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, bkey[g * 8 + c]);
              const uint32_t tile = (c & 1) ? (btile[g * 4 + (c >> 1)] >> 16) : (btile[g * 4 + (c >> 1)] & 0xFFFFu);
              const uint32_t cand = (m != 0u && bkey[g * 8 + c] == m) ? tile * BM + row : 0xFFFFFFFFu;
              const uint32_t vbest = __reduce_min_sync(0xFFFFFFFFu, cand);
              if (lane == 0 && m != 0u && bl < a.nreq)
                atomicMax(&sbest[bl], (static_cast<unsigned long long>(m) << 32) | (0xFFFFFFFFull - vbest));
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, a.tmem_cols);
  // one W2 launch covers one m-tile (<= MAXREQ_TILE requests): a CTA's keys per
  // request merge into the step's keys with one atomicMax each
  if (PICK && !*abort_flag)
    for (int bl = threadIdx.x; bl < a.nreq; bl += NTH)
      if (sbest[bl]) atomicMax(&a.best[bl], sbest[bl]);
}

// ---------------------------------------------------------------- SIMT kernels of a step

// GRU for every (request, unit): sums the split-K partials, applies the gates,
// keeps S (fp32) and writes its bf16 hi / lo halves (row stride 2*Hp) for the
// next tensor-core products.
// With a token->gate table, gi is the fed token's table row (b_ih included)
// instead of the W_ih X partials.
__global__ void __launch_bounds__(256) gru_step_kernel(const float* __restrict__ gi_part, int gi_splits,
                                                       const float* __restrict__ gh_part, int gh_splits,
                                                       const float* __restrict__ b_ih, const float* __restrict__ b_hh,
                                                       const float* __restrict__ table,
                                                       const int32_t* __restrict__ fed, float* __restrict__ S,
                                                       __nv_bfloat16* __restrict__ S2, int B, int H, int Hp) {
  griddep_launch_dependents();
  griddep_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * H) return;
  const int b = idx / H, j = idx % H;
  const size_t G3 = static_cast<size_t>(3) * H;
  const size_t gstride = static_cast<size_t>(B) * G3;
  float gi[3], gh[3];
#pragma unroll
  for (int g = 0; g < 3; ++g) {
    const size_t at = static_cast<size_t>(b) * G3 + static_cast<size_t>(g) * H + j;
    float si, sh = b_hh ? b_hh[g * H + j] : 0.f;
    if (table) {
      si = table[static_cast<size_t>(fed[b]) * G3 + static_cast<size_t>(g) * H + j];
    } else {
      si = b_ih ? b_ih[g * H + j] : 0.f;
#pragma unroll 4
      for (int s = 0; s < gi_splits; ++s) si += gi_part[s * gstride + at];
    }
#pragma unroll 4
    for (int s = 0; s < gh_splits; ++s) sh += gh_part[s * gstride + at];
    gi[g] = si;
    gh[g] = sh;
  }
  const float r = __fdividef(1.f, 1.f + __expf(-(gi[0] + gh[0])));
  const float z = __fdividef(1.f, 1.f + __expf(-(gi[1] + gh[1])));
  const float n = fmaf(2.f, __fdividef(1.f, 1.f + __expf(-2.f * (gi[2] + r * gh[2]))), -1.f);
  const float s_old = S[idx];
  const float s_new = (1.f - z) * n + z * s_old;
  S[idx] = s_new;
  const __nv_bfloat16 hi = __float2bfloat16_rn(s_new);
  S2[static_cast<size_t>(b) * 2 * Hp + j] = hi;
  S2[static_cast<size_t>(b) * 2 * Hp + Hp + j] = __float2bfloat16_rn(s_new - __bfloat162float(hi));
}

// u = SiLU(P + W1_s S') from the bottleneck GEMM's split-K partials and stage
// 1's P = W1_h h_i; written as interleaved bf16 rows U2[2b] = hi(u_b),
// U2[2b+1] = lo(u_b) for the W2 product.
__global__ void __launch_bounds__(256) silu_split_kernel(const float* __restrict__ upart, int splits,
                                                         const float* __restrict__ hp, int K, int step, int B, int r,
                                                         __nv_bfloat16* __restrict__ U2) {
  griddep_launch_dependents();
  griddep_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= B * r) return;
  const int b = idx / r, k = idx % r;
  float pre = hp[(static_cast<size_t>(b) * K + step) * r + k];
  const size_t sstride = static_cast<size_t>(B) * r;
#pragma unroll 4
  for (int s = 0; s < splits; ++s) pre += upart[s * sstride + idx];
  const float u = pre * __fdividef(1.f, 1.f + __expf(-pre));
  const __nv_bfloat16 hi = __float2bfloat16_rn(u);
  U2[static_cast<size_t>(2 * b) * r + k] = hi;
  U2[static_cast<size_t>(2 * b + 1) * r + k] = __float2bfloat16_rn(u - __bfloat162float(hi));
}

// Picks of this step, the next fed tokens and their embedding rows;
// verification after the last step.
__global__ void __launch_bounds__(256) pick_step_kernel(unsigned long long* best, int step, int K, int B, int V, int E,
                                                        const int32_t* __restrict__ anchor,
                                                        const int32_t* __restrict__ forced,
                                                        const int32_t* __restrict__ target, int32_t* draft,
                                                        int32_t* tau, const __nv_bfloat16* __restrict__ embed,
                                                        __nv_bfloat16* X, int32_t* fed_out, Control* ctl) {
  // one block per request: thread 0 decides the token, all threads copy the row
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.x;
  __shared__ int fed;
  if (threadIdx.x == 0) {
    int f;
    if (step < 0) {
      f = anchor[b];
    } else {
      const unsigned long long key = best[static_cast<size_t>(step) * B + b];
      const int t = static_cast<int>(argmax_key_index(key));
      draft[static_cast<size_t>(b) * K + step] = t;
      f = forced ? forced[static_cast<size_t>(b) * K + step] : t;
      if (step == K - 1 && target && tau) {
        int n = 0;
        while (n < K && draft[static_cast<size_t>(b) * K + n] == target[static_cast<size_t>(b) * K + n]) ++n;
        tau[b] = n;
      }
    }
    if (f < 0 || f >= V) {
      raise_error(ctl, ERRBIT_BAD_TOKEN);
      f = min(max(f, 0), V - 1);
    }
    fed = f;
    fed_out[b] = f;
  }
  __syncthreads();
  if (step + 1 >= K || X == nullptr) return;   // no embedding rows with a token->gate table
  const uint4* src = reinterpret_cast<const uint4*>(embed + static_cast<size_t>(fed) * E);
  uint4* dst = reinterpret_cast<uint4*>(X + static_cast<size_t>(b) * E);
  for (int q = threadIdx.x; q < E / 8; q += blockDim.x) dst[q] = __ldg(src + q);
}

// Pipeline depth, TMEM accumulator buffers and dynamic shared memory of one
// gemm_tc_kernel launch with BN columns per tile.
size_t gemm_plan(GArgs& g, bool pick) {
  const size_t stage_bytes = A_STAGE_BYTES + static_cast<size_t>(g.BN) * BK * 2;
  const size_t ring = pick ? static_cast<size_t>(NSLOT) * SLOT_BYTES : 0;
  g.stages = static_cast<int>((218 * 1024 - ring) / stage_bytes);
  if (g.stages > 8) g.stages = 8;
  g.nacc = 2;
  while (g.nacc < MAX_ACC && 2 * g.nacc * g.BN <= 512) g.nacc *= 2;
  g.tmem_cols = 32;
  while (g.tmem_cols < g.nacc * g.BN) g.tmem_cols <<= 1;
  return static_cast<size_t>(g.stages) * stage_bytes + ring + 1024 /*align*/ + 2048 /*barriers, keys*/;
}

using GemmKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, const GArgs);
GemmKernel gemm_kernel(int epi) {
  switch (epi) {
    case EPI_GREEDY: return gemm_tc_kernel<EPI_GREEDY>;
    case EPI_GREEDY_LOGITS: return gemm_tc_kernel<EPI_GREEDY_LOGITS>;
    case EPI_GUMBEL: return gemm_tc_kernel<EPI_GUMBEL>;
    case EPI_GUMBEL_LOGITS: return gemm_tc_kernel<EPI_GUMBEL_LOGITS>;
    default: return gemm_tc_kernel<EPI_PARTIAL>;
  }
}

// Launch with programmatic stream serialization: the kernel may start while the
// previous one finishes; it calls griddep_wait() before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Split count that brings a problem of `tiles` output tiles near one unit per SM.
int splits_for(int num_sms, int tiles, int num_kb) {
  const int cap = kLoopTcMaxSplits < num_kb ? kLoopTcMaxSplits : num_kb;
  return clampi(num_sms / (tiles > 0 ? tiles : 1), 1, cap);
}

// table[t, c] += bias[c] over a [rows, cols] fp32 table
__global__ void add_row_bias_kernel(float* __restrict__ table, const float* __restrict__ bias, size_t rows, int cols) {
  const size_t n = rows * static_cast<size_t>(cols);
  for (size_t q = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<size_t>(gridDim.x) * blockDim.x)
    table[q] += bias[q % cols];
}

}  // namespace

cudaError_t launch_add_row_bias(float* table, const float* bias, size_t rows, int cols, int num_sms,
                                cudaStream_t stream) {
  add_row_bias_kernel<<<num_sms * 4, 256, 0, stream>>>(table, bias, rows, cols);
  return cudaGetLastError();
}

bool loop_tc_supported(int E, int H, int d, int r, int V) {
  // every tensor map row stride and the W1 state-column base must be 16-byte
  // aligned; vocabulary tile indices must fit the epilogue's 16-bit fields
  return E % 8 == 0 && H % 8 == 0 && d % 8 == 0 && r % 8 == 0 && (V + BM - 1) / BM <= 65535;
}

cudaError_t run_loop_tc(const LoopTcArgs& L, cudaStream_t st) {
  const int B = L.B, K = L.K, E = L.E, H = L.H, r = L.r, V = L.V;
  const int G3 = 3 * H;
  const int Hp = loop_tc_padded_h(H);
  if (!loop_tc_supported(E, H, L.d, r, V)) return cudaErrorInvalidValue;
  cudaError_t e;
  // ---- tensor maps (fixed for the whole block)
  const int bn_gate = ((B + 15) / 16 * 16) > 256 ? 256 : (B + 15) / 16 * 16;
  const __nv_bfloat16* w1s = static_cast<const __nv_bfloat16*>(L.w1) + L.d;   // state columns of W1
  CUtensorMap tWih, tX, tWhh, tS2, tW1s, tW2;
  if (!make_tmap(&tWih, L.w_ih, G3, E, BM, E) || !make_tmap(&tX, L.X, B, E, bn_gate, E) ||
      !make_tmap(&tWhh, L.w_hh, G3, H, BM, H) || !make_tmap(&tS2, L.S2, B, 2 * Hp, bn_gate, 2 * Hp) ||
      !make_tmap(&tW1s, w1s, r, H, BM, L.d + H) || !make_tmap(&tW2, L.w2, V, r, BM, r))
    return cudaErrorInvalidValue;

  const int epi_w2 = (L.mode == 1 ? EPI_GUMBEL : EPI_GREEDY) + (L.logits ? 1 : 0);
  for (const int epi : {static_cast<int>(EPI_PARTIAL), epi_w2}) {
    e = cudaFuncSetAttribute(gemm_kernel(epi), cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
  }

  // ---- gate GEMMs: both problems split along K to about one unit per SM
  const int num_mt = (B + bn_gate - 1) / bn_gate;
  GArgs g;
  std::memset(&g, 0, sizeof(g));
  g.ctl = L.ctl;
  g.budget_ns = L.budget_ns;
  g.BN = bn_gate;
  const size_t gsm = gemm_plan(g, false);
  const int vt = (G3 + BM - 1) / BM;
  const int kb0 = (E + BK - 1) / BK, kb1 = 2 * Hp / BK;
  const int s0 = clampi(L.num_sms * kb0 / ((kb0 + kb1) * vt * num_mt), 1, kLoopTcMaxSplits < kb0 ? kLoopTcMaxSplits : kb0);
  const int s1 = clampi(L.num_sms * kb1 / ((kb0 + kb1) * vt * num_mt), 1, kLoopTcMaxSplits < kb1 ? kLoopTcMaxSplits : kb1);
  Prob& p0 = g.p[0];
  p0.nrows = G3; p0.M = B; p0.num_vt = vt; p0.num_mt = num_mt; p0.num_kb = kb0; p0.splits = s0; p0.a_kwrap = 0;
  p0.out = L.gi_part; p0.split_stride = static_cast<size_t>(B) * G3;
  Prob& p1 = g.p[1];
  p1.nrows = G3; p1.M = B; p1.num_vt = vt; p1.num_mt = num_mt; p1.num_kb = kb1; p1.splits = s1; p1.a_kwrap = Hp;
  p1.out = L.gh_part; p1.split_stride = static_cast<size_t>(B) * G3;
  // W_hh S alone (token->gate table): split to about one unit per SM
  GArgs gh = g;
  gh.nprob = 1;
  gh.p[0] = p1;
  const int sh1 = splits_for(L.num_sms, vt * num_mt, kb1);
  gh.p[0].splits = sh1;
  gh.units0 = gh.units = vt * num_mt * sh1;

  // ---- bottleneck GEMM: W1_s (r x H) against S' hi | lo
  GArgs bk = g;
  bk.nprob = 1;
  Prob& pb = bk.p[0];
  const int vtb = (r + BM - 1) / BM;
  pb.nrows = r; pb.M = B; pb.num_vt = vtb; pb.num_mt = num_mt; pb.num_kb = kb1;
  pb.splits = splits_for(L.num_sms, vtb * num_mt, kb1); pb.a_kwrap = Hp;
  pb.out = L.u_part; pb.split_stride = static_cast<size_t>(B) * r;
  bk.units0 = bk.units = vtb * num_mt * pb.splits;
  const int gridb = bk.units < L.num_sms ? bk.units : L.num_sms;

  // ---- initial state: S = 0 (with the pad columns of S2), keys = 0, X = anchor embeddings
  if ((e = cudaMemsetAsync(L.S, 0, static_cast<size_t>(B) * H * 4, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(L.S2, 0, static_cast<size_t>(B) * 2 * Hp * 2, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(L.best, 0, static_cast<size_t>(K) * B * 8, st)) != cudaSuccess) return e;
  __nv_bfloat16* Xg = L.gate_table ? nullptr : L.X;   // fed embeddings only when W_ih multiplies them
  e = launch_pdl(pick_step_kernel, dim3(B), dim3(256), 0, st, L.best, -1, K, B, V, E, L.anchor, L.forced, L.target,
                 L.draft, L.tau, static_cast<const __nv_bfloat16*>(L.embed), Xg, L.fed, L.ctl);
  if (e != cudaSuccess) return e;

  for (int i = 0; i < K; ++i) {
    // 1. gate GEMMs (W_hh S is zero at the first position: S = 0); with a
    //    token->gate table only W_hh S is multiplied
    if (!L.gate_table) {
      g.nprob = i == 0 ? 1 : 2;
      g.units0 = vt * num_mt * s0;
      g.units = g.units0 + (i == 0 ? 0 : vt * num_mt * s1);
      const int grid0 = g.units < L.num_sms ? g.units : L.num_sms;
      e = launch_pdl(gemm_tc_kernel<EPI_PARTIAL>, dim3(grid0), dim3(NTH), gsm, st, tWih, tX, tWhh, tS2, g);
      if (e != cudaSuccess) return e;
    } else if (i > 0) {
      const int gridh = gh.units < L.num_sms ? gh.units : L.num_sms;
      e = launch_pdl(gemm_tc_kernel<EPI_PARTIAL>, dim3(gridh), dim3(NTH), gsm, st, tWhh, tS2, tWhh, tS2, gh);
      if (e != cudaSuccess) return e;
    }
    // 2. GRU
    e = launch_pdl(gru_step_kernel, dim3((B * H + 255) / 256), dim3(256), 0, st, L.gi_part, s0, L.gh_part,
                   i == 0 ? 0 : (L.gate_table ? sh1 : s1), L.b_ih, L.b_hh, L.gate_table,
                   static_cast<const int32_t*>(L.fed), L.S, L.S2, B, H, Hp);
    if (e != cudaSuccess) return e;
    // 3. bottleneck product, 4. SiLU and the hi / lo split of u
    e = launch_pdl(gemm_tc_kernel<EPI_PARTIAL>, dim3(gridb), dim3(NTH), gsm, st, tW1s, tS2, tW1s, tS2, bk);
    if (e != cudaSuccess) return e;
    e = launch_pdl(silu_split_kernel, dim3((B * r + 255) / 256), dim3(256), 0, st, L.u_part, pb.splits, L.hp, K, i, B,
                   r, L.U2);
    if (e != cudaSuccess) return e;
    // 5. W2 GEMM + residual + pick, per chunk of requests
    for (int c0 = 0; c0 < B; c0 += MAXREQ_TILE) {
      const int nreq = B - c0 < MAXREQ_TILE ? B - c0 : MAXREQ_TILE;
      const int bn = (2 * nreq + 15) / 16 * 16;
      CUtensorMap tU;
      if (!make_tmap(&tU, L.U2 + static_cast<size_t>(2 * c0) * r, 2 * nreq, r, bn, r)) return cudaErrorInvalidValue;
      GArgs w;
      std::memset(&w, 0, sizeof(w));
      w.ctl = L.ctl;
      w.budget_ns = L.budget_ns;
      w.BN = bn;
      const size_t wsm = gemm_plan(w, true);
      Prob& q = w.p[0];
      q.nrows = V; q.M = 2 * nreq; q.num_vt = (V + BM - 1) / BM; q.num_mt = 1; q.num_kb = (r + BK - 1) / BK;
      q.splits = 1;
      w.nprob = 1;
      w.units0 = w.units = q.num_vt;
      w.base = L.base + static_cast<size_t>(c0) * K * V;
      w.logits = L.logits ? L.logits + static_cast<size_t>(c0) * K * V : nullptr;
      w.best = L.best + static_cast<size_t>(i) * B + c0;
      w.K = K; w.step = i; w.V = V; w.nreq = nreq; w.req0 = c0;
      w.temperature = L.temperature;
      w.seed = L.seed;
      const int gridw = w.units < L.num_sms ? w.units : L.num_sms;
      e = launch_pdl(gemm_kernel(epi_w2), dim3(gridw), dim3(NTH), wsm, st, tW2, tU, tW2, tU, w);
      if (e != cudaSuccess) return e;
    }
    // 6. picks, next fed tokens and embeddings (verification after the last position)
    e = launch_pdl(pick_step_kernel, dim3(B), dim3(256), 0, st, L.best, i, K, B, V, E, L.anchor, L.forced, L.target,
                   L.draft, L.tau, static_cast<const __nv_bfloat16*>(L.embed), Xg, L.fed, L.ctl);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace domino
