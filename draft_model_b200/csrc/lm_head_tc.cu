// Stage 1 of the Domino draft block on the tcgen05 tensor cores (sm_100a):
// base logits L^base[m, v] = sum_k W_lm[v, k] h[m, k] for every block position m
// (m = b*K + i), computed once per block (Domino study notes, gsyq.cn, §二.1(1);
// yhxrc.cn article, §三 第一个阶段).  The same launch also produces the
// hidden-state half of the bottleneck pre-activation, P[m, k] = W1[k, 0:d] h[m]
// (yhxrc.cn §四: W1 acts on [h_i ; S_{i-1}], and the h_i part depends on the
// backbone only), as two extra 128-row A tiles read from W1 with its row stride.
//
// Swap-AB formulation: the UMMA "A" operand is a 128-row tile of W_lm (vocabulary
// on the M side, so V = 151936 = 1187 x 128 tiles exactly) and "B" is a tile of
// the hidden states (BN = 16..256 block positions on the N side).  The fp32
// accumulator lives in tensor memory: TMEM lane = vocabulary row, column = block
// position, so the epilogue's tcgen05.ld hands every thread one vocabulary row
// and a warp stores 32 consecutive floats of one output row (coalesced).
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: 2-D tiled loads (128B swizzle) of A and B into a
//               STAGES-deep shared-memory ring (no multicast);
//   warp 1      TMEM allocator and single-thread MMA issuer
//               (tcgen05.mma.cta_group::1.kind::f16, K = 16 per instruction);
//   warps 2..5  epilogue: tcgen05.ld 32x32b from a double-buffered accumulator,
//               fp32 stores to HBM while the next tile accumulates.
// Every mbarrier wait is bounded; on expiry the kernel flags DOMINO_ERR_TIMEOUT,
// drains its copies and MMAs, frees TMEM and returns.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "domino_internal.h"
#include "tc_common.cuh"

namespace domino {
namespace {

using namespace tc;
constexpr int NTH = 192;
constexpr int kStageSubBlocks = 2;               // 64-wide k sub-blocks per pipeline stage

struct TcArgs {
  float* out;        // [M, V]
  float* out2;       // [M, rows2] (second A operand's products) or null
  float* sk_part;    // stream-K partial tiles [grid][BN][128] or null (whole tiles only)
  uint32_t* sk_flag; // [grid] partial-tile ready flags (zero between launches)
  Control* ctl;
  uint64_t budget_ns;
  int V, M, Kd;
  int BN;            // block positions per tile (multiple of 16, <= 256)
  int nk;            // 64-wide k sub-blocks per pipeline stage
  int stages;
  int tmem_cols;     // power of two >= 2*BN
  int num_vt, num_mt, num_kb;  // num_kb counts pipeline stages (nk sub-blocks each) per tile
  int rows2, num_vt2;  // second A operand: rows and 128-row tiles (0 = none)
};

// A contiguous run of k-stages of one tile handled by one CTA.  FULL runs cover
// the whole tile; with stream-K a CTA's first run may be the TAIL of a tile
// whose HEAD is the previous CTA's last run: the TAIL's owner parks its partial
// sums in global memory and the HEAD's owner adds them and stores the tile.
enum SegKind : int { SEG_FULL = 0, SEG_TAIL = 1, SEG_HEAD = 2 };
struct Seg {
  int t, kb0, kb1, kind;
};
struct SegIter {
  long long u, hi;  // stream-K: unit range (units = k-stages over all tiles)
  int t;            // whole-tile schedule: next tile
  bool sk;
  __device__ __forceinline__ bool next(const TcArgs& a, int ntiles, Seg& g) {
    if (sk) {
      if (u >= hi) return false;
      g.t = static_cast<int>(u / a.num_kb);
      g.kb0 = static_cast<int>(u % a.num_kb);
      g.kb1 = static_cast<int>(min(static_cast<long long>(a.num_kb), g.kb0 + (hi - u)));
      g.kind = (g.kb0 == 0 && g.kb1 == a.num_kb) ? SEG_FULL : (g.kb0 > 0 ? SEG_TAIL : SEG_HEAD);
      u += g.kb1 - g.kb0;
      return true;
    }
    if (t >= ntiles) return false;
    g.t = t;
    g.kb0 = 0;
    g.kb1 = a.num_kb;
    g.kind = SEG_FULL;
    t += gridDim.x;
    return true;
  }
};
__device__ __forceinline__ SegIter seg_begin(const TcArgs& a, int ntiles) {
  SegIter it;
  it.sk = a.sk_part != nullptr;
  const long long units = static_cast<long long>(ntiles) * a.num_kb;
  it.u = units * blockIdx.x / gridDim.x;
  it.hi = units * (blockIdx.x + 1) / gridDim.x;
  it.t = blockIdx.x;
  return it;
}

// Tile t -> (operand, vocabulary tile, position tile).  Tiles run position tile
// by position tile, each block being the W_lm tiles and then the second A
// operand's tiles of that position tile: with the k-stages split evenly over
// the CTAs, the CTAs on different position tiles then stream the same W_lm rows
// at about the same time, and the repeats are L2 hits.
__device__ __forceinline__ void tile_decode(const TcArgs& a, int t, bool& second, int& vt, int& mt) {
  const int per_mt = a.num_vt + a.num_vt2;
  mt = t / per_mt;
  const int rem = t % per_mt;
  second = rem >= a.num_vt;
  vt = second ? rem - a.num_vt : rem;
}

__global__ void __launch_bounds__(NTH, 1)
    lm_head_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                      const __grid_constant__ CUtensorMap tmB, const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment of every stage (the swizzle atom)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t b_sub_bytes = static_cast<uint32_t>(a.BN) * BK * 2;
  const uint32_t a_bytes = A_STAGE_BYTES * a.nk;          // nk A sub-tiles, then nk B sub-tiles
  const uint32_t stage_bytes = a_bytes + b_sub_bytes * a.nk;
  uint8_t* ctrl = smem + static_cast<size_t>(a.stages) * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + a.stages;
  uint64_t* tfull = empty + a.stages;   // [2]
  uint64_t* tempty = tfull + 2;         // [2]
  uint64_t* mma_done = tempty + 2;      // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = (a.num_vt + a.num_vt2) * a.num_mt;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    if (a.num_vt2) prefetch_tmap(&tmA2);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, a.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

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
      int it = 0;  // global k-stage counter
      int s = 0;   // ring slot of k-stage it
      uint32_t ph = 0;  // (it / stages) & 1
      bool ok = true;
      SegIter si = seg_begin(a, ntiles);
      Seg g;
      while (ok && si.next(a, ntiles, g)) {
        bool second;
        int vt, mt;
        tile_decode(a, g.t, second, vt, mt);
        const CUtensorMap* tA = second ? &tmA2 : &tmA;
        for (int kb = g.kb0; kb < g.kb1; ++kb, ++it) {
          if (it >= a.stages && !bounded_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
          uint8_t* sa = smem + static_cast<size_t>(s) * stage_bytes;
          uint8_t* sb = sa + a_bytes;
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          for (int j = 0; j < a.nk; ++j) {
            const int kc = (kb * a.nk + j) * BK;
            tma_load_2d(sa + j * A_STAGE_BYTES, tA, kc, vt * BM, &full[s]);
            tma_load_2d(sb + j * b_sub_bytes, &tmB, kc, mt * a.BN, &full[s]);
          }
          if (++s == a.stages) { s = 0; ph ^= 1u; }
        }
      }
      // drain copies that were issued but may still be in flight
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
      SegIter si = seg_begin(a, ntiles);
      Seg g;
      while (ok && si.next(a, ntiles, g)) {
        const int acc = local & 1;
        if (local >= 2 && !bounded_wait(&tempty[acc], ((local >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * a.BN);
        for (int kb = g.kb0; kb < g.kb1; ++kb, ++it) {
          if (!bounded_wait(&full[s], ph)) { ok = false; break; }
          tc_fence_after();
          // descriptors advance by (bytes >> 4) in their start-address field
          const uint64_t da = smem_desc_sw128(smem_u32(smem + static_cast<size_t>(s) * stage_bytes));
          const uint64_t db = da + (a_bytes >> 4);
          for (int j = 0; j < a.nk; ++j) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              tc_mma_bf16(d_tmem, da + ((j * A_STAGE_BYTES + kk * 32) >> 4), db + ((j * b_sub_bytes + kk * 32) >> 4),
                          idesc, (kb > g.kb0 || j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(&empty[s]);   // frees the stage once these MMAs have read it
          if (++s == a.stages) { s = 0; ph ^= 1u; }
        }
        if (ok) tc_commit(&tfull[acc]);
        ++local;
      }
      // every MMA issued by this thread must finish before TMEM is released
      tc_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(mma_done, 0)) {
        if (globaltimer_ns() - t0 > a.budget_ns) { raise_error(a.ctl, ERRBIT_TIMEOUT); break; }
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lane quarter = warp % 4
    const int q = warp & 3;
    int local = 0;
    SegIter si = seg_begin(a, ntiles);
    Seg g;
    while (si.next(a, ntiles, g)) {
      const int acc = local & 1;
      if (lane == 0) bounded_wait(&tfull[acc], (local >> 1) & 1);
      named_barrier(2, 128);          // the four epilogue warps take the same decision
      if (*abort_flag) break;
      tc_fence_after();
      bool second;
      int vt, mt;
      tile_decode(a, g.t, second, vt, mt);
      const int row = q * 32 + lane;                 // row of the 128-row tile
      const int v = vt * BM + row;
      const int nrows = second ? a.rows2 : a.V;
      float* dst = second ? a.out2 : a.out;
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * a.BN);
      if (g.kind == SEG_HEAD) {
        // the next CTA parked the tail of this tile: wait for its flag
        bool ready = true;
        if (threadIdx.x == 64) {
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_u32(&a.sk_flag[blockIdx.x + 1]) == 0u) {
            if (*abort_flag || globaltimer_ns() - t0 > a.budget_ns) {
              raise_error(a.ctl, ERRBIT_TIMEOUT);
              *abort_flag = 1;
              ready = false;
              break;
            }
          }
        }
        named_barrier(2, 128);
        ready = ready && !*abort_flag;
        if (!ready) break;
      }
      const float* park_in = a.sk_part + static_cast<size_t>(blockIdx.x + 1) * a.BN * BM;
      float* park_out = a.sk_part + static_cast<size_t>(blockIdx.x) * a.BN * BM;
      for (int cb = 0; cb < a.BN; cb += 64) {
        // a HEAD adds the parked tail: its 64 columns are loaded together, before
        // any store of this batch (the stores could alias them for the compiler,
        // which would otherwise serialise one load latency per column)
        float part[64];
        if (g.kind == SEG_HEAD) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            part[c] = cb + c < a.BN ? __ldcg(park_in + static_cast<size_t>(cb + c) * BM + row) : 0.f;
        }
#pragma unroll
        for (int c1 = 0; c1 < 64; c1 += 16) {
          const int c0 = cb + c1;
          if (c0 >= a.BN) break;
          float vals[16];
          tmem_ld16(trow + c0, vals);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int col = c0 + c;
            if (g.kind == SEG_TAIL) {
              park_out[static_cast<size_t>(col) * BM + row] = vals[c];
            } else {
              const float x = g.kind == SEG_HEAD ? vals[c] + part[c1 + c] : vals[c];
              const int m = mt * a.BN + col;
              if (v < nrows && m < a.M) dst[static_cast<size_t>(m) * nrows + v] = x;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (g.kind != SEG_FULL) {
        named_barrier(2, 128);   // all four epilogue warps done with the partial tile
        if (threadIdx.x == 64) {
          if (g.kind == SEG_TAIL) {
            __threadfence();
            asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(&a.sk_flag[blockIdx.x]), "r"(1u) : "memory");
          } else {
            st_relaxed_u32(&a.sk_flag[blockIdx.x + 1], 0u);   // consumed: clean for the next launch
          }
        }
      }
      ++local;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, a.tmem_cols);
}

}  // namespace

cudaError_t launch_lm_head_tc(const void* w_lm, const void* hidden, float* out, int V, int M, int Kd,
                              const void* w1, int rows2, int w1_stride, float* out2, float* sk_part,
                              uint32_t* sk_flag, Control* ctl, uint64_t budget_ns, int num_sms,
                              cudaStream_t stream) {
  TcArgs a;
  a.out = out;
  a.out2 = out2;
  a.rows2 = out2 ? rows2 : 0;
  a.ctl = ctl;
  a.budget_ns = budget_ns;
  a.V = V;
  a.M = M;
  a.Kd = Kd;
  int bn = (M + 15) / 16 * 16;
  a.BN = bn > 256 ? 256 : bn;
  int cols = 32;
  while (cols < 2 * a.BN) cols <<= 1;
  a.tmem_cols = cols;
  a.num_vt = out ? (V + BM - 1) / BM : 0;
  a.num_vt2 = out2 ? (rows2 + BM - 1) / BM : 0;
  a.num_mt = (M + a.BN - 1) / a.BN;
  a.nk = a.BN <= 64 ? kStageSubBlocks : 1;
  a.num_kb = (Kd + BK * a.nk - 1) / (BK * a.nk);
  const uint32_t stage_bytes = (A_STAGE_BYTES + static_cast<uint32_t>(a.BN) * BK * 2) * a.nk;
  const size_t budget = 220 * 1024;
  int stages = static_cast<int>((budget - 2048) / stage_bytes);
  if (stages > 12) stages = 12;
  if (stages < 2) return cudaErrorInvalidValue;
  a.stages = stages;
  const size_t smem = static_cast<size_t>(stages) * stage_bytes + 1024 /*align*/ + 256 /*barriers*/;

  CUtensorMap tmA, tmA2, tmB;
  if (!make_tmap(&tmA, out ? w_lm : w1, out ? V : rows2, Kd, BM, out ? Kd : w1_stride)) return cudaErrorInvalidValue;
  if (out2) {
    if (!make_tmap(&tmA2, w1, rows2, Kd, BM, w1_stride)) return cudaErrorInvalidValue;
  } else {
    tmA2 = tmA;
  }
  if (!make_tmap(&tmB, hidden, M, Kd, a.BN, Kd)) return cudaErrorInvalidValue;

  cudaError_t e = cudaFuncSetAttribute(lm_head_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int ntiles = (a.num_vt + a.num_vt2) * a.num_mt;
  if (ntiles == 0) return cudaSuccess;
  const int grid = ntiles < num_sms ? ntiles : num_sms;
  // stream-K when whole tiles would leave a ragged last wave and every CTA still
  // gets at least one tile's worth of k-stages (so a tile spans at most two CTAs)
  const long long units = static_cast<long long>(ntiles) * a.num_kb;
  const bool sk = sk_part && sk_flag && grid <= kLoopMaxGrid && ntiles % grid != 0 && units / grid >= a.num_kb;
  a.sk_part = sk ? sk_part : nullptr;
  a.sk_flag = sk ? sk_flag : nullptr;
  void* params[] = {&tmA, &tmA2, &tmB, &a};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(lm_head_tc_kernel), dim3(grid), dim3(NTH), params, smem,
                                     stream);
}

}  // namespace domino
