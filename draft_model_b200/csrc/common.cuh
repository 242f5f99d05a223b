// Device-side building blocks shared by the Domino kernels (sm_100a).
//
// Everything that waits on something another thread or the copy engine does is
// bounded by a %globaltimer budget: on expiry it raises DOMINO_ERR_TIMEOUT in the
// workspace error word and lets the caller return early, so no kernel can hang
// the GPU.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace domino {

// ---------------------------------------------------------------- error word bits
constexpr uint32_t ERRBIT_TIMEOUT = 1u;
constexpr uint32_t ERRBIT_BAD_TOKEN = 2u;

// Workspace control block (first 256 bytes of every workspace).
struct Control {
  uint32_t err;          // ERRBIT_* accumulated by device code
  uint32_t bar_count;    // grid barrier: arrivals during the current launch
  uint32_t bar_gen;      // CTAs that have left the current launch
  uint32_t pad0;
  uint64_t pad[30];
};
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

// ---------------------------------------------------------------- timing
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void raise_error(Control* ctl, uint32_t bit) {
  atomicOr(&ctl->err, bit);
}

// ---------------------------------------------------------------- memory-order helpers
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t atom_add_release_u32(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier for a co-resident (cooperatively launched) grid, executed by
// ONE thread per CTA (the caller brackets it with CTA barriers), in two halves
// so a CTA can do independent work between arriving and waiting.  The arrival
// counter only grows during a launch: barrier number k (0-based) completes when
// it reaches G*(k+1).  Arrival is a fire-and-forget release reduction; the wait
// polls with relaxed loads and ends with an acquire fence.  The last CTA to
// leave the kernel resets the counter (grid_exit), so every launch starts at 0.
__device__ __forceinline__ void grid_barrier_arrive(Control* ctl) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&ctl->bar_count) : "memory");
}
// Returns false if the wait ran out of budget (the error bit is raised).
__device__ __forceinline__ bool grid_barrier_wait(Control* ctl, uint32_t target, uint64_t budget_ns) {
  uint32_t spins = 0;
  uint64_t t0 = 0;
  while (true) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&ctl->bar_count) : "memory");
    if (static_cast<int32_t>(v - target) >= 0) break;
    if ((++spins & 31u) == 0u) {
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) t0 = now;
      else if (now - t0 > budget_ns) {
        raise_error(ctl, ERRBIT_TIMEOUT);
        return false;
      }
    }
  }
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
  return true;
}

// Called once per CTA (one thread) after its last barrier: the last CTA out
// resets the barrier counter for the next launch on this workspace.
__device__ __forceinline__ void grid_exit(Control* ctl, uint32_t nblocks) {
  const uint32_t n = atom_add_release_u32(&ctl->bar_gen, 1u) + 1u;
  if (n == nblocks) {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    st_relaxed_u32(&ctl->bar_count, 0u);
    st_relaxed_u32(&ctl->bar_gen, 0u);
  }
}

// ---------------------------------------------------------------- shared-memory mbarriers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}
// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Control* ctl, uint64_t budget_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > budget_ns) {
      raise_error(ctl, ERRBIT_TIMEOUT);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> shared (TMA engine, no tensor map, no multicast).
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// Bulk prefetch of a global range into L2 (no shared-memory destination).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// 4-byte asynchronous global -> shared copy (LDGSTS) and its group fences.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Programmatic dependent launch (kernels launched with programmatic stream
// serialization): let the next kernel in the stream start its prologue now, and
// wait until the kernel this one depends on has completed and its writes are
// visible.  Both are no-ops for a normally launched kernel.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Order-preserving map of a float onto uint32 (larger float -> larger integer).
__device__ __forceinline__ uint32_t orderable_u32(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Named barrier over a subset of warps (id != 0; count a multiple of 32).
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------- element access
// Widen 8 consecutive storage elements to fp32.  bf16 -> fp32 is exact: the
// bf16 bits are the top half of the fp32 bits.
__device__ __forceinline__ void widen8(const __nv_bfloat16* p, float* out) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    out[2 * k] = __uint_as_float(w[k] << 16);
    out[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void widen8(const float* p, float* out) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

// Warp reduce-scatter of 32 per-lane slots: afterwards lane l holds the sum over
// all lanes of slot l.  31 shuffles (butterfly that halves the slot set per stage).
__device__ __forceinline__ float warp_reduce_scatter32(float (&a)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float keep = upper ? a[j + half] : a[j];
      const float give = upper ? a[j] : a[j + half];
      a[j] = keep + __shfl_xor_sync(0xFFFFFFFFu, give, half);
    }
  }
  return a[0];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// ---------------------------------------------------------------- argmax keys
// Monotone map of an fp32 score to uint32 (larger score -> larger key), joined
// with the inverted index so that a 64-bit max prefers the lowest index on ties.
__device__ __forceinline__ uint64_t argmax_key(float score, uint32_t idx) {
  return (static_cast<uint64_t>(orderable_u32(score)) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - idx);
}
__device__ __forceinline__ uint32_t argmax_key_index(uint64_t key) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull);
}

// ---------------------------------------------------------------- Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
// (SC'11): ten rounds of two 32x32->64 multiplies with a Weyl-sequence key.
struct Philox4 {
  uint32_t x[4];
};
__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                                 uint32_t k1) {
  constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  constexpr uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t lo0 = M0 * c0, hi0 = __umulhi(M0, c0);
    const uint32_t lo1 = M1 * c2, hi1 = __umulhi(M1, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    k0 += W0; k1 += W1;
  }
  Philox4 out;
  out.x[0] = c0; out.x[1] = c1; out.x[2] = c2; out.x[3] = c3;
  return out;
}

// Gumbel noise for (seed, request b, 0-based position p, token j).
__device__ __forceinline__ float gumbel_noise(uint64_t seed, uint32_t b, uint32_t p, uint32_t j) {
  const Philox4 r = philox4x32_10(j >> 2, p, b, 0u, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  const uint32_t sel = j & 3u;
  const uint32_t w = sel == 0u ? r.x[0] : sel == 1u ? r.x[1] : sel == 2u ? r.x[2] : r.x[3];
  const float u = (static_cast<float>(w >> 9) * 2.0f + 1.0f) * 5.9604644775390625e-8f;  // 2^-24, exact
  return -logf(-logf(u));
}

}  // namespace domino
