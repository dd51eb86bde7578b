// psi_device.cuh - device building blocks of the Psi-Spec verify kernels
// (sm_100a): the counter RNG, order-preserving logit keys, 16-byte vector
// access, TMA bulk copies with mbarriers, and thread-block-cluster
// primitives (DSMEM address mapping, cluster barriers).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "psi_verify.h"

namespace psi {

constexpr int kThreads = 256;            // threads per CTA in every kernel
constexpr int kWarps = kThreads / 32;

// ---------------------------------------------------------------------------
// Counter RNG.  SplitMix64 (Steele, Lea & Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014): one output step adds the
// golden-gamma increment to the state and finalises it with Stafford's
// "Mix13" variant of the MurmurHash3 finaliser.  The verify step hashes the
// counters (seed, sequence, step, row, purpose) by chaining that step, and
// turns the top 24 bits into a float in [0, 1).
// ---------------------------------------------------------------------------
struct SplitMix64 {
  static constexpr uint64_t kGoldenGamma = 0x9E3779B97F4A7C15ull;
  static constexpr uint64_t kMul1 = 0xBF58476D1CE4E5B9ull;
  static constexpr uint64_t kMul2 = 0x94D049BB133111EBull;
  __device__ __forceinline__ static uint64_t step(uint64_t state) {
    uint64_t v = state + kGoldenGamma;
    v = (v ^ (v >> 30)) * kMul1;
    v = (v ^ (v >> 27)) * kMul2;
    return v ^ (v >> 31);
  }
};

__device__ __forceinline__ uint64_t counter_hash(uint64_t seed, uint64_t seq,
                                                 uint64_t step, uint64_t row,
                                                 uint64_t purpose) {
  const uint64_t words[4] = {seq, step, row, purpose};
  uint64_t h = SplitMix64::step(seed);
#pragma unroll
  for (int k = 0; k < 4; ++k) h = SplitMix64::step(h ^ words[k]);
  return h;
}

// 24 random bits scaled by 2^-24: exact in float, in [0, 1 - 2^-24].
__device__ __forceinline__ float uniform24(uint64_t seed, uint64_t seq,
                                           uint64_t step, uint64_t row,
                                           uint64_t purpose) {
  const uint32_t top = (uint32_t)(counter_hash(seed, seq, step, row, purpose) >> 40);
  return __uint2float_rn(top) * 5.9604644775390625e-08f;  // 2^-24
}

// ---------------------------------------------------------------------------
// Logit element types.  Kernels are templated on the raw bit type: uint16_t
// carries bfloat16, uint32_t carries float32.  A 16-byte vector holds kVec
// elements.  key() maps a value to an unsigned integer whose order is the
// numeric order (-0 and +0 share one key), so max/argmax/radix select work on
// integers.
// ---------------------------------------------------------------------------
template <typename Bits>
struct Elem;

template <>
struct Elem<uint16_t> {
  static constexpr int kVec = 8;
  static constexpr int kKeyBits = 16;
  static constexpr uint16_t kNegInf = 0xFF80u;
  __device__ __forceinline__ static float to_float(uint32_t b) {
    return __uint_as_float(b << 16);
  }
  __device__ __forceinline__ static uint32_t key(uint32_t b) {
    b = (b == 0x8000u) ? 0u : b;
    return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
  }
  // NaN or +inf (-inf is a valid logit)
  __device__ __forceinline__ static bool bad(uint32_t b) {
    return (b & 0x7FFFu) > 0x7F80u || b == 0x7F80u;
  }
};

template <>
struct Elem<uint32_t> {
  static constexpr int kVec = 4;
  static constexpr int kKeyBits = 32;
  static constexpr uint32_t kNegInf = 0xFF800000u;
  __device__ __forceinline__ static float to_float(uint32_t b) {
    return __uint_as_float(b);
  }
  __device__ __forceinline__ static uint32_t key(uint32_t b) {
    b = (b == 0x80000000u) ? 0u : b;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  }
  __device__ __forceinline__ static bool bad(uint32_t b) {
    return (b & 0x7FFFFFFFu) > 0x7F800000u || b == 0x7F800000u;
  }
};

// Element k (0..kVec-1) of a 16-byte vector.
template <typename Bits>
__device__ __forceinline__ uint32_t vec_elem(const uint4 &v, int k) {
  // selects rather than an indexed array, so a run-time k stays in registers
  const int q = sizeof(Bits) == 2 ? (k >> 1) : k;
  const uint32_t word = q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
  if constexpr (sizeof(Bits) == 2)
    return (k & 1) ? (word >> 16) : (word & 0xFFFFu);
  else
    return word;
}

// Cheap screen for "some element may be NaN/+-inf": true for every vector
// that holds one; exact check with Elem::bad() afterwards.
template <typename Bits>
__device__ __forceinline__ bool vec_maybe_nonfinite(const uint4 &v) {
  if constexpr (sizeof(Bits) == 2) {
    const uint32_t m = 0x7FFF7FFFu, add = 0x00800080u;
    const uint32_t t = ((v.x & m) + add) | ((v.y & m) + add) |
                       ((v.z & m) + add) | ((v.w & m) + add);
    return (t & 0x80008000u) != 0u;
  } else {
    const uint32_t m = 0x7FFFFFFFu, lim = 0x7F800000u;
    return (v.x & m) >= lim || (v.y & m) >= lim || (v.z & m) >= lim ||
           (v.w & m) >= lim;
  }
}

template <typename Bits>
__device__ __forceinline__ bool vec_has_bad(const uint4 &v) {
  if (!vec_maybe_nonfinite<Bits>(v)) return false;
  bool bad = false;
#pragma unroll
  for (int k = 0; k < Elem<Bits>::kVec; ++k) bad |= Elem<Bits>::bad(vec_elem<Bits>(v, k));
  return bad;
}

// Streaming 16-byte global load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with the PDL attribute
// (launch_pdl) may start while the kernel before it on the stream finishes:
// pdl_wait() returns once that kernel has completed and its memory writes are
// visible (at once for a kernel launched without the attribute), and
// pdl_trigger() lets the next kernel on the stream be launched early.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Shared memory, mbarriers and TMA bulk copies.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t arrivals) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(arrivals)
               : "memory");
}

// Make mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// One try: the thread may sleep until the phase completes, for at most
// `suspend_ns` (a hint), so waiting warps do not spin.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity,
                                              uint32_t suspend_ns = 20000u) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return done != 0u;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for an mbarrier phase, giving up after ~`limit_ns` nanoseconds.
// Returns false on timeout (the caller records it and carries on).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// Plain arrive on a local mbarrier (release at CTA scope).
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Arrive on an mbarrier of another CTA of the cluster (address from
// dsmem_map), releasing this thread's earlier shared::cluster stores.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// One test of a phase (no suspend hint), acquire at CTA scope.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0u;
}

// One test of a phase, acquire at cluster scope (the phase's arrivals came
// from other CTAs of the cluster, with their shared::cluster stores).
__device__ __forceinline__ bool mbar_test_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0u;
}

// Store into the shared memory of a CTA of the cluster (address from dsmem_map).
__device__ __forceinline__ void dsmem_st_f32(uint32_t cluster_addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}

__device__ __forceinline__ void dsmem_st_u64(uint32_t cluster_addr, uint64_t v) {
  asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(cluster_addr), "l"(v) : "memory");
}

// 16-byte shared-memory load.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// One bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src and bytes must be multiples of 16.  No multicast.
__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Hint: bring `bytes` of global memory at `src` into L2 (no data returned,
// no completion to wait for).  src and bytes must be multiples of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_sync() {
  cluster_arrive();
  cluster_wait();
}

// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_map(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ float dsmem_ld_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t dsmem_ld_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ double dsmem_ld_f64(uint32_t addr) {
  double v;
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t dsmem_ld_u64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// Reductions.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
  return __reduce_max_sync(0xFFFFFFFFu, v);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

}  // namespace psi
