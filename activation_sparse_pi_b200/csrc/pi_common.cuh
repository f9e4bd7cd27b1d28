// Device helpers shared by the sparse-FFN kernels (sm_100a).
//
// Data movement uses the sm_90+/sm_100 bulk-copy engine (cp.async.bulk,
// 1-D, global -> shared, completion counted on an mbarrier).  Every wait on
// an mbarrier is bounded: after kWaitLimit polls the kernel records
// kErrTimeout in the device error word and the caller bails out.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pi {

constexpr int kMaxBatch = 64;
constexpr int kErrTimeout = 1;
constexpr int kErrBadIndex = 2;
constexpr uint32_t kWaitLimit = 1u << 22;
// Suspend-hinted waits: each poll may sleep up to kSuspendNs before returning,
// so a waiting warp does not spin; kWaitLimitSleep polls bound the wait to
// about one second.
#ifndef PI_SUSPEND_NS
#define PI_SUSPEND_NS 2000
#endif
constexpr uint32_t kSuspendNs = PI_SUSPEND_NS;
constexpr uint32_t kWaitLimitSleep = (1u << 19) * (2000u / (PI_SUSPEND_NS < 2000 ? PI_SUSPEND_NS : 2000));

// Device error word (read and cleared by pi_device_error()).
__device__ int g_dev_error;

__device__ __forceinline__ void set_error(int code) { atomicOr(&g_dev_error, code); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}
// Bounded wait that lets the thread sleep between polls.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kWaitLimitSleep; ++it)
    if (mbar_try_wait_sleep(bar, parity)) return true;
  set_error(kErrTimeout);
  return false;
}

// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kWaitLimit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  set_error(kErrTimeout);
  return false;
}

// ------------------------------------------------------------- bulk copies
// 1-D bulk copy global -> shared; dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Same, with an L2 eviction-priority policy (streamed once: evict first).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Hint the L2 to fetch [src, src + bytes) (16-byte aligned, bytes % 16 == 0);
// no completion is tracked.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ------------------------------------------- programmatic dependent launch
// Wait until the preceding kernel in the stream has completed and its memory
// is visible (no-op when the kernel was not launched as a dependent).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the next kernel in the stream to start its prologue.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ----------------------------------------------------- 16-bit arithmetic
// DT: 0 = fp16, 1 = bf16.  A 32-bit word holds two consecutive elements, the
// lower-addressed one in the low half.
template <int DT>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
  if constexpr (DT == 0) {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  } else {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
}

// Only standard fp32 FMAs are used for 16-bit operands (each widened exactly
// to fp32, so products are exact): an earlier form of these kernels with the
// mixed-precision fma.f32.bf16 instruction faulted with "illegal instruction"
// in one kernel instantiation on B200.
// Sum of the 8 products of a 16-byte chunk of 16-bit weights with 8 fp32
// activations (two accumulation chains).
template <int DT>
__device__ __forceinline__ float dot8(const uint4& w, const float* x) {
  const float2 f0 = unpack2<DT>(w.x), f1 = unpack2<DT>(w.y);
  const float2 f2 = unpack2<DT>(w.z), f3 = unpack2<DT>(w.w);
  float a0 = f0.x * x[0], a1 = f0.y * x[1];
  a0 = fmaf(f1.x, x[2], a0); a1 = fmaf(f1.y, x[3], a1);
  a0 = fmaf(f2.x, x[4], a0); a1 = fmaf(f2.y, x[5], a1);
  a0 = fmaf(f3.x, x[6], a0); a1 = fmaf(f3.y, x[7], a1);
  return a0 + a1;
}

// Widen a 16-byte chunk of 16-bit activations to 8 fp32 values.
template <int DT>
__device__ __forceinline__ void widen8(const uint4& v, float* x) {
  const float2 f0 = unpack2<DT>(v.x), f1 = unpack2<DT>(v.y);
  const float2 f2 = unpack2<DT>(v.z), f3 = unpack2<DT>(v.w);
  x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
  x[4] = f2.x; x[5] = f2.y; x[6] = f3.x; x[7] = f3.y;
}

// Round an fp32 value to the 16-bit activation type (nearest even), as bits.
template <int DT>
__device__ __forceinline__ uint16_t round16(float v) {
  if constexpr (DT == 0) {
    return __half_as_ushort(__float2half_rn(v));
  } else {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

// Q4_0 nibble q (0..15) -> (q - 8) as an exact fp32: place q in the low
// mantissa bits of 2^23 and subtract 2^23 + 8.
__device__ __forceinline__ float q4_val(uint32_t q) {
  return __uint_as_float(0x4B000000u | q) - 8388616.0f;
}

// ------------------------------------------------------- plain loads
// 128-bit streaming load of read-only data (read once: no L1 allocation).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// The same load with an L2 eviction-priority policy (from createpolicy).
__device__ __forceinline__ uint4 ldg_stream_hint(const void* p, uint64_t policy) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(policy));
  return v;
}

// Ask the L2 for this CTA's share of a byte range (16-byte aligned start and
// size): bytes [cta * share, (cta + 1) * share), in pieces of at most 32 KB.
__device__ __forceinline__ void prefetch_l2_share(const uint8_t* base, size_t bytes, int cta,
                                                  int nctas) {
  if (!base || bytes == 0) return;
  const size_t share = ((bytes + nctas - 1) / nctas + 15) & ~size_t(15);
  const size_t lo = (size_t)cta * share;
  if (lo >= bytes) return;
  const size_t hi = lo + share < bytes ? lo + share : bytes;
  for (size_t o = lo; o < hi; o += 32768) {
    const size_t n = hi - o < 32768 ? hi - o : 32768;
    prefetch_l2(base + o, (uint32_t)n);
  }
}

// ------------------------------------------------------- grid barrier
// Barrier over all CTAs of a grid whose CTAs are all resident at once (the
// launcher sizes the grid from the occupancy calculator).  *count is a ticket
// counter: it is 0 before the first barrier of an API call and every barrier
// adds gridDim.x to it, so the k-th barrier (from 0) releases when it reaches
// (k + 1) * gridDim.x.  Every grid that uses one counter between two zeroings
// must have the same size.  The wait is bounded: on timeout the device error
// word records kErrTimeout and the call returns false.
constexpr uint32_t kGridWaitLimit = 1u << 21;  // about a second of polls

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ bool grid_barrier(uint32_t* count) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();  // this CTA's writes happen before its arrival
    const uint32_t ticket = atomicAdd(count, 1u);
    const uint32_t target = (ticket / gridDim.x + 1) * gridDim.x;
    uint32_t it = 0;
    while ((int32_t)(ld_acquire_gpu(count) - target) < 0) {
      if (++it == kGridWaitLimit) {
        set_error(kErrTimeout);
        ok = 0;
        break;
      }
      __nanosleep(32);
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// ------------------------------------------------------- warp reductions
// Transposed reduction of V values (V a power of two, V <= 32) across the
// warp.  Afterwards every lane holds the warp sum of value (lane >> (5 -
// log2 V)) in v[0].
template <int V>
__device__ __forceinline__ float warp_reduce_transposed(float (&v)[V]) {
  const int lane = threadIdx.x & 31;
  int n = V;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < n / 2) {
          float send = upper ? v[i] : v[i + n / 2];
          float keep = upper ? v[i + n / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return v[0];
}

template <int V>
__device__ __forceinline__ constexpr int log2c() {
  return V <= 1 ? 0 : 1 + log2c<V / 2>();
}

}  // namespace pi
