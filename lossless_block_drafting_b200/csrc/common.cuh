// Shared device helpers: status reporting, bounded mbarrier waits, argmax keys.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "orthrus.h"
#include "ptx.cuh"

namespace orthrus {

// A bounded wait gives up after `limit_ns` (the launch's wait limit: 2 s unless
// orthrus_set_wait_limit_ns changed it; the kernels' real waits take
// microseconds); the CTA then records ORTHRUS_ETIMEOUT and unwinds.
constexpr uint32_t kWaitMaxPolls = 1u << 30;

// Store `code` into *status if it is still 0 (first error wins).
__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// Limits below this select the kernels' short-wait instantiation (a watchdog
// or a test of the timeout path); the common path never pays for it.
constexpr uint64_t kShortWaitNs = 1000000ull;  // 1 ms

// Wait for the phase of `bar` with the given parity.  Returns false if the
// CTA-wide abort flag is raised or the wait runs out of time (which raises
// it).
//   kShort = false: one try_wait is the common path (it suspends the thread
//     until the phase completes or a hardware window ends); the abort flag and
//     the clock are looked at every 32 polls.
//   kShort = true (limit_ns < kShortWaitNs): every try_wait suspends the
//     thread for at most limit_ns, and flag and clock are looked at after
//     each, so the limit is noticed even when no hardware window would
//     outlast it.
template <bool kShort>
static __device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                      volatile int* abort_flag, int32_t* status,
                                                      uint64_t limit_ns) {
  if constexpr (kShort) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t polls = 0;; ++polls) {
      if (mbar_try_wait_for(bar, parity, static_cast<uint32_t>(limit_ns))) return true;
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns || polls > kWaitMaxPolls) {
        *abort_flag = 1;
        report(status, ORTHRUS_ETIMEOUT);
        return false;
      }
    }
  } else {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t polls = 1;; ++polls) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((polls & 31u) == 0) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns || polls > kWaitMaxPolls) {
          *abort_flag = 1;
          report(status, ORTHRUS_ETIMEOUT);
          return false;
        }
      }
    }
  }
}

// Warp-collective variant: every lane waits, and the warp proceeds only if all
// lanes succeeded, so warp-wide tcgen05 instructions after it are never
// reached by part of a warp.
template <bool kShort>
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile int* abort_flag, int32_t* status,
                                               uint64_t limit_ns) {
  if (!kShort && __all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;  // common case
  const bool ok = mbar_wait_bounded<kShort>(bar, parity, abort_flag, status, limit_ns);
  return __all_sync(0xFFFFFFFFu, ok);
}

// Wait that ignores the abort flag, used only to let in-flight asynchronous
// work (copies, MMAs) finish before the CTA exits; gives up after 200 ms.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, int32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) {
      report(status, ORTHRUS_ETIMEOUT);
      return;
    }
  }
}

// max(a, b, c) in one instruction (three-input form of max.f32).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Monotone map of fp32 onto uint32 (larger float -> larger key); -0 -> +0.
__device__ __forceinline__ uint32_t f32_order_key(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float f32_from_order_key(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// 64-bit argmax key: value in the high word, (0xFFFFFFFF - index) in the low
// word, so the maximum key is the maximum value at the SMALLEST index.  NaN
// values get key 0 (never chosen unless everything is NaN).
__device__ __forceinline__ uint64_t argmax_key(float v, uint32_t idx) {
  if (v != v) return 0ull;
  return (static_cast<uint64_t>(f32_order_key(v)) << 32) | (0xFFFFFFFFu - idx);
}
__device__ __forceinline__ int32_t key_index(uint64_t k) {
  return k == 0ull ? -1 : static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k));
}
__device__ __forceinline__ float key_value(uint64_t k) {
  return f32_from_order_key(static_cast<uint32_t>(k >> 32));
}

__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  uint32_t lo = static_cast<uint32_t>(v), hi = static_cast<uint32_t>(v >> 32);
  lo = __shfl_xor_sync(0xFFFFFFFFu, lo, m);
  hi = __shfl_xor_sync(0xFFFFFFFFu, hi, m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace orthrus
