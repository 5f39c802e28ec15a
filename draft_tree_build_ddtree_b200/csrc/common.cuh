// Shared device helpers of the DDTree round library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <utility>
#include <stdint.h>
#include <stdio.h>

#include "ddtree.h"

namespace ddt {

// The last host-side CUDA failure behind a DDTREE_ERR_CUDA return: the
// call that failed and the runtime's message (ddtree_last_error()).
inline char* last_error_buf() {
  static char buf[256] = "";
  return buf;
}
inline int cuda_fail(cudaError_t e, const char* where) {
  snprintf(last_error_buf(), 256, "%s: %s", where, cudaGetErrorString(e));
  return DDTREE_ERR_CUDA;
}
inline int cuda_fail_msg(const char* where) {
  snprintf(last_error_buf(), 256, "%s", where);
  return DDTREE_ERR_CUDA;
}

// Device status word read by ddtree_device_status(); bits DDTREE_STATUS_*.
__device__ unsigned int g_status;

__device__ __forceinline__ void flag_status(unsigned int bits) { atomicOr(&g_status, bits); }

// Programmatic dependent launch: a grid launched with programmatic stream
// serialization may start while the grid before it still runs; it must pass
// griddep_wait (which returns once that grid has completed and its writes are
// visible, and at once for a grid launched without the attribute) before it
// reads anything that grid writes.  griddep_launch_dependents lets such a
// dependent start as soon as every CTA of this grid has executed it.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch with programmatic stream serialization when `pdl` (the kernel then
// starts while the preceding kernel in the stream runs and must griddep_wait
// before reading its outputs); a plain launch otherwise.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_maybe_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Debug builds (-DDDTREE_DEBUG, libddtree_debug.so): internal indices are
// checked before they address memory; a violation sets
// DDTREE_STATUS_BOUNDS and the access is skipped, never a trap.  In release
// builds the check is `true`.
#ifdef DDTREE_DEBUG
__device__ __forceinline__ bool ddt_in_range(long long i, long long lo, long long hi) {
  if (i >= lo && i < hi) return true;
  flag_status(DDTREE_STATUS_BOUNDS);
  return false;
}
#define DDT_IN_RANGE(i, lo, hi) ddt::ddt_in_range((long long)(i), (long long)(lo), (long long)(hi))
#else
#define DDT_IN_RANGE(i, lo, hi) true
#endif

// ---------------------------------------------------------------------------
// Order-preserving integer keys: a > b as reals  <=>  key(a) > key(b).
// -0.0 maps to the key of +0.0; -inf is the smallest key of a real value.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t key16_of_bf16(uint16_t bits) {
  if (bits == 0x8000u) bits = 0;                       // -0.0 -> +0.0
  return (bits & 0x8000u) ? (uint32_t)(~bits & 0xFFFFu) : (uint32_t)(bits | 0x8000u);
}
__device__ __forceinline__ float bf16_of_key16(uint32_t key) {
  uint16_t bits = (key & 0x8000u) ? (uint16_t)(key & 0x7FFFu) : (uint16_t)(~key & 0xFFFFu);
  return __uint_as_float(((uint32_t)bits) << 16);
}
__device__ __forceinline__ uint32_t key32_of_f32(float x) {
  uint32_t bits = __float_as_uint(x);
  if (bits == 0x80000000u) bits = 0;                   // -0.0 -> +0.0
  return (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
}
__device__ __forceinline__ float f32_of_key32(uint32_t key) {
  uint32_t bits = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(bits);
}
__device__ __forceinline__ bool bf16_is_nan(uint16_t bits) {
  return (bits & 0x7F80u) == 0x7F80u && (bits & 0x007Fu) != 0;
}
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t bits) {
  return __uint_as_float(((uint32_t)bits) << 16);
}

// Order keys of the two bf16 values packed in a 32-bit word, two at a time:
// each 16-bit half becomes key16_of_bf16 of that half (-0.0 canonicalised).
__device__ __forceinline__ uint32_t key16x2_of_bf16x2(uint32_t w) {
  w &= ~__vcmpeq2(w, 0x80008000u);                      // -0.0 -> +0.0
  const uint32_t neg = ((w >> 15) & 0x00010001u) * 0xFFFFu;
  return w ^ (neg | 0x80008000u);
}
// Nonzero iff either half of the word is a bf16 NaN.
__device__ __forceinline__ uint32_t bf16x2_nan(uint32_t w) {
  return __vcmpgtu2(w & 0x7FFF7FFFu, 0x7F807F80u);
}

// 16-byte read-only global load that does not allocate in L1 (streamed once).
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Word k (0..3) of a 16-byte vector; k is a compile-time constant after
// unrolling, so this is a register select, not a memory access.
__device__ __forceinline__ uint32_t u32_at(const uint4& v, int k) {
  return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// ---------------------------------------------------------------------------
// Block-wide radix selection of the need-th largest key.
//
// Keys are `nbits` wide; `each(f)` calls f(key) for every key the thread
// holds (0 = empty).  Returns t, `above` (keys above t's final prefix) and
// `eq` (keys sharing the final prefix).  Either eq equals the remaining need
// (early exit: every key >= t is selected, t has zero low bits) or t is the
// exact value of the need-th key and the eq keys equal to it tie.
// ---------------------------------------------------------------------------
template <typename KeyT>
struct RadixOut {
  KeyT t;
  int above;
  int eq;
};

// Group form: the `gsize` threads with group-local ids `gtid` (its first 32
// form one warp) call it together and `sync()` is their barrier.
template <typename KeyT, typename Each, typename Sync>
__device__ __forceinline__ RadixOut<KeyT> radix_kth_g(Each each, int nbits, int need, uint32_t* hist, int* bcast,
                                                      int gtid, int gsize, Sync sync) {
  KeyT prefix = 0;
  int shift = nbits, above = 0, eq = 0;
  while (shift > 0) {
    const int width = shift < 8 ? shift : 8;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = gtid; i < 256; i += gsize) hist[i] = 0;
    sync();
    const int hi = shift + width;
    const bool top = hi >= (int)(8 * sizeof(KeyT));
    const KeyT want = top ? (KeyT)0 : (prefix >> hi);
    each([&](KeyT k) {
      if (k != 0 && (top || (k >> hi) == want)) atomicAdd(&hist[(uint32_t)(k >> shift) & dmask], 1u);
    });
    sync();
    if (gtid < 32) {
      uint32_t c[8];
      uint32_t mine = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = hist[8 * gtid + j]; mine += c[j]; }
      uint32_t incl = mine;   // keys in digits >= 8*lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
        if (gtid + o < 32) incl += v;
      }
      const uint32_t above_lane = incl - mine;
      const unsigned m = __ballot_sync(0xffffffffu, above_lane < (uint32_t)need && (uint32_t)need <= incl);
      if (m == 0 && gtid == 0) {          // fewer keys than need: all of them
        bcast[0] = 0;
        bcast[1] = (int)incl;
        bcast[2] = 0;
        bcast[3] = 0;
      }
      if (gtid == __ffs(m) - 1) {
        uint32_t ab = above_lane, cd = c[0];
        int d = 0;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
          if (ab + c[j] >= (uint32_t)need) { d = j; cd = c[j]; break; }
          ab += c[j];
        }
        bcast[0] = 8 * gtid + d;
        bcast[1] = (int)ab;
        bcast[2] = (int)cd;
        bcast[3] = 1;
      }
    }
    sync();
    const int digit = bcast[0], ab = bcast[1], cnt = bcast[2], ok = bcast[3];
    sync();
    if (!ok) return RadixOut<KeyT>{(KeyT)0, above + ab, 0};
    prefix |= ((KeyT)digit) << shift;
    need -= ab;
    above += ab;
    eq = cnt;
    if (cnt == need) break;
  }
  return RadixOut<KeyT>{prefix, above, eq};
}

template <typename KeyT, typename Each>
__device__ __forceinline__ RadixOut<KeyT> radix_kth(Each each, int nbits, int need, uint32_t* hist, int* bcast) {
  return radix_kth_g<KeyT>(each, nbits, need, hist, bcast, (int)threadIdx.x, (int)blockDim.x,
                           [] { __syncthreads(); });
}

// Barrier over `nthreads` threads (whole warps) on hardware barrier `id` (1..15).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}


}  // namespace ddt
