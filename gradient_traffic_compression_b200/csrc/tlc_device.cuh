// tlc_device.cuh -- device-side helpers shared by the compress and decode
// kernels: status-word publication for single-pass (decoupled look-back)
// scans, bounded waits, block-wide scans, and error reporting.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tlc.h"

namespace tlc {

constexpr int kWarp = 32;

__host__ __device__ __forceinline__ uint64_t umin64(uint64_t a, uint64_t b) { return a < b ? a : b; }

// ---------------------------------------------------------------------------
// Tile status words.  Each tile of a single-pass scan owns one 64-bit word:
// bits 62..63 hold the flag, the rest the tile's value.  A word is written
// first with its aggregate (flag 1) and later with its inclusive prefix
// (flag 2); both values are self-contained, so relaxed 64-bit accesses at
// GPU scope are enough (a reader sees one whole word or the other).
// ---------------------------------------------------------------------------
constexpr uint64_t kFlagShift = 62;
constexpr uint64_t kFlagAgg = 1ull << kFlagShift;
constexpr uint64_t kFlagPrefix = 2ull << kFlagShift;
constexpr uint64_t kValueMask = (1ull << kFlagShift) - 1;

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_u64(uint64_t *p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of the library is launched
// (launch_k) so that it may begin while the kernel before it on the stream
// is finishing.  Each kernel therefore calls pdl_wait() in every block
// before its first access to global memory (it returns once the previous
// grid has completed and its writes are visible; a kernel that ran without
// the overlap returns at once), and then pdl_trigger() to let the next
// kernel's blocks be placed as soon as all of its own blocks have started.
// Only shared memory may be touched before pdl_wait().
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_trigger();
}

// ---------------------------------------------------------------------------
// Debug build (compiled with -DTLC_DEBUG; build.py --debug makes
// libtlc_debug.so).  Bounds checks that never fault: a failing check records
// its location (source line | translation unit << 16) in this translation
// unit's device word, first failure kept, and the access it guards is
// skipped.  TLC_BOUND(c) guards a clamp that every build needs (c is always
// evaluated; valid inputs never fail it, so the debug build records when it
// does); TLC_CHECK(c) guards an index the code keeps in bounds by
// construction (evaluated in the debug build only).  The host reads the
// words through tlc_debug_fault().
// ---------------------------------------------------------------------------
#ifndef TLC_TU
#define TLC_TU 0
#endif
#ifdef TLC_DEBUG
static __device__ uint32_t g_tlc_debug_fault;  // one per translation unit
__device__ __forceinline__ bool debug_check(bool ok, uint32_t where) {
  if (!ok) atomicCAS(&g_tlc_debug_fault, 0u, where);
  return ok;
}
#define TLC_BOUND(c) (::tlc::debug_check((c), (uint32_t)__LINE__ | ((uint32_t)TLC_TU << 16)))
#define TLC_CHECK(c) (::tlc::debug_check((c), (uint32_t)__LINE__ | ((uint32_t)TLC_TU << 16)))
// Host side: this translation unit's word, optionally cleared.
#define TLC_DEFINE_DEBUG_READER(fn)                                  \
  uint32_t fn(bool reset) {                                          \
    uint32_t v = 0;                                                  \
    if (cudaMemcpyFromSymbol(&v, g_tlc_debug_fault, 4) != cudaSuccess) \
      v = 0xffffffffu;                                               \
    if (reset) {                                                     \
      const uint32_t z = 0;                                          \
      (void)cudaMemcpyToSymbol(g_tlc_debug_fault, &z, 4);            \
    }                                                                \
    return v;                                                        \
  }
#else
#define TLC_BOUND(c) (c)
#define TLC_CHECK(c) (true)
#define TLC_DEFINE_DEBUG_READER(fn) \
  uint32_t fn(bool) { return 0u; }
#endif

// Record a data-dependent failure; the first error wins, zero is never written.
__device__ __forceinline__ void report(int32_t *dev_status, int code) {
  if (dev_status) atomicCAS(reinterpret_cast<int *>(dev_status), 0, code);
}

// Poll a status word until its flag is set, at most `max_polls` times.
// Returns the word, or kFlagPrefix with value 0 after giving up (the caller
// then reports TLC_ERR_TIMEOUT; the result is wrong but every write stays
// in bounds, and later tiles can still finish).
__device__ __forceinline__ uint64_t wait_flag(const uint64_t *p, uint32_t max_polls,
                                              bool &timed_out) {
  uint64_t w = ld_relaxed_u64(p);
  uint32_t polls = 0;
  unsigned ns = 32;
  while ((w >> kFlagShift) == 0) {
    if (++polls >= max_polls) {
      timed_out = true;
      return kFlagPrefix;
    }
    __nanosleep(ns);
    if (ns < 512) ns <<= 1;
    w = ld_relaxed_u64(p);
  }
  return w;
}

// Look-back window: each lane of the looking-back warp reads V consecutive
// status words per round trip (32 * V tiles per trip): the words
// end - (lane*V + j), j = 0..V-1 (nearest first), with every load issued
// before any is waited on; indices below 0 read as `origin` (an inclusive
// prefix).  Then it waits (bounded) for any word that has no flag yet.
template <int V>
__device__ __forceinline__ void load_window(const uint64_t *status, int64_t end, uint64_t origin,
                                            uint32_t max_polls, bool &timed_out, uint64_t (&w)[V]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int64_t idx = end - (int64_t)(lane * V + j);
    w[j] = idx >= 0 ? ld_relaxed_u64(status + idx) : origin;
  }
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int64_t idx = end - (int64_t)(lane * V + j);
    if ((w[j] >> kFlagShift) == 0) w[j] = wait_flag(status + idx, max_polls, timed_out);
  }
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scans for blocks of kThreads threads (multiple of 32).
// `scratch` needs kThreads/32 + 1 words of shared memory.  Every thread
// receives the block total as well.
// ---------------------------------------------------------------------------
template <int kThreads>
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t v, uint32_t *scratch,
                                                        uint32_t &total) {
  constexpr int kWarps = kThreads / kWarp;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    uint32_t t = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += t;
  }
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kWarps ? scratch[lane] : 0;
    uint32_t wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      uint32_t t = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += t;
    }
    if (lane < kWarps) scratch[lane] = wi - w;   // exclusive warp offsets
    if (lane == kWarps - 1) scratch[kWarps] = wi;
  }
  __syncthreads();
  uint32_t r = scratch[warp] + inc - v;
  total = scratch[kWarps];
  __syncthreads();
  return r;
}

// Exclusive max-scan of signed values (identity -1); also returns the block max.
template <int kThreads>
__device__ __forceinline__ int32_t block_exclusive_max(int32_t v, int32_t *scratch,
                                                       int32_t &total) {
  constexpr int kWarps = kThreads / kWarp;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int32_t t = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc = max(inc, t);
  }
  int32_t exc_in_warp = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) exc_in_warp = -1;
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < kWarps ? scratch[lane] : -1;
    int32_t wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int32_t t = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi = max(wi, t);
    }
    int32_t we = __shfl_up_sync(0xffffffffu, wi, 1);
    if (lane == 0) we = -1;
    if (lane < kWarps) scratch[lane] = we;
    if (lane == kWarps - 1) scratch[kWarps] = wi;
  }
  __syncthreads();
  int32_t r = max(scratch[warp], exc_in_warp);
  total = scratch[kWarps];
  __syncthreads();
  return r;
}

}  // namespace tlc
