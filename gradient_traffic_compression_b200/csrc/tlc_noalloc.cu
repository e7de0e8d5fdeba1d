// tlc_noalloc.cu -- tlc_compress_noalloc: compression without any device
// allocation, for callers that cannot allocate device memory (see tlc.h).
//
// The two compress kernels need a little scratch: one 64-bit status word per
// compress tile (2048 byte groups), a tile ticket, and one partial maximum
// per block of the magnitude pass.  Here that scratch is a fixed array in the
// library's own device memory instead of a stream-ordered allocation.
#include <atomic>
#include <cstring>
#include <mutex>

#include "../../include/tlc.h"
#include "tlc_internal.h"

namespace {

// The scratch, in every device that loads the library, for the life of the
// process.  512 KiB holds the status words of n <= TLC_NOALLOC_MAX_N (52,429
// tiles) plus the partial maxima of devices with up to 3000 SMs.
constexpr size_t kScratchBytes = 512 * 1024;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
std::atomic<void *> g_scratch_ptr[kMaxDevices];

// Host code may not use g_noalloc_scratch as an address (on the host it only
// names the symbol); ask the runtime for the device address while that
// device is current.  The address is kept only once it has been obtained: a
// failed attempt (for example before the device has a context) returns
// nullptr, clears the runtime's last-error slot, and the next call tries
// again.
void *scratch_for_device(int d) {
  void *p = g_scratch_ptr[d].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lk(g_mu);
  p = g_scratch_ptr[d].load(std::memory_order_relaxed);
  if (p) return p;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return nullptr;
  }
  g_scratch_ptr[d].store(p, std::memory_order_release);
  return p;
}

}  // namespace

extern "C" tlc_status tlc_compress_noalloc(const float *x, size_t n, float s, float *err,
                                           uint8_t *out, size_t out_cap, uint64_t *out_len,
                                           int32_t *dev_status, tlc_stream_t stream) {
  if (!x || !err || !out || !out_len || n == 0 || n > TLC_NOALLOC_MAX_N)
    return TLC_ERR_INVALID_ARG;
  if (!(s >= 1.0f && s < 2.0f)) return TLC_ERR_INVALID_ARG;
  if (out_cap < tlc_compress_bound(n)) return TLC_ERR_INVALID_ARG;
  const size_t fb = n * sizeof(float);
  const auto ov = [](const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
  };
  if (ov(x, fb, err, fb) || ov(x, fb, out, out_cap) || ov(err, fb, out, out_cap))
    return TLC_ERR_INVALID_ARG;

  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return TLC_ERR_CUDA;
  const tlc::DeviceInfo *dev = tlc::device_info(d);
  if (!dev) return TLC_ERR_CUDA;
  void *scratch = scratch_for_device(d);
  if (!scratch) return TLC_ERR_CUDA;

  const uint32_t n_tiles = tlc::compress_tiles(n);
  const uint32_t n_part = tlc::compress_partials(*dev, n);
  if (tlc::compress_scratch_bytes(n_part, n_tiles) > kScratchBytes) return TLC_ERR_INVALID_ARG;
  // k_absmax clears the status words and the ticket before k_quant_zre reads
  // them, and writes every partial maximum that k_quant_zre reads, so nothing
  // left from an earlier call is used.
  int32_t *status_ptr =
      dev_status ? dev_status : tlc::compress_scratch_layout(scratch, n_part, n_tiles).spare_status;
  // the static scratch holds the look-back layout only, at any size
  const cudaError_t ce = tlc::launch_compress(*dev, x, n, s, err, out, out_cap, out_len,
                                              status_ptr, tlc::wait_limit(), scratch,
                                              reinterpret_cast<cudaStream_t>(stream), false);
  return ce == cudaSuccess ? TLC_OK : TLC_ERR_CUDA;
}
