// tlc_internal.h -- host-side interfaces between the C ABI (tlc_api.cu) and
// the kernel files.  Not installed; not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace tlc {

// Per-device facts, queried once per device and cached for the process.
struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int occ_quant_vec = 0;
  int occ_quant_scalar = 0;
  int occ_decode_write = 0;
  int occ_decode_acc = 0;
  cudaMemPool_t pool = nullptr;
};

// Scratch of one compress call, carved out of one stream-ordered allocation:
//   status[n_tiles] (u64, zeroed by k_absmax), ticket (u64 slot right after,
//   zeroed with it), partial[n_part] (u32), a spare status word.
struct CompressScratch {
  uint64_t *status;
  uint32_t *ticket;
  uint32_t *partial;
  int32_t *spare_status;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline size_t compress_scratch_bytes(uint32_t n_part, uint32_t n_tiles) {
  return align_up(8 * ((size_t)n_tiles + 1) + 4 * (size_t)n_part + 4, 256);
}

inline CompressScratch compress_scratch_layout(void *base, uint32_t n_part, uint32_t n_tiles) {
  CompressScratch s;
  s.status = static_cast<uint64_t *>(base);
  s.ticket = reinterpret_cast<uint32_t *>(s.status + n_tiles);
  s.partial = reinterpret_cast<uint32_t *>(s.status + n_tiles + 1);
  s.spare_status = reinterpret_cast<int32_t *>(s.partial + n_part);
  return s;
}

// Per-device facts for device d (initialised on first use); nullptr on error.
const DeviceInfo *device_info(int d);
// The current cross-block wait limit (polls).
uint32_t wait_limit();

// Kernel kinds for the optional per-launch timing (see tlc_kernel_timing).
enum KernelKind { kKindAbsmax = 0, kKindQuantZre, kKindDecodeWrite, kKindDecodeAccumulate,
                  kKindCount };
void timing_begin(int kind, cudaStream_t stream);
void timing_end(int kind, cudaStream_t stream);

uint32_t compress_tiles(uint64_t n);
uint32_t compress_partials(const DeviceInfo &dev, uint64_t n);
cudaError_t launch_compress(const DeviceInfo &dev, const float *x, uint64_t n, float s, float *err,
                            uint8_t *out, uint64_t out_cap, uint64_t *out_len,
                            int32_t *dev_status, uint32_t max_polls, void *scratch,
                            cudaStream_t stream);
int occupancy_quant(bool vec);

// Decode scratch per stream: status[tiles] (u64) then the ticket (u64 slot);
// both must be zero before the launch.
uint32_t decode_tiles_max(uint64_t cap, uint64_t groups);
inline size_t decode_scratch_words(uint32_t tiles) { return (size_t)tiles + 1; }
cudaError_t launch_decode(const DeviceInfo &dev, const uint8_t *in, const uint64_t *len_dev,
                          uint64_t cap, uint64_t n, float *y, bool accumulate,
                          int32_t *dev_status, uint32_t max_polls, uint64_t *status,
                          uint32_t *ticket, cudaStream_t stream);
cudaError_t launch_wait_test(uint64_t *status, uint32_t max_polls, int32_t *dev_status,
                             cudaStream_t stream);
int occupancy_decode(bool accumulate);

}  // namespace tlc
