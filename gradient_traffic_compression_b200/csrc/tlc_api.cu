// tlc_api.cu -- the C ABI (include/tlc.h): argument checks, scratch
// allocation from a per-device stream-ordered pool, and kernel launches.
// No host synchronisation happens here; all data-dependent checks run on the
// device and report through *dev_status.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/tlc.h"
#include "tlc_internal.h"

namespace {

constexpr uint32_t kDefaultPolls = 1u << 22;
std::atomic<uint32_t> g_wait_limit{0};

uint32_t wait_limit() {
  const uint32_t v = g_wait_limit.load(std::memory_order_relaxed);
  return v ? v : kDefaultPolls;
}

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
tlc::DeviceInfo g_dev[kMaxDevices];
cudaError_t g_dev_err[kMaxDevices];

void init_device(int d) {
  tlc::DeviceInfo &di = g_dev[d];
  cudaError_t e = cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, d);
  if (e == cudaSuccess) {
    di.occ_quant_vec = tlc::occupancy_quant(true);
    di.occ_quant_scalar = tlc::occupancy_quant(false);
    di.occ_decode_write = tlc::occupancy_decode(false);
    di.occ_decode_acc = tlc::occupancy_decode(true);
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = d;
    e = cudaMemPoolCreate(&di.pool, &props);
    if (e == cudaSuccess) {
      // keep freed scratch in the pool between calls
      uint64_t keep = UINT64_MAX;
      e = cudaMemPoolSetAttribute(di.pool, cudaMemPoolAttrReleaseThreshold, &keep);
    }
  }
  di.device = d;
  if (e == cudaSuccess) e = cudaGetLastError();
  g_dev_err[d] = e;
}

const tlc::DeviceInfo *current_device(cudaError_t &err) {
  int d = 0;
  err = cudaGetDevice(&d);
  if (err != cudaSuccess) return nullptr;
  if (d < 0 || d >= kMaxDevices) {
    err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::call_once(g_dev_once[d], init_device, d);
  err = g_dev_err[d];
  return err == cudaSuccess ? &g_dev[d] : nullptr;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

bool n_ok(size_t n) { return n >= 1 && n < (size_t(1) << 32); }

size_t groups_of(size_t n) { return (n + 4) / 5; }

// Stream-ordered scratch from the library's pool.
cudaError_t scratch_alloc(const tlc::DeviceInfo &dev, size_t bytes, void **p, cudaStream_t st) {
  return cudaMallocFromPoolAsync(p, bytes, dev.pool, st);
}

// ---- optional per-kernel timing -------------------------------------------
struct Timing {
  std::mutex mu;
  std::atomic<bool> on{false};
  struct Pending {
    int kind;
    cudaEvent_t b, e;
  };
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> spare;
  cudaEvent_t open_begin[tlc::kKindCount] = {};
  uint64_t launches[tlc::kKindCount] = {};
  double ms[tlc::kKindCount] = {};

  cudaEvent_t get() {
    if (!spare.empty()) {
      cudaEvent_t ev = spare.back();
      spare.pop_back();
      return ev;
    }
    cudaEvent_t ev = nullptr;
    cudaEventCreate(&ev);
    return ev;
  }
};
Timing g_timing;

const char *const kKindNames[tlc::kKindCount] = {"k_absmax", "k_quant_zre", "k_decode_write",
                                                 "k_decode_accumulate"};

}  // namespace

namespace tlc {
const DeviceInfo *device_info(int d) {
  if (d < 0 || d >= kMaxDevices) return nullptr;
  std::call_once(g_dev_once[d], init_device, d);
  return g_dev_err[d] == cudaSuccess ? &g_dev[d] : nullptr;
}
uint32_t wait_limit() { return ::wait_limit(); }

void timing_begin(int kind, cudaStream_t stream) {
  if (!g_timing.on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_timing.mu);
  cudaEvent_t ev = g_timing.get();
  cudaEventRecord(ev, stream);
  g_timing.open_begin[kind] = ev;
}
void timing_end(int kind, cudaStream_t stream) {
  if (!g_timing.on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_timing.mu);
  cudaEvent_t b = g_timing.open_begin[kind];
  if (!b) return;
  cudaEvent_t e = g_timing.get();
  cudaEventRecord(e, stream);
  g_timing.pending.push_back({kind, b, e});
  g_timing.open_begin[kind] = nullptr;
}
}  // namespace tlc

extern "C" {

void tlc_kernel_timing(int enable) {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  if (enable) {
    for (int k = 0; k < tlc::kKindCount; ++k) {
      g_timing.launches[k] = 0;
      g_timing.ms[k] = 0.0;
    }
  }
  g_timing.on.store(enable != 0, std::memory_order_relaxed);
}

int tlc_kernel_timing_read(uint64_t *launches, double *total_ms, int max_kinds) {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  for (auto &p : g_timing.pending) {
    float ms = 0.0f;
    if (cudaEventSynchronize(p.e) == cudaSuccess && cudaEventElapsedTime(&ms, p.b, p.e) == cudaSuccess) {
      g_timing.launches[p.kind] += 1;
      g_timing.ms[p.kind] += ms;
    }
    g_timing.spare.push_back(p.b);
    g_timing.spare.push_back(p.e);
  }
  g_timing.pending.clear();
  for (int k = 0; k < tlc::kKindCount && k < max_kinds; ++k) {
    if (launches) launches[k] = g_timing.launches[k];
    if (total_ms) total_ms[k] = g_timing.ms[k];
  }
  return tlc::kKindCount;
}

const char *tlc_kernel_name(int kind) {
  return (kind >= 0 && kind < tlc::kKindCount) ? kKindNames[kind] : nullptr;
}


size_t tlc_compress_bound(size_t n) { return n_ok(n) ? 4 + groups_of(n) : 0; }

const char *tlc_status_string(tlc_status s) {
  switch (s) {
    case TLC_OK: return "ok";
    case TLC_ERR_INVALID_ARG: return "invalid argument";
    case TLC_ERR_NONFINITE: return "non-finite value in x + err, or M*s overflows";
    case TLC_ERR_CORRUPT: return "corrupt stream";
    case TLC_ERR_TIMEOUT: return "cross-block wait timed out";
    case TLC_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char *tlc_version(void) { return "0.1.0"; }

void tlc_set_wait_limit(uint32_t max_polls) {
  g_wait_limit.store(max_polls, std::memory_order_relaxed);
}

tlc_status tlc_compress(const float *x, size_t n, float s, float *err, uint8_t *out,
                        size_t out_cap, uint64_t *out_len, int32_t *dev_status,
                        tlc_stream_t stream) {
  if (!x || !err || !out || !out_len || !n_ok(n)) return TLC_ERR_INVALID_ARG;
  if (!(s >= 1.0f && s < 2.0f)) return TLC_ERR_INVALID_ARG;  // also rejects NaN
  if (out_cap < tlc_compress_bound(n)) return TLC_ERR_INVALID_ARG;
  const size_t fb = n * sizeof(float);
  if (overlaps(x, fb, err, fb) || overlaps(x, fb, out, out_cap) || overlaps(err, fb, out, out_cap))
    return TLC_ERR_INVALID_ARG;

  cudaError_t ce;
  const tlc::DeviceInfo *dev = current_device(ce);
  if (!dev) return TLC_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t n_tiles = tlc::compress_tiles(n);
  const uint32_t n_part = tlc::compress_partials(*dev, n);
  void *scratch = nullptr;
  if (scratch_alloc(*dev, tlc::compress_scratch_bytes(n_part, n_tiles), &scratch, st) !=
      cudaSuccess)
    return TLC_ERR_CUDA;
  int32_t *status_ptr =
      dev_status ? dev_status : tlc::compress_scratch_layout(scratch, n_part, n_tiles).spare_status;
  ce = tlc::launch_compress(*dev, x, n, s, err, out, out_cap, out_len, status_ptr, wait_limit(),
                            scratch, st);
  const cudaError_t fe = cudaFreeAsync(scratch, st);
  return (ce == cudaSuccess && fe == cudaSuccess) ? TLC_OK : TLC_ERR_CUDA;
}

static tlc_status check_stream_arg(const uint8_t *in, size_t cap, bool len_on_device, size_t n) {
  if (!in || !n_ok(n) || cap < 4) return TLC_ERR_INVALID_ARG;
  if (!len_on_device && cap - 4 > groups_of(n)) return TLC_ERR_INVALID_ARG;
  return TLC_OK;
}

tlc_status tlc_decompress(const uint8_t *in, const uint64_t *in_len, size_t in_cap, size_t n,
                          float *y, int32_t *dev_status, tlc_stream_t stream) {
  if (!y) return TLC_ERR_INVALID_ARG;
  tlc_status v = check_stream_arg(in, in_cap, in_len != nullptr, n);
  if (v != TLC_OK) return v;
  if (overlaps(in, in_cap, y, n * sizeof(float))) return TLC_ERR_INVALID_ARG;

  cudaError_t ce;
  const tlc::DeviceInfo *dev = current_device(ce);
  if (!dev) return TLC_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t tiles = tlc::decode_tiles_max(in_cap, groups_of(n));
  const size_t words = tlc::decode_scratch_words(tiles);
  const size_t bytes = tlc::align_up(8 * words + 8, 256);
  void *scratch = nullptr;
  if (scratch_alloc(*dev, bytes, &scratch, st) != cudaSuccess) return TLC_ERR_CUDA;
  uint64_t *status = static_cast<uint64_t *>(scratch);
  int32_t *status_ptr = dev_status ? dev_status : reinterpret_cast<int32_t *>(status + words);
  ce = cudaMemsetAsync(scratch, 0, 8 * words, st);
  if (ce == cudaSuccess)
    ce = tlc::launch_decode(*dev, in, in_len, in_cap, n, y, false, status_ptr, wait_limit(),
                            status, reinterpret_cast<uint32_t *>(status + tiles), st);
  const cudaError_t fe = cudaFreeAsync(scratch, st);
  return (ce == cudaSuccess && fe == cudaSuccess) ? TLC_OK : TLC_ERR_CUDA;
}

tlc_status tlc_decompress_accumulate(const uint8_t *const *ins, const uint64_t *in_lens,
                                     const size_t *in_caps, int k, size_t n, float *acc,
                                     int32_t *dev_status, tlc_stream_t stream) {
  if (!ins || !in_caps || !acc || k < 1 || !n_ok(n)) return TLC_ERR_INVALID_ARG;
  for (int w = 0; w < k; ++w) {
    tlc_status v = check_stream_arg(ins[w], in_caps[w], in_lens != nullptr, n);
    if (v != TLC_OK) return v;
    if (overlaps(ins[w], in_caps[w], acc, n * sizeof(float))) return TLC_ERR_INVALID_ARG;
  }
  cudaError_t ce;
  const tlc::DeviceInfo *dev = current_device(ce);
  if (!dev) return TLC_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t g = groups_of(n);
  size_t total_words = 0;
  for (int w = 0; w < k; ++w)
    total_words += tlc::decode_scratch_words(tlc::decode_tiles_max(in_caps[w], g));
  const size_t bytes = tlc::align_up(8 * total_words + 8, 256);
  void *scratch = nullptr;
  if (scratch_alloc(*dev, bytes, &scratch, st) != cudaSuccess) return TLC_ERR_CUDA;
  uint64_t *base = static_cast<uint64_t *>(scratch);
  int32_t *status_ptr = dev_status ? dev_status : reinterpret_cast<int32_t *>(base + total_words);
  ce = cudaMemsetAsync(scratch, 0, 8 * total_words, st);
  size_t at = 0;
  for (int w = 0; w < k && ce == cudaSuccess; ++w) {
    const uint32_t tiles = tlc::decode_tiles_max(in_caps[w], g);
    uint64_t *status = base + at;
    ce = tlc::launch_decode(*dev, ins[w], in_lens ? in_lens + w : nullptr, in_caps[w], n, acc,
                            true, status_ptr, wait_limit(), status,
                            reinterpret_cast<uint32_t *>(status + tiles), st);
    at += tlc::decode_scratch_words(tiles);
  }
  const cudaError_t fe = cudaFreeAsync(scratch, st);
  return (ce == cudaSuccess && fe == cudaSuccess) ? TLC_OK : TLC_ERR_CUDA;
}

tlc_status tlc_test_wait_timeout(uint32_t max_polls, int32_t *dev_status, tlc_stream_t stream) {
  if (!max_polls || !dev_status) return TLC_ERR_INVALID_ARG;
  cudaError_t ce;
  const tlc::DeviceInfo *dev = current_device(ce);
  if (!dev) return TLC_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void *scratch = nullptr;
  if (scratch_alloc(*dev, 256, &scratch, st) != cudaSuccess) return TLC_ERR_CUDA;
  ce = cudaMemsetAsync(scratch, 0, 256, st);
  if (ce == cudaSuccess)
    ce = tlc::launch_wait_test(static_cast<uint64_t *>(scratch), max_polls, dev_status, st);
  const cudaError_t fe = cudaFreeAsync(scratch, st);
  return (ce == cudaSuccess && fe == cudaSuccess) ? TLC_OK : TLC_ERR_CUDA;
}

}  // extern "C"
