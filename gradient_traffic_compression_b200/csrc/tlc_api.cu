// tlc_api.cu -- the C ABI (include/tlc.h): argument checks, scratch
// allocation from a per-device stream-ordered pool, and kernel launches.
// No host synchronisation happens here; all data-dependent checks run on the
// device and report through *dev_status.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstddef>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/tlc.h"
#define TLC_TU 3
#include "tlc_device.cuh"
#include "tlc_internal.h"
#include <nvtx3/nvToolsExt.h>

namespace tlc {
TLC_DEFINE_DEBUG_READER(debug_fault_api)
uint32_t debug_fault_compress(bool reset);
uint32_t debug_fault_decode(bool reset);

#ifdef TLC_DEBUG
// Debug build: every scratch allocation gets kCanary bytes of 0xA5 on both
// sides; after the call's kernels, this kernel checks them.
constexpr size_t kCanary = 256;
__global__ void k_check_canaries(const uint8_t *base, size_t bytes) {
  for (size_t i = threadIdx.x; i < kCanary; i += blockDim.x) {
    (void)TLC_CHECK(base[i] == 0xA5);
    (void)TLC_CHECK(base[kCanary + bytes + i] == 0xA5);
  }
}
#endif
}  // namespace tlc

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
    di.occ_quant_batch = tlc::occupancy_quant_batch();
    di.occ_decode_batch_write = tlc::occupancy_decode_batch(false, false);
    di.occ_decode_batch_acc = tlc::occupancy_decode_batch(true, false);
    di.occ_decode_batch_ix_write = tlc::occupancy_decode_batch(false, true);
    di.occ_decode_batch_ix_acc = tlc::occupancy_decode_batch(true, true);
    tlc::occupancy_decode_ix(di.occ_decode_ix);
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

// A named NVTX range around each call that enqueues work, so profilers and
// timeline tools show the calls around their kernels (no cost without one).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

// Stream-ordered scratch from the library's pool.  (The debug build adds
// canaries on both sides and checks them when the scratch is freed.)
struct Scratch {
  void *base = nullptr;
  size_t bytes = 0;
};

cudaError_t scratch_alloc(const tlc::DeviceInfo &dev, size_t bytes, void **p, cudaStream_t st,
                          Scratch &sc) {
  sc.bytes = bytes;
#ifdef TLC_DEBUG
  cudaError_t e = cudaMallocFromPoolAsync(&sc.base, bytes + 2 * tlc::kCanary, dev.pool, st);
  if (e != cudaSuccess) return e;
  char *b = static_cast<char *>(sc.base);
  e = cudaMemsetAsync(b, 0xA5, tlc::kCanary, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(b + tlc::kCanary + bytes, 0xA5, tlc::kCanary, st);
  *p = b + tlc::kCanary;
  return e;
#else
  cudaError_t e = cudaMallocFromPoolAsync(&sc.base, bytes, dev.pool, st);
  *p = sc.base;
  return e;
#endif
}

cudaError_t scratch_free(Scratch &sc, cudaStream_t st) {
  if (!sc.base) return cudaSuccess;
#ifdef TLC_DEBUG
  tlc::k_check_canaries<<<1, 256, 0, st>>>(static_cast<const uint8_t *>(sc.base), sc.bytes);
#endif
  const cudaError_t e = cudaFreeAsync(sc.base, st);
  sc.base = nullptr;
  return e;
}

// ---- optional per-kernel timing -------------------------------------------
struct Timing {
  std::mutex mu;
  std::atomic<bool> on{false};
  uint32_t kinds = ~0u;  // kinds that get an event pair
  struct Pending {
    int kind;
    cudaEvent_t b, e;
  };
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> spare;
  cudaEvent_t open_begin[tlc::kKindCount] = {};
  uint64_t launches[tlc::kKindCount] = {};  // every launch while on
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

const char *const kKindNames[tlc::kKindCount] = {
    "k_absmax",    "k_quant_zre",    "k_decode_write",        "k_decode_accumulate",
    "k_zre_place", "k_decode_count", "k_decode_batch_prepare"};

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
  g_timing.launches[kind] += 1;
  if (!((g_timing.kinds >> kind) & 1u)) return;
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

void tlc_kernel_timing_kinds(uint32_t mask) {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  g_timing.kinds = mask;
}

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
    if (cudaEventSynchronize(p.e) == cudaSuccess && cudaEventElapsedTime(&ms, p.b, p.e) == cudaSuccess)
      g_timing.ms[p.kind] += ms;
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

const char *tlc_version(void) { return "0.2.0"; }

int tlc_debug_build(void) {
#ifdef TLC_DEBUG
  return 1;
#else
  return 0;
#endif
}

uint32_t tlc_debug_fault(int reset) {
  const uint32_t f[3] = {tlc::debug_fault_api(reset != 0), tlc::debug_fault_compress(reset != 0),
                         tlc::debug_fault_decode(reset != 0)};
  for (uint32_t v : f)
    if (v) return v;
  return 0;
}

void tlc_set_wait_limit(uint32_t max_polls) {
  g_wait_limit.store(max_polls, std::memory_order_relaxed);
}

static_assert(sizeof(tlc_compress_record) == sizeof(tlc::CompressRecord) &&
                  offsetof(tlc_compress_record, nonzeros) ==
                      offsetof(tlc::CompressRecord, nonzeros) &&
                  offsetof(tlc_compress_record, length) == offsetof(tlc::CompressRecord, length),
              "the public record and the kernels' record share one layout");

static tlc_status compress_call(const float *x, size_t n, float s, float *err, uint8_t *out,
                                size_t out_cap, uint64_t *out_len, int32_t *dev_status,
                                tlc::CompressRecord *rec, tlc_stream_t stream) {
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
  void *scratch = nullptr;
  Scratch sc;
  const bool deferred = tlc::compress_deferred(n);
  const size_t bytes = tlc::compress_scratch_bytes_for(*dev, n, deferred);
  if (scratch_alloc(*dev, bytes + 256, &scratch, st, sc) != cudaSuccess) return TLC_ERR_CUDA;
  // a status word for calls without one, past everything the kernels use
  int32_t *status_ptr =
      dev_status ? dev_status : reinterpret_cast<int32_t *>(static_cast<char *>(scratch) + bytes);
  ce = tlc::launch_compress(*dev, x, n, s, err, out, out_cap, out_len, status_ptr, wait_limit(),
                            scratch, st, deferred, rec);
  const cudaError_t fe = scratch_free(sc, st);
  return (ce == cudaSuccess && fe == cudaSuccess) ? TLC_OK : TLC_ERR_CUDA;
}

tlc_status tlc_compress(const float *x, size_t n, float s, float *err, uint8_t *out,
                        size_t out_cap, uint64_t *out_len, int32_t *dev_status,
                        tlc_stream_t stream) {
  NvtxRange nvtx("tlc_compress");
  return compress_call(x, n, s, err, out, out_cap, out_len, dev_status, nullptr, stream);
}

tlc_status tlc_compress_recorded(const float *x, size_t n, float s, float *err, uint8_t *out,
                                 size_t out_cap, uint64_t *out_len, int32_t *dev_status,
                                 tlc_compress_record *record, tlc_stream_t stream) {
  NvtxRange nvtx("tlc_compress_recorded");
  if (!record) return TLC_ERR_INVALID_ARG;
  return compress_call(x, n, s, err, out, out_cap, out_len, dev_status,
                       reinterpret_cast<tlc::CompressRecord *>(record), stream);
}

static tlc_status check_stream_arg(const uint8_t *in, size_t cap, bool len_on_device, size_t n) {
  if (!in || !n_ok(n) || cap < 4) return TLC_ERR_INVALID_ARG;
  if (!len_on_device && cap - 4 > groups_of(n)) return TLC_ERR_INVALID_ARG;
  return TLC_OK;
}

tlc_status tlc_decompress(const uint8_t *in, const uint64_t *in_len, size_t in_cap, size_t n,
                          float *y, int32_t *dev_status, tlc_stream_t stream) {
  NvtxRange nvtx("tlc_decompress");
  if (!y) return TLC_ERR_INVALID_ARG;
  tlc_status v = check_stream_arg(in, in_cap, in_len != nullptr, n);
  if (v != TLC_OK) return v;
  if (overlaps(in, in_cap, y, n * sizeof(float))) return TLC_ERR_INVALID_ARG;

  cudaError_t ce;
  const tlc::DeviceInfo *dev = current_device(ce);
  if (!dev) return TLC_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t tiles = tlc::decode_tiles_max(in_cap, groups_of(n));
  void *scratch = nullptr;
  Scratch sc;
  if (tlc::decode_deferred(tiles)) {
    // large stream: index, then decode
    const tlc::IndexedStream is = {in, in_len, in_cap};
    const size_t bytes = tlc::indexed_layout(&is, 1, n).total_bytes;
    if (scratch_alloc(*dev, bytes + 256, &scratch, st, sc) != cudaSuccess) return TLC_ERR_CUDA;
    int32_t *status_ptr =
        dev_status ? dev_status : reinterpret_cast<int32_t *>(static_cast<char *>(scratch) + bytes);
    ce = tlc::launch_decode_indexed(*dev, &is, 1, n, y, false, status_ptr, wait_limit(), scratch,
                                    st);
  } else {
    // small stream: one launch, tiles find their place by a look-back
    const size_t words = tlc::decode_scratch_words(tiles);
    const size_t bytes = tlc::align_up(8 * words + 8, 256);
    if (scratch_alloc(*dev, bytes, &scratch, st, sc) != cudaSuccess) return TLC_ERR_CUDA;
    uint64_t *status = static_cast<uint64_t *>(scratch);
    int32_t *status_ptr = dev_status ? dev_status : reinterpret_cast<int32_t *>(status + words);
    ce = cudaMemsetAsync(scratch, 0, 8 * words, st);
    if (ce == cudaSuccess)
      ce = tlc::launch_decode(*dev, in, in_len, in_cap, n, y, false, status_ptr, wait_limit(),
                              status, st);
  }
  const cudaError_t fe = scratch_free(sc, st);
  return (ce == cudaSuccess && fe == cudaSuccess) ? TLC_OK : TLC_ERR_CUDA;
}

tlc_status tlc_decompress_accumulate(const uint8_t *const *ins, const uint64_t *in_lens,
                                     const size_t *in_caps, int k, size_t n, float *acc,
                                     int32_t *dev_status, tlc_stream_t stream) {
  NvtxRange nvtx("tlc_decompress_accumulate");
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
  void *scratch = nullptr;
  Scratch sc;
  const uint32_t tiles0 = tlc::decode_tiles_max(in_caps[0], g);
  if (k == 1 && !tlc::decode_deferred(tiles0)) {
    // one small stream: one launch with a look-back
    const size_t words = tlc::decode_scratch_words(tiles0);
    const size_t bytes = tlc::align_up(8 * words + 8, 256);
    if (scratch_alloc(*dev, bytes, &scratch, st, sc) != cudaSuccess) return TLC_ERR_CUDA;
    uint64_t *base = static_cast<uint64_t *>(scratch);
    int32_t *status_ptr = dev_status ? dev_status : reinterpret_cast<int32_t *>(base + words);
    ce = cudaMemsetAsync(scratch, 0, 8 * words, st);
    if (ce == cudaSuccess)
      ce = tlc::launch_decode(*dev, ins[0], in_lens, in_caps[0], n, acc, true, status_ptr,
                              wait_limit(), base, st);
  } else {
    // index + one read-modify-write of acc per pass of up to kIndexPass
    // streams; passes run in stream order on `stream`, so the sum keeps
    // the worker order
    const int passes = (k + tlc::kIndexPass - 1) / tlc::kIndexPass;
    std::vector<tlc::IndexedStream> is(k);
    for (int w = 0; w < k; ++w) is[w] = {ins[w], in_lens ? in_lens + w : nullptr, in_caps[w]};
    size_t bytes = 0;
    for (int p = 0; p < passes; ++p) {
      const int kp = std::min(tlc::kIndexPass, k - p * tlc::kIndexPass);
      bytes = std::max(bytes, tlc::indexed_layout(&is[p * tlc::kIndexPass], kp, n).total_bytes);
    }
    if (scratch_alloc(*dev, bytes + 256, &scratch, st, sc) != cudaSuccess) return TLC_ERR_CUDA;
    int32_t *status_ptr =
        dev_status ? dev_status : reinterpret_cast<int32_t *>(static_cast<char *>(scratch) + bytes);
    ce = cudaSuccess;
    for (int p = 0; p < passes && ce == cudaSuccess; ++p) {
      const int kp = std::min(tlc::kIndexPass, k - p * tlc::kIndexPass);
      ce = tlc::launch_decode_indexed(*dev, &is[p * tlc::kIndexPass], kp, n, acc, true,
                                      status_ptr, wait_limit(), scratch, st);
    }
  }
  const cudaError_t fe = scratch_free(sc, st);
  return (ce == cudaSuccess && fe == cudaSuccess) ? TLC_OK : TLC_ERR_CUDA;
}

// ---- plans: a fixed list of tensors, one launch set per step ---------------

}  // extern "C"

struct tlc_plan_s {
  int device = -1;
  int count = 0;
  std::vector<uint64_t> offsets;  // count + 1 arena offsets
  bool has_inputs = false, has_outputs = false;
  void *dmem = nullptr;
  tlc::BatchPlanDev dev{};
  int32_t *spare_status = nullptr;
};

extern "C" {

tlc_status tlc_plan_create(int count, const size_t *ns, const float *const *xs,
                           float *const *errs, float *const *ys, tlc_plan *plan) {
  if (!plan) return TLC_ERR_INVALID_ARG;
  *plan = nullptr;
  if (count < 1 || !ns || (!xs && !ys) || (xs && !errs) || (!xs && errs))
    return TLC_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (!n_ok(ns[i])) return TLC_ERR_INVALID_ARG;
    if (xs && (!xs[i] || !errs[i])) return TLC_ERR_INVALID_ARG;
    if (ys && !ys[i]) return TLC_ERR_INVALID_ARG;
    const size_t fb = ns[i] * sizeof(float);
    if (xs && overlaps(xs[i], fb, errs[i], fb)) return TLC_ERR_INVALID_ARG;
  }
  cudaError_t ce;
  const tlc::DeviceInfo *dev = current_device(ce);
  if (!dev) return TLC_ERR_CUDA;

  std::vector<tlc::BatchTensor> T(count);
  std::vector<tlc::BatchChunk> chunks;
  std::vector<uint32_t> qtt, dtt, qct;
  std::vector<uint64_t> offsets(count + 1, 0);
  uint64_t n_dchunks = 0, n_qchunks = 0;
  for (int i = 0; i < count; ++i) {
    tlc::BatchTensor &t = T[i];
    t.x = xs ? xs[i] : nullptr;
    t.err = xs ? errs[i] : nullptr;
    t.y = ys ? ys[i] : nullptr;
    t.n = ns[i];
    t.groups = groups_of(ns[i]);
    t.cap = 4 + t.groups;
    t.arena_off = offsets[i];
    offsets[i + 1] = tlc::align_up(offsets[i] + t.cap, 16);
    t.q_tile_begin = (uint32_t)qtt.size();
    t.q_tiles = tlc::compress_tiles(t.n);
    for (uint32_t k = 0; k < t.q_tiles; ++k) qtt.push_back((uint32_t)i);
    t.q_chunk_begin = (uint32_t)n_qchunks;
    n_qchunks += tlc::compress_place_chunks(t.q_tiles);
    for (uint32_t k = 0; k < tlc::compress_place_chunks(t.q_tiles); ++k) qct.push_back((uint32_t)i);
    t.d_tile_begin = (uint32_t)dtt.size();
    t.d_tiles = tlc::decode_tiles_max(t.cap, t.groups);  // 512-byte units
    for (uint32_t k = 0; k < t.d_tiles; ++k) dtt.push_back((uint32_t)i);
    t.d_chunk_begin = (uint32_t)n_dchunks;
    t.d_chunks = (t.d_tiles + tlc::kDecodeChunkUnits - 1) / tlc::kDecodeChunkUnits;
    n_dchunks += t.d_chunks;
    t.vec_q = xs && (((reinterpret_cast<uintptr_t>(t.x) | reinterpret_cast<uintptr_t>(t.err)) &
                      15) == 0);
    t.vec_y = ys && ((reinterpret_cast<uintptr_t>(t.y) & 15) == 0);
    for (uint64_t b = 0; b < t.n; b += tlc::kBatchChunk) chunks.push_back({(uint32_t)i, 0u, b});
    if (qtt.size() >= (1ull << 31) || dtt.size() >= (1ull << 31) ||
        chunks.size() >= (1ull << 31) || n_dchunks + count >= (1ull << 31))
      return TLC_ERR_INVALID_ARG;
  }
  // device layout: tables, then the zeroed-per-call scratch of each direction
  const size_t sz_T = tlc::align_up(sizeof(tlc::BatchTensor) * count, 256);
  const size_t sz_C = tlc::align_up(sizeof(tlc::BatchChunk) * chunks.size(), 256);
  const size_t sz_Q = tlc::align_up(4 * qtt.size(), 256);
  const size_t sz_D = tlc::align_up(4 * dtt.size(), 256);
  const size_t sz_M = tlc::align_up(4 * (size_t)count + 8, 256);      // mbits, q_ticket
  const size_t sz_QS = tlc::align_up(8 * qtt.size(), 256);
  // decode: the ticket, per-tensor valid flags and (small plans, zeroed per
  // call) one look-back word per unit
  const bool d_ix = tlc::decode_deferred((uint32_t)dtt.size());
  const size_t d_head = tlc::align_up(4 + 4 * (size_t)count, 8);
  const size_t sz_DS = tlc::align_up(d_head + (d_ix ? 0 : 8 * dtt.size()), 256);
  const size_t sz_P = tlc::align_up(sizeof(tlc::BatchPrep) * count + 8, 256);  // prep, total
  // the index of indexed plans: units' first groups in their chunk, chunks'
  // first groups
  const size_t sz_E = d_ix ? tlc::align_up(4 * dtt.size(), 256) : 0;
  const size_t sz_S = d_ix ? tlc::align_up(4 * (n_dchunks + count), 256) : 0;
  // deferred placement of the compress side: chunk summaries, staging
  const bool q_def = xs && tlc::compress_deferred_tiles(qtt.size());
  const size_t sz_QC = q_def ? tlc::align_up(8 * n_qchunks, 256) : 0;
  const size_t sz_QT = q_def ? (size_t)tlc::compress_stage_bytes_per_tile() * qtt.size() : 0;
  const size_t sz_QCT = q_def ? tlc::align_up(4 * n_qchunks, 256) : 0;  // each chunk's tensor
  const size_t total = sz_T + sz_C + sz_Q + sz_D + sz_M + sz_QS + sz_DS + sz_P + 256 + sz_E +
                       sz_S + sz_QC + sz_QT + sz_QCT;
  tlc_plan_s *P = new tlc_plan_s();
  P->device = dev->device;
  P->count = count;
  P->offsets = offsets;
  P->has_inputs = xs != nullptr;
  P->has_outputs = ys != nullptr;
  if (cudaMalloc(&P->dmem, total) != cudaSuccess) {
    delete P;
    return TLC_ERR_CUDA;
  }
  char *b = static_cast<char *>(P->dmem);
  tlc::BatchPlanDev &D = P->dev;
  D.tensors = reinterpret_cast<tlc::BatchTensor *>(b);
  D.count = (uint32_t)count;
  D.chunks = reinterpret_cast<tlc::BatchChunk *>(b + sz_T);
  D.n_chunks = (uint32_t)chunks.size();
  D.q_tile_tensor = reinterpret_cast<uint32_t *>(b + sz_T + sz_C);
  D.n_q_tiles = (uint32_t)qtt.size();
  D.d_tile_tensor = reinterpret_cast<uint32_t *>(b + sz_T + sz_C + sz_Q);
  D.n_d_tiles = (uint32_t)dtt.size();
  char *zq = b + sz_T + sz_C + sz_Q + sz_D;
  D.mbits = reinterpret_cast<uint32_t *>(zq);
  D.q_ticket = reinterpret_cast<uint32_t *>(zq + 4 * (size_t)count);
  D.q_status = reinterpret_cast<uint64_t *>(zq + sz_M);
  D.q_zero_base = zq;
  D.q_zero_bytes = sz_M + 8 * qtt.size();
  char *zd = zq + sz_M + sz_QS;
  D.d_ticket = reinterpret_cast<uint32_t *>(zd);
  D.d_ok = reinterpret_cast<uint32_t *>(zd + 4);
  D.d_status = d_ix ? nullptr : reinterpret_cast<uint64_t *>(zd + d_head);
  D.d_zero_base = zd;
  D.d_zero_bytes = d_head + (d_ix ? 0 : 8 * dtt.size());
  D.d_prep = reinterpret_cast<tlc::BatchPrep *>(zd + sz_DS);
  D.d_total = reinterpret_cast<uint32_t *>(zd + sz_DS + sizeof(tlc::BatchPrep) * count);
  P->spare_status = reinterpret_cast<int32_t *>(zd + sz_DS + sz_P);
  D.d_loc = d_ix ? reinterpret_cast<uint32_t *>(zd + sz_DS + sz_P + 256) : nullptr;
  D.d_cpre = d_ix ? reinterpret_cast<uint32_t *>(zd + sz_DS + sz_P + 256 + sz_E) : nullptr;
  D.n_d_chunks = (uint32_t)n_dchunks;
  D.q_deferred = q_def;
  D.q_cagg = q_def ? reinterpret_cast<uint64_t *>(zd + sz_DS + sz_P + 256 + sz_E + sz_S) : nullptr;
  D.q_stage = q_def ? reinterpret_cast<uint8_t *>(zd + sz_DS + sz_P + 256 + sz_E + sz_S + sz_QC)
                    : nullptr;
  D.n_q_chunks = (uint32_t)n_qchunks;
  uint32_t *qct_dev = q_def ? reinterpret_cast<uint32_t *>(b + total - sz_QCT) : nullptr;
  D.q_chunk_tensor = qct_dev;
  ce = cudaMemcpy(b, T.data(), sizeof(tlc::BatchTensor) * count, cudaMemcpyHostToDevice);
  if (ce == cudaSuccess && !chunks.empty())
    ce = cudaMemcpy(b + sz_T, chunks.data(), sizeof(tlc::BatchChunk) * chunks.size(),
                    cudaMemcpyHostToDevice);
  if (ce == cudaSuccess)
    ce = cudaMemcpy(b + sz_T + sz_C, qtt.data(), 4 * qtt.size(), cudaMemcpyHostToDevice);
  if (ce == cudaSuccess)
    ce = cudaMemcpy(b + sz_T + sz_C + sz_Q, dtt.data(), 4 * dtt.size(), cudaMemcpyHostToDevice);
  if (ce == cudaSuccess && q_def)
    ce = cudaMemcpy(qct_dev, qct.data(), 4 * qct.size(), cudaMemcpyHostToDevice);
  if (ce != cudaSuccess) {
    cudaFree(P->dmem);
    delete P;
    return TLC_ERR_CUDA;
  }
  *plan = P;
  return TLC_OK;
}

void tlc_plan_destroy(tlc_plan plan) {
  if (!plan) return;
  int cur = -1;
  cudaGetDevice(&cur);
  if (cur != plan->device) cudaSetDevice(plan->device);
  cudaFree(plan->dmem);
  if (cur >= 0 && cur != plan->device) cudaSetDevice(cur);
  delete plan;
}

size_t tlc_plan_arena_bytes(tlc_plan plan) { return plan ? plan->offsets.back() : 0; }

size_t tlc_plan_stream_offset(tlc_plan plan, int i) {
  if (!plan || i < 0 || i >= plan->count) return (size_t)-1;
  return plan->offsets[i];
}

static const tlc::DeviceInfo *plan_device(tlc_plan plan) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != plan->device) return nullptr;
  return tlc::device_info(cur);
}

tlc_status tlc_compress_batch(tlc_plan plan, float s, uint8_t *arena, uint64_t *out_lens,
                              int32_t *dev_status, tlc_stream_t stream) {
  NvtxRange nvtx("tlc_compress_batch");
  if (!plan || !plan->has_inputs || !arena || !out_lens) return TLC_ERR_INVALID_ARG;
  if (!(s >= 1.0f && s < 2.0f)) return TLC_ERR_INVALID_ARG;
  const tlc::DeviceInfo *dev = plan_device(plan);
  if (!dev) return TLC_ERR_INVALID_ARG;
  const cudaError_t ce = tlc::launch_compress_batch(
      *dev, plan->dev, s, arena, out_lens, dev_status ? dev_status : plan->spare_status,
      wait_limit(), reinterpret_cast<cudaStream_t>(stream));
  return ce == cudaSuccess ? TLC_OK : TLC_ERR_CUDA;
}

tlc_status tlc_decompress_batch(tlc_plan plan, const uint8_t *arena, const uint64_t *in_lens,
                                int accumulate, int32_t *dev_status, tlc_stream_t stream) {
  NvtxRange nvtx("tlc_decompress_batch");
  if (!plan || !plan->has_outputs || !arena || !in_lens) return TLC_ERR_INVALID_ARG;
  const tlc::DeviceInfo *dev = plan_device(plan);
  if (!dev) return TLC_ERR_INVALID_ARG;
  const cudaError_t ce = tlc::launch_decode_batch(
      *dev, plan->dev, arena, in_lens, accumulate != 0,
      dev_status ? dev_status : plan->spare_status, wait_limit(),
      reinterpret_cast<cudaStream_t>(stream));
  return ce == cudaSuccess ? TLC_OK : TLC_ERR_CUDA;
}

static tlc_status run_wait_test(bool compress_side, uint32_t max_polls, int32_t *dev_status,
                                tlc_stream_t stream) {
  if (!max_polls || !dev_status) return TLC_ERR_INVALID_ARG;
  cudaError_t ce;
  const tlc::DeviceInfo *dev = current_device(ce);
  if (!dev) return TLC_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void *scratch = nullptr;
  Scratch sc;
  if (scratch_alloc(*dev, 256, &scratch, st, sc) != cudaSuccess) return TLC_ERR_CUDA;
  ce = cudaMemsetAsync(scratch, 0, 256, st);
  if (ce == cudaSuccess)
    ce = compress_side
             ? tlc::launch_compress_wait_test(static_cast<uint64_t *>(scratch), max_polls,
                                              dev_status, st)
             : tlc::launch_wait_test(static_cast<uint64_t *>(scratch), max_polls, dev_status, st);
  const cudaError_t fe = scratch_free(sc, st);
  return (ce == cudaSuccess && fe == cudaSuccess) ? TLC_OK : TLC_ERR_CUDA;
}

tlc_status tlc_test_wait_timeout(uint32_t max_polls, int32_t *dev_status, tlc_stream_t stream) {
  return run_wait_test(false, max_polls, dev_status, stream);
}

tlc_status tlc_test_compress_wait_timeout(uint32_t max_polls, int32_t *dev_status,
                                          tlc_stream_t stream) {
  return run_wait_test(true, max_polls, dev_status, stream);
}

}  // extern "C"
