// tlc_internal.h -- host-side interfaces between the C ABI (tlc_api.cu) and
// the kernel files.  Not installed; not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <utility>

namespace tlc {

// The per-call record of a compression (same layout as the public
// tlc_compress_record): written by the kernels, on the device.
struct CompressRecord {
  uint32_t m_bits;
  float scale;
  uint64_t nonzeros;
  uint64_t length;
};

// Per-device facts, queried once per device and cached for the process.
struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int occ_quant_vec = 0;
  int occ_quant_scalar = 0;
  int occ_decode_write = 0;
  int occ_decode_acc = 0;
  int occ_quant_batch = 0;
  int occ_decode_batch_write = 0;
  int occ_decode_batch_acc = 0;
  int occ_decode_batch_ix_write = 0;
  int occ_decode_batch_ix_acc = 0;
  int occ_decode_ix[5] = {};  // warp units (write, accumulate); sums of 2, 4, 8 streams
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

// The deferred-placement path appends, after the look-back layout (whose
// status words hold the tiles' summaries and the chunk and span counters
// there): the placement chunks' summaries (compress_place_chunks u64), the
// spans' summaries (compress_place_spans u64), a finite-step word, and a
// staging slot of compress_stage_bytes_per_tile() bytes per tile.
struct DeferredScratch {
  uint64_t *cagg;
  uint64_t *sagg;
  uint32_t *ok;
  uint8_t *stage;
};

// Staging bytes per tile of the deferred-placement path (one tile's groups).
uint32_t compress_stage_bytes_per_tile();
// Placement chunks (32 tiles) and spans (32 chunks) of the deferred path
// for n_tiles tiles.
uint32_t compress_place_chunks(uint32_t n_tiles);
uint32_t compress_place_spans(uint32_t n_tiles);

inline size_t deferred_head_bytes(uint32_t n_tiles) {
  return align_up(8 * ((size_t)compress_place_chunks(n_tiles) + compress_place_spans(n_tiles)) + 4,
                  256);
}

inline size_t deferred_scratch_bytes(uint32_t n_part, uint32_t n_tiles) {
  return compress_scratch_bytes(n_part, n_tiles) + deferred_head_bytes(n_tiles) +
         (size_t)n_tiles * compress_stage_bytes_per_tile();
}

inline DeferredScratch deferred_scratch_layout(void *base, uint32_t n_part, uint32_t n_tiles) {
  DeferredScratch d;
  char *p = static_cast<char *>(base) + compress_scratch_bytes(n_part, n_tiles);
  d.cagg = reinterpret_cast<uint64_t *>(p);
  d.sagg = d.cagg + compress_place_chunks(n_tiles);
  d.ok = reinterpret_cast<uint32_t *>(d.sagg + compress_place_spans(n_tiles));
  d.stage = reinterpret_cast<uint8_t *>(p + deferred_head_bytes(n_tiles));
  return d;
}

// ---- tensor lists (plans) ---------------------------------------------------
// Values per block of the batched magnitude pass (a multiple of 4 * 512).
constexpr uint32_t kBatchChunk = 8192;

// One tensor of a plan, as the batched kernels see it (device memory).
struct BatchTensor {
  const float *x;
  float *err;
  float *y;              // decompress target (or accumulation buffer)
  uint64_t n, groups;
  uint64_t arena_off;    // the tensor's stream slot in the arena
  uint64_t cap;          // slot size = 4 + ceil(n/5)
  uint32_t q_tile_begin, q_tiles;  // compress tiles (global numbering)
  uint32_t q_chunk_begin;          // 32-tile chunks of the deferred placement
  uint32_t d_tile_begin, d_tiles;  // decode 512-byte units (global numbering, upper
                                   // bound of the tiles of either mode)
  uint32_t d_chunk_begin, d_chunks;  // 64-unit chunks of the index (same)
  uint32_t vec_q;        // x and err 16-byte aligned
  uint32_t vec_y;        // y 16-byte aligned
};

// Per-tensor facts of one batched decode, written by the prepare kernel.
struct BatchPrep {
  uint64_t m;            // payload length (0 when the stream is corrupt)
  float scale;
  uint32_t act_begin;    // first tile in the compact numbering
  uint32_t cact_begin;   // first index chunk in the compact numbering
  uint32_t valid;        // the stream's length and header are valid
};

struct BatchChunk {
  uint32_t tensor;
  uint32_t pad;
  uint64_t start;        // first value of the chunk
};

// Device-side view of a plan: descriptor tables and scratch.
struct BatchPlanDev {
  const BatchTensor *tensors;
  uint32_t count;
  const BatchChunk *chunks;
  uint32_t n_chunks;
  const uint32_t *q_tile_tensor;
  uint32_t n_q_tiles;
  const uint32_t *d_tile_tensor;
  uint32_t n_d_tiles;
  uint32_t *mbits;        // per-tensor max bits
  uint32_t *q_ticket;
  uint64_t *q_status;
  void *q_zero_base;      // mbits, q_ticket and q_status, contiguous
  size_t q_zero_bytes;
  uint32_t *d_ticket;
  uint32_t *d_ok;         // indexed plans: per-tensor valid flags
  uint64_t *d_status;     // small plans: look-back words, one per unit
  void *d_zero_base;      // d_ticket, d_ok and d_status, contiguous (small plans
                          // clear them before each decode)
  size_t d_zero_bytes;
  BatchPrep *d_prep;      // count entries, rewritten by every decode call
  uint32_t *d_total;      // compact tile and chunk counts of the current decode call
  bool q_deferred;        // compress with deferred placement (n_q_tiles >= threshold)
  uint64_t *q_cagg;       // deferred placement: per 32-tile chunk summaries,
  uint8_t *q_stage;       // and the staged bytes, compress_stage_bytes_per_tile() per tile;
  uint32_t n_q_chunks;    // tile summaries and chunk counters sit in q_status
  const uint32_t *q_chunk_tensor;  // deferred placement: the tensor of each chunk
  uint32_t *d_loc;        // indexed plans: units' first groups within their chunk (per
                          // tensor d_tiles words from d_tile_begin)
  uint32_t *d_cpre;       // and chunks' first groups (per tensor d_chunks + 1 words from
                          // d_chunk_begin + tensor index)
  uint32_t n_d_chunks;
};

cudaError_t launch_compress_batch(const DeviceInfo &dev, const BatchPlanDev &p, float s,
                                  uint8_t *arena, uint64_t *out_lens, int32_t *dev_status,
                                  uint32_t max_polls, cudaStream_t stream);
cudaError_t launch_decode_batch(const DeviceInfo &dev, const BatchPlanDev &p,
                                const uint8_t *arena, const uint64_t *in_lens, bool accumulate,
                                int32_t *dev_status, uint32_t max_polls, cudaStream_t stream);
int occupancy_quant_batch();
int occupancy_decode_batch(bool accumulate, bool indexed);
uint32_t decode_tile_payload_bytes(bool accumulate);

// Per-device facts for device d (initialised on first use); nullptr on error.
const DeviceInfo *device_info(int d);
// The current cross-block wait limit (polls).
uint32_t wait_limit();

// Kernel kinds for the optional per-launch timing (see tlc_kernel_timing).
enum KernelKind { kKindAbsmax = 0, kKindQuantZre, kKindDecodeWrite, kKindDecodeAccumulate,
                  kKindZrePlace, kKindDecodeCount, kKindDecodePrepare, kKindCount };
// Launch a kernel that may overlap the end of the kernel before it on the
// stream (programmatic stream serialization); the kernel waits for that
// kernel's completion itself (pdl_wait) before touching global memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t stream, Args &&...args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

void timing_begin(int kind, cudaStream_t stream);
void timing_end(int kind, cudaStream_t stream);

uint32_t compress_tiles(uint64_t n);
uint32_t compress_partials(const DeviceInfo &dev, uint64_t n);
// Whether tlc_compress takes the deferred-placement path for n values, and
// whether a plan does, for its total tile count.
bool compress_deferred(uint64_t n);
bool compress_deferred_tiles(uint64_t n_tiles);
// Scratch bytes of one compress call.
size_t compress_scratch_bytes_for(const DeviceInfo &dev, uint64_t n, bool deferred);
// deferred: tiles stage their bytes and two small kernels place them (the
// scratch must then be compress_scratch_bytes_for(.., true) bytes); else
// tiles place their bytes themselves with a look-back over earlier tiles.
// rec: nullptr, or the call's record (device-writable).
cudaError_t launch_compress(const DeviceInfo &dev, const float *x, uint64_t n, float s, float *err,
                            uint8_t *out, uint64_t out_cap, uint64_t *out_len,
                            int32_t *dev_status, uint32_t max_polls, void *scratch,
                            cudaStream_t stream, bool deferred, CompressRecord *rec = nullptr);
int occupancy_quant(bool vec);

// Decode of one small stream (look-back): scratch of decode_scratch_words(
// tiles) u64 words, tiles = decode_tiles_max(cap, groups) 512-byte payload
// units (every tile is a whole number of units): status[tiles] then the
// ticket; all zero before the launch.
// Streams whose capacity spans decode_deferred(tiles) units or more, and
// sums of several streams, go through the index instead
// (launch_decode_indexed).
constexpr uint32_t kDecodeUnit = 512;
constexpr uint32_t kDecodeChunkUnits = 64;
uint32_t decode_tiles_max(uint64_t cap, uint64_t groups);
bool decode_deferred(uint32_t tiles);
inline size_t decode_scratch_words(uint32_t tiles) { return (size_t)tiles + 1; }

cudaError_t launch_decode(const DeviceInfo &dev, const uint8_t *in, const uint64_t *len_dev,
                          uint64_t cap, uint64_t n, float *y, bool accumulate,
                          int32_t *dev_status, uint32_t max_polls, uint64_t *scratch,
                          cudaStream_t stream);

// Indexed decode of up to kIndexPass streams of n values each: the index
// (a count and a scan launch), then one decode launch (dense output: exactly
// one stream; accumulate of one stream) or, for a sum of several streams
// (added in order), an entries launch and a sum-tile launch.  The scratch is
// indexed_layout(..).total_bytes bytes; nothing in it needs clearing.
constexpr int kIndexPass = 8;
struct IndexedStream {
  const uint8_t *in;
  const uint64_t *len_dev;  // or nullptr: cap is the exact length
  uint64_t cap;
};
struct IndexedLayout {
  size_t loc_off[kIndexPass], cpre_off[kIndexPass];
  size_t eloc_off[kIndexPass], ecpre_off[kIndexPass], list_off[kIndexPass], tfe_off[kIndexPass];
  size_t total_bytes;
};
IndexedLayout indexed_layout(const IndexedStream *s, int k, uint64_t n);
cudaError_t launch_decode_indexed(const DeviceInfo &dev, const IndexedStream *s, int k, uint64_t n,
                                  float *y, bool accumulate, int32_t *dev_status,
                                  uint32_t max_polls, void *scratch, cudaStream_t stream);
void occupancy_decode_ix(int occ[5]);
cudaError_t launch_wait_test(uint64_t *status, uint32_t max_polls, int32_t *dev_status,
                             cudaStream_t stream);
cudaError_t launch_compress_wait_test(uint64_t *status, uint32_t max_polls, int32_t *dev_status,
                                      cudaStream_t stream);
int occupancy_decode(bool accumulate);

}  // namespace tlc
