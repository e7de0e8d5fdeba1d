// tlc_decode.cu -- decompression kernels for the 3LC pipeline on sm_100a.
//
// Source: review page "3LC: Lightweight and Effective Traffic Compression for
// Distributed Machine Learning".  Decoding inverts "Proposed method" bullets
// 3 (zero-run encoding), 2 (quartic encoding) and 1 (dequantization to
// q * M * s); the Abstract's exchange of state changes between nodes is the
// receive side, where several workers' streams are summed.
//
// One kernel, k_decode, in two modes:
//   kWrite       dense output: y_i = +scale, -scale or +0.0
//   kAccumulate  acc_i += y_i only where q_i != 0 (acc keeps its bits at
//                zeros), one launch per worker stream, in worker order
// A tile is 1024 (kWrite) or 2048 (kAccumulate) payload bytes.  Per tile:
// expansion counts e_k (an escape byte b >= 243 stands for b - 241 groups of
// 121, any other byte for itself), a block scan, and a decoupled look-back
// over earlier tiles for the tile's first group index O.  The tile's groups
// are then expanded in shared memory (at most 14 bytes per payload byte) and
// walked as float4 columns with coalesced 128-bit accesses: written in kWrite
// mode, read-modify-written (all-zero columns skipped) in kAccumulate mode.
// An accumulate tile made mostly of escapes instead visits only its literal
// groups, so there work and traffic follow the non-zeros.
// For streams whose capacity holds 16384 or more 512-byte units (8 MiB), a
// counting kernel, k_decode_count, first writes the group count of every
// unit and of every 32-unit chunk; each tile then sums the counts before it
// (every thread a strided share) instead of looking back.  No tile waits on
// another, which measured 0.789 -> 0.459 ms (dense output) and 0.629 ->
// 0.505 ms (accumulate) on a dense 2^28-value stream, and 0.189 -> 0.178 /
// 0.040 -> 0.026 ms on the sparse config-3 stream, for about 0.011 ms per
// counting launch.  Below that size the extra launch costs more than the
// look-back on sparse streams.
// Every write is clamped to the ceil(n/5) groups of the tensor; a stream that
// does not expand to exactly that many groups is reported as corrupt.
#include "tlc_device.cuh"
#include "tlc_internal.h"

namespace tlc {

// Payload bytes per thread (1, 2 or a multiple of 4): small tiles balance the dense
// write mode best; the accumulate mode touches little memory per tile and
// prefers fewer, larger tiles.
#ifndef TLC_D_BYTES_WRITE
#define TLC_D_BYTES_WRITE 2
#endif
#ifndef TLC_D_BYTES_ACC
#define TLC_D_BYTES_ACC 8
#endif
constexpr int kDThreads = 256;
constexpr int kWrite = 0, kAccumulate = 1;
template <int kMode>
struct DecodeShape {
  static constexpr int kBytes = kMode == kWrite ? TLC_D_BYTES_WRITE : TLC_D_BYTES_ACC;
  static constexpr int kTile = kDThreads * kBytes;   // payload bytes per tile
  static constexpr int kMaxGroups = kTile * 14;      // largest expansion of a tile
};
#ifndef TLC_D_LOOKV
#define TLC_D_LOOKV 1
#endif
constexpr int kLookV = TLC_D_LOOKV;   // look-back words per lane per round trip
// Streams whose capacity allows this many 512-byte units or more get their
// tile prefixes from a counting pass (k_decode_count) instead of a look-back.
#ifndef TLC_DEFER_DECODE_MIN_TILES
#define TLC_DEFER_DECODE_MIN_TILES 16384
#endif
constexpr uint32_t kDecodeDeferMinTiles = TLC_DEFER_DECODE_MIN_TILES;
static_assert(kDecodeDeferMinTiles >= 4, "the deferred layout fits in tiles + 1 words");

size_t decode_smem_bytes(bool accumulate);

struct DecodeArgs {
  uint32_t *ecount;        // deferred prefixes only: each 512-byte unit's group count
  uint64_t *csum;          // and each 32-unit chunk's
  const uint8_t *in;
  const uint64_t *len_dev;
  uint64_t cap;
  uint64_t n;
  uint64_t groups;
  float *y;
  uint64_t *status;
  uint32_t *ticket;
  int32_t *dev_status;
  uint32_t max_polls;
};

__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
  return v;
}

// Exclusive prefix (in groups) of tile u, by warp 0.  Publishes the tile's
// aggregate first and its inclusive prefix last.  Each round trip reads
// 32 * kLookV earlier tiles' words.
__device__ uint64_t lookback_sum(uint64_t *status, uint32_t u, uint64_t E, uint32_t max_polls,
                                 bool &timed_out) {
  const int lane = threadIdx.x & 31;
  if (u == 0) {
    if (lane == 0) st_relaxed_u64(status, kFlagPrefix | E);
    return 0;
  }
  if (lane == 0) st_relaxed_u64(status + u, kFlagAgg | E);
  uint64_t sum = 0;
  int64_t end = (int64_t)u - 1;
  for (;;) {
    uint64_t w[kLookV];
    load_window(status, end, kFlagPrefix, max_polls, timed_out, w);
    // nearest prefix of this lane, and the sum up to and including it
    int jp = kLookV;
    uint64_t part = 0;
#pragma unroll
    for (int j = 0; j < kLookV; ++j) {
      if (jp == kLookV) {
        part += w[j] & kValueMask;
        if ((w[j] >> kFlagShift) == 2) jp = j;
      }
    }
    const uint32_t pmask = __ballot_sync(0xffffffffu, jp < kLookV);
    if (pmask) {
      const int pl = __ffs(pmask) - 1;
      sum += warp_sum_u64(lane <= pl ? part : 0);
      break;
    }
    sum += warp_sum_u64(part);
    end -= kWarp * kLookV;
  }
  if (lane == 0) st_relaxed_u64(status + u, kFlagPrefix | (sum + E));
  return sum;
}

// Base-3 digits of a quartic byte, two bits each; digit k belongs to the
// k-th value of the group (the first value is the most significant digit).
__device__ __forceinline__ uint16_t digits_of(uint32_t v) {
  const uint32_t d0 = v / 81u, d1 = (v / 27u) % 3u, d2 = (v / 9u) % 3u, d3 = (v / 3u) % 3u,
                 d4 = v % 3u;
  return (uint16_t)(d0 | (d1 << 2) | (d2 << 4) | (d3 << 6) | (d4 << 8));
}

__device__ __forceinline__ float dequant(uint32_t dig, float scale) {
  return dig == 1u ? 0.0f : (dig == 2u ? scale : -scale);
}

// One stream's decode job, as the tile function sees it.
struct DecodeJob {
  const uint8_t *payload;  // stream bytes after the 4-byte header
  uint64_t m;              // payload length
  uint64_t n, groups;
  float scale;
  float *y;                // output (kWrite) or accumulation buffer
  uint64_t *status;        // this stream's tile status words
  uint32_t n_tiles;        // tiles actually present: ceil(m / tile)
  bool vec;                // y is 16-byte aligned
  const uint32_t *ecount;  // deferred prefixes: group count per 512-byte unit
  const uint64_t *csum;    // and per chunk of kDecodeChunkUnits units
};

// Deferred prefixes: the first group index of the tile that starts at
// payload unit `unit` is the sum of the counts that k_decode_count wrote for
// the chunks before the unit's chunk and for the units before it in its
// chunk.  Every thread of the block sums a strided share; the result is this
// warp's partial sum (in every lane).  No wait.
__device__ __forceinline__ uint64_t prefix_share(const uint32_t *ecount, const uint64_t *csum,
                                                 uint32_t unit) {
  const uint32_t c = unit / kDecodeChunkUnits;
  uint64_t s = 0;
  for (uint32_t i = threadIdx.x; i < c; i += kDThreads) s += csum[i];
  const uint32_t t0 = c * kDecodeChunkUnits;
  if (threadIdx.x < kDecodeChunkUnits && t0 + threadIdx.x < unit) s += ecount[t0 + threadIdx.x];
  return warp_sum_u64(s);
}

struct DecodeSmem {
  uint16_t lut[256];       // base-3 digits of every quartic byte
  uint32_t scan[kDThreads / kWarp + 1];
  uint64_t o;
  uint64_t part[kDThreads / kWarp];  // per-warp partial prefixes (counting pass)
};

// Validate a stream (length and header) and return its payload length and
// scale.  Corrupt when the length is below 4 or above the readable capacity,
// the payload would be longer than the tensor's groups or empty, or the
// header is negative or not finite.
__device__ __forceinline__ bool read_stream_header(const uint8_t *in, const uint64_t *len_dev,
                                                   uint64_t cap, uint64_t groups, uint64_t &m,
                                                   float &scale) {
  const uint64_t L = len_dev ? *len_dev : cap;
  if (L < 4 || L > cap || L - 4 > groups || L == 4) return false;
  const uint32_t hb = (uint32_t)in[0] | ((uint32_t)in[1] << 8) | ((uint32_t)in[2] << 16) |
                      ((uint32_t)in[3] << 24);
  if (hb >= 0x7f800000u) return false;  // negative, infinite or NaN scale
  m = L - 4;
  scale = __uint_as_float(hb);
  return true;
}

// One tile of one stream; the whole block calls it and it ends synchronised.
// kDeferred: the tile's first group index comes from k_decode_count's
// counts instead of a look-back.
template <int kMode, bool kDeferred = false>
__device__ __forceinline__ void decode_tile(const DecodeJob &j, uint32_t u, DecodeSmem &sm,
                                            uint8_t *grp_s, int32_t *dev_status,
                                            uint32_t max_polls) {
  constexpr int kDBytes = DecodeShape<kMode>::kBytes;
  constexpr int kDTile = DecodeShape<kMode>::kTile;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float scale = j.scale;

  // ---- load the tile's payload bytes, expansion counts, block scan -------
  const uint64_t b0 = (uint64_t)u * kDTile + (uint64_t)threadIdx.x * kDBytes;
  uint32_t bw[(kDBytes + 3) / 4];
#pragma unroll
  for (int k = 0; k < (kDBytes + 3) / 4; ++k) bw[k] = 0x79797979u;
  int nvalid = 0;
  if (kDBytes % 4 == 0 && b0 + kDBytes <= j.m &&
      ((reinterpret_cast<uintptr_t>(j.payload + b0) & 3) == 0)) {
    const uint32_t *p32 = reinterpret_cast<const uint32_t *>(j.payload + b0);
#pragma unroll
    for (int k = 0; k < kDBytes / 4; ++k) bw[k] = __ldg(p32 + k);
    nvalid = kDBytes;
  } else {
#pragma unroll
    for (int k = 0; k < kDBytes; ++k) {
      if (b0 + k < j.m) {
        const uint32_t b = __ldg(j.payload + b0 + k);
        bw[k >> 2] = (bw[k >> 2] & ~(0xffu << (8 * (k & 3)))) | (b << (8 * (k & 3)));
        nvalid = k + 1;
      }
    }
  }
  uint32_t esum = 0;
  bool mine_lit = false;  // a literal group other than the all-zero 121
#pragma unroll
  for (int k = 0; k < kDBytes; ++k) {
    const uint32_t b = (bw[k >> 2] >> (8 * (k & 3))) & 0xffu;
    if (k < nvalid) {
      esum += b >= 243u ? b - 241u : 1u;
      mine_lit = mine_lit || (b < 243u && b != 121u);
    }
  }
  uint32_t E;
  const uint32_t off = block_exclusive_sum<kDThreads>(esum, sm.scan, E);
  // A tile without non-zero literals decodes to zeros only: plain zero
  // stores (dense output) or nothing at all (accumulate).  Otherwise dense
  // output expands the tile's groups in shared memory; so does the
  // accumulate mode when the tile is mostly literals (then a coalesced
  // float4 pass over acc is cheapest), while for escape-heavy tiles it visits
  // only the literal groups.
  const bool any_lit = __syncthreads_or(mine_lit) != 0;
  const bool expand = any_lit && (kMode == kWrite || E <= 4u * (uint32_t)kDTile);

  // ---- the tile's first group index ---------------------------------------
  // Counting pass: every thread sums a strided share of the counts before
  // the tile, then all threads pre-fill the zero groups.  Look-back: warp 0
  // looks back while the other warps pre-fill.
  if (kDeferred) {
    static_assert(kDTile % kDecodeUnit == 0 && kDecodeChunkUnits % (kDTile / kDecodeUnit) == 0,
                  "tiles are whole units and never straddle a chunk");
    const uint64_t p = prefix_share(j.ecount, j.csum, u * (uint32_t)(kDTile / kDecodeUnit));
    if (lane == 0) sm.part[warp] = p;
    if (expand) {
      const uint32_t words = (E + 15) / 16;
      for (uint32_t w = threadIdx.x; w < words; w += kDThreads)
        reinterpret_cast<uint4 *>(grp_s)[w] =
            make_uint4(0x79797979u, 0x79797979u, 0x79797979u, 0x79797979u);
    }
  } else if (warp == 0) {
    bool timed_out = false;
    const uint64_t O = lookback_sum(j.status, u, E, max_polls, timed_out);
    if (__any_sync(0xffffffffu, timed_out) && lane == 0) report(dev_status, TLC_ERR_TIMEOUT);
    if (lane == 0) sm.o = O;
  } else if (expand) {
    const uint32_t words = (E + 15) / 16;
    for (uint32_t w = threadIdx.x - kWarp; w < words; w += kDThreads - kWarp)
      reinterpret_cast<uint4 *>(grp_s)[w] =
          make_uint4(0x79797979u, 0x79797979u, 0x79797979u, 0x79797979u);
  }
  __syncthreads();
  uint64_t O;
  if (kDeferred) {
    O = 0;
#pragma unroll
    for (int w = 0; w < kDThreads / kWarp; ++w) O += sm.part[w];
  } else {
    O = sm.o;
  }
  if (threadIdx.x == 0) {
    const bool last = (u == j.n_tiles - 1);
    if (O + E > j.groups || (last && O + E != j.groups)) report(dev_status, TLC_ERR_CORRUPT);
  }
  const uint64_t Ec = O >= j.groups ? 0 : umin64(E, j.groups - O);

  if (!any_lit) {
    if (kMode == kWrite) {
      const uint64_t e_begin = 5 * O;
      const uint64_t e_end = umin64(5 * (O + Ec), j.n);
      const uint64_t v0 = (e_begin + 3) / 4, v1 = e_end / 4;
      if (e_end > e_begin) {
        if (!j.vec || v1 <= v0) {
          for (uint64_t e = e_begin + threadIdx.x; e < e_end; e += kDThreads) j.y[e] = 0.0f;
        } else {
          float4 *y4 = reinterpret_cast<float4 *>(j.y);
          for (uint64_t v = v0 + threadIdx.x; v < v1; v += kDThreads)
            y4[v] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          if (threadIdx.x < 4) {
            const uint64_t e = e_begin + threadIdx.x;
            if (e < 4 * v0) j.y[e] = 0.0f;
          } else if (threadIdx.x < 8) {
            const uint64_t e = 4 * v1 + (threadIdx.x - 4);
            if (e < e_end) j.y[e] = 0.0f;
          }
        }
      }
    }
  } else if (expand) {
    // literal bytes into the expanded group buffer
    uint32_t pos = off;
#pragma unroll
    for (int k = 0; k < kDBytes; ++k) {
      const uint32_t b = (bw[k >> 2] >> (8 * (k & 3))) & 0xffu;
      if (k < nvalid) {
        if (b >= 243u) {
          pos += b - 241u;
        } else {
          grp_s[pos] = (uint8_t)b;
          ++pos;
        }
      }
    }
    __syncthreads();
    // groups [O, O+Ec) -> values [5 O, min(5 (O+Ec), n))
    const uint64_t e_begin = 5 * O;
    const uint64_t e_end = umin64(5 * (O + Ec), j.n);
    if (e_end > e_begin) {
      const uint32_t o32 = (uint32_t)O;
      // one value: written (dense output) or added where non-zero (accumulate)
      auto put = [&](uint64_t e) {
        const uint32_t e32 = (uint32_t)e;
        const uint32_t g = e32 / 5u;
        const uint32_t dig = (sm.lut[grp_s[g - o32]] >> (2 * (e32 - 5u * g))) & 3u;
        if (kMode == kWrite)
          j.y[e] = dequant(dig, scale);
        else if (dig != 1u)
          j.y[e] = __fadd_rn(j.y[e], dequant(dig, scale));
      };
      const uint64_t v0 = (e_begin + 3) / 4, v1 = e_end / 4;
      if (!j.vec || v1 <= v0) {
        for (uint64_t e = e_begin + threadIdx.x; e < e_end; e += kDThreads) put(e);
      } else {
        // Values 4v..4v+3 lie in group g = 4v/5 (digits d0..) and, when
        // d0 >= 2, spill into group g+1; both groups' digit words are joined
        // so one shift lines the four digits up.
        float4 *y4 = reinterpret_cast<float4 *>(j.y);
        for (uint64_t v = v0 + threadIdx.x; v < v1; v += kDThreads) {
          const uint32_t e0 = (uint32_t)(4 * v);
          const uint32_t g = e0 / 5u;
          const uint32_t d0 = e0 - 5u * g;
          const uint32_t li = g - o32;
          const uint32_t c0 = grp_s[li];
          const uint32_t c1 = d0 >= 2u ? (uint32_t)grp_s[li + 1] : 121u;
          if (kMode == kWrite) {
            float4 o;
            if (c0 == 121u && c1 == 121u) {
              o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            } else {
              const uint32_t w =
                  ((uint32_t)sm.lut[c0] | ((uint32_t)sm.lut[c1] << 10)) >> (2u * d0);
              o.x = dequant(w & 3u, scale);
              o.y = dequant((w >> 2) & 3u, scale);
              o.z = dequant((w >> 4) & 3u, scale);
              o.w = dequant((w >> 6) & 3u, scale);
            }
            y4[v] = o;
          } else if (c0 != 121u || c1 != 121u) {
            const uint32_t w = ((uint32_t)sm.lut[c0] | ((uint32_t)sm.lut[c1] << 10)) >> (2u * d0);
            if ((w & 0xffu) != 0x55u) {  // some of the four digits is not zero
              float4 o = y4[v];
              if ((w & 3u) != 1u) o.x = __fadd_rn(o.x, dequant(w & 3u, scale));
              if (((w >> 2) & 3u) != 1u) o.y = __fadd_rn(o.y, dequant((w >> 2) & 3u, scale));
              if (((w >> 4) & 3u) != 1u) o.z = __fadd_rn(o.z, dequant((w >> 4) & 3u, scale));
              if (((w >> 6) & 3u) != 1u) o.w = __fadd_rn(o.w, dequant((w >> 6) & 3u, scale));
              y4[v] = o;
            }
          }
        }
        if (threadIdx.x < 4) {
          const uint64_t e = e_begin + threadIdx.x;
          if (e < 4 * v0) put(e);
        } else if (threadIdx.x < 8) {
          const uint64_t e = 4 * v1 + (threadIdx.x - 4);
          if (e < e_end) put(e);
        }
      }
    }
  } else {
    // accumulate, escape-heavy tile: visit only literal groups other than
    // the all-zero 121; each group's (up to five) acc values are loaded
    // before any is added
    uint64_t g = O + off;
#pragma unroll
    for (int k = 0; k < kDBytes; ++k) {
      const uint32_t b = (bw[k >> 2] >> (8 * (k & 3))) & 0xffu;
      if (k < nvalid) {
        if (b >= 243u) {
          g += b - 241u;
        } else {
          if (b != 121u && g < j.groups) {
            const uint16_t dg = digits_of(b);
            float v[5];
#pragma unroll
            for (int d = 0; d < 5; ++d) {
              const uint64_t e = 5 * g + d;
              v[d] = (((dg >> (2 * d)) & 3u) != 1u && e < j.n) ? j.y[e] : 0.0f;
            }
#pragma unroll
            for (int d = 0; d < 5; ++d) {
              const uint32_t dig = (dg >> (2 * d)) & 3u;
              const uint64_t e = 5 * g + d;
              if (dig != 1u && e < j.n) j.y[e] = __fadd_rn(v[d], dequant(dig, scale));
            }
          }
          ++g;
        }
      }
    }
  }
  __syncthreads();
}

template <int kMode, bool kVec, bool kDeferred>
__global__ void __launch_bounds__(kDThreads)
k_decode(const DecodeArgs a) {
  constexpr int kDTile = DecodeShape<kMode>::kTile;
  extern __shared__ __align__(16) uint8_t grp_s[];  // kMaxGroups + 16 bytes
  __shared__ DecodeSmem sm;
  __shared__ uint64_t m_s;
  __shared__ uint32_t tile_s;
  __shared__ float scale_s;
  __shared__ int ok_s;

  if (threadIdx.x == 0) {
    uint64_t m = 0;
    float scale = 0.0f;
    ok_s = read_stream_header(a.in, a.len_dev, a.cap, a.groups, m, scale) ? 1 : 0;
    m_s = m;
    scale_s = scale;
  }
  for (int v = threadIdx.x; v < 256; v += kDThreads) sm.lut[v] = v < 243 ? digits_of(v) : 0;
  __syncthreads();
  if (!ok_s) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(a.dev_status, TLC_ERR_CORRUPT);
    return;
  }
  DecodeJob job;
  job.payload = a.in + 4;
  job.m = m_s;
  job.n = a.n;
  job.groups = a.groups;
  job.scale = scale_s;
  job.y = a.y;
  job.status = a.status;
  job.n_tiles = (uint32_t)((job.m + kDTile - 1) / kDTile);
  job.vec = kVec;
  job.ecount = a.ecount;
  job.csum = a.csum;
  for (;;) {
    if (threadIdx.x == 0) tile_s = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t u = tile_s;
    if (u >= job.n_tiles) break;
    decode_tile<kMode, kDeferred>(job, u, sm, grp_s, a.dev_status, a.max_polls);
  }
}

// Deferred prefixes, first pass, for chunk c of one stream: the group count
// of each of its 512-byte payload units (one warp per unit, one 32-bit word
// per lane, every word loaded before any is counted) and of the chunk.
// Whole block; ends synchronised.
constexpr int kUnitsPerWarp = kDecodeChunkUnits / (kDThreads / kWarp);
static_assert(kDecodeUnit == 4 * kWarp * 4, "four words per lane per unit");
__device__ __forceinline__ void count_chunk(const uint8_t *payload, uint64_t m, uint32_t c,
                                            uint32_t *ecount, uint64_t *csum, uint32_t *wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t n_units = (uint32_t)((m + kDecodeUnit - 1) / kDecodeUnit);
  const bool al4 = (reinterpret_cast<uintptr_t>(payload) & 3) == 0;
  constexpr int kW = kUnitsPerWarp * (kDecodeUnit / (4 * kWarp));
  uint32_t w[kW];
  int nb[kW];
#pragma unroll
  for (int k = 0; k < kW; ++k) {
    const uint32_t unit = c * kDecodeChunkUnits + warp * kUnitsPerWarp + k / 4;
    const uint64_t p = (uint64_t)unit * kDecodeUnit + 4 * (uint64_t)(lane + kWarp * (k % 4));
    w[k] = 0;
    nb[k] = 0;
    if (al4 && p + 4 <= m) {
      w[k] = __ldg(reinterpret_cast<const uint32_t *>(payload + p));
      nb[k] = 4;
    } else {
      for (int q = 0; q < 4; ++q)
        if (p + q < m) {
          w[k] |= (uint32_t)__ldg(payload + p + q) << (8 * q);
          nb[k] = q + 1;
        }
    }
  }
  uint32_t wtot = 0;
#pragma unroll
  for (int i = 0; i < kUnitsPerWarp; ++i) {
    uint32_t e = 0;
#pragma unroll
    for (int k = 4 * i; k < 4 * i + 4; ++k)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t b = (w[k] >> (8 * q)) & 0xffu;
        if (q < nb[k]) e += b >= 243u ? b - 241u : 1u;
      }
    e = __reduce_add_sync(0xffffffffu, e);
    const uint32_t unit = c * kDecodeChunkUnits + warp * kUnitsPerWarp + i;
    if (lane == 0 && unit < n_units) ecount[unit] = e;
    wtot += e;
  }
  if (lane == 0) wsum[warp] = wtot;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t sum = 0;
#pragma unroll
    for (int v = 0; v < kDThreads / kWarp; ++v) sum += wsum[v];
    csum[c] = sum;
  }
  __syncthreads();
}

// Counting pass of one stream: blocks stride over the chunks that exist.
// Block 0 also clears k_decode's ticket.  A stream whose length or header is
// invalid is left to k_decode to report.
__global__ void __launch_bounds__(kDThreads) k_decode_count(const DecodeArgs a) {
  __shared__ uint64_t m_s;
  __shared__ int ok_s;
  __shared__ uint32_t wsum[kDThreads / kWarp];
  if (threadIdx.x == 0) {
    uint64_t m = 0;
    float scale = 0.0f;
    ok_s = read_stream_header(a.in, a.len_dev, a.cap, a.groups, m, scale) ? 1 : 0;
    m_s = m;
    if (blockIdx.x == 0) *a.ticket = 0;
  }
  __syncthreads();
  if (!ok_s) return;
  const uint64_t m = m_s;
  const uint32_t n_units = (uint32_t)((m + kDecodeUnit - 1) / kDecodeUnit);
  const uint32_t n_chunks = (n_units + kDecodeChunkUnits - 1) / kDecodeChunkUnits;
  for (uint32_t c = blockIdx.x; c < n_chunks; c += gridDim.x)
    count_chunk(a.in + 4, m, c, a.ecount, a.csum, wsum);
}

struct BatchDecodeArgs {
  const BatchTensor *tensors;
  uint32_t count;
  const BatchPrep *prep;        // per-tensor payload length, scale, first tile
  const uint32_t *total;        // tiles in the compact numbering
  uint32_t n_tiles;             // upper bound of total (sizes the grid)
  const uint8_t *arena;
  uint64_t *status;
  uint32_t *ticket;
  int32_t *dev_status;
  uint32_t max_polls;
  uint32_t *ecount;             // counting pass (plans of 16384 units and more)
  uint64_t *csum;
  uint32_t n_chunks;            // chunks of all tensors (upper bound)
};

constexpr int kPrepThreads = 1024;
constexpr uint32_t kSmemSearch = 2048;  // tensors whose first tiles fit in shared memory

// One block: validate every tensor's stream once, and number the tiles that
// actually exist (ceil(m / tile) per stream, 0 for a corrupt one)
// consecutively, tensor by tensor; the same for the counting pass's 32-unit
// chunks.  total[0] = tiles, total[1] = chunks.
__global__ void __launch_bounds__(kPrepThreads)
k_decode_batch_prepare(const BatchTensor *__restrict__ tensors, uint32_t count,
                       const uint8_t *__restrict__ arena, const uint64_t *__restrict__ in_lens,
                       uint32_t tile_bytes, BatchPrep *__restrict__ prep,
                       uint32_t *__restrict__ total, int32_t *dev_status) {
  __shared__ uint32_t scan_s[kPrepThreads / kWarp + 1];
  uint32_t base = 0, cbase = 0;
  for (uint32_t c0 = 0; c0 < count; c0 += kPrepThreads) {
    const uint32_t i = c0 + threadIdx.x;
    uint64_t m = 0;
    float scale = 0.0f;
    uint32_t tiles = 0, chunks = 0;
    if (i < count) {
      const BatchTensor &T = tensors[i];
      if (read_stream_header(arena + T.arena_off, in_lens + i, T.cap, T.groups, m, scale)) {
        tiles = (uint32_t)((m + tile_bytes - 1) / tile_bytes);
        const uint64_t units = (m + kDecodeUnit - 1) / kDecodeUnit;
        chunks = (uint32_t)((units + kDecodeChunkUnits - 1) / kDecodeChunkUnits);
      } else {
        m = 0;
        report(dev_status, TLC_ERR_CORRUPT);
      }
    }
    uint32_t sum, csum_all;
    const uint32_t off = block_exclusive_sum<kPrepThreads>(tiles, scan_s, sum);
    const uint32_t coff = block_exclusive_sum<kPrepThreads>(chunks, scan_s, csum_all);
    if (i < count) {
      BatchPrep p;
      p.m = m;
      p.scale = scale;
      p.act_begin = base + off;
      p.cact_begin = cbase + coff;
      p.pad = 0;
      prep[i] = p;
    }
    base += sum;
    cbase += csum_all;
  }
  if (threadIdx.x == 0) {
    total[0] = base;
    total[1] = cbase;
  }
}

// Decode the streams of a list of tensors from their arena slots: the tiles
// that exist, numbered tensor by tensor, taken in ticket order; each
// look-back is confined to its stream.  A tile's tensor is found by binary
// search over the tensors' first tiles.
template <int kMode, bool kDeferred>
__global__ void __launch_bounds__(kDThreads) k_decode_batch(const BatchDecodeArgs a) {
  constexpr int kDTile = DecodeShape<kMode>::kTile;
  extern __shared__ __align__(16) uint8_t grp_s[];
  __shared__ DecodeSmem sm;
  __shared__ uint32_t begin_s[kSmemSearch];
  __shared__ uint32_t tile_s;
  for (int v = threadIdx.x; v < 256; v += kDThreads) sm.lut[v] = v < 243 ? digits_of(v) : 0;
  const bool in_smem = a.count <= kSmemSearch;
  if (in_smem)
    for (uint32_t i = threadIdx.x; i < a.count; i += kDThreads) begin_s[i] = a.prep[i].act_begin;
  const uint32_t total = *a.total;
  for (;;) {
    if (threadIdx.x == 0) tile_s = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t u = tile_s;
    if (u >= total) break;
    // last tensor whose first tile is <= u (tensors without tiles are skipped
    // naturally: they share their first tile with the next tensor)
    uint32_t lo = 0, hi = a.count - 1;
    while (lo < hi) {
      const uint32_t mid = (lo + hi + 1) >> 1;
      const uint32_t b = in_smem ? begin_s[mid] : a.prep[mid].act_begin;
      if (b <= u) lo = mid; else hi = mid - 1;
    }
    const BatchTensor &T = a.tensors[lo];
    const BatchPrep &P = a.prep[lo];
    DecodeJob job;
    job.payload = a.arena + T.arena_off + 4;
    job.m = P.m;
    job.n = T.n;
    job.groups = T.groups;
    job.scale = P.scale;
    job.y = T.y;
    job.status = a.status + T.d_tile_begin;
    job.n_tiles = (uint32_t)((job.m + kDTile - 1) / kDTile);
    job.vec = T.vec_y != 0;
    job.ecount = kDeferred ? a.ecount + T.d_tile_begin : nullptr;
    job.csum = kDeferred ? a.csum + T.d_chunk_begin : nullptr;
    decode_tile<kMode, kDeferred>(job, u - P.act_begin, sm, grp_s, a.dev_status, a.max_polls);
  }
}

// Counting pass of a plan's streams: blocks stride over the chunks that
// exist, numbered tensor by tensor by the prepare kernel (a tensor's first
// chunk is found by binary search).  Block 0 also clears the decode ticket.
__global__ void __launch_bounds__(kDThreads) k_decode_batch_count(const BatchDecodeArgs a) {
  __shared__ uint32_t begin_s[kSmemSearch];
  __shared__ uint32_t wsum[kDThreads / kWarp];
  const bool in_smem = a.count <= kSmemSearch;
  if (in_smem)
    for (uint32_t i = threadIdx.x; i < a.count; i += kDThreads) begin_s[i] = a.prep[i].cact_begin;
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.ticket = 0;
  __syncthreads();
  const uint32_t total = a.total[1];
  for (uint32_t g = blockIdx.x; g < total; g += gridDim.x) {
    // last tensor whose first chunk is <= g (tensors without chunks share
    // their first chunk with the next tensor)
    uint32_t lo = 0, hi = a.count - 1;
    while (lo < hi) {
      const uint32_t mid = (lo + hi + 1) >> 1;
      const uint32_t b = in_smem ? begin_s[mid] : a.prep[mid].cact_begin;
      if (b <= g) lo = mid; else hi = mid - 1;
    }
    const BatchTensor &T = a.tensors[lo];
    const BatchPrep &P = a.prep[lo];
    count_chunk(a.arena + T.arena_off + 4, P.m, g - P.cact_begin, a.ecount + T.d_tile_begin,
                a.csum + T.d_chunk_begin, wsum);
  }
}

// Wait-limit check: tile 1 looks back at a tile 0 that never publishes.
__global__ void k_wait_test(uint64_t *status, uint32_t max_polls, int32_t *dev_status) {
  bool timed_out = false;
  (void)lookback_sum(status, 1, 0, max_polls, timed_out);
  if (__any_sync(0xffffffffu, timed_out) && threadIdx.x == 0) report(dev_status, TLC_ERR_TIMEOUT);
}

// ------------------------------------------------------------- launchers --
uint32_t decode_tiles_max(uint64_t cap, uint64_t groups) {
  // 512-byte units: at least as many as the tiles of either mode (tiles are
  // whole units), and the counting pass's unit count
  static_assert(DecodeShape<kWrite>::kTile % kDecodeUnit == 0 &&
                    DecodeShape<kAccumulate>::kTile % kDecodeUnit == 0,
                "tiles are whole units");
  uint64_t m = cap >= 4 ? cap - 4 : 0;
  if (m > groups) m = groups;
  uint64_t t = (m + kDecodeUnit - 1) / kDecodeUnit;
  return (uint32_t)(t < 1 ? 1 : t);
}

size_t decode_smem_bytes(bool accumulate) {
  return (size_t)(accumulate ? DecodeShape<kAccumulate>::kMaxGroups
                             : DecodeShape<kWrite>::kMaxGroups) + 16;
}

template <int kMode, bool kVec>
static cudaError_t launch_one(const DeviceInfo &dev, const DecodeArgs &a, uint32_t tiles,
                              bool deferred, cudaStream_t stream) {
  const size_t smem = decode_smem_bytes(kMode == kAccumulate);
  const int occ = kMode == kWrite ? dev.occ_decode_write : dev.occ_decode_acc;
  uint32_t grid = (uint32_t)dev.sm_count * (uint32_t)(occ > 0 ? occ : 1);
  if (grid > tiles) grid = tiles;
  if (deferred) {
    // tiles (the capacity's 512-byte units) bound the units that exist
    uint32_t cgrid = (tiles + kDecodeChunkUnits - 1) / kDecodeChunkUnits;
    if (cgrid > (uint32_t)dev.sm_count * 8) cgrid = (uint32_t)dev.sm_count * 8;
    timing_begin(kKindDecodeCount, stream);
    k_decode_count<<<cgrid, kDThreads, 0, stream>>>(a);
    timing_end(kKindDecodeCount, stream);
  }
  const int kind = kMode == kWrite ? kKindDecodeWrite : kKindDecodeAccumulate;
  timing_begin(kind, stream);
  if (deferred)
    k_decode<kMode, kVec, true><<<grid, kDThreads, smem, stream>>>(a);
  else
    k_decode<kMode, kVec, false><<<grid, kDThreads, smem, stream>>>(a);
  timing_end(kind, stream);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DeviceInfo &dev, const uint8_t *in, const uint64_t *len_dev,
                          uint64_t cap, uint64_t n, float *y, bool accumulate,
                          int32_t *dev_status, uint32_t max_polls, uint64_t *scratch,
                          cudaStream_t stream) {
  const uint64_t groups = (n + 4) / 5;
  const uint32_t tiles = decode_tiles_max(cap, groups);
  const bool deferred = decode_deferred(tiles);
  const DecodeScratch ds = decode_scratch_layout(scratch, tiles, deferred);
  DecodeArgs a;
  a.ecount = ds.ecount;
  a.csum = ds.csum;
  a.in = in;
  a.len_dev = len_dev;
  a.cap = cap;
  a.n = n;
  a.groups = groups;
  a.y = y;
  a.status = ds.status;
  a.ticket = ds.ticket;
  a.dev_status = dev_status;
  a.max_polls = max_polls;
  const bool vec = (reinterpret_cast<uintptr_t>(y) & 15) == 0;
  if (accumulate)
    return vec ? launch_one<kAccumulate, true>(dev, a, tiles, deferred, stream)
               : launch_one<kAccumulate, false>(dev, a, tiles, deferred, stream);
  return vec ? launch_one<kWrite, true>(dev, a, tiles, deferred, stream)
             : launch_one<kWrite, false>(dev, a, tiles, deferred, stream);
}

bool decode_deferred(uint32_t tiles) { return tiles >= kDecodeDeferMinTiles; }

uint32_t decode_tile_payload_bytes(bool accumulate) {
  return accumulate ? DecodeShape<kAccumulate>::kTile : DecodeShape<kWrite>::kTile;
}

template <int kMode>
static cudaError_t launch_batch_one(const DeviceInfo &dev, const BatchDecodeArgs &a,
                                    bool deferred, cudaStream_t stream) {
  const size_t smem = decode_smem_bytes(kMode == kAccumulate);
  const int occ = kMode == kWrite ? dev.occ_decode_batch_write : dev.occ_decode_batch_acc;
  uint32_t grid = (uint32_t)dev.sm_count * (uint32_t)(occ > 0 ? occ : 1);
  if (grid > a.n_tiles) grid = a.n_tiles;
  if (deferred) {
    uint32_t cgrid = a.n_chunks;
    if (cgrid > (uint32_t)dev.sm_count * 8) cgrid = (uint32_t)dev.sm_count * 8;
    timing_begin(kKindDecodeCount, stream);
    k_decode_batch_count<<<cgrid, kDThreads, 0, stream>>>(a);
    timing_end(kKindDecodeCount, stream);
  }
  const int kind = kMode == kWrite ? kKindDecodeWrite : kKindDecodeAccumulate;
  timing_begin(kind, stream);
  if (deferred)
    k_decode_batch<kMode, true><<<grid, kDThreads, smem, stream>>>(a);
  else
    k_decode_batch<kMode, false><<<grid, kDThreads, smem, stream>>>(a);
  timing_end(kind, stream);
  return cudaGetLastError();
}

cudaError_t launch_decode_batch(const DeviceInfo &dev, const BatchPlanDev &p,
                                const uint8_t *arena, const uint64_t *in_lens, bool accumulate,
                                int32_t *dev_status, uint32_t max_polls, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(p.d_zero_base, 0, p.d_zero_bytes, stream);
  if (e != cudaSuccess) return e;
  timing_begin(kKindDecodePrepare, stream);
  k_decode_batch_prepare<<<1, kPrepThreads, 0, stream>>>(
      p.tensors, p.count, arena, in_lens, decode_tile_payload_bytes(accumulate), p.d_prep,
      p.d_total, dev_status);
  timing_end(kKindDecodePrepare, stream);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BatchDecodeArgs a;
  a.tensors = p.tensors;
  a.count = p.count;
  a.prep = p.d_prep;
  a.total = p.d_total;
  a.arena = arena;
  a.status = p.d_status;
  a.ticket = p.d_ticket;
  a.n_tiles = p.n_d_tiles;
  a.dev_status = dev_status;
  a.max_polls = max_polls;
  a.ecount = p.d_ecount;
  a.csum = p.d_csum;
  a.n_chunks = p.n_d_chunks;
  const bool deferred = decode_deferred(p.n_d_tiles);
  return accumulate ? launch_batch_one<kAccumulate>(dev, a, deferred, stream)
                    : launch_batch_one<kWrite>(dev, a, deferred, stream);
}

int occupancy_decode_batch(bool accumulate) {
  int occ = 0;
  const size_t smem = decode_smem_bytes(accumulate);
  if (accumulate) {
    cudaFuncSetAttribute(k_decode_batch<kAccumulate, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode_batch<kAccumulate, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode_batch<kAccumulate, false>,
                                                  kDThreads, smem);
  } else {
    cudaFuncSetAttribute(k_decode_batch<kWrite, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode_batch<kWrite, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode_batch<kWrite, false>, kDThreads,
                                                  smem);
  }
  return occ;
}

cudaError_t launch_wait_test(uint64_t *status, uint32_t max_polls, int32_t *dev_status,
                             cudaStream_t stream) {
  k_wait_test<<<1, kWarp, 0, stream>>>(status, max_polls, dev_status);
  return cudaGetLastError();
}

int occupancy_decode(bool accumulate) {
  int occ = 0;
  const size_t smem = decode_smem_bytes(accumulate);
  if (accumulate) {
    cudaFuncSetAttribute(k_decode<kAccumulate, true, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode<kAccumulate, false, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode<kAccumulate, true, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode<kAccumulate, false, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode<kAccumulate, true, false>,
                                                  kDThreads, smem);
  } else {
    cudaFuncSetAttribute(k_decode<kWrite, true, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode<kWrite, false, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode<kWrite, true, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode<kWrite, false, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode<kWrite, true, false>, kDThreads,
                                                  smem);
  }
  return occ;
}

}  // namespace tlc
