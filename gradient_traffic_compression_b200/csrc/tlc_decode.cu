// tlc_decode.cu -- decompression kernels for the 3LC pipeline on sm_100a.
//
// Source: review page "3LC: Lightweight and Effective Traffic Compression for
// Distributed Machine Learning".  Decoding inverts "Proposed method" bullets
// 3 (zero-run encoding), 2 (quartic encoding) and 1 (dequantization to
// q * M * s); the Abstract's exchange of state changes between nodes is the
// receive side, where several workers' streams are summed.
//
// Two modes:
//   kWrite       dense output: y_i = +scale, -scale or +0.0
//   kAccumulate  acc_i += y_i only where q_i != 0 (acc keeps its bits at
//                zeros), streams in worker order
//
// Small streams (capacity below 8 MiB), one at a time: k_decode, one launch.
// A tile is 512 (kWrite) or 2048 (kAccumulate) payload bytes: per tile,
// expansion counts e_k (an escape byte b >= 243 stands for b - 241 groups of
// 121, any other byte for itself), a block scan, and a decoupled look-back
// over earlier tiles for the tile's first group index.
//
// Large streams, and several streams summed in one pass: an index, then the
// decode; no block of either kernel waits on another.
//   k_index_count   one block per 64-unit chunk of 512-byte payload units:
//                   each unit's first group relative to its chunk (loc[u])
//                   and the chunk's group count.
//   k_index_scan    one block per stream: the chunk counts scanned into each
//                   chunk's first group (cpre[c]) and the check that the
//                   stream expands to exactly ceil(n/5) groups (its valid
//                   flag); for sums of several streams the same for the
//                   non-zero literal groups ("entries").
//   k_decode_units  one stream: one warp per 512-byte unit, first group
//                   cpre[u / 64] + loc[u]; the unit's groups are expanded in
//                   the warp's shared memory and written (or added) as
//                   coalesced float4s from a table of two-digit value pairs.
//   k_index_entries 2..8 streams: one warp per unit writes the unit's entries
//                   (tile position and digit word) to the stream's list, in
//                   group order, and the first entry of every sum tile.
//   k_apply_entries 2..8 streams: tiles of 2048 groups; each stream's entries
//                   of the tile go to shared memory with a per-group stream
//                   mask, then each thread reads a marked group's acc values
//                   once, adds the streams' values in stream order and
//                   writes them once.
// The quartic bytes live only in shared memory.  Every write is clamped to
// the ceil(n/5) groups of the tensor; a stream that does not expand to
// exactly that many groups is reported as corrupt and left out.
#define TLC_TU 2
#include "tlc_device.cuh"
#include "tlc_internal.h"

namespace tlc {

TLC_DEFINE_DEBUG_READER(debug_fault_decode)

// Payload bytes per thread (1, 2 or a multiple of 4) of the small-stream
// tiles: small tiles balance the dense write mode best; the accumulate mode
// touches little memory per tile and prefers fewer, larger tiles.
#ifndef TLC_D_BYTES_WRITE
#define TLC_D_BYTES_WRITE 2
#endif
#ifndef TLC_D_BYTES_ACC
#define TLC_D_BYTES_ACC 8
#endif
constexpr int kDThreads = 256;
constexpr int kDWarps = kDThreads / kWarp;
constexpr int kWrite = 0, kAccumulate = 1;
template <int kMode>
struct DecodeShape {
  static constexpr int kBytes = kMode == kWrite ? TLC_D_BYTES_WRITE : TLC_D_BYTES_ACC;
  static constexpr int kTile = kDThreads * kBytes;   // payload bytes per tile
  static constexpr int kMaxGroups = kTile * 14;      // largest expansion of a tile
};
#ifndef TLC_D_LOOKV
#define TLC_D_LOOKV 4
#endif
constexpr int kLookV = TLC_D_LOOKV;   // look-back words per lane per round trip
// Streams whose capacity allows this many 512-byte units or more are
// decoded through the index.
#ifndef TLC_DEFER_DECODE_MIN_TILES
#define TLC_DEFER_DECODE_MIN_TILES 16384
#endif
constexpr uint32_t kDecodeDeferMinTiles = TLC_DEFER_DECODE_MIN_TILES;
static_assert(kDecodeUnit == 4 * kWarp * 4, "a unit is 16 bytes per lane of a warp");
static_assert(kDecodeChunkUnits == 2 * kWarp, "a chunk's units are two per lane of a warp");

size_t decode_smem_bytes(bool accumulate);

struct DecodeArgs {
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

// Exclusive prefix (a sum) of tile u of a single-pass scan, by one warp.
// Publishes the tile's aggregate first and its inclusive prefix last.  Each
// round trip reads 32 * kLookV earlier tiles' words.  Every lane gets the
// result.
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

__device__ __forceinline__ uint32_t expansion(uint32_t b) { return b >= 243u ? b - 241u : 1u; }

// The same for 16 bytes (four words) at once.  An escape byte 243..255
// (0xF3..0xFF: high nibble F, low nibble at least 3) stands for its low
// nibble - 1 groups, so 16 bytes expand to 16 + (the escapes' low nibbles)
// - 2 (the escapes).  esc_bits(w) has bit 7 of each escape byte of w set:
// the per-byte sums of its one add cannot carry.  Per byte lane the low
// nibbles add up to at most 60 and the escape counts to 4, so one multiply
// sums the four byte lanes.
__device__ __forceinline__ uint32_t esc_bits(uint32_t w) {
  return w & ((w & 0x7F7F7F7Fu) + 0x0D0D0D0Du) & 0x80808080u;
}
__device__ __forceinline__ uint32_t byte_lane_sum(uint32_t x) { return (x * 0x01010101u) >> 24; }
__device__ __forceinline__ uint32_t expansion16(const uint32_t (&w)[4]) {
  uint32_t lo = 0, cnt = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t e = esc_bits(w[k]) >> 7;  // 1 in each escape byte
    lo += w[k] & 0x0F0F0F0Fu & (e * 0x0Fu);
    cnt += e;
  }
  return 16u + byte_lane_sum(lo) - 2u * byte_lane_sum(cnt);
}

// Literal bytes other than the zero group 121 among 16 bytes: those that
// are neither escapes nor 121 (a zero byte of w ^ 0x79.., found without
// carries between bytes).
__device__ __forceinline__ uint32_t literals16(const uint32_t (&w)[4]) {
  uint32_t cnt = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t x = w[k] ^ 0x79797979u;
    const uint32_t nz = ((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x;  // bit 7: byte of x not zero
    cnt += ((~nz & 0x80808080u) | esc_bits(w[k])) >> 7;
  }
  return 16u - byte_lane_sum(cnt);
}

// One stream's decode job.
struct DecodeJob {
  const uint8_t *payload;  // stream bytes after the 4-byte header
  uint64_t m;              // payload length
  uint64_t n, groups;
  float scale;
  float *y;                // output (kWrite) or accumulation buffer
  uint64_t *status;        // small streams: this stream's tile status words
  uint32_t n_tiles;        // tiles (or units) actually present
  bool vec;                // y is 16-byte aligned
  const uint32_t *loc;     // indexed streams: units' first groups within their chunk
  const uint32_t *cpre;    // and chunks' first groups
};

struct DecodeSmem {
  uint16_t lut[256];       // base-3 digits of every quartic byte
  uint32_t scan[kDThreads / kWarp + 1];
  uint64_t o;
};

__device__ __forceinline__ void fill_lut(uint16_t *lut) {
  for (int v = threadIdx.x; v < 256; v += blockDim.x) lut[v] = v < 243 ? digits_of(v) : 0;
}

// A warp's scaled pair table: for every 4-bit word of two digits (2 bits
// each, first value lowest) the two values q * scale, q in {-1, 0, +1} (each
// product exact, +0.0 for q = 0; digit 3 never occurs), filled by lanes
// 0..15.  The 16 entries of 8 bytes fill the 32 banks once, so no pattern
// of lookups has a bank conflict.
__device__ __forceinline__ void fill_scaled_pairs(float2 *sp, float scale, int lane) {
  if (lane < 16) {
    auto q = [](uint32_t d) { return d == 0u ? -1.0f : (d == 2u ? 1.0f : 0.0f); };
    sp[lane] = make_float2(__fmul_rn(q(lane & 3u), scale), __fmul_rn(q((lane >> 2) & 3u), scale));
  }
  __syncwarp();
}
__device__ __forceinline__ float4 quad(const float2 *sp, uint32_t p8) {
  const float2 a = sp[p8 & 15u], b = sp[p8 >> 4];
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void add_quad(float4 &o, const float2 *sp, uint32_t p8) {
  const float4 p = quad(sp, p8);
  if ((p8 & 3u) != 1u) o.x = __fadd_rn(o.x, p.x);
  if (((p8 >> 2) & 3u) != 1u) o.y = __fadd_rn(o.y, p.y);
  if (((p8 >> 4) & 3u) != 1u) o.z = __fadd_rn(o.z, p.z);
  if (((p8 >> 6) & 3u) != 1u) o.w = __fadd_rn(o.w, p.w);
}

// Digit words in shared memory windows sit at swizzled positions: position
// p at p ^ (((p >> 6) & 7) << 1).  Lanes placing literals about 16
// positions apart then hit distinct banks, and the 26 consecutive positions
// a row of 32 float4s reads still do.  The swizzle stays inside each
// aligned block of 16 positions, so a window is filled in whole blocks.
__device__ __forceinline__ uint32_t wsw(uint32_t p) { return p ^ (((p >> 6) & 7u) << 1); }

// Validate a stream (length and header) and return its payload length and
// scale.  Corrupt when the length is below 4 or above the readable capacity,
// the payload would be longer than the tensor's groups or empty, or the
// header is negative or not finite (the encoder never writes such a header).
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

// Write values [e_begin, e_end) of groups whose quartic bytes sit in grp
// (grp[0] is group g_first), or add their non-zero values in accumulate
// mode.  Float4 columns with coalesced 128-bit accesses when y is 16-byte
// aligned, single values at the edges.  Values 4v..4v+3 lie in group g =
// 4v/5 (digits d0..) and, when d0 >= 2, spill into group g+1; both groups'
// digit words are joined so one shift lines the four digits up.
// The calling group of threads is a whole block (tid = threadIdx.x, nth =
// blockDim.x) or a whole warp (tid = lane, nth = 32).
template <int kMode>
__device__ __forceinline__ void emit_values(const uint8_t *grp, uint64_t g_first,
                                            uint64_t e_begin, uint64_t e_end, float *y, bool vec,
                                            float scale, const uint16_t *lut,
                                            uint32_t tid, uint32_t nth) {
  if (e_end <= e_begin) return;
  const uint32_t o32 = (uint32_t)g_first;
  auto put = [&](uint64_t e) {
    const uint32_t e32 = (uint32_t)e;
    const uint32_t g = e32 / 5u;
    const uint32_t dig = (lut[grp[g - o32]] >> (2 * (e32 - 5u * g))) & 3u;
    if (kMode == kWrite)
      y[e] = dequant(dig, scale);
    else if (dig != 1u)
      y[e] = __fadd_rn(y[e], dequant(dig, scale));
  };
  const uint64_t v0 = (e_begin + 3) / 4, v1 = e_end / 4;
  if (!vec || v1 <= v0) {
    for (uint64_t e = e_begin + tid; e < e_end; e += nth) put(e);
    return;
  }
  float4 *y4 = reinterpret_cast<float4 *>(y);
  for (uint64_t v = v0 + tid; v < v1; v += nth) {
    const uint32_t e0 = (uint32_t)(4 * v);
    const uint32_t g = e0 / 5u;
    const uint32_t d0 = e0 - 5u * g;
    const uint32_t li = g - o32;
    const uint32_t c0 = grp[li];
    const uint32_t c1 = d0 >= 2u ? (uint32_t)grp[li + 1] : 121u;
    if (kMode == kWrite) {
      float4 o;
      if (c0 == 121u && c1 == 121u) {
        o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      } else {
        const uint32_t w = ((uint32_t)lut[c0] | ((uint32_t)lut[c1] << 10)) >> (2u * d0);
        o.x = dequant(w & 3u, scale);
        o.y = dequant((w >> 2) & 3u, scale);
        o.z = dequant((w >> 4) & 3u, scale);
        o.w = dequant((w >> 6) & 3u, scale);
      }
      y4[v] = o;
    } else if (c0 != 121u || c1 != 121u) {
      const uint32_t w = ((uint32_t)lut[c0] | ((uint32_t)lut[c1] << 10)) >> (2u * d0);
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
  if (tid < 4) {
    const uint64_t e = e_begin + tid;
    if (e < 4 * v0) put(e);
  } else if (tid < 8) {
    const uint64_t e = 4 * v1 + (tid - 4);
    if (e < e_end) put(e);
  }
}

// Zeros over values [e_begin, e_end) (dense output of all-zero groups), by
// a block or a warp as emit_values.
__device__ __forceinline__ void emit_zeros(uint64_t e_begin, uint64_t e_end, float *y, bool vec,
                                           uint32_t tid, uint32_t nth) {
  if (e_end <= e_begin) return;
  const uint64_t v0 = (e_begin + 3) / 4, v1 = e_end / 4;
  if (!vec || v1 <= v0) {
    for (uint64_t e = e_begin + tid; e < e_end; e += nth) y[e] = 0.0f;
    return;
  }
  float4 *y4 = reinterpret_cast<float4 *>(y);
  for (uint64_t v = v0 + tid; v < v1; v += nth) y4[v] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (tid < 4) {
    const uint64_t e = e_begin + tid;
    if (e < 4 * v0) y[e] = 0.0f;
  } else if (tid < 8) {
    const uint64_t e = 4 * v1 + (tid - 4);
    if (e < e_end) y[e] = 0.0f;
  }
}

// One payload tile of one stream; the whole block calls it and it ends
// synchronised.  The tile's first group index comes from a decoupled
// look-back over the tiles before it (small streams) or, kIndexed, from the
// index (cpre and loc of its first unit; the index has checked the total).
template <int kMode, bool kIndexed = false>
__device__ __forceinline__ void decode_tile(const DecodeJob &j, uint32_t u, DecodeSmem &sm,
                                            uint8_t *grp_s, int32_t *dev_status,
                                            uint32_t max_polls) {
  constexpr int kDBytes = DecodeShape<kMode>::kBytes;
  constexpr int kDTile = DecodeShape<kMode>::kTile;
  static_assert(kDTile % kDecodeUnit == 0, "tiles are whole units");
  const int warp = threadIdx.x >> 5;
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
      esum += expansion(b);
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
  // Indexed: one lookup while every thread pre-fills the zero groups.
  // Look-back: warp 0 looks back while the other warps pre-fill.
  if (kIndexed) {
    constexpr uint32_t kTileUnits = kDTile / kDecodeUnit;
    if (threadIdx.x == 0)
      sm.o = (uint64_t)__ldg(j.cpre + (u * kTileUnits) / kDecodeChunkUnits) +
             __ldg(j.loc + u * kTileUnits);
    if (expand) {
      const uint32_t words = (E + 15) / 16;
      for (uint32_t w = threadIdx.x; w < words; w += kDThreads)
        reinterpret_cast<uint4 *>(grp_s)[w] =
            make_uint4(0x79797979u, 0x79797979u, 0x79797979u, 0x79797979u);
    }
  } else if (warp == 0) {
    bool timed_out = false;
    const uint64_t O = lookback_sum(j.status, u, E, max_polls, timed_out);
    if (__any_sync(0xffffffffu, timed_out) && threadIdx.x == 0) report(dev_status, TLC_ERR_TIMEOUT);
    if (threadIdx.x == 0) sm.o = O;
  } else if (expand) {
    const uint32_t words = (E + 15) / 16;
    for (uint32_t w = threadIdx.x - kWarp; w < words; w += kDThreads - kWarp)
      reinterpret_cast<uint4 *>(grp_s)[w] =
          make_uint4(0x79797979u, 0x79797979u, 0x79797979u, 0x79797979u);
  }
  __syncthreads();
  const uint64_t O = sm.o;
  if (!kIndexed && threadIdx.x == 0) {
    const bool last = (u == j.n_tiles - 1);
    if (O + E > j.groups || (last && O + E != j.groups)) report(dev_status, TLC_ERR_CORRUPT);
  }
  const uint64_t Ec = O >= j.groups ? 0 : umin64(E, j.groups - O);

  if (!any_lit) {
    if (kMode == kWrite)
      emit_zeros(5 * O, umin64(5 * (O + Ec), j.n), j.y, j.vec, threadIdx.x, kDThreads);
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
          if (TLC_CHECK(pos < (uint32_t)DecodeShape<kMode>::kMaxGroups)) grp_s[pos] = (uint8_t)b;
          ++pos;
        }
      }
    }
    __syncthreads();
    // groups [O, O+Ec) -> values [5 O, min(5 (O+Ec), n))
    emit_values<kMode>(grp_s, O, 5 * O, umin64(5 * (O + Ec), j.n), j.y, j.vec, scale, sm.lut,
                       threadIdx.x, kDThreads);
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

// Small streams: payload tiles in ticket order, each finding its first group
// by a decoupled look-back over the tiles before it.
template <int kMode, bool kVec>
__global__ void __launch_bounds__(kDThreads)
k_decode(const DecodeArgs a) {
  constexpr int kDTile = DecodeShape<kMode>::kTile;
  extern __shared__ __align__(16) uint8_t grp_s[];  // kMaxGroups + 16 bytes
  __shared__ DecodeSmem sm;
  __shared__ uint64_t m_s;
  __shared__ uint32_t tile_s;
  __shared__ float scale_s;
  __shared__ int ok_s;
  pdl_enter();

  if (threadIdx.x == 0) {
    uint64_t m = 0;
    float scale = 0.0f;
    ok_s = read_stream_header(a.in, a.len_dev, a.cap, a.groups, m, scale) ? 1 : 0;
    m_s = m;
    scale_s = scale;
  }
  fill_lut(sm.lut);
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
  for (;;) {
    if (threadIdx.x == 0) tile_s = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t u = tile_s;
    if (u >= job.n_tiles) break;
    decode_tile<kMode>(job, u, sm, grp_s, a.dev_status, a.max_polls);
  }
}

// Accumulate mode: values [e_begin, e_end) of the groups whose digit words
// (lut[] of their quartic bytes) sit in wd at swizzled positions counted
// from group g_first, added into acc by one warp where a digit is not zero:
// aligned float4s, two per lane loaded before either is added, each from
// the warp's scaled pair table (sp); single values at the ends, and
// everywhere when acc is not 16-byte aligned.  Values 4v..4v+3 lie in group
// g = 4v/5 (digits d0..) and, when d0 >= 2, spill into group g+1; both
// groups' digit words are joined so one shift lines the four digits up.
__device__ __forceinline__ void warp_accumulate(const uint16_t *wd, uint64_t g_first,
                                                uint64_t e_begin, uint64_t e_end, float *y,
                                                bool vec, float scale, const float2 *sp,
                                                int lane) {
  if (e_end <= e_begin) return;
  const uint32_t gf = (uint32_t)g_first;
  // n < 2^32, so value and float4 indices fit 32 bits
  auto put = [&](uint32_t e) {
    const uint32_t g = e / 5u;
    const uint32_t dig = (wd[wsw(g - gf)] >> (2 * (e - 5u * g))) & 3u;
    if (dig != 1u) y[e] = __fadd_rn(y[e], dequant(dig, scale));
  };
  auto digits8 = [&](uint32_t v) -> uint32_t {
    const uint32_t e0 = v << 2;
    const uint32_t g = e0 / 5u;
    const uint32_t d0 = e0 - 5u * g;
    const uint32_t li = g - gf;
    return (((uint32_t)wd[wsw(li)] | ((uint32_t)wd[wsw(li + 1)] << 10)) >> (2u * d0)) & 0xffu;
  };
  const uint32_t v0 = (uint32_t)((e_begin + 3) / 4), v1 = (uint32_t)(e_end / 4);
  if (!vec || v1 <= v0) {
    for (uint32_t e = (uint32_t)e_begin + lane; e < (uint32_t)e_end; e += kWarp) put(e);
    return;
  }
  float4 *y4 = reinterpret_cast<float4 *>(y);
  for (uint32_t v = v0 + lane; v < v1; v += 2 * kWarp) {
    const uint32_t vb = v + kWarp;
    const uint32_t pa = digits8(v);
    const uint32_t pb = vb < v1 ? digits8(vb) : 0x55u;
    float4 oa = make_float4(0.0f, 0.0f, 0.0f, 0.0f), ob = oa;
    if (pa != 0x55u) oa = y4[v];  // 0x55: four zero digits
    if (pb != 0x55u) ob = y4[vb];
    if (pa != 0x55u) {
      add_quad(oa, sp, pa);
      y4[v] = oa;
    }
    if (pb != 0x55u) {
      add_quad(ob, sp, pb);
      y4[vb] = ob;
    }
  }
  // the partial float4s at both ends, one value per lane
  const uint32_t h = 4 * v0 - (uint32_t)e_begin, t = (uint32_t)e_end - 4 * v1;  // each < 4
  if ((uint32_t)lane < h + t)
    put((uint32_t)lane < h ? (uint32_t)e_begin + lane : 4 * v1 + (lane - h));
}

// Dense output: the values [5 gb, min(5 (gb + wn), n)) of the groups
// [gb, gb + wn) whose digit words sit in wd at swizzled positions counted
// from gb & ~3, by one warp.  Each lane expands one whole batch of four
// groups 4a .. 4a + 3 (values 20a .. 20a + 19, float4s 5a .. 5a + 4) from one
// 8-byte read of their digit words (a multiple-of-4 position, so the four
// words share one aligned block that the swizzle at most swaps by halves)
// and the warp's scaled pair table, into `stage` (5 * 32 float4s); the warp
// then writes the staged float4s coalesced.  The values of partial batches
// at both ends, and every value when y is not 16-byte aligned, go singly.
constexpr int kStageQuads = 5 * kWarp;
__device__ __forceinline__ void warp_write(const uint16_t *wd, uint64_t gb, uint32_t wn,
                                           uint64_t n, float *y, bool vec, float scale,
                                           const float2 *sp, float4 *stage, int lane) {
  const uint64_t gal = gb & ~3ull;
  const uint64_t e_begin = 5 * gb, e_end = umin64(5 * (gb + wn), n);
  if (e_end <= e_begin) return;
  auto put = [&](uint64_t e) {
    const uint64_t g = e / 5;
    const uint32_t dig = (wd[wsw((uint32_t)(g - gal))] >> (2 * (uint32_t)(e - 5 * g))) & 3u;
    y[e] = dequant(dig, scale);
  };
  const uint64_t a_lo = (gb + 3) / 4, a_hi = umin64((gb + wn) / 4, n / 20);
  if (!vec || a_hi <= a_lo) {
    for (uint64_t e = e_begin + lane; e < e_end; e += kWarp) put(e);
    return;
  }
  // the partial batches' values: at most 15 at the start and 19 at the end
  const uint32_t h = (uint32_t)(20 * a_lo - e_begin), t = (uint32_t)(e_end - 20 * a_hi);
  for (uint32_t i = lane; i < h + t; i += kWarp) put(i < h ? e_begin + i : 20 * a_hi + (i - h));
  float4 *y4 = reinterpret_cast<float4 *>(y);
  const uint32_t p_lo = (uint32_t)(4 * a_lo - gal);  // window position of batch a_lo
  for (uint64_t a = a_lo; a < a_hi; a += kWarp) {
    const uint32_t nb = (uint32_t)umin64(kWarp, a_hi - a);
    if ((uint32_t)lane < nb) {
      const uint32_t q = wsw(p_lo + 4 * (uint32_t)(a - a_lo) + 4 * lane);
      const uint2 dw = *reinterpret_cast<const uint2 *>(wd + (q & ~3u));
      const uint32_t h0 = (q & 2u) ? dw.y : dw.x;  // words of groups 4a, 4a + 1
      const uint32_t h1 = (q & 2u) ? dw.x : dw.y;  // and 4a + 2, 4a + 3
      // the batch's 20 digits, two bits each: 16 in lo, 4 in hi
      const uint32_t w3 = h1 >> 16;
      const uint32_t lo = (h0 & 0x3ffu) | ((h0 >> 16) << 10) | ((h1 & 0x3ffu) << 20) | (w3 << 30);
      const uint32_t hi = w3 >> 2;
      float4 *sl = stage + 5 * lane;
      sl[0] = quad(sp, lo & 0xffu);
      sl[1] = quad(sp, (lo >> 8) & 0xffu);
      sl[2] = quad(sp, (lo >> 16) & 0xffu);
      sl[3] = quad(sp, lo >> 24);
      sl[4] = quad(sp, hi);
    }
    __syncwarp();
    float4 *dst = y4 + 5 * a;
    for (uint32_t i = lane; i < 5 * nb; i += kWarp) dst[i] = stage[i];
    __syncwarp();
  }
}

// ===================================================================== index
// The index of one stream: per 512-byte payload unit its first group,
// counted from the first group of its 64-unit chunk (loc); per chunk its
// group count, which the scan turns into the chunk's first group (cpre;
// cpre[n_chunks] is then the stream's total).  For sums of several streams
// the same for the non-zero literal groups ("entries": eloc, ecpre).  Two
// kernels: the count (one block per chunk, eight units per warp; no block
// waits on another) and the scan (one block per stream).

static_assert(kDecodeUnit == 4 * 4 * kWarp, "a unit is four 32-bit words per lane");
constexpr uint32_t kWarpUnits = 8;  // units one warp of the count takes
static_assert(kDecodeChunkUnits == kDWarps * kWarpUnits, "a chunk is one count block's units");

// Units u0 .. u0 + 7 of a payload of m bytes, by one warp (every load of
// the eight units issued before any count): lane i < 8 gets the group count
// of unit u0 + i, every other lane 0; bytes past the payload count 0.
// A unit wholly inside a 4-byte aligned payload is read as word lane + 32k
// (k < 4) of the unit, so every load is one coalesced 128-byte line; the
// payload's last unit, and every unit of an unaligned payload, byte by byte
// (lane L: bytes 16L .. 16L + 15).
// With kEnt, ent_out gets the same for the unit's non-zero literal groups.
template <bool kEnt>
__device__ __forceinline__ uint32_t count_units8(const uint8_t *payload, uint64_t m, uint64_t u0,
                                                 uint32_t &ent_out) {
  const uint32_t lane = threadIdx.x & 31;
  ent_out = 0u;
  if (u0 * kDecodeUnit >= m) return 0u;
  const uint64_t whole = m / kDecodeUnit - u0;  // units of this warp wholly inside (>= 0)
  const uint32_t n_word = (reinterpret_cast<uintptr_t>(payload) & 3) == 0
                              ? (uint32_t)umin64(whole, kWarpUnits) : 0u;
  const uint32_t *p32 = reinterpret_cast<const uint32_t *>(payload + u0 * kDecodeUnit) + lane;
  uint32_t w[kWarpUnits][4];
  if (n_word == kWarpUnits) {
#pragma unroll
    for (uint32_t i = 0; i < kWarpUnits; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) w[i][k] = __ldg(p32 + i * (kDecodeUnit / 4) + k * kWarp);
  } else {
    // byte loads where needed; a byte past the payload is read as a
    // literal 121 and its count taken off below
#pragma unroll
    for (uint32_t i = 0; i < kWarpUnits; ++i) {
      if (i < n_word) {
#pragma unroll
        for (int k = 0; k < 4; ++k) w[i][k] = __ldg(p32 + i * (kDecodeUnit / 4) + k * kWarp);
      } else {
        const uint64_t b0 = (u0 + i) * kDecodeUnit + 16ull * lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t x = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t p = b0 + 4 * k + j;
            x |= (p < m ? (uint32_t)__ldg(payload + p) : 121u) << (8 * j);
          }
          w[i][k] = x;
        }
      }
    }
  }
  // a unit expands to at most 512 * 14 < 2^16 groups and has at most 512
  // entries: two units per word, both counts from one pass over the words
  uint32_t pk[kWarpUnits / 2], pe[kWarpUnits / 2];
#pragma unroll
  for (uint32_t i = 0; i < kWarpUnits / 2; ++i) {
    pk[i] = expansion16(w[2 * i]) | (expansion16(w[2 * i + 1]) << 16);
    if (kEnt) pe[i] = literals16(w[2 * i]) | (literals16(w[2 * i + 1]) << 16);
  }
#pragma unroll
  for (uint32_t i = 0; i < kWarpUnits / 2; ++i) {
    pk[i] = __reduce_add_sync(0xffffffffu, pk[i]);
    if (kEnt) pe[i] = __reduce_add_sync(0xffffffffu, pe[i]);
  }
  const uint32_t h = (lane >> 1) & 3u;
  const uint32_t v = h == 0 ? pk[0] : (h == 1 ? pk[1] : (h == 2 ? pk[2] : pk[3]));
  uint32_t mine = lane < kWarpUnits ? ((lane & 1u) ? v >> 16 : v & 0xffffu) : 0u;
  // the padding bytes past the payload counted one group each (and, being
  // 121, no entry)
  if (lane < kWarpUnits) {
    const uint64_t ub = (u0 + lane) * kDecodeUnit;
    mine -= (uint32_t)(ub >= m ? kDecodeUnit : (ub + kDecodeUnit > m ? ub + kDecodeUnit - m : 0));
  }
  if (kEnt) {
    const uint32_t ve = h == 0 ? pe[0] : (h == 1 ? pe[1] : (h == 2 ? pe[2] : pe[3]));
    ent_out = lane < kWarpUnits ? ((lane & 1u) ? ve >> 16 : ve & 0xffffu) : 0u;
  }
  return mine;
}

// Chunk c (64 units) of a stream's payload of m bytes, by one block: warp w
// counts units 8w .. 8w + 7; loc[u] = the unit's first group counted from
// the chunk's first, cnt[c] = the chunk's group count (at most
// 64 * 512 * 14); with kEnt the same for entries in eloc and ecnt.
// wtot_s holds 2 * kDWarps words.  Ends synchronised.
__device__ __forceinline__ uint32_t scan8(uint32_t x, uint32_t lane) {
#pragma unroll
  for (uint32_t d = 1; d < kWarpUnits; d <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += t;
  }
  return x;
}
template <bool kEnt>
__device__ __forceinline__ void count_chunk(const uint8_t *payload, uint64_t m, uint32_t c,
                                            uint32_t *loc, uint32_t *cnt, uint32_t *eloc,
                                            uint32_t *ecnt, uint32_t *wtot_s) {
  const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t n_units = (m + kDecodeUnit - 1) / kDecodeUnit;
  const uint64_t u0 = (uint64_t)c * kDecodeChunkUnits + warp * kWarpUnits;
  uint32_t ent = 0;
  const uint32_t mine = count_units8<kEnt>(payload, m, u0, ent);
  const uint32_t inc = scan8(mine, lane), einc = scan8(ent, lane);
  if (lane == kWarpUnits - 1) {
    wtot_s[warp] = inc;
    wtot_s[kDWarps + warp] = einc;
  }
  __syncthreads();
  uint32_t off = 0, eoff = 0;
  for (uint32_t w = 0; w < warp; ++w) {
    off += wtot_s[w];
    eoff += wtot_s[kDWarps + w];
  }
  if (lane < kWarpUnits && u0 + lane < n_units) {
    loc[u0 + lane] = off + inc - mine;
    if (kEnt) eloc[u0 + lane] = eoff + einc - ent;
  }
  if (warp == kDWarps - 1 && lane == kWarpUnits - 1) {
    cnt[c] = off + inc;
    if (kEnt) ecnt[c] = eoff + einc;
  }
  __syncthreads();  // wtot_s is rewritten by the next chunk
}

// What the scan of one array of one stream writes.
struct IndexOut {
  uint32_t *cpre;      // chunk counts in, first groups (or entries) out, then the total
  uint32_t *ok;        // or nullptr: 1 when the stream expands to exactly `groups`, else 0
  uint64_t groups;
  uint32_t *tail;      // or nullptr: also gets the total
};

__device__ __forceinline__ uint32_t sat32(uint64_t v) { return (uint32_t)umin64(v, 0xffffffffull); }

// The stream's chunk counts, scanned by one block of kThreads into each
// chunk's first group (or entry) and the total, checked against the
// tensor's groups when s.ok is set.  In passes of up to kScanPer chunks per
// thread: each thread loads its contiguous share into registers (all loads
// issued first), then a block scan of the shares (64-bit: a corrupt
// stream's counts may add up past 2^32).  wsum holds kThreads / 32 + 1
// words.
constexpr int kScanPer = 8;
template <int kThreads>
__device__ void scan_chunks(const IndexOut &s, uint32_t n_chunks, uint64_t *wsum,
                            int32_t *dev_status) {
  constexpr int kWarps = kThreads / kWarp;
  static_assert(kWarps <= kWarp, "one warp scans the warp sums");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t carry = 0;
  for (uint32_t base = 0; base < n_chunks;) {
    const uint32_t per = min((uint32_t)kScanPer, (n_chunks - base + kThreads - 1) / kThreads);
    const uint32_t c0 = base + threadIdx.x * per;
    const uint32_t cend = min(c0 + per, n_chunks);
    base += kThreads * per;
    uint32_t v[kScanPer];
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) v[i] = c0 + i < cend ? __ldcg(s.cpre + c0 + i) : 0u;
    uint64_t sum = 0;
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) sum += v[i];
    uint64_t inc = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint64_t t = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += t;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const uint64_t x = lane < kWarps ? wsum[lane] : 0;
      uint64_t y = x;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint64_t t = __shfl_up_sync(0xffffffffu, y, d);
        if (lane >= d) y += t;
      }
      if (lane < kWarps) wsum[lane] = y - x;
      if (lane == 31) wsum[kWarps] = y;
    }
    __syncthreads();
    uint64_t run = carry + wsum[warp] + inc - sum;
    carry += wsum[kWarps];
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
      const uint32_t c = c0 + i;
      if (c < cend) {
        s.cpre[c] = sat32(run);
        run += v[i];
      }
    }
    __syncthreads();  // wsum is rewritten by the next pass
  }
  if (threadIdx.x == 0) {
    s.cpre[n_chunks] = sat32(carry);
    if (s.tail) *s.tail = sat32(carry);
    if (s.ok) {
      const bool ok = carry == s.groups;
      *s.ok = ok ? 1u : 0u;
      if (!ok) report(dev_status, TLC_ERR_CORRUPT);
    }
  }
}

// Up to kIndexPass streams of n values each, indexed and decoded by one
// launch sequence.  The entry arrays are set for sums of several streams.
struct IxStream {
  const uint8_t *in;
  const uint64_t *len_dev;
  uint64_t cap;
  uint32_t *loc;
  uint32_t *cpre;
  uint32_t *eloc;      // or nullptr: units' first entries within their chunk
  uint32_t *ecpre;     // chunks' first entries, then the total
  uint32_t *list;      // entries: (group - tile's first) << 16 | digit word, in group order
  uint32_t *tfe;       // per sum tile: its first entry; tfe[n_tiles] = the total
};
struct IxArgs {
  IxStream s[kIndexPass];
  int k;
  uint64_t n, groups;
  uint32_t *ticket2;   // decode tiles (cleared by the scan)
  uint32_t *ok;        // per stream (written by the scan)
  float *y;
  bool vec;
  int32_t *dev_status;
};

__device__ __forceinline__ uint32_t chunks_of(uint64_t m) {
  return (uint32_t)((m + (uint64_t)kDecodeUnit * kDecodeChunkUnits - 1) /
                    ((uint64_t)kDecodeUnit * kDecodeChunkUnits));
}

// Groups per tile of a sum of several streams.
#ifndef TLC_SUM_TILE
#define TLC_SUM_TILE 2048
#endif
constexpr uint32_t kSumTile = TLC_SUM_TILE;
static_assert(kSumTile % 16 == 0 && kSumTile <= 65536, "a tile position fits 16 bits");
__host__ __device__ __forceinline__ uint32_t sum_tiles(uint64_t groups) {
  return (uint32_t)((groups + kSumTile - 1) / kSumTile);
}

// Valid streams' payload lengths (0 for a corrupt one) into m_s and the
// running count of their `per(m)` items into pre_s (k + 1 words); whole
// block, ends synchronised.
template <typename F>
__device__ __forceinline__ void stream_prefix(const IxArgs &a, uint64_t *m_s, uint32_t *pre_s,
                                              F per) {
  if (threadIdx.x < (unsigned)a.k) {
    const IxStream &S = a.s[threadIdx.x];
    uint64_t m = 0;
    float scale = 0.0f;
    m_s[threadIdx.x] = read_stream_header(S.in, S.len_dev, S.cap, a.groups, m, scale) ? m : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    pre_s[0] = 0;
    for (int s = 0; s < a.k; ++s) pre_s[s + 1] = pre_s[s] + per(m_s[s]);
  }
  __syncthreads();
}

// Count of every stream: the chunks that exist (from each stream's length;
// none for a corrupt one), numbered stream by stream; block b takes chunks
// b, b + grid, ...
template <bool kEnt>
__global__ void __launch_bounds__(kDThreads, 4) k_index_count(const IxArgs a) {
  __shared__ uint64_t m_s[kIndexPass];
  __shared__ uint32_t pre_s[kIndexPass + 1];
  __shared__ uint32_t wtot_s[2 * kDWarps];
  pdl_enter();
  stream_prefix(a, m_s, pre_s, [](uint64_t m) { return chunks_of(m); });
  const uint32_t total = pre_s[a.k];
  for (uint32_t t = blockIdx.x; t < total; t += gridDim.x) {
    int s = 0;
    while (s + 1 < a.k && pre_s[s + 1] <= t) ++s;
    const IxStream &S = a.s[s];
    count_chunk<kEnt>(S.in + 4, m_s[s], t - pre_s[s], S.loc, S.cpre, S.eloc, S.ecpre, wtot_s);
  }
}

// Scan of every stream, block s for stream s (a corrupt stream gets ok = 0
// and a report); block 0 also clears the decode ticket.
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) k_index_scan(const IxArgs a) {
  __shared__ uint64_t wsum[kScanThreads / kWarp + 1];
  __shared__ uint64_t m_s;
  __shared__ int valid_s;
  pdl_enter();
  const int s = blockIdx.x;
  const IxStream &S = a.s[s];
  if (threadIdx.x == 0) {
    uint64_t m = 0;
    float scale = 0.0f;
    valid_s = read_stream_header(S.in, S.len_dev, S.cap, a.groups, m, scale) ? 1 : 0;
    m_s = m;
    if (s == 0) *a.ticket2 = 0u;
  }
  __syncthreads();
  if (!valid_s) {
    if (threadIdx.x == 0) {
      a.ok[s] = 0u;
      report(a.dev_status, TLC_ERR_CORRUPT);
    }
    return;
  }
  const uint32_t nc = chunks_of(m_s);
  const IndexOut io = {S.cpre, a.ok + s, a.groups, nullptr};
  scan_chunks<kScanThreads>(io, nc, wsum, a.dev_status);
  if (S.ecpre) {
    const IndexOut eo = {S.ecpre, nullptr, 0, S.tfe + sum_tiles(a.groups)};
    scan_chunks<kScanThreads>(eo, nc, wsum, a.dev_status);
  }
}

// ============================================================= warp units
// One 512-byte payload unit of an indexed stream, by one warp.  The unit's
// first group is cpre[u / 32] + loc[u].  Its groups are decoded in windows
// of kWarpGroups: the window is pre-filled with the zero group's digit word,
// the unit's literal groups in the window are placed as their digit words
// (lut[] of the byte) in the warp's own shared memory, and warp_write writes
// (or adds) the window's values; the float4s that straddle a window's or the
// unit's end become single values.  A unit without non-zero literals is
// plain zeros (dense output) or nothing (accumulate); an accumulate unit
// whose literals are few visits only its literal groups.  No warp waits on
// another.
#ifndef TLC_WARP_GROUPS
#define TLC_WARP_GROUPS 1024
#endif
constexpr uint32_t kWarpGroups = TLC_WARP_GROUPS;
static_assert(kWarpGroups % 16 == 0, "whole swizzle blocks of digit words");
constexpr uint32_t kZeroDigits2 = 0x01550155u;  // two digit words of the zero group 121
// A unit's literal-group list in the accumulate mode's sparse case (fewer
// than one literal group per 16 groups, so at most 14 * 512 / 16 entries)
// sits in the warp's window, one word per entry; an entry of a group past
// the tensor is kNoListEntry.
constexpr uint32_t kListCap = (kWarpGroups + 16) / 2;
static_assert(kListCap >= 14 * kDecodeUnit / 16, "a sparse unit's literal list fits the window");
static_assert(14 * kDecodeUnit <= (1u << 13), "a group offset within a unit fits 13 bits");
constexpr uint32_t kNoListEntry = 0xffffffffu;

__device__ __forceinline__ uint64_t unit_first_group(const uint32_t *cpre, const uint32_t *loc,
                                                     uint32_t u) {
  return (uint64_t)__ldg(cpre + (u / kDecodeChunkUnits)) + __ldg(loc + u);
}

// One unit by one warp; sp is the warp's scaled pair table (for j's scale),
// wd its window of digit words, stage its staging for dense output.
template <int kMode>
__device__ __forceinline__ void decode_unit(const DecodeJob &j, uint32_t u, const uint16_t *lut,
                                            const float2 *sp, uint16_t *wd, float4 *stage) {
  const int lane = threadIdx.x & 31;
  const uint64_t base = (uint64_t)u * kDecodeUnit + 16ull * lane;
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  int nb = 0;
  if (base < j.m) {
    const uint64_t left = j.m - base;
    const uint8_t *p = j.payload + base;
    if (left >= 16 && (reinterpret_cast<uintptr_t>(p) & 3) == 0) {
      const uint32_t *p32 = reinterpret_cast<const uint32_t *>(p);
#pragma unroll
      for (int k = 0; k < 4; ++k) w[k] = __ldg(p32 + k);
      nb = 16;
    } else {
      nb = (int)umin64(left, 16);
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (k < nb) w[k >> 2] |= (uint32_t)__ldg(p + k) << (8 * (k & 3));
    }
  }
  uint32_t e = 0, lits = 0;
  if (nb == 16) {
    e = expansion16(w);
    lits = literals16(w);
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k < nb) {
        const uint32_t b = (w[k >> 2] >> (8 * (k & 3))) & 0xffu;
        e += expansion(b);
        lits += (b < 243u && b != 121u) ? 1u : 0u;
      }
    }
  }
  uint32_t inc = e;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += t;
  }
  const uint32_t E = __shfl_sync(0xffffffffu, inc, 31);
  const uint32_t L = __reduce_add_sync(0xffffffffu, lits);
  const uint32_t excl = inc - e;
  const uint64_t O = unit_first_group(j.cpre, j.loc, u);
  const uint32_t Ec = O >= j.groups ? 0u : (uint32_t)umin64(E, j.groups - O);
  if (L == 0) {
    if (kMode == kWrite) emit_zeros(5 * O, umin64(5 * (O + Ec), j.n), j.y, j.vec, lane, kWarp);
    return;
  }
  if (kMode == kAccumulate && 16 * L < E) {
    // long zero runs around a few literals: the warp lists the unit's
    // literal groups in its window (in group order: the group's offset from
    // O in bits 0..12, its digit word in bits 13..22), then each lane takes
    // list entries i and i + 32 of every 64 and loads both groups' values
    // before adding to either, so no lane walks a run of literals alone
    uint32_t lpre = lits;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, lpre, d);
      if (lane >= d) lpre += t;
    }
    uint32_t *list = reinterpret_cast<uint32_t *>(wd);
    uint32_t at = lpre - lits, rel = excl;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k < nb) {
        const uint32_t b = (w[k >> 2] >> (8 * (k & 3))) & 0xffu;
        if (b >= 243u) {
          rel += b - 241u;
        } else {
          if (b != 121u && TLC_CHECK(at < kListCap))
            list[at++] = O + rel < j.groups ? rel | ((uint32_t)lut[b] << 13) : kNoListEntry;
          ++rel;
        }
      }
    }
    __syncwarp();
    for (uint32_t i = lane; i < L; i += 2 * kWarp) {
      const uint32_t ea = list[i];
      const uint32_t eb = i + kWarp < L ? list[i + kWarp] : kNoListEntry;
      // each group's values in acc and how many of its five exist (n may
      // end inside the last group)
      const uint64_t ea5 = 5 * (O + (ea & 0x1fffu)), eb5 = 5 * (O + (eb & 0x1fffu));
      float *ya = j.y + ea5, *yb = j.y + eb5;
      const uint32_t na = ea == kNoListEntry ? 0u : (uint32_t)umin64(5, j.n - ea5);
      const uint32_t nb2 = eb == kNoListEntry ? 0u : (uint32_t)umin64(5, j.n - eb5);
      const uint32_t da = ea >> 13, db = eb >> 13;
      float va[5], vb[5];
#pragma unroll
      for (int d = 0; d < 5; ++d) {
        va[d] = (((da >> (2 * d)) & 3u) != 1u && (uint32_t)d < na) ? ya[d] : 0.0f;
        vb[d] = (((db >> (2 * d)) & 3u) != 1u && (uint32_t)d < nb2) ? yb[d] : 0.0f;
      }
#pragma unroll
      for (int d = 0; d < 5; ++d) {
        const uint32_t qa = (da >> (2 * d)) & 3u, qb = (db >> (2 * d)) & 3u;
        if (qa != 1u && (uint32_t)d < na) ya[d] = __fadd_rn(va[d], dequant(qa, j.scale));
        if (qb != 1u && (uint32_t)d < nb2) yb[d] = __fadd_rn(vb[d], dequant(qb, j.scale));
      }
    }
    __syncwarp();  // the window is free again for the warp's next unit
    return;
  }
  for (uint32_t w0 = 0; w0 < Ec; w0 += kWarpGroups) {
    const uint32_t wn = min(kWarpGroups, Ec - w0);
    // window positions count from the window's first group rounded down to
    // a multiple of 4: groups at off .. off + wn - 1
    const uint64_t gb = O + w0;
    const uint32_t off = (uint32_t)(gb & 3u);
    // positions 0 .. off + wn (the last one read by a float4 that spills),
    // in whole swizzle blocks of 16
    for (uint32_t q = lane; q < 2 * ((off + wn) / 16 + 1); q += kWarp)
      reinterpret_cast<uint4 *>(wd)[q] = make_uint4(kZeroDigits2, kZeroDigits2, kZeroDigits2,
                                                    kZeroDigits2);
    __syncwarp();
    uint32_t pos = excl;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k < nb) {
        const uint32_t b = (w[k >> 2] >> (8 * (k & 3))) & 0xffu;
        if (b >= 243u) {
          pos += b - 241u;
        } else {
          if (pos - w0 < wn) wd[wsw(pos - w0 + off)] = lut[b];  // unsigned: pos in [w0, w0 + wn)
          ++pos;
        }
      }
    }
    __syncwarp();
    if (kMode == kWrite)
      warp_write(wd, gb, wn, j.n, j.y, j.vec, j.scale, sp, stage, lane);
    else
      warp_accumulate(wd, gb - off, 5 * gb, umin64(5 * (gb + wn), j.n), j.y, j.vec, j.scale, sp,
                      lane);
    __syncwarp();
  }
}

// Streams that expand to more than this many groups per payload byte on
// average are written by block-wide payload tiles instead of warp units.
#ifndef TLC_SPARSE_EXPANSION
#define TLC_SPARSE_EXPANSION 4
#endif

// Shared memory of a block of warp-unit decoders: per warp its scaled pair
// table, its window of digit words (positions up to kWarpGroups + 3, filled
// in whole swizzle blocks) and, for dense output, its staging.
template <int kMode>
struct UnitSmem {
  DecodeSmem d;   // digit table, block scan, a tile's first group
  float2 sp[kDWarps][16];
  __align__(16) uint16_t wd[kDWarps][kWarpGroups + 16];
  __align__(16) float4 stage[kMode == kWrite ? kDWarps : 1][kStageQuads];
};
static_assert(sizeof(UnitSmem<kWrite>::wd) >= DecodeShape<kWrite>::kMaxGroups + 16,
              "a dense-output payload tile's groups fit the warps' windows");

template <int kMode>
__device__ __forceinline__ float4 *unit_stage(UnitSmem<kMode> &sm, int warp) {
  return sm.stage[kMode == kWrite ? warp : 0];
}

// One indexed stream (dense output, or added into acc): warp w of block b
// takes units b * warps + w, then every (grid's warps)-th unit.  A sparse
// stream's dense output is written by whole blocks instead, one 512-byte
// payload tile (unit) per block in ticket order: its all-zero tiles are each
// one long run of zero stores, which a block writes faster than a warp.
// Blocks per SM the warp-unit kernels are compiled for: the accumulate
// emit keeps two float4s of acc per lane in flight, and the plan kernel
// tracks its tensor: both need the registers of 6 blocks.  Dense output
// runs 5 (its staging's shared memory).
template <int kMode>
constexpr int units_min_blocks(bool batch) {
  return kMode == kWrite ? 5 : 6;  // dense output: its staging allows 5 blocks
}

template <int kMode>
__global__ void __launch_bounds__(kDThreads, units_min_blocks<kMode>(false))
    k_decode_units(const IxArgs a) {
  __shared__ UnitSmem<kMode> sm;
  __shared__ DecodeJob job_s;
  __shared__ int ok_s;
  __shared__ uint32_t tile_s;
  fill_lut(sm.d.lut);
  pdl_enter();
  if (threadIdx.x == 0) {
    const IxStream &S = a.s[0];
    uint64_t m = 0;
    float scale = 0.0f;
    ok_s = a.ok[0] && read_stream_header(S.in, S.len_dev, S.cap, a.groups, m, scale);
    DecodeJob j;
    j.payload = S.in + 4;
    j.m = m;
    j.n = a.n;
    j.groups = a.groups;
    j.scale = scale;
    j.y = a.y;
    j.status = nullptr;
    j.n_tiles = (uint32_t)((m + kDecodeUnit - 1) / kDecodeUnit);
    j.vec = a.vec;
    j.loc = S.loc;
    j.cpre = S.cpre;
    job_s = j;
  }
  __syncthreads();
  if (!ok_s) return;
  if (kMode == kWrite && job_s.groups > (uint64_t)TLC_SPARSE_EXPANSION * job_s.m) {
    static_assert(DecodeShape<kWrite>::kTile == kDecodeUnit, "dense-output tiles are units");
    uint8_t *grp = reinterpret_cast<uint8_t *>(&sm.wd[0][0]);
    for (;;) {
      if (threadIdx.x == 0) tile_s = atomicAdd(a.ticket2, 1u);
      __syncthreads();
      const uint32_t t = tile_s;
      if (t >= job_s.n_tiles) break;
      decode_tile<kWrite, true>(job_s, t, sm.d, grp, a.dev_status, 0u);
    }
    return;
  }
  // the job stays in shared memory: its fields are read where they are used
  const int warp = threadIdx.x >> 5;
  const uint32_t nw = gridDim.x * kDWarps;
  fill_scaled_pairs(sm.sp[warp], job_s.scale, threadIdx.x & 31);
  for (uint32_t u = blockIdx.x * kDWarps + warp; u < job_s.n_tiles; u += nw)
    decode_unit<kMode>(job_s, u, sm.d.lut, sm.sp[warp], sm.wd[warp], unit_stage(sm, warp));
}

// ======================================================= sums of streams
// Entries: one warp per unit of every valid stream (numbered stream by
// stream).  Lane L takes the unit's bytes 16L .. 16L + 15; warp scans give
// its first group (cpre + loc) and first entry (ecpre + eloc).  Each
// non-zero literal group g becomes entry list[e] = (g mod kSumTile) << 16 |
// its digit word, and every tile boundary b * kSumTile that falls in the
// lane's groups gets tfe[b] = the index of the first entry at or after it.
// Units are disjoint runs of groups, so every entry and boundary is written
// once, and the list is in group order.
__global__ void __launch_bounds__(kDThreads) k_index_entries(const IxArgs a) {
  __shared__ uint64_t m_s[kIndexPass];
  __shared__ uint32_t pre_s[kIndexPass + 1];
  __shared__ uint16_t lut[256];
  fill_lut(lut);
  pdl_enter();
  stream_prefix(a, m_s, pre_s, [](uint64_t m) {
    return (uint32_t)((m + kDecodeUnit - 1) / kDecodeUnit);
  });
  const uint32_t total = pre_s[a.k];
  const int lane = threadIdx.x & 31;
  const uint32_t nw = gridDim.x * kDWarps;
  for (uint32_t t = blockIdx.x * kDWarps + (threadIdx.x >> 5); t < total; t += nw) {
    int s = 0;
    while (s + 1 < a.k && pre_s[s + 1] <= t) ++s;
    if (!a.ok[s]) continue;  // uniform in the warp
    const IxStream &S = a.s[s];
    const uint32_t u = t - pre_s[s];
    const uint64_t m = m_s[s];
    const uint8_t *payload = S.in + 4;
    const uint64_t base = (uint64_t)u * kDecodeUnit + 16ull * lane;
    uint32_t w[4] = {0x79797979u, 0x79797979u, 0x79797979u, 0x79797979u};
    int nb = 0;
    if (base < m) {
      const uint64_t left = m - base;
      const uint8_t *p = payload + base;
      if (left >= 16 && (reinterpret_cast<uintptr_t>(p) & 3) == 0) {
        const uint32_t *p32 = reinterpret_cast<const uint32_t *>(p);
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = __ldg(p32 + k);
        nb = 16;
      } else {
        nb = (int)umin64(left, 16);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (k < nb)
            w[k >> 2] = (w[k >> 2] & ~(0xffu << (8 * (k & 3)))) |
                        ((uint32_t)__ldg(p + k) << (8 * (k & 3)));
      }
    }
    const uint32_t c0 = u / kDecodeChunkUnits;
    const uint64_t g_unit = (uint64_t)__ldg(S.cpre + c0) + __ldg(S.loc + u);
    const uint64_t e_unit = (uint64_t)__ldg(S.ecpre + c0) + __ldg(S.eloc + u);
    // padding bytes (past the payload) are literal 121s: one group, no entry
    const uint32_t eg = nb > 0 ? expansion16(w) - (16u - (uint32_t)nb) : 0u;
    const uint32_t ee = nb > 0 ? literals16(w) : 0u;
    uint32_t ig = eg, ie = ee;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t tg = __shfl_up_sync(0xffffffffu, ig, d);
      const uint32_t te = __shfl_up_sync(0xffffffffu, ie, d);
      if (lane >= d) {
        ig += tg;
        ie += te;
      }
    }
    uint64_t g = g_unit + ig - eg;
    uint32_t e = (uint32_t)(e_unit + ie - ee);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k < nb) {
        const uint32_t b = (w[k >> 2] >> (8 * (k & 3))) & 0xffu;
        const uint32_t run = b >= 243u ? b - 241u : 1u;
        // a tile boundary among this byte's groups [g, g + run) (run < kSumTile)
        const uint64_t bnd = (g + kSumTile - 1) / kSumTile;
        if (bnd * kSumTile < g + run && TLC_CHECK(bnd <= sum_tiles(a.groups)))
          S.tfe[bnd] = e;
        if (b < 243u && b != 121u) {
          if (TLC_CHECK(e < m)) S.list[e] = ((uint32_t)(g % kSumTile) << 16) | lut[b];
          ++e;
        }
        g += run;
      }
    }
  }
}

// Sum tiles: kSumTile groups of acc, one block each (block b takes tiles
// b, b + grid, ...).  Every valid stream's entries of the tile
// [tfe[t], tfe[t + 1]) go to the tile's digit words in shared memory (kK *
// kSumTile words) and set the stream's bit in their group's mask byte.
// Then each thread takes whole groups: it reads the values of a marked
// group that some stream changes once, adds the marking streams' values in
// stream order and writes them once.  No value is touched by two threads,
// so the streams need no barrier between them.
// Groups of a thread whose acc values are loaded together, and the blocks
// per SM the kernel is compiled for.
#ifndef TLC_SUM_AT
#define TLC_SUM_AT 2
#endif
#ifndef TLC_SUM_MINB
#define TLC_SUM_MINB 5
#endif
template <int kK>
__global__ void __launch_bounds__(kDThreads, TLC_SUM_MINB) k_apply_entries(const IxArgs a) {
  extern __shared__ __align__(16) uint8_t dyn_s[];  // mask bytes, then digit words
  __shared__ float scale_s[kK];
  __shared__ const uint32_t *list_s[kK];  // per-lane stream choice: read from shared memory
  __shared__ uint32_t lo_s[kK], cnt_s[kK + 1];
  uint32_t *mask = reinterpret_cast<uint32_t *>(dyn_s);
  uint16_t *wd = reinterpret_cast<uint16_t *>(dyn_s + kSumTile);
  pdl_enter();
  if (threadIdx.x < (unsigned)kK) {
    float scale = 0.0f;
    const uint32_t *list = nullptr;
    if ((int)threadIdx.x < a.k) {
      const IxStream &S = a.s[threadIdx.x];
      uint64_t m = 0;
      list = S.list;
      if (!a.ok[threadIdx.x] || !read_stream_header(S.in, S.len_dev, S.cap, a.groups, m, scale))
        scale = -1.0f;  // left out
    }
    scale_s[threadIdx.x] = scale;
    list_s[threadIdx.x] = list;
  }
  __syncthreads();
  const uint32_t n_tiles = sum_tiles(a.groups);
  for (uint32_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const uint64_t g0 = (uint64_t)t * kSumTile;
    const uint32_t gn = (uint32_t)umin64(kSumTile, a.groups - g0);
    for (uint32_t i = threadIdx.x; i < kSumTile / 16; i += kDThreads)
      reinterpret_cast<uint4 *>(mask)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x < (unsigned)kK) {
      uint32_t lo = 0, hi = 0;
      if ((int)threadIdx.x < a.k && scale_s[threadIdx.x] >= 0.0f) {
        lo = __ldg(a.s[threadIdx.x].tfe + t);
        hi = __ldg(a.s[threadIdx.x].tfe + t + 1);
        if (hi < lo) hi = lo;
      }
      lo_s[threadIdx.x] = lo;
      cnt_s[threadIdx.x] = hi - lo;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t run = 0;
      for (int s = 0; s < kK; ++s) {
        const uint32_t c = cnt_s[s];
        cnt_s[s] = run;
        run += c;
      }
      cnt_s[kK] = run;
    }
    __syncthreads();
    const uint32_t all = cnt_s[kK];
    if (all == 0) continue;  // uniform; nothing here reads the tile's shared memory
    // the tile's entries of every stream, flattened
    for (uint32_t i = threadIdx.x; i < all; i += kDThreads) {
      int s = 0;
      while (s + 1 < kK && cnt_s[s + 1] <= i) ++s;
      const uint32_t ent = __ldg(list_s[s] + lo_s[s] + (i - cnt_s[s]));
      const uint32_t p = ent >> 16;
      if (TLC_CHECK(p < gn)) {
        wd[s * kSumTile + p] = (uint16_t)(ent & 0x3ffu);
        atomicOr(mask + (p >> 2), 1u << (8 * (p & 3) + s));
      }
    }
    __syncthreads();
    // this thread's groups are i = threadIdx.x + kDThreads * j; the marked
    // ones four at a time: first, from shared memory alone, which of their
    // values some stream changes, then those values loaded (all before any
    // add), the streams' values added in stream order, and written
    static_assert(kSumTile / kDThreads <= 32, "a thread's groups fit one word of bits");
    const uint8_t *mb = reinterpret_cast<const uint8_t *>(mask);
    uint32_t todo = 0;
#pragma unroll
    for (uint32_t j = 0; j < kSumTile / kDThreads; ++j) {
      const uint32_t i = threadIdx.x + kDThreads * j;
      if (i < gn && mb[i]) todo |= 1u << j;
    }
    while (todo) {
      constexpr int kAt = TLC_SUM_AT;
      uint32_t gi[kAt], tch[kAt];
#pragma unroll
      for (int q = 0; q < kAt; ++q) {
        gi[q] = 0u;
        tch[q] = 0u;
        if (todo) {
          const uint32_t i = threadIdx.x + kDThreads * (uint32_t)(__ffs(todo) - 1);
          todo &= todo - 1;
          gi[q] = i;
          uint32_t mk = mb[i], t = 0;
          while (mk) {
            const int st = __ffs(mk) - 1;
            mk &= mk - 1;
            const uint32_t dw = wd[st * kSumTile + i];
            // digit d is not zero (not 1): bit 2d of dw clear
#pragma unroll
            for (int d = 0; d < 5; ++d) t |= (((dw >> (2 * d)) & 1u) ^ 1u) << d;
          }
          const uint64_t e0 = 5 * (g0 + i);
          tch[q] = t & ((1u << (uint32_t)umin64(5, a.n - e0)) - 1u);  // the last group may be short
        }
      }
      float v[kAt][5];
#pragma unroll
      for (int q = 0; q < kAt; ++q) {
        const uint64_t e0 = 5 * (g0 + gi[q]);
#pragma unroll
        for (int d = 0; d < 5; ++d) v[q][d] = ((tch[q] >> d) & 1u) ? a.y[e0 + d] : 0.0f;
      }
#pragma unroll
      for (int q = 0; q < kAt; ++q) {
        if (!tch[q]) continue;
        const uint32_t i = gi[q];
        const uint64_t e0 = 5 * (g0 + i);
        uint32_t mk = mb[i];
        while (mk) {
          const int st = __ffs(mk) - 1;
          mk &= mk - 1;
          const uint32_t dw = wd[st * kSumTile + i];
          const float sc = scale_s[st];
#pragma unroll
          for (int d = 0; d < 5; ++d) {
            const uint32_t dig = (dw >> (2 * d)) & 3u;
            if (dig != 1u) v[q][d] = __fadd_rn(v[q][d], dequant(dig, sc));
          }
        }
#pragma unroll
        for (int d = 0; d < 5; ++d)
          if ((tch[q] >> d) & 1u) a.y[e0 + d] = v[q][d];
      }
    }
    __syncthreads();  // the tile's shared memory is rewritten by the next tile
  }
}

template <int kK>
constexpr size_t apply_smem_bytes() {
  return (size_t)kSumTile + (size_t)kK * kSumTile * sizeof(uint16_t);
}

// ================================================================= batches
struct BatchDecodeArgs {
  const BatchTensor *tensors;
  uint32_t count;
  const BatchPrep *prep;        // per-tensor payload length, scale, tiling, first tile
  const uint32_t *total;        // tiles and chunks in the compact numbering
  uint32_t n_tiles;             // upper bound of total[0] (sizes the grid)
  const uint8_t *arena;
  uint64_t *status;
  uint32_t *ticket;
  int32_t *dev_status;
  uint32_t max_polls;
  uint32_t *loc;                // indexed plans: units' first groups in their chunk,
  uint32_t *cpre;               // chunks' first groups (d_chunks + 1 per tensor),
  uint32_t *ok;                 // valid flags (written by the scan)
  uint32_t n_chunks;            // chunks of all tensors (upper bound)
};

constexpr int kPrepThreads = 1024;
constexpr uint32_t kSmemSearch = 2048;  // tensors whose first tiles fit in shared memory
constexpr uint32_t kSmemSearchUnits = 1024;  // the same in the warp-unit kernel (less room)

// One block: validate every tensor's stream once, and number the tiles that
// actually exist (ceil(m / tile_bytes) per stream, none for a corrupt one)
// consecutively, tensor by tensor; the same for the index's 64-unit chunks.
// total[0] = tiles, total[1] = chunks.
__global__ void __launch_bounds__(kPrepThreads)
k_decode_batch_prepare(const BatchTensor *__restrict__ tensors, uint32_t count,
                       const uint8_t *__restrict__ arena, const uint64_t *__restrict__ in_lens,
                       uint32_t tile_bytes, BatchPrep *__restrict__ prep,
                       uint32_t *__restrict__ total, int32_t *dev_status) {
  __shared__ uint32_t scan_s[kPrepThreads / kWarp + 1];
  pdl_enter();
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
      p.valid = m > 0 ? 1u : 0u;
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

// Last tensor whose first numbered item (begin) is <= u; tensors without
// items share their first item with the next tensor and are skipped.
__device__ __forceinline__ uint32_t find_tensor(const uint32_t *begin_s, bool in_smem,
                                                const BatchPrep *prep, uint32_t count, uint32_t u,
                                                bool chunks) {
  uint32_t lo = 0, hi = count - 1;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    const uint32_t b = in_smem ? begin_s[mid] : (chunks ? prep[mid].cact_begin
                                                          : prep[mid].act_begin);
    if (b <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Small plans: the payload tiles of every tensor in one ticket order, each
// look-back confined to its stream.
template <int kMode>
__global__ void __launch_bounds__(kDThreads) k_decode_batch(const BatchDecodeArgs a) {
  constexpr int kDTile = DecodeShape<kMode>::kTile;
  extern __shared__ __align__(16) uint8_t grp_s[];
  __shared__ DecodeSmem sm;
  __shared__ uint32_t begin_s[kSmemSearch];
  __shared__ uint32_t tile_s;
  fill_lut(sm.lut);
  pdl_enter();
  const bool in_smem = a.count <= kSmemSearch;
  if (in_smem)
    for (uint32_t i = threadIdx.x; i < a.count; i += kDThreads) begin_s[i] = a.prep[i].act_begin;
  const uint32_t total = *a.total;
  for (;;) {
    if (threadIdx.x == 0) tile_s = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t u = tile_s;
    if (u >= total) break;
    const uint32_t id = find_tensor(begin_s, in_smem, a.prep, a.count, u, false);
    const BatchTensor &T = a.tensors[id];
    const BatchPrep &P = a.prep[id];
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
    decode_tile<kMode>(job, u - P.act_begin, sm, grp_s, a.dev_status, a.max_polls);
  }
}

// Count of a plan's streams: the chunks that exist, numbered tensor by
// tensor by the prepare kernel; block b takes chunks b, b + grid, ...
__global__ void __launch_bounds__(kDThreads, 4) k_index_count_batch(const BatchDecodeArgs a) {
  __shared__ uint32_t begin_s[kSmemSearch];
  __shared__ uint32_t wtot_s[2 * kDWarps];
  pdl_enter();
  const bool in_smem = a.count <= kSmemSearch;
  if (in_smem)
    for (uint32_t i = threadIdx.x; i < a.count; i += kDThreads) begin_s[i] = a.prep[i].cact_begin;
  __syncthreads();
  const uint32_t total = a.total[1];
  for (uint32_t g = blockIdx.x; g < total; g += gridDim.x) {
    const uint32_t id = find_tensor(begin_s, in_smem, a.prep, a.count, g, true);
    const BatchTensor &T = a.tensors[id];
    const BatchPrep &P = a.prep[id];
    count_chunk<false>(a.arena + T.arena_off + 4, P.m, g - P.cact_begin, a.loc + T.d_tile_begin,
                       a.cpre + T.d_chunk_begin + id, nullptr, nullptr, wtot_s);
  }
}

// Scan of a plan's streams: block b takes tensors b, b + grid, ...; a
// tensor whose stream the prepare kernel found corrupt gets ok = 0.
__global__ void __launch_bounds__(kDThreads) k_index_scan_batch(const BatchDecodeArgs a) {
  __shared__ uint64_t wsum[kDWarps + 1];
  pdl_enter();
  for (uint32_t id = blockIdx.x; id < a.count; id += gridDim.x) {
    const BatchTensor &T = a.tensors[id];
    const BatchPrep &P = a.prep[id];
    if (!P.valid) {
      if (threadIdx.x == 0) a.ok[id] = 0u;
      continue;
    }
    const IndexOut io = {a.cpre + T.d_chunk_begin + id, a.ok + id, T.groups, nullptr};
    scan_chunks<kDThreads>(io, chunks_of(P.m), wsum, a.dev_status);
  }
}

// Large plans: every tensor's 512-byte units (numbered tensor by tensor by
// the prepare kernel), one warp per unit as in k_decode_units; a tensor the
// index did not mark valid is left out.
template <int kMode>
__global__ void __launch_bounds__(kDThreads, units_min_blocks<kMode>(true))
    k_decode_batch_units(const BatchDecodeArgs a) {
  __shared__ UnitSmem<kMode> sm;
  __shared__ uint32_t begin_s[kSmemSearchUnits];
  __shared__ DecodeJob jobs[kDWarps];  // each warp's current tensor
  fill_lut(sm.d.lut);
  pdl_enter();
  const bool in_smem = a.count <= kSmemSearchUnits;
  if (in_smem)
    for (uint32_t i = threadIdx.x; i < a.count; i += kDThreads) begin_s[i] = a.prep[i].act_begin;
  __syncthreads();
  const uint32_t total = *a.total;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t nw = gridDim.x * kDWarps;
  DecodeJob &j = jobs[warp];
  uint32_t cur = 0xffffffffu;
  for (uint32_t gu = blockIdx.x * kDWarps + warp; gu < total; gu += nw) {
    const uint32_t id = find_tensor(begin_s, in_smem, a.prep, a.count, gu, false);
    if (!a.ok[id]) continue;  // uniform in the warp
    const uint32_t first = in_smem ? begin_s[id] : a.prep[id].act_begin;
    if (id != cur) {
      __syncwarp();
      if (lane == 0) {
        const BatchTensor &T = a.tensors[id];
        const BatchPrep &P = a.prep[id];
        j.payload = a.arena + T.arena_off + 4;
        j.m = P.m;
        j.n = T.n;
        j.groups = T.groups;
        j.scale = P.scale;
        j.y = T.y;
        j.status = nullptr;
        j.n_tiles = (uint32_t)((P.m + kDecodeUnit - 1) / kDecodeUnit);
        j.vec = T.vec_y != 0;
        j.loc = a.loc + T.d_tile_begin;
        j.cpre = a.cpre + T.d_chunk_begin + id;
      }
      __syncwarp();
      fill_scaled_pairs(sm.sp[warp], j.scale, lane);
      cur = id;
    }
    decode_unit<kMode>(j, gu - first, sm.d.lut, sm.sp[warp], sm.wd[warp], unit_stage(sm, warp));
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
  // whole units), and the index's unit count
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

bool decode_deferred(uint32_t tiles) { return tiles >= kDecodeDeferMinTiles; }

uint32_t decode_tile_payload_bytes(bool accumulate) {
  return accumulate ? DecodeShape<kAccumulate>::kTile : DecodeShape<kWrite>::kTile;
}


static uint32_t persistent_grid(const DeviceInfo &dev, int occ, uint64_t work_blocks) {
  uint64_t grid = (uint64_t)dev.sm_count * (uint64_t)(occ > 0 ? occ : 1);
  if (grid > work_blocks) grid = work_blocks;
  return (uint32_t)(grid < 1 ? 1 : grid);
}

template <int kMode, bool kVec>
static cudaError_t launch_one(const DeviceInfo &dev, const DecodeArgs &a, uint32_t tiles,
                              cudaStream_t stream) {
  const size_t smem = decode_smem_bytes(kMode == kAccumulate);
  const int occ = kMode == kWrite ? dev.occ_decode_write : dev.occ_decode_acc;
  const int kind = kMode == kWrite ? kKindDecodeWrite : kKindDecodeAccumulate;
  timing_begin(kind, stream);
  launch_k(k_decode<kMode, kVec>, persistent_grid(dev, occ, tiles), kDThreads, smem, stream, a);
  timing_end(kind, stream);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DeviceInfo &dev, const uint8_t *in, const uint64_t *len_dev,
                          uint64_t cap, uint64_t n, float *y, bool accumulate,
                          int32_t *dev_status, uint32_t max_polls, uint64_t *scratch,
                          cudaStream_t stream) {
  const uint64_t groups = (n + 4) / 5;
  const uint32_t tiles = decode_tiles_max(cap, groups);
  DecodeArgs a;
  a.in = in;
  a.len_dev = len_dev;
  a.cap = cap;
  a.n = n;
  a.groups = groups;
  a.y = y;
  a.status = scratch;
  a.ticket = reinterpret_cast<uint32_t *>(scratch + tiles);
  a.dev_status = dev_status;
  a.max_polls = max_polls;
  const bool vec = (reinterpret_cast<uintptr_t>(y) & 15) == 0;
  if (accumulate)
    return vec ? launch_one<kAccumulate, true>(dev, a, tiles, stream)
               : launch_one<kAccumulate, false>(dev, a, tiles, stream);
  return vec ? launch_one<kWrite, true>(dev, a, tiles, stream)
             : launch_one<kWrite, false>(dev, a, tiles, stream);
}

// ---- indexed decode of up to kIndexPass streams --------------------------
// Scratch: [ticket2, ok[kIndexPass]] (written by the scan), then each
// stream's loc[] (one word per unit of its capacity) and cpre[] (one per
// chunk, plus the total); for two streams or more also eloc[], ecpre[],
// list[] (one word per possible entry: min(payload capacity, groups)) and
// tfe[] (one per sum tile, plus the total).
static size_t ix_head_bytes() { return align_up(4 + 4 * kIndexPass, 256); }

IndexedLayout indexed_layout(const IndexedStream *s, int k, uint64_t n) {
  IndexedLayout L = {};
  const uint64_t groups = (n + 4) / 5;
  size_t at = ix_head_bytes();
  for (int i = 0; i < k; ++i) {
    const uint32_t units = decode_tiles_max(s[i].cap, groups);
    const uint32_t chunks = (units + kDecodeChunkUnits - 1) / kDecodeChunkUnits;
    auto take = [&at](size_t words) {
      const size_t off = at;
      at = align_up(at + 4 * words, 16);
      return off;
    };
    L.loc_off[i] = take(units);
    L.cpre_off[i] = take((size_t)chunks + 1);
    if (k > 1) {
      const uint64_t mcap = s[i].cap >= 4 ? s[i].cap - 4 : 0;
      L.eloc_off[i] = take(units);
      L.ecpre_off[i] = take((size_t)chunks + 1);
      L.list_off[i] = take((size_t)(mcap < groups ? mcap : groups) + 1);
      L.tfe_off[i] = take((size_t)sum_tiles(groups) + 1);
    }
  }
  L.total_bytes = align_up(at, 256);
  return L;
}

// Blocks per SM: the warp-unit kernels (slots 0 dense output, 1
// accumulate) and each k_apply_entries instantiation (slots 2, 3, 4: up to
// 2, 4 and 8 streams), with their shared memory.
template <int kK>
static int apply_occupancy() {
  constexpr size_t smem = apply_smem_bytes<kK>();
  cudaFuncSetAttribute(k_apply_entries<kK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_apply_entries<kK>, kDThreads, smem);
  return occ;
}

void occupancy_decode_ix(int occ[5]) {
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ[0], k_decode_units<kWrite>, kDThreads, 0);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ[1], k_decode_units<kAccumulate>, kDThreads,
                                                0);
  occ[2] = apply_occupancy<2>();
  occ[3] = apply_occupancy<4>();
  occ[4] = apply_occupancy<8>();
}

template <int kK>
static cudaError_t launch_apply(const DeviceInfo &dev, const IxArgs &a, int occ_slot,
                               cudaStream_t stream) {
  constexpr size_t smem = apply_smem_bytes<kK>();
  const uint32_t grid = persistent_grid(dev, dev.occ_decode_ix[occ_slot], sum_tiles(a.groups));
  return launch_k(k_apply_entries<kK>, grid, kDThreads, smem, stream, a);
}

cudaError_t launch_decode_indexed(const DeviceInfo &dev, const IndexedStream *s, int k, uint64_t n,
                                  float *y, bool accumulate, int32_t *dev_status,
                                  uint32_t max_polls, void *scratch, cudaStream_t stream) {
  (void)max_polls;  // nothing in the indexed decode waits on another block
  if (k < 1 || k > kIndexPass || (!accumulate && k != 1)) return cudaErrorInvalidValue;
  const IndexedLayout L = indexed_layout(s, k, n);
  char *base = static_cast<char *>(scratch);
  IxArgs a;
  a.k = k;
  a.n = n;
  a.groups = (n + 4) / 5;
  a.ticket2 = reinterpret_cast<uint32_t *>(base);
  a.ok = reinterpret_cast<uint32_t *>(base + 4);
  a.y = y;
  a.vec = (reinterpret_cast<uintptr_t>(y) & 15) == 0;
  a.dev_status = dev_status;
  uint64_t chunks = 0, units_max = 0, units_all = 0;
  for (int i = 0; i < kIndexPass; ++i) {
    IxStream &S = a.s[i];
    S = IxStream{};
    if (i < k) {
      S.in = s[i].in;
      S.len_dev = s[i].len_dev;
      S.cap = s[i].cap;
      S.loc = reinterpret_cast<uint32_t *>(base + L.loc_off[i]);
      S.cpre = reinterpret_cast<uint32_t *>(base + L.cpre_off[i]);
      if (k > 1) {
        S.eloc = reinterpret_cast<uint32_t *>(base + L.eloc_off[i]);
        S.ecpre = reinterpret_cast<uint32_t *>(base + L.ecpre_off[i]);
        S.list = reinterpret_cast<uint32_t *>(base + L.list_off[i]);
        S.tfe = reinterpret_cast<uint32_t *>(base + L.tfe_off[i]);
      }
      const uint32_t units = decode_tiles_max(s[i].cap, a.groups);
      chunks += (units + kDecodeChunkUnits - 1) / kDecodeChunkUnits;
      units_all += units;
      if (units > units_max) units_max = units;
    }
  }
  timing_begin(kKindDecodeCount, stream);
  if (k > 1)
    launch_k(k_index_count<true>, persistent_grid(dev, 4, chunks), kDThreads, 0, stream, a);
  else
    launch_k(k_index_count<false>, persistent_grid(dev, 4, chunks), kDThreads, 0, stream, a);
  launch_k(k_index_scan, k, kScanThreads, 0, stream, a);
  timing_end(kKindDecodeCount, stream);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (k == 1) {
    // one warp per 512-byte unit
    const int kind = accumulate ? kKindDecodeAccumulate : kKindDecodeWrite;
    const uint32_t grid = persistent_grid(dev, dev.occ_decode_ix[accumulate ? 1 : 0],
                                          (units_max + kDWarps - 1) / kDWarps);
    timing_begin(kind, stream);
    if (accumulate)
      launch_k(k_decode_units<kAccumulate>, grid, kDThreads, 0, stream, a);
    else
      launch_k(k_decode_units<kWrite>, grid, kDThreads, 0, stream, a);
    timing_end(kind, stream);
    return cudaGetLastError();
  }
  // several streams: every stream's entries (one warp per unit), then the
  // sum tiles
  timing_begin(kKindDecodeAccumulate, stream);
  launch_k(k_index_entries, persistent_grid(dev, 8, (units_all + kDWarps - 1) / kDWarps),
           kDThreads, 0, stream, a);
  if (k == 2)
    e = launch_apply<2>(dev, a, 2, stream);
  else if (k <= 4)
    e = launch_apply<4>(dev, a, 3, stream);
  else
    e = launch_apply<8>(dev, a, 4, stream);
  timing_end(kKindDecodeAccumulate, stream);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ---- plans ----------------------------------------------------------------
template <int kMode>
static cudaError_t launch_batch_one(const DeviceInfo &dev, const BatchDecodeArgs &a,
                                    bool indexed, cudaStream_t stream) {
  const int kind = kMode == kWrite ? kKindDecodeWrite : kKindDecodeAccumulate;
  if (!indexed) {
    const size_t smem = decode_smem_bytes(kMode == kAccumulate);
    const int occ = kMode == kWrite ? dev.occ_decode_batch_write : dev.occ_decode_batch_acc;
    timing_begin(kind, stream);
    launch_k(k_decode_batch<kMode>, persistent_grid(dev, occ, a.n_tiles), kDThreads, smem, stream,
             a);
    timing_end(kind, stream);
    return cudaGetLastError();
  }
  timing_begin(kKindDecodeCount, stream);
  launch_k(k_index_count_batch, persistent_grid(dev, 4, a.n_chunks), kDThreads, 0, stream, a);
  launch_k(k_index_scan_batch, persistent_grid(dev, 8, a.count), kDThreads, 0, stream, a);
  timing_end(kKindDecodeCount, stream);
  const int occ = kMode == kWrite ? dev.occ_decode_batch_ix_write : dev.occ_decode_batch_ix_acc;
  timing_begin(kind, stream);
  launch_k(k_decode_batch_units<kMode>,
           persistent_grid(dev, occ, (a.n_tiles + kDWarps - 1) / kDWarps), kDThreads, 0, stream, a);
  timing_end(kind, stream);
  return cudaGetLastError();
}

cudaError_t launch_decode_batch(const DeviceInfo &dev, const BatchPlanDev &p,
                                const uint8_t *arena, const uint64_t *in_lens, bool accumulate,
                                int32_t *dev_status, uint32_t max_polls, cudaStream_t stream) {
  const bool indexed = decode_deferred(p.n_d_tiles);
  cudaError_t e = cudaSuccess;
  if (!indexed) {
    // the ticket and the look-back words (an indexed plan's scan writes
    // its valid flags, and its units need no ticket)
    e = cudaMemsetAsync(p.d_zero_base, 0, p.d_zero_bytes, stream);
    if (e != cudaSuccess) return e;
  }
  timing_begin(kKindDecodePrepare, stream);
  launch_k(k_decode_batch_prepare, 1, kPrepThreads, 0, stream, p.tensors, p.count, arena, in_lens,
           indexed ? kDecodeUnit : decode_tile_payload_bytes(accumulate), p.d_prep, p.d_total,
           dev_status);
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
  a.n_tiles = p.n_d_tiles;   // units (indexed) or an upper bound of the payload tiles
  a.dev_status = dev_status;
  a.max_polls = max_polls;
  a.loc = p.d_loc;
  a.cpre = p.d_cpre;
  a.ok = p.d_ok;
  a.n_chunks = p.n_d_chunks;
  return accumulate ? launch_batch_one<kAccumulate>(dev, a, indexed, stream)
                    : launch_batch_one<kWrite>(dev, a, indexed, stream);
}

template <int kMode>
static int batch_occupancy(bool indexed) {
  int occ = 0;
  if (indexed) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode_batch_units<kMode>, kDThreads,
                                                  0);
  } else {
    const size_t smem = decode_smem_bytes(kMode == kAccumulate);
    cudaFuncSetAttribute(k_decode_batch<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode_batch<kMode>, kDThreads, smem);
  }
  return occ;
}

int occupancy_decode_batch(bool accumulate, bool indexed) {
  return accumulate ? batch_occupancy<kAccumulate>(indexed) : batch_occupancy<kWrite>(indexed);
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
    cudaFuncSetAttribute(k_decode<kAccumulate, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_decode<kAccumulate, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode<kAccumulate, true>, kDThreads,
                                                  smem);
  } else {
    cudaFuncSetAttribute(k_decode<kWrite, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    cudaFuncSetAttribute(k_decode<kWrite, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode<kWrite, true>, kDThreads, smem);
  }
  return occ;
}

}  // namespace tlc
