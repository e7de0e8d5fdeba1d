// tlc_compress.cu -- compression kernels for the 3LC pipeline on sm_100a.
//
// Source: review page "3LC: Lightweight and Effective Traffic Compression for
// Distributed Machine Learning", section "Proposed method":
//   bullet 1  3-value quantization with sparsity multiplication and an
//             error-accumulation buffer  -> k_absmax + first half of k_quant_zre
//   bullet 2  quartic encoding (five ternary values per byte) -> k_quant_zre
//   bullet 3  zero-run encoding of all-zero byte groups       -> k_quant_zre
// bullet 5 of the same section asks for vectorised, byte-level processing
// with low overhead; here that is 128-bit coalesced loads, one pass per
// dependency, and a single-pass scan so no byte intermediate touches HBM.
//
// Two launches per call (three on the deferred-placement path, below):
//   k_absmax     x' = x + err and M = max|x'| (as a max over the uint32 bit
//                patterns of |x'|; NaN/Inf sort above every finite value).
//                It also clears the scan state that k_quant_zre uses.
//   k_quant_zre  per tile of 2048 byte groups (10240 values): recompute x',
//                q = round(x'/(M s)), err' = x' - q M s (written back), pack
//                the quartic bytes into shared memory, zero-run encode them,
//                and place the tile's output with a decoupled look-back over
//                earlier tiles.  Tiles are taken in order from a ticket
//                counter, so every tile a tile waits on is already running.
// Tensors of 768 tiles and more take a third launch instead of the
// per-tile look-back (the deferred-placement path): k_quant_zre tiles
// write their summary and stage the bytes that follow their leading run;
// the last tile of every 32-tile chunk to finish sums up the chunk, and the
// last chunk of every 32-chunk span the span; then k_zre_place, one block
// per chunk, composes the summaries before its chunk (spans, then chunks),
// scans its tiles' summaries and writes every tile's bytes in place; no
// block waits on another.
// The look-back inside k_quant_zre holds each tile's memory stream for a
// round trip to earlier tiles; moving it to a kernel with no other work
// measured 10-18% less time for the two kernels together than for the
// look-back k_quant_zre from 2^23 to 2^28 values (sparse and dense
// streams).  Below 768 tiles the look-back is as fast or faster.
//
// Zero-run emission order.  A maximal run of L bytes equal to 121 emits
// floor(L/14) bytes 255 (one at the end of each full chunk of 14), then, if
// L mod 14 = r != 0, one remainder byte (121 for r = 1, else 241 + r).  The
// remainder is written by the first non-121 byte after the run (just before
// that byte's own literal), or by the last tile at the end of the stream.
// The output sequence is the canonical one -- full chunks from the start of
// the run, remainder last -- but no tile needs to look at the next tile.
//
// Tile summary (aggregate) for a segment of bytes, as a function of the
// incoming run length t (mod 14) of 121-bytes that precede it:
//   all    the segment is entirely 121s (then A = its length)
//   A      length of its leading 121-run
//   R      bytes emitted from position A onwards (literals, full chunks of
//          runs that start inside, remainders before literals)
//   tc     length mod 14 of the trailing 121-run (if not all)
// emitted(t) = (all ? floor : ceil)((t + A) / 14) + R
// t_out(t)   = all ? (t + A) mod 14 : tc
// Two segments compose associatively (see compose()).
#define TLC_TU 1
#include "tlc_device.cuh"
#include "tlc_internal.h"

namespace tlc {

TLC_DEFINE_DEBUG_READER(debug_fault_compress)

// ------------------------------------------------------------ k_absmax ----
constexpr int kAbsThreads = 512;
constexpr int kAbsUnroll = 4;

__device__ __forceinline__ uint32_t abs_bits(float v) {
  return __float_as_uint(v) & 0x7fffffffu;
}

template <bool kVec>
__global__ void __launch_bounds__(kAbsThreads)
k_absmax(const float *__restrict__ x, const float *__restrict__ err, uint64_t n,
         uint32_t *__restrict__ partial, uint64_t *__restrict__ zero_words,
         uint32_t n_zero, CompressRecord *rec) {
  pdl_enter();
  if (rec && blockIdx.x == 0 && threadIdx.x == 0) rec->nonzeros = 0;
  uint32_t m = 0;
  const uint64_t gtid = (uint64_t)blockIdx.x * kAbsThreads + threadIdx.x;
  const uint64_t nth = (uint64_t)gridDim.x * kAbsThreads;
  if (kVec) {
    const uint64_t n4 = n >> 2;
    const float4 *x4 = reinterpret_cast<const float4 *>(x);
    const float4 *e4 = reinterpret_cast<const float4 *>(err);
    uint64_t i = gtid;
    for (; i + (kAbsUnroll - 1) * nth < n4; i += kAbsUnroll * nth) {
      float4 a[kAbsUnroll], b[kAbsUnroll];
#pragma unroll
      for (int u = 0; u < kAbsUnroll; ++u) {
        a[u] = __ldg(x4 + i + u * nth);
        b[u] = __ldg(e4 + i + u * nth);
      }
#pragma unroll
      for (int u = 0; u < kAbsUnroll; ++u) {
        m = max(m, abs_bits(__fadd_rn(a[u].x, b[u].x)));
        m = max(m, abs_bits(__fadd_rn(a[u].y, b[u].y)));
        m = max(m, abs_bits(__fadd_rn(a[u].z, b[u].z)));
        m = max(m, abs_bits(__fadd_rn(a[u].w, b[u].w)));
      }
    }
    for (; i < n4; i += nth) {
      const float4 a = __ldg(x4 + i), b = __ldg(e4 + i);
      m = max(m, abs_bits(__fadd_rn(a.x, b.x)));
      m = max(m, abs_bits(__fadd_rn(a.y, b.y)));
      m = max(m, abs_bits(__fadd_rn(a.z, b.z)));
      m = max(m, abs_bits(__fadd_rn(a.w, b.w)));
    }
    const uint64_t rem = n - (n4 << 2);
    if (gtid < rem) {
      const uint64_t k = (n4 << 2) + gtid;
      m = max(m, abs_bits(__fadd_rn(x[k], err[k])));
    }
  } else {
    for (uint64_t i = gtid; i < n; i += nth) m = max(m, abs_bits(__fadd_rn(x[i], err[i])));
  }
  for (uint64_t w = gtid; w < n_zero; w += nth) zero_words[w] = 0;

  __shared__ uint32_t wmax[kAbsThreads / kWarp];
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < kWarp) {
    uint32_t v = threadIdx.x < kAbsThreads / kWarp ? wmax[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xffffffffu, v);
    if (threadIdx.x == 0) partial[blockIdx.x] = v;
  }
}

// --------------------------------------------------------- k_quant_zre ----
// Tile shape (compile-time knobs; defaults are the tuned values).
#ifndef TLC_Q_ITERS
#define TLC_Q_ITERS 2
#endif
#ifndef TLC_Q_MINB
#define TLC_Q_MINB 6
#endif
constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / kWarp;
constexpr int kChunkElems = 640;   // one warp step: 32 lanes x 5 float4
constexpr int kChunkGroups = 128;  // = kChunkElems / 5
constexpr int kQIters = TLC_Q_ITERS;
constexpr int kTileGroups = kQWarps * kQIters * kChunkGroups;  // 2048 by default
constexpr uint64_t kTileElems = 5ull * kTileGroups;            // 10240 by default
constexpr int kZBytes = kTileGroups / kQThreads;               // 8 per thread by default
constexpr int kZWords = kZBytes / 4;                           // u32 words per thread
static_assert((kZBytes == 8 || kZBytes % 16 == 0) && kTileGroups < 65536, "tile shape");
#ifndef TLC_Q_LOOKV
#define TLC_Q_LOOKV 1
#endif
constexpr int kLookV = TLC_Q_LOOKV;  // look-back words per lane per round trip
// Tensors of at least this many tiles take the deferred-placement path.
#ifndef TLC_DEFER_MIN_TILES
#define TLC_DEFER_MIN_TILES 768
#endif
constexpr uint32_t kDeferMinTiles = TLC_DEFER_MIN_TILES;


struct ZAgg {
  uint32_t all, A, R, tc;
};

__device__ __forceinline__ uint64_t pack_agg(const ZAgg &a) {
  return kFlagAgg | (uint64_t)a.A | ((uint64_t)a.R << 16) | ((uint64_t)a.tc << 32) |
         ((uint64_t)a.all << 36);
}
__device__ __forceinline__ ZAgg unpack_agg(uint64_t w) {
  ZAgg a;
  a.A = (uint32_t)(w & 0xffffu);
  a.R = (uint32_t)((w >> 16) & 0xffffu);
  a.tc = (uint32_t)((w >> 32) & 0xfu);
  a.all = (uint32_t)((w >> 36) & 1u);
  return a;
}
// The same summary in 32 bits (A, R <= 4096 need 13 bits each), for the
// deferred path's summary array.
static_assert(kTileGroups < 8192, "A and R of a tile fit in 13 bits");
__device__ __forceinline__ uint32_t pack_agg32(const ZAgg &a) {
  return a.A | (a.R << 13) | (a.tc << 26) | (a.all << 31);
}
__device__ __forceinline__ ZAgg unpack_agg32(uint32_t w) {
  ZAgg a;
  a.A = w & 0x1fffu;
  a.R = (w >> 13) & 0x1fffu;
  a.tc = (w >> 26) & 0xfu;
  a.all = w >> 31;
  return a;
}
// Inclusive prefix: emitted count C (< 2^32) and run length mod 14.
__device__ __forceinline__ uint64_t pack_prefix(uint32_t C, uint32_t t) {
  return kFlagPrefix | (uint64_t)C | ((uint64_t)t << 32);
}

__device__ __forceinline__ uint32_t lead_count(const ZAgg &a, uint32_t t) {
  const uint32_t v = t + a.A;
  return a.all ? v / 14u : (v + 13u) / 14u;
}

__device__ __forceinline__ void eval_agg(uint32_t &C, uint32_t &t, const ZAgg &a) {
  C += lead_count(a, t) + a.R;
  t = a.all ? (t + a.A) % 14u : a.tc;
}

// Aggregate of segment a1 followed by segment a2.
__device__ __forceinline__ ZAgg compose(const ZAgg &a1, const ZAgg &a2) {
  ZAgg r;
  if (!a1.all) {
    r.all = 0;
    r.A = a1.A;
    r.R = a1.R + lead_count(a2, a1.tc) + a2.R;
    r.tc = a2.all ? (a1.tc + a2.A) % 14u : a2.tc;
  } else {
    r.all = a2.all;
    r.A = a1.A + a2.A;
    r.R = a2.R;
    r.tc = a2.tc;
  }
  return r;
}

__device__ __forceinline__ uint8_t remainder_byte(uint32_t r) {
  return r == 1 ? uint8_t(121) : uint8_t(241 + r);
}

// Rounding without the division.  With r = fl(x'/scale) the correctly
// rounded quotient and |x'| <= M <= scale, q = round(r) is non-zero exactly
// when fl(|x'|/scale) >= 1/2.  The fp32 neighbour below 1/2 is 1/2 - 2^-25,
// and the midpoint 1/2 - 2^-26 rounds to 1/2 (its even neighbour), so
//   fl(|x'|/scale) >= 1/2  <=>  |x'|/scale >= 1/2 - 2^-26
//                          <=>  |x'| >= scale * (1/2 - 2^-26)   (exact reals)
//                          <=>  |x'| >= T,  T = the least fp32 value that is
//                                            >= scale * (1/2 - 2^-26).
// scale has 24 significant bits and 1/2 - 2^-26 has 25, so the product is
// exact in fp64 and T is that product rounded towards +infinity.  The test
// gives the same q as the division for every input, subnormals included.
// M = 0 uses T = +inf (every q = 0, no division).
__device__ __forceinline__ float zero_band_threshold(float scale, bool mzero) {
  if (mzero) return __int_as_float(0x7f800000);
  const double t = __dmul_rn((double)scale, 0.5 - 0x1p-26);
  return __double2float_ru(t);
}

// One element: digit q+1 of round(x'/scale) with ties away from zero, and
// the updated error x' - q*scale.
__device__ __forceinline__ uint32_t quant_digit(float xp, float scale, float thr, float &e) {
  const bool nz = fabsf(xp) >= thr;
  const bool neg = __float_as_uint(xp) >> 31;
  e = nz ? __fsub_rn(xp, neg ? -scale : scale) : xp;
  return nz ? (neg ? 0u : 2u) : 1u;
}

// Quartic byte of five digits, first digit most significant (Horner in base 3).
__device__ __forceinline__ uint32_t pack_groups4(const uint32_t w[5]) {
  uint32_t out = 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t v = 0;
#pragma unroll
    for (int d = 0; d < 5; ++d) {
      const int i = 5 * g + d;
      v = v * 3u + ((w[i >> 2] >> (8 * (i & 3))) & 0xffu);
    }
    out |= v << (8 * g);
  }
  return out;
}

// ---- deferred placement: summaries of tiles and of 32-tile chunks ----------
// An aggregate with a validity bit, for warp scans (invalid = the identity
// of composition).
struct ZScan {
  uint32_t valid;
  ZAgg a;
};
__device__ __forceinline__ ZScan zcombine(const ZScan &x, const ZScan &y) {
  if (!x.valid) return y;
  if (!y.valid) return x;
  return {1u, compose(x.a, y.a)};
}
__device__ __forceinline__ ZScan zshfl_up(const ZScan &v, int d) {
  ZScan r;
  r.valid = __shfl_up_sync(0xffffffffu, v.valid, d);
  r.a.all = __shfl_up_sync(0xffffffffu, v.a.all, d);
  r.a.A = __shfl_up_sync(0xffffffffu, v.a.A, d);
  r.a.R = __shfl_up_sync(0xffffffffu, v.a.R, d);
  r.a.tc = __shfl_up_sync(0xffffffffu, v.a.tc, d);
  return r;
}

// The summary of a chunk of kPlaceTiles tiles, or of a span of kPlaceSpan
// chunks, in 64 bits (A, R < 2^24: a segment emits at most one byte per
// group), as the deferred path stores it.
constexpr int kPlaceTiles = 32;
constexpr int kPlaceSpan = 32;
static_assert((uint64_t)kPlaceSpan * kPlaceTiles * kTileGroups < (1u << 24),
              "span A and R fit in 24 bits");
struct ChunkCodec {
  __device__ static uint64_t pack(const ZAgg &a) {
    return (uint64_t)a.A | ((uint64_t)a.R << 24) | ((uint64_t)a.tc << 48) |
           ((uint64_t)a.all << 52);
  }
  __device__ static ZAgg unpack(uint64_t w) {
    ZAgg a;
    a.A = (uint32_t)(w & 0xffffffu);
    a.R = (uint32_t)((w >> 24) & 0xffffffu);
    a.tc = (uint32_t)((w >> 48) & 0xfu);
    a.all = (uint32_t)((w >> 52) & 1u);
    return a;
  }
};

// One tensor's compression job, as the tile function sees it.
struct TileJob {
  const float *x;
  float *err;
  uint64_t n;
  uint64_t groups;
  uint8_t *out;       // stream: header then payload
  uint64_t out_cap;
  uint64_t *out_len;
  uint64_t *status;   // this tensor's tile status words
  uint32_t n_tiles;
  bool vec;           // x and err are 16-byte aligned
  CompressRecord *rec;  // or nullptr: the call's record (non-zero count, length)
};

// The deferred-placement path's buffers for one tensor.
struct DeferJob {
  uint32_t *aggs;     // each tile's summary (pack_agg32),
  uint8_t *stage;     // kTileGroups staged bytes per tile,
  uint32_t *ccount;   // finished tiles per 32-tile chunk (starts at 0),
  uint64_t *cagg;     // each chunk's summary (ChunkCodec),
  uint32_t *scount;   // or nullptr: finished chunks per 32-chunk span (starts at 0)
  uint64_t *sagg;     // and each span's summary (ChunkCodec)
};

// Shared memory of one compress block.
struct QuantSmem {
  __align__(16) uint32_t dig[kQWarps][kChunkElems / 4];  // digits q+1, one byte per value
  __align__(16) uint32_t tile[kTileGroups / 4];          // the tile's quartic bytes
  uint32_t scan[kQWarps + 1];
  uint32_t A, cin, tin, last;
  uint32_t nzw[kQWarps];  // per-warp non-zero counts of a tile (recording calls)
};

__device__ __forceinline__ void put_out(const TileJob &j, uint64_t pos, uint8_t v) {
  if (TLC_BOUND(4 + pos < j.out_cap)) j.out[4 + pos] = v;
}

// Decoupled look-back for item t of a single-pass scan over status words,
// by one whole warp: publish the item's aggregate, combine earlier items'
// words until an inclusive prefix is found, publish this item's inclusive
// prefix, and return the exclusive prefix (emitted count, incoming run
// length mod 14) to every lane.  Each round trip reads 32 * kV earlier
// words: every lane first folds its kV words (oldest to nearest), then the
// lanes are folded in order.  Codec packs and unpacks aggregates.
struct TileCodec {
  __device__ static uint64_t pack(const ZAgg &a) { return pack_agg(a); }
  __device__ static ZAgg unpack(uint64_t w) { return unpack_agg(w); }
};

template <int kV, class Codec>
__device__ __forceinline__ void lookback_words(uint64_t *status, uint32_t t, const ZAgg &agg,
                                               uint32_t &cin, uint32_t &tin, int32_t *dev_status,
                                               uint32_t max_polls) {
  constexpr int kLookV = kV;
  const int lane = threadIdx.x & 31;
  if (t == 0) {
    if (lane == 0) {
      uint32_t C = 0, tt = 0;
      eval_agg(C, tt, agg);
      st_relaxed_u64(status, pack_prefix(C, tt));
    }
    cin = 0;
    tin = 0;
    return;
  }
  if (lane == 0) st_relaxed_u64(status + t, Codec::pack(agg));
  bool timed_out = false;
  bool have_suffix = false;
  ZAgg suffix = {0, 0, 0, 0};
  int64_t end = (int64_t)t - 1;
  uint32_t C = 0, tt = 0;
  for (;;) {
    uint64_t w[kLookV];
    load_window(status, end, pack_prefix(0, 0), max_polls, timed_out, w);
    int jp = kLookV;
    uint64_t wp = 0;
#pragma unroll
    for (int k = 0; k < kLookV; ++k)
      if (jp == kLookV && (w[k] >> kFlagShift) == 2) {
        jp = k;
        wp = w[k];
      }
    // this lane's words nearer than its prefix (or all of them), folded
    // from the oldest to the nearest
    ZAgg lagg = {1u, 0u, 0u, 0u};
    bool have = false;
#pragma unroll
    for (int k = kLookV - 1; k >= 0; --k) {
      if (k < jp) {
        const ZAgg ak = Codec::unpack(w[k]);
        lagg = have ? compose(lagg, ak) : ak;
        have = true;
      }
    }
    uint32_t lC = 0, lt = 0;  // this lane's state after its prefix
    if (jp < kLookV) {
      lC = (uint32_t)(wp & 0xffffffffu);
      lt = (uint32_t)((wp >> 32) & 0xfu);
      if (have) eval_agg(lC, lt, lagg);
    }
    const uint32_t pmask = __ballot_sync(0xffffffffu, jp < kLookV);
    const int pl = pmask ? __ffs(pmask) - 1 : kWarp;
    if (pmask) {
      C = __shfl_sync(0xffffffffu, lC, pl);
      tt = __shfl_sync(0xffffffffu, lt, pl);
    }
    // lanes pl-1 .. 0 (or 31 .. 0 without a prefix), oldest first
    ZAgg acc = {1u, 0u, 0u, 0u};
    bool acc_have = false;
    for (int l = pl - 1; l >= 0; --l) {
      ZAgg al;
      al.all = __shfl_sync(0xffffffffu, lagg.all, l);
      al.A = __shfl_sync(0xffffffffu, lagg.A, l);
      al.R = __shfl_sync(0xffffffffu, lagg.R, l);
      al.tc = __shfl_sync(0xffffffffu, lagg.tc, l);
      if (pmask) {
        eval_agg(C, tt, al);
      } else {
        acc = acc_have ? compose(acc, al) : al;
        acc_have = true;
      }
    }
    if (pmask) {
      if (have_suffix) eval_agg(C, tt, suffix);
      break;
    }
    suffix = have_suffix ? compose(acc, suffix) : acc;
    have_suffix = true;
    end -= kWarp * kLookV;
  }
  if (__any_sync(0xffffffffu, timed_out) && lane == 0) report(dev_status, TLC_ERR_TIMEOUT);
  if (lane == 0) {
    uint32_t Ci = C, ti = tt;
    eval_agg(Ci, ti, agg);
    st_relaxed_u64(status + t, pack_prefix(Ci, ti));
  }
  cin = C;
  tin = tt;
}

template <int kV>
__device__ __forceinline__ void lookback_warp(const TileJob &j, uint32_t t, const ZAgg &agg,
                                              uint32_t &cin, uint32_t &tin, int32_t *dev_status,
                                              uint32_t max_polls) {
  lookback_words<kV, TileCodec>(j.status, t, agg, cin, tin, dev_status, max_polls);
}

// The same, called by the whole block (warp 0 works); ends synchronised.
template <int kV>
__device__ __forceinline__ void lookback_tile(const TileJob &j, uint32_t t, const ZAgg &agg,
                                              uint32_t &cin, uint32_t &tin, QuantSmem &sm,
                                              int32_t *dev_status, uint32_t max_polls) {
  if ((threadIdx.x >> 5) == 0) {
    uint32_t c, ti;
    lookback_warp<kV>(j, t, agg, c, ti, dev_status, max_polls);
    if ((threadIdx.x & 31) == 0) {
      sm.cin = c;
      sm.tin = ti;
    }
  }
  __syncthreads();
  cin = sm.cin;
  tin = sm.tin;
}

// Stream header (first tile) and the closing remainder + length (last tile).
__device__ __forceinline__ void finish_tile(const TileJob &j, uint32_t t, const ZAgg &agg,
                                            uint32_t cin, uint32_t tin, float scale) {
  if (threadIdx.x != 0) return;
  if (t == 0) {
    const uint32_t sb = __float_as_uint(scale);
    j.out[0] = sb & 0xff;
    j.out[1] = (sb >> 8) & 0xff;
    j.out[2] = (sb >> 16) & 0xff;
    j.out[3] = (sb >> 24) & 0xff;
  }
  if (t == j.n_tiles - 1) {
    uint32_t C = cin, tt = tin;
    eval_agg(C, tt, agg);
    if (tt) put_out(j, C, remainder_byte(tt));
    *j.out_len = 4ull + C + (tt ? 1u : 0u);
    if (j.rec) j.rec->length = 4ull + C + (tt ? 1u : 0u);
  }
}

// One warp step: values [e0, e0 + 640) of a tensor -> err' written back and
// the 128 quartic bytes of these values, four per lane, returned packed
// (lane L holds groups 4L..4L+3 of the step).  `dig` is this warp's 640-byte
// shared buffer of digits.  Values past n count as zero (digit 1).
// Values with a non-zero digit among four digits (one per byte, 0..2, 1 is zero).
__device__ __forceinline__ uint32_t nonzero_digits(uint32_t dw) {
  const uint32_t x = dw ^ 0x01010101u;
  return __popc((x | (x >> 1)) & 0x01010101u);
}

// kCount: also add the number of non-zero q of the step's values to nz.
template <bool kCount>
__device__ __forceinline__ uint32_t quant_chunk(const float *x, float *err, uint64_t n,
                                                uint64_t e0, bool vec_full, float scale,
                                                float thr, uint32_t *dig, uint32_t &nz) {
  const int lane = threadIdx.x & 31;
  if (vec_full) {
    const float4 *x4 = reinterpret_cast<const float4 *>(x + e0);
    float4 *err4 = reinterpret_cast<float4 *>(err + e0);
    float4 xv[5], ev[5];
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      xv[k] = __ldg(x4 + lane + 32 * k);
      ev[k] = err4[lane + 32 * k];
    }
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      float4 o;
      uint32_t dw;
      dw = quant_digit(__fadd_rn(xv[k].x, ev[k].x), scale, thr, o.x);
      dw |= quant_digit(__fadd_rn(xv[k].y, ev[k].y), scale, thr, o.y) << 8;
      dw |= quant_digit(__fadd_rn(xv[k].z, ev[k].z), scale, thr, o.z) << 16;
      dw |= quant_digit(__fadd_rn(xv[k].w, ev[k].w), scale, thr, o.w) << 24;
      err4[lane + 32 * k] = o;
      dig[lane + 32 * k] = dw;
      if (kCount) nz += nonzero_digits(dw);
    }
  } else if (e0 < n) {
    // tail or unaligned step: scalar and bounds-checked
#pragma unroll 1
    for (int k = 0; k < 5; ++k) {
      uint32_t dw = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint64_t e = e0 + 4 * (uint64_t)(lane + 32 * k) + q;
        uint32_t d = 1;
        if (e < n) {
          float o;
          d = quant_digit(__fadd_rn(x[e], err[e]), scale, thr, o);
          err[e] = o;
        }
        dw |= d << (8 * q);
      }
      dig[lane + 32 * k] = dw;
      if (kCount) nz += nonzero_digits(dw);
    }
  } else {
    // step entirely past the end: all-zero groups
#pragma unroll
    for (int k = 0; k < 5; ++k) dig[lane + 32 * k] = 0x01010101u;
  }
  __syncwarp();
  uint32_t w5[5];
#pragma unroll
  for (int k = 0; k < 5; ++k) w5[k] = dig[5 * lane + k];
  const uint32_t packed = pack_groups4(w5);
  __syncwarp();
  return packed;
}

// Zero-run encoding of one tile of quartic bytes: every thread holds
// kZB consecutive bytes (p0 = threadIdx.x * kZB onwards) in qw; tgv bytes of
// the tile are valid.  Local analysis (block scans), decoupled look-back,
// emission, header / closing byte.  Whole block; ends synchronised.
//
// kDeferred: no look-back.  The tile stores its summary in dj.aggs[t] and the
// bytes it emits after its leading run (which do not depend on the incoming
// run) in its staging slot; k_zre_place later puts the prefix-dependent
// leading bytes and the staged bytes into the stream.
template <int kZB, int kV, bool kDeferred>
__device__ __forceinline__ void zre_encode_tile(const TileJob &j, const DeferJob &dj, uint32_t t,
                                                uint32_t tgv,
                                                const uint32_t (&qw)[kZB / 4], float scale,
                                                QuantSmem &sm, int32_t *dev_status,
                                                uint32_t max_polls) {
  constexpr int kZW = kZB / 4;
  bool mine_all = true;
#pragma unroll
  for (int w = 0; w < kZW; ++w) mine_all = mine_all && qw[w] == 0x79797979u;
  // bytes past tgv are all-zero (121) groups by construction
  const bool tile_all = __syncthreads_and(mine_all);
  if (kDeferred && tile_all) {
    if (threadIdx.x == 0) dj.aggs[t] = pack_agg32({1u, tgv, 0u, 0u});
    return;
  }
  if (!kDeferred && tile_all) {
    // Entirely 121s: only full 14-chunks of the run end inside the tile.
    const ZAgg agg = {1u, tgv, 0u, 0u};
    uint32_t cin, tin;
    lookback_tile<kV>(j, t, agg, cin, tin, sm, dev_status, max_polls);
    const uint32_t cnt = (tin + tgv) / 14u;
    for (uint32_t i = threadIdx.x; i < cnt; i += blockDim.x) put_out(j, (uint64_t)cin + i, 255);
    finish_tile(j, t, agg, cin, tin, scale);
    __syncthreads();
    return;
  }
  const int p0 = (int)threadIdx.x * kZB;
  int fnz = -1, lnz = -1;
#pragma unroll
  for (int k = 0; k < kZB; ++k) {
    const uint32_t b = (qw[k >> 2] >> (8 * (k & 3))) & 0xffu;
    const int p = p0 + k;
    if (p < (int)tgv && b != 121u) {
      if (fnz < 0) fnz = p;
      lnz = p;
    }
  }
  int32_t lnz_all;
  const int prev_in =
      block_exclusive_max<kQThreads>(lnz, reinterpret_cast<int32_t *>(sm.scan), lnz_all);
  if (prev_in < 0 && fnz >= 0) sm.A = (uint32_t)fnz;

  uint32_t cnt = 0;
  {
    int prev = prev_in;
#pragma unroll
    for (int k = 0; k < kZB; ++k) {
      const uint32_t b = (qw[k >> 2] >> (8 * (k & 3))) & 0xffu;
      const int p = p0 + k;
      if (p >= (int)tgv) break;
      if (b == 121u) {
        if (prev >= 0 && (p - prev - 1) % 14 == 13) ++cnt;
      } else {
        if (prev >= 0 && (p - 1 - prev) % 14 != 0) ++cnt;
        ++cnt;
        prev = p;
      }
    }
  }
  uint32_t R;
  const uint32_t off = block_exclusive_sum<kQThreads>(cnt, sm.scan, R);

  ZAgg agg;
  agg.all = lnz_all < 0 ? 1u : 0u;
  agg.A = agg.all ? tgv : sm.A;
  agg.R = R;
  agg.tc = agg.all ? 0u : (uint32_t)((int)tgv - 1 - lnz_all) % 14u;

  if constexpr (kDeferred) {
    if (threadIdx.x == 0) dj.aggs[t] = pack_agg32(agg);
    uint8_t *st = dj.stage + (uint64_t)t * kTileGroups;
    uint32_t k_out = off;
    // a tile emits at most one byte per group after its leading run
    auto stage = [&](uint8_t v) {
      if (TLC_CHECK(k_out < (uint32_t)kTileGroups)) st[k_out] = v;
      ++k_out;
    };
    int prev = prev_in;
#pragma unroll
    for (int k = 0; k < kZB; ++k) {
      const uint32_t b = (qw[k >> 2] >> (8 * (k & 3))) & 0xffu;
      const int p = p0 + k;
      if (p >= (int)tgv) break;
      if (prev < 0) {
        if (b != 121u) {  // the tile's first literal; the run before it is placed later
          stage((uint8_t)b);
          prev = p;
        }
      } else if (b == 121u) {
        if ((p - prev - 1) % 14 == 13) stage(255);
      } else {
        const uint32_t r = (uint32_t)(p - 1 - prev) % 14u;
        if (r) stage(remainder_byte(r));
        stage((uint8_t)b);
        prev = p;
      }
    }
    return;
  }

  uint32_t cin, tin;
  lookback_tile<kV>(j, t, agg, cin, tin, sm, dev_status, max_polls);

  {
    uint64_t k_out = (uint64_t)cin + lead_count(agg, tin) + off;
    int prev = prev_in;
#pragma unroll
    for (int k = 0; k < kZB; ++k) {
      const uint32_t b = (qw[k >> 2] >> (8 * (k & 3))) & 0xffu;
      const int p = p0 + k;
      if (p >= (int)tgv) break;
      if (b == 121u) {
        if (prev < 0) {
          if ((tin + p) % 14u == 13u) put_out(j, cin + (tin + p) / 14u, 255);
        } else if ((p - prev - 1) % 14 == 13) {
          put_out(j, k_out++, 255);
        }
      } else {
        if (prev < 0) {
          const uint32_t r = (tin + p) % 14u;
          if (r) put_out(j, cin + (tin + p) / 14u, remainder_byte(r));
        } else {
          const uint32_t r = (uint32_t)(p - 1 - prev) % 14u;
          if (r) put_out(j, k_out++, remainder_byte(r));
        }
        put_out(j, k_out++, (uint8_t)b);
        prev = p;
      }
    }
  }
  finish_tile(j, t, agg, cin, tin, scale);
  __syncthreads();
}

// One tile of kTileGroups byte groups (5 kTileGroups values) of one tensor, fused: quantize
// and update the error buffer, pack the quartic bytes into shared memory,
// then zero-run encode them.  Whole block; ends synchronised.
// kCount: the tile's non-zero values are added to the call's record.
template <bool kDeferred = false, bool kCount = false>
__device__ __forceinline__ void quant_tile(const TileJob &j, const DeferJob &dj, uint32_t t,
                                           float scale, float thr,
                                           QuantSmem &sm, int32_t *dev_status,
                                           uint32_t max_polls) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) sm.A = 0xffffffffu;
  const uint64_t g0 = (uint64_t)t * kTileGroups;
  const uint32_t tgv = (uint32_t)umin64(kTileGroups, j.groups - g0);
  const uint64_t e_tile = g0 * 5;
  const bool full = j.vec && (e_tile + kTileElems <= j.n);
  uint32_t nz = 0;
#pragma unroll 1
  for (int it = 0; it < kQIters; ++it) {
    const int c = it * kQWarps + warp;
    const uint64_t e0 = e_tile + (uint64_t)c * kChunkElems;
    sm.tile[c * (kChunkGroups / 4) + lane] =
        quant_chunk<kCount>(j.x, j.err, j.n, e0, full, scale, thr, sm.dig[warp], nz);
  }
  if (kCount) {
    nz = __reduce_add_sync(0xffffffffu, nz);
    if (lane == 0) sm.nzw[warp] = nz;
  }
  __syncthreads();
  if (kCount && threadIdx.x == 0) {
    uint32_t tot = 0;
#pragma unroll
    for (int w = 0; w < kQWarps; ++w) tot += sm.nzw[w];
    if (tot) atomicAdd(reinterpret_cast<unsigned long long *>(&j.rec->nonzeros),
                       (unsigned long long)tot);
  }
  uint32_t qw[kZWords];
  if constexpr (kZWords == 2) {
    const uint2 q2 = reinterpret_cast<const uint2 *>(sm.tile)[threadIdx.x];
    qw[0] = q2.x;
    qw[1] = q2.y;
  } else {
#pragma unroll
    for (int v = 0; v < kZWords / 4; ++v) {
      const uint4 q4 = reinterpret_cast<const uint4 *>(sm.tile)[threadIdx.x * (kZWords / 4) + v];
      qw[4 * v] = q4.x;
      qw[4 * v + 1] = q4.y;
      qw[4 * v + 2] = q4.z;
      qw[4 * v + 3] = q4.w;
    }
  }
  zre_encode_tile<kZBytes, kLookV, kDeferred>(j, dj, t, tgv, qw, scale, sm, dev_status,
                                              max_polls);
  if (kDeferred) {
    // The last tile of a 32-tile chunk to finish sums up the chunk (the
    // counter's atomic add orders every tile's summary before it).
    const uint32_t c = t / kPlaceTiles;
    if (threadIdx.x == 0) {
      if (t == 0) {
        const uint32_t sb = __float_as_uint(scale);
        j.out[0] = sb & 0xff;
        j.out[1] = (sb >> 8) & 0xff;
        j.out[2] = (sb >> 16) & 0xff;
        j.out[3] = (sb >> 24) & 0xff;
      }
      const uint32_t size = (uint32_t)umin64(kPlaceTiles, j.n_tiles - c * kPlaceTiles);
      __threadfence();
      sm.last = atomicAdd(dj.ccount + c, 1u) == size - 1 ? 1u : 0u;
    }
    __syncthreads();
    if (sm.last && warp == 0) {
      __threadfence();
      const uint32_t tt = c * kPlaceTiles + lane;
      ZScan v = {0u, {0u, 0u, 0u, 0u}};
      if (tt < j.n_tiles) v = {1u, unpack_agg32(__ldcg(dj.aggs + tt))};
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const ZScan o = zshfl_up(v, d);
        if (lane >= d) v = zcombine(o, v);
      }
      const uint64_t cw = ChunkCodec::pack(v.a);  // lane 31: the chunk's summary
      if (lane == 31) dj.cagg[c] = cw;
      if (dj.scount) {
        // The same one level up: the last chunk of a 32-chunk span to be
        // summed up sums up the span.
        const uint32_t sp = c / kPlaceSpan;
        const uint32_t n_chunks = (j.n_tiles + kPlaceTiles - 1) / kPlaceTiles;
        uint32_t slast = 0;
        if (lane == 31) {
          const uint32_t size = (uint32_t)umin64(kPlaceSpan, n_chunks - sp * kPlaceSpan);
          __threadfence();
          slast = atomicAdd(dj.scount + sp, 1u) == size - 1 ? 1u : 0u;
        }
        if (__shfl_sync(0xffffffffu, slast, 31)) {
          __threadfence();
          const uint32_t cc = sp * kPlaceSpan + lane;
          const uint64_t own = __shfl_sync(0xffffffffu, cw, 31);
          ZScan w = {0u, {0u, 0u, 0u, 0u}};
          if (cc < n_chunks) w = {1u, ChunkCodec::unpack(cc == c ? own : __ldcg(dj.cagg + cc))};
#pragma unroll
          for (int d = 1; d < 32; d <<= 1) {
            const ZScan o = zshfl_up(w, d);
            if (lane >= d) w = zcombine(o, w);
          }
          if (lane == 31) dj.sagg[sp] = ChunkCodec::pack(w.a);
        }
      }
    }
  }
}

// scale = M * s and the zero-band threshold from the bits of M; false when
// the step is non-finite (M not finite, or M * s overflows).
__device__ __forceinline__ bool scale_from_max(uint32_t mbits, float s, float &scale,
                                               float &thr) {
  if (mbits >= 0x7f800000u) return false;
  scale = __fmul_rn(__uint_as_float(mbits), s);
  if (!isfinite(scale)) return false;
  thr = zero_band_threshold(scale, mbits == 0);
  return true;
}

struct QuantArgs {
  uint32_t *aggs;    // deferred placement only: tile summaries,
  uint8_t *stage;    // staged bytes,
  uint32_t *ok;      // 1 if the step is finite (written by block 0),
  uint32_t *ccount;  // chunk counters,
  uint64_t *cagg;    // chunk summaries,
  uint32_t *scount;  // span counters and
  uint64_t *sagg;    // span summaries
  const float *x;
  float *err;
  uint64_t n;
  uint64_t groups;
  float s;
  const uint32_t *partial;
  uint32_t n_partial;
  uint8_t *out;
  uint64_t out_cap;
  uint64_t *out_len;
  uint64_t *status;
  uint32_t *ticket;
  uint32_t n_tiles;
  int32_t *dev_status;
  uint32_t max_polls;
  CompressRecord *rec;  // or nullptr
};

#if TLC_Q_MINB > 1
#define TLC_Q_BOUNDS __launch_bounds__(kQThreads, TLC_Q_MINB)
#else
#define TLC_Q_BOUNDS __launch_bounds__(kQThreads)
#endif

// kRecord: the call asked for a record (M, scale, non-zero count, length).
template <bool kVec, bool kDeferred, bool kRecord = false>
__global__ void TLC_Q_BOUNDS k_quant_zre(const QuantArgs a) {
  __shared__ QuantSmem sm;
  __shared__ uint32_t tile_id_s;
  __shared__ float scale_s, thr_s;
  __shared__ int ok_s;
  pdl_enter();

  // M from the per-block partial maxima of k_absmax.
  if (threadIdx.x < kWarp) {
    uint32_t mb = 0;
    for (uint32_t i = threadIdx.x; i < a.n_partial; i += kWarp) mb = max(mb, a.partial[i]);
    mb = __reduce_max_sync(0xffffffffu, mb);
    if (threadIdx.x == 0) {
      float scale = 0.0f, thr = 0.0f;
      ok_s = scale_from_max(mb, a.s, scale, thr) ? 1 : 0;
      scale_s = scale;
      thr_s = thr;
      if (kRecord && blockIdx.x == 0) {
        a.rec->m_bits = mb;
        a.rec->scale = ok_s ? scale : 0.0f;
      }
    }
  }
  __syncthreads();
  if (kDeferred && blockIdx.x == 0 && threadIdx.x == 0) *a.ok = ok_s;
  if (!ok_s) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      report(a.dev_status, TLC_ERR_NONFINITE);
      *a.out_len = 0;
      if (kRecord) a.rec->length = 0;
    }
    return;
  }
  const float scale = scale_s, thr = thr_s;
  const TileJob job = {a.x, a.err, a.n, a.groups, a.out, a.out_cap, a.out_len,
                       a.status, a.n_tiles, kVec, kRecord ? a.rec : nullptr};
  const DeferJob djob = {a.aggs, a.stage, a.ccount, a.cagg, a.scount, a.sagg};
  for (;;) {
    if (threadIdx.x == 0) tile_id_s = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t tk = tile_id_s;
    if (tk >= a.n_tiles) break;
    // Deferred tiles wait on no other tile, so they run last tile first:
    // k_absmax swept x and err front to back, and the end of both is still
    // in L2.  Look-back tiles keep ticket order (each waits on earlier ones).
    const uint32_t t = kDeferred ? a.n_tiles - 1 - tk : tk;
    quant_tile<kDeferred, kRecord>(job, djob, t, scale, thr, sm, a.dev_status, a.max_polls);
  }
}

// Warp-wide writes of a tile's bytes at any destination alignment: single
// bytes up to the first 16-byte boundary and after the last, 16-byte stores
// in between (other warps write the neighbouring bytes at the same time).
__device__ __forceinline__ void warp_fill_255(uint8_t *dst, uint32_t len, int lane) {
  const uint32_t head = (uint32_t)umin64(len, (16u - ((uint32_t)(uintptr_t)dst & 15u)) & 15u);
  if ((uint32_t)lane < head) dst[lane] = 255;
  const uint32_t nvec = (len - head) / 16u;
  uint4 *v = reinterpret_cast<uint4 *>(dst + head);
  for (uint32_t k = lane; k < nvec; k += kWarp) v[k] = make_uint4(~0u, ~0u, ~0u, ~0u);
  const uint32_t ts = head + 16u * nvec;
  if (ts + lane < len) dst[ts + lane] = 255;
}

// src is 16-byte aligned; every source word read lies in [src, src + len)
// rounded out to whole words.
__device__ __forceinline__ void warp_copy(uint8_t *dst, const uint8_t *__restrict__ src,
                                          uint32_t len, int lane) {
  const uint32_t head = (uint32_t)umin64(len, (16u - ((uint32_t)(uintptr_t)dst & 15u)) & 15u);
  if ((uint32_t)lane < head) dst[lane] = src[lane];
  const uint32_t nvec = (len - head) / 16u;
  const uint32_t sh = 8u * (head & 3u);
  const uint32_t *s32 = reinterpret_cast<const uint32_t *>(src) + (head >> 2);
  uint4 *v = reinterpret_cast<uint4 *>(dst + head);
#pragma unroll 4
  for (uint32_t k = lane; k < nvec; k += kWarp) {
    const uint32_t *w = s32 + 4 * k;
    const uint32_t w0 = w[0], w1 = w[1], w2 = w[2], w3 = w[3];
    const uint32_t w4 = sh ? w[4] : 0u;  // bytes up to head + 16k + 16 <= len
    v[k] = make_uint4(__funnelshift_r(w0, w1, sh), __funnelshift_r(w1, w2, sh),
                      __funnelshift_r(w2, w3, sh), __funnelshift_r(w3, w4, sh));
  }
  const uint32_t ts = head + 16u * nvec;
  if (ts + lane < len) dst[ts + lane] = src[ts + lane];
}

// The incoming prefix (emitted count C, run length mod 14) of chunk c:
// warp 0 composes the summaries of all earlier spans (each lane a
// contiguous share) and of the span's earlier chunks (one per lane), each by
// a warp scan.  Every lane returns the same prefix.
__device__ __forceinline__ void chunk_prefix(const uint64_t *__restrict__ cagg,
                                             const uint64_t *__restrict__ sagg, uint32_t c,
                                             int lane, uint32_t &C, uint32_t &tt) {
  const uint32_t sp = c / kPlaceSpan;
  const uint32_t per = (sp + kWarp - 1) / kWarp;
  const uint32_t pe = (uint32_t)umin64((uint64_t)(lane + 1) * per, sp);
  const uint32_t cc = sp * kPlaceSpan + lane;
  const uint64_t cw = cc < c ? cagg[cc] : 0;
  ZScan p = {0u, {0u, 0u, 0u, 0u}};
  for (uint32_t i = lane * per; i < pe; ++i) p = zcombine(p, {1u, ChunkCodec::unpack(sagg[i])});
  ZScan q = {0u, {0u, 0u, 0u, 0u}};
  if (cc < c) q = {1u, ChunkCodec::unpack(cw)};
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const ZScan o = zshfl_up(p, d);
    if (lane >= d) p = zcombine(o, p);
    const ZScan oq = zshfl_up(q, d);
    if (lane >= d) q = zcombine(oq, q);
  }
  C = 0;
  tt = 0;
  if (__shfl_sync(0xffffffffu, p.valid, 31)) {
    ZAgg pa;
    pa.all = __shfl_sync(0xffffffffu, p.a.all, 31);
    pa.A = __shfl_sync(0xffffffffu, p.a.A, 31);
    pa.R = __shfl_sync(0xffffffffu, p.a.R, 31);
    pa.tc = __shfl_sync(0xffffffffu, p.a.tc, 31);
    eval_agg(C, tt, pa);
  }
  if (__shfl_sync(0xffffffffu, q.valid, 31)) {
    ZAgg qa;
    qa.all = __shfl_sync(0xffffffffu, q.a.all, 31);
    qa.A = __shfl_sync(0xffffffffu, q.a.A, 31);
    qa.R = __shfl_sync(0xffffffffu, q.a.R, 31);
    qa.tc = __shfl_sync(0xffffffffu, q.a.tc, 31);
    eval_agg(C, tt, qa);
  }
}

// One tile's bytes in place, by one warp: the leading run's bytes (full
// 14-chunks as 255, then, if the run ends in the tile, its remainder byte)
// and the staged bytes, from the tile's incoming prefix (C, tin).
__device__ __forceinline__ void place_tile(const ZAgg &a, uint32_t C, uint32_t tin,
                                           const uint8_t *__restrict__ staged, uint8_t *out,
                                           uint64_t out_cap, int lane) {
  const uint32_t lead = lead_count(a, tin);
  const uint32_t r = (tin + a.A) % 14u;
  const bool rem = !a.all && r;  // the run ends in the tile with a remainder
  uint8_t *o = out + 4ull + C;
  const uint64_t room = out_cap > 4ull + C ? out_cap - 4ull - C : 0;
  (void)TLC_CHECK((uint64_t)lead + a.R <= room);  // the tile's bytes fit the stream
  warp_fill_255(o, (uint32_t)umin64(lead - (rem ? 1u : 0u), room), lane);
  if (rem && lane == 0 && TLC_BOUND(lead - 1 < room)) o[lead - 1] = remainder_byte(r);
  if (lead < room) warp_copy(o + lead, staged, (uint32_t)umin64(a.R, room - lead), lane);
}

// Warp 0 of a placement block: from the chunk's incoming prefix (C, tt),
// scan the chunk's nv tile summaries (w: lane l's tile l) and keep each
// tile's exclusive prefix and summary in shared memory.  Lane nv - 1 gets
// back in (C, tt) the state after the chunk's last tile.
__device__ __forceinline__ void scan_chunk_tiles(uint32_t w, uint32_t nv, int lane, uint32_t &C,
                                                 uint32_t &tt, uint32_t *tC, uint32_t *tT,
                                                 uint32_t *tA) {
  ZScan v = {0u, {0u, 0u, 0u, 0u}};
  if ((uint32_t)lane < nv) v = {1u, unpack_agg32(w)};
  ZScan inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const ZScan o = zshfl_up(inc, d);
    if (lane >= d) inc = zcombine(o, inc);
  }
  ZScan exc = zshfl_up(inc, 1);
  if (lane == 0) exc.valid = 0;
  if (exc.valid) eval_agg(C, tt, exc.a);
  tC[lane] = C;
  tT[lane] = tt;
  tA[lane] = w;
  if ((uint32_t)lane < nv) eval_agg(C, tt, v.a);
}

// Put the tiles' output in place, one block per 32-tile chunk.  Warp 0
// finds the chunk's incoming prefix (chunk_prefix), scans the chunk's own
// tile summaries (one per lane) and keeps every tile's exclusive prefix in
// shared memory; then each warp places every kPlaceWarps-th tile of the
// chunk.  The block of the last tile writes the closing remainder and the
// length.  No block waits on another, and one wave of blocks covers 2^28
// values (820 chunks).
constexpr int kPlaceWarps = 8;
constexpr int kPlaceThreads = kPlaceWarps * kWarp;
__global__ void __launch_bounds__(kPlaceThreads)
k_zre_place(const uint32_t *__restrict__ aggs, const uint64_t *__restrict__ cagg,
            const uint64_t *__restrict__ sagg, uint32_t n_tiles, const uint32_t *ok,
            const uint8_t *__restrict__ stage, uint8_t *out, uint64_t out_cap, uint64_t *out_len,
            CompressRecord *rec) {
  __shared__ uint32_t tC[kPlaceTiles], tT[kPlaceTiles], tA[kPlaceTiles];
  pdl_enter();
  if (!*ok) return;  // non-finite step: nothing was encoded
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t c = blockIdx.x;
  const uint32_t t0 = c * kPlaceTiles;
  const uint32_t nv = (uint32_t)umin64(kPlaceTiles, n_tiles - t0);
  if (warp == 0) {
    const uint32_t w = (uint32_t)lane < nv ? aggs[t0 + lane] : 0u;
    uint32_t C, tt;
    chunk_prefix(cagg, sagg, c, lane, C, tt);
    scan_chunk_tiles(w, nv, lane, C, tt, tC, tT, tA);
    if (t0 + nv == n_tiles && (uint32_t)lane == nv - 1) {
      // the stream's end: state after the last tile
      if (tt && TLC_BOUND(4ull + C < out_cap)) out[4 + C] = remainder_byte(tt);
      *out_len = 4ull + C + (tt ? 1u : 0u);
      if (rec) rec->length = 4ull + C + (tt ? 1u : 0u);
    }
  }
  __syncthreads();
  for (uint32_t k = warp; k < nv; k += kPlaceWarps)
    place_tile(unpack_agg32(tA[k]), tC[k], tT[k], stage + (uint64_t)(t0 + k) * kTileGroups, out,
               out_cap, lane);
}

// ------------------------------------------------- batched (tensor lists) --
// Magnitude pass over a list of tensors: one block per chunk of up to
// kBatchChunk values of one tensor, one atomic maximum per tensor.
__global__ void __launch_bounds__(kAbsThreads)
k_absmax_batch(const BatchTensor *__restrict__ tensors, const BatchChunk *__restrict__ chunks,
               uint32_t *__restrict__ mbits) {
  pdl_enter();
  const BatchChunk ch = chunks[blockIdx.x];
  const BatchTensor &T = tensors[ch.tensor];
  const uint64_t b = ch.start, e = umin64(ch.start + kBatchChunk, T.n);
  uint32_t m = 0;
  if (T.vec_q) {
    // b is a multiple of kBatchChunk, so x + b and err + b stay 16-byte aligned
    const uint64_t n4 = (e - b) >> 2;
    const float4 *x4 = reinterpret_cast<const float4 *>(T.x + b);
    const float4 *e4 = reinterpret_cast<const float4 *>(T.err + b);
    constexpr int kU = kBatchChunk / 4 / kAbsThreads;
    float4 xa[kU], ea[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const uint64_t i = threadIdx.x + (uint64_t)u * kAbsThreads;
      if (i < n4) {
        xa[u] = __ldg(x4 + i);
        ea[u] = __ldg(e4 + i);
      } else {
        xa[u] = ea[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      m = max(m, abs_bits(__fadd_rn(xa[u].x, ea[u].x)));
      m = max(m, abs_bits(__fadd_rn(xa[u].y, ea[u].y)));
      m = max(m, abs_bits(__fadd_rn(xa[u].z, ea[u].z)));
      m = max(m, abs_bits(__fadd_rn(xa[u].w, ea[u].w)));
    }
    const uint64_t r = b + (n4 << 2) + threadIdx.x;
    if (r < e) m = max(m, abs_bits(__fadd_rn(T.x[r], T.err[r])));
  } else {
    for (uint64_t i = b + threadIdx.x; i < e; i += kAbsThreads)
      m = max(m, abs_bits(__fadd_rn(T.x[i], T.err[i])));
  }
  __shared__ uint32_t wmax[kAbsThreads / kWarp];
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < kWarp) {
    uint32_t v = threadIdx.x < kAbsThreads / kWarp ? wmax[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xffffffffu, v);
    if (threadIdx.x == 0) atomicMax(mbits + ch.tensor, v);
  }
}

struct BatchQuantArgs {
  const BatchTensor *tensors;
  const uint32_t *tile_tensor;  // tensor of each global tile
  const uint32_t *mbits;        // per-tensor bits of M
  float s;
  uint8_t *arena;
  uint64_t *out_lens;
  uint64_t *status;             // all tensors' tile status words
  uint32_t *ticket;
  uint32_t n_tiles;             // over all tensors
  int32_t *dev_status;
  uint32_t max_polls;
  // deferred placement: tile summaries and chunk counters (in status),
  // chunk summaries, staging
  uint32_t *aggs;
  uint32_t *ccount;
  uint64_t *cagg;
  uint8_t *stage;
  const uint32_t *chunk_tensor;  // tensor of each chunk (global numbering)
  uint32_t n_chunks;
};

// Quantize + encode over a list of tensors: tiles of all tensors in one
// ticket order (tensor by tensor), each look-back confined to its tensor;
// with kDeferred, each tensor's tiles stage their bytes for
// k_zre_place_batch instead.
template <bool kDeferred>
__global__ void TLC_Q_BOUNDS k_quant_zre_batch(const BatchQuantArgs a) {
  __shared__ QuantSmem sm;
  __shared__ uint32_t tile_id_s;
  pdl_enter();
  for (;;) {
    if (threadIdx.x == 0) tile_id_s = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t tk = tile_id_s;
    if (tk >= a.n_tiles) break;
    const uint32_t u = kDeferred ? a.n_tiles - 1 - tk : tk;  // as in k_quant_zre
    const uint32_t id = a.tile_tensor[u];
    const BatchTensor &T = a.tensors[id];
    const uint32_t t = u - T.q_tile_begin;
    float scale = 0.0f, thr = 0.0f;
    if (!scale_from_max(a.mbits[id], a.s, scale, thr)) {
      if (t == 0 && threadIdx.x == 0) {
        report(a.dev_status, TLC_ERR_NONFINITE);
        a.out_lens[id] = 0;
      }
      __syncthreads();
      continue;
    }
    const TileJob job = {T.x,   T.err, T.n, T.groups, a.arena + T.arena_off, T.cap,
                         a.out_lens + id, a.status + T.q_tile_begin, T.q_tiles, T.vec_q != 0,
                         nullptr};
    if (kDeferred) {
      const DeferJob dj = {a.aggs + T.q_tile_begin,
                           a.stage + (uint64_t)T.q_tile_begin * kTileGroups,
                           a.ccount + T.q_chunk_begin, a.cagg + T.q_chunk_begin, nullptr,
                           nullptr};
      quant_tile<true>(job, dj, t, scale, thr, sm, a.dev_status, a.max_polls);
    } else {
      quant_tile<false>(job, DeferJob{}, t, scale, thr, sm, a.dev_status, a.max_polls);
    }
  }
}

// Deferred placement over a list of tensors, one block per 32-tile chunk
// (all tensors' chunks in one numbering, chunk_tensor naming each one's
// tensor): warp 0 composes the summaries of the tensor's earlier chunks
// (each lane a contiguous share, then a warp scan) and scans the chunk's
// tiles, then each warp places every kPlaceWarps-th tile of the chunk.  The
// block of a tensor's last tile writes the closing remainder byte and the
// length.  Tensors whose step is non-finite are skipped (k_quant_zre_batch
// set their length to 0).
__global__ void __launch_bounds__(kPlaceThreads) k_zre_place_batch(const BatchQuantArgs a) {
  __shared__ uint32_t tC[kPlaceTiles], tT[kPlaceTiles], tA[kPlaceTiles];
  pdl_enter();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t id = a.chunk_tensor[blockIdx.x];
  const BatchTensor &T = a.tensors[id];
  float scale = 0.0f, thr = 0.0f;
  if (!scale_from_max(a.mbits[id], a.s, scale, thr)) return;  // whole block
  const uint32_t c = blockIdx.x - T.q_chunk_begin;
  const uint32_t t0 = c * kPlaceTiles;
  const uint32_t nv = (uint32_t)umin64(kPlaceTiles, T.q_tiles - t0);
  uint8_t *out = a.arena + T.arena_off;
  const uint64_t out_cap = T.cap;
  if (warp == 0) {
    const uint32_t *aggs = a.aggs + T.q_tile_begin;
    const uint64_t *cagg = a.cagg + T.q_chunk_begin;
    const uint32_t w = (uint32_t)lane < nv ? aggs[t0 + lane] : 0u;
    // chunks [0, c) of this tensor: lane l folds [l * per, (l + 1) * per)
    const uint32_t per = (c + kWarp - 1) / kWarp;
    ZScan p = {0u, {0u, 0u, 0u, 0u}};
    const uint32_t pe = (uint32_t)umin64((uint64_t)(lane + 1) * per, c);
    for (uint32_t i = lane * per; i < pe; ++i) p = zcombine(p, {1u, ChunkCodec::unpack(cagg[i])});
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const ZScan o = zshfl_up(p, d);
      if (lane >= d) p = zcombine(o, p);
    }
    uint32_t C = 0, tt = 0;
    if (__shfl_sync(0xffffffffu, p.valid, 31)) {
      ZAgg pa;
      pa.all = __shfl_sync(0xffffffffu, p.a.all, 31);
      pa.A = __shfl_sync(0xffffffffu, p.a.A, 31);
      pa.R = __shfl_sync(0xffffffffu, p.a.R, 31);
      pa.tc = __shfl_sync(0xffffffffu, p.a.tc, 31);
      eval_agg(C, tt, pa);
    }
    scan_chunk_tiles(w, nv, lane, C, tt, tC, tT, tA);
    if (t0 + nv == T.q_tiles && (uint32_t)lane == nv - 1) {
      if (tt && TLC_BOUND(4ull + C < out_cap)) out[4 + C] = remainder_byte(tt);
      a.out_lens[id] = 4ull + C + (tt ? 1u : 0u);
    }
  }
  __syncthreads();
  for (uint32_t k = warp; k < nv; k += kPlaceWarps)
    place_tile(unpack_agg32(tA[k]), tC[k], tT[k],
               a.stage + (uint64_t)(T.q_tile_begin + t0 + k) * kTileGroups, out, out_cap, lane);
}

// Wait-limit check of the compress look-back: tile 1 looks back at a tile 0
// that never publishes (its status word stays 0); lookback_words reports
// TLC_ERR_TIMEOUT once the polls run out and returns a zero prefix.
__global__ void k_compress_wait_test(uint64_t *status, uint32_t max_polls, int32_t *dev_status) {
  const ZAgg agg = {0u, 0u, 1u, 0u};
  uint32_t cin = 0, tin = 0;
  lookback_words<kLookV, TileCodec>(status, 1, agg, cin, tin, dev_status, max_polls);
}

cudaError_t launch_compress_wait_test(uint64_t *status, uint32_t max_polls, int32_t *dev_status,
                                      cudaStream_t stream) {
  k_compress_wait_test<<<1, kWarp, 0, stream>>>(status, max_polls, dev_status);
  return cudaGetLastError();
}

// ------------------------------------------------------------- launcher ---
uint32_t compress_tiles(uint64_t n) {
  const uint64_t g = (n + 4) / 5;
  return (uint32_t)((g + kTileGroups - 1) / kTileGroups);
}

uint32_t compress_partials(const DeviceInfo &dev, uint64_t n) {
  const uint64_t per_block = (uint64_t)kAbsThreads * 4 * kAbsUnroll;
  uint64_t want = (n + per_block - 1) / per_block;
  const uint64_t cap = (uint64_t)dev.sm_count * 4;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return (uint32_t)want;
}

size_t compress_scratch_bytes_for(const DeviceInfo &dev, uint64_t n, bool deferred) {
  const uint32_t np = compress_partials(dev, n), nt = compress_tiles(n);
  return deferred ? deferred_scratch_bytes(np, nt) : compress_scratch_bytes(np, nt);
}

bool compress_deferred(uint64_t n) { return compress_tiles(n) >= kDeferMinTiles; }

bool compress_deferred_tiles(uint64_t n_tiles) { return n_tiles >= kDeferMinTiles; }

uint32_t compress_stage_bytes_per_tile() { return kTileGroups; }

uint32_t compress_place_chunks(uint32_t n_tiles) { return (n_tiles + kPlaceTiles - 1) / kPlaceTiles; }

uint32_t compress_place_spans(uint32_t n_tiles) {
  return (compress_place_chunks(n_tiles) + kPlaceSpan - 1) / kPlaceSpan;
}

cudaError_t launch_compress(const DeviceInfo &dev, const float *x, uint64_t n, float s,
                            float *err, uint8_t *out, uint64_t out_cap, uint64_t *out_len,
                            int32_t *dev_status, uint32_t max_polls, void *scratch,
                            cudaStream_t stream, bool deferred, CompressRecord *rec) {
  const uint32_t n_tiles = compress_tiles(n);
  const uint32_t n_part = compress_partials(dev, n);
  CompressScratch sc = compress_scratch_layout(scratch, n_part, n_tiles);
  const bool vec = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(err)) & 15) == 0;

  // status words and the ticket are cleared by k_absmax (ticket sits in
  // the word right after the status array).
  timing_begin(kKindAbsmax, stream);
  if (vec)
    launch_k(k_absmax<true>, n_part, kAbsThreads, 0, stream, x, err, n, sc.partial, sc.status,
             n_tiles + 1, rec);
  else
    launch_k(k_absmax<false>, n_part, kAbsThreads, 0, stream, x, err, n, sc.partial, sc.status,
             n_tiles + 1, rec);
  timing_end(kKindAbsmax, stream);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  QuantArgs qa;
  qa.x = x;
  qa.err = err;
  qa.n = n;
  qa.groups = (n + 4) / 5;
  qa.s = s;
  qa.partial = sc.partial;
  qa.n_partial = n_part;
  qa.out = out;
  qa.out_cap = out_cap;
  qa.out_len = out_len;
  qa.status = sc.status;
  qa.ticket = sc.ticket;
  qa.n_tiles = n_tiles;
  qa.dev_status = dev_status;
  qa.max_polls = max_polls;
  qa.rec = rec;

  // the deferred path keeps its tile summaries (u32 each) and then its
  // chunk counters where the look-back words would be: k_absmax clears
  // them, every tile writes its own summary
  qa.aggs = reinterpret_cast<uint32_t *>(sc.status);
  qa.stage = nullptr;
  qa.ok = nullptr;
  qa.ccount = nullptr;
  qa.cagg = nullptr;
  qa.scount = nullptr;
  qa.sagg = nullptr;
  DeferredScratch ds = {};
  if (deferred) {
    ds = deferred_scratch_layout(scratch, n_part, n_tiles);
    qa.stage = ds.stage;
    qa.ok = ds.ok;
    qa.cagg = ds.cagg;
    qa.sagg = ds.sagg;
    // the chunk counters, then the span counters, follow the summaries in
    // the (cleared) status area: n_tiles + chunks + spans < 2 * n_tiles
    qa.ccount = qa.aggs + n_tiles;
    qa.scount = qa.ccount + compress_place_chunks(n_tiles);
  }

  int occ = vec ? dev.occ_quant_vec : dev.occ_quant_scalar;
  uint32_t grid = (uint32_t)dev.sm_count * (uint32_t)(occ > 0 ? occ : 1);
  if (grid > n_tiles) grid = n_tiles;
  timing_begin(kKindQuantZre, stream);
  if (deferred) {
    if (rec)
      launch_k(vec ? k_quant_zre<true, true, true> : k_quant_zre<false, true, true>, grid,
               kQThreads, 0, stream, qa);
    else if (vec)
      launch_k(k_quant_zre<true, true>, grid, kQThreads, 0, stream, qa);
    else
      launch_k(k_quant_zre<false, true>, grid, kQThreads, 0, stream, qa);
    timing_end(kKindQuantZre, stream);
    timing_begin(kKindZrePlace, stream);
    launch_k(k_zre_place, compress_place_chunks(n_tiles), kPlaceThreads, 0, stream, qa.aggs,
             ds.cagg, ds.sagg, n_tiles, ds.ok, ds.stage, out, out_cap, out_len, rec);
    timing_end(kKindZrePlace, stream);
  } else {
    if (rec)
      launch_k(vec ? k_quant_zre<true, false, true> : k_quant_zre<false, false, true>, grid,
               kQThreads, 0, stream, qa);
    else if (vec)
      launch_k(k_quant_zre<true, false>, grid, kQThreads, 0, stream, qa);
    else
      launch_k(k_quant_zre<false, false>, grid, kQThreads, 0, stream, qa);
    timing_end(kKindQuantZre, stream);
  }
  return cudaGetLastError();
}

cudaError_t launch_compress_batch(const DeviceInfo &dev, const BatchPlanDev &p, float s,
                                  uint8_t *arena, uint64_t *out_lens, int32_t *dev_status,
                                  uint32_t max_polls, cudaStream_t stream) {
  // the per-tensor maxima, the ticket and the tile status words start at 0
  cudaError_t e = cudaMemsetAsync(p.q_zero_base, 0, p.q_zero_bytes, stream);
  if (e != cudaSuccess) return e;
  timing_begin(kKindAbsmax, stream);
  launch_k(k_absmax_batch, p.n_chunks, kAbsThreads, 0, stream, p.tensors, p.chunks, p.mbits);
  timing_end(kKindAbsmax, stream);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BatchQuantArgs qa;
  qa.tensors = p.tensors;
  qa.tile_tensor = p.q_tile_tensor;
  qa.mbits = p.mbits;
  qa.s = s;
  qa.arena = arena;
  qa.out_lens = out_lens;
  qa.status = p.q_status;
  qa.ticket = p.q_ticket;
  qa.n_tiles = p.n_q_tiles;
  qa.dev_status = dev_status;
  qa.max_polls = max_polls;
  qa.aggs = reinterpret_cast<uint32_t *>(p.q_status);  // cleared with the status words
  qa.ccount = qa.aggs + p.n_q_tiles;
  qa.cagg = p.q_cagg;
  qa.stage = p.q_stage;
  qa.chunk_tensor = p.q_chunk_tensor;
  qa.n_chunks = p.n_q_chunks;
  uint32_t grid = (uint32_t)dev.sm_count * (uint32_t)(dev.occ_quant_batch > 0 ? dev.occ_quant_batch : 1);
  if (grid > p.n_q_tiles) grid = p.n_q_tiles;
  timing_begin(kKindQuantZre, stream);
  if (p.q_deferred)
    launch_k(k_quant_zre_batch<true>, grid, kQThreads, 0, stream, qa);
  else
    launch_k(k_quant_zre_batch<false>, grid, kQThreads, 0, stream, qa);
  timing_end(kKindQuantZre, stream);
  if (p.q_deferred) {
    timing_begin(kKindZrePlace, stream);
    launch_k(k_zre_place_batch, p.n_q_chunks, kPlaceThreads, 0, stream, qa);
    timing_end(kKindZrePlace, stream);
  }
  return cudaGetLastError();
}

int occupancy_quant_batch() {
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_quant_zre_batch<false>, kQThreads, 0);
  return occ;
}

int occupancy_quant(bool vec) {
  int occ = 0;
  if (vec)
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_quant_zre<true, false>, kQThreads, 0);
  else
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_quant_zre<false, false>, kQThreads, 0);
  return occ;
}

}  // namespace tlc
