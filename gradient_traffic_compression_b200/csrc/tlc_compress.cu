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
// Two launches per call:
//   k_absmax     x' = x + err and M = max|x'| (as a max over the uint32 bit
//                patterns of |x'|; NaN/Inf sort above every finite value).
//                It also clears the scan state that k_quant_zre uses.
//   k_quant_zre  per tile of 4096 byte groups (20480 values): recompute x',
//                q = round(x'/(M s)), err' = x' - q M s (written back), pack
//                the quartic bytes into shared memory, zero-run encode them,
//                and place the tile's output with a decoupled look-back over
//                earlier tiles.  Tiles are taken in order from a ticket
//                counter, so every tile a tile waits on is already running.
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
#include "tlc_device.cuh"
#include "tlc_internal.h"

namespace tlc {

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
         uint32_t n_zero) {
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
#define TLC_Q_ITERS 4
#endif
#ifndef TLC_Q_MINB
#define TLC_Q_MINB 6
#endif
constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / kWarp;
constexpr int kChunkElems = 640;   // one warp step: 32 lanes x 5 float4
constexpr int kChunkGroups = 128;  // = kChunkElems / 5
constexpr int kQIters = TLC_Q_ITERS;
constexpr int kTileGroups = kQWarps * kQIters * kChunkGroups;  // 4096 by default
constexpr uint64_t kTileElems = 5ull * kTileGroups;            // 20480 by default
constexpr int kZBytes = kTileGroups / kQThreads;               // 16 per thread by default
constexpr int kZWords = kZBytes / 4;                           // u32 words per thread
static_assert((kZBytes == 8 || kZBytes % 16 == 0) && kTileGroups < 65536, "tile shape");
#ifndef TLC_Q_LOOKV
#define TLC_Q_LOOKV 1
#endif
constexpr int kLookV = TLC_Q_LOOKV;  // look-back words per lane per round trip


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
};

// Shared memory of one compress block.
struct QuantSmem {
  __align__(16) uint32_t dig[kQWarps][kChunkElems / 4];  // digits q+1, one byte per value
  __align__(16) uint32_t tile[kTileGroups / 4];          // the tile's quartic bytes
  uint32_t scan[kQWarps + 1];
  uint32_t A, cin, tin;
};

__device__ __forceinline__ void put_out(const TileJob &j, uint64_t pos, uint8_t v) {
  if (4 + pos < j.out_cap) j.out[4 + pos] = v;
}

// Decoupled look-back for tile t, by one whole warp: publish the tile's
// aggregate, combine earlier tiles' words until an inclusive prefix is
// found, publish this tile's inclusive prefix, and return the exclusive
// prefix (emitted count, incoming run length mod 14) to every lane.  Each
// round trip reads 32 * kV earlier words: every lane first folds its kV
// words (oldest to nearest), then the lanes are folded in order.
template <int kV>
__device__ __forceinline__ void lookback_warp(const TileJob &j, uint32_t t, const ZAgg &agg,
                                              uint32_t &cin, uint32_t &tin, int32_t *dev_status,
                                              uint32_t max_polls) {
  constexpr int kLookV = kV;
  const int lane = threadIdx.x & 31;
  if (t == 0) {
    if (lane == 0) {
      uint32_t C = 0, tt = 0;
      eval_agg(C, tt, agg);
      st_relaxed_u64(j.status, pack_prefix(C, tt));
    }
    cin = 0;
    tin = 0;
    return;
  }
  if (lane == 0) st_relaxed_u64(j.status + t, pack_agg(agg));
  bool timed_out = false;
  bool have_suffix = false;
  ZAgg suffix = {0, 0, 0, 0};
  int64_t end = (int64_t)t - 1;
  uint32_t C = 0, tt = 0;
  for (;;) {
    uint64_t w[kLookV];
    load_window(j.status, end, pack_prefix(0, 0), max_polls, timed_out, w);
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
        const ZAgg ak = unpack_agg(w[k]);
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
    st_relaxed_u64(j.status + t, pack_prefix(Ci, ti));
  }
  cin = C;
  tin = tt;
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
  }
}

// One warp step: values [e0, e0 + 640) of a tensor -> err' written back and
// the 128 quartic bytes of these values, four per lane, returned packed
// (lane L holds groups 4L..4L+3 of the step).  `dig` is this warp's 640-byte
// shared buffer of digits.  Values past n count as zero (digit 1).
__device__ __forceinline__ uint32_t quant_chunk(const float *x, float *err, uint64_t n,
                                                uint64_t e0, bool vec_full, float scale,
                                                float thr, uint32_t *dig) {
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
template <int kZB, int kV>
__device__ __forceinline__ void zre_encode_tile(const TileJob &j, uint32_t t, uint32_t tgv,
                                                const uint32_t (&qw)[kZB / 4], float scale,
                                                QuantSmem &sm, int32_t *dev_status,
                                                uint32_t max_polls) {
  constexpr int kZW = kZB / 4;
  bool mine_all = true;
#pragma unroll
  for (int w = 0; w < kZW; ++w) mine_all = mine_all && qw[w] == 0x79797979u;
  // bytes past tgv are all-zero (121) groups by construction
  if (__syncthreads_and(mine_all)) {
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

// One tile of 4096 byte groups (20480 values) of one tensor, fused: quantize
// and update the error buffer, pack the quartic bytes into shared memory,
// then zero-run encode them.  Whole block; ends synchronised.
__device__ __forceinline__ void quant_tile(const TileJob &j, uint32_t t, float scale, float thr,
                                           QuantSmem &sm, int32_t *dev_status,
                                           uint32_t max_polls) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) sm.A = 0xffffffffu;
  const uint64_t g0 = (uint64_t)t * kTileGroups;
  const uint32_t tgv = (uint32_t)umin64(kTileGroups, j.groups - g0);
  const uint64_t e_tile = g0 * 5;
  const bool full = j.vec && (e_tile + kTileElems <= j.n);
#pragma unroll 1
  for (int it = 0; it < kQIters; ++it) {
    const int c = it * kQWarps + warp;
    const uint64_t e0 = e_tile + (uint64_t)c * kChunkElems;
    sm.tile[c * (kChunkGroups / 4) + lane] =
        quant_chunk(j.x, j.err, j.n, e0, full, scale, thr, sm.dig[warp]);
  }
  __syncthreads();
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
  zre_encode_tile<kZBytes, kLookV>(j, t, tgv, qw, scale, sm, dev_status, max_polls);
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
};

#if TLC_Q_MINB > 1
#define TLC_Q_BOUNDS __launch_bounds__(kQThreads, TLC_Q_MINB)
#else
#define TLC_Q_BOUNDS __launch_bounds__(kQThreads)
#endif

template <bool kVec>
__global__ void TLC_Q_BOUNDS k_quant_zre(const QuantArgs a) {
  __shared__ QuantSmem sm;
  __shared__ uint32_t tile_id_s;
  __shared__ float scale_s, thr_s;
  __shared__ int ok_s;

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
    }
  }
  __syncthreads();
  if (!ok_s) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      report(a.dev_status, TLC_ERR_NONFINITE);
      *a.out_len = 0;
    }
    return;
  }
  const float scale = scale_s, thr = thr_s;
  const TileJob job = {a.x, a.err, a.n, a.groups, a.out, a.out_cap, a.out_len,
                       a.status, a.n_tiles, kVec};
  for (;;) {
    if (threadIdx.x == 0) tile_id_s = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t t = tile_id_s;
    if (t >= a.n_tiles) break;
    quant_tile(job, t, scale, thr, sm, a.dev_status, a.max_polls);
  }
}

// ------------------------------------------------- batched (tensor lists) --
// Magnitude pass over a list of tensors: one block per chunk of up to
// kBatchChunk values of one tensor, one atomic maximum per tensor.
__global__ void __launch_bounds__(kAbsThreads)
k_absmax_batch(const BatchTensor *__restrict__ tensors, const BatchChunk *__restrict__ chunks,
               uint32_t *__restrict__ mbits) {
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
};

// Quantize + encode over a list of tensors: tiles of all tensors in one
// ticket order (tensor by tensor), each look-back confined to its tensor.
__global__ void TLC_Q_BOUNDS k_quant_zre_batch(const BatchQuantArgs a) {
  __shared__ QuantSmem sm;
  __shared__ uint32_t tile_id_s;
  for (;;) {
    if (threadIdx.x == 0) tile_id_s = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const uint32_t u = tile_id_s;
    if (u >= a.n_tiles) break;
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
    const TileJob job = {T.x, T.err, T.n, T.groups, a.arena + T.arena_off, T.cap,
                         a.out_lens + id, a.status + T.q_tile_begin, T.q_tiles, T.vec_q != 0};
    quant_tile(job, t, scale, thr, sm, a.dev_status, a.max_polls);
  }
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

size_t compress_scratch_bytes_for(const DeviceInfo &dev, uint64_t n) {
  return compress_scratch_bytes(compress_partials(dev, n), compress_tiles(n));
}

cudaError_t launch_compress(const DeviceInfo &dev, const float *x, uint64_t n, float s,
                            float *err, uint8_t *out, uint64_t out_cap, uint64_t *out_len,
                            int32_t *dev_status, uint32_t max_polls, void *scratch,
                            cudaStream_t stream) {
  const uint32_t n_tiles = compress_tiles(n);
  const uint32_t n_part = compress_partials(dev, n);
  CompressScratch sc = compress_scratch_layout(scratch, n_part, n_tiles);
  const bool vec = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(err)) & 15) == 0;

  // status words and the ticket are cleared by k_absmax (ticket sits in
  // the word right after the status array).
  timing_begin(kKindAbsmax, stream);
  if (vec)
    k_absmax<true><<<n_part, kAbsThreads, 0, stream>>>(x, err, n, sc.partial, sc.status,
                                                        n_tiles + 1);
  else
    k_absmax<false><<<n_part, kAbsThreads, 0, stream>>>(x, err, n, sc.partial, sc.status,
                                                         n_tiles + 1);
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

  int occ = vec ? dev.occ_quant_vec : dev.occ_quant_scalar;
  uint32_t grid = (uint32_t)dev.sm_count * (uint32_t)(occ > 0 ? occ : 1);
  if (grid > n_tiles) grid = n_tiles;
  timing_begin(kKindQuantZre, stream);
  if (vec)
    k_quant_zre<true><<<grid, kQThreads, 0, stream>>>(qa);
  else
    k_quant_zre<false><<<grid, kQThreads, 0, stream>>>(qa);
  timing_end(kKindQuantZre, stream);
  return cudaGetLastError();
}

cudaError_t launch_compress_batch(const DeviceInfo &dev, const BatchPlanDev &p, float s,
                                  uint8_t *arena, uint64_t *out_lens, int32_t *dev_status,
                                  uint32_t max_polls, cudaStream_t stream) {
  // the per-tensor maxima, the ticket and the tile status words start at 0
  cudaError_t e = cudaMemsetAsync(p.q_zero_base, 0, p.q_zero_bytes, stream);
  if (e != cudaSuccess) return e;
  timing_begin(kKindAbsmax, stream);
  k_absmax_batch<<<p.n_chunks, kAbsThreads, 0, stream>>>(p.tensors, p.chunks, p.mbits);
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
  uint32_t grid = (uint32_t)dev.sm_count * (uint32_t)(dev.occ_quant_batch > 0 ? dev.occ_quant_batch : 1);
  if (grid > p.n_q_tiles) grid = p.n_q_tiles;
  timing_begin(kKindQuantZre, stream);
  k_quant_zre_batch<<<grid, kQThreads, 0, stream>>>(qa);
  timing_end(kKindQuantZre, stream);
  return cudaGetLastError();
}

int occupancy_quant_batch() {
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_quant_zre_batch, kQThreads, 0);
  return occ;
}

int occupancy_quant(bool vec) {
  int occ = 0;
  if (vec)
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_quant_zre<true>, kQThreads, 0);
  else
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_quant_zre<false>, kQThreads, 0);
  return occ;
}

}  // namespace tlc
