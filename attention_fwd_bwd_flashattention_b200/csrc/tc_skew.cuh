// Transformer-XL relation products moved from offset order to key order.
//
// "Fast and Exact Relative-Position Attention via Structure-Aware Kernels"
// (Abstract, technique (1), offset-aware tiling): the pairs of tile (m, n) read the
// offsets delta = i - j in 128 (m - n) + [-127, 127], i.e. two 128-offset blocks of r:
// block Delta = m - n (local offset c = il - jl for keys jl <= il) and block Delta - 1
// (c = il - jl + 128 for keys jl > il).
//
// The kernels compute each block's products transposed, r_b Q^T, so that TMEM lane =
// local offset c and TMEM column = query row il.  A warp then owns 32 offsets (its
// TMEM lane quarter g) of 32 query rows (its row quarter qt), and the thread of offset
// c writes the value of row il to key position jl = il - c (+128) of the padded fp32
// row rot[il * LD + jl]:
//   * for fixed il the 32 lanes write 32 consecutive words: no bank conflicts;
//   * the address is a per-thread base plus a compile-time offset;
//   * a warp whose offset quarter lies below its row quarter (g < qt) only reads
//     block Delta, one above it (g > qt) only block Delta - 1; only the four
//     diagonal warps (g == qt) need both and a per-lane choice.
// Each value is written as T * scl + vr (vrA / vrB: this thread's per-offset terms
// v.r of the two blocks, already multiplied by scl; SK_ADD mode: T + vr).  Positions of
// block Delta - 1 are left unwritten when it does not exist (hasB false: causal
// diagonal tile); the kernels mask those keys (j > i).
#pragma once

#include "tc_ptx.cuh"

namespace rp {
namespace tc {

// 32 products (one TMEM row segment) -> rows 32 qt + e, as T * scl + vr.  Modes:
// SK_PACKED f32x2 FMAs, SK_FMA scalar FMAs, SK_ADD T + vr (scl ignored).
enum { SK_PACKED = 0, SK_FMA = 1, SK_ADD = 2 };
template <int RS, int MODE, int OFF>
__device__ __forceinline__ void skew_store32(const uint32_t (&r)[32], float scl, float vr, float *dst) {
  if constexpr (MODE == SK_PACKED) {
    const uint64_t scl2 = f2(scl, scl), vr2 = f2(vr, vr);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      float lo, hi;
      f2_split(fma2(f2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), scl2, vr2), lo, hi);
      dst[e * RS + OFF] = lo;
      dst[(e + 1) * RS + OFF] = hi;
    }
  } else if constexpr (MODE == SK_FMA) {
#pragma unroll
    for (int e = 0; e < 32; ++e) dst[e * RS + OFF] = fmaf(__uint_as_float(r[e]), scl, vr);
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) dst[e * RS + OFF] = __uint_as_float(r[e]) + vr;
  }
}

template <int LD, int MODE = SK_PACKED>
__device__ __forceinline__ void txl_skew(uint32_t tl, uint32_t colA, uint32_t colB, bool hasB, int g, int qt, int lane,
                                         float scl, float vrA, float vrB, float *rot) {
  constexpr int RS = LD + 1;  // row il + 1 with key jl + 1: one padded row plus one word further
  const int c = 32 * g + lane;
  float *base = rot + 32 * qt * RS - c;  // row 32 qt, key 32 qt - c
  if (qt > g) {
    uint32_t r[32];
    tmem_ld32(tl + colA + 32 * qt, r);
    tmem_wait_ld();
    skew_store32<RS, MODE, 0>(r, scl, vrA, base);
  } else if (qt < g) {
    if (hasB) {
      uint32_t r[32];
      tmem_ld32(tl + colB + 32 * qt, r);
      tmem_wait_ld();
      skew_store32<RS, MODE, 128>(r, scl, vrB, base);
    }
  } else {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint32_t ra[16], rb[16];
      tmem_ld16(tl + colA + 32 * qt + 16 * hh, ra);
      if (hasB) {
        tmem_ld16(tl + colB + 32 * qt + 16 * hh, rb);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) rb[e] = 0u;
      }
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int ee = 16 * hh + e;
        const bool lo = lane <= ee;  // key jl = il - c >= 0: block Delta
        if constexpr (MODE == SK_ADD) {
          base[ee * RS + (lo ? 0 : 128)] = lo ? __uint_as_float(ra[e]) + vrA : __uint_as_float(rb[e]) + vrB;
        } else {
          base[ee * RS + (lo ? 0 : 128)] = lo ? fmaf(__uint_as_float(ra[e]), scl, vrA) : fmaf(__uint_as_float(rb[e]), scl, vrB);
        }
      }
    }
  }
}

}  // namespace tc
}  // namespace rp
