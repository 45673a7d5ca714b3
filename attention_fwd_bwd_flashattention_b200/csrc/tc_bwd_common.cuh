// Per-tile engine shared by the tensor-core backward kernels (sm_100a): launch
// shape, score / dS arithmetic, bounded warp-wide mbarrier waits and the control
// thread's bookkeeping of TMA loads in flight.
//
// Launch shape: 16 row warps (four threads per query row: warps w, w + 4, w + 8,
// w + 12 share TMEM lanes 32 (w & 3)..+31 and take 32 key columns each) and one
// control warp whose lane 0 issues every TMA load and tcgen05.mma.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace rp {
namespace tcb {

using namespace tc;

constexpr int TPR = 4;            // row threads per query row
constexpr int NC = 128 / TPR;     // key columns per row thread
constexpr int NSOFT = 128 * TPR;  // row threads
constexpr int CTRL_WARP = NSOFT / 32;
constexpr int NTHREADS = NSOFT + 32;
constexpr int ROT_LD = 132;
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Four log2-domain scores y = s c1 + (r' + u') - lse2 of consecutive keys, from the
// QK^T accumulator bits, the relative terms r' and u.k terms u' (both already
// multiplied by c1 = scale log2 e) and nlse = (-lse2, -lse2); two f32x2 pairs.
__device__ __forceinline__ void score_pairs(const uint32_t *s, float4 rr, float4 uk, uint64_t c12, uint64_t nlse, float (&y)[4]) {
  f2_split(fma2(f2(u2f(s[0]), u2f(s[1])), c12, add2(add2(f2(rr.x, rr.y), f2(uk.x, uk.y)), nlse)), y[0], y[1]);
  f2_split(fma2(f2(u2f(s[2]), u2f(s[3])), c12, add2(add2(f2(rr.z, rr.w), f2(uk.z, uk.w)), nlse)), y[2], y[3]);
}
// dS = P (dP - D) for four keys, nDv = (-D, -D).
__device__ __forceinline__ void ds_pairs(const float (&pr)[4], const uint32_t *dp, uint64_t nDv, float (&dd)[4]) {
  f2_split(mul2(f2(pr[0], pr[1]), add2(f2(u2f(dp[0]), u2f(dp[1])), nDv)), dd[0], dd[1]);
  f2_split(mul2(f2(pr[2], pr[3]), add2(f2(u2f(dp[2]), u2f(dp[3])), nDv)), dd[2], dd[3]);
}

// log2-domain LSE of query row i for P = 2^(y - lse2): rows past L and rows with no
// key (LSE = -inf) give +inf, i.e. P = 0
__device__ __forceinline__ float lse2_of(const Prm &p, int bh, int i) {
  if (i >= p.L) return INFINITY;
  const float l = p.lse[(size_t)bh * p.L + i];
  return l == -INFINITY ? INFINITY : l * LOG2E;
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *ab, int32_t *st) {
  const bool ok = mbar_wait(bar, parity, ab, st, RELPOS_ERR_TIMEOUT_DEV);
  return __all_sync(0xffffffffu, ok);
}

// Control-thread bookkeeping: TMA loads issued but not waited for are drained on exit.
struct Ctl {
  uint32_t pb[8], pp[8];
  int np;
  volatile int *ab;
  int32_t *st;
  __device__ void expect(uint32_t bar, uint32_t par, uint32_t bytes) {
    mbar_expect_tx(bar, bytes);
    pb[np] = bar;
    pp[np] = par;
    ++np;
  }
  __device__ bool wait(uint32_t bar, uint32_t par) { return mbar_wait(bar, par, ab, st, RELPOS_ERR_TIMEOUT_DEV); }
  __device__ bool wait_load(uint32_t bar, uint32_t par) {
    if (!wait(bar, par)) return false;
    for (int e = 0; e < np; ++e)
      if (pb[e] == bar && pp[e] == par) {
        pb[e] = pb[np - 1];
        pp[e] = pp[np - 1];
        --np;
        break;
      }
    return true;
  }
  __device__ void drain(uint32_t drain_bar) {
    umma_commit(drain_bar);
    volatile int none = 0;
    mbar_wait(drain_bar, 0, &none, st, RELPOS_ERR_TIMEOUT_DEV);
    for (int e = 0; e < np; ++e) mbar_wait(pb[e], pp[e], &none, st, RELPOS_ERR_TIMEOUT_DEV);
  }
};

// 32-byte store of eight words (the address 32-byte aligned): half the memory requests of
// two 16-byte stores when a warp's threads write 32 distinct rows
__device__ __forceinline__ void st_global_32B(void *ptr, const uint32_t *w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

}  // namespace tcb
}  // namespace rp
