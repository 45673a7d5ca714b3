// Tensor-core (tcgen05 / TMEM / TMA) backward pass of the per-offset bias
// mechanisms -- T5 buckets and ALiBi -- bf16, d = 64, sm_100a.  No atomics.
//
// S_ij = s q_i.k_j + b(j - i), with b one value per offset and head (T5: t[h,
// bucket(j - i)]; ALiBi: -m[h] |j - i|), laid out once per call for every offset of
// the sequence by the preparation kernel.  The bias is gathered by offset and never
// materialised as an L x L matrix (article "结构感知内核让相对位置注意力加速21倍",
// section "为什么相对位置注意力难做快").  A 128 x 128 tile (query tile m, key tile n)
// reads the 255 offsets 128 (n - m) + [-127, 127] ("Fast and Exact Relative-Position
// Attention via Structure-Aware Kernels", Abstract, technique (1), offset-aware
// tiling).  A tile is "flat" when all of its offsets share one bias value (T5 past its
// last logarithmic bucket on that side); every other tile is a band tile.
//
//   key-tile kernel   (one CTA per key tile, query tiles streamed): recomputes P and
//                     dS with the tile's bias window (a constant on flat tiles),
//                     dV += P^T dO and dK += dS^T Q, P / dS from smem as MN-major A
//                     operands.
//   query-tile kernel (one CTA per query tile, key tiles streamed): dQ += dS K (dS as
//                     the TMEM A operand) and this query tile's share of the bias
//                     gradient (offset-sharded, technique (3)): T5 sums dS per row on
//                     flat tiles (one bucket per side) and per offset on band tiles
//                     (the fp32 dS tile goes to smem and 255 threads add its diagonals
//                     in a fixed order), folding each band tile's 255 offset sums into
//                     its buckets at once (a bucket's offsets are consecutive: a
//                     segmented scan per warp, then the warps' carries), so a band of
//                     any width needs no per-offset storage; ALiBi sums dS_ij |j - i|
//                     per thread.  A fixed-order reduction over batches and query tiles
//                     finishes dt / dm.
#include <algorithm>
#include <climits>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_bwd_common.cuh"

namespace rp {
namespace tcbias {

using namespace tc;
using namespace tcb;

constexpr int NB_MAX = 64;  // T5 buckets (the boundary's limit)

struct BiasArgs {
  CUtensorMap mq, mk, mv, mdo;
  Prm p;                   // nT counts 128-row tiles
  float *part;             // [B,H,nT][nb] per-query-tile partial of dt (ALiBi: dm, nb = 1)
  int flat_pos, flat_neg;  // offsets >= flat_pos (<= -flat_neg) all have one bias value
};

__device__ __forceinline__ bool flat_tile(const BiasArgs &A, int m, int n) {
  if (n > m) return 128 * (n - m) - 127 >= A.flat_pos;
  if (n < m) return 128 * (m - n) - 127 >= A.flat_neg;
  return false;
}

// bias (times log2 e) of offset 128 (n - m) - 127 + k, zero outside the sequence
__device__ __forceinline__ float window_at(const Prm &p, int h, int m, int n, int k) {
  const int idx = 128 * (n - m) - 127 + k + p.L - 1;
  return (idx >= 0 && idx < 2 * p.L - 1) ? p.t5_bias[(size_t)h * (2 * p.L - 1) + idx] * LOG2E : 0.f;
}

// four log2-domain scores y = s c1 + b' - lse2 (b' = bias log2 e), two f32x2 pairs
__device__ __forceinline__ void score_bias4(const uint32_t *s, const float (&R)[4], uint64_t c12, uint64_t nlse,
                                            float (&y)[4]) {
  f2_split(fma2(f2(u2f(s[0]), u2f(s[1])), c12, add2(f2(R[0], R[1]), nlse)), y[0], y[1]);
  f2_split(fma2(f2(u2f(s[2]), u2f(s[3])), c12, add2(f2(R[2], R[3]), nlse)), y[2], y[3]);
}

// ============================================================================
// key-tile kernel: dK, dV
// ============================================================================
namespace kvb {
constexpr int OFF_K = 0, OFF_V = 16384, OFF_Q = 32768, OFF_DO = OFF_Q + 32768;
constexpr int OFF_PDS = OFF_DO + 32768;  // P tile, dS tile at +32768
constexpr int OFF_VEC = OFF_PDS + 65536;  // per tile, double-buffered: [lse2 | D | bias window (255)] x 512
constexpr int OFF_BAR = OFF_VEC + 4096;
constexpr int SMEM = OFF_BAR + 256 + 1024;
enum { B_KV = 0, B_ST0, B_ST1, B_SDP, B_SDPCONS, B_PDS, B_PDSFREE, B_DRAIN, NB };
constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 320;
static_assert(OFF_PDS % 1024 == 0, "swizzled operand tiles are 1024-byte aligned");
}  // namespace kvb

__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_bias_kv_kernel(const __grid_constant__ BiasArgs A) {
  using namespace kvb;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, n = (int)blockIdx.x / BH, h = bh % p.H;
  const int L = p.L, j0 = n * 128;
  const int mStart = p.causal ? n : 0, iters = p.nT - mStart;
  const int klen = key_len(p, bh / p.H);  // keys j >= klen of this batch are masked
  if (j0 >= klen) {  // a key tile of padding only: dK = dV = 0 (whole CTA, no barrier yet)
    for (int x = tid; x < 128 * (HD / 8); x += NTHREADS) {
      const int r = x / (HD / 8), c8 = x % (HD / 8);
      if (j0 + r < L) {
        const size_t off = ((size_t)bh * L + j0 + r) * HD + 8 * c8;
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dk + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dv + off) = make_uint4(0, 0, 0, 0);
      }
    }
    return;
  }
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NB + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NB);
  float *vec = (float *)(smem + OFF_VEC);
  int32_t *status = p.status;
  const float c1 = p.scale * LOG2E;

  if (tid == 0) {
    for (int k = 0; k < NB; ++k) mbar_init(BAR(k), (k == B_SDPCONS || k == B_PDS) ? NSOFT : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == CTRL_WARP) {
    if (lane == 0) {
      Ctl ctl;
      ctl.np = 0;
      ctl.ab = abort_flag;
      ctl.st = status;
      prefetch_tmap(&A.mq);
      prefetch_tmap(&A.mk);
      prefetch_tmap(&A.mv);
      prefetch_tmap(&A.mdo);
      const uint32_t idS = idesc_bf16(128, 128, false);
      const uint32_t idAcc = idesc_bf16(128, 64, true, true);
      ctl.expect(BAR(B_KV), 0, 32768);
      tma_load_3d(sbase + OFF_K, &A.mk, BAR(B_KV), 0, j0, bh);
      tma_load_3d(sbase + OFF_V, &A.mv, BAR(B_KV), 0, j0, bh);
      auto issue_stage = [&](int t) {
        const int m = mStart + t, st = t & 1;
        ctl.expect(BAR(B_ST0 + st), (uint32_t)((t >> 1) & 1), 32768u);
        tma_load_3d(sbase + OFF_Q + 16384 * st, &A.mq, BAR(B_ST0 + st), 0, m * 128, bh);
        tma_load_3d(sbase + OFF_DO + 16384 * st, &A.mdo, BAR(B_ST0 + st), 0, m * 128, bh);
      };
      auto issue_sdp = [&](int t) {
        const int st = t & 1;
        umma_k64(tbase + T_S, sbase + OFF_Q + 16384 * st, sbase + OFF_K, idS, false);
        umma_k64(tbase + T_DP, sbase + OFF_DO + 16384 * st, sbase + OFF_V, idS, false);
        umma_commit(BAR(B_SDP));
      };
      auto accumulate = [&](int t) {  // dV += P^T dO, dK += dS^T Q (P, dS in smem)
        const int st = t & 1;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t acc = (t > 0 || k > 0) ? 1u : 0u;
          umma_bf16(tbase + T_DV, sdesc_sw128(sbase + OFF_PDS + 2048 * k, 16384, 1024),
                    sdesc_sw128(sbase + OFF_DO + 16384 * st + 2048 * k, 16, 1024), idAcc, acc);
          umma_bf16(tbase + T_DK, sdesc_sw128(sbase + OFF_PDS + 32768 + 2048 * k, 16384, 1024),
                    sdesc_sw128(sbase + OFF_Q + 16384 * st + 2048 * k, 16, 1024), idAcc, acc);
        }
        umma_commit(BAR(B_PDSFREE));
      };
      issue_stage(0);
      if (iters > 1) issue_stage(1);
      bool ok = ctl.wait_load(BAR(B_KV), 0) && ctl.wait_load(BAR(B_ST0), 0);
      if (ok) {
        tc_fence_after();
        issue_sdp(0);
      }
      for (int t = 0; ok && t < iters; ++t) {
        if (t + 1 < iters) {  // S / dP(t) read by the rows: the next tile's products overlap their work
          if (!ctl.wait(BAR(B_SDPCONS), t & 1)) break;
          if (!ctl.wait_load(BAR(B_ST0 + ((t + 1) & 1)), ((t + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_sdp(t + 1);
        }
        if (!ctl.wait(BAR(B_PDS), t & 1)) break;
        tc_fence_after();
        accumulate(t);
        if (t + 2 < iters) {  // Q / dO(t) are free once its dV / dK MMAs are done
          if (!ctl.wait(BAR(B_PDSFREE), t & 1)) break;
          issue_stage(t + 2);
        }
      }
      ctl.drain(BAR(B_DRAIN));
    }
    __syncwarp();
  } else {
    const int g = warp & 3, qt = warp >> 2, il = 32 * g + lane, cb = NC * qt;
    const uint32_t tl = tbase + ((uint32_t)(g * 32) << 16);
    bool good = true;
    // per-tile terms staged through smem one tile ahead (one element per thread):
    // [lse2 of the 128 rows | D of the rows | bias window of the tile's 255 offsets]
    auto fetch1 = [&](int t) {
      const int m = mStart + t, i = m * 128 + (tid & 127);
      if (tid < 128) return lse2_of(p, bh, i);
      if (tid < 256) return (i < L) ? p.Dvec[(size_t)bh * L + i] : 0.f;
      return window_at(p, h, m, n, tid - 256);
    };
    if (tid < 511) vec[tid] = fetch1(0);
    for (int t = 0; t < iters; ++t) {
      const int m = mStart + t, i = m * 128 + il;
      const float *tv = vec + 512 * (t & 1);
      const float nv = (tid < 511 && t + 1 < iters) ? fetch1(t + 1) : 0.f;
      named_bar_sync(1, NSOFT);
      const bool flat = flat_tile(A, m, n);
      good = good && warp_wait(BAR(B_SDP), t & 1, abort_flag, status);
      uint32_t pk[NC / 2], dk[NC / 2];
      const bool need_mask = (p.causal && m == n) || (j0 + 128 > klen);
      if (good) {
        tc_fence_after();
        const float lse2 = tv[il], Dv = tv[128 + il], rflat = tv[256 + 127];
        const float *wrow = tv + 256 + 127 - il + cb;  // bias of key cb + x: wrow[x]
        const uint64_t c12 = f2(c1, c1), nlse = f2(-lse2, -lse2), nDv = f2(-Dv, -Dv);
        auto pds = [&](auto masked, auto banded) {
#pragma unroll
          for (int hq = 0; hq < NC / 8; ++hq) {
            uint32_t rs[8], rp[8];
            tmem_ld8(tl + T_S + cb + 8 * hq, rs);
            tmem_ld8(tl + T_DP + cb + 8 * hq, rp);
            tmem_wait_ld();
#pragma unroll
            for (int c4 = 0; c4 < 2; ++c4) {
              const int x0 = 8 * hq + 4 * c4;
              float R[4], y[4], pr[4], dd[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) R[e] = decltype(banded)::value ? wrow[x0 + e] : rflat;
              score_bias4(rs + 4 * c4, R, c12, nlse, y);
              if constexpr (decltype(masked)::value) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int j = j0 + cb + x0 + e;
                  if (j >= klen || (p.causal && j > i)) y[e] = -INFINITY;
                }
              }
#pragma unroll
              for (int e = 0; e < 4; ++e) pr[e] = ex2(y[e]);
              ds_pairs(pr, rp + 4 * c4, nDv, dd);
              pk[x0 / 2] = pack_bf16x2(pr[0], pr[1]);
              pk[x0 / 2 + 1] = pack_bf16x2(pr[2], pr[3]);
              dk[x0 / 2] = pack_bf16x2(dd[0], dd[1]);
              dk[x0 / 2 + 1] = pack_bf16x2(dd[2], dd[3]);
            }
          }
        };
        if (!flat) {
          if (need_mask) pds(std::true_type{}, std::true_type{}); else pds(std::false_type{}, std::true_type{});
        } else {
          if (need_mask) pds(std::true_type{}, std::false_type{}); else pds(std::false_type{}, std::false_type{});
        }
        tc_fence_before();
        mbar_arrive(BAR(B_SDPCONS));  // S / dP read: the next tile's products may overwrite them
      }
      // the P / dS tiles are rewritten once the previous tile's dV / dK MMAs have read them
      if (t >= 1) good = good && warp_wait(BAR(B_PDSFREE), (t - 1) & 1, abort_flag, status);
      if (good) {
#pragma unroll
        for (int cc = 0; cc < NC / 8; ++cc) {
          const int ch = (NC / 8) * (qt & 1) + cc;
          const uint32_t off = 16384 * (qt >> 1) + 128 * il + ((ch ^ (il & 7)) << 4);
          *reinterpret_cast<uint4 *>(smem + OFF_PDS + off) = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
          *reinterpret_cast<uint4 *>(smem + OFF_PDS + 32768 + off) =
              make_uint4(dk[4 * cc], dk[4 * cc + 1], dk[4 * cc + 2], dk[4 * cc + 3]);
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_PDS));
      }
      // buffer (t + 1) & 1 was last read in tile t - 1, before this tile's barrier
      if (tid < 511) vec[512 * ((t + 1) & 1) + tid] = nv;
    }
    // ---- epilogue: lanes are keys; this thread takes 16 of the 64 columns ----
    good = good && warp_wait(BAR(B_PDSFREE), (iters - 1) & 1, abort_flag, status);
    const int j = j0 + il;
    if (good) {
      tc_fence_after();
      uint32_t rv[16], rk[16];
      tmem_ld16(tl + T_DV + 16 * qt, rv);
      tmem_ld16(tl + T_DK + 16 * qt, rk);
      tmem_wait_ld();
      if (j < L) {
        __nv_bfloat16 *dvp = (__nv_bfloat16 *)p.dv + ((size_t)bh * L + j) * HD + 16 * qt;
        __nv_bfloat16 *dkp = (__nv_bfloat16 *)p.dk + ((size_t)bh * L + j) * HD + 16 * qt;
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          uint4 wv, wk;
          wv.x = pack_bf16x2(u2f(rv[8 * c8 + 0]), u2f(rv[8 * c8 + 1]));
          wv.y = pack_bf16x2(u2f(rv[8 * c8 + 2]), u2f(rv[8 * c8 + 3]));
          wv.z = pack_bf16x2(u2f(rv[8 * c8 + 4]), u2f(rv[8 * c8 + 5]));
          wv.w = pack_bf16x2(u2f(rv[8 * c8 + 6]), u2f(rv[8 * c8 + 7]));
          wk.x = pack_bf16x2(p.scale * u2f(rk[8 * c8 + 0]), p.scale * u2f(rk[8 * c8 + 1]));
          wk.y = pack_bf16x2(p.scale * u2f(rk[8 * c8 + 2]), p.scale * u2f(rk[8 * c8 + 3]));
          wk.z = pack_bf16x2(p.scale * u2f(rk[8 * c8 + 4]), p.scale * u2f(rk[8 * c8 + 5]));
          wk.w = pack_bf16x2(p.scale * u2f(rk[8 * c8 + 6]), p.scale * u2f(rk[8 * c8 + 7]));
          *reinterpret_cast<uint4 *>(dvp + 8 * c8) = wv;
          *reinterpret_cast<uint4 *>(dkp + 8 * c8) = wk;
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ============================================================================
// query-tile kernel: dQ and the per-query-tile partial of the bias gradient
// ============================================================================
namespace qb {
constexpr int OFF_Q = 0, OFF_DO = 16384, OFF_K = 32768, OFF_V = OFF_K + 32768;
constexpr int OFF_T = OFF_V + 32768;     // band tiles: fp32 dS, 128 rows x 132 (also the epilogue's scratch)
// T5 band tiles: per-bucket dS sums of this query tile (NB_MAX floats), then each warp's
// carry (the sum of its last run of equal buckets, that bucket, and its first bucket)
constexpr int OFF_G = OFF_T + 128 * ROT_LD * 4;
constexpr int OFF_GC = OFF_G + 4 * NB_MAX;
constexpr int OFF_VEC = OFF_GC + 3 * 4 * 8;      // bias window, double-buffered (2 x 256)
constexpr int OFF_BAR = OFF_VEC + 2048;
constexpr int SMEM = OFF_BAR + 256 + 1024;
enum { B_QD = 0, B_ST0, B_ST1, B_SDP, B_SDPCONS, B_PDS, B_DSFREE, B_DRAIN, NB };
constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256, T_DS = 320;
}  // namespace qb

__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_bias_q_kernel(const __grid_constant__ BiasArgs A) {
  using namespace qb;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, m = p.nT - 1 - (int)blockIdx.x / BH, h = bh % p.H;
  const int L = p.L, i0 = m * 128;
  const int klen = key_len(p, bh / p.H);  // keys j >= klen of this batch are masked; their tiles skipped
  const int nTiles = min(p.causal ? m + 1 : p.nT, (klen + 127) / 128);
  float *part = A.part + ((size_t)bh * p.nT + m) * p.nb;
  if (nTiles == 0) {  // no key at all: dQ = 0 and a zero partial (whole CTA, before any barrier)
    for (int x = tid; x < 128 * (HD / 8); x += NTHREADS) {
      const int r = x / (HD / 8), c8 = x % (HD / 8);
      if (i0 + r < L)
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dq + ((size_t)bh * L + i0 + r) * HD + 8 * c8) = make_uint4(0, 0, 0, 0);
    }
    if (tid < p.nb) part[tid] = 0.f;
    return;
  }
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NB + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NB);
  float *T = (float *)(smem + OFF_T);
  float *G = (float *)(smem + OFF_G);  // dt partial per bucket
  float *gc = (float *)(smem + OFF_GC);
  int *gcb = (int *)(smem + OFF_GC + 32), *gfb = (int *)(smem + OFF_GC + 64);
  float *vec = (float *)(smem + OFF_VEC);
  int32_t *status = p.status;
  const float c1 = p.scale * LOG2E;

  if (tid == 0) {
    for (int k = 0; k < NB; ++k) mbar_init(BAR(k), (k == B_SDPCONS || k == B_PDS) ? NSOFT : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int x = tid; x < NB_MAX; x += NTHREADS) G[x] = 0.f;
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == CTRL_WARP) {
    if (lane == 0) {
      Ctl ctl;
      ctl.np = 0;
      ctl.ab = abort_flag;
      ctl.st = status;
      prefetch_tmap(&A.mq);
      prefetch_tmap(&A.mk);
      prefetch_tmap(&A.mv);
      prefetch_tmap(&A.mdo);
      const uint32_t idS = idesc_bf16(128, 128, false);
      const uint32_t idDQ = idesc_bf16(128, 64, true);
      ctl.expect(BAR(B_QD), 0, 32768u);
      tma_load_3d(sbase + OFF_Q, &A.mq, BAR(B_QD), 0, i0, bh);
      tma_load_3d(sbase + OFF_DO, &A.mdo, BAR(B_QD), 0, i0, bh);
      auto issue_stage = [&](int n) {
        const int st = n & 1;
        ctl.expect(BAR(B_ST0 + st), (uint32_t)((n >> 1) & 1), 32768u);
        tma_load_3d(sbase + OFF_K + 16384 * st, &A.mk, BAR(B_ST0 + st), 0, n * 128, bh);
        tma_load_3d(sbase + OFF_V + 16384 * st, &A.mv, BAR(B_ST0 + st), 0, n * 128, bh);
      };
      auto issue_sdp = [&](int n) {
        const int st = n & 1;
        umma_k64(tbase + T_S, sbase + OFF_Q, sbase + OFF_K + 16384 * st, idS, false);
        umma_k64(tbase + T_DP, sbase + OFF_DO, sbase + OFF_V + 16384 * st, idS, false);
        umma_commit(BAR(B_SDP));
      };
      issue_stage(0);
      if (nTiles > 1) issue_stage(1);
      bool ok = ctl.wait_load(BAR(B_QD), 0) && ctl.wait_load(BAR(B_ST0), 0);
      if (ok) {
        tc_fence_after();
        issue_sdp(0);
      }
      for (int n = 0; ok && n < nTiles; ++n) {
        const int st = n & 1;
        if (n + 1 < nTiles) {  // S / dP(n) read by the rows
          if (!ctl.wait(BAR(B_SDPCONS), n & 1)) break;
          if (!ctl.wait_load(BAR(B_ST0 + (st ^ 1)), ((n + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_sdp(n + 1);
        }
        if (!ctl.wait(BAR(B_PDS), n & 1)) break;
        tc_fence_after();
        // dQ += dS K_n (dS from TMEM)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_bf16_ts(tbase + T_DQ, tbase + T_DS + 8 * k, sdesc_sw128(sbase + OFF_K + 16384 * st + 2048 * k, 16, 1024), idDQ,
                       (n > 0 || k > 0) ? 1u : 0u);
        umma_commit(BAR(B_DSFREE));
        if (n + 2 < nTiles) {  // K_n, V_n free once dS K_n is done
          if (!ctl.wait(BAR(B_DSFREE), n & 1)) break;
          issue_stage(n + 2);
        }
      }
      ctl.drain(BAR(B_DRAIN));
    }
    __syncwarp();
  } else {
    const int g = warp & 3, qt = warp >> 2, il = 32 * g + lane, cb = NC * qt;
    const int i = i0 + il;
    const uint32_t tl = tbase + ((uint32_t)(g * 32) << 16);
    const float lse2 = lse2_of(p, bh, i);
    const float Dv = (i < L) ? p.Dvec[(size_t)bh * L + i] : 0.f;
    const uint64_t c12 = f2(c1, c1), nlse = f2(-lse2, -lse2), nDv = f2(-Dv, -Dv);
    bool good = true;
    float sL = 0.f, sR = 0.f;  // T5: dS of flat tiles left / right of the diagonal
    float wsum = 0.f;          // ALiBi: sum of dS_ij |j - i|
    float nva = (tid < 255) ? window_at(p, h, m, 0, tid) : 0.f;
    for (int n = 0; n < nTiles; ++n) {
      const int j0 = n * 128;
      float *tv = vec + 256 * (n & 1);
      if (tid < 255) tv[tid] = nva;  // buffer n & 1 was last read in tile n - 2
      if (tid < 255 && n + 1 < nTiles) nva = window_at(p, h, m, n + 1, tid);
      named_bar_sync(1, NSOFT);
      const bool flat = flat_tile(A, m, n);
      good = good && warp_wait(BAR(B_SDP), n & 1, abort_flag, status);
      const bool need_mask = (p.causal && n == m) || (j0 + 128 > klen);
      const int d0 = j0 + cb - i;  // offset j - i of this thread's first key
      float x[NC];
      if (good) {
        tc_fence_after();
        const float rflat = tv[127];
        const float *wrow = tv + 127 - il + cb;
        auto pds = [&](auto masked, auto banded) {
#pragma unroll
          for (int hq = 0; hq < NC / 16; ++hq) {
            uint32_t rs[16], rp[16];
            tmem_ld16(tl + T_S + cb + 16 * hq, rs);
            tmem_ld16(tl + T_DP + cb + 16 * hq, rp);
            tmem_wait_ld();
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const int x0 = 16 * hq + 4 * c4;
              float R[4], y[4], pr[4], dd[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) R[e] = decltype(banded)::value ? wrow[x0 + e] : rflat;
              score_bias4(rs + 4 * c4, R, c12, nlse, y);
              if constexpr (decltype(masked)::value) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int j = j0 + cb + x0 + e;
                  if (j >= klen || (p.causal && j > i)) y[e] = -INFINITY;
                }
              }
#pragma unroll
              for (int e = 0; e < 4; ++e) pr[e] = ex2(y[e]);
              ds_pairs(pr, rp + 4 * c4, nDv, dd);
#pragma unroll
              for (int e = 0; e < 4; ++e) x[x0 + e] = dd[e];
            }
          }
        };
        if (!flat) {
          if (need_mask) pds(std::true_type{}, std::true_type{}); else pds(std::false_type{}, std::true_type{});
        } else {
          if (need_mask) pds(std::true_type{}, std::false_type{}); else pds(std::false_type{}, std::false_type{});
        }
        tc_fence_before();
        mbar_arrive(BAR(B_SDPCONS));
      } else {
#pragma unroll
        for (int e = 0; e < NC; ++e) x[e] = 0.f;
      }
      // ---- bias gradient of this tile ----
      if (p.alibi) {
        const float fd0 = (float)d0;
#pragma unroll
        for (int e = 0; e < NC; ++e) wsum = fmaf(x[e], fabsf(fd0 + (float)e), wsum);
      } else if (flat) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < NC; ++e) s += x[e];
        if (n < m) sL += s; else sR += s;
      }
      // ---- dS -> TMEM for dQ += dS K ----
      if (good) {
        uint32_t pk[NC / 2];
#pragma unroll
        for (int k = 0; k < NC / 2; ++k) pk[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
        // the previous tile's dS K MMAs read T_DS: wait for them (long done in practice)
        if (n >= 1 && !warp_wait(BAR(B_DSFREE), (n - 1) & 1, abort_flag, status)) good = false;
        if (good) {
          tmem_st16(tl + T_DS + 16 * qt, pk);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(BAR(B_PDS));
        }
      }
      // ---- T5 band tile: per-offset sums of dS, diagonals added in a fixed order ----
      if (!p.alibi && !flat) {
#pragma unroll
        for (int c4 = 0; c4 < NC / 4; ++c4)
          *reinterpret_cast<float4 *>(T + il * ROT_LD + cb + 4 * c4) =
              make_float4(x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]);
        named_bar_sync(2, NSOFT);
        // warps 0-7: thread tid takes the offset j - i = 128 (n - m) - 127 + tid (tid 255: none)
        float s = 0.f;
        int b = -1;
        bool last = false;  // this thread ends its bucket's run of offsets
        if (tid < 256) {
          const int delta = 128 * (n - m) - 127 + tid;
          if (tid < 255 && delta > -L && delta < L) b = p.t5_bkt[delta + L - 1];
          if (tid < 255) {
            for (int r = 0; r < 128; ++r) {
              const int c = r + tid - 127;
              if (c >= 0 && c < 128) s += T[r * ROT_LD + c];
            }
          }
          // inclusive scan within runs of equal buckets over the warp's 32 offsets (the
          // bucket is monotone in |j - i| on each side, so a bucket's offsets are consecutive)
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, o);
            const int bb = __shfl_up_sync(0xffffffffu, b, o);
            if (lane >= o && bb == b) s += y;
          }
          const int bn = __shfl_down_sync(0xffffffffu, b, 1);
          last = lane != 31 && bn != b;
          if (lane == 31) {
            gc[warp] = s;
            gcb[warp] = b;
          }
          if (lane == 0) gfb[warp] = b;
        }
        named_bar_sync(2, NSOFT);
        if (tid < 256 && b >= 0) {
          if (lane == 31) last = warp == 7 || gfb[warp + 1] != b;
          if (last) {  // the run's parts in the warps before this one, nearest first
            for (int w = warp - 1; w >= 0 && gfb[w + 1] == b && gcb[w] == b; --w) s += gc[w];
            G[b] += s;  // one thread per bucket per tile
          }
        }
      }
    }
    // ---- epilogue: dQ ----
    good = good && warp_wait(BAR(B_DSFREE), (nTiles - 1) & 1, abort_flag, status);  // every MMA done
    if (good) {
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tl + T_DQ + 16 * qt, r);
      tmem_wait_ld();
      if (i < L) {
        __nv_bfloat16 *dqp = (__nv_bfloat16 *)p.dq + ((size_t)bh * L + i) * HD + 16 * qt;
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          uint4 w;
          w.x = pack_bf16x2(p.scale * u2f(r[8 * c8 + 0]), p.scale * u2f(r[8 * c8 + 1]));
          w.y = pack_bf16x2(p.scale * u2f(r[8 * c8 + 2]), p.scale * u2f(r[8 * c8 + 3]));
          w.z = pack_bf16x2(p.scale * u2f(r[8 * c8 + 4]), p.scale * u2f(r[8 * c8 + 5]));
          w.w = pack_bf16x2(p.scale * u2f(r[8 * c8 + 6]), p.scale * u2f(r[8 * c8 + 7]));
          *reinterpret_cast<uint4 *>(dqp + 8 * c8) = w;
        }
      }
    }
    // ---- epilogue: this query tile's partial of dt / dm, in a fixed order ----
    // (T is free: its last readers passed the band barrier; the per-thread values go there)
    T[tid] = p.alibi ? wsum : sL;
    T[NSOFT + tid] = sR;
    named_bar_sync(1, NSOFT);
    if (warp < 2) {  // warp 0: sum of the first array, warp 1: of the second
      const float *src = T + NSOFT * warp;
      float s = 0.f;
      for (int r = 0; r < NSOFT / 32; ++r) s += src[32 * r + lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) T[2 * NSOFT + warp] = s;
    }
    named_bar_sync(1, NSOFT);
    if (p.alibi) {
      if (tid == 0) part[0] = -T[2 * NSOFT];  // dm = sum dS_ij (-|j - i|)
    } else {
      const float SL = T[2 * NSOFT], SR = T[2 * NSOFT + 1];
      const int bL = p.t5_bkt[0], bR = p.t5_bkt[2 * L - 2];  // buckets of the far offsets -(L - 1), L - 1
      if (tid < p.nb) part[tid] = G[tid] + (tid == bL ? SL : 0.f) + (tid == bR ? SR : 0.f);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// dt[h][b] (ALiBi: dm[h]) = sum over batches and query tiles of the partials, in a fixed
// order: one warp per output, lane l takes partials l, l + 32, ..., then a shuffle tree
__global__ void reduce_bias_kernel(Prm p, const float *part) {
  const int x = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (x >= p.H * p.nb) return;
  const int h = x / p.nb, b = x % p.nb, n = p.B * p.nT;
  float acc = 0.f;
  for (int t = lane; t < n; t += 32) {
    const int bb = t / p.nT, m = t % p.nT;
    acc += part[(((size_t)bb * p.H + h) * p.nT + m) * p.nb + b];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) p.drel0[x] = acc;
}

// Smallest a in [1, L - 1] from which every offset sign * a' (a' >= a) has the bias of
// offset sign * (L - 1) (the bucket is monotone in the distance on each side).
static int flat_from(const Prm &p, int sign) {
  if (p.L <= 1) return 1;
  const int target = t5_bucket(p, sign * (p.L - 1));
  int lo = 1, hi = p.L - 1;
  while (lo < hi) {
    const int mid = lo + (hi - lo) / 2;
    if (t5_bucket(p, sign * mid) == target) hi = mid; else lo = mid + 1;
  }
  return lo;
}

static void band_setup(const Prm &p, BiasArgs &a) {
  if (p.alibi) {  // ALiBi: no two offsets share a bias value, no flat tile
    a.flat_pos = a.flat_neg = INT_MAX / 4;
    return;
  }
  a.flat_pos = flat_from(p, 1);
  a.flat_neg = flat_from(p, -1);
}

}  // namespace tcbias

bool tc_make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t planes, uint32_t box_rows);

bool tc_bwd_bias_supported(const Prm &p) { return p.mech == M_T5 && p.nb <= tcbias::NB_MAX; }

cudaError_t tc_bwd_bias(const Prm &p0, cudaStream_t st) {
  using namespace tcbias;
  BiasArgs a;
  memset(&a, 0, sizeof(a));
  a.p = p0;
  a.p.nT = (p0.L + 127) / 128;
  a.part = p0.part_small;
  band_setup(p0, a);
  const uint64_t BH = (uint64_t)p0.B * p0.H;
  if (!(tc_make_map(&a.mq, p0.q, p0.L, BH, 128) && tc_make_map(&a.mk, p0.k, p0.L, BH, 128) &&
        tc_make_map(&a.mv, p0.v, p0.L, BH, 128) && tc_make_map(&a.mdo, p0.dout, p0.L, BH, 128)))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(tc_bwd_bias_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kvb::SMEM)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(tc_bwd_bias_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, qb::SMEM)) != cudaSuccess)
    return e;
  const unsigned tiles = (unsigned)(a.p.nT * BH);
  RP_TRACED("tc_bwd_bias_kv_kernel", st, tc_bwd_bias_kv_kernel<<<tiles, NTHREADS, kvb::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("tc_bwd_bias_q_kernel", st, tc_bwd_bias_q_kernel<<<tiles, NTHREADS, qb::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("reduce_bias_kernel", st, reduce_bias_kernel<<<(unsigned)((p0.H * p0.nb + 7) / 8), 256, 0, st>>>(a.p, a.part));
  return cudaGetLastError();
}

}  // namespace rp
