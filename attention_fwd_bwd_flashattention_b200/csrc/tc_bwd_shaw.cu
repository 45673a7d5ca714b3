// Tensor-core (tcgen05 / TMEM / TMA) backward pass of Shaw relative attention,
// bf16, d = 64, clip c <= 64, sm_100a.  No atomics.
//
// S_ij = s (q_i.k_j + q_i.a_rho) with rho = clip(j - i, -c, c) + c, a table of
// 2c + 1 rows per head ("Fast and Exact Relative-Position Attention via
// Structure-Aware Kernels", Abstract; Shaw's content-position term).  The per-row
// products QA[i][rho] = q_i.a_rho come from a preparation kernel (rows of 132 fp32,
// zero past rho = 2c).  Offset-aware tiling (Abstract, technique (1)): a 128 x 128 tile
// (query tile m, key tile n) holds offsets j - i = 128 (n - m) + [-127, 127]; it is a
// "band" tile when some of them are unclipped (128 |m - n| - 127 < c), and every
// other tile sees a single clipped table row (rho = 0 left of the queries, 2c right).
//
//   key-tile kernel   (one CTA per key tile, query tiles streamed): recomputes P and
//                     dS (band tiles gather QA by offset from the QA tile, loaded by
//                     TMA into padded smem rows; other tiles add one per-row value),
//                     dV += P^T dO and dK += dS^T Q (Shaw has no key-side term).
//   query-tile kernel (one CTA per query tile, key tiles streamed): dQ += dS K (dS as
//                     the TMEM A operand); on band tiles E[i][rho] = dS_ij for the
//                     unclipped pairs (zero elsewhere) and dQ += E a, G += E^T Q on
//                     the tensor core; clipped pairs are summed per row (left / right
//                     end) and applied to a_0 / a_2c at the end.  The CTA writes its
//                     partial of da (offset-sharded gradient, technique (3)); a fixed-
//                     order reduction over query tiles finishes da.
//
// Shaw's value-side table aV (O_i += sum_j P_ij aV_rho, the VAL variants): dP_ij gains
// DA[i][rho] = dO_i . aV_rho (a second per-row product table, gathered like QA but
// read from L2: band tiles by offset, other tiles one end value per row), so both
// kernels form dS = P (dP + DA - D); the query-tile kernel also writes P in offset order
// (Pe, into the E tile once E's MMAs are done) on band tiles and accumulates
// GV += Pe^T dO in TMEM, the clipped pairs' probability mass per row going to the end
// rows aV_0 / aV_2c: one daV partial per query tile, reduced in a fixed order.
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_bwd_common.cuh"

namespace rp {
namespace tcs {

using namespace tc;
using namespace tcb;

constexpr int QA_LD = 132;  // fp32 per QA row (rho = 0..2c, zero padded); TMA rows of 528 bytes

struct ShawArgs {
  CUtensorMap mq, mk, mv, mdo, ma, mqa;
  Prm p;            // nT counts 128-row tiles
  const float *qa;  // [B,H,L][132]
  const float *da;  // value side: [B,H,L][132] per-row products dO_i . aV_rho
  float *part;      // [B,H,nT][rows][64] da partial per query tile
  float *part_v;    // value side: [B,H,nT][rows][64] daV partial per query tile
};

__device__ __forceinline__ bool band_tile(int c, int m, int n) {
  const int d = m > n ? m - n : n - m;
  return 128 * d - 127 < c;
}

// ---------------------------------------------------------------------------
// QA[b,h,i][rho] = q_i . a_rho (and, for the value side, DA[b,h,i][rho] = dO_i . aV_rho):
// X[b,h,i][rho] = x_i . T_rho for rows x [B,H,L,64] and a table T [H,rows,64], rho < 132
// (rows past the table give 0).  One CTA per 128 rows of one (b,h): TMA brings the x tile
// and the table (n = 2c + 1 rows rounded up to 16, rows past the table read as zeros), one
// tcgen05 MMA (M = 128, N = n, K = 64) leaves the products in TMEM (the same products the
// forward computes for its QA tile), and each of the four warps writes its 32 rows.
// ---------------------------------------------------------------------------
struct QaArgs {
  CUtensorMap mx, mt;  // rows x (128-row boxes), table T (n-row box)
  Prm p;               // nT counts 128-row tiles
  float *out;          // [B,H,L][QA_LD]
  int n;               // table rows multiplied (a multiple of 16, <= 144)
};
namespace qat {
constexpr int OFF_X = 0, OFF_T = 16384;   // x tile 16 KB, table up to 144 x 128 B
constexpr int OFF_BAR = OFF_T + 144 * 128;
constexpr int SMEM = OFF_BAR + 64 + 1024;
}  // namespace qat
__global__ void __launch_bounds__(128, 1) shaw_qa_kernel(const __grid_constant__ QaArgs A) {
  using namespace qat;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, m = (int)blockIdx.x / BH, h = bh % p.H, i0 = m * 128;
  const uint32_t sbase = smem_u32(smem), bar = sbase + OFF_BAR;
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 20);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 16);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 8, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  if (tid == 0) {
    mbar_expect_tx(bar, 16384u + 128u * (uint32_t)A.n);
    tma_load_3d(sbase + OFF_X, &A.mx, bar, 0, i0, bh);
    tma_load_3d(sbase + OFF_T, &A.mt, bar, 0, 0, h);
    if (mbar_wait(bar, 0, abort_flag, p.status, RELPOS_ERR_TIMEOUT_DEV)) {
      tc_fence_after();
      umma_k64(tbase, sbase + OFF_X, sbase + OFF_T, idesc_bf16(128, A.n, false), false);
    } else {  // give the copies still in flight a bounded time to land before the CTA exits
      volatile int none = 0;
      mbar_wait(bar, 0, &none, p.status, RELPOS_ERR_TIMEOUT_DEV);
    }
    umma_commit(bar + 8);
  }
  __syncwarp();
  const bool good = warp_wait(bar + 8, 0, abort_flag, p.status) && !*abort_flag;
  const int i = i0 + 32 * warp + lane;
  if (good) {
    tc_fence_after();
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    float *out = A.out + ((size_t)bh * p.L + (i < p.L ? i : 0)) * QA_LD;
    for (int c0 = 0; c0 < QA_LD; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tl + c0, r);
      tmem_wait_ld();
      if (i < p.L) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int c = c0 + 4 * q;
          if (c < QA_LD)  // columns past the n multiplied (0 .. 3 of the last chunk) are zero
            *reinterpret_cast<float4 *>(out + c) =
                make_float4(c < A.n ? u2f(r[4 * q]) : 0.f, c + 1 < A.n ? u2f(r[4 * q + 1]) : 0.f,
                            c + 2 < A.n ? u2f(r[4 * q + 2]) : 0.f, c + 3 < A.n ? u2f(r[4 * q + 3]) : 0.f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

// log2-domain scores of four keys, y = (s + R) c1 - lse2, with the relation terms R
__device__ __forceinline__ void score4(const uint32_t *s, const float (&R)[4], uint64_t c12, uint64_t nlse, float (&y)[4]) {
  f2_split(fma2(add2(f2(u2f(s[0]), u2f(s[1])), f2(R[0], R[1])), c12, nlse), y[0], y[1]);
  f2_split(fma2(add2(f2(u2f(s[2]), u2f(s[3])), f2(R[2], R[3])), c12, nlse), y[2], y[3]);
}

// ============================================================================
// key-tile kernel: dK, dV
// ============================================================================
namespace kvs {
constexpr int OFF_K = 0, OFF_V = 16384, OFF_Q = 32768, OFF_DO = OFF_Q + 32768;
constexpr int OFF_ROT = OFF_DO + 32768;  // QA tile (128 x 132 fp32); P tile at +0, dS tile at +32768 after use
constexpr int OFF_VEC = OFF_ROT + 128 * QA_LD * 4;  // per tile, double-buffered: [lse2 | D | R_end] x 128
constexpr int OFF_BAR = OFF_VEC + 4096;
constexpr int SMEM = OFF_BAR + 256 + 1024;
enum { B_KV = 0, B_ST0, B_ST1, B_QA, B_SDP, B_SDPCONS, B_PDS, B_PDSFREE, B_DRAIN, NB };
constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 320;
}  // namespace kvs

// dS = P (dP + DA - D) for four keys (value side: DA the dO . aV terms), nDv = (-D, -D)
__device__ __forceinline__ void ds_pairs_da(const float (&pr)[4], const uint32_t *dp, const float *da, uint64_t nDv,
                                            float (&dd)[4]) {
  f2_split(mul2(f2(pr[0], pr[1]), add2(add2(f2(u2f(dp[0]), u2f(dp[1])), f2(da[0], da[1])), nDv)), dd[0], dd[1]);
  f2_split(mul2(f2(pr[2], pr[3]), add2(add2(f2(u2f(dp[2]), u2f(dp[3])), f2(da[2], da[3])), nDv)), dd[2], dd[3]);
}

template <bool VAL>
__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_shaw_kv_kernel(const __grid_constant__ ShawArgs A) {
  using namespace kvs;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, n = (int)blockIdx.x / BH;
  const int L = p.L, j0 = n * 128, cl = p.clip;
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
  float *rot = (float *)(smem + OFF_ROT);
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
      prefetch_tmap(&A.mqa);
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
      int qa_cnt = 0;  // band tiles whose QA tile was requested
      auto issue_qa = [&](int t) {
        // the rows wait for each QA tile; retire the previous one here (its phase is
        // complete by now) so that the exit drain only ever sees the latest
        if (qa_cnt > 0 && !ctl.wait_load(BAR(B_QA), (uint32_t)((qa_cnt - 1) & 1))) return;
        ctl.expect(BAR(B_QA), (uint32_t)(qa_cnt & 1), 128u * QA_LD * 4u);
        tma_load_3d(sbase + OFF_ROT, &A.mqa, BAR(B_QA), 0, (mStart + t) * 128, bh);
        ++qa_cnt;
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
          umma_bf16(tbase + T_DV, sdesc_sw128(sbase + OFF_ROT + 2048 * k, 16384, 1024),
                    sdesc_sw128(sbase + OFF_DO + 16384 * st + 2048 * k, 16, 1024), idAcc, acc);
          umma_bf16(tbase + T_DK, sdesc_sw128(sbase + OFF_ROT + 32768 + 2048 * k, 16384, 1024),
                    sdesc_sw128(sbase + OFF_Q + 16384 * st + 2048 * k, 16, 1024), idAcc, acc);
        }
        umma_commit(BAR(B_PDSFREE));
      };
      issue_stage(0);
      if (iters > 1) issue_stage(1);
      if (band_tile(cl, mStart, n)) issue_qa(0);
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
        const bool refill = t + 2 < iters, qa_next = t + 1 < iters && band_tile(cl, mStart + t + 1, n);
        if (refill || qa_next) {
          if (!ctl.wait(BAR(B_PDSFREE), t & 1)) break;  // Q / dO(t) and the P / dS tiles are free
          if (refill) issue_stage(t + 2);
          if (qa_next) issue_qa(t + 1);
        }
      }
      ctl.drain(BAR(B_DRAIN));
    }
    __syncwarp();
  } else {
    const int g = warp & 3, qt = warp >> 2, il = 32 * g + lane, cb = NC * qt;
    const uint32_t tl = tbase + ((uint32_t)(g * 32) << 16);
    const float *rrow = rot + il * QA_LD;
    bool good = true;
    int qa_cnt = 0;
    // per-tile row terms staged through smem one tile ahead (one element per thread):
    // [lse2 of the rows | D of the rows | QA of the clipped end row the tile sees
    //  | value side: DA of that end row]
    constexpr int NV = VAL ? 512 : 384;
    auto fetch1 = [&](int t) {
      const int m = mStart + t, r = tid & 127, w = tid >> 7, i = m * 128 + r;
      if (i >= L) return w == 0 ? INFINITY : 0.f;
      if (w == 0) return lse2_of(p, bh, i);
      if (w == 1) return p.Dvec[(size_t)bh * L + i];
      return (w == 2 ? A.qa : A.da)[((size_t)bh * L + i) * QA_LD + (m > n ? 0 : 2 * cl)];
    };
    if (tid < NV) vec[tid] = fetch1(0);
    for (int t = 0; t < iters; ++t) {
      const int m = mStart + t, i = m * 128 + il;
      const float *tv = vec + NV * (t & 1);
      const float nv = (tid < NV && t + 1 < iters) ? fetch1(t + 1) : 0.f;
      named_bar_sync(1, NSOFT);
      const bool band = band_tile(cl, m, n);
      // value side: row i of DA (dO_i . aV_rho), gathered by offset on band tiles; other tiles
      // take the row's end value
      const float *darow = (VAL && band && i < L) ? A.da + ((size_t)bh * L + i) * QA_LD + cl : nullptr;
      good = good && warp_wait(BAR(B_SDP), t & 1, abort_flag, status);
      if (band) {
        good = good && warp_wait(BAR(B_QA), qa_cnt & 1, abort_flag, status);
        ++qa_cnt;
      }
      uint32_t pk[NC / 2], dk[NC / 2];
      const bool need_mask = (p.causal && m == n) || (j0 + 128 > klen);
      const int d0 = j0 + cb - i;  // offset j - i of this thread's first key
      if (good) {
        tc_fence_after();
        const float lse2 = tv[il], Dv = tv[128 + il], rend = tv[256 + il];
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
              for (int e = 0; e < 4; ++e)
                R[e] = decltype(banded)::value ? rrow[iclamp(d0 + x0 + e, -cl, cl) + cl] : rend;
              score4(rs + 4 * c4, R, c12, nlse, y);
              if constexpr (decltype(masked)::value) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int j = j0 + cb + x0 + e;
                  if (j >= klen || (p.causal && j > i)) y[e] = -INFINITY;
                }
              }
#pragma unroll
              for (int e = 0; e < 4; ++e) pr[e] = ex2(y[e]);
              if constexpr (VAL) {
                float da4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) da4[e] = darow ? __ldg(darow + iclamp(d0 + x0 + e, -cl, cl)) : tv[384 + il];
                ds_pairs_da(pr, rp + 4 * c4, da4, nDv, dd);
              } else {
                ds_pairs(pr, rp + 4 * c4, nDv, dd);
              }
              pk[x0 / 2] = pack_bf16x2(pr[0], pr[1]);
              pk[x0 / 2 + 1] = pack_bf16x2(pr[2], pr[3]);
              dk[x0 / 2] = pack_bf16x2(dd[0], dd[1]);
              dk[x0 / 2 + 1] = pack_bf16x2(dd[2], dd[3]);
            }
          }
        };
        if (band) {
          if (need_mask) pds(std::true_type{}, std::true_type{}); else pds(std::false_type{}, std::true_type{});
        } else {
          if (need_mask) pds(std::true_type{}, std::false_type{}); else pds(std::false_type{}, std::false_type{});
        }
        tc_fence_before();
        mbar_arrive(BAR(B_SDPCONS));  // S / dP read: the next tile's products may overwrite them
      }
      named_bar_sync(1, NSOFT);  // every QA row read; the P / dS tiles overwrite them
      // ... once the previous tile's dV / dK MMAs have read its P / dS tiles
      if (t >= 1) good = good && warp_wait(BAR(B_PDSFREE), (t - 1) & 1, abort_flag, status);
      if (good) {
#pragma unroll
        for (int cc = 0; cc < NC / 8; ++cc) {
          const int ch = (NC / 8) * (qt & 1) + cc;
          const uint32_t off = 16384 * (qt >> 1) + 128 * il + ((ch ^ (il & 7)) << 4);
          *reinterpret_cast<uint4 *>(smem + OFF_ROT + off) = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
          *reinterpret_cast<uint4 *>(smem + OFF_ROT + 32768 + off) =
              make_uint4(dk[4 * cc], dk[4 * cc + 1], dk[4 * cc + 2], dk[4 * cc + 3]);
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_PDS));
      }
      if (tid < NV) vec[NV * ((t + 1) & 1) + tid] = nv;  // tile t - 1's terms were read before this tile's first barrier
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
// query-tile kernel: dQ and the per-query-tile da partial
// ============================================================================
namespace qs {
constexpr int OFF_Q = 0, OFF_DO = 16384, OFF_K = 32768, OFF_V = OFF_K + 32768;
constexpr int OFF_A = OFF_V + 32768;     // table rows 0..127 (B operand of E a)
constexpr int OFF_E = OFF_A + 16384;     // E tile, 128 x 128 bf16 (K-major, two 64-column halves)
constexpr int OFF_ROT = OFF_E + 32768;   // the CTA's QA rows, 128 x 132 fp32
constexpr int OFF_VEC = OFF_ROT + 128 * QA_LD * 4;  // clipped-sum exchange [2][4][128]
constexpr int OFF_BAR = OFF_VEC + 4096;
constexpr int SMEM = OFF_BAR + 256 + 1024;
// B_PEFULL / B_PEFREE (value side): Pe written into the E tile / GV MMAs done with it
enum { B_QD = 0, B_ST0, B_ST1, B_SDP, B_SDPCONS, B_PDS, B_EFREE, B_DSFREE, B_DRAIN, B_PEFULL, B_PEFREE, NB };
constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256, T_DS = 320, T_G = 384, T_GV = 448;
}  // namespace qs

// dS of this thread's NC keys into the offset-order tile E (row il): column
// (delta + c) & 127 for delta = j - i; unclipped pairs give their value, clipped
// ones 0 (the row's 128 keys hit every column once).  pk[k] = (v[2k], v[2k+1]) with v
// the masked values; C0 = column of v[0].  Aligned bf16 pairs; when C0 is odd the
// first and last value pair with a neighbouring thread's and are written alone.
__device__ __forceinline__ uint32_t Es_off(uint32_t t, uint32_t rowb, uint32_t r7) {  // t = 2 col, col even
  return ((t << 7) & 0x4000u) + rowb + ((t & 126u) ^ r7);
}
__device__ __forceinline__ void store_Es(uint8_t *E, int il, uint32_t C0, const uint32_t (&pk)[NC / 2]) {
  const bool odd = (C0 & 1u) != 0;
  const uint32_t rowb = 128u * (uint32_t)il, r7 = (uint32_t)(il & 7) << 4;
  const uint32_t sel = odd ? 0x5432u : 0x3210u;  // odd: (high half of pk[k], low half of pk[k+1])
  const uint32_t B0 = (C0 + (odd ? 1u : 0u)) & 127u;
#pragma unroll
  for (int k = 0; k < NC / 2 - 1; ++k) {
    const uint32_t col = (B0 + 2u * k) & 127u;
    *reinterpret_cast<uint32_t *>(E + Es_off(2u * col, rowb, r7)) = prmt(pk[k], pk[k + 1], sel);
  }
  if (!odd) {
    const uint32_t col = (B0 + 2u * (NC / 2 - 1)) & 127u;
    *reinterpret_cast<uint32_t *>(E + Es_off(2u * col, rowb, r7)) = pk[NC / 2 - 1];
  } else {
    const uint32_t c0 = (C0 - 1u) & 127u, c31 = (C0 + NC - 1) & 127u;  // high half of c0's pair, low half of c31's
    *reinterpret_cast<uint16_t *>(E + Es_off(2u * c0, rowb, r7) + 2u) = (uint16_t)(pk[0] & 0xFFFFu);
    *reinterpret_cast<uint16_t *>(E + Es_off(2u * c31, rowb, r7)) = (uint16_t)(pk[NC / 2 - 1] >> 16);
  }
}

template <bool VAL>
__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_shaw_q_kernel(const __grid_constant__ ShawArgs A) {
  using namespace qs;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, m = p.nT - 1 - (int)blockIdx.x / BH, h = bh % p.H;
  const int L = p.L, i0 = m * 128, cl = p.clip;
  const int klen = key_len(p, bh / p.H);  // keys j >= klen of this batch are masked; their tiles skipped
  const int nTiles = min(p.causal ? m + 1 : p.nT, (klen + 127) / 128);
  if (nTiles == 0) {  // no key at all: dQ = 0 and a zero da partial (whole CTA, before any barrier)
    for (int x = tid; x < 128 * (HD / 8); x += NTHREADS) {
      const int r = x / (HD / 8), c8 = x % (HD / 8);
      if (i0 + r < L)
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dq + ((size_t)bh * L + i0 + r) * HD + 8 * c8) = make_uint4(0, 0, 0, 0);
    }
    float *part = A.part + ((size_t)bh * p.nT + m) * (size_t)p.nrows * HD;
    for (int x = tid; x < p.nrows * HD; x += NTHREADS) part[x] = 0.f;
    if (VAL) {
      float *pv = A.part_v + ((size_t)bh * p.nT + m) * (size_t)p.nrows * HD;
      for (int x = tid; x < p.nrows * HD; x += NTHREADS) pv[x] = 0.f;
    }
    return;
  }
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NB + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NB);
  const float *rot = (const float *)(smem + OFF_ROT);
  float *vec = (float *)(smem + OFF_VEC);
  int32_t *status = p.status;
  const float c1 = p.scale * LOG2E;

  if (tid == 0) {
    for (int k = 0; k < NB; ++k) mbar_init(BAR(k), (k == B_SDPCONS || k == B_PDS || k == B_PEFULL) ? NSOFT : 1);
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
      prefetch_tmap(&A.ma);
      prefetch_tmap(&A.mqa);
      const uint32_t idS = idesc_bf16(128, 128, false);
      const uint32_t idDQ = idesc_bf16(128, 64, true);
      const uint32_t idG = idesc_bf16(128, 64, true, true);
      ctl.expect(BAR(B_QD), 0, 16384u * 3u + 128u * QA_LD * 4u);
      tma_load_3d(sbase + OFF_Q, &A.mq, BAR(B_QD), 0, i0, bh);
      tma_load_3d(sbase + OFF_DO, &A.mdo, BAR(B_QD), 0, i0, bh);
      tma_load_3d(sbase + OFF_A, &A.ma, BAR(B_QD), 0, 0, h);
      tma_load_3d(sbase + OFF_ROT, &A.mqa, BAR(B_QD), 0, i0, bh);
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
      int nband = 0;
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
        const bool bt = band_tile(cl, m, n);
        if (bt) {  // dQ += E a, G += E^T Q (E in smem)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            umma_bf16(tbase + T_DQ, sdesc_sw128(sbase + OFF_E + 16384 * (k >> 2) + 32 * (k & 3), 16, 1024),
                      sdesc_sw128(sbase + OFF_A + 2048 * k, 16, 1024), idDQ, (n > 0 || k > 0) ? 1u : 0u);
            umma_bf16(tbase + T_G, sdesc_sw128(sbase + OFF_E + 2048 * k, 16384, 1024),
                      sdesc_sw128(sbase + OFF_Q + 2048 * k, 16, 1024), idG, (nband > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(BAR(B_EFREE));
        }
        // dQ += dS K_n (dS from TMEM)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_bf16_ts(tbase + T_DQ, tbase + T_DS + 8 * k, sdesc_sw128(sbase + OFF_K + 16384 * st + 2048 * k, 16, 1024), idDQ,
                       (n > 0 || k > 0 || bt) ? 1u : 0u);
        umma_commit(BAR(B_DSFREE));
        if (VAL && bt) {  // GV += Pe^T dO, Pe written by the rows into the E tile once E's MMAs were done
          if (!ctl.wait(BAR(B_PEFULL), nband & 1)) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_bf16(tbase + T_GV, sdesc_sw128(sbase + OFF_E + 2048 * k, 16384, 1024),
                      sdesc_sw128(sbase + OFF_DO + 2048 * k, 16, 1024), idG, (nband > 0 || k > 0) ? 1u : 0u);
          umma_commit(BAR(B_PEFREE));
        }
        if (bt) ++nband;
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
    const float *rrow = rot + il * QA_LD;
    const float lse2 = lse2_of(p, bh, i);
    const float Dv = (i < L) ? p.Dvec[(size_t)bh * L + i] : 0.f;
    const uint64_t c12 = f2(c1, c1), nlse = f2(-lse2, -lse2), nDv = f2(-Dv, -Dv);
    bool good = warp_wait(BAR(B_QD), 0, abort_flag, status);
    float rsL = 0.f, rsR = 0.f;  // dS of clipped pairs, left (rho = 0) / right (rho = 2c)
    float psL = 0.f, psR = 0.f;  // value side: P of the clipped pairs, left / right
    // value side: row i of DA (dO_i . aV_rho), its end values and a pointer to the rest
    const float *darow = (VAL && i < L) ? A.da + ((size_t)bh * L + i) * QA_LD + cl : nullptr;
    const float daL = darow ? darow[-cl] : 0.f, daR = darow ? darow[cl] : 0.f;
    int nband = 0;
    for (int n = 0; n < nTiles; ++n) {
      const int j0 = n * 128;
      const bool band = band_tile(cl, m, n);
      const int d0 = j0 + cb - i;  // offset j - i of this thread's first key
      // clipped pairs: keys with j - i <= -c (left) or >= c (right); unclipped ones go to E
      const int eLo = max(0, 1 - cl - d0), eHi = min(NC - 1, cl - 1 - d0);  // unclipped: eLo..eHi
      const float dend = m > n ? daL : daR;  // value side: dO_i . aV of the row's clipped end
      uint32_t ppk[VAL ? NC / 2 : 1];  // value side, band tiles: P of the unclipped pairs (Pe), bf16 pairs
      good = good && warp_wait(BAR(B_SDP), n & 1, abort_flag, status);
      const bool need_mask = (p.causal && n == m) || (j0 + 128 > klen);
      float x[NC];
      if (good) {
        tc_fence_after();
        const float rend = band ? 0.f : rrow[m > n ? 0 : 2 * cl];
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
              for (int e = 0; e < 4; ++e)
                R[e] = decltype(banded)::value ? rrow[iclamp(d0 + x0 + e, -cl, cl) + cl] : rend;
              score4(rs + 4 * c4, R, c12, nlse, y);
              if constexpr (decltype(masked)::value) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int j = j0 + cb + x0 + e;
                  if (j >= klen || (p.causal && j > i)) y[e] = -INFINITY;
                }
              }
#pragma unroll
              for (int e = 0; e < 4; ++e) pr[e] = ex2(y[e]);
              if constexpr (VAL) {
                // dO_i . aV of the four keys: band tiles gather row i of DA by offset (L1 / L2)
                float da4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  da4[e] = (decltype(banded)::value && darow) ? __ldg(darow + iclamp(d0 + x0 + e, -cl, cl)) : dend;
                ds_pairs_da(pr, rp + 4 * c4, da4, nDv, dd);
                float pe[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int ee = x0 + e;
                  if (ee < eLo) psL += pr[e];
                  else if (ee > eHi) psR += pr[e];
                  pe[e] = (ee >= eLo && ee <= eHi) ? pr[e] : 0.f;
                }
                if constexpr (decltype(banded)::value) {
                  ppk[x0 / 2] = pack_bf16x2(pe[0], pe[1]);
                  ppk[x0 / 2 + 1] = pack_bf16x2(pe[2], pe[3]);
                }
              } else {
                ds_pairs(pr, rp + 4 * c4, nDv, dd);
              }
#pragma unroll
              for (int e = 0; e < 4; ++e) x[x0 + e] = dd[e];
            }
          }
        };
        if (band) {
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
#pragma unroll
      for (int e = 0; e < NC; ++e) {
        if (e < eLo) rsL += x[e];
        else if (e > eHi) rsR += x[e];
      }
      if (good) {
        uint32_t pk[NC / 2];
#pragma unroll
        for (int k = 0; k < NC / 2; ++k) pk[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
        // the previous tile's dS K MMAs read T_DS: wait for them (long done in practice)
        if (n >= 1 && !warp_wait(BAR(B_DSFREE), (n - 1) & 1, abort_flag, status)) good = false;
        if (good) tmem_st16(tl + T_DS + 16 * qt, pk);
        if (good && band) {
          // the E tile's last reader of the previous band tile: its E MMAs (value side: its GV MMAs)
          if (nband >= 1 && !warp_wait(BAR(VAL ? B_PEFREE : B_EFREE), (nband - 1) & 1, abort_flag, status)) good = false;
#pragma unroll
          for (int k = 0; k < NC / 2; ++k) {
            const float v0 = (2 * k >= eLo && 2 * k <= eHi) ? x[2 * k] : 0.f;
            const float v1 = (2 * k + 1 >= eLo && 2 * k + 1 <= eHi) ? x[2 * k + 1] : 0.f;
            pk[k] = pack_bf16x2(v0, v1);
          }
          if (good) store_Es(smem + OFF_E, il, (uint32_t)(d0 + cl) & 127u, pk);
        }
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_PDS));
        if constexpr (VAL) {
          if (band) {  // Pe into the E tile once this tile's E MMAs are done
            if (!warp_wait(BAR(B_EFREE), nband & 1, abort_flag, status)) good = false;
            if (good) {
              store_Es(smem + OFF_E, il, (uint32_t)(d0 + cl) & 127u, ppk);
              fence_async_smem();
              tc_fence_before();
              mbar_arrive(BAR(B_PEFULL));
            }
          }
        }
        if (band) ++nband;
      }
    }
    // ---- epilogue ----
    // clipped sums of the row: the four threads' parts, added in a fixed order
    vec[qt * 128 + il] = rsL;
    vec[512 + qt * 128 + il] = rsR;
    named_bar_sync(1, NSOFT);
    const float sL = ((vec[il] + vec[128 + il]) + vec[256 + il]) + vec[384 + il];
    const float sR = ((vec[512 + il] + vec[640 + il]) + vec[768 + il]) + vec[896 + il];
    good = good && warp_wait(BAR(B_DSFREE), (nTiles - 1) & 1, abort_flag, status);  // every MMA done
    if (VAL && nband > 0) good = good && warp_wait(BAR(B_PEFREE), (nband - 1) & 1, abort_flag, status);  // and GV's
    const __nv_bfloat16 *a = (const __nv_bfloat16 *)p.rel0 + (size_t)h * p.nrows * HD;
    if (good) {
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tl + T_DQ + 16 * qt, r);
      tmem_wait_ld();
      if (i < L) {
        __nv_bfloat16 *dqp = (__nv_bfloat16 *)p.dq + ((size_t)bh * L + i) * HD + 16 * qt;
        const __nv_bfloat16 *a0 = a + 16 * qt, *a1 = a + (size_t)(2 * cl) * HD + 16 * qt;
        float v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          v[e] = p.scale * (u2f(r[e]) + sL * __bfloat162float(a0[e]) + sR * __bfloat162float(a1[e]));
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          uint4 w;
          w.x = pack_bf16x2(v[8 * c8 + 0], v[8 * c8 + 1]);
          w.y = pack_bf16x2(v[8 * c8 + 2], v[8 * c8 + 3]);
          w.z = pack_bf16x2(v[8 * c8 + 4], v[8 * c8 + 5]);
          w.w = pack_bf16x2(v[8 * c8 + 6], v[8 * c8 + 7]);
          *reinterpret_cast<uint4 *>(dqp + 8 * c8) = w;
        }
      }
      // da partial: rows 1..2c-1 from G (TMEM lane = rho); the end rows below
      float *part = A.part + ((size_t)bh * p.nT + m) * (size_t)p.nrows * HD;
      uint32_t gr[16];
      tmem_ld16(tl + T_G + 16 * qt, gr);
      tmem_wait_ld();
      const int rho = il;
      if (rho >= 1 && rho <= 2 * cl - 1) {
#pragma unroll
        for (int e = 0; e < 16; ++e) part[(size_t)rho * HD + 16 * qt + e] = (nband > 0) ? p.scale * u2f(gr[e]) : 0.f;
      }
      if (VAL) {  // daV partial: rows 1..2c-1 from GV (TMEM lane = rho)
        float *pv = A.part_v + ((size_t)bh * p.nT + m) * (size_t)p.nrows * HD;
        tmem_ld16(tl + T_GV + 16 * qt, gr);
        tmem_wait_ld();
        if (rho >= 1 && rho <= 2 * cl - 1) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pv[(size_t)rho * HD + 16 * qt + e] = (nband > 0) ? u2f(gr[e]) : 0.f;
        }
      }
    }
    named_bar_sync(1, NSOFT);
    vec[il] = sL;  // row sums for the end rows of da (one copy per row)
    vec[128 + il] = sR;
    named_bar_sync(1, NSOFT);
    if (tid < 2 * HD) {  // da[0][d] = s sum_i sL_i q_i[d], da[2c][d] = s sum_i sR_i q_i[d]
      const int d = tid & (HD - 1), side = tid >> 6;
      const __nv_bfloat16 *qp = (const __nv_bfloat16 *)p.q + ((size_t)bh * L + i0) * HD + d;
      float acc = 0.f;
      for (int rr = 0; rr < 128 && i0 + rr < L; ++rr) acc = fmaf(vec[128 * side + rr], __bfloat162float(qp[(size_t)rr * HD]), acc);
      float *part = A.part + ((size_t)bh * p.nT + m) * (size_t)p.nrows * HD;
      part[(size_t)(side ? 2 * cl : 0) * HD + d] = p.scale * acc;
    }
    if (VAL) {  // daV[0][d] = sum_i psL_i dO_i[d], daV[2c][d] = sum_i psR_i dO_i[d] (row sums in a fixed order)
      named_bar_sync(1, NSOFT);
      vec[qt * 128 + il] = psL;
      vec[512 + qt * 128 + il] = psR;
      named_bar_sync(1, NSOFT);
      const float pL = ((vec[il] + vec[128 + il]) + vec[256 + il]) + vec[384 + il];
      const float pR = ((vec[512 + il] + vec[640 + il]) + vec[768 + il]) + vec[896 + il];
      named_bar_sync(1, NSOFT);
      vec[il] = pL;
      vec[128 + il] = pR;
      named_bar_sync(1, NSOFT);
      if (tid < 2 * HD) {
        const int d = tid & (HD - 1), side = tid >> 6;
        const __nv_bfloat16 *gp = (const __nv_bfloat16 *)p.dout + ((size_t)bh * L + i0) * HD + d;
        float acc = 0.f;
        for (int rr = 0; rr < 128 && i0 + rr < L; ++rr) acc = fmaf(vec[128 * side + rr], __bfloat162float(gp[(size_t)rr * HD]), acc);
        float *pv = A.part_v + ((size_t)bh * p.nT + m) * (size_t)p.nrows * HD;
        pv[(size_t)(side ? 2 * cl : 0) * HD + d] = acc;
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

// da (daV) = sum over batches and query tiles of the partials, in a fixed order
__global__ void reduce_shaw_kernel(Prm p, const float *part, float *out) {
  const size_t per = (size_t)p.nrows * HD;
  const size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= (size_t)p.H * per) return;
  const int h = (int)(x / per);
  const size_t re = x % per;
  float acc = 0.f;
  for (int b = 0; b < p.B; ++b)
    for (int t = 0; t < p.nT; ++t) acc += part[(((size_t)b * p.H + h) * p.nT + t) * per + re];
  out[x] = acc;
}

}  // namespace tcs

bool tc_make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t planes, uint32_t box_rows);
bool tc_make_map_f32_rows(CUtensorMap *m, const void *base, uint32_t row_len, uint64_t rows, uint64_t planes,
                          uint32_t box_rows);

bool tc_bwd_shaw_supported(const Prm &p) { return p.clip >= 1 && p.clip <= 64; }

size_t tc_bwd_shaw_qa_floats(const Prm &p) { return (size_t)p.B * p.H * p.L * tcs::QA_LD; }

template <bool VAL>
static cudaError_t run_shaw_bwd(const tcs::ShawArgs &a, cudaStream_t st) {
  using namespace tcs;
  cudaError_t e;
  auto kkv = tc_bwd_shaw_kv_kernel<VAL>;
  auto kq = tc_bwd_shaw_q_kernel<VAL>;
  if ((e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, kvs::SMEM)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, qs::SMEM)) != cudaSuccess) return e;
  const unsigned tiles = (unsigned)(a.p.nT * a.p.B * a.p.H);
  RP_TRACED("tc_bwd_shaw_kv_kernel", st, kkv<<<tiles, NTHREADS, kvs::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("tc_bwd_shaw_q_kernel", st, kq<<<tiles, NTHREADS, qs::SMEM, st>>>(a));
  return cudaGetLastError();
}

cudaError_t tc_bwd_shaw(const Prm &p0, const TcWork &w, cudaStream_t st) {
  using namespace tcs;
  typedef __nv_bfloat16 bf;
  ShawArgs a;
  memset(&a, 0, sizeof(a));
  a.p = p0;
  a.p.nT = (p0.L + 127) / 128;
  a.qa = w.qa;
  a.part = p0.part_row;
  if (p0.shaw_v) {
    a.da = w.da;
    a.part_v = p0.part_val;
  }
  const uint64_t BH = (uint64_t)p0.B * p0.H;
  if (!(tc_make_map(&a.mq, p0.q, p0.L, BH, 128) && tc_make_map(&a.mk, p0.k, p0.L, BH, 128) &&
        tc_make_map(&a.mv, p0.v, p0.L, BH, 128) && tc_make_map(&a.mdo, p0.dout, p0.L, BH, 128) &&
        tc_make_map(&a.ma, p0.rel0, p0.nrows, p0.H, 128) &&
        tc_make_map_f32_rows(&a.mqa, w.qa, QA_LD, p0.L, BH, 128)))
    return cudaErrorInvalidValue;
  cudaError_t e;
  const unsigned qa_blocks = (unsigned)(BH * a.p.nT);
  QaArgs qa;
  memset(&qa, 0, sizeof(qa));
  qa.p = a.p;
  qa.n = (2 * p0.clip + 1 + 15) / 16 * 16;
  qa.out = w.qa;
  qa.mx = a.mq;
  if (!tc_make_map(&qa.mt, p0.rel0, p0.nrows, p0.H, (uint32_t)qa.n)) return cudaErrorInvalidValue;
  if ((e = cudaFuncSetAttribute(shaw_qa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, qat::SMEM)) != cudaSuccess)
    return e;
  RP_TRACED("shaw_qa_kernel", st, shaw_qa_kernel<<<qa_blocks, 128, qat::SMEM, st>>>(qa));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p0.shaw_v) {  // DA = dO aV^T by row, for the value side
    qa.out = w.da;
    qa.mx = a.mdo;
    if (!tc_make_map(&qa.mt, p0.rel1, p0.nrows, p0.H, (uint32_t)qa.n)) return cudaErrorInvalidValue;
    RP_TRACED("shaw_qa_kernel", st, shaw_qa_kernel<<<qa_blocks, 128, qat::SMEM, st>>>(qa));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = p0.shaw_v ? run_shaw_bwd<true>(a, st) : run_shaw_bwd<false>(a, st)) != cudaSuccess) return e;
  const size_t n = (size_t)p0.H * p0.nrows * HD;
  RP_TRACED("reduce_shaw_kernel", st, reduce_shaw_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.p, a.part, p0.drel0));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p0.shaw_v) {
    RP_TRACED("reduce_shaw_kernel", st,
              reduce_shaw_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a.p, a.part_v, p0.drel1));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace rp
