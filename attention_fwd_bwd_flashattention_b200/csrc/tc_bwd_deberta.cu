// Tensor-core (tcgen05 / TMEM / TMA) backward pass of DeBERTa disentangled
// attention, bf16, d = 64, any span k, sm_100a.  No atomics.
//
// S_ij = s (q_i.k_j + q_i.Kr[rho] + k_j.Qr[rho']) with rho = clip(i - j + k, 0, W - 1)
// and rho' = clip(j - i + k, 0, W - 1), W = 2k table rows (DeBERTa's content-to-
// position and position-to-content terms, the decomposable relative terms whose
// query- and key-relation products are computed once and reused: "Fast and Exact
// Relative-Position Attention via Structure-Aware Kernels", Abstract, technique (2)).
//
// The gradients of the relation terms factor through two offset-ordered copies of dS,
//   M[i][r] = sum over j with rho(i, j) = r of dS_ij,
//   N[j][r] = sum over i with rho'(i, j) = r of dS_ij,
// dq_i += s sum_r M[i][r] Kr_r,  dk_j += s sum_r N[j][r] Qr_r,  dKr = s M^T Q,
// dQr = s N^T K.  An interior entry (1 <= r <= W - 2) is the single pair j = i + k - r
// (resp. i = j + k - r); the end columns hold the sums of the clipped pairs.  A 128 x 128
// tile (query tile m, key tile n) is "far" when all its pairs are clipped on both terms
// (128 |m - n| - 127 >= k); only the band of tiles around the diagonal touches interior
// entries (offset-aware tiling, technique (1)).
//
//   tables kernel    QKr = Q Kr^T and KQr = K Qr^T, fp32 [B,H,L][Wp] (one MMA per 256
//                    table rows, 512 per CTA).
// Rows of QKr, KQr, M and N are Wp = W rounded up to 64 entries long (the K steps of the
// rows kernel); the tables are read from copies padded with zero rows to Wp, so the
// entries past W are zero in M and N and never reach a gradient.
//   key-tile kernel  recomputes P and dS (band tiles gather both relation products by
//                    offset, far tiles add the clipped end products), dV += P^T dO,
//                    dK += dS^T Q, the clipped column sums of dS (far tiles: dS^T 1 on
//                    the tensor core; band tiles: warp butterflies) and writes N.
//   query-tile kernel the same recompute, dQ += dS K (dS as the TMEM A operand), the
//                    clipped row sums, and writes M.
//   rows kernel      dq = s (dQ + M Kr), dk = s (dK + N Qr), one 128-row tile per CTA.
//   table kernel     M^T Q and N^T K per (head, 128 table rows, 1024 data rows); a
//                    fixed-order reduction of these partials gives dKr and dQr
//                    ("offset-based gradient sharding", technique (3)).
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_bwd_common.cuh"

namespace rp {
namespace tcdeb {

using namespace tc;
using namespace tcb;

constexpr int CH = 1024;  // data rows per table-kernel CTA

struct DebArgs {
  CUtensorMap mq, mk, mv, mdo;  // [B,H,L,64], 128-row boxes
  CUtensorMap mkr256, mqr256;   // tables, 256-row boxes (tables kernel)
  CUtensorMap mkr64, mqr64;     // tables, 64-row boxes (rows kernel)
  CUtensorMap mM, mN;           // [B,H,L][Wp] bf16, 64 x 128 boxes
  Prm p;                        // nT counts 128-row tiles
  const float *qkr, *kqr;       // [B,H,L][Wp] relation products
  __nv_bfloat16 *M, *N;         // [B,H,L][Wp] offset-ordered dS
  float *dqc, *dkc;             // [B,H,L,64] dS K and dS^T Q
  float *part;                  // [2][H][W/128][B*nch][128][64] table-gradient partials
  int W, Wp, nbs, nch;          // table rows, row length of QKr / KQr / M / N, band tiles per side, chunks per plane
};

__device__ __forceinline__ bool far_left(int m, int n, int k) { return 128 * (m - n) - 127 >= k; }
__device__ __forceinline__ bool far_right(int m, int n, int k) { return 128 * (n - m) - 127 >= k; }

constexpr int RLD = 129;  // fp32 stride of the band tile's relation terms in smem (conflict-free rows and columns)

// Relation terms of band tile (i0, j0) into R[il * RLD + jl] = QKr[i][rho] + KQr[j][rho']
// (0 outside the sequence).  Warp w loads rows il = 8w .. 8w + 7 of QKr, then keys
// jl = 8w .. 8w + 7 of KQr; every load is a coalesced run of one table row and all of
// a warp's 32 loads of a phase are independent.  Ends with R complete for every row thread.
__device__ __forceinline__ void band_fill(const DebArgs &A, int bh, int i0, int j0, float *R, int warp, int lane) {
  const Prm &p = A.p;
  const int L = p.L, W = A.W, Wp = A.Wp, k = p.span;
  float v[32];
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int i = i0 + 8 * warp + rr;
    const float *row = A.qkr + ((size_t)bh * L + (i < L ? i : 0)) * Wp;
#pragma unroll
    for (int q = 0; q < 4; ++q) v[4 * rr + q] = (i < L) ? row[iclamp(i - j0 - (lane + 32 * q) + k, 0, W - 1)] : 0.f;
  }
#pragma unroll
  for (int rr = 0; rr < 8; ++rr)
#pragma unroll
    for (int q = 0; q < 4; ++q) R[(8 * warp + rr) * RLD + lane + 32 * q] = v[4 * rr + q];
  named_bar_sync(2, NSOFT);
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int j = j0 + 8 * warp + rr;
    const float *row = A.kqr + ((size_t)bh * L + (j < L ? j : 0)) * Wp;
#pragma unroll
    for (int q = 0; q < 4; ++q) v[4 * rr + q] = (j < L) ? row[iclamp(j - (i0 + lane + 32 * q) + k, 0, W - 1)] : 0.f;
  }
#pragma unroll
  for (int rr = 0; rr < 8; ++rr)
#pragma unroll
    for (int q = 0; q < 4; ++q) R[(lane + 32 * q) * RLD + 8 * warp + rr] += v[4 * rr + q];
  named_bar_sync(2, NSOFT);
}

// log2-domain scores y = (s_raw + R) c1 - lse2 of four keys
__device__ __forceinline__ void score_rel4(const uint32_t *s, const float (&R)[4], uint64_t c12, uint64_t nlse, float (&y)[4]) {
  f2_split(fma2(add2(f2(u2f(s[0]), u2f(s[1])), f2(R[0], R[1])), c12, nlse), y[0], y[1]);
  f2_split(fma2(add2(f2(u2f(s[2]), u2f(s[3])), f2(R[2], R[3])), c12, nlse), y[2], y[3]);
}

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Column sums over the warp's 32 rows: on entry v[c] is this lane's value of column c;
// on exit v[0] is the sum of column `lane` over the 32 lanes (31 shuffles, fixed order).
__device__ __forceinline__ float warp_colsum32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int e = 0; e < w; ++e) {
      const float send = up ? v[e] : v[e + w];
      const float keep = up ? v[e + w] : v[e];
      v[e] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

// ============================================================================
// tables kernel: QKr = Q Kr^T (side 0), KQr = K Qr^T (side 1)
// ============================================================================
// One CTA per 128 rows, side and 256 columns of the Wp: 256 TMEM columns each, and shared
// memory sized so that two CTAs share an SM (one writes its rows out while the other's
// loads and MMA run).
namespace tb {
constexpr int OFF_X = 0, OFF_T = 16384, OFF_BAR = OFF_T + 32768;
constexpr int SMEM = 100 * 1024;  // two CTAs per SM (256 TMEM columns each), never three
}  // namespace tb

__global__ void __launch_bounds__(128, 1) deb_tables_kernel(const __grid_constant__ DebArgs A) {
  using namespace tb;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int BH = p.B * p.H, side = blockIdx.y;
  const int bh = (int)blockIdx.x % BH, m = (int)blockIdx.x / BH, h = bh % p.H;
  // this CTA's 256 (or fewer) columns of the Wp
  const int L = p.L, Wp = A.Wp, col0 = 256 * (int)blockIdx.z, ncol = min(256, Wp - col0), i0 = m * 128;
  const int nchunk = 1;
  const uint32_t sbase = smem_u32(smem), bar = sbase + OFF_BAR;
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 32);
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
    const CUtensorMap *mx = side ? &A.mk : &A.mq, *mt = side ? &A.mqr256 : &A.mkr256;
    const int box = Wp < 256 ? Wp : 256;  // table rows per load (the map's box)
    mbar_expect_tx(bar, 16384u + 128u * (uint32_t)box * (uint32_t)nchunk);
    tma_load_3d(sbase + OFF_X, mx, bar, 0, i0, bh);
    for (int c = 0; c < nchunk; ++c) tma_load_3d(sbase + OFF_T + 32768 * c, mt, bar, 0, col0 + 256 * c, h);
    if (mbar_wait(bar, 0, abort_flag, p.status, RELPOS_ERR_TIMEOUT_DEV)) {
      tc_fence_after();
      for (int c = 0; c < nchunk; ++c) {
        const int nc = ncol - 256 * c < 256 ? ncol - 256 * c : 256;  // a multiple of 64
        umma_k64(tbase + 256 * c, sbase + OFF_X, sbase + OFF_T + 32768 * c, idesc_bf16(128, nc, false), false);
      }
    } else {  // give the copies still in flight a bounded time to land before the CTA exits
      volatile int none = 0;
      mbar_wait(bar, 0, &none, p.status, RELPOS_ERR_TIMEOUT_DEV);
    }
    umma_commit(bar + 8);
  }
  __syncwarp();
  const bool good = warp_wait(bar + 8, 0, abort_flag, p.status) && !*abort_flag;
  const int i = i0 + tid;
  float *out = (side ? (float *)A.kqr : (float *)A.qkr) + ((size_t)bh * L + i) * Wp + col0;
  if (good) {
    tc_fence_after();
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < ncol; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tl + c0, r);
      tmem_wait_ld();
      if (i < L) {  // rows of Wp floats (Wp a multiple of 64) in the workspace: 32-byte stores
#pragma unroll
        for (int q = 0; q < 4; ++q) st_global_32B(out + c0 + 8 * q, r + 8 * q);
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

// ============================================================================
// key-tile kernel: dV, dK (content part), N
// ============================================================================
namespace kvd {
constexpr int OFF_K = 0, OFF_V = 16384, OFF_Q = 32768, OFF_DO = OFF_Q + 32768;
constexpr int OFF_PDS = OFF_DO + 32768;  // P tile, dS tile at +32768; band tiles: relation terms (128 x RLD fp32) first
constexpr int OFF_ONES = OFF_PDS + 67584;  // 128 x 64 bf16 ones, MN-major swizzled (B of dS^T 1)
constexpr int OFF_VEC = OFF_ONES + 16384;  // per tile, double-buffered: [lse2 | D | c2p end product] x 384
constexpr int OFF_EK = OFF_VEC + 3072;     // p2c end products of the CTA's keys [2][128]
constexpr int OFF_RED = OFF_EK + 1024;     // band column sums [2 classes][4 row quarters][128]
constexpr int OFF_BAR = OFF_RED + 4096;
constexpr int SMEM = OFF_BAR + 256 + 1024;
enum { B_KV = 0, B_ST0, B_ST1, B_SDP, B_SDPCONS, B_PDS, B_PDSFREE, B_DRAIN, NB };
constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 320, T_C0 = 384, T_CW = 400;
static_assert(OFF_PDS % 1024 == 0 && OFF_ONES % 1024 == 0, "swizzled operand tiles are 1024-byte aligned");
}  // namespace kvd

__global__ void __launch_bounds__(NTHREADS, 1) deb_kv_kernel(const __grid_constant__ DebArgs A) {
  using namespace kvd;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, n = (int)blockIdx.x / BH;
  const int L = p.L, W = A.W, Wp = A.Wp, k = p.span, j0 = n * 128;
  const int mStart = p.causal ? n : 0, iters = p.nT - mStart;
  const int klen = key_len(p, bh / p.H);
  if (j0 >= klen) {  // a key tile of padding only: dK = dV = 0, N rows zero (whole CTA, no barrier yet)
    for (int x = tid; x < 128 * (HD / 8); x += NTHREADS) {
      const int r = x / (HD / 8), c8 = x % (HD / 8);
      if (j0 + r < L) {
        const size_t off = ((size_t)bh * L + j0 + r) * HD + 8 * c8;
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dv + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<float4 *>(A.dkc + off) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(A.dkc + off + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    for (int x = tid; x < 128 * (Wp / 8); x += NTHREADS) {
      const int r = x / (Wp / 8), c8 = x % (Wp / 8);
      if (j0 + r < L) *reinterpret_cast<uint4 *>(A.N + ((size_t)bh * L + j0 + r) * Wp + 8 * c8) = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NB + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NB);
  float *vec = (float *)(smem + OFF_VEC);
  float *ek = (float *)(smem + OFF_EK);
  float *red = (float *)(smem + OFF_RED);
  int32_t *status = p.status;
  const float c1 = p.scale * LOG2E;
  // far tiles of this key tile exist on the left (queries after the keys) / right
  const bool anyL = n + A.nbs + 1 < p.nT;
  const bool anyR = n - A.nbs - 1 >= mStart;

  if (tid == 0) {
    for (int q = 0; q < NB; ++q) mbar_init(BAR(q), (q == B_SDPCONS || q == B_PDS) ? NSOFT : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int x = tid; x < 16384 / 16; x += NTHREADS) {
    const uint32_t one2 = 0x3F803F80u;
    *reinterpret_cast<uint4 *>(smem + OFF_ONES + 16 * x) = make_uint4(one2, one2, one2, one2);
  }
  for (int x = tid; x < 1024; x += NTHREADS) red[x] = 0.f;
  if (tid < 256) {  // k_j . Qr_0 (far tiles left of the diagonal) and k_j . Qr_{W-1} (right)
    const int s = tid >> 7, j = j0 + (tid & 127);
    ek[tid] = (j < L) ? A.kqr[((size_t)bh * L + j) * Wp + (s ? W - 1 : 0)] : 0.f;
  }
  fence_async_smem();
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
      const uint32_t idC = idesc_bf16(128, 16, true, true);
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
      bool c0_on = false, cw_on = false;
      auto accumulate = [&](int t) {  // dV += P^T dO, dK += dS^T Q; far tiles: C += dS^T 1
        const int st = t & 1, m = mStart + t;
        const bool fl = far_left(m, n, k), fr = far_right(m, n, k);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t acc = (t > 0 || q > 0) ? 1u : 0u;
          umma_bf16(tbase + T_DV, sdesc_sw128(sbase + OFF_PDS + 2048 * q, 16384, 1024),
                    sdesc_sw128(sbase + OFF_DO + 16384 * st + 2048 * q, 16, 1024), idAcc, acc);
          umma_bf16(tbase + T_DK, sdesc_sw128(sbase + OFF_PDS + 32768 + 2048 * q, 16384, 1024),
                    sdesc_sw128(sbase + OFF_Q + 16384 * st + 2048 * q, 16, 1024), idAcc, acc);
        }
        if (fl || fr) {
          const bool on = fl ? c0_on : cw_on;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            umma_bf16(tbase + (fl ? T_C0 : T_CW), sdesc_sw128(sbase + OFF_PDS + 32768 + 2048 * q, 16384, 1024),
                      sdesc_sw128(sbase + OFF_ONES + 2048 * q, 16, 1024), idC, (on || q > 0) ? 1u : 0u);
          if (fl) c0_on = true; else cw_on = true;
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
        if (t + 1 < iters) {
          if (!ctl.wait(BAR(B_SDPCONS), t & 1)) break;
          if (!ctl.wait_load(BAR(B_ST0 + ((t + 1) & 1)), ((t + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_sdp(t + 1);
        }
        if (!ctl.wait(BAR(B_PDS), t & 1)) break;
        tc_fence_after();
        accumulate(t);
        if (t + 2 < iters) {
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
    float bandC0 = 0.f, bandCW = 0.f;  // threads tid < 128: clipped column sums of band tiles, key tid
    // per-tile row terms one tile ahead: [lse2 | D | c2p end product of the tile's side]
    auto fetch1 = [&](int t) {
      const int m = mStart + t, i = m * 128 + (tid & 127);
      if (tid < 128) return lse2_of(p, bh, i);
      if (i >= L) return 0.f;
      if (tid < 256) return p.Dvec[(size_t)bh * L + i];
      if (far_left(m, n, k)) return A.qkr[((size_t)bh * L + i) * Wp + W - 1];
      if (far_right(m, n, k)) return A.qkr[((size_t)bh * L + i) * Wp];
      return 0.f;
    };
    if (tid < 384) vec[tid] = fetch1(0);
    for (int t = 0; t < iters; ++t) {
      const int m = mStart + t, i = m * 128 + il;
      const float *tv = vec + 384 * (t & 1);
      const float nv = (tid < 384 && t + 1 < iters) ? fetch1(t + 1) : 0.f;
      named_bar_sync(1, NSOFT);
      const bool fl = far_left(m, n, k), fr = far_right(m, n, k), band = !fl && !fr;
      float *Rt = (float *)(smem + OFF_PDS);
      if (band) {  // the relation terms overwrite the P / dS tiles: the previous tile's MMAs must be done
        if (t >= 1) good = good && warp_wait(BAR(B_PDSFREE), (t - 1) & 1, abort_flag, status);
        band_fill(A, bh, m * 128, j0, Rt, warp, lane);
      }
      good = good && warp_wait(BAR(B_SDP), t & 1, abort_flag, status);
      uint32_t pk[NC / 2], dk[NC / 2];
      const bool need_mask = (p.causal && m == n) || (j0 + 128 > klen);
      if (good) {
        tc_fence_after();
        const float lse2 = tv[il], Dv = tv[128 + il], cE = tv[256 + il];
        const float *ekr = ek + (fl ? 0 : 128) + cb;
        const float *Rrow = Rt + il * RLD + cb;
        const uint64_t c12 = f2(c1, c1), nlse = f2(-lse2, -lse2), nDv = f2(-Dv, -Dv);
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
              if constexpr (decltype(banded)::value) {
#pragma unroll
                for (int e = 0; e < 4; ++e) R[e] = Rrow[x0 + e];
              } else {  // four keys' end products in one 16-byte load (aligned: cb, x0 multiples of 4)
                const float4 ev = *reinterpret_cast<const float4 *>(ekr + x0);
                R[0] = cE + ev.x;
                R[1] = cE + ev.y;
                R[2] = cE + ev.z;
                R[3] = cE + ev.w;
              }
              score_rel4(rs + 4 * c4, R, c12, nlse, y);
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
        if (band) {
          if (need_mask) pds(std::true_type{}, std::true_type{}); else pds(std::false_type{}, std::true_type{});
        } else {
          if (need_mask) pds(std::true_type{}, std::false_type{}); else pds(std::false_type{}, std::false_type{});
        }
        tc_fence_before();
        mbar_arrive(BAR(B_SDPCONS));
      } else {
#pragma unroll
        for (int e = 0; e < NC / 2; ++e) pk[e] = dk[e] = 0u;
      }
      if (band) named_bar_sync(1, NSOFT);  // every row has read the relation terms: P / dS may overwrite them
      else if (t >= 1) good = good && warp_wait(BAR(B_PDSFREE), (t - 1) & 1, abort_flag, status);
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
      if (band) {
        // N interior entries of this tile: N[j][j - i + k] = dS_ij (bf16, as in the MMA operand)
        const int r0 = j0 + cb - i + k;
#pragma unroll
        for (int x = 0; x < NC; ++x) {
          const int r = r0 + x, j = j0 + cb + x;
          if (r >= 1 && r <= W - 2 && j < L) {
            const uint32_t v = dk[x >> 1];
            *reinterpret_cast<uint16_t *>(A.N + ((size_t)bh * L + j) * Wp + r) = (uint16_t)((x & 1) ? (v >> 16) : (v & 0xFFFFu));
          }
        }
        // clipped column sums of the band tile: class 0 (i - j >= k), class W - 1 (j - i >= k - 1)
#pragma unroll
        for (int cls = 0; cls < 2; ++cls) {
          const bool present = cls == 0 ? 128 * (m - n) + 127 >= k : 128 * (n - m) + 127 >= k - 1;
          if (!present) continue;  // uniform over the CTA
          float v[32];
#pragma unroll
          for (int x = 0; x < NC; ++x) {
            const int r = r0 + x;
            const float d = (x & 1) ? bf_hi(dk[x >> 1]) : bf_lo(dk[x >> 1]);
            v[x] = (cls == 0 ? r <= 0 : r >= W - 1) ? d : 0.f;
          }
          red[cls * 512 + g * 128 + cb + lane] = warp_colsum32(v, lane);
        }
        named_bar_sync(2, NSOFT);
        if (tid < 128) {
          bandC0 += ((red[tid] + red[128 + tid]) + red[256 + tid]) + red[384 + tid];
          bandCW += ((red[512 + tid] + red[640 + tid]) + red[768 + tid]) + red[896 + tid];
        }
        named_bar_sync(2, NSOFT);
        if (tid < 128) {  // clear for the next band tile (an absent class leaves zeros)
#pragma unroll
          for (int q = 0; q < 8; ++q) red[128 * q + tid] = 0.f;
        }
      }
      if (tid < 384) vec[384 * ((t + 1) & 1) + tid] = nv;
    }
    // ---- zero the N entries of band query tiles this CTA did not visit ----
    for (int m = n - A.nbs; m <= n + A.nbs; ++m) {
      if (m >= mStart && m < p.nT) continue;
      const int r0 = j0 + cb - (m * 128 + il) + k;
#pragma unroll 4
      for (int x = 0; x < NC; ++x) {
        const int r = r0 + x, j = j0 + cb + x;
        if (r >= 1 && r <= W - 2 && j < L) *reinterpret_cast<uint16_t *>(A.N + ((size_t)bh * L + j) * Wp + r) = 0;
      }
    }
    // ---- epilogue: lanes are keys; this thread takes 16 of the 64 columns ----
    good = good && warp_wait(BAR(B_PDSFREE), (iters - 1) & 1, abort_flag, status);
    const int j = j0 + il;
    if (good) {
      tc_fence_after();
      uint32_t rv[16], rk[16];
      tmem_ld16(tl + T_DV + 16 * qt, rv);
      tmem_ld16(tl + T_DK + 16 * qt, rk);
      uint32_t rc0[16], rcw[16];
      tmem_ld16(tl + T_C0, rc0);
      tmem_ld16(tl + T_CW, rcw);
      tmem_wait_ld();
      if (j < L) {
        __nv_bfloat16 *dvp = (__nv_bfloat16 *)p.dv + ((size_t)bh * L + j) * HD + 16 * qt;
        float *dkp = A.dkc + ((size_t)bh * L + j) * HD + 16 * qt;
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          uint4 wv;
          wv.x = pack_bf16x2(u2f(rv[8 * c8 + 0]), u2f(rv[8 * c8 + 1]));
          wv.y = pack_bf16x2(u2f(rv[8 * c8 + 2]), u2f(rv[8 * c8 + 3]));
          wv.z = pack_bf16x2(u2f(rv[8 * c8 + 4]), u2f(rv[8 * c8 + 5]));
          wv.w = pack_bf16x2(u2f(rv[8 * c8 + 6]), u2f(rv[8 * c8 + 7]));
          *reinterpret_cast<uint4 *>(dvp + 8 * c8) = wv;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<float4 *>(dkp + 4 * q) = make_float4(u2f(rk[4 * q]), u2f(rk[4 * q + 1]), u2f(rk[4 * q + 2]), u2f(rk[4 * q + 3]));
        if (qt == 0) {  // N end columns: clipped column sums (far tiles from TMEM, band tiles from the butterflies)
          const float c0 = (anyL ? u2f(rc0[0]) : 0.f) + bandC0, cw = (anyR ? u2f(rcw[0]) : 0.f) + bandCW;
          __nv_bfloat16 *np = A.N + ((size_t)bh * L + j) * Wp;
          np[0] = __float2bfloat16_rn(c0);
          np[W - 1] = __float2bfloat16_rn(cw);
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
// query-tile kernel: dQ (content part), M
// ============================================================================
namespace qd {
constexpr int OFF_Q = 0, OFF_DO = 16384, OFF_K = 32768, OFF_V = OFF_K + 32768;
constexpr int OFF_R = OFF_V + 32768;     // band tiles: relation terms, then dS (128 x RLD fp32)
constexpr int OFF_VEC = OFF_R + 128 * RLD * 4;  // p2c end products of the tile's keys, double-buffered [2][128]
constexpr int OFF_RED = OFF_VEC + 1024;  // clipped row sums [2][4][128]
constexpr int OFF_BAR = OFF_RED + 4096;
constexpr int SMEM = OFF_BAR + 256 + 1024;  // over half the SM: one CTA per SM (512 TMEM columns each)
enum { B_QD = 0, B_ST0, B_ST1, B_SDP, B_SDPCONS, B_PDS, B_DSFREE, B_DRAIN, NB };
constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256, T_DS = 320;
static_assert(OFF_BAR + 256 + 1024 <= SMEM, "shared memory layout");
}  // namespace qd

__global__ void __launch_bounds__(NTHREADS, 1) deb_q_kernel(const __grid_constant__ DebArgs A) {
  using namespace qd;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, m = p.nT - 1 - (int)blockIdx.x / BH;
  const int L = p.L, W = A.W, Wp = A.Wp, k = p.span, i0 = m * 128;
  const int klen = key_len(p, bh / p.H);
  const int nTiles = min(p.causal ? m + 1 : p.nT, (klen + 127) / 128);
  if (nTiles == 0) {  // no key at all: dQ = 0, M rows zero (whole CTA, before any barrier)
    for (int x = tid; x < 128 * (HD / 4); x += NTHREADS) {
      const int r = x / (HD / 4), c4 = x % (HD / 4);
      if (i0 + r < L) *reinterpret_cast<float4 *>(A.dqc + ((size_t)bh * L + i0 + r) * HD + 4 * c4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int x = tid; x < 128 * (Wp / 8); x += NTHREADS) {
      const int r = x / (Wp / 8), c8 = x % (Wp / 8);
      if (i0 + r < L) *reinterpret_cast<uint4 *>(A.M + ((size_t)bh * L + i0 + r) * Wp + 8 * c8) = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NB + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NB);
  float *vec = (float *)(smem + OFF_VEC);
  float *red = (float *)(smem + OFF_RED);
  int32_t *status = p.status;
  const float c1 = p.scale * LOG2E;

  if (tid == 0) {
    for (int q = 0; q < NB; ++q) mbar_init(BAR(q), (q == B_SDPCONS || q == B_PDS) ? NSOFT : 1);
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
        if (n + 1 < nTiles) {
          if (!ctl.wait(BAR(B_SDPCONS), n & 1)) break;
          if (!ctl.wait_load(BAR(B_ST0 + (st ^ 1)), ((n + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_sdp(n + 1);
        }
        if (!ctl.wait(BAR(B_PDS), n & 1)) break;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 8; ++q)
          umma_bf16_ts(tbase + T_DQ, tbase + T_DS + 8 * q, sdesc_sw128(sbase + OFF_K + 16384 * st + 2048 * q, 16, 1024), idDQ,
                       (n > 0 || q > 0) ? 1u : 0u);
        umma_commit(BAR(B_DSFREE));
        if (n + 2 < nTiles) {
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
    const float cE0 = (i < L) ? A.qkr[((size_t)bh * L + i) * Wp] : 0.f;          // q_i . Kr_0
    const float cEW = (i < L) ? A.qkr[((size_t)bh * L + i) * Wp + W - 1] : 0.f;  // q_i . Kr_{W-1}
    const uint64_t c12 = f2(c1, c1), nlse = f2(-lse2, -lse2), nDv = f2(-Dv, -Dv);
    __nv_bfloat16 *mrow = A.M + ((size_t)bh * L + i) * Wp;
    bool good = true;
    float rs0 = 0.f, rsW = 0.f;  // clipped row sums: rho = 0 (j - i >= k), rho = W - 1 (i - j >= k - 1)
    // p2c end product of key tile n's keys for the tile's side, one tile ahead
    auto fetch_ek = [&](int n) {
      const int j = n * 128 + tid;
      if (tid >= 128 || j >= L) return 0.f;
      if (far_left(m, n, k)) return A.kqr[((size_t)bh * L + j) * Wp];
      if (far_right(m, n, k)) return A.kqr[((size_t)bh * L + j) * Wp + W - 1];
      return 0.f;
    };
    float nva = fetch_ek(0);
    for (int n = 0; n < nTiles; ++n) {
      const int j0 = n * 128;
      float *tv = vec + 128 * (n & 1);
      if (tid < 128) tv[tid] = nva;
      if (n + 1 < nTiles) nva = fetch_ek(n + 1);
      named_bar_sync(1, NSOFT);
      const bool fl = far_left(m, n, k), fr = far_right(m, n, k), band = !fl && !fr;
      float *Rt = (float *)(smem + OFF_R);
      if (band) band_fill(A, bh, i0, j0, Rt, warp, lane);
      good = good && warp_wait(BAR(B_SDP), n & 1, abort_flag, status);
      const bool need_mask = (p.causal && n == m) || (j0 + 128 > klen);
      float x[NC];
      if (good) {
        tc_fence_after();
        const float cE = fl ? cEW : cE0;
        const float *ekr = tv + cb;
        const float *Rrow = Rt + il * RLD + cb;
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
              if constexpr (decltype(banded)::value) {
#pragma unroll
                for (int e = 0; e < 4; ++e) R[e] = Rrow[x0 + e];
              } else {  // four keys' end products in one 16-byte load (aligned: cb, x0 multiples of 4)
                const float4 ev = *reinterpret_cast<const float4 *>(ekr + x0);
                R[0] = cE + ev.x;
                R[1] = cE + ev.y;
                R[2] = cE + ev.z;
                R[3] = cE + ev.w;
              }
              score_rel4(rs + 4 * c4, R, c12, nlse, y);
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
      uint32_t pk[NC / 2];
#pragma unroll
      for (int q = 0; q < NC / 2; ++q) pk[q] = pack_bf16x2(x[2 * q], x[2 * q + 1]);
      // ---- clipped row sums; band tiles: dS through smem into the M rows ----
      if (band) {
        const int r0 = i - j0 - cb + k;  // rho of this thread's first key (decreasing with the key)
#pragma unroll
        for (int e = 0; e < NC; ++e) {
          const int r = r0 - e;
          if (r <= 0) rs0 += x[e];
          else if (r >= W - 1) rsW += x[e];
        }
        named_bar_sync(2, NSOFT);  // every row has read the relation terms
#pragma unroll
        for (int e = 0; e < NC; ++e) Rt[il * RLD + cb + e] = x[e];
        named_bar_sync(2, NSOFT);
        // warp w writes rows 8w .. 8w + 7: M[i][rho] for the interior rho of the tile's keys
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int ir = i0 + 8 * warp + rr;
          if (ir >= L) continue;
          __nv_bfloat16 *mr = A.M + ((size_t)bh * L + ir) * Wp;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int jl = lane + 32 * q, r = ir - j0 - jl + k;
            if (r >= 1 && r <= W - 2) mr[r] = __float2bfloat16_rn(Rt[(8 * warp + rr) * RLD + jl]);
          }
        }
      } else {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < NC; ++e) s += x[e];
        if (fl) rsW += s; else rs0 += s;
      }
      // ---- dS -> TMEM for dQ += dS K ----
      if (good) {
        if (n >= 1 && !warp_wait(BAR(B_DSFREE), (n - 1) & 1, abort_flag, status)) good = false;
        if (good) {
          tmem_st16(tl + T_DS + 16 * qt, pk);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(BAR(B_PDS));
        }
      }
    }
    // ---- zero the M entries of band key tiles this CTA did not visit ----
    if (i < L) {
      for (int n = m - A.nbs; n <= m + A.nbs; ++n) {
        if (n >= 0 && n < nTiles) continue;
        const int r0 = i - n * 128 - cb + k;
#pragma unroll 4
        for (int e = 0; e < NC; ++e) {
          const int r = r0 - e;
          if (r >= 1 && r <= W - 2) *reinterpret_cast<uint16_t *>(mrow + r) = 0;
        }
      }
    }
    // ---- epilogue: dQ (content part) and the end columns of M ----
    good = good && warp_wait(BAR(B_DSFREE), (nTiles - 1) & 1, abort_flag, status);
    if (good) {
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tl + T_DQ + 16 * qt, r);
      tmem_wait_ld();
      if (i < L) {
        float *dqp = A.dqc + ((size_t)bh * L + i) * HD + 16 * qt;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<float4 *>(dqp + 4 * q) = make_float4(u2f(r[4 * q]), u2f(r[4 * q + 1]), u2f(r[4 * q + 2]), u2f(r[4 * q + 3]));
      }
    }
    red[qt * 128 + il] = rs0;
    red[512 + qt * 128 + il] = rsW;
    named_bar_sync(1, NSOFT);
    if (qt == 0 && i < L) {
      const float s0 = ((red[il] + red[128 + il]) + red[256 + il]) + red[384 + il];
      const float sW = ((red[512 + il] + red[640 + il]) + red[768 + il]) + red[896 + il];
      mrow[0] = __float2bfloat16_rn(s0);
      mrow[W - 1] = __float2bfloat16_rn(sW);
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
// rows kernel: dq = s (dQ + M Kr) (side 0), dk = s (dK + N Qr) (side 1)
// ============================================================================
// The Wp / 64 K steps are staged four at a time; a group's loads are issued once the
// previous group's MMAs are done with the staging buffers.
namespace rw {
constexpr int GK = 4;                   // K steps per group (96 KB: two CTAs per SM)
constexpr int OFF_X = 0;                // GK chunks of 128 rows x 64 columns (16 KB each)
constexpr int OFF_T = GK * 16384;       // GK chunks of 64 table rows x 64 (8 KB each)
constexpr int OFF_BAR = OFF_T + GK * 8192;
constexpr int SMEM = OFF_BAR + 256 + 1024;
}  // namespace rw

__global__ void __launch_bounds__(128, 1) deb_rows_kernel(const __grid_constant__ DebArgs A) {
  using namespace rw;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int BH = p.B * p.H, side = blockIdx.y;
  const int bh = (int)blockIdx.x % BH, m = (int)blockIdx.x / BH, h = bh % p.H;
  const int L = p.L, i0 = m * 128, nk = A.Wp / 64, ng = (nk + GK - 1) / GK;
  // bar: a group's loads landed; bar + 8: a group's MMAs done (staging free); bar + 24: all MMAs done
  const uint32_t sbase = smem_u32(smem), bar = sbase + OFF_BAR;
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 36);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 32);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 8, 1);
    mbar_init(bar + 24, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 64);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  if (tid == 0) {
    const CUtensorMap *mx = side ? &A.mN : &A.mM, *mt = side ? &A.mqr64 : &A.mkr64;
    const uint32_t id = idesc_bf16(128, 64, true);
    for (int gi = 0; gi < ng; ++gi) {
      const int c0 = GK * gi, nc = min(GK, nk - c0);
      const uint32_t ph = (uint32_t)(gi & 1);
      // the previous group's MMAs read the staging buffers: wait for them first
      if (gi > 0 && !mbar_wait(bar + 8, ph ^ 1u, abort_flag, p.status, RELPOS_ERR_TIMEOUT_DEV)) break;
      mbar_expect_tx(bar, (uint32_t)nc * (16384u + 8192u));
      for (int c = 0; c < nc; ++c) {
        tma_load_3d(sbase + OFF_X + 16384 * c, mx, bar, 64 * (c0 + c), i0, bh);
        tma_load_3d(sbase + OFF_T + 8192 * c, mt, bar, 0, 64 * (c0 + c), h);
      }
      if (!mbar_wait(bar, ph, abort_flag, p.status, RELPOS_ERR_TIMEOUT_DEV)) {
        // give the copies still in flight a bounded time to land before the CTA exits
        volatile int none = 0;
        mbar_wait(bar, ph, &none, p.status, RELPOS_ERR_TIMEOUT_DEV);
        break;
      }
      tc_fence_after();
      for (int c = 0; c < nc; ++c)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          umma_bf16(tbase, sdesc_sw128(sbase + OFF_X + 16384 * c + 32 * q, 16, 1024),
                    sdesc_sw128(sbase + OFF_T + 8192 * c + 2048 * q, 16, 1024), id, (c0 + c > 0 || q > 0) ? 1u : 0u);
      umma_commit(bar + 8);
    }
    umma_commit(bar + 24);
  }
  __syncwarp();
  const bool good = warp_wait(bar + 24, 0, abort_flag, p.status) && !*abort_flag;
  const int i = i0 + tid;
  if (good) {
    tc_fence_after();
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    uint32_t r[2][32];
    tmem_ld32(tl, r[0]);
    tmem_ld32(tl + 32, r[1]);
    tmem_wait_ld();
    if (i < L) {
      const float *cp = (side ? A.dkc : A.dqc) + ((size_t)bh * L + i) * HD;
      __nv_bfloat16 *op = (__nv_bfloat16 *)(side ? p.dk : p.dq) + ((size_t)bh * L + i) * HD;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const float4 a = *reinterpret_cast<const float4 *>(cp + 8 * c8);
        const float4 b = *reinterpret_cast<const float4 *>(cp + 8 * c8 + 4);
        const uint32_t *rr = r[c8 >> 2] + 8 * (c8 & 3);
        uint4 w;
        w.x = pack_bf16x2(p.scale * (a.x + u2f(rr[0])), p.scale * (a.y + u2f(rr[1])));
        w.y = pack_bf16x2(p.scale * (a.z + u2f(rr[2])), p.scale * (a.w + u2f(rr[3])));
        w.z = pack_bf16x2(p.scale * (b.x + u2f(rr[4])), p.scale * (b.y + u2f(rr[5])));
        w.w = pack_bf16x2(p.scale * (b.z + u2f(rr[6])), p.scale * (b.w + u2f(rr[7])));
        *reinterpret_cast<uint4 *>(op + 8 * c8) = w;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 64);
  }
}

// ============================================================================
// table kernel: partials of M^T Q (side 0, dKr) and N^T K (side 1, dQr)
// ============================================================================
namespace tk {
constexpr int NSTAGE = 3, STAGE = 49152;  // X: two 64-column boxes of 128 rows, Y: 128 x 64
constexpr int OFF_BAR = NSTAGE * STAGE;
constexpr int SMEM = OFF_BAR + 256 + 1024;
}  // namespace tk

__global__ void __launch_bounds__(128, 1) deb_table_kernel(const __grid_constant__ DebArgs A) {
  using namespace tk;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int nblk = (A.W + 127) / 128, side = blockIdx.z;
  const int h = (int)blockIdx.x / nblk, blk = (int)blockIdx.x % nblk;
  const int b = (int)blockIdx.y / A.nch, c = (int)blockIdx.y % A.nch, bh = b * p.H + h;
  const int rbase = c * CH, nsteps = CH / 128;
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto LD = [&](int s) { return bar0 + 8u * (uint32_t)s; };
  auto FR = [&](int s) { return bar0 + 8u * (uint32_t)(NSTAGE + s); };
  const uint32_t done = bar0 + 8u * 2 * NSTAGE;
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * (2 * NSTAGE + 1) + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * (2 * NSTAGE + 1));
  if (tid == 0) {
    for (int s = 0; s < 2 * NSTAGE + 1; ++s) mbar_init(bar0 + 8u * (uint32_t)s, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 64);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  if (tid == 0) {
    const CUtensorMap *mx = side ? &A.mN : &A.mM, *my = side ? &A.mk : &A.mq;
    int32_t *status = p.status;
    auto issue = [&](int s) {
      const int st = s % NSTAGE, row = rbase + 128 * s;
      const uint32_t dst = sbase + STAGE * st;
      mbar_expect_tx(LD(st), 49152u);
      tma_load_3d(dst, mx, LD(st), 128 * blk, row, bh);
      tma_load_3d(dst + 16384, mx, LD(st), 128 * blk + 64, row, bh);
      tma_load_3d(dst + 32768, my, LD(st), 0, row, bh);
    };
    const uint32_t id = idesc_bf16(128, 64, true, true);
    int issued = 0, waited = 0;  // loads issued / loads waited for (all are waited before exit)
    for (; issued < NSTAGE && issued < nsteps; ++issued) issue(issued);
    for (int s = 0; s < nsteps; ++s) {
      const int st = s % NSTAGE;
      if (!mbar_wait(LD(st), (uint32_t)((s / NSTAGE) & 1), abort_flag, status, RELPOS_ERR_TIMEOUT_DEV)) break;
      ++waited;
      tc_fence_after();
      const uint32_t xs = sbase + STAGE * st;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        umma_bf16(tbase, sdesc_sw128(xs + 2048 * q, 16384, 1024), sdesc_sw128(xs + 32768 + 2048 * q, 16, 1024), id,
                  (s > 0 || q > 0) ? 1u : 0u);
      umma_commit(FR(st));
      if (issued < nsteps) {  // refill this stage once its MMAs are done
        if (!mbar_wait(FR(st), (uint32_t)((s / NSTAGE) & 1), abort_flag, status, RELPOS_ERR_TIMEOUT_DEV)) break;
        issue(issued++);
      }
    }
    // every load issued is waited for (bounded) before the MMAs are drained
    volatile int none = 0;
    for (int s = waited; s < issued; ++s)
      mbar_wait(LD(s % NSTAGE), (uint32_t)((s / NSTAGE) & 1), &none, status, RELPOS_ERR_TIMEOUT_DEV);
    umma_commit(done);
  }
  __syncwarp();
  const bool good = warp_wait(done, 0, abort_flag, p.status) && !*abort_flag;
  if (good) {
    tc_fence_after();
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    uint32_t r[2][32];
    tmem_ld32(tl, r[0]);
    tmem_ld32(tl + 32, r[1]);
    tmem_wait_ld();
    float *out = A.part + ((((size_t)side * p.H + h) * nblk + blk) * ((size_t)p.B * A.nch) + (size_t)b * A.nch + c) * 128 * HD +
                 (size_t)tid * HD;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const uint32_t *rr = r[q >> 3] + 4 * (q & 7);
      *reinterpret_cast<float4 *>(out + 4 * q) = make_float4(u2f(rr[0]), u2f(rr[1]), u2f(rr[2]), u2f(rr[3]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 64);
  }
}

// dKr (side 0) / dQr (side 1) = s * sum over batches and chunks of the partials, fixed order
__global__ void reduce_deb_table_kernel(DebArgs A) {
  const Prm &p = A.p;
  const size_t per = (size_t)A.W * HD;
  const size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= 2 * (size_t)p.H * per) return;
  const int side = (int)(x / ((size_t)p.H * per));
  const size_t y = x % ((size_t)p.H * per);
  const int h = (int)(y / per), r = (int)((y % per) / HD), d = (int)(y % HD);
  const int nblk = (A.W + 127) / 128, blk = r / 128, rr = r % 128, nc = p.B * A.nch;
  const float *src = A.part + (((size_t)side * p.H + h) * nblk + blk) * (size_t)nc * 128 * HD + (size_t)rr * HD + d;
  float acc = 0.f;
  for (int q = 0; q < nc; ++q) acc += src[(size_t)q * 128 * HD];
  (side ? p.drel1 : p.drel0)[y] = p.scale * acc;
}

}  // namespace tcdeb

bool tc_make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t planes, uint32_t box_rows);
bool tc_make_map_bf16_wide(CUtensorMap *m, const void *base, uint32_t row_len, uint64_t rows, uint64_t planes,
                           uint32_t box_rows);

bool tc_bwd_deb_supported(const Prm &p) { return p.mech == M_DEB && p.span >= 1; }

static int deb_wp(const Prm &p) { return (2 * p.span + 63) / 64 * 64; }

void tc_bwd_deb_sizes(const Prm &p, size_t &table_elems, size_t &part_floats, size_t &pad_elems) {
  const size_t W = 2 * (size_t)p.span, Wp = (size_t)deb_wp(p), BH = (size_t)p.B * p.H;
  const size_t nch = ((size_t)p.L + tcdeb::CH - 1) / tcdeb::CH;
  table_elems = BH * p.L * Wp;
  part_floats = 2 * (size_t)p.H * ((W + 127) / 128) * p.B * nch * 128 * HD;
  pad_elems = 2 * (size_t)p.H * Wp * HD;  // Kr and Qr, zero rows W .. Wp - 1
}

cudaError_t tc_bwd_deb(const Prm &p0, const TcWork &w, cudaStream_t st) {
  using namespace tcdeb;
  DebArgs a;
  memset(&a, 0, sizeof(a));
  a.p = p0;
  a.p.nT = (p0.L + 127) / 128;
  a.W = 2 * p0.span;
  a.Wp = deb_wp(p0);
  a.nbs = (p0.span + 254) / 128 - 1;  // band tiles per side (also past the sequence ends: their M / N entries are zeroed)
  a.nch = (p0.L + CH - 1) / CH;
  a.qkr = w.qkr;
  a.kqr = w.kqr;
  a.M = (__nv_bfloat16 *)w.dM;
  a.N = (__nv_bfloat16 *)w.dN;
  a.dqc = w.dqc;
  a.dkc = w.dkc;
  a.part = w.dpart;
  const uint64_t BH = (uint64_t)p0.B * p0.H;
  // Kr and Qr copied into [H][Wp][64] tables whose rows W .. Wp - 1 are zero
  __nv_bfloat16 *kp = (__nv_bfloat16 *)w.dpad, *qp = kp + (size_t)p0.H * a.Wp * HD;
  cudaError_t e;
  const size_t rowb = (size_t)HD * 2, tabb = (size_t)a.W * rowb, padb = (size_t)a.Wp * rowb;
  if ((e = cudaMemsetAsync(w.dpad, 0, 2 * (size_t)p0.H * padb, st)) != cudaSuccess) return e;
  if ((e = cudaMemcpy2DAsync(kp, padb, p0.rel0, tabb, tabb, p0.H, cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  if ((e = cudaMemcpy2DAsync(qp, padb, p0.rel1, tabb, tabb, p0.H, cudaMemcpyDeviceToDevice, st)) != cudaSuccess) return e;
  if (a.Wp != a.W) {  // M and N columns W .. Wp - 1 (no kernel writes them) are zero: the rows kernel's K steps read them
    const size_t rows = (size_t)BH * p0.L, pitch = (size_t)a.Wp * 2, wb = (size_t)(a.Wp - a.W) * 2;
    if ((e = cudaMemset2DAsync(a.M + a.W, pitch, 0, wb, rows, st)) != cudaSuccess) return e;
    if ((e = cudaMemset2DAsync(a.N + a.W, pitch, 0, wb, rows, st)) != cudaSuccess) return e;
  }
  if (!(tc_make_map(&a.mq, p0.q, p0.L, BH, 128) && tc_make_map(&a.mk, p0.k, p0.L, BH, 128) &&
        tc_make_map(&a.mv, p0.v, p0.L, BH, 128) && tc_make_map(&a.mdo, p0.dout, p0.L, BH, 128) &&
        tc_make_map(&a.mkr256, kp, a.Wp, p0.H, std::min(a.Wp, 256)) &&
        tc_make_map(&a.mqr256, qp, a.Wp, p0.H, std::min(a.Wp, 256)) &&
        tc_make_map(&a.mkr64, kp, a.Wp, p0.H, 64) && tc_make_map(&a.mqr64, qp, a.Wp, p0.H, 64) &&
        tc_make_map_bf16_wide(&a.mM, a.M, a.Wp, p0.L, BH, 128) && tc_make_map_bf16_wide(&a.mN, a.N, a.Wp, p0.L, BH, 128)))
    return cudaErrorInvalidValue;
  if ((e = cudaFuncSetAttribute(deb_tables_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tb::SMEM)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(deb_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kvd::SMEM)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(deb_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, qd::SMEM)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(deb_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, rw::SMEM)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(deb_table_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tk::SMEM)) != cudaSuccess) return e;
  const unsigned tiles = (unsigned)(a.p.nT * BH);
  RP_TRACED("deb_tables_kernel", st, deb_tables_kernel<<<dim3(tiles, 2, (unsigned)((a.Wp + 255) / 256)), 128, tb::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("deb_kv_kernel", st, deb_kv_kernel<<<tiles, NTHREADS, kvd::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("deb_q_kernel", st, deb_q_kernel<<<tiles, NTHREADS, qd::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("deb_rows_kernel", st, deb_rows_kernel<<<dim3(tiles, 2), 128, rw::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("deb_table_kernel", st, deb_table_kernel<<<dim3((unsigned)(p0.H * ((a.W + 127) / 128)), (unsigned)(p0.B * a.nch), 2), 128, tk::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t n = 2 * (size_t)p0.H * a.W * HD;
  RP_TRACED("reduce_deb_table_kernel", st, reduce_deb_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a));
  return cudaGetLastError();
}

}  // namespace rp
