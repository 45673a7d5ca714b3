// Tensor-core (tcgen05 / TMEM / TMA) backward pass of Transformer-XL relative
// attention, bf16, d = 64, sm_100a.  No atomics anywhere.
//
// Three kernels share one per-tile engine (tc_bwd_common.cuh): four threads per query
// row in 16 row warps, and one control warp whose lane 0 issues every TMA load and
// tcgen05.mma.  For a 128 x 128 tile
// (query tile m, key tile n, Delta = m - n) the offsets are i - j = 128 Delta +
// [-127, 127], i.e. the two 128-offset blocks Delta and Delta - 1 of r; the rows
// recompute S = s((q + u).k + (q + v).r) exactly as the forward does (relation
// products by MMA, skewed into key order through padded smem rows), then
// P = exp(S - LSE), dP = dO V^T, dS = P (dP - D) with D = rowsum(dO o O).
//
//   key-tile kernel   (one CTA per key tile n, query tiles streamed):
//                     dV += P^T dO, dK += dS^T Q, c += dS^T 1 (column sums of dS),
//                     all with P / dS from smem as MN-major A operands; at the end
//                     dK += c u^T and a du partial sum_j c_j k_j.
//   query-tile kernel (one CTA per query tile m, key tiles streamed; the relation
//                     blocks are reused across key tiles as in the forward):
//                     dQ += dS K_n (dS as the TMEM A operand) + E_lo r_Delta +
//                     E_hi r_{Delta-1}, where E is dS moved into offset
//                     coordinates (E[i][c] = dS[i][i - c] by block).
//   diagonal kernel   (one CTA per chunk of a diagonal band Delta): every tile of
//                     the band reads the same two offset blocks, so the CTA keeps
//                     G += E^T Q and g += E^T 1 for both blocks in TMEM and writes one
//                     partial per chunk ("offset-based gradient sharding",
//                     "Fast and Exact Relative-Position Attention via Structure-Aware
//                     Kernels", Abstract, technique (3)).
// A fixed-order reduction turns the partials into dr = s (G + g v), dv = s sum g r
// and du = s sum_j c_j k_j.
//
// Stored tiles (whenever the buffer fits in 32 GiB): the query-tile kernel runs first and
// its row threads also write every tile's P and dS (bf16, 64 KB per tile) to a workspace
// buffer; the key-tile and diagonal work then stream those tiles instead of recomputing
// S, P and dS (tc_bwd_kvs_kernel: dV, [dK | c] MMAs only; tc_bwd_dgs_kernel: E rebuilt in
// smem from the stored dS, then the G MMAs).  The results are bitwise the same.
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tc_skew.cuh"
#include "tc_bwd_common.cuh"

namespace rp {
namespace tcb {

using namespace tc;

struct BwdArgs {
  CUtensorMap mq, mk, mv, mdo, mr;
  Prm p;                 // nT counts 128-row tiles
  const float *uk, *vr;  // u.k_j [B,H,L], v.r_rho [H,rows]
  float *part_kv;        // [B,H,nT][64]  du partial per key tile
  float *part_dg;        // [B,H,nbands,nchunk][2][65][128] diagonal partials (G then g)
  float *part_uv;        // [H][ceil(rows / 32)][64] dv partials per 32-offset tile
  int dg_ch, dg_nchunk, nbands;
  CUtensorMap mpd;       // stored P / dS tiles: [planes][128][64] bf16, four 16 KB planes per tile
  __nv_bfloat16 *pd;     // (P keys 0-63, P keys 64-127, dS likewise) and their base
  int pd_stored;         // 1: the query-tile kernel stores P and dS; dK / dV and dr come from them
  int n_kvs;             // streaming launch: CTAs of the key-tile role (the rest run the diagonal role)
};

// First of the four 16 KB planes of tile (m, n) of (batch, head) bh in the stored-tile
// buffer: causal tiles n <= m row by row, else all.
__device__ __forceinline__ int tile_plane(const Prm &p, int bh, int m, int n) {
  const int ntiles = p.causal ? p.nT * (p.nT + 1) / 2 : p.nT * p.nT;
  const int idx = p.causal ? m * (m + 1) / 2 + n : m * p.nT + n;
  return (bh * ntiles + idx) * 4;
}

constexpr int DG_STRIDE = 2 * 128 * 65;

// dS of this thread's NC keys (jl = cb + e, e = 0..NC-1) of row il, written into
// the two 128x128 bf16 operand tiles of the relation products in offset order
// (128-byte-swizzled K-major, 64-column halves 16 KB apart; E_lo at E, E_hi at
// E + 32768).  In the combined offset c' = il - jl + 128, c' >= 128 is E_lo column
// c' - 128 (keys jl <= il) and c' < 128 is E_hi column c' (keys jl > il); the value's
// partner c' ^ 128 in the other tile gets 0, so both tiles are fully rewritten.
// x[e] sits at c' = C0 - e, C0 = il - cb + 128: values go out as aligned bf16 pairs;
// when C0 is even the first and last value pair with a neighbouring thread's and
// are written alone.  The positions of values and zeros are the same for every tile, so
// a kernel whose E tiles hold nothing else zeroes them once and passes ZERO = false.
__device__ __forceinline__ uint32_t E_off(uint32_t t, uint32_t rowb, uint32_t r7) {  // t = 2 c', c' even
  return (((t << 7) & 0xC000u) ^ 0x8000u) + rowb + ((t & 126u) ^ r7);
}
// pk[k] = bf16 pair (x[2k+1] low, x[2k] high) of the thread's values
template <bool ZERO = true>
__device__ __forceinline__ void store_E(uint8_t *E, int il, int cb, const uint32_t (&pk)[NC / 2]) {
  const uint32_t C0 = (uint32_t)(il - cb + 128);
  const bool ev = (C0 & 1u) == 0;
  const uint32_t rowb = 128u * (uint32_t)il, r7 = (uint32_t)(il & 7) << 4;
  const uint32_t T0 = 2u * ((C0 - 1u) & ~1u);  // 2 c' of the first whole pair
  // pk[k] = (x[2k+1], x[2k]) is the pair at c' = C0 - 2k - 1 when C0 is odd; when it
  // is even the pair at c' = C0 - 2k - 2 is (x[2k+2], x[2k+1]): high half of pk[k+1],
  // low half of pk[k], picked by one byte permute
  const uint32_t sel = ev ? 0x1076u : 0x3210u;
#pragma unroll
  for (int k = 0; k < NC / 2 - 1; ++k) {
    const uint32_t off = E_off(T0 - 4u * k, rowb, r7);
    *reinterpret_cast<uint32_t *>(E + off) = prmt(pk[k], pk[k + 1], sel);
    if (ZERO) *reinterpret_cast<uint32_t *>(E + (off ^ 0x8000u)) = 0u;
  }
  if (!ev) {
    const uint32_t off = E_off(T0 - 4u * (NC / 2 - 1), rowb, r7);
    *reinterpret_cast<uint32_t *>(E + off) = pk[NC / 2 - 1];
    if (ZERO) *reinterpret_cast<uint32_t *>(E + (off ^ 0x8000u)) = 0u;
  } else {
    const uint32_t o0 = E_off(2u * C0, rowb, r7), o1 = E_off(2u * (C0 - NC), rowb, r7) + 2u;
    *reinterpret_cast<uint16_t *>(E + o0) = (uint16_t)(pk[0] >> 16);
    if (ZERO) *reinterpret_cast<uint16_t *>(E + (o0 ^ 0x8000u)) = 0;
    *reinterpret_cast<uint16_t *>(E + o1) = (uint16_t)(pk[NC / 2 - 1] & 0xFFFFu);
    if (ZERO) *reinterpret_cast<uint16_t *>(E + (o1 ^ 0x8000u)) = 0;
  }
}

// Offset block b of r (rows 128 b + off .. +127) exists unless causal and b < 0.
__device__ __forceinline__ bool block_valid(const Prm &p, int b) { return !(p.causal && b < 0); }
__device__ __forceinline__ int slot3(int b) { return ((b % 3) + 3) % 3; }

// ============================================================================
// key-tile kernel: dK, dV, column sums of dS
// ============================================================================
namespace kv {
// relation blocks in a 2-slot ring (block b in slot b & 1): the load of block D + 1
// replaces block D - 1 only after T(t), its last reader, has been consumed
constexpr int OFF_K = 0, OFF_V = 16384, OFF_Q = 32768, OFF_DO = OFF_Q + 32768, OFF_R = OFF_DO + 32768;
constexpr int OFF_ROT = OFF_R + 2 * 16384;            // rot rows; P tile at +0, dS tile at +32768
// 128 x 64 bf16 ones in the MN-major 128-byte-swizzled layout: the second N atom of
// the dK MMA's B operand [Q_m | 1], so that columns 64..79 of dK give c = dS^T 1
constexpr int OFF_ONES = OFF_ROT + 128 * ROT_LD * 4;
// uk[128] (then the du column sums), then per-tile row / offset terms, double-buffered:
// [lse2 | D | v.r block D | v.r block D - 1] x 128
constexpr int OFF_VEC = OFF_ONES + 16384;
constexpr int OFF_BAR = OFF_VEC + 8192;
constexpr int SMEM = OFF_BAR + 256 + 1024;
static_assert(OFF_ONES % 1024 == 0, "swizzled operand tiles are 1024-byte aligned");
enum { B_KV = 0, B_ST0, B_ST1, B_TFULL, B_TCONS, B_SDP, B_SDPCONS, B_PDS, B_PDSFREE, B_DRAIN, NB };
constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 320;  // dK | c: 80 columns
}  // namespace kv

__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_kv_kernel(const __grid_constant__ BwdArgs A) {
  using namespace kv;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 1-D grid: key tiles with the most causal query tiles first, over every head
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, n = (int)blockIdx.x / BH, h = bh % p.H;
  const int L = p.L, j0 = n * 128;
  // query tiles holding only Transformer-XL memory placeholders (rows < mem_len) are skipped
  const int mStart = max(p.causal ? n : 0, p.mem_len / 128), iters = p.nT - mStart;
  const int klen = key_len(p, bh / p.H);  // keys j >= klen of this batch are masked
  if (j0 >= klen) {  // a key tile of padding only: dK = dV = 0, no du contribution (whole CTA, no barrier yet)
    for (int x = tid; x < 128 * (HD / 8); x += NTHREADS) {
      const int r = x / (HD / 8), c8 = x % (HD / 8);
      if (j0 + r < L) {
        const size_t off = ((size_t)bh * L + j0 + r) * HD + 8 * c8;
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dk + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dv + off) = make_uint4(0, 0, 0, 0);
      }
    }
    if (tid < HD) A.part_kv[((size_t)bh * p.nT + n) * HD + tid] = 0.f;
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
    mbar_init(BAR(B_KV), 1);
    mbar_init(BAR(B_ST0), 1);
    mbar_init(BAR(B_ST1), 1);
    mbar_init(BAR(B_TFULL), 1);
    mbar_init(BAR(B_TCONS), NSOFT);
    mbar_init(BAR(B_SDP), 1);
    mbar_init(BAR(B_SDPCONS), NSOFT);
    mbar_init(BAR(B_PDS), NSOFT);
    mbar_init(BAR(B_PDSFREE), 1);
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  // all-ones B operand for the column sums (any swizzle of all-ones is all-ones)
  for (int x = tid; x < 16384 / 16; x += NTHREADS) {
    const uint32_t one2 = 0x3F803F80u;
    *reinterpret_cast<uint4 *>(smem + OFF_ONES + 16 * x) = make_uint4(one2, one2, one2, one2);
  }
  if (tid < 128) vec[tid] = (j0 + tid < L) ? A.uk[(size_t)bh * L + j0 + tid] * c1 : 0.f;  // u.k, pre-scaled
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
      prefetch_tmap(&A.mr);
      const uint32_t idS = idesc_bf16(128, 128, false);
      const uint32_t idAcc = idesc_bf16(128, 64, true, true);
      const uint32_t idK = idesc_bf16(128, 80, true, true);
      ctl.expect(BAR(B_KV), 0, 32768);
      tma_load_3d(sbase + OFF_K, &A.mk, BAR(B_KV), 0, j0, bh);
      tma_load_3d(sbase + OFF_V, &A.mv, BAR(B_KV), 0, j0, bh);
      auto issue_stage = [&](int t) {
        const int m = mStart + t, D = m - n, st = t & 1;
        const bool bA = block_valid(p, D), bB = (t == 0) && block_valid(p, D - 1);
        ctl.expect(BAR(B_ST0 + st), (uint32_t)((t >> 1) & 1), 32768u + (bA ? 16384u : 0u) + (bB ? 16384u : 0u));
        tma_load_3d(sbase + OFF_Q + 16384 * st, &A.mq, BAR(B_ST0 + st), 0, m * 128, bh);
        tma_load_3d(sbase + OFF_DO + 16384 * st, &A.mdo, BAR(B_ST0 + st), 0, m * 128, bh);
        if (bA) tma_load_3d(sbase + OFF_R + 16384 * (D & 1), &A.mr, BAR(B_ST0 + st), 0, 128 * D + p.off, h);
        if (bB) tma_load_3d(sbase + OFF_R + 16384 * ((D - 1) & 1), &A.mr, BAR(B_ST0 + st), 0, 128 * (D - 1) + p.off, h);
      };
      auto accumulate = [&](int t) {  // dV += P^T dO, [dK | c] += dS^T [Q | 1] of tile t (P, dS in smem)
        const int st = t & 1;
        const uint32_t lbo = (uint32_t)(OFF_ONES - OFF_Q - 16384 * st);  // Q atom -> ones atom
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t acc = (t > 0 || k > 0) ? 1u : 0u;
          umma_bf16(tbase + T_DV, sdesc_sw128(sbase + OFF_ROT + 2048 * k, 16384, 1024),
                    sdesc_sw128(sbase + OFF_DO + 16384 * st + 2048 * k, 16, 1024), idAcc, acc);
          umma_bf16(tbase + T_DK, sdesc_sw128(sbase + OFF_ROT + 32768 + 2048 * k, 16384, 1024),
                    sdesc_sw128(sbase + OFF_Q + 16384 * st + 2048 * k, lbo, 1024), idK, acc);
        }
        umma_commit(BAR(B_PDSFREE));
      };
      // relation products of tile t, transposed (lane = offset, column = query row);
      // they overwrite S / dP of tile t - 1, which the rows have read by then
      auto issue_T = [&](int t) {
        const int D = mStart + t - n, st = t & 1;
        if (block_valid(p, D)) umma_k64(tbase + 0, sbase + OFF_R + 16384 * (D & 1), sbase + OFF_Q + 16384 * st, idS, false);
        if (block_valid(p, D - 1))
          umma_k64(tbase + 128, sbase + OFF_R + 16384 * ((D - 1) & 1), sbase + OFF_Q + 16384 * st, idS, false);
        umma_commit(BAR(B_TFULL));
      };
      issue_stage(0);
      bool ok = ctl.wait_load(BAR(B_ST0), 0) && ctl.wait_load(BAR(B_KV), 0);
      if (ok) {
        tc_fence_after();
        issue_T(0);
      }
      for (int t = 0; ok && t < iters; ++t) {
        const int st = t & 1;
        if (!ctl.wait(BAR(B_TCONS), t & 1)) break;
        tc_fence_after();
        umma_k64(tbase + T_S, sbase + OFF_Q + 16384 * st, sbase + OFF_K, idS, false);
        umma_k64(tbase + T_DP, sbase + OFF_DO + 16384 * st, sbase + OFF_V, idS, false);
        umma_commit(BAR(B_SDP));
        if (t == 0 && iters > 1) issue_stage(1);  // T(0) consumed: block D0 - 1's slot is free
        if (t + 1 < iters) {  // S / dP(t) read by the rows: T(t + 1) overlaps their P / dS stores
          if (!ctl.wait(BAR(B_SDPCONS), t & 1)) break;
          if (!ctl.wait_load(BAR(B_ST0 + (st ^ 1)), ((t + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_T(t + 1);
        }
        if (!ctl.wait(BAR(B_PDS), t & 1)) break;
        tc_fence_after();
        accumulate(t);
        if (t + 2 < iters) {  // Q / dO of tile t and relation block D (last read by T(t + 1)) are free
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
    float *rrow = rot + il * ROT_LD;
    bool good = true;
    // per-tile terms staged through smem one tile ahead, one element per thread:
    // [lse2 of the 128 rows | D of the rows | c1 v.r of block D's 128 offsets | same, block D - 1]
    auto fetch1 = [&](int t) {
      const int m = mStart + t, D = m - n, r = tid & 127, w = tid >> 7;
      const int i = m * 128 + r, ro = 128 * (w == 2 ? D : D - 1) + r + p.off;
      if (w == 0) return lse2_of(p, bh, i);
      if (w == 1) return (i < L) ? p.Dvec[(size_t)bh * L + i] : 0.f;
      return (ro >= 0 && ro < p.nrows) ? A.vr[(size_t)h * p.nrows + ro] * c1 : 0.f;
    };
    vec[128 + tid] = fetch1(0);
    named_bar_sync(1, NSOFT);  // tile 0's terms; later tiles' are written before the previous tile's last barrier
    for (int t = 0; t < iters; ++t) {
      const int m = mStart + t, D = m - n, i = m * 128 + il;
      const float *tv = vec + 128 + 512 * (t & 1);
      const float nv = (t + 1 < iters) ? fetch1(t + 1) : 0.f;
      good = good && warp_wait(BAR(B_TFULL), t & 1, abort_flag, status);
      if (t >= 1) good = good && warp_wait(BAR(B_PDSFREE), (t - 1) & 1, abort_flag, status);
      const bool hasA = block_valid(p, D), hasB = block_valid(p, D - 1);
      if (good) {
        tc_fence_after();
        if (hasA) {
          txl_skew<ROT_LD>(tl, 0, 128, hasB, g, qt, lane, c1, tv[256 + il], tv[384 + il], rot);
        } else {
#pragma unroll
          for (int c = 0; c < NC; ++c) rrow[(il - cb - c) & 127] = 0.f;
        }
        tc_fence_before();
        mbar_arrive(BAR(B_TCONS));
      }
      named_bar_sync(1, NSOFT);
      good = good && warp_wait(BAR(B_SDP), t & 1, abort_flag, status);
      // P and dS of this thread's NC keys, packed to bf16 pairs as they are made
      uint32_t pk[NC / 2], dk[NC / 2];
      const bool need_mask = (p.causal && m == n) || (j0 + 128 > klen);
      if (good) {
        tc_fence_after();
        const float lse2 = tv[il], Dv = tv[128 + il];
        const uint64_t c12 = f2(c1, c1), nlse = f2(-lse2, -lse2), nDv = f2(-Dv, -Dv);
        auto pds = [&](auto masked) {
#pragma unroll
          for (int hq = 0; hq < NC / 8; ++hq) {
            uint32_t rs[8], rp[8];
            tmem_ld8(tl + T_S + cb + 8 * hq, rs);
            tmem_ld8(tl + T_DP + cb + 8 * hq, rp);
            tmem_wait_ld();
#pragma unroll
            for (int c4 = 0; c4 < 2; ++c4) {
              const int x0 = 8 * hq + 4 * c4;
              const float4 rr = *reinterpret_cast<const float4 *>(rrow + cb + x0);
              const float4 uk = *reinterpret_cast<const float4 *>(vec + cb + x0);
              float y[4], pr[4], dd[4];
              score_pairs(rs + 4 * c4, rr, uk, c12, nlse, y);
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
        if (need_mask) pds(std::true_type{}); else pds(std::false_type{});
        tc_fence_before();
        mbar_arrive(BAR(B_SDPCONS));  // S / dP read: T(t + 1) may overwrite them
      }
      // tile t + 1's terms into the other buffer (tile t - 1's, read before the previous
      // tile's last barrier); the barrier below makes them visible
      vec[128 + 512 * ((t + 1) & 1) + tid] = nv;
      named_bar_sync(1, NSOFT);  // every rot row read; the P / dS tiles overwrite them
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
    }
    // ---- epilogue: lanes are keys now; this thread takes 16 of the 64 columns ----
    good = good && warp_wait(BAR(B_PDSFREE), (iters - 1) & 1, abort_flag, status);
    const int j = j0 + il;
    float csum = 0.f;
    if (good) {
      tc_fence_after();
      uint32_t rv[16], rk[16], rc[16];
      tmem_ld16(tl + T_DV + 16 * qt, rv);
      tmem_ld16(tl + T_DK + 16 * qt, rk);
      tmem_ld16(tl + T_DK + 64, rc);
      tmem_wait_ld();
      csum = u2f(rc[0]);
      if (j < L) {
        const __nv_bfloat16 *u = (const __nv_bfloat16 *)p.rel1 + (size_t)h * HD + 16 * qt;
        __nv_bfloat16 *dvp = (__nv_bfloat16 *)p.dv + ((size_t)bh * L + j) * HD + 16 * qt;
        __nv_bfloat16 *dkp = (__nv_bfloat16 *)p.dk + ((size_t)bh * L + j) * HD + 16 * qt;
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          float kv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) kv[e] = p.scale * (u2f(rk[8 * c8 + e]) + csum * __bfloat162float(u[8 * c8 + e]));
          uint4 wv, wk;
          wv.x = pack_bf16x2(u2f(rv[8 * c8 + 0]), u2f(rv[8 * c8 + 1]));
          wv.y = pack_bf16x2(u2f(rv[8 * c8 + 2]), u2f(rv[8 * c8 + 3]));
          wv.z = pack_bf16x2(u2f(rv[8 * c8 + 4]), u2f(rv[8 * c8 + 5]));
          wv.w = pack_bf16x2(u2f(rv[8 * c8 + 6]), u2f(rv[8 * c8 + 7]));
          wk.x = pack_bf16x2(kv[0], kv[1]);
          wk.y = pack_bf16x2(kv[2], kv[3]);
          wk.z = pack_bf16x2(kv[4], kv[5]);
          wk.w = pack_bf16x2(kv[6], kv[7]);
          if (dcheck((size_t)(dvp + 8 * c8 - (__nv_bfloat16 *)p.dv) + 8 <= (size_t)BH * L * HD, status)) {
            *reinterpret_cast<uint4 *>(dvp + 8 * c8) = wv;
            *reinterpret_cast<uint4 *>(dkp + 8 * c8) = wk;
          }
        }
      } else {
        csum = 0.f;
      }
    }
    // du partial: s * sum_j c_j k_j over this key tile (fixed order)
    named_bar_sync(1, NSOFT);
    if (qt == 0) vec[il] = csum;
    named_bar_sync(1, NSOFT);
    if (tid < HD) {
      const __nv_bfloat16 *kp = (const __nv_bfloat16 *)p.k + (size_t)bh * L * HD;
      float acc = 0.f;
      for (int jj = 0; jj < 128 && j0 + jj < L; ++jj) acc = fmaf(vec[jj], __bfloat162float(kp[(size_t)(j0 + jj) * HD + tid]), acc);
      A.part_kv[((size_t)bh * p.nT + n) * HD + tid] = p.scale * acc;
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
// key-tile kernel from stored P / dS: dV += P^T dO, [dK | c] += dS^T [Q | 1] streaming the
// query-tile kernel's tiles (no recompute); the same epilogue as tc_bwd_kv_kernel
// ============================================================================
namespace kvs {
constexpr int OFF_P = 0;                    // 2 stages x 64 KB: P (two 64-key halves), dS at +32 KB
constexpr int OFF_Q = 2 * 65536;            // 2 stages x 16 KB
constexpr int OFF_DO = OFF_Q + 32768;       // 2 stages x 16 KB
constexpr int OFF_ONES = OFF_DO + 32768;    // 128 x 64 bf16 ones (second N atom of [Q | 1])
constexpr int OFF_VEC = OFF_ONES + 16384;   // c_j of the tile's keys (du)
constexpr int OFF_BAR = OFF_VEC + 512;
constexpr int SMEM = OFF_BAR + 256 + 1024;
constexpr int NTH = 160;  // four epilogue warps (TMEM lane quarters = keys) and one control warp
enum { B_LD0 = 0, B_LD1, B_FR0, B_FR1, B_DONE, B_DRAIN, NB };
constexpr uint32_t T_DV = 0, T_DK = 64;  // dK | c: 80 columns
}  // namespace kvs

// Body of the key-tile role for CTA index `cta` of its role.  Warps 0-3 (epilogue) and 4
// (control) work; any further warps of the block only pass its two block barriers.
__device__ __forceinline__ void kvs_body(const BwdArgs &A, uint8_t *smem, int cta) {
  using namespace kvs;
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nth = (int)blockDim.x;
  const int BH = p.B * p.H;
  const int bh = cta % BH, n = cta / BH, h = bh % p.H;
  const int L = p.L, j0 = n * 128;
  // query tiles holding only Transformer-XL memory placeholders (rows < mem_len) are skipped
  const int mStart = max(p.causal ? n : 0, p.mem_len / 128), iters = p.nT - mStart;
  const int klen = key_len(p, bh / p.H);
  if (j0 >= klen) {  // a key tile of padding only: dK = dV = 0, no du contribution (whole CTA, no barrier yet)
    for (int x = tid; x < 128 * (HD / 8); x += nth) {
      const int r = x / (HD / 8), c8 = x % (HD / 8);
      if (j0 + r < L) {
        const size_t off = ((size_t)bh * L + j0 + r) * HD + 8 * c8;
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dk + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dv + off) = make_uint4(0, 0, 0, 0);
      }
    }
    if (tid < HD) A.part_kv[((size_t)bh * p.nT + n) * HD + tid] = 0.f;
    return;
  }
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NB + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NB);
  float *vec = (float *)(smem + OFF_VEC);
  int32_t *status = p.status;
  if (tid == 0) {
    for (int k = 0; k < NB; ++k) mbar_init(BAR(k), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int x = tid; x < 16384 / 16; x += nth) {
    const uint32_t one2 = 0x3F803F80u;
    *reinterpret_cast<uint4 *>(smem + OFF_ONES + 16 * x) = make_uint4(one2, one2, one2, one2);
  }
  fence_async_smem();
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  if (warp == 4) {
    if (lane == 0) {
      Ctl ctl;
      ctl.np = 0;
      ctl.ab = abort_flag;
      ctl.st = status;
      prefetch_tmap(&A.mpd);
      prefetch_tmap(&A.mq);
      prefetch_tmap(&A.mdo);
      const uint32_t idAcc = idesc_bf16(128, 64, true, true);
      const uint32_t idK = idesc_bf16(128, 80, true, true);
      auto issue = [&](int t) {
        const int st = t & 1, m = mStart + t, pl = tile_plane(p, bh, m, n);
        ctl.expect(BAR(B_LD0 + st), (uint32_t)((t >> 1) & 1), 65536u + 32768u);
#pragma unroll
        for (int q = 0; q < 4; ++q) tma_load_3d(sbase + OFF_P + 65536 * st + 16384 * q, &A.mpd, BAR(B_LD0 + st), 0, 0, pl + q);
        tma_load_3d(sbase + OFF_Q + 16384 * st, &A.mq, BAR(B_LD0 + st), 0, m * 128, bh);
        tma_load_3d(sbase + OFF_DO + 16384 * st, &A.mdo, BAR(B_LD0 + st), 0, m * 128, bh);
      };
      issue(0);
      if (iters > 1) issue(1);
      for (int t = 0; t < iters; ++t) {
        const int st = t & 1;
        if (!ctl.wait_load(BAR(B_LD0 + st), (uint32_t)((t >> 1) & 1))) break;
        tc_fence_after();
        const uint32_t lbo = (uint32_t)(OFF_ONES - OFF_Q - 16384 * st);  // Q atom -> ones atom
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t acc = (t > 0 || k > 0) ? 1u : 0u;
          umma_bf16(tbase + T_DV, sdesc_sw128(sbase + OFF_P + 65536 * st + 2048 * k, 16384, 1024),
                    sdesc_sw128(sbase + OFF_DO + 16384 * st + 2048 * k, 16, 1024), idAcc, acc);
          umma_bf16(tbase + T_DK, sdesc_sw128(sbase + OFF_P + 65536 * st + 32768 + 2048 * k, 16384, 1024),
                    sdesc_sw128(sbase + OFF_Q + 16384 * st + 2048 * k, lbo, 1024), idK, acc);
        }
        umma_commit(BAR(B_FR0 + st));
        if (t + 2 < iters) {  // this stage is free once its MMAs are done
          if (!ctl.wait(BAR(B_FR0 + st), (uint32_t)((t >> 1) & 1))) break;
          issue(t + 2);
        }
      }
      umma_commit(BAR(B_DONE));
      ctl.drain(BAR(B_DRAIN));
    }
    __syncwarp();
  } else if (warp < 4) {  // epilogue: lane il is key j0 + il; this thread takes all 64 columns
    const int il = 32 * warp + lane, j = j0 + il;
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    float csum = 0.f;
    if (warp_wait(BAR(B_DONE), 0, abort_flag, status)) {
      tc_fence_after();
      uint32_t c8r[8];
      tmem_ld8(tl + T_DK + 64, c8r);
      tmem_wait_ld();
      csum = j < L ? u2f(c8r[0]) : 0.f;
      const __nv_bfloat16 *u = (const __nv_bfloat16 *)p.rel1 + (size_t)h * HD;
#pragma unroll
      for (int c0 = 0; c0 < HD; c0 += 32) {
        uint32_t rv[32], rk[32];
        tmem_ld32(tl + T_DV + c0, rv);
        tmem_ld32(tl + T_DK + c0, rk);
        tmem_wait_ld();
        if (j < L) {
          __nv_bfloat16 *dvp = (__nv_bfloat16 *)p.dv + ((size_t)bh * L + j) * HD + c0;
          __nv_bfloat16 *dkp = (__nv_bfloat16 *)p.dk + ((size_t)bh * L + j) * HD + c0;
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float kv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) kv[e] = p.scale * (u2f(rk[8 * c8 + e]) + csum * __bfloat162float(u[c0 + 8 * c8 + e]));
            uint4 wv, wk;
            wv.x = pack_bf16x2(u2f(rv[8 * c8 + 0]), u2f(rv[8 * c8 + 1]));
            wv.y = pack_bf16x2(u2f(rv[8 * c8 + 2]), u2f(rv[8 * c8 + 3]));
            wv.z = pack_bf16x2(u2f(rv[8 * c8 + 4]), u2f(rv[8 * c8 + 5]));
            wv.w = pack_bf16x2(u2f(rv[8 * c8 + 6]), u2f(rv[8 * c8 + 7]));
            wk.x = pack_bf16x2(kv[0], kv[1]);
            wk.y = pack_bf16x2(kv[2], kv[3]);
            wk.z = pack_bf16x2(kv[4], kv[5]);
            wk.w = pack_bf16x2(kv[6], kv[7]);
            if (dcheck((size_t)(dvp + 8 * c8 - (__nv_bfloat16 *)p.dv) + 8 <= (size_t)BH * L * HD, status)) {
              *reinterpret_cast<uint4 *>(dvp + 8 * c8) = wv;
              *reinterpret_cast<uint4 *>(dkp + 8 * c8) = wk;
            }
          }
        }
      }
    }
    // du partial: s * sum_j c_j k_j over this key tile (fixed order)
    vec[il] = csum;
    named_bar_sync(1, 128);
    if (tid < HD) {
      const __nv_bfloat16 *kp = (const __nv_bfloat16 *)p.k + (size_t)bh * L * HD;
      float acc = 0.f;
      for (int jj = 0; jj < 128 && j0 + jj < L; ++jj) acc = fmaf(vec[jj], __bfloat162float(kp[(size_t)(j0 + jj) * HD + tid]), acc);
      A.part_kv[((size_t)bh * p.nT + n) * HD + tid] = p.scale * acc;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

__global__ void __launch_bounds__(kvs::NTH, 1) tc_bwd_kvs_kernel(const __grid_constant__ BwdArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  kvs_body(A, (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023), (int)blockIdx.x);
}

// ============================================================================
// query-tile kernel: dQ
// ============================================================================
namespace qk {
constexpr int OFF_Q = 0, OFF_DO = 16384, OFF_K = 32768, OFF_V = OFF_K + 32768, OFF_R = OFF_V + 32768;
constexpr int OFF_ROT = OFF_R + 3 * 16384;  // rot rows; E_lo at +0, E_hi at +32768
constexpr int OFF_VEC = OFF_ROT + 128 * ROT_LD * 4;
constexpr int OFF_BAR = OFF_VEC + 4096;
constexpr int SMEM = OFF_BAR + 256 + 1024;
enum { B_QD = 0, B_ST0, B_ST1, B_SFULL, B_TCONS, B_DPF, B_DPCONS, B_PDS, B_PDSFREE, B_DSFREE, B_DRAIN, NB };
constexpr uint32_t T_S = 0, T_REL = 128, T_DQ = 384, T_DS = 448;
}  // namespace qk

__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_q_kernel(const __grid_constant__ BwdArgs A) {
  using namespace qk;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, m = p.nT - 1 - (int)blockIdx.x / BH, h = bh % p.H;
  const int L = p.L, i0 = m * 128;
  const int klen = key_len(p, bh / p.H);  // keys j >= klen of this batch are masked; their tiles skipped
  const int nTiles = min(p.causal ? m + 1 : p.nT, (klen + 127) / 128);
  if (nTiles == 0) {  // no key at all: dQ = 0 (whole CTA, before any barrier)
    for (int x = tid; x < 128 * (HD / 8); x += NTHREADS) {
      const int r = x / (HD / 8), c8 = x % (HD / 8);
      if (i0 + r < L)
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.dq + ((size_t)bh * L + i0 + r) * HD + 8 * c8) = make_uint4(0, 0, 0, 0);
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
    mbar_init(BAR(B_QD), 1);
    mbar_init(BAR(B_ST0), 1);
    mbar_init(BAR(B_ST1), 1);
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_TCONS), NSOFT);
    mbar_init(BAR(B_DPF), 1);
    mbar_init(BAR(B_DPCONS), NSOFT);
    mbar_init(BAR(B_PDS), NSOFT);
    mbar_init(BAR(B_PDSFREE), 1);
    mbar_init(BAR(B_DSFREE), 1);
    mbar_init(BAR(B_DRAIN), 1);
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
      prefetch_tmap(&A.mr);
      const uint32_t idS = idesc_bf16(128, 128, false);
      const uint32_t idDQ = idesc_bf16(128, 64, true);
      ctl.expect(BAR(B_QD), 0, 32768);
      tma_load_3d(sbase + OFF_Q, &A.mq, BAR(B_QD), 0, i0, bh);
      tma_load_3d(sbase + OFF_DO, &A.mdo, BAR(B_QD), 0, i0, bh);
      auto issue_stage = [&](int n) {  // K_n, V_n and the relation block tile n adds
        const int st = n & 1, D = m - n;
        const bool b0 = (n == 0) && block_valid(p, D), b1 = block_valid(p, D - 1);
        ctl.expect(BAR(B_ST0 + st), (uint32_t)((n >> 1) & 1), 32768u + (b0 ? 16384u : 0u) + (b1 ? 16384u : 0u));
        tma_load_3d(sbase + OFF_K + 16384 * st, &A.mk, BAR(B_ST0 + st), 0, n * 128, bh);
        tma_load_3d(sbase + OFF_V + 16384 * st, &A.mv, BAR(B_ST0 + st), 0, n * 128, bh);
        if (b0) tma_load_3d(sbase + OFF_R + 16384 * slot3(D), &A.mr, BAR(B_ST0 + st), 0, 128 * D + p.off, h);
        if (b1) tma_load_3d(sbase + OFF_R + 16384 * slot3(D - 1), &A.mr, BAR(B_ST0 + st), 0, 128 * (D - 1) + p.off, h);
      };
      issue_stage(0);
      if (nTiles > 1) issue_stage(1);
      bool ok = ctl.wait_load(BAR(B_QD), 0) && ctl.wait_load(BAR(B_ST0), 0);
      if (ok) {
        tc_fence_after();
        umma_k64(tbase + T_S, sbase + OFF_Q, sbase + OFF_K, idS, false);
        // relation products transposed (lane = offset, column = query row)
        if (block_valid(p, m)) umma_k64(tbase + T_REL + 128 * (m & 1), sbase + OFF_R + 16384 * slot3(m), sbase + OFF_Q, idS, false);
        if (block_valid(p, m - 1))
          umma_k64(tbase + T_REL + 128 * ((m - 1) & 1), sbase + OFF_R + 16384 * slot3(m - 1), sbase + OFF_Q, idS, false);
        umma_commit(BAR(B_SFULL));
      }
      for (int n = 0; ok && n < nTiles; ++n) {
        const int st = n & 1, D = m - n;
        const uint32_t slotA = T_REL + 128 * (D & 1);  // block D's products; reused for dP(n)
        if (!ctl.wait(BAR(B_TCONS), n & 1)) break;
        tc_fence_after();
        umma_k64(tbase + slotA, sbase + OFF_DO, sbase + OFF_V + 16384 * st, idS, false);  // dP(n)
        umma_commit(BAR(B_DPF));
        if (n + 1 < nTiles) {
          if (!ctl.wait_load(BAR(B_ST0 + (st ^ 1)), ((n + 1) >> 1) & 1)) break;
          umma_k64(tbase + T_S, sbase + OFF_Q, sbase + OFF_K + 16384 * (st ^ 1), idS, false);  // S(n+1)
          // relation block D - 2 for tile n + 1 into the slot dP(n) used, once the rows have
          // read dP(n): it runs under their dS / E stores
          if (!ctl.wait(BAR(B_DPCONS), n & 1)) break;
          tc_fence_after();
          if (block_valid(p, D - 2))
            umma_k64(tbase + slotA, sbase + OFF_R + 16384 * slot3(D - 2), sbase + OFF_Q, idS, false);
          umma_commit(BAR(B_SFULL));
        }
        if (!ctl.wait(BAR(B_PDS), n & 1)) break;
        tc_fence_after();
        // dQ += E_lo r_D + E_hi r_{D-1} (E in smem, freed first so the rows can skew the
        // next tile), then dQ += dS K_n (dS in TMEM)
        uint32_t acc = n > 0 ? 1u : 0u;
        if (block_valid(p, D)) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_bf16(tbase + T_DQ, sdesc_sw128(sbase + OFF_ROT + 16384 * (k >> 2) + 32 * (k & 3), 16, 1024),
                      sdesc_sw128(sbase + OFF_R + 16384 * slot3(D) + 2048 * k, 16, 1024), idDQ, (acc || k > 0) ? 1u : 0u);
          acc = 1u;
        }
        if (block_valid(p, D - 1)) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_bf16(tbase + T_DQ, sdesc_sw128(sbase + OFF_ROT + 32768 + 16384 * (k >> 2) + 32 * (k & 3), 16, 1024),
                      sdesc_sw128(sbase + OFF_R + 16384 * slot3(D - 1) + 2048 * k, 16, 1024), idDQ, (acc || k > 0) ? 1u : 0u);
          acc = 1u;
        }
        umma_commit(BAR(B_PDSFREE));
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_bf16_ts(tbase + T_DQ, tbase + T_DS + 8 * k, sdesc_sw128(sbase + OFF_K + 16384 * st + 2048 * k, 16, 1024), idDQ,
                       (acc || k > 0) ? 1u : 0u);
        umma_commit(BAR(B_DSFREE));
        if (n + 2 < nTiles) {  // K_n, V_n and the tile's relation block slot are free once dS K_n is done
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
    float *rrow = rot + il * ROT_LD;
    const float lse2 = lse2_of(p, bh, i);
    const float Dv = (i < L) ? p.Dvec[(size_t)bh * L + i] : 0.f;
    const uint64_t c12 = f2(c1, c1), nlse = f2(-lse2, -lse2), nDv = f2(-Dv, -Dv);
    bool good = true;
    // per key tile, staged through smem one tile ahead (one element per thread, double-
    // buffered): [c1 u.k of the keys | c1 v.r of block D's offsets | same, block D - 1]
    auto fetch1 = [&](int n) {
      const int j0 = n * 128, D = m - n, r = tid & 127, w = tid >> 7;
      if (w == 0) return (j0 + r < L) ? A.uk[(size_t)bh * L + j0 + r] * c1 : 0.f;
      const int ro = 128 * (w == 1 ? D : D - 1) + r + p.off;
      return (ro >= 0 && ro < p.nrows) ? A.vr[(size_t)h * p.nrows + ro] * c1 : 0.f;
    };
    if (tid < 384) vec[tid] = fetch1(0);
    named_bar_sync(1, NSOFT);  // tile 0's terms; later tiles' are written before the previous tile's last barrier
    for (int n = 0; n < nTiles; ++n) {
      const int j0 = n * 128, D = m - n;
      const float *tu = vec + 384 * (n & 1);
      const float nv = (tid < 384 && n + 1 < nTiles) ? fetch1(n + 1) : 0.f;
      good = good && warp_wait(BAR(B_SFULL), n & 1, abort_flag, status);
      if (n >= 1) good = good && warp_wait(BAR(B_PDSFREE), (n - 1) & 1, abort_flag, status);
      const bool hasA = block_valid(p, D), hasB = block_valid(p, D - 1);
      float x[NC];
      if (good) {
        tc_fence_after();
        if (hasA) {
          txl_skew<ROT_LD>(tl, T_REL + 128 * (D & 1), T_REL + 128 * ((D - 1) & 1), hasB, g, qt, lane, c1, tu[128 + il],
                           tu[256 + il], rot);
        } else {
#pragma unroll
          for (int c = 0; c < NC; ++c) rrow[(il - cb - c) & 127] = 0.f;
        }
        uint32_t r[32];
        tmem_ld32(tl + T_S + cb, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < NC; ++e) x[e] = u2f(r[e]);
        tc_fence_before();
        mbar_arrive(BAR(B_TCONS));
      } else {
#pragma unroll
        for (int e = 0; e < NC; ++e) x[e] = 0.f;
      }
      named_bar_sync(1, NSOFT);
      const bool need_mask = (p.causal && n == m) || (j0 + 128 > klen);
      auto probs = [&](auto masked) {  // x <- P = 2^(s c1 + r' + u' - lse2)
#pragma unroll
        for (int c4 = 0; c4 < NC / 4; ++c4) {
          const float4 rr = *reinterpret_cast<const float4 *>(rrow + cb + 4 * c4);
          const float4 uk = *reinterpret_cast<const float4 *>(tu + cb + 4 * c4);
          const uint32_t sb[4] = {__float_as_uint(x[4 * c4]), __float_as_uint(x[4 * c4 + 1]), __float_as_uint(x[4 * c4 + 2]),
                                  __float_as_uint(x[4 * c4 + 3])};
          float y[4];
          score_pairs(sb, rr, uk, c12, nlse, y);
          if constexpr (decltype(masked)::value) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = j0 + cb + 4 * c4 + e;
              if (j >= klen || (p.causal && j > i)) y[e] = -INFINITY;
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) x[4 * c4 + e] = ex2(y[e]);
        }
      };
      if (need_mask) probs(std::true_type{}); else probs(std::false_type{});
      // row-major bf16 P / dS planes of this tile for the key-tile kernel: row il, keys cb .. cb + 31
      __nv_bfloat16 *pdrow = A.pd_stored ? A.pd + (size_t)(tile_plane(p, bh, m, n) + (qt >> 1)) * 8192 + il * 64 + 32 * (qt & 1)
                                         : nullptr;
      // elements of the stored-tile buffer: four 8192-element planes per stored tile
      const size_t pd_elems = (size_t)BH * (p.causal ? p.nT * (p.nT + 1) / 2 : p.nT * p.nT) * 4 * 8192;
      // (pdrow is 64-byte aligned: 16 KB planes, 128-byte rows, 64-byte halves of a row)
      if (A.pd_stored && good && dcheck((size_t)(pdrow - A.pd) + 2 * 8192 + NC <= pd_elems, status)) {
#pragma unroll
        for (int c16 = 0; c16 < NC / 16; ++c16) {
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(x[16 * c16 + 2 * e], x[16 * c16 + 2 * e + 1]);
          st_global_32B(pdrow + 16 * c16, w);
        }
      }
      good = good && warp_wait(BAR(B_DPF), n & 1, abort_flag, status);
      if (good) {
        tc_fence_after();
        uint32_t r[32];
        tmem_ld32(tl + T_REL + 128 * (D & 1) + cb, r);
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < NC / 4; ++c4) {
          const float pr[4] = {x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]};
          float dd[4];
          ds_pairs(pr, r + 4 * c4, nDv, dd);
#pragma unroll
          for (int e = 0; e < 4; ++e) x[4 * c4 + e] = dd[e];
        }
        tc_fence_before();
        mbar_arrive(BAR(B_DPCONS));  // dP(n) read: the next relation block may overwrite it
      }
      // tile n + 1's terms into the other buffer (tile n - 1's, read before the previous
      // tile's last barrier); the barrier below makes them visible
      if (tid < 384) vec[384 * ((n + 1) & 1) + tid] = nv;
      named_bar_sync(1, NSOFT);  // every rot row read: E overwrites them
      if (good) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
        if (A.pd_stored && dcheck((size_t)(pdrow - A.pd) + 2 * 8192 + NC <= pd_elems, status)) {
#pragma unroll
          for (int c16 = 0; c16 < NC / 16; ++c16) st_global_32B(pdrow + 2 * 8192 + 16 * c16, pk + 8 * c16);
        }
        // the previous tile's dS K MMAs read T_DS: wait for them (long done in practice)
        if (n >= 1 && !warp_wait(BAR(B_DSFREE), (n - 1) & 1, abort_flag, status)) good = false;
        if (good) tmem_st16(tl + T_DS + 16 * qt, pk);
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = prmt(pk[e], pk[e], 0x1032u);  // swap halves: (x[2e+1], x[2e])
        store_E(smem + OFF_ROT, il, cb, pk);
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_PDS));
      }
    }
    good = good && warp_wait(BAR(B_DSFREE), (nTiles - 1) & 1, abort_flag, status);  // last dQ MMAs done
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
          if (dcheck((size_t)(dqp + 8 * c8 - (__nv_bfloat16 *)p.dq) + 8 <= (size_t)BH * L * HD, status))
            *reinterpret_cast<uint4 *>(dqp + 8 * c8) = w;
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
// diagonal kernel: per-offset sums G = sum dS q and g = sum dS for dr
// ============================================================================
namespace dg {
constexpr int OFF_Q = 0, OFF_DO = 32768, OFF_K = 65536, OFF_V = OFF_K + 16384, OFF_R = OFF_V + 16384;
constexpr int OFF_ROT = OFF_R + 32768;  // rot rows; E_lo at +0, E_hi at +32768
// 128 x 64 bf16 ones in the MN-major 128-byte-swizzled layout: the second N atom
// of the G MMAs' B operand [Q_m | 1], so that columns 64..79 of G give g = E^T 1
constexpr int OFF_ONES = OFF_ROT + 128 * ROT_LD * 4;
constexpr int OFF_VEC = OFF_ONES + 16384;
constexpr int OFF_BAR = OFF_VEC + 4096;
constexpr int SMEM = OFF_BAR + 256 + 1024;
static_assert(OFF_ONES % 1024 == 0, "swizzled operand tiles are 1024-byte aligned");
enum { B_R = 0, B_ST0, B_ST1, B_KV, B_KVFREE, B_TFULL, B_TCONS, B_SDP, B_SDPCONS, B_PDS, B_PDSFREE, B_DRAIN, NB };
constexpr uint32_t T_S = 0, T_DP = 128, T_GLO = 256, T_GHI = 336;  // G | g: 80 columns each
}  // namespace dg

__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_diag_kernel(const __grid_constant__ BwdArgs A) {
  using namespace dg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 1-D grid: longest bands first (causal: D = 0, 1, ...; otherwise 0, 1, -1, 2, -2, ...)
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, rr0 = (int)blockIdx.x / BH;
  const int chunk = rr0 % A.dg_nchunk, rank = rr0 / A.dg_nchunk;
  const int D = p.causal ? rank : ((rank & 1) ? (rank + 1) / 2 : -(rank / 2));
  const int band = p.causal ? D : D + (p.nT - 1);
  const int b = bh / p.H, h = bh % p.H;
  const int mlo = max(0, D), mhi = min(p.nT - 1, p.nT - 1 + D);
  const int mc = mlo + chunk * A.dg_ch, m1a = min(mhi, mc + A.dg_ch - 1);
  if (mc > m1a) return;  // no such chunk (never read): whole CTA, before any barrier or TMEM allocation
  const int m0 = max(mc, p.mem_len / 128);  // memory-placeholder query tiles are skipped
  // keys j >= klen of this batch are masked: tiles whose key tile m - D lies past them are skipped
  const int klen = key_len(p, bh / p.H);
  const int m1 = min(m1a, (klen + 127) / 128 - 1 + D);
  if (m0 > m1) {  // the chunk's tiles are all padding: a zero partial
    float *part = A.part_dg + (((size_t)bh * A.nbands + band) * A.dg_nchunk + chunk) * DG_STRIDE;
    for (int x = tid; x < DG_STRIDE; x += NTHREADS) part[x] = 0.f;
    return;
  }
  const int iters = m1 - m0 + 1;
  const int L = p.L;
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NB + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NB);
  float *rot = (float *)(smem + OFF_ROT);
  float *vec = (float *)(smem + OFF_VEC);
  int32_t *status = p.status;
  const float c1 = p.scale * LOG2E;
  const bool hasA = block_valid(p, D), hasB = block_valid(p, D - 1);
  (void)b;

  if (tid == 0) {
    for (int k = 0; k < NB; ++k) mbar_init(BAR(k), (k == B_TCONS || k == B_SDPCONS || k == B_PDS) ? NSOFT : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int x = tid; x < 16384 / 16; x += NTHREADS) {
    const uint32_t one2 = 0x3F803F80u;
    *reinterpret_cast<uint4 *>(smem + OFF_ONES + 16 * x) = make_uint4(one2, one2, one2, one2);
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
      prefetch_tmap(&A.mr);
      const uint32_t idS = idesc_bf16(128, 128, false);
      const uint32_t idG = idesc_bf16(128, 80, true, true);
      ctl.expect(BAR(B_R), 0, (hasA ? 16384u : 0u) + (hasB ? 16384u : 0u));
      if (hasA) tma_load_3d(sbase + OFF_R, &A.mr, BAR(B_R), 0, 128 * D + p.off, h);
      if (hasB) tma_load_3d(sbase + OFF_R + 16384, &A.mr, BAR(B_R), 0, 128 * (D - 1) + p.off, h);
      auto issue_qd = [&](int t) {
        const int m = m0 + t, st = t & 1;
        ctl.expect(BAR(B_ST0 + st), (uint32_t)((t >> 1) & 1), 32768);
        tma_load_3d(sbase + OFF_Q + 16384 * st, &A.mq, BAR(B_ST0 + st), 0, m * 128, bh);
        tma_load_3d(sbase + OFF_DO + 16384 * st, &A.mdo, BAR(B_ST0 + st), 0, m * 128, bh);
      };
      auto issue_kv = [&](int t) {
        const int nn = m0 + t - D;
        ctl.expect(BAR(B_KV), (uint32_t)(t & 1), 32768);
        tma_load_3d(sbase + OFF_K, &A.mk, BAR(B_KV), 0, nn * 128, bh);
        tma_load_3d(sbase + OFF_V, &A.mv, BAR(B_KV), 0, nn * 128, bh);
      };
      auto accumulate = [&](int t) {  // [G | g]_lo, [G | g]_hi += E^T [Q_t | 1]
        const int st = t & 1;
        const uint32_t lbo = (uint32_t)(OFF_ONES - OFF_Q - 16384 * st);  // Q atom -> ones atom
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t acc = (t > 0 || k > 0) ? 1u : 0u;
          const uint64_t bq = sdesc_sw128(sbase + OFF_Q + 16384 * st + 2048 * k, lbo, 1024);
          const uint64_t elo = sdesc_sw128(sbase + OFF_ROT + 2048 * k, 16384, 1024);
          const uint64_t ehi = sdesc_sw128(sbase + OFF_ROT + 32768 + 2048 * k, 16384, 1024);
          umma_bf16(tbase + T_GLO, elo, bq, idG, acc);
          umma_bf16(tbase + T_GHI, ehi, bq, idG, acc);
        }
        umma_commit(BAR(B_PDSFREE));
      };
      issue_qd(0);
      issue_kv(0);
      if (iters > 1) issue_qd(1);
      // relation products of tile t, transposed (lane = offset, column = query row);
      // they overwrite S / dP of tile t - 1, which the rows have read by then
      auto issue_T = [&](int t) {
        const int st = t & 1;
        if (hasA) umma_k64(tbase + 0, sbase + OFF_R, sbase + OFF_Q + 16384 * st, idS, false);
        if (hasB) umma_k64(tbase + 128, sbase + OFF_R + 16384, sbase + OFF_Q + 16384 * st, idS, false);
        umma_commit(BAR(B_TFULL));
      };
      bool ok = ctl.wait_load(BAR(B_R), 0) && ctl.wait_load(BAR(B_ST0), 0);
      if (ok) {
        tc_fence_after();
        issue_T(0);
      }
      for (int t = 0; ok && t < iters; ++t) {
        const int st = t & 1;
        if (!ctl.wait(BAR(B_TCONS), t & 1)) break;
        if (!ctl.wait_load(BAR(B_KV), t & 1)) break;
        tc_fence_after();
        umma_k64(tbase + T_S, sbase + OFF_Q + 16384 * st, sbase + OFF_K, idS, false);
        umma_k64(tbase + T_DP, sbase + OFF_DO + 16384 * st, sbase + OFF_V, idS, false);
        umma_commit(BAR(B_SDP));
        umma_commit(BAR(B_KVFREE));
        if (t + 1 < iters) {
          if (!ctl.wait(BAR(B_KVFREE), t & 1)) break;
          issue_kv(t + 1);
          // S / dP(t) read by the rows: T(t + 1) overlaps their dS / E stores
          if (!ctl.wait(BAR(B_SDPCONS), t & 1)) break;
          if (!ctl.wait_load(BAR(B_ST0 + (st ^ 1)), ((t + 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_T(t + 1);
        }
        if (!ctl.wait(BAR(B_PDS), t & 1)) break;
        tc_fence_after();
        accumulate(t);
        if (t + 2 < iters) {  // Q / dO of tile t are free once G(t) is done
          if (!ctl.wait(BAR(B_PDSFREE), t & 1)) break;
          issue_qd(t + 2);
        }
      }
      ctl.drain(BAR(B_DRAIN));
    }
    __syncwarp();
  } else {
    const int g = warp & 3, qt = warp >> 2, il = 32 * g + lane, cb = NC * qt;
    const uint32_t tl = tbase + ((uint32_t)(g * 32) << 16);
    float *rrow = rot + il * ROT_LD;
    bool good = true;
    // smem terms: c1 v.r of the band's two blocks (offset r: [r], [128 + r], fixed), then
    // per tile, double-buffered and staged one tile ahead (one element per thread):
    // [lse2 of the rows | D of the rows | c1 u.k of the keys]
    if (tid < 256) {
      const int ro = 128 * (tid < 128 ? D : D - 1) + (tid & 127) + p.off;
      vec[tid] = (ro >= 0 && ro < p.nrows) ? A.vr[(size_t)h * p.nrows + ro] * c1 : 0.f;
    }
    auto fetch1 = [&](int t) {
      const int m = m0 + t, r = tid & 127, w = tid >> 7, i = m * 128 + r, j = (m - D) * 128 + r;
      if (w == 0) return lse2_of(p, bh, i);
      if (w == 1) return (i < L) ? p.Dvec[(size_t)bh * L + i] : 0.f;
      return (j < L) ? A.uk[(size_t)bh * L + j] * c1 : 0.f;
    };
    if (tid < 384) vec[256 + tid] = fetch1(0);
    named_bar_sync(1, NSOFT);  // the band's terms and tile 0's; later tiles' are written before the previous tile's last barrier
    for (int t = 0; t < iters; ++t) {
      const int m = m0 + t, nn = m - D, i = m * 128 + il, j0 = nn * 128;
      const float *tv = vec + 256 + 384 * (t & 1), *tu = tv + 256;
      const float nv = (tid < 384 && t + 1 < iters) ? fetch1(t + 1) : 0.f;
      good = good && warp_wait(BAR(B_TFULL), t & 1, abort_flag, status);
      if (t >= 1) good = good && warp_wait(BAR(B_PDSFREE), (t - 1) & 1, abort_flag, status);
      if (good) {
        tc_fence_after();
        if (hasA) {
          txl_skew<ROT_LD>(tl, 0, 128, hasB, g, qt, lane, c1, vec[il], vec[128 + il], rot);
        } else {
#pragma unroll
          for (int c = 0; c < NC; ++c) rrow[(il - cb - c) & 127] = 0.f;
        }
        tc_fence_before();
        mbar_arrive(BAR(B_TCONS));
      }
      named_bar_sync(1, NSOFT);
      good = good && warp_wait(BAR(B_SDP), t & 1, abort_flag, status);
      uint32_t ds[NC / 2];  // dS as bf16 pairs (x[2k+1] low, x[2k] high)
      const bool need_mask = (p.causal && m == nn) || (j0 + 128 > klen);
      if (good) {
        tc_fence_after();
        const float lse2 = tv[il], Dv = tv[128 + il];
        const uint64_t c12 = f2(c1, c1), nlse = f2(-lse2, -lse2), nDv = f2(-Dv, -Dv);
        auto pds = [&](auto masked) {
#pragma unroll
          for (int hq = 0; hq < NC / 16; ++hq) {
            uint32_t rs[16], rp[16];
            tmem_ld16(tl + T_S + cb + 16 * hq, rs);
            tmem_ld16(tl + T_DP + cb + 16 * hq, rp);
            tmem_wait_ld();
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const int x0 = 16 * hq + 4 * c4;
              const float4 rr = *reinterpret_cast<const float4 *>(rrow + cb + x0);
              const float4 uk = *reinterpret_cast<const float4 *>(tu + cb + x0);
              float y[4], pr[4], dd[4];
              score_pairs(rs + 4 * c4, rr, uk, c12, nlse, y);
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
              ds[x0 / 2] = pack_bf16x2(dd[1], dd[0]);
              ds[x0 / 2 + 1] = pack_bf16x2(dd[3], dd[2]);
            }
          }
        };
        if (need_mask) pds(std::true_type{}); else pds(std::false_type{});
        tc_fence_before();
        mbar_arrive(BAR(B_SDPCONS));  // S / dP read: T(t + 1) may overwrite them
      } else {
#pragma unroll
        for (int x = 0; x < NC / 2; ++x) ds[x] = 0u;
      }
      // tile t + 1's terms into the other buffer (tile t - 1's, read before the previous
      // tile's last barrier); the barrier below makes them visible
      if (tid < 384) vec[256 + 384 * ((t + 1) & 1) + tid] = nv;
      named_bar_sync(1, NSOFT);  // every rot row read: E overwrites them
      if (good) {
        store_E(smem + OFF_ROT, il, cb, ds);
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_PDS));
      }
    }
    // ---- epilogue: lane il now is offset c = il of both blocks; 16 columns per thread ----
    good = good && warp_wait(BAR(B_PDSFREE), (iters - 1) & 1, abort_flag, status);
    if (good) {
      tc_fence_after();
      uint32_t rlo[16], rhi[16], glo[16], ghi[16];
      tmem_ld16(tl + T_GLO + 16 * qt, rlo);
      tmem_ld16(tl + T_GHI + 16 * qt, rhi);
      tmem_ld16(tl + T_GLO + 64, glo);
      tmem_ld16(tl + T_GHI + 64, ghi);
      tmem_wait_ld();
      // partial layout [block lo / hi][65][128 offsets]: G columns 0..63, then g
      float *part = A.part_dg + (((size_t)bh * A.nbands + band) * A.dg_nchunk + chunk) * DG_STRIDE;
      const bool part_ok = dcheck(
          (size_t)(part - A.part_dg) + DG_STRIDE <= (size_t)BH * A.nbands * A.dg_nchunk * DG_STRIDE, status);
#pragma unroll
      for (int e = 0; e < 16 && part_ok; ++e) {
        part[(size_t)(16 * qt + e) * 128 + il] = u2f(rlo[e]);
        part[(size_t)(65 + 16 * qt + e) * 128 + il] = u2f(rhi[e]);
      }
      if (qt == 0 && part_ok) {
        part[(size_t)64 * 128 + il] = u2f(glo[0]);
        part[(size_t)(65 + 64) * 128 + il] = u2f(ghi[0]);
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
// diagonal kernel from the stored dS tiles: the same partials as tc_bwd_diag_kernel with
// no recompute of S, P or dS -- the rows rebuild E (offset order) from each stored dS tile
// ============================================================================
namespace dgs {
constexpr int OFF_DS = 0;                  // 2 stages x 32 KB: dS (two 64-key halves)
constexpr int OFF_Q = 2 * 32768;           // 2 stages x 16 KB
constexpr int OFF_E = OFF_Q + 32768;       // E_lo, E_hi (64 KB)
constexpr int OFF_ONES = OFF_E + 65536;    // 128 x 64 bf16 ones (second N atom of [Q | 1])
constexpr int OFF_BAR = OFF_ONES + 16384;
constexpr int SMEM = OFF_BAR + 256 + 1024;
enum { B_LD0 = 0, B_LD1, B_EFULL, B_EFREE, B_DRAIN, NB };
constexpr uint32_t T_GLO = 0, T_GHI = 128;  // G | g: 80 columns each
}  // namespace dgs

// Body of the diagonal role for CTA index `cta` of its role (NTHREADS threads).
__device__ __forceinline__ void dgs_body(const BwdArgs &A, uint8_t *smem, int cta) {
  using namespace dgs;
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BH = p.B * p.H;
  const int bh = cta % BH, rr0 = cta / BH;
  const int chunk = rr0 % A.dg_nchunk, rank = rr0 / A.dg_nchunk;
  const int D = p.causal ? rank : ((rank & 1) ? (rank + 1) / 2 : -(rank / 2));
  const int band = p.causal ? D : D + (p.nT - 1);
  const int mlo = max(0, D), mhi = min(p.nT - 1, p.nT - 1 + D);
  const int mc = mlo + chunk * A.dg_ch, m1a = min(mhi, mc + A.dg_ch - 1);
  if (mc > m1a) return;  // no such chunk (never read)
  const int m0 = max(mc, p.mem_len / 128);  // memory-placeholder query tiles are skipped
  const int klen = key_len(p, bh / p.H);
  const int m1 = min(m1a, (klen + 127) / 128 - 1 + D);  // the tiles the query-tile kernel stored
  float *part = A.part_dg + (((size_t)bh * A.nbands + band) * A.dg_nchunk + chunk) * DG_STRIDE;
  if (m0 > m1) {  // the chunk's tiles are all padding: a zero partial
    for (int x = tid; x < DG_STRIDE; x += NTHREADS) part[x] = 0.f;
    return;
  }
  const int iters = m1 - m0 + 1;
  const uint32_t sbase = smem_u32(smem), bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NB + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NB);
  int32_t *status = p.status;
  if (tid == 0) {
    for (int k = 0; k < NB; ++k) mbar_init(BAR(k), k == B_EFULL ? NSOFT : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  for (int x = tid; x < 16384 / 16; x += NTHREADS) {
    const uint32_t one2 = 0x3F803F80u;
    *reinterpret_cast<uint4 *>(smem + OFF_ONES + 16 * x) = make_uint4(one2, one2, one2, one2);
  }
  // E's zero entries sit at the same places in every tile: written once here, the rows
  // then write only the values (store_E<false>)
  for (int x = tid; x < 65536 / 16; x += NTHREADS) *reinterpret_cast<uint4 *>(smem + OFF_E + 16 * x) = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 256);
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
      prefetch_tmap(&A.mpd);
      prefetch_tmap(&A.mq);
      const uint32_t idG = idesc_bf16(128, 80, true, true);
      auto issue = [&](int t) {  // dS planes of tile (m, m - D) and Q_m
        const int st = t & 1, m = m0 + t, pl = tile_plane(p, bh, m, m - D);
        ctl.expect(BAR(B_LD0 + st), (uint32_t)((t >> 1) & 1), 32768u + 16384u);
        tma_load_3d(sbase + OFF_DS + 32768 * st, &A.mpd, BAR(B_LD0 + st), 0, 0, pl + 2);
        tma_load_3d(sbase + OFF_DS + 32768 * st + 16384, &A.mpd, BAR(B_LD0 + st), 0, 0, pl + 3);
        tma_load_3d(sbase + OFF_Q + 16384 * st, &A.mq, BAR(B_LD0 + st), 0, m * 128, bh);
      };
      issue(0);
      if (iters > 1) issue(1);
      for (int t = 0; t < iters; ++t) {
        const int st = t & 1;
        if (!ctl.wait_load(BAR(B_LD0 + st), (uint32_t)((t >> 1) & 1))) break;
        if (!ctl.wait(BAR(B_EFULL), t & 1)) break;  // the rows have built E(t) (and read dS(t))
        tc_fence_after();
        const uint32_t lbo = (uint32_t)(OFF_ONES - OFF_Q - 16384 * st);  // Q atom -> ones atom
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // [G | g]_lo, [G | g]_hi += E^T [Q | 1]
          const uint32_t acc = (t > 0 || k > 0) ? 1u : 0u;
          const uint64_t bq = sdesc_sw128(sbase + OFF_Q + 16384 * st + 2048 * k, lbo, 1024);
          umma_bf16(tbase + T_GLO, sdesc_sw128(sbase + OFF_E + 2048 * k, 16384, 1024), bq, idG, acc);
          umma_bf16(tbase + T_GHI, sdesc_sw128(sbase + OFF_E + 32768 + 2048 * k, 16384, 1024), bq, idG, acc);
        }
        umma_commit(BAR(B_EFREE));
        if (t + 2 < iters) {  // stage st (dS read by the rows, Q by these MMAs) is free
          if (!ctl.wait(BAR(B_EFREE), t & 1)) break;
          issue(t + 2);
        }
      }
      ctl.drain(BAR(B_DRAIN));
    }
    __syncwarp();
  } else {
    const int g = warp & 3, qt = warp >> 2, il = 32 * g + lane, cb = NC * qt;
    const uint32_t tl = tbase + ((uint32_t)(g * 32) << 16);
    bool good = true;
    for (int t = 0; t < iters; ++t) {
      const int st = t & 1;
      good = good && warp_wait(BAR(B_LD0 + st), (uint32_t)((t >> 1) & 1), abort_flag, status);
      if (t >= 1) good = good && warp_wait(BAR(B_EFREE), (t - 1) & 1, abort_flag, status);  // E(t - 1) read
      if (good) {
        // this thread's 32 dS values (row il, keys cb .. cb + 31) from the swizzled stage,
        // as bf16 pairs (x[2k+1] low, x[2k] high) for store_E
        uint32_t ds[NC / 2];
        const uint8_t *src = smem + OFF_DS + 32768 * st + 16384 * (qt >> 1) + 128 * il;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v = *reinterpret_cast<const uint4 *>(src + (((4 * (qt & 1) + c) ^ (il & 7)) << 4));
          ds[4 * c] = prmt(v.x, v.x, 0x1032u);
          ds[4 * c + 1] = prmt(v.y, v.y, 0x1032u);
          ds[4 * c + 2] = prmt(v.z, v.z, 0x1032u);
          ds[4 * c + 3] = prmt(v.w, v.w, 0x1032u);
        }
        store_E<false>(smem + OFF_E, il, cb, ds);
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(BAR(B_EFULL));
      }
    }
    // ---- epilogue: lane il is offset c = il of both blocks; 16 columns per thread ----
    good = good && warp_wait(BAR(B_EFREE), (iters - 1) & 1, abort_flag, status);
    if (good) {
      tc_fence_after();
      uint32_t rlo[16], rhi[16], glo[16], ghi[16];
      tmem_ld16(tl + T_GLO + 16 * qt, rlo);
      tmem_ld16(tl + T_GHI + 16 * qt, rhi);
      tmem_ld16(tl + T_GLO + 64, glo);
      tmem_ld16(tl + T_GHI + 64, ghi);
      tmem_wait_ld();
      const bool part_ok = dcheck(
          (size_t)(part - A.part_dg) + DG_STRIDE <= (size_t)BH * A.nbands * A.dg_nchunk * DG_STRIDE, status);
#pragma unroll
      for (int e = 0; e < 16 && part_ok; ++e) {
        part[(size_t)(16 * qt + e) * 128 + il] = u2f(rlo[e]);
        part[(size_t)(65 + 16 * qt + e) * 128 + il] = u2f(rhi[e]);
      }
      if (qt == 0 && part_ok) {
        part[(size_t)64 * 128 + il] = u2f(glo[0]);
        part[(size_t)(65 + 64) * 128 + il] = u2f(ghi[0]);
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_dgs_kernel(const __grid_constant__ BwdArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  dgs_body(A, (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023), (int)blockIdx.x);
}

// Both streaming roles in one launch.  They are independent (each only reads the stored
// tiles and Q / dO) and bound differently -- the key-tile role by DRAM bandwidth, the
// diagonal role by latency -- so their CTAs are interleaved in the grid (the k-th
// key-tile CTA at index ~ k * gridDim / n_kvs, each role keeping its own heaviest-first
// order) and the scheduler runs them side by side.
constexpr int STREAM_SMEM = kvs::SMEM > dgs::SMEM ? kvs::SMEM : dgs::SMEM;

__global__ void __launch_bounds__(NTHREADS, 1) tc_bwd_stream_kernel(const __grid_constant__ BwdArgs A) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint64_t c = blockIdx.x, total = gridDim.x, nk = (uint64_t)A.n_kvs;
  const int before = (int)(c * nk / total), upto = (int)((c + 1) * nk / total);  // key-tile CTAs in [0, c) / [0, c]
  if (upto > before)
    kvs_body(A, smem, before);
  else
    dgs_body(A, smem, (int)c - before);
}

// dr[h][rho][e] = s (sum G + (sum g) v[e]) over the batch, the bands holding
// offset delta = rho - off (as block D or D - 1) and their chunks, in a fixed order.
// One CTA per 32 consecutive offsets (the lanes; the partials are offset-contiguous,
// so each warp load is one 128-byte run) and 8 warps of 8 columns e each.  The CTA
// also writes the dv partial of its 32 offsets, sum_rho (sum g)_rho r_rho[e], reduced
// over the lanes by a fixed shuffle tree.
__global__ void __launch_bounds__(256) reduce_dr_kernel(BwdArgs A) {
  const Prm &p = A.p;
  const int ntile = (p.nrows + 31) / 32;
  const int h = (int)blockIdx.x / ntile, tile = (int)blockIdx.x % ntile;
  const int lane = threadIdx.x & 31, eg = threadIdx.x >> 5;
  const int rho = 32 * tile + lane;
  const bool ok = rho < p.nrows;
  float acc[8], gs = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
  if (ok) {
    const int delta = rho - p.off;
    const int blk = delta >= 0 ? delta / 128 : -((-delta + 127) / 128);
    const int c = delta - 128 * blk;
    for (int bb = 0; bb < p.B; ++bb) {
      const size_t bh = (size_t)bb * p.H + h;
      for (int w = 0; w < 2; ++w) {  // w = 0: band blk (block = D); w = 1: band blk + 1 (block = D - 1)
        const int D = blk + w;
        const int band = p.causal ? D : D + (p.nT - 1);
        if (band < 0 || band >= A.nbands) continue;
        const int len = p.nT - (D < 0 ? -D : D);
        const int nch = (len + A.dg_ch - 1) / A.dg_ch;
        const float *part = A.part_dg + (bh * A.nbands + band) * A.dg_nchunk * DG_STRIDE + (size_t)(65 * w) * 128 + c;
        // up to four chunks' loads in flight before their (in-order) accumulation
        for (int ch = 0; ch < nch; ch += 4) {
          float v[4][9];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float *pu = part + (size_t)(ch + u) * DG_STRIDE;
            const bool have = ch + u < nch;
#pragma unroll
            for (int k = 0; k < 8; ++k) v[u][k] = have ? __ldg(pu + (size_t)(8 * eg + k) * 128) : 0.f;
            v[u][8] = have ? __ldg(pu + (size_t)64 * 128) : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] += v[u][k];
            gs += v[u][8];
          }
        }
      }
    }
  }
  const __nv_bfloat16 *vv = (const __nv_bfloat16 *)p.rel2 + (size_t)h * HD + 8 * eg;
  const __nv_bfloat16 *rr = (const __nv_bfloat16 *)p.rel0 + ((size_t)h * p.nrows + (ok ? rho : 0)) * HD + 8 * eg;
  float pv[8];
  if (ok) {
    float *out = p.drel0 + ((size_t)h * p.nrows + rho) * HD + 8 * eg;
    // the r row (16-byte aligned: the boundary checks the table's alignment) in one load
    const uint4 rw4 = __ldg(reinterpret_cast<const uint4 *>(rr));
    const uint32_t rw[4] = {rw4.x, rw4.y, rw4.z, rw4.w};
    uint32_t ob[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      ob[k] = __float_as_uint(p.scale * (acc[k] + gs * __bfloat162float(vv[k])));
      pv[k] = gs * ((k & 1) ? __uint_as_float(rw[k >> 1] & 0xFFFF0000u) : __uint_as_float(rw[k >> 1] << 16));
    }
    // a warp's 32 lanes write 32 rows: one 32-byte store each when the gradient buffer allows
    if ((reinterpret_cast<uintptr_t>(out) & 31u) == 0) {
      st_global_32B(out, ob);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) out[k] = __uint_as_float(ob[k]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) pv[k] = 0.f;
  }
  // sum over the 32 lanes of eight values in 9 shuffles: halve the set at xor 16, 8, 4
  // (each lane keeps the half its bit selects), then finish at xor 2, 1; lane 4k ends
  // with the sum of value k (a fixed order)
  {
    const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0, b2 = (lane & 4) != 0;
    float h4[4], h3[2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float send = b4 ? pv[j] : pv[j + 4], keep = b4 ? pv[j + 4] : pv[j];
      h4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float send = b3 ? h4[j] : h4[j + 2], keep = b3 ? h4[j + 2] : h4[j];
      h3[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float h2 = (b2 ? h3[1] : h3[0]) + __shfl_xor_sync(0xffffffffu, b2 ? h3[0] : h3[1], 4);
    h2 += __shfl_xor_sync(0xffffffffu, h2, 2);
    h2 += __shfl_xor_sync(0xffffffffu, h2, 1);
    if ((lane & 3) == 0) A.part_uv[((size_t)h * ntile + tile) * HD + 8 * eg + (lane >> 2)] = h2;
  }
}

// dv[h][e] = s * sum over the 32-offset tiles of the dv partials; du[h][e] = sum over
// (batch, key tile) of the du partials.  One CTA per head: 4 strided partial sums per
// column, combined in a fixed order.
__global__ void __launch_bounds__(256) reduce_uv_kernel(BwdArgs A) {
  const Prm &p = A.p;
  __shared__ float red[2][4][HD];
  const int h = blockIdx.x, e = threadIdx.x & (HD - 1), part = threadIdx.x >> 6;
  const int ntile = (p.nrows + 31) / 32, nkv = p.B * p.nT;
  float dv = 0.f, du = 0.f;
  for (int t = part; t < ntile; t += 4) dv += A.part_uv[((size_t)h * ntile + t) * HD + e];
  for (int x = part; x < nkv; x += 4) {
    const int bb = x / p.nT, n = x % p.nT;
    du += A.part_kv[(((size_t)bb * p.H + h) * p.nT + n) * HD + e];
  }
  red[0][part][e] = dv;
  red[1][part][e] = du;
  __syncthreads();
  if (part == 0) {
    p.drel2[(size_t)h * HD + e] = p.scale * (((red[0][0][e] + red[0][1][e]) + red[0][2][e]) + red[0][3][e]);
    p.drel1[(size_t)h * HD + e] = ((red[1][0][e] + red[1][1][e]) + red[1][2][e]) + red[1][3][e];
  }
}

}  // namespace tcb

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------
// Diagonal bands of tiles and their chunks (one diagonal-role CTA and one partial per
// (batch, head, band, chunk)).  Bands are split only until there are about four diagonal
// CTAs per SM: longer chunks write fewer partials and set up (E's zeros, TMEM) fewer
// times, while the key-tile role fills the SMs beside them.  Measured at Transformer-XL
// causal 8K, H = 8 (512 bands): 5 chunks per band 1.570 ms per step, 2 chunks 1.533,
// 1 chunk 1.518.
void tc_bwd_shape(const Prm &p, int &nT, int &nbands, int &ch, int &nchunk) {
  nT = (p.L + 127) / 128;
  nbands = p.causal ? nT : 2 * nT - 1;
  long long cap = 4 * 148 / ((long long)p.B * p.H * nbands);
  int nch = (nT + 3) / 4;
  if (cap < nch) nch = (int)(cap < 1 ? 1 : cap);
  ch = (nT + nch - 1) / nch;
  nchunk = (nT + ch - 1) / ch;
}

// Bytes of the stored P / dS tile buffer: 64 KB per tile of the backward, or 0 when over
// 32 GiB (the key-tile and diagonal kernels then recompute S, P and dS).
size_t tc_bwd_tile_bytes(const Prm &p) {
  const size_t nT = ((size_t)p.L + 127) / 128;
  const size_t ntiles = p.causal ? nT * (nT + 1) / 2 : nT * nT;
  const size_t bytes = (size_t)p.B * p.H * ntiles * 65536;
  return bytes <= ((size_t)32 << 30) ? bytes : 0;
}

size_t tc_bwd_part_floats(const Prm &p, size_t &kv_floats) {
  int nT, nbands, ch, nchunk;
  tc_bwd_shape(p, nT, nbands, ch, nchunk);
  kv_floats = (size_t)p.B * p.H * nT * HD;
  return (size_t)p.B * p.H * nbands * nchunk * tcb::DG_STRIDE;
}

bool tc_make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t planes, uint32_t box_rows);

cudaError_t tc_bwd(const Prm &p0, const TcWork &w, cudaStream_t st) {
  using namespace tcb;
  BwdArgs a;
  memset(&a, 0, sizeof(a));
  a.p = p0;
  int nT, nbands, ch, nchunk;
  tc_bwd_shape(p0, nT, nbands, ch, nchunk);
  a.p.nT = nT;
  a.nbands = nbands;
  a.dg_ch = ch;
  a.dg_nchunk = nchunk;
  a.uk = w.uk;
  a.vr = w.vr;
  a.part_kv = w.part_kv;
  a.part_dg = w.part_dg;
  a.part_uv = w.part_uv;
  a.p.part_small = w.part_kv;
  const uint64_t BH = (uint64_t)p0.B * p0.H;
  a.pd_stored = w.pdtiles != nullptr;
  a.pd = (__nv_bfloat16 *)w.pdtiles;
  if (a.pd_stored && !tc_make_map(&a.mpd, w.pdtiles, 128, tc_bwd_tile_bytes(p0) / 16384, 128)) return cudaErrorInvalidValue;
  if (!(tc_make_map(&a.mq, p0.q, p0.L, BH, 128) && tc_make_map(&a.mk, p0.k, p0.L, BH, 128) &&
        tc_make_map(&a.mv, p0.v, p0.L, BH, 128) && tc_make_map(&a.mdo, p0.dout, p0.L, BH, 128) &&
        tc_make_map(&a.mr, p0.rel0, p0.nrows, p0.H, 128)))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if ((e = tc_prep(a.p, w, st)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(tc_bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kv::SMEM)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(tc_bwd_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, qk::SMEM)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(tc_bwd_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dg::SMEM)) != cudaSuccess)
    return e;
  const unsigned tiles = (unsigned)(nT * p0.H * p0.B);
  const unsigned qtiles = (unsigned)((nT - p0.mem_len / 128) * p0.H * p0.B);  // no memory-placeholder query tiles
  const unsigned diag_ctas = (unsigned)(nbands * nchunk * p0.B * p0.H);
  if (a.pd_stored) {  // the query-tile kernel first; then both roles streaming its P / dS tiles
    if ((e = cudaFuncSetAttribute(tc_bwd_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, STREAM_SMEM)) !=
        cudaSuccess)
      return e;
    RP_TRACED("tc_bwd_q_kernel", st, tc_bwd_q_kernel<<<qtiles, NTHREADS, qk::SMEM, st>>>(a));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    a.n_kvs = (int)tiles;
    RP_TRACED("tc_bwd_stream_kernel", st, tc_bwd_stream_kernel<<<tiles + diag_ctas, NTHREADS, STREAM_SMEM, st>>>(a));
  } else {
    RP_TRACED("tc_bwd_kv_kernel", st, tc_bwd_kv_kernel<<<tiles, NTHREADS, kv::SMEM, st>>>(a));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    RP_TRACED("tc_bwd_q_kernel", st, tc_bwd_q_kernel<<<qtiles, NTHREADS, qk::SMEM, st>>>(a));
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (!a.pd_stored) RP_TRACED("tc_bwd_diag_kernel", st, tc_bwd_diag_kernel<<<diag_ctas, NTHREADS, dg::SMEM, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("reduce_dr_kernel", st, reduce_dr_kernel<<<(unsigned)(p0.H * ((p0.nrows + 31) / 32)), 256, 0, st>>>(a));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("reduce_uv_kernel", st, reduce_uv_kernel<<<p0.H, 256, 0, st>>>(a));
  return cudaGetLastError();
}

}  // namespace rp
