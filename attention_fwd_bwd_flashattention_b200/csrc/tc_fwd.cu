// Tensor-core (tcgen05 / TMEM / TMA) forward kernel of relative-position
// attention for bf16 inputs, d = 64, on sm_100a.
//
// One CTA per 128-row query tile (heaviest causal tiles launched first), nine
// warps:
//   warps 0-15 "softmax": four threads per query row (warps w, w + 4, w + 8, w + 12
//              share TMEM lanes 32 (w & 3)..+31 and take 32 key columns each).
//              They read S = Q K^T and the relation products from TMEM, add the
//              relative term gathered by offset, run the online softmax (row max
//              exchanged through smem; lazy rescale of O only when the running max
//              grows by more than 2^8), and write P (bf16 pairs) into TMEM, where the
//              PV MMA reads it as its A operand.
//   warp 16    lane 0 issues every TMA load (Q, K, V, relation-table windows,
//              2-stage K and V rings on separate barriers) and every tcgen05.mma, and
//              signals through mbarriers and tcgen05.commit.
// TMEM (512 columns): S [0,128), relation products [128,384), O [384,448), P [448,512).
//
// Relation stage per mechanism ("Fast and Exact Relative-Position Attention via
// Structure-Aware Kernels", Abstract, techniques (1) and (2)):
//   T5       per-tile window of the per-offset bias vector (255 values) in smem.
//   Shaw     QA = Q a^T (129 products per row) computed once per query tile by one
//            MMA and kept in smem; each pair reads its clipped column.
//   TXL      the offsets of tile (m, n) are 128 (m - n) + [-127, 127]: two
//            128-offset blocks of r.  Block b's products r_b Q^T are computed by
//            one 128x128x64 MMA and reused by the two consecutive key tiles that
//            need it, so each key tile adds exactly one new block.  Each row's
//            products are computed transposed (lane = offset) and written into
//            key order through padded smem rows.
//   DeBERTa  tiles within the span: c2p = Q Kr_win^T (255 offsets) rotated per row,
//            p2c = K Qr_win^T computed with keys as rows and transposed through
//            smem; tiles outside the span use per-row / per-key end products.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tc_skew.cuh"

namespace rp {
namespace tc {

constexpr int BM = 128, BN = 128;
constexpr int TPR = 4;             // softmax threads per query row
constexpr int NC = 128 / TPR;      // key columns per softmax thread
constexpr int NSOFT = 128 * TPR;   // softmax threads
constexpr int CTRL_WARP = NSOFT / 32;
constexpr int NTHREADS = NSOFT + 32;
constexpr int ROT_LD = 132;  // fp32 stride of the per-row skew buffer (conflict-free rotations)

constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + 16384;    // 2 stages
constexpr int OFF_V = OFF_K + 32768;    // 2 stages
constexpr int OFF_P = OFF_V + 32768;    // two 64-key halves of P
constexpr int OFF_R = OFF_P + 32768;    // relation-table staging (2 x 16 KB or one 32 KB window)
constexpr int OFF_ROT = OFF_R + 32768;  // 128 x ROT_LD fp32
constexpr int OFF_VEC = OFF_ROT + 128 * ROT_LD * 4;  // 2 x 512 fp32 per-tile vectors
constexpr int OFF_RED = OFF_VEC + 2 * 512 * 4;  // 2 x TPR x 128 fp32 row-max exchange
constexpr int OFF_BAR = OFF_RED + 2 * TPR * 128 * 4;
constexpr int SMEM_USED = OFF_BAR + 256;
constexpr int SMEM_BYTES = SMEM_USED + 1024;

// B_K0 / B_K1: K (and the Transformer-XL relation block) of the even / odd key tiles;
// B_V0 / B_V1: V of the even / odd key tiles (loaded on their own schedule)
enum {
  B_Q = 0, B_K0 = 1, B_K1 = 2, B_SFULL = 3, B_SFREE = 4, B_PFULL = 5, B_PV = 6, B_PLOAD = 7, B_PFULLPRO = 8,
  B_PFREEPRO = 9, B_RLOAD = 10, B_RFREE = 11, B_GFULL = 12, B_DRAIN = 13, B_V0 = 14, B_V1 = 15, B_RLOAD2 = 16,
  NBARS = 17
};
// P (bf16 pairs) lives in TMEM columns [448, 512) as the PV MMA's A operand (no P smem
// traffic).  The P smem tile then holds: DeBERTa's p2c table window (OFF_R holds the c2p
// one; B_RLOAD / B_RLOAD2), Shaw's value side's offset-ordered P (Pe), Transformer-XL's
// first relation block.
constexpr uint32_t TM_PD = 448;

constexpr uint32_t TM_S = 0, TM_REL = 128, TM_O = 384, TM_COLS = 512;

struct FwdArgs {
  CUtensorMap mq, mk, mv, mt0, mt1;
  Prm p;
  const float *uk, *vr, *c2pE, *p2cE;
  int shaw_n;  // N of the Shaw QA MMA (2c + 1 rounded up to 16)
};

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// A wait whose result is the same on all 32 lanes (tcgen05.ld/st are warp-collective).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *ab, int32_t *st) {
  const bool ok = mbar_wait(bar, parity, ab, st, RELPOS_ERR_TIMEOUT_DEV);
  return __all_sync(0xffffffffu, ok);
}

// Shaw's value side: this thread's NC probabilities of row il written into the
// offset-order tile Pe at column (delta + c) & 127 (delta = j - i), in the layout of the
// P tile (128-byte-swizzled K-major, 64-column halves 16 KB apart).  Clipped pairs are
// passed as 0, so the row's 128 keys fill every column once.  pk[k] = (v[2k], v[2k+1]);
// C0 = column of v[0].  Aligned bf16 pairs; when C0 is odd the first and the last value
// share their pair with a neighbouring thread's and are written alone.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t pe_off(uint32_t t, uint32_t rowb, uint32_t r7) {  // t = 2 col, col even
  return ((t << 7) & 0x4000u) + rowb + ((t & 126u) ^ r7);
}
__device__ __forceinline__ void store_pe(uint8_t *E, int il, uint32_t C0, const uint32_t (&pk)[NC / 2]) {
  const bool odd = (C0 & 1u) != 0;
  const uint32_t rowb = 128u * (uint32_t)il, r7 = (uint32_t)(il & 7) << 4;
  const uint32_t sel = odd ? 0x5432u : 0x3210u;  // odd: (high half of pk[k], low half of pk[k+1])
  const uint32_t B0 = (C0 + (odd ? 1u : 0u)) & 127u;
#pragma unroll
  for (int k = 0; k < NC / 2 - 1; ++k) {
    const uint32_t col = (B0 + 2u * k) & 127u;
    *reinterpret_cast<uint32_t *>(E + pe_off(2u * col, rowb, r7)) = prmt(pk[k], pk[k + 1], sel);
  }
  if (!odd) {
    const uint32_t col = (B0 + 2u * (NC / 2 - 1)) & 127u;
    *reinterpret_cast<uint32_t *>(E + pe_off(2u * col, rowb, r7)) = pk[NC / 2 - 1];
  } else {
    const uint32_t c0 = (C0 - 1u) & 127u, c31 = (C0 + NC - 1) & 127u;
    *reinterpret_cast<uint16_t *>(E + pe_off(2u * c0, rowb, r7) + 2u) = (uint16_t)(pk[0] & 0xFFFFu);
    *reinterpret_cast<uint16_t *>(E + pe_off(2u * c31, rowb, r7)) = (uint16_t)(pk[NC / 2 - 1] >> 16);
  }
}

// Shaw band tile: some of its offsets 128 (n - m) + [-127, 127] are unclipped.
__device__ __forceinline__ bool shaw_band(int clip, int m, int n) {
  const int D = m - n;
  return 128 * (D < 0 ? -D : D) - 127 < clip;
}

// VAL (Shaw only): the value-side table aV (rel1) adds sum_j P_ij aV[clip(j - i) + c] to
// every O_i: band tiles through one more MMA O += Pe aV[0..127] with P in offset order,
// the clipped pairs through two per-row sums applied to aV[0] / aV[2c] in the epilogue.
template <int MECH, bool VAL = false>
__global__ void __launch_bounds__(NTHREADS, 1) tc_fwd_kernel(const __grid_constant__ FwdArgs A) {
  constexpr bool SV = MECH == M_SHAW && VAL;
  constexpr uint32_t TMP = TM_PD;  // P in TMEM (the PV MMA's A operand)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const Prm &p = A.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 1-D grid, heaviest (longest causal) query tiles of every head first
  const int BH = p.B * p.H;
  const int bh = (int)blockIdx.x % BH, m = p.nT - 1 - (int)blockIdx.x / BH;
  const int h = bh % p.H;
  const int L = p.L, i0 = m * BM;
  // keys j >= klen of this batch are masked; key tiles past them are skipped
  const int klen = key_len(p, bh / p.H);
  const int nTiles = min(p.causal ? m + 1 : p.nT, (klen + BN - 1) / BN);
  if (nTiles == 0) {  // no key at all: O = 0, LSE = -inf (whole CTA, before any barrier)
    for (int x = tid; x < BM * (HD / 8); x += NTHREADS) {
      const int r = x / (HD / 8), c8 = x % (HD / 8);
      if (i0 + r < L)
        *reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.out + ((size_t)bh * L + i0 + r) * HD + 8 * c8) = make_uint4(0, 0, 0, 0);
    }
    if (tid < BM && i0 + tid < L) p.lse[(size_t)bh * L + i0 + tid] = -INFINITY;
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  volatile int *abort_flag = (volatile int *)(smem + OFF_BAR + 8 * NBARS + 4);
  uint32_t *tmem_slot = (uint32_t *)(smem + OFF_BAR + 8 * NBARS);
  float *rot = (float *)(smem + OFF_ROT);
  float *vec = (float *)(smem + OFF_VEC);

  if (tid == 0) {
    mbar_init(BAR(B_Q), 1);
    mbar_init(BAR(B_K0), 1);
    mbar_init(BAR(B_K1), 1);
    mbar_init(BAR(B_V0), 1);
    mbar_init(BAR(B_V1), 1);
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_SFREE), NSOFT);
    mbar_init(BAR(B_PFULL), NSOFT);
    mbar_init(BAR(B_PV), 1);
    mbar_init(BAR(B_PLOAD), 1);
    mbar_init(BAR(B_PFULLPRO), 1);
    mbar_init(BAR(B_PFREEPRO), NSOFT);
    mbar_init(BAR(B_RLOAD), 1);
    mbar_init(BAR(B_RLOAD2), 1);
    mbar_init(BAR(B_RFREE), NSOFT);
    mbar_init(BAR(B_GFULL), 1);
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), TM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  int32_t *status = p.status;
  const float c1 = p.scale * 1.4426950408889634f;  // scale * log2(e)

  if (warp == CTRL_WARP) {
    // ======================= TMA + MMA issuer ==========================
    if (lane == 0) {
      prefetch_tmap(&A.mq);
      prefetch_tmap(&A.mk);
      prefetch_tmap(&A.mv);
      if (MECH != M_T5) prefetch_tmap(&A.mt0);
      if (MECH == M_DEB) prefetch_tmap(&A.mt1);
      const uint32_t idS = idesc_bf16(128, 128, false);
      const uint32_t idPV = idesc_bf16(128, 64, true);
      const uint32_t idW = idesc_bf16(128, 256, false);
      // TMA loads issued but not yet waited for, drained before exit on abort
      uint32_t pend_bar[10];
      uint32_t pend_par[10];
      int npend = 0;
      auto expect = [&](int bi, uint32_t par, uint32_t bytes) {
        mbar_expect_tx(BAR(bi), bytes);
        pend_bar[npend] = BAR(bi);
        pend_par[npend] = par;
        ++npend;
      };
      auto waited = [&](uint32_t bar) {  // drop one pending entry of this barrier
        for (int e = 0; e < npend; ++e)
          if (pend_bar[e] == bar) {
            pend_bar[e] = pend_bar[npend - 1];
            pend_par[e] = pend_par[npend - 1];
            --npend;
            return;
          }
      };
      auto wait_load = [&](int bi, uint32_t par) {
        const bool r = mbar_wait(BAR(bi), par, abort_flag, status, RELPOS_ERR_TIMEOUT_DEV);
        if (r) waited(BAR(bi));
        return r;
      };
      auto wait_bar = [&](int bi, uint32_t par) { return mbar_wait(BAR(bi), par, abort_flag, status, RELPOS_ERR_TIMEOUT_DEV); };

      expect(B_Q, 0, 16384);
      tma_load_3d(sbase + OFF_Q, &A.mq, BAR(B_Q), 0, i0, bh);
      int band_cnt = 0;
      bool ok = true;
      if (MECH == M_SHAW) {
        expect(B_PLOAD, 0, (uint32_t)A.shaw_n * 128u);
        tma_load_3d(sbase + OFF_R, &A.mt0, BAR(B_PLOAD), 0, 0, h);
        ok = wait_load(B_Q, 0) && wait_load(B_PLOAD, 0);
        if (ok) {
          tc_fence_after();
          umma_k64(tbase + TM_REL, sbase + OFF_Q, sbase + OFF_R, idesc_bf16(128, A.shaw_n, false), false);
          umma_commit(BAR(B_PFULLPRO));
          ok = wait_bar(B_PFREEPRO, 0);
        }
        if (SV && ok) {  // the QA MMA is done with the table a: aV rows 0..127 take its place
          expect(B_PLOAD, 1, 16384);
          tma_load_3d(sbase + OFF_R, &A.mt1, BAR(B_PLOAD), 0, 0, h);
        }
      }
      if (MECH == M_TXL) {  // first relation block: offsets 128 m + [0, 128)
        expect(B_PLOAD, 0, 16384);
        tma_load_3d(sbase + OFF_P, &A.mt0, BAR(B_PLOAD), 0, 128 * m + p.off, h);
      }
      // DeBERTa band tile: some offsets of tile (m, n) are inside the span
      auto deb_band = [&](int n) {
        const int D = m - n;
        return 128 * (D < 0 ? -D : D) - 127 < p.span;
      };
      // both table windows of band tile n (c2p: Kr rows into OFF_R; p2c: Qr rows into the P
      // smem tile, free because P lives in TMEM), phase = the band tile's index & 1
      auto issue_win = [&](int n) {
        const int D = m - n;
        const uint32_t ph = (uint32_t)(band_cnt & 1);
        expect(B_RLOAD, ph, 32768);
        tma_load_3d(sbase + OFF_R, &A.mt0, BAR(B_RLOAD), 0, p.span + 128 * D - 127, h);
        expect(B_RLOAD2, ph, 32768);
        tma_load_3d(sbase + OFF_P, &A.mt1, BAR(B_RLOAD2), 0, p.span - 128 * D - 127, h);
      };
      auto needs_new_block = [&](int n) {  // TXL: block (m - n - 1), unless it is entirely masked
        return !(p.causal && m - n - 1 < 0);
      };
      // K(n) and the relation block tile n adds (TXL) go into stage n & 1 as soon as S(n - 2),
      // their previous reader, is complete; V(n) goes into stage n & 1 once PV(n - 2) is: the
      // loads of a key tile are issued about one tile ahead of their first use
      auto issue_k = [&](int n) {
        const int st = n & 1;
        uint32_t bytes = 16384;
        if (MECH == M_TXL && needs_new_block(n)) bytes += 16384;
        expect(B_K0 + st, (uint32_t)((n >> 1) & 1), bytes);
        tma_load_3d(sbase + OFF_K + 16384 * st, &A.mk, BAR(B_K0 + st), 0, n * BN, bh);
        if (MECH == M_TXL && needs_new_block(n))
          tma_load_3d(sbase + OFF_R + 16384 * st, &A.mt0, BAR(B_K0 + st), 0, 128 * (m - n - 1) + p.off, h);
      };
      auto issue_v = [&](int n) {
        const int st = n & 1;
        expect(B_V0 + st, (uint32_t)((n >> 1) & 1), 16384);
        tma_load_3d(sbase + OFF_V + 16384 * st, &A.mv, BAR(B_V0 + st), 0, n * BN, bh);
      };
      auto issue_pv = [&](int n) {  // O (+)= P(n) V(n)
        const int ps = n & 1;
        // P from TMEM; Shaw's value side on band tiles also O += Pe aV (Pe in the P smem tile)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_bf16_ts(tbase + TM_O, tbase + TMP + 8 * k, sdesc_sw128(sbase + OFF_V + 16384 * ps + 2048 * k, 16, 1024),
                       idPV, (n > 0 || k > 0) ? 1u : 0u);
        if (SV && shaw_band(p.clip, m, n)) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_bf16(tbase + TM_O, sdesc_sw128(sbase + OFF_P + 16384 * (k >> 2) + 32 * (k & 3), 16, 1024),
                      sdesc_sw128(sbase + OFF_R + 2048 * k, 16, 1024), idPV, 1u);
        }
        umma_commit(BAR(B_PV));
      };
      if (ok) {
        issue_k(0);
        issue_v(0);
        if (nTiles > 1) {
          issue_k(1);
          issue_v(1);
        }
      }
      if (SV && ok) ok = wait_load(B_PLOAD, 1);  // aV staged before the first PV
      if (MECH == M_DEB && ok && deb_band(0)) issue_win(0);
      for (int n = 0; ok && n < nTiles; ++n) {
        const int st = n & 1;
        const int Delta = m - n;
        if (!wait_load(B_K0 + st, (n >> 1) & 1)) break;
        if (n == 0) {
          if (MECH != M_SHAW && !wait_load(B_Q, 0)) break;
          if (MECH == M_TXL && !wait_load(B_PLOAD, 0)) break;
        } else if (!wait_bar(B_SFREE, (n - 1) & 1)) {
          break;
        }
        tc_fence_after();
        umma_k64(tbase + TM_S, sbase + OFF_Q, sbase + OFF_K + 16384 * st, idS, false);
        if (MECH == M_TXL) {
          // relation products transposed (lane = offset, column = query row)
          if (n == 0) umma_k64(tbase + TM_REL + 128 * (m & 1), sbase + OFF_P, sbase + OFF_Q, idS, false);
          if (needs_new_block(n))
            umma_k64(tbase + TM_REL + 128 * ((Delta - 1) & 1), sbase + OFF_R + 16384 * st, sbase + OFF_Q, idS, false);
        }
        const bool band = (MECH == M_DEB) && deb_band(n);
        if (band) {  // c2p window, prefetched (issue_win)
          if (!wait_load(B_RLOAD, (uint32_t)(band_cnt & 1))) break;
          umma_k64(tbase + TM_REL, sbase + OFF_Q, sbase + OFF_R, idW, false);
        }
        umma_commit(BAR(B_SFULL));
        // K(n + 1) into the stage of tile n - 1: the rows released S(n - 1) (B_SFREE), so
        // S(n - 1) and every MMA committed with it (and DeBERTa's p2c product of tile n - 1,
        // which the rows read before that release) are complete
        if (n >= 1 && n + 1 < nTiles) issue_k(n + 1);
        if (band) {  // p2c once the rows have read c2p; its window was prefetched with c2p's
          if (!wait_bar(B_RFREE, band_cnt & 1)) break;
          if (!wait_load(B_RLOAD2, (uint32_t)(band_cnt & 1))) break;
          tc_fence_after();
          umma_k64(tbase + TM_REL, sbase + OFF_K + 16384 * st, sbase + OFF_P, idW, false);
          umma_commit(BAR(B_GFULL));
          ++band_cnt;
        }
        // the next band tile's two table windows, as soon as this tile's relation MMAs (the
        // windows' last readers, committed to B_GFULL) are done
        if (MECH == M_DEB && n + 1 < nTiles && deb_band(n + 1)) {
          if (band && !wait_bar(B_GFULL, (band_cnt - 1) & 1)) break;
          issue_win(n + 1);
        }
        // V(n) into the stage of tile n - 2 once PV(n - 2) is complete (committed one tile ago)
        if (n >= 2) {
          if (!wait_bar(B_PV, (n - 2) & 1)) break;
          issue_v(n);
        }
        if (n >= 1) {
          if (!wait_bar(B_PFULL, (n - 1) & 1)) break;
          if (!wait_load(B_V0 + ((n - 1) & 1), ((n - 1) >> 1) & 1)) break;
          tc_fence_after();
          issue_pv(n - 1);
        }
      }
      if (ok && !*abort_flag && wait_bar(B_PFULL, (nTiles - 1) & 1) &&
          wait_load(B_V0 + ((nTiles - 1) & 1), ((nTiles - 1) >> 1) & 1)) {
        tc_fence_after();
        issue_pv(nTiles - 1);
      }
      // drain: every MMA issued by this thread, then every TMA load still in flight
      umma_commit(BAR(B_DRAIN));
      volatile int no_abort = 0;
      mbar_wait(BAR(B_DRAIN), 0, &no_abort, status, RELPOS_ERR_TIMEOUT_DEV);
      for (int e = 0; e < npend; ++e) mbar_wait(pend_bar[e], pend_par[e], &no_abort, status, RELPOS_ERR_TIMEOUT_DEV);
    }
    __syncwarp();
  } else {
    // ========================== softmax warps ===========================
    // warp w: TMEM lanes 32 (w & 3) .. +31 (query rows), key columns [NC qt, NC qt + NC), qt = w >> 2
    const int g = warp & 3, qt = warp >> 2;
    const int il = 32 * g + lane, i = i0 + il;
    const int cb = NC * qt;  // first key column of this thread
    const uint32_t tl = tbase + ((uint32_t)(g * 32) << 16);
    float *rrow = rot + il * ROT_LD;
    float *red = (float *)(smem + OFF_RED);
    float m2 = -INFINITY, lsum = 0.f;
    float sL = 0.f, sR = 0.f;  // Shaw value side: mass of the row's keys clipped left (delta <= -c) / right (>= c)
    float cE0 = 0.f, cE1 = 0.f;
    bool good = true;  // warp-uniform: false once any wait of the CTA ran out
    if (MECH == M_DEB && i < L) {
      cE0 = A.c2pE[((size_t)bh * L + i) * 2 + 0];
      cE1 = A.c2pE[((size_t)bh * L + i) * 2 + 1];
    }
    if (MECH == M_SHAW) {  // QA row -> smem (kept for the whole CTA); 32-column chunks split by thread
      good = warp_wait(BAR(B_PFULLPRO), 0, abort_flag, status);
      if (good) {
        tc_fence_after();
        const int nq = (2 * p.clip + 1 + 31) / 32;
        for (int q = qt; q < nq; q += TPR) {
          uint32_t r[32];
          tmem_ld32(tl + TM_REL + 32 * q, r);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t)
            if (32 * q + t < ROT_LD) rrow[32 * q + t] = u2f(r[t]);
        }
        tc_fence_before();
        mbar_arrive(BAR(B_PFREEPRO));
      }
      named_bar_sync(1, NSOFT);
    }
    int band_cnt = 0;
    // per-tile vectors, fetched one key tile ahead (one element per thread)
    auto fetch_vec = [&](int n) {
      const int j0 = n * BN;
      float va = 0.f;
      if (MECH == M_TXL) {  // u.k, pre-scaled by c1
        if (tid < 128 && j0 + tid < L) va = A.uk[(size_t)bh * L + j0 + tid] * c1;
      } else if (MECH == M_T5) {
        const int idx = j0 - i0 - 127 + tid + L - 1;
        if (tid < 255 && idx >= 0 && idx < 2 * L - 1) va = p.t5_bias[(size_t)h * (2 * L - 1) + idx];
      } else if (MECH == M_DEB) {
        const int j = j0 + (tid >> 1);
        if (tid < 256 && j < L) va = A.p2cE[((size_t)bh * L + j) * 2 + (tid & 1)];
      }
      return va;
    };
    // TXL: v.r of the tile's two offset blocks, one value per thread tid < 256, staged in
    // smem one tile ahead (slots 128 .. 383 of the tile's vector buffer)
    auto fetch_vr1 = [&](int n) {
      if (MECH != M_TXL || tid >= 256) return 0.f;
      const int ro = 128 * (tid < 128 ? m - n : m - n - 1) + (tid & 127) + p.off;
      return (ro >= 0 && ro < p.nrows) ? A.vr[(size_t)h * p.nrows + ro] * c1 : 0.f;
    };
    float nva = fetch_vec(0);
    if (MECH == M_TXL) {
      if (tid < 256) vec[128 + tid] = fetch_vr1(0);
      named_bar_sync(1, NSOFT);
    }
    for (int n = 0; n < nTiles; ++n) {
      const int j0 = n * BN, Delta = m - n;
      float *tv = vec + 512 * (n & 1);
      if ((MECH == M_TXL && tid < 128) || (MECH == M_T5 && tid < 255) || (MECH == M_DEB && tid < 256)) tv[tid] = nva;
      const float nvr = (n + 1 < nTiles) ? fetch_vr1(n + 1) : 0.f;
      if (n + 1 < nTiles) nva = fetch_vec(n + 1);
      // the per-tile vectors written above are read only after a later barrier of this tile
      // (Transformer-XL: the one after the skew; the other mechanisms: this one)
      if (MECH != M_TXL) named_bar_sync(1, NSOFT);
      good = good && warp_wait(BAR(B_SFULL), n & 1, abort_flag, status);
      float x[NC];
      uint32_t rs[32];  // S row segment; its registers are valid only after tcgen05.wait::ld
      if (good) {
        tc_fence_after();
        tmem_ld32(tl + TM_S + cb, rs);
        // Transformer-XL: the relation block's load (in the skew below) is issued before this
        // one is waited for, so that the two TMEM latencies overlap
        if (MECH != M_TXL) {
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < NC; ++t) x[t] = u2f(rs[t]);
        }
      } else {
#pragma unroll
        for (int t = 0; t < NC; ++t) x[t] = 0.f;
      }
      // ---- relative term, gathered by offset ----
      if (MECH == M_TXL) {
        if (good) {
          const bool hasB = !(p.causal && Delta == 0);
          // relation terms in key order, already c1 (T + v.r); its tcgen05.wait::ld also
          // completes the S load above
          txl_skew<ROT_LD, SK_PACKED>(tl, TM_REL + 128 * (Delta & 1), TM_REL + 128 * ((Delta - 1) & 1), hasB, g, qt, lane,
                                      c1, tv[128 + il], tv[256 + il], rot);
          tmem_wait_ld();  // when the skew had no load to wait for (no block Delta - 1 for this warp)
#pragma unroll
          for (int t = 0; t < NC; ++t) x[t] = u2f(rs[t]);
          tc_fence_before();
          mbar_arrive(BAR(B_SFREE));
        }
        named_bar_sync(1, NSOFT);
        // log2-domain score s c1 + (r' + u'): one f32x2 add and one f32x2 FMA per two keys
        const uint64_t c12 = f2(c1, c1);
#pragma unroll
        for (int c4 = 0; c4 < NC / 4; ++c4) {
          const float4 rr = *reinterpret_cast<const float4 *>(rrow + cb + 4 * c4);
          const float4 uk = *reinterpret_cast<const float4 *>(tv + cb + 4 * c4);
          f2_split(fma2(f2(x[4 * c4 + 0], x[4 * c4 + 1]), c12, add2(f2(rr.x, rr.y), f2(uk.x, uk.y))), x[4 * c4 + 0],
                   x[4 * c4 + 1]);
          f2_split(fma2(f2(x[4 * c4 + 2], x[4 * c4 + 3]), c12, add2(f2(rr.z, rr.w), f2(uk.z, uk.w))), x[4 * c4 + 2],
                   x[4 * c4 + 3]);
        }
      } else if (MECH == M_T5) {
        if (good) {
          tc_fence_before();
          mbar_arrive(BAR(B_SFREE));
        }
        const float lg = 1.4426950408889634f;
        const float *bw = tv + cb - il + 127;
#pragma unroll
        for (int t = 0; t < NC; ++t) x[t] = x[t] * c1 + bw[t] * lg;
      } else if (MECH == M_SHAW) {
        if (good) {
          tc_fence_before();
          mbar_arrive(BAR(B_SFREE));
        }
        const int d0 = j0 + cb - i;
#pragma unroll
        for (int t = 0; t < NC; ++t) x[t] = (x[t] + rrow[iclamp(d0 + t, -p.clip, p.clip) + p.clip]) * c1;
      } else {  // DeBERTa
        const bool band = 128 * (Delta < 0 ? -Delta : Delta) - 127 < p.span;
        if (band) {
          // c2p: window column w (Kr row lo + w) belongs to key il + 127 - w; this
          // thread handles w in [64 qt, 64 qt + 64)
          if (good) {
            const int lo = p.span + 128 * Delta - 127;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t r[32];
              tmem_ld32(tl + TM_REL + 64 * qt + 32 * q, r);
              tmem_wait_ld();
#pragma unroll
              for (int t = 0; t < 32; ++t) {
                const int w = 64 * qt + 32 * q + t;
                if (w >= il && w <= il + 127) {
                  const int rho = lo + w;
                  rrow[il + 127 - w] = (rho < 0) ? cE0 : (rho > 2 * p.span - 1 ? cE1 : u2f(r[t]));
                }
              }
            }
            tc_fence_before();
            mbar_arrive(BAR(B_RFREE));
          }
          named_bar_sync(1, NSOFT);
#pragma unroll
          for (int t = 0; t < NC; ++t) x[t] += rrow[cb + t];
          named_bar_sync(1, NSOFT);
          good = good && warp_wait(BAR(B_GFULL), band_cnt & 1, abort_flag, status);
          ++band_cnt;
          if (good) {
            tc_fence_after();
            // TMEM lane il now holds key il of the tile: K_j . Qr_win; window column w
            // belongs to query il + 127 - w
            const int lo2 = p.span - 128 * Delta - 127;
            const float e0 = tv[2 * il], e1 = tv[2 * il + 1];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t r[32];
              tmem_ld32(tl + TM_REL + 64 * qt + 32 * q, r);
              tmem_wait_ld();
#pragma unroll
              for (int t = 0; t < 32; ++t) {
                const int w = 64 * qt + 32 * q + t;
                if (w >= il && w <= il + 127) {
                  const int rho = lo2 + w;
                  rot[(il + 127 - w) * ROT_LD + il] = (rho < 0) ? e0 : (rho > 2 * p.span - 1 ? e1 : u2f(r[t]));
                }
              }
            }
            tc_fence_before();
            mbar_arrive(BAR(B_SFREE));
          }
          named_bar_sync(1, NSOFT);
#pragma unroll
          for (int t = 0; t < NC; ++t) x[t] = (x[t] + rrow[cb + t]) * c1;
        } else {
          if (good) {
            tc_fence_before();
            mbar_arrive(BAR(B_SFREE));
          }
          const float c2p = Delta > 0 ? cE1 : cE0;
          const int sel = Delta < 0 ? 1 : 0;
#pragma unroll
          for (int t = 0; t < NC; ++t) x[t] = (x[t] + c2p + tv[2 * (cb + t) + sel]) * c1;
        }
      }
      // ---- mask (diagonal / ragged tiles only), row max over the row's threads ----
      const bool need_mask = (p.causal && n == m) || (j0 + BN > klen);
      float mt = -INFINITY;
      if (need_mask) {
#pragma unroll
        for (int t = 0; t < NC; ++t) {
          const int j = j0 + cb + t;
          if (j >= klen || (p.causal && j > i)) x[t] = -INFINITY;
        }
      }
#pragma unroll
      for (int t = 0; t < NC; t += 2) mt = fmax3(mt, x[t], x[t + 1]);
      float *rd = red + TPR * 128 * (n & 1);
      rd[128 * qt + il] = mt;
      // the next tile's v.r into the other buffer (read last by tile n - 1's skew)
      if (MECH == M_TXL && tid < 256 && n + 1 < nTiles) vec[512 * ((n + 1) & 1) + 128 + tid] = nvr;
      named_bar_sync(1, NSOFT);
      mt = rd[il];
#pragma unroll
      for (int u = 1; u < TPR; ++u) mt = fmaxf(mt, rd[128 * u + il]);
      if (n == 0) {
        m2 = mt;
      } else {
        const bool need = mt > m2 + 8.f;  // identical in every thread of the row
        if (__any_sync(0xffffffffu, need)) {
          good = good && warp_wait(BAR(B_PV), (n - 1) & 1, abort_flag, status);
          const float alpha = need ? ex2(m2 - mt) : 1.f;
          if (good) {
            tc_fence_after();
            uint32_t r[16];
            tmem_ld16(tl + TM_O + 16 * qt, r);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 16; ++t) r[t] = __float_as_uint(u2f(r[t]) * alpha);
            tmem_st16(tl + TM_O + 16 * qt, r);
            tmem_wait_st();
          }
          if (need) {
            lsum *= alpha;
            if (SV) {
              sL *= alpha;
              sR *= alpha;
            }
            m2 = mt;
          }
        }
      }
      const float msub = (m2 == -INFINITY) ? 0.f : m2;
      {
        const uint64_t nm = f2(-msub, -msub);
        uint64_t ls = f2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < NC; t += 2) {
          float a, b;
          f2_split(add2(f2(x[t], x[t + 1]), nm), a, b);
          x[t] = ex2(a);
          x[t + 1] = ex2(b);
          ls = add2(ls, f2(x[t], x[t + 1]));
        }
        float l0, l1;
        f2_split(ls, l0, l1);
        lsum += l0 + l1;
      }
      if (n >= 1) good = good && warp_wait(BAR(B_PV), (n - 1) & 1, abort_flag, status);
      if constexpr (SV) {
        const int d0 = j0 + cb - i;  // delta of this thread's first key
        const int eLo = max(0, 1 - p.clip - d0), eHi = min(NC - 1, p.clip - 1 - d0);  // unclipped: eLo..eHi
#pragma unroll
        for (int e = 0; e < NC; ++e) {
          if (e < eLo) sL += x[e];
          else if (e > eHi) sR += x[e];
        }
        if (good) {
          uint32_t pk[NC / 2];
#pragma unroll
          for (int k = 0; k < NC / 2; ++k) pk[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
          tmem_st16(tl + TM_PD + 16 * qt, pk);
          if (shaw_band(p.clip, m, n)) {
#pragma unroll
            for (int k = 0; k < NC / 2; ++k) {
              const float v0 = (2 * k >= eLo && 2 * k <= eHi) ? x[2 * k] : 0.f;
              const float v1 = (2 * k + 1 >= eLo && 2 * k + 1 <= eHi) ? x[2 * k + 1] : 0.f;
              pk[k] = pack_bf16x2(v0, v1);
            }
            store_pe(smem + OFF_P, il, (uint32_t)(d0 + p.clip) & 127u, pk);
          }
          tmem_wait_st();
          fence_async_smem();
          tc_fence_before();
          mbar_arrive(BAR(B_PFULL));
        }
      } else if (good) {  // P (bf16 pairs) into TMEM for the PV MMA, eight columns at a time
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) pk[k] = pack_bf16x2(x[16 * hh + 2 * k], x[16 * hh + 2 * k + 1]);
          tmem_st8(tl + TM_PD + 16 * qt + 8 * hh, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(B_PFULL));
      }
    }
    // ---- epilogue: O / l (l summed over the row's threads), LSE ----
    float *rl = red + TPR * 128 * (nTiles & 1);
    rl[128 * qt + il] = lsum;
    if (SV) {  // the per-tile vector buffer is unused by Shaw: it carries the clipped sums
      vec[128 * qt + il] = sL;
      vec[512 + 128 * qt + il] = sR;
    }
    named_bar_sync(1, NSOFT);
    float ltot = 0.f, sLt = 0.f, sRt = 0.f;
#pragma unroll
    for (int u = 0; u < TPR; ++u) ltot += rl[128 * u + il];
    if (SV) {
#pragma unroll
      for (int u = 0; u < TPR; ++u) {
        sLt += vec[128 * u + il];
        sRt += vec[512 + 128 * u + il];
      }
    }
    good = good && warp_wait(BAR(B_PV), (nTiles - 1) & 1, abort_flag, status);
    if (good) {
      tc_fence_after();
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      __nv_bfloat16 *orow = (__nv_bfloat16 *)p.out + ((size_t)bh * L + i) * HD + 16 * qt;
      uint32_t r[16];
      tmem_ld16(tl + TM_O + 16 * qt, r);
      tmem_wait_ld();
      if (SV) {  // clipped pairs: O += sL aV[0] + sR aV[2c]
        const __nv_bfloat16 *a0 = (const __nv_bfloat16 *)p.rel1 + (size_t)h * p.nrows * HD + 16 * qt;
        const __nv_bfloat16 *a1 = a0 + (size_t)(2 * p.clip) * HD;
#pragma unroll
        for (int e = 0; e < 16; ++e)
          r[e] = __float_as_uint(u2f(r[e]) + sLt * __bfloat162float(a0[e]) + sRt * __bfloat162float(a1[e]));
      }
      if (i < L) {
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          uint4 v;
          v.x = pack_bf16x2(u2f(r[8 * c8 + 0]) * inv, u2f(r[8 * c8 + 1]) * inv);
          v.y = pack_bf16x2(u2f(r[8 * c8 + 2]) * inv, u2f(r[8 * c8 + 3]) * inv);
          v.z = pack_bf16x2(u2f(r[8 * c8 + 4]) * inv, u2f(r[8 * c8 + 5]) * inv);
          v.w = pack_bf16x2(u2f(r[8 * c8 + 6]) * inv, u2f(r[8 * c8 + 7]) * inv);
          if (dcheck((size_t)(orow + 8 * c8 - (__nv_bfloat16 *)p.out) + 8 <= (size_t)BH * L * HD, status))
            *reinterpret_cast<uint4 *>(orow + 8 * c8) = v;
        }
        if (qt == 0 && dcheck((size_t)bh * L + i < (size_t)BH * L, status))
          p.lse[(size_t)bh * L + i] = ltot > 0.f ? (m2 + log2f(ltot)) * 0.6931471805599453f : -INFINITY;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TM_COLS);
  }
}

// Per-call products for the tensor-core forward: Transformer-XL u.k_j and v.r_rho,
// DeBERTa end-row products q_i.Kr[0], q_i.Kr[2k-1], k_j.Qr[0], k_j.Qr[2k-1].
// Per-row / per-offset products of the relation stage.  Eight threads share one
// 64-element row (eight consecutive elements each, so a warp reads four whole rows),
// and the partial dot products are combined by a fixed shuffle tree.
//   TXL      uk[b,h,j] = u_h . k_j  and  vr[h,rho] = v_h . r_rho
//   DeBERTa  c2pE[b,h,i] = (q_i . Kr_0, q_i . Kr_last), p2cE[b,h,j] = (k_j . Qr_0, k_j . Qr_last)
// a . b over eight bf16: a is 16-byte aligned (a row of q, k or a table, which the tensor-core
// path requires aligned) and read in one load; b (a per-head vector or a table row) may be
// read element by element
template <bool B_ALIGNED = false>
__device__ __forceinline__ float dot8(const __nv_bfloat16 *a, const __nv_bfloat16 *b) {
  const uint4 av = __ldg(reinterpret_cast<const uint4 *>(a));
  const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
  uint32_t bw[4];
  if constexpr (B_ALIGNED) {
    const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(b));
    bw[0] = bv.x;
    bw[1] = bv.y;
    bw[2] = bv.z;
    bw[3] = bv.w;
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float alo = __uint_as_float(aw[c] << 16), ahi = __uint_as_float(aw[c] & 0xFFFF0000u);
    float blo, bhi;
    if constexpr (B_ALIGNED) {
      blo = __uint_as_float(bw[c] << 16);
      bhi = __uint_as_float(bw[c] & 0xFFFF0000u);
    } else {
      blo = __bfloat162float(b[2 * c]);
      bhi = __bfloat162float(b[2 * c + 1]);
    }
    s = fmaf(alo, blo, s);
    s = fmaf(ahi, bhi, s);
  }
  return s;
}
__device__ __forceinline__ float sum8(float x) {  // over the eight threads of a row
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}
__global__ void __launch_bounds__(256) tc_prep_kernel(Prm p, float *uk, float *vr, float *c2pE, float *p2cE) {
  typedef __nv_bfloat16 bf;
  const size_t row = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 3;
  const int sub = threadIdx.x & 7;
  const size_t rows = (size_t)p.B * p.H * p.L;
  if (p.mech == M_TXL) {
    const size_t nr = rows + (size_t)p.H * p.nrows;  // key rows, then table rows
    float a = 0.f;
    if (row < rows) {
      const int h = (int)((row / p.L) % p.H);
      a = dot8((const bf *)p.k + row * HD + 8 * sub, (const bf *)p.rel1 + (size_t)h * HD + 8 * sub);
    } else if (row < nr) {
      const size_t rr = row - rows;
      const int h = (int)(rr / p.nrows);
      a = dot8((const bf *)p.rel0 + rr * HD + 8 * sub, (const bf *)p.rel2 + (size_t)h * HD + 8 * sub);
    }
    a = sum8(a);
    if (sub == 0) {
      if (row < rows) uk[row] = a;
      else if (row < nr) vr[row - rows] = a;
    }
  } else if (p.mech == M_DEB) {
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
    if (row < rows) {
      const int h = (int)((row / p.L) % p.H);
      const bf *q = (const bf *)p.q + row * HD + 8 * sub, *k = (const bf *)p.k + row * HD + 8 * sub;
      const bf *Kr = (const bf *)p.rel0 + (size_t)h * p.nrows * HD + 8 * sub;
      const bf *Qr = (const bf *)p.rel1 + (size_t)h * p.nrows * HD + 8 * sub;
      const size_t last = (size_t)(p.nrows - 1) * HD;
      a0 = dot8<true>(q, Kr);
      a1 = dot8<true>(q, Kr + last);
      b0 = dot8<true>(k, Qr);
      b1 = dot8<true>(k, Qr + last);
    }
    a0 = sum8(a0);
    a1 = sum8(a1);
    b0 = sum8(b0);
    b1 = sum8(b1);
    if (row < rows && sub == 0) {
      c2pE[2 * row] = a0;
      c2pE[2 * row + 1] = a1;
      p2cE[2 * row] = b0;
      p2cE[2 * row + 1] = b1;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)f;
  }
  return fn;
}

// [planes][rows][64] bf16 viewed as a 3D tensor; box = 64 x box_rows x 1, 128B swizzle,
// rows outside [0, rows) read as zeros.
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t planes, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, rows, planes};
  cuuint64_t strides[2] = {64 * 2, rows * 64 * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MECH, bool VAL = false>
static cudaError_t launch_fwd_t(const FwdArgs &a, cudaStream_t st) {
  auto k = tc_fwd_kernel<MECH, VAL>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // query tiles holding only Transformer-XL memory placeholders (rows < mem_len) are not launched
  RP_TRACED("tc_fwd_kernel", st, k<<<(unsigned)((a.p.nT - a.p.mem_len / BM) * a.p.H * a.p.B), NTHREADS, SMEM_BYTES, st>>>(a));
  return cudaGetLastError();
}

}  // namespace tc

// [planes][rows][row_len] fp32 rows (row_len * 4 bytes a multiple of 16), no swizzle;
// box = row_len x box_rows x 1 lands as contiguous padded rows; rows outside
// [0, rows) read as zeros.
bool tc_make_map_f32_rows(CUtensorMap *m, const void *base, uint32_t row_len, uint64_t rows, uint64_t planes,
                          uint32_t box_rows) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc || (row_len * 4u) % 16u != 0 || row_len > 256) return false;
  cuuint64_t dims[3] = {row_len, rows, planes};
  cuuint64_t strides[2] = {(cuuint64_t)row_len * 4, (cuuint64_t)rows * row_len * 4};
  cuuint32_t box[3] = {row_len, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tc_make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t planes, uint32_t box_rows) {
  return tc::make_map(m, base, rows, planes, box_rows);
}

// [planes][rows][row_len] bf16 (row_len a multiple of 64); box = 64 x box_rows x 1 at any
// 64-element column offset, 128B swizzle; rows and columns outside the tensor read as zeros.
bool tc_make_map_bf16_wide(CUtensorMap *m, const void *base, uint32_t row_len, uint64_t rows, uint64_t planes,
                           uint32_t box_rows) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc || row_len % 64u != 0) return false;
  cuuint64_t dims[3] = {row_len, rows, planes};
  cuuint64_t strides[2] = {(cuuint64_t)row_len * 2, (cuuint64_t)rows * row_len * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t tc_prep(const Prm &p, const TcWork &w, cudaStream_t st) {
  if (p.mech != M_TXL && p.mech != M_DEB) return cudaSuccess;
  const size_t rows = (size_t)p.B * p.H * p.L + (p.mech == M_TXL ? (size_t)p.H * p.nrows : 0);
  RP_TRACED("tc_prep_kernel", st, tc::tc_prep_kernel<<<(unsigned)((8 * rows + 255) / 256), 256, 0, st>>>(p, w.uk, w.vr, w.c2pE, w.p2cE));
  return cudaGetLastError();
}

bool tc_supported(const Prm &p) {
  if (p.mech == M_SHAW && 2 * p.clip + 1 > 131) return false;  // QA row must fit the 132-float smem row
  if (p.shaw_v && p.clip > 64) return false;  // the unclipped offsets 1 .. 2c - 1 must fit the 128 columns of Pe
  return true;
}

cudaError_t tc_fwd(const Prm &p, const TcWork &w, cudaStream_t st) {
  using namespace tc;
  FwdArgs a;
  memset(&a, 0, sizeof(a));
  a.p = p;
  a.p.nT = (p.L + BM - 1) / BM;  // 128-row tiles
  a.uk = w.uk;
  a.vr = w.vr;
  a.c2pE = w.c2pE;
  a.p2cE = w.p2cE;
  const uint64_t BH = (uint64_t)p.B * p.H;
  bool ok = make_map(&a.mq, p.q, p.L, BH, 128) && make_map(&a.mk, p.k, p.L, BH, 128) && make_map(&a.mv, p.v, p.L, BH, 128);
  if (p.mech == M_TXL) ok = ok && make_map(&a.mt0, p.rel0, p.nrows, p.H, 128);
  if (p.mech == M_SHAW) {
    a.shaw_n = ((2 * p.clip + 1) + 15) / 16 * 16;
    ok = ok && make_map(&a.mt0, p.rel0, p.nrows, p.H, a.shaw_n);
    if (p.shaw_v) ok = ok && make_map(&a.mt1, p.rel1, p.nrows, p.H, 128);  // aV rows 0..127 (past 2c: zeros)
  }
  if (p.mech == M_DEB) ok = ok && make_map(&a.mt0, p.rel0, p.nrows, p.H, 256) && make_map(&a.mt1, p.rel1, p.nrows, p.H, 256);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = tc_prep(p, w, st);
  if (e != cudaSuccess) return e;
  switch (p.mech) {
    case M_T5: return launch_fwd_t<M_T5>(a, st);
    case M_SHAW: return p.shaw_v ? launch_fwd_t<M_SHAW, true>(a, st) : launch_fwd_t<M_SHAW>(a, st);
    case M_TXL: return launch_fwd_t<M_TXL>(a, st);
    default: return launch_fwd_t<M_DEB>(a, st);
  }
}

}  // namespace rp
