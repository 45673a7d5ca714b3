// Shared definitions of the relative-position attention kernels (sm_100a).
//
// Notation follows "Fast and Exact Relative-Position Attention via
// Structure-Aware Kernels" (Abstract) and the article
// "结构感知内核让相对位置注意力加速21倍" (section "为什么相对位置注意力难做快"):
// S_ij = scale * q_i.k_j + R_ij, with R the mechanism's relative term.  For a
// pair (i, j) the offset is delta = j - i; each mechanism reads a table row
// rho(delta) that is monotone in delta, so a tile of queries x keys touches a
// contiguous window of offsets and a contiguous window of table rows (the
// "offset-aware tiling" of the Abstract, technique (1); article section
// "1. 偏移感知分块").
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace rp {

constexpr int HD = 64;  // head dimension supported by every kernel
constexpr int RELPOS_ERR_TIMEOUT_DEV = -5;  // value of RELPOS_ERR_TIMEOUT written to the device status word
constexpr int RELPOS_ERR_BOUNDS_DEV = -7;   // value of RELPOS_ERR_BOUNDS (debug build)

// Index check of the debug build (RELPOS_DEBUG): true when the access may go ahead.  A
// failed check writes RELPOS_ERR_BOUNDS to the status word and the caller skips the
// access; control flow is otherwise unchanged, so every barrier stays balanced.  In the
// release build it is the constant true and the check disappears.
__device__ __forceinline__ bool dcheck(bool ok, int32_t *status) {
#ifdef RELPOS_DEBUG
  if (!ok && status) *status = RELPOS_ERR_BOUNDS_DEV;
  return ok;
#else
  (void)status;
  (void)ok;
  return true;
#endif
}

enum { M_T5 = 0, M_SHAW = 1, M_TXL = 2, M_DEB = 3 };

// Parameters of one call, passed by value to every kernel.
struct Prm {
  int mech, causal, B, H, L;
  int nrows;   // rows of the (row side) relative table of one head
  int off;     // Transformer-XL: row of offset delta is -delta + off
  float scale;
  // T5 buckets: exact-distance buckets below `me`, then thresholds thr[0..nthr)
  // (smallest distance of log buckets me+1, me+2, ...), capped at half-1.
  int nb, bidir, half, me, nthr;
  int thr[32];
  // ALiBi runs on the T5 per-offset path (mech M_T5, one "bucket"): its bias vector
  // is -m[h] |delta| and its slope gradient weights each offset's dS sum by -|delta|.
  int alibi;
  int clip;   // Shaw clip c
  int shaw_v;  // Shaw: value-side table rel1 = aV (O_i += sum_j P_ij aV[row(j - i)])
  int mem_len, esize;  // host bookkeeping: Transformer-XL memory length (L counts it), element bytes
  int span;   // DeBERTa span k
  int nT;     // number of 64-row tiles
  int diag_ch, diag_nchunk, nbands;  // Transformer-XL diagonal shards
  // tensors
  const void *q, *k, *v, *o, *dout;
  const void *rel0, *rel1, *rel2;
  void *out, *dq, *dk, *dv;
  float *lse, *drel0, *drel1, *drel2;
  // workspace
  float *t5_bias;      // [H][2L-1]   t[h, bucket(delta)] (ALiBi: -m[h] |delta|) at delta + L - 1
  int *t5_bkt;         // [2L-1]      bucket(delta) (ALiBi: 0)
  float *Dvec;         // [B][H][L]   D_i = dO_i . O_i
  float *part_row;     // per (b,h,query tile) partial of the query-side table gradient
  float *part_col;     // per (b,h,key tile) partial of the key-side table gradient
  float *part_small;   // T5 bucket partials / Transformer-XL du partials
  float *part_diag;    // Transformer-XL per-diagonal-shard partials
  float *part_val;     // Shaw value term: per (b,h,query tile) partial of daV
  float *gtot;         // Transformer-XL [H][n_off] diagonal sums of dS
  int *status;
  const int *seqlens_k;  // [B] key lengths (device), or null: every batch has L keys
  int klen;              // this CTA's key length (set by kernels that mask keys)
};

// Key length of batch b: keys j >= key_len are masked (variable-length batches).
__device__ __forceinline__ int key_len(const Prm &p, int b) {
  if (!p.seqlens_k) return p.L;
  const int v = p.seqlens_k[b];
  return v < 0 ? 0 : (v > p.L ? p.L : v);
}

// ---------------------------------------------------------------------------
// element access
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ldf(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void stf(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, size_t i, float x) { p[i] = __float2bfloat16_rn(x); }

// ---------------------------------------------------------------------------
// T5 bucket of n = j - i (integer thresholds computed exactly on the host)
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int t5_bucket(const Prm &p, int n) {
  int base = 0, a;
  if (p.bidir) {
    base = n > 0 ? p.half : 0;
    a = n < 0 ? -n : n;
  } else {
    a = n < 0 ? -n : 0;
  }
  if (a < p.me) return base + a;
  int t = 0;
  for (int s = 0; s < p.nthr; ++s)
    if (a >= p.thr[s]) t = s + 1;
  int bk = p.me + t;
  if (bk > p.half - 1) bk = p.half - 1;
  return base + bk;
}

__host__ __device__ __forceinline__ int iclamp(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Query-side table row of offset delta = j - i (Shaw a, Transformer-XL r,
// DeBERTa Kr).  Transformer-XL rows outside [0, nrows) belong to masked or
// padded pairs only.
template <int MECH>
__device__ __forceinline__ int rho_row(const Prm &p, int delta) {
  if (MECH == M_SHAW) return iclamp(delta, -p.clip, p.clip) + p.clip;
  if (MECH == M_TXL) return -delta + p.off;
  return iclamp(-delta + p.span, 0, 2 * p.span - 1);  // DeBERTa c2p
}
// Key-side table row (DeBERTa Qr) of offset delta = j - i.
__device__ __forceinline__ int rho_col(const Prm &p, int delta) { return iclamp(delta + p.span, 0, 2 * p.span - 1); }

// Table-row window [lo, lo+n) that the offsets delta in [dmin, dmax] read.
template <int MECH>
__device__ __forceinline__ void row_window(const Prm &p, int dmin, int dmax, int &lo, int &n) {
  int a = rho_row<MECH>(p, dmin), b = rho_row<MECH>(p, dmax);
  int l = a < b ? a : b, h = a < b ? b : a;
  if (l < 0) l = 0;
  if (h > p.nrows - 1) h = p.nrows - 1;
  lo = l;
  n = h >= l ? h - l + 1 : 0;
}
__device__ __forceinline__ void col_window(const Prm &p, int dmin, int dmax, int &lo, int &n) {
  lo = rho_col(p, dmin);
  n = rho_col(p, dmax) - lo + 1;
}

// Does the mechanism clip offsets onto end rows 0 and nrows-1?
template <int MECH>
__device__ __forceinline__ bool has_ends() { return MECH == M_SHAW || MECH == M_DEB; }

}  // namespace rp
