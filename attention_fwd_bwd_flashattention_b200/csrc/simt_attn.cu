// CUDA-core (fp32 FFMA) kernels for relative-position attention, forward and
// backward, all four mechanisms.  This is the float32 path of the library (and the
// bfloat16 path of the cases the tensor-core kernels do not take).  Like every other
// kernel of the library it is checked against the fp64 CPU oracle, element by element
// on the same inputs; no kernel serves as another's reference.
//
// The structure is the method's, at 64 x 64 tiles:
//  * offset-aware tiling: a query tile x key tile pair touches the offset window
//    delta = j - i in [j0 - i0 - 63, j0 - i0 + 63] and a contiguous window of
//    table rows ("Fast and Exact Relative-Position Attention via Structure-Aware
//    Kernels", Abstract, technique (1)),
//  * relation products only for that window: W = X . Tab_window^T (one small GEMM
//    per tile) gathered into the score tile by offset (technique (2); article
//    "结构感知内核让相对位置注意力加速21倍", section "2. 复用查询—键关系乘积"),
//  * online softmax with the relative term added before the running max (article
//    section "结构感知分块如何保持精确性"),
//  * a backward pass with no atomics: dK/dV in a key-tile-parallel kernel, dQ in a
//    query-tile-parallel kernel, relative-table gradients accumulated in per-shard
//    partials (per query tile, per key tile, or per diagonal band of tiles for
//    Transformer-XL) and merged by a fixed-order reduction (technique (3); article
//    section "3. 基于偏移的梯度分片").
#include "common.cuh"
#include "kernels.h"

namespace rp {
namespace simt {

constexpr int BM = 64, BN = 64, NT = 256, LDX = HD + 1, WS = 145, TROWS = 128;
constexpr float LOG2E = 1.4426950408889634f;

// aux (small per-tile vectors) layout, in floats
constexpr int A_U = 0, A_V = 64, A_UK = 128, A_VT = 192, A_BIAS = 320, A_LSE = 448, A_D = 512, A_G = 576,
              A_ACC = 704, A_CS = 768, A_SIZE = 1024;

struct Sm {
  float *Q, *K, *V, *dO, *T, *W, *P, *dS, *aux;
};

constexpr int SMEM_FLOATS = 4 * BM * LDX + TROWS * LDX + BM * WS + 2 * BM * LDX + A_SIZE;
constexpr size_t SMEM_BYTES = SMEM_FLOATS * sizeof(float);

__device__ __forceinline__ Sm carve(float *s) {
  Sm m;
  m.Q = s;
  m.K = m.Q + BM * LDX;
  m.V = m.K + BN * LDX;
  m.dO = m.V + BN * LDX;
  m.T = m.dO + BM * LDX;
  m.W = m.T + TROWS * LDX;
  m.P = m.W + BM * WS;
  m.dS = m.P + BM * LDX;
  m.aux = m.dS + BM * LDX;
  return m;
}

// ---------------------------------------------------------------------------
// register-tiled smem GEMMs; thread (ty, tx) owns rows ty + 16a, cols tx + 16b
// ---------------------------------------------------------------------------
// acc[a][b] += sum_k A[(ty+16a)*lda + k] * B[(tx+16b)*ldb + k]
template <int NA, int NB>
__device__ __forceinline__ void mm_nt(const float *A, int lda, const float *B, int ldb, int K, float (&acc)[NA][NB]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 4
  for (int kk = 0; kk < K; ++kk) {
    float a[NA], b[NB];
#pragma unroll
    for (int i = 0; i < NA; ++i) a[i] = A[(ty + 16 * i) * lda + kk];
#pragma unroll
    for (int j = 0; j < NB; ++j) b[j] = B[(tx + 16 * j) * ldb + kk];
#pragma unroll
    for (int i = 0; i < NA; ++i)
#pragma unroll
      for (int j = 0; j < NB; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}
// acc[a][b] += sum_k A[(ty+16a)*lda + k] * B[k*ldb + tx+16b]
template <int NA, int NB>
__device__ __forceinline__ void mm_nn(const float *A, int lda, const float *B, int ldb, int K, float (&acc)[NA][NB]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 4
  for (int kk = 0; kk < K; ++kk) {
    float a[NA], b[NB];
#pragma unroll
    for (int i = 0; i < NA; ++i) a[i] = A[(ty + 16 * i) * lda + kk];
#pragma unroll
    for (int j = 0; j < NB; ++j) b[j] = B[kk * ldb + tx + 16 * j];
#pragma unroll
    for (int i = 0; i < NA; ++i)
#pragma unroll
      for (int j = 0; j < NB; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}
// acc[a][b] += sum_k A[k*lda + ty+16a] * B[k*ldb + tx+16b]
template <int NA, int NB>
__device__ __forceinline__ void mm_tn(const float *A, int lda, const float *B, int ldb, int K, float (&acc)[NA][NB]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 4
  for (int kk = 0; kk < K; ++kk) {
    float a[NA], b[NB];
#pragma unroll
    for (int i = 0; i < NA; ++i) a[i] = A[kk * lda + ty + 16 * i];
#pragma unroll
    for (int j = 0; j < NB; ++j) b[j] = B[kk * ldb + tx + 16 * j];
#pragma unroll
    for (int i = 0; i < NA; ++i)
#pragma unroll
      for (int j = 0; j < NB; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

__device__ __forceinline__ float hsum16(float x) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float hmax16(float x) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// rows [r0, r0+64) of a [L, 64] matrix into dst[64][LDX] (zeros past L)
template <class T>
__device__ __forceinline__ void load_rows(const T *src, int r0, int L, float *dst) {
  for (int x = threadIdx.x; x < 64 * HD; x += NT) {
    int r = x >> 6, c = x & 63;
    dst[r * LDX + c] = (r0 + r < L) ? ldf(src, (size_t)(r0 + r) * HD + c) : 0.f;
  }
}
// table rows [lo, lo+n) of one head into dst[TROWS][LDX]
template <class T>
__device__ __forceinline__ void load_tab(const T *tab, int lo, int n, float *dst) {
  for (int x = threadIdx.x; x < n * HD; x += NT) {
    int w = x >> 6, c = x & 63;
    dst[w * LDX + c] = ldf(tab, (size_t)(lo + w) * HD + c);
  }
}
template <class T>
__device__ __forceinline__ void load_vec64(const T *src, float *dst) {
  if (threadIdx.x < HD) dst[threadIdx.x] = ldf(src, threadIdx.x);
}

// T5: bias window aux[A_BIAS + w] = bias(delta = dmin + w), w in [0, 127)
__device__ __forceinline__ void load_bias_window(const Prm &p, const Sm &sm, int h, int dmin) {
  if (threadIdx.x < TROWS) {
    int idx = dmin + (int)threadIdx.x + p.L - 1;
    sm.aux[A_BIAS + threadIdx.x] = (idx >= 0 && idx < 2 * p.L - 1) ? p.t5_bias[(size_t)h * (2 * p.L - 1) + idx] : 0.f;
  }
}

// W[r][w] = X_r . T_w for r in [0,64), w in [0, nw)   (thread: 4 rows x 8 window cols)
__device__ __forceinline__ void window_gemm(const float *X, const float *T, int nw, float *W) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  mm_nt<4, 8>(X, LDX, T, LDX, HD, acc);
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b)
      if (tx + 16 * b < nw) W[(ty + 16 * a) * WS + tx + 16 * b] = acc[a][b];
}

// ---------------------------------------------------------------------------
// Score tile S (scaled, relative term added, masked) for queries [i0, i0+64)
// and keys [j0, j0+64).  TRANS = false: S[a][b] is (query ty+16a, key tx+16b);
// TRANS = true: (key ty+16a, query tx+16b).  Q and K tiles must be in smem.
// Contains __syncthreads(); must be called by the whole block.
// ---------------------------------------------------------------------------
template <int MECH, bool TRANS, class T>
__device__ __forceinline__ void scores(const Prm &p, const Sm &sm, int h, int i0, int j0, float (&S)[4][4]) {
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) S[a][b] = 0.f;
  if (TRANS)
    mm_nt<4, 4>(sm.K, LDX, sm.Q, LDX, HD, S);
  else
    mm_nt<4, 4>(sm.Q, LDX, sm.K, LDX, HD, S);
  const int dmin = j0 - (i0 + BM - 1), dmax = j0 + BN - 1 - i0;
  if (MECH == M_TXL && tid < BN) {  // u . k_j for this key tile
    float acc = 0.f;
    for (int kk = 0; kk < HD; ++kk) acc = fmaf(sm.aux[A_U + kk], sm.K[tid * LDX + kk], acc);
    sm.aux[A_UK + tid] = acc;
  }
  if (MECH != M_T5) {
    int lo, nw;
    row_window<MECH>(p, dmin, dmax, lo, nw);
    load_tab((const T *)p.rel0 + (size_t)h * p.nrows * HD, lo, nw, sm.T);
    __syncthreads();
    if (MECH == M_TXL && tid < nw) {  // v . r_rho for the window rows
      float acc = 0.f;
      for (int kk = 0; kk < HD; ++kk) acc = fmaf(sm.aux[A_V + kk], sm.T[tid * LDX + kk], acc);
      sm.aux[A_VT + tid] = acc;
    }
    window_gemm(sm.Q, sm.T, nw, sm.W);
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int r = TRANS ? tx + 16 * b : ty + 16 * a, c = TRANS ? ty + 16 * a : tx + 16 * b;
        const int w = rho_row<MECH>(p, (j0 + c) - (i0 + r)) - lo;
        if (w >= 0 && w < nw) {
          float x = sm.W[r * WS + w];
          if (MECH == M_TXL) x += sm.aux[A_VT + w];
          S[a][b] += x;
        }
      }
    if (MECH == M_DEB) {
      __syncthreads();
      int lo2, nw2;
      col_window(p, dmin, dmax, lo2, nw2);
      load_tab((const T *)p.rel1 + (size_t)h * p.nrows * HD, lo2, nw2, sm.T);
      __syncthreads();
      window_gemm(sm.K, sm.T, nw2, sm.W);
      __syncthreads();
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int r = TRANS ? tx + 16 * b : ty + 16 * a, c = TRANS ? ty + 16 * a : tx + 16 * b;
          S[a][b] += sm.W[c * WS + rho_col(p, (j0 + c) - (i0 + r)) - lo2];
        }
    }
    if (MECH == M_TXL) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) S[a][b] += sm.aux[A_UK + (TRANS ? ty + 16 * a : tx + 16 * b)];
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r = TRANS ? tx + 16 * b : ty + 16 * a, c = TRANS ? ty + 16 * a : tx + 16 * b;
      const int i = i0 + r, j = j0 + c;
      float s = S[a][b] * p.scale;
      if (MECH == M_T5) s += sm.aux[A_BIAS + (j - i) - dmin];
      if (i >= p.L || j >= p.klen || (p.causal && j > i)) s = -INFINITY;
      S[a][b] = s;
    }
}

template <int MECH, bool COLSIDE, bool TRANS>
__device__ __forceinline__ void scatter_E(const Prm &p, const float (&dS)[4][4], float *E, int i0, int j0, int lo, int nw);
__device__ __forceinline__ void zero_W(float *W, int nw);

// ---------------------------------------------------------------------------
// forward: one CTA per (query tile, head, batch)
// ---------------------------------------------------------------------------
template <int MECH, class T>
__global__ void __launch_bounds__(NT, 1) fwd_kernel(Prm p) {
  p.klen = key_len(p, blockIdx.z);
  extern __shared__ float smem[];
  const Sm sm = carve(smem);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m = (int)blockIdx.x + p.mem_len / BM, h = blockIdx.y, b = blockIdx.z;  // memory-placeholder tiles skipped
  const int L = p.L, i0 = m * BM;
  const size_t base = ((size_t)b * p.H + h) * (size_t)L * HD;
  const T *Qg = (const T *)p.q + base, *Kg = (const T *)p.k + base, *Vg = (const T *)p.v + base;
  load_rows(Qg, i0, L, sm.Q);
  if (MECH == M_TXL) {
    load_vec64((const T *)p.rel1 + (size_t)h * HD, sm.aux + A_U);
    load_vec64((const T *)p.rel2 + (size_t)h * HD, sm.aux + A_V);
  }
  float O[4][4], mrow[4], lrow[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    mrow[a] = -INFINITY;
    lrow[a] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) O[a][e] = 0.f;
  }
  int nEnd = p.nT;
  if (p.causal) nEnd = min(p.nT, (i0 + BM - 1) / BN + 1);
  for (int n = 0; n < nEnd; ++n) {
    const int j0 = n * BN;
    __syncthreads();
    load_rows(Kg, j0, L, sm.K);
    load_rows(Vg, j0, L, sm.V);
    if (MECH == M_T5) load_bias_window(p, sm, h, j0 - (i0 + BM - 1));
    __syncthreads();
    float S[4][4];
    scores<MECH, false, T>(p, sm, h, i0, j0, S);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float mx = fmaxf(fmaxf(S[a][0], S[a][1]), fmaxf(S[a][2], S[a][3]));
      mx = hmax16(mx);
      const float mnew = fmaxf(mrow[a], mx);
      const float muse = (mnew == -INFINITY) ? 0.f : mnew;
      const float alpha = exp2f((mrow[a] - muse) * LOG2E);
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        S[a][c] = exp2f((S[a][c] - muse) * LOG2E);
        sum += S[a][c];
      }
      sum = hsum16(sum);
      lrow[a] = lrow[a] * alpha + sum;
#pragma unroll
      for (int e = 0; e < 4; ++e) O[a][e] *= alpha;
      mrow[a] = mnew;
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) sm.P[(ty + 16 * a) * LDX + tx + 16 * c] = S[a][c];
    __syncthreads();
    mm_nn<4, 4>(sm.P, LDX, sm.V, LDX, BN, O);
    if (MECH == M_SHAW && p.shaw_v) {
      // value term: O_i += sum_rho Pe[i][rho] aV_rho, Pe = P by table row (window of the tile)
      int lo, nw;
      row_window<MECH>(p, j0 - (i0 + BM - 1), j0 + BN - 1 - i0, lo, nw);
      zero_W(sm.W, 0);
      __syncthreads();
      scatter_E<MECH, false, false>(p, S, sm.W, i0, j0, lo, nw);
      load_tab((const T *)p.rel1 + (size_t)h * p.nrows * HD, lo, nw, sm.T);
      __syncthreads();
      mm_nn<4, 4>(sm.W, WS, sm.T, LDX, nw, O);
    }
  }
  T *Og = (T *)p.out + base;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
    if (i < L) {
      const float inv = lrow[a] > 0.f ? 1.f / lrow[a] : 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) stf(Og, (size_t)i * HD + tx + 16 * e, O[a][e] * inv);
      if (tx == 0)
        p.lse[((size_t)b * p.H + h) * L + i] = lrow[a] > 0.f ? mrow[a] + logf(lrow[a]) : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------------------
// backward helpers
// ---------------------------------------------------------------------------
// P and dS of a tile from S; rows of the (query) statistics come from aux.
template <bool TRANS>
__device__ __forceinline__ void probs_and_ds(const Sm &sm, float (&S)[4][4], const float (&dP)[4][4], float (&dS)[4][4]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r = TRANS ? tx + 16 * b : ty + 16 * a;
      const float pr = exp2f((S[a][b] - sm.aux[A_LSE + r]) * LOG2E);  // S = -inf -> 0
      S[a][b] = pr;
      dS[a][b] = pr * (dP[a][b] - sm.aux[A_D + r]);
    }
}

// LSE and D of query rows [i0, i0+64) into aux (0 past L).
__device__ __forceinline__ void load_row_stats(const Prm &p, const Sm &sm, size_t bh, int i0) {
  if (threadIdx.x < BM) {
    const int i = i0 + threadIdx.x;
    const bool ok = i < p.L;
    float l = ok ? p.lse[bh * p.L + i] : 0.f;
    if (l == -INFINITY) l = 0.f;  // empty rows have P = 0 already (S = -inf)
    sm.aux[A_LSE + threadIdx.x] = l;
    sm.aux[A_D + threadIdx.x] = ok ? p.Dvec[bh * p.L + i] : 0.f;
  }
}

// Scatter a dS tile into E[x][rho - lo] (row space of the table window), where
// x is this thread's register row (query for the query side, key for the key
// side).  Pairs that fall on an end row of a clipping table are summed across
// the 16 lanes of the row in a fixed butterfly order.  E must be zeroed first.
template <int MECH, bool COLSIDE, bool TRANS>
__device__ __forceinline__ void scatter_E(const Prm &p, const float (&dS)[4][4], float *E, int i0, int j0, int lo, int nw) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int last = p.nrows - 1;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    float e0 = 0.f, e1 = 0.f;
    const int x = ty + 16 * a;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r = TRANS ? tx + 16 * b : x, c = TRANS ? x : tx + 16 * b;
      const int i = i0 + r, j = j0 + c;
      if (i >= p.L || j >= p.klen || (p.causal && j > i)) continue;
      const int rho = COLSIDE ? rho_col(p, j - i) : rho_row<MECH>(p, j - i);
      if (has_ends<MECH>() && rho == 0)
        e0 += dS[a][b];
      else if (has_ends<MECH>() && rho == last)
        e1 += dS[a][b];
      else
        E[x * WS + rho - lo] = dS[a][b];
    }
    if (has_ends<MECH>()) {
      e0 = hsum16(e0);
      e1 = hsum16(e1);
      if (tx == 0) {
        if (lo == 0) E[x * WS] += e0;
        if (lo + nw - 1 == last) E[x * WS + last - lo] += e1;
      }
    }
  }
}

// Shaw value term in dP: dP_ij += dO_i . aV[row(j - i)] for the tile's pairs (TRANS as in
// scores()).  The window products dO . aV_w come from one small GEMM; contains
// __syncthreads() and uses T / W, which scores() has finished with.
template <bool TRANS, class T>
__device__ __forceinline__ void value_dp(const Prm &p, const Sm &sm, int h, int i0, int j0, int dmin, int dmax,
                                         float (&dP)[4][4]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  int lo, nw;
  row_window<M_SHAW>(p, dmin, dmax, lo, nw);
  __syncthreads();
  load_tab((const T *)p.rel1 + (size_t)h * p.nrows * HD, lo, nw, sm.T);
  __syncthreads();
  window_gemm(sm.dO, sm.T, nw, sm.W);  // W[r][w] = dO_r . aV_{lo + w}
  __syncthreads();
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r = TRANS ? tx + 16 * b : ty + 16 * a, c = TRANS ? ty + 16 * a : tx + 16 * b;
      const int w = rho_row<M_SHAW>(p, (j0 + c) - (i0 + r)) - lo;
      if (w >= 0 && w < nw) dP[a][b] += sm.W[r * WS + w];
    }
}

__device__ __forceinline__ void zero_W(float *W, int nw) {
  for (int x = threadIdx.x; x < BM * WS; x += NT) W[x] = 0.f;
  (void)nw;
}

// ---------------------------------------------------------------------------
// D_i = dO_i . O_i
// ---------------------------------------------------------------------------
// eight threads per 64-element row (a warp reads four whole rows), fixed shuffle tree
template <class T>
__global__ void __launch_bounds__(256) dvec_kernel(Prm p) {
  const size_t n = (size_t)p.B * p.H * p.L;
  const size_t row = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 3;
  const int sub = threadIdx.x & 7;
  float acc = 0.f;
  if (row < n) {
    const T *o = (const T *)p.o + row * HD + 8 * sub, *g = (const T *)p.dout + row * HD + 8 * sub;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc = fmaf(ldf(o, c), ldf(g, c), acc);
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (row < n && sub == 0) p.Dvec[row] = acc;
}

// ---------------------------------------------------------------------------
// dQ (+ query-side table partials): one CTA per (query tile, head, batch)
// ---------------------------------------------------------------------------
template <int MECH, class T>
__global__ void __launch_bounds__(NT, 1) bwd_q_kernel(Prm p) {
  p.klen = key_len(p, blockIdx.z);
  extern __shared__ float smem[];
  const Sm sm = carve(smem);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m = (int)blockIdx.x + p.mem_len / BM, h = blockIdx.y, b = blockIdx.z;  // memory-placeholder tiles skipped
  const int L = p.L, i0 = m * BM;
  const size_t bh = (size_t)b * p.H + h, base = bh * (size_t)L * HD;
  const T *Qg = (const T *)p.q + base, *Kg = (const T *)p.k + base, *Vg = (const T *)p.v + base,
          *dOg = (const T *)p.dout + base;
  load_rows(Qg, i0, L, sm.Q);
  load_rows(dOg, i0, L, sm.dO);
  load_row_stats(p, sm, bh, i0);
  if (MECH == M_TXL) {
    load_vec64((const T *)p.rel1 + (size_t)h * HD, sm.aux + A_U);
    load_vec64((const T *)p.rel2 + (size_t)h * HD, sm.aux + A_V);
  }
  // this CTA's partial of the query-side table gradient (Shaw a, DeBERTa Kr)
  float *part = nullptr;
  float *partv = nullptr;  // Shaw value term: daV partial of this CTA
  if (MECH == M_SHAW || MECH == M_DEB) {
    part = p.part_row + (bh * p.nT + m) * (size_t)p.nrows * HD;
    for (int x = tid; x < p.nrows * HD; x += NT) part[x] = 0.f;
  }
  if (MECH == M_SHAW && p.shaw_v) {
    partv = p.part_val + (bh * p.nT + m) * (size_t)p.nrows * HD;
    for (int x = tid; x < p.nrows * HD; x += NT) partv[x] = 0.f;
  }
  if (MECH == M_T5 && tid < 64) sm.aux[A_ACC + tid] = 0.f;
  float dQ[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) dQ[a][e] = 0.f;
  int nEnd = p.nT;
  if (p.causal) nEnd = min(p.nT, (i0 + BM - 1) / BN + 1);
  for (int n = 0; n < nEnd; ++n) {
    const int j0 = n * BN;
    const int dmin = j0 - (i0 + BM - 1), dmax = j0 + BN - 1 - i0;
    __syncthreads();
    load_rows(Kg, j0, L, sm.K);
    load_rows(Vg, j0, L, sm.V);
    if (MECH == M_T5) load_bias_window(p, sm, h, dmin);
    __syncthreads();
    float S[4][4], dP[4][4], dS[4][4];
    scores<MECH, false, T>(p, sm, h, i0, j0, S);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) dP[a][c] = 0.f;
    mm_nt<4, 4>(sm.dO, LDX, sm.V, LDX, HD, dP);
    if (MECH == M_SHAW && p.shaw_v) value_dp<false, T>(p, sm, h, i0, j0, dmin, dmax, dP);
    probs_and_ds<false>(sm, S, dP, dS);
    __syncthreads();  // everyone is done reading W / T of the score stage
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) sm.dS[(ty + 16 * a) * LDX + tx + 16 * c] = dS[a][c];
    zero_W(sm.W, 0);
    __syncthreads();
    mm_nn<4, 4>(sm.dS, LDX, sm.K, LDX, BN, dQ);
    if (MECH == M_T5) {
      // diagonal sums g(delta) of dS, then folded into buckets in a fixed order
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int r = ty + 16 * a, cc = tx + 16 * c;
          sm.W[r * WS + (cc - r) + (BM - 1)] = dS[a][c];
        }
      __syncthreads();
      if (tid < TROWS - 1) {
        float g = 0.f;
        for (int r = 0; r < BM; ++r) g += sm.W[r * WS + tid];
        sm.aux[A_G + tid] = g;
      }
      __syncthreads();
      if (tid < p.nb) {
        float acc = sm.aux[A_ACC + tid];
        for (int w = 0; w < TROWS - 1; ++w) {
          const int delta = dmin + w;
          if (delta > -p.L && delta < p.L && p.t5_bkt[delta + p.L - 1] == tid)
            acc += p.alibi ? -fabsf((float)delta) * sm.aux[A_G + w] : sm.aux[A_G + w];
        }
        sm.aux[A_ACC + tid] = acc;
      }
    } else {
      int lo, nw;
      row_window<MECH>(p, dmin, dmax, lo, nw);
      scatter_E<MECH, false, false>(p, dS, sm.W, i0, j0, lo, nw);
      load_tab((const T *)p.rel0 + (size_t)h * p.nrows * HD, lo, nw, sm.T);
      __syncthreads();
      mm_nn<4, 4>(sm.W, WS, sm.T, LDX, nw, dQ);  // dq_i += sum_rho E[i][rho] Tab[rho]
      if (MECH == M_SHAW || MECH == M_DEB) {
        float G[8][4];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int e = 0; e < 4; ++e) G[a][e] = 0.f;
        mm_tn<8, 4>(sm.W, WS, sm.Q, LDX, BM, G);  // G[rho][e] = sum_i E[i][rho] q_i[e]
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const int w = ty + 16 * a;
          if (w < nw) {
#pragma unroll
            for (int e = 0; e < 4; ++e) part[(size_t)(lo + w) * HD + tx + 16 * e] += p.scale * G[a][e];
          }
        }
        if (MECH == M_SHAW && p.shaw_v) {  // daV[rho] += sum_i Pe[i][rho] dO_i (Pe: P by table row)
          __syncthreads();
          zero_W(sm.W, 0);
          __syncthreads();
          scatter_E<MECH, false, false>(p, S, sm.W, i0, j0, lo, nw);
          __syncthreads();
#pragma unroll
          for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int e = 0; e < 4; ++e) G[a][e] = 0.f;
          mm_tn<8, 4>(sm.W, WS, sm.dO, LDX, BM, G);
#pragma unroll
          for (int a = 0; a < 8; ++a) {
            const int w = ty + 16 * a;
            if (w < nw) {
#pragma unroll
              for (int e = 0; e < 4; ++e) partv[(size_t)(lo + w) * HD + tx + 16 * e] += G[a][e];
            }
          }
        }
      }
    }
  }
  T *dQg = (T *)p.dq + base;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
    if (i < L) {
#pragma unroll
      for (int e = 0; e < 4; ++e) stf(dQg, (size_t)i * HD + tx + 16 * e, p.scale * dQ[a][e]);
    }
  }
  if (MECH == M_T5) {
    __syncthreads();
    if (tid < p.nb) p.part_small[(bh * p.nT + m) * p.nb + tid] = sm.aux[A_ACC + tid];
  }
}

// ---------------------------------------------------------------------------
// dK, dV (+ key-side partials): one CTA per (key tile, head, batch); the
// register tile is transposed (rows are keys) so key-side sums are lane-local.
// ---------------------------------------------------------------------------
template <int MECH, class T>
__global__ void __launch_bounds__(NT, 1) bwd_kv_kernel(Prm p) {
  p.klen = key_len(p, blockIdx.z);
  extern __shared__ float smem[];
  const Sm sm = carve(smem);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int L = p.L, j0 = n * BN;
  const size_t bh = (size_t)b * p.H + h, base = bh * (size_t)L * HD;
  const T *Qg = (const T *)p.q + base, *Kg = (const T *)p.k + base, *Vg = (const T *)p.v + base,
          *dOg = (const T *)p.dout + base;
  load_rows(Kg, j0, L, sm.K);
  load_rows(Vg, j0, L, sm.V);
  if (MECH == M_TXL) {
    load_vec64((const T *)p.rel1 + (size_t)h * HD, sm.aux + A_U);
    load_vec64((const T *)p.rel2 + (size_t)h * HD, sm.aux + A_V);
  }
  float *part = nullptr;
  if (MECH == M_DEB) {
    part = p.part_col + (bh * p.nT + n) * (size_t)p.nrows * HD;
    for (int x = tid; x < p.nrows * HD; x += NT) part[x] = 0.f;
  }
  float dK[4][4], dV[4][4], cs[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    cs[a] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) dK[a][e] = dV[a][e] = 0.f;
  }
  const int mStart = max(p.causal ? n : 0, p.mem_len / BM);  // memory-placeholder query tiles skipped
  for (int m = mStart; m < p.nT; ++m) {
    const int i0 = m * BM;
    const int dmin = j0 - (i0 + BM - 1), dmax = j0 + BN - 1 - i0;
    __syncthreads();
    load_rows(Qg, i0, L, sm.Q);
    load_rows(dOg, i0, L, sm.dO);
    load_row_stats(p, sm, bh, i0);
    if (MECH == M_T5) load_bias_window(p, sm, h, dmin);
    __syncthreads();
    float S[4][4], dP[4][4], dS[4][4];
    scores<MECH, true, T>(p, sm, h, i0, j0, S);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) dP[a][c] = 0.f;
    mm_nt<4, 4>(sm.V, LDX, sm.dO, LDX, HD, dP);
    if (MECH == M_SHAW && p.shaw_v) value_dp<true, T>(p, sm, h, i0, j0, dmin, dmax, dP);
    probs_and_ds<true>(sm, S, dP, dS);
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sm.P[(ty + 16 * a) * LDX + tx + 16 * c] = S[a][c];
        sm.dS[(ty + 16 * a) * LDX + tx + 16 * c] = dS[a][c];
        if (MECH == M_TXL) cs[a] += dS[a][c];
      }
    if (MECH == M_DEB) zero_W(sm.W, 0);
    __syncthreads();
    mm_nn<4, 4>(sm.P, LDX, sm.dO, LDX, BM, dV);
    mm_nn<4, 4>(sm.dS, LDX, sm.Q, LDX, BM, dK);
    if (MECH == M_DEB) {
      int lo2, nw2;
      col_window(p, dmin, dmax, lo2, nw2);
      scatter_E<MECH, true, true>(p, dS, sm.W, i0, j0, lo2, nw2);
      load_tab((const T *)p.rel1 + (size_t)h * p.nrows * HD, lo2, nw2, sm.T);
      __syncthreads();
      mm_nn<4, 4>(sm.W, WS, sm.T, LDX, nw2, dK);  // dk_j += sum_rho E'[j][rho] Qr[rho]
      float G[8][4];
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) G[a][e] = 0.f;
      mm_tn<8, 4>(sm.W, WS, sm.K, LDX, BN, G);  // G[rho][e] = sum_j E'[j][rho] k_j[e]
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const int w = ty + 16 * a;
        if (w < nw2) {
#pragma unroll
          for (int e = 0; e < 4; ++e) part[(size_t)(lo2 + w) * HD + tx + 16 * e] += p.scale * G[a][e];
        }
      }
    }
  }
  if (MECH == M_TXL) {
    // (q_i + u) . k_j: dk_j gets (sum_i dS_ij) u; du gets sum_j (sum_i dS_ij) k_j
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float c = hsum16(cs[a]);
#pragma unroll
      for (int e = 0; e < 4; ++e) dK[a][e] = fmaf(c, sm.aux[A_U + tx + 16 * e], dK[a][e]);
      if (tx == 0) sm.aux[A_CS + ty + 16 * a] = c;
    }
    __syncthreads();
    if (tid < HD) {
      float acc = 0.f;
      for (int c = 0; c < BN; ++c) acc = fmaf(sm.aux[A_CS + c], sm.K[c * LDX + tid], acc);
      p.part_small[(bh * p.nT + n) * HD + tid] = p.scale * acc;
    }
  }
  T *dKg = (T *)p.dk + base, *dVg = (T *)p.dv + base;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int j = j0 + ty + 16 * a;
    if (j < L) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        stf(dKg, (size_t)j * HD + tx + 16 * e, p.scale * dK[a][e]);
        stf(dVg, (size_t)j * HD + tx + 16 * e, dV[a][e]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Transformer-XL dr: one CTA per (diagonal band of tiles, chunk of the band,
// batch*head).  Every tile of band Delta = m - n reads the same 127 offsets, so
// the CTA keeps sum_i dS_ij q_i and sum dS_ij per offset in registers across
// its tiles and writes one partial (offset-based gradient sharding).
// ---------------------------------------------------------------------------
template <class T>
__global__ void __launch_bounds__(NT, 1) bwd_diag_kernel(Prm p) {
  p.klen = key_len(p, blockIdx.z / p.H);
  extern __shared__ float smem[];
  const Sm sm = carve(smem);
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int band = blockIdx.x, chunk = blockIdx.y, bhi = blockIdx.z;
  const int b = bhi / p.H, h = bhi % p.H;
  const int Delta = p.causal ? band : band - (p.nT - 1);
  const int mlo = max(0, Delta), mhi = min(p.nT - 1, p.nT - 1 + Delta);
  const int m0 = mlo + chunk * p.diag_ch, m1 = min(mhi, m0 + p.diag_ch - 1);
  if (m0 > m1) return;  // no such chunk (never read)
  const int mfirst = max(m0, p.mem_len / BM);  // memory-placeholder query tiles skipped (the partial still written)
  const int L = p.L;
  const size_t bh = (size_t)b * p.H + h, base = bh * (size_t)L * HD;
  const T *Qg = (const T *)p.q + base, *Kg = (const T *)p.k + base, *Vg = (const T *)p.v + base,
          *dOg = (const T *)p.dout + base;
  load_vec64((const T *)p.rel1 + (size_t)h * HD, sm.aux + A_U);
  load_vec64((const T *)p.rel2 + (size_t)h * HD, sm.aux + A_V);
  float G[8][4], g = 0.f;
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) G[a][e] = 0.f;
  for (int m = mfirst; m <= m1; ++m) {
    const int n = m - Delta, i0 = m * BM, j0 = n * BN;
    __syncthreads();
    load_rows(Qg, i0, L, sm.Q);
    load_rows(dOg, i0, L, sm.dO);
    load_rows(Kg, j0, L, sm.K);
    load_rows(Vg, j0, L, sm.V);
    load_row_stats(p, sm, bh, i0);
    __syncthreads();
    float S[4][4], dP[4][4], dS[4][4];
    scores<M_TXL, false, T>(p, sm, h, i0, j0, S);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) dP[a][c] = 0.f;
    mm_nt<4, 4>(sm.dO, LDX, sm.V, LDX, HD, dP);
    probs_and_ds<false>(sm, S, dP, dS);
    __syncthreads();
    zero_W(sm.W, 0);
    __syncthreads();
    // E[r][w], w = r - c + 63 <-> table row (i - j) + off = 64 Delta - 63 + off + w
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = ty + 16 * a, cc = tx + 16 * c;
        sm.W[r * WS + r - cc + (BN - 1)] = dS[a][c];
      }
    __syncthreads();
    mm_tn<8, 4>(sm.W, WS, sm.Q, LDX, BM, G);
    if (tid < TROWS - 1)
      for (int r = 0; r < BM; ++r) g += sm.W[r * WS + tid];
  }
  float *part = p.part_diag + ((bh * p.nbands + band) * (size_t)p.diag_nchunk + chunk) * (size_t)(TROWS * (HD + 1));
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) part[(size_t)(ty + 16 * a) * HD + tx + 16 * e] = G[a][e];
  if (tid < TROWS) part[TROWS * HD + tid] = (tid < TROWS - 1) ? g : 0.f;
}

// ---------------------------------------------------------------------------
// fixed-order reductions of the partials
// ---------------------------------------------------------------------------
__global__ void reduce_t5_kernel(Prm p) {  // dt[h][bk] = sum_{b, m} partial
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= p.H * p.nb) return;
  const int h = x / p.nb, bk = x % p.nb;
  float acc = 0.f;
  for (int b = 0; b < p.B; ++b)
    for (int m = 0; m < p.nT; ++m) acc += p.part_small[(((size_t)b * p.H + h) * p.nT + m) * p.nb + bk];
  p.drel0[x] = acc;
}

// out[h][rho][e] = sum_{b, tile} part[((b*H + h)*nT + tile)][rho][e]
__global__ void reduce_tiles_kernel(Prm p, const float *part, float *out) {
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

// Transformer-XL: dr[h][rho] = scale * (sum_shards G + g v), g -> gtot; du from key-tile partials
template <class T>
__global__ void reduce_txl_dr_kernel(Prm p) {
  const size_t per = (size_t)p.nrows * HD;
  const size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= (size_t)p.H * per) return;
  const int h = (int)(x / per), rho = (int)((x % per) / HD), e = (int)(x % HD);
  float acc = 0.f, gs = 0.f;
  const int rel = rho - p.off;  // = i - j
  // bands whose window [64D - 63, 64D + 63] holds rel
  const int dlo = (rel - 63 >= 0) ? (rel - 63 + 63) / 64 : -((63 - rel) / 64);
  for (int b = 0; b < p.B; ++b) {
    const size_t bh = (size_t)b * p.H + h;
    for (int D = dlo; D <= dlo + 2; ++D) {
      const int w = rel - 64 * D + 63;
      if (w < 0 || w > 126) continue;
      const int band = p.causal ? D : D + (p.nT - 1);
      if (band < 0 || band >= p.nbands) continue;
      const int len = p.nT - (D < 0 ? -D : D);
      const int nch = (len + p.diag_ch - 1) / p.diag_ch;
      for (int c = 0; c < nch; ++c) {
        const float *part = p.part_diag + ((bh * p.nbands + band) * (size_t)p.diag_nchunk + c) * (size_t)(TROWS * (HD + 1));
        acc += part[(size_t)w * HD + e];
        gs += part[TROWS * HD + w];
      }
    }
  }
  const float vv = ldf((const T *)p.rel2 + (size_t)h * HD, e);
  p.drel0[x] = p.scale * (acc + gs * vv);
  if (e == 0) p.gtot[(size_t)h * p.nrows + rho] = gs;
}

// dv[h][e] = scale * sum_rho gtot[h][rho] r[h][rho][e]  (block-wide fixed-order tree)
// du[h][e] = sum_{b, n} part_small[(b*H + h)*nT + n][e]
template <class T>
__global__ void reduce_txl_uv_kernel(Prm p) {
  __shared__ float red[256];
  const int h = blockIdx.x / HD, e = blockIdx.x % HD;
  const T *r = (const T *)p.rel0 + (size_t)h * p.nrows * HD;
  float acc = 0.f;
  for (int rho = threadIdx.x; rho < p.nrows; rho += 256) acc = fmaf(p.gtot[(size_t)h * p.nrows + rho], ldf(r, (size_t)rho * HD + e), acc);
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    p.drel2[(size_t)h * HD + e] = p.scale * red[0];
    float du = 0.f;
    for (int b = 0; b < p.B; ++b)
      for (int n = 0; n < p.nT; ++n) du += p.part_small[(((size_t)b * p.H + h) * p.nT + n) * HD + e];
    p.drel1[(size_t)h * HD + e] = du;
  }
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
template <int MECH, class T>
static cudaError_t run_fwd_t(const Prm &p, cudaStream_t st) {
  auto k = fwd_kernel<MECH, T>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nT - p.mem_len / BM, p.H, p.B);  // no memory-placeholder query tiles
  RP_TRACED("simt_fwd_kernel", st, k<<<grid, NT, SMEM_BYTES, st>>>(p));
  return cudaGetLastError();
}

template <int MECH, class T>
static cudaError_t run_bwd_t(const Prm &p, cudaStream_t st) {
  cudaError_t e;
  const size_t rows = (size_t)p.B * p.H * p.L;
  RP_TRACED("dvec_kernel", st, dvec_kernel<T><<<(unsigned)((8 * rows + 255) / 256), 256, 0, st>>>(p));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  auto kq = bwd_q_kernel<MECH, T>;
  auto kkv = bwd_kv_kernel<MECH, T>;
  if ((e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES)) != cudaSuccess) return e;
  dim3 grid(p.nT, p.H, p.B), gq(p.nT - p.mem_len / BM, p.H, p.B);  // no memory-placeholder query tiles
  RP_TRACED("simt_bwd_kv_kernel", st, kkv<<<grid, NT, SMEM_BYTES, st>>>(p));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  RP_TRACED("simt_bwd_q_kernel", st, kq<<<gq, NT, SMEM_BYTES, st>>>(p));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (MECH == M_TXL) {
    auto kd = bwd_diag_kernel<T>;
    if ((e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES)) != cudaSuccess) return e;
    dim3 gd(p.nbands, p.diag_nchunk, p.B * p.H);
    RP_TRACED("simt_bwd_diag_kernel", st, kd<<<gd, NT, SMEM_BYTES, st>>>(p));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t n = (size_t)p.H * p.nrows * HD;
    RP_TRACED("reduce_txl_dr_kernel", st, reduce_txl_dr_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    RP_TRACED("reduce_txl_uv_kernel", st, reduce_txl_uv_kernel<T><<<p.H * HD, 256, 0, st>>>(p));
    return cudaGetLastError();
  }
  if (MECH == M_T5) {
    RP_TRACED("reduce_t5_kernel", st, reduce_t5_kernel<<<(p.H * p.nb + 255) / 256, 256, 0, st>>>(p));
    return cudaGetLastError();
  }
  const size_t n = (size_t)p.H * p.nrows * HD;
  RP_TRACED("reduce_tiles_kernel", st, reduce_tiles_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p, p.part_row, p.drel0));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (MECH == M_SHAW && p.shaw_v) {
    RP_TRACED("reduce_tiles_kernel", st, reduce_tiles_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p, p.part_val, p.drel1));
    return cudaGetLastError();
  }
  if (MECH == M_DEB) {
    RP_TRACED("reduce_tiles_kernel", st, reduce_tiles_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p, p.part_col, p.drel1));
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace simt

// T5 per-offset bucket and bias vectors (the method's per-call preprocessing):
// bkt[delta + L - 1] = bucket(delta), bias[h][delta + L - 1] = t[h][bucket(delta)];
// ALiBi: bkt = 0 and bias = -m[h] |delta| (one slope per head, rel0 = m[H]).
__global__ void t5_prep_kernel(Prm p) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  const int n = 2 * p.L - 1;
  if (x >= n) return;
  const float *t = (const float *)p.rel0;
  if (p.alibi) {
    const float dist = (float)abs(x - (p.L - 1));
    p.t5_bkt[x] = 0;
    for (int h = 0; h < p.H; ++h) p.t5_bias[(size_t)h * n + x] = -(t[h] * dist);
    return;
  }
  const int bk = t5_bucket(p, x - (p.L - 1));
  p.t5_bkt[x] = bk;
  for (int h = 0; h < p.H; ++h) p.t5_bias[(size_t)h * n + x] = t[h * p.nb + bk];
}

cudaError_t launch_dvec(const Prm &p, bool bf16, cudaStream_t st) {
  const size_t rows = (size_t)p.B * p.H * p.L;
  if (bf16)
    RP_TRACED("dvec_kernel", st, simt::dvec_kernel<__nv_bfloat16><<<(unsigned)((8 * rows + 255) / 256), 256, 0, st>>>(p));
  else
    RP_TRACED("dvec_kernel", st, simt::dvec_kernel<float><<<(unsigned)((8 * rows + 255) / 256), 256, 0, st>>>(p));
  return cudaGetLastError();
}

cudaError_t launch_t5_prep(const Prm &p, cudaStream_t st) {
  const int n = 2 * p.L - 1;
  RP_TRACED("t5_prep_kernel", st, t5_prep_kernel<<<(n + 255) / 256, 256, 0, st>>>(p));
  return cudaGetLastError();
}

cudaError_t simt_fwd(const Prm &p, bool bf16, cudaStream_t st) {
  using bf = __nv_bfloat16;
  switch (p.mech) {
    case M_T5: return bf16 ? simt::run_fwd_t<M_T5, bf>(p, st) : simt::run_fwd_t<M_T5, float>(p, st);
    case M_SHAW: return bf16 ? simt::run_fwd_t<M_SHAW, bf>(p, st) : simt::run_fwd_t<M_SHAW, float>(p, st);
    case M_TXL: return bf16 ? simt::run_fwd_t<M_TXL, bf>(p, st) : simt::run_fwd_t<M_TXL, float>(p, st);
    default: return bf16 ? simt::run_fwd_t<M_DEB, bf>(p, st) : simt::run_fwd_t<M_DEB, float>(p, st);
  }
}

cudaError_t simt_bwd(const Prm &p, bool bf16, cudaStream_t st) {
  using bf = __nv_bfloat16;
  switch (p.mech) {
    case M_T5: return bf16 ? simt::run_bwd_t<M_T5, bf>(p, st) : simt::run_bwd_t<M_T5, float>(p, st);
    case M_SHAW: return bf16 ? simt::run_bwd_t<M_SHAW, bf>(p, st) : simt::run_bwd_t<M_SHAW, float>(p, st);
    case M_TXL: return bf16 ? simt::run_bwd_t<M_TXL, bf>(p, st) : simt::run_bwd_t<M_TXL, float>(p, st);
    default: return bf16 ? simt::run_bwd_t<M_DEB, bf>(p, st) : simt::run_bwd_t<M_DEB, float>(p, st);
  }
}

}  // namespace rp
