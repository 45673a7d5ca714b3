// Shaw relative positions with a wide clip, on the Transformer-XL relation-block kernels.
//
// Shaw, Uszkoreit and Vaswani's key-side term q_i . a[clip(j - i, -c, c) + c] (the Hugging
// Face page of "Fast and Exact Relative-Position Attention via Structure-Aware Kernels"
// lists it with Transformer-XL among the mechanisms of one offset-indexed family) is the
// Transformer-XL relation term q_i . r_{i-j} of the table with one row per offset:
//   r[rho] = a[clip(off - rho, -c, c) + c],   rho = i - j + off
// (off = 0 causal, L - 1 otherwise), with the content and position biases u = v = 0.  The
// gradient of row a[c'] is the sum of dr over the offsets that row stands for: one offset
// for an interior row, every offset at or beyond the clip for the two end rows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace rp {
namespace {

// r[h][rho] = a[h][clip(off - rho) + c]: 16 bytes (8 bf16) per thread
__global__ void shaw_expand_kernel(const uint4 *a, uint4 *r, int H, int rows, int off, int clip) {
  const size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t n = (size_t)H * rows * (HD / 8);
  if (x >= n) return;
  const int c8 = (int)(x % (HD / 8));
  const size_t hr = x / (HD / 8);
  const int rho = (int)(hr % rows), h = (int)(hr / rows);
  int d = off - rho;  // j - i
  d = d < -clip ? -clip : (d > clip ? clip : d);
  r[x] = a[((size_t)h * (2 * clip + 1) + d + clip) * (HD / 8) + c8];
}

// da[h][c'][e] = sum of dr[h][rho][e] over the offsets rho of row c'.  One CTA per (h, c');
// four groups of 64 threads take every fourth offset of the range, then the four partial
// sums are added in group order (a fixed order: the result does not depend on timing).
__global__ void __launch_bounds__(256) shaw_collapse_kernel(const float *dr, float *da, int rows, int off, int clip) {
  __shared__ float part[4][HD];
  const int nr = 2 * clip + 1;
  const int h = (int)blockIdx.x / nr, cp = (int)blockIdx.x % nr;
  const int e = threadIdx.x & (HD - 1), grp = threadIdx.x >> 6;
  // offsets rho = off - delta with delta = cp - c, every delta <= -c (cp = 0) or >= c (cp = 2c)
  int lo, hi;
  if (cp == 0) {
    lo = off + clip;
    hi = rows - 1;
  } else if (cp == 2 * clip) {
    lo = 0;
    hi = off - clip;
  } else {
    lo = hi = off - (cp - clip);
  }
  lo = lo < 0 ? 0 : lo;
  hi = hi > rows - 1 ? rows - 1 : hi;
  float s = 0.f;
  for (int rho = lo + grp; rho <= hi; rho += 4) s += dr[((size_t)h * rows + rho) * HD + e];
  part[grp][e] = s;
  __syncthreads();
  if (grp == 0) da[((size_t)h * nr + cp) * HD + e] = ((part[0][e] + part[1][e]) + part[2][e]) + part[3][e];
}

}  // namespace

cudaError_t launch_shaw_expand(const Prm &p, const Prm &t, void *xtab, cudaStream_t st) {
  const size_t n = (size_t)p.H * t.nrows * (HD / 8);
  RP_TRACED("shaw_expand_kernel", st,
            shaw_expand_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>((const uint4 *)p.rel0, (uint4 *)xtab, p.H,
                                                                             t.nrows, t.off, p.clip));
  return cudaGetLastError();
}

cudaError_t launch_shaw_collapse(const Prm &p, const Prm &t, const float *xdr, float *da, cudaStream_t st) {
  RP_TRACED("shaw_collapse_kernel", st,
            shaw_collapse_kernel<<<(unsigned)(p.H * (2 * p.clip + 1)), 256, 0, st>>>(xdr, da, t.nrows, t.off, p.clip));
  return cudaGetLastError();
}

}  // namespace rp
