// C ABI of the relative-position attention library: argument validation,
// workspace layout and dispatch to the kernels.  Declared in relpos_attn.h.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <vector>

#include <cuda.h>

#include "relpos_attn.h"
#include "common.cuh"
#include "kernels.h"

namespace {

using rp::Prm;

constexpr int kVersion = 10800;  // 1.1.0: seqlens_k; 1.2.0: RELPOS_ALIBI; 1.3.0: shaw_value; 1.4.0: mem_len; 1.5.0: relpos_selftest_wait; 1.6.0: relpos_trace_begin / _end; 1.7.0: relpos_last_cuda_error, RELPOS_ERR_BOUNDS; 1.8.0: Shaw c > 64 on the tensor cores
constexpr int kTile = 64;        // query/key tile of the CUDA-core kernels
constexpr int kMaxL = 1 << 20;

// ---- exact T5 thresholds -------------------------------------------------
// Little-endian base-2^32 big integers, just enough for a^x * b^y comparisons.
typedef std::vector<uint32_t> Big;
static void big_mul(Big &x, uint32_t m) {
  uint64_t carry = 0;
  for (auto &d : x) {
    uint64_t t = (uint64_t)d * m + carry;
    d = (uint32_t)t;
    carry = t >> 32;
  }
  if (carry) x.push_back((uint32_t)carry);
}
static Big big_powmul(uint32_t a, int ea, uint32_t b, int eb) {
  Big x(1, 1u);
  for (int i = 0; i < ea; ++i) big_mul(x, a);
  for (int i = 0; i < eb; ++i) big_mul(x, b);
  while (x.size() > 1 && x.back() == 0) x.pop_back();
  return x;
}
static int big_cmp(const Big &x, const Big &y) {
  if (x.size() != y.size()) return x.size() < y.size() ? -1 : 1;
  for (size_t i = x.size(); i-- > 0;)
    if (x[i] != y[i]) return x[i] < y[i] ? -1 : 1;
  return 0;
}
// Is bucket offset t reached at distance a?  (a/me)^span >= (md/me)^t
static bool t5_reached(uint32_t a, int t, uint32_t me, uint32_t md, int span) {
  return big_cmp(big_powmul(a, span, me, t), big_powmul(me, span, md, t)) >= 0;
}

static int fill_t5(const relpos_params_t *P, Prm &p) {
  const int nb = P->t5_num_buckets, md = P->t5_max_distance;
  const int bidir = P->t5_bidirectional ? 1 : 0;
  if (nb < 2 || nb > 64 || (bidir && nb < 4)) return RELPOS_ERR_INVALID_ARG;
  p.nb = nb;
  p.bidir = bidir;
  p.half = bidir ? nb / 2 : nb;
  p.me = p.half / 2;
  if (p.me < 1 || md <= p.me) return RELPOS_ERR_INVALID_ARG;
  const int span = p.half - p.me;
  p.nthr = span - 1;
  if (p.nthr > 32) return RELPOS_ERR_INVALID_ARG;
  for (int t = 1; t <= p.nthr; ++t) {
    // smallest a in [me, md] with bucket offset >= t (monotone in a)
    uint32_t lo = (uint32_t)p.me, hi = (uint32_t)md;
    while (lo < hi) {
      uint32_t mid = lo + (hi - lo) / 2;
      if (t5_reached(mid, t, (uint32_t)p.me, (uint32_t)md, span))
        hi = mid;
      else
        lo = mid + 1;
    }
    p.thr[t - 1] = (int)lo;
  }
  return RELPOS_OK;
}

// Transformer-XL diagonal bands of tiles and their chunking for the relation-gradient partials
static void set_bands(Prm &p) {
  p.nbands = p.causal ? p.nT : 2 * p.nT - 1;
  long long cap = 4000 / ((long long)p.B * p.H * p.nbands);
  int nch = (int)((p.nT + 7) / 8);
  if (cap < nch) nch = (int)(cap < 1 ? 1 : cap);
  p.diag_ch = (p.nT + nch - 1) / nch;
  p.diag_nchunk = (p.nT + p.diag_ch - 1) / p.diag_ch;
}

static int validate_and_fill(const relpos_params_t *P, Prm &p) {
  if (!P) return RELPOS_ERR_INVALID_ARG;
  memset(&p, 0, sizeof(p));
  if (P->mech < RELPOS_T5 || P->mech > RELPOS_ALIBI) return RELPOS_ERR_INVALID_ARG;
  if (P->dtype != RELPOS_F32 && P->dtype != RELPOS_BF16) return RELPOS_ERR_INVALID_ARG;
  if (P->causal != 0 && P->causal != 1) return RELPOS_ERR_INVALID_ARG;
  if (P->kernel_path < RELPOS_PATH_AUTO || P->kernel_path > RELPOS_PATH_TC) return RELPOS_ERR_INVALID_ARG;
  if (P->d != rp::HD) return RELPOS_ERR_INVALID_ARG;
  if (P->B < 1 || P->H < 1 || P->L < 1 || P->L > kMaxL) return RELPOS_ERR_INVALID_ARG;
  if (P->B > 65535 || P->H > 65535 || P->B * P->H > 65535) return RELPOS_ERR_INVALID_ARG;  // no overflow: both <= 2^16
  if (!isfinite(P->scale)) return RELPOS_ERR_INVALID_ARG;
  if (P->shaw_value != 0 && (P->shaw_value != 1 || P->mech != RELPOS_SHAW)) return RELPOS_ERR_INVALID_ARG;
  if (P->mem_len < 0 || P->mem_len > kMaxL - P->L) return RELPOS_ERR_INVALID_ARG;
  if (P->mem_len > 0 && (P->mech != RELPOS_TXL || P->causal != 1)) return RELPOS_ERR_INVALID_ARG;
  // ALiBi is a per-offset bias like T5's: it runs on the T5 kernels with one slope
  // per head in place of the bucket table
  p.mech = P->mech == RELPOS_ALIBI ? (int)rp::M_T5 : P->mech;
  p.causal = P->causal;
  p.B = (int)P->B;
  p.H = (int)P->H;
  p.L = (int)(P->L + P->mem_len);  // the kernels see the memory and the segment as one causal sequence
  p.mem_len = (int)P->mem_len;
  p.esize = P->dtype == RELPOS_BF16 ? 2 : 4;
  p.scale = P->scale;
  p.seqlens_k = P->seqlens_k;
  p.nT = (p.L + kTile - 1) / kTile;
  switch (P->mech) {
    case RELPOS_T5: {
      int e = fill_t5(P, p);
      if (e) return e;
      p.nrows = p.nb;
      break;
    }
    case RELPOS_ALIBI:
      p.alibi = 1;
      p.nb = 1;
      p.nrows = 1;
      break;
    case RELPOS_SHAW:
      if (P->shaw_clip < 0 || P->shaw_clip > 4096) return RELPOS_ERR_INVALID_ARG;
      p.clip = P->shaw_clip;
      p.nrows = 2 * p.clip + 1;
      p.shaw_v = P->shaw_value;
      break;
    case RELPOS_TXL:
      p.nrows = p.causal ? p.L : 2 * p.L - 1;
      p.off = p.causal ? 0 : p.L - 1;
      break;
    default:
      if (P->deberta_span < 1 || P->deberta_span > 4096) return RELPOS_ERR_INVALID_ARG;
      p.span = P->deberta_span;
      p.nrows = 2 * p.span;
      break;
  }
  if (p.mech == rp::M_TXL) set_bands(p);
  return RELPOS_OK;
}

// Shaw with a clip over 64 (and no value-side table): the relative term s q_i . a[clip(j - i)]
// is the Transformer-XL relation term s q_i . r_{i-j} of the table expanded to one row per
// offset, r_rho = a[clip(-(rho - off)) + c], with u = v = 0; the gradient of a is the
// expanded table's gradient summed over the offsets each row of a stands for.  It runs on
// the relation-block kernels, whose tiles need no per-clip layout.
static bool shaw_wide(const Prm &p) { return p.mech == rp::M_SHAW && !p.shaw_v && p.clip > 64; }

static Prm txl_view(const Prm &p) {
  Prm t = p;
  t.mech = rp::M_TXL;
  t.nrows = p.causal ? p.L : 2 * p.L - 1;
  t.off = p.causal ? 0 : p.L - 1;
  set_bands(t);
  return t;
}

// Which kernel family runs pass `pass` (0 forward, 1 backward) of a call.
static bool use_tc(const relpos_params_t *P, const Prm &p, int pass) {
  if (P->dtype != RELPOS_BF16 || P->kernel_path == RELPOS_PATH_SIMT) return false;
  if (shaw_wide(p)) return true;
  if (pass == 1)
    return p.mech == rp::M_TXL || (p.mech == rp::M_SHAW && rp::tc_bwd_shaw_supported(p)) ||
           (p.mech == rp::M_T5 && rp::tc_bwd_bias_supported(p)) || (p.mech == rp::M_DEB && rp::tc_bwd_deb_supported(p));
  return rp::tc_supported(p);
}

// ---- workspace layout ------------------------------------------------------
struct Layout {
  size_t t5_bias, t5_bkt, dvec, part_row, part_col, part_small, part_diag, gtot, part_val;
  size_t uk, vr, c2pE, p2cE;  // tensor-core products
  size_t part_kv, part_dg, part_uv, qa, da;  // tensor-core backward partials / products
  size_t qkr, kqr, dM, dN, dqc, dkc, dpart, dpad;  // DeBERTa tensor-core backward
  size_t pdtiles;                            // Transformer-XL tensor-core backward: stored P / dS tiles (0: none)
  size_t mq, mo, mlse, mdo, mdq;             // Transformer-XL memory: query-side tensors padded to M + L rows
  size_t xtab, xzero, xdr, xduv;             // wide-clip Shaw: expanded table, zero u / v, its gradients
  size_t total;
};
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// lean: the smallest backward workspace (no stored P / dS tiles)
static Layout layout_of(const Prm &p, int pass, bool tc, bool lean = false);

// wide-clip Shaw: the Transformer-XL layout of the same shape, then the expanded table
// (bf16 [H][rows][d]), the zero u / v vector (bf16 [H][d]) and, for the backward, the
// expanded table's gradient and the u / v gradients (fp32, discarded)
static Layout wide_layout(const Prm &p, int pass, bool lean) {
  const Prm t = txl_view(p);
  Layout l = layout_of(t, pass, true, lean);
  size_t off = l.total;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off += align256(bytes);
    return at;
  };
  const size_t tab = (size_t)p.H * t.nrows * rp::HD;
  l.xtab = take(2 * tab);
  l.xzero = take(2 * (size_t)p.H * rp::HD);
  if (pass == 1) {
    l.xdr = take(sizeof(float) * tab);
    l.xduv = take(sizeof(float) * 2 * (size_t)p.H * rp::HD);
  }
  l.total = off;
  return l;
}

static Layout layout_of(const Prm &p, int pass, bool tc, bool lean) {
  if (tc && shaw_wide(p)) return wide_layout(p, pass, lean);
  Layout l;
  memset(&l, 0, sizeof(l));
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off += align256(bytes);
    return at;
  };
  const size_t BH = (size_t)p.B * p.H;
  if (p.mech == rp::M_T5) {
    l.t5_bias = take(sizeof(float) * (size_t)p.H * (2 * (size_t)p.L - 1));
    l.t5_bkt = take(sizeof(int) * (2 * (size_t)p.L - 1));
  }
  if (pass == 0 && tc) {
    if (p.mech == rp::M_TXL) {
      l.uk = take(sizeof(float) * BH * p.L);
      l.vr = take(sizeof(float) * (size_t)p.H * p.nrows);
    }
    if (p.mech == rp::M_DEB) {
      l.c2pE = take(sizeof(float) * BH * p.L * 2);
      l.p2cE = take(sizeof(float) * BH * p.L * 2);
    }
  }
  if (pass == 1 && tc && p.mech == rp::M_DEB) {  // tensor-core backward (DeBERTa)
    size_t tab = 0, partf = 0, padn = 0;
    rp::tc_bwd_deb_sizes(p, tab, partf, padn);
    l.dvec = take(sizeof(float) * BH * p.L);
    l.qkr = take(sizeof(float) * tab);
    l.kqr = take(sizeof(float) * tab);
    l.dM = take(2 * tab);
    l.dN = take(2 * tab);
    l.dqc = take(sizeof(float) * BH * p.L * rp::HD);
    l.dkc = take(sizeof(float) * BH * p.L * rp::HD);
    l.dpart = take(sizeof(float) * partf);
    l.dpad = take(2 * padn);
  } else if (pass == 1 && tc && p.mech == rp::M_T5) {  // tensor-core backward (T5, ALiBi): per-query-tile partials
    l.dvec = take(sizeof(float) * BH * p.L);
    l.part_small = take(sizeof(float) * BH * (size_t)((p.L + 127) / 128) * p.nb);
  } else if (pass == 1 && tc && p.mech == rp::M_SHAW) {  // tensor-core backward (Shaw)
    l.dvec = take(sizeof(float) * BH * p.L);
    l.qa = take(sizeof(float) * rp::tc_bwd_shaw_qa_floats(p));
    l.part_row = take(sizeof(float) * BH * (size_t)((p.L + 127) / 128) * p.nrows * rp::HD);
    if (p.shaw_v) {  // value side: dO . aV by row and the daV partials
      l.da = take(sizeof(float) * rp::tc_bwd_shaw_qa_floats(p));
      l.part_val = take(sizeof(float) * BH * (size_t)((p.L + 127) / 128) * p.nrows * rp::HD);
    }
  } else if (pass == 1 && tc) {  // tensor-core backward (Transformer-XL)
    size_t kvf = 0;
    const size_t dgf = rp::tc_bwd_part_floats(p, kvf);
    l.dvec = take(sizeof(float) * BH * p.L);
    l.uk = take(sizeof(float) * BH * p.L);
    l.vr = take(sizeof(float) * (size_t)p.H * p.nrows);
    l.part_kv = take(sizeof(float) * kvf);
    l.part_dg = take(sizeof(float) * dgf);
    l.part_uv = take(sizeof(float) * (size_t)p.H * ((p.nrows + 31) / 32) * rp::HD);
    const size_t eb = lean ? 0 : rp::tc_bwd_tile_bytes(p);
    if (eb) l.pdtiles = take(eb);
  } else if (pass == 1) {
    l.dvec = take(sizeof(float) * BH * p.L);
    const size_t tab = (size_t)p.nrows * rp::HD;
    switch (p.mech) {
      case rp::M_T5: l.part_small = take(sizeof(float) * BH * p.nT * p.nb); break;
      case rp::M_SHAW:
        l.part_row = take(sizeof(float) * BH * p.nT * tab);
        if (p.shaw_v) l.part_val = take(sizeof(float) * BH * p.nT * tab);
        break;
      case rp::M_DEB:
        l.part_row = take(sizeof(float) * BH * p.nT * tab);
        l.part_col = take(sizeof(float) * BH * p.nT * tab);
        break;
      default:
        l.part_small = take(sizeof(float) * BH * p.nT * rp::HD);
        l.part_diag = take(sizeof(float) * BH * p.nbands * p.diag_nchunk * 128 * (rp::HD + 1));
        l.gtot = take(sizeof(float) * (size_t)p.H * p.nrows);
        break;
    }
  }
  if (p.mem_len > 0) {  // the query-side tensors at M + L rows, the first M rows placeholders
    const size_t rows = BH * (size_t)p.L, rb = (size_t)p.esize * rp::HD;
    l.mq = take(rows * rb);
    l.mo = take(rows * rb);
    l.mlse = take(rows * sizeof(float));
    if (pass == 1) {
      l.mdo = take(rows * rb);
      l.mdq = take(rows * rb);
    }
  }
  l.total = off;
  return l;
}

static void bind_workspace(Prm &p, const Layout &l, void *ws) {
  char *b = (char *)ws;
  if (p.mech == rp::M_T5) {
    p.t5_bias = (float *)(b + l.t5_bias);
    p.t5_bkt = (int *)(b + l.t5_bkt);
  }
  p.Dvec = (float *)(b + l.dvec);
  p.part_row = (float *)(b + l.part_row);
  p.part_col = (float *)(b + l.part_col);
  p.part_small = (float *)(b + l.part_small);
  p.part_diag = (float *)(b + l.part_diag);
  p.gtot = (float *)(b + l.gtot);
  p.part_val = (float *)(b + l.part_val);
}

static rp::TcWork tc_work(const Layout &l, void *ws) {
  char *b = (char *)ws;
  rp::TcWork w;
  w.uk = (float *)(b + l.uk);
  w.vr = (float *)(b + l.vr);
  w.c2pE = (float *)(b + l.c2pE);
  w.p2cE = (float *)(b + l.p2cE);
  w.part_kv = (float *)(b + l.part_kv);
  w.part_dg = (float *)(b + l.part_dg);
  w.part_uv = (float *)(b + l.part_uv);
  w.qa = (float *)(b + l.qa);
  w.da = (float *)(b + l.da);
  w.qkr = (float *)(b + l.qkr);
  w.kqr = (float *)(b + l.kqr);
  w.dqc = (float *)(b + l.dqc);
  w.dkc = (float *)(b + l.dkc);
  w.dpart = (float *)(b + l.dpart);
  w.dM = b + l.dM;
  w.dN = b + l.dN;
  w.dpad = b + l.dpad;
  w.pdtiles = l.pdtiles ? b + l.pdtiles : nullptr;
  return w;
}

static bool aligned16(const void *x) { return ((uintptr_t)x & 15) == 0; }

static int rel_count(const Prm &p) {
  return p.mech == rp::M_TXL ? 3 : ((p.mech == rp::M_DEB || p.shaw_v) ? 2 : 1);
}

// The calling thread's CUDA context.  The runtime binds the current device's primary
// context lazily, on the first runtime call that needs it, but the tensor-map encoder (a
// driver call, made before any launch) needs a current context already: in a host thread
// that has made no CUDA call yet it would fail.  When no context is current, make the
// current device's primary context current (cudaSetDevice on the device cudaGetDevice
// reports: what the runtime's lazy binding would do); a current context is left alone.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
static int ensure_context() {
  static CtxGetCurrentFn fn = [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return (CtxGetCurrentFn) nullptr;
    }
    return (CtxGetCurrentFn)f;
  }();
  CUcontext ctx = nullptr;
  if (fn && fn(&ctx) == CUDA_SUCCESS && ctx) return RELPOS_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return RELPOS_ERR_CUDA;
  }
  return RELPOS_OK;
}

// CUDA error behind this thread's last RELPOS_ERR_LAUNCH (relpos_last_cuda_error)
static thread_local int t_last_cuda = 0;

static int to_status(cudaError_t e) {
  if (e == cudaSuccess) return RELPOS_OK;
  t_last_cuda = (int)e;
  cudaGetLastError();  // clear a sticky launch-configuration error
  return RELPOS_ERR_LAUNCH;
}

__global__ void fill_f32_kernel(float *x, size_t n, float v) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) x[i] = v;
}

// Transformer-XL memory: a [B,H,L,..] tensor into rows M .. M + L - 1 of each (batch, head)
// plane of a [B,H,M+L,..] one (rows 0 .. M - 1 set to zero), and back.
static cudaError_t pad_rows(void *dst, const void *src, size_t rb, const Prm &p, cudaStream_t st) {
  const int M = p.mem_len, Ls = p.L - M, BH = p.B * p.H;
  cudaError_t e = cudaMemsetAsync(dst, 0, (size_t)BH * p.L * rb, st);
  if (e != cudaSuccess) return e;
  return cudaMemcpy2DAsync((char *)dst + (size_t)M * rb, (size_t)p.L * rb, src, (size_t)Ls * rb, (size_t)Ls * rb, BH,
                           cudaMemcpyDeviceToDevice, st);
}
static cudaError_t unpad_rows(void *dst, const void *src, size_t rb, const Prm &p, cudaStream_t st) {
  const int M = p.mem_len, Ls = p.L - M, BH = p.B * p.H;
  return cudaMemcpy2DAsync(dst, (size_t)Ls * rb, (const char *)src + (size_t)M * rb, (size_t)p.L * rb, (size_t)Ls * rb, BH,
                           cudaMemcpyDeviceToDevice, st);
}

// wide-clip Shaw: the expanded table of the Transformer-XL view t (rel0 of t) from a (rel0
// of p), the zero u / v vector (rel1 = rel2 of t)
static cudaError_t wide_tables(const Prm &p, Prm &t, void *xtab, void *xzero, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(xzero, 0, 2 * (size_t)p.H * rp::HD, st);
  if (e != cudaSuccess) return e;
  if ((e = rp::launch_shaw_expand(p, t, xtab, st)) != cudaSuccess) return e;
  t.rel0 = xtab;
  t.rel1 = xzero;
  t.rel2 = xzero;
  return cudaSuccess;
}

}  // namespace

extern "C" int relpos_attn_workspace_size(const relpos_params_t *params, int pass, size_t *bytes) {
  Prm p;
  if (!bytes || pass < 0 || pass > 2) return RELPOS_ERR_INVALID_ARG;
  int e = validate_and_fill(params, p);
  if (e) return e;
  const int ps = pass == 0 ? 0 : 1;
  *bytes = layout_of(p, ps, use_tc(params, p, ps), pass == 2).total;
  return RELPOS_OK;
}

// seqlens_k is read by the kernels: it must be device (or managed) memory; a host
// pointer is rejected here rather than faulting on the device.
static int check_seqlens(const relpos_params_t *P) {
  if (!P->seqlens_k) return RELPOS_OK;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, P->seqlens_k) != cudaSuccess) {
    cudaGetLastError();  // reset the runtime's last-error state after the failed query
    return RELPOS_ERR_INVALID_ARG;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) ? RELPOS_OK : RELPOS_ERR_INVALID_ARG;
}

extern "C" int relpos_attn_fwd(const relpos_params_t *params, const void *q, const void *k, const void *v,
                               const void *const rel[3], void *o, float *lse, void *workspace,
                               size_t workspace_bytes, int32_t *dev_status, void *stream) {
  cudaGetLastError();  // an error left by an earlier, unrelated call in this thread is not ours
  Prm p;
  int e = validate_and_fill(params, p);
  if (e) return e;
  if (!q || !k || !v || !rel || !o || !lse) return RELPOS_ERR_INVALID_ARG;
  for (int i = 0; i < rel_count(p); ++i)
    if (!rel[i]) return RELPOS_ERR_INVALID_ARG;
  if ((e = check_seqlens(params))) return e;
  const bool tc = use_tc(params, p, 0);
  if (params->kernel_path == RELPOS_PATH_TC && !tc) return RELPOS_ERR_UNSUPPORTED;
  if (tc) {  // TMA needs 16-byte aligned tensors
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(rel[0]) ||
        ((p.mech == rp::M_DEB || p.shaw_v) && !aligned16(rel[1])))
      return RELPOS_ERR_INVALID_ARG;
  }
  const Layout l = layout_of(p, 0, tc);
  if (l.total > 0 && (!workspace || workspace_bytes < l.total || ((uintptr_t)workspace & 255))) return RELPOS_ERR_WORKSPACE;
  if ((e = ensure_context())) return e;  // argument errors are all found above
  bind_workspace(p, l, workspace);
  cudaStream_t st = (cudaStream_t)stream;
  p.q = q;
  p.k = k;
  p.v = v;
  p.rel0 = rel[0];
  p.rel1 = rel_count(p) > 1 ? rel[1] : nullptr;
  p.rel2 = rel_count(p) > 2 ? rel[2] : nullptr;
  p.out = o;
  p.lse = lse;
  p.status = dev_status;
  const size_t rb = (size_t)p.esize * rp::HD;
  char *wb = (char *)workspace;
  if (p.mem_len > 0) {  // the segment's queries at rows M .. M + L - 1 of the padded sequence
    if ((e = to_status(pad_rows(wb + l.mq, q, rb, p, st)))) return e;
    p.q = wb + l.mq;
    p.out = wb + l.mo;
    p.lse = (float *)(wb + l.mlse);
  }
  const bool bf16 = params->dtype == RELPOS_BF16;
  if (tc && shaw_wide(p)) {
    Prm t = txl_view(p);
    if ((e = to_status(wide_tables(p, t, wb + l.xtab, wb + l.xzero, st)))) return e;
    return to_status(rp::tc_fwd(t, tc_work(l, workspace), st));
  }
  if (p.mech == rp::M_T5 && (e = to_status(rp::launch_t5_prep(p, st)))) return e;
  e = tc ? to_status(rp::tc_fwd(p, tc_work(l, workspace), st)) : to_status(rp::simt_fwd(p, bf16, st));
  if (e || p.mem_len == 0) return e;
  if ((e = to_status(unpad_rows(o, wb + l.mo, rb, p, st)))) return e;
  return to_status(unpad_rows(lse, wb + l.mlse, sizeof(float), p, st));
}

extern "C" int relpos_attn_bwd(const relpos_params_t *params, const void *q, const void *k, const void *v,
                               const void *const rel[3], const void *o, const float *lse, const void *dout,
                               void *dq, void *dk, void *dv, float *const drel[3], void *workspace,
                               size_t workspace_bytes, int32_t *dev_status, void *stream) {
  cudaGetLastError();  // an error left by an earlier, unrelated call in this thread is not ours
  Prm p;
  int e = validate_and_fill(params, p);
  if (e) return e;
  if (!q || !k || !v || !rel || !o || !lse || !dout || !dq || !dk || !dv || !drel) return RELPOS_ERR_INVALID_ARG;
  for (int i = 0; i < rel_count(p); ++i)
    if (!rel[i] || !drel[i]) return RELPOS_ERR_INVALID_ARG;
  if ((e = check_seqlens(params))) return e;
  const bool tc = use_tc(params, p, 1);
  if (params->kernel_path == RELPOS_PATH_TC && !tc) return RELPOS_ERR_UNSUPPORTED;
  Layout l = layout_of(p, 1, tc);
  if (workspace_bytes < l.total && l.pdtiles) l = layout_of(p, 1, tc, true);  // too small for the stored tiles: recompute
  if (!workspace || workspace_bytes < l.total || ((uintptr_t)workspace & 255)) return RELPOS_ERR_WORKSPACE;
  bind_workspace(p, l, workspace);
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.dout = dout;
  p.rel0 = rel[0];
  p.rel1 = rel_count(p) > 1 ? rel[1] : nullptr;
  p.rel2 = rel_count(p) > 2 ? rel[2] : nullptr;
  p.lse = (float *)lse;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.drel0 = drel[0];
  p.drel1 = rel_count(p) > 1 ? drel[1] : nullptr;
  p.drel2 = rel_count(p) > 2 ? drel[2] : nullptr;
  p.status = dev_status;
  cudaStream_t st = (cudaStream_t)stream;
  const bool bf16 = params->dtype == RELPOS_BF16;
  if (tc) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(rel[0]))
      return RELPOS_ERR_INVALID_ARG;
    if ((p.mech == rp::M_DEB || p.shaw_v) && !aligned16(rel[1])) return RELPOS_ERR_INVALID_ARG;
  }
  if ((e = ensure_context())) return e;  // argument errors are all found above
  const size_t rb = (size_t)p.esize * rp::HD;
  char *wb = (char *)workspace;
  if (p.mem_len > 0) {  // placeholder rows 0 .. M - 1: zero q, O and dO, LSE = +inf, so P = 0 and dS = 0 there
    if ((e = to_status(pad_rows(wb + l.mq, q, rb, p, st)))) return e;
    if ((e = to_status(pad_rows(wb + l.mo, o, rb, p, st)))) return e;
    if ((e = to_status(pad_rows(wb + l.mdo, dout, rb, p, st)))) return e;
    const size_t n = (size_t)p.B * p.H * p.L;
    RP_TRACED("fill_f32_kernel", st, fill_f32_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>((float *)(wb + l.mlse), n, INFINITY));
    if ((e = to_status(cudaGetLastError()))) return e;
    if ((e = to_status(cudaMemcpy2DAsync(wb + l.mlse + (size_t)p.mem_len * sizeof(float), (size_t)p.L * sizeof(float), lse,
                                         (size_t)(p.L - p.mem_len) * sizeof(float), (size_t)(p.L - p.mem_len) * sizeof(float),
                                         (size_t)p.B * p.H, cudaMemcpyDeviceToDevice, st))))
      return e;
    p.q = wb + l.mq;
    p.o = wb + l.mo;
    p.dout = wb + l.mdo;
    p.lse = (float *)(wb + l.mlse);
    p.dq = wb + l.mdq;
  }
  if (tc && shaw_wide(p)) {
    Prm t = txl_view(p);
    if ((e = to_status(wide_tables(p, t, wb + l.xtab, wb + l.xzero, st)))) return e;
    t.drel0 = (float *)(wb + l.xdr);
    t.drel1 = (float *)(wb + l.xduv);
    t.drel2 = t.drel1 + (size_t)p.H * rp::HD;
    if ((e = to_status(rp::launch_dvec(t, bf16, st)))) return e;
    if ((e = to_status(rp::tc_bwd(t, tc_work(l, workspace), st)))) return e;
    return to_status(rp::launch_shaw_collapse(p, t, t.drel0, p.drel0, st));
  }
  if (tc) {
    if ((e = to_status(rp::launch_dvec(p, bf16, st)))) return e;
    if (p.mech == rp::M_SHAW) {
      e = to_status(rp::tc_bwd_shaw(p, tc_work(l, workspace), st));
    } else if (p.mech == rp::M_DEB) {
      e = to_status(rp::tc_bwd_deb(p, tc_work(l, workspace), st));
    } else if (p.mech == rp::M_T5) {
      if ((e = to_status(rp::launch_t5_prep(p, st)))) return e;
      e = to_status(rp::tc_bwd_bias(p, st));
    } else {
      e = to_status(rp::tc_bwd(p, tc_work(l, workspace), st));
    }
  } else {
    if (p.mech == rp::M_T5 && (e = to_status(rp::launch_t5_prep(p, st)))) return e;
    e = to_status(rp::simt_bwd(p, bf16, st));
  }
  if (e || p.mem_len == 0) return e;
  return to_status(unpad_rows(dq, wb + l.mdq, rb, p, st));
}

extern "C" int relpos_attn_resolved_path(const relpos_params_t *params, int pass) {
  Prm p;
  if (pass != 0 && pass != 1) return RELPOS_ERR_INVALID_ARG;
  int e = validate_and_fill(params, p);
  if (e) return e;
  const bool tc = use_tc(params, p, pass);
  if (params->kernel_path == RELPOS_PATH_TC && !tc) return RELPOS_ERR_UNSUPPORTED;
  return tc ? RELPOS_PATH_TC : RELPOS_PATH_SIMT;
}

extern "C" const char *relpos_strerror(int status) {
  switch (status) {
    case RELPOS_OK: return "ok";
    case RELPOS_ERR_INVALID_ARG: return "invalid argument";
    case RELPOS_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case RELPOS_ERR_UNSUPPORTED: return "unsupported configuration";
    case RELPOS_ERR_LAUNCH: return "kernel launch failed";
    case RELPOS_ERR_TIMEOUT: return "a bounded device wait ran out";
    case RELPOS_ERR_CUDA: return "CUDA runtime error";
    case RELPOS_ERR_BOUNDS: return "an index check of the debug build failed (the access was skipped)";
    default: return "unknown status";
  }
}

extern "C" int relpos_attn_version(void) { return kVersion; }

extern "C" int relpos_last_cuda_error(void) { return t_last_cuda; }
