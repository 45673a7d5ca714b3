// Internal launchers behind the C ABI (not exported).
#pragma once
#include <cuda_runtime.h>
#include "common.cuh"

namespace rp {
// Every kernel launch of the library goes through RP_TRACED: an NVTX range around the
// launch and, when the calling thread registered a trace (relpos_trace_begin), CUDA
// events on the launch stream before and after the kernel.
void trace_pre(const char *name, cudaStream_t st);
void trace_post(cudaStream_t st);
#define RP_TRACED(name, st, ...)   \
  do {                             \
    ::rp::trace_pre(name, st);     \
    __VA_ARGS__;                   \
    ::rp::trace_post(st);          \
  } while (0)

cudaError_t launch_t5_prep(const Prm &p, cudaStream_t st);
cudaError_t simt_fwd(const Prm &p, bool bf16, cudaStream_t st);
cudaError_t simt_bwd(const Prm &p, bool bf16, cudaStream_t st);

// tensor-core (bf16) path
struct TcWork {
  float *uk, *vr, *c2pE, *p2cE;  // per-call products (Transformer-XL, DeBERTa)
  float *part_kv, *part_dg;      // backward partials (Transformer-XL)
  float *part_uv;                // [H][ceil(rows / 32)][64] dv partials per 32-offset tile
  float *qa;                     // Shaw backward: [B,H,L][132] per-row products q_i . a_rho
  float *da;                     // Shaw value side: [B,H,L][132] per-row products dO_i . aV_rho
  void *pdtiles;                 // Transformer-XL backward: the query-tile kernel's P / dS tiles (or null)
  // DeBERTa backward: relation products QKr, KQr and dS K, dS^T Q (fp32), the
  // offset-ordered dS copies M, N (bf16, [B,H,L][2k]) and the table-gradient partials
  float *qkr, *kqr, *dqc, *dkc, *dpart;
  void *dM, *dN, *dpad;  // dpad: Kr, Qr padded with zero rows to a multiple of 64 (bf16)
};
bool tc_supported(const Prm &p);
cudaError_t tc_prep(const Prm &p, const TcWork &w, cudaStream_t st);
cudaError_t tc_fwd(const Prm &p, const TcWork &w, cudaStream_t st);
cudaError_t tc_bwd(const Prm &p, const TcWork &w, cudaStream_t st);
size_t tc_bwd_part_floats(const Prm &p, size_t &kv_floats);
size_t tc_bwd_tile_bytes(const Prm &p);
bool tc_bwd_shaw_supported(const Prm &p);
size_t tc_bwd_shaw_qa_floats(const Prm &p);
cudaError_t tc_bwd_shaw(const Prm &p, const TcWork &w, cudaStream_t st);
bool tc_bwd_deb_supported(const Prm &p);
void tc_bwd_deb_sizes(const Prm &p, size_t &table_elems, size_t &part_floats, size_t &pad_elems);
cudaError_t tc_bwd_deb(const Prm &p, const TcWork &w, cudaStream_t st);
bool tc_bwd_bias_supported(const Prm &p);
cudaError_t tc_bwd_bias(const Prm &p, cudaStream_t st);
cudaError_t launch_dvec(const Prm &p, bool bf16, cudaStream_t st);
// wide-clip Shaw on the Transformer-XL kernels (view t): the table expanded to one row per
// offset, and its gradient summed back into the 2c + 1 rows
cudaError_t launch_shaw_expand(const Prm &p, const Prm &t, void *xtab, cudaStream_t st);
cudaError_t launch_shaw_collapse(const Prm &p, const Prm &t, const float *xdr, float *da, cudaStream_t st);
}  // namespace rp
