// Internal launchers behind the C ABI (not exported).
#pragma once
#include <cuda_runtime.h>
#include "common.cuh"

namespace rp {
cudaError_t launch_t5_prep(const Prm &p, cudaStream_t st);
cudaError_t simt_fwd(const Prm &p, bool bf16, cudaStream_t st);
cudaError_t simt_bwd(const Prm &p, bool bf16, cudaStream_t st);

// tensor-core (bf16) path
struct TcWork {
  float *uk, *vr, *c2pE, *p2cE;  // per-call products (Transformer-XL, DeBERTa)
  float *part_kv, *part_dg;      // backward partials (Transformer-XL)
  float *part_uv;                // [H][ceil(rows / 32)][64] dv partials per 32-offset tile
  float *qa;                     // Shaw backward: [B,H,L][132] per-row products q_i . a_rho
};
bool tc_supported(const Prm &p);
cudaError_t tc_prep(const Prm &p, const TcWork &w, cudaStream_t st);
cudaError_t tc_fwd(const Prm &p, const TcWork &w, cudaStream_t st);
cudaError_t tc_bwd(const Prm &p, const TcWork &w, cudaStream_t st);
size_t tc_bwd_part_floats(const Prm &p, size_t &kv_floats);
bool tc_bwd_shaw_supported(const Prm &p);
size_t tc_bwd_shaw_qa_floats(const Prm &p);
cudaError_t tc_bwd_shaw(const Prm &p, const TcWork &w, cudaStream_t st);
bool tc_bwd_bias_supported(const Prm &p);
cudaError_t tc_bwd_bias(const Prm &p, cudaStream_t st);
cudaError_t launch_dvec(const Prm &p, bool bf16, cudaStream_t st);
}  // namespace rp
