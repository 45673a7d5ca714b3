// Internal launchers behind the C ABI (not exported).
#pragma once
#include <cuda_runtime.h>
#include "common.cuh"

namespace rp {
cudaError_t launch_t5_prep(const Prm &p, cudaStream_t st);
cudaError_t simt_fwd(const Prm &p, bool bf16, cudaStream_t st);
cudaError_t simt_bwd(const Prm &p, bool bf16, cudaStream_t st);
}  // namespace rp
