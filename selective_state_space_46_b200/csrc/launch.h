// Internal host-side launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>

#include "decode.cuh"
#include "scan.cuh"

namespace mssm {

// dtype: 0 = fp32 storage, 1 = bf16 storage.  Return the launch error, if any.
cudaError_t launch_scan_chunk_state(const ScanArgs& a, int dtype, bool softplus, cudaStream_t s);
cudaError_t launch_scan_out(const ScanArgs& a, int dtype, bool has_z, bool softplus, cudaStream_t s);
cudaError_t launch_state_update(const DecodeArgs& a, int dtype, bool has_z, cudaStream_t s);

}  // namespace mssm
