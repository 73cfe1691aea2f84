// Instantiation of the zero-order-hold selective scan kernels.
#include "scan_dispatch.cuh"

namespace mssm {

cudaError_t launch_scan_chained_zoh(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp,
                                    cudaStream_t s) {
  return ScanDispatch<true>::chained(a, grid, rpt, dtype, has_z, sp, s);
}

cudaError_t launch_scan_fused_zoh(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp,
                                  cudaStream_t s) {
  return ScanDispatch<true>::fused(a, grid, rpt, dtype, has_z, sp, s);
}

cudaError_t launch_scan_split_zoh(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp,
                                  cudaStream_t s) {
  return ScanDispatch<true>::split(a, grid, rpt, dtype, has_z, sp, s);
}

cudaError_t launch_scan_chunk_state_zoh(const ScanArgs& a, int rows, int rpt, int dtype, bool sp, cudaStream_t s) {
  return ScanDispatch<true>::chunk_state(a, rows, rpt, dtype, sp, s);
}

cudaError_t launch_scan_out_zoh(const ScanArgs& a, int rows, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
  return ScanDispatch<true>::out(a, rows, rpt, dtype, has_z, sp, s);
}

}  // namespace mssm
