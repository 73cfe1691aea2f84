// Instantiation and launch of the selective scan kernels (Euler discretisation
// here; the zero-order-hold kernels are instantiated in scan_zoh.cu).
#include "scan_dispatch.cuh"

namespace mssm {

cudaError_t launch_scan_chained(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
  if (a.zoh) return launch_scan_chained_zoh(a, grid, rpt, dtype, has_z, sp, s);
  return ScanDispatch<false>::chained(a, grid, rpt, dtype, has_z, sp, s);
}

cudaError_t launch_scan_fused(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
  if (a.zoh) return launch_scan_fused_zoh(a, grid, rpt, dtype, has_z, sp, s);
  return ScanDispatch<false>::fused(a, grid, rpt, dtype, has_z, sp, s);
}

cudaError_t launch_scan_split(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
  if (a.zoh) return launch_scan_split_zoh(a, grid, rpt, dtype, has_z, sp, s);
  return ScanDispatch<false>::split(a, grid, rpt, dtype, has_z, sp, s);
}

cudaError_t launch_scan_chunk_state(const ScanArgs& a, int rows, int rpt, int dtype, bool sp, cudaStream_t s) {
  if (a.zoh) return launch_scan_chunk_state_zoh(a, rows, rpt, dtype, sp, s);
  return ScanDispatch<false>::chunk_state(a, rows, rpt, dtype, sp, s);
}

cudaError_t launch_scan_out(const ScanArgs& a, int rows, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
  if (a.zoh) return launch_scan_out_zoh(a, rows, rpt, dtype, has_z, sp, s);
  return ScanDispatch<false>::out(a, rows, rpt, dtype, has_z, sp, s);
}

}  // namespace mssm
