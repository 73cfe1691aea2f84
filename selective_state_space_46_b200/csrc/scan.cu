// Instantiation and launch of the selective scan kernels.
#include "launch.h"

namespace mssm {

template <typename T, bool SP>
static cudaError_t chunk_state_t(const ScanArgs& a, cudaStream_t s) {
  dim3 g(a.Bt * a.tiles_per_batch, a.nseg - 1);
  scan_chunk_state_kernel<T, SP><<<g, kRows, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename T, bool HAS_Z, bool SP>
static cudaError_t out_t(const ScanArgs& a, cudaStream_t s) {
  dim3 g(a.Bt * a.tiles_per_batch, a.nseg);
  scan_out_kernel<T, HAS_Z, SP><<<g, kRows, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_scan_chunk_state(const ScanArgs& a, int dtype, bool softplus, cudaStream_t s) {
  if (dtype == 1) return softplus ? chunk_state_t<uint16_t, true>(a, s) : chunk_state_t<uint16_t, false>(a, s);
  return softplus ? chunk_state_t<float, true>(a, s) : chunk_state_t<float, false>(a, s);
}

cudaError_t launch_scan_out(const ScanArgs& a, int dtype, bool has_z, bool softplus, cudaStream_t s) {
  if (dtype == 1) {
    if (has_z) return softplus ? out_t<uint16_t, true, true>(a, s) : out_t<uint16_t, true, false>(a, s);
    return softplus ? out_t<uint16_t, false, true>(a, s) : out_t<uint16_t, false, false>(a, s);
  }
  if (has_z) return softplus ? out_t<float, true, true>(a, s) : out_t<float, true, false>(a, s);
  return softplus ? out_t<float, false, true>(a, s) : out_t<float, false, false>(a, s);
}

}  // namespace mssm
