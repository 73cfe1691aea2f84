// Instantiation and launch of the backward scan kernels: pass A (the chunk summaries both
// ways and their folds) and pass B (the per-chunk recompute and backward sweep).
#include "launch.h"

namespace mssm {

template <typename T, bool HAS_Z, int CHUNK>
static cudaError_t bwd_t(const BwdArgs& a, cudaStream_t s) {
  const unsigned tiles = unsigned(a.Bt * a.tiles_per_batch);
  if (a.nseg > 1) {
    scan_bwd_summary_kernel<T, HAS_Z, CHUNK><<<dim3(tiles, a.nseg), kBwdRows, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  scan_bwd_kernel<T, HAS_Z, CHUNK><<<dim3(tiles, a.nseg), kBwdRows, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename T, bool HAS_Z>
static cudaError_t bwd_c(const BwdArgs& a, cudaStream_t s) {
  if (a.chunk == kBwdChunkShort) return bwd_t<T, HAS_Z, kBwdChunkShort>(a, s);
  if (a.chunk == kBwdChunk) return bwd_t<T, HAS_Z, kBwdChunk>(a, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_scan_bwd(const BwdArgs& a, int dtype, bool has_z, cudaStream_t s) {
  if (dtype == 1) return has_z ? bwd_c<uint16_t, true>(a, s) : bwd_c<uint16_t, false>(a, s);
  return has_z ? bwd_c<float, true>(a, s) : bwd_c<float, false>(a, s);
}

}  // namespace mssm
