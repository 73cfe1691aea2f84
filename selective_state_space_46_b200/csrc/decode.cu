// Instantiation and launch of the decode state-update kernel.
#include "launch.h"

namespace mssm {

template <typename T, bool HAS_Z>
static cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t s) {
  const int64_t threads = int64_t(a.Bt) * a.D * 4;
  const int64_t blocks = (threads + kDecodeThreads - 1) / kDecodeThreads;
  state_update_kernel<T, HAS_Z><<<unsigned(blocks), kDecodeThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_state_update(const DecodeArgs& a, int dtype, bool has_z, cudaStream_t s) {
  if (dtype == 1) return has_z ? launch_decode_t<uint16_t, true>(a, s) : launch_decode_t<uint16_t, false>(a, s);
  return has_z ? launch_decode_t<float, true>(a, s) : launch_decode_t<float, false>(a, s);
}

}  // namespace mssm
