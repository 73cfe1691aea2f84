// Instantiation and launch of the causal conv1d kernels.
#include "launch.h"

namespace mssm {

template <typename T, int K>
static cudaError_t conv_t(const ConvArgs& a, int items, bool silu, cudaStream_t s) {
  const int64_t rows = int64_t(a.Bt) * a.D;
  dim3 g(unsigned((rows + kConvWarps - 1) / kConvWarps), unsigned(items));
  if (silu)
    causal_conv1d_kernel<T, K, true><<<g, 32 * kConvWarps, 0, s>>>(a);
  else
    causal_conv1d_kernel<T, K, false><<<g, 32 * kConvWarps, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t conv_k(const ConvArgs& a, int items, bool silu, cudaStream_t s) {
  switch (a.K) {
    case 1: return conv_t<T, 1>(a, items, silu, s);
    case 2: return conv_t<T, 2>(a, items, silu, s);
    case 3: return conv_t<T, 3>(a, items, silu, s);
    default: return conv_t<T, 4>(a, items, silu, s);
  }
}

cudaError_t launch_causal_conv1d(const ConvArgs& a, int items, int dtype, bool silu, cudaStream_t s) {
  return dtype == 1 ? conv_k<uint16_t>(a, items, silu, s) : conv_k<float>(a, items, silu, s);
}

template <typename T>
static cudaError_t update_t(const ConvUpdateArgs& a, cudaStream_t s) {
  const int64_t rows = int64_t(a.Bt) * a.D;
  const unsigned g = unsigned((rows + 255) / 256);
  switch (a.K) {
    case 2: causal_conv1d_update_kernel<T, 2><<<g, 256, 0, s>>>(a); break;
    case 3: causal_conv1d_update_kernel<T, 3><<<g, 256, 0, s>>>(a); break;
    default: causal_conv1d_update_kernel<T, 4><<<g, 256, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_causal_conv1d_update(const ConvUpdateArgs& a, int dtype, cudaStream_t s) {
  return dtype == 1 ? update_t<uint16_t>(a, s) : update_t<float>(a, s);
}

}  // namespace mssm
