// Instantiation and launch of the decode state-update kernels; the device error word.
#include "launch.h"

namespace mssm {

__device__ unsigned int g_device_error = 0u;

// Address of each device's copy of the error word, looked up once per device
// (the caller serialises launches, so the cache needs no lock of its own).
static void* g_error_word_cache[64] = {};
// per device: SM count once the streaming kernels' shared-memory opt-in is set (0: not yet)
static int g_stream_sms[64] = {};

static int g_address_generation = 0;

void forget_device_addresses() {
  for (void*& p : g_error_word_cache) p = nullptr;
  for (int& v : g_stream_sms) v = 0;  // a reset also drops the kernels' attributes
  ++g_address_generation;
}

int device_address_generation() { return g_address_generation; }

cudaError_t device_error_word(unsigned int** out) {
  void** cache = g_error_word_cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!cache[dev]) {
    e = cudaGetSymbolAddress(&cache[dev], g_device_error);
    if (e != cudaSuccess) return e;
  }
  *out = static_cast<unsigned int*>(cache[dev]);
  return cudaSuccess;
}

// SM count and the streaming kernels' shared-memory opt-in, once per device
static cudaError_t stream_setup(int* sms) {
  int* sm_cache = g_stream_sms;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!sm_cache[dev]) {
    int v = 0;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int b16 = kWsWarps * kWsBufs * int(StreamSlot<uint16_t>::kBytes);
    const int b32 = kWsWarps * kWsBufs * int(StreamSlot<float>::kBytes);
    if ((e = cudaFuncSetAttribute(state_update_stream_kernel<uint16_t, true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, b16)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(state_update_stream_kernel<uint16_t, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, b16)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(state_update_stream_kernel<float, true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, b32)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(state_update_stream_kernel<float, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, b32)) != cudaSuccess)
      return e;
    sm_cache[dev] = v;
  }
  *sms = sm_cache[dev];
  return cudaSuccess;
}

// Batch groups of the streaming kernel: as many CTAs per channel block as fill the
// resident slots, but no more groups than batches.
int stream_groups(int Bt, int D, int sms) {
  const int nblk = (D + kWsRows - 1) / kWsRows;
  int groups = (sms * kStreamCtasPerSm * kWsWarps) / nblk;
  if (groups < 1) groups = 1;
  if (groups > Bt) groups = Bt;
  // same number of batches per CTA with as few groups as that needs
  const int per = (Bt + groups - 1) / groups;
  return (Bt + per - 1) / per;
}

template <typename T, bool HAS_Z>
static cudaError_t launch_decode_t(DecodeArgs a, DecodePath path, cudaStream_t s) {
  cudaError_t e = device_error_word(&a.err);
  if (e != cudaSuccess) return e;
  const int64_t rows = int64_t(a.Bt) * a.D;
  const int64_t blocks = (rows + kDecodeThreads - 1) / kDecodeThreads;
  if (path == DecodePath::kStream) {
    int sms = 0;
    if ((e = stream_setup(&sms)) != cudaSuccess) return e;
    a.groups = stream_groups(a.Bt, a.D, sms);
    const int64_t warps = int64_t((a.D + kWsRows - 1) / kWsRows) * a.groups;
    state_update_stream_kernel<T, HAS_Z><<<unsigned((warps + kWsWarps - 1) / kWsWarps), kWsWarps * 32,
                                           kWsWarps * kWsBufs * StreamSlot<T>::kBytes, s>>>(a);
  } else if (path == DecodePath::kBulkTile) {
    state_update_bulk_kernel<T, HAS_Z><<<unsigned(blocks), kDecodeThreads, 0, s>>>(a);
  } else {
    state_update_kernel<T, HAS_Z><<<unsigned(blocks), kDecodeThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_state_update(const DecodeArgs& a, int dtype, bool has_z, DecodePath path, cudaStream_t s) {
  if (dtype == 1) return has_z ? launch_decode_t<uint16_t, true>(a, path, s) : launch_decode_t<uint16_t, false>(a, path, s);
  return has_z ? launch_decode_t<float, true>(a, path, s) : launch_decode_t<float, false>(a, path, s);
}

cudaError_t read_device_error(unsigned int* value, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess || !clear || *value == 0u) return e;
  const unsigned int zero = 0u;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace mssm
