// Host-side dispatch of the scan kernels over their template parameters, for
// one discretisation (ZOH) per translation unit: scan.cu instantiates the
// Euler kernels and scan_zoh.cu the zero-order-hold ones, so the two compile
// in parallel.
//
// Row tiles: `rows` channels per tile, `rpt` rows per thread, so rows / rpt
// threads per CTA.  Supported: (32, 1), (64, 1), (64, 2), (128, 2); two rows per
// thread are built for bf16 I/O only (fp32 I/O is the small-problem path).
#pragma once

#include "launch.h"

namespace mssm {

// Lets `kernel` use `bytes` of dynamic shared memory (above the 48 KB default), once per
// device, and again after mssm_shutdown (a device reset drops it).  set_gen: the caller's
// own per-device record for this kernel (the address generation it was set in, + 1).
template <typename K>
cudaError_t opt_in_smem(K kernel, int bytes, int (&set_gen)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int gen = device_address_generation() + 1;
  if (set_gen[dev] != gen) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    set_gen[dev] = gen;
  }
  return cudaSuccess;
}

template <bool ZOH>
struct ScanDispatch {
  template <typename T, int NT, int R, bool SP>
  static cudaError_t chunk_state_t(const ScanArgs& a, cudaStream_t s) {
    dim3 g(a.Bt * a.tiles_per_batch, a.nseg - 1);
    // packed sequences take the forward-sweep summaries (their chunks may start inside a block)
    if constexpr (ZOH) {
      scan_chunk_state_kernel<T, NT, R, SP, true, true><<<g, NT, 0, s>>>(a);
    } else {
      if (a.cu_seqlens)
        scan_chunk_state_kernel<T, NT, R, SP, false, true><<<g, NT, 0, s>>>(a);
      else
        scan_chunk_state_kernel<T, NT, R, SP, false, false><<<g, NT, 0, s>>>(a);
    }
    return cudaGetLastError();
  }
  template <typename T, int NT, int R, bool HAS_Z, bool SP>
  static cudaError_t out_t(const ScanArgs& a, cudaStream_t s) {
    dim3 g(a.Bt * a.tiles_per_batch, a.nseg);
    if (a.nseg > 1 && a.cu_seqlens) {
      // Packed sequences, right after the chunk-summary kernel: a programmatic dependent
      // launch, so that the CTAs' prologue overlaps that kernel's long carry folds (they
      // read the carries after griddep_wait).  Measured on B200: 387 -> 364 us for 32
      // packed sequences; on plain batches whose forward grid fits one wave it cost 6%
      // (the early CTAs are placed unevenly over the SMs), so they launch normally.
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = g;
      cfg.blockDim = dim3(NT);
      cfg.dynamicSmemBytes = 0;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, scan_out_kernel<T, NT, R, HAS_Z, SP, ZOH>, a);
    }
    scan_out_kernel<T, NT, R, HAS_Z, SP, ZOH><<<g, NT, 0, s>>>(a);
    return cudaGetLastError();
  }
  template <typename T, int R, bool HAS_Z, bool SP>
  static cudaError_t chained_t(const ScanArgs& a, int grid, cudaStream_t s) {
    scan_out_chained_kernel<T, R, HAS_Z, SP, ZOH><<<grid, 32, 0, s>>>(a);
    return cudaGetLastError();
  }
  template <typename T, int R, bool HAS_Z, bool SP>
  static cudaError_t fused_t(const ScanArgs& a, int grid, cudaStream_t s) {
    scan_fused_kernel<T, R, HAS_Z, SP, ZOH><<<grid, 32, 0, s>>>(a);
    return cudaGetLastError();
  }

  template <typename T, int R, bool HAS_Z, bool SP>
  static cudaError_t split_t(const ScanArgs& a, int grid, cudaStream_t s) {
    constexpr int bytes = split_smem_bytes<R>();
    static int set_gen[64] = {};  // one record per kernel instantiation
    cudaError_t e = opt_in_smem(scan_split_kernel<T, R, HAS_Z, SP, ZOH>, bytes, set_gen);
    if (e != cudaSuccess) return e;
    scan_split_kernel<T, R, HAS_Z, SP, ZOH><<<grid, 32 * kSplitWarps, bytes, s>>>(a);
    return cudaGetLastError();
  }

  // ---- runtime -> template parameters
  template <typename T, int R>
  static cudaError_t split_r(const ScanArgs& a, int grid, bool has_z, bool sp, cudaStream_t s) {
    if (has_z) return sp ? split_t<T, R, true, true>(a, grid, s) : split_t<T, R, true, false>(a, grid, s);
    return sp ? split_t<T, R, false, true>(a, grid, s) : split_t<T, R, false, false>(a, grid, s);
  }
  template <typename T, int R>
  static cudaError_t fused_r(const ScanArgs& a, int grid, bool has_z, bool sp, cudaStream_t s) {
    if (has_z) return sp ? fused_t<T, R, true, true>(a, grid, s) : fused_t<T, R, true, false>(a, grid, s);
    return sp ? fused_t<T, R, false, true>(a, grid, s) : fused_t<T, R, false, false>(a, grid, s);
  }
  template <typename T, int R>
  static cudaError_t chained_r(const ScanArgs& a, int grid, bool has_z, bool sp, cudaStream_t s) {
    if (has_z) return sp ? chained_t<T, R, true, true>(a, grid, s) : chained_t<T, R, true, false>(a, grid, s);
    return sp ? chained_t<T, R, false, true>(a, grid, s) : chained_t<T, R, false, false>(a, grid, s);
  }
  template <typename T, int NT, int R>
  static cudaError_t chunk_state_r(const ScanArgs& a, bool sp, cudaStream_t s) {
    return sp ? chunk_state_t<T, NT, R, true>(a, s) : chunk_state_t<T, NT, R, false>(a, s);
  }
  template <typename T, int NT, int R>
  static cudaError_t out_r(const ScanArgs& a, bool has_z, bool sp, cudaStream_t s) {
    if (has_z) return sp ? out_t<T, NT, R, true, true>(a, s) : out_t<T, NT, R, true, false>(a, s);
    return sp ? out_t<T, NT, R, false, true>(a, s) : out_t<T, NT, R, false, false>(a, s);
  }

  static cudaError_t fused(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
    if (dtype == 1)
      return rpt == 2 ? fused_r<uint16_t, 2>(a, grid, has_z, sp, s) : fused_r<uint16_t, 1>(a, grid, has_z, sp, s);
    if (rpt != 1) return cudaErrorInvalidConfiguration;
    return fused_r<float, 1>(a, grid, has_z, sp, s);
  }
  static cudaError_t split(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
    if (dtype == 1)
      return rpt == 2 ? split_r<uint16_t, 2>(a, grid, has_z, sp, s) : split_r<uint16_t, 1>(a, grid, has_z, sp, s);
    if (rpt != 1) return cudaErrorInvalidConfiguration;
    return split_r<float, 1>(a, grid, has_z, sp, s);
  }
  static cudaError_t chained(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
    if (dtype == 1)
      return rpt == 2 ? chained_r<uint16_t, 2>(a, grid, has_z, sp, s) : chained_r<uint16_t, 1>(a, grid, has_z, sp, s);
    if (rpt != 1) return cudaErrorInvalidConfiguration;
    return chained_r<float, 1>(a, grid, has_z, sp, s);
  }
  static cudaError_t chunk_state(const ScanArgs& a, int rows, int rpt, int dtype, bool sp, cudaStream_t s) {
    if (dtype == 1) {
      if (rpt == 1) return rows == 32 ? chunk_state_r<uint16_t, 32, 1>(a, sp, s) : chunk_state_r<uint16_t, 64, 1>(a, sp, s);
      return rows == 64 ? chunk_state_r<uint16_t, 32, 2>(a, sp, s) : chunk_state_r<uint16_t, 64, 2>(a, sp, s);
    }
    if (rpt != 1) return cudaErrorInvalidConfiguration;
    return rows == 32 ? chunk_state_r<float, 32, 1>(a, sp, s) : chunk_state_r<float, 64, 1>(a, sp, s);
  }
  static cudaError_t out(const ScanArgs& a, int rows, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s) {
    if (dtype == 1) {
      if (rpt == 1) return rows == 32 ? out_r<uint16_t, 32, 1>(a, has_z, sp, s) : out_r<uint16_t, 64, 1>(a, has_z, sp, s);
      return rows == 64 ? out_r<uint16_t, 32, 2>(a, has_z, sp, s) : out_r<uint16_t, 64, 2>(a, has_z, sp, s);
    }
    if (rpt != 1) return cudaErrorInvalidConfiguration;
    return rows == 32 ? out_r<float, 32, 1>(a, has_z, sp, s) : out_r<float, 64, 1>(a, has_z, sp, s);
  }
};

// the zero-order-hold launches, defined in scan_zoh.cu
cudaError_t launch_scan_chunk_state_zoh(const ScanArgs& a, int rows, int rpt, int dtype, bool sp, cudaStream_t s);
cudaError_t launch_scan_out_zoh(const ScanArgs& a, int rows, int rpt, int dtype, bool has_z, bool sp, cudaStream_t s);
cudaError_t launch_scan_chained_zoh(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp,
                                    cudaStream_t s);
cudaError_t launch_scan_fused_zoh(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp,
                                  cudaStream_t s);
cudaError_t launch_scan_split_zoh(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool sp,
                                  cudaStream_t s);

}  // namespace mssm
