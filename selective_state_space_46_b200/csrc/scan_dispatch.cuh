// Host-side dispatch of the scan kernels over their template parameters, for
// one discretisation (ZOH) per translation unit: scan.cu instantiates the
// Euler kernels and scan_zoh.cu the zero-order-hold ones, so the two compile
// in parallel.
#pragma once

#include "launch.h"

namespace mssm {

template <bool ZOH>
struct ScanDispatch {
  template <typename T, int ROWS, bool SP>
  static cudaError_t chunk_state_t(const ScanArgs& a, cudaStream_t s) {
    dim3 g(a.Bt * a.tiles_per_batch, a.nseg - 1);
    // packed sequences take the forward-sweep summaries (their chunks may start inside a block)
    if constexpr (ZOH) {
      scan_chunk_state_kernel<T, ROWS, SP, true, true><<<g, ROWS, 0, s>>>(a);
    } else {
      if (a.cu_seqlens)
        scan_chunk_state_kernel<T, ROWS, SP, false, true><<<g, ROWS, 0, s>>>(a);
      else
        scan_chunk_state_kernel<T, ROWS, SP, false, false><<<g, ROWS, 0, s>>>(a);
    }
    return cudaGetLastError();
  }
  template <typename T, int ROWS, bool HAS_Z, bool SP>
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
      cfg.blockDim = dim3(ROWS);
      cfg.dynamicSmemBytes = 0;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, scan_out_kernel<T, ROWS, HAS_Z, SP, ZOH>, a);
    }
    scan_out_kernel<T, ROWS, HAS_Z, SP, ZOH><<<g, ROWS, 0, s>>>(a);
    return cudaGetLastError();
  }
  template <typename T, bool HAS_Z, bool SP>
  static cudaError_t chained_t(const ScanArgs& a, int grid, cudaStream_t s) {
    scan_out_chained_kernel<T, HAS_Z, SP, ZOH><<<grid, 32, 0, s>>>(a);
    return cudaGetLastError();
  }
  template <typename T, bool HAS_Z, bool SP>
  static cudaError_t fused_t(const ScanArgs& a, int grid, cudaStream_t s) {
    scan_fused_kernel<T, HAS_Z, SP, ZOH><<<grid, 32, 0, s>>>(a);
    return cudaGetLastError();
  }
  template <typename T>
  static cudaError_t fused_d(const ScanArgs& a, int grid, bool has_z, bool sp, cudaStream_t s) {
    if (has_z) return sp ? fused_t<T, true, true>(a, grid, s) : fused_t<T, true, false>(a, grid, s);
    return sp ? fused_t<T, false, true>(a, grid, s) : fused_t<T, false, false>(a, grid, s);
  }
  static cudaError_t fused(const ScanArgs& a, int grid, int dtype, bool has_z, bool sp, cudaStream_t s) {
    return dtype == 1 ? fused_d<uint16_t>(a, grid, has_z, sp, s) : fused_d<float>(a, grid, has_z, sp, s);
  }
  template <typename T>
  static cudaError_t chained_d(const ScanArgs& a, int grid, bool has_z, bool sp, cudaStream_t s) {
    if (has_z) return sp ? chained_t<T, true, true>(a, grid, s) : chained_t<T, true, false>(a, grid, s);
    return sp ? chained_t<T, false, true>(a, grid, s) : chained_t<T, false, false>(a, grid, s);
  }
  template <typename T, int ROWS>
  static cudaError_t chunk_state_d(const ScanArgs& a, bool sp, cudaStream_t s) {
    return sp ? chunk_state_t<T, ROWS, true>(a, s) : chunk_state_t<T, ROWS, false>(a, s);
  }
  template <typename T, int ROWS>
  static cudaError_t out_d(const ScanArgs& a, bool has_z, bool sp, cudaStream_t s) {
    if (has_z) return sp ? out_t<T, ROWS, true, true>(a, s) : out_t<T, ROWS, true, false>(a, s);
    return sp ? out_t<T, ROWS, false, true>(a, s) : out_t<T, ROWS, false, false>(a, s);
  }
  static cudaError_t chained(const ScanArgs& a, int grid, int dtype, bool has_z, bool sp, cudaStream_t s) {
    return dtype == 1 ? chained_d<uint16_t>(a, grid, has_z, sp, s) : chained_d<float>(a, grid, has_z, sp, s);
  }
  static cudaError_t chunk_state(const ScanArgs& a, int rows, int dtype, bool sp, cudaStream_t s) {
    if (dtype == 1) return rows == 32 ? chunk_state_d<uint16_t, 32>(a, sp, s) : chunk_state_d<uint16_t, 64>(a, sp, s);
    return rows == 32 ? chunk_state_d<float, 32>(a, sp, s) : chunk_state_d<float, 64>(a, sp, s);
  }
  static cudaError_t out(const ScanArgs& a, int rows, int dtype, bool has_z, bool sp, cudaStream_t s) {
    if (dtype == 1) return rows == 32 ? out_d<uint16_t, 32>(a, has_z, sp, s) : out_d<uint16_t, 64>(a, has_z, sp, s);
    return rows == 32 ? out_d<float, 32>(a, has_z, sp, s) : out_d<float, 64>(a, has_z, sp, s);
  }
};

// the zero-order-hold launches, defined in scan_zoh.cu
cudaError_t launch_scan_chunk_state_zoh(const ScanArgs& a, int rows, int dtype, bool sp, cudaStream_t s);
cudaError_t launch_scan_out_zoh(const ScanArgs& a, int rows, int dtype, bool has_z, bool sp, cudaStream_t s);
cudaError_t launch_scan_chained_zoh(const ScanArgs& a, int grid, int dtype, bool has_z, bool sp, cudaStream_t s);
cudaError_t launch_scan_fused_zoh(const ScanArgs& a, int grid, int dtype, bool has_z, bool sp, cudaStream_t s);

}  // namespace mssm
