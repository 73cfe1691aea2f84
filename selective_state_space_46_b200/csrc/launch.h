// Internal host-side launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>

#include "bwd.cuh"
#include "conv.cuh"
#include "decode.cuh"
#include "scan.cuh"

namespace mssm {

// dtype: 0 = fp32 storage, 1 = bf16 storage.  Return the launch error, if any.
// rows: channels per row tile (32, 64 or 128), rpt: rows per thread (1 or 2; 2 for bf16 only),
// so rows / rpt threads per CTA; the grid is (Bt * tiles_per_batch, nseg [- 1]).
cudaError_t launch_scan_chunk_state(const ScanArgs& a, int rows, int rpt, int dtype, bool softplus, cudaStream_t s);
cudaError_t launch_scan_out(const ScanArgs& a, int rows, int rpt, int dtype, bool has_z, bool softplus,
                            cudaStream_t s);
// Persistent chained forward kernel (row tiles of 32 * rpt channels), `grid` one-warp CTAs.
cudaError_t launch_scan_chained(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool softplus,
                                cudaStream_t s);
// Fused single-pass (look-back) kernel (row tiles of 32 * rpt channels), `grid` one-warp CTAs.
cudaError_t launch_scan_fused(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool softplus,
                              cudaStream_t s);
// Split-chunk kernel (row tiles of 32 * rpt channels), `grid` persistent CTAs of kSplitWarps
// warps; seg_len is kSplitWarps sub-segments.
cudaError_t launch_scan_split(const ScanArgs& a, int grid, int rpt, int dtype, bool has_z, bool softplus,
                              cudaStream_t s);
// Device address of this device's error word (cached per device).
cudaError_t device_error_word(unsigned int** out);
// Drops every cached device address of a module symbol (after this, the next call looks
// them up again: a device reset may load the module at another address).
void forget_device_addresses();
// Incremented by forget_device_addresses: caches of per-device setup compare against it.
int device_address_generation();
// bulk: the state is one contiguous [rows][16] range (bulk-copy kernel), else one thread per row.
enum class DecodePath { kStream, kBulkTile, kPerRow };
cudaError_t launch_state_update(const DecodeArgs& a, int dtype, bool has_z, DecodePath path, cudaStream_t s);
// Causal conv1d + SiLU: grid (ceil(rows / kConvWarps), items); one decode step of it.
cudaError_t launch_causal_conv1d(const ConvArgs& a, int items, int dtype, bool silu, cudaStream_t s);
cudaError_t launch_causal_conv1d_update(const ConvUpdateArgs& a, int dtype, cudaStream_t s);
// Backward scan: pass A (chunk summaries both ways and their folds, when there is more than
// one chunk) and pass B (recompute and backward sweep per chunk).
cudaError_t launch_scan_bwd(const BwdArgs& a, int dtype, bool has_z, cudaStream_t s);
// Reads (and optionally clears) the current device's error word.
cudaError_t read_device_error(unsigned int* value, bool clear);

}  // namespace mssm
