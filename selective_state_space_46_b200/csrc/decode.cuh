// One-token selective state update (decode), sm_100a.
//
// The recurrent view of the selective SSM ("State Space Models in Large
// Language Models ...", section Discretization, recurrent view; "SSM vs
// Attention: The Decision Page", the cost model's fixed-size state): per row
// (b, d), delta = softplus(dt + bias), h_n <- exp(delta A_dn) h_n + delta B_n x,
// y = C . h + D x, times silu(z); h is read and written in place.
//
// The step moves 64 + 64 bytes of fp32 state per row against 16 exponentials,
// so it is HBM-bound and the design goal is bytes in flight.
//  * Contiguous state (the usual [Bt, D, 16] layout): a CTA owns 256 rows, whose
//    16 KB of state is one contiguous range.  One thread issues a single bulk
//    copy (cp.async.bulk, completion counted on an mbarrier) into shared memory,
//    so every resident CTA keeps 16 KB in flight from one instruction, while
//    all threads load their x/dt/z and A/B/C.  Each thread then updates its row
//    in shared memory (the four 16-byte quarters are visited in a lane-rotated
//    order, which makes the accesses bank-conflict free) and one thread writes
//    the tile back with a bulk store.  The mbarrier wait is bounded: if it gives
//    up, the CTA records an error in a device word (read by mssm_get_error),
//    waits a bounded time more for its copy, and leaves its rows untouched.
//  * Any other layout: one thread per row with 128-bit loads where aligned.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace mssm {

constexpr int kDecodeThreads = 256;            // rows per CTA
constexpr int kDecodeSpinLimit = 1 << 22;      // bounded mbarrier polls

struct DecodeArgs {
  float* state;
  int64_t st_sb, st_sd;  // n stride 1
  const void* x;
  const void* dt;
  const void* z;
  void* out;
  int64_t x_sb, x_sd, dt_sb, dt_sd, z_sb, z_sd, o_sb, o_sd;
  const float* A;
  int64_t A_sd, A_sn;
  const void* B;
  const void* C;
  int64_t B_sb, B_sn, C_sb, C_sn;
  const float* Dskip;
  int64_t D_s;
  const float* bias;
  int64_t bias_s;
  int Bt, D;
  int softplus;
  int vec_state;  // every row's state starts 16-byte aligned
  int vec_A;      // A rows 16-byte aligned with unit n stride
  int vec_BC;     // B and C rows 16-byte aligned with unit n stride
  unsigned int* err;  // device error word: bit 0 = a bulk copy did not complete in time
};

template <typename T>
__device__ __forceinline__ float ld_elem(const void* base, int64_t off) {
  return Elem<T>::load(static_cast<const T*>(base) + off);
}

// 4 consecutive values (n stride 1, aligned) or strided scalars
template <typename T>
__device__ __forceinline__ float4 load4(const void* base, int64_t off, int64_t stride, bool vec) {
  const T* p = static_cast<const T*>(base) + off;
  if (vec) {
    if constexpr (sizeof(T) == 2) {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
      return make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
    } else {
      return __ldg(reinterpret_cast<const float4*>(p));
    }
  }
  return make_float4(Elem<T>::load(p), Elem<T>::load(p + stride), Elem<T>::load(p + 2 * stride),
                     Elem<T>::load(p + 3 * stride));
}

// Per-row scalars of the update.
struct DecodeRow {
  int b, d;
  float x, dt, w, dl2;
};

// rows < 2^31 (checked on the host), so the row splits with 32-bit arithmetic
template <typename T>
__device__ __forceinline__ DecodeRow decode_row_scalars(const DecodeArgs& p, uint32_t row) {
  DecodeRow r;
  r.b = int(row / uint32_t(p.D));
  r.d = int(row - uint32_t(r.b) * uint32_t(p.D));
  r.x = ld_elem<T>(p.x, int64_t(r.b) * p.x_sb + int64_t(r.d) * p.x_sd);
  float dt = ld_elem<T>(p.dt, int64_t(r.b) * p.dt_sb + int64_t(r.d) * p.dt_sd);
  if (p.bias) dt += p.bias[int64_t(r.d) * p.bias_s];
  if (p.softplus) dt = softplus_f(dt);
  r.dt = dt;
  r.w = dt * r.x;
  r.dl2 = dt * kLog2e;
  return r;
}

// Update one 16-byte quarter q (states 4q..4q+3); returns the partial readout.
template <typename T>
__device__ __forceinline__ float decode_quarter(const DecodeArgs& p, const DecodeRow& r, int q, float4& h) {
  const float4 a = load4<float>(p.A, int64_t(r.d) * p.A_sd + int64_t(4 * q) * p.A_sn, p.A_sn, p.vec_A != 0);
  const float4 bv = load4<T>(p.B, int64_t(r.b) * p.B_sb + int64_t(4 * q) * p.B_sn, p.B_sn, p.vec_BC != 0);
  const float4 cv = load4<T>(p.C, int64_t(r.b) * p.C_sb + int64_t(4 * q) * p.C_sn, p.C_sn, p.vec_BC != 0);
  h.x = fmaf(ex2f(r.dl2 * a.x), h.x, r.w * bv.x);
  h.y = fmaf(ex2f(r.dl2 * a.y), h.y, r.w * bv.y);
  h.z = fmaf(ex2f(r.dl2 * a.z), h.z, r.w * bv.z);
  h.w = fmaf(ex2f(r.dl2 * a.w), h.w, r.w * bv.w);
  return fmaf(cv.x, h.x, fmaf(cv.y, h.y, fmaf(cv.z, h.z, cv.w * h.w)));
}

template <typename T, bool HAS_Z>
__device__ __forceinline__ void decode_finish(const DecodeArgs& p, const DecodeRow& r, float y) {
  if (p.Dskip) y = fmaf(p.Dskip[int64_t(r.d) * p.D_s], r.x, y);
  if constexpr (HAS_Z) y *= gate_f<T>(ld_elem<T>(p.z, int64_t(r.b) * p.z_sb + int64_t(r.d) * p.z_sd));
  T* o = static_cast<T*>(p.out) + int64_t(r.b) * p.o_sb + int64_t(r.d) * p.o_sd;
  if constexpr (sizeof(T) == 2) {
    *o = f_to_bf16(y);
  } else {
    *o = y;
  }
}

// ---------------------------------------------------------------------------
// contiguous state: bulk copy in, update in shared memory, bulk copy out
// ---------------------------------------------------------------------------
template <typename T, bool HAS_Z>
__global__ void __launch_bounds__(kDecodeThreads) state_update_bulk_kernel(const DecodeArgs p) {
  __shared__ __align__(128) float st_s[kDecodeThreads * kN];
  __shared__ __align__(8) unsigned long long mbar;
  const int tid = threadIdx.x;
  const int64_t rows = int64_t(p.Bt) * p.D;
  const int64_t r0 = int64_t(blockIdx.x) * kDecodeThreads;
  const int nrows = int(rows - r0 < kDecodeThreads ? rows - r0 : kDecodeThreads);
  const uint32_t bytes = uint32_t(nrows) * kN * 4;
  float* gtile = p.state + r0 * kN;  // contiguous layout: row r starts at r * 16
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(st_s));
  const uint32_t mb = static_cast<uint32_t>(__cvta_generic_to_shared(&mbar));

  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mb) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(sbase), "l"(gtile), "r"(bytes), "r"(mb) : "memory");
  }

  const bool live = tid < nrows;
  DecodeRow r{};
  if (live) r = decode_row_scalars<T>(p, uint32_t(r0) + uint32_t(tid));

  uint32_t done = 0;
  for (int it = 0; it < kDecodeSpinLimit && !done; ++it) {
    asm volatile("{\n .reg .pred pr;\n mbarrier.try_wait.parity.shared::cta.b64 pr, [%1], 0;\n selp.u32 %0, 1, 0, pr;\n}"
                 : "=r"(done) : "r"(mb) : "memory");
  }
  if (!__syncthreads_and(done)) {
    // give up: record the error, give the copy a bounded time more, leave the rows untouched
    if (tid == 0) atomicOr(p.err, 1u);
    for (int it = 0; it < kDecodeSpinLimit && !done; ++it) {
      asm volatile("{\n .reg .pred pr;\n mbarrier.try_wait.parity.shared::cta.b64 pr, [%1], 0;\n selp.u32 %0, 1, 0, pr;\n}"
                   : "=r"(done) : "r"(mb) : "memory");
    }
    return;
  }

  if (live) {
    float4* hs = reinterpret_cast<float4*>(st_s + tid * kN);
    float y = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int q = (k + (tid >> 1)) & 3;  // lane-rotated quarter order: conflict-free
      float4 h = hs[q];
      y += decode_quarter<T>(p, r, q, h);
      hs[q] = h;
    }
    decode_finish<T, HAS_Z>(p, r, y);
  }
  // make the generic-proxy shared-memory writes visible to the bulk copy, then store
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (tid == 0) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gtile), "r"(sbase), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }
}

// ---------------------------------------------------------------------------
// contiguous state, persistent streaming form: a grid of a few CTAs per SM,
// each walking its tiles (blockIdx.x, blockIdx.x + gridDim.x, ...) through a
// ring of kStreamBufs shared-memory tiles.  kStreamBufs - 1 bulk loads are kept
// in flight ahead of the tile being updated, and the bulk store of a tile
// overlaps the next tiles; so every SM keeps its share of the bytes moving for the whole
// launch, with no per-CTA ramp-up or tail wave.
// ---------------------------------------------------------------------------
constexpr int kStreamBufs = 4;        // tiles resident per CTA
constexpr int kStreamAhead = kStreamBufs - 1;
constexpr int kStreamCtasPerSm = 3;   // 3 x 64 KB shared memory, 768 threads, <= 85 registers
constexpr int kStreamTileBytes = kDecodeThreads * kN * 4;

__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t mb, uint32_t parity) {
  uint32_t done;
  asm volatile("{\n .reg .pred pr;\n mbarrier.try_wait.parity.shared::cta.b64 pr, [%1], %2;\n selp.u32 %0, 1, 0, pr;\n}"
               : "=r"(done) : "r"(mb), "r"(parity) : "memory");
  return done;
}

template <typename T, bool HAS_Z>
__global__ void __launch_bounds__(kDecodeThreads, kStreamCtasPerSm) state_update_stream_kernel(const DecodeArgs p) {
  extern __shared__ __align__(128) float ring_s[];  // kStreamBufs x [kDecodeThreads][16]
  __shared__ __align__(8) unsigned long long mbar[kStreamBufs];
  const int tid = threadIdx.x;
  const uint32_t rows = uint32_t(p.Bt) * uint32_t(p.D);
  const uint32_t ntiles = (rows + kDecodeThreads - 1) / kDecodeThreads;
  if (blockIdx.x >= ntiles) return;
  const uint32_t mine = (ntiles - 1 - blockIdx.x) / gridDim.x + 1;  // tiles of this CTA
  const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(ring_s));
  const uint32_t mb0 = static_cast<uint32_t>(__cvta_generic_to_shared(&mbar[0]));

  // tile i of this CTA: global tile blockIdx.x + i * gridDim.x; the last tile may be partial
  auto tile_rows = [&](uint32_t i) {
    const uint32_t r0 = (blockIdx.x + i * gridDim.x) * uint32_t(kDecodeThreads);
    return rows - r0 < uint32_t(kDecodeThreads) ? rows - r0 : uint32_t(kDecodeThreads);
  };
  auto tile_ptr = [&](uint32_t i) {
    return p.state + size_t(blockIdx.x + i * gridDim.x) * kDecodeThreads * kN;
  };
  auto issue_load = [&](uint32_t i) {  // one thread
    const uint32_t buf = i % kStreamBufs;
    const uint32_t bytes = tile_rows(i) * kN * 4;
    const uint32_t mb = mb0 + buf * 8;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(ring + buf * kStreamTileBytes), "l"(tile_ptr(i)), "r"(bytes), "r"(mb) : "memory");
  };

  if (tid == 0) {
#pragma unroll
    for (int k = 0; k < kStreamBufs; ++k)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mb0 + 8 * k) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0) {
    for (uint32_t j = 0; j < uint32_t(kStreamAhead) && j < mine; ++j) issue_load(j);
  }

  uint32_t i = 0;
  bool ok = true;
  for (; i < mine; ++i) {
    const uint32_t buf = i % kStreamBufs;
    const uint32_t nrows = tile_rows(i);
    const bool live = uint32_t(tid) < nrows;
    DecodeRow r{};
    if (live) r = decode_row_scalars<T>(p, (blockIdx.x + i * gridDim.x) * uint32_t(kDecodeThreads) + tid);

    uint32_t done = 0;
    const uint32_t parity = (i / kStreamBufs) & 1u;
    for (int it = 0; it < kDecodeSpinLimit && !done; ++it) done = mbar_try_wait(mb0 + buf * 8, parity);
    if (!__syncthreads_and(done)) {
      ok = false;
      break;
    }
    if (live) {
      float4* hs = reinterpret_cast<float4*>(ring_s + buf * (kDecodeThreads * kN) + tid * kN);
      float y = 0.0f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = (k + (tid >> 1)) & 3;  // lane-rotated quarter order: conflict-free
        float4 h = hs[q];
        y += decode_quarter<T>(p, r, q, h);
        hs[q] = h;
      }
      decode_finish<T, HAS_Z>(p, r, y);
    }
    // generic-proxy writes of this tile -> visible to the bulk store
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                   ::"l"(tile_ptr(i)), "r"(ring + buf * kStreamTileBytes), "r"(nrows * kN * 4) : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      if (i + kStreamAhead < mine) {
        // tile i + kStreamAhead reuses the buffer of tile i - 1, whose store is the older of
        // the (at most) two stores in flight
        asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        issue_load(i + kStreamAhead);
      }
    }
  }
  if (!ok && tid == 0) {
    // record the error; give the loads still in flight (tiles i .. i + kStreamAhead - 1) a
    // bounded time to land
    atomicOr(p.err, 1u);
    for (uint32_t j = i; j < i + kStreamAhead && j < mine; ++j) {
      uint32_t done = 0;
      for (int it = 0; it < kDecodeSpinLimit && !done; ++it)
        done = mbar_try_wait(mb0 + (j % kStreamBufs) * 8, (j / kStreamBufs) & 1u);
    }
  }
  if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// any layout: one thread per row
// ---------------------------------------------------------------------------
template <typename T, bool HAS_Z>
__global__ void __launch_bounds__(kDecodeThreads) state_update_kernel(const DecodeArgs p) {
  const uint32_t row = blockIdx.x * uint32_t(kDecodeThreads) + threadIdx.x;
  const uint32_t rows = uint32_t(p.Bt) * uint32_t(p.D);
  if (row >= rows) return;
  const int b = int(row / uint32_t(p.D));
  const int d = int(row - uint32_t(b) * uint32_t(p.D));
  float* st = p.state + int64_t(b) * p.st_sb + int64_t(d) * p.st_sd;
  float4 h[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (p.vec_state) {
      h[q] = __ldcs(reinterpret_cast<const float4*>(st) + q);
    } else {
      h[q] = make_float4(st[4 * q], st[4 * q + 1], st[4 * q + 2], st[4 * q + 3]);
    }
  }
  const DecodeRow r = decode_row_scalars<T>(p, row);
  float y = 0.0f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    y += decode_quarter<T>(p, r, q, h[q]);
    if (p.vec_state) {
      __stcs(reinterpret_cast<float4*>(st) + q, h[q]);
    } else {
      st[4 * q] = h[q].x; st[4 * q + 1] = h[q].y; st[4 * q + 2] = h[q].z; st[4 * q + 3] = h[q].w;
    }
  }
  decode_finish<T, HAS_Z>(p, r, y);
}

}  // namespace mssm
