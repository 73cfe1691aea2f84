// One-token selective state update (decode), sm_100a.
//
// The recurrent view of the selective SSM ("State Space Models in Large
// Language Models ...", section Discretization, recurrent view; "SSM vs
// Attention: The Decision Page", the cost model's fixed-size state): per row
// (b, d), delta = softplus(dt + bias), h_n <- exp(delta A_dn) h_n + delta B_n x,
// y = C . h + D x, times silu(z); h is read and written in place.
//
// The step moves 64 + 64 bytes of fp32 state per row against 16 exponentials,
// so it is HBM-bound.  Four threads own one row, one 16-byte quarter of its
// state each: a warp reads and writes eight rows' states as 512 contiguous
// bytes, with one 128-bit load and one 128-bit store per thread.  The partial
// readouts of the four quarters are summed with two butterfly shuffles.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace mssm {

constexpr int kDecodeThreads = 256;  // 64 rows per CTA

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
};

template <typename T>
__device__ __forceinline__ float ld_elem(const void* base, int64_t off) {
  return Elem<T>::load(static_cast<const T*>(base) + off);
}

template <typename T, bool HAS_Z>
__global__ void __launch_bounds__(kDecodeThreads) state_update_kernel(const DecodeArgs p) {
  const int64_t gid = int64_t(blockIdx.x) * kDecodeThreads + threadIdx.x;
  const int64_t row = gid >> 2;
  const int q = int(gid & 3);
  const int64_t rows = int64_t(p.Bt) * p.D;
  // Lanes past the last row compute on a clamped row and store nothing, so the
  // whole warp stays converged for the shuffles below.
  const bool live = row < rows;
  const int64_t rr = live ? row : rows - 1;
  const int b = int(rr / p.D);
  const int d = int(rr - int64_t(b) * p.D);

  float* st = p.state + int64_t(b) * p.st_sb + int64_t(d) * p.st_sd + 4 * q;
  float4 h;
  if (p.vec_state) {
    h = __ldcs(reinterpret_cast<const float4*>(st));
  } else {
    h = make_float4(st[0], st[1], st[2], st[3]);
  }
  const float xv = ld_elem<T>(p.x, int64_t(b) * p.x_sb + int64_t(d) * p.x_sd);
  float dt = ld_elem<T>(p.dt, int64_t(b) * p.dt_sb + int64_t(d) * p.dt_sd);
  if (p.bias) dt += p.bias[int64_t(d) * p.bias_s];
  if (p.softplus) dt = softplus_f(dt);
  const float* Ar = p.A + int64_t(d) * p.A_sd + int64_t(4 * q) * p.A_sn;
  const float a0 = Ar[0], a1 = Ar[p.A_sn], a2 = Ar[2 * p.A_sn], a3 = Ar[3 * p.A_sn];
  const int64_t bo = int64_t(b) * p.B_sb + int64_t(4 * q) * p.B_sn;
  const int64_t co = int64_t(b) * p.C_sb + int64_t(4 * q) * p.C_sn;
  const float b0 = ld_elem<T>(p.B, bo), b1 = ld_elem<T>(p.B, bo + p.B_sn);
  const float b2 = ld_elem<T>(p.B, bo + 2 * p.B_sn), b3 = ld_elem<T>(p.B, bo + 3 * p.B_sn);
  const float c0 = ld_elem<T>(p.C, co), c1 = ld_elem<T>(p.C, co + p.C_sn);
  const float c2 = ld_elem<T>(p.C, co + 2 * p.C_sn), c3 = ld_elem<T>(p.C, co + 3 * p.C_sn);

  const float w = dt * xv;
  const float dl2 = dt * kLog2e;
  h.x = fmaf(ex2f(dl2 * a0), h.x, w * b0);
  h.y = fmaf(ex2f(dl2 * a1), h.y, w * b1);
  h.z = fmaf(ex2f(dl2 * a2), h.z, w * b2);
  h.w = fmaf(ex2f(dl2 * a3), h.w, w * b3);
  float y = fmaf(c0, h.x, fmaf(c1, h.y, fmaf(c2, h.z, c3 * h.w)));
  y += __shfl_xor_sync(0xffffffffu, y, 1);
  y += __shfl_xor_sync(0xffffffffu, y, 2);

  if (!live) return;
  if (p.vec_state) {
    __stcs(reinterpret_cast<float4*>(st), h);
  } else {
    st[0] = h.x; st[1] = h.y; st[2] = h.z; st[3] = h.w;
  }
  if (q == 0) {
    if (p.Dskip) y = fmaf(p.Dskip[int64_t(d) * p.D_s], xv, y);
    if constexpr (HAS_Z) y *= silu_f(ld_elem<T>(p.z, int64_t(b) * p.z_sb + int64_t(d) * p.z_sd));
    T* o = static_cast<T*>(p.out) + int64_t(b) * p.o_sb + int64_t(d) * p.o_sd;
    if constexpr (sizeof(T) == 2) {
      *o = f_to_bf16(y);
    } else {
      *o = y;
    }
  }
}

}  // namespace mssm
