// Causal depthwise conv1d + SiLU, the step that produces the scan's input u
// ("Linear Attention vs Softmax Attention ...", section Implementation: the
// listed layer's grouped Conv1d, one group per channel, kernel size K, padding
// K - 1 and the output truncated to the first L steps, then SiLU), sm_100a.
//
//   out[b,d,t] = act(bias[d] + sum_{k<K} w[d,k] x[b,d,t-(K-1)+k]),  x = 0 before the start
//
// The work is HBM-bound: 2 + 2 bytes per element in bf16 against K FMAs and one
// SFU operation; the taps and the SiLU run on packed f32x2 pairs of outputs, so a
// warp spends few enough issue slots per element for its compute to hide under the
// loads of the other warps.  A warp item is one row (b, d) over kConvPieces pieces of 32
// lanes x one 16-byte block.  Each lane issues the loads of all its blocks up
// front, then per piece takes the K - 1 inputs before its block from the lane
// below by shuffle (lane 0: from the previous piece, or loaded for the first)
// and stores one 16-byte block of outputs, so every access is a fully used
// 512-byte warp transaction.  Packed
// sequences (cu_seqlens) restart at every sequence start: inputs before it read
// as zero, and blocks are aligned to the row, not to the sequence, with the
// outputs outside the sequence left unwritten.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace mssm {

constexpr int kConvMaxK = 4;
constexpr int kConvWarps = 4;   // rows per CTA
constexpr int kConvPieces = 8;  // pieces of 32 blocks per warp item

struct ConvArgs {
  const void* x;
  void* out;
  int64_t x_sb, x_sd, o_sb, o_sd;  // element strides, L stride 1
  const float* w;
  int64_t w_sd, w_sk;
  const float* bias;
  int64_t bias_s;
  int Bt, D, L, K;   // Bt: batches, or packed sequences (data batch 0)
  int vec;           // x and out rows start 16-byte aligned
  const int* cu_seqlens;
  unsigned* err;     // device error word: bit 2 = inconsistent cu_seqlens
};

template <typename T>
__device__ __forceinline__ void conv_unpack(const uint4& v, float* f) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf16lo(w[i]);
      f[2 * i + 1] = bf16hi(w[i]);
    }
  } else {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
}

template <typename T, int K, bool SILU>
__global__ void __launch_bounds__(32 * kConvWarps) causal_conv1d_kernel(const ConvArgs p) {
  constexpr int S = 16 / int(sizeof(T));  // steps per 16-byte block
  constexpr int P = 32 * S;               // steps per warp piece
  const int lane = threadIdx.x & 31;
  const uint32_t row = blockIdx.x * uint32_t(kConvWarps) + (threadIdx.x >> 5);
  if (row >= uint32_t(p.Bt) * uint32_t(p.D)) return;  // whole warps
  const int vb = int(row / uint32_t(p.D));
  const int d = int(row - uint32_t(vb) * uint32_t(p.D));

  // the steps of this row's sequence: [tb, te)
  int b = vb, tb = 0, te = p.L;
  if (p.cu_seqlens) {
    int a = __ldg(p.cu_seqlens + vb), e = __ldg(p.cu_seqlens + vb + 1);
    if ((a < 0 || a > p.L || e < a || e > p.L) && lane == 0 && p.err) atomicOr(p.err, 4u);
    a = min(max(a, 0), p.L);
    e = min(max(e, a), p.L);
    b = 0;
    tb = a;
    te = e;
  }
  const int t0 = tb + int(blockIdx.y) * (kConvPieces * P);  // this item's outputs: [t0, t1)
  if (t0 >= te) return;
  const int t1 = min(te, t0 + kConvPieces * P);
  const int ta = t0 - t0 % S;  // first block, aligned to the row

  const T* xr = static_cast<const T*>(p.x) + int64_t(b) * p.x_sb + int64_t(d) * p.x_sd;
  T* orow = static_cast<T*>(p.out) + int64_t(b) * p.o_sb + int64_t(d) * p.o_sd;
  // inputs at steps before tb are zero; steps at or after te are never needed
  auto x_at = [&](int t) -> float { return (t >= tb && t < te) ? Elem<T>::load(xr + t) : 0.0f; };

  // every piece's block is loaded up front: kConvPieces independent loads in flight per lane
  uint4 raw[kConvPieces];
#pragma unroll
  for (int q = 0; q < kConvPieces; ++q) {
    const int tl = ta + q * P + lane * S;
    raw[q] = (p.vec && tl >= tb && tl + S <= te) ? __ldg(reinterpret_cast<const uint4*>(xr + tl))
                                                 : make_uint4(0u, 0u, 0u, 0u);
  }
  f2_t w2[K];  // tap weights, broadcast to both lanes of a pair
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const float wk = p.w[int64_t(d) * p.w_sd + int64_t(k) * p.w_sk];
    w2[k] = f2(wk, wk);
  }
  const float bias = p.bias ? p.bias[int64_t(d) * p.bias_s] : 0.0f;
  const f2_t bias2 = f2(bias, bias);
  const f2_t half2 = f2(0.5f, 0.5f);
  // lane 0's halo for the first piece: the K - 1 inputs before ta
  float carry[kConvMaxK - 1];
#pragma unroll
  for (int k = 0; k < K - 1; ++k) carry[k] = lane == 0 ? x_at(ta - (K - 1) + k) : 0.0f;

#pragma unroll
  for (int q = 0; q < kConvPieces; ++q) {
    const int tp = ta + q * P;
    if (tp >= t1) break;  // warp-uniform
    const int tl = tp + lane * S;  // this lane's block
    // xe[0 .. K-2]: the K - 1 inputs before the block (halo), xe[K-1 ..]: the block
    float xe[S + kConvMaxK - 1];
    float* xv = xe + (K - 1);
    if (p.vec && tl >= tb && tl + S <= te) {
      conv_unpack<T>(raw[q], xv);
    } else {  // a block cut by the sequence's edges, or an unaligned row
#pragma unroll
      for (int j = 0; j < S; ++j) xv[j] = x_at(tl + j);
    }
    // halo: the last K - 1 inputs of the lane below; lane 0 takes the carried ones
#pragma unroll
    for (int k = 0; k < K - 1; ++k) {
      const float up = __shfl_up_sync(0xffffffffu, xv[S - (K - 1) + k], 1);
      xe[k] = lane == 0 ? carry[k] : up;
    }
#pragma unroll
    for (int k = 0; k < K - 1; ++k) carry[k] = __shfl_sync(0xffffffffu, xv[S - (K - 1) + k], 31);

    // outputs in pairs (y_j, y_j+1) on the packed f32x2 pipe: tap k reads the input
    // pair (xe[j + k], xe[j + k + 1])
    float y[S];
#pragma unroll
    for (int j = 0; j < S; j += 2) {
      f2_t acc = bias2;
#pragma unroll
      for (int k = 0; k < K; ++k) acc = fma2(w2[k], f2(xe[j + k], xe[j + k + 1]), acc);
      if constexpr (SILU && sizeof(T) == 2) {
        // silu(a) = h (1 + tanh h), h = a / 2, on both lanes of the pair
        const f2_t h = mul2(acc, half2);
        float hlo, hhi;
        f2split(h, hlo, hhi);
        float tlo, thi;
        asm("tanh.approx.f32 %0, %1;" : "=f"(tlo) : "f"(hlo));
        asm("tanh.approx.f32 %0, %1;" : "=f"(thi) : "f"(hhi));
        acc = fma2(h, f2(tlo, thi), h);
      }
      f2split(acc, y[j], y[j + 1]);
      if constexpr (SILU && sizeof(T) == 4) {
        y[j] = gate_f<T>(y[j]);  // exact form for fp32 outputs
        y[j + 1] = gate_f<T>(y[j + 1]);
      }
    }
    // store the outputs in [t0, t1)
    if (p.vec && tl >= t0 && tl + S <= t1) {
      if constexpr (sizeof(T) == 2) {
        *reinterpret_cast<uint4*>(orow + tl) = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                                                          pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
      } else {
        *reinterpret_cast<float4*>(orow + tl) = make_float4(y[0], y[1], y[2], y[3]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < S; ++j) {
        const int t = tl + j;
        if (t >= t0 && t < t1) {
          if constexpr (sizeof(T) == 2) {
            orow[t] = f_to_bf16(y[j]);
          } else {
            orow[t] = y[j];
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// One decode step of the conv: state [Bt, D, K-1] holds the previous K-1 inputs,
// oldest first; out = act(bias + sum_k w_k window_k) over window = [state, x];
// the state then drops its oldest input and takes x.  One thread per row.
// ---------------------------------------------------------------------------
struct ConvUpdateArgs {
  void* state;
  int64_t st_sb, st_sd, st_sk;
  const void* x;
  void* out;
  int64_t x_sb, x_sd, o_sb, o_sd;
  const float* w;
  int64_t w_sd, w_sk;
  const float* bias;
  int64_t bias_s;
  int Bt, D, K;
  int silu;
};

template <typename T, int K>
__global__ void __launch_bounds__(256) causal_conv1d_update_kernel(const ConvUpdateArgs p) {
  const uint32_t row = blockIdx.x * 256u + threadIdx.x;
  if (row >= uint32_t(p.Bt) * uint32_t(p.D)) return;
  const int b = int(row / uint32_t(p.D));
  const int d = int(row - uint32_t(b) * uint32_t(p.D));
  T* st = static_cast<T*>(p.state) + int64_t(b) * p.st_sb + int64_t(d) * p.st_sd;
  float win[K];
#pragma unroll
  for (int k = 0; k < K - 1; ++k) win[k] = Elem<T>::load(st + int64_t(k) * p.st_sk);
  const T xin = static_cast<const T*>(p.x)[int64_t(b) * p.x_sb + int64_t(d) * p.x_sd];
  win[K - 1] = Elem<T>::load(&xin);
  float acc = p.bias ? p.bias[int64_t(d) * p.bias_s] : 0.0f;
#pragma unroll
  for (int k = 0; k < K; ++k) acc = fmaf(p.w[int64_t(d) * p.w_sd + int64_t(k) * p.w_sk], win[k], acc);
  const float y = p.silu ? gate_f<T>(acc) : acc;
  T* o = static_cast<T*>(p.out) + int64_t(b) * p.o_sb + int64_t(d) * p.o_sd;
  if constexpr (sizeof(T) == 2) {
    *o = f_to_bf16(y);
  } else {
    *o = y;
  }
  // shift the window: the stored values are inputs, kept in their own dtype (exact)
#pragma unroll
  for (int k = 0; k < K - 2; ++k) st[int64_t(k) * p.st_sk] = st[int64_t(k + 1) * p.st_sk];
  if (K > 1) st[int64_t(K - 2) * p.st_sk] = xin;
}

}  // namespace mssm
