// Selective scan forward kernels and their launcher (sm_100a).
//
// The scan is the Mamba-1 selective state space recurrence: per row (b, d) and
// state n, h_t = exp(delta_t A_dn) h_(t-1) + delta_t B_tn u_t, y_t = C_t . h_t +
// D_d u_t, times silu(z_t) ("Linear Attention vs Softmax Attention: Can RWKV or
// Mamba Replace Transformers?", section Implementation; "State Space Models in
// Large Language Models ...", section Dynamic Parameterization for
// delta = softplus(parameter + linear)).
//
// Work decomposition
//  * One thread owns one row (b, d) and keeps its 16-wide state in registers
//    as eight packed fp32 pairs; rows of one CTA are 64 consecutive channels
//    of the same batch, so the CTA stages B and C of that batch once per
//    32-step chunk in shared memory (converted to fp32, laid out [t][B0..15,
//    C0..15]) and every row reads them as warp-wide broadcasts.
//  * u / delta / z are streamed per row along L with 16-byte vector loads and
//    one 16-step block of prefetch; y is written with 16-byte vector stores.
//  * Long sequences are split into chunks of seg_len steps.  The per-position
//    affine maps (A_bar_t, B_bar_t u_t) compose associatively ("Mamba selective
//    state space", section "Selectivity Removes the Convolution Shortcut; Scan
//    Restores Parallelism"), so a chunk is summarised by (S, H): S = sum of
//    delta over the chunk (the chunk's decay is exp(A_n S)) and H = the chunk's
//    end state from a zero start.  Kernel 1 computes (S, H) for every chunk but
//    the last with a backward sweep (2 flops per state and step instead of 3),
//    and the last CTA of a row tile to finish folds the summaries into carried
//    states (no CTA ever waits on another).  Kernel 2 re-runs every chunk
//    forward from its carried state and writes y and the final state.
//  * Structured A (A_dn == (n+1) A_d0 exactly, the S4D-real initialisation the
//    pages use) computes exp(delta A_dn) as powers of one exponential; any
//    other A takes one SFU exponential per state.  The choice is uniform per CTA.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace mssm {

constexpr int kRows = 64;   // rows (threads) per CTA
constexpr int kTC = 32;     // steps per staged B/C chunk
constexpr int kSegQuant = 64;  // chunk lengths of the length split are multiples of this

struct ScanArgs {
  const void* u;
  const void* delta;
  const void* z;
  void* out;
  int64_t u_sb, u_sd, dl_sb, dl_sd, z_sb, z_sd, o_sb, o_sd;  // element strides, L stride 1
  const void* B;
  const void* C;
  int64_t B_sb, B_sn, C_sb, C_sn;
  const float* A;
  int64_t A_sd, A_sn;
  const float* Dskip;
  int64_t D_s;
  const float* bias;
  int64_t bias_s;
  float* last_state;
  int64_t ls_sb, ls_sd;  // n stride 1
  int Bt, D, L;
  int force_general;
  int nseg, seg_len;
  int tiles_per_batch;
  int vec_rows;  // u/delta/z/out row starts are 16-byte aligned
  int vec_bc;    // B/C row starts are 16-byte aligned
  // carry workspace, used when nseg > 1
  float* ws_H;          // [nseg-1][ntiles*kRows][16]: chunk end state, then carried state
  float* ws_S;          // [nseg-1][ntiles*kRows]: sum of delta over the chunk
  unsigned* ws_count;   // [ntiles]: arrivals of kernel-1 CTAs, reset by the last one
};

// ---------------------------------------------------------------------------
// per-row 16-step (bf16) / 8-step (fp32) blocks of u, delta, z: 32 bytes each
// ---------------------------------------------------------------------------
template <typename T> struct Blk {
  static constexpr int kSteps = 32 / int(sizeof(T));
  uint32_t w[8];
  __device__ __forceinline__ float at(int j) const {
    if constexpr (sizeof(T) == 2) {
      return (j & 1) ? bf16hi(w[j >> 1]) : bf16lo(w[j >> 1]);
    } else {
      return __uint_as_float(w[j]);
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = 0u;
  }
  // Load steps [t, t + kSteps) of a row; steps at or past t_end read as 0.
  __device__ __forceinline__ void load(const T* row, int t, int t_end, bool vec) {
    if (vec && t + kSteps <= t_end) {
      const uint4* p = reinterpret_cast<const uint4*>(row + t);
      const uint4 a = __ldg(p), b = __ldg(p + 1);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else {
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t lo = (t + 2 * i < t_end) ? uint32_t(__ldg(row + t + 2 * i)) : 0u;
          const uint32_t hi = (t + 2 * i + 1 < t_end) ? uint32_t(__ldg(row + t + 2 * i + 1)) : 0u;
          w[i] = lo | (hi << 16);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          w[i] = (t + i < t_end) ? __float_as_uint(__ldg(row + t + i)) : 0u;
      }
    }
  }
};

// Store steps [t, t + kSteps) of y (fp32 values), clipped at t_end.
template <typename T>
__device__ __forceinline__ void store_block(T* row, int t, int t_end, bool vec, const float* y) {
  constexpr int S = Blk<T>::kSteps;
  if constexpr (sizeof(T) == 2) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
    if (vec && t + S <= t_end) {
      uint4* p = reinterpret_cast<uint4*>(row + t);
      p[0] = make_uint4(w[0], w[1], w[2], w[3]);
      p[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (t + 2 * i < t_end) row[t + 2 * i] = uint16_t(w[i] & 0xffffu);
        if (t + 2 * i + 1 < t_end) row[t + 2 * i + 1] = uint16_t(w[i] >> 16);
      }
    }
  } else {
    if (vec && t + S <= t_end) {
      float4* p = reinterpret_cast<float4*>(row + t);
      p[0] = make_float4(y[0], y[1], y[2], y[3]);
      p[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (t + i < t_end) row[t + i] = y[i];
    }
  }
}

// ---------------------------------------------------------------------------
// B/C staging: a kTC-step chunk of NR rows (B rows 0..15 then C rows 0..15)
// loaded by the CTA's 64 threads into registers, then written transposed to
// shared memory as fp32 [t][row].
// ---------------------------------------------------------------------------
template <typename T, int NR> struct BCStage {
  static constexpr int kVals = NR * kTC / kRows;     // values per thread (16 or 8)
  static constexpr int kWords = kVals * int(sizeof(T)) / 4;
  static constexpr int kThreadsPerRow = kTC / kVals;  // 2 or 4
  uint32_t w[kWords];

  __device__ __forceinline__ void load(const ScanArgs& p, int b, int cs, int t_end) {
    const int tid = threadIdx.x;
    const int r = tid / kThreadsPerRow;
    const int t = cs + (tid % kThreadsPerRow) * kVals;
    const T* base = (r < 16) ? static_cast<const T*>(p.B) + int64_t(b) * p.B_sb + int64_t(r) * p.B_sn
                             : static_cast<const T*>(p.C) + int64_t(b) * p.C_sb + int64_t(r - 16) * p.C_sn;
    if (p.vec_bc && t + kVals <= t_end) {
      const uint4* q = reinterpret_cast<const uint4*>(base + t);
#pragma unroll
      for (int i = 0; i < kWords / 4; ++i) {
        const uint4 v = __ldg(q + i);
        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
      }
    } else {
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < kWords; ++i) {
          const uint32_t lo = (t + 2 * i < t_end) ? uint32_t(__ldg(base + t + 2 * i)) : 0u;
          const uint32_t hi = (t + 2 * i + 1 < t_end) ? uint32_t(__ldg(base + t + 2 * i + 1)) : 0u;
          w[i] = lo | (hi << 16);
        }
      } else {
#pragma unroll
        for (int i = 0; i < kWords; ++i)
          w[i] = (t + i < t_end) ? __float_as_uint(__ldg(base + t + i)) : 0u;
      }
    }
  }

  __device__ __forceinline__ void store(float* s) const {  // s: [kTC][32] floats
    const int tid = threadIdx.x;
    const int r = tid / kThreadsPerRow;
    const int t = (tid % kThreadsPerRow) * kVals;
#pragma unroll
    for (int j = 0; j < kVals; ++j) {
      float v;
      if constexpr (sizeof(T) == 2) {
        v = (j & 1) ? bf16hi(w[j >> 1]) : bf16lo(w[j >> 1]);
      } else {
        v = __uint_as_float(w[j]);
      }
      s[(t + j) * 32 + r] = v;
    }
  }
};

// ---------------------------------------------------------------------------
// exp(delta * A_dn) for the row's 16 states, as 8 packed pairs
// ---------------------------------------------------------------------------
template <bool STRUCT>
__device__ __forceinline__ void decay_pairs(float dt, float a2_0, const f2_t (&A2p)[8], f2_t (&dA)[8]) {
  if constexpr (STRUCT) {
    // exp(dt (n+1) A_0) = a^(n+1), a = exp(dt A_0): one SFU op, 15 multiplies, depth 4
    const float a = ex2f(dt * a2_0);
    const float a2 = a * a;
    dA[0] = f2(a, a2);
    const f2_t s2 = f2(a2, a2);
    dA[1] = mul2(dA[0], s2);
    const float a4 = f2hi(dA[1]);
    const f2_t s4 = f2(a4, a4);
    dA[2] = mul2(dA[0], s4);
    dA[3] = mul2(dA[1], s4);
    const float a8 = f2hi(dA[3]);
    const f2_t s8 = f2(a8, a8);
    dA[4] = mul2(dA[0], s8);
    dA[5] = mul2(dA[1], s8);
    dA[6] = mul2(dA[2], s8);
    dA[7] = mul2(dA[3], s8);
  } else {
    const f2_t d2 = f2(dt, dt);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float lo, hi;
      f2split(mul2(d2, A2p[k]), lo, hi);
      dA[k] = f2(ex2f(lo), ex2f(hi));
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 2: forward sweep of one chunk from its carried state, fused epilogue.
// ---------------------------------------------------------------------------
// One block of S steps.  PARTIAL: the block runs past t1; the steps past the
// end become identity steps (delta = 0 gives A_bar = 1 and no input), so the
// state is exactly the state at t1 - 1.
template <typename T, bool HAS_Z, bool SOFTPLUS, bool STRUCT, bool PARTIAL>
__device__ __forceinline__ void forward_block(const float* bcrow, int valid, const Blk<T>& cu,
                                              const Blk<T>& cd, const Blk<T>& cz, float bias,
                                              float Dd, float a2_0, const f2_t (&A2p)[8],
                                              f2_t (&h2)[8], float* ybuf) {
  constexpr int S = Blk<T>::kSteps;
#pragma unroll
  for (int j = 0; j < S; ++j) {
    float uu = cu.at(j);
    float dt = cd.at(j) + bias;
    if constexpr (SOFTPLUS) dt = softplus_f(dt);
    if constexpr (PARTIAL) {
      if (j >= valid) {
        dt = 0.0f;
        uu = 0.0f;
      }
    }
    f2_t dA[8];
    decay_pairs<STRUCT>(dt, a2_0, A2p, dA);
    const float w = dt * uu;
    const f2_t w2 = f2(w, w);
    const ulonglong2* q = reinterpret_cast<const ulonglong2*>(bcrow + j * 32);
    f2_t yA = 0ull, yB = 0ull;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const ulonglong2 bb = q[k];      // B pairs (2k, 2k+1) of states 4k..4k+3
      const ulonglong2 cc = q[4 + k];  // C pairs
      h2[2 * k] = fma2(dA[2 * k], h2[2 * k], mul2(w2, bb.x));
      h2[2 * k + 1] = fma2(dA[2 * k + 1], h2[2 * k + 1], mul2(w2, bb.y));
      yA = (k == 0) ? mul2(cc.x, h2[0]) : fma2(cc.x, h2[2 * k], yA);
      yB = (k == 0) ? mul2(cc.y, h2[1]) : fma2(cc.y, h2[2 * k + 1], yB);
    }
    float y0, y1, y2, y3;
    f2split(yA, y0, y1);
    f2split(yB, y2, y3);
    float y = ((y0 + y1) + (y2 + y3)) + Dd * uu;
    if constexpr (HAS_Z) y *= silu_f(cz.at(j));
    ybuf[j] = y;
  }
}

template <typename T, bool HAS_Z, bool SOFTPLUS, bool STRUCT>
__device__ __forceinline__ void forward_chunk(const ScanArgs& p, float (*bc_s)[kTC * 32], int b,
                                              int t0, int t1, const T* urow, const T* dlrow,
                                              const T* zrow, T* orow, bool row_ok, float bias,
                                              float Dd, float a2_0, const f2_t (&A2p)[8],
                                              f2_t (&h2)[8]) {
  constexpr int S = Blk<T>::kSteps;
  const bool vec = p.vec_rows != 0;
  BCStage<T, 32> stage;
  const int nchunks = (t1 - t0 + kTC - 1) / kTC;
  if (nchunks <= 0) return;
  stage.load(p, b, t0, t1);
  stage.store(bc_s[0]);
  __syncthreads();

  Blk<T> cu, cd, cz;
  cu.load(urow, t0, t1, vec);
  cd.load(dlrow, t0, t1, vec);
  if constexpr (HAS_Z) cz.load(zrow, t0, t1, vec);
  else cz.zero();

  for (int c = 0; c < nchunks; ++c) {
    const int cs = t0 + c * kTC;
    const int ce = min(t1, cs + kTC);
    if (c + 1 < nchunks) stage.load(p, b, cs + kTC, t1);
    const float* bcb = bc_s[c & 1];
    for (int tb = cs; tb < ce; tb += S) {
      Blk<T> nu, nd, nz;
      const int tn = tb + S;
      if (tn < t1) {
        nu.load(urow, tn, t1, vec);
        nd.load(dlrow, tn, t1, vec);
        if constexpr (HAS_Z) nz.load(zrow, tn, t1, vec);
        else nz.zero();
      } else {
        nu.zero();
        nd.zero();
        nz.zero();
      }
      float ybuf[S];
      const float* bcrow = bcb + (tb - cs) * 32;
      if (tb + S <= t1)
        forward_block<T, HAS_Z, SOFTPLUS, STRUCT, false>(bcrow, S, cu, cd, cz, bias, Dd, a2_0, A2p, h2, ybuf);
      else
        forward_block<T, HAS_Z, SOFTPLUS, STRUCT, true>(bcrow, t1 - tb, cu, cd, cz, bias, Dd, a2_0, A2p, h2, ybuf);
      if (row_ok) store_block<T>(orow, tb, t1, vec, ybuf);
      cu = nu;
      cd = nd;
      cz = nz;
    }
    if (c + 1 < nchunks) stage.store(bc_s[(c + 1) & 1]);
    __syncthreads();
  }
}

template <typename T, bool HAS_Z, bool SOFTPLUS>
__global__ void __launch_bounds__(kRows) scan_out_kernel(const ScanArgs p) {
  __shared__ __align__(16) float bc_s[2][kTC * 32];
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int seg = blockIdx.y;
  const int b = tile / p.tiles_per_batch;
  const int d = (tile - b * p.tiles_per_batch) * kRows + tid;
  const bool row_ok = d < p.D;
  const int dc = row_ok ? d : p.D - 1;
  const int t0 = seg * p.seg_len;
  const int t1 = min(p.L, t0 + p.seg_len);

  const T* urow = static_cast<const T*>(p.u) + int64_t(b) * p.u_sb + int64_t(dc) * p.u_sd;
  const T* dlrow = static_cast<const T*>(p.delta) + int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
  const T* zrow = HAS_Z ? static_cast<const T*>(p.z) + int64_t(b) * p.z_sb + int64_t(dc) * p.z_sd : nullptr;
  T* orow = static_cast<T*>(p.out) + int64_t(b) * p.o_sb + int64_t(dc) * p.o_sd;

  const float bias = p.bias ? p.bias[int64_t(dc) * p.bias_s] : 0.0f;
  const float Dd = p.Dskip ? p.Dskip[int64_t(dc) * p.D_s] : 0.0f;
  const float* Ar = p.A + int64_t(dc) * p.A_sd;
  f2_t A2p[8];
  bool st = true;
  const float A0 = Ar[0];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float lo = Ar[int64_t(2 * k) * p.A_sn], hi = Ar[int64_t(2 * k + 1) * p.A_sn];
    st = st && (lo == float(2 * k + 1) * A0) && (hi == float(2 * k + 2) * A0);
    A2p[k] = f2(lo * kLog2e, hi * kLog2e);
  }
  const bool structured = __syncthreads_and(st) && !p.force_general;
  const float a2_0 = A0 * kLog2e;

  f2_t h2[8];
  if (seg > 0) {
    const int64_t rowg = int64_t(tile) * kRows + tid;
    const float4* src = reinterpret_cast<const float4*>(p.ws_H + (int64_t(seg - 1) * p.Bt * p.tiles_per_batch * kRows + rowg) * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldcg(src + i);
      h2[2 * i] = f2(v.x, v.y);
      h2[2 * i + 1] = f2(v.z, v.w);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) h2[k] = 0ull;
  }

  if (structured)
    forward_chunk<T, HAS_Z, SOFTPLUS, true>(p, bc_s, b, t0, t1, urow, dlrow, zrow, orow, row_ok,
                                            bias, Dd, a2_0, A2p, h2);
  else
    forward_chunk<T, HAS_Z, SOFTPLUS, false>(p, bc_s, b, t0, t1, urow, dlrow, zrow, orow, row_ok,
                                             bias, Dd, a2_0, A2p, h2);

  if (seg == p.nseg - 1 && row_ok && p.last_state) {
    float* dst = p.last_state + int64_t(b) * p.ls_sb + int64_t(d) * p.ls_sd;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float lo, hi;
      f2split(h2[k], lo, hi);
      dst[2 * k] = lo;
      dst[2 * k + 1] = hi;
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 1: chunk summaries (S, H) by a backward sweep, then the carry fold.
//   H_n = sum_s delta_s u_s B_sn exp(A_n sum_{s<r<=end} delta_r),  S = sum_s delta_s
// ---------------------------------------------------------------------------
template <typename T, bool SOFTPLUS, bool STRUCT>
__device__ __forceinline__ void backward_chunk(const ScanArgs& p, float (*bc_s)[kTC * 32], int b,
                                               int t0, int t1, const T* urow, const T* dlrow,
                                               float bias, float a2_0, const f2_t (&A2p)[8],
                                               f2_t (&H2)[8], float& S) {
  constexpr int SB = Blk<T>::kSteps;
  const bool vec = p.vec_rows != 0;
  BCStage<T, 32> stage;  // rows 16..31 (C) are staged but unused here
  const int nchunks = (t1 - t0) / kTC;  // chunks of kernel 1 are always full
  float Tacc = 0.0f;                    // sum of delta over steps after the current one
  stage.load(p, b, t0 + (nchunks - 1) * kTC, t1);
  stage.store(bc_s[0]);
  __syncthreads();
  Blk<T> cu, cd;
  {
    const int tl = t1 - SB;
    cu.load(urow, tl, t1, vec);
    cd.load(dlrow, tl, t1, vec);
  }
  for (int ci = 0; ci < nchunks; ++ci) {
    const int c = nchunks - 1 - ci;
    const int cs = t0 + c * kTC;
    if (c > 0) stage.load(p, b, cs - kTC, t1);
    const float* bcb = bc_s[ci & 1];
    for (int tb = cs + kTC - SB; tb >= cs; tb -= SB) {
      Blk<T> nu, nd;
      const int tn = tb - SB;
      if (tn >= t0) {
        nu.load(urow, tn, t1, vec);
        nd.load(dlrow, tn, t1, vec);
      } else {
        nu.zero();
        nd.zero();
      }
#pragma unroll
      for (int jj = 0; jj < SB; ++jj) {
        const int j = SB - 1 - jj;
        float dt = cd.at(j) + bias;
        if constexpr (SOFTPLUS) dt = softplus_f(dt);
        const float w = dt * cu.at(j);
        const ulonglong2* q = reinterpret_cast<const ulonglong2*>(bcb + (tb + j - cs) * 32);
        f2_t v[8];
        if constexpr (STRUCT) {
          const float pi = ex2f(a2_0 * Tacc);   // prod_{r>t} A_bar_r,0
          const float pi2 = pi * pi;
          v[0] = mul2(f2(w, w), f2(pi, pi2));   // (w pi, w pi^2)
          const f2_t s2 = f2(pi2, pi2);
#pragma unroll
          for (int k = 1; k < 8; ++k) v[k] = mul2(v[k - 1], s2);
        } else {
          const f2_t T2 = f2(Tacc, Tacc);
          const f2_t w2 = f2(w, w);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float lo, hi;
            f2split(mul2(T2, A2p[k]), lo, hi);
            v[k] = mul2(w2, f2(ex2f(lo), ex2f(hi)));
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const ulonglong2 bb = q[k];
          H2[2 * k] = fma2(v[2 * k], bb.x, H2[2 * k]);
          H2[2 * k + 1] = fma2(v[2 * k + 1], bb.y, H2[2 * k + 1]);
        }
        Tacc += dt;
      }
      cu = nu;
      cd = nd;
    }
    if (c > 0) stage.store(bc_s[(ci + 1) & 1]);
    __syncthreads();
  }
  S = Tacc;
}

template <typename T, bool SOFTPLUS>
__global__ void __launch_bounds__(kRows) scan_chunk_state_kernel(const ScanArgs p) {
  __shared__ __align__(16) float bc_s[2][kTC * 32];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int seg = blockIdx.y;  // 0 .. nseg-2
  const int b = tile / p.tiles_per_batch;
  const int d = (tile - b * p.tiles_per_batch) * kRows + tid;
  const int dc = d < p.D ? d : p.D - 1;
  const int t0 = seg * p.seg_len;
  const int t1 = t0 + p.seg_len;

  const T* urow = static_cast<const T*>(p.u) + int64_t(b) * p.u_sb + int64_t(dc) * p.u_sd;
  const T* dlrow = static_cast<const T*>(p.delta) + int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
  const float bias = p.bias ? p.bias[int64_t(dc) * p.bias_s] : 0.0f;
  const float* Ar = p.A + int64_t(dc) * p.A_sd;
  f2_t A2p[8];
  bool st = true;
  const float A0 = Ar[0];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float lo = Ar[int64_t(2 * k) * p.A_sn], hi = Ar[int64_t(2 * k + 1) * p.A_sn];
    st = st && (lo == float(2 * k + 1) * A0) && (hi == float(2 * k + 2) * A0);
    A2p[k] = f2(lo * kLog2e, hi * kLog2e);
  }
  const bool structured = __syncthreads_and(st) && !p.force_general;
  const float a2_0 = A0 * kLog2e;

  f2_t H2[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) H2[k] = 0ull;
  float S = 0.0f;
  if (structured)
    backward_chunk<T, SOFTPLUS, true>(p, bc_s, b, t0, t1, urow, dlrow, bias, a2_0, A2p, H2, S);
  else
    backward_chunk<T, SOFTPLUS, false>(p, bc_s, b, t0, t1, urow, dlrow, bias, a2_0, A2p, H2, S);

  const int64_t rows_total = int64_t(p.Bt) * p.tiles_per_batch * kRows;
  const int64_t rowg = int64_t(tile) * kRows + tid;
  {
    float4* dst = reinterpret_cast<float4*>(p.ws_H + (int64_t(seg) * rows_total + rowg) * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a, bq, c, dd;
      f2split(H2[2 * i], a, bq);
      f2split(H2[2 * i + 1], c, dd);
      __stcg(dst + i, make_float4(a, bq, c, dd));
    }
    __stcg(p.ws_S + int64_t(seg) * rows_total + rowg, S);
  }

  // The last kernel-1 CTA of this row tile folds the chunk summaries, in chunk
  // order, into carried states: prefix_k = exp(A S_k) prefix_(k-1) + H_k, stored
  // over H_k.  Nobody waits: the fold runs in whichever CTA arrives last.
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.ws_count[tile], 1u) == unsigned(p.nseg - 2));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  f2_t h[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) h[k] = 0ull;
  for (int k = 0; k < p.nseg - 1; ++k) {
    float4* rec = reinterpret_cast<float4*>(p.ws_H + (int64_t(k) * rows_total + rowg) * kN);
    const float Sk = __ldcg(p.ws_S + int64_t(k) * rows_total + rowg);
    const f2_t S2 = f2(Sk, Sk);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldcg(rec + i);
      float e0, e1, e2, e3;
      f2split(mul2(S2, A2p[2 * i]), e0, e1);
      f2split(mul2(S2, A2p[2 * i + 1]), e2, e3);
      h[2 * i] = fma2(f2(ex2f(e0), ex2f(e1)), h[2 * i], f2(v.x, v.y));
      h[2 * i + 1] = fma2(f2(ex2f(e2), ex2f(e3)), h[2 * i + 1], f2(v.z, v.w));
      float a, bq, c, dd;
      f2split(h[2 * i], a, bq);
      f2split(h[2 * i + 1], c, dd);
      __stcg(rec + i, make_float4(a, bq, c, dd));
    }
  }
  if (tid == 0) p.ws_count[tile] = 0u;
}

}  // namespace mssm
