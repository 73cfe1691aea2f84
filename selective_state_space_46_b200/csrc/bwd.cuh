// Backward of the selective scan (Euler discretisation, zero initial state), sm_100a.
//
// The forward per row (b, d) and state n is h_t = a_t h_(t-1) + dt_t B_t u_t with
// a_t = exp(dt_t A_n), y_t = C_t . h_t + D u_t, out_t = y_t silu(z_t).  Its reverse-mode
// chain rule runs from the last step to the first with g = dLoss/dh_t:
//   gy = dout silu(z);  g += gy C_t;  dC_t += gy h_t;  ddt += g (A a h_(t-1) + B_t u_t);
//   dA += g dt a h_(t-1);  dB_t += g dt u;  du += g dt B_t (+ gy D);  g *= a.
// The fused forward never stores the states, so the backward recomputes them
// ("Mamba selective state space", the hardware-aware scan: intermediates are
// recomputed in the backward pass instead of being written).
//
// Two chunk-parallel passes over chunks of kBwdChunk steps (kBwdChunkShort when there are
// many row tiles), one thread per row:
//  A. scan_bwd_summary_kernel: one backward sweep over every chunk gives its forward
//     summary H_c (the state it leaves from a zero start), its reverse summary G_c
//     (the gradient it sends to the chunk before from a zero incoming gradient) and
//     S_c (its summed step); the last CTA of a row tile folds them forwards into
//     every chunk's start state and backwards, Q_(c-1) = exp(A S_c) Q_c + G_c, into
//     every chunk's incoming gradient Q_c;
//  B. scan_bwd_kernel: every chunk recomputes its states forward from its start
//     state, window by window (the states after a window's even steps held in
//     registers, the windows' start states in shared memory),
//     and sweeps them backwards from Q_c, writing du, ddelta, dz and accumulating
//     dA, dD, dbias (per row, then one atomic add per CTA) and dB, dC (a
//     transpose-reduction over the warp's 32 rows through shared memory, then one
//     atomic add per lane and step).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace mssm {

constexpr int kBwdChunk = 64;       // steps per chunk
constexpr int kBwdChunkShort = 32;  // steps per chunk when there are many row tiles
constexpr int kBwdShortChunkTiles = 1024;  // from this many row tiles on, 32-step chunks
constexpr int kBwdRows = 32;   // rows per CTA (one warp)

struct BwdArgs {
  const void* u;
  const void* delta;
  const void* z;
  const void* dout;
  int64_t u_sb, u_sd, dl_sb, dl_sd, z_sb, z_sd, g_sb, g_sd;  // L stride 1
  const void* B;
  const void* C;
  int64_t B_sb, B_sn, C_sb, C_sn;  // L stride 1
  const float* A;
  int64_t A_sd, A_sn;
  const float* Dskip;
  int64_t D_s;
  const float* bias;
  int64_t bias_s;
  void* du;
  void* ddelta;
  void* dz;
  int64_t du_sb, du_sd, dd_sb, dd_sd, dz_sb, dz_sd;
  float* dA;  // [D, N] contiguous, accumulated
  float* dB;  // [Bt, N, L] contiguous, accumulated
  float* dC;
  float* dD;     // [D], accumulated, or null
  float* dbias;  // [D], accumulated, or null
  int Bt, D, L;
  int softplus;
  int nseg, tiles_per_batch;
  int chunk;          // steps per chunk: kBwdChunk or kBwdChunkShort
  int vec_rows;       // u, delta, dout, z, du, ddelta, dz rows start 16-byte aligned
  int force_general;  // never take the structured-A powers
  float* hstart;    // [nseg-1][rows][16]: chunk k's summary H_k, then (folded) chunk k+1's start state
  float* ws_G;      // [nseg][rows][16]: outgoing gradient summary G_c of chunk c
  float* ws_S;      // [nseg][rows]: summed step S_c of chunk c
  float* ws_Q;      // [nseg][rows][16]: incoming gradient of chunk c (the fold)
  unsigned* ws_count;  // [tiles]: pass A arrivals, reset by the folding CTA
};

// dt of one step: softplus(delta + bias) or delta + bias; also sigmoid(delta + bias), the
// derivative of softplus (1 without softplus)
__device__ __forceinline__ float bwd_dt(float raw, float bias, bool softplus, float& dsp) {
  const float v = raw + bias;
  if (!softplus) {
    dsp = 1.0f;
    return v;
  }
  const float e = ex2f(-v * kLog2e);
  dsp = rcpf(1.0f + e);  // sigmoid(v)
  return softplus_f(v);
}

// silu(z) and its derivative sigma(z) (1 + z (1 - sigma(z)))
__device__ __forceinline__ void bwd_silu(float z, float& s, float& ds) {
  const float sg = rcpf(1.0f + ex2f(-z * kLog2e));
  s = z * sg;
  ds = sg * fmaf(z, 1.0f - sg, 1.0f);
}

// Row constants: A as packed pairs (natural units, and times log2 e), skip, bias, and
// whether A is structured, A_n = (n + 1) A_0 exactly.
struct BwdRow {
  f2_t A[kN / 2], A2[kN / 2];
  float A2_0;  // A_0 log2 e
  float Dd, bias;
  bool structured;
};
__device__ __forceinline__ void bwd_row(const BwdArgs& p, int d, BwdRow& r) {
  float a[kN];
#pragma unroll
  for (int n = 0; n < kN; ++n) a[n] = p.A[int64_t(d) * p.A_sd + int64_t(n) * p.A_sn];
  r.structured = true;
#pragma unroll
  for (int n = 1; n < kN; ++n) r.structured = r.structured && (a[n] == float(n + 1) * a[0]);
#pragma unroll
  for (int k = 0; k < kN / 2; ++k) {
    r.A[k] = f2(a[2 * k], a[2 * k + 1]);
    r.A2[k] = f2(a[2 * k] * kLog2e, a[2 * k + 1] * kLog2e);
  }
  r.A2_0 = a[0] * kLog2e;
  r.Dd = p.Dskip ? p.Dskip[int64_t(d) * p.D_s] : 0.0f;
  r.bias = p.bias ? p.bias[int64_t(d) * p.bias_s] : 0.0f;
}

// B and C of steps [t0, t0 + CHUNK) of batch b into shared memory, fp32 [t][32]
// (B in 0..15, C in 16..31); zero past L.  Each of the 32 threads loads one row of B or C,
// as 16-byte blocks where the row's chunk is whole and aligned.
template <typename T, int CHUNK>
__device__ __forceinline__ void bwd_stage_bc(const BwdArgs& p, int b, int t0, float (*bc)[32]) {
  const int r = threadIdx.x;
  const T* base = r < 16 ? static_cast<const T*>(p.B) + int64_t(b) * p.B_sb + int64_t(r) * p.B_sn
                         : static_cast<const T*>(p.C) + int64_t(b) * p.C_sb + int64_t(r - 16) * p.C_sn;
  constexpr int kPer = 16 / int(sizeof(T));  // elements per 16-byte block
  if (t0 + CHUNK <= p.L && (reinterpret_cast<uintptr_t>(base + t0) & 15) == 0) {
    const uint4* src = reinterpret_cast<const uint4*>(base + t0);
    uint4 v[CHUNK / kPer];
#pragma unroll
    for (int i = 0; i < CHUNK / kPer; ++i) v[i] = __ldg(src + i);
#pragma unroll
    for (int i = 0; i < CHUNK / kPer; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          bc[i * 8 + 2 * e][r] = bf16lo(w[e]);
          bc[i * 8 + 2 * e + 1][r] = bf16hi(w[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) bc[i * 4 + e][r] = __uint_as_float(w[e]);
      }
    }
    return;
  }
  for (int j = 0; j < CHUNK; ++j) {
    const int t = t0 + j;
    bc[j][r] = t < p.L ? Elem<T>::load(base + t) : 0.0f;
  }
}

// Reduce 32 per-lane quantities v[0..31] over the warp through a 4 KB shared buffer
// s[32][32]: lane i writes v[q] to s[q][i] (one bank per lane), then sums row i with
// eight 16-byte loads, taken in the order chunk ^ (i % 8) so that the eight lanes of a
// quarter-warp read eight different chunks, and packed adds.  Lane i returns the sum of
// v[i] over all lanes.  The buffer must be free on entry; it is free again on return.
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32], float* s) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int q = 0; q < 32; ++q) s[q * 32 + lane] = v[q];
  __syncwarp();
  const ulonglong2* row = reinterpret_cast<const ulonglong2*>(s + lane * 32);
  f2_t acc[4];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const ulonglong2 x = row[c ^ (lane & 7)];
    if (c < 2) {
      acc[2 * c] = x.x;
      acc[2 * c + 1] = x.y;
    } else {
      acc[2 * (c & 1)] = add2(acc[2 * (c & 1)], x.x);
      acc[2 * (c & 1) + 1] = add2(acc[2 * (c & 1) + 1], x.y);
    }
  }
  __syncwarp();
  float lo, hi;
  f2split(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), lo, hi);
  return lo + hi;
}

// ---------------------------------------------------------------------------
// pass B: recompute the chunk's states and sweep them backwards.  The chunk is
// walked in windows of kBwdWin steps: a first forward sweep leaves each window's
// start state in shared memory (2 KB per window for the warp); then, window by
// window from the last, the window's states are recomputed into registers and
// swept backwards.  The window's inputs are read once, as 16-byte blocks where the
// rows allow.
// ---------------------------------------------------------------------------
constexpr int kBwdWin = 8;

// steps [t, t + kBwdWin) of a row (zero past t_end)
template <typename T>
__device__ __forceinline__ void bwd_load_win(const void* base, int64_t off, int t, int t_end, bool vec,
                                             float (&v)[kBwdWin]) {
  const T* row = static_cast<const T*>(base) + off;
  if (vec && t + kBwdWin <= t_end) {
    if constexpr (sizeof(T) == 2) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + t));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16lo(ws[i]);
        v[2 * i + 1] = bf16hi(ws[i]);
      }
    } else {
      const float4 a = __ldg(reinterpret_cast<const float4*>(row + t));
      const float4 b = __ldg(reinterpret_cast<const float4*>(row + t) + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kBwdWin; ++j) v[j] = t + j < t_end ? Elem<T>::load(row + t + j) : 0.0f;
  }
}

// A window's raw 16-byte blocks of one row (kBwdWin steps), fetched ahead of their use.
template <typename T>
struct WinBuf {
  uint4 q[kBwdWin * sizeof(T) / 16];
};

template <typename T>
__device__ __forceinline__ void bwd_fetch_win(const void* base, int64_t off, int t, int t_end, bool vec,
                                              WinBuf<T>& wb) {
  if (vec && t + kBwdWin <= t_end) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(base) + off + t);
#pragma unroll
    for (int i = 0; i < int(kBwdWin * sizeof(T) / 16); ++i) wb.q[i] = __ldg(src + i);
  }
}

// the window's values from its fetched blocks (or, for a partial window or an unaligned row,
// by plain loads now)
template <typename T>
__device__ __forceinline__ void bwd_unpack_win(const void* base, int64_t off, int t, int t_end, bool vec,
                                               const WinBuf<T>& wb, float (&v)[kBwdWin]) {
  if (vec && t + kBwdWin <= t_end) {
    if constexpr (sizeof(T) == 2) {
      const uint32_t ws[4] = {wb.q[0].x, wb.q[0].y, wb.q[0].z, wb.q[0].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16lo(ws[i]);
        v[2 * i + 1] = bf16hi(ws[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        v[4 * i] = __uint_as_float(wb.q[i].x);
        v[4 * i + 1] = __uint_as_float(wb.q[i].y);
        v[4 * i + 2] = __uint_as_float(wb.q[i].z);
        v[4 * i + 3] = __uint_as_float(wb.q[i].w);
      }
    }
  } else {
    const T* row = static_cast<const T*>(base) + off;
#pragma unroll
    for (int j = 0; j < kBwdWin; ++j) v[j] = t + j < t_end ? Elem<T>::load(row + t + j) : 0.0f;
  }
}

// steps [t, t + kBwdWin) of an output row, clipped at t_end
template <typename T>
__device__ __forceinline__ void bwd_store_win(void* base, int64_t off, int t, int t_end, bool vec,
                                              const float (&v)[kBwdWin]) {
  T* row = static_cast<T*>(base) + off;
  if (vec && t + kBwdWin <= t_end) {
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<uint4*>(row + t) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                      pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    } else {
      reinterpret_cast<float4*>(row + t)[0] = make_float4(v[0], v[1], v[2], v[3]);
      reinterpret_cast<float4*>(row + t)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < kBwdWin; ++j) {
      if (t + j < t_end) {
        if constexpr (sizeof(T) == 2) {
          row[t + j] = f_to_bf16(v[j]);
        } else {
          row[t + j] = v[j];
        }
      }
    }
  }
}

// a_n = exp(dt A_n) for the 16 states as 8 pairs (a_2k, a_2k+1).  Structured A: the
// powers x^1 .. x^16 of x = exp(dt A_0) by a tree of depth 4 (x^2, x^4, x^8 broadcast
// over the pairs); otherwise one SFU exponential per state.
template <bool STRUCT>
__device__ __forceinline__ void bwd_decay(float dt, const BwdRow& r, f2_t (&a)[kN / 2]) {
  if constexpr (STRUCT) {
    const float x1 = ex2f(dt * r.A2_0);
    const float x2 = x1 * x1, x4 = x2 * x2, x8 = x4 * x4;
    a[0] = f2(x1, x2);
    a[1] = mul2(a[0], f2(x2, x2));
    const f2_t q4 = f2(x4, x4);
    a[2] = mul2(a[0], q4);
    a[3] = mul2(a[1], q4);
    const f2_t q8 = f2(x8, x8);
#pragma unroll
    for (int k = 0; k < 4; ++k) a[4 + k] = mul2(a[k], q8);
  } else {
    const f2_t d2 = f2(dt, dt);
#pragma unroll
    for (int k = 0; k < kN / 2; ++k) {
      float lo, hi;
      f2split(mul2(d2, r.A2[k]), lo, hi);
      a[k] = f2(ex2f(lo), ex2f(hi));
    }
  }
}

// ---------------------------------------------------------------------------
// pass A: one backward sweep over chunk c gives both of its summaries, sharing the
// step's dt and decay powers: the forward one, H_c = sum_t (prod_(s>t) a_s) dt_t u_t B_t
// (the state the chunk leaves from a zero start, accumulated with the running product
// P of the later steps' decays), and the reverse one, G_c (the gradient the chunk sends
// to the one before from a zero incoming gradient: g = a (g + gy C) from the last step
// to the first), plus S_c = sum_t dt_t.  The last CTA of a row tile to arrive folds
// them: forwards, start_(c+1) = exp(A S_c) start_c + H_c from start_0 = 0, and
// backwards, Q_(c-1) = exp(A S_c) Q_c + G_c from Q_(nseg-1) = 0.  Windows of kBwdWin
// steps, 16-byte loads of u, delta, dout and z where the rows allow, the 16 states as 8
// packed pairs.
// ---------------------------------------------------------------------------
template <typename T, bool HAS_Z, bool STRUCT>
__device__ __forceinline__ void bwd_summary_chunk(const BwdArgs& p, const BwdRow& r, const float (*bc)[32], int b,
                                                  int dc, int t0, int t1, f2_t (&H)[kN / 2], f2_t (&g2)[kN / 2],
                                                  float& ssum) {
  const int64_t uo = int64_t(b) * p.u_sb + int64_t(dc) * p.u_sd;
  const int64_t ro = int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
  const int64_t go = int64_t(b) * p.g_sb + int64_t(dc) * p.g_sd;
  const int64_t zo = int64_t(b) * p.z_sb + int64_t(dc) * p.z_sd;
  const bool vin = p.vec_rows != 0;
  f2_t P[kN / 2];
#pragma unroll
  for (int k = 0; k < kN / 2; ++k) P[k] = f2(1.0f, 1.0f);
  const int nwin = (t1 - t0 + kBwdWin - 1) / kBwdWin;
  // the inputs of window w are fetched while window w + 1 is swept
  WinBuf<T> nu, nd, ng, nz;
  {
    const int tw = t0 + (nwin - 1) * kBwdWin;
    bwd_fetch_win<T>(p.u, uo, tw, t1, vin, nu);
    bwd_fetch_win<T>(p.delta, ro, tw, t1, vin, nd);
    bwd_fetch_win<T>(p.dout, go, tw, t1, vin, ng);
    if constexpr (HAS_Z) bwd_fetch_win<T>(p.z, zo, tw, t1, vin, nz);
  }
  for (int w = nwin - 1; w >= 0; --w) {
    const int tw = t0 + w * kBwdWin;
    const WinBuf<T> cu = nu, cd = nd, cg = ng, cz = nz;
    if (w > 0) {
      bwd_fetch_win<T>(p.u, uo, tw - kBwdWin, t1, vin, nu);
      bwd_fetch_win<T>(p.delta, ro, tw - kBwdWin, t1, vin, nd);
      bwd_fetch_win<T>(p.dout, go, tw - kBwdWin, t1, vin, ng);
      if constexpr (HAS_Z) bwd_fetch_win<T>(p.z, zo, tw - kBwdWin, t1, vin, nz);
    }
    float uu[kBwdWin], dl[kBwdWin], gd[kBwdWin], zz[kBwdWin];
    bwd_unpack_win<T>(p.u, uo, tw, t1, vin, cu, uu);
    bwd_unpack_win<T>(p.delta, ro, tw, t1, vin, cd, dl);
    bwd_unpack_win<T>(p.dout, go, tw, t1, vin, cg, gd);
    if constexpr (HAS_Z) bwd_unpack_win<T>(p.z, zo, tw, t1, vin, cz, zz);
#pragma unroll
    for (int j = kBwdWin - 1; j >= 0; --j) {
      if (tw + j >= t1) continue;  // past the end of the sequence (a partial last window)
      float dsp;  // unused here
      const float dt = bwd_dt(dl[j], r.bias, p.softplus, dsp);
      float gy = gd[j];
      if constexpr (HAS_Z) {
        float sv, ds;
        bwd_silu(zz[j], sv, ds);
        gy *= sv;
      }
      f2_t a[kN / 2];
      bwd_decay<STRUCT>(dt, r, a);
      const f2_t gy2 = f2(gy, gy), w2 = f2(dt * uu[j], dt * uu[j]);
      const ulonglong2* q = reinterpret_cast<const ulonglong2*>(bc[tw - t0 + j]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const ulonglong2 bb = q[k], cc = q[4 + k];  // B and C pairs (4k, 4k+1), (4k+2, 4k+3)
        H[2 * k] = fma2(P[2 * k], mul2(w2, bb.x), H[2 * k]);
        H[2 * k + 1] = fma2(P[2 * k + 1], mul2(w2, bb.y), H[2 * k + 1]);
        P[2 * k] = mul2(P[2 * k], a[2 * k]);
        P[2 * k + 1] = mul2(P[2 * k + 1], a[2 * k + 1]);
        g2[2 * k] = mul2(a[2 * k], fma2(gy2, cc.x, g2[2 * k]));
        g2[2 * k + 1] = mul2(a[2 * k + 1], fma2(gy2, cc.y, g2[2 * k + 1]));
      }
      ssum += dt;
    }
  }
}

__device__ __forceinline__ void bwd_store16(float* dst, const f2_t (&v)[kN / 2]) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float x0, x1, x2, x3;
    f2split(v[2 * i], x0, x1);
    f2split(v[2 * i + 1], x2, x3);
    __stcg(d4 + i, make_float4(x0, x1, x2, x3));
  }
}

__device__ __forceinline__ void bwd_load16(const float* src, float4 (&v)[4]) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __ldcg(s4 + i);
}

template <typename T, bool HAS_Z, int CHUNK>
__global__ void __launch_bounds__(kBwdRows) scan_bwd_summary_kernel(const BwdArgs p) {
  __shared__ __align__(16) float bc_s[CHUNK][32];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int c = blockIdx.y;
  const int b = tile / p.tiles_per_batch;
  const int d = (tile - b * p.tiles_per_batch) * kBwdRows + tid;
  const int dc = d < p.D ? d : p.D - 1;
  const int t0 = c * CHUNK;
  const int t1 = min(p.L, t0 + CHUNK);
  BwdRow r;
  bwd_row(p, dc, r);
  const bool structured = __syncthreads_and(r.structured) && !p.force_general;
  bwd_stage_bc<T, CHUNK>(p, b, t0, bc_s);
  __syncthreads();

  f2_t H[kN / 2], g2[kN / 2];
#pragma unroll
  for (int k = 0; k < kN / 2; ++k) H[k] = g2[k] = f2(0.0f, 0.0f);
  float ssum = 0.0f;
  if (structured)
    bwd_summary_chunk<T, HAS_Z, true>(p, r, bc_s, b, dc, t0, t1, H, g2, ssum);
  else
    bwd_summary_chunk<T, HAS_Z, false>(p, r, bc_s, b, dc, t0, t1, H, g2, ssum);
  const int64_t rows_total = int64_t(p.Bt) * p.tiles_per_batch * kBwdRows;
  const int64_t rowg = int64_t(tile) * kBwdRows + tid;
  // the first chunk sends no gradient back, and the last one's end state starts nothing
  if (c + 1 < p.nseg) bwd_store16(p.hstart + (int64_t(c) * rows_total + rowg) * kN, H);
  if (c > 0) bwd_store16(p.ws_G + (int64_t(c) * rows_total + rowg) * kN, g2);
  __stcg(p.ws_S + int64_t(c) * rows_total + rowg, ssum);

  // the last CTA of the row tile to arrive folds both ways
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.ws_count[tile], 1u) == unsigned(p.nseg - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  auto decay_of = [&](float sk, f2_t (&a)[kN / 2]) {
    if (structured)
      bwd_decay<true>(sk, r, a);
    else
      bwd_decay<false>(sk, r, a);
  };
  // forwards: hstart[k] (the start state of chunk k + 1) = exp(A S_k) hstart[k - 1] + H_k, in place
  {
    f2_t h[kN / 2];
#pragma unroll
    for (int k = 0; k < kN / 2; ++k) h[k] = f2(0.0f, 0.0f);
    float s_cur = __ldcg(p.ws_S + rowg);
    float4 h_cur[4];
    bwd_load16(p.hstart + rowg * kN, h_cur);
    for (int k = 0; k + 1 < p.nseg; ++k) {
      float s_nx = 0.0f;
      float4 h_nx[4] = {};
      if (k + 2 < p.nseg) {  // the next chunk's summary, fetched while this one is applied
        s_nx = __ldcg(p.ws_S + int64_t(k + 1) * rows_total + rowg);
        bwd_load16(p.hstart + (int64_t(k + 1) * rows_total + rowg) * kN, h_nx);
      }
      f2_t a[kN / 2];
      decay_of(s_cur, a);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        h[2 * i] = fma2(a[2 * i], h[2 * i], f2(h_cur[i].x, h_cur[i].y));
        h[2 * i + 1] = fma2(a[2 * i + 1], h[2 * i + 1], f2(h_cur[i].z, h_cur[i].w));
      }
      bwd_store16(p.hstart + (int64_t(k) * rows_total + rowg) * kN, h);
      s_cur = s_nx;
#pragma unroll
      for (int i = 0; i < 4; ++i) h_cur[i] = h_nx[i];
    }
  }
  // backwards: Q_(nseg-1) = 0, Q_(k-1) = exp(A S_k) Q_k + G_k
  {
    f2_t q[kN / 2];
#pragma unroll
    for (int k = 0; k < kN / 2; ++k) q[k] = f2(0.0f, 0.0f);
    float s_cur = __ldcg(p.ws_S + int64_t(p.nseg - 1) * rows_total + rowg);
    float4 g_cur[4];
    bwd_load16(p.ws_G + (int64_t(p.nseg - 1) * rows_total + rowg) * kN, g_cur);
    for (int k = p.nseg - 1; k >= 0; --k) {
      bwd_store16(p.ws_Q + (int64_t(k) * rows_total + rowg) * kN, q);
      if (k == 0) break;
      float s_nx = 0.0f;
      float4 g_nx[4] = {};
      if (k > 1) {
        s_nx = __ldcg(p.ws_S + int64_t(k - 1) * rows_total + rowg);
        bwd_load16(p.ws_G + (int64_t(k - 1) * rows_total + rowg) * kN, g_nx);
      }
      f2_t a[kN / 2];
      decay_of(s_cur, a);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        q[2 * i] = fma2(a[2 * i], q[2 * i], f2(g_cur[i].x, g_cur[i].y));
        q[2 * i + 1] = fma2(a[2 * i + 1], q[2 * i + 1], f2(g_cur[i].z, g_cur[i].w));
      }
      s_cur = s_nx;
#pragma unroll
      for (int i = 0; i < 4; ++i) g_cur[i] = g_nx[i];
    }
  }
  if (tid == 0) p.ws_count[tile] = 0u;
}

// One step of the states' forward recurrence on the 8 pairs: h = a h + (dt u) B.
__device__ __forceinline__ void bwd_fwd_step(const f2_t (&a)[kN / 2], float wv, const float* bcrow,
                                             const f2_t (&hin)[kN / 2], f2_t (&hout)[kN / 2]) {
  const f2_t w2 = f2(wv, wv);
  const ulonglong2* q = reinterpret_cast<const ulonglong2*>(bcrow);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const ulonglong2 bb = q[k];  // B pairs (4k, 4k+1), (4k+2, 4k+3)
    hout[2 * k] = fma2(a[2 * k], hin[2 * k], mul2(w2, bb.x));
    hout[2 * k + 1] = fma2(a[2 * k + 1], hin[2 * k + 1], mul2(w2, bb.y));
  }
}

// The backward sweep of one chunk.  Registers hold a window's states after its even steps
// only (he[i] = h after 2i of its steps, he[0] its start); the chain rule needs, at step
// j, the state after the step (h_post) and a_j h_pre, which is h_post - (dt u)_j B_j, so
// a state after an odd step is never needed before the step itself recomputes it.  The
// window start states live in shared memory, [window][pair][lane] (2 KB per window).
template <typename T, bool HAS_Z, bool STRUCT>
__device__ __forceinline__ void bwd_chunk(const BwdArgs& p, const BwdRow& r, const float (*bc)[32],
                                          f2_t (*hwin)[kN / 2][kBwdRows], int b, bool row_ok, int dc, int t0, int t1,
                                          f2_t (&h)[kN / 2], f2_t (&g)[kN / 2], f2_t (&dA)[kN / 2],
                                          float& dDacc, float& dbacc) {
  const int tid = threadIdx.x;
  const int64_t uo = int64_t(b) * p.u_sb + int64_t(dc) * p.u_sd;
  const int64_t ro = int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
  const int64_t go = int64_t(b) * p.g_sb + int64_t(dc) * p.g_sd;
  const int64_t zo = int64_t(b) * p.z_sb + int64_t(dc) * p.z_sd;
  const int64_t duo = int64_t(b) * p.du_sb + int64_t(dc) * p.du_sd;
  const int64_t ddo = int64_t(b) * p.dd_sb + int64_t(dc) * p.dd_sd;
  const int64_t dzo = int64_t(b) * p.dz_sb + int64_t(dc) * p.dz_sd;
  const bool vin = p.vec_rows != 0;
  const int nwin = (t1 - t0 + kBwdWin - 1) / kBwdWin;
  // forward: every window's start state but the last one's to the scratch; h ends as the
  // last window's start state
  for (int w = 0; w + 1 < nwin; ++w) {
#pragma unroll
    for (int k = 0; k < kN / 2; ++k) hwin[w][k][tid] = h[k];
    const int tw = t0 + w * kBwdWin;
    float uu[kBwdWin], dl[kBwdWin];
    bwd_load_win<T>(p.u, uo, tw, t1, vin, uu);
    bwd_load_win<T>(p.delta, ro, tw, t1, vin, dl);
#pragma unroll
    for (int j = 0; j < kBwdWin; ++j) {
      float dsp;  // unused here
      const float dt = bwd_dt(dl[j], r.bias, p.softplus, dsp);
      f2_t a[kN / 2];
      bwd_decay<STRUCT>(dt, r, a);
      bwd_fwd_step(a, dt * uu[j], bc[tw - t0 + j], h, h);
    }
  }
  // backward, window by window
  for (int w = nwin - 1; w >= 0; --w) {
    const int tw = t0 + w * kBwdWin;
    f2_t he[kBwdWin / 2 + 1][kN / 2];
    if (w + 1 == nwin) {
#pragma unroll
      for (int k = 0; k < kN / 2; ++k) he[0][k] = h[k];
    } else {
#pragma unroll
      for (int k = 0; k < kN / 2; ++k) he[0][k] = hwin[w][k][tid];
    }
    // slots w (just read, or never written for the last window) and w + 1 (read for the
    // window before) are free: the 4 KB buffer of the dB/dC reduction
    __syncwarp();
    float* red_s = reinterpret_cast<float*>(&hwin[w][0][0]);
    float uu[kBwdWin], dl[kBwdWin], go_[kBwdWin], zz[kBwdWin];
    bwd_load_win<T>(p.u, uo, tw, t1, vin, uu);
    bwd_load_win<T>(p.delta, ro, tw, t1, vin, dl);
    bwd_load_win<T>(p.dout, go, tw, t1, vin, go_);
    if constexpr (HAS_Z) bwd_load_win<T>(p.z, zo, tw, t1, vin, zz);
    // recompute the window's states; keep those after its even steps
    {
      f2_t odd[kN / 2];
#pragma unroll
      for (int j = 0; j < kBwdWin; ++j) {
        float dsp;  // unused here
        const float dt = bwd_dt(dl[j], r.bias, p.softplus, dsp);
        f2_t a[kN / 2];
        bwd_decay<STRUCT>(dt, r, a);
        if (j % 2 == 0)
          bwd_fwd_step(a, dt * uu[j], bc[tw - t0 + j], he[j / 2], odd);
        else
          bwd_fwd_step(a, dt * uu[j], bc[tw - t0 + j], odd, he[j / 2 + 1]);
      }
    }
    float du_w[kBwdWin], dd_w[kBwdWin], dz_w[kBwdWin];
#pragma unroll
    for (int j = kBwdWin - 1; j >= 0; --j) {
      const int t = tw + j;
      if (t >= t1) {  // past the end of the sequence (the last window may be partial)
        du_w[j] = 0.0f; dd_w[j] = 0.0f; dz_w[j] = 0.0f;
        continue;
      }
      float dsp;
      const float dt = bwd_dt(dl[j], r.bias, p.softplus, dsp);
      f2_t a[kN / 2];
      bwd_decay<STRUCT>(dt, r, a);
      // B pairs at q[0..3], C pairs at q[4..7], read where they are used
      const ulonglong2* q = reinterpret_cast<const ulonglong2*>(bc[t - t0]);
      const float wv = dt * uu[j];
      // post: the state after step j; ah: a_j times the state before it
      f2_t post[kN / 2], ah[kN / 2];
#pragma unroll
      for (int k = 0; k < kN / 2; ++k) {
        const ulonglong2 bb = q[k >> 1];
        const f2_t Bk = (k & 1) ? bb.y : bb.x;
        if (j % 2 == 0) {
          ah[k] = mul2(a[k], he[j / 2][k]);
          post[k] = fma2(f2(wv, wv), Bk, ah[k]);
        } else {
          post[k] = he[j / 2 + 1][k];
          ah[k] = fma2(f2(-wv, -wv), Bk, post[k]);
        }
      }
      float gy = go_[j];
      if constexpr (HAS_Z) {
        f2_t ya = f2(0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const ulonglong2 cc = q[4 + k];
          ya = fma2(cc.x, post[2 * k], ya);
          ya = fma2(cc.y, post[2 * k + 1], ya);
        }
        float y0, y1;
        f2split(ya, y0, y1);
        const float yv = fmaf(r.Dd, uu[j], y0 + y1);
        float sv, ds;
        bwd_silu(zz[j], sv, ds);
        dz_w[j] = go_[j] * yv * ds;
        gy = go_[j] * sv;
      }
      dDacc = fmaf(gy, uu[j], dDacc);
      // rows past D contribute nothing to the channel sums dB and dC
      const float gym = row_ok ? gy : 0.0f, um = row_ok ? uu[j] : 0.0f;
      const f2_t gy2 = f2(gy, gy), gym2 = f2(gym, gym), u2 = f2(uu[j], uu[j]), um2 = f2(um, um);
      const f2_t dt2 = f2(dt, dt);
      f2_t ddt2 = f2(0.0f, 0.0f), du2 = f2(0.0f, 0.0f);
      float red[32];  // dB (0..15) and dC (16..31) of this row and step
#pragma unroll
      for (int k = 0; k < kN / 2; ++k) {
        const ulonglong2 bb = q[k >> 1], cc = q[4 + (k >> 1)];
        const f2_t Bk = (k & 1) ? bb.y : bb.x, Ck = (k & 1) ? cc.y : cc.x;
        g[k] = fma2(gy2, Ck, g[k]);
        f2split(mul2(gym2, post[k]), red[16 + 2 * k], red[17 + 2 * k]);
        const f2_t gah = mul2(g[k], ah[k]);
        ddt2 = fma2(g[k], mul2(Bk, u2), fma2(r.A[k], gah, ddt2));
        dA[k] = fma2(gah, dt2, dA[k]);
        const f2_t gdt = mul2(g[k], dt2);
        f2split(mul2(gdt, um2), red[2 * k], red[2 * k + 1]);
        du2 = fma2(gdt, Bk, du2);
        g[k] = mul2(g[k], a[k]);
      }
      float t0v, t1v, u0v, u1v;
      f2split(ddt2, t0v, t1v);
      f2split(du2, u0v, u1v);
      const float draw = (t0v + t1v) * dsp;
      dbacc += draw;
      du_w[j] = fmaf(gy, r.Dd, u0v + u1v);
      dd_w[j] = draw;
      const float tot = warp_transpose_sum(red, red_s);
      float* dst = tid < 16 ? p.dB + (int64_t(b) * kN + tid) * p.L + t
                            : p.dC + (int64_t(b) * kN + (tid - 16)) * p.L + t;
      atomicAdd(dst, tot);
    }
    if (row_ok) {
      const bool vout = p.vec_rows != 0;
      bwd_store_win<T>(p.du, duo, tw, t1, vout, du_w);
      bwd_store_win<T>(p.ddelta, ddo, tw, t1, vout, dd_w);
      if constexpr (HAS_Z) bwd_store_win<T>(p.dz, dzo, tw, t1, vout, dz_w);
    }
  }
}

// pass B's register cap per thread, which sets its occupancy (one-warp CTAs, 65536 registers
// per SM)
#ifndef MSSM_BWD_MAXNREG
#define MSSM_BWD_MAXNREG 255
#endif
template <typename T, bool HAS_Z, int CHUNK>
__global__ void __maxnreg__(MSSM_BWD_MAXNREG) scan_bwd_kernel(const BwdArgs p) {
  __shared__ __align__(16) float bc_s[CHUNK][32];
  // window start states, and one spare slot so that two free slots always follow window w
  __shared__ __align__(16) f2_t hwin[CHUNK / kBwdWin + 1][kN / 2][kBwdRows];
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int c = blockIdx.y;
  const int b = tile / p.tiles_per_batch;
  const int d = (tile - b * p.tiles_per_batch) * kBwdRows + tid;
  const bool row_ok = d < p.D;
  const int dc = row_ok ? d : p.D - 1;
  const int t0 = c * CHUNK;
  const int t1 = min(p.L, t0 + CHUNK);
  const int64_t rows_total = int64_t(p.Bt) * p.tiles_per_batch * kBwdRows;
  const int64_t rowg = int64_t(tile) * kBwdRows + tid;
  BwdRow r;
  bwd_row(p, dc, r);
  const bool structured = __syncthreads_and(r.structured) && !p.force_general;
  bwd_stage_bc<T, CHUNK>(p, b, t0, bc_s);
  __syncthreads();

  f2_t h[kN / 2], g[kN / 2], dA[kN / 2];
  {
    const float4* hsrc = reinterpret_cast<const float4*>(p.hstart + (int64_t(c - 1) * rows_total + rowg) * kN);
    const float4* qsrc = reinterpret_cast<const float4*>(p.ws_Q + (int64_t(c) * rows_total + rowg) * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 hv = c > 0 ? __ldcg(hsrc + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 qv = c + 1 < p.nseg ? __ldcg(qsrc + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      h[2 * i] = f2(hv.x, hv.y); h[2 * i + 1] = f2(hv.z, hv.w);
      g[2 * i] = f2(qv.x, qv.y); g[2 * i + 1] = f2(qv.z, qv.w);
    }
  }
#pragma unroll
  for (int k = 0; k < kN / 2; ++k) dA[k] = f2(0.0f, 0.0f);
  float dDacc = 0.0f, dbacc = 0.0f;
  if (structured)
    bwd_chunk<T, HAS_Z, true>(p, r, bc_s, hwin, b, row_ok, dc, t0, t1, h, g, dA, dDacc, dbacc);
  else
    bwd_chunk<T, HAS_Z, false>(p, r, bc_s, hwin, b, row_ok, dc, t0, t1, h, g, dA, dDacc, dbacc);
  if (row_ok) {
#pragma unroll
    for (int k = 0; k < kN / 2; ++k) {
      float lo, hi;
      f2split(dA[k], lo, hi);
      atomicAdd(p.dA + int64_t(d) * kN + 2 * k, lo);
      atomicAdd(p.dA + int64_t(d) * kN + 2 * k + 1, hi);
    }
    if (p.dD) atomicAdd(p.dD + d, dDacc);
    if (p.dbias) atomicAdd(p.dbias + d, dbacc);
  }
}

}  // namespace mssm
