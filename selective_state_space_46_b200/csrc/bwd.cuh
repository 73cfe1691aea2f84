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
// Three chunk-parallel passes over chunks of kBwdChunk steps, one thread per row:
//  A. the forward chunk summaries and their fold (scan_chunk_state_kernel) give
//     every chunk's start state;
//  B. scan_bwd_summary_kernel: every chunk but the first runs the g recurrence
//     from a zero incoming gradient, giving G_c (what it sends to the chunk
//     before) and S_c (its summed step); the last CTA of a row tile folds them
//     backwards, Q_(c-1) = exp(A S_c) Q_c + G_c, into each chunk's incoming Q_c;
//  C. scan_bwd_kernel: every chunk recomputes its states forward from its start
//     state, window by window (kBwdWin steps held in registers, the windows' start
//     states in shared memory), and sweeps them backwards from Q_c, writing du,
//     ddelta, dz and accumulating dA, dD, dbias (per row, then one atomic add per
//     CTA) and dB, dC (a transpose-reduction over the warp's 32 rows through shared
//     memory, then one atomic add per lane and step).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace mssm {

constexpr int kBwdChunk = 64;  // steps per chunk (the forward summaries' quantum)
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
  int vec_rows;       // u, delta, dout, z, du, ddelta, dz rows start 16-byte aligned
  int force_general;  // never take the structured-A powers
  const float* hstart;  // [nseg-1][rows][16]: start state of chunk k+1 at k (pass A)
  float* ws_G;          // [nseg][rows][16]: pass B outgoing gradient of chunk c
  float* ws_S;          // [nseg][rows]: pass B summed step of chunk c
  float* ws_Q;          // [nseg][rows][16]: incoming gradient of chunk c (pass B fold)
  unsigned* ws_count;   // [tiles]: pass B arrivals, reset by the folding CTA
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

// B and C of steps [t0, t0 + kBwdChunk) of batch b into shared memory, fp32 [t][32]
// (B in 0..15, C in 16..31); zero past L.  Each of the 32 threads loads one row of B or C.
template <typename T>
__device__ __forceinline__ void bwd_stage_bc(const BwdArgs& p, int b, int t0, float (*bc)[32]) {
  const int r = threadIdx.x;
  const T* base = r < 16 ? static_cast<const T*>(p.B) + int64_t(b) * p.B_sb + int64_t(r) * p.B_sn
                         : static_cast<const T*>(p.C) + int64_t(b) * p.C_sb + int64_t(r - 16) * p.C_sn;
  for (int j = 0; j < kBwdChunk; ++j) {
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
// pass C: recompute the chunk's states and sweep them backwards.  The chunk is
// walked in windows of kBwdWin steps: a first forward sweep leaves each window's
// start state in shared memory (2 KB per window for the warp); then, window by
// window from the last, the window's kBwdWin states are recomputed into
// registers and swept backwards.  The window's inputs are read once, as 16-byte
// blocks where the rows allow.
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
// pass B: the g recurrence of chunk c >= 1 from a zero incoming gradient, walked
// backwards in windows of kBwdWin steps (16-byte loads of delta, dout and z where
// the rows allow) with the 16 states as 8 packed pairs; then the fold, by the last
// CTA of the row tile to arrive.
// ---------------------------------------------------------------------------

// C of steps [t0, t0 + kBwdChunk) of batch b into shared memory, fp32 [t][16]; zero past L.
// Thread i loads row i % 16 over one half of the steps.
template <typename T>
__device__ __forceinline__ void bwd_stage_c(const BwdArgs& p, int b, int t0, float (*cs)[kN]) {
  const int n = threadIdx.x & (kN - 1);
  const int j0 = (threadIdx.x / kN) * (kBwdChunk / 2);
  const T* base = static_cast<const T*>(p.C) + int64_t(b) * p.C_sb + int64_t(n) * p.C_sn;
#pragma unroll 8
  for (int j = j0; j < j0 + kBwdChunk / 2; ++j) {
    const int t = t0 + j;
    cs[j][n] = t < p.L ? Elem<T>::load(base + t) : 0.0f;
  }
}

template <typename T, bool HAS_Z, bool STRUCT>
__device__ __forceinline__ void bwd_summary_chunk(const BwdArgs& p, const BwdRow& r, const float (*cs)[kN], int b,
                                                  int dc, int t0, int t1, f2_t (&g2)[8], float& ssum) {
  const int64_t ro = int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
  const int64_t go = int64_t(b) * p.g_sb + int64_t(dc) * p.g_sd;
  const int64_t zo = int64_t(b) * p.z_sb + int64_t(dc) * p.z_sd;
  const bool vin = p.vec_rows != 0;
  const int nwin = (t1 - t0 + kBwdWin - 1) / kBwdWin;
  for (int w = nwin - 1; w >= 0; --w) {
    const int tw = t0 + w * kBwdWin;
    float dl[kBwdWin], gd[kBwdWin], zz[kBwdWin];
    bwd_load_win<T>(p.delta, ro, tw, t1, vin, dl);
    bwd_load_win<T>(p.dout, go, tw, t1, vin, gd);
    if constexpr (HAS_Z) bwd_load_win<T>(p.z, zo, tw, t1, vin, zz);
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
      const f2_t gy2 = f2(gy, gy);
      const ulonglong2* cq = reinterpret_cast<const ulonglong2*>(cs[tw - t0 + j]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const ulonglong2 cc = cq[k];  // C pairs (4k, 4k+1), (4k+2, 4k+3)
        g2[2 * k] = mul2(a[2 * k], fma2(gy2, cc.x, g2[2 * k]));
        g2[2 * k + 1] = mul2(a[2 * k + 1], fma2(gy2, cc.y, g2[2 * k + 1]));
      }
      ssum += dt;
    }
  }
}

template <typename T, bool HAS_Z>
__global__ void __launch_bounds__(kBwdRows) scan_bwd_summary_kernel(const BwdArgs p) {
  __shared__ __align__(16) float cs[kBwdChunk][kN];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int c = blockIdx.y + 1;
  const int b = tile / p.tiles_per_batch;
  const int d = (tile - b * p.tiles_per_batch) * kBwdRows + tid;
  const int dc = d < p.D ? d : p.D - 1;
  const int t0 = c * kBwdChunk;
  const int t1 = min(p.L, t0 + kBwdChunk);
  BwdRow r;
  bwd_row(p, dc, r);
  const bool structured = __syncthreads_and(r.structured) && !p.force_general;
  bwd_stage_c<T>(p, b, t0, cs);
  __syncthreads();

  f2_t g2[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) g2[k] = f2(0.0f, 0.0f);
  float ssum = 0.0f;
  if (structured)
    bwd_summary_chunk<T, HAS_Z, true>(p, r, cs, b, dc, t0, t1, g2, ssum);
  else
    bwd_summary_chunk<T, HAS_Z, false>(p, r, cs, b, dc, t0, t1, g2, ssum);
  const int64_t rows_total = int64_t(p.Bt) * p.tiles_per_batch * kBwdRows;
  const int64_t rowg = int64_t(tile) * kBwdRows + tid;
  {
    float gv[kN];
#pragma unroll
    for (int k = 0; k < 8; ++k) f2split(g2[k], gv[2 * k], gv[2 * k + 1]);
    float4* dst = reinterpret_cast<float4*>(p.ws_G + (int64_t(c) * rows_total + rowg) * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) __stcg(dst + i, make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]));
    __stcg(p.ws_S + int64_t(c) * rows_total + rowg, ssum);
  }
  // the last CTA of the row tile folds backwards: Q_(nseg-1) = 0, Q_(c-1) = exp(A S_c) Q_c + G_c,
  // with chunk c-1's summary fetched while chunk c's is applied
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.ws_count[tile], 1u) == unsigned(p.nseg - 2));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  auto fetch = [&](int k, float& sk, float4 (&gk)[4]) {
    sk = __ldcg(p.ws_S + int64_t(k) * rows_total + rowg);
    const float4* gs = reinterpret_cast<const float4*>(p.ws_G + (int64_t(k) * rows_total + rowg) * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) gk[i] = __ldcg(gs + i);
  };
  f2_t q[kN / 2];
#pragma unroll
  for (int k = 0; k < kN / 2; ++k) q[k] = f2(0.0f, 0.0f);
  float s_cur = 0.0f;
  float4 g_cur[4];
  fetch(p.nseg - 1, s_cur, g_cur);
  for (int k = p.nseg - 1; k >= 0; --k) {
    float4* qd = reinterpret_cast<float4*>(p.ws_Q + (int64_t(k) * rows_total + rowg) * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float q0, q1, q2, q3;
      f2split(q[2 * i], q0, q1);
      f2split(q[2 * i + 1], q2, q3);
      __stcg(qd + i, make_float4(q0, q1, q2, q3));
    }
    if (k == 0) break;
    float s_nx = 0.0f;
    float4 g_nx[4] = {};
    if (k > 1) fetch(k - 1, s_nx, g_nx);
    f2_t a[kN / 2];
    if (structured)
      bwd_decay<true>(s_cur, r, a);
    else
      bwd_decay<false>(s_cur, r, a);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      q[2 * i] = fma2(a[2 * i], q[2 * i], f2(g_cur[i].x, g_cur[i].y));
      q[2 * i + 1] = fma2(a[2 * i + 1], q[2 * i + 1], f2(g_cur[i].z, g_cur[i].w));
    }
    s_cur = s_nx;
#pragma unroll
    for (int i = 0; i < 4; ++i) g_cur[i] = g_nx[i];
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

template <typename T, bool HAS_Z, bool STRUCT>
__device__ __forceinline__ void bwd_chunk(const BwdArgs& p, const BwdRow& r, const float (*bc)[32],
                                          f2_t (*hwin)[kN / 2][kBwdRows], int b, bool row_ok, int dc, int t0,
                                          int t1, f2_t (&h)[kN / 2], f2_t (&g)[kN / 2], f2_t (&dA)[kN / 2],
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
  // forward: every window's start state
  for (int w = 0; w < nwin; ++w) {
#pragma unroll
    for (int k = 0; k < kN / 2; ++k) hwin[w][k][tid] = h[k];
    if (w + 1 == nwin) break;
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
    float uu[kBwdWin], dl[kBwdWin], go_[kBwdWin], zz[kBwdWin];
    bwd_load_win<T>(p.u, uo, tw, t1, vin, uu);
    bwd_load_win<T>(p.delta, ro, tw, t1, vin, dl);
    bwd_load_win<T>(p.dout, go, tw, t1, vin, go_);
    if constexpr (HAS_Z) bwd_load_win<T>(p.z, zo, tw, t1, vin, zz);
    // recompute the window's states into registers
    f2_t hs[kBwdWin + 1][kN / 2];  // hs[0]: the window's start state, hs[j + 1]: after step j
#pragma unroll
    for (int k = 0; k < kN / 2; ++k) hs[0][k] = hwin[w][k][tid];
    // slots w (just read) and w + 1 (read for the window before) are free: the 4 KB buffer
    // of the dB/dC reduction
    __syncwarp();
    float* red_s = reinterpret_cast<float*>(&hwin[w][0][0]);
#pragma unroll
    for (int j = 0; j < kBwdWin; ++j) {
      float dsp;  // unused here
      const float dt = bwd_dt(dl[j], r.bias, p.softplus, dsp);
      f2_t a[kN / 2];
      bwd_decay<STRUCT>(dt, r, a);
      bwd_fwd_step(a, dt * uu[j], bc[tw - t0 + j], hs[j], hs[j + 1]);
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
      float gy = go_[j];
      if constexpr (HAS_Z) {
        f2_t ya = f2(0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const ulonglong2 cc = q[4 + k];
          ya = fma2(cc.x, hs[j + 1][2 * k], ya);
          ya = fma2(cc.y, hs[j + 1][2 * k + 1], ya);
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
        f2split(mul2(gym2, hs[j + 1][k]), red[16 + 2 * k], red[17 + 2 * k]);
        const f2_t gah = mul2(mul2(g[k], a[k]), hs[j][k]);
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

template <typename T, bool HAS_Z>
__global__ void __launch_bounds__(kBwdRows) scan_bwd_kernel(const BwdArgs p) {
  __shared__ __align__(16) float bc_s[kBwdChunk][32];
  // window start states, and one spare slot so that two free slots always follow window w
  __shared__ __align__(16) f2_t hwin[kBwdChunk / kBwdWin + 1][kN / 2][kBwdRows];
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int c = blockIdx.y;
  const int b = tile / p.tiles_per_batch;
  const int d = (tile - b * p.tiles_per_batch) * kBwdRows + tid;
  const bool row_ok = d < p.D;
  const int dc = row_ok ? d : p.D - 1;
  const int t0 = c * kBwdChunk;
  const int t1 = min(p.L, t0 + kBwdChunk);
  const int64_t rows_total = int64_t(p.Bt) * p.tiles_per_batch * kBwdRows;
  const int64_t rowg = int64_t(tile) * kBwdRows + tid;
  BwdRow r;
  bwd_row(p, dc, r);
  const bool structured = __syncthreads_and(r.structured) && !p.force_general;
  bwd_stage_bc<T>(p, b, t0, bc_s);
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
