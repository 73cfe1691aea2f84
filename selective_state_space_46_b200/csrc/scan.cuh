// Selective scan forward kernels (sm_100a).
//
// The scan is the Mamba-1 selective state space recurrence: per row (b, d) and
// state n, h_t = exp(delta_t A_dn) h_(t-1) + delta_t B_tn u_t, y_t = C_t . h_t +
// D_d u_t, times silu(z_t) ("Linear Attention vs Softmax Attention: Can RWKV or
// Mamba Replace Transformers?", section Implementation; "State Space Models in
// Large Language Models ...", section Dynamic Parameterization for
// delta = softplus(parameter + linear)).
//
// Work decomposition
//  * One thread owns one row (b, d) and keeps its 16-wide state in registers as
//    eight packed fp32 pairs (fma.rn.f32x2).  A CTA is ROWS (32 or 64)
//    consecutive channels of one batch; it stages that batch's B and C once per
//    32-step chunk in shared memory (fp32, [t][B0..15, C0..15]) and every row
//    reads them as warp-wide broadcasts.
//  * u / delta_raw / z are streamed per row in 16-byte blocks (8 bf16 or 4 fp32
//    steps) by cp.async into a per-thread shared-memory slot ring four blocks
//    deep; each thread reads only its own slots, so the stream needs no barrier
//    and holds no registers while in flight.  y leaves as one 16-byte store per
//    block.
//  * Arithmetic runs in base 2: s = delta / ln 2 comes straight out of the
//    softplus (bias folded into one FMA), exp(delta A) = 2^(s A), and the ln 2
//    that s lacks is folded into B when B is staged, so delta*B*u = s*u*(ln2 B).
//  * Long sequences are split into chunks of seg_len steps.  The per-position
//    affine maps (A_bar_t, B_bar_t u_t) compose associatively ("Mamba selective
//    state space", section "Selectivity Removes the Convolution Shortcut; Scan
//    Restores Parallelism"), so a chunk is summarised by (S, H): S = sum of s
//    over the chunk (its decay is 2^(A_n S)) and H = its end state from zero.
//    Kernel 1 computes (S, H) for every chunk but the last with a backward sweep
//    (H_n = sum_t s_t u_t ln2 B_tn 2^(A_n sum_{r>t} s_r): two FP32 operations per
//    state and step), and the last CTA of a row tile to finish folds the
//    summaries into carried states; no CTA ever waits on another.  Kernel 2 runs
//    every chunk forward from its carried state and writes y and the final state.
//  * Structured A (A_dn == (n+1) A_d0 exactly, the S4D-real initialisation the
//    pages use) computes 2^(s A_dn) as powers of one exponential; any other A
//    takes one SFU exponential per state.  The choice is uniform per CTA.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace mssm {

constexpr int kTC = 32;         // steps per staged B/C chunk
constexpr int kSegQuant = 64;   // chunk lengths of the length split are multiples of this
constexpr int kStages = 4;      // depth of the per-thread cp.async ring (16-byte blocks)

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
  const float* h0;       // [Bt, D, 16] initial state (n stride 1), or null for zero
  int64_t h0_sb, h0_sd;
  int vec_h0;            // h0 rows are 16-byte aligned
  int zoh;               // zero-order-hold input gain (exp(delta A) - 1) / A instead of delta
  int Bt, D, L;
  int force_general;
  int nseg, seg_len;
  int tiles_per_batch;   // ceil(D / ROWS)
  int vec_rows;          // u/delta/z/out row starts are 16-byte aligned
  int vec_bc;            // B/C row starts are 16-byte aligned
  int vec_ls;            // last_state rows are 16-byte aligned
  // carry workspace, used when nseg > 1 (rows_total = Bt * tiles_per_batch * ROWS)
  float* ws_H;           // [nseg-1][rows_total][16]: chunk end state, then carried state
  float* ws_S;           // [nseg-1][rows_total]: sum of delta / ln2 over the chunk
  unsigned* ws_count;    // [Bt * tiles_per_batch]: kernel-1 arrivals, reset by the last one
  // chained schedule (scan_out_chained_kernel), zeroed before each launch
  unsigned* ch_ticket;   // work-item counter
  unsigned* ch_flags;    // [tiles]: chunks of the tile whose carried state is published
  float* ch_carry;       // [tiles * 32][16]: carried state between consecutive chunks
  // fused schedule (scan_fused_kernel): per (tile, chunk) flags (zeroed before each launch),
  // summaries and end states; the ticket is ch_ticket
  unsigned* lb_flags;    // [tiles][nseg]: 1 = summary published, 2 = end state published
  float* lb_S;           // [tiles][nseg][32]
  float* lb_H;           // [tiles][nseg][32][16]
  float* lb_I;           // [tiles][nseg][32][16]
  unsigned* err;         // device error word: bit 1 = a chained wait gave up
  int test_no_publish;   // test hook: the chained kernel publishes no carried states
  // packed variable-length sequences: Bt is the sequence count, the data has one batch row,
  // sequence v covers steps cu_seqlens[v] .. cu_seqlens[v+1] - 1 of it (null: plain batches)
  const int* cu_seqlens;
};

// The steps of virtual batch v: data batch row b, first step tb, length len, and the
// index of its last chunk.  Offsets outside [0, L], decreasing offsets, or a sequence
// longer than the planned nseg * seg_len are clamped and flagged (error word bit 2).
struct SeqRange {
  int b, tb, len, last_seg;
};
__device__ __forceinline__ SeqRange seq_range(const ScanArgs& p, int v) {
  SeqRange r;
  if (!p.cu_seqlens) {
    r.b = v;
    r.tb = 0;
    r.len = p.L;
  } else {
    int a = __ldg(p.cu_seqlens + v), e = __ldg(p.cu_seqlens + v + 1);
    const int cap = p.nseg * p.seg_len;
    bool bad = a < 0 || a > p.L || e < a || e > p.L || e - a > cap;
    a = min(max(a, 0), p.L);
    e = min(max(e, a), p.L);
    if (e - a > cap) e = a + cap;
    if (bad && threadIdx.x == 0 && p.err) atomicOr(p.err, 4u);
    r.b = 0;
    r.tb = a;
    r.len = e - a;
  }
  r.last_seg = r.len > 0 ? (r.len - 1) / p.seg_len : 0;
  return r;
}

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
// Programmatic dependent launch: a grid launched with programmatic stream serialization may
// start while the grid before it in the stream still runs; griddep_wait() returns once that
// grid has completed and its writes are visible (at once for a grid launched without it).
// griddep_launch_dependents() lets the next such grid start before this one ends.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// bf16 halves of a 32-bit word widened to fp32 with a byte permute (ALU pipe)
__device__ __forceinline__ float bf_lo(uint32_t w) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, 0x1044;" : "=r"(r) : "r"(w));
  return __uint_as_float(r);
}
__device__ __forceinline__ float bf_hi(uint32_t w) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, 0x3244;" : "=r"(r) : "r"(w));
  return __uint_as_float(r);
}

// element j of a 16-byte block
template <typename T>
__device__ __forceinline__ float blk_at(const uint4& v, int j) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if constexpr (sizeof(T) == 2) {
    return (j & 1) ? bf_hi(w[j >> 1]) : bf_lo(w[j >> 1]);
  } else {
    return __uint_as_float(w[j]);
  }
}

// softplus in base 2: returns softplus(v) / ln2 given v2 = v * log2(e).
//  * v > 20: v (remainder below 2.1e-9, PyTorch's softplus threshold).
//  * PRECISE (fp32 I/O), e = e^v < 2^-6: the series e - e^2/2 + e^3/3 (scaled by
//    log2 e), whose truncation error is below e^4/4 (relative < 2^-20); avoids
//    forming 1 + e.
//  * otherwise log2(1 + e), within the SFU's 2^-22 absolute error: < 2e-5 relative
//    for a result >= log2(1 + 2^-6).  Without PRECISE (bf16 I/O) this form is used
//    for small e too: the rounding of 1 + e and the SFU add up to an absolute error
//    below 3.3e-7 in the result (2.3e-7 in the step), whose effect on an output is
//    far below the rounding of a bf16 value.
template <bool PRECISE = true>
__device__ __forceinline__ float softplus2(float v2) {
  const float e = ex2f(v2);
  const float big = lg2f(1.0f + e);
  float r = big;
  if constexpr (PRECISE) {
    const float small = e * fmaf(e, fmaf(e, 0.48089834696298783f, -0.72134752044448170f), 1.4426950408889634f);
    r = (e < 0.015625f) ? small : big;
  }
  return (v2 > 28.853900817779268f) ? v2 : r;
}

// ---------------------------------------------------------------------------
// B/C staging: a kTC-step chunk of B rows 0..15 and C rows 0..15 loaded by the
// CTA's ROWS threads into registers, then written transposed to shared memory
// as fp32 [t][32] with B pre-multiplied by ln 2.
// ---------------------------------------------------------------------------
template <typename T, int ROWS> struct BCStage {
  static constexpr int kVals = 32 * kTC / ROWS;        // values per thread: 16 or 32
  static constexpr int kWords = kVals * int(sizeof(T)) / 4;
  static constexpr int kThreadsPerRow = kTC / kVals;   // 2 or 1
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

  // B rows are scaled for the discretisation: ln 2 (Euler, base-2 step s), 1 / (n + 1)
  // (zero-order hold on the structured-A path), or 1 (zero-order hold, general A)
  __device__ __forceinline__ void store(float* s, int bmode = 0) const {  // s: [kTC][32]
    const int tid = threadIdx.x;
    const int r = tid / kThreadsPerRow;
    const int t = (tid % kThreadsPerRow) * kVals;
    const float scale = (r >= 16) ? 1.0f : bmode == 0 ? kLn2 : bmode == 1 ? 1.0f / float(r + 1) : 1.0f;
#pragma unroll
    for (int j = 0; j < kVals; ++j) {
      float v;
      if constexpr (sizeof(T) == 2) {
        v = (j & 1) ? bf_hi(w[j >> 1]) : bf_lo(w[j >> 1]);
      } else {
        v = __uint_as_float(w[j]);
      }
      s[(t + j) * 32 + r] = v * scale;
    }
  }
};

// Fetch the 16-byte block of a row starting at step t into a shared slot:
// cp.async when aligned and complete, else synchronous element loads (zero past t_end).
template <typename T>
__device__ __forceinline__ void fetch_block(uint4* slot, const T* row, int t, int t_end, bool vec) {
  constexpr int S = 16 / int(sizeof(T));
  if (vec && t + S <= t_end) {
    cp_async16(smem_u32(slot), row + t);
  } else {
    uint32_t w[4];
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = (t + 2 * i < t_end) ? uint32_t(__ldg(row + t + 2 * i)) : 0u;
        const uint32_t hi = (t + 2 * i + 1 < t_end) ? uint32_t(__ldg(row + t + 2 * i + 1)) : 0u;
        w[i] = lo | (hi << 16);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = (t + i < t_end) ? __float_as_uint(__ldg(row + t + i)) : 0u;
    }
    *slot = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Store a block of y (S steps of fp32 values) at step t, clipped to [t_lo, t_end).
template <typename T>
__device__ __forceinline__ void store_block(T* row, int t, int t_lo, int t_end, bool vec, const float* y) {
  constexpr int S = 16 / int(sizeof(T));
  const bool whole = vec && t >= t_lo && t + S <= t_end;
  if constexpr (sizeof(T) == 2) {
    const uint32_t w0 = pack_bf16x2(y[0], y[1]), w1 = pack_bf16x2(y[2], y[3]);
    const uint32_t w2 = pack_bf16x2(y[4], y[5]), w3 = pack_bf16x2(y[6], y[7]);
    if (whole) {
      *reinterpret_cast<uint4*>(row + t) = make_uint4(w0, w1, w2, w3);
    } else {
      const uint32_t w[4] = {w0, w1, w2, w3};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ta = t + 2 * i, tb = t + 2 * i + 1;
        if (ta >= t_lo && ta < t_end) row[ta] = uint16_t(w[i] & 0xffffu);
        if (tb >= t_lo && tb < t_end) row[tb] = uint16_t(w[i] >> 16);
      }
    }
  } else {
    if (whole) {
      *reinterpret_cast<float4*>(row + t) = make_float4(y[0], y[1], y[2], y[3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (t + i >= t_lo && t + i < t_end) row[t + i] = y[i];
    }
  }
}

// Powers a^1 .. a^16 as eight pairs (a^(2k+1), a^(2k+2)); 15 multiplies, depth 4.
__device__ __forceinline__ void powers16(float a, f2_t (&dA)[8]) {
  const float a2 = a * a;
  const float a3 = a2 * a, a4 = a2 * a2;
  const float a5 = a4 * a, a6 = a4 * a2, a7 = a4 * a3, a8 = a4 * a4;
  dA[0] = f2(a, a2);
  dA[1] = f2(a3, a4);
  dA[2] = f2(a5, a6);
  dA[3] = f2(a7, a8);
  dA[4] = f2(a8 * a, a8 * a2);
  dA[5] = f2(a8 * a3, a8 * a4);
  dA[6] = f2(a8 * a5, a8 * a6);
  dA[7] = f2(a8 * a7, a8 * a8);
}

// Per-row constants of the scan.
struct RowParams {
  float bias2;   // bias * log2(e)
  float Dd;      // skip weight
  float A0;      // A[d, 0]
  float invA0;   // 1 / A[d, 0] (0 when A[d, 0] = 0)
  f2_t Ap[8];    // A[d, n] pairs (general path)
};

template <bool STRUCT>
__device__ __forceinline__ void decay(float s, const RowParams& rp, f2_t (&dA)[8]) {
  if constexpr (STRUCT) {
    powers16(ex2f(s * rp.A0), dA);
  } else {
    const f2_t s2 = f2(s, s);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float lo, hi;
      f2split(mul2(s2, rp.Ap[k]), lo, hi);
      dA[k] = f2(ex2f(lo), ex2f(hi));
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 2: forward sweep of one chunk from its carried state, fused epilogue.
//
// Software-pipelined over 16-byte blocks of S steps: while block k runs its
// recurrence (FMA pipe), block k+1's per-step scalars (softplus, decay base,
// s*u: SFU-heavy) are computed in the same loop body, so the two overlap.
// ---------------------------------------------------------------------------

// Per-step scalars of one block: x = decay base 2^(s A_0) (structured A) or s
// (general A), w = s * u.  PARTIAL: steps before `lo` or at or past `valid` become
// identity steps (s = 0: A_bar = 1 and no input).
//
// Zero-order hold (ZOH): the input term of state n is G_n B_n u with G_n =
// (exp(delta A_n) - 1) / A_n.  Structured A: exp(delta A_n) - 1 = E (1 + a + ... + a^n)
// with a = exp(delta A_0) and E = a - 1, and A_n = (n+1) A_0, so G_n B_n u =
// (E / A_0) u * P_n * B_n / (n+1) with P_n = sum_{i<=n} a^i: w = (E / A_0) u here
// (E / A_0 = delta phi(delta A_0), see zoh_gain_f), B is staged divided by n + 1, and
// the recurrence forms w P_n by a running FMA over the powers it already has.
// General A: w = u and the recurrence takes G_n per state.  sv[j] = s (for the sum S).
template <typename T, bool SOFTPLUS, bool STRUCT, bool PARTIAL, bool ZOH = false>
__device__ __forceinline__ void block_scalars(const uint4& ru, const uint4& rd, int lo, int valid,
                                              const RowParams& rp, float* x, float* w, float* sv = nullptr) {
  constexpr int S = 16 / int(sizeof(T));
#pragma unroll
  for (int j = 0; j < S; ++j) {
    const float v2 = fmaf(blk_at<T>(rd, j), kLog2e, rp.bias2);
    float s = SOFTPLUS ? softplus2<sizeof(T) == 4>(v2) : v2;
    float uu = blk_at<T>(ru, j);
    if constexpr (PARTIAL) {
      const bool in = j >= lo && j < valid;
      s = in ? s : 0.0f;
      uu = in ? uu : 0.0f;
    }
    x[j] = STRUCT ? ex2f(s * rp.A0) : s;
    if constexpr (!ZOH) {
      w[j] = s * uu;
    } else if constexpr (STRUCT) {
      const float dt = s * kLn2;
      w[j] = zoh_gain_f(x[j], dt, rp.A0, rp.invA0) * uu;
    } else {
      w[j] = uu;
    }
    if (sv) sv[j] = s;
  }
}

// Recurrence and readout of one block; yout[j] = C_t . h_t (before skip and gate).
// READOUT = false: the recurrence only (chunk summaries by a forward sweep).
// invA: 1 / A[d, n] pairs, used by the zero-order hold on the general path only.
template <typename T, bool STRUCT, bool ZOH = false, bool READOUT = true>
__device__ __forceinline__ void block_recurrence(const float* bcrow, const float* x, const float* w,
                                                 const RowParams& rp, f2_t (&h2)[8], float* yout,
                                                 const f2_t* invA = nullptr) {
  constexpr int S = 16 / int(sizeof(T));
#pragma unroll
  for (int j = 0; j < S; ++j) {
    f2_t dA[8];
    f2_t gw[8];  // ZOH: per-state multiplier of the staged B
    if constexpr (STRUCT) {
      powers16(x[j], dA);
      if constexpr (ZOH) {
        // w P_n, n = 0..15, as a running FMA over a^1 .. a^15
        float run = w[j];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float alo, ahi;
          f2split(dA[k], alo, ahi);  // a^(2k+1), a^(2k+2)
          const float p_lo = run;
          const float p_hi = fmaf(w[j], alo, p_lo);
          run = fmaf(w[j], ahi, p_hi);
          gw[k] = f2(p_lo, p_hi);
        }
      }
    } else {
      const f2_t s2 = f2(x[j], x[j]);
      const float dt = x[j] * kLn2;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float lo, hi;
        f2split(mul2(s2, rp.Ap[k]), lo, hi);
        const float elo = ex2f(lo), ehi = ex2f(hi);
        dA[k] = f2(elo, ehi);
        if constexpr (ZOH) {
          float alo, ahi, ilo, ihi;
          f2split(rp.Ap[k], alo, ahi);
          f2split(invA[k], ilo, ihi);
          gw[k] = f2(zoh_gain_f(elo, dt, alo, ilo) * w[j], zoh_gain_f(ehi, dt, ahi, ihi) * w[j]);
        }
      }
    }
    const f2_t w2 = f2(w[j], w[j]);
    const ulonglong2* q = reinterpret_cast<const ulonglong2*>(bcrow + j * 32);
    f2_t ya = 0ull;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const ulonglong2 bb = q[k];      // scaled B, pairs (4k, 4k+1), (4k+2, 4k+3)
      const ulonglong2 cc = q[4 + k];  // C pairs
      const f2_t m0 = ZOH ? gw[2 * k] : w2;
      const f2_t m1 = ZOH ? gw[2 * k + 1] : w2;
      h2[2 * k] = fma2(dA[2 * k], h2[2 * k], mul2(m0, bb.x));
      h2[2 * k + 1] = fma2(dA[2 * k + 1], h2[2 * k + 1], mul2(m1, bb.y));
      if constexpr (READOUT) {
        ya = (k == 0) ? mul2(cc.x, h2[0]) : fma2(cc.x, h2[2 * k], ya);
        ya = fma2(cc.y, h2[2 * k + 1], ya);
      }
    }
    if constexpr (READOUT) {
      float a0, a1;
      f2split(ya, a0, a1);
      yout[j] = a0 + a1;
    }
  }
}

// READOUT = false: no output, no z; ssum returns the sum of s over the steps (the
// chunk-summary sweep of the zero-order-hold discretisation).
template <typename T, int ROWS, bool HAS_Z, bool SOFTPLUS, bool STRUCT, bool ZOH = false, bool READOUT = true>
__device__ __forceinline__ void forward_chunk(const ScanArgs& p, float (*bc_s)[kTC * 32], uint4* slots,
                                              int b, int t0, int t1, const T* urow, const T* dlrow,
                                              const T* zrow, T* orow, bool row_ok, const RowParams& rp,
                                              f2_t (&h2)[8], float* ssum = nullptr, const float* carry = nullptr) {
  constexpr int S = 16 / int(sizeof(T));
  constexpr bool LOAD_Z = HAS_Z && READOUT;
  const int bmode = !ZOH ? 0 : STRUCT ? 1 : 2;
  f2_t invA[8];
  if constexpr (ZOH && !STRUCT) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float lo, hi;
      f2split(rp.Ap[k], lo, hi);
      invA[k] = f2(lo != 0.0f ? rcpf(lo) : 0.0f, hi != 0.0f ? rcpf(hi) : 0.0f);
    }
  }
  float sacc = 0.0f;
  constexpr int kBlkPerChunk = kTC / S;
  const int tid = threadIdx.x;
  const bool vec = p.vec_rows != 0;
  auto take_carry = [&]() {
    if (!carry) return;
    griddep_wait();
    const float4* src = reinterpret_cast<const float4*>(carry);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldcg(src + i);
      h2[2 * i] = f2(v.x, v.y);
      h2[2 * i + 1] = f2(v.z, v.w);
    }
  };
  if (t1 <= t0) {
    take_carry();
    return;
  }
  // blocks are aligned to S-step boundaries of the row; a chunk that starts inside a block
  // (packed sequences) runs its first `head` steps as identity steps and stores nothing there
  const int ta = t0 - t0 % S;
  const int head = t0 - ta;
  const int nblk = (t1 - ta + S - 1) / S;
  const int nchunks = (t1 - ta + kTC - 1) / kTC;

  auto slot = [&](int stage, int tensor) { return slots + (stage * 3 + tensor) * ROWS + tid; };
  auto issue = [&](int k) {
    const int t = ta + k * S;
    const int st = k % kStages;
    fetch_block<T>(slot(st, 0), urow, t, t1, vec);
    fetch_block<T>(slot(st, 1), dlrow, t, t1, vec);
    if constexpr (LOAD_Z) fetch_block<T>(slot(st, 2), zrow, t, t1, vec);
  };
  auto scalars = [&](int k, const uint4& ru, const uint4& rd, float* x, float* w) {
    const int valid = t1 - (ta + k * S);
    const int lo = k == 0 ? head : 0;
    float sv[S];
    if (valid >= S && lo == 0)
      block_scalars<T, SOFTPLUS, STRUCT, false, ZOH>(ru, rd, 0, S, rp, x, w, READOUT ? nullptr : sv);
    else
      block_scalars<T, SOFTPLUS, STRUCT, true, ZOH>(ru, rd, lo, valid, rp, x, w, READOUT ? nullptr : sv);
    if constexpr (!READOUT) {
#pragma unroll
      for (int j = 0; j < S; ++j) sacc += sv[j];
    }
  };
#pragma unroll
  for (int k = 0; k < kStages - 1; ++k) {
    if (k < nblk) issue(k);
    cp_commit();
  }

  BCStage<T, ROWS> stage;
  stage.load(p, b, ta, t1);
  stage.store(bc_s[0], bmode);

  // block 0's scalars
  cp_wait<kStages - 2>();
  uint4 ru = *slot(0, 0);
  uint4 rz = LOAD_Z ? *slot(0, 2) : make_uint4(0u, 0u, 0u, 0u);
  float xc[S], wc[S];
  scalars(0, ru, *slot(0, 1), xc, wc);
  __syncthreads();
  // the carried start state is the previous kernel's output: everything above (row
  // constants, B/C staging, the first input fetches) may overlap that kernel's tail
  take_carry();

  int k = 0;
  for (int c = 0; c < nchunks; ++c) {
    const int cs = ta + c * kTC;
    if (c + 1 < nchunks) stage.load(p, b, cs + kTC, t1);
    const float* bcb = bc_s[c & 1];
#pragma unroll 1
    for (int kb = 0; kb < kBlkPerChunk && k < nblk; ++kb, ++k) {
      // next block: fetch further ahead, then its scalars (independent of this block's recurrence)
      if (k + kStages - 1 < nblk) issue(k + kStages - 1);
      cp_commit();
      float xn[S], wn[S];
      uint4 run = make_uint4(0u, 0u, 0u, 0u), rzn = make_uint4(0u, 0u, 0u, 0u);
      if (k + 1 < nblk) {
        cp_wait<kStages - 2>();
        const int st = (k + 1) % kStages;
        run = *slot(st, 0);
        if constexpr (LOAD_Z) rzn = *slot(st, 2);
        scalars(k + 1, run, *slot(st, 1), xn, wn);
      }
      // this block: recurrence, readout, skip, gate, store
      float y[S];
      block_recurrence<T, STRUCT, ZOH, READOUT>(bcb + kb * S * 32, xc, wc, rp, h2, y, invA);
      if constexpr (READOUT) {
#pragma unroll
        for (int j = 0; j < S; ++j) {
          float v = fmaf(rp.Dd, blk_at<T>(ru, j), y[j]);
          if constexpr (HAS_Z) v *= gate_f<T>(blk_at<T>(rz, j));
          y[j] = v;
        }
        if (row_ok) store_block<T>(orow, ta + k * S, t0, t1, vec, y);
      }
#pragma unroll
      for (int j = 0; j < S; ++j) {
        xc[j] = xn[j];
        wc[j] = wn[j];
      }
      ru = run;
      rz = rzn;
    }
    if (c + 1 < nchunks) stage.store(bc_s[(c + 1) & 1], bmode);
    __syncthreads();
  }
  cp_wait<0>();
  if (ssum) *ssum = sacc;
}

template <int ROWS>
__device__ __forceinline__ bool load_row_params(const ScanArgs& p, int dc, RowParams& rp) {
  const float bias = p.bias ? p.bias[int64_t(dc) * p.bias_s] : 0.0f;
  rp.bias2 = bias * kLog2e;
  rp.Dd = p.Dskip ? p.Dskip[int64_t(dc) * p.D_s] : 0.0f;
  const float* Ar = p.A + int64_t(dc) * p.A_sd;
  rp.A0 = Ar[0];
  rp.invA0 = rp.A0 != 0.0f ? 1.0f / rp.A0 : 0.0f;
  bool st = true;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float lo = Ar[int64_t(2 * k) * p.A_sn], hi = Ar[int64_t(2 * k + 1) * p.A_sn];
    st = st && (lo == float(2 * k + 1) * rp.A0) && (hi == float(2 * k + 2) * rp.A0);
    rp.Ap[k] = f2(lo, hi);
  }
  return st;
}

// The initial state of row (b, d): h0[b, d, :] when given, else zero.
__device__ __forceinline__ void load_h0(const ScanArgs& p, int b, int d, f2_t (&h2)[8]) {
  if (!p.h0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) h2[k] = 0ull;
    return;
  }
  const float* src = p.h0 + int64_t(b) * p.h0_sb + int64_t(d) * p.h0_sd;
  if (p.vec_h0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(src) + i);
      h2[2 * i] = f2(v.x, v.y);
      h2[2 * i + 1] = f2(v.z, v.w);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) h2[k] = f2(__ldg(src + 2 * k), __ldg(src + 2 * k + 1));
  }
}

// The forward sweep with the A path chosen at run time (uniform per CTA).
template <typename T, int ROWS, bool HAS_Z, bool SOFTPLUS, bool ZOH>
__device__ __forceinline__ void forward_any(const ScanArgs& p, float (*bc_s)[kTC * 32], uint4* slots, int b,
                                            int t0, int t1, const T* urow, const T* dlrow, const T* zrow, T* orow,
                                            bool row_ok, const RowParams& rp, bool structured, f2_t (&h2)[8],
                                            const float* carry = nullptr) {
  if (structured)
    forward_chunk<T, ROWS, HAS_Z, SOFTPLUS, true, ZOH>(p, bc_s, slots, b, t0, t1, urow, dlrow, zrow, orow,
                                                       row_ok, rp, h2, nullptr, carry);
  else
    forward_chunk<T, ROWS, HAS_Z, SOFTPLUS, false, ZOH>(p, bc_s, slots, b, t0, t1, urow, dlrow, zrow, orow,
                                                        row_ok, rp, h2, nullptr, carry);
}

// 64-row CTAs are used when the grid must fill 16 warps per SM (128 registers);
// 32-row CTAs when the rows alone limit occupancy, so they may use up to 224.
template <typename T, int ROWS, bool HAS_Z, bool SOFTPLUS, bool ZOH>
__global__ void __launch_bounds__(ROWS, ROWS == 32 ? 9 : 8) scan_out_kernel(const ScanArgs p) {
  __shared__ __align__(16) float bc_s[2][kTC * 32];
  __shared__ __align__(16) uint4 slots[kStages * 3 * ROWS];
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int seg = blockIdx.y;
  const int vb = tile / p.tiles_per_batch;  // batch, or sequence of a packed batch
  const SeqRange sr = seq_range(p, vb);
  if (seg > sr.last_seg) return;  // past the end of a shorter packed sequence
  const int b = sr.b;
  const int d = (tile - vb * p.tiles_per_batch) * ROWS + tid;
  const bool row_ok = d < p.D;
  const int dc = row_ok ? d : p.D - 1;
  const int t0 = sr.tb + seg * p.seg_len;
  const int t1 = sr.tb + min(sr.len, (seg + 1) * p.seg_len);

  const T* urow = static_cast<const T*>(p.u) + int64_t(b) * p.u_sb + int64_t(dc) * p.u_sd;
  const T* dlrow = static_cast<const T*>(p.delta) + int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
  const T* zrow = HAS_Z ? static_cast<const T*>(p.z) + int64_t(b) * p.z_sb + int64_t(dc) * p.z_sd : nullptr;
  T* orow = static_cast<T*>(p.out) + int64_t(b) * p.o_sb + int64_t(dc) * p.o_sd;

  RowParams rp;
  const bool st = load_row_params<ROWS>(p, dc, rp);
  const bool structured = __syncthreads_and(st) && !p.force_general;

  // chunk 0 starts from h0 (an input); a later chunk from the carry the summary kernel
  // folded, read inside forward_chunk once that kernel has completed (this grid may be
  // launched while it still runs)
  f2_t h2[8];
  const float* carry = nullptr;
  if (seg > 0) {
    const int64_t rows_total = int64_t(p.Bt) * p.tiles_per_batch * ROWS;
    const int64_t rowg = int64_t(tile) * ROWS + tid;
    carry = p.ws_H + (int64_t(seg - 1) * rows_total + rowg) * kN;
#pragma unroll
    for (int k = 0; k < 8; ++k) h2[k] = 0ull;
  } else {
    load_h0(p, vb, dc, h2);
  }

  forward_any<T, ROWS, HAS_Z, SOFTPLUS, ZOH>(p, bc_s, slots, b, t0, t1, urow, dlrow, zrow, orow, row_ok, rp,
                                             structured, h2, carry);

  if (seg == sr.last_seg && row_ok && p.last_state) {
    float* dst = p.last_state + int64_t(vb) * p.ls_sb + int64_t(d) * p.ls_sd;
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) f2split(h2[k], v[2 * k], v[2 * k + 1]);
    if (p.vec_ls) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
#pragma unroll
      for (int n = 0; n < 16; ++n) dst[n] = v[n];
    }
  }
}

// ---------------------------------------------------------------------------
// Chained persistent forward kernel.
//
// For shapes with many row tiles, splitting L only to balance the work is
// cheaper done by hand-over than by chunk summaries: work items are (tile,
// chunk) pairs taken in chunk-major order from an atomic ticket by a grid of
// persistent one-warp CTAs; an item starts from the state its tile's previous
// chunk published (st.release / ld.acquire on a per-tile flag) and publishes
// its own end state.  The grid is never larger than the number of tiles, so an
// item's predecessor was taken at least a full grid's worth of items earlier
// and has finished: the wait is a bound that is not expected to be reached.
// If it is (kChainSpinLimit polls with nanosleep back-off), the item sets bit 1
// of the device error word (mssm_get_error reports MSSM_ERR_TIMEOUT) and runs
// from a zero state.  Every SM sub-partition then does the same amount of work
// instead of the 3-versus-2 warps a fixed grid leaves on some of them.
// ---------------------------------------------------------------------------
constexpr int kChainSpinLimit = 1 << 20;

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <typename T, bool HAS_Z, bool SOFTPLUS, bool ZOH>
__global__ void __launch_bounds__(32, 8) scan_out_chained_kernel(const ScanArgs p) {
  constexpr int ROWS = 32;
  __shared__ __align__(16) float bc_s[2][kTC * 32];
  __shared__ __align__(16) uint4 slots[kStages * 3 * ROWS];
  __shared__ int s_item;
  __shared__ int s_ok;
  const int tid = threadIdx.x;
  const int ntiles = p.Bt * p.tiles_per_batch;
  const int nitems = ntiles * p.nseg;
  for (;;) {
    if (tid == 0) s_item = int(atomicAdd(p.ch_ticket, 1u));
    __syncthreads();
    const int item = s_item;
    if (item >= nitems) break;
    const int c = item / ntiles;
    const int tile = item - c * ntiles;
    const int vb = tile / p.tiles_per_batch;  // batch, or sequence of a packed batch
    const SeqRange sr = seq_range(p, vb);
    __syncthreads();                         // every thread has read s_item
    if (c > sr.last_seg) continue;           // past the end of a shorter packed sequence
    const int b = sr.b;
    const int d = (tile - vb * p.tiles_per_batch) * ROWS + tid;
    const bool row_ok = d < p.D;
    const int dc = row_ok ? d : p.D - 1;
    const int t0 = sr.tb + c * p.seg_len;
    const int t1 = sr.tb + min(sr.len, (c + 1) * p.seg_len);
    const T* urow = static_cast<const T*>(p.u) + int64_t(b) * p.u_sb + int64_t(dc) * p.u_sd;
    const T* dlrow = static_cast<const T*>(p.delta) + int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
    const T* zrow = HAS_Z ? static_cast<const T*>(p.z) + int64_t(b) * p.z_sb + int64_t(dc) * p.z_sd : nullptr;
    T* orow = static_cast<T*>(p.out) + int64_t(b) * p.o_sb + int64_t(dc) * p.o_sd;
    RowParams rp;
    const bool st = load_row_params<ROWS>(p, dc, rp);

    f2_t h2[8];
    if (c == 0) {
      load_h0(p, vb, dc, h2);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) h2[k] = 0ull;
    }
    if (c > 0) {
      if (tid == 0) {
        unsigned v = ld_acquire_u32(p.ch_flags + tile);
        for (int it = 0; v < unsigned(c) && it < kChainSpinLimit; ++it) {
          __nanosleep(64);
          v = ld_acquire_u32(p.ch_flags + tile);
        }
        s_ok = v >= unsigned(c);
        if (!s_ok) atomicOr(p.err, 2u);
      }
      __syncthreads();
      if (s_ok) {
        const float4* src = reinterpret_cast<const float4*>(p.ch_carry + (int64_t(tile) * ROWS + tid) * kN);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 v = __ldcg(src + i);
          h2[2 * i] = f2(v.x, v.y);
          h2[2 * i + 1] = f2(v.z, v.w);
        }
      }
    }
    const bool structured = __syncthreads_and(st) && !p.force_general;
    forward_any<T, ROWS, HAS_Z, SOFTPLUS, ZOH>(p, bc_s, slots, b, t0, t1, urow, dlrow, zrow, orow, row_ok, rp,
                                               structured, h2);
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) f2split(h2[k], v[2 * k], v[2 * k + 1]);
    if (c == sr.last_seg) {
      if (row_ok && p.last_state) {
        float* dst = p.last_state + int64_t(vb) * p.ls_sb + int64_t(d) * p.ls_sd;
        if (p.vec_ls) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
#pragma unroll
          for (int n = 0; n < 16; ++n) dst[n] = v[n];
        }
      }
    } else {
      float4* dst = reinterpret_cast<float4*>(p.ch_carry + (int64_t(tile) * ROWS + tid) * kN);
#pragma unroll
      for (int i = 0; i < 4; ++i) __stcg(dst + i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
      __threadfence();
      __syncthreads();
      if (tid == 0 && !p.test_no_publish) st_release_u32(p.ch_flags + tile, unsigned(c + 1));
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Kernel 1: chunk summaries (S, H) by a backward sweep, then the carry fold.
// ---------------------------------------------------------------------------
// Per-step scalars of a block for the backward sweep: s and w = s * u.
template <typename T, bool SOFTPLUS>
__device__ __forceinline__ void block_scalars_bwd(const uint4& ru, const uint4& rd, const RowParams& rp,
                                                  float* sv, float* wv) {
  constexpr int S = 16 / int(sizeof(T));
#pragma unroll
  for (int j = 0; j < S; ++j) {
    const float v2 = fmaf(blk_at<T>(rd, j), kLog2e, rp.bias2);
    const float s = SOFTPLUS ? softplus2<sizeof(T) == 4>(v2) : v2;
    sv[j] = s;
    wv[j] = s * blk_at<T>(ru, j);
  }
}

template <typename T, int ROWS, bool SOFTPLUS, bool STRUCT>
__device__ __forceinline__ void backward_chunk(const ScanArgs& p, float (*bc_s)[kTC * 32], uint4* slots,
                                               int b, int t0, int t1, const T* urow, const T* dlrow,
                                               const RowParams& rp, f2_t (&H2)[8], float& Ssum) {
  constexpr int S = 16 / int(sizeof(T));
  constexpr int kBlkPerChunk = kTC / S;
  const int tid = threadIdx.x;
  const bool vec = p.vec_rows != 0;
  const int nblk = (t1 - t0) / S;          // chunks of kernel 1 are always full
  const int nchunks = (t1 - t0) / kTC;
  auto slot = [&](int stage, int tensor) { return slots + (stage * 3 + tensor) * ROWS + tid; };
  // the i-th block issued is block nblk-1-i (backwards), into stage i % kStages
  auto issue = [&](int i) {
    const int t = t0 + (nblk - 1 - i) * S;
    const int st = i % kStages;
    fetch_block<T>(slot(st, 0), urow, t, t1, vec);
    fetch_block<T>(slot(st, 1), dlrow, t, t1, vec);
  };
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < nblk) issue(i);
    cp_commit();
  }
  BCStage<T, ROWS> stage;  // C rows are staged too but unused here
  stage.load(p, b, t0 + (nchunks - 1) * kTC, t1);
  stage.store(bc_s[0]);
  cp_wait<kStages - 2>();
  float sc[S], wc[S];
  block_scalars_bwd<T, SOFTPLUS>(*slot(0, 0), *slot(0, 1), rp, sc, wc);
  __syncthreads();

  float Tacc = 0.0f;  // sum of s over the steps after the current one
  int i = 0;
  for (int ci = 0; ci < nchunks; ++ci) {
    const int c = nchunks - 1 - ci;
    const int cs = t0 + c * kTC;
    if (c > 0) stage.load(p, b, cs - kTC, t1);
    const float* bcb = bc_s[ci & 1];
#pragma unroll 1
    for (int kb = kBlkPerChunk - 1; kb >= 0; --kb, ++i) {
      if (i + kStages - 1 < nblk) issue(i + kStages - 1);
      cp_commit();
      float sn[S], wn[S];
      if (i + 1 < nblk) {
        cp_wait<kStages - 2>();
        const int st = (i + 1) % kStages;
        block_scalars_bwd<T, SOFTPLUS>(*slot(st, 0), *slot(st, 1), rp, sn, wn);
      }
      // suffix sums: T_j = Tacc + sum_{j < r < S} s_r (independent exponent inputs)
      float Tj[S];
      Tj[S - 1] = Tacc;
#pragma unroll
      for (int j = S - 2; j >= 0; --j) Tj[j] = Tj[j + 1] + sc[j + 1];
      Tacc = Tj[0] + sc[0];
#pragma unroll
      for (int j = 0; j < S; ++j) {
        const ulonglong2* q = reinterpret_cast<const ulonglong2*>(bcb + (kb * S + j) * 32);
        const float w = wc[j];
        f2_t v[8];
        if constexpr (STRUCT) {
          // v_n = w pi^(n+1), pi = 2^(A_0 T_j) = prod_{r>t} A_bar_r,0: pairs by a tree of
          // depth 3 over the broadcast powers pi^2, pi^4, pi^8
          const float pi = ex2f(rp.A0 * Tj[j]);
          const float pi2 = pi * pi, pi4 = pi2 * pi2, pi8 = pi4 * pi4;
          v[0] = f2(w * pi, w * pi2);
          v[1] = mul2(v[0], f2(pi2, pi2));
          const f2_t q4 = f2(pi4, pi4);
          v[2] = mul2(v[0], q4);
          v[3] = mul2(v[1], q4);
          const f2_t q8 = f2(pi8, pi8);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) v[4 + kk] = mul2(v[kk], q8);
        } else {
          const f2_t T2 = f2(Tj[j], Tj[j]);
          const f2_t w2 = f2(w, w);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            float lo, hi;
            f2split(mul2(T2, rp.Ap[kk]), lo, hi);
            v[kk] = mul2(w2, f2(ex2f(lo), ex2f(hi)));
          }
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const ulonglong2 bb = q[kk];
          H2[2 * kk] = fma2(v[2 * kk], bb.x, H2[2 * kk]);
          H2[2 * kk + 1] = fma2(v[2 * kk + 1], bb.y, H2[2 * kk + 1]);
        }
      }
#pragma unroll
      for (int j = 0; j < S; ++j) {
        sc[j] = sn[j];
        wc[j] = wn[j];
      }
    }
    if (c > 0) stage.store(bc_s[(ci + 1) & 1]);
    __syncthreads();
  }
  cp_wait<0>();
  Ssum = Tacc;
}

// FWD: summaries by the forward sweep (zero-order hold, packed sequences whose chunks start
// inside a 16-byte block); otherwise by the cheaper backward sweep.
template <typename T, int ROWS, bool SOFTPLUS, bool ZOH, bool FWD>
__global__ void __launch_bounds__(ROWS, 512 / ROWS) scan_chunk_state_kernel(const ScanArgs p) {
  __shared__ __align__(16) float bc_s[2][kTC * 32];
  __shared__ __align__(16) uint4 slots[kStages * 3 * ROWS];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int seg = blockIdx.y;  // 0 .. nseg-2
  const int vb = tile / p.tiles_per_batch;  // batch, or sequence of a packed batch
  const SeqRange sr = seq_range(p, vb);
  if (seg >= sr.last_seg) return;  // the last chunk of a sequence needs no summary
  const int b = sr.b;
  const int d = (tile - vb * p.tiles_per_batch) * ROWS + tid;
  const int dc = d < p.D ? d : p.D - 1;
  const int t0 = sr.tb + seg * p.seg_len;
  const int t1 = t0 + p.seg_len;  // not the last chunk: always full

  const T* urow = static_cast<const T*>(p.u) + int64_t(b) * p.u_sb + int64_t(dc) * p.u_sd;
  const T* dlrow = static_cast<const T*>(p.delta) + int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
  RowParams rp;
  const bool st = load_row_params<ROWS>(p, dc, rp);
  const bool structured = __syncthreads_and(st) && !p.force_general;

  f2_t H2[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) H2[k] = 0ull;
  float Ssum = 0.0f;
  if constexpr (ZOH || FWD) {
    // the summary is the chunk's end state from zero by a forward sweep (for the zero-order
    // hold the backward form would need every step's own powers as well as the suffix decay)
    if (structured)
      forward_chunk<T, ROWS, false, SOFTPLUS, true, ZOH, false>(p, bc_s, slots, b, t0, t1, urow, dlrow, nullptr,
                                                                nullptr, false, rp, H2, &Ssum);
    else
      forward_chunk<T, ROWS, false, SOFTPLUS, false, ZOH, false>(p, bc_s, slots, b, t0, t1, urow, dlrow,
                                                                 nullptr, nullptr, false, rp, H2, &Ssum);
  } else if (structured) {
    backward_chunk<T, ROWS, SOFTPLUS, true>(p, bc_s, slots, b, t0, t1, urow, dlrow, rp, H2, Ssum);
  } else {
    backward_chunk<T, ROWS, SOFTPLUS, false>(p, bc_s, slots, b, t0, t1, urow, dlrow, rp, H2, Ssum);
  }

  const int64_t rows_total = int64_t(p.Bt) * p.tiles_per_batch * ROWS;
  const int64_t rowg = int64_t(tile) * ROWS + tid;
  {
    float4* dst = reinterpret_cast<float4*>(p.ws_H + (int64_t(seg) * rows_total + rowg) * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a, bq, c, dd;
      f2split(H2[2 * i], a, bq);
      f2split(H2[2 * i + 1], c, dd);
      __stcg(dst + i, make_float4(a, bq, c, dd));
    }
    __stcg(p.ws_S + int64_t(seg) * rows_total + rowg, Ssum);
  }
  // The forward kernel that follows may start once every CTA has got here: its CTAs then
  // take the places of the CTAs that exit and run their prologue during the folds below.
  // (Triggering earlier would let them hold registers beside this kernel's CTAs and push
  // part of their grid into a second wave.)  They read the folded carries only after
  // griddep_wait(), which waits for this whole grid.
  griddep_launch_dependents();

  // The last kernel-1 CTA of this row tile folds the chunk summaries, in chunk
  // order, into carried states: prefix_k = 2^(A S_k) prefix_(k-1) + H_k, stored
  // over H_k.  Nobody waits: the fold runs in whichever CTA arrives last.
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&p.ws_count[tile], 1u) == unsigned(sr.last_seg - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  f2_t h[8];
  load_h0(p, vb, dc, h);
  const int nrec = sr.last_seg;
  // records are prefetched one ahead so the serial walk waits on arithmetic, not on L2
  float4 nv[4];
  float nS = 0.0f;
  {
    const float4* rec = reinterpret_cast<const float4*>(p.ws_H + rowg * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) nv[i] = __ldcg(rec + i);
    nS = __ldcg(p.ws_S + rowg);
  }
  for (int k = 0; k < nrec; ++k) {
    float4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = nv[i];
    const float Sk = nS;
    if (k + 1 < nrec) {
      const float4* nrec_p = reinterpret_cast<const float4*>(p.ws_H + (int64_t(k + 1) * rows_total + rowg) * kN);
#pragma unroll
      for (int i = 0; i < 4; ++i) nv[i] = __ldcg(nrec_p + i);
      nS = __ldcg(p.ws_S + int64_t(k + 1) * rows_total + rowg);
    }
    float4* rec = reinterpret_cast<float4*>(p.ws_H + (int64_t(k) * rows_total + rowg) * kN);
    const f2_t S2 = f2(Sk, Sk);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float e0, e1, e2, e3;
      f2split(mul2(S2, rp.Ap[2 * i]), e0, e1);
      f2split(mul2(S2, rp.Ap[2 * i + 1]), e2, e3);
      h[2 * i] = fma2(f2(ex2f(e0), ex2f(e1)), h[2 * i], f2(v[i].x, v[i].y));
      h[2 * i + 1] = fma2(f2(ex2f(e2), ex2f(e3)), h[2 * i + 1], f2(v[i].z, v[i].w));
      float a, bq, c, dd;
      f2split(h[2 * i], a, bq);
      f2split(h[2 * i + 1], c, dd);
      __stcg(rec + i, make_float4(a, bq, c, dd));
    }
  }
  if (tid == 0) p.ws_count[tile] = 0u;
}



}  // namespace mssm

namespace mssm {

// ---------------------------------------------------------------------------
// Fused single-pass schedule: chunk summaries, carries and the forward sweep in
// one persistent kernel (a decoupled look-back over the chunks of a row tile).
//
// Work items (tile, chunk) are taken in chunk-major order from an atomic ticket.
// An item of chunk c first summarises its chunk (S_c, H_c) -- unless it is the
// last chunk, whose summary nobody reads -- and publishes it (flag 1), then looks
// back over chunks c-1, c-2, ... composing their published summaries until it
// meets a published end state (flag 2), which gives its start state; it then
// publishes its own end state (flag 2) and runs the forward sweep.  Chunk 0's
// end state follows from its summary and h0 without looking back.  Every wait is
// on an item taken earlier, whose own waits are on items earlier still, so the
// waits always end; each is bounded anyway (kChainSpinLimit polls): if one gives
// up, the item records bit 1 of the device error word and treats the missing
// prefix as a zero state.  Records: flags [tiles][nseg], S [tiles][nseg][32],
// H and end states [tiles][nseg][32][16].
// ---------------------------------------------------------------------------
template <bool STRUCT>
__device__ __forceinline__ void lb_decay(float S, const RowParams& rp, f2_t (&e)[8]) {
  // 2^(S A_n): the chunk's decay over summed base-2 step S
  const f2_t S2 = f2(S, S);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float lo, hi;
    f2split(mul2(S2, rp.Ap[k]), lo, hi);
    e[k] = f2(ex2f(lo), ex2f(hi));
  }
}

template <typename T, bool HAS_Z, bool SOFTPLUS, bool ZOH>
__global__ void __launch_bounds__(32, 8) scan_fused_kernel(const ScanArgs p) {
  constexpr int ROWS = 32;
  __shared__ __align__(16) float bc_s[2][kTC * 32];
  __shared__ __align__(16) uint4 slots[kStages * 3 * ROWS];
  __shared__ int s_item;
  __shared__ unsigned s_flag;
  const int tid = threadIdx.x;
  const int ntiles = p.Bt * p.tiles_per_batch;
  const int nitems = ntiles * p.nseg;
  for (;;) {
    if (tid == 0) s_item = int(atomicAdd(p.ch_ticket, 1u));
    __syncthreads();
    const int item = s_item;
    if (item >= nitems) break;
    const int c = item / ntiles;
    const int tile = item - c * ntiles;
    const int b = tile / p.tiles_per_batch;
    const int d = (tile - b * p.tiles_per_batch) * ROWS + tid;
    const bool row_ok = d < p.D;
    const int dc = row_ok ? d : p.D - 1;
    const int t0 = c * p.seg_len;
    const int t1 = min(p.L, t0 + p.seg_len);
    const T* urow = static_cast<const T*>(p.u) + int64_t(b) * p.u_sb + int64_t(dc) * p.u_sd;
    const T* dlrow = static_cast<const T*>(p.delta) + int64_t(b) * p.dl_sb + int64_t(dc) * p.dl_sd;
    const T* zrow = HAS_Z ? static_cast<const T*>(p.z) + int64_t(b) * p.z_sb + int64_t(dc) * p.z_sd : nullptr;
    T* orow = static_cast<T*>(p.out) + int64_t(b) * p.o_sb + int64_t(dc) * p.o_sd;
    RowParams rp;
    const bool st = load_row_params<ROWS>(p, dc, rp);
    const bool structured = __syncthreads_and(st) && !p.force_general;
    const int64_t recbase = int64_t(tile) * p.nseg;  // record of chunk k: (recbase + k) * ROWS + tid
    const bool publish = !p.test_no_publish;

    auto store16 = [&](float* dst, const f2_t (&v)[8]) {
      float4* q = reinterpret_cast<float4*>(dst);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a0, a1, a2, a3;
        f2split(v[2 * i], a0, a1);
        f2split(v[2 * i + 1], a2, a3);
        __stcg(q + i, make_float4(a0, a1, a2, a3));
      }
    };
    auto load16 = [&](const float* src, f2_t (&v)[8]) {
      const float4* q = reinterpret_cast<const float4*>(src);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = __ldcg(q + i);
        v[2 * i] = f2(x.x, x.y);
        v[2 * i + 1] = f2(x.z, x.w);
      }
    };
    auto release = [&](int k, unsigned flag) {  // records of chunk k written by every thread
      __threadfence();
      __syncthreads();
      if (tid == 0 && publish) st_release_u32(p.lb_flags + recbase + k, flag);
    };

    // 1. this chunk's summary (not for the last chunk: nobody reads it)
    f2_t H[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) H[k] = 0ull;
    float S = 0.0f;
    const bool last = c == p.nseg - 1;
    if (!last) {
      if constexpr (ZOH) {
        if (structured)
          forward_chunk<T, ROWS, false, SOFTPLUS, true, true, false>(p, bc_s, slots, b, t0, t1, urow, dlrow,
                                                                     nullptr, nullptr, false, rp, H, &S);
        else
          forward_chunk<T, ROWS, false, SOFTPLUS, false, true, false>(p, bc_s, slots, b, t0, t1, urow, dlrow,
                                                                      nullptr, nullptr, false, rp, H, &S);
      } else {
        if (structured)
          backward_chunk<T, ROWS, SOFTPLUS, true>(p, bc_s, slots, b, t0, t1, urow, dlrow, rp, H, S);
        else
          backward_chunk<T, ROWS, SOFTPLUS, false>(p, bc_s, slots, b, t0, t1, urow, dlrow, rp, H, S);
      }
    }
    const int64_t myrec = (recbase + c) * ROWS + tid;
    f2_t carry[8];
    if (c == 0) {
      load_h0(p, b, dc, carry);
    } else {
      if (!last) {
        store16(p.lb_H + myrec * kN, H);
        __stcg(p.lb_S + myrec, S);
        release(c, 1u);
      }
      // 2. look back: compose the published summaries of chunks c-1, c-2, ... (later ones
      // first) until a published end state; (Sacc, Hacc) is the map of the chunks in between
      f2_t Hacc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) Hacc[k] = 0ull;
      float Sacc = 0.0f;
      bool found = false;
      for (int k = c - 1; k >= 0; --k) {
        if (tid == 0) {
          unsigned v = ld_acquire_u32(p.lb_flags + recbase + k);
          for (int it = 0; v == 0u && it < kChainSpinLimit; ++it) {
            __nanosleep(64);
            v = ld_acquire_u32(p.lb_flags + recbase + k);
          }
          if (v == 0u) atomicOr(p.err, 2u);
          s_flag = v;
        }
        __syncthreads();
        const unsigned f = s_flag;
        __syncthreads();
        if (f == 0u) break;  // gave up: the prefix before chunk k is taken as zero
        const int64_t rk = (recbase + k) * ROWS + tid;
        f2_t e[8];
        lb_decay<true>(Sacc, rp, e);
        f2_t v[8];
        if (f >= 2u) {
          load16(p.lb_I + rk * kN, v);
#pragma unroll
          for (int q = 0; q < 8; ++q) Hacc[q] = fma2(e[q], v[q], Hacc[q]);
          found = true;
          break;
        }
        load16(p.lb_H + rk * kN, v);
#pragma unroll
        for (int q = 0; q < 8; ++q) Hacc[q] = fma2(e[q], v[q], Hacc[q]);
        Sacc += __ldcg(p.lb_S + rk);
      }
      (void)found;
#pragma unroll
      for (int q = 0; q < 8; ++q) carry[q] = Hacc[q];
    }
    // this chunk's end state for the chunks after it: 2^(A S) carry + H
    if (!last) {
      f2_t e[8], I[8];
      lb_decay<true>(S, rp, e);
#pragma unroll
      for (int q = 0; q < 8; ++q) I[q] = fma2(e[q], carry[q], H[q]);
      store16(p.lb_I + myrec * kN, I);
      release(c, 2u);
    }

    // 3. the forward sweep from the carried state
    forward_any<T, ROWS, HAS_Z, SOFTPLUS, ZOH>(p, bc_s, slots, b, t0, t1, urow, dlrow, zrow, orow, row_ok, rp,
                                               structured, carry);
    if (last && row_ok && p.last_state) {
      float* dst = p.last_state + int64_t(b) * p.ls_sb + int64_t(d) * p.ls_sd;
      float v[16];
#pragma unroll
      for (int k = 0; k < 8; ++k) f2split(carry[k], v[2 * k], v[2 * k + 1]);
      if (p.vec_ls) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      } else {
#pragma unroll
        for (int n = 0; n < 16; ++n) dst[n] = v[n];
      }
    }
    __syncthreads();
  }
}

}  // namespace mssm
