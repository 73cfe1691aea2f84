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
  int groups;     // streaming kernel: batch groups (CTAs per channel block)
  int zoh;        // zero-order-hold input gain (exp(dt A) - 1) / A instead of dt
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

// One state: h <- exp(dt a) h + g x b, g = dt (Euler) or (exp(dt a) - 1) / a (zero-order hold).
__device__ __forceinline__ float decode_state(bool zoh, float h, float a, float b, float dt, float dl2, float x,
                                              float w) {
  const float e = ex2f(dl2 * a);
  if (zoh) return fmaf(e, h, zoh_gain_f(e, dt, a, a != 0.0f ? rcpf(a) : 0.0f) * x * b);
  return fmaf(e, h, w * b);
}

// Update one 16-byte quarter q (states 4q..4q+3); returns the partial readout.
template <typename T>
__device__ __forceinline__ float decode_quarter(const DecodeArgs& p, const DecodeRow& r, int q, float4& h) {
  const float4 a = load4<float>(p.A, int64_t(r.d) * p.A_sd + int64_t(4 * q) * p.A_sn, p.A_sn, p.vec_A != 0);
  const float4 bv = load4<T>(p.B, int64_t(r.b) * p.B_sb + int64_t(4 * q) * p.B_sn, p.B_sn, p.vec_BC != 0);
  const float4 cv = load4<T>(p.C, int64_t(r.b) * p.C_sb + int64_t(4 * q) * p.C_sn, p.C_sn, p.vec_BC != 0);
  const bool zoh = p.zoh != 0;
  h.x = decode_state(zoh, h.x, a.x, bv.x, r.dt, r.dl2, r.x, r.w);
  h.y = decode_state(zoh, h.y, a.y, bv.y, r.dt, r.dl2, r.x, r.w);
  h.z = decode_state(zoh, h.z, a.z, bv.z, r.dt, r.dl2, r.x, r.w);
  h.w = decode_state(zoh, h.w, a.w, bv.w, r.dt, r.dl2, r.x, r.w);
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
// persistent streaming form.  Every warp owns one block of 32 channels and walks
// the batches b = g, g + G, g + 2G, ... of that block (g, G: its batch group and
// the group count), independently of the other warps of its CTA.  Per (batch,
// channel block) tile, lane 0 issues bulk copies of everything the tile reads --
// the contiguous 2 KB of state, the x / dt / z runs of the block and the batch's
// B and C rows -- into one slot of the warp's own shared-memory ring, all counted
// on the slot's mbarrier; kWsAhead tiles are in flight ahead of the one being
// updated, and the updated state leaves by a bulk store that overlaps the
// following tiles.  A, the skip weight and the bias of a lane's channel are
// loaded once into registers.  The only waits in the loop are the (bounded)
// mbarrier waits the ring hides and warp-level syncs: no warp waits for another
// (a CTA-wide tile synchronised all 128 threads twice per tile, which was the
// kernel's largest stall).
//
// Needs: contiguous 16-byte-aligned state; x, dt (and z) with unit channel
// stride, 16-byte-aligned batch rows and D a multiple of 16 / sizeof(T); B and
// C with unit n stride and 16-byte-aligned batch rows (the host checks all).
// ---------------------------------------------------------------------------
constexpr int kWsRows = 32;          // channels per warp, one lane each
constexpr int kWsWarps = 4;          // warps per CTA
constexpr int kWsBufs = 6;           // ring slots per warp
constexpr int kWsAhead = kWsBufs - 1;
constexpr int kStreamCtasPerSm = 3;  // 3 x 4 warps x 6 slots of <= 2.5 KB of shared memory

template <typename T>
struct StreamSlot {
  static constexpr uint32_t kState = 0;
  static constexpr uint32_t kX = kWsRows * kN * 4;
  static constexpr uint32_t kDt = kX + kWsRows * sizeof(T);
  static constexpr uint32_t kZ = kDt + kWsRows * sizeof(T);
  static constexpr uint32_t kB = kZ + kWsRows * sizeof(T);
  static constexpr uint32_t kC = kB + kN * sizeof(T);
  static constexpr uint32_t kBytes = kC + kN * sizeof(T);
  static_assert(kBytes % 16 == 0 && kX % 16 == 0 && kDt % 16 == 0 && kZ % 16 == 0 && kB % 16 == 0 &&
                    kC % 16 == 0,
                "slot layout must keep 16-byte alignment");
};

// One wait on a ring slot's mbarrier: the warp sleeps until the phase completes or about
// kStreamWaitHintNs pass (instead of re-polling), so warps that wait for their data take no
// issue slots from the warps that have theirs.
constexpr uint32_t kStreamWaitHintNs = 2000;
constexpr int kStreamWaitLimit = 1 << 19;  // bounded: at most about a second of waiting
__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t mb, uint32_t parity) {
  uint32_t done;
  asm volatile("{\n .reg .pred pr;\n mbarrier.try_wait.parity.shared::cta.b64 pr, [%1], %2, %3;\n selp.u32 %0, 1, 0, pr;\n}"
               : "=r"(done) : "r"(mb), "r"(parity), "r"(kStreamWaitHintNs) : "memory");
  return done;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t mb) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(mb) : "memory");
}

// value j of a run of T stored in shared memory
template <typename T>
__device__ __forceinline__ float smem_elem(const unsigned char* base, int j) {
  return Elem<T>::load(reinterpret_cast<const T*>(base) + j);
}

// values 4q .. 4q+3 of a 16-value run of T in shared memory (16-byte aligned), one load
template <typename T>
__device__ __forceinline__ void smem_quarter(const unsigned char* base, int q, float (&v)[4]) {
  if constexpr (sizeof(T) == 2) {
    const uint2 w = *reinterpret_cast<const uint2*>(base + q * 8);
    v[0] = bf16lo(w.x); v[1] = bf16hi(w.x); v[2] = bf16lo(w.y); v[3] = bf16hi(w.y);
  } else {
    const float4 w = *reinterpret_cast<const float4*>(base + q * 16);
    v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
  }
}

template <typename T, bool HAS_Z>
__global__ void __launch_bounds__(kWsWarps * 32, kStreamCtasPerSm) state_update_stream_kernel(const DecodeArgs p) {
  using L = StreamSlot<T>;
  extern __shared__ __align__(128) unsigned char ring_s[];  // kWsWarps x kWsBufs slots of L::kBytes
  __shared__ __align__(8) unsigned long long mbar[kWsWarps][kWsBufs];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nblk = (p.D + kWsRows - 1) / kWsRows;
  const int gw = int(blockIdx.x) * kWsWarps + warp;
  const int cb = gw % nblk;
  const int g = gw / nblk;
  // a whole warp leaves here (nothing below synchronises more than one warp)
  if (g >= p.Bt || g >= p.groups) return;
  const int c0 = cb * kWsRows;
  const int nrows = p.D - c0 < kWsRows ? p.D - c0 : kWsRows;
  const uint32_t mine = uint32_t(p.Bt - 1 - g) / uint32_t(p.groups) + 1;  // batches of this warp
  const bool live = lane < nrows;
  const int d = c0 + (live ? lane : nrows - 1);
  unsigned char* wring = ring_s + warp * (kWsBufs * L::kBytes);
  const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(wring));
  const uint32_t mb0 = static_cast<uint32_t>(__cvta_generic_to_shared(&mbar[warp][0]));
  constexpr uint32_t ES = sizeof(T);
  const uint32_t run_bytes = uint32_t(nrows) * ES;  // a multiple of 16 (D % (16 / ES) == 0)
  const uint32_t tile_bytes = uint32_t(nrows) * kN * 4 + (HAS_Z ? 3u : 2u) * run_bytes + 2u * kN * ES;

  auto issue = [&](uint32_t i) {  // lane 0
    const int64_t b = int64_t(g) + int64_t(i) * p.groups;
    const uint32_t slot = ring + (i % kWsBufs) * L::kBytes;
    const uint32_t mb = mb0 + (i % kWsBufs) * 8;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb), "r"(tile_bytes) : "memory");
    bulk_load(slot + L::kState, p.state + (b * p.D + c0) * kN, uint32_t(nrows) * kN * 4, mb);
    bulk_load(slot + L::kX, static_cast<const T*>(p.x) + b * p.x_sb + c0, run_bytes, mb);
    bulk_load(slot + L::kDt, static_cast<const T*>(p.dt) + b * p.dt_sb + c0, run_bytes, mb);
    if constexpr (HAS_Z) bulk_load(slot + L::kZ, static_cast<const T*>(p.z) + b * p.z_sb + c0, run_bytes, mb);
    bulk_load(slot + L::kB, static_cast<const T*>(p.B) + b * p.B_sb, kN * ES, mb);
    bulk_load(slot + L::kC, static_cast<const T*>(p.C) + b * p.C_sb, kN * ES, mb);
  };

  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < kWsBufs; ++k)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mb0 + 8 * k) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (uint32_t j = 0; j < uint32_t(kWsAhead) && j < mine; ++j) issue(j);
  }
  __syncwarp();

  // per-channel constants, once per warp.  The state row is visited in the lane-rotated
  // quarter order q = (kq + rot) & 3 (bank-conflict free), so A is stored pre-rotated:
  // a2r[4 kq + e] = A[d, 4 q + e] * log2(e), and the loop indexes it with constants.
  const int rot = (lane >> 1) & 3;
  float a2r[kN];
  {
    const float* Ar = p.A + int64_t(d) * p.A_sd;
#pragma unroll
    for (int kq = 0; kq < 4; ++kq)
#pragma unroll
      for (int e = 0; e < 4; ++e) a2r[4 * kq + e] = Ar[int64_t(4 * ((kq + rot) & 3) + e) * p.A_sn] * kLog2e;
  }
  const float bias = p.bias ? p.bias[int64_t(d) * p.bias_s] : 0.0f;
  const float Dd = p.Dskip ? p.Dskip[int64_t(d) * p.D_s] : 0.0f;

  uint32_t i = 0;
  bool ok = true;
  for (; i < mine; ++i) {
    const uint32_t k = i % kWsBufs;
    unsigned char* slot = wring + k * L::kBytes;
    uint32_t done = 0;
    for (int it = 0; it < kStreamWaitLimit && !done; ++it) done = mbar_try_wait(mb0 + k * 8, (i / kWsBufs) & 1u);
    if (!__all_sync(0xffffffffu, done)) {
      ok = false;
      break;
    }
    if (live) {
      const int64_t b = int64_t(g) + int64_t(i) * p.groups;
      const float x = smem_elem<T>(slot + L::kX, lane);
      float dt = smem_elem<T>(slot + L::kDt, lane) + bias;
      if (p.softplus) dt = softplus_f(dt);
      const float w = dt * x;
      float4* hs = reinterpret_cast<float4*>(slot + L::kState + lane * (kN * 4));
      float y = 0.0f;
#pragma unroll
      for (int kq = 0; kq < 4; ++kq) {
        const int q = (kq + rot) & 3;
        float4 h = hs[q];
        float hv[4] = {h.x, h.y, h.z, h.w};
        float bq[4], cq[4];  // B and C of states 4q .. 4q+3, one shared load each
        smem_quarter<T>(slot + L::kB, q, bq);
        smem_quarter<T>(slot + L::kC, q, cq);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float ed = ex2f(dt * a2r[4 * kq + e]);
          float gn = w;
          if (p.zoh) {
            const float an = a2r[4 * kq + e] * kLn2;
            gn = zoh_gain_f(ed, dt, an, an != 0.0f ? rcpf(an) : 0.0f) * x;
          }
          hv[e] = fmaf(ed, hv[e], gn * bq[e]);
          y = fmaf(cq[e], hv[e], y);
        }
        hs[q] = make_float4(hv[0], hv[1], hv[2], hv[3]);
      }
      y = fmaf(Dd, x, y);
      if constexpr (HAS_Z) y *= gate_f<T>(smem_elem<T>(slot + L::kZ, lane));
      T* o = static_cast<T*>(p.out) + b * p.o_sb + int64_t(d) * p.o_sd;
      if constexpr (sizeof(T) == 2) {
        *o = f_to_bf16(y);
      } else {
        *o = y;
      }
    }
    // generic-proxy accesses of this slot -> ordered before the bulk store and the next bulk load
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
      const int64_t b = int64_t(g) + int64_t(i) * p.groups;
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                   ::"l"(p.state + (b * p.D + c0) * kN), "r"(ring + k * L::kBytes + L::kState),
                   "r"(uint32_t(nrows) * kN * 4) : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      if (i + kWsAhead < mine) {
        // tile i + kWsAhead takes the slot of tile i - 1, whose store is the older of
        // the (at most) two stores in flight
        asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        issue(i + kWsAhead);
      }
    }
  }
  if (!ok && lane == 0) {
    // record the error; give the loads still in flight (tiles i .. i + kWsAhead - 1) a
    // bounded time to land before the warp's slots can be released
    atomicOr(p.err, 1u);
    for (uint32_t j = i; j < i + kWsAhead && j < mine; ++j) {
      uint32_t done = 0;
      for (int it = 0; it < kStreamWaitLimit && !done; ++it)
        done = mbar_try_wait(mb0 + (j % kWsBufs) * 8, (j / kWsBufs) & 1u);
    }
  }
  if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
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
