// C ABI of libmssm.so: argument validation, dtype/shape dispatch, the carry
// workspace, status codes.  Every compute step runs in the kernels of scan.cu
// and decode.cu; nothing here touches tensor contents on the host.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/mssm.h"
#include "launch.h"

namespace {

thread_local std::string g_last_error;

mssm_status fail(mssm_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

mssm_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MSSM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

std::mutex g_mu;
int g_force_general = 0;
int64_t g_chunk_len = 0;
int g_schedule = -1;
int g_rows_per_cta = 0;     // 0 automatic, else 32, 64 or 128
int g_rows_per_thread = 0;  // 0 automatic, else 1 or 2
int g_decode_path = 0;  // MSSM_OPT_DECODE_PATH
int g_test_hooks = 0;   // MSSM_OPT_TEST_HOOKS  // -1 automatic, else the forced LaunchShape mode

// ---- launch accounting and optional per-kernel event timing (diagnostics)
int64_t g_launches[MSSM_KERNEL_KINDS] = {};
int g_timing = 0;
struct TimedLaunch {
  int kind;
  cudaEvent_t a, b;
};
std::vector<TimedLaunch> g_pending;
std::vector<cudaEvent_t> g_event_pool;
double g_time_ms[MSSM_KERNEL_KINDS] = {};
int64_t g_timed[MSSM_KERNEL_KINDS] = {};

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Launch through `fn`, counting it and, when timing is on, bracketing it with
// events recorded on the same stream.  Caller holds g_mu.
template <typename F>
cudaError_t tracked(int kind, cudaStream_t s, F&& fn) {
  cudaEvent_t a = nullptr, b = nullptr;
  if (g_timing) {
    a = take_event();
    b = take_event();
    if (a && b && cudaEventRecord(a, s) != cudaSuccess) a = nullptr;
  }
  cudaError_t e = fn();
  if (e != cudaSuccess) return e;
  ++g_launches[kind];
  if (g_timing && a && b && cudaEventRecord(b, s) == cudaSuccess) g_pending.push_back({kind, a, b});
  return cudaSuccess;
}

struct DeviceState {
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int64_t count_cap = 0;  // arrival counters at the start of ws (a region only counters ever use)
  int sm_count = 0;
  void* bwd_ws = nullptr;  // the backward scan's checkpoints and chunk gradients
  size_t bwd_bytes = 0;
};
std::vector<DeviceState> g_dev;

DeviceState* device_state(int dev) {
  if (dev < 0) return nullptr;
  if (int(g_dev.size()) <= dev) g_dev.resize(dev + 1);
  DeviceState& s = g_dev[dev];
  if (s.sm_count == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    s.sm_count = v;
  }
  return &s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t esize(int dtype) { return dtype == MSSM_BF16 ? 2 : 4; }  // f32, i32: 4

const char* dname(int dtype) {
  return dtype == MSSM_BF16 ? "bf16" : dtype == MSSM_F32 ? "f32" : dtype == MSSM_I32 ? "i32" : "?";
}

// Shape/dtype check of one tensor.  shape entries < 0 are not checked.
mssm_status check(const mssm_tensor* t, const char* name, int ndim, const int64_t* shape,
                  int dtype, bool inner_contig) {
  if (!t) return fail(MSSM_ERR_INVALID_ARG, "%s: null tensor descriptor", name);
  if (t->ndim != ndim) return fail(MSSM_ERR_INVALID_ARG, "%s: expected %d dims, got %d", name, ndim, t->ndim);
  int64_t numel = 1;
  for (int i = 0; i < ndim; ++i) {
    if (t->shape[i] < 0) return fail(MSSM_ERR_INVALID_ARG, "%s: negative size in dim %d", name, i);
    if (shape[i] >= 0 && t->shape[i] != shape[i])
      return fail(MSSM_ERR_INVALID_ARG, "%s: dim %d is %lld, expected %lld", name, i,
                  (long long)t->shape[i], (long long)shape[i]);
    numel *= t->shape[i];
  }
  if (t->dtype != dtype)
    return fail(MSSM_ERR_INVALID_ARG, "%s: dtype %s, expected %s", name, dname(t->dtype), dname(dtype));
  if (numel > 0 && !t->data) return fail(MSSM_ERR_INVALID_ARG, "%s: null data pointer", name);
  if (inner_contig && numel > 0 && t->shape[ndim - 1] > 1 && t->stride[ndim - 1] != 1)
    return fail(MSSM_ERR_UNSUPPORTED, "%s: innermost stride must be 1", name);
  if (!aligned16(t->data) && (reinterpret_cast<uintptr_t>(t->data) % esize(dtype)) != 0)
    return fail(MSSM_ERR_INVALID_ARG, "%s: data pointer not aligned to its element size", name);
  return MSSM_OK;
}

// rows of a [.., .., L] tensor start on 16-byte boundaries
bool rows_vec(const mssm_tensor* t) {
  const int64_t es = int64_t(esize(t->dtype));
  return aligned16(t->data) && (t->stride[0] * es) % 16 == 0 && (t->stride[1] * es) % 16 == 0;
}

bool same_ptr(const mssm_tensor* a, const mssm_tensor* b) {
  return a && b && a->data && a->data == b->data;
}

// Launch shape of the scan.
//   mode 0: one forward kernel over whole sequences (nseg == 1)
//   mode 1: chunk-summary kernel + forward kernel over nseg chunks
//   mode 2: persistent chained forward kernel (`grid` one-warp CTAs)
//   mode 3: fused single pass (`grid` one-warp CTAs)
//   mode 4: split chunks (`grid` persistent CTAs of kSplitWarps warps; a chunk of seg steps is
//           kSplitWarps sub-segments summarised, combined and swept by one warp each)
// rows: channels per row tile; rpt: rows per thread (rows / rpt threads per CTA).
struct LaunchShape {
  int mode;
  int rows;
  int rpt;
  int64_t seg, nseg;
  int grid;
};

int64_t round_seg(int64_t v) {
  v = ((v + mssm::kSegQuant - 1) / mssm::kSegQuant) * mssm::kSegQuant;
  return v < mssm::kSegQuant ? mssm::kSegQuant : v;
}

// Cost model, in cycles of the busiest SM sub-partition (SMSP).  Measured on B200:
// cycles per 32 elements one SMSP spends on the forward sweep (cyc_out) and on the
// chunk summaries (cyc_sum), by rows per thread and by the warps resident on the SMSP
// (one warp cannot hide its own latencies; two or more reach the same rate).  A CTA
// costs kStart cycles of start-up latency per wave, a launch kLaunch, a chained work
// item kItem, and the carry fold kFold per chunk.  Grid kernels run their CTAs in waves
// of at most out_ctas per SM (register and shared-memory limited) and put
// ceil(warps / 4) warps on the busiest SMSP.
//
// Packed sequences (total_len >= 0: the sum of the Bt sequence lengths, each at most L)
// count only the chunks that hold steps, about total_len / seg + Bt per row tile column,
// and pay the forward-sweep summary.  A chained tile runs its chunks one after another,
// so the chained schedule costs at least nseg items, which is what rules it out for a
// few long sequences among short ones.
struct TileKind {
  int rows, rpt;
};
// Measured on B200 (bf16 I/O, gate, softplus + bias, structured A), SMSP cycles per 32
// elements by the warps resident on the busiest SMSP: forward sweep, one row per thread,
// about 160 with two warps (the chained kernel at 8 per SM), 147 with four (64-row CTAs at
// 16 per SM); two rows per thread 150 with three or more but 221 with one (half the warps
// for the same rows); chunk summaries 86 (one row per thread) and 95 (two).  One warp per
// SMSP is extrapolated.  The split-chunk schedule costs a forward sweep, a summary and about 14
// cycles of composition and hand-over per 32 elements.
double cyc_out(int rpt, int64_t k) {
  if (rpt == 1) return k <= 1 ? 190.0 : k == 2 ? 160.0 : k == 3 ? 155.0 : 147.0;
  return k <= 1 ? 221.0 : k == 2 ? 185.0 : 150.0;
}
double cyc_sum(int rpt, int64_t k, bool fwd_sweep) {
  if (fwd_sweep) return cyc_out(rpt, k) * 0.7;  // measured 0.67-0.73 of the forward kernel
  if (rpt == 1) return k <= 1 ? 110.0 : k == 2 ? 95.0 : 86.0;
  return k <= 1 ? 120.0 : k == 2 ? 105.0 : 95.0;
}
constexpr double kSplitCombine = 14.0;
int out_ctas(int rows, int rpt) {  // resident CTAs per SM of the grid kernels
  if (rpt == 1) return rows == 32 ? 9 : 8;
  return rows == 64 ? 12 : 6;
}

LaunchShape choose_shape(int64_t Bt, int64_t D, int64_t L, int sms, int64_t forced_seg, int forced_mode,
                         int forced_rows, int forced_rpt, int dtype, int64_t total_len = -1) {
  // kCta: each CTA's own start (its first B/C stage and input blocks arriving), paid by every
  // warp of the busiest SMSP in turn
  constexpr double kStart = 4000.0, kLaunch = 6000.0, kItem = 4000.0, kFold = 200.0, kCta = 3000.0;
  const bool packed = total_len >= 0;
  // forced tile shapes that do not exist fall back to the nearest that does
  if (dtype != MSSM_BF16) {
    if (forced_rpt == 2) forced_rpt = 1;
    if (forced_rows == 128) forced_rows = 64;
  }
  if ((forced_rows == 32 && forced_rpt == 2) || (forced_rows == 128 && forced_rpt == 1)) forced_rpt = 0;
  // row tile kinds: two rows per thread are built for bf16 I/O only, and are planned only
  // when forced (measured no faster than one row per thread on any benchmark shape)
  std::vector<TileKind> kinds = {{32, 1}, {64, 1}};
  if (dtype == MSSM_BF16 && (forced_rpt == 2 || forced_rows == 128)) {
    kinds.push_back({64, 2});
    kinds.push_back({128, 2});
  }
  auto grid_time = [&](int64_t ctas, const TileKind& tk, double steps, bool sum) {
    const int nt = tk.rows / tk.rpt;
    const int64_t max_cta = out_ctas(tk.rows, tk.rpt);
    const int64_t on_sm = (ctas + sms - 1) / sms;
    const int64_t waves = (on_sm + max_cta - 1) / max_cta;
    const int64_t resident = on_sm < max_cta ? on_sm : max_cta;
    const int64_t k = (resident * (nt / 32) + 3) / 4;
    const double cyc = sum ? cyc_sum(tk.rpt, k, packed) : cyc_out(tk.rpt, k);
    return double(waves) * (double(k) * (steps * tk.rpt * cyc + kCta) + kStart) + kLaunch;
  };
  const int def_rows = forced_rows ? forced_rows : (forced_rpt == 2 ? 64 : 32);
  const int def_rpt = forced_rpt ? forced_rpt : (def_rows == 128 ? 2 : 1);
  LaunchShape best{0, def_rows, def_rpt, L > 0 ? L : 1, 1, 0};
  double best_cost = -1.0;
  auto consider = [&](const LaunchShape& sh, double cost) {
    if (forced_mode >= 0 && sh.mode != forced_mode) return;
    if (best_cost < 0.0 || cost < best_cost * 0.999) {
      best_cost = cost;
      best = sh;
    }
  };
  for (const TileKind& tk : kinds) {
    if (forced_rows && tk.rows != forced_rows) continue;
    if (forced_rpt && tk.rpt != forced_rpt) continue;
    const int64_t tpb = (D + tk.rows - 1) / tk.rows;
    const int64_t tiles = Bt * tpb;
    const bool one_warp = tk.rows / tk.rpt == 32;  // tile kinds of the persistent kernels
    for (int64_t want = 1; want <= 64; ++want) {
      int64_t seg = forced_seg > 0 ? forced_seg : round_seg((L + want - 1) / want);
      int64_t nseg = L > 0 ? (L + seg - 1) / seg : 1;
      while (nseg > 65535) {
        seg *= 2;
        nseg = (L + seg - 1) / seg;
      }
      if (forced_mode == 0) nseg = 1, seg = L > 0 ? L : 1;
      // CTAs (items) that hold steps; the rest of a packed grid exits at once
      int64_t out_items = tiles * nseg, sum_items = tiles * (nseg - 1);
      if (packed) {
        out_items = std::min<int64_t>(out_items, tpb * ((total_len + seg - 1) / seg + Bt));
        sum_items = std::min<int64_t>(sum_items, tpb * (total_len / seg));
      }
      double cost = grid_time(out_items, tk, double(seg), false);
      if (nseg > 1) cost += grid_time(sum_items, tk, double(seg), true) + kFold * double(nseg);
      if (packed) {
        // packed sequences: most CTAs hold fewer than seg steps, so count the work itself
        // (every tile sweeps and summarises total_len steps, each CTA's warps pay their
        // start) at the SMSP rate of a full SM of this kind, plus a tail of kPackedTail of
        // one item's duration (the last items run on a draining GPU), and no less than
        // that duration (a chunk of the longest sequence is swept by one warp).  Fitted to the
        // chunk-length sweep of 32 sequences of up to 4096 steps (27048 in all) x 1536
        // channels: 4-6% above the measured times at chunks of 128 to 512, in their order.
        constexpr double kPackedTail = 0.15;
        const double smsps = 4.0 * double(sms), wpt = double(tk.rows / tk.rpt) / 32.0;
        const int64_t kf = (int64_t(out_ctas(tk.rows, tk.rpt)) * (tk.rows / tk.rpt / 32) + 3) / 4;
        const double c_out = tk.rpt * cyc_out(tk.rpt, kf), c_sum = tk.rpt * cyc_sum(tk.rpt, kf, true);
        const double per_step = double(tpb) * wpt * double(total_len) / smsps;
        cost = per_step * c_out + double(out_items) * wpt * kCta / smsps + kStart + kLaunch;
        if (nseg > 1)
          cost += per_step * c_sum + double(sum_items) * wpt * kCta / smsps + kStart + kLaunch + kFold * double(nseg);
        const double item = double(seg) * double(kf) * (c_out + (nseg > 1 ? c_sum : 0.0));
        cost = std::max(cost + kPackedTail * item, item);  // ... and never below one item's own sweep
      }
      consider(LaunchShape{nseg > 1 ? 1 : 0, tk.rows, tk.rpt, seg, nseg, 0}, cost);
      if (one_warp && nseg > 1) {
        const int64_t cap = int64_t(tk.rpt == 1 ? 8 : 12) * sms;  // resident one-warp CTAs
        // fused single pass (forced only): persistent one-warp CTAs
        if (forced_mode == 3 && !packed)
          consider(LaunchShape{3, tk.rows, tk.rpt, seg, nseg, int(std::min<int64_t>(tiles * nseg, cap))}, 0.0);
        // chained, forced: never more CTAs than tiles
        if (forced_mode == 2 && tiles < cap)
          consider(LaunchShape{2, tk.rows, tk.rpt, seg, nseg, int(std::min<int64_t>(tiles, cap))}, 0.0);
        // split chunks (forced only: measured slower than summaries + forward on every
        // benchmark shape): a chunk is kSplitWarps sub-segments of whole summary blocks
        if (forced_mode == 4 && !packed && seg % (mssm::kSplitWarps * mssm::kSegQuant) == 0) {
          const int64_t grid = std::min<int64_t>(tiles * nseg, int64_t(3) * sms);
          const int64_t k = 3;  // warps per SMSP (3 CTAs of 4 warps per SM)
          const int64_t rounds = (tiles * nseg + grid - 1) / grid;
          const double sub = double(seg) / mssm::kSplitWarps;
          const double item =
              sub * tk.rpt * (cyc_out(tk.rpt, k) + cyc_sum(tk.rpt, k, false) + kSplitCombine) * double(k) + kItem;
          consider(LaunchShape{4, tk.rows, tk.rpt, seg, nseg, int(grid)},
                   double(rounds) * item + kLaunch + kStart * double(nseg));
        }
        const int64_t per_sm = std::min<int64_t>(tiles / sms, tk.rpt == 1 ? 8 : 12);
        if (per_sm >= 4) {
          // each CTA takes whole items from a ticket, so the items run in about items / grid
          // rounds plus a tail of a quarter round (fitted to the measured chunk-length choices
          // of 8 x 5120 x 1024, 64 x 1536 x 512, 8 x 5120 x 4096 and 8 x 5120 x 16384), and in
          // no fewer rounds than the tile's chain of chunks; k warps share an SMSP
          constexpr double kChainTail = 0.25;
          const int64_t grid = per_sm * sms;
          const int64_t k = (per_sm + 3) / 4;
          const double rounds = std::max(double(out_items) / double(grid) + kChainTail, double(nseg));
          const double item = double(seg) * tk.rpt * cyc_out(tk.rpt, k) * double(k) + kItem;
          consider(LaunchShape{2, tk.rows, tk.rpt, seg, nseg, int(grid)}, rounds * item + kLaunch);
        }
      }
      if (forced_mode == 0 || forced_seg > 0 || L <= mssm::kSegQuant) break;
    }
  }
  return best;
}

}  // namespace

extern "C" {

const char* mssm_version(void) { return "0.1.0"; }

const char* mssm_status_string(mssm_status s) {
  switch (s) {
    case MSSM_OK: return "MSSM_OK";
    case MSSM_ERR_INVALID_ARG: return "MSSM_ERR_INVALID_ARG";
    case MSSM_ERR_UNSUPPORTED: return "MSSM_ERR_UNSUPPORTED";
    case MSSM_ERR_CUDA: return "MSSM_ERR_CUDA";
    case MSSM_ERR_TIMEOUT: return "MSSM_ERR_TIMEOUT";
  }
  return "MSSM_ERR_UNKNOWN";
}

const char* mssm_last_error(void) { return g_last_error.c_str(); }

mssm_status mssm_set_option(int option, int64_t value) {
  std::lock_guard<std::mutex> lk(g_mu);
  switch (option) {
    case MSSM_OPT_FORCE_GENERAL_A:
      if (value != 0 && value != 1) return fail(MSSM_ERR_INVALID_ARG, "FORCE_GENERAL_A takes 0 or 1");
      g_force_general = int(value);
      return MSSM_OK;
    case MSSM_OPT_CHUNK_LEN:
      if (value < 0 || value % mssm::kSegQuant != 0 || value > (int64_t(1) << 30))
        return fail(MSSM_ERR_INVALID_ARG, "CHUNK_LEN must be 0 or a positive multiple of %d", mssm::kSegQuant);
      g_chunk_len = value;
      return MSSM_OK;
    case MSSM_OPT_SCHEDULE:
      if (value < 0 || value > 5) return fail(MSSM_ERR_INVALID_ARG, "SCHEDULE takes 0 (automatic) to 5");
      g_schedule = int(value) - 1;
      return MSSM_OK;
    case MSSM_OPT_ROWS_PER_CTA:
      if (value != 0 && value != 32 && value != 64 && value != 128)
        return fail(MSSM_ERR_INVALID_ARG, "ROWS_PER_CTA takes 0, 32, 64 or 128");
      g_rows_per_cta = int(value);
      return MSSM_OK;
    case MSSM_OPT_ROWS_PER_THREAD:
      if (value < 0 || value > 2) return fail(MSSM_ERR_INVALID_ARG, "ROWS_PER_THREAD takes 0, 1 or 2");
      g_rows_per_thread = int(value);
      return MSSM_OK;
    case MSSM_OPT_TEST_HOOKS:
      if (value < 0 || value > 1) return fail(MSSM_ERR_INVALID_ARG, "TEST_HOOKS takes 0 or 1");
      g_test_hooks = int(value);
      return MSSM_OK;
    case MSSM_OPT_DECODE_PATH:
      if (value < 0 || value > 3) return fail(MSSM_ERR_INVALID_ARG, "DECODE_PATH takes 0 (automatic) to 3");
      g_decode_path = int(value);
      return MSSM_OK;
    case MSSM_OPT_KERNEL_TIMING:
      if (value != 0 && value != 1) return fail(MSSM_ERR_INVALID_ARG, "KERNEL_TIMING takes 0 or 1");
      g_timing = int(value);
      return MSSM_OK;
  }
  return fail(MSSM_ERR_INVALID_ARG, "unknown option %d", option);
}

}  // extern "C"

namespace {

// Validation and kernel arguments of a scan call, shared by both scan entry points.
struct ScanCall {
  mssm::ScanArgs a{};
  int dtype = 0;
  bool has_z = false;
  bool softplus = false;
  bool noop = false;       // Bt * D == 0: nothing to launch
  int64_t Bt = 0, D = 0, L = 0;  // as planned: packed sequences plan S x D x max_seqlen
  int64_t total_len = -1;        // packed sequences: their summed length (the packed row's T)
};

// state_batches: the leading size of last_state (and h0) when it is not Bt (packed
// sequences: their count), else -1.
mssm_status scan_prepare(const mssm_tensor* u, const mssm_tensor* delta, const mssm_tensor* A,
                         const mssm_tensor* B, const mssm_tensor* C, const mssm_tensor* D,
                         const mssm_tensor* z, const mssm_tensor* delta_bias, int softplus_flag,
                         mssm_tensor* out, mssm_tensor* last_state, ScanCall& call,
                         int64_t state_batches = -1) {
  if (!u) return fail(MSSM_ERR_INVALID_ARG, "u: null tensor descriptor");
  if (u->ndim != 3) return fail(MSSM_ERR_INVALID_ARG, "u: expected 3 dims [Bt, D, L]");
  const int dt = u->dtype;
  if (dt != MSSM_F32 && dt != MSSM_BF16) return fail(MSSM_ERR_INVALID_ARG, "u: dtype must be f32 or bf16");
  if (!A || A->ndim != 2) return fail(MSSM_ERR_INVALID_ARG, "A: expected 2 dims [D, N]");
  const int64_t Bt = u->shape[0], Dd = u->shape[1], L = u->shape[2], N = A->shape[1];
  if (N != mssm::kN)
    return fail(MSSM_ERR_UNSUPPORTED, "state size N = %lld; this build supports N = %d", (long long)N, mssm::kN);
  const int64_t s_bdl[3] = {Bt, Dd, L}, s_bnl[3] = {Bt, N, L}, s_dn[2] = {Dd, N}, s_d[1] = {Dd},
                s_bdn[3] = {state_batches >= 0 ? state_batches : Bt, Dd, N};
  mssm_status st;
  if ((st = check(u, "u", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if ((st = check(delta, "delta", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if ((st = check(A, "A", 2, s_dn, MSSM_F32, false)) != MSSM_OK) return st;
  if ((st = check(B, "B", 3, s_bnl, dt, true)) != MSSM_OK) return st;
  if ((st = check(C, "C", 3, s_bnl, dt, true)) != MSSM_OK) return st;
  if (D && (st = check(D, "D", 1, s_d, MSSM_F32, false)) != MSSM_OK) return st;
  if (z && (st = check(z, "z", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if (delta_bias && (st = check(delta_bias, "delta_bias", 1, s_d, MSSM_F32, false)) != MSSM_OK) return st;
  if ((st = check(out, "out", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if (last_state && (st = check(last_state, "last_state", 3, s_bdn, MSSM_F32, true)) != MSSM_OK) return st;
  if (Bt > INT32_MAX || Dd > INT32_MAX || L > INT32_MAX - 2 * mssm::kSegQuant)
    return fail(MSSM_ERR_UNSUPPORTED, "Bt, D and L must each fit in 31 bits");
  if (Bt * Dd > int64_t(INT32_MAX) || (state_batches >= 0 && state_batches * Dd > int64_t(INT32_MAX)))
    return fail(MSSM_ERR_UNSUPPORTED, "Bt * D (or the sequence count * D) must fit in 31 bits");
  const mssm_tensor* ins[] = {u, delta, B, C, z, A, D, delta_bias};
  for (const mssm_tensor* t : ins)
    if (same_ptr(out, t)) return fail(MSSM_ERR_INVALID_ARG, "out must not alias an input");
  if (last_state)
    for (const mssm_tensor* t : ins)
      if (same_ptr(last_state, t)) return fail(MSSM_ERR_INVALID_ARG, "last_state must not alias an input");
  call.dtype = dt;
  call.has_z = z != nullptr;
  call.softplus = softplus_flag != 0;
  call.Bt = Bt;
  call.D = Dd;
  call.L = L;
  call.noop = (Bt == 0 || Dd == 0);
  if (call.noop) return MSSM_OK;

  mssm::ScanArgs& a = call.a;
  a.u = u->data; a.delta = delta->data; a.z = z ? z->data : nullptr; a.out = out->data;
  a.u_sb = u->stride[0]; a.u_sd = u->stride[1];
  a.dl_sb = delta->stride[0]; a.dl_sd = delta->stride[1];
  a.z_sb = z ? z->stride[0] : 0; a.z_sd = z ? z->stride[1] : 0;
  a.o_sb = out->stride[0]; a.o_sd = out->stride[1];
  a.B = B->data; a.C = C->data;
  a.B_sb = B->stride[0]; a.B_sn = B->stride[1]; a.C_sb = C->stride[0]; a.C_sn = C->stride[1];
  a.A = static_cast<const float*>(A->data); a.A_sd = A->stride[0]; a.A_sn = A->stride[1];
  a.Dskip = D ? static_cast<const float*>(D->data) : nullptr; a.D_s = D ? D->stride[0] : 0;
  a.bias = delta_bias ? static_cast<const float*>(delta_bias->data) : nullptr;
  a.bias_s = delta_bias ? delta_bias->stride[0] : 0;
  a.last_state = last_state ? static_cast<float*>(last_state->data) : nullptr;
  a.ls_sb = last_state ? last_state->stride[0] : 0; a.ls_sd = last_state ? last_state->stride[1] : 0;
  a.Bt = int(Bt); a.D = int(Dd); a.L = int(L);
  a.vec_rows = rows_vec(u) && rows_vec(delta) && rows_vec(out) && (!z || rows_vec(z));
  a.vec_bc = rows_vec(B) && rows_vec(C);
  a.vec_ls = last_state && aligned16(last_state->data) && (last_state->stride[0] * 4) % 16 == 0 &&
             (last_state->stride[1] * 4) % 16 == 0;
  return MSSM_OK;
}

// First checks of an mssm_scan_ext; returns the packed-sequence count through nseq
// (-1 without cu_seqlens).
mssm_status scan_ext_header(const mssm_scan_ext* ext, int64_t* nseq) {
  *nseq = -1;
  if (!ext) return MSSM_OK;
  if (ext->struct_size < int32_t(sizeof(mssm_scan_ext)))
    return fail(MSSM_ERR_INVALID_ARG, "ext->struct_size = %d; expected at least %d", int(ext->struct_size),
                int(sizeof(mssm_scan_ext)));
  if (ext->discretization != MSSM_DISC_EULER && ext->discretization != MSSM_DISC_ZOH)
    return fail(MSSM_ERR_INVALID_ARG, "ext->discretization must be MSSM_DISC_EULER or MSSM_DISC_ZOH");
  const mssm_tensor* cu = ext->cu_seqlens;
  if (cu) {
    const int64_t any[1] = {-1};
    mssm_status st = check(cu, "cu_seqlens", 1, any, MSSM_I32, true);
    if (st != MSSM_OK) return st;
    if (cu->shape[0] < 1) return fail(MSSM_ERR_INVALID_ARG, "cu_seqlens: expected S + 1 >= 1 offsets");
    if (cu->shape[0] - 1 > INT32_MAX) return fail(MSSM_ERR_UNSUPPORTED, "too many sequences");
    *nseq = cu->shape[0] - 1;
  }
  return MSSM_OK;
}

// The optional inputs of mssm_selective_scan_fwd_ex: initial state, discretisation and
// packed sequences (after scan_prepare has checked the main tensors).
mssm_status scan_prepare_ext(const mssm_scan_ext* ext, const mssm_tensor* out, const mssm_tensor* last_state,
                             ScanCall& call) {
  if (!ext) return MSSM_OK;
  call.a.zoh = ext->discretization == MSSM_DISC_ZOH;
  const mssm_tensor* cu = ext->cu_seqlens;
  if (cu) {
    if (call.Bt != 1)
      return fail(MSSM_ERR_INVALID_ARG, "with cu_seqlens, u/delta/z/out must be [1, D, T] (got Bt = %lld)",
                  (long long)call.Bt);
    const int64_t S = cu->shape[0] - 1;
    if (ext->max_seqlen < 0 || ext->max_seqlen > call.L)
      return fail(MSSM_ERR_INVALID_ARG, "max_seqlen = %lld must lie in [0, T = %lld]",
                  (long long)ext->max_seqlen, (long long)call.L);
    // plan as S independent rows of max_seqlen steps; the kernels read each sequence's range
    call.total_len = call.L;
    call.Bt = S;
    call.L = ext->max_seqlen;
    call.noop = (S == 0 || call.D == 0);
    call.a.Bt = int(S);
    call.a.cu_seqlens = static_cast<const int*>(cu->data);
  }
  const mssm_tensor* h0 = ext->h0;
  if (h0) {
    const int64_t s_bdn[3] = {call.Bt, call.D, mssm::kN};
    mssm_status st = check(h0, "h0", 3, s_bdn, MSSM_F32, true);
    if (st != MSSM_OK) return st;
    if (same_ptr(h0, out) || same_ptr(h0, last_state))
      return fail(MSSM_ERR_INVALID_ARG, "h0 must not alias out or last_state");
    if (call.noop) return MSSM_OK;
    call.a.h0 = static_cast<const float*>(h0->data);
    call.a.h0_sb = h0->stride[0];
    call.a.h0_sd = h0->stride[1];
    call.a.vec_h0 = aligned16(h0->data) && (h0->stride[0] * 4) % 16 == 0 && (h0->stride[1] * 4) % 16 == 0;
  }
  return MSSM_OK;
}

// Plans the launch (caller holds g_mu) and returns the carry workspace layout.
struct ScanPlan {
  int mode = 0;
  int rows_per_cta = 64;
  int rpt = 1;            // rows per thread
  int grid = 0;
  int64_t nseg = 1;
  // mode 1: arrival counters, chunk sums, chunk end states
  // mode 2: ticket + per-tile flags (count_bytes, zeroed per call), carried states (h_bytes)
  size_t count_bytes = 0, s_bytes = 0, h_bytes = 0;
  size_t need() const { return mode != 0 ? count_bytes + s_bytes + h_bytes : 0; }
};

ScanPlan scan_plan(ScanCall& call, int sm_count) {
  mssm::ScanArgs& a = call.a;
  a.force_general = g_force_general;
  a.test_no_publish = g_test_hooks & 1;
  const LaunchShape shape = choose_shape(call.Bt, call.D, call.L, sm_count, g_chunk_len, g_schedule, g_rows_per_cta,
                                         g_rows_per_thread, call.dtype, call.total_len);
  ScanPlan plan;
  plan.mode = shape.mode;
  plan.rows_per_cta = shape.rows;
  plan.rpt = shape.rpt;
  plan.grid = shape.grid;
  plan.nseg = shape.nseg;
  a.tiles_per_batch = int((call.D + shape.rows - 1) / shape.rows);
  const int64_t tiles = call.Bt * a.tiles_per_batch;
  a.seg_len = int(shape.seg);
  a.nseg = int(shape.nseg);
  if (shape.mode == 1) {
    const int64_t rows_total = tiles * shape.rows;
    plan.count_bytes = ((size_t(tiles) * 4 + 255) / 256) * 256;
    plan.s_bytes = ((size_t(shape.nseg - 1) * rows_total * 4 + 255) / 256) * 256;
    plan.h_bytes = size_t(shape.nseg - 1) * rows_total * mssm::kN * 4;
  } else if (shape.mode == 2 || shape.mode == 4) {
    plan.count_bytes = ((size_t(tiles + 1) * 4 + 255) / 256) * 256;
    plan.h_bytes = size_t(tiles) * shape.rows * mssm::kN * 4;
  } else if (shape.mode == 3) {
    const size_t recs = size_t(tiles) * size_t(shape.nseg);
    plan.count_bytes = ((size_t(recs + 1) * 4 + 255) / 256) * 256;
    plan.s_bytes = ((recs * shape.rows * 4 + 255) / 256) * 256;
    plan.h_bytes = 2 * recs * shape.rows * mssm::kN * 4;  // summaries and end states
  }
  return plan;
}

void scan_bind_workspace(mssm::ScanArgs& a, const ScanPlan& plan, void* ws) {
  char* base = static_cast<char*>(ws);
  if (plan.mode == 2 || plan.mode == 4) {
    a.ch_ticket = reinterpret_cast<unsigned*>(base);
    a.ch_flags = reinterpret_cast<unsigned*>(base) + 1;
    a.ch_carry = reinterpret_cast<float*>(base + plan.count_bytes);
    return;
  }
  if (plan.mode == 3) {
    a.ch_ticket = reinterpret_cast<unsigned*>(base);
    a.lb_flags = reinterpret_cast<unsigned*>(base) + 1;
    a.lb_S = reinterpret_cast<float*>(base + plan.count_bytes);
    a.lb_H = reinterpret_cast<float*>(base + plan.count_bytes + plan.s_bytes);
    a.lb_I = a.lb_H + plan.h_bytes / 8;
    return;
  }

  a.ws_count = reinterpret_cast<unsigned*>(base);
  a.ws_S = reinterpret_cast<float*>(base + plan.count_bytes);
  a.ws_H = reinterpret_cast<float*>(base + plan.count_bytes + plan.s_bytes);
}

// The kernel launches of a planned call (caller holds g_mu).  `ws` is the
// workspace base the plan was bound to (mode 2 zeroes its ticket and flags).
mssm_status scan_launch(ScanCall& call, const ScanPlan& plan, void* ws, cudaStream_t s) {
  cudaError_t e = mssm::device_error_word(&call.a.err);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  if (plan.mode == 3) {
    e = cudaMemsetAsync(ws, 0, plan.count_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(fused schedule flags)");
    e = tracked(MSSM_KERNEL_SCAN_OUT, s, [&] {
      return mssm::launch_scan_fused(call.a, plan.grid, plan.rpt, call.dtype, call.has_z, call.softplus, s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "fused scan kernel launch");
    return MSSM_OK;
  }
  if (plan.mode == 4) {
    e = cudaMemsetAsync(ws, 0, plan.count_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(split schedule flags)");
    e = tracked(MSSM_KERNEL_SCAN_OUT, s, [&] {
      return mssm::launch_scan_split(call.a, plan.grid, plan.rpt, call.dtype, call.has_z, call.softplus, s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "split scan kernel launch");
    return MSSM_OK;
  }
  if (plan.mode == 2) {
    e = cudaMemsetAsync(ws, 0, plan.count_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(chained schedule flags)");
    e = tracked(MSSM_KERNEL_SCAN_OUT, s, [&] {
      return mssm::launch_scan_chained(call.a, plan.grid, plan.rpt, call.dtype, call.has_z, call.softplus, s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "chained scan kernel launch");
    return MSSM_OK;
  }
  if (plan.nseg > 1) {
    e = tracked(MSSM_KERNEL_SCAN_CHUNK_STATE, s, [&] {
      return mssm::launch_scan_chunk_state(call.a, plan.rows_per_cta, plan.rpt, call.dtype, call.softplus, s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "chunk-state kernel launch");
  }
  e = tracked(MSSM_KERNEL_SCAN_OUT, s, [&] {
    return mssm::launch_scan_out(call.a, plan.rows_per_cta, plan.rpt, call.dtype, call.has_z, call.softplus, s);
  });
  if (e != cudaSuccess) return cuda_fail(e, "scan kernel launch");
  return MSSM_OK;
}

// The allocating scan of a prepared call: plan, grow the workspace if needed, launch.
mssm_status scan_fwd_impl(ScanCall& call, void* stream) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = device_state(dev);
  const ScanPlan plan = scan_plan(call, ds->sm_count);
  if (plan.mode >= 2) {
    // ticket, flags and carried states: zeroed by scan_launch where they must be
    const size_t need = plan.need() + size_t(ds->count_cap) * 4;
    if (ds->ws_bytes < need) {
      if (ds->ws) {
        e = cudaFree(ds->ws);  // synchronises the device
        ds->ws = nullptr;
        ds->ws_bytes = 0;
        ds->count_cap = 0;
        if (e != cudaSuccess) return cuda_fail(e, "cudaFree(workspace)");
      }
      e = cudaMalloc(&ds->ws, need);
      if (e != cudaSuccess) {
        ds->ws = nullptr;
        return cuda_fail(e, "cudaMalloc(workspace)");
      }
      ds->ws_bytes = need;
      e = cudaMemsetAsync(ds->ws, 0, need, s);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
    }
    // after the arrival counters of mode 1, which must keep their zeros
    void* base = static_cast<char*>(ds->ws) + size_t(ds->count_cap) * 4;
    scan_bind_workspace(call.a, plan, base);
    return scan_launch(call, plan, base, s);
  }
  if (plan.nseg > 1) {
    // The arrival counters keep a region of their own at the start of the
    // workspace, sized for the most row tiles seen so far: they start at zero
    // and every complete call leaves them at zero, so they are never cleared
    // per call.  (Sharing the counters' bytes with the summaries of a call with
    // more tiles would leave non-zero counters behind.)
    const int64_t tiles = plan.count_bytes / 4;
    const int64_t cap = tiles > ds->count_cap ? tiles : ds->count_cap;
    ScanPlan layout = plan;
    layout.count_bytes = ((size_t(cap) * 4 + 255) / 256) * 256;
    const size_t need = layout.need();
    if (ds->ws_bytes < need || cap > ds->count_cap) {
      if (ds->ws) {
        e = cudaFree(ds->ws);  // synchronises the device
        ds->ws = nullptr;
        ds->ws_bytes = 0;
        ds->count_cap = 0;
        if (e != cudaSuccess) return cuda_fail(e, "cudaFree(workspace)");
      }
      e = cudaMalloc(&ds->ws, need);
      if (e != cudaSuccess) {
        ds->ws = nullptr;
        return cuda_fail(e, "cudaMalloc(workspace)");
      }
      ds->ws_bytes = need;
      ds->count_cap = int64_t(layout.count_bytes / 4);
      e = cudaMemsetAsync(ds->ws, 0, need, s);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
    }
    layout.count_bytes = size_t(ds->count_cap) * 4;
    scan_bind_workspace(call.a, layout, ds->ws);
  }
  return scan_launch(call, plan, ds->ws, s);
}

}  // namespace

extern "C" {

mssm_status mssm_selective_scan_fwd(const mssm_tensor* u, const mssm_tensor* delta,
                                    const mssm_tensor* A, const mssm_tensor* B,
                                    const mssm_tensor* C, const mssm_tensor* D,
                                    const mssm_tensor* z, const mssm_tensor* delta_bias,
                                    int softplus_flag, mssm_tensor* out, mssm_tensor* last_state,
                                    void* stream) {
  ScanCall call;
  mssm_status st = scan_prepare(u, delta, A, B, C, D, z, delta_bias, softplus_flag, out, last_state, call);
  if (st != MSSM_OK || call.noop) return st;
  return scan_fwd_impl(call, stream);
}

mssm_status mssm_selective_scan_fwd_ex(const mssm_tensor* u, const mssm_tensor* delta,
                                       const mssm_tensor* A, const mssm_tensor* B,
                                       const mssm_tensor* C, const mssm_tensor* D,
                                       const mssm_tensor* z, const mssm_tensor* delta_bias,
                                       int softplus_flag, const mssm_scan_ext* ext, mssm_tensor* out,
                                       mssm_tensor* last_state, void* stream) {
  int64_t nseq = -1;
  mssm_status st = scan_ext_header(ext, &nseq);
  if (st != MSSM_OK) return st;
  ScanCall call;
  st = scan_prepare(u, delta, A, B, C, D, z, delta_bias, softplus_flag, out, last_state, call, nseq);
  if (st != MSSM_OK) return st;
  if ((st = scan_prepare_ext(ext, out, last_state, call)) != MSSM_OK || call.noop) return st;
  return scan_fwd_impl(call, stream);
}

// ---------------------------------------------------------------------------
// Scan without any allocation.  Its carry scratch is a fixed array in the
// library's device image instead of a cudaMalloc'd workspace.  The array lives
// on every GPU that loads this library, from module load until process exit.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[64] = {};  // per-device address of g_noalloc_scratch, set up on first use
int g_noalloc_sms[64] = {};    // per-device SM count, set up on first use

}  // namespace

extern "C" {

mssm_status mssm_selective_scan_fwd_noalloc(const mssm_tensor* u, const mssm_tensor* delta,
                                            const mssm_tensor* A, const mssm_tensor* B,
                                            const mssm_tensor* C, const mssm_tensor* D,
                                            const mssm_tensor* z, const mssm_tensor* delta_bias,
                                            int softplus_flag, mssm_tensor* out,
                                            mssm_tensor* last_state, void* stream) {
  ScanCall call;
  mssm_status st = scan_prepare(u, delta, A, B, C, D, z, delta_bias, softplus_flag, out, last_state, call);
  if (st != MSSM_OK || call.noop) return st;

  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MSSM_ERR_UNSUPPORTED, "device index %d out of range", dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_sms[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_noalloc_sms[dev] = v;
  }
  const ScanPlan plan = scan_plan(call, g_noalloc_sms[dev]);
  if (plan.mode != 0) {
    const size_t need = plan.need();
    if (need > kNoAllocScratchBytes)
      return fail(MSSM_ERR_UNSUPPORTED,
                  "this problem needs %zu bytes of carry scratch; the no-allocation scan has a fixed "
                  "%zu-byte array (use mssm_selective_scan_fwd, or a longer MSSM_OPT_CHUNK_LEN)",
                  need, kNoAllocScratchBytes);
    // First use on this device: look up the array's device address with this
    // device current.  Host code must never pass &g_noalloc_scratch itself.
    if (!g_noalloc_ptr[dev]) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
      g_noalloc_ptr[dev] = ptr;
    }
    // The array keeps whatever the previous call left: zero the arrival
    // counters (the chained schedule zeroes its own ticket and flags).
    if (plan.mode == 1) {
      e = cudaMemsetAsync(g_noalloc_ptr[dev], 0, plan.count_bytes, s);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(no-allocation scratch counters)");
    }
    scan_bind_workspace(call.a, plan, g_noalloc_ptr[dev]);
  }
  return scan_launch(call, plan, g_noalloc_ptr[dev], s);
}

static mssm_status state_update_impl(mssm_tensor* state, const mssm_tensor* x, const mssm_tensor* dt_t,
                                     const mssm_tensor* A, const mssm_tensor* B, const mssm_tensor* C,
                                     const mssm_tensor* D, const mssm_tensor* z, const mssm_tensor* bias,
                                     int softplus_flag, int discretization, mssm_tensor* out, void* stream) {
  if (discretization != MSSM_DISC_EULER && discretization != MSSM_DISC_ZOH)
    return fail(MSSM_ERR_INVALID_ARG, "discretization must be MSSM_DISC_EULER or MSSM_DISC_ZOH");
  if (!x) return fail(MSSM_ERR_INVALID_ARG, "x: null tensor descriptor");
  if (x->ndim != 2) return fail(MSSM_ERR_INVALID_ARG, "x: expected 2 dims [Bt, D]");
  const int dt = x->dtype;
  if (dt != MSSM_F32 && dt != MSSM_BF16) return fail(MSSM_ERR_INVALID_ARG, "x: dtype must be f32 or bf16");
  if (!A || A->ndim != 2) return fail(MSSM_ERR_INVALID_ARG, "A: expected 2 dims [D, N]");
  const int64_t Bt = x->shape[0], Dd = x->shape[1], N = A->shape[1];
  if (N != mssm::kN)
    return fail(MSSM_ERR_UNSUPPORTED, "state size N = %lld; this build supports N = %d", (long long)N, mssm::kN);
  const int64_t s_bd[2] = {Bt, Dd}, s_bn[2] = {Bt, N}, s_dn[2] = {Dd, N}, s_d[1] = {Dd}, s_bdn[3] = {Bt, Dd, N};
  mssm_status st;
  if ((st = check(state, "state", 3, s_bdn, MSSM_F32, true)) != MSSM_OK) return st;
  if ((st = check(x, "x", 2, s_bd, dt, false)) != MSSM_OK) return st;
  if ((st = check(dt_t, "dt", 2, s_bd, dt, false)) != MSSM_OK) return st;
  if ((st = check(A, "A", 2, s_dn, MSSM_F32, false)) != MSSM_OK) return st;
  if ((st = check(B, "B", 2, s_bn, dt, false)) != MSSM_OK) return st;
  if ((st = check(C, "C", 2, s_bn, dt, false)) != MSSM_OK) return st;
  if (D && (st = check(D, "D", 1, s_d, MSSM_F32, false)) != MSSM_OK) return st;
  if (z && (st = check(z, "z", 2, s_bd, dt, false)) != MSSM_OK) return st;
  if (bias && (st = check(bias, "dt_bias", 1, s_d, MSSM_F32, false)) != MSSM_OK) return st;
  if ((st = check(out, "out", 2, s_bd, dt, false)) != MSSM_OK) return st;
  if (Bt > INT32_MAX || Dd > INT32_MAX) return fail(MSSM_ERR_UNSUPPORTED, "Bt and D must fit in 31 bits");
  const mssm_tensor* ins[] = {x, dt_t, A, B, C, D, z, bias};
  for (const mssm_tensor* t : ins) {
    if (same_ptr(out, t)) return fail(MSSM_ERR_INVALID_ARG, "out must not alias an input");
    if (same_ptr(state, t)) return fail(MSSM_ERR_INVALID_ARG, "state must not alias an input");
  }
  if (same_ptr(out, state)) return fail(MSSM_ERR_INVALID_ARG, "out must not alias state");
  if (Bt == 0 || Dd == 0) return MSSM_OK;
  if (Bt * Dd > int64_t(INT32_MAX)) return fail(MSSM_ERR_UNSUPPORTED, "Bt * D must fit in 31 bits");

  mssm::DecodeArgs a{};
  a.state = static_cast<float*>(state->data);
  a.st_sb = state->stride[0]; a.st_sd = state->stride[1];
  a.x = x->data; a.dt = dt_t->data; a.z = z ? z->data : nullptr; a.out = out->data;
  a.x_sb = x->stride[0]; a.x_sd = x->stride[1];
  a.dt_sb = dt_t->stride[0]; a.dt_sd = dt_t->stride[1];
  a.z_sb = z ? z->stride[0] : 0; a.z_sd = z ? z->stride[1] : 0;
  a.o_sb = out->stride[0]; a.o_sd = out->stride[1];
  a.A = static_cast<const float*>(A->data); a.A_sd = A->stride[0]; a.A_sn = A->stride[1];
  a.B = B->data; a.C = C->data;
  a.B_sb = B->stride[0]; a.B_sn = B->stride[1]; a.C_sb = C->stride[0]; a.C_sn = C->stride[1];
  a.Dskip = D ? static_cast<const float*>(D->data) : nullptr; a.D_s = D ? D->stride[0] : 0;
  a.bias = bias ? static_cast<const float*>(bias->data) : nullptr; a.bias_s = bias ? bias->stride[0] : 0;
  a.Bt = int(Bt); a.D = int(Dd);
  a.softplus = softplus_flag != 0;
  a.zoh = discretization == MSSM_DISC_ZOH;
  a.vec_state = aligned16(state->data) && (state->stride[0] * 4) % 16 == 0 && (state->stride[1] * 4) % 16 == 0;
  a.vec_A = aligned16(A->data) && A->stride[1] == 1 && (A->stride[0] * 4) % 16 == 0;
  const int64_t es = int64_t(esize(dt));
  a.vec_BC = aligned16(B->data) && aligned16(C->data) && B->stride[1] == 1 && C->stride[1] == 1 &&
             (B->stride[0] * es) % 16 == 0 && (C->stride[0] * es) % 16 == 0;

  // one contiguous [rows][16] state range, 16-byte aligned: the bulk-copy kernels
  const bool contiguous = aligned16(state->data) && state->stride[1] == mssm::kN && state->stride[0] == Dd * mssm::kN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  // every per-row input a contiguous, 16-byte aligned run per batch: the streaming kernel
  auto runs = [&](const mssm_tensor* t) {
    return !t || (aligned16(t->data) && t->stride[1] == 1 && (t->stride[0] * es) % 16 == 0);
  };
  const bool streamable = contiguous && runs(x) && runs(dt_t) && runs(z) && a.vec_BC &&
                          (Dd * es) % 16 == 0;
  mssm::DecodePath path = mssm::DecodePath::kPerRow;
  if (g_decode_path != 3 && contiguous) {
    path = (g_decode_path == 2 || !streamable) ? mssm::DecodePath::kBulkTile : mssm::DecodePath::kStream;
  }
  cudaError_t e = tracked(MSSM_KERNEL_STATE_UPDATE, s,
                          [&] { return mssm::launch_state_update(a, dt, z != nullptr, path, s); });
  if (e != cudaSuccess) return cuda_fail(e, "state update launch");
  return MSSM_OK;
}

mssm_status mssm_state_update(mssm_tensor* state, const mssm_tensor* x, const mssm_tensor* dt,
                              const mssm_tensor* A, const mssm_tensor* B, const mssm_tensor* C,
                              const mssm_tensor* D, const mssm_tensor* z, mssm_tensor* out,
                              void* stream) {
  return state_update_impl(state, x, dt, A, B, C, D, z, nullptr, 1, MSSM_DISC_EULER, out, stream);
}

mssm_status mssm_state_update_ex(mssm_tensor* state, const mssm_tensor* x, const mssm_tensor* dt,
                                 const mssm_tensor* A, const mssm_tensor* B, const mssm_tensor* C,
                                 const mssm_tensor* D, const mssm_tensor* z, const mssm_tensor* dt_bias,
                                 int softplus_flag, int discretization, mssm_tensor* out, void* stream) {
  return state_update_impl(state, x, dt, A, B, C, D, z, dt_bias, softplus_flag, discretization, out, stream);
}

mssm_status mssm_selective_scan_bwd(const mssm_tensor* u, const mssm_tensor* delta, const mssm_tensor* A,
                                    const mssm_tensor* B, const mssm_tensor* C, const mssm_tensor* D,
                                    const mssm_tensor* z, const mssm_tensor* delta_bias, int softplus_flag,
                                    const mssm_tensor* dout, mssm_tensor* du, mssm_tensor* ddelta,
                                    mssm_tensor* dA, mssm_tensor* dB, mssm_tensor* dC, mssm_tensor* dD,
                                    mssm_tensor* dz, mssm_tensor* ddelta_bias, void* stream) {
  // the forward's checks, with dout in the place of out (its shape, dtype and layout)
  ScanCall call;
  mssm_status st = scan_prepare(u, delta, A, B, C, D, z, delta_bias, softplus_flag,
                                const_cast<mssm_tensor*>(dout), nullptr, call);
  if (st != MSSM_OK) return st;
  const int dt = u->dtype;
  const int64_t Bt = u->shape[0], Dd = u->shape[1], L = u->shape[2], N = mssm::kN;
  const int64_t s_bdl[3] = {Bt, Dd, L}, s_bnl[3] = {Bt, N, L}, s_dn[2] = {Dd, N}, s_d[1] = {Dd};
  if ((st = check(du, "du", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if ((st = check(ddelta, "ddelta", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if ((st = check(dA, "dA", 2, s_dn, MSSM_F32, true)) != MSSM_OK) return st;
  if ((st = check(dB, "dB", 3, s_bnl, MSSM_F32, true)) != MSSM_OK) return st;
  if ((st = check(dC, "dC", 3, s_bnl, MSSM_F32, true)) != MSSM_OK) return st;
  if (!D != !dD) return fail(MSSM_ERR_INVALID_ARG, "dD must be given exactly when D is");
  if (!z != !dz) return fail(MSSM_ERR_INVALID_ARG, "dz must be given exactly when z is");
  if (!delta_bias != !ddelta_bias)
    return fail(MSSM_ERR_INVALID_ARG, "ddelta_bias must be given exactly when delta_bias is");
  if (dD && (st = check(dD, "dD", 1, s_d, MSSM_F32, true)) != MSSM_OK) return st;
  if (dz && (st = check(dz, "dz", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if (ddelta_bias && (st = check(ddelta_bias, "ddelta_bias", 1, s_d, MSSM_F32, true)) != MSSM_OK) return st;
  // the accumulated gradients are zeroed and atomically added: they must be dense
  auto dense = [](const mssm_tensor* t) {
    int64_t want = 1;
    for (int i = t->ndim - 1; i >= 0; --i) {
      if (t->shape[i] > 1 && t->stride[i] != want) return false;
      want *= t->shape[i];
    }
    return true;
  };
  for (const mssm_tensor* t : {static_cast<const mssm_tensor*>(dA), static_cast<const mssm_tensor*>(dB),
                               static_cast<const mssm_tensor*>(dC), static_cast<const mssm_tensor*>(dD),
                               static_cast<const mssm_tensor*>(ddelta_bias)})
    if (t && !dense(t)) return fail(MSSM_ERR_UNSUPPORTED, "dA, dB, dC, dD and ddelta_bias must be dense");
  const mssm_tensor* ins[] = {u, delta, A, B, C, D, z, delta_bias, dout};
  const mssm_tensor* outs[] = {du, ddelta, dA, dB, dC, dD, dz, ddelta_bias};
  for (const mssm_tensor* o : outs) {
    if (!o) continue;
    for (const mssm_tensor* i : ins)
      if (same_ptr(o, i)) return fail(MSSM_ERR_INVALID_ARG, "gradients must not alias the inputs");
    for (const mssm_tensor* o2 : outs)
      if (o2 != o && same_ptr(o, o2)) return fail(MSSM_ERR_INVALID_ARG, "gradients must not alias each other");
  }
  // chunk length: 32 steps once there are many row tiles (the shorter forward sweep of pass B
  // then pays; measured 6.72 against 6.95 ms on 8 x 5120 x 4096, 1280 tiles), else 64 (with
  // few tiles the per-chunk costs dominate: 315 against 340 us on 2 x 1536 x 2048, 96 tiles);
  // then the grid limits, checked before anything is launched
  const int64_t tpb = (Dd + mssm::kBwdRows - 1) / mssm::kBwdRows;
  const int64_t tiles = Bt * tpb, rows_total = tiles * mssm::kBwdRows;
  int chunk = tiles >= mssm::kBwdShortChunkTiles ? mssm::kBwdChunkShort : mssm::kBwdChunk;
  if ((L + chunk - 1) / chunk > 65535) chunk = mssm::kBwdChunk;  // long sequences keep 64
  const int64_t nseg = (L + chunk - 1) / chunk;
  if (nseg > 65535 || tiles > INT32_MAX) return fail(MSSM_ERR_UNSUPPORTED, "problem too large for the backward grid");
  if (call.noop) return MSSM_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  // zero the accumulated gradients
  cudaError_t e = cudaSuccess;
  auto zero = [&](const mssm_tensor* t, size_t elems) {
    if (t && e == cudaSuccess && elems) e = cudaMemsetAsync(t->data, 0, elems * 4, s);
  };
  zero(dA, size_t(Dd * N));
  zero(dB, size_t(Bt * N * L));
  zero(dC, size_t(Bt * N * L));
  zero(dD, size_t(Dd));
  zero(ddelta_bias, size_t(Dd));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(gradients)");
  if (L == 0) return MSSM_OK;

  // workspace: the chunk summaries (H then the start states, G, S), the incoming gradients Q,
  // and the arrival counters
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  const size_t cnt_b = al(size_t(tiles) * 4);
  const size_t h_b = al(size_t(nseg - 1) * rows_total * mssm::kN * 4);
  const size_t g_b = al(size_t(nseg) * rows_total * mssm::kN * 4), s_b = al(size_t(nseg) * rows_total * 4);
  const size_t need = cnt_b + h_b + 2 * g_b + s_b;
  int dev = -1;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  DeviceState* ds = device_state(dev);
  if (ds->bwd_bytes < need) {
    if (ds->bwd_ws) {
      e = cudaFree(ds->bwd_ws);  // synchronises the device
      ds->bwd_ws = nullptr;
      ds->bwd_bytes = 0;
      if (e != cudaSuccess) return cuda_fail(e, "cudaFree(backward workspace)");
    }
    if ((e = cudaMalloc(&ds->bwd_ws, need)) != cudaSuccess) {
      ds->bwd_ws = nullptr;
      return cuda_fail(e, "cudaMalloc(backward workspace)");
    }
    ds->bwd_bytes = need;
  }
  char* base = static_cast<char*>(ds->bwd_ws);
  unsigned* cnt = reinterpret_cast<unsigned*>(base);
  float* hA = reinterpret_cast<float*>(base + cnt_b);
  float* gB = reinterpret_cast<float*>(base + cnt_b + h_b);
  float* qB = reinterpret_cast<float*>(base + cnt_b + h_b + g_b);
  float* sB = reinterpret_cast<float*>(base + cnt_b + h_b + 2 * g_b);
  if ((e = cudaMemsetAsync(base, 0, cnt_b, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(counters)");

  mssm::BwdArgs b{};
  b.u = u->data; b.delta = delta->data; b.z = z ? z->data : nullptr; b.dout = dout->data;
  b.u_sb = u->stride[0]; b.u_sd = u->stride[1]; b.dl_sb = delta->stride[0]; b.dl_sd = delta->stride[1];
  b.z_sb = z ? z->stride[0] : 0; b.z_sd = z ? z->stride[1] : 0;
  b.g_sb = dout->stride[0]; b.g_sd = dout->stride[1];
  b.B = B->data; b.C = C->data;
  b.B_sb = B->stride[0]; b.B_sn = B->stride[1]; b.C_sb = C->stride[0]; b.C_sn = C->stride[1];
  b.A = static_cast<const float*>(A->data); b.A_sd = A->stride[0]; b.A_sn = A->stride[1];
  b.Dskip = D ? static_cast<const float*>(D->data) : nullptr; b.D_s = D ? D->stride[0] : 0;
  b.bias = delta_bias ? static_cast<const float*>(delta_bias->data) : nullptr;
  b.bias_s = delta_bias ? delta_bias->stride[0] : 0;
  b.du = du->data; b.ddelta = ddelta->data; b.dz = dz ? dz->data : nullptr;
  b.du_sb = du->stride[0]; b.du_sd = du->stride[1]; b.dd_sb = ddelta->stride[0]; b.dd_sd = ddelta->stride[1];
  b.dz_sb = dz ? dz->stride[0] : 0; b.dz_sd = dz ? dz->stride[1] : 0;
  b.dA = static_cast<float*>(dA->data); b.dB = static_cast<float*>(dB->data); b.dC = static_cast<float*>(dC->data);
  b.dD = dD ? static_cast<float*>(dD->data) : nullptr;
  b.dbias = ddelta_bias ? static_cast<float*>(ddelta_bias->data) : nullptr;
  b.Bt = int(Bt); b.D = int(Dd); b.L = int(L);
  b.softplus = softplus_flag != 0;
  b.nseg = int(nseg); b.tiles_per_batch = int(tpb); b.chunk = chunk;
  b.hstart = hA; b.ws_G = gB; b.ws_S = sB; b.ws_Q = qB; b.ws_count = cnt;
  b.vec_rows = rows_vec(u) && rows_vec(delta) && rows_vec(dout) && rows_vec(du) && rows_vec(ddelta) &&
               (!z || (rows_vec(z) && rows_vec(dz)));
  b.force_general = g_force_general;
  e = tracked(MSSM_KERNEL_SCAN_BWD, s, [&] { return mssm::launch_scan_bwd(b, dt, z != nullptr, s); });
  if (e != cudaSuccess) return cuda_fail(e, "backward scan kernel launch");
  return MSSM_OK;
}

mssm_status mssm_causal_conv1d_fwd(const mssm_tensor* x, const mssm_tensor* weight, const mssm_tensor* bias,
                                   const mssm_tensor* cu_seqlens, int64_t max_seqlen, int silu_flag,
                                   mssm_tensor* out, void* stream) {
  if (!x) return fail(MSSM_ERR_INVALID_ARG, "x: null tensor descriptor");
  if (x->ndim != 3) return fail(MSSM_ERR_INVALID_ARG, "x: expected 3 dims [Bt, D, L]");
  const int dt = x->dtype;
  if (dt != MSSM_F32 && dt != MSSM_BF16) return fail(MSSM_ERR_INVALID_ARG, "x: dtype must be f32 or bf16");
  if (!weight || weight->ndim != 2) return fail(MSSM_ERR_INVALID_ARG, "weight: expected 2 dims [D, K]");
  const int64_t Bt = x->shape[0], Dd = x->shape[1], L = x->shape[2], K = weight->shape[1];
  if (K < 1 || K > mssm::kConvMaxK)
    return fail(MSSM_ERR_UNSUPPORTED, "kernel size K = %lld; this build supports 1..%d", (long long)K,
                mssm::kConvMaxK);
  const int64_t s_bdl[3] = {Bt, Dd, L}, s_dk[2] = {Dd, K}, s_d[1] = {Dd}, any[1] = {-1};
  mssm_status st;
  if ((st = check(x, "x", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if ((st = check(out, "out", 3, s_bdl, dt, true)) != MSSM_OK) return st;
  if ((st = check(weight, "weight", 2, s_dk, MSSM_F32, false)) != MSSM_OK) return st;
  if (bias && (st = check(bias, "bias", 1, s_d, MSSM_F32, false)) != MSSM_OK) return st;
  if (same_ptr(out, x)) return fail(MSSM_ERR_INVALID_ARG, "out must not alias x");
  if (Bt > INT32_MAX || Dd > INT32_MAX || L > INT32_MAX / 2 || Bt * Dd > int64_t(INT32_MAX))
    return fail(MSSM_ERR_UNSUPPORTED, "size too large");
  int64_t S = Bt, Lmax = L;
  if (cu_seqlens) {
    if ((st = check(cu_seqlens, "cu_seqlens", 1, any, MSSM_I32, true)) != MSSM_OK) return st;
    if (cu_seqlens->shape[0] < 1) return fail(MSSM_ERR_INVALID_ARG, "cu_seqlens: expected S + 1 >= 1 offsets");
    if (Bt != 1) return fail(MSSM_ERR_INVALID_ARG, "with cu_seqlens, x must be [1, D, T]");
    if (max_seqlen < 0 || max_seqlen > L) return fail(MSSM_ERR_INVALID_ARG, "max_seqlen must lie in [0, T]");
    S = cu_seqlens->shape[0] - 1;
    Lmax = max_seqlen;
    if (S * Dd > int64_t(INT32_MAX)) return fail(MSSM_ERR_UNSUPPORTED, "S * D must fit in 31 bits");
  }
  if (S == 0 || Dd == 0 || Lmax == 0) return MSSM_OK;

  mssm::ConvArgs a{};
  a.x = x->data; a.out = out->data;
  a.x_sb = x->stride[0]; a.x_sd = x->stride[1]; a.o_sb = out->stride[0]; a.o_sd = out->stride[1];
  a.w = static_cast<const float*>(weight->data); a.w_sd = weight->stride[0]; a.w_sk = weight->stride[1];
  a.bias = bias ? static_cast<const float*>(bias->data) : nullptr; a.bias_s = bias ? bias->stride[0] : 0;
  a.Bt = int(S); a.D = int(Dd); a.L = int(L); a.K = int(K);
  a.vec = rows_vec(x) && rows_vec(out);
  a.cu_seqlens = cu_seqlens ? static_cast<const int*>(cu_seqlens->data) : nullptr;
  cudaError_t e = mssm::device_error_word(&a.err);
  if (e != cudaSuccess) return cuda_fail(e, "device error word");
  // warp items of kConvPieces pieces of 32 16-byte blocks
  const int64_t item = int64_t(mssm::kConvPieces) * 32 * (16 / int64_t(esize(dt)));
  const int64_t items64 = (Lmax + item - 1) / item;
  if (items64 > 65535) return fail(MSSM_ERR_UNSUPPORTED, "sequence too long for the conv grid (%lld pieces)",
                                   (long long)items64);
  const int items = int(items64);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  e = tracked(MSSM_KERNEL_CONV, s, [&] { return mssm::launch_causal_conv1d(a, items, dt, silu_flag != 0, s); });
  if (e != cudaSuccess) return cuda_fail(e, "conv1d kernel launch");
  return MSSM_OK;
}

mssm_status mssm_causal_conv1d_update(mssm_tensor* conv_state, const mssm_tensor* x, const mssm_tensor* weight,
                                      const mssm_tensor* bias, int silu_flag, mssm_tensor* out, void* stream) {
  if (!x) return fail(MSSM_ERR_INVALID_ARG, "x: null tensor descriptor");
  if (x->ndim != 2) return fail(MSSM_ERR_INVALID_ARG, "x: expected 2 dims [Bt, D]");
  const int dt = x->dtype;
  if (dt != MSSM_F32 && dt != MSSM_BF16) return fail(MSSM_ERR_INVALID_ARG, "x: dtype must be f32 or bf16");
  if (!weight || weight->ndim != 2) return fail(MSSM_ERR_INVALID_ARG, "weight: expected 2 dims [D, K]");
  const int64_t Bt = x->shape[0], Dd = x->shape[1], K = weight->shape[1];
  if (K < 2 || K > mssm::kConvMaxK)
    return fail(MSSM_ERR_UNSUPPORTED, "kernel size K = %lld; the update supports 2..%d", (long long)K,
                mssm::kConvMaxK);
  const int64_t s_bd[2] = {Bt, Dd}, s_dk[2] = {Dd, K}, s_d[1] = {Dd}, s_st[3] = {Bt, Dd, K - 1};
  mssm_status st;
  if ((st = check(x, "x", 2, s_bd, dt, false)) != MSSM_OK) return st;
  if ((st = check(out, "out", 2, s_bd, dt, false)) != MSSM_OK) return st;
  if ((st = check(conv_state, "conv_state", 3, s_st, dt, false)) != MSSM_OK) return st;
  if ((st = check(weight, "weight", 2, s_dk, MSSM_F32, false)) != MSSM_OK) return st;
  if (bias && (st = check(bias, "bias", 1, s_d, MSSM_F32, false)) != MSSM_OK) return st;
  if (same_ptr(out, x) || same_ptr(out, conv_state) || same_ptr(conv_state, x))
    return fail(MSSM_ERR_INVALID_ARG, "out, x and conv_state must not alias");
  if (Bt * Dd > int64_t(INT32_MAX)) return fail(MSSM_ERR_UNSUPPORTED, "Bt * D must fit in 31 bits");
  if (Bt == 0 || Dd == 0) return MSSM_OK;
  mssm::ConvUpdateArgs a{};
  a.state = conv_state->data;
  a.st_sb = conv_state->stride[0]; a.st_sd = conv_state->stride[1]; a.st_sk = conv_state->stride[2];
  a.x = x->data; a.out = out->data;
  a.x_sb = x->stride[0]; a.x_sd = x->stride[1]; a.o_sb = out->stride[0]; a.o_sd = out->stride[1];
  a.w = static_cast<const float*>(weight->data); a.w_sd = weight->stride[0]; a.w_sk = weight->stride[1];
  a.bias = bias ? static_cast<const float*>(bias->data) : nullptr; a.bias_s = bias ? bias->stride[0] : 0;
  a.Bt = int(Bt); a.D = int(Dd); a.K = int(K);
  a.silu = silu_flag != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_mu);
  cudaError_t e = tracked(MSSM_KERNEL_CONV, s, [&] { return mssm::launch_causal_conv1d_update(a, dt, s); });
  if (e != cudaSuccess) return cuda_fail(e, "conv1d update kernel launch");
  return MSSM_OK;
}

mssm_status mssm_scan_plan(int64_t Bt, int64_t D, int64_t L, int sm_count, int* rows_per_cta,
                           int64_t* chunk_len, int64_t* n_chunks, int* schedule) {
  return mssm_scan_plan_packed(Bt, D, L, -1, sm_count, rows_per_cta, chunk_len, n_chunks, schedule);
}

mssm_status mssm_scan_plan_packed(int64_t S, int64_t D, int64_t max_seqlen, int64_t total_len, int sm_count,
                                  int* rows_per_cta, int64_t* chunk_len, int64_t* n_chunks, int* schedule) {
  mssm_scan_plan_info info;
  info.struct_size = int32_t(sizeof(info));
  mssm_status st = mssm_scan_plan_query(S, D, max_seqlen, total_len, MSSM_BF16, sm_count, &info);
  if (st != MSSM_OK) return st;
  if (rows_per_cta) *rows_per_cta = info.rows_per_cta;
  if (chunk_len) *chunk_len = info.chunk_len;
  if (n_chunks) *n_chunks = info.n_chunks;
  if (schedule) *schedule = info.schedule;
  return MSSM_OK;
}

mssm_status mssm_scan_plan_query(int64_t S, int64_t D, int64_t max_seqlen, int64_t total_len, int io_dtype,
                                 int sm_count, mssm_scan_plan_info* info) {
  const int64_t Bt = S, L = max_seqlen;
  if (!info) return fail(MSSM_ERR_INVALID_ARG, "info: null pointer");
  if (info->struct_size < int32_t(sizeof(mssm_scan_plan_info)))
    return fail(MSSM_ERR_INVALID_ARG, "info->struct_size = %d; expected at least %d", int(info->struct_size),
                int(sizeof(mssm_scan_plan_info)));
  if (Bt < 0 || D < 0 || L < 0) return fail(MSSM_ERR_INVALID_ARG, "negative size");
  if (io_dtype != MSSM_F32 && io_dtype != MSSM_BF16) return fail(MSSM_ERR_INVALID_ARG, "io_dtype must be f32 or bf16");
  if (sm_count <= 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    sm_count = v;
  }
  int64_t forced;
  int forced_mode, forced_rows, forced_rpt;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    forced = g_chunk_len;
    forced_mode = g_schedule;
    forced_rows = g_rows_per_cta;
    forced_rpt = g_rows_per_thread;
  }
  const LaunchShape sh =
      choose_shape(Bt, D, L, sm_count, forced, forced_mode, forced_rows, forced_rpt, io_dtype, total_len);
  info->schedule = sh.mode;
  info->rows_per_cta = sh.rows;
  info->rows_per_thread = sh.rpt;
  info->chunk_len = sh.seg;
  info->n_chunks = sh.nseg;
  info->grid = sh.grid;
  return MSSM_OK;
}

mssm_status mssm_kernel_stats(int64_t launches[MSSM_KERNEL_KINDS], int64_t timed[MSSM_KERNEL_KINDS],
                              double ms[MSSM_KERNEL_KINDS], int reset) {
  std::lock_guard<std::mutex> lk(g_mu);
  mssm_status st = MSSM_OK;
  for (const TimedLaunch& t : g_pending) {
    float v = 0.0f;
    cudaError_t e = cudaEventSynchronize(t.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&v, t.a, t.b);
    if (e != cudaSuccess) {
      st = cuda_fail(e, "kernel timing events");
    } else {
      g_time_ms[t.kind] += v;
      g_timed[t.kind] += 1;
    }
    g_event_pool.push_back(t.a);
    g_event_pool.push_back(t.b);
  }
  g_pending.clear();
  for (int k = 0; k < MSSM_KERNEL_KINDS; ++k) {
    if (launches) launches[k] = g_launches[k];
    if (timed) timed[k] = g_timed[k];
    if (ms) ms[k] = g_time_ms[k];
    if (reset) {
      g_launches[k] = 0;
      g_timed[k] = 0;
      g_time_ms[k] = 0.0;
    }
  }
  return st;
}

mssm_status mssm_get_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "asynchronous kernel error");
  unsigned int word = 0u;
  e = mssm::read_device_error(&word, true);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word & 1u)
    return fail(MSSM_ERR_TIMEOUT, "a decode bulk copy did not complete within its bounded wait; "
                "the state rows of that tile were left unchanged");
  if (word & 2u)
    return fail(MSSM_ERR_TIMEOUT, "a chained scan chunk gave up waiting for the previous chunk's "
                "carried state and ran from a zero state");
  if (word & 4u)
    return fail(MSSM_ERR_INVALID_ARG, "cu_seqlens held an offset outside [0, T], a decreasing offset "
                "or a sequence longer than max_seqlen; the scan outputs are undefined");
  return MSSM_OK;
}

mssm_status mssm_shutdown(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  mssm_status st = MSSM_OK;
  int prev = -1;
  if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
  for (size_t i = 0; i < g_dev.size(); ++i) {
    if (!g_dev[i].ws && !g_dev[i].bwd_ws) continue;
    cudaSetDevice(int(i));
    if (g_dev[i].ws) {
      cudaError_t e = cudaFree(g_dev[i].ws);
      if (e != cudaSuccess) st = cuda_fail(e, "cudaFree(workspace)");
    }
    if (g_dev[i].bwd_ws) {
      cudaError_t e = cudaFree(g_dev[i].bwd_ws);
      if (e != cudaSuccess) st = cuda_fail(e, "cudaFree(backward workspace)");
    }
    g_dev[i].ws = nullptr;
    g_dev[i].ws_bytes = 0;
    g_dev[i].count_cap = 0;
    g_dev[i].bwd_ws = nullptr;
    g_dev[i].bwd_bytes = 0;
  }
  // Cached addresses of module symbols (the no-allocation scratch, the error word) are only
  // valid while the module stays loaded; look them up again after a device reset.
  for (int i = 0; i < 64; ++i) {
    g_noalloc_ptr[i] = nullptr;
    g_noalloc_sms[i] = 0;
  }
  mssm::forget_device_addresses();
  if (prev >= 0) cudaSetDevice(prev);
  return st;
}

}  // extern "C"
