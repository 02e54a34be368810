// The extern "C" boundary: argument validation, problem geometry, workspace
// layout and kernel launches.  Every entry point validates synchronously and
// launches nothing on invalid input; see include/vmoba.h for the contract.
#include <atomic>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "pairs.cuh"

using namespace vmoba;

namespace {

std::atomic<unsigned long long> g_launches{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Fills P from the public shape; returns VMOBA_OK or a status.
int make_prob(const vmoba_shape* sh, Prob* P) {
  if (!sh) return VMOBA_ERR_ARG;
  if (sh->dtype != VMOBA_BF16 && sh->dtype != VMOBA_F32) return VMOBA_ERR_DTYPE;
  if (sh->T < 1 || sh->H < 1 || sh->W < 1 || sh->n_heads < 1 || sh->n_heads > 128)
    return VMOBA_ERR_SHAPE;
  if (sh->head_dim != 64 && sh->head_dim != 128) return VMOBA_ERR_SHAPE;
  if (sh->mode < 0 || sh->mode > 2) return VMOBA_ERR_ARG;
  int bt, bh, bw;
  if (sh->mode == 0) { bt = sh->bt; bh = sh->H; bw = sh->W; }
  else if (sh->mode == 1) { bt = sh->T; bh = sh->bh; bw = sh->bw; }
  else { bt = sh->bt; bh = sh->bh; bw = sh->bw; }
  if (bt < 1 || bh < 1 || bw < 1) return VMOBA_ERR_SHAPE;
  if (sh->T % bt || sh->H % bh || sh->W % bw) return VMOBA_ERR_SHAPE;
  const long long s = (long long)sh->T * sh->H * sh->W;
  if (s > (long long)kMaxTiles * kTile) return VMOBA_ERR_SHAPE;
  Prob p{};
  p.T = sh->T; p.H = sh->H; p.W = sh->W; p.s = (int)s;
  p.n_h = sh->n_heads; p.d = sh->head_dim; p.mode = sh->mode; p.dtype = sh->dtype;
  p.bt = bt; p.bh = bh; p.bw = bw;
  p.nbt = sh->T / bt; p.nbh = sh->H / bh; p.nbw = sh->W / bw;
  p.Nb = p.nbt * p.nbh * p.nbw;
  p.L = bt * bh * bw;
  if (p.Nb > kMaxBlocks) return VMOBA_ERR_SHAPE;
  if ((long long)p.s * p.Nb >= (1LL << 31)) return VMOBA_ERR_SHAPE;
  p.Wb = (p.Nb + 31) / 32;
  p.n_qt = (p.s + kTile - 1) / kTile;
  p.Wqt = (p.n_qt + 31) / 32;
  p.cap = (uint32_t)((long long)p.s * p.Nb);     // every pair of a head (at most)
  *P = p;
  return VMOBA_OK;
}

// Pair slots per head that a workspace of ws_bytes holds: every pair of the
// head if it fits, else the largest capacity whose layout fits (the layout
// grows with the capacity), 0 if not even one pair does.  Every call of a
// layer passes the same ws_bytes, so all derive the same layout.
uint32_t fit_capacity(Prob P, size_t ws_bytes) {
  const uint32_t full = P.cap;
  if (ws_layout(P).total <= ws_bytes) return full;
  uint32_t lo = 0, hi = full;
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo + 1) / 2;
    P.cap = mid;
    if (ws_layout(P).total <= ws_bytes) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Checks the workspace and fixes the layer's pair capacity from its size.
int check_ws(Prob& P, const void* ws, size_t ws_bytes, WsLayout* L) {
  if (!ws || !aligned16(ws)) return VMOBA_ERR_WORKSPACE;
  const uint32_t cap = fit_capacity(P, ws_bytes);
  if (cap == 0) return VMOBA_ERR_WORKSPACE;
  P.cap = cap;
  *L = ws_layout(P);
  return VMOBA_OK;
}

// The CUDA error behind the calling thread's last VMOBA_ERR_CUDA.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return VMOBA_OK;
  g_last_cuda_error = e;
  return VMOBA_ERR_CUDA;
}

// The runtime's last-error slot is per host thread and the launchers read it
// after their launches; drop whatever another caller on this thread left
// there so it is not reported as ours (errors that break the context
// persist and still surface on our own launches).
void drop_stale_error() { (void)cudaGetLastError(); }

ItemBufs item_bufs(const Prob& P, void* ws, const WsLayout& L) {
  ItemBufs b{};
  b.rows = item_rows_capacity(P);
  char* p = ws_ptr<char>(ws, L.items);
  b.qh = reinterpret_cast<__half*>(p);
  p += align_up(b.rows * P.d * sizeof(__half), 256);
  b.doh = reinterpret_cast<__half*>(p);
  p += align_up(b.rows * P.d * sizeof(__half), 256);
  b.l2g = reinterpret_cast<float*>(p);
  p += align_up(b.rows * sizeof(float), 256);
  b.dg = reinterpret_cast<float*>(p);
  return b;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

}  // namespace

namespace {
std::atomic<long long> g_wait_budget{0};
std::atomic<int> g_skip_loads{0};
}  // namespace

namespace vmoba {
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n); }
long long debug_wait_budget() { return g_wait_budget.load(); }
int debug_skip_loads() { return g_skip_loads.load(); }
}  // namespace vmoba

extern "C" {

unsigned long long vmoba_kernel_launches(void) { return g_launches.load(); }


int vmoba_mode_for_layer(int layer_idx) { return layer_idx < 0 ? -1 : layer_idx % 3; }

int vmoba_num_blocks(const vmoba_shape* shape) {
  Prob P;
  int rc = make_prob(shape, &P);
  return rc == VMOBA_OK ? P.Nb : rc;
}

size_t vmoba_workspace_size(const vmoba_shape* shape) {
  Prob P;
  if (make_prob(shape, &P) != VMOBA_OK) return 0;
  return ws_layout(P).total;
}

size_t vmoba_workspace_size_bounded(const vmoba_shape* shape, double max_pair_fraction) {
  Prob P;
  if (make_prob(shape, &P) != VMOBA_OK) return 0;
  if (!(max_pair_fraction > 0.0) || std::isnan(max_pair_fraction)) return 0;
  // fraction of the pool, a relative margin for rounding in the selection's
  // mass sums and a few pairs more; never beyond the whole pool
  const double pool = (double)P.s * (double)P.Nb;
  const double want = std::floor(max_pair_fraction * pool * (1.0 + 1e-4)) + 64.0;
  if (want < pool) P.cap = (uint32_t)want;
  return ws_layout(P).total;
}

size_t vmoba_bwd_workspace_size(const vmoba_shape* shape) {
  Prob P;
  if (make_prob(shape, &P) != VMOBA_OK) return 0;
  return bwd_blk_ws_bytes(P);   // rowD and LSE*log2(e), [n_h][s] fp32 each
}

int vmoba_partition(const vmoba_shape* shape, const void* k, const void* v, void* k_perm,
                    void* v_perm, float* blocks, cudaStream_t stream) {
  Prob P;
  int rc = make_prob(shape, &P);
  if (rc != VMOBA_OK) return rc;
  if (!k || !v || !k_perm || !v_perm || !blocks) return VMOBA_ERR_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_perm) || !aligned16(v_perm) ||
      !aligned16(blocks))
    return VMOBA_ERR_ARG;
  drop_stale_error();
  return cuda_status(launch_partition(P, k, v, k_perm, v_perm, blocks, stream));
}

int vmoba_score_select(const vmoba_shape* shape, const void* q, const float* blocks, float tau,
                       float scale, uint32_t* sel_bits, vmoba_head_stats* stats, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  Prob P;
  int rc = make_prob(shape, &P);
  if (rc != VMOBA_OK) return rc;
  if (!q || !blocks || !sel_bits || !stats) return VMOBA_ERR_ARG;
  if (!aligned16(q) || !aligned16(blocks)) return VMOBA_ERR_ARG;   // 16-byte vector loads
  if (!(tau > 0.0f) || std::isnan(tau)) return VMOBA_ERR_ARG;
  if (std::isnan(scale) || std::isinf(scale)) return VMOBA_ERR_ARG;
  WsLayout L;
  if ((rc = check_ws(P, ws, ws_bytes, &L)) != VMOBA_OK) return rc;
  if (scale <= 0.0f) scale = 1.0f / std::sqrt((float)P.d);
  // tau at or above the whole pool keeps every pair; 2 can never be reached
  const float tau_dev = tau >= 1.0f ? 2.0f : tau;
  drop_stale_error();
  return cuda_status(
      launch_score_select(P, q, blocks, tau_dev, scale, sel_bits, stats, ws, L, num_sms(),
                          stream));
}

int vmoba_score_select_variant(const vmoba_shape* shape, const void* q, const float* blocks,
                               int variant, double param, float scale, uint32_t* sel_bits,
                               vmoba_head_stats* stats, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  Prob P;
  int rc = make_prob(shape, &P);
  if (rc != VMOBA_OK) return rc;
  if (!q || !blocks || !sel_bits || !stats) return VMOBA_ERR_ARG;
  if (!aligned16(q) || !aligned16(blocks)) return VMOBA_ERR_ARG;   // 16-byte vector loads
  if (std::isnan(param) || std::isnan(scale) || std::isinf(scale)) return VMOBA_ERR_ARG;
  const bool topk = variant == VMOBA_SELECT_TOPK_GLOBAL || variant == VMOBA_SELECT_TOPK_LOCAL;
  if (variant < VMOBA_SELECT_THRESHOLD_GLOBAL || variant > VMOBA_SELECT_ROWNORM_GLOBAL)
    return VMOBA_ERR_ARG;
  if (topk ? !(param >= 1.0 && param == std::floor(param) && param < 9.0e15) : !(param > 0.0))
    return VMOBA_ERR_ARG;
  WsLayout L;
  if ((rc = check_ws(P, ws, ws_bytes, &L)) != VMOBA_OK) return rc;
  if (scale <= 0.0f) scale = 1.0f / std::sqrt((float)P.d);
  const double pool = (double)P.s * (double)P.Nb;
  drop_stale_error();
  switch (variant) {
    case VMOBA_SELECT_THRESHOLD_GLOBAL: {
      const float tau_dev = param >= 1.0 ? 2.0f : (float)param;
      return cuda_status(launch_score_select(P, q, blocks, tau_dev, scale, sel_bits, stats, ws,
                                             L, num_sms(), stream));
    }
    case VMOBA_SELECT_ROWNORM_GLOBAL: {
      const float tau_dev = param >= 1.0 ? 2.0f : (float)param;
      return cuda_status(launch_score_select(P, q, blocks, tau_dev, scale, sel_bits, stats, ws,
                                             L, num_sms(), stream, 0, 0.0, true));
    }
    case VMOBA_SELECT_TOPK_GLOBAL:
      // k at or above the pool keeps every pair (the walk can never reach pool + 1)
      return cuda_status(launch_score_select(P, q, blocks, 0.0f, scale, sel_bits, stats, ws, L,
                                             num_sms(), stream, 1,
                                             param >= pool ? pool + 1.0 : param));
    default: {
      cudaError_t e = launch_score_pool(P, q, blocks, scale, ws, L, num_sms(), stream);
      if (e != cudaSuccess) return cuda_status(e);
      const double p = topk ? param : (param >= 1.0 ? 2.0 : param);
      return cuda_status(launch_select_local(P, topk ? 1 : 0, p, sel_bits, stats, ws, L, stream));
    }
  }
}

int vmoba_build_plan(const vmoba_shape* shape, const uint32_t* sel_bits, void* ws,
                     size_t ws_bytes, cudaStream_t stream) {
  Prob P;
  int rc = make_prob(shape, &P);
  if (rc != VMOBA_OK) return rc;
  if (!sel_bits) return VMOBA_ERR_ARG;
  WsLayout L;
  if ((rc = check_ws(P, ws, ws_bytes, &L)) != VMOBA_OK) return rc;
  drop_stale_error();
  return cuda_status(launch_plan(P, sel_bits, ws, L, stream));
}

int vmoba_attn_fwd(const vmoba_shape* shape, const void* q, const void* k_perm,
                   const void* v_perm, const uint32_t* sel_bits, void* ws, size_t ws_bytes,
                   float scale, void* out, float* lse, cudaStream_t stream) {
  Prob P;
  int rc = make_prob(shape, &P);
  if (rc != VMOBA_OK) return rc;
  if (!q || !k_perm || !v_perm || !sel_bits || !out || !lse) return VMOBA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_perm) || !aligned16(v_perm) || !aligned16(out))
    return VMOBA_ERR_ARG;
  if (std::isnan(scale) || std::isinf(scale)) return VMOBA_ERR_ARG;
  WsLayout L;
  if ((rc = check_ws(P, ws, ws_bytes, &L)) != VMOBA_OK) return rc;
  if (scale <= 0.0f) scale = 1.0f / std::sqrt((float)P.d);
  // bf16 runs on the tensor cores; fp32 I/O (whose 1e-4 bar rules out
  // TF32) runs on the CUDA cores
  drop_stale_error();
  if (uses_blk_path(P))
    return cuda_status(launch_attn_fwd_blk(
        P, q, k_perm, v_perm, sel_bits, pairs_view(P, ws_ptr<char>(ws, L.pairs)),
        ws_ptr<char>(ws, L.part), item_bufs(P, ws, L), scale, out, ws_ptr<float>(ws, L.o32),
        lse, ws_ptr<int>(ws, L.status), num_sms(), stream));
  return cuda_status(
      launch_attn_fwd_simt(P, q, k_perm, v_perm, sel_bits, ws, L, scale, out, lse, stream));
}

int vmoba_attn_bwd(const vmoba_shape* shape, const void* q, const void* k_perm,
                   const void* v_perm, const uint32_t* sel_bits, void* ws, size_t ws_bytes,
                   float scale, const float* lse, const void* dout, void* dq, void* dk,
                   void* dv, void* ws_bwd, size_t ws_bwd_bytes, cudaStream_t stream) {
  Prob P;
  int rc = make_prob(shape, &P);
  if (rc != VMOBA_OK) return rc;
  if (!q || !k_perm || !v_perm || !sel_bits || !lse || !dout || !dq || !dk || !dv)
    return VMOBA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_perm) || !aligned16(v_perm) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return VMOBA_ERR_ARG;
  if (std::isnan(scale) || std::isinf(scale)) return VMOBA_ERR_ARG;
  WsLayout L;
  if ((rc = check_ws(P, ws, ws_bytes, &L)) != VMOBA_OK) return rc;
  if (!ws_bwd || ws_bwd_bytes < vmoba_bwd_workspace_size(shape) || !aligned16(ws_bwd))
    return VMOBA_ERR_WORKSPACE;
  if (scale <= 0.0f) scale = 1.0f / std::sqrt((float)P.d);
  drop_stale_error();
  if (uses_blk_path(P))
    return cuda_status(launch_attn_bwd_blk(
        P, q, k_perm, v_perm, sel_bits, pairs_view(P, ws_ptr<char>(ws, L.pairs)),
        ws_ptr<char>(ws, L.part), item_bufs(P, ws, L), ws_ptr<float>(ws, L.o32), lse, dout, dq,
        dk, dv, ws_bwd, scale, ws_ptr<int>(ws, L.status), num_sms(), stream));
  return cuda_status(launch_attn_bwd_simt(P, q, k_perm, v_perm, sel_bits, ws, L, scale, lse,
                                          dout, dq, dk, dv, static_cast<float*>(ws_bwd),
                                          stream));
}

int vmoba_get_status(void* ws, int* device_status, cudaStream_t stream) {
  if (!ws || !device_status) return VMOBA_ERR_ARG;
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return VMOBA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return VMOBA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyAsync(ws, &zero, sizeof(int), cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return VMOBA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return VMOBA_ERR_CUDA;
  *device_status = v;
  return VMOBA_OK;
}

const char* vmoba_last_cuda_error(void) { return cudaGetErrorName(g_last_cuda_error); }

int vmoba_debug_set_wait(long long wait_cycles, int skip_forward_loads) {
  if (wait_cycles < 0 || (skip_forward_loads != 0 && skip_forward_loads != 1))
    return VMOBA_ERR_ARG;
  g_wait_budget.store(wait_cycles);
  g_skip_loads.store(skip_forward_loads);
  return VMOBA_OK;
}

const char* vmoba_status_string(int status) {
  switch (status) {
    case VMOBA_OK: return "ok";
    case VMOBA_ERR_ARG: return "invalid argument";
    case VMOBA_ERR_SHAPE: return "unsupported shape (box must divide T,H,W; head_dim 64 or 128)";
    case VMOBA_ERR_DTYPE: return "unsupported dtype";
    case VMOBA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case VMOBA_ERR_CUDA: return "CUDA runtime error";
    case VMOBA_ERR_TIMEOUT: return "bounded device wait timed out";
    case VMOBA_ERR_NOT_IMPLEMENTED: return "not implemented";
    case VMOBA_ERR_DEVICE: return "device is not sm_100";
    default: return "unknown status";
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Selection without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc when they want a selection: an engine
// that reserves all device memory into its own pool at start-up and forbids
// later allocations (so it cannot hand out a workspace of its own), or a
// plugin loaded into a host program that gives it no allocator.  For them
// vmoba_score_select_static keeps the score pool, the radix histograms and
// the per-head search state in a fixed array of device memory that belongs
// to the library (kStaticSelectScratch bytes on every GPU whose copy of this
// library's device code is loaded, held until the process exits).  Only this
// entry point uses the array; every other call keeps using caller memory.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr size_t kStaticSelectScratch = VMOBA_STATIC_SELECT_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_select_scratch[kStaticSelectScratch];

constexpr int kMaxStaticDevices = 64;
std::mutex g_static_mu;
void* g_static_addr[kMaxStaticDevices] = {};

// Device address of the scratch array on the current device.  Host code may
// not pass g_select_scratch itself to a kernel: on the host that name is a
// stand-in symbol, not a device address.  Resolved once per device.
int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VMOBA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxStaticDevices) return VMOBA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr)
      return VMOBA_ERR_CUDA;
    g_static_addr[dev] = p;
  }
  *out = g_static_addr[dev];
  return VMOBA_OK;
}

// The selection's part of the workspace layout, packed into the static array:
// the device status word, the search state and histograms, the fp32 score
// pool and, for bf16 inputs, the bf16 split of the block means.
WsLayout static_select_layout(const Prob& P) {
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  w.status = take(256);
  w.sel_state = take(sizeof(SelState) * P.n_h);
  w.hist_count = take(sizeof(uint32_t) * kHistBins * P.n_h);
  w.hist_mass = take(sizeof(double) * kHistBins * P.n_h);
  w.scores = take(sizeof(float) * (size_t)P.n_h * P.s * P.Nb);
  if (P.dtype == VMOBA_BF16) w.bsplit = take(sel_split_bytes(P));
  w.total = off;
  return w;
}

}  // namespace

extern "C" {

int vmoba_score_select_static(const vmoba_shape* shape, const void* q, const float* blocks,
                              float tau, float scale, uint32_t* sel_bits,
                              vmoba_head_stats* stats, cudaStream_t stream) {
  Prob P;
  int rc = make_prob(shape, &P);
  if (rc != VMOBA_OK) return rc;
  if (!q || !blocks || !sel_bits || !stats) return VMOBA_ERR_ARG;
  if (!aligned16(q) || !aligned16(blocks)) return VMOBA_ERR_ARG;   // 16-byte vector loads
  if (!(tau > 0.0f) || std::isnan(tau)) return VMOBA_ERR_ARG;
  if (std::isnan(scale) || std::isinf(scale)) return VMOBA_ERR_ARG;
  const WsLayout L = static_select_layout(P);
  if (L.total > kStaticSelectScratch) return VMOBA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((rc = static_scratch(&scratch)) != VMOBA_OK) return rc;
  if (scale <= 0.0f) scale = 1.0f / std::sqrt((float)P.d);
  const float tau_dev = tau >= 1.0f ? 2.0f : tau;
  // the first kernel of the selection clears the histograms and the search
  // state; the score pool and the split of B are fully overwritten before
  // they are read
  drop_stale_error();
  return cuda_status(launch_score_select(P, q, blocks, tau_dev, scale, sel_bits, stats, scratch,
                                         L, num_sms(), stream));
}

}  // extern "C"
