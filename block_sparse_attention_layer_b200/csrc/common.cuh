// Internal definitions shared by the VMoBA kernels and the C ABI.
//
// Geometry of one layer (VMoBA notes, key design 1): the (T, H, W) latent is
// cut into N_b equal boxes (bt, bh, bw); blocks are numbered row-major over
// the (T/bt, H/bh, W/bw) grid and tokens inside a block keep (t, y, x) order.
// "Partition order" position p = j*L + r lists block j's r-th token.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/vmoba.h"

namespace vmoba {

constexpr int kTile = 128;          // query / key tile (rows) used by the plan
constexpr int kHistBits0 = 11;      // radix digits of the 32-bit ordered score key
constexpr int kHistBins = 2048;
constexpr int kMaxBlocks = 1024;    // N_b limit (bitmap row <= 32 words)
constexpr int kMaxTiles = 8192;     // ceil(s/128) limit

struct Prob {
  int T, H, W, s;
  int n_h, d, mode, dtype;
  int bt, bh, bw;                   // box of the mode
  int nbt, nbh, nbw;                // box grid
  int Nb, L;                        // number of blocks, tokens per block
  int Wb;                           // bitmap words per query row
  int n_qt;                         // 128-row tiles (queries and keys alike)
  int Wqt;                          // words of a tile bitmap (ceil(n_qt/32))
  uint32_t cap;                     // (query, block) pair slots per head in the workspace
};

// Original token of partition position p.
__host__ __device__ __forceinline__ int perm_token(const Prob& P, int p) {
  int j = p / P.L, r = p - j * P.L;
  int pw = j % P.nbw, q = j / P.nbw;
  int ph = q % P.nbh, pt = q / P.nbh;
  int hw = P.bh * P.bw;
  int tt = r / hw, rr = r - tt * hw;
  int yy = rr / P.bw, xx = rr - yy * P.bw;
  int t = pt * P.bt + tt, y = ph * P.bh + yy, x = pw * P.bw + xx;
  return (t * P.H + y) * P.W + x;
}

// Order-preserving map float -> uint32 (larger float <=> larger key); -0 and
// +0 map to one key.
__host__ __device__ __forceinline__ uint32_t f2key(float f) {
  f = f + 0.0f;
  uint32_t b;
#ifdef __CUDA_ARCH__
  b = __float_as_uint(f);
#else
  memcpy(&b, &f, 4);
#endif
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__host__ __device__ __forceinline__ float key2f(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
#ifdef __CUDA_ARCH__
  return __uint_as_float(b);
#else
  float f;
  memcpy(&f, &b, 4);
  return f;
#endif
}

// Per-head state of the threshold search (lives in the workspace).
struct SelState {
  uint32_t max_key;      // ordered key of max S (atomicMax by the score kernel)
  uint32_t prefix;       // resolved high bits of the cut key / cut index
  uint32_t cut_key;      // ordered key of the last selected score
  uint32_t idx_cut;      // ties at cut_key: flat indices <= idx_cut are kept
  uint32_t tie_count;    // elements whose key equals cut_key
  uint32_t tie_take;     // how many of them are kept (remaining, during tie passes)
  int state;             // 0 searching, 1 resolved, 2 every pair selected
  int pad;
  double Z;              // sum exp(S - max S) over the pool
  double target;         // tau * Z
  double mass_above;     // mass of keys above the current prefix bucket
  unsigned long long count_above;
  unsigned long long n_selected;
  double mass_selected;
};

// Byte offsets inside the caller's workspace (all 256-byte aligned).
struct WsLayout {
  size_t status, sel_state, hist_count, hist_mass, scores;
  size_t bsplit;         // bf16 hi / lo split of the block means (tensor-core score passes)
  size_t qt_kt_bits, qt_work, kt_qt_bits, kt_work;
  size_t o32;            // fp32 copy of the forward output, [s][n_h][d]
  size_t pairs;          // pair lists of the selection (pairs.cu)
  size_t part;           // per-pair partial results of one head (block-major kernels)
  size_t items;          // item-ordered Q / dO / LSE / D copies of one head
  size_t total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t pairs_ws_bytes(const Prob& P);
size_t blk_partial_bytes(const Prob& P);
// Rows per head and half of the bf16 split of the block means (N_b rounded
// up to 128) and its bytes ([n_h][hi, lo][rows][d]).
int sel_split_rows(const Prob& P);
size_t sel_split_bytes(const Prob& P);
size_t item_bufs_bytes(const Prob& P);
// bf16 (head_dim 64 or 128) runs the block-major tensor-core kernels; fp32
// I/O (whose 1e-4 bar rules out TF32) runs on the CUDA cores.
inline bool uses_blk_path(const Prob& P) { return P.dtype == VMOBA_BF16; }

inline WsLayout ws_layout(const Prob& P) {
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  w.status = take(256);
  w.sel_state = take(sizeof(SelState) * P.n_h);
  w.hist_count = take(sizeof(uint32_t) * kHistBins * P.n_h);
  w.hist_mass = take(sizeof(double) * kHistBins * P.n_h);
  w.scores = take(sizeof(float) * (size_t)P.n_h * P.s * P.Nb);
  w.bsplit = take(sel_split_bytes(P));
  const bool tiles = !uses_blk_path(P);     // tile plan of the CUDA-core kernels
  w.qt_kt_bits = take(tiles ? sizeof(uint32_t) * (size_t)P.n_h * P.n_qt * P.Wqt : 0);
  w.qt_work = take(tiles ? sizeof(uint32_t) * (size_t)P.n_h * P.n_qt : 0);
  w.kt_qt_bits = take(tiles ? sizeof(uint32_t) * (size_t)P.n_h * P.n_qt * P.Wqt : 0);
  w.kt_work = take(tiles ? sizeof(uint32_t) * (size_t)P.n_h * P.n_qt : 0);
  w.o32 = take(sizeof(float) * (size_t)P.n_h * P.s * P.d);
  w.pairs = take(pairs_ws_bytes(P));
  w.part = take(uses_blk_path(P) ? blk_partial_bytes(P) : 0);
  w.items = take(uses_blk_path(P) ? item_bufs_bytes(P) : 0);
  w.total = off;
  return w;
}

template <typename T>
inline T* ws_ptr(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

// Brackets one kernel launch with CUDA events on its stream while tracing is
// enabled (vmoba_trace_enable); a no-op otherwise.
class TraceScope {
 public:
  TraceScope(const char* name, cudaStream_t st);
  ~TraceScope();
 private:
  cudaStream_t stream_;
  void* a_;
  const char* name_ = nullptr;
};
#define VMOBA_TRACE(name, st) ::vmoba::TraceScope _vmoba_trace_scope_((name), (st))

// Kernels launched by this library since load (diagnostics; see
// vmoba_kernel_launches).  Every launch wrapper adds what it launched.
void count_launches(int n);

// Wait settings of vmoba_debug_set_wait (0 = defaults).
long long debug_wait_budget();
int debug_skip_loads();

// ---- launch wrappers (one per kernel family; defined in the .cu files) ----
cudaError_t launch_partition(const Prob& P, const void* k, const void* v, void* kp, void* vp,
                             float* blocks, cudaStream_t st);
// by_count = 0: the method's mass threshold tau; by_count = 1: the kcount
// highest pairs of each head's pool (top-k global), same ranking and ties;
// rownorm: the pool normalised per query row first (a selection variant).
cudaError_t launch_score_select(const Prob& P, const void* q, const float* blocks, float tau,
                                float scale, uint32_t* sel, vmoba_head_stats* stats, void* ws,
                                const WsLayout& L, int num_sms, cudaStream_t st,
                                int by_count = 0, double kcount = 0.0, bool rownorm = false);
// bf16 Q: the score pool S = scale q b^T of every head on the tensor cores
// (score_tc.cu), written to `pool` with each head's max in st[h].max_key;
// bsplit receives the bf16 hi / lo split of the block means.
cudaError_t launch_score_pool_tc(const Prob& P, const void* q, const float* blocks, float scale,
                                 void* bsplit, float* pool, SelState* st, int* status,
                                 int num_sms, cudaStream_t stream);
// The score pool S = scale q b^T of every head into the workspace.
cudaError_t launch_score_pool(const Prob& P, const void* q, const float* blocks, float scale,
                              void* ws, const WsLayout& L, int num_sms, cudaStream_t st);
// Per-query-row selection (threshold local / top-k local); scores in the
// workspace pool, per-row scratch in the forward-output copy.
cudaError_t launch_select_local(const Prob& P, int topk, double param, uint32_t* sel,
                                vmoba_head_stats* stats, void* ws, const WsLayout& L,
                                cudaStream_t st);
cudaError_t launch_plan(const Prob& P, const uint32_t* sel, void* ws, const WsLayout& L,
                        cudaStream_t st);
cudaError_t launch_attn_fwd_simt(const Prob& P, const void* q, const void* kp, const void* vp,
                                 const uint32_t* sel, void* ws, const WsLayout& L, float scale,
                                 void* out, float* lse, cudaStream_t st);
cudaError_t launch_attn_bwd_simt(const Prob& P, const void* q, const void* kp, const void* vp,
                                 const uint32_t* sel, void* ws, const WsLayout& L, float scale,
                                 const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                 float* rowD, cudaStream_t st);

}  // namespace vmoba
