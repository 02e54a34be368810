/*
 * vmoba.h -- C ABI of the B200 (sm_100a) VMoBA per-layer sparse attention.
 *
 * The method (VMoBA: Mixture-of-Block Attention for Video Diffusion Models;
 * papernotes.org ICLR 2026 notes, "overall framework" and key designs 1-3;
 * paperlayer.ai digest, sections 3.1-3.4) replaces one full self-attention of
 * a video DiT.  Q/K/V of a (T, H, W) video latent go in; an output of
 * full-attention shape comes out.  Per layer l it
 *   1. rearranges the keys into blocks of the layer's partition mode
 *      (l mod 3: 1D temporal, 2D spatial across all frames, 3D local patch)
 *      and mean-pools every block into B                  -> vmoba_partition
 *   2. scores every query of a head against every block, S = scale*q.b,
 *   3. ranks the head's whole s x N_b pool and keeps pairs in descending
 *      order until the normalised cumulative similarity reaches tau
 *                                                          -> vmoba_score_select
 *   4. runs attention over the selected (query, block) pairs only
 *                                         -> vmoba_build_plan, vmoba_attn_fwd,
 *                                            vmoba_attn_bwd
 *
 * Conventions shared by every call
 * --------------------------------
 * Tokens are frame-major: token n = t*H*W + y*W + x.  s = T*H*W.
 * Q, K, V, O, dO, dQ, dK, dV are [s][n_heads][head_dim] row-major (one
 * sample; loop or offset pointers for a batch).  K', V' (keys/values in
 * partition order) are [n_heads][s][head_dim].  Blocks are numbered
 * row-major over the (T/bt', H/bh', W/bw') box grid; inside a block tokens
 * keep (t, y, x) order.  dtype VMOBA_BF16 = bf16 storage, VMOBA_F32 = fp32;
 * all accumulation is fp32 or wider.
 * Selection bitmap sel_bits: [n_heads][s][ceil(N_b/32)] uint32, bit (j%32)
 * of word (j/32) of row i set iff query i (original order) attends block j.
 * Normalisation of the pool (the pages name it but print no formula; the
 * reading taken): p = exp(S - max S) / sum exp(S - max S) over the head's
 * whole pool; ties rank by (query asc, block asc); ">=" tau stops.
 *
 * Ownership: the caller allocates every buffer (device memory unless noted);
 * the library never allocates, frees or synchronises.  Every compute call
 * is asynchronous on the given stream.
 * Errors: invalid arguments return a negative vmoba_status synchronously,
 * before anything is launched.  A launch failure returns VMOBA_ERR_CUDA.
 * Faults detected on the device (a bounded wait that ran out) are latched in
 * a status word inside the workspace: read it with vmoba_get_status.
 * Workspace contents are private; the same workspace must be passed to
 * vmoba_score_select, vmoba_build_plan, vmoba_attn_fwd and vmoba_attn_bwd of
 * one layer, and no two calls may use one workspace concurrently.
 */
#ifndef VMOBA_H_
#define VMOBA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vmoba_status {
  VMOBA_OK = 0,
  VMOBA_ERR_ARG = -1,             /* null pointer, bad tau/scale, misaligned pointer */
  VMOBA_ERR_SHAPE = -2,           /* box does not divide (T,H,W); unsupported head_dim */
  VMOBA_ERR_DTYPE = -3,           /* dtype not VMOBA_BF16 / VMOBA_F32 */
  VMOBA_ERR_WORKSPACE = -4,       /* workspace pointer null or smaller than required */
  VMOBA_ERR_CUDA = -5,            /* a CUDA runtime call or launch failed */
  VMOBA_ERR_TIMEOUT = -6,         /* a bounded device wait ran out (device status) */
  VMOBA_ERR_NOT_IMPLEMENTED = -7, /* combination not built (e.g. this dtype/head_dim) */
  VMOBA_ERR_DEVICE = -8           /* current device is not sm_100 */
} vmoba_status;

enum { VMOBA_BF16 = 0, VMOBA_F32 = 1 };

/* Size of the library-owned device scratch of vmoba_score_select_static. */
#define VMOBA_STATIC_SELECT_SCRATCH_BYTES ((size_t)16 << 20)

/* One layer's problem.  mode: 0 = 1D (box bt x H x W), 1 = 2D (T x bh x bw),
 * 2 = 3D (bt x bh x bw); the fields the mode does not use are ignored.
 * head_dim must be 64 or 128. */
typedef struct vmoba_shape {
  int T, H, W;
  int n_heads, head_dim;
  int mode;
  int bt, bh, bw;
  int dtype;
} vmoba_shape;

/* Per-head selection result (written to device memory by vmoba_score_select).
 * n_selected = k*, the number of (query, block) pairs kept; mass = their
 * normalised cumulative similarity (>= tau unless every pair is kept);
 * cut_score = S of the last pair kept. */
typedef struct vmoba_head_stats {
  long long n_selected;
  double mass;
  float cut_score;
  int all_selected;               /* 1 when tau reached the whole pool */
} vmoba_head_stats;

/* Partition mode of layer l: l mod 3 (notes, key design 1).  -1 if l < 0. */
int vmoba_mode_for_layer(int layer_idx);

/* N_b of the shape's mode, or a negative vmoba_status. */
int vmoba_num_blocks(const vmoba_shape* shape);

/* Bytes of workspace for score_select / build_plan / attn_fwd / attn_bwd
 * (one buffer serves them all), or 0 for an invalid shape.  This size holds
 * the pair lists and per-pair buffers for every (query, block) pair of every
 * head being selected. */
size_t vmoba_workspace_size(const vmoba_shape* shape);

/* The same for selections that keep at most max_pair_fraction of each head's
 * s x N_b pairs (plus a small margin), or 0 for an invalid shape or a
 * fraction <= 0 / NaN; at or above the whole pool it equals
 * vmoba_workspace_size.  The method's threshold selection keeps fewer than
 * tau * s * N_b + 1 pairs per head (the cumulative rule stops within the
 * first tau of the mass, and the sorted prefix carries at least its share of
 * it), so max_pair_fraction = tau suffices for it; top-k global needs k /
 * (s N_b); the local variants can keep more.  Every call of a layer derives
 * the pair capacity from the ws_bytes it is given (the largest the buffer
 * holds).  If a selection keeps more pairs in a head than that capacity,
 * vmoba_build_plan leaves the head empty (its attention outputs and
 * gradients are zero) and latches VMOBA_ERR_WORKSPACE in the device status
 * word (vmoba_get_status); nothing is read or written past the buffers. */
size_t vmoba_workspace_size_bounded(const vmoba_shape* shape, double max_pair_fraction);

/* Bytes of the extra backward workspace, or 0: the row terms D and -LSE
 * log2(e) ([n_heads][s] fp32 each) and, for bf16 layers, fp16 copies of K'
 * and V' (the backward's tensor-core MMAs take fp16 operands). */
size_t vmoba_bwd_workspace_size(const vmoba_shape* shape);

/* Step 1 (notes, key design 1: "rearrange K in (T H W), B = mean(K')").
 * k, v: [s][n_heads][d] (dtype).  Writes k_perm, v_perm: [n_heads][s][d]
 * (dtype; exact copies in partition order) and blocks: [n_heads][N_b][d]
 * fp32 block means (fp64 accumulation).  All pointers 16-byte aligned. */
int vmoba_partition(const vmoba_shape* shape, const void* k, const void* v,
                    void* k_perm, void* v_perm, float* blocks, cudaStream_t stream);

/* Steps 2-3 (notes, key design 2: per-head global pool q_i b_i^T; key design
 * 3: k = min{k' : cumulative normalised similarity >= tau}; digest 3.3-3.4).
 * q: [s][n_heads][d] (dtype); blocks from vmoba_partition.  tau in (0, 1]
 * (tau >= the pool's total keeps every pair; tau <= 0 or NaN ->
 * VMOBA_ERR_ARG).  scale <= 0 selects 1/sqrt(head_dim).  q and blocks must
 * be 16-byte aligned (VMOBA_ERR_ARG otherwise: the kernels read them in
 * 16-byte vectors).  Writes sel_bits (layout above, fully overwritten) and
 * stats[n_heads] (device).  The pool is ranked by an exact on-device radix
 * select over (score desc, index asc); no host sort and no host round trip. */
int vmoba_score_select(const vmoba_shape* shape, const void* q, const float* blocks,
                       float tau, float scale, uint32_t* sel_bits,
                       vmoba_head_stats* stats, void* ws, size_t ws_bytes,
                       cudaStream_t stream);

/* The ablation's selection variants (notes, ablation table; digest App. A),
 * the research alternatives to step 3 -- no counterpart is needed on the
 * method's own path.  variant:
 *   VMOBA_SELECT_THRESHOLD_GLOBAL  the method itself (= vmoba_score_select),
 *                                  param = tau;
 *   VMOBA_SELECT_TOPK_GLOBAL       "topk + global": the param = k highest
 *                                  pairs of each head's pool, ranked (score
 *                                  desc, index asc) like the method;
 *   VMOBA_SELECT_THRESHOLD_LOCAL   "threshold + local": per query row, the
 *                                  shortest prefix of its own blocks (score
 *                                  desc, block asc) whose mass under the
 *                                  row's own softmax reaches param = tau;
 *   VMOBA_SELECT_TOPK_LOCAL        "topk + local" (about MoBA's selection;
 *                                  the training-free runs use it on 3D
 *                                  blocks): per query row its first
 *                                  min(param = k, N_b) blocks;
 *   VMOBA_SELECT_ROWNORM_GLOBAL    the method's global pool and cumulative
 *                                  rule under the other reading of
 *                                  "normalised similarity": each query's
 *                                  scores normalised by a softmax over its
 *                                  own N_b blocks and divided by s, so
 *                                  every query carries 1/s of the head's
 *                                  mass; param = tau.  Ranked by that value
 *                                  (ties by index); cut_score is the log row
 *                                  softmax of the last pair kept.
 * tau must be > 0 (>= 1 keeps everything); k a whole number >= 1 (at or
 * above the pool / N_b keeps everything); anything else, or an unknown
 * variant, -> VMOBA_ERR_ARG.  Same buffers, alignment rule and outputs as
 * vmoba_score_select.  stats of the local variants: n_selected = pairs,
 * mass = mean kept mass per row under the row softmax, cut_score = NaN
 * (each row has its own cut); the per-row bookkeeping uses workspace that
 * vmoba_attn_fwd overwrites later. */
enum {
  VMOBA_SELECT_THRESHOLD_GLOBAL = 0,
  VMOBA_SELECT_TOPK_GLOBAL = 1,
  VMOBA_SELECT_THRESHOLD_LOCAL = 2,
  VMOBA_SELECT_TOPK_LOCAL = 3,
  VMOBA_SELECT_ROWNORM_GLOBAL = 4
};
int vmoba_score_select_variant(const vmoba_shape* shape, const void* q, const float* blocks,
                               int variant, double param, float scale, uint32_t* sel_bits,
                               vmoba_head_stats* stats, void* ws, size_t ws_bytes,
                               cudaStream_t stream);

/* Step 4a: from any selection bitmap (vmoba_score_select's, or one the
 * caller built), build the tile work lists the attention kernels walk:
 * per 128-query tile (queries in partition order) the key tiles its rows
 * touch, and per key tile the query tiles that touch it. */
int vmoba_build_plan(const vmoba_shape* shape, const uint32_t* sel_bits,
                     void* ws, size_t ws_bytes, cudaStream_t stream);

/* Step 4b (notes, overall framework: attention only over the selected
 * blocks, output of full-attention shape, heads concatenated).
 * For query i: LSE_i = log sum_{n : block(n) selected for i} exp(scale q_i.k_n),
 * O_i = softmax-weighted sum of v_n; a row with no selected block gets
 * O = 0 and LSE = -inf.  q: [s][n_heads][d]; k_perm, v_perm from
 * vmoba_partition; sel_bits the bitmap the plan was built from.  Writes
 * out [s][n_heads][d] (dtype) and lse [n_heads][s] fp32 (natural log), and
 * keeps an fp32 copy of O in the workspace for vmoba_attn_bwd.
 * Range: the bf16 (tensor-core) path keeps each (query, block) partial
 * result as O/l in fp16 (a convex combination of V rows, so |O/l| <= max|V|);
 * inputs with |V| above 65504, the largest finite fp16, are outside its
 * contract (their partials overflow to inf).  The fp32 path has no such
 * limit. */
int vmoba_attn_fwd(const vmoba_shape* shape, const void* q, const void* k_perm,
                   const void* v_perm, const uint32_t* sel_bits, void* ws,
                   size_t ws_bytes, float scale, void* out, float* lse,
                   cudaStream_t stream);

/* Step 4c: gradients through the selected pairs, mask held constant (the
 * pages add no loss and route no gradient through selection).
 * D_i = dO_i.O_i, dS = P*(dP - D), dQ = scale dS K, dK = scale dS^T Q,
 * dV = P^T dO.  D is taken from the fp32 output copy the preceding
 * vmoba_attn_fwd left in ws (the same ws, sel_bits and inputs are
 * required), so the bf16 rounding of the stored output does not enter the
 * gradients.  lse from vmoba_attn_fwd; dout [s][n_heads][d].  Writes dq, dk,
 * dv [s][n_heads][d] (dtype, original token order; a key no selected query
 * attends gets zeros).  ws_bwd: vmoba_bwd_workspace_size bytes.
 * Range: the bf16 / tensor-core path computes on fp16 copies of Q, dO, K'
 * and V' with fp16 P and dS, and keeps each (query, block) share of dQ (the
 * block's sum of dS k_n, before the scale) in fp16; values above 65504 in
 * magnitude are outside its contract.  The fp32 path has no such limit. */
int vmoba_attn_bwd(const vmoba_shape* shape, const void* q, const void* k_perm,
                   const void* v_perm, const uint32_t* sel_bits, void* ws,
                   size_t ws_bytes, float scale, const float* lse, const void* dout,
                   void* dq, void* dk, void* dv, void* ws_bwd, size_t ws_bwd_bytes,
                   cudaStream_t stream);

/* Reads the workspace's device status word (synchronises the stream) into
 * *device_status (VMOBA_OK or VMOBA_ERR_TIMEOUT) and clears it.
 * vmoba_build_plan also clears it (a new plan starts clean). */
int vmoba_get_status(void* ws, int* device_status, cudaStream_t stream);

/* Diagnostics for tests of the bounded-wait path.  wait_cycles > 0 replaces
 * the spin budget of every bounded device wait (about one second of SM clock
 * by default) for attention launches made after the call; 0 restores it.
 * skip_forward_loads = 1 makes the tensor-core forward's key/value producer
 * issue no loads, so that its consumers' waits run out with no copy or MMA
 * in flight and latch VMOBA_ERR_TIMEOUT (the outputs of such a call are
 * garbage); 0 restores normal operation.  Process-wide, meant for tests:
 * set it only while no other thread launches.  Returns VMOBA_ERR_ARG for a
 * negative budget or a flag other than 0 / 1. */
int vmoba_debug_set_wait(long long wait_cycles, int skip_forward_loads);

/* Selection for callers that cannot allocate device memory.
 * Same contract and results as vmoba_score_select, but the score pool, the
 * radix histograms and the per-head search state live in a fixed 16 MiB
 * array of device memory owned by the library, so no workspace is passed
 * and nothing is allocated by the call.  Meant for callers such as an
 * engine that has pooled all device memory at start-up and forbids later
 * cudaMalloc, or a plugin that is given no allocator.  This entry point has
 * no counterpart in the paper: it only changes where scratch memory lives.
 * - The array is committed on a device when the CUDA runtime loads the
 *   library's device code there.  With lazy module loading (the CUDA 12
 *   default) that can happen at this entry point's first call on the
 *   device, so make one warm-up call on each device before reserving a
 *   memory pool that leaves no room for 16 MiB; the array then stays
 *   committed until the process exits.
 * - Problems whose scratch exceeds VMOBA_STATIC_SELECT_SCRATCH_BYTES return
 *   VMOBA_ERR_WORKSPACE without launching anything.  The scratch is the fp32
 *   score pool (4*n_heads*s*N_b bytes), for bf16 inputs the bf16 hi / lo
 *   split of the block means (4 * n_heads * N_b' * head_dim bytes, N_b' =
 *   N_b rounded up to 128), and about 24.6 KB per head of histograms and
 *   search state; e.g. 4 heads x 2048 tokens x 64 blocks (2.2 MB) fits,
 *   12 heads x 55296 tokens x 24 blocks (64 MB) does not.
 * - The array is committed on a device when the CUDA runtime loads the
 *   library's device code there.  With lazy module loading (the CUDA 12
 *   default) that can happen at this entry point's first call on the
 *   device, so make one warm-up call on each device before reserving a
 *   memory pool that leaves no room for 16 MiB; the array then stays
 *   committed until the process exits.
 * - Problems whose scratch exceeds VMOBA_STATIC_SELECT_SCRATCH_BYTES return
 *   VMOBA_ERR_WORKSPACE without launching anything.  For bf16 inputs the
 *   scratch is the bf16 hi / lo split of the block means (4 * n_heads *
 *   N_b' * head_dim bytes, N_b' = N_b rounded up to 128; the score pool is
 *   recomputed, never stored) plus about 24.6 KB per head of histograms and
 *   search state: 12 heads x 288 blocks x 128 (2.7 MB) fits, 128 heads x
 *   1024 blocks x 128 (67 MB) does not.  For fp32 inputs the fp32 score pool
 *   (4 * n_heads * s * N_b bytes) takes the split's place: 2 heads x 256
 *   tokens x 8 blocks fits, 12 heads x 55296 tokens x 24 blocks does not.
 * - The array is committed on a device when the CUDA runtime loads the
 *   library's device code there.  With lazy module loading (the CUDA 12
 *   default) that can happen at this entry point's first call on the
 *   device, so make one warm-up call on each device before reserving a
 *   memory pool that leaves no room for 16 MiB; the array then stays
 *   committed until the process exits.
 * - Problems whose scratch exceeds VMOBA_STATIC_SELECT_SCRATCH_BYTES return
 *   VMOBA_ERR_WORKSPACE without launching anything.  The scratch is the fp32
 *   score pool (4*n_heads*s*N_b bytes) plus about 24.6 KB per head of
 *   histograms and search state; e.g. 4 heads x 2048 tokens x 64 blocks
 *   (2.1 MB) fits, 12 heads x 55296 tokens x 24 blocks (64 MB) does not.
 * - The first call on a device looks up the array's device address on that
 *   device (a CUDA runtime query) and caches it; make that first call before
 *   any stream capture.  cudaDeviceReset invalidates the cached address:
 *   do not call this entry point on a device after resetting it.
 * - Every call on a device shares the one array: calls that may run at the
 *   same time on the GPU (different streams, other host threads) race and
 *   corrupt each other's results.  Serialise them.
 * - Inputs and outputs (q, blocks, sel_bits, stats) are caller memory, as in
 *   vmoba_score_select. */
int vmoba_score_select_static(const vmoba_shape* shape, const void* q, const float* blocks,
                              float tau, float scale, uint32_t* sel_bits,
                              vmoba_head_stats* stats, cudaStream_t stream);

/* Number of CUDA kernels this library has launched since it was loaded
 * (host-side counter, thread-safe; diagnostics for launch accounting). */
unsigned long long vmoba_kernel_launches(void);

/* Per-kernel device timing (diagnostics).  While enabled, every kernel the
 * library launches is bracketed by two CUDA events on its own stream. */
typedef struct vmoba_trace_entry {
  char name[48];        /* kernel name */
  int launches;         /* launches since the last read */
  double ms;            /* summed device time of those launches */
} vmoba_trace_entry;

/* Turns tracing on (nonzero) or off.  Always VMOBA_OK. */
int vmoba_trace_enable(int on);

/* Waits for the traced launches, writes up to max_entries aggregated
 * entries (one per kernel name) and clears the trace.  Returns the number of
 * distinct kernel names (may exceed max_entries; out may be NULL). */
int vmoba_trace_read(vmoba_trace_entry* out, int max_entries);

/* Static text of a vmoba_status code. */
const char* vmoba_status_string(int status);

/* Name of the CUDA error (e.g. "cudaErrorInvalidValue") behind the calling
 * host thread's most recent VMOBA_ERR_CUDA, or "cudaSuccess" if none.  Each
 * compute call first drops any error another caller left in the thread's
 * runtime error slot, so a returned VMOBA_ERR_CUDA is the library's own. */
const char* vmoba_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* VMOBA_H_ */
