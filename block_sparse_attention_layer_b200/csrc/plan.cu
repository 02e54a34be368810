// Tile work lists for the sparse attention kernels, built from a selection
// bitmap (the (query, block) pair mask of VMoBA notes, key design 2).
//
// Queries and keys are both walked in partition order in tiles of 128
// positions, so a query tile holds spatially coherent tokens of one box
// region.  For query tile t of head h the union of its rows' selected blocks
// is turned into the set of key tiles those blocks overlap
// (qt_kt_bits[h][t], a bitmap over key tiles); the transpose
// (kt_qt_bits[h][kt]) lists the query tiles that touch key tile kt, which
// the key-stationary backward walks.  Per-row masking inside a tile is done
// by the attention kernels from the bitmap itself.
#include "common.cuh"
#include "pairs.cuh"

namespace vmoba {
namespace {

__global__ void k_plan_clear(uint32_t* __restrict__ kt_qt, uint32_t* __restrict__ kt_work,
                             size_t n_bits_words, size_t n_work, int* __restrict__ status) {
  // a new plan starts with a clean device status word
  if (blockIdx.x == 0 && threadIdx.x == 0) *status = VMOBA_OK;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_bits_words;
       i += (size_t)gridDim.x * blockDim.x)
    kt_qt[i] = 0u;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_work;
       i += (size_t)gridDim.x * blockDim.x)
    kt_work[i] = 0u;
}

// One CTA (128 threads = 128 rows) per (query tile, head).
__global__ void __launch_bounds__(kTile)
k_plan_tiles(Prob P, const uint32_t* __restrict__ sel, uint32_t* __restrict__ qt_kt,
             uint32_t* __restrict__ qt_work, uint32_t* __restrict__ kt_qt,
             uint32_t* __restrict__ kt_work) {
  __shared__ uint32_t uni[kMaxBlocks / 32];
  __shared__ uint32_t kts[kMaxTiles / 32];
  const int t = blockIdx.x, h = blockIdx.y;
  for (int w = threadIdx.x; w < P.Wb; w += blockDim.x) uni[w] = 0u;
  for (int w = threadIdx.x; w < P.Wqt; w += blockDim.x) kts[w] = 0u;
  __syncthreads();
  const int p = t * kTile + threadIdx.x;
  if (p < P.s) {
    const int i = perm_token(P, p);
    const uint32_t* row = sel + ((size_t)h * P.s + i) * P.Wb;
    for (int w = 0; w < P.Wb; ++w) {
      uint32_t bits = __ldg(row + w);
      if (bits) atomicOr(&uni[w], bits);
    }
  }
  __syncthreads();
  // every selected block marks the key tiles it overlaps
  for (int j = threadIdx.x; j < P.Nb; j += blockDim.x) {
    if (!((uni[j >> 5] >> (j & 31)) & 1u)) continue;
    const int k0 = (j * P.L) / kTile;
    const int k1 = (j * P.L + P.L - 1) / kTile;
    for (int kt = k0; kt <= k1; ++kt) atomicOr(&kts[kt >> 5], 1u << (kt & 31));
  }
  __syncthreads();
  uint32_t* out = qt_kt + ((size_t)h * P.n_qt + t) * P.Wqt;
  int cnt = 0;
  for (int w = threadIdx.x; w < P.Wqt; w += blockDim.x) {
    const uint32_t bits = kts[w];
    out[w] = bits;
    cnt += __popc(bits);
    uint32_t b = bits;
    while (b) {
      const int kt = w * 32 + __ffs(b) - 1;
      b &= b - 1;
      atomicOr(&kt_qt[((size_t)h * P.n_qt + kt) * P.Wqt + (t >> 5)], 1u << (t & 31));
      atomicAdd(&kt_work[(size_t)h * P.n_qt + kt], 1u);
    }
  }
  // block reduce of the key-tile count
  __shared__ int red[kTile / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < kTile / 32; ++w) tot += red[w];
    qt_work[(size_t)h * P.n_qt + t] = (uint32_t)tot;
  }
}

}  // namespace

cudaError_t launch_plan(const Prob& P, const uint32_t* sel, void* ws, const WsLayout& L,
                        cudaStream_t st) {
  uint32_t* qt_kt = ws_ptr<uint32_t>(ws, L.qt_kt_bits);
  uint32_t* qt_work = ws_ptr<uint32_t>(ws, L.qt_work);
  uint32_t* kt_qt = ws_ptr<uint32_t>(ws, L.kt_qt_bits);
  uint32_t* kt_work = ws_ptr<uint32_t>(ws, L.kt_work);
  // the tile bitmaps serve the CUDA-core kernels only; the tensor-core
  // kernels walk the pair lists
  const bool tiles = !uses_blk_path(P);
  const size_t nbw = tiles ? (size_t)P.n_h * P.n_qt * P.Wqt : 0;
  const size_t nw = tiles ? (size_t)P.n_h * P.n_qt : 0;
  {
    VMOBA_TRACE("k_plan_clear", st);
    k_plan_clear<<<tiles ? 148 : 1, 256, 0, st>>>(kt_qt, kt_work, nbw, nw,
                                                   ws_ptr<int>(ws, L.status));
  }
  if (tiles) {
    dim3 grid(P.n_qt, P.n_h);
    VMOBA_TRACE("k_plan_tiles", st);
    k_plan_tiles<<<grid, kTile, 0, st>>>(P, sel, qt_kt, qt_work, kt_qt, kt_work);
  }
  count_launches(tiles ? 2 : 1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_pairs(P, sel, pairs_view(P, ws_ptr<char>(ws, L.pairs)), ws_ptr<int>(ws, L.status),
                      st);
}

}  // namespace vmoba
