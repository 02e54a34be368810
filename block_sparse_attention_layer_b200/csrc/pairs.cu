// Pair lists of the selection bitmap (the (query, block) mask of VMoBA notes,
// key design 2), built on the device for the block-major attention kernels.
//
// For every head h:
//   row_cnt[i]   number of blocks query i selected;
//   row_off[i]   exclusive prefix of row_cnt: the pairs of query i occupy
//                slots row_off[i] .. row_off[i]+row_cnt[i]-1, in block order
//                ("CSR");
//   col_off[j]   start of block j's query list in col_rows ("CSC"), queries
//                in ascending order (deterministic);
//   item_off[j]  first work item of block j: its query list cut into tiles of
//                128 queries; item_off[N_b] = number of work items;
//   slot_row     for every CSR slot, the item row of that (query, block) pair:
//                128 item_off[j] + its position in block j's list.  The
//                attention kernels write partial results item by item (whole
//                128-row tiles) and the merges read them through slot_row in
//                each query's block order;
//   pitem_off[j] the same for pairs of consecutive tiles (256 queries);
//   blk_order    the blocks by list length, longest first (ties: lower j
//                first), so that kernels launching one CTA per block start
//                the longest ones first.
// Rows are processed in chunks of 256 (8 warps x 32 rows); per-chunk column
// counts give each chunk's base inside every block list, and warp ballots
// give each row's rank inside the chunk.
#include "common.cuh"
#include "pairs.cuh"

namespace vmoba {
namespace {

constexpr int kChunkRows = 256;

// Per (chunk, head): column counts of the chunk and the row popcounts.
__global__ void __launch_bounds__(kChunkRows)
k_pairs_count(Prob P, const uint32_t* __restrict__ sel, uint32_t* __restrict__ row_cnt,
              uint32_t* __restrict__ chunk_cnt, int n_chunks) {
  __shared__ uint32_t cc[kMaxBlocks];
  const int c = blockIdx.x, h = blockIdx.y;
  for (int j = threadIdx.x; j < P.Nb; j += blockDim.x) cc[j] = 0u;
  __syncthreads();
  const int i = c * kChunkRows + threadIdx.x;
  const int lane = threadIdx.x & 31;
  uint32_t n = 0;
  for (int w = 0; w < P.Wb; ++w) {
    const uint32_t bits = (i < P.s) ? __ldg(sel + ((size_t)h * P.s + i) * P.Wb + w) : 0u;
    n += __popc(bits);
    // column counts of this warp's 32 rows, one ballot per column of the word
    const int jmax = min(32, P.Nb - w * 32);
    for (int b = 0; b < jmax; ++b) {
      const unsigned m = __ballot_sync(0xffffffffu, (bits >> b) & 1u);
      if (lane == 0 && m) atomicAdd(&cc[w * 32 + b], (uint32_t)__popc(m));
    }
  }
  if (i < P.s) row_cnt[(size_t)h * P.s + i] = n;
  __syncthreads();
  for (int j = threadIdx.x; j < P.Nb; j += blockDim.x)
    chunk_cnt[((size_t)h * n_chunks + c) * P.Nb + j] = cc[j];
}

// Block-wide exclusive scan helper (blockDim.x == 1024).
__device__ uint32_t block_excl_scan(uint32_t v, uint32_t* sh, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = sh[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sh[lane] = s;
  }
  __syncthreads();
  const uint32_t before = (warp > 0 ? sh[warp - 1] : 0u) + x - v;
  *total = sh[31];
  __syncthreads();
  return before;
}

// One CTA (1024 threads) per head: column totals and offsets, chunk bases,
// work-item offsets, and the row offsets (CSR).
__global__ void __launch_bounds__(1024)
k_pairs_scan(Prob P, uint32_t* __restrict__ row_cnt, uint32_t* __restrict__ chunk_cnt,
             int n_chunks, uint32_t* __restrict__ row_off, uint32_t* __restrict__ col_off,
             uint32_t* __restrict__ item_off, uint32_t* __restrict__ pitem_off,
             uint32_t* __restrict__ head_totals, uint32_t* __restrict__ blk_order,
             int* __restrict__ status) {
  __shared__ uint32_t sh[32];
  __shared__ uint32_t len[kMaxBlocks];
  const int h = blockIdx.x, t = threadIdx.x;
  uint32_t* cc = chunk_cnt + (size_t)h * n_chunks * P.Nb;
  // column totals (one thread per block)
  uint32_t tot = 0;
  if (t < P.Nb)
    for (int c = 0; c < n_chunks; ++c) tot += cc[(size_t)c * P.Nb + t];
  uint32_t all;
  const uint32_t off = block_excl_scan(t < P.Nb ? tot : 0u, sh, &all);
  if (all > P.cap) {
    // more pairs than the workspace holds: the head is left empty (every
    // count and offset 0, so the attention kernels do nothing for it and its
    // outputs are zero) and the device status word says why
    for (int j = t; j <= P.Nb; j += blockDim.x) {
      col_off[(size_t)h * (P.Nb + 1) + j] = 0u;
      item_off[(size_t)h * (P.Nb + 1) + j] = 0u;
      pitem_off[(size_t)h * (P.Nb + 1) + j] = 0u;
      if (j < P.Nb) blk_order[(size_t)h * P.Nb + j] = (uint32_t)j;
    }
    for (int i = t; i < P.s; i += blockDim.x) {
      row_cnt[(size_t)h * P.s + i] = 0u;
      row_off[(size_t)h * (P.s + 1) + i] = 0u;
    }
    if (t == 0) {
      row_off[(size_t)h * (P.s + 1) + P.s] = 0u;
      head_totals[4 * h] = head_totals[4 * h + 1] = head_totals[4 * h + 2] = 0u;
      head_totals[4 * h + 3] = 1u;             // overflow: k_pairs_fill skips the head
      atomicExch(status, (int)VMOBA_ERR_WORKSPACE);
    }
    return;
  }
  const uint32_t tiles = t < P.Nb ? (tot + kTile - 1) / kTile : 0u;
  uint32_t n_items, n_pitems;
  const uint32_t ioff = block_excl_scan(tiles, sh, &n_items);
  const uint32_t poff = block_excl_scan((tiles + 1) / 2, sh, &n_pitems);
  if (t < P.Nb) len[t] = tot;
  __syncthreads();
  if (t < P.Nb) {
    uint32_t rank = 0;
    for (int u = 0; u < P.Nb; ++u) rank += (len[u] > tot || (len[u] == tot && u < t)) ? 1u : 0u;
    blk_order[(size_t)h * P.Nb + rank] = (uint32_t)t;
  }
  if (t < P.Nb) {
    col_off[(size_t)h * (P.Nb + 1) + t] = off;
    item_off[(size_t)h * (P.Nb + 1) + t] = ioff;
    pitem_off[(size_t)h * (P.Nb + 1) + t] = poff;
    // chunk bases in place: base of chunk c in block t's list
    uint32_t run = off;
    for (int c = 0; c < n_chunks; ++c) {
      const uint32_t v = cc[(size_t)c * P.Nb + t];
      cc[(size_t)c * P.Nb + t] = run;
      run += v;
    }
  }
  if (t == 0) {
    col_off[(size_t)h * (P.Nb + 1) + P.Nb] = all;
    item_off[(size_t)h * (P.Nb + 1) + P.Nb] = n_items;
    pitem_off[(size_t)h * (P.Nb + 1) + P.Nb] = n_pitems;
    head_totals[4 * h] = all;
    head_totals[4 * h + 1] = n_items;
    head_totals[4 * h + 2] = n_pitems;
    head_totals[4 * h + 3] = 0u;
  }
  // row offsets: exclusive scan of row_cnt over s rows, 1024 at a time
  uint32_t carry = 0;
  for (int base = 0; base < P.s; base += 1024) {
    const int i = base + t;
    const uint32_t v = i < P.s ? row_cnt[(size_t)h * P.s + i] : 0u;
    uint32_t sum;
    const uint32_t ex = block_excl_scan(v, sh, &sum);
    if (i < P.s) row_off[(size_t)h * (P.s + 1) + i] = carry + ex;
    carry += sum;
  }
  if (t == 0) row_off[(size_t)h * (P.s + 1) + P.s] = carry;
}

// Per (chunk, head): write every row of the chunk into the lists of the
// blocks it selected, at chunk base + rank among the chunk's rows, and the
// item row of that entry at the row's pair slot (its CSR offset plus the
// blocks below j it selected).
__global__ void __launch_bounds__(kChunkRows)
k_pairs_fill(Prob P, const uint32_t* __restrict__ sel, const uint32_t* __restrict__ chunk_base,
             const uint32_t* __restrict__ head_totals, int n_chunks,
             const uint32_t* __restrict__ row_off,
             const uint32_t* __restrict__ col_off, const uint32_t* __restrict__ item_off,
             uint32_t* __restrict__ col_rows, uint32_t* __restrict__ slot_row) {
  __shared__ uint32_t wcnt[kChunkRows / 32][32];
  const int c = blockIdx.x, h = blockIdx.y;
  if (head_totals[4 * h + 3] != 0u) return;      // the head overflowed the workspace
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = c * kChunkRows + threadIdx.x;
  const uint32_t* cb = chunk_base + ((size_t)h * n_chunks + c) * P.Nb;
  uint32_t* rows = col_rows + (size_t)h * P.cap;
  uint32_t* srow = slot_row + (size_t)h * P.cap;
  const uint32_t* coff = col_off + (size_t)h * (P.Nb + 1);
  const uint32_t* ioff = item_off + (size_t)h * (P.Nb + 1);
  uint32_t slot = (i < P.s) ? __ldg(row_off + (size_t)h * (P.s + 1) + i) : 0u;
  for (int w = 0; w < P.Wb; ++w) {
    const uint32_t bits = (i < P.s) ? __ldg(sel + ((size_t)h * P.s + i) * P.Wb + w) : 0u;
    const int jmax = min(32, P.Nb - w * 32);
    // counts of each warp for the 32 columns of this word
    for (int b = 0; b < jmax; ++b) {
      const unsigned m = __ballot_sync(0xffffffffu, (bits >> b) & 1u);
      if (lane == b) wcnt[warp][b] = __popc(m);
    }
    __syncthreads();
    // prefix over warps -> base of each warp for each column
    if (warp == 0 && lane < jmax) {
      uint32_t run = cb[w * 32 + lane];
      for (int ww = 0; ww < kChunkRows / 32; ++ww) {
        const uint32_t v = wcnt[ww][lane];
        wcnt[ww][lane] = run;
        run += v;
      }
    }
    __syncthreads();
    for (int b = 0; b < jmax; ++b) {
      const unsigned m = __ballot_sync(0xffffffffu, (bits >> b) & 1u);
      if ((bits >> b) & 1u) {
        const uint32_t rank = __popc(m & ((1u << lane) - 1u));
        const uint32_t e = wcnt[warp][b] + rank;    // entry of block j's list
        const int j = w * 32 + b;
        rows[e] = (uint32_t)i;
        srow[slot++] = kTile * __ldg(ioff + j) + (e - __ldg(coff + j));
      }
    }
    __syncthreads();
  }
}

}  // namespace

size_t pairs_ws_bytes(const Prob& P) {
  const int n_chunks = (P.s + kChunkRows - 1) / kChunkRows;
  size_t b = 0;
  auto take = [&](size_t x) { b += align_up(x, 256); };
  take(sizeof(uint32_t) * (size_t)P.n_h * P.s);                 // row_cnt
  take(sizeof(uint32_t) * (size_t)P.n_h * (P.s + 1));           // row_off
  take(sizeof(uint32_t) * (size_t)P.n_h * (P.Nb + 1));          // col_off
  take(sizeof(uint32_t) * (size_t)P.n_h * (P.Nb + 1));          // item_off
  take(sizeof(uint32_t) * (size_t)P.n_h * (P.Nb + 1));          // pitem_off
  take(sizeof(uint32_t) * 4 * P.n_h);                           // head totals
  take(sizeof(uint32_t) * (size_t)P.n_h * n_chunks * P.Nb);     // chunk counts / bases
  take(sizeof(uint32_t) * (size_t)P.n_h * P.cap);               // col_rows
  take(sizeof(uint32_t) * (size_t)P.n_h * P.cap);               // slot_row
  take(sizeof(uint32_t) * (size_t)P.n_h * P.Nb);                // blk_order
  return b;
}

PairsView pairs_view(const Prob& P, void* base) {
  const int n_chunks = (P.s + kChunkRows - 1) / kChunkRows;
  PairsView v{};
  char* p = static_cast<char*>(base);
  auto take = [&](size_t x) { char* r = p; p += align_up(x, 256); return reinterpret_cast<uint32_t*>(r); };
  v.row_cnt = take(sizeof(uint32_t) * (size_t)P.n_h * P.s);
  v.row_off = take(sizeof(uint32_t) * (size_t)P.n_h * (P.s + 1));
  v.col_off = take(sizeof(uint32_t) * (size_t)P.n_h * (P.Nb + 1));
  v.item_off = take(sizeof(uint32_t) * (size_t)P.n_h * (P.Nb + 1));
  v.pitem_off = take(sizeof(uint32_t) * (size_t)P.n_h * (P.Nb + 1));
  v.head_totals = take(sizeof(uint32_t) * 4 * P.n_h);
  v.chunk = take(sizeof(uint32_t) * (size_t)P.n_h * n_chunks * P.Nb);
  v.col_rows = take(sizeof(uint32_t) * (size_t)P.n_h * P.cap);
  v.slot_row = take(sizeof(uint32_t) * (size_t)P.n_h * P.cap);
  v.blk_order = take(sizeof(uint32_t) * (size_t)P.n_h * P.Nb);
  v.n_chunks = n_chunks;
  return v;
}

cudaError_t launch_pairs(const Prob& P, const uint32_t* sel, const PairsView& v, int* status,
                         cudaStream_t st) {
  dim3 g(v.n_chunks, P.n_h);
  {
    VMOBA_TRACE("k_pairs_count", st);
    k_pairs_count<<<g, kChunkRows, 0, st>>>(P, sel, v.row_cnt, v.chunk, v.n_chunks);
  }
  {
    VMOBA_TRACE("k_pairs_scan", st);
    k_pairs_scan<<<P.n_h, 1024, 0, st>>>(P, v.row_cnt, v.chunk, v.n_chunks, v.row_off, v.col_off,
                                         v.item_off, v.pitem_off, v.head_totals, v.blk_order,
                                         status);
  }
  {
    VMOBA_TRACE("k_pairs_fill", st);
    k_pairs_fill<<<g, kChunkRows, 0, st>>>(P, sel, v.chunk, v.head_totals, v.n_chunks, v.row_off,
                                           v.col_off,
                                           v.item_off, v.col_rows, v.slot_row);
  }
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace vmoba
