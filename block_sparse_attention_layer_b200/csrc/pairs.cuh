// Device pair lists of a selection bitmap (see pairs.cu).
#pragma once

#include "common.cuh"

namespace vmoba {

struct PairsView {
  uint32_t* row_cnt;      // [n_h][s]
  uint32_t* row_off;      // [n_h][s+1]   CSR offsets (pair slots of each query)
  uint32_t* col_off;      // [n_h][N_b+1] start of each block's query list
  uint32_t* item_off;     // [n_h][N_b+1] first 128-query work item of each block
  uint32_t* pitem_off;    // [n_h][N_b+1] first pair of work items (256 queries) of each block
  uint32_t* head_totals;  // [n_h][4]     pairs, work items, item pairs, 0
  uint32_t* chunk;        // [n_h][chunks][N_b] scratch (chunk bases)
  uint32_t* col_rows;     // [n_h][s*N_b] query lists, block by block
  uint32_t* slot_row;     // [n_h][s*N_b] item row of each CSR pair slot
  uint32_t* blk_order;    // [n_h][N_b]   blocks by query-list length, longest first
  int n_chunks;
};

// A work item: block j and one tile of up to 128 queries of its list.
struct WorkItem {
  int j;                  // block
  int count;              // queries in the tile (0 when the tile does not exist)
  uint32_t first;         // index of the tile's first entry in col_rows
};

// Block j with off[j] <= n < off[j+1], for a non-decreasing offset array
// (off[N_b] > n), scanned forward from `hint` (off[hint] <= n); `hint`
// becomes j.  Every role of a CTA visits its work in increasing order, so the
// scan passes only the blocks finished since its last item.  kWarp: the
// whole warp takes 32 entries per coalesced step (n warp-uniform, all lanes
// present); otherwise one thread steps one entry at a time.
template <bool kWarp>
__device__ __forceinline__ int find_block(const uint32_t* off, int Nb, uint32_t n, int& hint) {
  int j = hint;
  if (kWarp) {
    const int lane = threadIdx.x & 31;
    for (;;) {
      const int jj = j + 1 + lane;
      // entries <= n form a prefix of the window (off is non-decreasing)
      const uint32_t m = __ballot_sync(0xffffffffu, jj <= Nb && __ldg(off + jj) <= n);
      if (m != 0xffffffffu) {
        j += __popc(m);
        break;
      }
      j += 32;
    }
  } else {
    while (__ldg(off + j + 1) <= n) ++j;
  }
  hint = j;
  return j;
}

// Work item n of head h (n < head_totals[4h+1]); `hint` as in find_block
// (0 before a role's first item).
template <bool kWarp>
__device__ __forceinline__ WorkItem decode_item(const PairsView& pv, const Prob& P, int h, int n,
                                                int& hint) {
  const uint32_t* item_off = pv.item_off + (size_t)h * (P.Nb + 1);
  const uint32_t* col_off = pv.col_off + (size_t)h * (P.Nb + 1);
  const int j = find_block<kWarp>(item_off, P.Nb, (uint32_t)n, hint);
  WorkItem it;
  it.j = j;
  const int g = n - (int)__ldg(item_off + j);
  const uint32_t c0 = __ldg(col_off + j), c1 = __ldg(col_off + j + 1);
  it.first = c0 + (uint32_t)g * kTile;
  it.count = min(kTile, (int)(c1 - it.first));
  return it;
}

// Item pair p of head h: tiles 2q and 2q+1 of one block's list (the second
// may be absent).  Returns the first tile; *second gets the other (count 0
// when absent) and *n0 the first tile's work-item index.  `hint` as in
// find_block, over the pair offsets.
template <bool kWarp>
__device__ __forceinline__ WorkItem decode_item_pair(const PairsView& pv, const Prob& P, int h,
                                                     int p, WorkItem* second, int* n0,
                                                     int& hint) {
  const uint32_t* pitem_off = pv.pitem_off + (size_t)h * (P.Nb + 1);
  const uint32_t* item_off = pv.item_off + (size_t)h * (P.Nb + 1);
  const uint32_t* col_off = pv.col_off + (size_t)h * (P.Nb + 1);
  const int j = find_block<kWarp>(pitem_off, P.Nb, (uint32_t)p, hint);
  const int q = p - (int)__ldg(pitem_off + j);
  const uint32_t c0 = __ldg(col_off + j), c1 = __ldg(col_off + j + 1);
  WorkItem a, b;
  a.j = b.j = j;
  a.first = c0 + (uint32_t)q * 2 * kTile;
  b.first = a.first + kTile;
  a.count = min(kTile, (int)(c1 - a.first));
  b.count = c1 > b.first ? min(kTile, (int)(c1 - b.first)) : 0;
  *n0 = (int)__ldg(item_off + j) + 2 * q;
  *second = b;
  return a;
}

// Item-ordered copies (gather.cu) for the backward passes: fp16 rows of Q and
// dO (the bf16 inputs converted; their MMAs take fp16), fp32 -LSE*log2e and D.
struct ItemBufs {
  __half* qh;
  __half* doh;
  float* l2g;
  float* dg;
  size_t rows;   // capacity
};

size_t pairs_ws_bytes(const Prob& P);
PairsView pairs_view(const Prob& P, void* base);
// Builds the pair lists; a head with more pairs than P.cap is left empty and
// VMOBA_ERR_WORKSPACE is latched in *status.
cudaError_t launch_pairs(const Prob& P, const uint32_t* sel, const PairsView& v, int* status,
                         cudaStream_t st);

cudaError_t launch_attn_fwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                                const uint32_t* sel, const PairsView& pv, void* part,
                                const ItemBufs& ib, float scale, void* out, float* o32,
                                float* lse, int* status, int num_sms, cudaStream_t st);

size_t item_rows_capacity(const Prob& P);
cudaError_t launch_gather_items(const Prob& P, int h, const PairsView& pv,
                                const __nv_bfloat16* a, const __nv_bfloat16* b,
                                __half* ah, __half* bh, const float* fa,
                                const float* fb, float* fag, float* fbg, float fa_pad,
                                int num_sms, cudaStream_t st);

size_t bwd_blk_ws_bytes(const Prob& P);
cudaError_t launch_attn_bwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                                const uint32_t* sel, const PairsView& pv, void* part,
                                const ItemBufs& ib, const float* o32, const float* lse,
                                const void* dout, void* dq, void* dk, void* dv, void* ws_bwd,
                                float scale, int* status, int num_sms, cudaStream_t st);

}  // namespace vmoba
