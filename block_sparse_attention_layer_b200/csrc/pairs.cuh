// Device pair lists of a selection bitmap (see pairs.cu).
#pragma once

#include "common.cuh"

namespace vmoba {

struct PairsView {
  uint32_t* row_cnt;      // [n_h][s]
  uint32_t* row_off;      // [n_h][s+1]   CSR offsets (pair slots of each query)
  uint32_t* col_off;      // [n_h][N_b+1] start of each block's query list
  uint32_t* item_off;     // [n_h][N_b+1] first 128-query work item of each block
  uint32_t* head_totals;  // [n_h][2]     pairs, work items
  uint32_t* chunk;        // [n_h][chunks][N_b] scratch (chunk bases)
  uint32_t* col_rows;     // [n_h][s*N_b] query lists, block by block
  int n_chunks;
};

// Item-ordered copies (gather.cu): bf16 rows of Q and dO, fp32 LSE*log2e and D.
struct ItemBufs {
  __nv_bfloat16* qg;
  __nv_bfloat16* dog;
  float* l2g;
  float* dg;
  size_t rows;   // capacity
};

size_t pairs_ws_bytes(const Prob& P);
PairsView pairs_view(const Prob& P, void* base);
cudaError_t launch_pairs(const Prob& P, const uint32_t* sel, const PairsView& v, cudaStream_t st);

cudaError_t launch_attn_fwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                                const uint32_t* sel, const PairsView& pv, void* part,
                                const ItemBufs& ib, float scale, void* out, float* o32,
                                float* lse, int* status, int num_sms, cudaStream_t st);

size_t item_rows_capacity(const Prob& P);
cudaError_t launch_gather_items(const Prob& P, int h, const PairsView& pv,
                                const __nv_bfloat16* a, const __nv_bfloat16* b,
                                __nv_bfloat16* ag, __nv_bfloat16* bg, const float* fa,
                                const float* fb, float* fag, float* fbg, float fa_pad,
                                int num_sms, cudaStream_t st);

size_t bwd_blk_ws_bytes(const Prob& P);
cudaError_t launch_attn_bwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                                const uint32_t* sel, const PairsView& pv, void* part,
                                const ItemBufs& ib, const float* o32, const float* lse,
                                const void* dout, void* dq, void* dk, void* dv, void* ws_bwd,
                                float scale, int* status, int num_sms, cudaStream_t st);

// Pair slot of (query i, block j) for a selected pair: CSR offset of the row
// plus the number of blocks below j the row selected.
__device__ __forceinline__ uint32_t pair_slot(const uint32_t* __restrict__ row_off_h,
                                              const uint32_t* __restrict__ sel_row, int Wb,
                                              int i, int j) {
  uint32_t r = 0;
  const int wj = j >> 5;
  for (int w = 0; w < wj; ++w) r += __popc(__ldg(sel_row + w));
  r += __popc(__ldg(sel_row + wj) & ((1u << (j & 31)) - 1u));
  (void)Wb;
  return __ldg(row_off_h + i) + r;
}

}  // namespace vmoba
