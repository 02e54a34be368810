// Item-ordered copies of the rows the backward kernels read as tiles.
//
// Work item n of a head (block j, query tile g of block j's list) covers rows
// [128 n, 128 n + 128) of the copy: row r holds the r-th query of the tile,
// rows past the list end are zero.  The backward kernels (dQ pass, dK/dV
// pass) then fetch query tiles with plain 2-D TMA instead of scattered
// loads; the forward gathers its own query rows from Q.  Q and dO are
// stored in fp16 (exact within fp16's range), the operand type of the
// backward's MMAs.  With no row source (a == nullptr) only the per-row
// values are rewritten.  One warp per item; D / 8 lanes x 16 bytes move a row
// of head_dim D, 4 instructions in flight per source, at most 64 registers a
// thread so that four 256-thread CTAs share an SM (8 in flight at 88
// registers, two CTAs per SM, were 8 % slower on the 3D layers).
#include "tc_prims.cuh"
#include "pairs.cuh"

namespace vmoba {
namespace {

constexpr int kInFlight = 4;             // warp instructions in flight per batch

template <int D>
__global__ void __launch_bounds__(256, 4)
k_gather_items(Prob P, int h, PairsView pv, const __nv_bfloat16* __restrict__ a,
               const __nv_bfloat16* __restrict__ b, __half* __restrict__ ah,
               __half* __restrict__ bh, const float* __restrict__ fa,
               const float* __restrict__ fb, float* __restrict__ fag, float* __restrict__ fbg,
               float fa_pad) {
  const uint32_t* col_rows = pv.col_rows + (size_t)h * P.cap;
  const int n_items = (int)__ldg(pv.head_totals + 4 * h + 1);
  const int lane = threadIdx.x & 31;
  constexpr int kLpr = D / 8, kRpi = 32 / kLpr;  // lanes per row, rows per instruction
  const int half = lane / kLpr, c = lane % kLpr;  // row of the instruction's kRpi, 16-byte chunk
  const int warps = (gridDim.x * blockDim.x) >> 5;
  int hint = 0;
  for (int n = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; n < n_items; n += warps) {
    const WorkItem it = decode_item<true>(pv, P, h, n, hint);
    const int count = it.count;
    const uint32_t* rows = col_rows + it.first;
    const size_t base = (size_t)n * kTile;
    for (int r0 = 0; a != nullptr && r0 < kTile; r0 += kRpi * kInFlight) {
      uint4 va[kInFlight], vb[kInFlight];
#pragma unroll
      for (int u = 0; u < kInFlight; ++u) {
        const int r = r0 + kRpi * u + half;
        va[u] = make_uint4(0u, 0u, 0u, 0u);
        vb[u] = make_uint4(0u, 0u, 0u, 0u);
        if (r < count) {
          const size_t src = ((size_t)__ldg(rows + r) * P.n_h + h) * D;
          va[u] = __ldg(reinterpret_cast<const uint4*>(a + src) + c);
          if (b) vb[u] = __ldg(reinterpret_cast<const uint4*>(b + src) + c);
        }
      }
#pragma unroll
      for (int u = 0; u < kInFlight; ++u) {
        const size_t dst = (base + r0 + kRpi * u + half) * D;
        reinterpret_cast<uint4*>(ah + dst)[c] = tc::bf16x8_to_f16x8(va[u]);
        if (b) reinterpret_cast<uint4*>(bh + dst)[c] = tc::bf16x8_to_f16x8(vb[u]);
      }
    }
    if (fa) {
      for (int r = lane; r < kTile; r += 32) {
        float x = fa_pad, y = 0.f;
        if (r < count) {
          const uint32_t i = __ldg(rows + r);
          x = __ldg(fa + (size_t)h * P.s + i);
          y = __ldg(fb + (size_t)h * P.s + i);
        }
        fag[base + r] = x;
        fbg[base + r] = y;
      }
    }
  }
}

}  // namespace

size_t item_rows_capacity(const Prob& P) {
  // at most one partial tile per block beyond the pairs themselves
  return (size_t)P.cap + (size_t)kTile * P.Nb;
}

cudaError_t launch_gather_items(const Prob& P, int h, const PairsView& pv,
                                const __nv_bfloat16* a, const __nv_bfloat16* b,
                                __half* ah, __half* bh, const float* fa,
                                const float* fb, float* fag, float* fbg, float fa_pad,
                                int num_sms, cudaStream_t st) {
  {
    VMOBA_TRACE("k_gather_items", st);
    if (P.d == 128)
      k_gather_items<128><<<num_sms * 8, 256, 0, st>>>(P, h, pv, a, b, ah, bh, fa, fb, fag, fbg,
                                                       fa_pad);
    else
      k_gather_items<64><<<num_sms * 8, 256, 0, st>>>(P, h, pv, a, b, ah, bh, fa, fb, fag, fbg,
                                                      fa_pad);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace vmoba

namespace vmoba {

size_t item_bufs_bytes(const Prob& P) {
  const size_t rows = item_rows_capacity(P);
  return 2 * align_up(rows * P.d * sizeof(__half), 256) +
         2 * align_up(rows * sizeof(float), 256);
}

}  // namespace vmoba
