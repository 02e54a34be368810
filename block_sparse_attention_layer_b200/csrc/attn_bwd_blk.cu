// Sparse attention backward, block-major, on the 5th-generation tensor cores
// (bf16, head_dim D = 64 or 128).  The selection mask is held constant (the pages add
// no loss and route no gradient through it):
//   P = exp(scale q.k - LSE),  D_i = dO_i . O_i,  dS = P (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO   (selected pairs only).
//
// Two passes over the pair lists (pairs.cu), no atomics, deterministic:
//  * dQ pass: a work item is (block j, 128 queries of block j's list); it
//    walks the block's keys in chunks of 128: S = Q K^T, dP = dO V^T, then
//    dS in TMEM and dQ += dS K.  The per-pair partial dQ goes to the item's
//    rows (128 n + r) by asynchronous TMA stores of each warp's staging
//    tile; a merge sums each query's partials, found through the pair lists'
//    slot -> item row map, in ascending block order.
//  * dK/dV pass: a work item is (block j, 128-key tile of block j); it walks
//    all query tiles of block j's list: S^T = K Q^T, dP^T = V dO^T,
//    P^T and dS^T in TMEM, dV += P^T dO, dK += dS^T Q; dK, dV of the tile's
//    keys are complete at the end and are written in original key order.
// Both passes take fp16 operands: dK and dV sum over every query of a
// block's list (tens of thousands in the large layers), and with P and dS
// rounded to bf16 (8 significant bits) the rounding alone moves them by more
// than 2e-2; fp16 (11 bits) keeps it near 1/8 of that.  K' and V' are
// copied to fp16 once per call and the query tiles come from fp16
// item-ordered copies (exact conversions of the bf16 inputs within fp16's
// range, |x| <= 65504; P is in [0, 1] and dS = P (dP - D) must stay below
// 65504 too).  Its D_i is the sum of P dP over the row's
//    selected keys, accumulated by the dQ pass, not dO_i . O_i from the
//    forward's output copy: dK sums D's error times P q over every query of
//    the list, and the output copy carries the forward's bf16 P.
// D_i comes from the forward's fp32 output copy.
#include "tc_prims.cuh"
#include "pairs.cuh"

namespace vmoba {
namespace {

using namespace tc;

// 128 rows x 64 bf16: one 128-byte swizzle atom wide; a 128-row tile of
// head_dim D is D / 64 of them side by side
constexpr uint32_t kHalf = 128 * 64 * 2;
template <int D>
constexpr uint32_t tile_bytes() { return (D / 64) * kHalf; }
// 384 threads: warp 0 TMA, warp 1 MMA, warps 4-7 and 8-11 two softmax
// warpgroups that split each tile's 128 columns 64/64 (a warp reaches TMEM
// lanes 32*(warp % 4) .. +32, so both groups cover all 128 rows).
constexpr int kThreads = 384;
constexpr int kSoftmaxWarps = 8;
// Column of the packed bf16 operand (P, P^T, dS, dS^T) for 16-wide step kk:
// group g writes its 64 columns, packed two per 32-bit column, at 64 g.
__device__ __forceinline__ uint32_t packed_col(int kk) { return (kk >> 2) * 64 + (kk & 3) * 8; }
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------- D_i, lse2
// rowD[h][i] = dO_i . O_i (fp32 output copy); nlse2[h][i] = -LSE_i * log2(e),
// so that P = 2^(S scale log2(e) + nlse2) is one fused multiply-add and ex2.
template <int D>
__global__ void k_bwd_rows(Prob P, const float* __restrict__ o32,
                           const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
                           float* __restrict__ rowD, float* __restrict__ lse2) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= P.s * P.n_h) return;
  const int i = warp / P.n_h, h = warp - i * P.n_h;
  float acc;
  if constexpr (D == 128) {
    const float4 a = reinterpret_cast<const float4*>(o32 + (size_t)warp * D)[lane];
    const uint2 b = reinterpret_cast<const uint2*>(dout + (size_t)warp * D)[lane];
    acc = a.x * __uint_as_float(b.x << 16) + a.y * __uint_as_float(b.x & 0xFFFF0000u) +
          a.z * __uint_as_float(b.y << 16) + a.w * __uint_as_float(b.y & 0xFFFF0000u);
  } else {
    const float2 a = reinterpret_cast<const float2*>(o32 + (size_t)warp * D)[lane];
    const uint32_t b = reinterpret_cast<const uint32_t*>(dout + (size_t)warp * D)[lane];
    acc = a.x * __uint_as_float(b << 16) + a.y * __uint_as_float(b & 0xFFFF0000u);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) {
    rowD[(size_t)h * P.s + i] = acc;
    lse2[(size_t)h * P.s + i] = -lse[(size_t)h * P.s + i] * kLog2e;
  }
}

// =====================================================================
// dQ pass.  Roles: warp 0 TMA (the item's Q and dO tiles from the
// item-ordered copies, then the block's K, V chunks), warp 1 MMA, warps
// 4-7 / 8-11 softmax of key columns 0-63 / 64-127 + epilogue (warps 2-3
// idle).  Per chunk J the softmax reads S(J) and frees it, forms P(J), then
// dS(J) = P (dP - D) once dP(J) is there.  Two TMEM schedules, dQ at
// [384,384+D) in both:
//  - long blocks (more than two key chunks): S double-buffered at [0,128),
//    [128,256), dP (then dS) at [256,384); issue order S(J+1), dQ(J),
//    dP(J+1): S(J+1) runs while dS(J) is formed, dP(J+1) while P(J+1) is;
//  - short blocks (DB): S at [0,128), dP double-buffered at [128,256),
//    [256,384); issue order S(J+1), dP(J+1), dQ(J): chunk J+1's MMAs need
//    not wait for dQ(J) to take dS(J) out of a shared dP buffer.  With long
//    blocks this order asks for K(J+2) right after dQ(J) is issued, before
//    the two-stage K ring can refill, which costs more than it gains.
// =====================================================================
struct DqBars {
  uint64_t full_k[2], empty_k[2], full_v[2], empty_v[2];
  uint64_t s_full[2], s_free[2], dp_full[2], ds_full[2];
  uint64_t qd_full, qd_empty, dq_final, dq_free;
  uint32_t tmem_base;
  int abort;
};
constexpr uint32_t kStageB = 32 * 32 * 4;     // epilogue staging per softmax warp
template <int D>
constexpr size_t dq_smem() {
  return 1024 + 2 * tile_bytes<D>() /*Q,dO*/ + 4 * tile_bytes<D>() /*K,V x2*/ + 8 * kStageB +
         sizeof(DqBars) + 64;
}
static_assert(dq_smem<128>() <= 232448, "shared memory per CTA");

template <int D, bool DB>
__global__ void __launch_bounds__(kThreads, 1)
k_bwd_dq_blk(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
             const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
             const __grid_constant__ CUtensorMap tm_pd, Prob P, int h, PairsView pv,
             const float* __restrict__ dg, const float* __restrict__ l2g, float sl2,
             float* __restrict__ part_d, Watch wt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr uint32_t kTileB = tile_bytes<D>();
  uint8_t* sQ = smem;
  uint8_t* sO = sQ + kTileB;              // dO tile
  uint8_t* sK = sO + kTileB;              // 2 stages
  uint8_t* sV = sK + 2 * kTileB;          // 2 stages
  uint8_t* sStage = sV + 2 * kTileB;      // 8 x kStageB
  DqBars* bars = reinterpret_cast<DqBars*>(sStage + 8 * kStageB);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = (int)__ldg(pv.head_totals + 4 * h + 1);
  const int nch = (P.L + kTile - 1) / kTile;
  const int kc_last = P.L - (nch - 1) * kTile;        // keys in the last chunk
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->full_k[i], 1); mbar_init(&bars->empty_k[i], 1);
      mbar_init(&bars->full_v[i], 1); mbar_init(&bars->empty_v[i], 1);
      mbar_init(&bars->s_full[i], 1); mbar_init(&bars->s_free[i], kSoftmaxWarps);
      mbar_init(&bars->dp_full[i], 1); mbar_init(&bars->ds_full[i], kSoftmaxWarps);
    }
    mbar_init(&bars->qd_full, 1);
    mbar_init(&bars->qd_empty, 1);
    mbar_init(&bars->dq_final, 1);
    mbar_init(&bars->dq_free, kSoftmaxWarps);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tDQ = tmem + 384;
  // TMEM column of S(J) and of dP(J), and the barrier slot / phase parity of
  // chunk J's S and dP barriers, for the two schedules above
  auto tS = [&](int J) -> uint32_t { return DB ? tmem : tmem + 128 * (uint32_t)(J & 1); };
  auto tdP = [&](int J) -> uint32_t {
    return DB ? tmem + 128 + 128 * (uint32_t)(J & 1) : tmem + 256;
  };
  auto s_slot = [](int J) { return DB ? 0 : (J & 1); };
  auto s_par = [](int J) -> uint32_t { return DB ? (J & 1) : ((J >> 1) & 1); };
  auto d_slot = [](int J) { return DB ? (J & 1) : 0; };
  auto d_par = [](int J) -> uint32_t { return DB ? ((J >> 1) & 1) : (J & 1); };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_o);
      int J = 0, it_local = 0, hint = 0;
      bool ok = true;
      for (int n = blockIdx.x; n < n_items && ok; n += G, ++it_local) {
        const WorkItem it = decode_item<false>(pv, P, h, n, hint);
        if (it_local >= 1) ok = mbar_wait(&bars->qd_empty, (it_local - 1) & 1, wt, abort);
        if (!ok) break;
        mbar_expect_tx(&bars->qd_full, 2 * kTileB);
        tma_load_2d(sQ, &tm_q, &bars->qd_full, 0, n * kTile);
        if (D == 128) tma_load_2d(sQ + kHalf, &tm_q, &bars->qd_full, 64, n * kTile);
        tma_load_2d(sO, &tm_o, &bars->qd_full, 0, n * kTile);
        if (D == 128) tma_load_2d(sO + kHalf, &tm_o, &bars->qd_full, 64, n * kTile);
        for (int c = 0; c < nch && ok; ++c, ++J) {
          const int row = h * P.s + it.j * P.L + c * kTile;
          const int st = J & 1;
          if (J >= 2) ok = mbar_wait(&bars->empty_k[st], ((J >> 1) - 1) & 1, wt, abort);
          if (!ok) break;
          mbar_expect_tx(&bars->full_k[st], kTileB);
          tma_load_2d(sK + st * kTileB, &tm_k, &bars->full_k[st], 0, row);
          if (D == 128) tma_load_2d(sK + st * kTileB + kHalf, &tm_k, &bars->full_k[st], 64, row);
          if (J >= 2) ok = mbar_wait(&bars->empty_v[st], ((J >> 1) - 1) & 1, wt, abort);
          if (!ok) break;
          mbar_expect_tx(&bars->full_v[st], kTileB);
          tma_load_2d(sV + st * kTileB, &tm_v, &bars->full_v[st], 0, row);
          if (D == 128) tma_load_2d(sV + st * kTileB + kHalf, &tm_v, &bars->full_v[st], 64, row);
        }
        if (ok && n + G < n_items) {
          // the next item's Q / dO into L2 behind this item's loads (one buffer in smem)
          for (int x = 0; x < D; x += 64) {
            tma_prefetch_l2_2d(&tm_q, x, (n + G) * kTile);
            tma_prefetch_l2_2d(&tm_o, x, (n + G) * kTile);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idSS = idesc_f16(128, 128, false, false);
      const uint32_t idSS_last = idesc_f16(128, (kc_last + 15) & ~15, false, false);
      const uint32_t idDQ = idesc_f16(128, D, false, true);
      const int ks_last = (kc_last + 15) / 16;
      const uint32_t qb = smem_u32(sQ), ob = smem_u32(sO);
      const int my_items = blockIdx.x < n_items ? (n_items - 1 - blockIdx.x) / G + 1 : 0;
      const int total = my_items * nch;                 // chunks of this CTA
      bool ok = true;
      // S(J) = Q K^T; the chunk's first S of an item waits for its Q / dO,
      // every S for the softmax to have read the S it overwrites
      auto issue_s = [&](int J) -> bool {
        const int st = J & 1, c = J % nch, itl = J / nch;
        if (c == 0 && !mbar_wait(&bars->qd_full, itl & 1, wt, abort)) return false;
        const int prev = DB ? J - 1 : J - 2;
        if (prev >= 0 && !mbar_wait(&bars->s_free[s_slot(prev)], s_par(prev), wt, abort))
          return false;
        if (!mbar_wait(&bars->full_k[st], (J >> 1) & 1, wt, abort)) return false;
        tc_fence_after();
        const uint32_t kb = smem_u32(sK + st * kTileB);
        const uint32_t idc = c == nch - 1 ? idSS_last : idSS;   // N = the chunk's keys
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tS(J), desc_sw128(qb + off, 16, 1024), desc_sw128(kb + off, 16, 1024), idc,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[s_slot(J)]);
        return true;
      };
      // dP(J) = dO V^T; overwrites dS(J-1) (DB: dS(J-2)), whose dQ MMA was
      // issued before
      auto issue_dp = [&](int J) -> bool {
        const int st = J & 1, c = J % nch;
        if (!mbar_wait(&bars->full_v[st], (J >> 1) & 1, wt, abort)) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(sV + st * kTileB);
        const uint32_t idc = c == nch - 1 ? idSS_last : idSS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tdP(J), desc_sw128(ob + off, 16, 1024), desc_sw128(vb + off, 16, 1024), idc,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->empty_v[st]);
        mma_commit(&bars->dp_full[d_slot(J)]);
        if (c == nch - 1) mma_commit(&bars->qd_empty);  // item's last reader of Q / dO
        return true;
      };
      // dQ += dS(J) K(J); dS packed over the dP columns
      auto issue_dq = [&](int J) -> bool {
        const int st = J & 1, c = J % nch, itl = J / nch;
        if (!mbar_wait(&bars->ds_full[d_slot(J)], d_par(J), wt, abort)) return false;
        if (c == 0 && itl > 0 && !mbar_wait(&bars->dq_free, (itl - 1) & 1, wt, abort))
          return false;
        tc_fence_after();
        const uint32_t kb = smem_u32(sK + st * kTileB);
        const int ks = c == nch - 1 ? ks_last : 8;
        for (int kk = 0; kk < ks; ++kk)
          mma_ts(tDQ, tdP(J) + packed_col(kk), desc_sw128(kb + kk * 2048, kHalf, 1024), idDQ,
                 (c > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty_k[st]);
        if (c == nch - 1) mma_commit(&bars->dq_final);
        return true;
      };
      if (total > 0) ok = issue_s(0) && issue_dp(0);
      for (int J = 0; J < total && ok; ++J) {
        const bool more = J + 1 < total;
        if (more && (J + 1) % nch == 0) {
          // next item: its Q / dO arrive after this item's last dP, so issue dQ first
          ok = issue_dq(J) && issue_s(J + 1) && issue_dp(J + 1);
        } else if (more) {
          ok = DB ? (issue_s(J + 1) && issue_dp(J + 1) && issue_dq(J))
                  : (issue_s(J + 1) && issue_dq(J) && issue_dp(J + 1));
        } else {
          ok = issue_dq(J);
        }
      }
    }
  } else if (warp >= 4) {
    const int wq = warp & 3, wg = (warp - 4) >> 2;   // lane quarter, column group
    const int r = wq * 32 + lane;
    const int cb = 64 * wg;                         // this group's key columns
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    float* stg = reinterpret_cast<float*>(sStage + (warp - 4) * kStageB);
    const uint64_t sl2x2 = f32x2(sl2, sl2);
    int J = 0, it_local = 0;
    bool ok = true;
    // -LSE log2(e) and D of the row in item nn (the item-ordered copies hold
    // -inf and 0 past the tile's queries); loaded one item ahead, before the
    // epilogue, so their latency is off the critical path
    auto fetch = [&](int nn, float& l2, float& d) {
      l2 = __ldg(l2g + (size_t)nn * kTile + r);
      d = __ldg(dg + (size_t)nn * kTile + r);
    };
    float nx_l2 = -INFINITY, nx_d = 0.f;
    if (blockIdx.x < n_items) fetch(blockIdx.x, nx_l2, nx_d);
    for (int n = blockIdx.x; n < n_items && ok; n += G, ++it_local) {
      const uint64_t nl2x2 = f32x2(nx_l2, nx_l2), Dx2 = f32x2(nx_d, nx_d);
      // sum of P dP over the group's keys of this block: the block's share of
      // D_i = dO_i . O_i = sum_k P_ik dP_ik, exact to fp32 (the D used above
      // comes from the forward's output copy); the dQ merge adds the shares
      // up and the dK/dV pass uses that sum
      uint64_t dacc = f32x2(0.f, 0.f);
      for (int c = 0; c < nch; ++c, ++J) {
        const int sb = s_slot(J), db = d_slot(J);
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], s_par(J), wt, abort));
        if (!ok) break;
        tc_fence_after();
        const int lim = (c == nch - 1 ? kc_last : kTile) - cb;   // valid columns of this group
        if (lim <= 0) {
          // no key of this chunk in the group's columns: the dQ MMA reads none of them
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->s_free[sb]);
          ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full[db], d_par(J), wt, abort));
          if (!ok) break;
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->ds_full[db]);
          continue;
        }
        const bool full = lim >= 64;
        // P for the group's 64 key columns; rows past the tile's end give P = 0
        uint32_t pr[64];
        tmem_ld32(tS(J) + lane_off + cb, pr);
        tmem_ld32(tS(J) + lane_off + cb + 32, pr + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[sb]);   // S may be overwritten now
        if (full) {
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float2 t = f32x2_split(
                fma_x2(f32x2(__uint_as_float(pr[e]), __uint_as_float(pr[e + 1])), sl2x2, nl2x2));
            pr[e] = __float_as_uint(fast_exp2(t.x));
            pr[e + 1] = __float_as_uint(fast_exp2(t.y));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float2 t = f32x2_split(
                fma_x2(f32x2(__uint_as_float(pr[e]), __uint_as_float(pr[e + 1])), sl2x2, nl2x2));
            // columns past the chunk's keys: S is not written there, P = 0
            pr[e] = __float_as_uint(e < lim ? fast_exp2(t.x) : 0.f);
            pr[e + 1] = __float_as_uint(e + 1 < lim ? fast_exp2(t.y) : 0.f);
          }
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full[db], d_par(J), wt, abort));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {                  // 32 dP columns per wait
          uint32_t dp[32];
          tmem_ld32(tdP(J) + lane_off + cb + hh * 32, dp);
          tmem_ld_wait();
          uint32_t pk[16];
          if (full) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int x = hh * 32 + e;
              const uint64_t dp2 = f32x2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1]));
              const uint64_t p2 = f32x2(__uint_as_float(pr[x]), __uint_as_float(pr[x + 1]));
              const float2 ds = f32x2_split(mul_x2(p2, sub_x2(dp2, Dx2)));
              pk[e >> 1] = pack_f16x2(ds.x, ds.y);
              dacc = fma_x2(p2, dp2, dacc);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int x = hh * 32 + e;
              // dP past the chunk's keys is stale; P = 0 there must not meet it
              const uint64_t dp2 = f32x2(x < lim ? __uint_as_float(dp[e]) : 0.f,
                                         x + 1 < lim ? __uint_as_float(dp[e + 1]) : 0.f);
              const uint64_t p2 = f32x2(__uint_as_float(pr[x]), __uint_as_float(pr[x + 1]));
              const float2 ds = f32x2_split(mul_x2(p2, sub_x2(dp2, Dx2)));
              pk[e >> 1] = pack_f16x2(ds.x, ds.y);
              dacc = fma_x2(p2, dp2, dacc);
            }
          }
          // dS into the group's columns [cb + 16 hh, +16): dP columns already read
          tmem_st16(tdP(J) + lane_off + cb + hh * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->ds_full[db]);
      }
      if (!ok) break;
      if (n + G < n_items) fetch(n + G, nx_l2, nx_d);
      {
        const float2 dsum = f32x2_split(dacc);
        part_d[((size_t)n * kTile + r) * 2 + wg] = dsum.x + dsum.y;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dq_final, it_local & 1, wt, abort));
      if (!ok) break;
      tc_fence_after();
      // the partial leaves rounded to fp16 (the merge adds the partials in
      // fp32): a thread's 64 columns of its row are one 128-byte staging
      // row, and each warp's 32 rows one asynchronous store; the groups take
      // columns 0-63 / 64-127 (head_dim 64: group 0 takes all of them)
      if (D == 128 || wg == 0) {
        const int c0 = D == 128 ? 64 * wg : 0;
        uint32_t xr[64];
        tmem_ld32(tDQ + lane_off + c0, xr);
        tmem_ld32(tDQ + lane_off + c0 + 32, xr + 32);
        tmem_ld_wait();
        // the staging tile is free once the previous store has read it
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
        // row `lane` into the staging tile in the 128-byte swizzle of the
        // store's tensor map: 16-byte granule g at g ^ (row & 7)
        uint32_t* stw = reinterpret_cast<uint32_t*>(stg);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          uint4 u;
          u.x = pack_f16x2(__uint_as_float(xr[8 * g]), __uint_as_float(xr[8 * g + 1]));
          u.y = pack_f16x2(__uint_as_float(xr[8 * g + 2]), __uint_as_float(xr[8 * g + 3]));
          u.z = pack_f16x2(__uint_as_float(xr[8 * g + 4]), __uint_as_float(xr[8 * g + 5]));
          u.w = pack_f16x2(__uint_as_float(xr[8 * g + 6]), __uint_as_float(xr[8 * g + 7]));
          *reinterpret_cast<uint4*>(stw + lane * 32 + ((g ^ (lane & 7)) << 2)) = u;
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_pd, stw, c0, n * kTile + wq * 32);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_free);
    }
    if (lane == 0) bulk_wait_all();      // partials in global memory before the CTA retires
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// dQ_i = scale * sum_j partial_ij; one warp per row, the two half-warps take
// alternate blocks (in ascending order, D / 16 fp16 dims per lane) and add
// their sums at the end.  The partials sit at the pairs' item rows
// (slot_row).
template <int D>
__global__ void __launch_bounds__(256)
k_bwd_dq_merge(Prob P, int h, PairsView pv, const __half* __restrict__ part_dq,
               const float2* __restrict__ part_d, float scale, __nv_bfloat16* __restrict__ dq,
               float* __restrict__ rowD) {
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (i >= P.s) return;
  const uint32_t off = __ldg(pv.row_off + (size_t)h * (P.s + 1) + i);
  const uint32_t cnt = __ldg(pv.row_cnt + (size_t)h * P.s + i);
  const uint32_t* srow = pv.slot_row + (size_t)h * P.cap + off;
  // D_i as the sum of the pass's P dP shares (lane-parallel over the pairs,
  // then a warp sum), replacing the value computed from the output copy
  float dsum = 0.f;
  for (uint32_t k = lane; k < cnt; k += 32) {
    const float2 v = part_d[__ldg(srow + k)];
    dsum += v.x + v.y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  if (lane == 0 && cnt > 0) rowD[(size_t)h * P.s + i] = dsum;
  constexpr int V = D / 16;
  const int hw = lane >> 4, hl = lane & 15;
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
#pragma unroll 4
  for (uint32_t k = hw; k < cnt; k += 2) {
    const uint32_t row = __ldg(srow + k);
    uint32_t u[V / 2];
    if constexpr (V == 8) {
      const uint4 x = reinterpret_cast<const uint4*>(part_dq + (size_t)row * D)[hl];
      u[0] = x.x;
      u[1] = x.y;
      u[2] = x.z;
      u[3] = x.w;
    } else {
      const uint2 x = reinterpret_cast<const uint2*>(part_dq + (size_t)row * D)[hl];
      u[0] = x.x;
      u[1] = x.y;
    }
#pragma unroll
    for (int e = 0; e < V / 2; ++e) {
      const float2 a = unpack_f16x2(u[e]);
      acc[2 * e] += a.x;
      acc[2 * e + 1] += a.y;
    }
  }
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  if (hw == 0) {
    __nv_bfloat16* dst = dq + ((size_t)i * P.n_h + h) * D;
    if constexpr (V == 8) {
      reinterpret_cast<uint4*>(dst)[hl] =
          make_uint4(pack_bf16x2(acc[0] * scale, acc[1] * scale),
                     pack_bf16x2(acc[2] * scale, acc[3] * scale),
                     pack_bf16x2(acc[4] * scale, acc[5] * scale),
                     pack_bf16x2(acc[6] * scale, acc[7] * scale));
    } else {
      reinterpret_cast<uint2*>(dst)[hl] = make_uint2(pack_bf16x2(acc[0] * scale, acc[1] * scale),
                                                     pack_bf16x2(acc[2] * scale, acc[3] * scale));
    }
  }
}

// =====================================================================
// dK/dV pass.  Item = (key tile kt of block j, head h), one CTA each.
// TMEM: S^T [0,128) (then P^T), dP^T [128,256) (then dS^T), dV [256,256+D),
// dK [384,384+D).  Two softmax warpgroups split each query tile's columns
// 64 / 64.  The tile's work is cut where its dependencies allow:
//   S^T(g)  -> P^T(g) (exponentials)            -> dV(g) += P^T dO
//   dP^T(g) -> dS^T(g) = P^T (dP^T - D)          -> dK(g) += dS^T Q
// and the MMA issue order is dV(g), S^T(g+1), dK(g), dP^T(g+1): the next
// S^T runs while dS^T(g) is formed, dP^T(g+1) while P^T(g+1) is.  Each MMA
// overwrites only columns whose readers were issued before it.
// Roles: warp 0 loads the K/V tile once, then each query tile's Q and dO
// (TMA, item-ordered copies) and -LSE log2(e), D (bulk copies) into two
// buffers; warp 1 MMA; warps 4-7 / 8-11 softmax of query columns 0-63 /
// 64-127 (one key row per thread) and the epilogue (dV / dK).
// =====================================================================
struct KvBars {
  uint64_t kv_full;
  uint64_t qd_full[2], qd_empty[2];
  uint64_t st_full, dpt_full, p_full, ds_full;
  uint64_t acc_final;
  uint32_t tmem_base;
  int abort;
};
template <int D>
constexpr size_t kv_smem() {
  return 1024 + 2 * tile_bytes<D>() /*K,V*/ + 4 * tile_bytes<D>() /*Q,dO x2*/ +
         2 * 2 * kTile * sizeof(float) /*nlse2, D x2*/ + sizeof(KvBars) + 64;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_bwd_dkdv_blk(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
               Prob P, int h, PairsView pv, const float* __restrict__ dg,
               const float* __restrict__ l2g, float sl2, float scale,
               __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
               Watch wt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr uint32_t kTileB = tile_bytes<D>();
  uint8_t* sK = smem;
  uint8_t* sV = sK + kTileB;
  uint8_t* sQ = sV + kTileB;           // 2 buffers
  uint8_t* sO = sQ + 2 * kTileB;       // 2 buffers
  float* sL = reinterpret_cast<float*>(sO + 2 * kTileB);   // [2][128] -lse2
  float* sD = sL + 2 * kTile;                              // [2][128] D
  KvBars* bars = reinterpret_cast<KvBars*>(sD + 2 * kTile);
  volatile int* abort = &bars->abort;

  // longest query lists first (the hardware hands out CTAs in index order)
  const int nkt = (P.L + kTile - 1) / kTile;
  const int rk = blockIdx.x / nkt, kt = blockIdx.x - rk * nkt;
  const int j = (int)__ldg(pv.blk_order + (size_t)h * P.Nb + rk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t* col_off = pv.col_off + (size_t)h * (P.Nb + 1);
  const int item0 = (int)__ldg(pv.item_off + (size_t)h * (P.Nb + 1) + j);
  const int c0 = (int)__ldg(col_off + j), c1 = (int)__ldg(col_off + j + 1);
  const int nq = c1 - c0;
  const int ng = (nq + kTile - 1) / kTile;           // query tiles of block j
  const int key0 = j * P.L + kt * kTile;             // first key (partition order)
  const int nkeys = min(kTile, P.L - kt * kTile);    // keys of this tile inside block j

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int i = 0; i < 2; ++i) { mbar_init(&bars->qd_full[i], 1); mbar_init(&bars->qd_empty[i], 1); }
    mbar_init(&bars->st_full, 1);
    mbar_init(&bars->dpt_full, 1);
    mbar_init(&bars->p_full, kSoftmaxWarps);
    mbar_init(&bars->ds_full, kSoftmaxWarps);
    mbar_init(&bars->acc_final, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tS = tmem, tP = tmem + 128, tV = tmem + 256, tK = tmem + 384;

  if (warp == 0) {
    if (lane == 0 && ng > 0) {
      const int row = h * P.s + key0;
      mbar_expect_tx(&bars->kv_full, 2 * kTileB);
      tma_load_2d(sK, &tm_k, &bars->kv_full, 0, row);
      if (D == 128) tma_load_2d(sK + kHalf, &tm_k, &bars->kv_full, 64, row);
      tma_load_2d(sV, &tm_v, &bars->kv_full, 0, row);
      if (D == 128) tma_load_2d(sV + kHalf, &tm_v, &bars->kv_full, 64, row);
      bool ok = true;
      for (int g = 0; g < ng && ok; ++g) {
        const int b = g & 1;
        if (g >= 2) ok = mbar_wait(&bars->qd_empty[b], ((g >> 1) - 1) & 1, wt, abort);
        if (!ok) break;
        const int qrow = (item0 + g) * kTile;
        mbar_expect_tx(&bars->qd_full[b], 2 * kTileB + 2 * kTile * sizeof(float));
        tma_load_2d(sQ + b * kTileB, &tm_q, &bars->qd_full[b], 0, qrow);
        if (D == 128) tma_load_2d(sQ + b * kTileB + kHalf, &tm_q, &bars->qd_full[b], 64, qrow);
        tma_load_2d(sO + b * kTileB, &tm_o, &bars->qd_full[b], 0, qrow);
        if (D == 128) tma_load_2d(sO + b * kTileB + kHalf, &tm_o, &bars->qd_full[b], 64, qrow);
        bulk_load(sL + b * kTile, l2g + qrow, kTile * sizeof(float), &bars->qd_full[b]);
        bulk_load(sD + b * kTile, dg + qrow, kTile * sizeof(float), &bars->qd_full[b]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && ng > 0) {
      const uint32_t idSS = idesc_f16(128, 128, false, false);
      const uint32_t idAcc = idesc_f16(128, D, false, true);
      const uint32_t kb = smem_u32(sK), vb = smem_u32(sV);
      // S^T = K Q^T (or dP^T = V dO^T): keys x queries, K-major both sides
      auto issue_ss = [&](uint32_t tD, uint32_t ab, uint32_t bb) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tD, desc_sw128(ab + off, 16, 1024), desc_sw128(bb + off, 16, 1024), idSS,
                 kk > 0 ? 1u : 0u);
        }
      };
      // acc += A^T B with A^T packed in TMEM, B = Q or dO (queries = reduction, MN-major)
      auto issue_acc = [&](uint32_t tD, uint32_t tA, uint32_t bb, int g) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tD, tA + packed_col(kk), desc_sw128(bb + kk * 2048, kHalf, 1024), idAcc,
                 (g > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(&bars->kv_full, 0, wt, abort) &&
                mbar_wait(&bars->qd_full[0], 0, wt, abort);
      if (ok) {
        tc_fence_after();
        issue_ss(tS, kb, smem_u32(sQ));
        mma_commit(&bars->st_full);
        issue_ss(tP, vb, smem_u32(sO));
        mma_commit(&bars->dpt_full);
      }
      for (int g = 0; g < ng && ok; ++g) {
        const int b = g & 1;
        const bool more = g + 1 < ng;
        const uint32_t qb = smem_u32(sQ + b * kTileB), ob = smem_u32(sO + b * kTileB);
        if (!mbar_wait(&bars->p_full, g & 1, wt, abort)) { ok = false; break; }
        tc_fence_after();
        issue_acc(tV, tS, ob, g);                       // dV += P^T dO
        if (more) {
          if (!mbar_wait(&bars->qd_full[b ^ 1], ((g + 1) >> 1) & 1, wt, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_ss(tS, kb, smem_u32(sQ + (b ^ 1) * kTileB));   // S^T(g+1)
          mma_commit(&bars->st_full);
        }
        if (!mbar_wait(&bars->ds_full, g & 1, wt, abort)) { ok = false; break; }
        tc_fence_after();
        issue_acc(tK, tP, qb, g);                       // dK += dS^T Q
        mma_commit(&bars->qd_empty[b]);
        if (more) {
          issue_ss(tP, vb, smem_u32(sO + (b ^ 1) * kTileB));   // dP^T(g+1)
          mma_commit(&bars->dpt_full);
        }
      }
      if (ok) mma_commit(&bars->acc_final);
    }
  } else if (warp >= 4) {
    const int wq = warp & 3, wg = (warp - 4) >> 2;   // lane quarter, query-column group
    const int c = wq * 32 + lane;                     // key row of this thread
    const int cb = 64 * wg;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const bool kvalid = c < nkeys;
    const uint64_t sl2x2 = f32x2(sl2, sl2);
    bool ok = true;
    for (int g = 0; g < ng && ok; ++g) {
      const int b = g & 1;
      // qd_full also covers sL / sD of this tile
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->qd_full[b], (g >> 1) & 1, wt, abort));
      if (!ok) break;
      const float* NL = sL + b * kTile + cb;
      const float* Dq = sD + b * kTile + cb;
      // -LSE log2(e) of the first 32 query columns read ahead of the S^T wait
      // (the other 32 are read as they are used; all 64 would spill)
      float4 nlr[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) nlr[x] = *reinterpret_cast<const float4*>(NL + 4 * x);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->st_full, g & 1, wt, abort));
      if (!ok) break;
      tc_fence_after();
      // P^T for the group's 64 query columns (kept in fp32 for dS^T);
      // rows of keys past the tile's end are computed but never stored
      uint32_t pr[64];
      tmem_ld32(tS + lane_off + cb, pr);
      tmem_ld32(tS + lane_off + cb + 32, pr + 32);
      tmem_ld_wait();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pp[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int x = hh * 32 + e;
          const float4 nl = hh == 0 ? nlr[x >> 2] : *reinterpret_cast<const float4*>(NL + x);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int y = x + 2 * u;
            const float2 t = f32x2_split(
                fma_x2(f32x2(__uint_as_float(pr[y]), __uint_as_float(pr[y + 1])), sl2x2,
                       u ? f32x2(nl.z, nl.w) : f32x2(nl.x, nl.y)));
            const float p0 = fast_exp2(t.x), p1 = fast_exp2(t.y);
            pr[y] = __float_as_uint(p0);
            pr[y + 1] = __float_as_uint(p1);
            pp[(e >> 1) + u] = pack_f16x2(p0, p1);
          }
        }
        // P^T into the group's columns [cb + 16 hh, +16) (S^T already read)
        tmem_st16(tS + lane_off + cb + hh * 16, pp);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
      // likewise D of the first 32 query columns, ahead of the dP^T wait
      float4 ddr[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) ddr[x] = *reinterpret_cast<const float4*>(Dq + 4 * x);
      // dS^T = P^T (dP^T - D)
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dpt_full, g & 1, wt, abort));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t xp[32];
        tmem_ld32(tP + lane_off + cb + hh * 32, xp);
        tmem_ld_wait();
        uint32_t pd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const int x = hh * 32 + e;
          const float4 dd = hh == 0 ? ddr[x >> 2] : *reinterpret_cast<const float4*>(Dq + x);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int y = e + 2 * u;
            const uint64_t dp = sub_x2(f32x2(__uint_as_float(xp[y]), __uint_as_float(xp[y + 1])),
                                       u ? f32x2(dd.z, dd.w) : f32x2(dd.x, dd.y));
            const float2 ds = f32x2_split(mul_x2(
                f32x2(__uint_as_float(pr[x + 2 * u]), __uint_as_float(pr[x + 2 * u + 1])), dp));
            pd[(e >> 1) + u] = pack_f16x2(ds.x, ds.y);
          }
        }
        // dS^T into the group's columns [cb + 16 hh, +16) (dP^T already read)
        tmem_st16(tP + lane_off + cb + hh * 16, pd);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_full);
    }
    // epilogue: dK (x scale) and dV of the tile's keys, original key order
    const bool have = ng > 0 && ok &&
                      __all_sync(0xffffffffu, mbar_wait(&bars->acc_final, 0, wt, abort));
    if (ng == 0 || have) {
      if (have) tc_fence_after();
      const int pk = key0 + c;
      const int n = kvalid ? perm_token(P, pk) : 0;
      {                                               // group 0: dV, group 1: dK
        const int half = wg == 0 ? 1 : 0;
        const uint32_t base = half == 0 ? tK : tV;
        const float f = half == 0 ? scale : 1.0f;
        __nv_bfloat16* dst = (half == 0 ? dk : dv) + ((size_t)n * P.n_h + h) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t xr[32];
          if (have) {
            tmem_ld32(base + lane_off + cc * 32, xr);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) xr[e] = 0u;
          }
          if (kvalid) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(xr[e]) * f, __uint_as_float(xr[e + 1]) * f);
              u.y = pack_bf16x2(__uint_as_float(xr[e + 2]) * f, __uint_as_float(xr[e + 3]) * f);
              u.z = pack_bf16x2(__uint_as_float(xr[e + 4]) * f, __uint_as_float(xr[e + 5]) * f);
              u.w = pack_bf16x2(__uint_as_float(xr[e + 6]) * f, __uint_as_float(xr[e + 7]) * f);
              d4[e / 8] = u;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

namespace {
// bf16 -> fp16 of a contiguous array, 16 bytes per step (n a multiple of 8)
__global__ void k_to_f16(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n16;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = tc::bf16x8_to_f16x8(__ldg(src + i));
}
}  // namespace

size_t bwd_blk_ws_bytes(const Prob& P) {
  // rowD + lse2 ([n_h][s] fp32 each); for the tensor-core path also fp16
  // copies of K' and V' ([n_h][s][d] each)
  size_t b = 2 * align_up(sizeof(float) * (size_t)P.n_h * P.s, 256);
  if (uses_blk_path(P)) b += 2 * align_up(sizeof(__half) * (size_t)P.n_h * P.s * P.d, 256);
  return b;
}

namespace {

template <int D>
cudaError_t bwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                    const PairsView& pv, void* part, const ItemBufs& ib, const float* o32,
                    const float* lse, const void* dout, void* dq, void* dk, void* dv,
                    void* ws_bwd, float scale, int* status, int num_sms, cudaStream_t st) {
  CUtensorMap tk, tv, tq, to, tpd;
  const uint64_t rows = (uint64_t)P.n_h * P.s;
  __half* part_dq = static_cast<__half*>(part);
  // fp16 copies of K' and V' (the backward's MMAs take fp16 operands)
  const size_t f32_bytes = align_up(sizeof(float) * (size_t)P.n_h * P.s, 256);
  __half* kh = reinterpret_cast<__half*>(static_cast<char*>(ws_bwd) + 2 * f32_bytes);
  __half* vh = reinterpret_cast<__half*>(
      reinterpret_cast<char*>(kh) + align_up(sizeof(__half) * (size_t)P.n_h * P.s * D, 256));
  // the dQ pass's per-pair shares of D (two per item row), where the
  // forward kept its (m, l)
  float* part_d = reinterpret_cast<float*>(
      static_cast<char*>(part) + align_up(item_rows_capacity(P) * D * sizeof(__half), 256));
  const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (!make_tmap_2d(&tk, kh, f16, 2, rows, D, 64, 128) ||
      !make_tmap_2d(&tv, vh, f16, 2, rows, D, 64, 128) ||
      !make_tmap_2d(&tq, ib.qh, f16, 2, ib.rows, D, 64, 128) ||
      !make_tmap_2d(&to, ib.doh, f16, 2, ib.rows, D, 64, 128) ||
      !make_tmap_2d(&tpd, part_dq, f16, 2, item_rows_capacity(P), D, 64, 32))
    return cudaErrorInvalidValue;
  float* rowD = static_cast<float*>(ws_bwd);
  float* lse2 = reinterpret_cast<float*>(static_cast<char*>(ws_bwd) +
                                         align_up(sizeof(float) * (size_t)P.n_h * P.s, 256));
  {
    VMOBA_TRACE("k_to_f16", st);
    const size_t n16 = (size_t)P.n_h * P.s * D / 8;
    k_to_f16<<<num_sms * 8, 256, 0, st>>>(static_cast<const uint4*>(kp),
                                          reinterpret_cast<uint4*>(kh), n16);
    k_to_f16<<<num_sms * 8, 256, 0, st>>>(static_cast<const uint4*>(vp),
                                          reinterpret_cast<uint4*>(vh), n16);
  }
  const int warps = P.s * P.n_h;
  {
    VMOBA_TRACE("k_bwd_rows", st);
    k_bwd_rows<D><<<(warps + 7) / 8, 256, 0, st>>>(
        P, o32, static_cast<const __nv_bfloat16*>(dout), lse, rowD, lse2);
  }
  cudaError_t e = cudaFuncSetAttribute(k_bwd_dq_blk<D, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)dq_smem<D>());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_bwd_dq_blk<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)dq_smem<D>());
  if (e != cudaSuccess) return e;
  // blocks of at most two key chunks take the double-buffered dP schedule
  const bool dq_db = (P.L + kTile - 1) / kTile <= 2;
  e = cudaFuncSetAttribute(k_bwd_dkdv_blk<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kv_smem<D>());
  if (e != cudaSuccess) return e;
  const float sl2 = scale * kLog2e;
  const int nkt = (P.L + kTile - 1) / kTile;
  for (int h = 0; h < P.n_h; ++h) {
    // padding rows get -LSE log2(e) = -inf, so their P is exactly 0
    e = launch_gather_items(P, h, pv, static_cast<const __nv_bfloat16*>(q),
                            static_cast<const __nv_bfloat16*>(dout), ib.qh, ib.doh, lse2, rowD,
                            ib.l2g, ib.dg, -INFINITY, num_sms, st);
    if (e != cudaSuccess) return e;
    {
      VMOBA_TRACE("k_bwd_dq_blk", st);
      if (dq_db)
        k_bwd_dq_blk<D, true><<<num_sms, kThreads, dq_smem<D>(), st>>>(
            tk, tv, tq, to, tpd, P, h, pv, ib.dg, ib.l2g, sl2, part_d, make_watch(status));
      else
        k_bwd_dq_blk<D, false><<<num_sms, kThreads, dq_smem<D>(), st>>>(
            tk, tv, tq, to, tpd, P, h, pv, ib.dg, ib.l2g, sl2, part_d, make_watch(status));
    }
    {
      VMOBA_TRACE("k_bwd_dq_merge", st);
      k_bwd_dq_merge<D><<<(P.s + 7) / 8, 256, 0, st>>>(
          P, h, pv, part_dq, reinterpret_cast<const float2*>(part_d), scale,
          static_cast<__nv_bfloat16*>(dq), rowD);
    }
    // the exact D of this head into item order for the dK/dV pass
    e = launch_gather_items(P, h, pv, nullptr, nullptr, nullptr, nullptr, lse2, rowD, ib.l2g,
                            ib.dg, -INFINITY, num_sms, st);
    if (e != cudaSuccess) return e;
    {
      VMOBA_TRACE("k_bwd_dkdv_blk", st);
      k_bwd_dkdv_blk<D><<<P.Nb * nkt, kThreads, kv_smem<D>(), st>>>(
          tk, tv, tq, to, P, h, pv, ib.dg, ib.l2g, sl2, scale, static_cast<__nv_bfloat16*>(dk),
          static_cast<__nv_bfloat16*>(dv), make_watch(status));
    }
  }
  count_launches(3 + 4 * P.n_h);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                                const uint32_t* sel, const PairsView& pv, void* part,
                                const ItemBufs& ib, const float* o32, const float* lse,
                                const void* dout, void* dq, void* dk, void* dv, void* ws_bwd,
                                float scale, int* status, int num_sms, cudaStream_t st) {
  (void)sel;
  return P.d == 128 ? bwd_blk<128>(P, q, kp, vp, pv, part, ib, o32, lse, dout, dq, dk, dv, ws_bwd,
                                   scale, status, num_sms, st)
                    : bwd_blk<64>(P, q, kp, vp, pv, part, ib, o32, lse, dout, dq, dk, dv, ws_bwd,
                                  scale, status, num_sms, st);
}

}  // namespace vmoba
