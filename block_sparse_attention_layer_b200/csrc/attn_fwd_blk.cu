// Sparse attention forward, block-major, on the 5th-generation tensor cores
// (bf16, head_dim D = 64 or 128).
//
// VMoBA notes, overall framework: attention only over the selected
// (query, block) pairs.  A work item is (block j, one tile of 128 queries
// from block j's query list); every query of the tile selected block j, so
// the tile attends all keys of the block with no per-row masking and no
// wasted pairs.  The item computes, for each of its queries, the partial
// softmax state of block j (running max m, sum l, and O / l) over the
// block's keys in chunks of 128 and stores it at the item's rows (row
// 128 n + r for row r of item n): (m, l) in fp32, O / l in fp16 -- a convex
// combination of V rows, so |O / l| <= max |V| and fp16 keeps it to 2^-12
// relative, below the bf16 output's rounding.  O / l leaves through the
// staging tiles as asynchronous TMA stores of 32 rows x 64 columns.  A merge
// kernel then combines the partials of each query (found through the pair
// lists' slot -> item row map) with log-sum-exp weights into O, its fp32
// copy and LSE.
//
// Persistent kernel, one head per launch.  A CTA takes PAIRS of work items
// (two consecutive 128-query tiles A, B of one block's list) so that every
// K / V chunk it loads serves 256 queries; CTA b takes pairs b, b + G, ...
// (static round-robin: all pairs of a layer cost about the same).
// Roles (384 threads):
//   warp 0      TMA producer: the block's K / V chunks (2-stage rings);
//   warp 1      TMEM owner (512 columns) and single-thread MMA issuer;
//   warps 2-3   query gather: the pair's two query tiles straight from Q by
//               cp.async (a softmax warpgroup must start at a multiple of 4,
//               which leaves these two warps to the copy);
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: one query
//               row per thread, lazy 2^8 rescale of O, then the tile's
//               epilogue (partials out through a per-warp staging tile and
//               an asynchronous TMA store).
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+D), O_B [384,384+D).
// The MMA issue order per chunk c is PV_A(c), S_A(c+1), PV_B(c), S_B(c+1):
// while one warpgroup computes exponentials the tensor core serves the other.
// P is written as bf16 pairs over the first half of its own S columns; the
// next S of the same tile is issued after the PV that reads P, and MMAs of
// one CTA execute in issue order.
// The last chunk of a block whose size is not a multiple of 128 runs with
// N = its key count rounded up to 16 (S) and that many 16-key steps (PV).
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
constexpr int kThreads = 384;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStageB = 32 * 32 * 4;     // per softmax warp: 32 rows x 32 fp32
constexpr uint32_t kGatherThreads = 64;       // warps 2-3 gather the query tiles

struct Bars {
  uint64_t full_k[2], empty_k[2], full_v[2], empty_v[2];
  uint64_t q_full[2], q_empty[2];                          // per query tile of the pair
  uint64_t s_full[2], p_full[2], o_final[2], o_free[2];   // per tile of the pair
  uint32_t tmem_base;
  int abort;
};

template <int D>
constexpr size_t fwd_smem() {
  return 1024 + 2 * tile_bytes<D>() /*Q pair*/ + 2 * tile_bytes<D>() /*K*/ +
         2 * tile_bytes<D>() /*V*/ + 8 * kStageB + sizeof(Bars) + 64;
}
static_assert(fwd_smem<128>() <= 232448, "shared memory per CTA");

// One chunk of softmax for one row: P = 2^(S sl2 - m) over the chunk's kc
// valid keys (NC columns loaded), written as bf16 pairs over S's first NC/2
// columns; running max / sum updated, O rescaled when the max grew by more
// than 2^8.
template <int NC, int D>
__device__ __forceinline__ void softmax_chunk(uint32_t tS, uint32_t tO, int kc, float sl2,
                                              float& m_run, float& l_run) {
  uint32_t xr[NC];
#pragma unroll
  for (int g = 0; g < NC / 32; ++g) tmem_ld32(tS + g * 32, xr + g * 32);
  tmem_ld_wait();
  const bool full = kc >= NC;
  float mt = -INFINITY;
#pragma unroll
  for (int e = 0; e < NC; ++e)
    mt = fmaxf(mt, (full || e < kc) ? __uint_as_float(xr[e]) : -INFINITY);
  const float mt2 = mt * sl2;
  const bool grows = m_run == -INFINITY || mt2 > m_run + kRescaleLog2;
  const bool rescale = grows && m_run > -INFINITY;
  const float m_new = grows ? fmaxf(mt2, m_run) : m_run;
  float lsum = 0.f;
#pragma unroll
  for (int c4 = 0; c4 < NC / 32; ++c4) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int col = c4 * 32 + e;
      const float a = (full || col < kc) ? fast_exp2(fmaf(__uint_as_float(xr[col]), sl2, -m_new))
                                         : 0.f;
      const float b = (full || col + 1 < kc)
                          ? fast_exp2(fmaf(__uint_as_float(xr[col + 1]), sl2, -m_new)) : 0.f;
      lsum += a + b;
      pk[e >> 1] = pack_bf16x2(a, b);
    }
    tmem_st16(tS + c4 * 16, pk);
  }
  // O rescale after the S row is consumed (fewer live registers); O holds
  // the previous chunks' PV, complete since this S was issued after it
  float f = 1.0f;
  if (__any_sync(0xffffffffu, rescale)) {
    f = rescale ? fast_exp2(m_run - m_new) : 1.0f;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t ob[32];
      tmem_ld32(tO + cc * 32, ob);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) ob[e] = __float_as_uint(__uint_as_float(ob[e]) * f);
      tmem_st32(tO + cc * 32, ob);
    }
  }
  m_run = m_new;
  l_run = fmaf(l_run, f, lsum);
  tmem_st_wait();
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_fwd_blk(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
          const __grid_constant__ CUtensorMap tm_po, const __nv_bfloat16* __restrict__ q,
          Prob P, int h, PairsView pv, float sl2, float2* __restrict__ part_ml,
          Watch wt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr uint32_t kTileB = tile_bytes<D>();
  uint8_t* sQ = smem;                       // tiles A, B
  uint8_t* sK = sQ + 2 * kTileB;            // 2 stages
  uint8_t* sV = sK + 2 * kTileB;            // 2 stages
  uint8_t* sStage = sV + 2 * kTileB;        // 8 x kStageB
  Bars* bars = reinterpret_cast<Bars*>(sStage + 8 * kStageB);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pairs = (int)__ldg(pv.head_totals + 4 * h + 2);
  const int nch = (P.L + kTile - 1) / kTile;          // key chunks per block
  const int kc_last = P.L - (nch - 1) * kTile;        // keys in the last chunk
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->full_k[i], 1); mbar_init(&bars->empty_k[i], 1);
      mbar_init(&bars->full_v[i], 1); mbar_init(&bars->empty_v[i], 1);
      mbar_init(&bars->s_full[i], 1); mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->o_final[i], 1); mbar_init(&bars->o_free[i], 4);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->q_full[t], kGatherThreads);
      mbar_init(&bars->q_empty[t], 1);
    }
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // (wt.skip_loads: diagnostics for the timeout path -- nothing is issued,
    // so the MMA warp's first wait runs out with no copy in flight)
    if (lane == 0 && !wt.skip_loads) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int J = 0, hint = 0;
      bool ok = true;
      for (int p = blockIdx.x; p < n_pairs && ok; p += G) {
        WorkItem b;
        int n0;
        const WorkItem a = decode_item_pair<false>(pv, P, h, p, &b, &n0, hint);
        for (int c = 0; c < nch && ok; ++c, ++J) {
          const int row = h * P.s + a.j * P.L + c * kTile;
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
      }
    }
  } else if (warp == 2 || warp == 3) {
    // -------------------------------------------------------- query gather
    // The pair's query rows straight from Q (one head's rows stay in L2):
    // warp w copies rows [64 w, 64 w + 64) of each tile, kRps rows per step
    // (D / 8 lanes x 16 bytes per row), into the 128-byte-swizzled layout
    // the MMA descriptors read (16-byte granule g of row r at g ^ (r & 7));
    // rows past the tile's queries are zero-filled.
    constexpr int kLpr = D / 8, kRps = 32 / kLpr;     // lanes per row, rows per step
    const int w = warp - 2, c = lane % kLpr, hr = lane / kLpr;
    const uint32_t* col_rows = pv.col_rows + (size_t)h * P.cap;
    const uint32_t qbase = smem_u32(sQ);
    int it_local = 0, hint = 0;
    bool ok = true;
    for (int p = blockIdx.x; p < n_pairs && ok; p += G, ++it_local) {
      WorkItem tb;
      int n0;
      const WorkItem ta = decode_item_pair<true>(pv, P, h, p, &tb, &n0, hint);
      // tile by tile: the next pair's tile A is copied while this pair's
      // tile B is still being read
#pragma unroll 1
      for (int t = 0; t < 2 && ok; ++t) {
        const WorkItem m = t == 0 ? ta : tb;
        if (it_local >= 1)
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&bars->q_empty[t], (it_local - 1) & 1, wt, abort));
        if (!ok) break;
        if (m.count == 0) {                        // no tile B in this pair
          mbar_arrive(&bars->q_full[t]);
          continue;
        }
        const int base = 64 * w;
        // query indices of the warp's 64 rows, one per lane and half
        const uint32_t idx0 =
            base + lane < m.count ? __ldg(col_rows + m.first + base + lane) : 0u;
        const uint32_t idx1 =
            base + 32 + lane < m.count ? __ldg(col_rows + m.first + base + 32 + lane) : 0u;
        const uint32_t tbase = qbase + t * kTileB + (c >> 3) * kHalf;
#pragma unroll 4
        for (int k = 0; k < 64 / kRps; ++k) {
          const int rr = kRps * k + hr;             // row within the warp's 64
          const uint32_t i0 = __shfl_sync(0xffffffffu, idx0, rr & 31);
          const uint32_t i1 = __shfl_sync(0xffffffffu, idx1, rr & 31);
          const int r = base + rr;
          const bool in = r < m.count;
          const uint32_t i = in ? (rr < 32 ? i0 : i1) : 0u;
          cp_async16(tbase + r * 128 + (((c & 7) ^ (r & 7)) << 4),
                     q + ((size_t)i * P.n_h + h) * D + c * 8, in ? 16u : 0u);
        }
        // copies landed, made visible to the tensor core's (async) proxy
        cp_async_wait_all();
        fence_proxy_async();
        mbar_arrive(&bars->q_full[t]);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 128, false, false);
      const uint32_t idS_last = idesc_bf16(128, (kc_last + 15) & ~15, false, false);
      const uint32_t idPV = idesc_bf16(128, D, false, true);
      const int ks_last = (kc_last + 15) / 16;
      int Jk = 0;                 // chunks through the K / V rings
      int Js[2] = {0, 0};         // S / P rounds per tile
      int It[2] = {0, 0};         // items per tile
      bool ok = true;
      auto issue_s = [&](int t, uint32_t kb, bool last) {
        const uint32_t qbase = smem_u32(sQ + t * kTileB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tmem + t * 128, desc_sw128(qbase + off, 16, 1024), desc_sw128(kb + off, 16, 1024),
                 last ? idS_last : idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[t]);
      };
      auto issue_pv = [&](int t, uint32_t vb, int c) {
        const int ks = c == nch - 1 ? ks_last : 8;
        for (int kk = 0; kk < ks; ++kk)
          mma_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8,
                 desc_sw128(vb + kk * 2048, kHalf, 1024), idPV, (c > 0 || kk > 0) ? 1u : 0u);
        if (c == nch - 1) mma_commit(&bars->o_final[t]);
      };
      int hint = 0;
      for (int p = blockIdx.x, it_local = 0; p < n_pairs && ok; p += G, ++it_local) {
        WorkItem b;
        int n0;
        decode_item_pair<false>(pv, P, h, p, &b, &n0, hint);
        const int nt = b.count > 0 ? 2 : 1;
        {
          const int st = Jk & 1;
          if (!mbar_wait(&bars->full_k[st], (Jk >> 1) & 1, wt, abort)) { ok = false; break; }
          const uint32_t kb = smem_u32(sK + st * kTileB);
          for (int t = 0; t < 2 && ok; ++t) {
            // every pair passes both tiles' barriers; an absent tile B is
            // released at once
            if (!mbar_wait(&bars->q_full[t], it_local & 1, wt, abort)) { ok = false; break; }
            tc_fence_after();
            if (t < nt) issue_s(t, kb, nch == 1);
            if (t >= nt || nch == 1) mma_commit(&bars->q_empty[t]);
          }
          if (!ok) break;
          mma_commit(&bars->empty_k[st]);
        }
        for (int c = 0; c < nch && ok; ++c) {
          const int Jc = Jk + c, stc = Jc & 1, st1 = (Jc + 1) & 1;
          const bool more = c + 1 < nch;
          if (!mbar_wait(&bars->full_v[stc], (Jc >> 1) & 1, wt, abort)) { ok = false; break; }
          uint32_t kb1 = 0;
          for (int t = 0; t < nt && ok; ++t) {
            if (c == 0 && It[t] > 0 &&
                !mbar_wait(&bars->o_free[t], (It[t] - 1) & 1, wt, abort)) { ok = false; break; }
            if (!mbar_wait(&bars->p_full[t], Js[t] & 1, wt, abort)) { ok = false; break; }
            ++Js[t];
            tc_fence_after();
            issue_pv(t, smem_u32(sV + stc * kTileB), c);
            if (more) {
              if (t == 0) {
                if (!mbar_wait(&bars->full_k[st1], ((Jc + 1) >> 1) & 1, wt, abort)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                kb1 = smem_u32(sK + st1 * kTileB);
              }
              issue_s(t, kb1, c + 1 == nch - 1);
              if (c + 1 == nch - 1) mma_commit(&bars->q_empty[t]);   // tile t's last S
            }
          }
          if (!ok) break;
          mma_commit(&bars->empty_v[stc]);
          if (more) mma_commit(&bars->empty_k[st1]);
        }
        Jk += nch;
        for (int t = 0; t < nt; ++t) ++It[t];
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------- softmax + epilogue
    const int t = (warp - 4) >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + t * 128 + lane_off, tO = tmem + 256 + t * 128 + lane_off;
    float* stg = reinterpret_cast<float*>(sStage + (warp - 4) * kStageB);
    int Js = 0, It = 0;
    bool ok = true;
    // this tile of pair pp: its work item and query count; decoded one pair
    // ahead, before the epilogue, so the decode is off the critical path
    int hint = 0;
    auto fetch = [&](int pp, int& n, int& cnt) {
      WorkItem bb;
      int nn;
      const WorkItem aa = decode_item_pair<true>(pv, P, h, pp, &bb, &nn, hint);
      n = nn + t;
      cnt = t == 0 ? aa.count : bb.count;
    };
    int nx_n = 0, nx_cnt = 0;
    if (blockIdx.x < n_pairs) fetch(blockIdx.x, nx_n, nx_cnt);
    for (int p = blockIdx.x; p < n_pairs && ok; p += G) {
      const int n = nx_n, cnt = nx_cnt;
      if (cnt == 0) {                              // no tile B in this pair
        if (p + G < n_pairs) fetch(p + G, nx_n, nx_cnt);
        continue;
      }
      const bool valid = r < cnt;
      float m_run = -INFINITY, l_run = 0.f;
      for (int c = 0; c < nch; ++c, ++Js) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], Js & 1, wt, abort));
        if (!ok) break;
        tc_fence_after();
        const int kc = c == nch - 1 ? kc_last : kTile;
        if (kc > 64) softmax_chunk<128, D>(tS, tO, kc, sl2, m_run, l_run);
        else softmax_chunk<64, D>(tS, tO, kc, sl2, m_run, l_run);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[t]);
      }
      if (!ok) break;
      if (p + G < n_pairs) fetch(p + G, nx_n, nx_cnt);
      // epilogue: partial state of (query, block j) into the item's rows
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_final[t], It & 1, wt, abort));
      ++It;
      if (!ok) break;
      tc_fence_after();
      if (valid) part_ml[(size_t)n * kTile + r] = make_float2(m_run, l_run);
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      uint32_t* stw = reinterpret_cast<uint32_t*>(stg);
#pragma unroll 1
      for (int cc = 0; cc < D / 64; ++cc) {          // 64 columns: 128 fp16 bytes per row
        uint32_t ob[64];
        tmem_ld32(tO + cc * 64, ob);
        tmem_ld32(tO + cc * 64 + 32, ob + 32);
        tmem_ld_wait();
        // the staging tile is free once the previous store has read it
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
        // row `lane` into the staging tile in the 128-byte swizzle of the
        // store's tensor map: 16-byte granule g at g ^ (row & 7)
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          uint4 u;
          u.x = pack_f16x2(__uint_as_float(ob[8 * g]) * inv_l, __uint_as_float(ob[8 * g + 1]) * inv_l);
          u.y = pack_f16x2(__uint_as_float(ob[8 * g + 2]) * inv_l,
                           __uint_as_float(ob[8 * g + 3]) * inv_l);
          u.z = pack_f16x2(__uint_as_float(ob[8 * g + 4]) * inv_l,
                           __uint_as_float(ob[8 * g + 5]) * inv_l);
          u.w = pack_f16x2(__uint_as_float(ob[8 * g + 6]) * inv_l,
                           __uint_as_float(ob[8 * g + 7]) * inv_l);
          *reinterpret_cast<uint4*>(stw + lane * 32 + ((g ^ (lane & 7)) << 2)) = u;
        }
        fence_proxy_async();
        __syncwarp();
        // the warp's 32 item rows, 64 columns, in one asynchronous store
        if (lane == 0) {
          tma_store_2d(&tm_po, stw, cc * 64, n * kTile + wq * 32);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_free[t]);
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

// Combine the partial (m, l, O / l) of every query's selected blocks:
// O_i = sum_j 2^(m_j - M) l_j (O / l)_j / sum_j 2^(m_j - M) l_j,
// LSE_i = (M + log2 sum_j 2^(m_j - M) l_j) ln 2.
// One warp per query row: the two half-warps take alternate blocks (in
// ascending order, D / 16 dims per lane) and add their sums at the end; the
// partials sit at the pairs' item rows (slot_row).
// Memory-bound: eight 256-thread CTAs per SM (at most 32 registers a thread)
// keep enough row loads in flight (5 per SM at 48 registers were 22 % slower).
template <int D>
__global__ void __launch_bounds__(256, 8)
k_fwd_merge(Prob P, int h, PairsView pv, const __half* __restrict__ part_o,
            const float2* __restrict__ part_ml, __nv_bfloat16* __restrict__ out,
            float* __restrict__ o32, float* __restrict__ lse) {
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (i >= P.s) return;
  const uint32_t off = __ldg(pv.row_off + (size_t)h * (P.s + 1) + i);
  const uint32_t cnt = __ldg(pv.row_cnt + (size_t)h * P.s + i);
  const uint32_t* srow = pv.slot_row + (size_t)h * P.cap + off;
  // lane k takes pairs k, k + 32, ...: item rows and (m, l) are loaded
  // lane-parallel and broadcast to the warp by shuffles
  uint32_t row0 = 0u;
  float2 ml0 = make_float2(-INFINITY, 0.f);
  if ((uint32_t)lane < cnt) {
    row0 = __ldg(srow + lane);
    ml0 = part_ml[row0];
  }
  float M = ml0.x;
  for (uint32_t b = 32 + lane; b < cnt; b += 32) M = fmaxf(M, part_ml[__ldg(srow + b)].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  // each half-warp reads one pair's row (V fp16 values per lane, one vector
  // load), so a warp instruction covers two pairs; the halves meet at the end
  constexpr int V = D / 16;
  const int hw = lane >> 4, hl = lane & 15;
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  float Lsum = 0.f;
  for (uint32_t b = 0; b < cnt; b += 32) {
    uint32_t my_row = row0;
    float2 ml = ml0;
    if (b > 0) {
      my_row = 0u;
      ml = make_float2(-INFINITY, 0.f);
      if (b + lane < cnt) {
        my_row = __ldg(srow + b + lane);
        ml = part_ml[my_row];
      }
    }
    const float my_w = b + lane < cnt ? exp2f(ml.x - M) * ml.y : 0.f;
    const int kn = (int)min(32u, cnt - b);
#pragma unroll 4
    for (int k = 0; k < kn; k += 2) {
      const int kk = k + hw;                 // <= kn <= 32
      const uint32_t row = __shfl_sync(0xffffffffu, my_row, kk & 31);
      const float w = __shfl_sync(0xffffffffu, my_w, kk & 31);
      if (kk < kn) {
        Lsum += w;
        uint32_t u[V / 2];
        if constexpr (V == 8) {
          const uint4 x = reinterpret_cast<const uint4*>(part_o + (size_t)row * D)[hl];
          u[0] = x.x;
          u[1] = x.y;
          u[2] = x.z;
          u[3] = x.w;
        } else {
          const uint2 x = reinterpret_cast<const uint2*>(part_o + (size_t)row * D)[hl];
          u[0] = x.x;
          u[1] = x.y;
        }
#pragma unroll
        for (int e = 0; e < V / 2; ++e) {
          const float2 a = unpack_f16x2(u[e]);
          acc[2 * e] = fmaf(w, a.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(w, a.y, acc[2 * e + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  Lsum += __shfl_xor_sync(0xffffffffu, Lsum, 16);
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  const size_t row = ((size_t)i * P.n_h + h) * D;
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] *= inv;
  if (hw == 0) {
    if constexpr (V == 8) {
      reinterpret_cast<float4*>(o32 + row)[2 * hl] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      reinterpret_cast<float4*>(o32 + row)[2 * hl + 1] =
          make_float4(acc[4], acc[5], acc[6], acc[7]);
      reinterpret_cast<uint4*>(out + row)[hl] =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                     pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    } else {
      reinterpret_cast<float4*>(o32 + row)[hl] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      reinterpret_cast<uint2*>(out + row)[hl] =
          make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
    }
  }
  if (lane == 0)
    lse[(size_t)h * P.s + i] = Lsum > 0.f ? (M + log2f(Lsum)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace

size_t blk_partial_bytes(const Prob& P) {
  // one head's partials, one row per work-item row (item_rows_capacity rows):
  // d fp16 (forward O / l, dQ pass), then the forward's (m, l) or the dQ
  // pass's two shares of D
  const size_t rows = item_rows_capacity(P);
  return align_up(rows * P.d * sizeof(__half), 256) + align_up(rows * sizeof(float2), 256);
}

namespace {

template <int D>
cudaError_t fwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                    const PairsView& pv, void* part, float scale, void* out, float* o32,
                    float* lse, int* status, int num_sms, cudaStream_t st) {
  CUtensorMap tk, tv, tpo;
  const uint64_t rows = (uint64_t)P.n_h * P.s;
  const size_t prows = item_rows_capacity(P);
  __half* part_o = static_cast<__half*>(part);    // fp16 O / l, then (m, l) at a fixed offset
  float2* part_ml = reinterpret_cast<float2*>(
      static_cast<char*>(part) + align_up(prows * D * sizeof(__half), 256));
  if (!make_tmap_bf16_2d(&tk, kp, rows, D, 128) || !make_tmap_bf16_2d(&tv, vp, rows, D, 128) ||
      !make_tmap_2d(&tpo, part_o, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, prows, D, 64, 32))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_fwd_blk<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)fwd_smem<D>());
  if (e != cudaSuccess) return e;
  const float sl2 = scale * 1.4426950408889634f;
  for (int h = 0; h < P.n_h; ++h) {
    {
      VMOBA_TRACE("k_fwd_blk", st);
      k_fwd_blk<D><<<num_sms, kThreads, fwd_smem<D>(), st>>>(
          tk, tv, tpo, static_cast<const __nv_bfloat16*>(q), P, h, pv, sl2, part_ml,
          make_watch(status));
    }
    {
      VMOBA_TRACE("k_fwd_merge", st);
      k_fwd_merge<D><<<(P.s + 7) / 8, 256, 0, st>>>(P, h, pv, part_o, part_ml,
                                                    static_cast<__nv_bfloat16*>(out), o32, lse);
    }
  }
  count_launches(2 * P.n_h);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                                const uint32_t* sel, const PairsView& pv, void* part,
                                const ItemBufs& ib, float scale, void* out, float* o32,
                                float* lse, int* status, int num_sms, cudaStream_t st) {
  (void)sel;
  (void)ib;
  return P.d == 128 ? fwd_blk<128>(P, q, kp, vp, pv, part, scale, out, o32, lse, status, num_sms, st)
                    : fwd_blk<64>(P, q, kp, vp, pv, part, scale, out, o32, lse, status, num_sms, st);
}

}  // namespace vmoba
