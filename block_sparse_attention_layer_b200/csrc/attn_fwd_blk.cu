// Sparse attention forward, block-major, on the 5th-generation tensor cores
// (bf16, head_dim 128).
//
// VMoBA notes, overall framework: attention only over the selected
// (query, block) pairs.  A work item is (block j, one tile of 128 queries
// from block j's query list); every query of the tile selected block j, so
// the tile attends all keys of the block with no per-row masking and no
// wasted pairs.  The item computes, for each of its queries, the partial
// softmax state of block j (running max m, sum l, unnormalised O) over the
// block's keys in chunks of 128 and stores it in the pair's slot.  A merge
// kernel then combines the partials of each query with log-sum-exp weights
// into O, its fp32 copy and LSE.
//
// Persistent kernel, one head per launch: CTA b takes items b, b + G, ...
// (all items of a layer cost the same, so a static round-robin balances).
// Roles (256 threads):
//   warp 0      TMA producer of the block's K / V chunks (2-stage rings);
//   warp 1      TMEM owner (512 columns) and single-thread MMA issuer:
//               S = Q K^T into two S buffers; O += P V with P read from TMEM;
//   (warps 2-3 idle: the softmax warpgroup must start at a multiple of 4)
// Query tiles come by TMA from the item-ordered copy of Q (gather.cu) into
// two Q buffers, loaded by the producer ahead of the item.
//   warps 4-7   softmax: one query row per thread, lazy 2^8 rescale of O,
//               then the item's epilogue (partials out).
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384).
#include "tc_prims.cuh"
#include "pairs.cuh"

namespace vmoba {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr uint32_t kHalf = 128 * 64 * 2;
constexpr uint32_t kTileB = 2 * kHalf;
constexpr int kThreads = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kTmemCols = 512;

struct Bars {
  uint64_t full_k[2], empty_k[2], full_v[2], empty_v[2];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t o_final, o_free;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = 1024 + 2 * kTileB /*Q x2*/ + 2 * kTileB /*K*/ + 2 * kTileB /*V*/ +
                              sizeof(Bars) + 64;

struct Item {
  int j, count;           // block, queries in this tile (1..128)
  const uint32_t* rows;   // the tile's query indices
};

__device__ __forceinline__ Item decode_item(const Prob& P, int n, const uint32_t* item_off,
                                            const uint32_t* col_off, const uint32_t* col_rows) {
  // largest j with item_off[j] <= n (item_off is non-decreasing, item_off[0] = 0)
  int lo = 0, hi = P.Nb;   // invariant: item_off[lo] <= n < item_off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(item_off + mid) <= (uint32_t)n) lo = mid; else hi = mid;
  }
  Item it;
  it.j = lo;
  const int g = n - (int)__ldg(item_off + lo);
  const int c0 = (int)__ldg(col_off + lo), c1 = (int)__ldg(col_off + lo + 1);
  it.count = min(kTile, c1 - c0 - g * kTile);
  it.rows = col_rows + c0 + g * kTile;
  return it;
}

__global__ void __launch_bounds__(kThreads, 1)
k_fwd_blk(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
          const __grid_constant__ CUtensorMap tm_q, Prob P, int h,
          const uint32_t* __restrict__ sel,
          PairsView pv, float sl2, float* __restrict__ part_o, float2* __restrict__ part_ml,
          int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                       // 2 buffers
  uint8_t* sK = sQ + 2 * kTileB;
  uint8_t* sV = sK + 2 * kTileB;
  Bars* bars = reinterpret_cast<Bars*>(sV + 2 * kTileB);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t* item_off = pv.item_off + (size_t)h * (P.Nb + 1);
  const uint32_t* col_off = pv.col_off + (size_t)h * (P.Nb + 1);
  const uint32_t* col_rows = pv.col_rows + (size_t)h * P.s * P.Nb;
  const uint32_t* row_off = pv.row_off + (size_t)h * (P.s + 1);
  const int n_items = (int)__ldg(pv.head_totals + 2 * h + 1);
  const int nch = (P.L + kTile - 1) / kTile;          // key chunks per block
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->full_k[i], 1); mbar_init(&bars->empty_k[i], 1);
      mbar_init(&bars->full_v[i], 1); mbar_init(&bars->empty_v[i], 1);
      mbar_init(&bars->s_full[i], 1); mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->o_done[i], 1);
      mbar_init(&bars->q_full[i], 1); mbar_init(&bars->q_empty[i], 1);
    }
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->o_free, 4);
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
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      int J = 0, it_local = 0;
      bool ok = true;
      for (int n = blockIdx.x; n < n_items && ok; n += G, ++it_local) {
        const Item it = decode_item(P, n, item_off, col_off, col_rows);
        const int qb = it_local & 1;
        if (it_local >= 2)
          ok = mbar_wait(&bars->q_empty[qb], ((it_local >> 1) - 1) & 1, status, abort);
        if (!ok) break;
        mbar_expect_tx(&bars->q_full[qb], kTileB);
        tma_load_2d(sQ + qb * kTileB, &tm_q, &bars->q_full[qb], 0, n * kTile);
        tma_load_2d(sQ + qb * kTileB + kHalf, &tm_q, &bars->q_full[qb], 64, n * kTile);
        for (int c = 0; c < nch && ok; ++c, ++J) {
          const int row = h * P.s + it.j * P.L + c * kTile;
          const int st = J & 1;
          if (J >= 2) ok = mbar_wait(&bars->empty_k[st], ((J >> 1) - 1) & 1, status, abort);
          if (!ok) break;
          mbar_expect_tx(&bars->full_k[st], kTileB);
          tma_load_2d(sK + st * kTileB, &tm_k, &bars->full_k[st], 0, row);
          tma_load_2d(sK + st * kTileB + kHalf, &tm_k, &bars->full_k[st], 64, row);
          if (J >= 2) ok = mbar_wait(&bars->empty_v[st], ((J >> 1) - 1) & 1, status, abort);
          if (!ok) break;
          mbar_expect_tx(&bars->full_v[st], kTileB);
          tma_load_2d(sV + st * kTileB, &tm_v, &bars->full_v[st], 0, row);
          tma_load_2d(sV + st * kTileB + kHalf, &tm_v, &bars->full_v[st], 64, row);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 128, false, false);
      const uint32_t idPV = idesc_bf16(128, 128, false, true);
      int J = 0, it_local = 0;
      int prev_c = -1, prev_it = -1;   // chunk / item of the chunk whose PV is pending
      bool ok = true;
      auto issue_pv = [&](int Jp, int cp, int itp) -> bool {
        const int sb = Jp & 1;
        if (!mbar_wait(&bars->p_full[sb], (Jp >> 1) & 1, status, abort)) return false;
        if (!mbar_wait(&bars->full_v[sb], (Jp >> 1) & 1, status, abort)) return false;
        if (cp == 0 && itp > 0 && !mbar_wait(&bars->o_free, (itp - 1) & 1, status, abort))
          return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(sV + sb * kTileB);
        const uint32_t tP = tmem + sb * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tO, tP + kk * 8, desc_sw128(vb + kk * 2048, kHalf, 1024), idPV,
                 (cp > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty_v[sb]);
        mma_commit(&bars->o_done[sb]);
        if (cp == nch - 1) mma_commit(&bars->o_final);
        return true;
      };
      for (int n = blockIdx.x; n < n_items && ok; n += G, ++it_local) {
        const int qb = it_local & 1;
        if (!mbar_wait(&bars->q_full[qb], (it_local >> 1) & 1, status, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qbase = smem_u32(sQ + qb * kTileB);
        for (int c = 0; c < nch && ok; ++c, ++J) {
          const int st = J & 1;
          if (!mbar_wait(&bars->full_k[st], (J >> 1) & 1, status, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kb = smem_u32(sK + st * kTileB);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            mma_ss(tmem + st * 128, desc_sw128(qbase + off, 16, 1024),
                   desc_sw128(kb + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->empty_k[st]);
          mma_commit(&bars->s_full[st]);
          if (c == nch - 1) mma_commit(&bars->q_empty[qb]);
          if (J > 0) ok = issue_pv(J - 1, prev_c, prev_it);
          prev_c = c;
          prev_it = it_local;
        }
      }
      if (ok && J > 0) issue_pv(J - 1, prev_c, prev_it);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------- softmax + epilogue
    const int wq = warp - 4;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    int J = 0, it_local = 0;
    bool ok = true;
    for (int n = blockIdx.x; n < n_items && ok; n += G, ++it_local) {
      const Item it = decode_item(P, n, item_off, col_off, col_rows);
      float m_run = -INFINITY, l_run = 0.f;
      for (int c = 0; c < nch; ++c, ++J) {
        const int sb = J & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], (J >> 1) & 1, status, abort));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + sb * 128 + lane_off;
        const int lim = P.L - c * kTile;        // keys of this chunk inside block j
        const bool full = lim >= kTile;         // uniform over the CTA
        // the whole S row in registers: four loads, one wait
        uint32_t xr[128];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tS + c4 * 32, xr + c4 * 32);
        tmem_ld_wait();
        float mt = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; ++e)
          mt = fmaxf(mt, (full || e < lim) ? __uint_as_float(xr[e]) : -INFINITY);
        const float mt2 = mt * sl2;
        const bool grows = m_run == -INFINITY || mt2 > m_run + kRescaleLog2;
        const bool rescale = grows && m_run > -INFINITY;
        const float m_new = grows ? fmaxf(mt2, m_run) : m_run;
        if (__any_sync(0xffffffffu, rescale)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[(J - 1) & 1], ((J - 1) >> 1) & 1,
                                                 status, abort));
          if (!ok) break;
          tc_fence_after();
          const float f = rescale ? exp2f(m_run - m_new) : 1.0f;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t ob[32];
            tmem_ld32(tO + cc * 32 + lane_off, ob);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) ob[e] = __float_as_uint(__uint_as_float(ob[e]) * f);
            tmem_st32(tO + cc * 32 + lane_off, ob);
          }
          tmem_st_wait();
          l_run *= f;
        }
        m_run = m_new;
        float lsum = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int col = c4 * 32 + e;
            const float a = (full || col < lim)
                                ? exp2f(fmaf(__uint_as_float(xr[col]), sl2, -m_run)) : 0.f;
            const float b = (full || col + 1 < lim)
                                ? exp2f(fmaf(__uint_as_float(xr[col + 1]), sl2, -m_run)) : 0.f;
            lsum += a + b;
            pk[e >> 1] = pack_bf16x2(a, b);
          }
          tmem_st16(tS + c4 * 16, pk);
        }
        l_run += lsum;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[sb]);
      }
      if (!ok) break;
      // epilogue: partial state of (query, block j) into the pair's slot
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_final, it_local & 1, status, abort));
      if (!ok) break;
      tc_fence_after();
      const bool valid = r < it.count;
      size_t slot = 0;
      if (valid) {
        const uint32_t i = __ldg(it.rows + r);
        slot = pair_slot(row_off, sel + ((size_t)h * P.s + i) * P.Wb, P.Wb, (int)i, it.j);
        part_ml[slot] = make_float2(m_run, l_run);
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t ob[32];
        tmem_ld32(tO + cc * 32 + lane_off, ob);
        tmem_ld_wait();
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(part_o + slot * kD + cc * 32);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            dst[e / 4] = make_float4(__uint_as_float(ob[e]), __uint_as_float(ob[e + 1]),
                                     __uint_as_float(ob[e + 2]), __uint_as_float(ob[e + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_free);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Combine the partial (m, l, O) of every query's selected blocks:
// O_i = sum_j 2^(m_j - M) O_j / sum_j 2^(m_j - M) l_j, LSE_i = (M + log2 L) ln 2.
// One warp per query row, four dims per lane, blocks in ascending order.
__global__ void __launch_bounds__(256)
k_fwd_merge(Prob P, int h, PairsView pv, const float* __restrict__ part_o,
            const float2* __restrict__ part_ml, __nv_bfloat16* __restrict__ out,
            float* __restrict__ o32, float* __restrict__ lse) {
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (i >= P.s) return;
  const uint32_t off = __ldg(pv.row_off + (size_t)h * (P.s + 1) + i);
  const uint32_t cnt = __ldg(pv.row_cnt + (size_t)h * P.s + i);
  float M = -INFINITY;
  for (uint32_t k = 0; k < cnt; ++k) M = fmaxf(M, part_ml[off + k].x);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float Lsum = 0.f;
  for (uint32_t k = 0; k < cnt; ++k) {
    const float2 ml = part_ml[off + k];
    const float w = exp2f(ml.x - M);
    Lsum = fmaf(w, ml.y, Lsum);
    const float4 o = reinterpret_cast<const float4*>(part_o + (size_t)(off + k) * 128)[lane];
    acc.x = fmaf(w, o.x, acc.x); acc.y = fmaf(w, o.y, acc.y);
    acc.z = fmaf(w, o.z, acc.z); acc.w = fmaf(w, o.w, acc.w);
  }
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
  const size_t row = ((size_t)i * P.n_h + h) * 128;
  reinterpret_cast<float4*>(o32 + row)[lane] = acc;
  uint2 b;
  b.x = pack_bf16x2(acc.x, acc.y);
  b.y = pack_bf16x2(acc.z, acc.w);
  reinterpret_cast<uint2*>(out + row)[lane] = b;
  if (lane == 0)
    lse[(size_t)h * P.s + i] = Lsum > 0.f ? (M + log2f(Lsum)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace

size_t blk_partial_bytes(const Prob& P) {
  // one head's worst case: every (query, block) pair selected
  return align_up((size_t)P.s * P.Nb * 128 * sizeof(float), 256) +
         align_up((size_t)P.s * P.Nb * sizeof(float2), 256);
}

cudaError_t launch_attn_fwd_blk(const Prob& P, const void* q, const void* kp, const void* vp,
                                const uint32_t* sel, const PairsView& pv, void* part,
                                const ItemBufs& ib, float scale, void* out, float* o32,
                                float* lse, int* status, int num_sms, cudaStream_t st) {
  CUtensorMap tk, tv, tq;
  const uint64_t rows = (uint64_t)P.n_h * P.s;
  if (!make_tmap_bf16_2d(&tk, kp, rows, kD, 128) || !make_tmap_bf16_2d(&tv, vp, rows, kD, 128) ||
      !make_tmap_bf16_2d(&tq, ib.qg, ib.rows, kD, 128))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_fwd_blk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  float* part_o = static_cast<float*>(part);
  float2* part_ml = reinterpret_cast<float2*>(
      static_cast<char*>(part) + align_up((size_t)P.s * P.Nb * 128 * sizeof(float), 256));
  const float sl2 = scale * 1.4426950408889634f;
  for (int h = 0; h < P.n_h; ++h) {
    e = launch_gather_items(P, h, pv, static_cast<const __nv_bfloat16*>(q), nullptr, ib.qg,
                            nullptr, nullptr, nullptr, nullptr, nullptr, 0.f, num_sms, st);
    if (e != cudaSuccess) return e;
    {
      VMOBA_TRACE("k_fwd_blk", st);
      k_fwd_blk<<<num_sms, kThreads, kSmemBytes, st>>>(tk, tv, tq, P, h, sel, pv, sl2, part_o,
                                                        part_ml, status);
    }
    {
      VMOBA_TRACE("k_fwd_merge", st);
      k_fwd_merge<<<(P.s + 7) / 8, 256, 0, st>>>(P, h, pv, part_o, part_ml,
                                                 static_cast<__nv_bfloat16*>(out), o32, lse);
    }
  }
  count_launches(2 * P.n_h);
  return cudaGetLastError();
}

}  // namespace vmoba
