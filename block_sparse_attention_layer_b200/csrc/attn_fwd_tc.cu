// Sparse attention forward on the 5th-generation tensor cores (bf16, d = 128).
//
// Computes, over the selected (query, block) pairs only (VMoBA notes,
// overall framework), O_i = softmax_i(scale q_i K_sel^T) V_sel and
// LSE_i, with online softmax.  One CTA per (128-query tile, head); queries
// in partition order.  The key tiles the tile's rows touch come from the
// plan (qt_kt bitmap); inside a tile each row masks the keys of blocks it
// did not select.
//
// Roles (256 threads):
//   warp 0        TMA producer: K and V tiles (128 keys x 128 d, two 64-column
//                 128B-swizzled boxes each) into a 2-stage ring per operand;
//   warp 1        TMEM owner (512 columns) and single-thread MMA issuer:
//                 S_j = Q K_j^T into one of two S buffers, then
//                 O += P_{j-1} V_{j-1} with P read from TMEM;
//   warps 4..7    softmax: thread r owns query row r (TMEM lane r), reads its
//                 S row with tcgen05.ld, masks, keeps running max / sum,
//                 writes bf16 P back over S, rescales O in TMEM only when the
//                 running max grows by more than 2^8; epilogue writes O, its
//                 fp32 copy and LSE in original token order.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384).
#include "tc_prims.cuh"

namespace vmoba {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kKStages = 2, kVStages = 2;
constexpr uint32_t kHalf = 128 * 64 * 2;          // one 128-row x 64-col bf16 box
constexpr uint32_t kTileB = 2 * kHalf;            // 128 x 128 bf16
constexpr int kThreads = 256;
constexpr float kRescaleLog2 = 8.0f;              // lazy rescale threshold (factor 256)
constexpr uint32_t kTmemCols = 512;

struct FwdBars {
  uint64_t full_k[kKStages], empty_k[kKStages], full_v[kVStages], empty_v[kVStages];
  uint64_t s_full[2], p_full[2], o_done[2], o_final;
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ constexpr size_t fwd_fixed_smem() {
  return 1024 /*align slack*/ + kTileB /*Q*/ + kKStages * kTileB + kVStages * kTileB;
}

__device__ __forceinline__ bool row_bit(const uint32_t* words, int b) {
  return (words[b >> 5] >> (b & 31)) & 1u;
}

__global__ void __launch_bounds__(kThreads, 1)
k_fwd_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
         Prob P, const __nv_bfloat16* __restrict__ q, const uint32_t* __restrict__ sel,
         const uint32_t* __restrict__ qt_kt, float sl2, __nv_bfloat16* __restrict__ out,
         float* __restrict__ o32, float* __restrict__ lse, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kTileB;
  uint8_t* sV = sK + kKStages * kTileB;
  uint32_t* srow = reinterpret_cast<uint32_t*>(sV + kVStages * kTileB);
  FwdBars* bars = reinterpret_cast<FwdBars*>(
      (reinterpret_cast<uintptr_t>(srow + kTile * P.Wb) + 15) & ~static_cast<uintptr_t>(15));
  volatile int* abort = &bars->abort;

  const int t = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t* tiles = qt_kt + ((size_t)h * P.n_qt + t) * P.Wqt;
  int n_kt = 0;
  for (int w = 0; w < P.Wqt; ++w) n_kt += __popc(__ldg(tiles + w));

  // Q tile (partition order; zero rows past s) -> 128B-swizzled K-major smem
  for (int idx = threadIdx.x; idx < kTile * 16; idx += kThreads) {
    const int r = idx >> 4, c = idx & 15;
    const int p = t * kTile + r;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (p < P.s) {
      const int i = perm_token(P, p);
      val = __ldg(reinterpret_cast<const uint4*>(q + ((size_t)i * P.n_h + h) * kD) + c);
    }
    *reinterpret_cast<uint4*>(sQ + (c >> 3) * kHalf + sw128_off(r, c & 7)) = val;
  }
  for (int idx = threadIdx.x; idx < kTile * P.Wb; idx += kThreads) {
    const int rr = idx / P.Wb, w = idx - rr * P.Wb;
    const int pp = t * kTile + rr;
    srow[idx] = (pp < P.s) ? __ldg(sel + ((size_t)h * P.s + perm_token(P, pp)) * P.Wb + w) : 0u;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kKStages; ++i) { mbar_init(&bars->full_k[i], 1); mbar_init(&bars->empty_k[i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&bars->full_v[i], 1); mbar_init(&bars->empty_v[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);      // one arrive per softmax warp
      mbar_init(&bars->o_done[i], 1);
    }
    mbar_init(&bars->o_final, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_kt > 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int j = 0;
      bool ok = true;
      for (int w = 0; w < P.Wqt && ok; ++w) {
        uint32_t bits = __ldg(tiles + w);
        while (bits && ok) {
          const int kt = w * 32 + __ffs(bits) - 1;
          bits &= bits - 1;
          const int row = h * P.s + kt * kTile;
          const int ks = j % kKStages, vs = j % kVStages;
          if (j >= kKStages)
            ok = mbar_wait(&bars->empty_k[ks], ((j / kKStages) - 1) & 1, status, abort);
          if (!ok) break;
          mbar_expect_tx(&bars->full_k[ks], kTileB);
          tma_load_2d(sK + ks * kTileB, &tm_k, &bars->full_k[ks], 0, row);
          tma_load_2d(sK + ks * kTileB + kHalf, &tm_k, &bars->full_k[ks], 64, row);
          if (j >= kVStages)
            ok = mbar_wait(&bars->empty_v[vs], ((j / kVStages) - 1) & 1, status, abort);
          if (!ok) break;
          mbar_expect_tx(&bars->full_v[vs], kTileB);
          tma_load_2d(sV + vs * kTileB, &tm_v, &bars->full_v[vs], 0, row);
          tma_load_2d(sV + vs * kTileB + kHalf, &tm_v, &bars->full_v[vs], 64, row);
          ++j;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n_kt > 0) {
      const uint32_t idS = idesc_bf16(128, 128, false, false);
      const uint32_t idPV = idesc_bf16(128, 128, false, true);
      const uint32_t qb = smem_u32(sQ);
      auto issue_pv = [&](int i) -> bool {
        const int sb = i & 1, vs = i % kVStages;
        if (!mbar_wait(&bars->p_full[sb], (i >> 1) & 1, status, abort)) return false;
        if (!mbar_wait(&bars->full_v[vs], (i / kVStages) & 1, status, abort)) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(sV + vs * kTileB);
        const uint32_t tP = tmem + sb * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: P columns [8kk, 8kk+8)
          mma_ts(tO, tP + kk * 8, desc_sw128(vb + kk * 2048, kHalf, 1024), idPV,
                 (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty_v[vs]);
        mma_commit(&bars->o_done[sb]);
        return true;
      };
      bool ok = true;
      for (int j = 0; j < n_kt && ok; ++j) {
        const int ks = j % kKStages, sb = j & 1;
        if (!mbar_wait(&bars->full_k[ks], (j / kKStages) & 1, status, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = smem_u32(sK + ks * kTileB);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 16 of d per step, 4 steps per 64-column box
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_ss(tmem + sb * 128, desc_sw128(qb + off, 16, 1024), desc_sw128(kb + off, 16, 1024),
                 idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->empty_k[ks]);
        mma_commit(&bars->s_full[sb]);
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok) ok = issue_pv(n_kt - 1);
      if (ok) mma_commit(&bars->o_final);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------- softmax rows
    const int wq = warp - 4;
    const int r = wq * 32 + lane;
    const int p = t * kTile + r;
    const bool valid = p < P.s;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t* my_sel = srow + r * P.Wb;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int j = 0;
    for (int w = 0; w < P.Wqt && ok; ++w) {
      uint32_t bits = __ldg(tiles + w);
      while (bits) {
        const int kt = w * 32 + __ffs(bits) - 1;
        bits &= bits - 1;
        const int sb = j & 1;
        ok = mbar_wait(&bars->s_full[sb], (j >> 1) & 1, status, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + sb * 128 + lane_off;
        // keys of blocks this row did not select (and keys past s) are masked
        const int p0 = kt * kTile;
        const int plast = min(p0 + kTile - 1, P.s - 1);
        const int b0 = p0 / P.L, b1 = plast / P.L;
        bool all = valid && (p0 + kTile <= P.s), any = false;
        if (valid) {
          for (int b = b0; b <= b1; ++b) {
            const bool on = row_bit(my_sel, b);
            all = all && on;
            any = any || on;
          }
        }
        const int lim = P.s - p0;   // columns >= lim are past s
        // Every tcgen05.ld/st below is executed by all 32 lanes (they are
        // warp-collective); per-row decisions only predicate the arithmetic.
        // pass 1: row max over allowed columns, 32 TMEM columns at a time
        float mt = -INFINITY;
        {
          int b = b0, nb = (b0 + 1) * P.L - p0;
          bool cur = any && row_bit(my_sel, b0);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t xr[32];
            tmem_ld32(tS + c4 * 32, xr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int c = c4 * 32 + e;
              bool ok_c = any;
              if (any && !all) {
                if (c == nb) { ++b; cur = (b <= b1) && row_bit(my_sel, b); nb += P.L; }
                ok_c = cur && c < lim;
              }
              if (ok_c) mt = fmaxf(mt, __uint_as_float(xr[e]));
            }
          }
        }
        const float mt2 = mt * sl2;
        const bool grows = mt2 > -INFINITY && (m_run == -INFINITY || mt2 > m_run + kRescaleLog2);
        const bool rescale = grows && m_run > -INFINITY;
        const float m_new = grows ? fmaxf(mt2, m_run) : m_run;
        if (__any_sync(0xffffffffu, rescale)) {
          // some row of this warp moves its max: bring PV_{j-1} home, rescale O rows
          ok = mbar_wait(&bars->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, status, abort);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const float f = rescale ? exp2f(m_run - m_new) : 1.0f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t ob[32];
            tmem_ld32(tO + c * 32 + lane_off, ob);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) ob[e] = __float_as_uint(__uint_as_float(ob[e]) * f);
            tmem_st32(tO + c * 32 + lane_off, ob);
          }
          tmem_st_wait();
          l_run *= f;
        }
        m_run = m_new;
        // pass 2: P = exp2(S*scale*log2e - m) as bf16 pairs; P chunk c4 lands in
        // columns [16 c4, 16 c4 + 16), already read, so it never clobbers unread S
        float lsum = 0.f;
        {
          const bool live = any && m_run > -INFINITY;
          int b = b0, nb = (b0 + 1) * P.L - p0;
          bool cur = live && row_bit(my_sel, b0);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t xr[32];
            tmem_ld32(tS + c4 * 32, xr);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float pe[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int c = c4 * 32 + e + u;
                bool ok_c = live;
                if (live && !all) {
                  if (c == nb) { ++b; cur = (b <= b1) && row_bit(my_sel, b); nb += P.L; }
                  ok_c = cur && c < lim;
                }
                pe[u] = ok_c ? exp2f(fmaf(__uint_as_float(xr[e + u]), sl2, -m_run)) : 0.f;
              }
              lsum += pe[0] + pe[1];
              pk[e >> 1] = pack_bf16x2(pe[0], pe[1]);
            }
            tmem_st16(tS + c4 * 16, pk);
          }
        }
        l_run += lsum;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[sb]);
        ++j;
      }
    }
    // ------------------------------------------------------------ epilogue
    const int i = valid ? perm_token(P, p) : 0;
    if (n_kt > 0 && ok) {
      const bool fin = __all_sync(0xffffffffu, mbar_wait(&bars->o_final, 0, status, abort));
      if (fin) {
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ob[32];
          tmem_ld32(tO + c * 32 + lane_off, ob);
          tmem_ld_wait();
          if (valid) {
            float* fr = o32 + ((size_t)i * P.n_h + h) * kD + c * 32;
            uint4* br = reinterpret_cast<uint4*>(out + ((size_t)i * P.n_h + h) * kD + c * 32);
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 v4 = make_float4(__uint_as_float(ob[e]) * inv, __uint_as_float(ob[e + 1]) * inv,
                                      __uint_as_float(ob[e + 2]) * inv,
                                      __uint_as_float(ob[e + 3]) * inv);
              *reinterpret_cast<float4*>(fr + e) = v4;
            }
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(ob[e]) * inv, __uint_as_float(ob[e + 1]) * inv);
              u.y = pack_bf16x2(__uint_as_float(ob[e + 2]) * inv, __uint_as_float(ob[e + 3]) * inv);
              u.z = pack_bf16x2(__uint_as_float(ob[e + 4]) * inv, __uint_as_float(ob[e + 5]) * inv);
              u.w = pack_bf16x2(__uint_as_float(ob[e + 6]) * inv, __uint_as_float(ob[e + 7]) * inv);
              br[e / 8] = u;
            }
          }
        }
        if (valid)
          lse[(size_t)h * P.s + i] = l_run > 0.f ? (m_run + log2f(l_run)) * 0.6931471805599453f
                                                 : -INFINITY;
      }
    } else if (n_kt == 0 && valid) {
      // no key tile for the whole query tile: every row is empty
      float* fr = o32 + ((size_t)i * P.n_h + h) * kD;
      uint4* br = reinterpret_cast<uint4*>(out + ((size_t)i * P.n_h + h) * kD);
      for (int e = 0; e < kD; e += 4) *reinterpret_cast<float4*>(fr + e) = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int e = 0; e < kD / 8; ++e) br[e] = make_uint4(0u, 0u, 0u, 0u);
      lse[(size_t)h * P.s + i] = -INFINITY;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool fwd_tc_supported(const Prob& P) { return P.dtype == VMOBA_BF16 && P.d == 128; }

size_t fwd_tc_smem(const Prob& P) {
  return fwd_fixed_smem() + sizeof(uint32_t) * kTile * P.Wb + sizeof(FwdBars) + 16;
}

cudaError_t launch_attn_fwd_tc(const Prob& P, const void* q, const void* kp, const void* vp,
                               const uint32_t* sel, void* ws, const WsLayout& L, float scale,
                               void* out, float* lse, cudaStream_t st) {
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)P.n_h * P.s;
  if (!make_tmap_bf16_2d(&tk, kp, rows, kD, 128) || !make_tmap_bf16_2d(&tv, vp, rows, kD, 128))
    return cudaErrorInvalidValue;
  const size_t smem = fwd_tc_smem(P);
  cudaError_t e = cudaFuncSetAttribute(k_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(P.n_qt, P.n_h);
  k_fwd_tc<<<grid, kThreads, smem, st>>>(
      tk, tv, P, static_cast<const __nv_bfloat16*>(q), sel, ws_ptr<uint32_t>(ws, L.qt_kt_bits),
      scale * 1.4426950408889634f, static_cast<__nv_bfloat16*>(out), ws_ptr<float>(ws, L.o32),
      lse, ws_ptr<int>(ws, L.status));
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace vmoba
