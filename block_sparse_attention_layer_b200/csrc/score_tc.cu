// Step 2 of the layer on the 5th-generation tensor cores (bf16 Q, head_dim
// 64 or 128): the per-head score pool S = scale * q_i b_j^T of every query
// and block, written once, with each head's max, for the selection passes.
//
// VMoBA notes, key design 2 (one global pool of all s x N_b query-block
// pairs per head, S^ = q_i b_i^T).
//
// Q is exactly bf16; the fp32 block means are split as B = B_hi + B_lo with
// B_hi = bf16(B) and B_lo = bf16(B - B_hi), and both products accumulate in
// fp32 in TMEM (kind::f16 MMAs), which keeps S within about 1e-6 relative of
// the fp32 dot product.  Q is read one 128-query tile at a time by TMA
// straight from the [s][n_h][d] input.
//
// Persistent CTAs, cph per head (CTA b: head b / cph, query tiles b % cph,
// + cph, ...); 384 threads: warp 0 TMA producer, warp 1 TMEM owner and MMA
// issuer, warps 4-11 epilogue (warp w reads TMEM lanes 32 (w % 4) .. +32 and
// columns 64 ((w - 4) / 4) .. +64 of each 128-block chunk) writing the
// scores and the running max.  Two TMEM accumulators (256 columns) let the
// MMAs of the next chunk run while the epilogue reads the current one.  B
// chunks stay resident in shared memory when a head has at most 256 blocks;
// otherwise they stream through a two-stage ring.
//
// (Running the selection's histogram passes straight off the accumulator,
// with no pool in memory, was measured slower: at one CTA per SM the
// histogram's shared-memory atomics could not hide their latency, where the
// stored-pool kernels run many CTAs per SM.)
#include "tc_prims.cuh"

namespace vmoba {
namespace {

using namespace tc;

constexpr int kThreads = 384;
constexpr int kEpiThreads = 256;

template <int D>
struct Geo {
  static constexpr uint32_t kHalf = 128 * 64 * 2;          // 128 rows x 64 bf16, 128B-swizzled
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQ = kHalves * kHalf;           // one 128-query tile
  static constexpr uint32_t kB = 2 * kHalves * kHalf;       // one 128-block chunk, hi + lo
  static constexpr uint32_t kStage = 8 * 32 * 32 * 4;      // epilogue: 32 x 32 fp32 per warp
  static constexpr size_t kSmem = 1024 + 2 * kQ + 2 * kB + kStage + 256;
};
static_assert(Geo<128>::kSmem <= 232448, "shared memory per CTA");

struct PoolBars {
  uint64_t q_full[2], q_empty[2], b_full[2], b_empty[2], acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(PoolBars) <= 256, "barrier block");

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_score_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_b,
           Prob P, int NbP, int cph, float scale, SelState* __restrict__ st,
           float* __restrict__ pool, Watch wt) {
  using G = Geo<D>;
  const int h = blockIdx.x / cph, k0 = blockIdx.x - h * cph;
  const int n_qt = (P.s + 127) / 128;
  if (h >= P.n_h || k0 >= n_qt) return;                     // no tile: nothing loaded

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                                       // 2 tiles
  uint8_t* sB = sQ + 2 * G::kQ;                             // 2 chunks
  float* sStage = reinterpret_cast<float*>(sB + 2 * G::kB);  // 8 x 32 x 32 floats
  PoolBars* bars = reinterpret_cast<PoolBars*>(sB + 2 * G::kB + G::kStage);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb16 = (P.Nb + 15) & ~15;
  const int nch = (nb16 + 127) / 128;                       // 128-block chunks
  const bool resident = nch <= 2;
  const int my_tiles = (n_qt - 1 - k0) / cph + 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1); mbar_init(&bars->q_empty[i], 1);
      mbar_init(&bars->b_full[i], 1); mbar_init(&bars->b_empty[i], 1);
      mbar_init(&bars->acc_full[i], 1); mbar_init(&bars->acc_empty[i], kEpiThreads / 32);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_b);
      auto load_b = [&](int c, int stage) {
        const int row_hi = (h * 2) * NbP + c * 128, row_lo = (h * 2 + 1) * NbP + c * 128;
        uint8_t* dst = sB + stage * G::kB;
        mbar_expect_tx(&bars->b_full[stage], G::kB);
#pragma unroll
        for (int hf = 0; hf < G::kHalves; ++hf) {
          tma_load_2d(dst + hf * G::kHalf, &tm_b, &bars->b_full[stage], 64 * hf, row_hi);
          tma_load_2d(dst + (G::kHalves + hf) * G::kHalf, &tm_b, &bars->b_full[stage], 64 * hf,
                      row_lo);
        }
      };
      if (resident)
        for (int c = 0; c < nch; ++c) load_b(c, c);
      bool ok = true;
      int J = 0;
      for (int it = 0; it < my_tiles && ok; ++it) {
        const int t = k0 + it * cph, qs = it & 1;
        if (it >= 2) ok = mbar_wait(&bars->q_empty[qs], ((it >> 1) - 1) & 1, wt, abort);
        if (!ok) break;
        mbar_expect_tx(&bars->q_full[qs], G::kQ);
#pragma unroll
        for (int hf = 0; hf < G::kHalves; ++hf)
          tma_load_2d(sQ + qs * G::kQ + hf * G::kHalf, &tm_q, &bars->q_full[qs], h * D + 64 * hf,
                      t * 128);
        if (!resident) {
          for (int c = 0; c < nch && ok; ++c, ++J) {
            const int bs = J & 1;
            if (J >= 2) ok = mbar_wait(&bars->b_empty[bs], ((J >> 1) - 1) & 1, wt, abort);
            if (ok) load_b(c, bs);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      int A = 0, J = 0;
      for (int it = 0; it < my_tiles && ok; ++it) {
        const int qs = it & 1;
        if (!mbar_wait(&bars->q_full[qs], (it >> 1) & 1, wt, abort)) { ok = false; break; }
        const uint32_t qb = smem_u32(sQ + qs * G::kQ);
        for (int c = 0; c < nch && ok; ++c, ++A) {
          const int as = A & 1;
          if (A >= 2 && !mbar_wait(&bars->acc_empty[as], ((A >> 1) - 1) & 1, wt, abort)) {
            ok = false;
            break;
          }
          const int bs = resident ? c : (J & 1);
          const uint32_t par = resident ? 0u : (uint32_t)((J >> 1) & 1);
          if (!mbar_wait(&bars->b_full[bs], par, wt, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t bb = smem_u32(sB + bs * G::kB);
          const int n = min(128, nb16 - c * 128);
          const uint32_t idesc = idesc_bf16(128, n, false, false);
#pragma unroll
          for (int part = 0; part < 2; ++part) {              // B_hi, then B_lo
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * G::kHalf + (kk & 3) * 32;
              mma_ss(tmem + as * 128, desc_sw128(qb + off, 16, 1024),
                     desc_sw128(bb + part * G::kHalves * G::kHalf + off, 16, 1024), idesc,
                     (part > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(&bars->acc_full[as]);
          if (!resident) {
            mma_commit(&bars->b_empty[bs]);
            ++J;
          }
        }
        if (ok) mma_commit(&bars->q_empty[qs]);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int wq = warp & 3, g = (warp - 4) >> 2;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    // the warp's 32 rows x 32 columns pass through a staging tile (column e
    // of row r at r * 32 + (e ^ r): conflict-free by row and by column) and
    // leave one row per store instruction, 128 contiguous bytes, whatever
    // N_b's alignment
    float* stg = sStage + (warp - 4) * 1024;
    float vmax = -INFINITY;
    bool ok = true;
    int A = 0;
    for (int it = 0; it < my_tiles && ok; ++it) {
      const int t = k0 + it * cph;
      const int i0 = t * 128 + wq * 32;                       // the warp's first query row
      const bool row_ok = i0 + lane < P.s;                     // this thread's row
      const int nrows = min(32, P.s - i0);
      for (int c = 0; c < nch; ++c, ++A) {
        const int as = A & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->acc_full[as], (A >> 1) & 1, wt, abort));
        if (!ok) break;
        tc_fence_after();
        const int j0 = c * 128 + g * 64;                      // first block of the warp's columns
        const int vc = max(0, min(64, P.Nb - j0));            // valid blocks among them
        if (vc > 0) {
          uint32_t xr[64];
          tmem_ld32(tmem + as * 128 + lane_off + g * 64, xr);
          if (vc > 32) tmem_ld32(tmem + as * 128 + lane_off + g * 64 + 32, xr + 32);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (32 * u >= vc) break;
            const int ve = min(32, vc - 32 * u);
            __syncwarp();                                     // the last half's reads are done
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float x = __uint_as_float(xr[32 * u + e]) * scale;
              stg[lane * 32 + (e ^ lane)] = x;
              if (row_ok && e < ve) vmax = fmaxf(vmax, x);
            }
            __syncwarp();
            float* dst = pool + ((size_t)h * P.s + i0) * P.Nb + j0 + 32 * u + lane;
            if (lane < ve) {
#pragma unroll 4
              for (int r = 0; r < nrows; ++r) dst[(size_t)r * P.Nb] = stg[r * 32 + (lane ^ r)];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty[as]);
      }
    }
    // per-head max as an ordered key, one atomic per warp
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    if (lane == 0 && vmax > -INFINITY) atomicMax(&st[h].max_key, f2key(vmax));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// B = B_hi + B_lo in bf16, [n_h][2][NbP][D] (hi rows, then lo rows), blocks
// past N_b zero.
template <int D>
__global__ void k_split_blocks(Prob P, int NbP, const float* __restrict__ B,
                               __nv_bfloat16* __restrict__ bs) {
  const size_t n = (size_t)P.n_h * NbP * D;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(e % D);
    const size_t r = e / D;
    const int j = (int)(r % NbP), h = (int)(r / NbP);
    const float x = j < P.Nb ? B[((size_t)h * P.Nb + j) * D + k] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
    bs[(((size_t)h * 2) * NbP + j) * D + k] = hi;
    bs[(((size_t)h * 2 + 1) * NbP + j) * D + k] = lo;
  }
}

template <int D>
cudaError_t pool_tc(const Prob& P, const void* q, const float* blocks, float scale, void* bsplit,
                    float* pool, SelState* st, int* status, int num_sms, cudaStream_t stream) {
  const int NbP = sel_split_rows(P);
  {
    VMOBA_TRACE("k_split_blocks", stream);
    k_split_blocks<D><<<num_sms * 2, 256, 0, stream>>>(P, NbP, blocks,
                                                       static_cast<__nv_bfloat16*>(bsplit));
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tb;
  if (!make_tmap_bf16_2d(&tq, q, (uint64_t)P.s, (uint64_t)P.n_h * D, 128) ||
      !make_tmap_bf16_2d(&tb, bsplit, (uint64_t)P.n_h * 2 * NbP, D, 128))
    return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(k_score_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Geo<D>::kSmem);
  if (e != cudaSuccess) return e;
  const int cph = max(1, num_sms / P.n_h);
  {
    VMOBA_TRACE("k_score_tc", stream);
    k_score_tc<D><<<P.n_h * cph, kThreads, Geo<D>::kSmem, stream>>>(
        tq, tb, P, NbP, cph, scale, st, pool, make_watch(status));
  }
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace

int sel_split_rows(const Prob& P) { return (P.Nb + 127) / 128 * 128; }

size_t sel_split_bytes(const Prob& P) {
  return (size_t)P.n_h * 2 * sel_split_rows(P) * P.d * sizeof(__nv_bfloat16);
}

cudaError_t launch_score_pool_tc(const Prob& P, const void* q, const float* blocks, float scale,
                                 void* bsplit, float* pool, SelState* st, int* status,
                                 int num_sms, cudaStream_t stream) {
  return P.d == 128 ? pool_tc<128>(P, q, blocks, scale, bsplit, pool, st, status, num_sms, stream)
                    : pool_tc<64>(P, q, blocks, scale, bsplit, pool, st, status, num_sms, stream);
}

}  // namespace vmoba
