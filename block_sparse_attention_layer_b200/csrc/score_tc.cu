// Steps 2-3 of the layer on the 5th-generation tensor cores (bf16 Q, head_dim
// 64 or 128): the per-head score pool S = scale * q_i b_j^T, recomputed tile
// by tile in every pass of the selection instead of being written to memory.
//
// VMoBA notes, key design 2 (one global pool of all s x N_b query-block
// pairs per head, Ŝ = q_i b_i^T) and key design 3 (keep pairs in descending
// order until the normalised cumulative similarity reaches tau).
//
// Q is exactly bf16; the fp32 block means are split as B = B_hi + B_lo with
// B_hi = bf16(B) and B_lo = bf16(B - B_hi), and both products accumulate in
// fp32 in TMEM (kind::f16 MMAs), which keeps S within about 1e-6 relative of
// the fp32 dot product.  A pass reads Q (one 128-query tile at a time, by
// TMA straight from the [s][n_h][d] input) and the head's split B, and runs
// one of these epilogues on each 128 x 128 accumulator:
//   kMax        per-head max of S (ordered-key atomicMax, one per warp);
//   kHist0..2   radix histogram of the 32-bit order-preserving key of S over
//               the elements still in the candidate bucket: count and mass
//               exp(S - max S) per digit (fp32 per tile in shared memory,
//               folded into fp64 per CTA, fp64 atomics to global once);
//   kTie0..2    count-only radix histogram of the flat index i*N_b + j of the
//               elements whose key equals the cut (exact ties);
//   kEmit       the selection bitmap, one 32-bit word per 32 blocks of a row;
//   kPool       S itself, written to the workspace pool, and the head max.
// The digit walks between passes are the one-warp scans of score_select.cu.
//
// Persistent CTAs, cph per head (CTA b: head b / cph, query tiles b % cph,
// + cph, ...); 384 threads: warp 0 TMA producer, warp 1 TMEM owner and MMA
// issuer, warps 4-11 epilogue (warp w reads TMEM lanes 32 (w % 4) .. +32 and
// columns 64 ((w - 4) / 4) .. +64 of each 128-block chunk).  Two TMEM
// accumulators (256 columns) let the MMAs of the next chunk run while the
// epilogue reads the current one.  B chunks stay resident in shared memory
// when a head has at most 256 blocks; otherwise they stream through a
// two-stage ring.
#include "tc_prims.cuh"

namespace vmoba {
namespace {

using namespace tc;

constexpr int kThreads = 384;
constexpr int kEpiThreads = 256;
constexpr int kBins = kHistBins;
constexpr float kLog2e = 1.4426950408889634f;

enum SelPass {
  kMax = 0, kHist0 = 1, kHist1 = 2, kHist2 = 3, kTie0 = 4, kTie1 = 5, kTie2 = 6,
  kEmit = 7, kPool = 8
};
// SelState::state values (score_select.cu)
constexpr int kStSearch = 0, kStAll = 2, kStTies = 3;

template <int D>
struct Geo {
  static constexpr uint32_t kHalf = 128 * 64 * 2;          // 128 rows x 64 bf16, 128B-swizzled
  static constexpr int kHalves = D / 64;
  static constexpr uint32_t kQ = kHalves * kHalf;           // one 128-query tile
  static constexpr uint32_t kB = 2 * kHalves * kHalf;       // one 128-block chunk, hi + lo
  static constexpr size_t kSmem = 1024 + 2 * kQ + 2 * kB +
                                  kBins * (sizeof(uint32_t) + sizeof(float) + sizeof(double)) +
                                  256;
};
static_assert(Geo<128>::kSmem <= 232448, "shared memory per CTA");

struct SelBars {
  uint64_t q_full[2], q_empty[2], b_full[2], b_empty[2], acc_full[2], acc_empty[2];
  uint64_t adds_done, fold_done;       // epilogue warps: a tile's histogram adds / fp64 fold
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SelBars) <= 256, "barrier block");

template <int PASS>
__device__ __forceinline__ bool radix_digit(uint32_t key, uint32_t prefix, uint32_t& dig) {
  // three digits of 11, 11 and 10 bits, most significant first; a digit
  // counts only if the bits above it equal the resolved prefix
  constexpr int p = (PASS >= kTie0) ? PASS - kTie0 : PASS - kHist0;
  if (p == 0) { dig = key >> 21; return true; }
  if (p == 1) { dig = (key >> 10) & 2047u; return (key >> 21) == prefix; }
  dig = key & 1023u;
  return (key >> 10) == prefix;
}

template <int D, int PASS>
__global__ void __launch_bounds__(kThreads, 1)
k_score_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_b,
           Prob P, int NbP, int cph, float scale, SelState* __restrict__ st,
           uint32_t* __restrict__ hc, double* __restrict__ hm, uint32_t* __restrict__ sel,
           float* __restrict__ pool, Watch wt) {
  using G = Geo<D>;
  const int h = blockIdx.x / cph, k0 = blockIdx.x - h * cph;
  const int n_qt = (P.s + 127) / 128;
  if (h >= P.n_h || k0 >= n_qt) return;                     // no tile: nothing loaded
  const int state = st[h].state;
  if (PASS >= kHist0 && PASS <= kHist2 && state != kStSearch) return;
  if (PASS >= kTie0 && PASS <= kTie2 && state != kStTies) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                                       // 2 tiles
  uint8_t* sB = sQ + 2 * G::kQ;                             // 2 chunks
  uint32_t* hcnt = reinterpret_cast<uint32_t*>(sB + 2 * G::kB);
  float* hm32 = reinterpret_cast<float*>(hcnt + kBins);
  double* hm64 = reinterpret_cast<double*>(hm32 + kBins);
  SelBars* bars = reinterpret_cast<SelBars*>(hm64 + kBins);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb16 = (P.Nb + 15) & ~15;
  const int nch = (nb16 + 127) / 128;                       // 128-block chunks
  const bool resident = nch <= 2;
  const int my_tiles = (n_qt - 1 - k0) / cph + 1;

  constexpr bool kHist = PASS >= kHist0 && PASS <= kHist2;
  constexpr bool kTie = PASS >= kTie0 && PASS <= kTie2;
  if (kHist || kTie)
    for (int b = threadIdx.x; b < kBins; b += kThreads) {
      hcnt[b] = 0u;
      hm32[b] = 0.f;
      hm64[b] = 0.0;
    }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1); mbar_init(&bars->q_empty[i], 1);
      mbar_init(&bars->b_full[i], 1); mbar_init(&bars->b_empty[i], 1);
      mbar_init(&bars->acc_full[i], 1); mbar_init(&bars->acc_empty[i], kEpiThreads / 32);
    }
    mbar_init(&bars->adds_done, kEpiThreads / 32);
    mbar_init(&bars->fold_done, kEpiThreads / 32);
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
    const int et = threadIdx.x - 128;                       // 0..255
    const int wq = warp & 3, g = (warp - 4) >> 2;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    // all eight epilogue warps past a point: bounded, so that a warp that gave
    // up on a timed-out wait cannot leave the others blocked
    auto epi_sync = [&](uint64_t* bar, int phase) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
      return __all_sync(0xffffffffu, mbar_wait(bar, (uint32_t)(phase & 1), wt, abort));
    };
    int n_sync = 0;
    const SelState S0 = st[h];
    const uint32_t prefix = S0.prefix, cut = S0.cut_key, idx_cut = S0.idx_cut;
    const float ml2 = key2f(S0.max_key) * kLog2e;           // log2(e) max S
    const float sl2 = scale * kLog2e;
    float vmax = -INFINITY;
    bool ok = true;
    int A = 0;
    for (int it = 0; it < my_tiles && ok; ++it) {
      const int t = k0 + it * cph;
      const int i = t * 128 + wq * 32 + lane;                 // this thread's query row
      const bool row_ok = i < P.s;
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
            uint32_t word = 0u;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (e >= ve || !row_ok) continue;
              const int j = j0 + 32 * u + e;
              const float x = __uint_as_float(xr[32 * u + e]) * scale;
              if (PASS == kMax) {
                vmax = fmaxf(vmax, x);
              } else if (kHist) {
                uint32_t dig;
                if (radix_digit<PASS>(f2key(x), prefix, dig)) {
                  atomicAdd(&hcnt[dig], 1u);
                  atomicAdd(&hm32[dig], fast_exp2(fmaf(__uint_as_float(xr[32 * u + e]), sl2,
                                                       -ml2)));
                }
              } else if (kTie) {
                uint32_t dig;
                if (f2key(x) == cut &&
                    radix_digit<PASS>((uint32_t)((size_t)i * P.Nb + j), prefix, dig))
                  atomicAdd(&hcnt[dig], 1u);
              } else if (PASS == kEmit) {
                const uint32_t key = f2key(x);
                const uint32_t idx = (uint32_t)((size_t)i * P.Nb + j);
                const bool on = state == kStAll || key > cut || (key == cut && idx <= idx_cut);
                word |= (on ? 1u : 0u) << e;
              } else {                                         // kPool
                pool[((size_t)h * P.s + i) * P.Nb + j] = x;
                vmax = fmaxf(vmax, x);
              }
            }
            if (PASS == kEmit && row_ok)
              sel[((size_t)h * P.s + i) * P.Wb + (j0 >> 5) + u] = word;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty[as]);
      }
      if (kHist && ok) {
        // fold this tile's fp32 masses into the CTA's fp64 sums (each thread
        // its own bins, once every warp's adds of the tile are in)
        ok = epi_sync(&bars->adds_done, n_sync);
        if (!ok) break;
        for (int b = et; b < kBins; b += kEpiThreads) {
          const float v = hm32[b];
          if (v != 0.f) {
            hm64[b] += (double)v;
            hm32[b] = 0.f;
          }
        }
        ok = epi_sync(&bars->fold_done, n_sync);
        ++n_sync;
      }
    }
    if (kTie && ok) ok = epi_sync(&bars->adds_done, n_sync);
    if (PASS == kMax || PASS == kPool) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      if (lane == 0 && vmax > -INFINITY) atomicMax(&st[h].max_key, f2key(vmax));
    }
    if ((kHist || kTie) && ok) {
      // every add and fold is in: each thread sends its own bins
      for (int b = et; b < kBins; b += kEpiThreads) {
        if (hcnt[b]) {
          atomicAdd(&hc[h * kBins + b], hcnt[b]);
          if (kHist) atomicAdd(&hm[h * kBins + b], hm64[b]);
        }
      }
    }
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

template <int D, int PASS>
cudaError_t launch_pass(const Prob& P, int NbP, const CUtensorMap& tq, const CUtensorMap& tb,
                        float scale, SelState* st, uint32_t* hc, double* hm, uint32_t* sel,
                        float* pool, int* status, int num_sms, cudaStream_t stream,
                        const char* name) {
  cudaError_t e = cudaFuncSetAttribute(k_score_tc<D, PASS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Geo<D>::kSmem);
  if (e != cudaSuccess) return e;
  const int cph = max(1, num_sms / P.n_h);
  VMOBA_TRACE(name, stream);
  k_score_tc<D, PASS><<<P.n_h * cph, kThreads, Geo<D>::kSmem, stream>>>(
      tq, tb, P, NbP, cph, scale, st, hc, hm, sel, pool, make_watch(status));
  return cudaGetLastError();
}

template <int D>
cudaError_t run_passes(const Prob& P, const void* q, const float* blocks, float scale,
                       const SelPassOps& ops, cudaStream_t stream) {
  const int NbP = sel_split_rows(P);
  {
    VMOBA_TRACE("k_split_blocks", stream);
    k_split_blocks<D><<<ops.num_sms * 2, 256, 0, stream>>>(
        P, NbP, blocks, static_cast<__nv_bfloat16*>(ops.bsplit));
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tb;
  if (!make_tmap_bf16_2d(&tq, q, (uint64_t)P.s, (uint64_t)P.n_h * D, 128) ||
      !make_tmap_bf16_2d(&tb, ops.bsplit, (uint64_t)P.n_h * 2 * NbP, D, 128))
    return cudaErrorInvalidValue;
  int launches = 1;
#define VMOBA_PASS(ID, NAME)                                                                   \
  do {                                                                                         \
    e = launch_pass<D, ID>(P, NbP, tq, tb, scale, ops.st, ops.hc, ops.hm, ops.sel, ops.pool,  \
                           ops.status, ops.num_sms, stream, NAME);                             \
    ++launches;                                                                                \
    if (e != cudaSuccess) return e;                                                            \
  } while (0)
  if (ops.pool_only) {
    VMOBA_PASS(kPool, "k_score_tc_pool");
    count_launches(launches);
    return cudaSuccess;
  }
  VMOBA_PASS(kMax, "k_score_tc_max");
  for (int p = 0; p < 3; ++p) {
    if (p == 0) VMOBA_PASS(kHist0, "k_score_tc_hist");
    if (p == 1) VMOBA_PASS(kHist1, "k_score_tc_hist");
    if (p == 2) VMOBA_PASS(kHist2, "k_score_tc_hist");
    if ((e = ops.scan(p, stream)) != cudaSuccess) return e;
  }
  for (int p = 0; p < 3; ++p) {
    if (p == 0) VMOBA_PASS(kTie0, "k_score_tc_tie");
    if (p == 1) VMOBA_PASS(kTie1, "k_score_tc_tie");
    if (p == 2) VMOBA_PASS(kTie2, "k_score_tc_tie");
    if ((e = ops.tie_scan(p, stream)) != cudaSuccess) return e;
  }
  VMOBA_PASS(kEmit, "k_score_tc_emit");
#undef VMOBA_PASS
  count_launches(launches);
  return cudaSuccess;
}

}  // namespace

int sel_split_rows(const Prob& P) { return (P.Nb + 127) / 128 * 128; }

size_t sel_split_bytes(const Prob& P) {
  return (size_t)P.n_h * 2 * sel_split_rows(P) * P.d * sizeof(__nv_bfloat16);
}

cudaError_t launch_score_passes_tc(const Prob& P, const void* q, const float* blocks,
                                   float scale, const SelPassOps& ops, cudaStream_t stream) {
  return P.d == 128 ? run_passes<128>(P, q, blocks, scale, ops, stream)
                    : run_passes<64>(P, q, blocks, scale, ops, stream);
}

}  // namespace vmoba
