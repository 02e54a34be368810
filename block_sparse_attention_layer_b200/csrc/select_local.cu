// Per-query-row block selection: the ablation's "threshold + local" and
// "topk + local" variants (VMoBA notes, ablation table; "topk + local" is
// about MoBA's selection, and digest App. A runs it training-free on 3D
// blocks).  Instead of one pool per head, each query row i ranks its own N_b
// scores S[i][.] (S desc, block asc):
//   threshold local: p = softmax of the row (same temperature as the pool),
//                    keep the shortest prefix whose mass reaches tau (the
//                    whole row if rounding leaves the total short);
//   top-k local:     keep the first min(k, N_b) blocks.
// The scores are the pool the score kernel wrote (fp32).  One warp per row:
// keys (~ordered score << 32 | block) are sorted ascending in shared memory
// by a bitonic network, the prefix rule is applied on the sorted order with
// fp64 sums, and the row's bitmap words are built in shared memory.  Per-row
// counts and kept masses go to scratch and a second kernel reduces them per
// head in a fixed order, so the stats are bitwise repeatable.
#include "common.cuh"

namespace vmoba {
namespace {

constexpr int kLocalWarps = 8;

template <int N>
__device__ __forceinline__ void warp_bitonic_sort(uint64_t* a, int lane) {
  for (int size = 2; size <= N; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncwarp();
      for (int t = lane; t < N / 2; t += 32) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const uint64_t x = a[lo], y = a[hi];
        if ((x > y) == asc) { a[lo] = y; a[hi] = x; }
      }
    }
  }
  __syncwarp();
}

// N = N_b rounded up to a power of two (>= 32).
template <int N>
__global__ void __launch_bounds__(32 * kLocalWarps)
k_select_local(Prob P, const float* __restrict__ S, int topk, double param,
               uint32_t* __restrict__ sel, uint32_t* __restrict__ row_cnt,
               double* __restrict__ row_mass) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* keys = reinterpret_cast<uint64_t*>(smem) + (size_t)warp * N;
  uint32_t* bits = reinterpret_cast<uint32_t*>(reinterpret_cast<uint64_t*>(smem) +
                                               (size_t)kLocalWarps * N) + warp * 32;
  constexpr int kSeg = N / 32;          // sorted elements per lane (contiguous)
  const long long rows = (long long)P.n_h * P.s;
  for (long long r = (long long)blockIdx.x * kLocalWarps + warp; r < rows;
       r += (long long)gridDim.x * kLocalWarps) {
    const float* row = S + (size_t)r * P.Nb;
    float mx = -INFINITY;
    for (int j = lane; j < N; j += 32) {
      uint64_t key = ~0ull;
      if (j < P.Nb) {
        const float x = __ldg(row + j);
        mx = fmaxf(mx, x);
        key = ((uint64_t)(~f2key(x)) << 32) | (uint32_t)j;
      }
      keys[j] = key;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    warp_bitonic_sort<N>(keys, lane);
    // the lane's contiguous run of the sorted order: masses (fp64 sums of
    // fp32 exponentials, as the pool selection)
    double seg = 0.0;
    for (int u = 0; u < kSeg; ++u) {
      const int t = lane * kSeg + u;
      if (t < P.Nb) seg += (double)expf(key2f(~(uint32_t)(keys[t] >> 32)) - mx);
    }
    double before = seg;          // exclusive scan of the runs over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, before, o);
      if (lane >= o) before += y;
    }
    const double Z = __shfl_sync(0xffffffffu, before, 31);
    before -= seg;
    const double target = param * Z;
    const int kk = topk ? (int)fmin(param, (double)P.Nb) : 0;
    if (lane < 32 && lane < P.Wb) bits[lane] = 0u;
    __syncwarp();
    uint32_t cnt = 0;
    double kept = 0.0;
    double run = before;
    for (int u = 0; u < kSeg; ++u) {
      const int t = lane * kSeg + u;
      if (t >= P.Nb) break;
      const double p = (double)expf(key2f(~(uint32_t)(keys[t] >> 32)) - mx);
      // keep t while the mass ranked before it is still short of the target
      const bool on = topk ? t < kk : run < target;
      if (on) {
        const uint32_t j = (uint32_t)keys[t];
        atomicOr(&bits[j >> 5], 1u << (j & 31));
        ++cnt;
        kept += p;
      }
      run += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      kept += __shfl_xor_sync(0xffffffffu, kept, o);
    }
    __syncwarp();
    if (lane < P.Wb) sel[(size_t)r * P.Wb + lane] = bits[lane];
    if (lane == 0) {
      row_cnt[r] = cnt;
      row_mass[r] = Z > 0.0 ? kept / Z : 0.0;
    }
    __syncwarp();
  }
}

// Per head, in a fixed order: pairs kept and the mean kept mass per row.
__global__ void __launch_bounds__(1024)
k_local_stats(Prob P, const uint32_t* __restrict__ row_cnt, const double* __restrict__ row_mass,
              vmoba_head_stats* __restrict__ out) {
  __shared__ unsigned long long sc[1024];
  __shared__ double sm[1024];
  const int h = blockIdx.x, t = threadIdx.x;
  unsigned long long c = 0;
  double m = 0.0;
  for (int i = t; i < P.s; i += 1024) {
    c += row_cnt[(size_t)h * P.s + i];
    m += row_mass[(size_t)h * P.s + i];
  }
  sc[t] = c;
  sm[t] = m;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (t < w) { sc[t] += sc[t + w]; sm[t] += sm[t + w]; }
    __syncthreads();
  }
  if (t == 0) {
    vmoba_head_stats o;
    o.n_selected = (long long)sc[0];
    o.mass = sm[0] / (double)P.s;
    o.cut_score = nanf("");
    o.all_selected = sc[0] == (unsigned long long)P.s * P.Nb ? 1 : 0;
    out[h] = o;
  }
}

template <int N>
cudaError_t run_local(const Prob& P, const float* S, int topk, double param, uint32_t* sel,
                      uint32_t* rc, double* rm, cudaStream_t st) {
  const size_t smem = sizeof(uint64_t) * kLocalWarps * N + sizeof(uint32_t) * kLocalWarps * 32;
  cudaError_t e = cudaFuncSetAttribute(k_select_local<N>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)P.n_h * P.s;
  const int grid = (int)((rows + kLocalWarps - 1) / kLocalWarps);
  {
    VMOBA_TRACE("k_select_local", st);
    k_select_local<N><<<grid, 32 * kLocalWarps, smem, st>>>(P, S, topk, param, sel, rc, rm);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_local(const Prob& P, int topk, double param, uint32_t* sel,
                                vmoba_head_stats* stats, void* ws, const WsLayout& L,
                                cudaStream_t st) {
  const float* S = ws_ptr<float>(ws, L.scores);
  // per-row scratch in the forward-output copy (written only by the forward)
  uint32_t* rc = ws_ptr<uint32_t>(ws, L.o32);
  double* rm = reinterpret_cast<double*>(
      ws_ptr<char>(ws, L.o32) + align_up(sizeof(uint32_t) * (size_t)P.n_h * P.s, 256));
  cudaError_t e;
  if (P.Nb <= 32) e = run_local<32>(P, S, topk, param, sel, rc, rm, st);
  else if (P.Nb <= 64) e = run_local<64>(P, S, topk, param, sel, rc, rm, st);
  else if (P.Nb <= 128) e = run_local<128>(P, S, topk, param, sel, rc, rm, st);
  else if (P.Nb <= 256) e = run_local<256>(P, S, topk, param, sel, rc, rm, st);
  else if (P.Nb <= 512) e = run_local<512>(P, S, topk, param, sel, rc, rm, st);
  else e = run_local<1024>(P, S, topk, param, sel, rc, rm, st);
  if (e != cudaSuccess) return e;
  {
    VMOBA_TRACE("k_local_stats", st);
    k_local_stats<<<P.n_h, 1024, 0, st>>>(P, rc, rm, stats);
  }
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace vmoba
