// Steps 2-3 of the layer: the per-head score pool S = scale * q_i b_i^T and
// the global threshold selection over it.
//
// VMoBA notes, key design 2 (global block selection: one pool of all s x N_b
// query-block pairs per head) and key design 3 (k = min{k' : cumulative
// normalised similarity >= tau}); digest sections 3.3 and 3.4.
//
// "Normalised" is read as p = exp(S - max S) / Z over the head's whole pool,
// Z = sum exp(S - max S).  The cut is found without sorting: an exact radix
// select over the 32-bit order-preserving key of each fp32 score, three
// passes of 11/11/10 bits.  Each pass histograms (count, sum of exp(S - m))
// per digit for the elements still in the candidate bucket; a one-warp scan
// per head walks the digits from the top until the mass reaches tau * Z.
// Exact ties at the cut are ranked by flat index i*N_b + j (ascending) with
// three more count-only radix passes that return at once unless needed.
//
// The pool is written once -- by the tensor cores for bf16 inputs
// (score_tc.cu; every workload of the method), with fp32 FMAs on the CUDA
// cores for fp32 inputs, whose 1e-4 output bar the bf16 split of Q could not
// meet -- and read by each pass: init -> pool (and max) -> {hist, scan} x 3
// -> {tie_hist, tie_scan} x 3 -> emit -> stats.
//
// The ablation's "topk + global" variant (VMoBA notes, ablation table) runs
// the same passes with the digit walk counting pairs instead of mass: the
// cut is then the k-th pair of the same ranking; the masses still ride
// along for the stats (a last-pass bucket holds one score value, so its
// share of the mass is exact).
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "tc_prims.cuh"

namespace vmoba {
namespace {

constexpr int kSel_Search = 0, kSel_Resolved = 1, kSel_All = 2, kSel_Ties = 3;

// Element k of a 16-byte vector held as four 32-bit words.
template <typename E>
__device__ __forceinline__ float word_elem(const uint32_t* w, int k);
template <>
__device__ __forceinline__ float word_elem<float>(const uint32_t* w, int k) {
  return __uint_as_float(w[k]);
}

__global__ void k_init(SelState* st, uint32_t* hc, unsigned long long* hm, int n_h) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_h * kHistBins;
       i += gridDim.x * blockDim.x) {
    hc[i] = 0u;
    hm[i] = 0ull;
  }
  if (blockIdx.x == 0 && threadIdx.x < n_h) {
    SelState s{};
    s.max_key = 0u;
    s.idx_cut = 0xFFFFFFFFu;
    s.state = kSel_Search;
    st[threadIdx.x] = s;
  }
}

// ---------------------------------------------------------------- scores
// 128 queries x 64 blocks per CTA step, 256 threads (16 x 16), 8 queries x
// 4 blocks per thread, fp32 FMA over d in pairs of queries (fma.rn.f32x2:
// two round-to-nearest FMAs, the same results as scalar ones in the same
// order).  Q tile and B chunk are staged transposed in shared memory: 16-byte
// global loads, one row per lane, so the transposed stores hit 32 distinct
// banks (row pitches 132 and 68 floats).  Per d step a thread reads two
// query float4s (a broadcast across its half-warp) and one block float4.
constexpr int kSQ = 128, kSB = 64, kQPad = 132, kBPad = 68;

template <typename E, int D>
__global__ void __launch_bounds__(256)
k_score(Prob P, const E* __restrict__ q, const float* __restrict__ B, float scale,
        float* __restrict__ S, SelState* __restrict__ st) {
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;                  // [D][kQPad]
  float* Bs = sm + D * kQPad;      // [D][kBPad]
  const int i0 = blockIdx.x * kSQ, h = blockIdx.y;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;

  // Q: 16-byte vectors of V elements; item = (vector g, query r), r fastest
  constexpr int V = 16 / (int)sizeof(E);
  for (int id = threadIdx.x; id < kSQ * (D / V); id += 256) {
    const int r = id % kSQ, g = id / kSQ, i = i0 + r;
    float x[V];
    if (i < P.s) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(q + ((size_t)i * P.n_h + h) * D) + g);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < V; ++k) x[k] = word_elem<E>(w, k);
    } else {
#pragma unroll
      for (int k = 0; k < V; ++k) x[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < V; ++k) Qs[(g * V + k) * kQPad + r] = x[k];
  }
  float vmax = -INFINITY;
  const float* Bh = B + (size_t)h * P.Nb * D;
  for (int j0 = 0; j0 < P.Nb; j0 += kSB) {
    __syncthreads();
    for (int id = threadIdx.x; id < kSB * (D / 4); id += 256) {
      const int r = id % kSB, g = id / kSB, j = j0 + r;
      const float4 v = j < P.Nb ? __ldg(reinterpret_cast<const float4*>(Bh + (size_t)j * D) + g)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      Bs[(4 * g + 0) * kBPad + r] = v.x;
      Bs[(4 * g + 1) * kBPad + r] = v.y;
      Bs[(4 * g + 2) * kBPad + r] = v.z;
      Bs[(4 * g + 3) * kBPad + r] = v.w;
    }
    __syncthreads();
    uint64_t acc[4][4];            // [query pair (2a, 2a+1)][block b]
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0ull;
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      const float4 q0 = *reinterpret_cast<const float4*>(Qs + c * kQPad + 8 * ty);
      const float4 q1 = *reinterpret_cast<const float4*>(Qs + c * kQPad + 8 * ty + 4);
      const float4 bb = *reinterpret_cast<const float4*>(Bs + c * kBPad + 4 * tx);
      const uint64_t qp[4] = {tc::f32x2(q0.x, q0.y), tc::f32x2(q0.z, q0.w),
                              tc::f32x2(q1.x, q1.y), tc::f32x2(q1.z, q1.w)};
      const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint64_t b2 = tc::f32x2(bv[b], bv[b]);
#pragma unroll
        for (int a = 0; a < 4; ++a) acc[a][b] = tc::fma_x2(qp[a], b2, acc[a][b]);
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = i0 + 8 * ty + 2 * a + e;
        if (i >= P.s) continue;
        float* row = S + ((size_t)h * P.s + i) * P.Nb;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int j = j0 + 4 * tx + b;
          if (j < P.Nb) {
            const float2 pr = tc::f32x2_split(acc[a][b]);
            const float x = (e ? pr.y : pr.x) * scale;
            row[j] = x;
            vmax = fmaxf(vmax, x);
          }
        }
      }
    }
  }
  // per-head maximum -> ordered key, one atomic per warp
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  if ((threadIdx.x & 31) == 0 && vmax > -INFINITY) atomicMax(&st[h].max_key, f2key(vmax));
}

// ------------------------------------------------------------- histograms
constexpr int kHistThreads = 256;
constexpr int kHistChunk = 64 * 1024;   // pool elements per CTA
// Bucket masses are summed in fixed point, so that their values do not depend
// on the order in which the atomics land: a CTA adds each element's mass
// exp(x - max) <= 1 as an integer multiple of 2^-kMassBitsCta (2^16 elements
// of at most 2^47 each stay below 2^63), in three 16-bit parts with 32-bit
// shared atomics (faster than fp32 shared atomics, and than 64-bit ones),
// then adds its bucket totals, rounded to 2^-F (F = 63 - ceil(log2 pool), at
// most kMassBitsCta), into the head's 64-bit global buckets, which therefore
// cannot overflow either.  An element's mass is off by at most 2^-48 (about
// 4e-15 of the head's largest), far below the fp32 rounding of the scores.
constexpr int kMassBitsCta = 47;
static_assert(kHistChunk == 1 << (63 - kMassBitsCta), "per-CTA fixed-point range");

template <int PASS>
__device__ __forceinline__ bool digit_of(uint32_t key, uint32_t prefix, uint32_t& dig) {
  if (PASS == 0) { dig = key >> 21; return true; }
  if (PASS == 1) { dig = (key >> 10) & 2047u; return (key >> 21) == prefix; }
  dig = key & 1023u;
  return (key >> 10) == prefix;
}

template <int PASS>
__global__ void __launch_bounds__(kHistThreads)
k_hist(Prob P, const float* __restrict__ S, SelState* __restrict__ st, uint32_t* __restrict__ hc,
       unsigned long long* __restrict__ hm, int shift) {
  // the mass in three 16-bit parts, each summed by 32-bit shared atomics
  // (at most 2^16 elements of at most 2^16 each: no part overflows)
  __shared__ uint32_t cnt[kHistBins], m0[kHistBins], m1[kHistBins], m2[kHistBins];
  const int h = blockIdx.y;
  if (st[h].state != kSel_Search) return;
  for (int b = threadIdx.x; b < kHistBins; b += kHistThreads) {
    cnt[b] = 0u;
    m0[b] = 0u;
    m1[b] = 0u;
    m2[b] = 0u;
  }
  __syncthreads();
  const float m = key2f(st[h].max_key);
  const uint32_t prefix = st[h].prefix;
  const size_t pool = (size_t)P.s * P.Nb;
  const float* base = S + (size_t)h * pool;
  const size_t beg = (size_t)blockIdx.x * kHistChunk;
  const size_t end = min(beg + (size_t)kHistChunk, pool);
  auto add = [&](float x) {
    uint32_t dig;
    if (digit_of<PASS>(f2key(x), prefix, dig)) {
      atomicAdd(&cnt[dig], 1u);
      const unsigned long long v = __float2ull_rn(expf(x - m) * 140737488355328.f);   // 2^47
      atomicAdd(&m0[dig], (uint32_t)(v & 0xFFFFu));
      atomicAdd(&m1[dig], (uint32_t)((v >> 16) & 0xFFFFu));
      atomicAdd(&m2[dig], (uint32_t)(v >> 32));
    }
  };
  if ((pool & 3) == 0) {
    // 16-byte loads: the head's pool starts 16-byte aligned and beg, end
    // are multiples of 4
    const float4* b4 = reinterpret_cast<const float4*>(base);
    for (size_t f = beg / 4 + threadIdx.x; f < end / 4; f += kHistThreads) {
      const float4 v = __ldg(b4 + f);
      add(v.x);
      add(v.y);
      add(v.z);
      add(v.w);
    }
  } else {
    for (size_t f = beg + threadIdx.x; f < end; f += kHistThreads) add(__ldg(base + f));
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kHistBins; b += kHistThreads) {
    if (cnt[b]) {
      atomicAdd(&hc[h * kHistBins + b], cnt[b]);
      const unsigned long long v = (unsigned long long)m0[b] + ((unsigned long long)m1[b] << 16) +
                                   ((unsigned long long)m2[b] << 32);
      atomicAdd(&hm[h * kHistBins + b], shift == 0 ? v : (v + (1ull << (shift - 1))) >> shift);
    }
  }
}

// One warp per head: walk the digits from the top, stop where the mass
// reaches the target, record the bucket and the mass/count strictly above.
template <int PASS>
__global__ void __launch_bounds__(32)
k_scan(Prob P, SelState* __restrict__ st, uint32_t* __restrict__ hc,
       unsigned long long* __restrict__ hm, double qinv, float tau, int by_count, double kcount) {
  const int h = blockIdx.x, lane = threadIdx.x;
  SelState& S = st[h];
  if (S.state != kSel_Search) return;
  uint32_t* c = hc + h * kHistBins;
  unsigned long long* mi = hm + h * kHistBins;
  // bucket mass as a double (fixed point, quantum qinv)
  auto mm = [&](int d) { return (double)mi[d] * qinv; };
  const int nb = (PASS == 2) ? 1024 : 2048;
  const int per = nb / 32;
  // lane l owns digits nb-1-l*per ... nb-per-l*per (descending)
  unsigned long long li = 0;
  unsigned long long lc = 0;
  for (int k = 0; k < per; ++k) {
    int d = nb - 1 - lane * per - k;
    li += mi[d];
    lc += c[d];
  }
  const double lm = (double)li * qinv;
  double above = S.mass_above, target = S.target;
  unsigned long long cabove = S.count_above;
  if (PASS == 0) {
    double tot = lm;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    above = 0.0;
    cabove = 0;
    target = by_count ? kcount : (double)tau * tot;
    if (lane == 0) { S.Z = tot; S.target = target; }
  }
  // the walk stops where the running mass (or pair count) reaches the target
  auto reach = [&](double m, unsigned long long cnt) {
    return by_count ? (double)cnt >= target : m >= target;
  };
  double incl = lm;
  unsigned long long cincl = lc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double y = __shfl_up_sync(0xffffffffu, incl, o);
    unsigned long long yc = __shfl_up_sync(0xffffffffu, cincl, o);
    if (lane >= o) { incl += y; cincl += yc; }
  }
  const unsigned ball = __ballot_sync(0xffffffffu, reach(above + incl, cabove + cincl));
  const unsigned nz = __ballot_sync(0xffffffffu, lc > 0);
  if (nz == 0u || (ball == 0u && PASS == 0)) {
    // tau reaches the whole pool: every pair is selected
    if (lane == 0) {
      S.state = kSel_All;
      S.n_selected = (unsigned long long)P.s * P.Nb;
      S.mass_selected = S.Z;
    }
    return;
  }
  // deciding lane: first lane whose running mass reaches the target (or, on a
  // rounding shortfall, the last lane holding elements), moved forward to a
  // lane that holds elements
  int fl = ball ? (__ffs(ball) - 1) : (31 - __clz(nz));
  const unsigned later = nz & (0xffffffffu << fl);
  fl = later ? (__ffs(later) - 1) : (31 - __clz(nz));
  int chosen = -1;
  double acc = 0.0;
  unsigned long long cacc = 0;
  if (lane == fl) {
    acc = above + (incl - lm);
    cacc = cabove + (cincl - lc);
    int last = -1;
    double acc_last = 0.0;
    unsigned long long cacc_last = 0;
    for (int k = 0; k < per; ++k) {
      int d = nb - 1 - lane * per - k;
      if (c[d]) {
        if (reach(acc + mm(d), cacc + c[d])) { chosen = d; break; }
        last = d;
        acc_last = acc;
        cacc_last = cacc;
      }
      acc += mm(d);
      cacc += c[d];
    }
    if (chosen < 0) { chosen = last; acc = acc_last; cacc = cacc_last; }
  }
  chosen = __shfl_sync(0xffffffffu, chosen, fl);
  acc = __shfl_sync(0xffffffffu, acc, fl);
  cacc = __shfl_sync(0xffffffffu, cacc, fl);
  if (lane == 0) {
    const uint32_t pre = (PASS == 0) ? (uint32_t)chosen
                                     : ((S.prefix << (PASS == 1 ? 11 : 10)) | (uint32_t)chosen);
    S.prefix = pre;
    S.mass_above = acc;
    S.count_above = cacc;
    if (PASS == 2) {
      const uint32_t nt = c[chosen];
      const double e = mm(chosen) / (double)nt;   // one score value: equal shares
      const double need = by_count ? target - (double)cacc : target - acc;
      const double rr = by_count ? need : ((need > 0.0 && e > 0.0) ? ceil(need / e) : 1.0);
      const uint32_t r = (rr < 1.0) ? 1u : (rr >= (double)nt ? nt : (uint32_t)rr);
      S.cut_key = pre;
      S.tie_count = nt;
      S.n_selected = cacc + r;
      S.mass_selected = acc + (double)r * e;
      if (r == nt) {
        S.state = kSel_Resolved;
        S.idx_cut = 0xFFFFFFFFu;
      } else {
        S.state = kSel_Ties;
        S.tie_take = r;
        S.prefix = 0u;
      }
    }
  }
  __syncwarp();
  for (int d = lane; d < kHistBins; d += 32) { c[d] = 0u; mi[d] = 0ull; }
}

// ---- ties at the cut: rank by flat index (count-only radix select) ----
template <int TP>
__global__ void __launch_bounds__(kHistThreads)
k_tie_hist(Prob P, const float* __restrict__ S, SelState* __restrict__ st, uint32_t* __restrict__ hc) {
  __shared__ uint32_t cnt[kHistBins];
  const int h = blockIdx.y;
  if (st[h].state != kSel_Ties) return;
  for (int b = threadIdx.x; b < kHistBins; b += kHistThreads) cnt[b] = 0u;
  __syncthreads();
  const uint32_t cut = st[h].cut_key, prefix = st[h].prefix;
  const size_t pool = (size_t)P.s * P.Nb;
  const float* base = S + (size_t)h * pool;
  const size_t beg = (size_t)blockIdx.x * kHistChunk;
  const size_t end = min(beg + (size_t)kHistChunk, pool);
  auto add = [&](float x, size_t f) {
    if (f2key(x) != cut) return;
    uint32_t dig;
    if (digit_of<TP>((uint32_t)f, prefix, dig)) atomicAdd(&cnt[dig], 1u);
  };
  if ((pool & 3) == 0) {
    // 16-byte loads, as in the mass histogram
    const float4* b4 = reinterpret_cast<const float4*>(base);
    for (size_t f = beg / 4 + threadIdx.x; f < end / 4; f += kHistThreads) {
      const float4 v = __ldg(b4 + f);
      add(v.x, 4 * f);
      add(v.y, 4 * f + 1);
      add(v.z, 4 * f + 2);
      add(v.w, 4 * f + 3);
    }
  } else {
    for (size_t f = beg + threadIdx.x; f < end; f += kHistThreads) add(__ldg(base + f), f);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kHistBins; b += kHistThreads)
    if (cnt[b]) atomicAdd(&hc[h * kHistBins + b], cnt[b]);
}

template <int TP>
__global__ void __launch_bounds__(32)
k_tie_scan(SelState* __restrict__ st, uint32_t* __restrict__ hc) {
  const int h = blockIdx.x, lane = threadIdx.x;
  SelState& S = st[h];
  if (S.state != kSel_Ties) return;
  uint32_t* c = hc + h * kHistBins;
  const int nb = (TP == 2) ? 1024 : 2048;
  const int per = nb / 32;
  unsigned long long lc = 0;
  for (int k = 0; k < per; ++k) lc += c[lane * per + k];       // ascending digits
  unsigned long long incl = lc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned long long take = S.tie_take;
  unsigned ball = __ballot_sync(0xffffffffu, incl >= take);
  const int fl = ball ? (__ffs(ball) - 1) : 31;
  int chosen = -1;
  unsigned long long before = 0;
  if (lane == fl) {
    unsigned long long acc = incl - lc;
    for (int k = 0; k < per; ++k) {
      int d = lane * per + k;
      if (acc + c[d] >= take) { chosen = d; break; }
      acc += c[d];
    }
    if (chosen < 0) chosen = lane * per + per - 1;
    before = acc;
  }
  chosen = __shfl_sync(0xffffffffu, chosen, fl);
  before = __shfl_sync(0xffffffffu, before, fl);
  if (lane == 0) {
    const uint32_t pre = (TP == 0) ? (uint32_t)chosen
                                   : ((S.prefix << (TP == 1 ? 11 : 10)) | (uint32_t)chosen);
    S.prefix = pre;
    S.tie_take = (uint32_t)(take - before);
    if (TP == 2) {
      S.idx_cut = pre;
      S.state = kSel_Resolved;
    }
  }
  __syncwarp();
  for (int d = lane; d < kHistBins; d += 32) c[d] = 0u;
}

// ------------------------------------------------------------------ emit
// One warp per (row, 32-block word): bit j set iff pair (i, j) is selected.
// Vector form of the bitmap pass for N_b a multiple of V (every row starts
// 4 V-byte aligned): lane l holds blocks V l .. V l + V - 1 of each 32 V-block
// span, and 32 / V lanes' V-bit groups make one 32-bit word.
template <int V>
__device__ __forceinline__ void emit_rows_vec(const Prob& P, const float* __restrict__ S,
                                              uint32_t* __restrict__ sel, int h, int warp,
                                              int lane, int state, uint32_t cut, uint32_t idx_cut,
                                              int rows_per_cta) {
  constexpr int kLpw = 32 / V;                        // lanes per bitmap word
  for (int rr = warp; rr < rows_per_cta; rr += 8) {
    const int i = blockIdx.x * rows_per_cta + rr;
    if (i >= P.s) break;
    const float* row = S + ((size_t)h * P.s + i) * P.Nb;
    for (int j0 = 0; j0 < P.Nb; j0 += 32 * V) {
      const int j = j0 + V * lane;
      uint32_t bits = 0u;
      if (j < P.Nb) {
        if (state == kSel_All) {
          bits = (1u << V) - 1u;
        } else {
          float xs[V];
          if constexpr (V == 4) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(row + j));
            xs[0] = v.x;
            xs[1] = v.y;
            xs[2] = v.z;
            xs[3] = v.w;
          } else {
            const float2 v = __ldg(reinterpret_cast<const float2*>(row + j));
            xs[0] = v.x;
            xs[1] = v.y;
          }
#pragma unroll
          for (int e = 0; e < V; ++e) {
            const uint32_t key = f2key(xs[e]);
            const uint32_t idx = (uint32_t)((size_t)i * P.Nb + j + e);
            if (key > cut || (key == cut && idx <= idx_cut)) bits |= 1u << e;
          }
        }
      }
      uint32_t word = bits << (V * (lane & (kLpw - 1)));
#pragma unroll
      for (int o = 1; o < kLpw; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
      const int w = (j0 >> 5) + lane / kLpw;
      if ((lane & (kLpw - 1)) == 0 && w < P.Wb) sel[((size_t)h * P.s + i) * P.Wb + w] = word;
    }
  }
}

__global__ void __launch_bounds__(256)
k_emit(Prob P, const float* __restrict__ S, const SelState* __restrict__ st,
       uint32_t* __restrict__ sel) {
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int state = st[h].state;
  const uint32_t cut = st[h].cut_key, idx_cut = st[h].idx_cut;
  const int rows_per_cta = 8 * 4;
  if ((P.Nb & 1) == 0) {
    if ((P.Nb & 3) == 0)
      emit_rows_vec<4>(P, S, sel, h, warp, lane, state, cut, idx_cut, rows_per_cta);
    else
      emit_rows_vec<2>(P, S, sel, h, warp, lane, state, cut, idx_cut, rows_per_cta);
    return;
  }
  for (int rr = warp; rr < rows_per_cta; rr += 8) {
    const int i = blockIdx.x * rows_per_cta + rr;
    if (i >= P.s) break;
    const float* row = S + ((size_t)h * P.s + i) * P.Nb;
    for (int w = 0; w < P.Wb; ++w) {
      const int j = w * 32 + lane;
      bool on = false;
      if (j < P.Nb) {
        if (state == kSel_All) {
          on = true;
        } else {
          uint32_t key = f2key(__ldg(row + j));
          uint32_t idx = (uint32_t)((size_t)i * P.Nb + j);
          on = key > cut || (key == cut && idx <= idx_cut);
        }
      }
      unsigned bits = __ballot_sync(0xffffffffu, on);
      if (lane == 0) sel[((size_t)h * P.s + i) * P.Wb + w] = bits;
    }
  }
}

// The per-query reading of "normalised similarity" (a selection variant):
// each row of the stored pool becomes its log softmax over the row's N_b
// blocks, S_ij <- S_ij - log sum_j' exp S_ij', in place, and the per-head max
// of the result is recorded.  Ranking the head's pool by this value is
// ranking it by p_ij = softmax_j(S_i.) / s, and exp(S' - max S') is p up to
// one factor per head, so the method's passes below then apply the
// cumulative rule to p unchanged.  One warp per row.
__global__ void __launch_bounds__(256)
k_rownorm(Prob P, float* __restrict__ S, SelState* __restrict__ st) {
  const int lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);   // h * s + i
  if (row >= (size_t)P.n_h * P.s) return;
  const int h = (int)(row / (size_t)P.s);
  float* r = S + row * P.Nb;
  float m = -INFINITY;
  for (int j = lane; j < P.Nb; j += 32) m = fmaxf(m, r[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float z = 0.f;
  for (int j = lane; j < P.Nb; j += 32) z += expf(r[j] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const float lse = m + logf(z);
  float mx = -INFINITY;
  for (int j = lane; j < P.Nb; j += 32) {
    const float v = r[j] - lse;
    r[j] = v;
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) atomicMax(&st[h].max_key, f2key(mx));
}

__global__ void k_stats(Prob P, const SelState* __restrict__ st, vmoba_head_stats* __restrict__ out) {
  const int h = threadIdx.x;
  if (h >= P.n_h) return;
  const SelState S = st[h];
  vmoba_head_stats o;
  o.n_selected = (long long)S.n_selected;
  o.mass = S.Z > 0.0 ? S.mass_selected / S.Z : 0.0;
  o.all_selected = S.state == kSel_All ? 1 : 0;
  o.cut_score = S.state == kSel_All ? -INFINITY : key2f(S.cut_key);
  out[h] = o;
}

template <typename E, int D>
cudaError_t launch_score(const Prob& P, const void* q, const float* B, float scale, float* S,
                         SelState* st, cudaStream_t stream) {
  const size_t smem = sizeof(float) * D * (kQPad + kBPad);
  cudaError_t e = cudaFuncSetAttribute(k_score<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((P.s + kSQ - 1) / kSQ, P.n_h);
  {
    VMOBA_TRACE("k_score", stream);
    k_score<E, D><<<grid, 256, smem, stream>>>(P, static_cast<const E*>(q), B, scale, S, st);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_pool(const Prob& P, const void* q, const float* blocks, float scale,
                              void* ws, const WsLayout& L, int num_sms, cudaStream_t stream) {
  SelState* st = ws_ptr<SelState>(ws, L.sel_state);
  {
    VMOBA_TRACE("k_init", stream);
    k_init<<<64, 256, 0, stream>>>(st, ws_ptr<uint32_t>(ws, L.hist_count),
                                   ws_ptr<unsigned long long>(ws, L.hist_mass), P.n_h);
  }
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  float* S = ws_ptr<float>(ws, L.scores);
  if (P.dtype == VMOBA_BF16)
    return launch_score_pool_tc(P, q, blocks, scale, ws_ptr<void>(ws, L.bsplit), S, st,
                                ws_ptr<int>(ws, L.status), num_sms, stream);
  e = (P.d == 128) ? launch_score<float, 128>(P, q, blocks, scale, S, st, stream)
                   : launch_score<float, 64>(P, q, blocks, scale, S, st, stream);
  count_launches(1);
  return e;
}

cudaError_t launch_score_select(const Prob& P, const void* q, const float* blocks, float tau,
                                float scale, uint32_t* sel, vmoba_head_stats* stats, void* ws,
                                const WsLayout& L, int num_sms, cudaStream_t stream,
                                int by_count, double kcount, bool rownorm) {
  SelState* st = ws_ptr<SelState>(ws, L.sel_state);
  uint32_t* hc = ws_ptr<uint32_t>(ws, L.hist_count);
  unsigned long long* hm = ws_ptr<unsigned long long>(ws, L.hist_mass);
  // global fixed-point scale of the bucket masses (see kMassBitsCta)
  const size_t pool_elems = (size_t)P.s * P.Nb;
  const int lg = pool_elems <= 1 ? 0 : 64 - __builtin_clzll((unsigned long long)(pool_elems - 1));
  const int fbits = std::min(kMassBitsCta, 63 - lg);
  const int shift = kMassBitsCta - fbits;
  const double qinv = std::ldexp(1.0, -fbits);

  {
    VMOBA_TRACE("k_init", stream);
    k_init<<<64, 256, 0, stream>>>(st, hc, hm, P.n_h);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int launches = 1;
  auto scan = [&](int pass, cudaStream_t s) -> cudaError_t {
    VMOBA_TRACE("k_scan", s);
    if (pass == 0) k_scan<0><<<P.n_h, 32, 0, s>>>(P, st, hc, hm, qinv, tau, by_count, kcount);
    if (pass == 1) k_scan<1><<<P.n_h, 32, 0, s>>>(P, st, hc, hm, qinv, tau, by_count, kcount);
    if (pass == 2) k_scan<2><<<P.n_h, 32, 0, s>>>(P, st, hc, hm, qinv, tau, by_count, kcount);
    ++launches;
    return cudaGetLastError();
  };
  auto tie_scan = [&](int pass, cudaStream_t s) -> cudaError_t {
    VMOBA_TRACE("k_tie_scan", s);
    if (pass == 0) k_tie_scan<0><<<P.n_h, 32, 0, s>>>(st, hc);
    if (pass == 1) k_tie_scan<1><<<P.n_h, 32, 0, s>>>(st, hc);
    if (pass == 2) k_tie_scan<2><<<P.n_h, 32, 0, s>>>(st, hc);
    ++launches;
    return cudaGetLastError();
  };

  if (P.dtype == VMOBA_BF16) {
    // the tensor cores write the pool (and each head's max) once; the radix
    // passes below read it with many CTAs per SM, whose shared-memory
    // histogram atomics hide each other's latency
    e = launch_score_pool_tc(P, q, blocks, scale, ws_ptr<void>(ws, L.bsplit),
                             ws_ptr<float>(ws, L.scores), st, ws_ptr<int>(ws, L.status), num_sms,
                             stream);
    if (e != cudaSuccess) return e;
  }
  {
    // fp32 I/O: the pool is computed once with fp32 FMAs and read by each
    // pass (bf16 with the per-query normalisation: written above)
    float* S = ws_ptr<float>(ws, L.scores);
    if (P.dtype != VMOBA_BF16) {
      e = (P.d == 128) ? launch_score<float, 128>(P, q, blocks, scale, S, st, stream)
                       : launch_score<float, 64>(P, q, blocks, scale, S, st, stream);
      if (e != cudaSuccess) return e;
      ++launches;
    }
    if (rownorm) {
      // the max of the normalised pool replaces the raw one
      {
        VMOBA_TRACE("k_init", stream);
        k_init<<<64, 256, 0, stream>>>(st, hc, hm, P.n_h);
      }
      ++launches;
      VMOBA_TRACE("k_rownorm", stream);
      k_rownorm<<<(unsigned)(((size_t)P.n_h * P.s + 7) / 8), 256, 0, stream>>>(P, S, st);
      ++launches;
    }
    const size_t pool = (size_t)P.s * P.Nb;
    dim3 hgrid((unsigned)((pool + kHistChunk - 1) / kHistChunk), P.n_h);
    for (int pass = 0; pass < 3; ++pass) {
      {
        VMOBA_TRACE("k_hist", stream);
        if (pass == 0) k_hist<0><<<hgrid, kHistThreads, 0, stream>>>(P, S, st, hc, hm, shift);
        if (pass == 1) k_hist<1><<<hgrid, kHistThreads, 0, stream>>>(P, S, st, hc, hm, shift);
        if (pass == 2) k_hist<2><<<hgrid, kHistThreads, 0, stream>>>(P, S, st, hc, hm, shift);
      }
      ++launches;
      if ((e = scan(pass, stream)) != cudaSuccess) return e;
    }
    for (int pass = 0; pass < 3; ++pass) {
      {
        VMOBA_TRACE("k_tie_hist", stream);
        if (pass == 0) k_tie_hist<0><<<hgrid, kHistThreads, 0, stream>>>(P, S, st, hc);
        if (pass == 1) k_tie_hist<1><<<hgrid, kHistThreads, 0, stream>>>(P, S, st, hc);
        if (pass == 2) k_tie_hist<2><<<hgrid, kHistThreads, 0, stream>>>(P, S, st, hc);
      }
      ++launches;
      if ((e = tie_scan(pass, stream)) != cudaSuccess) return e;
    }
    dim3 egrid((P.s + 31) / 32, P.n_h);
    {
      VMOBA_TRACE("k_emit", stream);
      k_emit<<<egrid, 256, 0, stream>>>(P, S, st, sel);
    }
    ++launches;
  }
  {
    VMOBA_TRACE("k_stats", stream);
    k_stats<<<1, 128, 0, stream>>>(P, st, stats);
  }
  ++launches;
  count_launches(launches);
  return cudaGetLastError();
}

}  // namespace vmoba
