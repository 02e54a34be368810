// Sparse attention forward/backward over the selected (query, block) pairs,
// fp32 CUDA-core (FMA) kernels.  They serve fp32 I/O, whose tolerance
// (1e-4 against fp64) rules out TF32 tensor-core math, and head_dim 64.
//
// Definition (VMoBA notes, overall framework: attention only on the
// selected blocks, output of full-attention shape): for query i,
// LSE_i = log sum_{n : block(n) selected for i} exp(scale q_i.k_n) and
// O_i the softmax-weighted sum of v_n; rows with nothing selected give
// O = 0, LSE = -inf.  Backward holds the mask constant:
// D_i = dO_i.O_i, dS = P (dP - D), dQ = scale dS K, dK = scale dS^T Q,
// dV = P^T dO.
//
// Layout: a 128-row query tile in partition order, TPR = head_dim/32
// threads per row, each owning 32 consecutive columns; dot products reduce
// over the TPR lanes with shuffles.  Key tiles come from the plan
// (qt_kt_bits); keys are staged through shared memory 32 at a time with a
// padded row layout (33 floats per 32-column segment).
#include "common.cuh"

namespace vmoba {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kChunk = 32;    // keys (fwd, dq) or query rows (dkdv) staged per step

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename E> __device__ __forceinline__ E from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

template <int TPR>
__device__ __forceinline__ float row_sum(float v) {
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ bool sel_bit(const uint32_t* words, int j) {
  return (words[j >> 5] >> (j & 31)) & 1u;
}

template <int D>
struct Seg {  // padded shared-memory row: TPR segments of 33 floats
  static constexpr int TPR = D / 32;
  static constexpr int ROW = TPR * 33;
  __device__ static int at(int row, int part, int x) { return row * ROW + part * 33 + x; }
};

// Stage rows [p0, p0+kChunk) of a [n_h][s][D] tensor (partition order) as fp32.
template <typename E, int D>
__device__ void stage_perm_rows(const Prob& P, const E* __restrict__ src, int h, int p0,
                                float* dst) {
  for (int idx = threadIdx.x; idx < kChunk * D; idx += blockDim.x) {
    int r = idx / D, c = idx - r * D;
    int p = p0 + r;
    float v = (p < P.s) ? to_f(src[((size_t)h * P.s + p) * D + c]) : 0.f;
    dst[Seg<D>::at(r, c >> 5, c & 31)] = v;
  }
}

// Stage query rows of partition positions [p0, p0+kChunk) from a [s][n_h][D]
// tensor in original order.
template <typename E, int D>
__device__ void stage_orig_rows(const Prob& P, const E* __restrict__ src, int h, int p0,
                                float* dst) {
  for (int idx = threadIdx.x; idx < kChunk * D; idx += blockDim.x) {
    int r = idx / D, c = idx - r * D;
    int p = p0 + r;
    float v = 0.f;
    if (p < P.s) v = to_f(src[((size_t)perm_token(P, p) * P.n_h + h) * D + c]);
    dst[Seg<D>::at(r, c >> 5, c & 31)] = v;
  }
}

// ------------------------------------------------------------------ fwd
template <typename E, int D>
__global__ void __launch_bounds__(kTile * (D / 32))
k_fwd_simt(Prob P, const E* __restrict__ q, const E* __restrict__ kp, const E* __restrict__ vp,
           const uint32_t* __restrict__ sel, const uint32_t* __restrict__ qt_kt, float scale,
           E* __restrict__ out, float* __restrict__ o32, float* __restrict__ lse) {
  constexpr int TPR = D / 32;
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Vs = Ks + kChunk * Seg<D>::ROW;
  int* kblk = reinterpret_cast<int*>(Vs + kChunk * Seg<D>::ROW);
  uint32_t* srow = reinterpret_cast<uint32_t*>(kblk + kChunk);   // [kTile][Wb]

  const int t = blockIdx.x, h = blockIdx.y;
  const int r = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int p = t * kTile + r;
  const bool valid = p < P.s;
  const int i = valid ? perm_token(P, p) : 0;
  const float sl2 = scale * kLog2e;

  float qv[32], o[32];
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    qv[x] = valid ? to_f(q[((size_t)i * P.n_h + h) * D + part * 32 + x]) * sl2 : 0.f;
    o[x] = 0.f;
  }
  for (int idx = threadIdx.x; idx < kTile * P.Wb; idx += blockDim.x) {
    int rr = idx / P.Wb, w = idx - rr * P.Wb;
    int pp = t * kTile + rr;
    srow[idx] = (pp < P.s) ? sel[((size_t)h * P.s + perm_token(P, pp)) * P.Wb + w] : 0u;
  }
  float m = -INFINITY, l = 0.f;
  const uint32_t* tiles = qt_kt + ((size_t)h * P.n_qt + t) * P.Wqt;
  for (int w = 0; w < P.Wqt; ++w) {
    uint32_t bits = tiles[w];
    while (bits) {
      const int kt = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1;
      for (int kc = 0; kc < kTile; kc += kChunk) {
        const int k0 = kt * kTile + kc;
        __syncthreads();
        stage_perm_rows<E, D>(P, kp, h, k0, Ks);
        stage_perm_rows<E, D>(P, vp, h, k0, Vs);
        for (int c = threadIdx.x; c < kChunk; c += blockDim.x)
          kblk[c] = (k0 + c < P.s) ? (k0 + c) / P.L : -1;
        __syncthreads();
        float sc[kChunk];
        float cmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < kChunk; ++c) {
          float a = 0.f;
#pragma unroll
          for (int x = 0; x < 32; ++x) a = fmaf(qv[x], Ks[Seg<D>::at(c, part, x)], a);
          a = row_sum<TPR>(a);
          const int j = kblk[c];
          const bool ok = valid && j >= 0 && sel_bit(srow + r * P.Wb, j);
          sc[c] = ok ? a : -INFINITY;
          cmax = fmaxf(cmax, sc[c]);
        }
        if (cmax > -INFINITY) {
          const float mn = fmaxf(m, cmax);
          const float corr = exp2f(m - mn);
          l *= corr;
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] *= corr;
          m = mn;
#pragma unroll
          for (int c = 0; c < kChunk; ++c) {
            const float pe = exp2f(sc[c] - m);
            l += pe;
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = fmaf(pe, Vs[Seg<D>::at(c, part, x)], o[x]);
          }
        }
      }
    }
  }
  if (!valid) return;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  E* orow = out + ((size_t)i * P.n_h + h) * D + part * 32;
  float* frow = o32 + ((size_t)i * P.n_h + h) * D + part * 32;
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    orow[x] = from_f<E>(o[x] * inv);
    frow[x] = o[x] * inv;
  }
  if (part == 0) lse[(size_t)h * P.s + i] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
}

// ------------------------------------------------------------- bwd: D_i
// D_i = dO_i . O_i with the forward's fp32 output (the stored bf16 output
// would put its rounding, 2^-9 relative, into every dS of the row).
template <typename E, int D>
__global__ void k_bwd_rowdot(Prob P, const float* __restrict__ o, const E* __restrict__ dout,
                             float* __restrict__ rowD) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= P.s * P.n_h) return;
  const int i = warp / P.n_h, h = warp - i * P.n_h;
  const float* a = o + (size_t)warp * D;
  const E* b = dout + (size_t)warp * D;
  float acc = 0.f;
  for (int x = lane; x < D; x += 32) acc = fmaf(a[x], to_f(b[x]), acc);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) rowD[(size_t)h * P.s + i] = acc;
}

// ---------------------------------------------------- bwd: dQ (by query)
template <typename E, int D>
__global__ void __launch_bounds__(kTile * (D / 32))
k_bwd_dq_simt(Prob P, const E* __restrict__ q, const E* __restrict__ kp,
              const E* __restrict__ vp, const uint32_t* __restrict__ sel,
              const uint32_t* __restrict__ qt_kt, float scale, const float* __restrict__ lse,
              const E* __restrict__ dout, const float* __restrict__ rowD, E* __restrict__ dq) {
  constexpr int TPR = D / 32;
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;
  float* Vs = Ks + kChunk * Seg<D>::ROW;
  int* kblk = reinterpret_cast<int*>(Vs + kChunk * Seg<D>::ROW);
  uint32_t* srow = reinterpret_cast<uint32_t*>(kblk + kChunk);

  const int t = blockIdx.x, h = blockIdx.y;
  const int r = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int p = t * kTile + r;
  const bool valid = p < P.s;
  const int i = valid ? perm_token(P, p) : 0;
  const float sl2 = scale * kLog2e;
  float qv[32], dov[32], g[32];
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    const size_t off = ((size_t)i * P.n_h + h) * D + part * 32 + x;
    qv[x] = valid ? to_f(q[off]) * sl2 : 0.f;
    dov[x] = valid ? to_f(dout[off]) : 0.f;
    g[x] = 0.f;
  }
  const float lse2 = valid ? lse[(size_t)h * P.s + i] * kLog2e : -INFINITY;
  const float Di = valid ? rowD[(size_t)h * P.s + i] : 0.f;
  for (int idx = threadIdx.x; idx < kTile * P.Wb; idx += blockDim.x) {
    int rr = idx / P.Wb, w = idx - rr * P.Wb;
    int pp = t * kTile + rr;
    srow[idx] = (pp < P.s) ? sel[((size_t)h * P.s + perm_token(P, pp)) * P.Wb + w] : 0u;
  }
  const uint32_t* tiles = qt_kt + ((size_t)h * P.n_qt + t) * P.Wqt;
  for (int w = 0; w < P.Wqt; ++w) {
    uint32_t bits = tiles[w];
    while (bits) {
      const int kt = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1;
      for (int kc = 0; kc < kTile; kc += kChunk) {
        const int k0 = kt * kTile + kc;
        __syncthreads();
        stage_perm_rows<E, D>(P, kp, h, k0, Ks);
        stage_perm_rows<E, D>(P, vp, h, k0, Vs);
        for (int c = threadIdx.x; c < kChunk; c += blockDim.x)
          kblk[c] = (k0 + c < P.s) ? (k0 + c) / P.L : -1;
        __syncthreads();
#pragma unroll 4
        for (int c = 0; c < kChunk; ++c) {
          float a = 0.f, dp = 0.f;
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            a = fmaf(qv[x], Ks[Seg<D>::at(c, part, x)], a);
            dp = fmaf(dov[x], Vs[Seg<D>::at(c, part, x)], dp);
          }
          a = row_sum<TPR>(a);
          dp = row_sum<TPR>(dp);
          const int j = kblk[c];
          const bool ok = valid && j >= 0 && sel_bit(srow + r * P.Wb, j);
          const float pr = ok ? exp2f(a - lse2) : 0.f;
          const float ds = pr * (dp - Di);
#pragma unroll
          for (int x = 0; x < 32; ++x) g[x] = fmaf(ds, Ks[Seg<D>::at(c, part, x)], g[x]);
        }
      }
    }
  }
  if (!valid) return;
  E* row = dq + ((size_t)i * P.n_h + h) * D + part * 32;
#pragma unroll
  for (int x = 0; x < 32; ++x) row[x] = from_f<E>(g[x] * scale);
}

// ------------------------------------------------- bwd: dK, dV (by key)
// KR keys per CTA (KR * D/32 threads) keep the four 32-float accumulators in
// registers: 64 keys at head_dim 128, 128 keys at head_dim 64.
template <typename E, int D, int KR>
__global__ void __launch_bounds__(KR * (D / 32))
k_bwd_dkdv_simt(Prob P, const E* __restrict__ q, const E* __restrict__ kp,
                const E* __restrict__ vp, const uint32_t* __restrict__ sel,
                const uint32_t* __restrict__ kt_qt, float scale, const float* __restrict__ lse,
                const E* __restrict__ dout, const float* __restrict__ rowD, E* __restrict__ dk,
                E* __restrict__ dv) {
  constexpr int TPR = D / 32;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* Os = Qs + kChunk * Seg<D>::ROW;             // dO rows
  float* l2s = Os + kChunk * Seg<D>::ROW;
  float* Ds = l2s + kChunk;
  uint32_t* srow = reinterpret_cast<uint32_t*>(Ds + kChunk);   // [kChunk][Wb]

  const int h = blockIdx.y;
  const int kt = (blockIdx.x * KR) / kTile;
  const int c = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int pk = blockIdx.x * KR + c;
  const bool kvalid = pk < P.s;
  const int blk = kvalid ? pk / P.L : 0;
  const float sl2 = scale * kLog2e;
  float kv[32], vv[32], gk[32], gv[32];
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    const size_t off = ((size_t)h * P.s + (kvalid ? pk : 0)) * D + part * 32 + x;
    kv[x] = kvalid ? to_f(kp[off]) * sl2 : 0.f;
    vv[x] = kvalid ? to_f(vp[off]) : 0.f;
    gk[x] = 0.f;
    gv[x] = 0.f;
  }
  const uint32_t* qts = kt_qt + ((size_t)h * P.n_qt + kt) * P.Wqt;
  for (int w = 0; w < P.Wqt; ++w) {
    uint32_t bits = qts[w];
    while (bits) {
      const int qt = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1;
      for (int rc = 0; rc < kTile; rc += kChunk) {
        const int p0 = qt * kTile + rc;
        __syncthreads();
        stage_orig_rows<E, D>(P, q, h, p0, Qs);
        stage_orig_rows<E, D>(P, dout, h, p0, Os);
        for (int rr = threadIdx.x; rr < kChunk; rr += blockDim.x) {
          const int pp = p0 + rr;
          const int ii = pp < P.s ? perm_token(P, pp) : 0;
          l2s[rr] = pp < P.s ? lse[(size_t)h * P.s + ii] * kLog2e : -INFINITY;
          Ds[rr] = pp < P.s ? rowD[(size_t)h * P.s + ii] : 0.f;
        }
        for (int idx = threadIdx.x; idx < kChunk * P.Wb; idx += blockDim.x) {
          int rr = idx / P.Wb, ww = idx - rr * P.Wb;
          int pp = p0 + rr;
          srow[idx] = (pp < P.s) ? sel[((size_t)h * P.s + perm_token(P, pp)) * P.Wb + ww] : 0u;
        }
        __syncthreads();
#pragma unroll 4
        for (int rr = 0; rr < kChunk; ++rr) {
          float a = 0.f, dp = 0.f;
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            a = fmaf(kv[x], Qs[Seg<D>::at(rr, part, x)], a);
            dp = fmaf(vv[x], Os[Seg<D>::at(rr, part, x)], dp);
          }
          a = row_sum<TPR>(a);
          dp = row_sum<TPR>(dp);
          const bool ok = kvalid && sel_bit(srow + rr * P.Wb, blk);
          const float pr = ok ? exp2f(a - l2s[rr]) : 0.f;
          const float ds = pr * (dp - Ds[rr]);
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            gv[x] = fmaf(pr, Os[Seg<D>::at(rr, part, x)], gv[x]);
            gk[x] = fmaf(ds, Qs[Seg<D>::at(rr, part, x)], gk[x]);
          }
        }
      }
    }
  }
  if (!kvalid) return;
  const int n = perm_token(P, pk);
  E* rk = dk + ((size_t)n * P.n_h + h) * D + part * 32;
  E* rv = dv + ((size_t)n * P.n_h + h) * D + part * 32;
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    rk[x] = from_f<E>(gk[x] * scale);
    rv[x] = from_f<E>(gv[x]);
  }
}

template <int D>
size_t fwd_smem(const Prob& P) {
  return sizeof(float) * 2 * kChunk * Seg<D>::ROW + sizeof(int) * kChunk +
         sizeof(uint32_t) * kTile * P.Wb;
}
template <int D>
size_t dkdv_smem(const Prob& P) {
  return sizeof(float) * (2 * kChunk * Seg<D>::ROW + 2 * kChunk) +
         sizeof(uint32_t) * kChunk * P.Wb;
}

template <typename E, int D>
cudaError_t fwd_t(const Prob& P, const void* q, const void* kp, const void* vp,
                  const uint32_t* sel, const uint32_t* qt_kt, float scale, void* out, float* o32,
                  float* lse, cudaStream_t st) {
  const size_t smem = fwd_smem<D>(P);
  cudaError_t e = cudaFuncSetAttribute(k_fwd_simt<E, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(P.n_qt, P.n_h);
  {
    VMOBA_TRACE("k_fwd_simt", st);
    k_fwd_simt<E, D><<<grid, kTile * (D / 32), smem, st>>>(
        P, static_cast<const E*>(q), static_cast<const E*>(kp), static_cast<const E*>(vp), sel,
        qt_kt, scale, static_cast<E*>(out), o32, lse);
  }
  count_launches(1);
  return cudaGetLastError();
}

template <typename E, int D>
cudaError_t bwd_t(const Prob& P, const void* q, const void* kp, const void* vp,
                  const uint32_t* sel, const uint32_t* qt_kt, const uint32_t* kt_qt, float scale,
                  const float* o32, const float* lse, const void* dout, void* dq, void* dk,
                  void* dv, float* rowD, cudaStream_t st) {
  const int warps = P.s * P.n_h;
  {
    VMOBA_TRACE("k_bwd_rowdot", st);
    k_bwd_rowdot<E, D><<<(warps + 7) / 8, 256, 0, st>>>(P, o32, static_cast<const E*>(dout),
                                                         rowD);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t s1 = fwd_smem<D>(P);
  e = cudaFuncSetAttribute(k_bwd_dq_simt<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)s1);
  if (e != cudaSuccess) return e;
  dim3 grid(P.n_qt, P.n_h);
  {
    VMOBA_TRACE("k_bwd_dq_simt", st);
    k_bwd_dq_simt<E, D><<<grid, kTile * (D / 32), s1, st>>>(
        P, static_cast<const E*>(q), static_cast<const E*>(kp), static_cast<const E*>(vp), sel,
        qt_kt, scale, lse, static_cast<const E*>(dout), rowD, static_cast<E*>(dq));
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  constexpr int KR = D == 128 ? 64 : 128;
  const size_t s2 = dkdv_smem<D>(P);
  e = cudaFuncSetAttribute(k_bwd_dkdv_simt<E, D, KR>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
  if (e != cudaSuccess) return e;
  dim3 kgrid(P.n_qt * (kTile / KR), P.n_h);
  {
    VMOBA_TRACE("k_bwd_dkdv_simt", st);
    k_bwd_dkdv_simt<E, D, KR><<<kgrid, KR * (D / 32), s2, st>>>(
        P, static_cast<const E*>(q), static_cast<const E*>(kp), static_cast<const E*>(vp), sel,
        kt_qt, scale, lse, static_cast<const E*>(dout), rowD, static_cast<E*>(dk),
        static_cast<E*>(dv));
  }
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_simt(const Prob& P, const void* q, const void* kp, const void* vp,
                                 const uint32_t* sel, void* ws, const WsLayout& L, float scale,
                                 void* out, float* lse, cudaStream_t st) {
  const uint32_t* qt_kt = ws_ptr<uint32_t>(ws, L.qt_kt_bits);
  float* o32 = ws_ptr<float>(ws, L.o32);
  if (P.dtype == VMOBA_BF16)
    return P.d == 128
               ? fwd_t<__nv_bfloat16, 128>(P, q, kp, vp, sel, qt_kt, scale, out, o32, lse, st)
               : fwd_t<__nv_bfloat16, 64>(P, q, kp, vp, sel, qt_kt, scale, out, o32, lse, st);
  return P.d == 128 ? fwd_t<float, 128>(P, q, kp, vp, sel, qt_kt, scale, out, o32, lse, st)
                    : fwd_t<float, 64>(P, q, kp, vp, sel, qt_kt, scale, out, o32, lse, st);
}

cudaError_t launch_attn_bwd_simt(const Prob& P, const void* q, const void* kp, const void* vp,
                                 const uint32_t* sel, void* ws, const WsLayout& L, float scale,
                                 const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                 float* rowD, cudaStream_t st) {
  const uint32_t* qt_kt = ws_ptr<uint32_t>(ws, L.qt_kt_bits);
  const uint32_t* kt_qt = ws_ptr<uint32_t>(ws, L.kt_qt_bits);
  const float* o32 = ws_ptr<float>(ws, L.o32);
  if (P.dtype == VMOBA_BF16)
    return P.d == 128 ? bwd_t<__nv_bfloat16, 128>(P, q, kp, vp, sel, qt_kt, kt_qt, scale, o32,
                                                  lse, dout, dq, dk, dv, rowD, st)
                      : bwd_t<__nv_bfloat16, 64>(P, q, kp, vp, sel, qt_kt, kt_qt, scale, o32,
                                                 lse, dout, dq, dk, dv, rowD, st);
  return P.d == 128 ? bwd_t<float, 128>(P, q, kp, vp, sel, qt_kt, kt_qt, scale, o32, lse, dout,
                                        dq, dk, dv, rowD, st)
                    : bwd_t<float, 64>(P, q, kp, vp, sel, qt_kt, kt_qt, scale, o32, lse, dout,
                                       dq, dk, dv, rowD, st);
}

}  // namespace vmoba
