// Step 1 of the layer: key/value rearrange for the layer's partition mode and
// the mean-pool of every key block (VMoBA notes, key design 1:
// "rearrange K in (T H W), then B = mean(K')").
//
// One CTA per (block j, head h).  Each warp moves whole token rows (d
// elements, 16-byte vectors, 16/32 lanes per row so two rows move per warp
// instruction at d*elem = 256 B) from the [s][n_h][d] inputs to the
// block-contiguous [n_h][s][d] outputs and accumulates the key row into fp64
// per-lane column sums; a shared-memory pass reduces the warps.  HBM bound:
// 2 reads + 2 writes of d*elem bytes per token and head.
#include "common.cuh"

namespace vmoba {
namespace {

template <typename E>
struct Vec16;  // 16 bytes of E as an array of floats
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void to_f(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void to_f(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

constexpr int kWarps = 8;

template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32)
k_partition_pool(Prob P, const E* __restrict__ k, const E* __restrict__ v,
                 E* __restrict__ kp, E* __restrict__ vp, float* __restrict__ blocks) {
  constexpr int CH = D * sizeof(E) / 16;         // 16-byte chunks per row
  static_assert(CH >= 1 && CH <= 32 && 32 % CH == 0, "row must be 16..512 bytes");
  constexpr int RPW = 32 / CH;                   // rows per warp instruction
  constexpr int NV = Vec16<E>::N;                // columns per chunk
  __shared__ double red[kWarps * RPW][D];

  const int j = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / CH, ch = lane % CH;
  const int p0 = j * P.L;

  double acc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) acc[i] = 0.0;

  const size_t in_row = (size_t)P.n_h * D;       // elements between tokens in k/v
  for (int r = warp * RPW + sub; r < P.L; r += kWarps * RPW) {
    const int p = p0 + r;
    const int n = perm_token(P, p);
    const uint4* ks = reinterpret_cast<const uint4*>(k + (size_t)n * in_row + (size_t)h * D) + ch;
    const uint4* vs = reinterpret_cast<const uint4*>(v + (size_t)n * in_row + (size_t)h * D) + ch;
    uint4 kv = __ldg(ks);
    uint4 vv = __ldg(vs);
    uint4* kd = reinterpret_cast<uint4*>(kp + ((size_t)h * P.s + p) * D) + ch;
    uint4* vd = reinterpret_cast<uint4*>(vp + ((size_t)h * P.s + p) * D) + ch;
    *kd = kv;
    *vd = vv;
    float f[NV];
    Vec16<E>::to_f(kv, f);
#pragma unroll
    for (int i = 0; i < NV; ++i) acc[i] += (double)f[i];
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) red[warp * RPW + sub][ch * NV + i] = acc[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    double sum = 0.0;
#pragma unroll 4
    for (int w = 0; w < kWarps * RPW; ++w) sum += red[w][c];
    blocks[((size_t)h * P.Nb + j) * D + c] = (float)(sum / (double)P.L);
  }
}

template <typename E, int D>
cudaError_t launch_t(const Prob& P, const void* k, const void* v, void* kp, void* vp,
                     float* blocks, cudaStream_t st) {
  dim3 grid(P.Nb, P.n_h);
  {
    VMOBA_TRACE("k_partition_pool", st);
    k_partition_pool<E, D><<<grid, kWarps * 32, 0, st>>>(
        P, static_cast<const E*>(k), static_cast<const E*>(v), static_cast<E*>(kp),
        static_cast<E*>(vp), blocks);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_partition(const Prob& P, const void* k, const void* v, void* kp, void* vp,
                             float* blocks, cudaStream_t st) {
  if (P.dtype == VMOBA_BF16) {
    if (P.d == 128) return launch_t<__nv_bfloat16, 128>(P, k, v, kp, vp, blocks, st);
    if (P.d == 64) return launch_t<__nv_bfloat16, 64>(P, k, v, kp, vp, blocks, st);
  } else {
    if (P.d == 128) return launch_t<float, 128>(P, k, v, kp, vp, blocks, st);
    if (P.d == 64) return launch_t<float, 64>(P, k, v, kp, vp, blocks, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vmoba
