// Grouped SIMT GEMM for the Newton-Schulz iteration: fp32 FMA accumulation,
// operands stored as fp32 (MUON_GEMM_FP32) or bf16 (MUON_GEMM_BF16_SIMT).
//
// Newton-Schulz step ("源码实现", zeropower_via_newtonschulz5):
//   A = X X^T (GK_GRAM), B = b A + c A^2 (GK_SQR), X' = a X + B X (GK_UPD).
#include "kernels.h"

namespace am {

AM_CHECK_READER(read_and_clear_check_gemm_simt)

namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ int find_group(const GemmLaunch& L, int tile) {
  int g = 0;
  while (g + 1 < L.num_groups && L.g[g + 1].tile_begin <= tile) ++g;
  return g;
}

template <typename T>
__global__ void __launch_bounds__(NT) k_gemm_simt(const GemmLaunch L) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int gi = find_group(L, blockIdx.x);
  const GemmGroup& g = L.g[gi];
  int t = blockIdx.x - g.tile_begin;
  const int b = t / g.tiles_per_mat;
  t -= b * g.tiles_per_mat;
  const int tm = t / g.tiles_n, tn = t % g.tiles_n;
  const int m0 = tm * BM, n0 = tn * BN;
  const T* A = reinterpret_cast<const T*>(g.A) + (int64_t)b * g.sa;
  const T* B = reinterpret_cast<const T*>(g.B) + (int64_t)b * g.sb;
  const bool b_nt = g.kind != GK_UPD;      // GRAM / SQR: B stored N x K
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += BK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int idx = tid + r * NT;
      {  // A tile: (m, k) at A[m * lda + k]
        const int mm = idx / BK, kk = idx % BK;
        const int gm = m0 + mm, gk = k0 + kk;
        As[kk][mm] = (gm < g.M && gk < g.K && AM_IN((int64_t)b * g.sa + (int64_t)gm * g.lda + gk, 1, (int64_t)g.count * g.sa))
                         ? to_f(A[(int64_t)gm * g.lda + gk]) : 0.f;
      }
      if (b_nt) {  // (k, n) at B[n * ldb + k]
        const int nn = idx / BK, kk = idx % BK;
        const int gn = n0 + nn, gk = k0 + kk;
        Bs[kk][nn] = (gn < g.N && gk < g.K && AM_IN((int64_t)b * g.sb + (int64_t)gn * g.ldb + gk, 1, (int64_t)g.count * g.sb))
                         ? to_f(B[(int64_t)gn * g.ldb + gk]) : 0.f;
      } else {     // (k, n) at B[k * ldb + n]
        const int kk = idx / BN, nn = idx % BN;
        const int gn = n0 + nn, gk = k0 + kk;
        Bs[kk][nn] = (gn < g.N && gk < g.K && AM_IN((int64_t)b * g.sb + (int64_t)gk * g.ldb + gn, 1, (int64_t)g.count * g.sb))
                         ? to_f(B[(int64_t)gk * g.ldb + gn]) : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
  float alpha = g.alpha0, beta = g.beta0;
  if (g.rho) {
    const float r = g.rho[b];
    for (int p = 0; p < g.pa; ++p) alpha *= r;
    for (int p = 0; p < g.pb; ++p) beta *= r;
  }
  T* C = reinterpret_cast<T*>(g.C) + (int64_t)b * g.sc;
  const T* E = g.E ? reinterpret_cast<const T*>(g.E) + (int64_t)b * g.se : nullptr;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty + 16 * i;
    if (gm >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx + 16 * j;
      if (gn >= g.N) continue;
      float v = alpha * acc[i][j];
      if (E && AM_IN((int64_t)b * g.se + (int64_t)gm * g.lde + gn, 1, (int64_t)g.count * g.se))
        v += beta * to_f(E[(int64_t)gm * g.lde + gn]);
      if (AM_IN((int64_t)b * g.sc + (int64_t)gm * g.ldc + gn, 1, (int64_t)g.count * g.sc))
        C[(int64_t)gm * g.ldc + gn] = from_f<T>(v);
    }
  }
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmLaunch& L, cudaStream_t st) {
  if (L.total_tiles == 0) return cudaSuccess;
  if (L.dtype == kBF16) k_gemm_simt<__nv_bfloat16><<<L.total_tiles, NT, 0, st>>>(L);
  else k_gemm_simt<float><<<L.total_tiles, NT, 0, st>>>(L);
  return cudaGetLastError();
}

}  // namespace am
