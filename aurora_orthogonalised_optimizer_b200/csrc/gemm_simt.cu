// Grouped SIMT GEMM for the Newton-Schulz iteration: fp32 FMA accumulation,
// operands stored as fp32 (MUON_GEMM_FP32) or bf16 (MUON_GEMM_BF16_SIMT).
//
// Newton-Schulz step ("源码实现", zeropower_via_newtonschulz5 of the Track 3
// Aurora write-up): A = X X^T (GK_GRAM), B = b A + c A^2 (GK_SQR),
// X' = a X + B X (GK_UPD).
//
// A block computes a 128 x 128 tile with 256 threads.  Thread (ty, tx) of the
// 16 x 16 grid owns the 8 x 8 outputs at rows {0, 64} + 4 ty + {0..3} and
// columns {0, 64} + 4 tx + {0..3} of the tile, so each step of k reads its
// operands from shared memory as four float4 (two of them broadcast across
// the warp).  K advances 8 at a time through two shared-memory buffers: the
// next 8-deep slices of the two operands are loaded into registers (four
// consecutive elements per thread and operand, one vector load where the row
// allows it) while the current slices are multiplied.  The symmetric kinds
// (X X^T, A A) run only the tiles on or above the diagonal and store each
// element of the upper triangle at (m, n) and at (n, m), so the stored
// product is exactly symmetric.
#include "kernels.h"

namespace am {

AM_CHECK_READER(read_and_clear_check_gemm_simt)

namespace {

constexpr int TT = kSimtTile;       // tile edge (rows and columns)
constexpr int TK = 8;               // k per shared-memory slice
constexpr int NT = 256;
constexpr int LDS = TT + 4;         // padded slice row (floats)

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Four consecutive elements at p as fp32 (p 16-byte aligned for fp32,
// 8-byte aligned for bf16).
__device__ __forceinline__ float4 ld4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                     __uint_as_float(v.y & 0xFFFF0000u));
}

__device__ __forceinline__ int find_group(const GemmLaunch& L, int tile) {
  int g = 0;
  while (g + 1 < L.num_groups && L.g[g + 1].tile_begin <= tile) ++g;
  return g;
}

// Tile t of the upper triangle of a T x T grid of tiles, row by row.
__device__ __forceinline__ void tri_tile(int t, int T, int& tm, int& tn) {
  int r = 0;
  while (t >= T - r) {
    t -= T - r;
    ++r;
  }
  tm = r;
  tn = r + t;
}

// Four consecutive elements of an operand row at p, the first in column c
// of `cols`; zeros past the row's end or when the row is outside the matrix.
// `vec`: the quad is aligned for one vector load.  `base`, `ext`: the
// group's batched tensor, for the checked build's index test.
template <typename T>
__device__ __forceinline__ float4 ld_quad(const T* p, bool row_ok, int c, int cols, bool vec, const T* base,
                                          int64_t ext) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!row_ok) return v;
  if (vec && c + 3 < cols) {
    if (AM_IN(p - base, 4, ext)) v = ld4(p);
    return v;
  }
  float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (c + i < cols && AM_IN(p - base + i, 1, ext)) e[i] = to_f(p[i]);
  return make_float4(e[0], e[1], e[2], e[3]);
}

// SYM: Gram / square (B stored N x K, symmetric output, upper-triangle
// tiles); otherwise the update (B stored K x N).
template <typename T, bool SYM>
__global__ void __launch_bounds__(NT, 2) k_gemm_simt(const GemmLaunch L) {
  __shared__ __align__(16) float As[2][TK][LDS];
  __shared__ __align__(16) float Bs[2][TK][LDS];
  const int gi = find_group(L, blockIdx.x);
  const GemmGroup& g = L.g[gi];
  int t = blockIdx.x - g.tile_begin;
  const int b = t / g.tiles_per_mat;
  t -= b * g.tiles_per_mat;
  int tm, tn;
  if constexpr (SYM) {
    tri_tile(t, g.tiles_m, tm, tn);
  } else {
    tm = t / g.tiles_n;
    tn = t % g.tiles_n;
  }
  const int m0 = tm * TT, n0 = tn * TT;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const T* gA = reinterpret_cast<const T*>(g.A);
  const T* gB = reinterpret_cast<const T*>(g.B);
  // a quad can be read with one vector load when every quad's element
  // offset is a multiple of 4 and the base is aligned for a quad
  constexpr uintptr_t kQuadBytes = 4 * sizeof(T);
  const bool a_vec = ((g.lda | g.sa) & 3) == 0 && (reinterpret_cast<uintptr_t>(gA) % kQuadBytes) == 0;
  const bool b_vec = ((g.ldb | g.sb) & 3) == 0 && (reinterpret_cast<uintptr_t>(gB) % kQuadBytes) == 0;

  // This thread's slice elements.  K-contiguous operands (A, and B of the
  // symmetric kinds): row tid / 2, k 4 (tid % 2) .. +3.  The update's B (K x
  // N, N contiguous): k tid / 32, columns 4 (tid % 32) .. +3.
  const int kr = tid >> 1, kq = (tid & 1) * 4;
  const int nk = tid >> 5, nq = (tid & 31) * 4;
  const bool a_row = m0 + kr < g.M;
  const T* pa = gA + (int64_t)b * g.sa + (int64_t)(a_row ? m0 + kr : 0) * g.lda + kq;
  const bool b_row = SYM ? n0 + kr < g.N : true;
  const T* pb = SYM ? gB + (int64_t)b * g.sb + (int64_t)(b_row ? n0 + kr : 0) * g.ldb + kq
                    : gB + (int64_t)b * g.sb + (int64_t)nk * g.ldb + n0 + nq;
  const int64_t b_step = SYM ? TK : TK * g.ldb;
  auto load_a = [&](int k0) {
    return ld_quad<T>(pa + k0, a_row, k0 + kq, g.K, a_vec, gA, (int64_t)g.count * g.sa);
  };
  auto load_b = [&](int k0, const T* q) {
    if constexpr (SYM) return ld_quad<T>(q, b_row, k0 + kq, g.K, b_vec, gB, (int64_t)g.count * g.sb);
    else return ld_quad<T>(q, k0 + nk < g.K, n0 + nq, g.N, b_vec, gB, (int64_t)g.count * g.sb);
  };
  auto store = [&](int buf, float4 va, float4 vb) {
    As[buf][kq + 0][kr] = va.x;
    As[buf][kq + 1][kr] = va.y;
    As[buf][kq + 2][kr] = va.z;
    As[buf][kq + 3][kr] = va.w;
    if constexpr (SYM) {
      Bs[buf][kq + 0][kr] = vb.x;
      Bs[buf][kq + 1][kr] = vb.y;
      Bs[buf][kq + 2][kr] = vb.z;
      Bs[buf][kq + 3][kr] = vb.w;
    } else {
      *reinterpret_cast<float4*>(&Bs[buf][nk][nq]) = vb;
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  store(0, load_a(0), load_b(0, pb));
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < g.K; k0 += TK) {
    const bool more = k0 + TK < g.K;
    float4 na = make_float4(0.f, 0.f, 0.f, 0.f), nb = na;
    if (more) {
      pb += b_step;
      na = load_a(k0 + TK);
      nb = load_b(k0 + TK, pb);
    }
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][4 * ty]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + 4 * ty]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + 4 * tx]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (more) store(buf ^ 1, na, nb);
    __syncthreads();
    buf ^= 1;
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
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i >> 2) * 64 + 4 * ty + (i & 3);
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + (j >> 2) * 64 + 4 * tx + (j & 3);
      if (n >= g.N || (SYM && n < m)) continue;
      float v = alpha * acc[i][j];
      if (E && AM_IN((int64_t)b * g.se + (int64_t)m * g.lde + n, 1, (int64_t)g.count * g.se))
        v += beta * to_f(E[(int64_t)m * g.lde + n]);
      const T o = from_f<T>(v);
      if (AM_IN((int64_t)b * g.sc + (int64_t)m * g.ldc + n, 1, (int64_t)g.count * g.sc))
        C[(int64_t)m * g.ldc + n] = o;
      if (SYM && n != m && AM_IN((int64_t)b * g.sc + (int64_t)n * g.ldc + m, 1, (int64_t)g.count * g.sc))
        C[(int64_t)n * g.ldc + m] = o;
    }
  }
}

}  // namespace

int simt_tile_count(int kind, int M, int N, int* tiles_m, int* tiles_n) {
  *tiles_m = (M + kSimtTile - 1) / kSimtTile;
  *tiles_n = (N + kSimtTile - 1) / kSimtTile;
  if (kind != GK_UPD) return *tiles_m * (*tiles_m + 1) / 2;   // upper triangle (M == N)
  return *tiles_m * *tiles_n;
}

cudaError_t launch_gemm_simt(const GemmLaunch& L, cudaStream_t st) {
  if (L.total_tiles == 0) return cudaSuccess;
  // every group of a launch has the same kind
  const bool sym = L.g[0].kind != GK_UPD;
  if (L.dtype == kBF16) {
    if (sym) k_gemm_simt<__nv_bfloat16, true><<<L.total_tiles, NT, 0, st>>>(L);
    else k_gemm_simt<__nv_bfloat16, false><<<L.total_tiles, NT, 0, st>>>(L);
  } else {
    if (sym) k_gemm_simt<float, true><<<L.total_tiles, NT, 0, st>>>(L);
    else k_gemm_simt<float, false><<<L.total_tiles, NT, 0, st>>>(L);
  }
  return cudaGetLastError();
}

}  // namespace am
