// Shared device-side helpers of libaurora_muon: dtype access, reductions,
// the sticky status word and the per-launch matrix tables.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/aurora_muon.h"

namespace am {

constexpr int kF32 = MUON_F32;
constexpr int kBF16 = MUON_BF16;

// ---------------------------------------------------------------- dtype access
__device__ __forceinline__ float ld_as_f32(const void* p, int64_t i, int dt) {
  if (dt == kBF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}
__device__ __forceinline__ void st_from_f32(void* p, int64_t i, int dt, float v) {
  if (dt == kBF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(p)[i] = v;
}
__host__ __device__ __forceinline__ int dt_bytes(int dt) { return dt == kBF16 ? 2 : 4; }

// 8 consecutive elements p[i .. i+7] as floats; i a multiple of 8 and the
// array 16-byte aligned (one 16-byte load for bf16, two for fp32).
__device__ __forceinline__ void ld8(const void* p, int64_t i, int dt, float (&v)[8]) {
  if (dt == kBF16) {
    const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + i);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[2 * h] = __uint_as_float(ww[h] << 16);
      v[2 * h + 1] = __uint_as_float(ww[h] & 0xFFFF0000u);
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    const float4 b = *(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}
__device__ __forceinline__ void st8(void* p, int64_t i, int dt, const float (&v)[8]) {
  if (dt == kBF16) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * h], v[2 * h + 1]);
      w[h] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p) + i) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    float4* q = reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i);
    q[0] = make_float4(v[0], v[1], v[2], v[3]);
    q[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}
// Masked variants: only elements k < cnt (cnt <= 8) are touched; others read 0.
__device__ __forceinline__ void ld8m(const void* p, int64_t i, int dt, int cnt, float (&v)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = k < cnt ? ld_as_f32(p, i + k, dt) : 0.f;
}
__device__ __forceinline__ void st8m(void* p, int64_t i, int dt, int cnt, const float (&v)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    if (k < cnt) st_from_f32(p, i + k, dt, v[k]);
}
// Vector or masked access of the 8-group starting at column j of a row of
// length n (row start index `row_off`); vec: rows are 16-byte aligned.
__device__ __forceinline__ void ld8r(const void* p, int64_t row_off, int64_t j, int64_t n, bool vec, int dt,
                                     float (&v)[8]) {
  if (vec && j + 8 <= n) ld8(p, row_off + j, dt, v);
  else ld8m(p, row_off + j, dt, (int)(n - j < 8 ? (n - j > 0 ? n - j : 0) : 8), v);
}
__device__ __forceinline__ void st8r(void* p, int64_t row_off, int64_t j, int64_t n, bool vec, int dt,
                                     const float (&v)[8]) {
  if (vec && j + 8 <= n) st8(p, row_off + j, dt, v);
  else st8m(p, row_off + j, dt, (int)(n - j < 8 ? (n - j > 0 ? n - j : 0) : 8), v);
}

// ---------------------------------------------------------------- checked build
// Built with AURORA_MUON_CHECKED (build.py --checked -> libaurora_muon_checked.so),
// every global access of the streaming, power-iteration, GEMM-epilogue,
// SIMT-GEMM and AdamW kernels first tests its element range
// [first, first + count) against the extent of the buffer it addresses (TMA
// loads and stores are bounded by their tensor maps).  A failed test records
// the source line in the file's sticky check word (first failure wins) and the access is
// skipped (loads read zeros), so nothing outside a buffer is touched; the
// host reads the words through muon_last_device_status (MUON_ERR_BOUNDS).
// In the normal build the test is the constant true and compiles away.
#ifdef AURORA_MUON_CHECKED
static __device__ unsigned int g_check_line = 0;
__device__ __noinline__ inline void check_fail(unsigned int line) { atomicCAS(&g_check_line, 0u, line); }
__device__ __forceinline__ bool in_range(int64_t first, int64_t count, int64_t extent, unsigned int line) {
  if (first >= 0 && count >= 0 && first + count <= extent) return true;
  check_fail(line);
  return false;
}
#define AM_IN(first, count, extent) ::am::in_range((int64_t)(first), (int64_t)(count), (int64_t)(extent), __LINE__)
// Host: read and clear this file's check word (current device).
#define AM_CHECK_READER(fn)                                                        \
  cudaError_t fn(unsigned int* out) {                                              \
    unsigned int v = 0, zero = 0;                                                  \
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_check_line, sizeof(v));             \
    if (e != cudaSuccess) return e;                                                \
    *out = v;                                                                      \
    return v ? cudaMemcpyToSymbol(g_check_line, &zero, sizeof(zero)) : cudaSuccess; \
  }
#else
#define AM_IN(first, count, extent) true
#define AM_CHECK_READER(fn)             \
  cudaError_t fn(unsigned int* out) {   \
    *out = 0;                           \
    return cudaSuccess;                 \
  }
#endif
// Elements of the 8-group at column j of a row of length n (0 to 8).
__device__ __forceinline__ int64_t cnt8(int64_t n, int64_t j) { return n - j >= 8 ? 8 : (n - j > 0 ? n - j : 0); }
// Extents of the per-matrix buffers (elements).
#define AM_EXT_ORIG(d) ((d).m * (d).n)                 /* W, G, M, V */
#define AM_EXT_X(d) ((d).s * (d).ldl)                  /* uX, UX, X0 */
#define AM_EXT_VEC(d) ((((d).l > (d).s ? (d).l : (d).s) + 63) / 64 * 64)   /* vec0, vec1 */

// Checked forms of the access helpers: `ext` is the extent (elements) of the
// buffer p points to.  A range outside it is skipped (a load gives zeros).
#define ld8c(ext, p, i, dt, v)                                  \
  do {                                                          \
    if (AM_IN((i), 8, (ext))) ::am::ld8((p), (i), (dt), (v));   \
    else for (int _q = 0; _q < 8; ++_q) (v)[_q] = 0.f;          \
  } while (0)
#define st8c(ext, p, i, dt, v)                                  \
  do {                                                          \
    if (AM_IN((i), 8, (ext))) ::am::st8((p), (i), (dt), (v));   \
  } while (0)
#define ld8rc(ext, p, row_off, j, n, vec, dt, v)                                        \
  do {                                                                                  \
    if (AM_IN((row_off) + (j), ::am::cnt8((n), (j)), (ext)))                            \
      ::am::ld8r((p), (row_off), (j), (n), (vec), (dt), (v));                           \
    else for (int _q = 0; _q < 8; ++_q) (v)[_q] = 0.f;                                  \
  } while (0)
#define st8rc(ext, p, row_off, j, n, vec, dt, v)                                        \
  do {                                                                                  \
    if (AM_IN((row_off) + (j), ::am::cnt8((n), (j)), (ext)))                            \
      ::am::st8r((p), (row_off), (j), (n), (vec), (dt), (v));                           \
  } while (0)
// 16 bytes (8 bf16) at element i of a bf16 buffer through the read-only path
__device__ __forceinline__ uint4 ldg8bf(int64_t ext, const __nv_bfloat16* p, int64_t i, unsigned int line) {
#ifdef AURORA_MUON_CHECKED
  if (!in_range(i, 8, ext, line)) return make_uint4(0, 0, 0, 0);
#endif
  return __ldg(reinterpret_cast<const uint4*>(p + i));
}
#define LDG8BF(ext, p, i) ::am::ldg8bf((ext), (p), (i), __LINE__)

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Deterministic block sum of one double per thread (blockDim.x multiple of 32,
// at most 1024).  Every thread gets the result.
__device__ __forceinline__ double block_sum(double v, double* smem32) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) smem32[wid] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < nw; ++w) t += smem32[w];
  return t;
}

// ---------------------------------------------------------------- tables
// Matrix descriptor for the element-wise / reduction kernels.  Original
// orientation is m x n; the "X orientation" is s x l (s = min, l = max), the
// transpose of the original when the matrix is tall (m > n).
struct MatDesc {
  void* W;            // param (param dtype), original orientation
  const void* G;      // grad / input (grad dtype), original orientation
  float* M;           // momentum fp32, original orientation
  float* V;           // optional fp32 output, original orientation
  void* uX;           // u in X orientation (ns dtype), leading dim ldl
  void* UX;           // polar output in X orientation (ns dtype), leading dim ldl
  void* X0;           // scaled Newton-Schulz input (ns dtype), leading dim ldl
  float* D;           // Aurora column scale (length l)
  float* vec0;        // power-iteration vectors (length >= l), two of them
  float* vec1;
  float* rho_slot;    // bucket-ordered copy of rho read by the GEMM epilogues
  float* gvp;         // fused power iteration: one partial X^T z (ldl floats) per row item
  float* colsq;       // Aurora D: column sums of squares (X orientation) per row block, room for
                      // [ceil(s / 32)][round64(l)] floats: of uX per 128 rows for the D init,
                      // of U per 32 rows (written by the last update GEMM) for the D update
  int64_t m, n, s, l, ldl;
  int tall;           // m > n
  int idx;            // matrix index (scalar block row)
  int part;           // first partial slot of this matrix
  int nslots;         // partial slots owned by this matrix (from part on)
  int nblk;           // blocks of this matrix in the current launch
  int flag;           // launch-specific per-matrix flag
  int gv_rows;        // fused power iteration: rows of X per item
};

constexpr int kMaxMatsPerLaunch = 96;

struct MatTable {
  int count;
  int ns_dtype;       // dtype of uX / UX / X0
  int param_dtype;
  int grad_dtype;
  int blk_prefix[kMaxMatsPerLaunch + 1];
  MatDesc mats[kMaxMatsPerLaunch];
};

__device__ __forceinline__ int find_mat(const MatTable& t, int blk) {
  int lo = 0, hi = t.count - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (t.blk_prefix[mid] <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Per-matrix scalar block (doubles), indexed by MatDesc::idx.
enum ScalarSlot {
  S_SUM_U2 = 0,    // |u|_F^2
  S_SUM_W2,        // |W|_F^2
  S_SUM_X02,       // |X0|_F^2 of the scaled NS input
  S_RHO,           // 1 / (|X0|_F + ns_eps)
  S_SIGMA,         // operator-norm estimate
  S_SUM_UU2,       // |U|_F^2 of the polar output
  S_DOT_UUX,       // <U, u>
  S_COEF_U,        // final coefficient of U in V
  S_COEF_u,        // final coefficient of u in V
  S_VNORM2,        // scratch
  S_COUNT = 16
};

}  // namespace am
