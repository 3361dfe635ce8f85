// HBM-bound stages of the optimizer step: momentum/Nesterov prologue,
// Aurora column scales, scaled Newton-Schulz input, power-iteration
// matrix-vector passes, Frobenius / dot reductions, the per-matrix scalar
// algebra and the fused parameter epilogue.
//
// Method: "modded-nanogpt Track 3 优化实录：Aurora 行均衡 polar + Contra-Muon +
// u/w-floor …", sections "组合优化栈" (muon_update), "源码实现"
// (aurora_orthogonalize) and "u/w-floor".
//
// Every reduction is deterministic: per-block partials in a fixed order,
// combined in double precision by a second pass.
#include "common.cuh"
#include "kernels.h"

namespace am {

constexpr int kTile = 64;       // element-wise tile edge
constexpr int kEwThreads = 256; // 8 column groups of 8 elements x 32 row lanes
constexpr int kWarps = kEwThreads / 32;

// Warp-level partial sums (no block barrier): lane 0 of each warp writes
// its warp's sums to partials[((slot) * kWarps + warp) * nq + q].
__device__ __forceinline__ void warp_partials(double* partials, int64_t slot, int nq, float a, float b) {
  const double A = warp_sum((double)a);
  const double B = nq > 1 ? warp_sum((double)b) : 0.0;
  if ((threadIdx.x & 31) == 0) {
    double* p = partials + (slot * kWarps + (threadIdx.x >> 5)) * nq;
    p[0] = A;
    if (nq > 1) p[1] = B;
  }
}

// ============================================================================
// prologue: m <- m + (1-mu)(g-m); u = Nesterov ? g + mu(m-g) : m; write u in
// the X orientation (transposed through shared memory for tall matrices);
// per-warp partials of |u|^2 and |W|^2.
// mode 0: optimizer step (uses G, M, W);  mode 1: u = G (input staging).
// A block owns a 64 x 64 tile; thread t handles the 8-element groups
// (row t/8 + 32k, columns 8 (t%8) .. +7), k = 0, 1, with 16-byte accesses.
// All loads are issued before any store (the buffers may alias as far as the
// compiler knows).
// ============================================================================
__global__ void __launch_bounds__(kEwThreads, 4)
k_prologue(const MatTable t, int mode, float mu, int nesterov, int want_w2, double* partials) {
  __shared__ float tile[kTile][kTile + 1];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int nt = (int)(((d.m + kTile - 1) / kTile) * ((d.n + kTile - 1) / kTile));
  const int b0 = (blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  for (int b = b0; b < b0 + kEwTilesPerCta && b < nt; ++b) {
    if (b != b0) __syncthreads();   // shared tile reused by the next tile
    const int64_t tiles_c = (d.n + kTile - 1) / kTile;
    const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
    const int rg = threadIdx.x >> 3, cg = threadIdx.x & 7;
    const bool vec = (d.n & 7) == 0;
    const bool xvec = (d.ldl & 7) == 0;
    const int64_t j = c0 + 8 * cg;
    const bool in0 = r0 + rg < d.m && j < d.n, in1 = r0 + rg + 32 < d.m && j < d.n;
    const int64_t ro0 = (r0 + rg) * d.n, ro1 = (r0 + rg + 32) * d.n;
    float g0[8], g1[8], m0[8], m1[8], w0[8], w1[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) g0[e] = g1[e] = m0[e] = m1[e] = w0[e] = w1[e] = 0.f;
    if (in0) ld8rc(AM_EXT_ORIG(d), d.G, ro0, j, d.n, vec, t.grad_dtype, g0);
    if (in1) ld8rc(AM_EXT_ORIG(d), d.G, ro1, j, d.n, vec, t.grad_dtype, g1);
    if (mode == 0) {
      if (in0) ld8rc(AM_EXT_ORIG(d), d.M, ro0, j, d.n, vec, kF32, m0);
      if (in1) ld8rc(AM_EXT_ORIG(d), d.M, ro1, j, d.n, vec, kF32, m1);
      if (want_w2) {
        if (in0) ld8rc(AM_EXT_ORIG(d), d.W, ro0, j, d.n, vec, t.param_dtype, w0);
        if (in1) ld8rc(AM_EXT_ORIG(d), d.W, ro1, j, d.n, vec, t.param_dtype, w1);
      }
    }
    float su2 = 0.f, sw2 = 0.f;
    float u0[8], u1[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (mode == 0) {
        m0[e] = m0[e] + (1.f - mu) * (g0[e] - m0[e]);
        m1[e] = m1[e] + (1.f - mu) * (g1[e] - m1[e]);
        u0[e] = nesterov ? g0[e] + mu * (m0[e] - g0[e]) : m0[e];
        u1[e] = nesterov ? g1[e] + mu * (m1[e] - g1[e]) : m1[e];
      } else {
        u0[e] = g0[e];
        u1[e] = g1[e];
      }
      su2 += u0[e] * u0[e] + u1[e] * u1[e];
      sw2 += w0[e] * w0[e] + w1[e] * w1[e];
    }
    if (mode == 0) {
      if (in0) st8rc(AM_EXT_ORIG(d), d.M, ro0, j, d.n, vec, kF32, m0);
      if (in1) st8rc(AM_EXT_ORIG(d), d.M, ro1, j, d.n, vec, kF32, m1);
    }
    if (!d.tall) {
      if (in0) st8rc(AM_EXT_X(d), d.uX, (r0 + rg) * d.ldl, j, d.n, xvec, t.ns_dtype, u0);
      if (in1) st8rc(AM_EXT_X(d), d.uX, (r0 + rg + 32) * d.ldl, j, d.n, xvec, t.ns_dtype, u1);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        tile[rg][8 * cg + e] = u0[e];
        tile[rg + 32][8 * cg + e] = u1[e];
      }
      __syncthreads();
      // X row = original column c0 + xr; X columns = original rows r0 + 8 cg ..
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int xr = rg + 32 * k;
        const int64_t xi = c0 + xr, xj = r0 + 8 * cg;
        if (xi < d.n && xj < d.m) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = tile[8 * cg + e][xr];
          st8rc(AM_EXT_X(d), d.uX, xi * d.ldl, xj, d.m, xvec, t.ns_dtype, v);
        }
      }
    }
    if (AM_IN(b, 1, d.nslots)) warp_partials(partials, d.part + b, 2, su2, sw2);
  }
}

// Sum the per-warp partials of each matrix into its scalar block.  Layout:
// partials[((part + block) * 8 + warp) * nq + q]; slot < 0 skips q.
__global__ void k_finalize_sums(const MatTable t, const double* partials, int nq, int slot0,
                                int slot1, double* scal) {
  __shared__ double red[32];
  const MatDesc& d = t.mats[blockIdx.x];
  for (int q = 0; q < nq; ++q) {
    const int slot = q == 0 ? slot0 : slot1;
    double s = 0.0;
    const int64_t n = (int64_t)d.nblk * kWarps;
    for (int64_t k = threadIdx.x; k < n; k += blockDim.x)
      if (AM_IN(k, 1, (int64_t)d.nslots * kWarps)) s += partials[((int64_t)d.part * kWarps + k) * nq + q];
    s = block_sum(s, red);
    if (threadIdx.x == 0 && slot >= 0) scal[d.idx * S_COUNT + slot] = s;
  }
}

// ============================================================================
// Aurora D update from a pass over U (the FP32 / SIMT modes; the tensor-core
// mode takes the column sums from the GEMM epilogue): per column j of the X
// orientation (= a row of the tall-oriented matrix) sum_i U_ij^2, then
// row_sq = max(sum, pp_eps^2) and D_j *= (target / row_sq)^beta with
// target = s / l ["源码实现"].
// A block owns kColStrip = 256 columns; each warp streams every 8th row with
// one 16-byte load (8 columns) per lane, so a warp reads 512 contiguous bytes.
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_colnorm(const MatTable t, float pp_eps, float beta) {
  __shared__ float part[kWarps][kColStrip];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t j = (int64_t)b * kColStrip + 8 * lane;
  const void* X = d.UX;
  const bool vec = (d.ldl & 7) == 0;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (j < d.l) {
#pragma unroll 4
    for (int64_t i = w; i < d.s; i += kWarps) {
      float x[8];
      ld8rc(AM_EXT_X(d), X, i * d.ldl, j, d.l, vec, t.ns_dtype, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += x[e] * x[e];
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[w][8 * lane + e] = acc[e];
  __syncthreads();
  const int64_t jj = (int64_t)b * kColStrip + threadIdx.x;
  if (jj < d.l) {
    float sum = 0.f;
#pragma unroll
    for (int r = 0; r < kWarps; ++r) sum += part[r][threadIdx.x];
    if (!AM_IN(jj, 1, d.l)) return;
    const float row_sq = fmaxf(sum, pp_eps * pp_eps);
    const float target = (float)d.s / (float)d.l;
    d.D[jj] = d.D[jj] * powf(target / row_sq, beta);
  }
}

// Column sums of squares of uX over kColsqRows-row blocks, into
// MatDesc::colsq ([ceil(s / kColsqRows)][round64(l)] floats): a block covers
// 8 kColsqRows rows x 256 columns, warp w rows kColsqRows w .. of them, each
// lane 8 columns (one 16-byte load per row).  Blocks of bounded length
// instead of one block walking every row of a column strip (whose last wave
// leaves most of the GPU idle).
__global__ void __launch_bounds__(kEwThreads, 4)
k_colsq_partial(const MatTable t) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t strips = (d.l + kColStrip - 1) / kColStrip;
  const int64_t b = blockIdx.x - t.blk_prefix[mi];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t rb = (b / strips) * 8 + w;                  // row block of this warp
  const int64_t j = (b % strips) * kColStrip + 8 * lane;
  const int64_t i0 = rb * kColsqRows;
  if (i0 >= d.s || j >= d.l) return;
  const int64_t i1 = min(d.s, i0 + kColsqRows);
  const bool vec = (d.ldl & 7) == 0;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
  for (int64_t i = i0; i < i1; ++i) {
    float x[8];
    ld8rc(AM_EXT_X(d), d.uX, i * d.ldl, j, d.l, vec, t.ns_dtype, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += x[e] * x[e];
  }
  float* q = d.colsq + rb * ((d.l + 63) / 64 * 64) + j;     // j + 8 <= round64(l)
  if (!AM_IN(rb * ((d.l + 63) / 64 * 64) + j, 8, ((d.s + 31) / 32) * ((d.l + 63) / 64 * 64))) return;
  // (ceil(s / kColsqRows) row blocks fit the buffer sized for 32-row blocks)
  reinterpret_cast<float4*>(q)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  reinterpret_cast<float4*>(q)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// Aurora D from the partial column sums in MatDesc::colsq (written per
// kColsqRows-row block by k_colsq_partial from uX, or per 32-row block by the
// last update GEMM of the previous polar from U): one thread per column sums
// the ceil(s / rows) partials in block order (deterministic).
//   mode 0 (D init):  D_j = 1 / max(sqrt(sum), pp_eps)
//   mode 1 (D update): D_j *= (target / max(sum, pp_eps^2))^beta, target = s / l
__global__ void __launch_bounds__(kColStrip)
k_colsq_update(const MatTable t, int mode, int rows, float pp_eps, float beta) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t j = (int64_t)(blockIdx.x - t.blk_prefix[mi]) * kColStrip + threadIdx.x;
  if (j >= d.l) return;
  const int64_t nb = (d.s + rows - 1) / rows, ldq = (d.l + 63) / 64 * 64;
  const float* q = d.colsq + j;
  float sum = 0.f;
  for (int64_t b = 0; b < nb; ++b)
    if (AM_IN(b * ldq + j, 1, nb * ldq)) sum += q[b * ldq];
  if (!AM_IN(j, 1, d.l)) return;
  if (mode == 0) {
    d.D[j] = 1.f / fmaxf(sqrtf(sum), pp_eps);
  } else {
    const float row_sq = fmaxf(sum, pp_eps * pp_eps);
    const float target = (float)d.s / (float)d.l;
    d.D[j] = d.D[j] * powf(target / row_sq, beta);
  }
}

// X0 = uX * diag(D) in the NS dtype, with per-warp partials of |X0|^2.
// 64 x 64 tiles of the X orientation, 8-element groups.
__global__ void __launch_bounds__(kEwThreads)
k_scale_cols(const MatTable t, double* partials) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int nt = (int)(((d.s + kTile - 1) / kTile) * ((d.l + kTile - 1) / kTile));
  const int b0 = (blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  for (int b = b0; b < b0 + kEwTilesPerCta && b < nt; ++b) {
    const int64_t tiles_c = (d.l + kTile - 1) / kTile;
    const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
    const int rg = threadIdx.x >> 3, cg = threadIdx.x & 7;
    const int64_t j = c0 + 8 * cg;
    const bool vec = (d.ldl & 7) == 0;
    float s2 = 0.f;
    if (j < d.l) {
      const bool in0 = r0 + rg < d.s, in1 = r0 + rg + 32 < d.s;
      const int64_t ro0 = (r0 + rg) * d.ldl, ro1 = (r0 + rg + 32) * d.ldl;
      float dj[8], x0[8], x1[8];
      ld8rc(d.l, d.D, 0, j, d.l, true, kF32, dj);
      if (in0) ld8rc(AM_EXT_X(d), d.uX, ro0, j, d.l, vec, t.ns_dtype, x0);
      if (in1) ld8rc(AM_EXT_X(d), d.uX, ro1, j, d.l, vec, t.ns_dtype, x1);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x0[e] = in0 ? x0[e] * dj[e] : 0.f;
        x1[e] = in1 ? x1[e] * dj[e] : 0.f;
        s2 += x0[e] * x0[e] + x1[e] * x1[e];
      }
      if (in0) st8rc(AM_EXT_X(d), d.X0, ro0, j, d.l, vec, t.ns_dtype, x0);
      if (in1) st8rc(AM_EXT_X(d), d.X0, ro1, j, d.l, vec, t.ns_dtype, x1);
    }
    if (AM_IN(b, 1, d.nslots)) warp_partials(partials, d.part + b, 1, s2, 0.f);
  }
}

// Per-matrix scalar algebra (one thread per matrix).
//  op 0: rho = 1 / (sqrt(scal[src]) + ns_eps)
//  op 1: final coefficients of V = cU U + cu u (optimizer step)
//  op 2: cU = 1, cu = 0 (plain polar output)
//  op 3: cU = 0, cu = 1 / max(sigma, 1e-10) (operator-norm normalisation)
//  op 4: u/w floor on an existing update: S_SUM_U2 holds |U|^2, S_SUM_W2 |W|^2
__global__ void k_scalars(const MatTable t, int op, int src_slot, float ns_eps, float contra,
                          float target_uw, double* scal) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= t.count) return;
  const MatDesc& d = t.mats[k];
  double* S = scal + (int64_t)d.idx * S_COUNT;
  if (op == 0) {
    S[S_RHO] = 1.0 / (sqrt(S[src_slot]) + (double)ns_eps);
  } else if (op == 1) {
    const double m = (double)d.m, n = (double)d.n;
    const double F2 = S[S_SUM_UU2];
    const double F = sqrt(F2);
    double cU = 1.0, cu = 0.0, vnorm;
    if (contra != 0.f) {
      // V = U - (C/2) u / sigma';  |V|^2 = F^2 - C <U,u>/sigma' + (C^2/4) |u|^2 / sigma'^2
      const double sg = fmax(S[S_SIGMA], 1e-10);
      const double h = 0.5 * (double)contra / sg;
      double v2 = F2 - 2.0 * h * S[S_DOT_UUX] + h * h * S[S_SUM_U2];
      v2 = fmax(v2, 0.0);
      const double r = F / fmax(sqrt(v2), 1e-10);   // Frobenius restore
      cU = r;
      cu = -h * r;
      vnorm = sqrt(v2) * r;
    } else {
      vnorm = F;
    }
    const double asp = sqrt(fmax(1.0, m / n));
    cU *= asp; cu *= asp; vnorm *= asp;
    if (target_uw > 0.f) {
      const double pw = fmax(sqrt(S[S_SUM_W2]), 1e-8);
      const double pu = fmax(vnorm, 1e-8);
      if (pu / pw < (double)target_uw) {
        const double f = (double)target_uw * pw / pu;
        cU *= f; cu *= f;
      }
    }
    S[S_COEF_U] = cU;
    S[S_COEF_u] = cu;
  } else if (op == 2) {
    S[S_COEF_U] = 1.0;
    S[S_COEF_u] = 0.0;
  } else if (op == 3) {
    S[S_COEF_U] = 0.0;
    S[S_COEF_u] = 1.0 / fmax(S[S_SIGMA], 1e-10);
  } else if (op == 4) {
    const double pw = fmax(sqrt(S[S_SUM_W2]), 1e-8);
    const double pu = fmax(sqrt(S[S_SUM_U2]), 1e-8);
    S[S_COEF_U] = (pu / pw < (double)target_uw) ? (double)target_uw * pw / pu : 1.0;
  }
}

// ============================================================================
// Power iteration ("组合优化栈": scale_to_unit_operator_norm, 5 iterations).
// On the X orientation Q (s x l):
//   flag 0 (row dot):  out_i = sum_j Q_ij x_j   (x length l, out length s)
//                      one warp per kMatvecRowsPerWarp rows, 8-element groups per lane
//   flag 1 (col dot):  out_j = sum_i Q_ij y_i   (y length s, out length l)
//                      kColDotStrip columns per block, 32 row lanes
// `dir` selects vec0 -> vec1 (0) or vec1 -> vec0 (1).  The vectors are
// 16-byte aligned with length padded to a multiple of 64.
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_matvec(const MatTable t, int dir) {
  __shared__ float smem[32 * (kColDotStrip + 1)];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const float* in = dir == 0 ? d.vec0 : d.vec1;
  float* out = dir == 0 ? d.vec1 : d.vec0;
  const bool vec = (d.ldl & 7) == 0;
  if (d.flag == 0) {
    // each warp reduces kMatvecRowsPerWarp rows, loading the vector chunk once
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t i0 = (int64_t)b * kMatvecRowsPerCta + w * kMatvecRowsPerWarp;
    float acc[kMatvecRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kMatvecRowsPerWarp; ++r) acc[r] = 0.f;
    if (i0 < d.s) {
#pragma unroll 2
      for (int64_t j = 8 * lane; j < d.l; j += 256) {
        float v[8];
        ld8rc(AM_EXT_VEC(d), in, 0, j, d.l, true, kF32, v);
#pragma unroll
        for (int r = 0; r < kMatvecRowsPerWarp; ++r) {
          if (i0 + r < d.s) {
            float x[8];
            ld8rc(AM_EXT_X(d), d.uX, (i0 + r) * d.ldl, j, d.l, vec, t.ns_dtype, x);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[r] += x[e] * v[e];
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kMatvecRowsPerWarp; ++r) {
        const float a = warp_sum(acc[r]);
        if (lane == 0 && i0 + r < d.s && AM_IN(i0 + r, 1, AM_EXT_VEC(d))) out[i0 + r] = a;
      }
    }
  } else {
    // kColDotStrip = 64 columns: 8 groups of 8 columns x 32 row lanes
    float (*part)[kColDotStrip + 1] = reinterpret_cast<float (*)[kColDotStrip + 1]>(smem);
    const int cg = threadIdx.x & 7, rl = threadIdx.x >> 3;
    const int64_t j = (int64_t)b * kColDotStrip + 8 * cg;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (j < d.l) {
#pragma unroll 4
      for (int64_t i = rl; i < d.s; i += 32) {
        float x[8];
        ld8rc(AM_EXT_X(d), d.uX, i * d.ldl, j, d.l, vec, t.ns_dtype, x);
        const float y = AM_IN(i, 1, AM_EXT_VEC(d)) ? in[i] : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += x[e] * y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[rl][8 * cg + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < kColDotStrip) {
      const int64_t jj = (int64_t)b * kColDotStrip + threadIdx.x;
      if (jj < d.l && AM_IN(jj, 1, AM_EXT_VEC(d))) {
        float sum = 0.f;
        for (int r = 0; r < 32; ++r) sum += part[r][threadIdx.x];
        out[jj] = sum;
      }
    }
  }
}

// One block per matrix on the vector of length len (flag 0: l, 1: s; `which`
// picks vec0/vec1).  mode 0: fill with 1/sqrt(len);  mode 1: normalise to
// unit length (guarded by 1e-30);  mode 2: store the norm as sigma.
__global__ void k_vecop(const MatTable t, int which, int mode, int len_is_s_when_flag0,
                        double* scal) {
  __shared__ double red[32];
  const MatDesc& d = t.mats[blockIdx.x];
  float* v = which == 0 ? d.vec0 : d.vec1;
  const bool is_s = (d.flag == 0) == (len_is_s_when_flag0 != 0);
  const int64_t len = is_s ? d.s : d.l;
  if (mode == 0) {
    const float c = (float)(1.0 / sqrt((double)len));
    for (int64_t i = threadIdx.x; i < len; i += blockDim.x) v[i] = c;
    return;
  }
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < len; i += blockDim.x) s += (double)v[i] * v[i];
  s = block_sum(s, red);
  const double nrm = sqrt(s);
  if (mode == 1) {
    const float inv = (float)(1.0 / fmax(nrm, 1e-30));
    for (int64_t i = threadIdx.x; i < len; i += blockDim.x) v[i] *= inv;
  } else if (threadIdx.x == 0) {
    scal[d.idx * S_COUNT + S_SIGMA] = nrm;
  }
}

// ============================================================================
// <U,U> and <U,u> over the X orientation, per-warp partials (2 per warp).
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_dots(const MatTable t, double* partials) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int nt = (int)(((d.s + kTile - 1) / kTile) * ((d.l + kTile - 1) / kTile));
  const int b0 = (blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  for (int b = b0; b < b0 + kEwTilesPerCta && b < nt; ++b) {
    const int64_t tiles_c = (d.l + kTile - 1) / kTile;
    const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
    const int rg = threadIdx.x >> 3, cg = threadIdx.x & 7;
    const int64_t j = c0 + 8 * cg;
    const bool vec = (d.ldl & 7) == 0;
    float a = 0.f, c = 0.f;
    if (j < d.l) {
      const bool in0 = r0 + rg < d.s, in1 = r0 + rg + 32 < d.s;
      const int64_t ro0 = (r0 + rg) * d.ldl, ro1 = (r0 + rg + 32) * d.ldl;
      float U0[8], u0[8], U1[8], u1[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) U0[e] = u0[e] = U1[e] = u1[e] = 0.f;
      if (in0) { ld8rc(AM_EXT_X(d), d.UX, ro0, j, d.l, vec, t.ns_dtype, U0); ld8rc(AM_EXT_X(d), d.uX, ro0, j, d.l, vec, t.ns_dtype, u0); }
      if (in1) { ld8rc(AM_EXT_X(d), d.UX, ro1, j, d.l, vec, t.ns_dtype, U1); ld8rc(AM_EXT_X(d), d.uX, ro1, j, d.l, vec, t.ns_dtype, u1); }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        a += U0[e] * U0[e] + U1[e] * U1[e];
        c += U0[e] * u0[e] + U1[e] * u1[e];
      }
    }
    if (AM_IN(b, 1, d.nslots)) warp_partials(partials, d.part + b, 2, a, c);
  }
}

// ============================================================================
// Fused epilogue, original orientation: V = cU U + cu u (U, u read from the
// X orientation, transposed through shared memory for tall matrices);
// optional fp32 V output; optional W <- W - lr V in the param dtype.
// 64 x 64 tiles, 8-element groups with 16-byte accesses.
// ============================================================================
__global__ void __launch_bounds__(kEwThreads, 4)
k_epilogue(const MatTable t, float lr, int update_w, const double* scal) {
  __shared__ float tV[kTile][kTile + 1];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int nt = (int)(((d.m + kTile - 1) / kTile) * ((d.n + kTile - 1) / kTile));
  const int b0 = (blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  const float cU = (float)scal[d.idx * S_COUNT + S_COEF_U];
  const float cu = (float)scal[d.idx * S_COUNT + S_COEF_u];
  const bool need_U = cU != 0.f, need_u = cu != 0.f;
  const bool vec = (d.n & 7) == 0;
  const bool xvec = (d.ldl & 7) == 0;
  const int rg = threadIdx.x >> 3, cg = threadIdx.x & 7;
  for (int b = b0; b < b0 + kEwTilesPerCta && b < nt; ++b) {
    if (b != b0) __syncthreads();   // shared tile reused by the next tile
    const int64_t tiles_c = (d.n + kTile - 1) / kTile;
    const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
    const int64_t j = c0 + 8 * cg;
    float v[2][8], w[2][8];
    bool in[2];
    // parameter rows first: their loads overlap the transpose below
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t i = r0 + rg + 32 * k;
      in[k] = i < d.m && j < d.n;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[k][e] = w[k][e] = 0.f;
      if (in[k] && update_w) ld8rc(AM_EXT_ORIG(d), d.W, i * d.n, j, d.n, vec, t.param_dtype, w[k]);
    }
    if (d.tall) {
      // V = cU U + cu u is formed in the X orientation (X tile rows = original
      // columns c0 + xr, X tile columns = original rows r0 + 8 cg ..) and
      // transposed through one shared tile
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int64_t xi = c0 + rg + 32 * k, xj = r0 + 8 * cg;
        float xU[8], xu[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) xU[e] = xu[e] = 0.f;
        if (xi < d.n && xj < d.m) {
          if (need_U) ld8rc(AM_EXT_X(d), d.UX, xi * d.ldl, xj, d.m, xvec, t.ns_dtype, xU);
          if (need_u) ld8rc(AM_EXT_X(d), d.uX, xi * d.ldl, xj, d.m, xvec, t.ns_dtype, xu);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) tV[rg + 32 * k][8 * cg + e] = cU * xU[e] + cu * xu[e];
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) v[k][e] = tV[8 * cg + e][rg + 32 * k];
    } else {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int64_t i = r0 + rg + 32 * k;
        if (!in[k]) continue;
        float U[8], u[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) U[e] = u[e] = 0.f;
        if (need_U) ld8rc(AM_EXT_X(d), d.UX, i * d.ldl, j, d.n, xvec, t.ns_dtype, U);
        if (need_u) ld8rc(AM_EXT_X(d), d.uX, i * d.ldl, j, d.n, xvec, t.ns_dtype, u);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[k][e] = cU * U[e] + cu * u[e];
      }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (!in[k]) continue;
      const int64_t ro = (r0 + rg + 32 * k) * d.n;
#pragma unroll
      for (int e = 0; e < 8; ++e) w[k][e] -= lr * v[k][e];
      if (d.V) st8rc(AM_EXT_ORIG(d), d.V, ro, j, d.n, vec, kF32, v[k]);
      if (update_w) st8rc(AM_EXT_ORIG(d), d.W, ro, j, d.n, vec, t.param_dtype, w[k]);
    }
  }
}

// Tall matrices whose edges are multiples of 64, bf16 params and bf16
// Newton-Schulz storage (the common case): the same epilogue with every load
// issued one tile ahead of its use (packed bf16 in registers), and two shared
// tiles so each tile needs one barrier.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float (&v)[8]) {
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    v[2 * h] = __uint_as_float(ww[h] << 16);
    v[2 * h + 1] = __uint_as_float(ww[h] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(kEwThreads, 3)
k_epilogue_tall_bf16(const MatTable t, float lr, int update_w, const double* scal) {
  __shared__ float tV[2][kTile][kTile + 1];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t tiles_c = d.n / kTile;
  const int nt = (int)((d.m / kTile) * tiles_c);
  const int b0 = (blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  const int b1 = min(b0 + kEwTilesPerCta, nt);
  const float cU = (float)scal[d.idx * S_COUNT + S_COEF_U];
  const float cu = (float)scal[d.idx * S_COUNT + S_COEF_u];
  const bool need_U = cU != 0.f, need_u = cu != 0.f;
  const int rg = threadIdx.x >> 3, cg = threadIdx.x & 7;
  const __nv_bfloat16* W = reinterpret_cast<const __nv_bfloat16*>(d.W);
  const __nv_bfloat16* UX = reinterpret_cast<const __nv_bfloat16*>(d.UX);
  const __nv_bfloat16* uX = reinterpret_cast<const __nv_bfloat16*>(d.uX);
  // per tile: W rows r0 + rg (+32) at columns c0 + 8 cg; X rows c0 + rg (+32)
  // of U and u at columns r0 + 8 cg
  auto load = [&](int b, uint4 (&w)[2], uint4 (&xU)[2], uint4 (&xu)[2]) {
    const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t i = r0 + rg + 32 * k, xi = c0 + rg + 32 * k;
      w[k] = update_w ? LDG8BF(AM_EXT_ORIG(d), W, i * d.n + c0 + 8 * cg) : make_uint4(0, 0, 0, 0);
      xU[k] = need_U ? LDG8BF(AM_EXT_X(d), UX, xi * d.ldl + r0 + 8 * cg) : make_uint4(0, 0, 0, 0);
      xu[k] = need_u ? LDG8BF(AM_EXT_X(d), uX, xi * d.ldl + r0 + 8 * cg) : make_uint4(0, 0, 0, 0);
    }
  };
  auto process = [&](int b, int buf, const uint4 (&w)[2], const uint4 (&xU)[2], const uint4 (&xu)[2]) {
    const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      float U[8], u[8];
      bf16x8_to_f32(xU[k], U);
      bf16x8_to_f32(xu[k], u);
#pragma unroll
      for (int e = 0; e < 8; ++e) tV[buf][rg + 32 * k][8 * cg + e] = cU * U[e] + cu * u[e];
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t ro = (r0 + rg + 32 * k) * d.n + c0 + 8 * cg;
      float v[8], wf[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = tV[buf][8 * cg + e][rg + 32 * k];
      if (d.V) st8c(AM_EXT_ORIG(d), d.V, ro, kF32, v);
      if (update_w) {
        bf16x8_to_f32(w[k], wf);
#pragma unroll
        for (int e = 0; e < 8; ++e) wf[e] -= lr * v[e];
        st8c(AM_EXT_ORIG(d), d.W, ro, kBF16, wf);
      }
    }
  };
  if (b0 >= b1) return;
  uint4 wa[2], Ua[2], ua[2], wb[2], Ub[2], ub[2];
  load(b0, wa, Ua, ua);
  for (int b = b0; b < b1; b += 2) {
    if (b + 1 < b1) load(b + 1, wb, Ub, ub);
    process(b, 0, wa, Ua, ua);
    if (b + 1 >= b1) break;
    if (b + 2 < b1) load(b + 2, wa, Ua, ua);
    process(b + 1, 1, wb, Ub, ub);
  }
}

// ============================================================================
// Flat streaming variants for matrices whose rows are contiguous and a
// multiple of 8 elements long (no transposition needed): a block walks
// kEwTilesPerCta chunks of kFlatChunk consecutive elements, each thread
// moving two 8-element groups per chunk with 16-byte accesses.  Partials:
// one slot per chunk, like the tiled kernels' one slot per tile.
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_prologue_flat(const MatTable t, int mode, float mu, int nesterov, int want_w2, double* partials) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t total = d.m * d.n;
  const int64_t c0 = (int64_t)(blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  for (int64_t c = c0; c < c0 + kEwTilesPerCta && c * kFlatChunk < total; ++c) {
    float su2 = 0.f, sw2 = 0.f;
    float g[2][8], m[2][8], w[2][8];
    bool in[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = c * kFlatChunk + 8 * (threadIdx.x + kEwThreads * k);
      in[k] = e < total;
#pragma unroll
      for (int q = 0; q < 8; ++q) g[k][q] = m[k][q] = w[k][q] = 0.f;
      if (!in[k]) continue;
      ld8c(AM_EXT_ORIG(d), d.G, e, t.grad_dtype, g[k]);
      if (mode == 0) {
        ld8c(AM_EXT_ORIG(d), d.M, e, kF32, m[k]);
        if (want_w2) ld8c(AM_EXT_ORIG(d), d.W, e, t.param_dtype, w[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (!in[k]) continue;
      const int64_t e = c * kFlatChunk + 8 * (threadIdx.x + kEwThreads * k);
      float u[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (mode == 0) {
          m[k][q] = m[k][q] + (1.f - mu) * (g[k][q] - m[k][q]);
          u[q] = nesterov ? g[k][q] + mu * (m[k][q] - g[k][q]) : m[k][q];
        } else {
          u[q] = g[k][q];
        }
        su2 += u[q] * u[q];
        sw2 += w[k][q] * w[k][q];
      }
      if (mode == 0) st8c(AM_EXT_ORIG(d), d.M, e, kF32, m[k]);
      st8c(AM_EXT_X(d), d.uX, e, t.ns_dtype, u);
    }
    if (AM_IN(c, 1, d.nslots)) warp_partials(partials, d.part + c, 2, su2, sw2);
  }
}

__global__ void __launch_bounds__(kEwThreads)
k_scale_cols_flat(const MatTable t, double* partials) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t total = d.s * d.l;
  const int64_t c0 = (int64_t)(blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  // column of each of this thread's two 8-groups, advanced chunk by chunk
  // (one division per block instead of one per group)
  const int64_t step = kFlatChunk % d.l;
  int64_t col[2] = {(c0 * kFlatChunk + 8 * threadIdx.x) % d.l,
                    (c0 * kFlatChunk + 8 * (threadIdx.x + kEwThreads)) % d.l};
  for (int64_t c = c0; c < c0 + kEwTilesPerCta && c * kFlatChunk < total; ++c) {
    float s2 = 0.f;
    float x[2][8], dj[2][8];
    bool in[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = c * kFlatChunk + 8 * (threadIdx.x + kEwThreads * k);
      in[k] = e < total;
      if (in[k]) {
        ld8c(AM_EXT_X(d), d.uX, e, t.ns_dtype, x[k]);
        ld8c(d.l, d.D, col[k], kF32, dj[k]);
      }
      col[k] += step;
      if (col[k] >= d.l) col[k] -= d.l;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (!in[k]) continue;
      const int64_t e = c * kFlatChunk + 8 * (threadIdx.x + kEwThreads * k);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        x[k][q] *= dj[k][q];
        s2 += x[k][q] * x[k][q];
      }
      st8c(AM_EXT_X(d), d.X0, e, t.ns_dtype, x[k]);
    }
    if (AM_IN(c, 1, d.nslots)) warp_partials(partials, d.part + c, 1, s2, 0.f);
  }
}

// bf16 Newton-Schulz storage, rows contiguous: X0 = uX diag(D) by column
// strips.  A block owns kStripCols columns (8 per thread) over kStripRows
// rows; each thread loads its 8 column scales once and walks its columns down
// the rows, four rows' loads in flight, one 16-byte load and one store per
// row (the chunk-wise kernel above re-reads the scales for every 8 elements;
// its bf16 form ran at 77% of HBM against this one's 100% under ncu).
// Partial |X0|^2 per warp, one slot per block.
__global__ void __launch_bounds__(kEwThreads, 4)
k_scale_cols_strip_bf16(const MatTable t, double* partials) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t strips = (d.l + kStripCols - 1) / kStripCols;
  const int64_t b = blockIdx.x - t.blk_prefix[mi];
  const int64_t j = (b % strips) * kStripCols + 8 * threadIdx.x;
  const int64_t i0 = (b / strips) * kStripRows, i1 = min(d.s, i0 + kStripRows);
  const __nv_bfloat16* uX = reinterpret_cast<const __nv_bfloat16*>(d.uX);
  float s2 = 0.f;
  if (j < d.l) {                                     // l is a multiple of 8: the whole group is inside
    float dd[8];
    ld8c(d.l, d.D, j, kF32, dd);
    for (int64_t i = i0; i < i1; i += 4) {
      uint4 x[4];
#pragma unroll
      for (int r = 0; r < 4; ++r)
        x[r] = i + r < i1 ? LDG8BF(AM_EXT_X(d), uX, (i + r) * d.ldl + j) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (i + r >= i1) break;
        float v[8];
        bf16x8_to_f32(x[r], v);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          v[q] *= dd[q];
          s2 += v[q] * v[q];
        }
        st8c(AM_EXT_X(d), d.X0, (i + r) * d.ldl + j, kBF16, v);
      }
    }
  }
  if (AM_IN(b, 1, d.nslots)) warp_partials(partials, d.part + b, 1, s2, 0.f);
}

__global__ void __launch_bounds__(kEwThreads)
k_dots_flat(const MatTable t, double* partials) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t total = d.s * d.l;
  const int64_t c0 = (int64_t)(blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  for (int64_t c = c0; c < c0 + kEwTilesPerCta && c * kFlatChunk < total; ++c) {
    float a = 0.f, cc = 0.f;
    float U[2][8], u[2][8];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = c * kFlatChunk + 8 * (threadIdx.x + kEwThreads * k);
#pragma unroll
      for (int q = 0; q < 8; ++q) U[k][q] = u[k][q] = 0.f;
      if (e < total) {
        ld8c(AM_EXT_X(d), d.UX, e, t.ns_dtype, U[k]);
        ld8c(AM_EXT_X(d), d.uX, e, t.ns_dtype, u[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        a += U[k][q] * U[k][q];
        cc += U[k][q] * u[k][q];
      }
    if (AM_IN(c, 1, d.nslots)) warp_partials(partials, d.part + c, 2, a, cc);
  }
}

__global__ void __launch_bounds__(kEwThreads)
k_epilogue_flat(const MatTable t, float lr, int update_w, const double* scal) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t total = d.m * d.n;
  const float cU = (float)scal[d.idx * S_COUNT + S_COEF_U];
  const float cu = (float)scal[d.idx * S_COUNT + S_COEF_u];
  const bool need_U = cU != 0.f, need_u = cu != 0.f;
  const int64_t c0 = (int64_t)(blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  for (int64_t c = c0; c < c0 + kEwTilesPerCta && c * kFlatChunk < total; ++c) {
    float U[2][8], u[2][8], w[2][8];
    bool in[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = c * kFlatChunk + 8 * (threadIdx.x + kEwThreads * k);
      in[k] = e < total;
#pragma unroll
      for (int q = 0; q < 8; ++q) U[k][q] = u[k][q] = w[k][q] = 0.f;
      if (!in[k]) continue;
      if (need_U) ld8c(AM_EXT_X(d), d.UX, e, t.ns_dtype, U[k]);
      if (need_u) ld8c(AM_EXT_X(d), d.uX, e, t.ns_dtype, u[k]);
      if (update_w) ld8c(AM_EXT_ORIG(d), d.W, e, t.param_dtype, w[k]);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (!in[k]) continue;
      const int64_t e = c * kFlatChunk + 8 * (threadIdx.x + kEwThreads * k);
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[q] = cU * U[k][q] + cu * u[k][q];
        w[k][q] -= lr * v[q];
      }
      if (d.V) st8c(AM_EXT_ORIG(d), d.V, e, kF32, v);
      if (update_w) st8c(AM_EXT_ORIG(d), d.W, e, t.param_dtype, w[k]);
    }
  }
}

// Optimizer-step prologue for tall matrices whose edges are multiples of 64,
// bf16 grads, params and Newton-Schulz storage: the same arithmetic as
// k_prologue with each tile's loads issued while the previous tile is
// processed, and two shared tiles (one barrier per tile).
__global__ void __launch_bounds__(kEwThreads, 2)
k_prologue_tall_bf16(const MatTable t, float mu, int nesterov, int want_w2, double* partials) {
  __shared__ float tile[2][kTile][kTile + 1];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t tiles_c = d.n / kTile;
  const int nt = (int)((d.m / kTile) * tiles_c);
  const int b0 = (blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  const int b1 = min(b0 + kEwTilesPerCta, nt);
  const int rg = threadIdx.x >> 3, cg = threadIdx.x & 7;
  const __nv_bfloat16* G = reinterpret_cast<const __nv_bfloat16*>(d.G);
  const __nv_bfloat16* W = reinterpret_cast<const __nv_bfloat16*>(d.W);
  struct Raw { uint4 g[2]; float4 m[2][2]; uint4 w[2]; };
  auto load = [&](int b, Raw& r) {
    const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = (r0 + rg + 32 * k) * d.n + c0 + 8 * cg;
      r.g[k] = LDG8BF(AM_EXT_ORIG(d), G, e);
      if (AM_IN(e, 8, AM_EXT_ORIG(d))) {
        r.m[k][0] = reinterpret_cast<const float4*>(d.M + e)[0];
        r.m[k][1] = reinterpret_cast<const float4*>(d.M + e)[1];
      } else {
        r.m[k][0] = r.m[k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      r.w[k] = want_w2 ? LDG8BF(AM_EXT_ORIG(d), W, e) : make_uint4(0, 0, 0, 0);
    }
  };
  auto process = [&](int b, int buf, const Raw& r) {
    const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
    float g[2][8], m[2][8], w[2][8], u[2][8];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      bf16x8_to_f32(r.g[k], g[k]);
      bf16x8_to_f32(r.w[k], w[k]);
      m[k][0] = r.m[k][0].x; m[k][1] = r.m[k][0].y; m[k][2] = r.m[k][0].z; m[k][3] = r.m[k][0].w;
      m[k][4] = r.m[k][1].x; m[k][5] = r.m[k][1].y; m[k][6] = r.m[k][1].z; m[k][7] = r.m[k][1].w;
    }
    float su2 = 0.f, sw2 = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        m[k][e] = m[k][e] + (1.f - mu) * (g[k][e] - m[k][e]);
        u[k][e] = nesterov ? g[k][e] + mu * (m[k][e] - g[k][e]) : m[k][e];
      }
      su2 += u[0][e] * u[0][e] + u[1][e] * u[1][e];
      sw2 += w[0][e] * w[0][e] + w[1][e] * w[1][e];
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      st8c(AM_EXT_ORIG(d), d.M, (r0 + rg + 32 * k) * d.n + c0 + 8 * cg, kF32, m[k]);
#pragma unroll
      for (int e = 0; e < 8; ++e) tile[buf][rg + 32 * k][8 * cg + e] = u[k][e];
    }
    __syncthreads();
    // X row = original column c0 + xr; X columns = original rows r0 + 8 cg ..
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int xr = rg + 32 * k;
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = tile[buf][8 * cg + e][xr];
      st8c(AM_EXT_X(d), d.uX, (c0 + xr) * d.ldl + r0 + 8 * cg, kBF16, v);
    }
    if (AM_IN(b, 1, d.nslots)) warp_partials(partials, d.part + b, 2, su2, sw2);
  };
  if (b0 >= b1) return;
  Raw ra, rb;
  load(b0, ra);
  for (int b = b0; b < b1; b += 2) {
    if (b + 1 < b1) load(b + 1, rb);
    process(b, 0, ra);
    if (b + 1 >= b1) break;
    if (b + 2 < b1) load(b + 2, ra);
    process(b + 1, 1, rb);
  }
}

// bf16 params and bf16 Newton-Schulz storage: the same flat epilogue with
// each chunk's loads issued while the previous chunk is processed.
__global__ void __launch_bounds__(kEwThreads)
k_epilogue_flat_bf16(const MatTable t, float lr, int update_w, const double* scal) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int64_t total = d.m * d.n;
  const float cU = (float)scal[d.idx * S_COUNT + S_COEF_U];
  const float cu = (float)scal[d.idx * S_COUNT + S_COEF_u];
  const bool need_U = cU != 0.f, need_u = cu != 0.f;
  const int64_t c0 = (int64_t)(blockIdx.x - t.blk_prefix[mi]) * kEwTilesPerCta;
  const int64_t c1 = min(c0 + kEwTilesPerCta, (total + kFlatChunk - 1) / kFlatChunk);
  const __nv_bfloat16* UX = reinterpret_cast<const __nv_bfloat16*>(d.UX);
  const __nv_bfloat16* uX = reinterpret_cast<const __nv_bfloat16*>(d.uX);
  const __nv_bfloat16* W = reinterpret_cast<const __nv_bfloat16*>(d.W);
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  // element offset of group k of chunk c for this thread (total is a multiple of 8)
  auto off = [&](int64_t c, int k) { return c * kFlatChunk + 8 * (threadIdx.x + kEwThreads * k); };
  auto load = [&](int64_t c, uint4 (&a)[2], uint4 (&b)[2], uint4 (&w)[2]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = off(c, k);
      const bool in = e < total;
      a[k] = in && need_U ? LDG8BF(AM_EXT_X(d), UX, e) : z4;
      b[k] = in && need_u ? LDG8BF(AM_EXT_X(d), uX, e) : z4;
      w[k] = in && update_w ? LDG8BF(AM_EXT_ORIG(d), W, e) : z4;
    }
  };
  auto process = [&](int64_t c, const uint4 (&a)[2], const uint4 (&b)[2], const uint4 (&w)[2]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = off(c, k);
      if (e >= total) continue;
      float U[8], u[8], wf[8], v[8];
      bf16x8_to_f32(a[k], U);
      bf16x8_to_f32(b[k], u);
      bf16x8_to_f32(w[k], wf);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[q] = cU * U[q] + cu * u[q];
        wf[q] -= lr * v[q];
      }
      if (d.V) st8c(AM_EXT_ORIG(d), d.V, e, kF32, v);
      if (update_w) st8c(AM_EXT_ORIG(d), d.W, e, kBF16, wf);
    }
  };
  if (c0 >= c1) return;
  uint4 aa[2], ba[2], wa[2], ab[2], bb[2], wb[2];
  load(c0, aa, ba, wa);
  for (int64_t c = c0; c < c1; c += 2) {
    if (c + 1 < c1) load(c + 1, ab, bb, wb);
    process(c, aa, ba, wa);
    if (c + 1 >= c1) break;
    if (c + 2 < c1) load(c + 2, aa, ba, wa);
    process(c + 1, ab, bb, wb);
  }
}

// ============================================================================
// u/w floor on caller-provided fp32 updates (entry point uw_floor_apply):
// partial |W|^2 and |V|^2 over the flat original layout (4096 elements per
// block, 16-byte accesses), then V *= coef.
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_sumsq_wv(const MatTable t, double* partials) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const int64_t total = d.m * d.n;
  float sw = 0.f, sv = 0.f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int64_t e0 = (int64_t)b * 4096 + 8 * (threadIdx.x + 256 * k);
    if (e0 < total) {
      float w[8], v[8];
      ld8rc(AM_EXT_ORIG(d), d.W, 0, e0, total, true, t.param_dtype, w);
      ld8rc(AM_EXT_ORIG(d), d.V, 0, e0, total, true, kF32, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sw += w[e] * w[e];
        sv += v[e] * v[e];
      }
    }
  }
  if (AM_IN(b, 1, d.nslots)) warp_partials(partials, d.part + b, 2, sv, sw);
}

__global__ void __launch_bounds__(kEwThreads)
k_scale_v(const MatTable t, const double* scal) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const float c = (float)scal[d.idx * S_COUNT + S_COEF_U];
  if (c == 1.f) return;
  const int64_t total = d.m * d.n;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int64_t e0 = (int64_t)b * 4096 + 8 * (threadIdx.x + 256 * k);
    if (e0 < total) {
      float v[8];
      ld8rc(AM_EXT_ORIG(d), d.V, 0, e0, total, true, kF32, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] *= c;
      st8rc(AM_EXT_ORIG(d), d.V, 0, e0, total, true, kF32, v);
    }
  }
}

// rho (double, scalar block) -> bucket-ordered float slot for the GEMMs.
__global__ void k_copy_rho(const MatTable t, const double* scal) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= t.count) return;
  const MatDesc& d = t.mats[k];
  *d.rho_slot = (float)scal[d.idx * S_COUNT + S_RHO];
}

__global__ void k_sigma_out(const MatTable t, const double* scal, float* sigma_out) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= t.count) return;
  sigma_out[t.mats[k].idx] = (float)scal[t.mats[k].idx * S_COUNT + S_SIGMA];
}

AM_CHECK_READER(read_and_clear_check_elementwise)

// Tests the element range [5, 6) against an extent of 4 and touches no
// memory: in the checked build the test fails and is recorded.
__global__ void k_bounds_selftest() {
  const int64_t first = 5 + (int64_t)threadIdx.x;
  if (!AM_IN(first, 1, 4)) return;
}

cudaError_t launch_bounds_selftest(cudaStream_t st) {
  k_bounds_selftest<<<1, 1, 0, st>>>();
  return cudaGetLastError();
}

// ============================================================================
// launch wrappers
// ============================================================================
cudaError_t launch_prologue(const MatTable& t, int nblk, int mode, float mu, int nesterov,
                            int want_w2, double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_prologue<<<nblk, kEwThreads, 0, st>>>(t, mode, mu, nesterov, want_w2, partials);
  return cudaGetLastError();
}
cudaError_t launch_finalize_sums(const MatTable& t, const double* partials, int nq, int slot0,
                                 int slot1, double* scal, cudaStream_t st) {
  if (t.count == 0) return cudaSuccess;
  k_finalize_sums<<<t.count, 256, 0, st>>>(t, partials, nq, slot0, slot1, scal);
  return cudaGetLastError();
}
cudaError_t launch_prologue_flat(const MatTable& t, int nblk, int mode, float mu, int nesterov, int want_w2,
                                 double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_prologue_flat<<<nblk, kEwThreads, 0, st>>>(t, mode, mu, nesterov, want_w2, partials);
  return cudaGetLastError();
}
cudaError_t launch_scale_cols_flat(const MatTable& t, int nblk, double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_scale_cols_flat<<<nblk, kEwThreads, 0, st>>>(t, partials);
  return cudaGetLastError();
}
cudaError_t launch_dots_flat(const MatTable& t, int nblk, double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_dots_flat<<<nblk, kEwThreads, 0, st>>>(t, partials);
  return cudaGetLastError();
}
cudaError_t launch_epilogue_flat(const MatTable& t, int nblk, float lr, int update_w, const double* scal,
                                 cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_epilogue_flat<<<nblk, kEwThreads, 0, st>>>(t, lr, update_w, scal);
  return cudaGetLastError();
}
cudaError_t launch_colnorm(const MatTable& t, int nblk, float pp_eps, float beta, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_colnorm<<<nblk, kEwThreads, 0, st>>>(t, pp_eps, beta);
  return cudaGetLastError();
}
cudaError_t launch_colsq_partial(const MatTable& t, int nblk, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_colsq_partial<<<nblk, kEwThreads, 0, st>>>(t);
  return cudaGetLastError();
}
cudaError_t launch_colsq_update(const MatTable& t, int nblk, int mode, float pp_eps, float beta, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_colsq_update<<<nblk, kColStrip, 0, st>>>(t, mode, mode == 0 ? kColsqRows : 32, pp_eps, beta);
  return cudaGetLastError();
}
cudaError_t launch_scale_cols(const MatTable& t, int nblk, double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_scale_cols<<<nblk, kEwThreads, 0, st>>>(t, partials);
  return cudaGetLastError();
}
cudaError_t launch_scalars(const MatTable& t, int op, int src_slot, float ns_eps, float contra,
                           float target_uw, double* scal, cudaStream_t st) {
  if (t.count == 0) return cudaSuccess;
  k_scalars<<<(t.count + 127) / 128, 128, 0, st>>>(t, op, src_slot, ns_eps, contra, target_uw, scal);
  return cudaGetLastError();
}
cudaError_t launch_matvec(const MatTable& t, int nblk, int dir, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_matvec<<<nblk, kEwThreads, 0, st>>>(t, dir);
  return cudaGetLastError();
}
cudaError_t launch_vecop(const MatTable& t, int which, int mode, int len_is_s_when_flag0,
                         double* scal, cudaStream_t st) {
  if (t.count == 0) return cudaSuccess;
  k_vecop<<<t.count, 256, 0, st>>>(t, which, mode, len_is_s_when_flag0, scal);
  return cudaGetLastError();
}
cudaError_t launch_dots(const MatTable& t, int nblk, double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_dots<<<nblk, kEwThreads, 0, st>>>(t, partials);
  return cudaGetLastError();
}
cudaError_t launch_epilogue(const MatTable& t, int nblk, float lr, int update_w, const double* scal,
                            cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_epilogue<<<nblk, kEwThreads, 0, st>>>(t, lr, update_w, scal);
  return cudaGetLastError();
}
cudaError_t launch_prologue_tall_bf16(const MatTable& t, int nblk, float mu, int nesterov, int want_w2,
                                      double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_prologue_tall_bf16<<<nblk, kEwThreads, 0, st>>>(t, mu, nesterov, want_w2, partials);
  return cudaGetLastError();
}
cudaError_t launch_scale_cols_strip_bf16(const MatTable& t, int nblk, double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_scale_cols_strip_bf16<<<nblk, kEwThreads, 0, st>>>(t, partials);
  return cudaGetLastError();
}
cudaError_t launch_epilogue_flat_bf16(const MatTable& t, int nblk, float lr, int update_w, const double* scal,
                                      cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_epilogue_flat_bf16<<<nblk, kEwThreads, 0, st>>>(t, lr, update_w, scal);
  return cudaGetLastError();
}
cudaError_t launch_epilogue_tall_bf16(const MatTable& t, int nblk, float lr, int update_w, const double* scal,
                                      cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_epilogue_tall_bf16<<<nblk, kEwThreads, 0, st>>>(t, lr, update_w, scal);
  return cudaGetLastError();
}
cudaError_t launch_sumsq_wv(const MatTable& t, int nblk, double* partials, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_sumsq_wv<<<nblk, kEwThreads, 0, st>>>(t, partials);
  return cudaGetLastError();
}
cudaError_t launch_scale_v(const MatTable& t, int nblk, const double* scal, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_scale_v<<<nblk, kEwThreads, 0, st>>>(t, scal);
  return cudaGetLastError();
}

cudaError_t launch_sigma_out(const MatTable& t, const double* scal, float* sigma_out, cudaStream_t st) {
  if (t.count == 0) return cudaSuccess;
  k_sigma_out<<<(t.count + 127) / 128, 128, 0, st>>>(t, scal, sigma_out);
  return cudaGetLastError();
}
cudaError_t launch_copy_rho(const MatTable& t, const double* scal, cudaStream_t st) {
  if (t.count == 0) return cudaSuccess;
  k_copy_rho<<<(t.count + 127) / 128, 128, 0, st>>>(t, scal);
  return cudaGetLastError();
}

}  // namespace am
