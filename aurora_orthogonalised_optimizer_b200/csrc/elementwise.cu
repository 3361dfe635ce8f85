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
constexpr int kEwThreads = 256; // 64 columns x 4 row lanes

// ============================================================================
// prologue: m <- m + (1-mu)(g-m); u = Nesterov ? g + mu(m-g) : m; write u in
// the X orientation (transposed through shared memory for tall matrices);
// per-block partials of |u|^2 and |W|^2.
// mode 0: optimizer step (uses G, M, W);  mode 1: u = G (input staging).
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_prologue(const MatTable t, int mode, float mu, int nesterov, int want_w2, double* partials) {
  __shared__ float tile[kTile][kTile + 1];
  __shared__ double red[32];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const int64_t tiles_c = (d.n + kTile - 1) / kTile;
  const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
  float su2 = 0.f, sw2 = 0.f;
  const int64_t j = c0 + tx;
#pragma unroll 4
  for (int rr = ty; rr < kTile; rr += 4) {
    const int64_t i = r0 + rr;
    float u = 0.f;
    if (i < d.m && j < d.n) {
      const int64_t e = i * d.n + j;
      const float g = ld_as_f32(d.G, e, t.grad_dtype);
      if (mode == 0) {
        const float m0 = d.M[e];
        const float m1 = m0 + (1.f - mu) * (g - m0);
        d.M[e] = m1;
        u = nesterov ? g + mu * (m1 - g) : m1;
        if (want_w2) { const float w = ld_as_f32(d.W, e, t.param_dtype); sw2 += w * w; }
      } else {
        u = g;
      }
      su2 += u * u;
      if (!d.tall) st_from_f32(d.uX, i * d.ldl + j, t.ns_dtype, u);
    }
    tile[rr][tx] = u;
  }
  if (d.tall) {
    __syncthreads();
    // X row = original column c0 + rr, X column = original row r0 + tx
#pragma unroll 4
    for (int rr = ty; rr < kTile; rr += 4) {
      const int64_t xi = c0 + rr, xj = r0 + tx;
      if (xi < d.n && xj < d.m) st_from_f32(d.uX, xi * d.ldl + xj, t.ns_dtype, tile[tx][rr]);
    }
  }
  const double a = block_sum((double)su2, red);
  const double w = block_sum((double)sw2, red);
  if (threadIdx.x == 0) {
    partials[(int64_t)(d.part + b) * 2 + 0] = a;
    partials[(int64_t)(d.part + b) * 2 + 1] = w;
  }
}

// Sum the per-block partials of each matrix into its scalar block.
// partials are laid out [slot q of nq] per block.  dst_slot[q] < 0 skips q.
__global__ void k_finalize_sums(const MatTable t, const double* partials, int nq, int slot0,
                                int slot1, double* scal) {
  __shared__ double red[32];
  const MatDesc& d = t.mats[blockIdx.x];
  for (int q = 0; q < nq; ++q) {
    const int slot = q == 0 ? slot0 : slot1;
    double s = 0.0;
    for (int b = threadIdx.x; b < d.nblk; b += blockDim.x) s += partials[(int64_t)(d.part + b) * nq + q];
    s = block_sum(s, red);
    if (threadIdx.x == 0 && slot >= 0) scal[d.idx * S_COUNT + slot] = s;
  }
}

// ============================================================================
// Column reductions over the X orientation (s x l): per column j of X
// (= a row of the tall-oriented matrix), sum_i X_ij^2.
//   mode 0 (D init):  D_j = 1 / max(sqrt(sum), pp_eps)              ["源码实现"]
//   mode 1 (D update): row_sq = max(sum, pp_eps^2);
//                      D_j *= (target / row_sq)^beta, target = s / l
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_colnorm(const MatTable t, int mode, float pp_eps, float beta) {
  __shared__ float part[4][kTile];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
  const int64_t j = (int64_t)b * kTile + tx;
  const void* X = mode == 0 ? d.uX : d.UX;
  float acc = 0.f;
  if (j < d.l)
    for (int64_t i = ty; i < d.s; i += 4) {
      const float x = ld_as_f32(X, i * d.ldl + j, t.ns_dtype);
      acc += x * x;
    }
  part[ty][tx] = acc;
  __syncthreads();
  if (ty == 0 && j < d.l) {
    const float sum = ((part[0][tx] + part[1][tx]) + part[2][tx]) + part[3][tx];
    if (mode == 0) {
      d.D[j] = 1.f / fmaxf(sqrtf(sum), pp_eps);
    } else {
      const float row_sq = fmaxf(sum, pp_eps * pp_eps);
      const float target = (float)d.s / (float)d.l;
      d.D[j] = d.D[j] * powf(target / row_sq, beta);
    }
  }
}

// X0 = uX * diag(D) in the NS dtype, with per-block partials of |X0|^2.
__global__ void __launch_bounds__(kEwThreads)
k_scale_cols(const MatTable t, double* partials) {
  __shared__ double red[32];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const int64_t tiles_c = (d.l + kTile - 1) / kTile;
  const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
  const int64_t j = c0 + tx;
  float s2 = 0.f;
  if (j < d.l) {
    const float dj = d.D[j];
    for (int rr = ty; rr < kTile; rr += 4) {
      const int64_t i = r0 + rr;
      if (i < d.s) {
        const float x = ld_as_f32(d.uX, i * d.ldl + j, t.ns_dtype) * dj;
        s2 += x * x;
        st_from_f32(d.X0, i * d.ldl + j, t.ns_dtype, x);
      }
    }
  }
  const double a = block_sum((double)s2, red);
  if (threadIdx.x == 0) partials[d.part + b] = a;
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
//   flag 1 (col dot):  out_j = sum_i Q_ij y_i   (y length s, out length l)
// `dir` selects vec0 -> vec1 (0) or vec1 -> vec0 (1).
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_matvec(const MatTable t, int dir) {
  __shared__ float part[4][kTile];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const float* in = dir == 0 ? d.vec0 : d.vec1;
  float* out = dir == 0 ? d.vec1 : d.vec0;
  if (d.flag == 0) {
    // 8 warps, one row each
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t i = (int64_t)b * 8 + w;
    if (i < d.s) {
      float acc = 0.f;
      for (int64_t j = lane; j < d.l; j += 32) acc += ld_as_f32(d.uX, i * d.ldl + j, t.ns_dtype) * in[j];
      acc = warp_sum(acc);
      if (lane == 0) out[i] = acc;
    }
  } else {
    const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
    const int64_t j = (int64_t)b * kTile + tx;
    float acc = 0.f;
    if (j < d.l)
      for (int64_t i = ty; i < d.s; i += 4) acc += ld_as_f32(d.uX, i * d.ldl + j, t.ns_dtype) * in[i];
    part[ty][tx] = acc;
    __syncthreads();
    if (ty == 0 && j < d.l) out[j] = ((part[0][tx] + part[1][tx]) + part[2][tx]) + part[3][tx];
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
// <U,U> and <U,u> over the X orientation, per-block partials (2 per block).
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_dots(const MatTable t, double* partials) {
  __shared__ double red[32];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const int64_t tiles_c = (d.l + kTile - 1) / kTile;
  const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
  const int64_t j = c0 + tx;
  float a = 0.f, c = 0.f;
  if (j < d.l)
    for (int rr = ty; rr < kTile; rr += 4) {
      const int64_t i = r0 + rr;
      if (i < d.s) {
        const float U = ld_as_f32(d.UX, i * d.ldl + j, t.ns_dtype);
        const float u = ld_as_f32(d.uX, i * d.ldl + j, t.ns_dtype);
        a += U * U;
        c += U * u;
      }
    }
  const double A = block_sum((double)a, red);
  const double C = block_sum((double)c, red);
  if (threadIdx.x == 0) {
    partials[(int64_t)(d.part + b) * 2 + 0] = A;
    partials[(int64_t)(d.part + b) * 2 + 1] = C;
  }
}

// ============================================================================
// Fused epilogue, original orientation: V = cU U + cu u (U, u read from the
// X orientation, transposed through shared memory for tall matrices);
// optional fp32 V output; optional W <- W - lr V in the param dtype.
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_epilogue(const MatTable t, float lr, int update_w, const double* scal) {
  __shared__ float tU[kTile][kTile + 1];
  __shared__ float tu[kTile][kTile + 1];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const int64_t tiles_c = (d.n + kTile - 1) / kTile;
  const int64_t r0 = (b / tiles_c) * kTile, c0 = (b % tiles_c) * kTile;
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
  const float cU = (float)scal[d.idx * S_COUNT + S_COEF_U];
  const float cu = (float)scal[d.idx * S_COUNT + S_COEF_u];
  const bool need_u = cu != 0.f;
  if (d.tall) {
    // X tile rows = original columns c0.., X tile cols = original rows r0..
    for (int rr = ty; rr < kTile; rr += 4) {
      const int64_t xi = c0 + rr, xj = r0 + tx;
      const bool in = xi < d.n && xj < d.m;
      tU[rr][tx] = in && cU != 0.f ? ld_as_f32(d.UX, xi * d.ldl + xj, t.ns_dtype) : 0.f;
      tu[rr][tx] = in && need_u ? ld_as_f32(d.uX, xi * d.ldl + xj, t.ns_dtype) : 0.f;
    }
    __syncthreads();
  }
  const int64_t j = c0 + tx;
  for (int rr = ty; rr < kTile; rr += 4) {
    const int64_t i = r0 + rr;
    if (i >= d.m || j >= d.n) continue;
    float U, u;
    if (d.tall) {
      U = tU[tx][rr];
      u = tu[tx][rr];
    } else {
      U = cU != 0.f ? ld_as_f32(d.UX, i * d.ldl + j, t.ns_dtype) : 0.f;
      u = need_u ? ld_as_f32(d.uX, i * d.ldl + j, t.ns_dtype) : 0.f;
    }
    const float v = cU * U + cu * u;
    const int64_t e = i * d.n + j;
    if (d.V) d.V[e] = v;
    if (update_w) {
      const float w = ld_as_f32(d.W, e, t.param_dtype);
      st_from_f32(d.W, e, t.param_dtype, w - lr * v);
    }
  }
}

// ============================================================================
// u/w floor on caller-provided fp32 updates (entry point uw_floor_apply):
// partial |W|^2 and |V|^2 over the original orientation, then V *= coef.
// ============================================================================
__global__ void __launch_bounds__(kEwThreads)
k_sumsq_wv(const MatTable t, double* partials) {
  __shared__ double red[32];
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const int64_t total = d.m * d.n;
  float sw = 0.f, sv = 0.f;
  for (int64_t e = (int64_t)b * 4096 + threadIdx.x; e < total && e < (int64_t)(b + 1) * 4096;
       e += blockDim.x) {
    const float w = ld_as_f32(d.W, e, t.param_dtype);
    const float v = d.V[e];
    sw += w * w;
    sv += v * v;
  }
  const double W2 = block_sum((double)sw, red);
  const double V2 = block_sum((double)sv, red);
  if (threadIdx.x == 0) {
    partials[(int64_t)(d.part + b) * 2 + 0] = V2;
    partials[(int64_t)(d.part + b) * 2 + 1] = W2;
  }
}

__global__ void __launch_bounds__(kEwThreads)
k_scale_v(const MatTable t, const double* scal) {
  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int b = blockIdx.x - t.blk_prefix[mi];
  const float c = (float)scal[d.idx * S_COUNT + S_COEF_U];
  if (c == 1.f) return;
  const int64_t total = d.m * d.n;
  for (int64_t e = (int64_t)b * 4096 + threadIdx.x; e < total && e < (int64_t)(b + 1) * 4096;
       e += blockDim.x)
    d.V[e] *= c;
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
cudaError_t launch_colnorm(const MatTable& t, int nblk, int mode, float pp_eps, float beta,
                           cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  k_colnorm<<<nblk, kEwThreads, 0, st>>>(t, mode, pp_eps, beta);
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
