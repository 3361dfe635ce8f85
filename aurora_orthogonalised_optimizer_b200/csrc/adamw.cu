// Auxiliary AdamW for the non-matrix parameters (token embedding, output
// projection, value embeddings, 1-D gains): one fused multi-tensor launch.
//
// Method: the Track 3 Aurora write-up ("完整的超参配置表" and the paragraph on
// where the hyper-parameters sit) hands these parameters to AdamW with betas
// (0.8, 0.95), eps 1e-10, weight_decay 0, fused; the update is the
// decoupled-weight-decay Adam of torch.optim.AdamW:
//   p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2
//   p <- p - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
//
// HBM-bound: each element is read once and written once (param, two fp32
// states) plus one gradient read.  A block owns 2048 x ITERS consecutive
// elements of one tensor; each thread moves 8-element groups with 16-byte
// accesses, all loads issued before any store.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "common.cuh"

namespace am {
namespace {

constexpr int kAwThreads = 256;
constexpr int kAwMaxTensors = 192;
// A block owns kAwThreads * 8 * ITERS consecutive elements of one tensor.
template <int ITERS>
__host__ __device__ constexpr int64_t aw_chunk() { return (int64_t)kAwThreads * 8 * ITERS; }

struct AwTensor {
  void* p;
  const void* g;
  float* m;
  float* v;
  int64_t numel;
  float step_size;    // lr / (1 - b1^t)
  float decay;        // 1 - lr wd
};

struct AwTable {
  int count;
  int param_dtype, grad_dtype;
  float beta1, beta2, eps, inv_sqrt_bc2;
  int blk_prefix[kAwMaxTensors + 1];
  AwTensor t[kAwMaxTensors];
};

__device__ __forceinline__ void adamw8(float (&p)[8], const float (&g)[8], float (&m)[8], float (&v)[8],
                                       const AwTable& T, const AwTensor& d) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    m[e] = T.beta1 * m[e] + (1.f - T.beta1) * g[e];
    v[e] = T.beta2 * v[e] + (1.f - T.beta2) * g[e] * g[e];
    const float denom = sqrtf(v[e]) * T.inv_sqrt_bc2 + T.eps;
    p[e] = p[e] * d.decay - d.step_size * (m[e] / denom);
  }
}

template <int ITERS>
__global__ void __launch_bounds__(kAwThreads) k_adamw(const AwTable T) {
  constexpr int kAwIters = ITERS;
  constexpr int64_t kAwChunk = aw_chunk<ITERS>();
  int lo = 0, hi = T.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (T.blk_prefix[mid] <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
  }
  const AwTensor& d = T.t[lo];
  const int64_t base = (int64_t)(blockIdx.x - T.blk_prefix[lo]) * kAwChunk;
  // all loads first (the four arrays may alias as far as the compiler knows)
  float p[kAwIters][8], g[kAwIters][8], m[kAwIters][8], v[kAwIters][8];
  int cnt[kAwIters];
#pragma unroll
  for (int k = 0; k < kAwIters; ++k) {
    const int64_t j = base + 8 * (threadIdx.x + kAwThreads * k);
    const int64_t left = d.numel - j;
    cnt[k] = left <= 0 ? 0 : (left >= 8 ? 8 : (int)left);
    if (cnt[k] > 0 && !AM_IN(j, cnt[k], d.numel)) cnt[k] = 0;
    if (cnt[k] == 8) {
      ld8(d.p, j, T.param_dtype, p[k]);
      ld8(d.g, j, T.grad_dtype, g[k]);
      ld8(d.m, j, kF32, m[k]);
      ld8(d.v, j, kF32, v[k]);
    } else {
      ld8m(d.p, j, T.param_dtype, cnt[k], p[k]);
      ld8m(d.g, j, T.grad_dtype, cnt[k], g[k]);
      ld8m(d.m, j, kF32, cnt[k], m[k]);
      ld8m(d.v, j, kF32, cnt[k], v[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < kAwIters; ++k) {
    if (cnt[k] == 0) continue;
    adamw8(p[k], g[k], m[k], v[k], T, d);
    const int64_t j = base + 8 * (threadIdx.x + kAwThreads * k);
    if (cnt[k] == 8) {
      st8(d.p, j, T.param_dtype, p[k]);
      st8(d.m, j, kF32, m[k]);
      st8(d.v, j, kF32, v[k]);
    } else {
      st8m(d.p, j, T.param_dtype, cnt[k], p[k]);
      st8m(d.m, j, kF32, cnt[k], m[k]);
      st8m(d.v, j, kF32, cnt[k], v[k]);
    }
  }
}

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// 8-element groups per thread: 1 by default (48 registers, 5 blocks per SM);
// AURORA_MUON_AW_ITERS=2 or 4 selects the wider variants (tuning only).
int aw_iters() {
  static const int it = [] {
    const char* e = std::getenv("AURORA_MUON_AW_ITERS");
    const int v = e ? std::atoi(e) : 1;
    return (v == 2 || v == 4) ? v : 1;
  }();
  return it;
}

}  // namespace

AM_CHECK_READER(read_and_clear_check_adamw)

}  // namespace am

using namespace am;

extern "C" {

void adamw_config_default(adamw_config* c) {
  if (!c) return;
  std::memset(c, 0, sizeof(*c));
  c->lr = 0.01f;
  c->beta1 = 0.8f;
  c->beta2 = 0.95f;
  c->eps = 1e-10f;
  c->weight_decay = 0.0f;
  c->step = 1;
  c->param_dtype = MUON_BF16;
  c->grad_dtype = MUON_BF16;
}

muon_status adamw_step(const adamw_config* cfg, int n, const int64_t* numels, const float* lrs,
                       void* const* params, const void* const* grads, float* const* exp_avg,
                       float* const* exp_avg_sq, void* stream) {
  if (!cfg || n < 0) return MUON_ERR_INVALID_ARG;
  if (cfg->step < 1 || !(cfg->beta1 >= 0.f && cfg->beta1 < 1.f) || !(cfg->beta2 >= 0.f && cfg->beta2 < 1.f) ||
      !(cfg->eps >= 0.f) || !(cfg->weight_decay >= 0.f))
    return MUON_ERR_INVALID_ARG;
  if (cfg->param_dtype < 0 || cfg->param_dtype > 1 || cfg->grad_dtype < 0 || cfg->grad_dtype > 1)
    return MUON_ERR_INVALID_ARG;
  if (n == 0) return MUON_OK;
  if (!numels || !params || !grads || !exp_avg || !exp_avg_sq) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (numels[i] < 0) return MUON_ERR_INVALID_ARG;
    if (numels[i] == 0) continue;
    if (!params[i] || !grads[i] || !exp_avg[i] || !exp_avg_sq[i]) return MUON_ERR_INVALID_ARG;
    if (!aligned16(params[i]) || !aligned16(grads[i]) || !aligned16(exp_avg[i]) || !aligned16(exp_avg_sq[i]))
      return MUON_ERR_INVALID_ARG;
  }
  const double bc1 = 1.0 - std::pow((double)cfg->beta1, (double)cfg->step);
  const double bc2 = 1.0 - std::pow((double)cfg->beta2, (double)cfg->step);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int iters = aw_iters();
  const int64_t chunk = (int64_t)kAwThreads * 8 * iters;
  int i = 0;
  while (i < n) {
    AwTable T;
    std::memset(&T, 0, sizeof(T));
    T.param_dtype = cfg->param_dtype;
    T.grad_dtype = cfg->grad_dtype;
    T.beta1 = cfg->beta1;
    T.beta2 = cfg->beta2;
    T.eps = cfg->eps;
    T.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
    int blocks = 0;
    while (i < n && T.count < kAwMaxTensors) {
      if (numels[i] > 0) {
        const double lr = lrs ? (double)lrs[i] : (double)cfg->lr;
        AwTensor& d = T.t[T.count];
        d.p = params[i];
        d.g = grads[i];
        d.m = exp_avg[i];
        d.v = exp_avg_sq[i];
        d.numel = numels[i];
        d.step_size = (float)(lr / bc1);
        d.decay = (float)(1.0 - lr * (double)cfg->weight_decay);
        T.blk_prefix[T.count] = blocks;
        blocks += (int)((numels[i] + chunk - 1) / chunk);
        ++T.count;
      }
      ++i;
    }
    T.blk_prefix[T.count] = blocks;
    if (T.count == 0) continue;
    if (iters == 4) k_adamw<4><<<blocks, kAwThreads, 0, st>>>(T);
    else if (iters == 2) k_adamw<2><<<blocks, kAwThreads, 0, st>>>(T);
    else k_adamw<1><<<blocks, kAwThreads, 0, st>>>(T);
    if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  }
  return MUON_OK;
}

}  // extern "C"
