// opnorm_normalize_noalloc: the operator-norm normalisation of
// opnorm_normalize, for callers that cannot hand the library a workspace.
//
// Some callers cannot allocate device memory at the point where they need
// this step: code running under a framework whose memory manager owns the
// whole device (a raw cudaMalloc there fails or fragments the pool), and
// latency-bound loops that must not enter the allocator after start-up
// (cudaMalloc can synchronise the device and take unbounded time).  This
// entry point needs no workspace: its scratch (the two power-iteration
// vectors of every matrix and a per-matrix scalar block) lives in the
// file-scope device array below, which every GPU that loads the library
// holds until the process exits.
//
// The power iteration runs directly on the caller's input (its own dtype and
// orientation), so no staging copy of the matrix is needed.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "kernels.h"

namespace am {

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;   // 1 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_opnorm_scratch[kScratchBytes];

// Device address of g_opnorm_scratch on the current device, looked up once
// per device (with that device current) on the first call made on it and
// kept for the life of the process.  A cudaDeviceReset reloads the module
// and can move the array, so none may come between calls.
cudaError_t scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_opnorm_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

inline size_t round64(int64_t x) { return (size_t)((x + 63) / 64 * 64); }

}  // namespace

}  // namespace am

using namespace am;

extern "C" muon_status opnorm_normalize_noalloc(const muon_config* cfg, int n, const muon_shape* shapes,
                                                const void* const* in, int in_dtype, float* const* out,
                                                float* sigma_out, void* stream) {
  if (!cfg || cfg->power_iters < 1) return MUON_ERR_INVALID_ARG;
  if (in_dtype != MUON_F32 && in_dtype != MUON_BF16) return MUON_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && (!shapes || !in))) return MUON_ERR_INVALID_ARG;
  if (n == 0) return MUON_OK;
  if (sigma_out && ((uintptr_t)sigma_out & 15u)) return MUON_ERR_INVALID_ARG;
  // scratch layout: n scalar blocks (S_COUNT doubles), then per matrix the
  // vector over its columns and the vector over its rows (floats, 64-aligned)
  size_t need = (size_t)n * S_COUNT * sizeof(double);
  for (int i = 0; i < n; ++i) {
    const int64_t m = shapes[i].rows, k = shapes[i].cols;
    if (m <= 0 || k <= 0) return MUON_ERR_INVALID_ARG;
    // the same edge bound as the workspace entry points; it also keeps each
    // term of the sum below far from wrapping around
    if (m > (int64_t)1 << 31 || k > (int64_t)1 << 31) return MUON_ERR_INVALID_ARG;
    if (!in[i] || ((uintptr_t)in[i] & 15u)) return MUON_ERR_INVALID_ARG;
    if (out && out[i] && ((uintptr_t)out[i] & 15u)) return MUON_ERR_INVALID_ARG;
    need += sizeof(float) * (round64(k) + round64(m));
  }
  if (need > kScratchBytes) return MUON_ERR_UNSUPPORTED;   // beyond the static scratch

  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return MUON_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  double* scal = reinterpret_cast<double*>(base);
  // every call shares the scratch: start each call from a cleared scalar block
  if (cudaMemsetAsync(scal, 0, (size_t)n * S_COUNT * sizeof(double), st) != cudaSuccess) return MUON_ERR_CUDA;

  // per-matrix descriptors on the caller's input in its own orientation:
  // rows play the role of s, columns of l, v runs over the columns.
  float* vecs = reinterpret_cast<float*>(scal + (size_t)n * S_COUNT);
  size_t voff = 0;
  for (int c0 = 0; c0 < n; c0 += kMaxMatsPerLaunch) {
    const int cnt = std::min(kMaxMatsPerLaunch, n - c0);
    MatTable t;
    std::memset(&t, 0, sizeof(t));
    t.count = cnt;
    t.ns_dtype = in_dtype;
    t.param_dtype = in_dtype;
    t.grad_dtype = in_dtype;
    for (int k = 0; k < cnt; ++k) {
      const int i = c0 + k;
      MatDesc& d = t.mats[k];
      d.m = d.s = shapes[i].rows;
      d.n = d.l = shapes[i].cols;
      d.ldl = shapes[i].cols;
      d.tall = 0;
      d.idx = i;
      d.uX = const_cast<void*>(in[i]);
      d.V = out ? out[i] : nullptr;
      d.vec0 = vecs + voff;
      voff += round64(d.l);
      d.vec1 = vecs + voff;
      voff += round64(d.s);
    }
    auto blocks = [&](int pass) {   // pass 0: vector ops, 1: row dot, 2: column dot
      int tot = 0;
      for (int k = 0; k < cnt; ++k) {
        MatDesc& d = t.mats[k];
        d.flag = pass == 2 ? 1 : 0;
        d.nblk = pass == 1 ? (int)((d.s + kMatvecRowsPerCta - 1) / kMatvecRowsPerCta)
                 : pass == 2 ? (int)((d.l + kColDotStrip - 1) / kColDotStrip) : 0;
        t.blk_prefix[k] = tot;
        tot += d.nblk;
      }
      t.blk_prefix[cnt] = tot;
      return tot;
    };
    blocks(0);
    if (launch_vecop(t, 0, 0, 0, scal, st) != cudaSuccess) return MUON_ERR_CUDA;   // v = 1/sqrt(cols)
    for (int it = 0; it < cfg->power_iters; ++it) {
      int nb = blocks(1);
      if (launch_matvec(t, nb, 0, st) != cudaSuccess) return MUON_ERR_CUDA;     // t = A v
      nb = blocks(2);
      if (launch_matvec(t, nb, 1, st) != cudaSuccess) return MUON_ERR_CUDA;     // w = A^T t
      blocks(0);
      if (launch_vecop(t, 0, 1, 0, scal, st) != cudaSuccess) return MUON_ERR_CUDA;  // v = w / |w|
    }
    int nb = blocks(1);
    if (launch_matvec(t, nb, 0, st) != cudaSuccess) return MUON_ERR_CUDA;       // t = A v
    blocks(0);
    if (launch_vecop(t, 1, 2, 1, scal, st) != cudaSuccess) return MUON_ERR_CUDA;  // sigma = |t|
    if (sigma_out && launch_sigma_out(t, scal, sigma_out, st) != cudaSuccess) return MUON_ERR_CUDA;
    if (out) {
      if (launch_scalars(t, 3, 0, 0.f, 0.f, 0.f, scal, st) != cudaSuccess) return MUON_ERR_CUDA;
      int tiles = 0;
      for (int k = 0; k < cnt; ++k) {
        MatDesc& d = t.mats[k];
        d.nblk = (int)((((d.m + 63) / 64) * ((d.n + 63) / 64) + kEwTilesPerCta - 1) / kEwTilesPerCta);
        t.blk_prefix[k] = tiles;
        tiles += d.nblk;
      }
      t.blk_prefix[cnt] = tiles;
      if (launch_epilogue(t, tiles, 0.f, 0, scal, st) != cudaSuccess) return MUON_ERR_CUDA;
    }
  }
  return MUON_OK;
}
