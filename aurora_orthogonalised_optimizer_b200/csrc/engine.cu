// Host engine of libaurora_muon: argument validation, shape bucketing,
// workspace carving, the stage sequence of one optimizer step, and the C ABI
// declared in include/aurora_muon.h.
//
// Stage order of muon_step (Track 3 write-up, "组合优化栈" + "u/w-floor"):
//   prologue (momentum, Nesterov, u in X orientation, |u|^2, |W|^2)
//   [contra]  power iteration on u -> sigma
//   [aurora]  D init from the tall-oriented row norms of u
//   polar loop: scaled input X0 -> rho; ns_steps x {Gram, square, update}
//               [aurora, not last] D update from the row norms of U
//   <U,U>, <U,u> (tensor-core mode: formed by the last update GEMM of each
//   matrix's final polar) -> per-matrix coefficients -> fused epilogue
//   W <- W - lr V
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "kernels.h"

using namespace am;

namespace {

constexpr size_t kAlign = 1024;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round8(int64_t x) { return (x + 7) / 8 * 8; }
inline int64_t round64(int64_t x) { return (x + 63) / 64 * 64; }

struct MatPlan {
  int64_t m, n, s, l;
  int tall, bucket, bidx;
  int64_t part;      // first partial block slot
  int64_t gv_rows;   // fused power iteration: rows of X per item
  int64_t gv_off;    // and the offset (floats) of this matrix's item partials
};

struct BucketPlan {
  int64_t s, l, ldl, lds;
  std::vector<int> members;
  size_t off_uX, off_P, off_Q, off_A, off_B, off_D, off_v0, off_v1, off_rho;
  size_t off_dots;       // fused <U,U>, <U,u> partials of the last update GEMM (16 doubles per tile)
  size_t off_colsq;      // Aurora D: per 32-row block column sums of squares (uX, then U)
  bool colsq = false;    // the bucket has that buffer
  bool colsq_gemm = false;  // its D updates read sums the last update GEMM wrote
  int64_t dot_tiles;     // tiles per member reserved there (both tensor-core variants fit)
};

struct Plan {
  int ns_dtype = kBF16;
  int nsb = 2;
  std::vector<MatPlan> mats;
  std::vector<BucketPlan> buckets;
  size_t off_scal = 0, off_partials = 0, off_gv = 0, off_dots = 0, off_sched = 0, total = 0;
};

// Rows per item of the fused power-iteration pass: items of about
// total / (148 x 8) elements (a few waves of one block per SM), kept between
// 64 Ki and 1 Mi elements; the partial X^T z per item then costs at most
// ~2% of the item's bytes.
int64_t gv_rows_for(int64_t s, int64_t l, int64_t total_elems) {
  const int64_t item = std::min<int64_t>(std::max<int64_t>(total_elems / (148 * 8), 1 << 16), 1 << 20);
  return std::max<int64_t>(1, std::min<int64_t>(s, cdiv(item, l)));
}

int ns_dtype_of(const muon_config* c) { return c->gemm_mode == MUON_GEMM_FP32 ? kF32 : kBF16; }

Plan make_plan(const muon_config* cfg, int n, const muon_shape* shapes) {
  Plan p;
  p.ns_dtype = ns_dtype_of(cfg);
  p.nsb = dt_bytes(p.ns_dtype);
  std::map<std::pair<int64_t, int64_t>, int> bmap;
  int64_t part = 0, gv = 0, total_elems = 0;
  for (int i = 0; i < n; ++i) total_elems += shapes[i].rows * shapes[i].cols;
  for (int i = 0; i < n; ++i) {
    MatPlan mp;
    mp.m = shapes[i].rows;
    mp.n = shapes[i].cols;
    mp.s = std::min(mp.m, mp.n);
    mp.l = std::max(mp.m, mp.n);
    mp.tall = mp.m > mp.n;
    auto key = std::make_pair(mp.s, mp.l);
    auto it = bmap.find(key);
    if (it == bmap.end()) {
      BucketPlan b{};
      b.s = mp.s;
      b.l = mp.l;
      b.ldl = round8(mp.l);
      b.lds = round8(mp.s);
      p.buckets.push_back(b);
      it = bmap.emplace(key, (int)p.buckets.size() - 1).first;
    }
    mp.bucket = it->second;
    mp.bidx = (int)p.buckets[mp.bucket].members.size();
    p.buckets[mp.bucket].members.push_back(i);
    mp.part = part;
    const int64_t tiles = cdiv(mp.m, 64) * cdiv(mp.n, 64);
    part += std::max(tiles, cdiv(mp.m * mp.n, 4096));
    mp.gv_rows = gv_rows_for(mp.s, mp.l, total_elems);
    mp.gv_off = gv;
    gv += cdiv(mp.s, mp.gv_rows) * round8(mp.l);
    p.mats.push_back(mp);
  }
  size_t off = 0;
  for (auto& b : p.buckets) {
    const size_t cnt = b.members.size();
    const size_t xbytes = cnt * (size_t)b.s * (size_t)b.ldl * p.nsb;
    const size_t abytes = cnt * (size_t)b.s * (size_t)b.lds * p.nsb;
    b.off_uX = off; off = align_up(off + xbytes);
    b.off_P = off;  off = align_up(off + xbytes);
    b.off_Q = off;  off = align_up(off + xbytes);
    b.off_A = off;  off = align_up(off + abytes);
    b.off_B = off;  off = align_up(off + abytes);
    const size_t vbytes = cnt * (size_t)round64(b.l) * 4;   // per-matrix vectors, 256-byte aligned
    b.off_D = off;  off = align_up(off + vbytes);
    b.off_v0 = off; off = align_up(off + vbytes);
    b.off_v1 = off; off = align_up(off + vbytes);
    b.off_rho = off; off = align_up(off + cnt * 4);
  }
  // per-tile reduction slots of the fused dots (tensor-core mode only)
  p.off_dots = off;
  for (auto& b : p.buckets) {
    int tm, tn;
    b.dot_tiles = 0;
    if (cfg->gemm_mode == MUON_GEMM_BF16)
      b.dot_tiles = std::max(tc_tile_count(GK_UPD, (int)b.s, (int)b.l, true, &tm, &tn),
                             tc_tile_count(GK_UPD, (int)b.s, (int)b.l, false, &tm, &tn));
    b.off_dots = off;
    off = align_up(off + b.members.size() * (size_t)b.dot_tiles * 16 * sizeof(double));
  }
  // column sums of squares per row block for Aurora's D (non-square
  // buckets), sized for 32-row blocks: formed from uX for the D init; for the
  // D updates, written by the last update GEMM of each non-final polar in the
  // tensor-core mode
  for (auto& b : p.buckets) {
    b.colsq = cfg->aurora && b.s != b.l;
    b.colsq_gemm = b.colsq && cfg->gemm_mode == MUON_GEMM_BF16 && cfg->pp_iterations > 1;
    b.off_colsq = off;
    if (b.colsq) off = align_up(off + b.members.size() * (size_t)cdiv(b.s, 32) * (size_t)round64(b.l) * sizeof(float));
  }
  p.off_scal = off;
  off = align_up(off + (size_t)n * S_COUNT * sizeof(double));
  p.off_partials = off;
  off = align_up(off + (size_t)part * 8 /*warps*/ * 2 * sizeof(double));
  p.off_gv = off;
  off = align_up(off + (size_t)gv * sizeof(float));
  p.off_sched = off;                                   // the tensor-core GEMM's tile counter
  off = align_up(off + sizeof(unsigned int));
  p.total = off;
  return p;
}

// ---------------------------------------------------------------- validation
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

muon_status check_config(const muon_config* c, bool need_ns, bool need_pp, bool need_pi) {
  if (!c) return MUON_ERR_INVALID_ARG;
  if (c->gemm_mode < 0 || c->gemm_mode > 2) return MUON_ERR_INVALID_ARG;
  if (c->param_dtype < 0 || c->param_dtype > 1 || c->grad_dtype < 0 || c->grad_dtype > 1)
    return MUON_ERR_INVALID_ARG;
  if (need_ns && c->ns_steps < 1) return MUON_ERR_INVALID_ARG;
  if (need_pp && c->pp_iterations < 1) return MUON_ERR_INVALID_ARG;
  if (need_pi && c->power_iters < 1) return MUON_ERR_INVALID_ARG;
  if (c->weight_decay != 0.f) return MUON_ERR_INVALID_ARG;
  if (!(c->ns_eps >= 0.f) || !(c->pp_eps > 0.f) || !(c->target_uw >= 0.f)) return MUON_ERR_INVALID_ARG;
  return MUON_OK;
}

muon_status check_shapes(int n, const muon_shape* shapes) {
  if (n < 0) return MUON_ERR_INVALID_ARG;
  if (n > 0 && !shapes) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (shapes[i].rows <= 0 || shapes[i].cols <= 0) return MUON_ERR_INVALID_ARG;
    if (shapes[i].rows > (int64_t)1 << 31 || shapes[i].cols > (int64_t)1 << 31) return MUON_ERR_INVALID_ARG;
    if (std::min(shapes[i].rows, shapes[i].cols) > 32768) return MUON_ERR_UNSUPPORTED;
  }
  return MUON_OK;
}

template <class P>
muon_status check_ptrs(int n, P const* arr, bool allow_null_array, bool allow_null_entry) {
  if (n == 0) return MUON_OK;
  if (!arr) return allow_null_array ? MUON_OK : MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (!arr[i]) { if (allow_null_entry) continue; return MUON_ERR_INVALID_ARG; }
    if (!aligned16((const void*)arr[i])) return MUON_ERR_INVALID_ARG;
  }
  return MUON_OK;
}

muon_status check_ws(const Plan& p, void* ws, size_t bytes) {
  if (p.total == 0) return MUON_OK;
  if (!ws || bytes < p.total || !aligned16(ws)) return MUON_ERR_WORKSPACE;
  return MUON_OK;
}

// ---------------------------------------------------------------- device info
int num_sms_current() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> g(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cache[dev] = sms;
  return sms;
}

// Tensor-core GEMM variant: SM pairs (256 x 256 tiles) unless the
// environment sets AURORA_MUON_TC_PAIR=0 (single-SM 128 x 256 tiles).
bool tc_pair() {
  static const bool pair = [] {
    const char* e = std::getenv("AURORA_MUON_TC_PAIR");
    return !(e && e[0] == '0');
  }();
  return pair;
}

// ---------------------------------------------------------------- tracing
// The tc_kind_* classes time the same tensor-core launches as ns_gemm_tc,
// split by GEMM kind (Gram, square, update); they are not extra launches.
enum ProfClass {
  PC_GEMM_TC = 0, PC_GEMM_SIMT, PC_PROLOGUE, PC_POWER, PC_AURORA, PC_REDUCE, PC_EPILOGUE,
  PC_TC_GRAM, PC_TC_SQR, PC_TC_UPD, PC_COUNT
};
const char* const kProfNames[PC_COUNT] = {"ns_gemm_tc", "ns_gemm_simt", "prologue", "power_iter",
                                          "aurora_rows", "reductions", "epilogue",
                                          "tc_kind_gram", "tc_kind_square", "tc_kind_update"};

struct ProfRecord {
  int cls;
  cudaEvent_t a, b;
  double flops, bytes;
};

struct ProfState {
  std::mutex mu;
  bool on = false;
  std::vector<ProfRecord> recs;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pool;
  size_t used = 0;
} g_prof;

// Brackets one launch with events when tracing is on.
struct ProfScope {
  ProfRecord rec{};
  bool active = false;
  cudaStream_t st;
  ProfScope(int cls, double flops, double bytes, cudaStream_t s) : st(s) {
    std::lock_guard<std::mutex> g(g_prof.mu);
    if (!g_prof.on) return;
    if (g_prof.used == g_prof.pool.size()) {
      cudaEvent_t a, b;
      if (cudaEventCreate(&a) != cudaSuccess) return;
      if (cudaEventCreate(&b) != cudaSuccess) { cudaEventDestroy(a); return; }
      g_prof.pool.emplace_back(a, b);
    }
    auto ev = g_prof.pool[g_prof.used++];
    rec = ProfRecord{cls, ev.first, ev.second, flops, bytes};
    active = cudaEventRecord(rec.a, st) == cudaSuccess;
  }
  ~ProfScope() {
    if (!active) return;
    cudaEventRecord(rec.b, st);
    std::lock_guard<std::mutex> g(g_prof.mu);
    g_prof.recs.push_back(rec);
  }
};

// ---------------------------------------------------------------- context
struct Ctx {
  const muon_config* cfg;
  const Plan* plan;
  char* ws;
  cudaStream_t st;
  double* scal;
  double* partials;
  unsigned int* sched;    // tile counter of the tensor-core GEMM launches
  void* const* W;
  const void* const* G;
  float* const* M;
  float* const* V;
  int param_dtype, grad_dtype;
  bool fuse_dots;    // the last update GEMM of each bucket's final polar forms <U,U>, <U,u>
};

template <class T> T* wsp(const Ctx& c, size_t off) { return reinterpret_cast<T*>(c.ws + off); }

MatDesc make_desc(const Ctx& c, int i) {
  const MatPlan& mp = c.plan->mats[i];
  const BucketPlan& b = c.plan->buckets[mp.bucket];
  const int nsb = c.plan->nsb;
  const size_t xo = (size_t)mp.bidx * b.s * b.ldl * nsb;
  MatDesc d{};
  d.W = c.W ? c.W[i] : nullptr;
  d.G = c.G ? c.G[i] : nullptr;
  d.M = c.M ? c.M[i] : nullptr;
  d.V = c.V ? c.V[i] : nullptr;
  d.uX = c.ws + b.off_uX + xo;
  const bool odd = (c.cfg->ns_steps & 1) != 0;
  d.UX = c.ws + (odd ? b.off_P : b.off_Q) + xo;
  d.X0 = c.ws + b.off_Q + xo;
  const size_t vo = (size_t)mp.bidx * (size_t)round64(b.l);
  d.D = wsp<float>(c, b.off_D) + vo;
  d.vec0 = wsp<float>(c, b.off_v0) + vo;
  d.vec1 = wsp<float>(c, b.off_v1) + vo;
  d.rho_slot = wsp<float>(c, b.off_rho) + mp.bidx;
  d.gvp = wsp<float>(c, c.plan->off_gv) + mp.gv_off;
  d.colsq = b.colsq ? wsp<float>(c, b.off_colsq) + (size_t)mp.bidx * (size_t)cdiv(b.s, 32) * (size_t)round64(b.l)
                    : nullptr;
  d.gv_rows = (int)mp.gv_rows;
  d.m = mp.m; d.n = mp.n; d.s = mp.s; d.l = mp.l; d.ldl = b.ldl;
  d.tall = mp.tall;
  d.idx = i;
  d.part = (int)mp.part;
  d.nslots = (int)std::max(cdiv(mp.m, 64) * cdiv(mp.n, 64), cdiv(mp.m * mp.n, 4096));
  return d;
}

// Run `launch(table, nblk_total)` over `ids` in chunks of at most
// kMaxMatsPerLaunch matrices; blocks(d) gives each matrix's block count and
// may set d.flag.
template <class BlocksFn, class LaunchFn>
cudaError_t for_chunks(const Ctx& c, const std::vector<int>& ids, BlocksFn blocks, LaunchFn launch) {
  size_t k = 0;
  while (k < ids.size()) {
    MatTable t;
    std::memset(&t, 0, sizeof(t));
    t.ns_dtype = c.plan->ns_dtype;
    t.param_dtype = c.param_dtype;
    t.grad_dtype = c.grad_dtype;
    int total = 0;
    while (k < ids.size() && t.count < kMaxMatsPerLaunch) {
      MatDesc d = make_desc(c, ids[k]);
      d.nblk = (int)blocks(d);
      t.blk_prefix[t.count] = total;
      total += d.nblk;
      t.mats[t.count++] = d;
      ++k;
    }
    t.blk_prefix[t.count] = total;
    cudaError_t e = launch(t, total);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

double table_elems(const MatTable& t) {
  double e = 0;
  for (int i = 0; i < t.count; ++i) e += (double)t.mats[i].m * (double)t.mats[i].n;
  return e;
}

int64_t tiles_orig(const MatDesc& d) { return cdiv(d.m, 64) * cdiv(d.n, 64); }
int64_t tiles_x(const MatDesc& d) { return cdiv(d.s, 64) * cdiv(d.l, 64); }
// blocks of a streaming launch (kEwTilesPerCta tiles each)
int64_t blocks_orig(const MatDesc& d) { return cdiv(tiles_orig(d), kEwTilesPerCta); }
int64_t blocks_x(const MatDesc& d) { return cdiv(tiles_x(d), kEwTilesPerCta); }
// Flat streaming applies when rows are contiguous, a multiple of 8 long and
// (original orientation) need no transposition into the X orientation.
bool flat_orig(const MatDesc& d) { return !d.tall && (d.n & 7) == 0 && d.ldl == d.n; }
bool flat_x(const MatDesc& d) { return (d.l & 7) == 0 && d.ldl == d.l; }
int64_t fblocks_orig(const MatDesc& d) { return cdiv(cdiv(d.m * d.n, kFlatChunk), kEwTilesPerCta); }
int64_t fblocks_x(const MatDesc& d) { return cdiv(cdiv(d.s * d.l, kFlatChunk), kEwTilesPerCta); }
// partial-sum slots a stage leaves per matrix (one per tile or per flat chunk)
int64_t slots_orig(const MatDesc& d) { return flat_orig(d) ? cdiv(d.m * d.n, kFlatChunk) : tiles_orig(d); }
int64_t slots_x(const MatDesc& d) { return flat_x(d) ? cdiv(d.s * d.l, kFlatChunk) : tiles_x(d); }

// Split ids by a predicate on their descriptors.
template <class Pred>
std::pair<std::vector<int>, std::vector<int>> split_ids(const Ctx& c, const std::vector<int>& ids, Pred pred) {
  std::pair<std::vector<int>, std::vector<int>> r;
  for (int i : ids) (pred(make_desc(c, i)) ? r.first : r.second).push_back(i);
  return r;
}

#define CK(expr)                                   \
  do {                                             \
    cudaError_t _e = (expr);                       \
    if (_e != cudaSuccess) return MUON_ERR_CUDA;   \
  } while (0)

// ---------------------------------------------------------------- stages
muon_status stage_prologue(const Ctx& c, const std::vector<int>& ids, int mode, bool want_w2) {
  const double per_elem = dt_bytes(c.grad_dtype) + c.plan->nsb + (mode == 0 ? 8.0 : 0.0) +
                          (want_w2 ? dt_bytes(c.param_dtype) : 0.0);
  const auto fl = split_ids(c, ids, flat_orig);
  CK(for_chunks(c, fl.first, fblocks_orig, [&](const MatTable& t, int nb) {
    ProfScope ps(PC_PROLOGUE, 0.0, per_elem * table_elems(t), c.st);
    return launch_prologue_flat(t, nb, mode, c.cfg->mu, c.cfg->nesterov, want_w2 ? 1 : 0, c.partials, c.st);
  }));
  // tall: the bf16 kernel that loads one tile ahead when the edges are whole tiles
  const bool bf16_all = mode == 0 && c.grad_dtype == kBF16 && c.plan->ns_dtype == kBF16 &&
                        (!want_w2 || c.param_dtype == kBF16);
  const auto tl = split_ids(c, fl.second, [bf16_all](const MatDesc& d) {
    return bf16_all && d.tall && d.m % 64 == 0 && d.n % 64 == 0 && d.ldl == d.m;
  });
  CK(for_chunks(c, tl.first, blocks_orig, [&](const MatTable& t, int nb) {
    ProfScope ps(PC_PROLOGUE, 0.0, per_elem * table_elems(t), c.st);
    return launch_prologue_tall_bf16(t, nb, c.cfg->mu, c.cfg->nesterov, want_w2 ? 1 : 0, c.partials, c.st);
  }));
  CK(for_chunks(c, tl.second, blocks_orig, [&](const MatTable& t, int nb) {
    ProfScope ps(PC_PROLOGUE, 0.0, per_elem * table_elems(t), c.st);
    return launch_prologue(t, nb, mode, c.cfg->mu, c.cfg->nesterov, want_w2 ? 1 : 0, c.partials, c.st);
  }));
  CK(for_chunks(c, ids, slots_orig, [&](const MatTable& t, int) {
    ProfScope ps(PC_REDUCE, 0.0, 0.0, c.st);
    return launch_finalize_sums(t, c.partials, 2, S_SUM_U2, want_w2 ? S_SUM_W2 : -1, c.scal, c.st);
  }));
  return MUON_OK;
}

// Power iteration on u (X orientation): sigma in S_SIGMA.
// With A the stored matrix and v over A's columns: t = A v, w = A^T t.
// Wide/square (X = A): t is a row dot of X, w a column dot.
// Tall (X = A^T):      t is a column dot of X, w a row dot.
// k_matvec flag: 0 = row dot (in: l, out: s), 1 = column dot (in: s, out: l).
// Separate row-dot and column-dot passes: two reads of X per iteration.  Used
// for rows longer than the fused pass takes.
muon_status stage_power_iteration_2pass(const Ctx& c, const std::vector<int>& ids, int iters) {
  auto vec_blocks = [](MatDesc& d) -> int64_t { d.flag = d.tall ? 1 : 0; return 0; };
  auto vecop = [&](int which, int mode, int len_is_s_when_flag0) {
    return for_chunks(c, ids, vec_blocks, [&](const MatTable& t, int) {
      ProfScope ps(PC_POWER, 0.0, 0.0, c.st);
      return launch_vecop(t, which, mode, len_is_s_when_flag0, c.scal, c.st);
    });
  };
  auto pass = [&](bool first, int dir) {
    return for_chunks(c, ids, [first](MatDesc& d) -> int64_t {
      const bool rowdot = first ? !d.tall : (bool)d.tall;
      d.flag = rowdot ? 0 : 1;
      return rowdot ? cdiv(d.s, kMatvecRowsPerCta) : cdiv(d.l, kColDotStrip);
    }, [&](const MatTable& t, int nb) {
      ProfScope ps(PC_POWER, 2.0 * table_elems(t), c.plan->nsb * table_elems(t), c.st);
      return launch_matvec(t, nb, dir, c.st);
    });
  };
  CK(vecop(0, 0, 0));          // v = ones / sqrt(len(v)) on vec0
  for (int k = 0; k < iters; ++k) {
    CK(pass(true, 0));         // t = A v    (vec0 -> vec1)
    CK(pass(false, 1));        // w = A^T t  (vec1 -> vec0)
    CK(vecop(0, 1, 0));        // v = w / |w|
  }
  CK(pass(true, 0));           // t = A v
  CK(vecop(1, 2, 1));          // sigma = |t|
  return MUON_OK;
}

// Fused passes (powiter.cu): one read of X per iteration, six in all.
//   wide (v over l in vec0):   [z = X v -> vec1, vec0 = X^T z / |X^T z|] x iters;
//                              z = X v -> vec1; sigma = |vec1| (over s).
//   tall (v over s in vec0):   vec1 = X^T v0 (= A v0);
//                              [z = X vec1 -> vec0, vec1 = X^T z / |z|] x iters;
//                              sigma = |vec1| (over l).
muon_status stage_power_iteration(const Ctx& c, const std::vector<int>& ids, int iters) {
  const int64_t max_ldl = gv_max_ldl(c.plan->ns_dtype);
  const auto fz = split_ids(c, ids, [max_ldl](const MatDesc& d) { return d.ldl <= max_ldl; });
  if (!fz.second.empty()) {
    muon_status s = stage_power_iteration_2pass(c, fz.second, iters);
    if (s != MUON_OK) return s;
  }
  const std::vector<int>& all = fz.first;
  if (all.empty()) return MUON_OK;
  const auto tw = split_ids(c, all, [](const MatDesc& d) { return d.tall != 0; });
  auto vec_blocks = [](MatDesc& d) -> int64_t { d.flag = d.tall ? 1 : 0; return 0; };
  auto items = [](MatDesc& d) -> int64_t { d.flag = d.tall ? 1 : 0; return cdiv(d.s, d.gv_rows); };
  auto pass = [&](const std::vector<int>& v, int mode) {
    return for_chunks(c, v, items, [&](const MatTable& t, int nb) {
      const double fl = (mode == GV_DOT_ACC ? 4.0 : 2.0) * table_elems(t);
      ProfScope ps(PC_POWER, fl, c.plan->nsb * table_elems(t), c.st);
      return launch_gramvec(t, nb, mode, c.st);
    });
  };
  auto reduce = [&](const std::vector<int>& v, int normalise) {
    return for_chunks(c, v, vec_blocks, [&](const MatTable& t, int) {
      ProfScope ps(PC_POWER, 0.0, 0.0, c.st);
      return launch_gv_reduce(t, normalise, c.st);
    });
  };
  auto vecop = [&](int which, int mode, int len_is_s_when_flag0) {
    return for_chunks(c, all, vec_blocks, [&](const MatTable& t, int) {
      ProfScope ps(PC_POWER, 0.0, 0.0, c.st);
      return launch_vecop(t, which, mode, len_is_s_when_flag0, c.scal, c.st);
    });
  };
  CK(vecop(0, 0, 0));                                   // v0 = 1/sqrt(len) (wide: l, tall: s)
  if (!tw.first.empty()) {
    CK(pass(tw.first, GV_ACC));                         // tall: X^T v0
    CK(reduce(tw.first, 0));
  }
  for (int k = 0; k < iters; ++k) {
    CK(pass(all, GV_DOT_ACC));
    CK(reduce(all, 1));
  }
  if (!tw.second.empty()) CK(pass(tw.second, GV_DOT));  // wide: z = X v
  CK(vecop(1, 2, 1));                                   // sigma = |vec1|
  return MUON_OK;
}

// Algorithmic flops of a launch: 2 K per useful output element; the
// symmetric kinds need only the s (s + 1) / 2 elements of one triangle.
double gemm_flops(const GemmLaunch& L) {
  double f = 0;
  for (int g = 0; g < L.num_groups; ++g) {
    const GemmGroup& G = L.g[g];
    const double outs = (G.kind == GK_UPD) ? (double)G.M * G.N : 0.5 * (double)G.M * (G.M + 1);
    f += 2.0 * G.K * outs * G.count;
  }
  return f;
}

muon_status gemm_launch(const Ctx& c, GemmLaunch& L) {
  if (L.num_groups == 0) return MUON_OK;
  if (c.cfg->gemm_mode == MUON_GEMM_BF16) {
    alignas(64) unsigned char maps[kMaxGemmGroups * 3 * 128];
    if (!tc_encode_maps(L, tc_pair(), maps)) return MUON_ERR_CUDA;
    L.tile_ctr = c.sched;
    CK(cudaMemsetAsync(c.sched, 0, sizeof(unsigned int), c.st));
    ProfScope ps(PC_GEMM_TC, gemm_flops(L), 0.0, c.st);
    ProfScope pk(PC_TC_GRAM + L.g[0].kind, gemm_flops(L), 0.0, c.st);   // every group of a launch has one kind
    CK(launch_gemm_tc(L, maps, num_sms_current(), tc_pair(), c.st));
  } else {
    ProfScope ps(PC_GEMM_SIMT, gemm_flops(L), 0.0, c.st);
    CK(launch_gemm_simt(L, c.st));
  }
  L.num_groups = 0;
  L.total_tiles = 0;
  return MUON_OK;
}

void add_group(const Ctx& c, GemmLaunch& L, GemmGroup g) {
  if (c.cfg->gemm_mode == MUON_GEMM_BF16) {
    g.tiles_per_mat = tc_tile_count(g.kind, g.M, g.N, tc_pair(), &g.tiles_m, &g.tiles_n);
  } else {
    g.tiles_per_mat = simt_tile_count(g.kind, g.M, g.N, &g.tiles_m, &g.tiles_n);
  }
  g.tile_begin = L.total_tiles;
  L.g[L.num_groups++] = g;
  L.total_tiles += g.tiles_per_mat * g.count;
}

// ns_steps Newton-Schulz iterations on every matrix of the given buckets.
// it = 0 reads X0 scaled by rho: uX, or Q for the buckets flagged in
// x0_in_Q (Aurora's D-scaled input); the iterates ping-pong P (even it),
// Q (odd it).
muon_status stage_newton_schulz(const Ctx& c, const std::vector<int>& bucket_ids_in,
                                const std::vector<bool>& x0_in_Q_in, const std::vector<bool>& final_in) {
  const Plan& p = *c.plan;
  const float a = c.cfg->ns_a, bc = c.cfg->ns_b, cc = c.cfg->ns_c;
  // Longest tiles first: the persistent kernel deals tiles round-robin in
  // group order, so big-K groups up front shorten the launch's tail.
  std::vector<size_t> order(bucket_ids_in.size());
  for (size_t k = 0; k < order.size(); ++k) order[k] = k;
  std::stable_sort(order.begin(), order.end(), [&](size_t x, size_t y) {
    const BucketPlan& bx = p.buckets[bucket_ids_in[x]];
    const BucketPlan& by = p.buckets[bucket_ids_in[y]];
    return bx.s != by.s ? bx.s > by.s : bx.l > by.l;
  });
  std::vector<int> bucket_ids;
  std::vector<bool> x0_in_Q, final_polar;
  for (size_t k : order) {
    bucket_ids.push_back(bucket_ids_in[k]);
    x0_in_Q.push_back(x0_in_Q_in[k]);
    final_polar.push_back(final_in[k]);
  }
  const bool tc = c.cfg->gemm_mode == MUON_GEMM_BF16;
  for (int it = 0; it < c.cfg->ns_steps; ++it) {
    for (int kind = 0; kind < 3; ++kind) {
      GemmLaunch L;
      std::memset(&L, 0, sizeof(L));
      L.dtype = p.ns_dtype;
      for (size_t k = 0; k < bucket_ids.size(); ++k) {
        const BucketPlan& b = p.buckets[bucket_ids[k]];
        char* X_in = c.ws + (it == 0 ? (x0_in_Q[k] ? b.off_Q : b.off_uX) : ((it & 1) ? b.off_P : b.off_Q));
        char* X_out = c.ws + ((it & 1) ? b.off_Q : b.off_P);
        char* Ab = c.ws + b.off_A;
        char* Bb = c.ws + b.off_B;
        const int64_t sx = b.s * b.ldl, ss = b.s * b.lds;
        GemmGroup g{};
        g.kind = kind;
        g.count = (int)b.members.size();
        g.rho = wsp<float>(c, b.off_rho);
        if (kind == GK_GRAM) {
          g.M = (int)b.s; g.N = (int)b.s; g.K = (int)b.l;
          g.A = X_in; g.lda = b.ldl; g.sa = sx;
          g.B = X_in; g.ldb = b.ldl; g.sb = sx;
          g.C = Ab; g.ldc = b.lds; g.sc = ss;
          g.alpha0 = 1.f; g.pa = it == 0 ? 2 : 0;
        } else if (kind == GK_SQR) {
          g.M = (int)b.s; g.N = (int)b.s; g.K = (int)b.s;
          g.A = Ab; g.lda = b.lds; g.sa = ss;
          g.B = Ab; g.ldb = b.lds; g.sb = ss;
          g.C = Bb; g.ldc = b.lds; g.sc = ss;
          g.E = Ab; g.lde = b.lds; g.se = ss;
          g.alpha0 = cc; g.beta0 = bc;
          g.rho = nullptr;
        } else {
          g.M = (int)b.s; g.N = (int)b.l; g.K = (int)b.s;
          g.A = Bb; g.lda = b.lds; g.sa = ss;
          g.B = X_in; g.ldb = b.ldl; g.sb = sx;
          g.C = X_out; g.ldc = b.ldl; g.sc = sx;
          g.E = X_in; g.lde = b.ldl; g.se = sx;
          g.alpha0 = 1.f; g.beta0 = a;
          g.pa = g.pb = it == 0 ? 1 : 0;
          if (tc && c.fuse_dots && final_polar[k] && it == c.cfg->ns_steps - 1) {
            g.dotu = c.ws + b.off_uX;
            g.dotp = wsp<double>(c, b.off_dots);
          }
          if (tc && b.colsq_gemm && !final_polar[k] && it == c.cfg->ns_steps - 1) {
            // Aurora's next D update reads these column sums instead of U, and
            // nothing else reads this polar's U: it is not stored
            g.colsq = wsp<float>(c, b.off_colsq);
            g.colsq_ld = round64(b.l);
            g.colsq_batch = cdiv(b.s, 32) * round64(b.l);
            g.no_store = 1;
          }
        }
        add_group(c, L, g);
        if (L.num_groups == kMaxGemmGroups) {
          muon_status s = gemm_launch(c, L);
          if (s != MUON_OK) return s;
        }
      }
      muon_status s = gemm_launch(c, L);
      if (s != MUON_OK) return s;
    }
  }
  return MUON_OK;
}

std::vector<int> ids_of_buckets(const Plan& p, const std::vector<int>& bids) {
  std::vector<int> ids;
  for (int b : bids) for (int i : p.buckets[b].members) ids.push_back(i);
  return ids;
}

// Polar factor of u (in X orientation) for every matrix; result in UX.
// Square matrices (and every matrix without Aurora) take one plain polar of
// u; with Aurora the non-square ones take pp_iterations polars of D-scaled u.
// The first polar of both kinds runs in the same grouped launches.
muon_status stage_polar(const Ctx& c, bool aurora) {
  const Plan& p = *c.plan;
  std::vector<int> plain_b, eq_b;
  for (int b = 0; b < (int)p.buckets.size(); ++b)
    ((aurora && p.buckets[b].s != p.buckets[b].l) ? eq_b : plain_b).push_back(b);
  const float eps = c.cfg->ns_eps;
  const float pe = c.cfg->pp_eps, beta = c.cfg->pp_beta;
  const std::vector<int> plain_ids = ids_of_buckets(p, plain_b), eq_ids = ids_of_buckets(p, eq_b);
  if (!plain_ids.empty())
    CK(for_chunks(c, plain_ids, [](const MatDesc&) { return (int64_t)0; }, [&](const MatTable& t, int) {
      ProfScope ps(PC_REDUCE, 0.0, 0.0, c.st);
      cudaError_t e = launch_scalars(t, 0, S_SUM_U2, eps, 0.f, 0.f, c.scal, c.st);
      if (e != cudaSuccess) return e;
      return launch_copy_rho(t, c.scal, c.st);
    }));
  // bytes of the column-sum partials (one float per column per row block)
  auto colsq_bytes = [](const MatTable& t, int rows) {
    double q = 0.0;
    for (int i = 0; i < t.count; ++i) q += 4.0 * (double)cdiv(t.mats[i].s, rows) * (double)t.mats[i].l;
    return q;
  };
  if (!eq_ids.empty()) {
    // D init: column sums of squares of uX per kColsqRows-row block, then their sum
    CK(for_chunks(c, eq_ids, [](const MatDesc& d) { return cdiv(d.s, 8 * kColsqRows) * cdiv(d.l, kColStrip); },
                  [&](const MatTable& t, int nb) {
      ProfScope ps(PC_AURORA, 0.0, c.plan->nsb * table_elems(t) + colsq_bytes(t, kColsqRows), c.st);
      return launch_colsq_partial(t, nb, c.st);
    }));
    CK(for_chunks(c, eq_ids, [](const MatDesc& d) { return cdiv(d.l, kColStrip); }, [&](const MatTable& t, int nb) {
      ProfScope ps(PC_AURORA, 0.0, colsq_bytes(t, kColsqRows), c.st);
      return launch_colsq_update(t, nb, 0, pe, beta, c.st);
    }));
  }
  const int rounds = eq_b.empty() ? 1 : c.cfg->pp_iterations;
  for (int k = 0; k < rounds; ++k) {
    if (!eq_ids.empty()) {
      // bf16 storage with contiguous rows: by column strips; else flat chunks
      // or 64 x 64 tiles.  The partial slots each form leaves differ, and the
      // sum below reads exactly those.
      const bool bf16 = c.plan->ns_dtype == kBF16;
      auto strip_blocks = [](const MatDesc& d) { return cdiv(d.l, kStripCols) * cdiv(d.s, kStripRows); };
      const auto fx = split_ids(c, eq_ids, flat_x);
      CK(for_chunks(c, fx.first, [&](const MatDesc& d) { return bf16 ? strip_blocks(d) : fblocks_x(d); },
                    [&](const MatTable& t, int nb) {
        ProfScope ps(PC_AURORA, 0.0, 2.0 * c.plan->nsb * table_elems(t), c.st);
        return bf16 ? launch_scale_cols_strip_bf16(t, nb, c.partials, c.st)
                    : launch_scale_cols_flat(t, nb, c.partials, c.st);
      }));
      CK(for_chunks(c, fx.second, blocks_x, [&](const MatTable& t, int nb) {
        ProfScope ps(PC_AURORA, 0.0, 2.0 * c.plan->nsb * table_elems(t), c.st);
        return launch_scale_cols(t, nb, c.partials, c.st);
      }));
      CK(for_chunks(c, eq_ids, [&](const MatDesc& d) { return bf16 && flat_x(d) ? strip_blocks(d) : slots_x(d); },
                    [&](const MatTable& t, int) {
        ProfScope ps(PC_REDUCE, 0.0, 0.0, c.st);
        cudaError_t e = launch_finalize_sums(t, c.partials, 1, S_SUM_X02, -1, c.scal, c.st);
        if (e != cudaSuccess) return e;
        e = launch_scalars(t, 0, S_SUM_X02, eps, 0.f, 0.f, c.scal, c.st);
        if (e != cudaSuccess) return e;
        return launch_copy_rho(t, c.scal, c.st);
      }));
    }
    std::vector<int> bids = eq_b;
    std::vector<bool> in_q(eq_b.size(), true), fin(eq_b.size(), k == rounds - 1);
    if (k == 0)
      for (int b : plain_b) { bids.push_back(b); in_q.push_back(false); fin.push_back(true); }
    muon_status s = stage_newton_schulz(c, bids, in_q, fin);
    if (s != MUON_OK) return s;
    if (k < rounds - 1) {
      // D update: from the column sums the last update GEMM wrote (tensor-core
      // mode), else from a pass over U
      const bool tcq = c.cfg->gemm_mode == MUON_GEMM_BF16;
      const auto fq = split_ids(c, eq_ids, [tcq](const MatDesc& d) { return tcq && d.colsq != nullptr; });
      CK(for_chunks(c, fq.first, [](const MatDesc& d) { return cdiv(d.l, kColStrip); }, [&](const MatTable& t, int nb) {
        ProfScope ps(PC_AURORA, 0.0, colsq_bytes(t, 32), c.st);
        return launch_colsq_update(t, nb, 1, pe, beta, c.st);
      }));
      CK(for_chunks(c, fq.second, [](const MatDesc& d) { return cdiv(d.l, kColStrip); }, [&](const MatTable& t, int nb) {
        ProfScope ps(PC_AURORA, 0.0, c.plan->nsb * table_elems(t), c.st);
        return launch_colnorm(t, nb, pe, beta, c.st);
      }));
    }
  }
  return MUON_OK;
}

std::vector<int> iota_ids(int n) {
  std::vector<int> v(n);
  for (int i = 0; i < n; ++i) v[i] = i;
  return v;
}

// Write V = cU U + cu u (original orientation) and optionally W.
muon_status stage_epilogue(const Ctx& c, const std::vector<int>& ids, bool update_w, float lr) {
  const bool need_u = c.cfg->contra != 0.f || !update_w;
  const double per_elem = c.plan->nsb * (need_u ? 2.0 : 1.0) + (update_w ? 2.0 * dt_bytes(c.param_dtype) : 0.0) +
                          (c.V ? 4.0 : 0.0);
  const auto fl = split_ids(c, ids, flat_orig);
  // bf16 params and NS storage: the kernels that load one chunk / tile ahead
  const bool bf16_both = c.param_dtype == kBF16 && c.plan->ns_dtype == kBF16;
  CK(for_chunks(c, fl.first, fblocks_orig, [&](const MatTable& t, int nb) {
    ProfScope ps(PC_EPILOGUE, 0.0, per_elem * table_elems(t), c.st);
    return bf16_both ? launch_epilogue_flat_bf16(t, nb, lr, update_w ? 1 : 0, c.scal, c.st)
                     : launch_epilogue_flat(t, nb, lr, update_w ? 1 : 0, c.scal, c.st);
  }));
  // tall matrices: the prefetching bf16 kernel when the edges are whole tiles
  const auto tl = split_ids(c, fl.second, [bf16_both](const MatDesc& d) {
    return bf16_both && d.tall && d.m % 64 == 0 && d.n % 64 == 0 && d.ldl == d.m;
  });
  CK(for_chunks(c, tl.first, blocks_orig, [&](const MatTable& t, int nb) {
    ProfScope ps(PC_EPILOGUE, 0.0, per_elem * table_elems(t), c.st);
    return launch_epilogue_tall_bf16(t, nb, lr, update_w ? 1 : 0, c.scal, c.st);
  }));
  CK(for_chunks(c, tl.second, blocks_orig, [&](const MatTable& t, int nb) {
    ProfScope ps(PC_EPILOGUE, 0.0, per_elem * table_elems(t), c.st);
    return launch_epilogue(t, nb, lr, update_w ? 1 : 0, c.scal, c.st);
  }));
  return MUON_OK;
}

muon_status stage_dots(const Ctx& c, const std::vector<int>& ids) {
  const auto fx = split_ids(c, ids, flat_x);
  CK(for_chunks(c, fx.first, fblocks_x, [&](const MatTable& t, int nb) {
    ProfScope ps(PC_REDUCE, 0.0, 2.0 * c.plan->nsb * table_elems(t), c.st);
    return launch_dots_flat(t, nb, c.partials, c.st);
  }));
  CK(for_chunks(c, fx.second, blocks_x, [&](const MatTable& t, int nb) {
    ProfScope ps(PC_REDUCE, 0.0, 2.0 * c.plan->nsb * table_elems(t), c.st);
    return launch_dots(t, nb, c.partials, c.st);
  }));
  CK(for_chunks(c, ids, slots_x, [&](const MatTable& t, int) {
    ProfScope ps(PC_REDUCE, 0.0, 0.0, c.st);
    return launch_finalize_sums(t, c.partials, 2, S_SUM_UU2, S_DOT_UUX, c.scal, c.st);
  }));
  return MUON_OK;
}

// <U,U> and <U,u> from the slots the last update GEMM of the final polar
// filled (tensor-core mode): one block of 8 warp slots per output tile.
muon_status stage_dots_fused(const Ctx& c, const std::vector<int>& ids) {
  const Plan& p = *c.plan;
  const bool pair = tc_pair();
  CK(for_chunks(c, ids, [&](MatDesc& d) -> int64_t {
    const BucketPlan& b = p.buckets[p.mats[d.idx].bucket];
    int tm, tn;
    const int64_t tpm = tc_tile_count(GK_UPD, (int)b.s, (int)b.l, pair, &tm, &tn);
    d.part = (int)((b.off_dots - p.off_dots) / (16 * sizeof(double)) + (size_t)p.mats[d.idx].bidx * tpm);
    return tpm;
  }, [&](const MatTable& t, int) {
    ProfScope ps(PC_REDUCE, 0.0, 0.0, c.st);
    return launch_finalize_sums(t, wsp<double>(c, p.off_dots), 2, S_SUM_UU2, S_DOT_UUX, c.scal, c.st);
  }));
  return MUON_OK;
}

muon_status set_coeffs(const Ctx& c, const std::vector<int>& ids, int op) {
  CK(for_chunks(c, ids, [](const MatDesc&) { return (int64_t)0; }, [&](const MatTable& t, int) {
    ProfScope ps(PC_REDUCE, 0.0, 0.0, c.st);
    return launch_scalars(t, op, 0, c.cfg->ns_eps, c.cfg->contra, c.cfg->target_uw, c.scal, c.st);
  }));
  return MUON_OK;
}

Ctx make_ctx(const muon_config* cfg, const Plan& p, void* ws, void* stream) {
  Ctx c{};
  c.cfg = cfg;
  c.plan = &p;
  c.ws = reinterpret_cast<char*>(ws);
  c.st = reinterpret_cast<cudaStream_t>(stream);
  c.scal = reinterpret_cast<double*>(c.ws + p.off_scal);
  c.partials = reinterpret_cast<double*>(c.ws + p.off_partials);
  c.sched = reinterpret_cast<unsigned int*>(c.ws + p.off_sched);
  c.param_dtype = cfg->param_dtype;
  c.grad_dtype = cfg->grad_dtype;
  return c;
}

// Shared front half of ns_polar / aurora_polar / opnorm_normalize.
muon_status stage_input(Ctx& c, int n, const void* const* in, int in_dtype) {
  c.G = in;
  c.grad_dtype = in_dtype;
  return stage_prologue(c, iota_ids(n), 1, false);
}

}  // namespace

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

void muon_config_default(muon_config* c) {
  if (!c) return;
  std::memset(c, 0, sizeof(*c));
  c->lr = 0.0375f;
  c->mu = 0.95f;
  c->nesterov = 1;
  c->ns_steps = 12;
  c->ns_a = 2.0f;
  c->ns_b = -1.5f;
  c->ns_c = 0.5f;
  c->ns_eps = 1e-7f;
  c->aurora = 1;
  c->pp_iterations = 2;
  c->pp_beta = 0.5f;
  c->pp_eps = 1e-7f;
  c->contra = 0.4f;
  c->power_iters = 5;
  c->target_uw = 0.35f;
  c->weight_decay = 0.0f;
  c->gemm_mode = MUON_GEMM_BF16;
  c->param_dtype = MUON_BF16;
  c->grad_dtype = MUON_BF16;
}

const char* muon_status_string(muon_status s) {
  switch (s) {
    case MUON_OK: return "ok";
    case MUON_ERR_INVALID_ARG: return "invalid argument";
    case MUON_ERR_UNSUPPORTED: return "unsupported request";
    case MUON_ERR_WORKSPACE: return "workspace missing or too small";
    case MUON_ERR_CUDA: return "CUDA error";
    case MUON_ERR_TIMEOUT: return "device-side wait timed out";
    case MUON_ERR_BOUNDS: return "index outside its buffer (checked build)";
  }
  return "unknown status";
}

size_t muon_workspace_size(const muon_config* cfg, int n, const muon_shape* shapes) {
  if (!cfg || n <= 0 || !shapes || check_shapes(n, shapes) != MUON_OK) return 0;
  return make_plan(cfg, n, shapes).total;
}

muon_status muon_step(const muon_config* cfg, int n, const muon_shape* shapes, void* const* params,
                      const void* const* grads, float* const* momentum, float* const* update_out,
                      void* workspace, size_t workspace_bytes, void* stream) {
  muon_status s = check_config(cfg, true, cfg && cfg->aurora, cfg && cfg->contra != 0.f);
  if (s != MUON_OK) return s;
  if ((s = check_shapes(n, shapes)) != MUON_OK) return s;
  if (n == 0) return MUON_OK;
  if ((s = check_ptrs(n, params, false, false)) != MUON_OK) return s;
  if ((s = check_ptrs(n, grads, false, false)) != MUON_OK) return s;
  if ((s = check_ptrs(n, momentum, false, false)) != MUON_OK) return s;
  if ((s = check_ptrs(n, update_out, true, true)) != MUON_OK) return s;
  const Plan p = make_plan(cfg, n, shapes);
  if ((s = check_ws(p, workspace, workspace_bytes)) != MUON_OK) return s;

  Ctx c = make_ctx(cfg, p, workspace, stream);
  c.W = params;
  c.G = grads;
  c.M = momentum;
  c.V = update_out;
  const std::vector<int> ids = iota_ids(n);
  if ((s = stage_prologue(c, ids, 0, cfg->target_uw > 0.f)) != MUON_OK) return s;
  if (cfg->contra != 0.f && (s = stage_power_iteration(c, ids, cfg->power_iters)) != MUON_OK) return s;
  c.fuse_dots = cfg->gemm_mode == MUON_GEMM_BF16;
  if ((s = stage_polar(c, cfg->aurora != 0)) != MUON_OK) return s;
  if ((s = c.fuse_dots ? stage_dots_fused(c, ids) : stage_dots(c, ids)) != MUON_OK) return s;
  if ((s = set_coeffs(c, ids, 1)) != MUON_OK) return s;
  return stage_epilogue(c, ids, true, cfg->lr);
}

static muon_status polar_entry(const muon_config* cfg, int n, const muon_shape* shapes,
                               const void* const* in, int in_dtype, float* const* out, void* ws,
                               size_t ws_bytes, void* stream, bool aurora) {
  muon_status s = check_config(cfg, true, aurora, false);
  if (s != MUON_OK) return s;
  if (in_dtype < 0 || in_dtype > 1) return MUON_ERR_INVALID_ARG;
  if ((s = check_shapes(n, shapes)) != MUON_OK) return s;
  if (n == 0) return MUON_OK;
  if ((s = check_ptrs(n, in, false, false)) != MUON_OK) return s;
  if ((s = check_ptrs(n, out, false, false)) != MUON_OK) return s;
  const Plan p = make_plan(cfg, n, shapes);
  if ((s = check_ws(p, ws, ws_bytes)) != MUON_OK) return s;
  Ctx c = make_ctx(cfg, p, ws, stream);
  c.V = out;
  const std::vector<int> ids = iota_ids(n);
  if ((s = stage_input(c, n, in, in_dtype)) != MUON_OK) return s;
  if ((s = stage_polar(c, aurora)) != MUON_OK) return s;
  if ((s = set_coeffs(c, ids, 2)) != MUON_OK) return s;
  return stage_epilogue(c, ids, false, 0.f);
}

muon_status ns_polar(const muon_config* cfg, int n, const muon_shape* shapes, const void* const* in,
                     int in_dtype, float* const* out, void* ws, size_t ws_bytes, void* stream) {
  return polar_entry(cfg, n, shapes, in, in_dtype, out, ws, ws_bytes, stream, false);
}

muon_status aurora_polar(const muon_config* cfg, int n, const muon_shape* shapes,
                         const void* const* in, int in_dtype, float* const* out, void* ws,
                         size_t ws_bytes, void* stream) {
  return polar_entry(cfg, n, shapes, in, in_dtype, out, ws, ws_bytes, stream, true);
}

muon_status opnorm_normalize(const muon_config* cfg, int n, const muon_shape* shapes,
                             const void* const* in, int in_dtype, float* const* out,
                             float* sigma_out, void* ws, size_t ws_bytes, void* stream) {
  muon_status s = check_config(cfg, false, false, true);
  if (s != MUON_OK) return s;
  if (in_dtype < 0 || in_dtype > 1) return MUON_ERR_INVALID_ARG;
  if ((s = check_shapes(n, shapes)) != MUON_OK) return s;
  if (n == 0) return MUON_OK;
  if ((s = check_ptrs(n, in, false, false)) != MUON_OK) return s;
  if ((s = check_ptrs(n, out, true, true)) != MUON_OK) return s;
  if (sigma_out && !aligned16(sigma_out)) return MUON_ERR_INVALID_ARG;
  const Plan p = make_plan(cfg, n, shapes);
  if ((s = check_ws(p, ws, ws_bytes)) != MUON_OK) return s;
  Ctx c = make_ctx(cfg, p, ws, stream);
  c.V = out;
  const std::vector<int> ids = iota_ids(n);
  if ((s = stage_input(c, n, in, in_dtype)) != MUON_OK) return s;
  if ((s = stage_power_iteration(c, ids, cfg->power_iters)) != MUON_OK) return s;
  if (sigma_out) {
    CK(for_chunks(c, ids, [](const MatDesc&) { return (int64_t)0; }, [&](const MatTable& t, int) {
      return launch_sigma_out(t, c.scal, sigma_out, c.st);
    }));
  }
  if (out) {
    if ((s = set_coeffs(c, ids, 3)) != MUON_OK) return s;
    if ((s = stage_epilogue(c, ids, false, 0.f)) != MUON_OK) return s;
  }
  return MUON_OK;
}

muon_status uw_floor_apply(const muon_config* cfg, int n, const muon_shape* shapes,
                           const void* const* params, float* const* updates, void* ws,
                           size_t ws_bytes, void* stream) {
  if (!cfg) return MUON_ERR_INVALID_ARG;
  if (cfg->param_dtype < 0 || cfg->param_dtype > 1 || !(cfg->target_uw >= 0.f)) return MUON_ERR_INVALID_ARG;
  muon_status s = check_shapes(n, shapes);
  if (s != MUON_OK) return s;
  if (n == 0) return MUON_OK;
  if ((s = check_ptrs(n, params, false, false)) != MUON_OK) return s;
  if ((s = check_ptrs(n, updates, false, false)) != MUON_OK) return s;
  const Plan p = make_plan(cfg, n, shapes);
  if ((s = check_ws(p, ws, ws_bytes)) != MUON_OK) return s;
  Ctx c = make_ctx(cfg, p, ws, stream);
  c.W = const_cast<void* const*>(params);
  c.V = updates;
  const std::vector<int> ids = iota_ids(n);
  auto blocks = [](const MatDesc& d) { return cdiv(d.m * d.n, 4096); };
  CK(for_chunks(c, ids, blocks, [&](const MatTable& t, int nb) { return launch_sumsq_wv(t, nb, c.partials, c.st); }));
  CK(for_chunks(c, ids, blocks, [&](const MatTable& t, int) {
    cudaError_t e = launch_finalize_sums(t, c.partials, 2, S_SUM_U2, S_SUM_W2, c.scal, c.st);
    if (e != cudaSuccess) return e;
    return launch_scalars(t, 4, 0, 0.f, 0.f, cfg->target_uw, c.scal, c.st);
  }));
  CK(for_chunks(c, ids, blocks, [&](const MatTable& t, int nb) { return launch_scale_v(t, nb, c.scal, c.st); }));
  return MUON_OK;
}

void muon_profile_enable(int on) {
  std::lock_guard<std::mutex> g(g_prof.mu);
  if (on) {
    g_prof.recs.clear();
    g_prof.used = 0;
  }
  g_prof.on = on != 0;
}

int muon_profile_read(muon_profile_entry* out, int max_entries) {
  std::lock_guard<std::mutex> g(g_prof.mu);
  muon_profile_entry tot[PC_COUNT];
  std::memset(tot, 0, sizeof(tot));
  for (int k = 0; k < PC_COUNT; ++k) std::snprintf(tot[k].name, sizeof(tot[k].name), "%s", kProfNames[k]);
  for (const ProfRecord& r : g_prof.recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -1;
    tot[r.cls].launches += 1;
    tot[r.cls].ms += ms;
    tot[r.cls].flops += r.flops;
    tot[r.cls].bytes += r.bytes;
  }
  int w = 0;
  for (int k = 0; k < PC_COUNT && w < max_entries; ++k) out[w++] = tot[k];
  return w;
}

muon_status muon_selftest_wait_timeout(long long max_cycles, void* stream) {
  const long long lim = std::min(std::max(max_cycles, 1000LL), 4000000000LL);
  return launch_wait_selftest(lim, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

// the first failed index test seen by muon_last_device_status (file * 100000 + line)
static unsigned int g_last_check_line = 0;

muon_status muon_last_device_status(void* stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MUON_ERR_CUDA;
  unsigned int v = 0, w = 0;
  if (read_and_clear_device_status(&v) != cudaSuccess) return MUON_ERR_CUDA;
  if (read_and_clear_gv_status(&w) != cudaSuccess) return MUON_ERR_CUDA;
  // the first failed index test, as file * 100000 + line (files in this order, from 1)
  unsigned int line = 0;
  cudaError_t (*const readers[])(unsigned int*) = {read_and_clear_check_elementwise, read_and_clear_check_powiter,
                                                   read_and_clear_check_gemm_tc, read_and_clear_check_gemm_simt,
                                                   read_and_clear_check_adamw};
  for (unsigned int f = 0; f < 5; ++f) {
    unsigned int q = 0;
    if (readers[f](&q) != cudaSuccess) return MUON_ERR_CUDA;
    if (q && !line) line = (f + 1) * 100000u + q;
  }
  if (line) g_last_check_line = line;
  if (v != 0) return static_cast<muon_status>(v);
  if (w != 0) return static_cast<muon_status>(w);
  return line ? MUON_ERR_BOUNDS : MUON_OK;
}

int muon_build_checked(void) {
#ifdef AURORA_MUON_CHECKED
  return 1;
#else
  return 0;
#endif
}

int muon_last_check_line(void) {
  const unsigned int l = g_last_check_line;
  g_last_check_line = 0;
  return (int)l;
}

muon_status muon_selftest_bounds_check(void* stream) {
  return launch_bounds_selftest(reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

}  // extern "C"
