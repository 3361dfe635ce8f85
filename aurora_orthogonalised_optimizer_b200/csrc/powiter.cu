// Power iteration of the Contra-Muon operator-norm estimate, one read of the
// stored update per iteration.
//
// Method (Track 3 Aurora write-up, "组合优化栈 / Contra-Muon"): sigma, the
// largest singular value of the momentum update A = u, is estimated by
// power iterations v <- A^T A v / |A^T A v| started from v = 1/sqrt(n) over
// A's columns, then sigma = |A v|; N = u / sigma.
//
// Let X be the s x l orientation of A (X = A when A is wide or square,
// X = A^T when it is tall) and x_i its rows.  One pass over the rows gives
// both z = X y (z_i = x_i . y) and X^T z = sum_i z_i x_i from the same loaded
// row, so an iteration costs one read of X instead of two:
//   wide  (v over l):  pass with y = v  -> z = A v,  X^T z = A^T A v;
//                      then v <- X^T z / |X^T z|.
//   tall  (v over s):  carry t = A v = X^T v (over l) instead of v;
//                      pass with y = t  -> z = X t = A^T A v,
//                      X^T z / |z| = A v_next = t_next.
// Wide: 5 fused passes and a final z = X v (sigma = |z|).  Tall: a first
// X^T v0 pass (z given) and 5 fused passes (sigma = |t|).  Six reads of X in
// both cases, where separate row-dot and column-dot passes take eleven.
//
// Kernel k_gramvec: a block owns a range of rows of one matrix (an "item");
// its thread 0 streams the rows into a 4-stage ring of shared-memory stages
// with bulk asynchronous copies (cp.async.bulk, completion on an mbarrier);
// the 16 warps form teams of TW warps, R = 2 rows per team per stage, each
// thread holding 8-column chunks of y and of the X^T z accumulator in
// registers.  The row dot is a warp sum, plus an mbarrier-synchronised sum
// over the team's warps when TW > 1.  Each item writes one partial X^T z
// vector; k_gv_reduce sums an item's partials in a fixed order
// (deterministic) and applies the normalisation.  Every wait is bounded: on
// expiry the block records MUON_ERR_TIMEOUT in its status word and returns.
#include <algorithm>
#include <mutex>
#include <set>

#include "kernels.h"

namespace am {

// Sticky status word of the kernels in this file (first error wins).
__device__ unsigned int g_gv_status = 0;

namespace {

constexpr int kGvWarps = 16;
constexpr int kGvThreads = 32 * kGvWarps;            // thread 0 also issues the copies
constexpr int kGvStages = 4;
constexpr uint32_t kGvStageBytes = 49152;                      // NT x R rows of a group
constexpr uint32_t kGvRingBytes = kGvStages * kGvStageBytes;
constexpr int kGvRowsMax = 2;                                   // R: rows per team per group
constexpr long long kGvWaitLimit = 2000000000LL;               // ~1 s at B200 clocks

struct GvCtl {
  unsigned long long full[kGvStages];
  unsigned long long empty[kGvStages];
  unsigned long long team[8];
  float red[2][kGvRowsMax][kGvWarps];   // per-warp partial dots, by team-phase parity
  int abort;
};
constexpr size_t kGvSmemBytes = kGvRingBytes + sizeof(GvCtl);

__device__ __forceinline__ uint32_t s_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void gv_raise(unsigned int code) { atomicCAS(&g_gv_status, 0u, code); }
// elements of a matrix's per-item partials of X^T z (one ldl row per item)
__device__ __forceinline__ int64_t gv_ext(const MatDesc& d) { return (d.s + d.gv_rows - 1) / d.gv_rows * d.ldl; }
__device__ __forceinline__ void mb_init(uint32_t a, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mb_arrive(uint32_t a) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ void mb_expect_tx(uint32_t a, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mb_try(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false on timeout (recorded) or when another warp aborted.
__device__ __forceinline__ bool mb_wait(uint32_t a, uint32_t parity, volatile int* abort_flag) {
  if (mb_try(a, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mb_try(a, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kGvWaitLimit) {
        *abort_flag = 1;
        gv_raise(MUON_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
// Bulk copy of `bytes` (multiple of 16) from global to this block's shared
// memory; completion is counted on the mbarrier at `mbar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(mbar)
      : "memory");
}

// Two fp32 lanes in one 64-bit register, and the paired fused multiply-add
// of sm_100 (two independent round-to-nearest fp32 FMAs).
__device__ __forceinline__ unsigned long long pk2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 upk2(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// Non-blocking probe of an mbarrier phase.
__device__ __forceinline__ bool mb_test(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}

template <bool BF16>
struct GvTraits {
  static constexpr int kKcMax = BF16 ? 3 : 2;          // 8-element chunks per thread
  static constexpr int kChunkBytes = BF16 ? 16 : 32;
  static constexpr int kWords = BF16 ? 4 : 8;          // 32-bit words per chunk
};

// A chunk of 8 elements from shared memory as raw words; words holding
// elements at or beyond `valid` (< 8 only in a row's last chunk) are zeroed.
template <bool BF16>
__device__ __forceinline__ void ld_chunk_words(const unsigned char* p, int valid, uint32_t (&w)[GvTraits<BF16>::kWords]) {
  if constexpr (BF16) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    if (valid < 8) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        if (2 * h >= valid) w[h] = 0u;
        else if (2 * h + 1 >= valid) w[h] &= 0xFFFFu;
      }
    }
  } else {
    const uint4 a = reinterpret_cast<const uint4*>(p)[0];
    const uint4 b = reinterpret_cast<const uint4*>(p)[1];
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    if (valid < 8) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (e >= valid) w[e] = 0u;
    }
  }
}
// Element pair h (elements 2h, 2h+1) of a chunk as a packed fp32 pair.
template <bool BF16>
__device__ __forceinline__ unsigned long long chunk_pair(const uint32_t (&w)[GvTraits<BF16>::kWords], int h) {
  if constexpr (BF16) return pk2(__uint_as_float(w[h] << 16), __uint_as_float(w[h] & 0xFFFF0000u));
  else return pk2(__uint_as_float(w[2 * h]), __uint_as_float(w[2 * h + 1]));
}

// Team width: the fewest warps (a power of two, at most 16) whose threads
// cover the row's 8-column chunks with at most KCMAX chunks each.
template <int KCMAX>
__host__ __device__ __forceinline__ int gv_team_warps(int64_t ldl) {
  const int64_t chunks = ldl / 8;
  int tw = 1;
  while (tw < kGvWarps && (int64_t)tw * 32 * KCMAX < chunks) tw *= 2;
  return tw;
}

// mode: GV_DOT_ACC, GV_DOT, GV_ACC (see kernels.h).
//
// A group (one ring stage) holds R consecutive rows per team.  A warp copies
// its chunks of the team's R rows from shared memory into registers as fp32
// pairs and releases the stage at once, so the ring's other stages stay in
// flight; the dots of the R rows are independent FMA chains; the team's
// partial dots meet in shared memory behind one team-mbarrier phase per
// group (two slot sets by phase parity: a warp publishes group g+1 only after
// it has seen group g's phase complete); then z * x is accumulated from the
// same registers.  Thread 0 also issues the copies: without blocking
// whenever the stage of the next group is free, and blocking only for the
// group it is about to read.
template <bool BF16>
__global__ void __launch_bounds__(kGvThreads, 1) k_gramvec(const MatTable t, int mode) {
  using Tr = GvTraits<BF16>;
  constexpr int KCMAX = Tr::kKcMax;
  constexpr int RM = kGvRowsMax;
  extern __shared__ __align__(128) unsigned char gv_smem[];
  GvCtl* ctl = reinterpret_cast<GvCtl*>(gv_smem + kGvRingBytes);
  const uint32_t ring = s_u32(gv_smem);

  const int mi = find_mat(t, blockIdx.x);
  const MatDesc& d = t.mats[mi];
  const int item = blockIdx.x - t.blk_prefix[mi];
  const int64_t r0 = (int64_t)item * d.gv_rows;
  const int64_t r1 = min(d.s, r0 + (int64_t)d.gv_rows);
  const int C = (int)(d.ldl / 8);                          // 8-column chunks per row
  const int TW = gv_team_warps<KCMAX>(d.ldl);
  const int NT = kGvWarps / TW;                            // teams
  const int KC = (C + 32 * TW - 1) / (32 * TW);
  const uint32_t row_bytes = (uint32_t)C * Tr::kChunkBytes;
  const int R = (int)min((uint32_t)RM, kGvStageBytes / ((uint32_t)NT * row_bytes));
  const int rows_per_group = NT * R;
  const int groups = (int)((r1 - r0 + rows_per_group - 1) / rows_per_group);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int team = warp / TW, wt = warp % TW, tt = wt * 32 + lane;
  const bool reduce_team = TW > 1 && mode != GV_ACC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGvStages; ++s) {
      mb_init(s_u32(&ctl->full[s]), 1);
      mb_init(s_u32(&ctl->empty[s]), kGvWarps);
    }
    for (int k = 0; k < 8; ++k) mb_init(s_u32(&ctl->team[k]), (uint32_t)TW);
    ctl->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int* abort_flag = &ctl->abort;

  float* yv = d.tall ? d.vec1 : d.vec0;     // vector over l (input of z = X y)
  float* zv = d.tall ? d.vec0 : d.vec1;     // vector over s

  // ---------------------------------------------------------------- copies
  // group g -> stage g % kGvStages; its rows are contiguous in X and in the stage
  const unsigned char* src = reinterpret_cast<const unsigned char*>(d.uX);
  auto issue = [&](int g) {
    const int s = g % kGvStages;
    const int64_t row0 = r0 + (int64_t)g * rows_per_group;
    const int nrows = (int)min((int64_t)rows_per_group, r1 - row0);
    const uint32_t fb = s_u32(&ctl->full[s]);
    // the group's rows are consecutive in X and in the stage: one copy (one
    // large bulk copy streams faster than one per row, and far faster than
    // smaller pieces)
    if (!AM_IN(row0 * d.ldl, (int64_t)nrows * d.ldl, AM_EXT_X(d))) return;   // (the wait then times out)
    mb_expect_tx(fb, (uint32_t)nrows * row_bytes);
    bulk_g2s(ring + (uint32_t)s * kGvStageBytes, src + row0 * (int64_t)row_bytes, (uint32_t)nrows * row_bytes, fb);
  };
  int issued = 0;
  if (threadIdx.x == 0)
    for (; issued < groups && issued < kGvStages; ++issued) issue(issued);
  // thread 0: issue every group whose stage all warps have released (group
  // issued - kGvStages); wait only while group `need` is not yet issued
  auto refill = [&](int need) -> bool {
    while (issued < groups) {
      const int gp = issued - kGvStages;
      const uint32_t eb = s_u32(&ctl->empty[gp % kGvStages]);
      const uint32_t ph = (uint32_t)(gp / kGvStages) & 1u;
      if (issued <= need) {
        if (!mb_wait(eb, ph, abort_flag)) return false;
      } else if (!mb_test(eb, ph)) {
        break;
      }
      issue(issued++);
    }
    return true;
  };

  // ---------------------------------------------------------------- rows
  // this thread's chunks: byte offset in a row, and elements inside l (8 but
  // in a row's last chunk when l is not a multiple of 8; 0 = no chunk)
  uint32_t coff[KCMAX];
  int cval[KCMAX];
  unsigned long long y2[KCMAX][4], acc2[KCMAX][4];
#pragma unroll
  for (int k = 0; k < KCMAX; ++k) {
    const int c = tt + k * 32 * TW;
    const int64_t j = 8 * (int64_t)c;
    coff[k] = (uint32_t)c * Tr::kChunkBytes;
    cval[k] = (k < KC && c < C) ? (int)min((int64_t)8, d.l - j) : 0;
    float yy[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (mode != GV_ACC && cval[k] == 8 && AM_IN(j, 8, AM_EXT_VEC(d))) {
      const float4 a = reinterpret_cast<const float4*>(yv + j)[0];
      const float4 b = reinterpret_cast<const float4*>(yv + j)[1];
      yy[0] = a.x; yy[1] = a.y; yy[2] = a.z; yy[3] = a.w;
      yy[4] = b.x; yy[5] = b.y; yy[6] = b.z; yy[7] = b.w;
    } else if (mode != GV_ACC) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (e < cval[k] && AM_IN(j + e, 1, AM_EXT_VEC(d))) yy[e] = yv[j + e];
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      y2[k][h] = pk2(yy[2 * h], yy[2 * h + 1]);
      acc2[k][h] = 0ull;
    }
  }

  const uint32_t team_bar = s_u32(&ctl->team[team < 8 ? team : 0]);
  uint32_t par = 0;
  bool ok = true;
  for (int g = 0; g < groups; ++g) {
    if (threadIdx.x == 0 && !refill(g)) { ok = false; break; }
    const int s = g % kGvStages;
    const uint32_t ph = (uint32_t)(g / kGvStages) & 1u;
    if (!mb_wait(s_u32(&ctl->full[s]), ph, abort_flag)) { ok = false; break; }
    const int64_t i0 = r0 + (int64_t)g * rows_per_group + (int64_t)team * R;
    const int nr = (int)max((int64_t)0, min((int64_t)R, r1 - i0));
    // rows -> registers (fp32 pairs), then the stage goes back to the producer
    unsigned long long x2[RM][KCMAX][4];
    const unsigned char* tbase = gv_smem + (size_t)s * kGvStageBytes + (size_t)team * R * row_bytes;
#pragma unroll
    for (int r = 0; r < RM; ++r) {
#pragma unroll
      for (int k = 0; k < KCMAX; ++k) {
        if (r < nr && cval[k] > 0) {
          uint32_t w[Tr::kWords];
          ld_chunk_words<BF16>(tbase + (size_t)r * row_bytes + coff[k], cval[k], w);
#pragma unroll
          for (int h = 0; h < 4; ++h) x2[r][k][h] = chunk_pair<BF16>(w, h);
        } else {
#pragma unroll
          for (int h = 0; h < 4; ++h) x2[r][k][h] = 0ull;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mb_arrive(s_u32(&ctl->empty[s]));
    if (nr == 0) continue;
    float z[RM];
    if (mode == GV_ACC) {
#pragma unroll
      for (int r = 0; r < RM; ++r) z[r] = r < nr && AM_IN(i0 + r, 1, AM_EXT_VEC(d)) ? zv[i0 + r] : 0.f;
    } else {
      unsigned long long p2[RM];
#pragma unroll
      for (int r = 0; r < RM; ++r) p2[r] = 0ull;
#pragma unroll
      for (int k = 0; k < KCMAX; ++k)
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
          for (int r = 0; r < RM; ++r) p2[r] = fma2(x2[r][k][h], y2[k][h], p2[r]);
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        const float2 q = upk2(p2[r]);
        z[r] = q.x + q.y;
      }
#pragma unroll
      for (int r = 0; r < RM; ++r) z[r] = warp_sum(z[r]);
      if (reduce_team) {
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < RM; ++r) ctl->red[par][r][warp] = z[r];
          mb_arrive(team_bar);
        }
        if (!mb_wait(team_bar, par, abort_flag)) { ok = false; break; }
#pragma unroll
        for (int r = 0; r < RM; ++r) z[r] = lane < TW ? ctl->red[par][r][team * TW + lane] : 0.f;
#pragma unroll
        for (int r = 0; r < RM; ++r) z[r] = warp_sum(z[r]);
        par ^= 1u;
      }
      if (tt == 0)
#pragma unroll
        for (int r = 0; r < RM; ++r)
          if (r < nr && AM_IN(i0 + r, 1, AM_EXT_VEC(d))) zv[i0 + r] = z[r];
    }
    if (mode != GV_DOT) {
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        const unsigned long long z2 = pk2(z[r], z[r]);   // z = 0 for rows past the item's end
#pragma unroll
        for (int k = 0; k < KCMAX; ++k)
#pragma unroll
          for (int h = 0; h < 4; ++h) acc2[k][h] = fma2(z2, x2[r][k][h], acc2[k][h]);
      }
    }
  }
  if (threadIdx.x == 0 && *abort_flag) {
    // copies still in flight after an abort land before the block moves on
    for (int k = 0; k < kGvStages && k < issued; ++k) {
      const int g = issued - 1 - k;
      const uint32_t a = s_u32(&ctl->full[g % kGvStages]), ph = (uint32_t)(g / kGvStages) & 1u;
      const long long t0 = clock64();
      while (!mb_try(a, ph) && clock64() - t0 < kGvWaitLimit) {}
    }
  }

  // every warp is done and every copy has landed: the ring is free
  __syncthreads();
  if (*abort_flag || mode == GV_DOT) return;
  float* part = d.gvp + (int64_t)item * d.ldl;
  float* dst = NT == 1 ? part : reinterpret_cast<float*>(gv_smem) + (int64_t)team * d.ldl;
#pragma unroll
  for (int k = 0; k < KCMAX; ++k) {
    if (cval[k] > 0) {
      const float2 a0 = upk2(acc2[k][0]), a1 = upk2(acc2[k][1]), a2 = upk2(acc2[k][2]), a3 = upk2(acc2[k][3]);
      float4* q = reinterpret_cast<float4*>(dst + 8 * (int64_t)(tt + k * 32 * TW));
      if (NT == 1 ? AM_IN((int64_t)item * d.ldl + 8 * (int64_t)(tt + k * 32 * TW), 8, gv_ext(d))
                  : AM_IN((int64_t)team * d.ldl + 8 * (int64_t)(tt + k * 32 * TW), 8, (int64_t)NT * d.ldl)) {
        q[0] = make_float4(a0.x, a0.y, a1.x, a1.y);
        q[1] = make_float4(a2.x, a2.y, a3.x, a3.y);
      }
    }
  }
  if (NT == 1) return;
  // several teams: combine their accumulators (staged in the ring) in team order
  __syncthreads();
  const float* comb = reinterpret_cast<const float*>(gv_smem);
  for (int j4 = threadIdx.x; j4 < 2 * C; j4 += blockDim.x) {
    float4 sum = reinterpret_cast<const float4*>(comb)[j4];
    for (int tm = 1; tm < NT; ++tm) {
      const float4 v = reinterpret_cast<const float4*>(comb + (int64_t)tm * d.ldl)[j4];
      sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
    }
    if (AM_IN((int64_t)item * d.ldl + 4 * (int64_t)j4, 4, gv_ext(d))) reinterpret_cast<float4*>(part)[j4] = sum;
  }
}

// One block per matrix: sum the item partials of X^T z in item order into
// the vector over l (tall: vec1, wide: vec0); with `normalise`, scale it by
// 1 / max(|z|, 1e-30) (tall: z = vec0 over s) or by its own inverse norm
// (wide), the norm accumulated in double.
__global__ void __launch_bounds__(512) k_gv_reduce(const MatTable t, int normalise) {
  __shared__ double red[32];
  const MatDesc& d = t.mats[blockIdx.x];
  const int P = (int)((d.s + d.gv_rows - 1) / d.gv_rows);
  const int C = (int)(d.ldl / 8);
  float* out = d.tall ? d.vec1 : d.vec0;
  double ss = 0.0;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const float* p = d.gvp + 8 * (int64_t)c;
#pragma unroll 6
    for (int q = 0; q < P; ++q) {   // item order: the sum is the same on every run
      if (!AM_IN((int64_t)q * d.ldl + 8 * (int64_t)c, 8, gv_ext(d))) continue;
      const float4 a = __ldg(reinterpret_cast<const float4*>(p + (int64_t)q * d.ldl));
      const float4 b = __ldg(reinterpret_cast<const float4*>(p + (int64_t)q * d.ldl) + 1);
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    const int64_t j = 8 * (int64_t)c;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (j + e < d.l && AM_IN(j + e, 1, AM_EXT_VEC(d))) {
        out[j + e] = v[e];
        ss += (double)v[e] * v[e];
      }
    }
  }
  if (!normalise) return;
  if (d.tall) {
    ss = 0.0;
    for (int64_t i = threadIdx.x; i < d.s; i += blockDim.x)
      if (AM_IN(i, 1, AM_EXT_VEC(d))) ss += (double)d.vec0[i] * d.vec0[i];
  }
  ss = block_sum(ss, red);
  const float inv = (float)(1.0 / fmax(sqrt(ss), 1e-30));
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const int64_t j = 8 * (int64_t)c;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (j + e < d.l && AM_IN(j + e, 1, AM_EXT_VEC(d))) out[j + e] *= inv;
  }
}

template <bool BF16>
cudaError_t gv_prepare() {
  static std::mutex mu;
  static std::set<int> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  if (done.count(dev)) return cudaSuccess;
  e = cudaFuncSetAttribute(k_gramvec<BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGvSmemBytes);
  if (e == cudaSuccess) done.insert(dev);
  return e;
}

}  // namespace

int64_t gv_max_ldl(int ns_dtype) {
  return ns_dtype == kBF16 ? (int64_t)kGvWarps * 32 * GvTraits<true>::kKcMax * 8
                           : (int64_t)kGvWarps * 32 * GvTraits<false>::kKcMax * 8;
}

cudaError_t launch_gramvec(const MatTable& t, int nblk, int mode, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  cudaError_t e;
  if (t.ns_dtype == kBF16) {
    if ((e = gv_prepare<true>()) != cudaSuccess) return e;
    k_gramvec<true><<<nblk, kGvThreads, kGvSmemBytes, st>>>(t, mode);
  } else {
    if ((e = gv_prepare<false>()) != cudaSuccess) return e;
    k_gramvec<false><<<nblk, kGvThreads, kGvSmemBytes, st>>>(t, mode);
  }
  return cudaGetLastError();
}

cudaError_t launch_gv_reduce(const MatTable& t, int normalise, cudaStream_t st) {
  if (t.count == 0) return cudaSuccess;
  k_gv_reduce<<<t.count, 512, 0, st>>>(t, normalise);
  return cudaGetLastError();
}

AM_CHECK_READER(read_and_clear_check_powiter)

cudaError_t read_and_clear_gv_status(unsigned int* out) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_gv_status, sizeof(v));
  if (e != cudaSuccess) return e;
  *out = v;
  if (v != 0) e = cudaMemcpyToSymbol(g_gv_status, &zero, sizeof(zero));
  return e;
}

}  // namespace am
