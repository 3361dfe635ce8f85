// Grouped Newton-Schulz GEMMs on the sm_100a tensor cores.
//
// Newton-Schulz step ("源码实现", zeropower_via_newtonschulz5 of the Track 3
// Aurora write-up): A = X X^T, B = b A + c A^2, X' = a X + B X, with bf16
// operands and fp32 accumulation.
//
// Kernel design (persistent, warp-specialised, one CTA per SM), in two
// variants selected at compile time:
//   * single-SM (PAIR = false): a CTA computes a 128 x 256 tile with
//     tcgen05.mma.cta_group::1 (M = 128, N = 256); 4-stage smem ring of a
//     128 x 64 A tile and a 256 x 64 B tile.
//   * SM pair (PAIR = true): a cluster of two CTAs computes a 256 x 256 tile
//     with tcgen05.mma.cta_group::2 (M = 256, N = 256) issued by the even
//     ("leader") CTA.  Each CTA TMA-loads its own 128 rows of A and its own
//     128 columns of B into its own shared memory (no multicast; the loads of
//     both CTAs complete on the leader's barrier) and owns 128 rows of the
//     fp32 accumulator in its TMEM.  6-stage ring of 2 x 16 KiB per CTA.
//     Per FLOP this halves the B traffic of each SM.
// Tiles are taken in launch order from a device counter (L.tile_ctr) as each
// CTA (pair) frees up, so the tiles in flight at any moment are neighbours
// in that order and their operands stay in L2; with a fixed round-robin
// deal, the units drift apart over hundreds of waves and the operands of
// several matrices compete for L2 (about 3x the operand bytes read from
// DRAM on the 168-matrix step).
// Roles: warp 0 = TMA producer (one lane); warp 1 = TMEM allocator and MMA
// issuer (one lane of the leader); warps 2..5 = epilogue.  Two 256-column
// TMEM accumulators let the epilogue of one tile overlap the main loop of the
// next.  Epilogue: tcgen05.ld 32 lanes x 32 columns per warp,
// alpha*acc + beta*E, a 32 x 32 bf16 block staged in shared memory with the
// 64-byte swizzle, TMA bulk-tensor store.  A and A^2 are symmetric: only tiles
// touching the upper triangle run; each stores its upper blocks directly and
// mirrored (the transposed block built from 8 x 8 tiles with ldmatrix.trans /
// stmatrix), and the diagonal block is completed from its own upper triangle,
// so every element is written exactly once.
// Operand majorness: Gram and square read both operands K-major; the update
// reads X as an MN-major B operand (X is [K][N] with N contiguous).
// Every mbarrier wait is bounded: on expiry the CTA records MUON_ERR_TIMEOUT,
// drains its own copies and MMAs (again bounded), frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>

#include "kernels.h"

namespace am {

AM_CHECK_READER(read_and_clear_check_gemm_tc)

// Sticky per-device status word (a muon_status code; the first error wins).
__device__ unsigned int g_device_status = 0;

namespace {

__device__ __forceinline__ void raise_status(unsigned int code) { atomicCAS(&g_device_status, 0u, code); }

constexpr int TBN = 256, TBK = 64;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;                   // 2 accumulators x 256 fp32 columns
constexpr uint32_t kOutTileBytes = 32 * 32 * 2;       // one staged 32x32 bf16 output block
constexpr uint32_t kOutBytes = 4 /*warps*/ * 4 /*2 parities x {direct, mirror}*/ * kOutTileBytes;
constexpr long long kWaitLimitCycles = 2000000000LL;  // ~1 s at B200 clocks
constexpr int kTq = 4;                                // slots of the tile-index ring
// threads that free each ring slot: the MMA issuer and the four epilogue
// warps of the leader CTA, and (SM pair) the producer and the four epilogue
// warps of the peer
template <bool PAIR>
constexpr uint32_t kTqTakers = PAIR ? 10u : 5u;

// Per-variant geometry (see the file comment).
template <bool PAIR>
struct Geo {
  static constexpr int kTileM = PAIR ? 256 : 128;                       // rows of a tile
  static constexpr int kStages = PAIR ? 6 : 4;
  static constexpr uint32_t kABytes = 128 * TBK * 2;                    // per CTA: 128 rows x 64
  static constexpr uint32_t kBRows = PAIR ? 128 : 256;                  // B rows (N) per CTA
  static constexpr uint32_t kBBytes = kBRows * TBK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTxBytes = (PAIR ? 2 : 1) * kStageBytes;    // lands on the leader's barrier
  static constexpr size_t kSmemBytes = 1024 + kStages * (size_t)kStageBytes + kOutBytes + 512;
};
static_assert(Geo<true>::kSmemBytes <= 232448 && Geo<false>::kSmemBytes <= 232448, "shared memory budget");

struct TcParams {
  CUtensorMap maps[3 * kMaxGemmGroups];   // per group: operand A, operand B, output C
  GemmLaunch L;
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t a) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t a, uint32_t parity) {
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
// The same with acquire at cluster scope: the phase was completed by a
// release from another CTA of the cluster whose shared-memory writes the
// waiter then reads.
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; returns false (and raises the abort flag) on timeout or when
// another role already aborted.  `cl`: acquire at cluster scope.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity, volatile int* abort_flag,
                                          long long limit = kWaitLimitCycles, bool cl = false) {
  auto try_once = [&]() { return cl ? mbar_try_wait_cl(a, parity) : mbar_try_wait(a, parity); };
  if (try_once()) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (try_once()) return true;
    if ((i & 255u) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > limit) {
        *abort_flag = 1;
        raise_status(MUON_ERR_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t mbar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void ld_shared_v4(uint32_t a, uint32_t& x, uint32_t& y, uint32_t& z, uint32_t& w) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(x), "=r"(y), "=r"(z), "=r"(w) : "r"(a) : "memory");
}
// Byte offset of (row r, byte b) inside a 32 x 64-byte block stored with the
// TMA 64-byte swizzle: 16-byte chunk index XOR ((r >> 1) & 3).
__device__ __forceinline__ uint32_t swz64(int r, int b) {
  return (uint32_t)(r * 64 + ((((b >> 4) ^ (r >> 1)) & 3) << 4) + (b & 15));
}
// Four 8 x 8 tiles of 16-bit values between shared memory and registers; in
// registers lane t holds row t / 4, columns 2 (t % 4) and 2 (t % 4) + 1 of
// tile i in x_i, and lanes 8i .. 8i + 7 give the addresses of tile i's rows.
// The load transposes each tile.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t a, uint32_t& x0, uint32_t& x1, uint32_t& x2, uint32_t& x3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
               : "r"(a)
               : "memory");
}
__device__ __forceinline__ void stsm_x4(uint32_t a, uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x0), "r"(x1), "r"(x2),
               "r"(x3)
               : "memory");
}
// dst <- the transpose of the 32 x 32 block of 16-bit values at src (both
// 64-byte swizzled).  Step a moves tiles (a, 0..3) of src to tiles (0..3, a)
// of dst, each transposed on the way through registers.
__device__ __forceinline__ void transpose_block32(uint32_t src, uint32_t dst, int lane) {
  const int m = lane >> 3, rr = lane & 7;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    uint32_t x0, x1, x2, x3;
    ldsm_x4_trans(src + swz64(8 * a + rr, 16 * m), x0, x1, x2, x3);
    stsm_x4(dst + swz64(8 * m + rr, 16 * a), x0, x1, x2, x3);
  }
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 32 consecutive bf16 of one row of E (cols col0.., masked to < N) -> 4 x uint4.
__device__ __forceinline__ void load_e_chunk(const __nv_bfloat16* erow, int col0, int N, uint4 (&out)[4]) {
  const __nv_bfloat16* e = erow + col0;
  if (col0 + 32 <= N) {
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) out[j4] = __ldg(reinterpret_cast<const uint4*>(e) + j4);
  } else {
    uint32_t w[16] = {};
    for (int j = 0; j < 32 && col0 + j < N; ++j) {
      const uint32_t h = __bfloat16_as_ushort(e[j]);
      w[j >> 1] |= h << (16 * (j & 1));
    }
    for (int j4 = 0; j4 < 4; ++j4) out[j4] = make_uint4(w[4 * j4], w[4 * j4 + 1], w[4 * j4 + 2], w[4 * j4 + 3]);
  }
}

// ---------------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
// Arrive on a peer CTA's barrier, ordering this thread's earlier shared-memory
// writes to the peer (st.shared::cluster) before it at cluster scope.
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t a) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t a) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(a) : "memory");
}
// TMA load into this CTA's shared memory whose completion is signalled on a
// barrier of either CTA of the pair (`mbar` is a shared::cluster address).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t mbar, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
template <bool PAIR>
__device__ __forceinline__ void tc_commit_g(uint32_t mbar) {
  if constexpr (PAIR)
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
  else
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}
template <bool PAIR>
__device__ __forceinline__ void tc_mma_g(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  if constexpr (PAIR)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
template <bool PAIR>
__device__ __forceinline__ void tmem_alloc_g(uint32_t slot_saddr) {
  if constexpr (PAIR) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_saddr),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  } else {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_saddr),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
}
template <bool PAIR>
__device__ __forceinline__ void tmem_dealloc_g(uint32_t taddr) {
  if constexpr (PAIR)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(kTmemCols) : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(kTmemCols) : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets (all >> 4), version 1, 128-byte swizzle (layout 2).
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor, kind::f16: D fp32, A/B bf16, M = m, N = 256.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t b_mn_major, uint32_t m) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major << 16) | ((uint32_t)(TBN >> 3) << 17) |
         ((m >> 4) << 24);
}

// ---------------------------------------------------------------- scheduling
__device__ __forceinline__ bool symmetric_kind(int kind) { return kind == GK_GRAM || kind == GK_SQR; }

struct TileInfo {
  int g, b, m0, n0, nkb;
};

// Symmetric kinds enumerate, column block by column block, the row blocks
// whose tile touches the upper triangle: tm <= 2 tn + 1 for 128-row tiles,
// tm <= tn for 256-row tiles.
template <bool PAIR>
__device__ __forceinline__ TileInfo decode_tile(const GemmLaunch& L, int tile) {
  int g = 0;
  while (g + 1 < L.num_groups && L.g[g + 1].tile_begin <= tile) ++g;
  const GemmGroup& G = L.g[g];
  int t = tile - G.tile_begin;
  const int b = t / G.tiles_per_mat;
  t -= b * G.tiles_per_mat;
  int tm, tn;
  if (symmetric_kind(G.kind)) {
    tn = 0;
    for (;;) {
      const int cnt = PAIR ? min(tn + 1, G.tiles_m) : min(2 * tn + 2, G.tiles_m);
      if (t < cnt) break;
      t -= cnt;
      ++tn;
    }
    tm = t;
  } else {
    // column strips of X outermost: the concurrently running tiles share one
    // strip of the B operand (read from HBM about once) and all of A (s x s)
    tm = t % G.tiles_m;
    tn = t / G.tiles_m;
  }
  TileInfo ti;
  ti.g = g;
  ti.b = b;
  ti.m0 = tm * Geo<PAIR>::kTileM;
  ti.n0 = tn * TBN;
  ti.nkb = (G.K + TBK - 1) / TBK;
  return ti;
}

__device__ __forceinline__ float bf16_bits_to_f(uint32_t h) { return __uint_as_float(h << 16); }

// ---------------------------------------------------------------- kernel
template <bool PAIR>
__global__ void __launch_bounds__(kThreads, 1) k_gemm_tc(const __grid_constant__ TcParams P) {
  using Gm = Geo<PAIR>;
  constexpr int S = Gm::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sA = base;                                 // S x 16 KiB
  const uint32_t sB = base + S * Gm::kABytes;               // S x kBBytes
  const uint32_t sOut = sB + S * Gm::kBBytes;               // 32 KiB of output staging
  uint8_t* ctl = smem + S * Gm::kStageBytes + kOutBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ctl);        // full[S], empty[S], tfull[2], tempty[2], drain
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * S;
  const uint32_t tfull0 = empty0 + 8 * S, tempty0 = tfull0 + 16, drain = tempty0 + 16;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(ctl + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 196);
  // ring of tile indices: full[kTq], empty[kTq], index[kTq]
  const uint32_t tqf0 = smem_u32(ctl + 256), tqe0 = tqf0 + 8 * kTq;
  const uint32_t tq_addr = tqe0 + 8 * kTq;
  volatile int* tq = reinterpret_cast<volatile int*>(ctl + 256 + 16 * kTq);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GemmLaunch& L = P.L;
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, (PAIR ? 2 : 1) * 4);   // one arrive per epilogue warp of each CTA
    }
    mbar_init(drain, 1);
    for (int k = 0; k < kTq; ++k) {
      mbar_init(tqf0 + 8 * k, 1);
      mbar_init(tqe0 + 8 * k, kTqTakers<PAIR>);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < L.num_groups; ++g)
      for (int k = 0; k < 3; ++k)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.maps[3 * g + k])) : "memory");
  }
  if (warp == 1) tmem_alloc_g<PAIR>(smem_u32(const_cast<uint32_t*>(tmem_slot)));
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();    // peer barriers initialised before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // The tile sequence.  The leader CTA's producer takes each next tile index
  // from L.tile_ctr as it starts a tile and publishes it in its ring slot
  // (and, SM pair, in the peer CTA's); the MMA issuer, the epilogue warps and
  // the peer's producer read the slots in order and free each on the
  // leader's barrier.  -1 ends the sequence; -2 means a wait gave up.
  auto tq_advance = [&](int& qi, uint32_t& qph) {
    if (++qi == kTq) { qi = 0; qph ^= 1u; }
  };
  auto tq_publish = [&](int& qi, uint32_t& qph) -> int {
    // (the peer's frees are released at cluster scope: acquire at cluster scope)
    if (!mbar_wait(tqe0 + 8 * qi, qph ^ 1u, abort_flag, kWaitLimitCycles, PAIR)) return -2;
    int t = (int)atomicAdd(L.tile_ctr, 1u);
    if (t >= L.total_tiles) t = -1;
    tq[qi] = t;
    if constexpr (PAIR) {
      st_cluster_u32(map_to_rank(tq_addr + 4 * qi, 1), (uint32_t)t);
      mbar_arrive_release_cluster(map_to_rank(tqf0 + 8 * qi, 1));
    }
    mbar_arrive(tqf0 + 8 * qi);
    tq_advance(qi, qph);
    return t;
  };
  auto tq_read = [&](int qi, uint32_t qph) -> int {
    if (!mbar_wait(tqf0 + 8 * qi, qph, abort_flag, kWaitLimitCycles, PAIR)) return -2;
    return tq[qi];
  };
  auto tq_free = [&](int qi) {   // after the slot's index has been read
    if constexpr (PAIR) {
      if (leader) mbar_arrive(tqe0 + 8 * qi);
      else mbar_arrive_release_cluster(map_to_rank(tqe0 + 8 * qi, 0));
    } else {
      mbar_arrive(tqe0 + 8 * qi);
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      for (;;) {
        int tile;
        if (leader) {
          tile = tq_publish(qi, qph);
        } else {
          tile = tq_read(qi, qph);
          if (tile != -2) tq_free(qi);
          tq_advance(qi, qph);
        }
        if (tile == -2) { ok = false; break; }
        if (tile < 0) break;
        const TileInfo ti = decode_tile<PAIR>(L, tile);
        const GemmGroup& G = L.g[ti.g];
        const CUtensorMap* mA = &P.maps[3 * ti.g];
        const CUtensorMap* mB = &P.maps[3 * ti.g + 1];
        const bool upd = G.kind == GK_UPD;
        const int arow = ti.m0 + (int)rank * 128;
        const int bcol = ti.n0 + (int)rank * (int)Gm::kBRows;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t fb_local = full0 + 8 * stage;
          if (leader) mbar_expect_tx(fb_local, Gm::kTxBytes);
          const uint32_t fb = PAIR ? map_to_rank(fb_local, 0) : fb_local;
          const uint32_t a_dst = sA + stage * Gm::kABytes, b_dst = sB + stage * Gm::kBBytes;
          if constexpr (PAIR) {
            tma_load_3d_pair(a_dst, mA, fb, kb * TBK, arow, ti.b);
            if (upd) {
#pragma unroll
              for (int j = 0; j < (int)Gm::kBRows / 64; ++j)
                tma_load_3d_pair(b_dst + j * (64 * TBK * 2), mB, fb, bcol + 64 * j, kb * TBK, ti.b);
            } else {
              tma_load_3d_pair(b_dst, mB, fb, kb * TBK, bcol, ti.b);
            }
          } else {
            tma_load_3d(a_dst, mA, fb, kb * TBK, arow, ti.b);
            if (upd) {
#pragma unroll
              for (int j = 0; j < (int)Gm::kBRows / 64; ++j)
                tma_load_3d(b_dst + j * (64 * TBK * 2), mB, fb, bcol + 64 * j, kb * TBK, ti.b);
            } else {
              tma_load_3d(b_dst, mB, fb, kb * TBK, bcol, ti.b);
            }
          }
          ++issued;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      if (!ok && leader) {
        // drain: wait (bounded) for every stage's most recent loads (of both
        // CTAs of a pair, which complete on this barrier) to land
        for (uint32_t k = 0; k < (uint32_t)S && k < issued; ++k) {
          const uint32_t idx = issued - 1 - k;
          const uint32_t st = idx % S, ph = (idx / S) & 1u;
          const long long t0 = clock64();
          while (!mbar_try_wait(full0 + 8 * st, ph) && clock64() - t0 < kWaitLimitCycles) {}
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, any = false;
      int it = 0;
      int qi = 0;
      uint32_t qph = 0;
      for (;; ++it) {
        const int tile = tq_read(qi, qph);
        if (tile == -2) { ok = false; break; }
        tq_free(qi);
        tq_advance(qi, qph);
        if (tile < 0) break;
        const TileInfo ti = decode_tile<PAIR>(L, tile);
        const bool upd = L.g[ti.g].kind == GK_UPD;
        const uint32_t idesc = make_idesc(upd ? 1u : 0u, (uint32_t)Gm::kTileM);
        const int acc = it & 1;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TBN);
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = sA + stage * Gm::kABytes, b0 = sB + stage * Gm::kBBytes;
#pragma unroll
          for (int k = 0; k < TBK / 16; ++k) {
            const uint64_t ad = make_sdesc(a0 + k * 32, 16, 1024);
            const uint64_t bd = upd ? make_sdesc(b0 + k * 16 * 128, 64 * TBK * 2, 1024)
                                    : make_sdesc(b0 + k * 32, 16, 1024);
            tc_mma_g<PAIR>(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
            any = true;
          }
          tc_commit_g<PAIR>(empty0 + 8 * stage);
          if constexpr (PAIR) tc_commit_g<PAIR>(map_to_rank(empty0 + 8 * stage, 1));
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_g<PAIR>(tfull0 + 8 * acc);
        if constexpr (PAIR) tc_commit_g<PAIR>(map_to_rank(tfull0 + 8 * acc, 1));
        if (acc == 1) acc_phase ^= 1u;
      }
      if (!ok && any) {
        tc_commit_g<PAIR>(drain);
        const long long t0 = clock64();
        while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitLimitCycles) {}
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp owns 32 rows (its TMEM lane quadrant) and walks the tile in
    // 32-column chunks: TMEM -> registers -> alpha*acc + beta*E -> bf16 ->
    // a 32x32 block staged in shared memory (64-byte swizzle) -> TMA store.
    // Symmetric kinds also store the transposed block (mirror); the block on
    // the diagonal is completed from its own upper triangle in shared memory.
    const int q = warp & 3;                          // TMEM lane quadrant of this warp
    const uint32_t wbuf = sOut + (uint32_t)(warp - 2) * 4u * kOutTileBytes;
    const uint32_t tempty_leader0 = PAIR ? map_to_rank(tempty0, 0) : tempty0;
    uint32_t acc_phase = 0, par = 0;
    int it = 0;
    int qi = 0;
    uint32_t qph = 0;
    for (;; ++it) {
      // lane 0 takes the next index for the warp
      int tile = 0;
      if (lane == 0) {
        tile = tq_read(qi, qph);
        if (tile != -2) tq_free(qi);
      }
      tile = __shfl_sync(0xffffffffu, tile, 0);
      tq_advance(qi, qph);
      if (tile < 0) break;
      const TileInfo ti = decode_tile<PAIR>(L, tile);
      const GemmGroup& G = L.g[ti.g];
      const int acc = it & 1;
      if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag)) break;
      tc_fence_after();
      float alpha = G.alpha0, beta = G.beta0;
      if (G.rho) {
        const float r = G.rho[ti.b];
        for (int p = 0; p < G.pa; ++p) alpha *= r;
        for (int p = 0; p < G.pb; ++p) beta *= r;
      }
      const int r0 = ti.m0 + (int)rank * 128 + q * 32;   // first row of this warp's strip
      const int row = r0 + lane;
      const bool sym = symmetric_kind(G.kind);
      const CUtensorMap* mC = &P.maps[3 * ti.g + 2];
      const __nv_bfloat16* Erow =
          (G.E && row < G.M) ? reinterpret_cast<const __nv_bfloat16*>(G.E) + (int64_t)ti.b * G.se +
                                   (int64_t)row * G.lde
                             : nullptr;
      // chunk ch is needed when it is inside N and (symmetric) not below the diagonal
      auto wanted = [&](int ch) {
        const int c0 = ti.n0 + ch * 32;
        return r0 < G.M && c0 < G.N && !(sym && c0 < r0);
      };
      // fused reductions of the output against itself and against dotu
      const bool dots = G.dotp != nullptr;
      const __nv_bfloat16* Urow =
          (dots && row < G.M) ? reinterpret_cast<const __nv_bfloat16*>(G.dotu) + (int64_t)ti.b * G.sc +
                                    (int64_t)row * G.ldc
                              : nullptr;
      float s_cc = 0.f, s_cu = 0.f;
      uint4 en[4] = {}, un[4] = {};
      int next = 0;
      while (next < TBN / 32 && !wanted(next)) ++next;
      // element range of a 32-column chunk of this lane's row (for the checked build)
      auto e_ok = [&](int64_t ld, int64_t stride, int col) {
        return AM_IN((int64_t)ti.b * stride + (int64_t)row * ld + col, min(32, G.N - col), (int64_t)G.count * stride);
      };
      if (next < TBN / 32 && Erow && e_ok(G.lde, G.se, ti.n0 + next * 32)) load_e_chunk(Erow, ti.n0 + next * 32, G.N, en);
      if (next < TBN / 32 && Urow && e_ok(G.ldc, G.sc, ti.n0 + next * 32)) load_e_chunk(Urow, ti.n0 + next * 32, G.N, un);
      while (next < TBN / 32) {
        const int ch = next;
        const int col0 = ti.n0 + ch * 32;
        const uint4 ec[4] = {en[0], en[1], en[2], en[3]};
        const uint4 uc[4] = {un[0], un[1], un[2], un[3]};
        ++next;
        while (next < TBN / 32 && !wanted(next)) ++next;
        if (next < TBN / 32 && Erow && e_ok(G.lde, G.se, ti.n0 + next * 32)) load_e_chunk(Erow, ti.n0 + next * 32, G.N, en);
        if (next < TBN / 32 && Urow && e_ok(G.ldc, G.sc, ti.n0 + next * 32)) load_e_chunk(Urow, ti.n0 + next * 32, G.N, un);
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TBN + ch * 32), r);
        uint32_t pk[16];
        {
          const uint32_t ew[16] = {ec[0].x, ec[0].y, ec[0].z, ec[0].w, ec[1].x, ec[1].y, ec[1].z, ec[1].w,
                                   ec[2].x, ec[2].y, ec[2].z, ec[2].w, ec[3].x, ec[3].y, ec[3].z, ec[3].w};
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            float v0 = alpha * __uint_as_float(r[2 * h]), v1 = alpha * __uint_as_float(r[2 * h + 1]);
            if (Erow) {
              v0 += beta * bf16_bits_to_f(ew[h] & 0xFFFFu);
              v1 += beta * bf16_bits_to_f(ew[h] >> 16);
            }
            const __nv_bfloat162 p2 = __floats2bfloat162_rn(v0, v1);
            pk[h] = *reinterpret_cast<const uint32_t*>(&p2);
          }
        }
        if (Urow) {
          // columns past N hold 0 in both (zero-filled operands and addend)
          const uint32_t uw[16] = {uc[0].x, uc[0].y, uc[0].z, uc[0].w, uc[1].x, uc[1].y, uc[1].z, uc[1].w,
                                   uc[2].x, uc[2].y, uc[2].z, uc[2].w, uc[3].x, uc[3].y, uc[3].z, uc[3].w};
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const float v0 = bf16_bits_to_f(pk[h] & 0xFFFFu), v1 = bf16_bits_to_f(pk[h] >> 16);
            s_cc = fmaf(v0, v0, fmaf(v1, v1, s_cc));
            s_cu = fmaf(v0, bf16_bits_to_f(uw[h] & 0xFFFFu), fmaf(v1, bf16_bits_to_f(uw[h] >> 16), s_cu));
          }
        }
        // staging buffers of this parity are free once the group issued two
        // chunks ago has been read by the TMA unit
        if (lane == 0) bulk_wait_read1();
        __syncwarp();
        const uint32_t dbuf = wbuf + par * 2u * kOutTileBytes, mbuf = dbuf + kOutTileBytes;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(dbuf + swz64(lane, 16 * c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        const bool diag = sym && col0 == r0;
        const bool mirror = sym && col0 > r0;
        if (diag || mirror) {
          // the transposed block: the mirror's store, or (diagonal block)
          // the source of its lower part
          __syncwarp();
          transpose_block32(dbuf, mbuf, lane);
        }
        if (diag) {
          __syncwarp();
          // lower part of the diagonal block <- its upper part: row `lane`
          // takes the columns left of the diagonal from the transposed copy
          uint32_t tw[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) ld_shared_v4(mbuf + swz64(lane, 16 * c), tw[4 * c], tw[4 * c + 1], tw[4 * c + 2], tw[4 * c + 3]);
#pragma unroll
          for (int w = 0; w < 16; ++w) {
            if (2 * w + 1 < lane) pk[w] = tw[w];
            else if (2 * w < lane) pk[w] = (pk[w] & 0xFFFF0000u) | (tw[w] & 0xFFFFu);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c)
            st_shared_v4(dbuf + swz64(lane, 16 * c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        if (G.colsq) {
          // column sums of the squared stored values of this 32 x 32 block:
          // lane l sums columns 2 (l % 16), +1 over rows 16 (l / 16) .. +15
          __syncwarp();
          const int cp = lane & 15, rh = lane >> 4;
          float q0 = 0.f, q1 = 0.f;
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const uint32_t w = ld_shared_u32(dbuf + swz64(16 * rh + r, 4 * cp));
            const float v0 = bf16_bits_to_f(w & 0xFFFFu), v1 = bf16_bits_to_f(w >> 16);
            q0 = fmaf(v0, v0, q0);
            q1 = fmaf(v1, v1, q1);
          }
          q0 += __shfl_xor_sync(0xffffffffu, q0, 16);
          q1 += __shfl_xor_sync(0xffffffffu, q1, 16);
          const int64_t qo = (int64_t)ti.b * G.colsq_batch + (int64_t)(r0 >> 5) * G.colsq_ld + col0 + 2 * cp;
          if (lane < 16 && AM_IN(qo, 2, (int64_t)G.count * G.colsq_batch))
            *reinterpret_cast<float2*>(G.colsq + qo) = make_float2(q0, q1);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0 && !G.no_store) {
          tma_store_3d(mC, dbuf, col0, r0, ti.b);
          if (mirror) tma_store_3d(mC, mbuf, r0, col0, ti.b);
          bulk_commit();
        }
        par ^= 1u;
      }
      if (dots) {
        // one slot per (tile, epilogue warp of the pair); unused slots of the
        // single-SM variant are written as zero
        s_cc = warp_sum(s_cc);
        s_cu = warp_sum(s_cu);
        if (lane == 0) {
          const int tin = ti.m0 / Gm::kTileM + G.tiles_m * (ti.n0 / TBN);
          const int64_t so = ((int64_t)ti.b * G.tiles_per_mat + tin) * 16;
          double* slot = G.dotp + so;
          const int w = (int)rank * 4 + q;
          if (AM_IN(so, 16, (int64_t)G.count * G.tiles_per_mat * 16)) {
            slot[2 * w] = (double)s_cc;
            slot[2 * w + 1] = (double)s_cu;
            if (!PAIR) {
              slot[2 * (w + 4)] = 0.0;
              slot[2 * (w + 4) + 1] = 0.0;
            }
          }
        }
      }
      // this warp's TMEM reads of the accumulator are complete: release it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) mbar_arrive_cluster(tempty_leader0 + 8 * acc);
        else mbar_arrive(tempty0 + 8 * acc);
      }
      if (acc == 1) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // the leader's MMAs write the peer's TMEM: free it only after both are done
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_g<PAIR>(tmem_base);
  }
}

// Exercises the timeout path of mbar_wait: one thread waits on a barrier
// that nothing ever arrives on; after `limit` cycles the wait gives up and
// records MUON_ERR_TIMEOUT.
__global__ void k_wait_selftest(long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, limit);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t ld_elems,
               uint64_t batch_elems, uint32_t box0, uint32_t box1,
               CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = get_encode();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {ld_elems * 2, batch_elems * 2};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Per-device launch facts for one kernel variant: the shared-memory opt-in
// and the number of CTA pairs that can be resident at once.
struct DeviceFacts {
  cudaError_t err = cudaSuccess;
  int units = 0;
};

template <bool PAIR>
DeviceFacts device_facts(int num_sms) {
  static std::mutex mu;
  static std::map<int, DeviceFacts> cache;
  int dev = 0;
  DeviceFacts f;
  if ((f.err = cudaGetDevice(&dev)) != cudaSuccess) return f;
  std::lock_guard<std::mutex> g(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  f.err = cudaFuncSetAttribute(k_gemm_tc<PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)Geo<PAIR>::kSmemBytes);
  if (f.err == cudaSuccess) {
    if constexpr (PAIR) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = Geo<PAIR>::kSmemBytes;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      f.err = cudaOccupancyMaxActiveClusters(&clusters, k_gemm_tc<PAIR>, &cfg);
      f.units = clusters;
    } else {
      f.units = num_sms;
    }
  }
  if (f.err == cudaSuccess && f.units <= 0) f.err = cudaErrorInvalidConfiguration;
  cache[dev] = f;
  return f;
}

}  // namespace

cudaError_t launch_wait_selftest(long long limit_cycles, cudaStream_t st) {
  k_wait_selftest<<<1, 32, 0, st>>>(limit_cycles);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_status(unsigned int* out) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v));
  if (e != cudaSuccess) return e;
  *out = v;
  if (v != 0) e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
  return e;
}

int tc_tile_count(int kind, int M, int N, bool pair, int* tiles_m, int* tiles_n) {
  const int tile_m = pair ? 256 : 128;
  const int tm = (M + tile_m - 1) / tile_m, tn = (N + TBN - 1) / TBN;
  *tiles_m = tm;
  *tiles_n = tn;
  if (kind == GK_UPD) return tm * tn;
  int c = 0;
  for (int j = 0; j < tn; ++j) c += std::min(pair ? j + 1 : 2 * j + 2, tm);
  return c;
}

bool tc_encode_maps(const GemmLaunch& L, bool pair, void* maps_out) {
  CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(maps_out);
  const uint32_t brows = pair ? 128 : 256;
  for (int g = 0; g < L.num_groups; ++g) {
    const GemmGroup& G = L.g[g];
    if (!encode_3d(&maps[3 * g], G.A, G.K, G.M, G.count, G.lda, G.sa, TBK, 128)) return false;
    bool ok;
    if (G.kind == GK_UPD)
      ok = encode_3d(&maps[3 * g + 1], G.B, G.N, G.K, G.count, G.ldb, G.sb, 64, TBK);
    else
      ok = encode_3d(&maps[3 * g + 1], G.B, G.K, G.N, G.count, G.ldb, G.sb, TBK, brows);
    if (!ok) return false;
    if (!encode_3d(&maps[3 * g + 2], G.C, G.N, G.M, G.count, G.ldc, G.sc, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return false;
  }
  return true;
}

cudaError_t launch_gemm_tc(const GemmLaunch& L, const void* maps, int num_sms, bool pair, cudaStream_t st) {
  if (L.total_tiles == 0) return cudaSuccess;
  TcParams* P = new TcParams;
  std::memcpy(P->maps, maps, sizeof(CUtensorMap) * 3 * L.num_groups);
  P->L = L;
  cudaError_t e;
  if (pair) {
    const DeviceFacts f = device_facts<true>(num_sms);
    if (f.err != cudaSuccess) { delete P; return f.err; }
    const int clusters = std::min(f.units, L.total_tiles);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Geo<true>::kSmemBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_gemm_tc<true>, *P);
  } else {
    const DeviceFacts f = device_facts<false>(num_sms);
    if (f.err != cudaSuccess) { delete P; return f.err; }
    const int grid = std::min(f.units, L.total_tiles);
    k_gemm_tc<false><<<grid, kThreads, Geo<false>::kSmemBytes, st>>>(*P);
    e = cudaGetLastError();
  }
  delete P;
  return e;
}

}  // namespace am
