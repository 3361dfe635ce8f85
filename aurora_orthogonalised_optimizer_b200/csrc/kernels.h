// Internal launch interface between the host engine and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace am {

// ---------------------------------------------------------------- GEMM groups
// One group = one shape bucket of `count` same-shape matrices stored as a
// batched tensor [count][rows][ld].  All operands use the Newton-Schulz dtype.
enum GemmKind {
  GK_GRAM = 0,   // C[s x s] = alpha * X X^T          (A = X, B = X, K = l)
  GK_SQR = 1,    // C[s x s] = alpha * A A + beta * E (E = A), symmetric A
  GK_UPD = 2     // C[s x l] = alpha * B X + beta * E (E = X), K = s
};

struct GemmGroup {
  int kind;
  int count;
  int M, N, K;
  int tiles_m, tiles_n, tiles_per_mat;
  int tile_begin;                 // first tile of this group in the launch
  const void* A; int64_t lda, sa; // operand A: [count][M][lda], K contiguous
  const void* B; int64_t ldb, sb; // operand B: GRAM/SQR: [count][N][ldb] (K contiguous);
                                  //            UPD: [count][K][ldb] (N contiguous)
  void* C; int64_t ldc, sc;
  const void* E; int64_t lde, se; // epilogue addend (may be null)
  const float* rho;               // per-batch normalisation scale (may be null)
  float alpha0, beta0;            // alpha = alpha0 * rho^pa, beta = beta0 * rho^pb
  int pa, pb;
  // Update kind, tensor-core path only: when dotp is set the epilogue also
  // forms per-warp partials of <C, C> and <C, dotu> (dotu laid out like C,
  // bf16) over the stored bf16 values:
  // dotp[((b * tiles_per_mat + tile) * 8 + warp) * 2 + {0, 1}].
  const void* dotu;
  double* dotp;
  // Update kind, tensor-core path only: when colsq is set the epilogue also
  // writes, per 32-row block of C, the column sums of the squared stored
  // bf16 values: colsq[b * colsq_batch + (row / 32) * colsq_ld + col].
  float* colsq;
  int64_t colsq_ld, colsq_batch;
  int no_store;                   // C itself is not needed (only colsq): skip its stores
};

constexpr int kMaxGemmGroups = 16;

struct GemmLaunch {
  int num_groups;
  int total_tiles;
  int dtype;                      // kF32 or kBF16
  // tensor-core path: the next tile to take (device counter, zero at launch);
  // each CTA (pair) takes tiles in this order as it frees up
  unsigned int* tile_ctr;
  GemmGroup g[kMaxGemmGroups];
};

// SIMT grouped GEMM (fp32 FMA accumulation; bf16 or fp32 storage): tiles of
// kSimtTile x kSimtTile outputs; the symmetric kinds run only the tiles on or
// above the diagonal (simt_tile_count gives a group's tiles per matrix).
constexpr int kSimtTile = 128;
int simt_tile_count(int kind, int M, int N, int* tiles_m, int* tiles_n);
cudaError_t launch_gemm_simt(const GemmLaunch& L, cudaStream_t st);

// tcgen05 grouped GEMM (bf16 operands, fp32 accumulation in TMEM, TMA loads).
// `maps` holds three CUtensorMap (128 B each) per group: operand A, operand B, output C.
// `pair` selects the SM-pair variant (clusters of two CTAs, 256 x 256 tiles).
cudaError_t launch_gemm_tc(const GemmLaunch& L, const void* maps, int num_sms, bool pair, cudaStream_t st);
bool tc_encode_maps(const GemmLaunch& L, bool pair, void* maps_out);  // host: builds the tensor maps
int tc_tile_count(int kind, int M, int N, bool pair, int* tiles_m, int* tiles_n);
cudaError_t read_and_clear_device_status(unsigned int* out);  // current device
cudaError_t launch_wait_selftest(long long limit_cycles, cudaStream_t st);

// ---------------------------------------------------------------- element-wise
// Streaming kernels work on 64 x 64 tiles; a block walks kEwTilesPerCta
// consecutive tiles of one matrix (launch ceil(tiles / kEwTilesPerCta)
// blocks per matrix); reductions still leave one set of partials per tile.
constexpr int kEwTilesPerCta = 4;
// Flat variants (rows contiguous, length a multiple of 8): chunks of
// kFlatChunk elements, one partial slot per chunk.
constexpr int64_t kFlatChunk = 4096;
// Row-dot pass of the power iteration: 8 warps x kMatvecRowsPerWarp rows.
constexpr int kMatvecRowsPerWarp = 4;
constexpr int kMatvecRowsPerCta = 8 * kMatvecRowsPerWarp;
// Column reductions (Aurora column norms, power-iteration column dots):
// one block per kColStrip columns of the X orientation.
constexpr int kColStrip = 256;
// Power-iteration column dots: one block per kColDotStrip columns.
constexpr int kColDotStrip = 64;
cudaError_t launch_prologue(const MatTable& t, int nblk, int mode, float mu, int nesterov,
                            int want_w2, double* partials, cudaStream_t st);
cudaError_t launch_finalize_sums(const MatTable& t, const double* partials, int nq, int slot0,
                                 int slot1, double* scal, cudaStream_t st);
// Aurora D update from a pass over U (FP32 / SIMT modes).
cudaError_t launch_colnorm(const MatTable& t, int nblk, float pp_eps, float beta, cudaStream_t st);
cudaError_t launch_scale_cols(const MatTable& t, int nblk, double* partials, cudaStream_t st);
// Aurora D from per-row-block column sums of squares (MatDesc::colsq):
// k_colsq_partial forms them from uX per kColsqRows rows (blocks of
// 8 kColsqRows rows x kColStrip columns); the last update GEMM of a
// non-final polar forms them from U per 32 rows.  launch_colsq_update (one
// block per kColStrip columns) sums them: mode 0 D init (kColsqRows-row
// partials), mode 1 D update (32-row partials).
constexpr int kColsqRows = 128;
cudaError_t launch_colsq_partial(const MatTable& t, int nblk, cudaStream_t st);
cudaError_t launch_colsq_update(const MatTable& t, int nblk, int mode, float pp_eps, float beta, cudaStream_t st);
cudaError_t launch_scalars(const MatTable& t, int op, int src_slot, float ns_eps, float contra,
                           float target_uw, double* scal, cudaStream_t st);
cudaError_t launch_matvec(const MatTable& t, int nblk, int dir, cudaStream_t st);
cudaError_t launch_vecop(const MatTable& t, int which, int mode, int len_is_s_when_flag0,
                         double* scal, cudaStream_t st);
cudaError_t launch_dots(const MatTable& t, int nblk, double* partials, cudaStream_t st);
cudaError_t launch_epilogue(const MatTable& t, int nblk, float lr, int update_w, const double* scal,
                            cudaStream_t st);
// Optimizer-step prologue, tall, m and n multiples of 64, bf16 grads / params / NS storage.
cudaError_t launch_prologue_tall_bf16(const MatTable& t, int nblk, float mu, int nesterov, int want_w2,
                                      double* partials, cudaStream_t st);
// Aurora input scaling with bf16 NS storage and contiguous rows, by column
// strips: blocks of kStripCols columns x kStripRows rows,
// one partial slot per block (cdiv(l, kStripCols) * cdiv(s, kStripRows) of
// them, never more than the matrix's 64 x 64 tiles).
constexpr int kStripCols = 2048, kStripRows = 64;
cudaError_t launch_scale_cols_strip_bf16(const MatTable& t, int nblk, double* partials, cudaStream_t st);
// Flat (wide / square, rows a multiple of 8) and bf16 params and NS storage.
cudaError_t launch_epilogue_flat_bf16(const MatTable& t, int nblk, float lr, int update_w, const double* scal,
                                      cudaStream_t st);
// Tall matrices with m, n multiples of 64, bf16 params and bf16 NS storage.
cudaError_t launch_epilogue_tall_bf16(const MatTable& t, int nblk, float lr, int update_w, const double* scal,
                                      cudaStream_t st);
cudaError_t launch_sumsq_wv(const MatTable& t, int nblk, double* partials, cudaStream_t st);
cudaError_t launch_scale_v(const MatTable& t, int nblk, const double* scal, cudaStream_t st);
cudaError_t launch_copy_rho(const MatTable& t, const double* scal, cudaStream_t st);
cudaError_t launch_prologue_flat(const MatTable& t, int nblk, int mode, float mu, int nesterov, int want_w2,
                                 double* partials, cudaStream_t st);
cudaError_t launch_scale_cols_flat(const MatTable& t, int nblk, double* partials, cudaStream_t st);
cudaError_t launch_dots_flat(const MatTable& t, int nblk, double* partials, cudaStream_t st);
cudaError_t launch_epilogue_flat(const MatTable& t, int nblk, float lr, int update_w, const double* scal,
                                 cudaStream_t st);
// Fused power-iteration pass (powiter.cu): one read of X (s x l) per pass.
enum GramVecMode {
  GV_DOT_ACC = 0,   // z = X y (written), partial X^T z
  GV_DOT = 1,       // z = X y only
  GV_ACC = 2        // partial X^T z with z given
};
int64_t gv_max_ldl(int ns_dtype);   // longest row (elements, padded) the fused pass takes
cudaError_t launch_gramvec(const MatTable& t, int nblk, int mode, cudaStream_t st);
cudaError_t launch_gv_reduce(const MatTable& t, int normalise, cudaStream_t st);
cudaError_t read_and_clear_gv_status(unsigned int* out);
cudaError_t launch_sigma_out(const MatTable& t, const double* scal, float* sigma_out, cudaStream_t st);

// Checked build: read and clear each file's check word (source line of the
// first failed index test, 0 if none; always 0 in the normal build).
cudaError_t read_and_clear_check_elementwise(unsigned int* out);
cudaError_t read_and_clear_check_powiter(unsigned int* out);
cudaError_t read_and_clear_check_gemm_tc(unsigned int* out);
cudaError_t read_and_clear_check_gemm_simt(unsigned int* out);
cudaError_t read_and_clear_check_adamw(unsigned int* out);
cudaError_t launch_bounds_selftest(cudaStream_t st);

}  // namespace am
