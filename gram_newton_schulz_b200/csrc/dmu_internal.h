// Internal types shared by the planner (plan.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dmu.h"

namespace dmu {

// ---------------------------------------------------------------- tiles
// One CTA computes a BM x BN fp32 tile in TMEM with tcgen05.mma
// (M = 128, N = 256, K = 16 per instruction), K-blocks of BK = 64 bf16
// (one 128-byte swizzle atom per row).
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int A_PART_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_PART_BYTES = BN * BK * 2;  // 32 KB
constexpr int GEMM_THREADS = 320;          // TMA warp, MMA warp, 8 epilogue warps
constexpr int EPI_WARPS = 8;               // two per TMEM lane quarter, each on half the columns
constexpr int TMEM_COLS = 512;             // two BN-column accumulators

constexpr int MAX_MAPS = 16;
constexpr int MAX_PROBS = 8;

// Gram-space storage slots (each a bf16 matrix); hi/lo pairs.
enum GramSlot : int {
  SLOT_G_HI = 0, SLOT_G_LO, SLOT_R_HI, SLOT_R_LO, SLOT_T_HI, SLOT_T_LO,
  SLOT_PA_HI, SLOT_PA_LO, SLOT_PB_HI, SLOT_PB_LO, NUM_SLOTS
};
// fp32 path: one fp32 matrix per quantity.
enum GramSlotF32 : int { FSLOT_G = 0, FSLOT_R, FSLOT_T, FSLOT_PA, FSLOT_PB, NUM_FSLOTS };

enum Epi : int { EPI_GRAM = 0, EPI_UPDATE = 1 };
enum AlphaMode : int { ALPHA_CONST = 0, ALPHA_INV2 = 1, ALPHA_INV = 2 };

// Term bits: which bf16 products the MMA warp issues per K slice.
enum Terms : int { TERM_HH = 1, TERM_HL = 2, TERM_LH = 4 };

// Operand kind of a tensor-core launch: bf16 (kind::f16, K = 16 per MMA)
// or tf32 (kind::tf32 on fp32 storage, K = 8 per MMA).  Either way a
// K-block is one 128-byte swizzle row: 64 bf16 or 32 fp32 elements.
enum MmaKind : int { KIND_BF16 = 0, KIND_TF32 = 1, KIND_F16 = 2 };

// Storage format of an epilogue input/output matrix: bf16 hi/lo pair,
// fp32, or fp16 hi/lo pair (values pre-scaled by a power of two chosen by
// the planner so fp16's exponent range holds them).
enum Fmt : int { FMT_PAIR = 0, FMT_F32 = 1, FMT_PAIR_H = 2 };

// One grouped-GEMM problem: `count` independent matrices of the same
// geometry.  Output tile (bi, bj) of matrix `mat` is
//   D[i][j] = sum_k A(i, k) * B(j, k),   i in [0, M), j in [0, N)
// where A and B are read by TMA from 3-D tensor maps; z = base + mat.
struct GemmProblem {
  int count, M, N, K;
  int tiles_m, tiles_n, tiles_per_mat;
  int tile_begin;       // first global tile index of this problem
  int sym;              // upper-triangle tiles only, mirrored write (M == N)
  int a_map, b_map;     // indices into GemmParams::maps
  int a_mn, b_mn;       // 1: operand is MN-major (M/N contiguous)
  // Half-stored symmetric operands: only 256 x 256 blocks (r, c) with
  // r <= c hold data.  A K-atom of rows in block r and columns in block c
  // is read directly (K-major, *_map) when r <= c, else as the transposed
  // block (MN-major, *_map_t).  half_out: the output is written half-stored
  // (whole tiles, no mirror).
  int half_a, half_b, half_out;
  int a_map_t, b_map_t;
  int a_z[2], b_z[2];   // z base of the hi and lo parts
  int terms;            // Terms bits
  // epilogue
  int epi;
  int alpha_mode;
  float alpha, beta, gamma, gamma2;
  const float* inv;     // per-matrix 1/(||M||+eps), indexed by inv_base + mat
  int inv_base;
  // EPI_GRAM: out = alpha' * acc + beta * Cin + gamma * I  (bf16 hi/lo pair)
  const __nv_bfloat16* cin_hi;
  const __nv_bfloat16* cin_lo;
  __nv_bfloat16* out_hi;
  __nv_bfloat16* out_lo;   // may be null
  __nv_bfloat16* out2_hi;  // optional second output out + gamma2 * I
  __nv_bfloat16* out2_lo;
  long long ld;            // row stride (elements) of Cin/out
  long long mat_stride;    // matrix stride (elements) of Cin/out
  int cin_fmt, out_fmt, out2_fmt;  // Fmt of Cin, out, out2
  float scale2;            // out2 = scale2 * out + gamma2 * I
  const float* cin_f;      // FMT_F32 variants of Cin / out / out2
  float* out_f;
  float* out2_f;
  // EPI_UPDATE: W += alpha * inv * acc in W's layout; O = inv * acc
  void* const* w_ptrs;     // device table, indexed by ptr_base + mat
  float* const* o_ptrs;    // device table (may be null)
  int ptr_base;
  int w_f32;               // W is fp32 (else bf16)
  int w_transposed;        // output tile is W^T (tall matrix)
  long long w_cols;        // W's row length
};

struct __align__(64) GemmParams {
  CUtensorMap maps[MAX_MAPS];
  GemmProblem prob[MAX_PROBS];
  int nprob;
  int total_tiles;
  unsigned int* status;    // device status word
  long long timeout_ns;    // bounded-wait limit
};

// ---------------------------------------------------------------- momentum
struct MomChunk {
  long long start;  // first element (flat, row-major) within the matrix
  int slot;         // matrix slot (bucket order)
  int len;          // elements in this chunk
};

struct MomMat {     // per-slot geometry for the momentum/normalise pass
  long long rows, cols, ldc;
  long long mb_off;     // element offset of this matrix's image in the Mb area
  int chunk_begin, chunk_end;
};

constexpr int MOM_CHUNK = 16384;

// ---------------------------------------------------------------- fp32 path
struct SimtProblem {
  int count, M, N, K;
  int sym;
  // A(i,k) = a + mat*a_ms + i*a_si + k*a_sk ; same for B(j,k)
  const float* a; long long a_ms, a_si, a_sk;
  const float* b; long long b_ms, b_si, b_sk;
  int epi, alpha_mode;
  float alpha, beta, gamma, gamma2;
  const float* inv; int inv_base;
  const float* cin; float* out; float* out2;
  long long ld, mat_stride;
  void* const* w_ptrs; float* const* o_ptrs; int ptr_base;
  int w_f32, w_transposed; long long w_cols;
};

// ---------------------------------------------------------------- launchers
// Single-CTA tensor-core launch: 128 x tbn tiles, tbn = 256 or 128.
cudaError_t launch_gemm_tc(const GemmParams& p, int na, int nb, int kind, int num_sms, int tbn,
                           cudaStream_t s);
// CTA-pair variant: 256 x 256 tiles (tiles_* of every problem computed with
// a 256-row block), clusters of 2 CTAs, tcgen05.mma.cta_group::2.  `kat`:
// K atoms per stage of the one-MMA-per-slice fp16 kernels (1, 2, or 0 for
// the default of 3); other configurations ignore it.
cudaError_t launch_gemm_tc2(const GemmParams& p, int na, int nb, int kind, int num_sms, int kat, int tn,
                            cudaStream_t s);
cudaError_t gemm_tc_configure();
cudaError_t launch_wait_selftest(unsigned int* status, long long timeout_ns, cudaStream_t s);
int gemm_tc_stages(int na, int nb);

// Per-chunk partial sums: MOM_PARTIALS_PER_CHUNK floats per momentum chunk.
constexpr int MOM_PARTIALS_PER_CHUNK = 8;
cudaError_t launch_momentum(const MomChunk* chunks, int nchunks, const MomMat* mats,
                            const void* const* grads, float* const* momenta, int grad_f32,
                            void* mb, int mb_f32, float beta, float gscale, const float* iscale,
                            int* fix_count, float* partial, int vec_ok, int num_sms, long long timeout_ns,
                            unsigned int* status, cudaStream_t s);
cudaError_t momentum_configure();
cudaError_t launch_norm_finalize(const MomMat* mats, int nmats, const float* partial,
                                 float eps, float* inv, float* iscale, float* inv_img, int* fix,
                                 int* fix_count, unsigned int* status, cudaStream_t s);
cudaError_t launch_image_fix(const MomChunk* chunks, int nchunks, const MomMat* mats, const void* const* grads,
                             float* const* momenta, float gscale, void* mb, const float* iscale, const int* fix,
                             const int* fix_count, int vec_ok, int num_sms, cudaStream_t s);
cudaError_t launch_simt_gemm(const SimtProblem& p, cudaStream_t s);
cudaError_t launch_identity16(void* hi, void* lo, int count, int m, long long ld, long long mat_stride, int f16,
                              cudaStream_t s);
cudaError_t launch_identity_f32(float* p, int count, int m, long long ld, long long mat_stride,
                                cudaStream_t s);
// Test-hook conversions; `half` reads a half-stored symmetric matrix
// (element (r, c) with block(r) > block(c) comes from (c, r)).
cudaError_t launch_pair_to_f32(const __nv_bfloat16* hi, const __nv_bfloat16* lo, long long rows,
                               long long cols, long long ld, float* out, cudaStream_t s, int half = 0);
cudaError_t launch_pair_h_to_f32(const void* hi, const void* lo, long long rows, long long cols, long long ld,
                                 float scale, float* out, cudaStream_t s, int half = 0);
cudaError_t launch_f32_copy2d(const float* src, long long rows, long long cols, long long ld,
                              float* out, cudaStream_t s);
constexpr int HALF_BLOCK = 256;  // block size of half-stored symmetric matrices

}  // namespace dmu

namespace dmu {
// ---------------------------------------------------------------- on-chip recursion (m <= 128)
// One shape bucket whose whole Gram recursion runs in one CTA per matrix
// (SYRK from the momentum image, K steps of the R-form recursion with
// G/T, R and P held in shared memory as bf16 hi/lo pairs); only the final
// P is written, as an fp16 hi/lo pair into the class's final-P area.
constexpr int ONCHIP_MAX_M = 128;
struct OnchipProblem {
  int count;            // matrices of the bucket
  int m, n;             // m = min(rows, cols) <= 128, n = max
  int tall;             // the iterated X is Mb^T (MN-major image reads)
  int map;              // image tensor map (K-major box 64 x 128, or MN-major 64 x 64)
  int inv_base;         // index of the bucket's first matrix in `inv`
  int mat_begin;        // first global matrix index of this problem
  __half* p_hi;         // final P of the bucket's first matrix, fp16 hi/lo pair
  __half* p_lo;
  long long ld, mat_stride;
};

struct __align__(64) OnchipParams {
  CUtensorMap maps[MAX_MAPS];
  OnchipProblem prob[MAX_PROBS];
  int nprob;
  int total;            // matrices over all problems
  const float* inv;
  float a, b, c;        // recursion coefficients
  int steps;            // K >= 1
  unsigned int* status;
  long long timeout_ns;
};

cudaError_t onchip_configure();
cudaError_t launch_gram_onchip(const OnchipParams& p, int num_sms, cudaStream_t s);
}  // namespace dmu
