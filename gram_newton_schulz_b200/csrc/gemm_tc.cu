// Grouped bf16 GEMM on the 5th-generation tensor cores (tcgen05), sm_100a.
//
// Every product of the Muon update is one "problem" here:
//   * the Gram matrix G0 = s^2 X X^T (SYRK: only upper-triangle tiles,
//     mirrored on write) -- DMuon page, section 2.2 (Gram-space recursion,
//     SYRK-style symmetric path); Dion3 review, section 3 (symmetric GEMM);
//   * the Gram-space products G G, R G, R P, T R of the recursion
//     Q = aI + bG + cG^2, G <- QGQ, P <- QP, written as R = Q - aI so the
//     identity terms are applied exactly in the fp32 epilogue:
//       R = bG + c(GG),  T = aG + RG,  G' = aT + TR,  P' = aP + RP
//     (all operands are polynomials in G0, hence symmetric and commuting;
//     only upper tiles are computed);
//   * the final O = P X0 with the weight update fused in the epilogue.
//
// Structure (one CTA per SM, persistent, static round-robin over tiles):
//   warp 0     TMA producer: 3-D tensor maps, 128-byte swizzle, a ring of
//              shared-memory stages guarded by full/empty mbarriers;
//   warp 1     MMA issuer: one thread issues tcgen05.mma (M=128, N=256,
//              K=16) into one of two TMEM accumulators (2 x 256 columns);
//   warps 2-9  epilogue: tcgen05.ld of their 32-lane quarter (two warps per
//              quarter, each on half of the tile's columns), fp32 affine
//              epilogue, hi/lo split, direct stores; in diagonal tiles the
//              mirror images move as 8 x 8 block transposes through a
//              per-warp shared scratch; the epilogue of tile t overlaps
//              the main loop of tile t+1.
// Operand precision: each stage holds up to two bf16 parts of A (hi, lo)
// and of B; the problem's term bits choose hi*hi, hi*lo, lo*hi.
// Every mbarrier wait is bounded by a wall-clock limit; on expiry the CTA
// sets DMU_FLAG_TIMEOUT in the status word and winds down.
#include <cuda_fp16.h>

#include "dmu_internal.h"
#include "ptx.cuh"

namespace dmu {

// Per-warp shared scratch of the symmetric diagonal-tile epilogue (block
// transposes of the mirror images), after the barrier area.
constexpr int EPI_SCRATCH_BYTES = EPI_WARPS * 2048;

template <int NA, int NB, int TBN = BN>
struct TcCfg {  // stage geometry is the same for both operand kinds
  static constexpr int B_PART = TBN * BK * 2;  // TBN rows of one 128-byte K row
  static constexpr int STAGE_BYTES = NA * A_PART_BYTES + NB * B_PART;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + EPI_SCRATCH_BYTES;
  static_assert(STAGES >= 2 && STAGES <= 13, "stage count (barrier area holds 13)");
  static_assert(TBN == 128 || TBN == 256, "tile width");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

struct TileCoord {
  int pi, mat, bi, bj;
};

template <int TBM, int TBN = BN>
__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int t) {
  TileCoord c;
  int pi = 0;
  while (pi + 1 < p.nprob && t >= p.prob[pi + 1].tile_begin) ++pi;
  const GemmProblem& pr = p.prob[pi];
  int local = t - pr.tile_begin;
  int mat = local / pr.tiles_per_mat;
  int tl = local - mat * pr.tiles_per_mat;
  int bi, bj;
  if (!pr.sym) {
    bi = tl % pr.tiles_m;
    bj = tl / pr.tiles_m;
  } else {
    // column block bj holds row blocks 0 .. min(tiles_m, ((bj+1)*TBN-1)/TBM + 1) - 1
    bj = 0;
    for (;;) {
      int cnt = min(pr.tiles_m, ((bj + 1) * TBN - 1) / TBM + 1);
      if (tl < cnt) break;
      tl -= cnt;
      ++bj;
    }
    bi = tl;
  }
  c.pi = pi;
  c.mat = mat;
  c.bi = bi;
  c.bj = bj;
  return c;
}

// Bounded wait on an mbarrier phase.  Returns false when the CTA is
// winding down (this or another role timed out).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         const GemmParams& p) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (;;) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if ((long long)(ptx::globaltimer() - t0) > p.timeout_ns) {
      *abort_flag = 1;
      atomicOr(p.status, DMU_FLAG_TIMEOUT);
      return false;
    }
  }
}

// ------------------------------------------------------------- epilogue
__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float2 t = __bfloat1622float2(h[q]);
    f[2 * q] = t.x;
    f[2 * q + 1] = t.y;
  }
}

// hi = RN(v), lo = RN(v - hi), two values per packed conversion (v - hi is
// exact in fp32, so the pair carries v to 16 + 8 bits).
__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&hi);
  __nv_bfloat162* l = reinterpret_cast<__nv_bfloat162*>(&lo);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 hq = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
    const float2 f = __bfloat1622float2(hq);
    h[q] = hq;
    l[q] = __floats2bfloat162_rn(__fsub_rn(v[2 * q], f.x), __fsub_rn(v[2 * q + 1], f.y));
  }
}

__device__ __forceinline__ void unpack8_h(const uint4& u, float* f) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float2 t = __half22float2(h[q]);
    f[2 * q] = t.x;
    f[2 * q + 1] = t.y;
  }
}

__device__ __forceinline__ void split8_h(const float* v, uint4& hi, uint4& lo) {
  __half2* h = reinterpret_cast<__half2*>(&hi);
  __half2* l = reinterpret_cast<__half2*>(&lo);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __half2 hq = __floats2half2_rn(v[2 * q], v[2 * q + 1]);
    const float2 f = __half22float2(hq);
    h[q] = hq;
    l[q] = __floats2half2_rn(__fsub_rn(v[2 * q], f.x), __fsub_rn(v[2 * q + 1], f.y));
  }
}

__device__ __forceinline__ void store_pair_h(__half* hi, __half* lo, long long off, float v) {
  __half h = __float2half_rn(v);
  hi[off] = h;
  if (lo) lo[off] = __float2half_rn(v - __half2float(h));
}

// Store value v at (i, j) of a hi/lo pair.
__device__ __forceinline__ void store_pair(__nv_bfloat16* hi, __nv_bfloat16* lo, long long off,
                                           float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi[off] = h;
  if (lo) lo[off] = __float2bfloat16_rn(v - bf2f(h));
}

// Columns per epilogue chunk (one tcgen05.ld of 32 lanes x CW columns).
constexpr int CW = 16;

// 16-byte global load that asks L2 to fetch the surrounding 256 bytes from
// DRAM.  An epilogue thread reads its row 32 bytes per chunk, a chunk at a
// time; with the hint the first chunk brings the warp's whole 256-byte row
// segment in at once, instead of one 32-byte sector at a time.
__device__ __forceinline__ uint4 ld_row16(const void* p) {
  uint4 r;
  asm volatile("ld.global.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p)
               : "memory");
  return r;
}

// Symmetric diagonal tiles: the mirror images (j, i), i < j, of a chunk's
// upper elements are moved as 8 x 8 blocks through a per-warp shared-memory
// scratch (ldmatrix .trans / stmatrix) and written as 16-byte rows, instead
// of one 2-byte store per element.  Scratch per epilogue warp: 32 source rows
// x 32 bytes (the chunk as the lanes computed it) and 16 destination rows x
// 64 bytes (its transpose); 16-byte segments are XOR-swizzled so that the
// 8-row accesses of ldmatrix / stmatrix fall on distinct banks.
constexpr int TRI_SCRATCH = 2048;
static_assert(EPI_SCRATCH_BYTES == EPI_WARPS * TRI_SCRATCH, "scratch per epilogue warp");
static_assert(CW == 16, "the block-transpose mirror moves 32 x 16 chunks");
__device__ __forceinline__ uint32_t tri_src(uint32_t scr, int r, int seg) {
  return scr + r * 32 + ((seg ^ ((r >> 2) & 1)) << 4);
}
__device__ __forceinline__ uint32_t tri_dst(uint32_t scr, int r, int seg) {
  return scr + 1024 + r * 64 + ((seg ^ ((r >> 1) & 3)) << 4);
}

// One 16-bit part (hi or lo) of the mirror images of a 32 x CW chunk (rows
// row_lo .. row_lo + 31, one per lane, x0 / x1 = this lane's 16 packed
// values; columns col0 .. col0 + 15; the whole chunk inside the matrix).
// Destination rows R = col0 .. col0 + 15, 8-column segments C0 = row_lo +
// 8 s: segments left of the diagonal are written from the transpose, the
// segment holding (R, R) merges the transpose (C < R) with row R's own
// values (C >= R, from the source rows), segments right of it are skipped.
// om is the matrix's base; in-matrix offsets fit 32 bits (m <= 65536, so
// row * ld + column < 2^32).  Warp-collective; the lanes' direct stores
// precede it.
__device__ __forceinline__ void tri_mirror_part(uint16_t* om, uint32_t ld, int row_lo, int col0, int lane, uint4 x0,
                                                uint4 x1, uint32_t scr) {
  ptx::sts128(tri_src(scr, lane, 0), x0);
  ptx::sts128(tri_src(scr, lane, 1), x1);
  __syncwarp();
#pragma unroll
  for (int cb = 0; cb < 2; ++cb) {
    // matrix rb = lanes 8 rb .. 8 rb + 7, columns 8 cb .. 8 cb + 7; its
    // transpose is destination rows 8 cb .. 8 cb + 7, segment rb
    uint32_t t[4];
    ptx::ldsm_x4_trans(tri_src(scr, lane, cb), t);
    ptx::stsm_x4(tri_dst(scr, 8 * cb + (lane & 7), lane >> 3), t);
  }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int s = lane + 32 * h, dr = s >> 2, sg = s & 3;
    const int R = col0 + dr, C0 = row_lo + 8 * sg;
    if (C0 > R) continue;
    uint4 val = ptx::lds128(tri_dst(scr, dr, sg));
    if (C0 + 7 >= R) {
      const uint4 d = ptx::lds128(tri_src(scr, R - row_lo, (C0 - col0) >> 3));
      const int e0 = R - C0;  // elements e >= e0 lie on or right of the diagonal
      uint32_t* pv = reinterpret_cast<uint32_t*>(&val);
      const uint32_t* pd = reinterpret_cast<const uint32_t*>(&d);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t keep = (2 * w < e0 ? 0x0000FFFFu : 0u) | (2 * w + 1 < e0 ? 0xFFFF0000u : 0u);
        pv[w] = (pv[w] & keep) | (pd[w] & ~keep);
      }
    }
    *reinterpret_cast<uint4*>(om + ((uint32_t)R * ld + (uint32_t)C0)) = val;
  }
  __syncwarp();
}

// The Cin row segment of one chunk (16 values of row i), loaded ahead of its
// use so that its latency overlaps the previous chunk's epilogue (or, for a
// tile's first chunk, the main loop): a 16-bit pair as raw[0..1] (hi) and
// raw[2..3] (lo), or fp32 as raw[0..3].  `ok` is set only for a whole chunk
// inside the matrix with an input to read; other chunks load per element.
// Cin is never written by the launch that reads it, so loading early is safe.
struct CinRow {
  uint4 raw[4];
  bool ok;
};

__device__ __forceinline__ void cin_fetch(const GemmProblem& pr, int mat, int i, int col0, CinRow& c) {
  c.ok = false;
  if (i >= pr.M || col0 + CW > pr.N) return;
  const long long off = (long long)mat * pr.mat_stride + (long long)i * pr.ld + col0;
  if (pr.cin_fmt == FMT_F32 && pr.cin_f) {
    const uint4* pf = reinterpret_cast<const uint4*>(pr.cin_f + off);
#pragma unroll
    for (int q = 0; q < 4; ++q) c.raw[q] = ld_row16(pf + q);
    c.ok = true;
  } else if ((pr.cin_fmt == FMT_PAIR_H || pr.cin_fmt == FMT_PAIR) && pr.cin_hi) {
    // both 16-bit formats are addressed as 2-byte elements
    const uint4* ph = reinterpret_cast<const uint4*>(pr.cin_hi + off);
    c.raw[0] = ld_row16(ph);
    c.raw[1] = ld_row16(ph + 1);
    if (pr.cin_lo) {
      const uint4* pl = reinterpret_cast<const uint4*>(pr.cin_lo + off);
      c.raw[2] = ld_row16(pl);
      c.raw[3] = ld_row16(pl + 1);
    } else {
      c.raw[2] = make_uint4(0u, 0u, 0u, 0u);  // +0 in both formats: hi + 0 = hi exactly
      c.raw[3] = c.raw[2];
    }
    c.ok = true;
  }
}

// One CW-column chunk of a Gram-space output tile for the thread's row i.
// Input and outputs are bf16 hi/lo pairs (FMT_PAIR) or fp32 (FMT_F32).
// Every rounding step is explicit (__fmul_rn, __fadd_rn, __fmaf_rn), so the
// on-chip recursion, which repeats this arithmetic, gets the same bits
// whatever fused multiply-adds the compiler would otherwise form.
// `tri`: store only i <= j and mirror (symmetric outputs, except the
// off-diagonal tiles of half-stored outputs, which are written whole).
__device__ __forceinline__ void epi_gram_chunk(const GemmProblem& pr, int mat, int i, int col0,
                                               const uint32_t (&r)[CW], bool tri, uint32_t scr,
                                               const CinRow& cin) {
  const int M = pr.M, N = pr.N;
  const int lane = (int)(threadIdx.x & 31u);
  const int row_lo = i - lane;
  // whole-chunk symmetric diagonal tiles take the block-transpose mirror
  // (warp-uniform: every lane of the chunk lies inside the matrix)
  const bool fast = tri && scr != 0u && col0 + CW <= N && row_lo + 32 <= M;
  if (i >= M) return;
  float coef = pr.alpha;
  if (pr.alpha_mode == ALPHA_INV2) {
    float s = pr.inv[pr.inv_base + mat];
    coef *= s * s;
  } else if (pr.alpha_mode == ALPHA_INV) {
    coef *= pr.inv[pr.inv_base + mat];
  }
  float v[CW];
#pragma unroll
  for (int c = 0; c < CW; ++c) v[c] = __fmul_rn(coef, __uint_as_float(r[c]));

  const long long mbase = (long long)mat * pr.mat_stride;
  const long long rowoff = mbase + (long long)i * pr.ld;
  const bool full = (col0 + CW <= N);
  const bool all_upper = !tri || (i <= col0);

  if (cin.ok) {
    // the whole chunk's row segment, loaded by cin_fetch
    if (pr.cin_fmt == FMT_F32) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[4 * q] = __fmaf_rn(pr.beta, __uint_as_float(cin.raw[q].x), v[4 * q]);
        v[4 * q + 1] = __fmaf_rn(pr.beta, __uint_as_float(cin.raw[q].y), v[4 * q + 1]);
        v[4 * q + 2] = __fmaf_rn(pr.beta, __uint_as_float(cin.raw[q].z), v[4 * q + 2]);
        v[4 * q + 3] = __fmaf_rn(pr.beta, __uint_as_float(cin.raw[q].w), v[4 * q + 3]);
      }
    } else {
#pragma unroll
      for (int q = 0; q < CW / 8; ++q) {
        float fh[8], fl[8];
        if (pr.cin_fmt == FMT_PAIR_H) {
          unpack8_h(cin.raw[q], fh);
          unpack8_h(cin.raw[2 + q], fl);
        } else {
          unpack8(cin.raw[q], fh);
          unpack8(cin.raw[2 + q], fl);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * q + e] = __fmaf_rn(pr.beta, __fadd_rn(fh[e], fl[e]), v[8 * q + e]);
      }
    }
  } else if (!full) {
    // ragged chunk: per-element loads of the columns inside the matrix
    if (pr.cin_fmt == FMT_F32 && pr.cin_f) {
#pragma unroll
      for (int c = 0; c < CW; ++c)
        if (col0 + c < N) v[c] = __fmaf_rn(pr.beta, pr.cin_f[rowoff + col0 + c], v[c]);
    } else if (pr.cin_fmt == FMT_PAIR_H && pr.cin_hi) {
      const __half* ch = reinterpret_cast<const __half*>(pr.cin_hi);
      const __half* cl = reinterpret_cast<const __half*>(pr.cin_lo);
#pragma unroll
      for (int c = 0; c < CW; ++c)
        if (col0 + c < N) {
          float x = __half2float(ch[rowoff + col0 + c]);
          if (cl) x = __fadd_rn(x, __half2float(cl[rowoff + col0 + c]));
          v[c] = __fmaf_rn(pr.beta, x, v[c]);
        }
    } else if (pr.cin_fmt == FMT_PAIR && pr.cin_hi) {
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        if (col0 + c < N) {
          float x = bf2f(pr.cin_hi[rowoff + col0 + c]);
          if (pr.cin_lo) x = __fadd_rn(x, bf2f(pr.cin_lo[rowoff + col0 + c]));
          v[c] = __fmaf_rn(pr.beta, x, v[c]);
        }
      }
    }
  }
  const int dc = i - col0;  // diagonal column within the chunk
  if (dc >= 0 && dc < CW) {
#pragma unroll
    for (int c = 0; c < CW; ++c)
      if (c == dc) v[c] = __fadd_rn(v[c], pr.gamma);
  }

  for (int pass = 0; pass < 2; ++pass) {
    const int fmt = pass == 0 ? pr.out_fmt : pr.out2_fmt;
    if (pass == 1) {
      if (!pr.out2_hi && !pr.out2_f) break;
#pragma unroll
      for (int c = 0; c < CW; ++c) v[c] = __fmaf_rn(v[c], pr.scale2, c == dc ? pr.gamma2 : 0.f);
    }
    if (fmt == FMT_PAIR_H) {
      __half* oh = reinterpret_cast<__half*>(pass == 0 ? pr.out_hi : pr.out2_hi);
      __half* ol = reinterpret_cast<__half*>(pass == 0 ? pr.out_lo : pr.out2_lo);
      if (!oh) continue;
      if (fast) {
        uint4 h0, l0, h1, l1;
        split8_h(v, h0, l0);
        split8_h(v + 8, h1, l1);
        // rows above the chunk's diagonal 16 x 16 block and inside it store
        // all 16 values (the block's lower half is rewritten by the mirror)
        if (i < col0 + CW) {
          uint4* dh = reinterpret_cast<uint4*>(oh + rowoff + col0);
          dh[0] = h0;
          dh[1] = h1;
          if (ol) {
            uint4* dl = reinterpret_cast<uint4*>(ol + rowoff + col0);
            dl[0] = l0;
            dl[1] = l1;
          }
        }
        tri_mirror_part(reinterpret_cast<uint16_t*>(oh) + mbase, (uint32_t)pr.ld, row_lo, col0, lane, h0, h1, scr);
        if (ol) tri_mirror_part(reinterpret_cast<uint16_t*>(ol) + mbase, (uint32_t)pr.ld, row_lo, col0, lane, l0, l1, scr);
        continue;
      }
      if (full && all_upper) {
        uint4* dh = reinterpret_cast<uint4*>(oh + rowoff + col0);
        uint4* dl = ol ? reinterpret_cast<uint4*>(ol + rowoff + col0) : nullptr;
#pragma unroll
        for (int q = 0; q < CW / 8; ++q) {
          uint4 h, l;
          split8_h(v + 8 * q, h, l);
          dh[q] = h;
          if (dl) dl[q] = l;
        }
      } else {
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          const int j = col0 + c;
          if (j < N && (!tri || i <= j)) store_pair_h(oh, ol, rowoff + j, v[c]);
        }
      }
      if (tri) {
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          const int j = col0 + c;
          if (j < N && i < j) store_pair_h(oh, ol, mbase + (long long)j * pr.ld + i, v[c]);
        }
      }
      continue;
    }
    if (fmt == FMT_F32) {
      float* of = pass == 0 ? pr.out_f : pr.out2_f;
      if (!of) continue;
      if (full && all_upper) {
        float4* d4 = reinterpret_cast<float4*>(of + rowoff + col0);
#pragma unroll
        for (int q = 0; q < CW / 4; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          const int j = col0 + c;
          if (j < N && (!tri || i <= j)) of[rowoff + j] = v[c];
        }
      }
      if (tri) {
#pragma unroll
        for (int c = 0; c < CW; ++c) {
          const int j = col0 + c;
          if (j < N && i < j) of[mbase + (long long)j * pr.ld + i] = v[c];
        }
      }
      continue;
    }
    __nv_bfloat16* oh = pass == 0 ? pr.out_hi : pr.out2_hi;
    __nv_bfloat16* ol = pass == 0 ? pr.out_lo : pr.out2_lo;
    if (!oh) continue;
    if (fast) {
      uint4 h0, l0, h1, l1;
      split8(v, h0, l0);
      split8(v + 8, h1, l1);
      if (i < col0 + CW) {
        uint4* dh = reinterpret_cast<uint4*>(oh + rowoff + col0);
        dh[0] = h0;
        dh[1] = h1;
        if (ol) {
          uint4* dl = reinterpret_cast<uint4*>(ol + rowoff + col0);
          dl[0] = l0;
          dl[1] = l1;
        }
      }
      tri_mirror_part(reinterpret_cast<uint16_t*>(oh) + mbase, (uint32_t)pr.ld, row_lo, col0, lane, h0, h1, scr);
      if (ol) tri_mirror_part(reinterpret_cast<uint16_t*>(ol) + mbase, (uint32_t)pr.ld, row_lo, col0, lane, l0, l1, scr);
      continue;
    }
    // direct stores (i, j), j >= i when symmetric
    if (full && all_upper) {
      uint4* dh = reinterpret_cast<uint4*>(oh + rowoff + col0);
      uint4* dl = ol ? reinterpret_cast<uint4*>(ol + rowoff + col0) : nullptr;
#pragma unroll
      for (int q = 0; q < CW / 8; ++q) {
        uint4 h, l;
        split8(v + 8 * q, h, l);
        dh[q] = h;
        if (dl) dl[q] = l;
      }
    } else {
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        const int j = col0 + c;
        if (j < N && (!tri || i <= j)) store_pair(oh, ol, rowoff + j, v[c]);
      }
    }
    // mirrored stores (j, i) for j > i: consecutive lanes write consecutive
    // columns of row j, so each store instruction is coalesced.
    if (tri) {
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        const int j = col0 + c;
        if (j < N && i < j) store_pair(oh, ol, mbase + (long long)j * pr.ld + i, v[c]);
      }
    }
  }
}

// Gram products whose input (if any) and output are 16-bit hi/lo pairs and
// that have no second output -- every product of the split-bf16 and
// scaled-fp16 classes, and the SYRK -- take a specialised chunk epilogue:
// the formats are template parameters, the tile-uniform fields are read
// once per tile into GramTile, and in-matrix offsets are 32-bit.  The
// arithmetic is epi_gram_chunk's, operation for operation, so the bits are
// the same; other problems, and chunks at a ragged matrix edge, keep
// epi_gram_chunk.
struct GramTile {
  const uint16_t* cin_hi;  // this matrix's input pair (null: no input; lo may be null)
  const uint16_t* cin_lo;
  uint16_t* out_hi;        // this matrix's output pair (lo may be null)
  uint16_t* out_lo;
  float coef, beta, gamma;
  uint32_t ld;
  int kind;                // GRAM_GENERAL: epi_gram_chunk; else the formats
};
enum GramKind : int { GRAM_GENERAL = 0, GRAM_BB = 1, GRAM_HH = 2, GRAM_BH = 3 };  // Cin (or none) -> out formats

__device__ __forceinline__ GramTile gram_tile(const GemmProblem& pr, int mat) {
  GramTile g;
  g.kind = GRAM_GENERAL;
  g.cin_hi = g.cin_lo = nullptr;
  g.out_hi = g.out_lo = nullptr;
  g.coef = g.beta = g.gamma = 0.f;
  g.ld = 0;
  if (pr.epi != EPI_GRAM || !pr.out_hi || pr.out_fmt == FMT_F32 || pr.out2_hi || pr.out2_f) return g;
  if (pr.cin_fmt == FMT_F32) return g;
  const bool cin_h = pr.cin_hi && pr.cin_fmt == FMT_PAIR_H, out_h = pr.out_fmt == FMT_PAIR_H;
  if (cin_h && !out_h) return g;
  g.kind = out_h ? (pr.cin_hi && !cin_h ? GRAM_BH : GRAM_HH) : GRAM_BB;
  const long long mbase = (long long)mat * pr.mat_stride;
  g.out_hi = reinterpret_cast<uint16_t*>(pr.out_hi) + mbase;
  g.out_lo = pr.out_lo ? reinterpret_cast<uint16_t*>(pr.out_lo) + mbase : nullptr;
  if (pr.cin_hi) {
    g.cin_hi = reinterpret_cast<const uint16_t*>(pr.cin_hi) + mbase;
    g.cin_lo = pr.cin_lo ? reinterpret_cast<const uint16_t*>(pr.cin_lo) + mbase : nullptr;
  }
  float coef = pr.alpha;
  if (pr.alpha_mode == ALPHA_INV2) {
    float sv = pr.inv[pr.inv_base + mat];
    coef *= sv * sv;
  } else if (pr.alpha_mode == ALPHA_INV) {
    coef *= pr.inv[pr.inv_base + mat];
  }
  g.coef = coef;
  g.beta = pr.beta;
  g.gamma = pr.gamma;
  g.ld = (uint32_t)pr.ld;
  return g;
}

// The row segment of a chunk's input pair (see CinRow), for gram_tile16.
__device__ __forceinline__ void cin16_fetch(const GramTile& g, int i, int col0, CinRow& c) {
  c.ok = g.cin_hi != nullptr;
  if (!c.ok) return;
  const uint32_t off = (uint32_t)i * g.ld + (uint32_t)col0;
  const uint4* ph = reinterpret_cast<const uint4*>(g.cin_hi + off);
  c.raw[0] = ld_row16(ph);
  c.raw[1] = ld_row16(ph + 1);
  if (g.cin_lo) {
    const uint4* pl = reinterpret_cast<const uint4*>(g.cin_lo + off);
    c.raw[2] = ld_row16(pl);
    c.raw[3] = ld_row16(pl + 1);
  } else {
    c.raw[2] = make_uint4(0u, 0u, 0u, 0u);
    c.raw[3] = c.raw[2];
  }
}

// A warp's chunks [c_lo, c_hi) of one tile of a GramTile product, every
// chunk whole (all 32 rows and 16 columns inside the matrix).  tmem: the
// accumulator's column 0 in this warp's lane quarter; col_base: the tile's
// first column; chunks with col0 < tri_end are symmetric diagonal chunks
// (mirrored); cin: the first chunk's input, already loaded.  The next
// chunk's input is loaded as soon as this chunk's has been consumed, so
// one CinRow is live at a time.
template <bool CIN_H, bool OUT_H>
__device__ __forceinline__ void gram_tile16(const GramTile& g, uint32_t tmem, int col_base, int c_lo, int c_hi,
                                            int row_lo, int lane, int tri_end, uint32_t scr, CinRow cin) {
  const int i = row_lo + lane;
  const bool has_cin = g.cin_hi != nullptr;
  for (int ch = c_lo; ch < c_hi; ++ch) {
    const int col0 = col_base + ch * CW;
    uint32_t r[CW];
    ptx::tmem_ld16(tmem + (uint32_t)(ch * CW), r);
    ptx::tmem_wait_ld();
    float v[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) v[c] = __fmul_rn(g.coef, __uint_as_float(r[c]));
    if (has_cin) {
#pragma unroll
      for (int q = 0; q < CW / 8; ++q) {
        float fh[8], fl[8];
        if (CIN_H) {
          unpack8_h(cin.raw[q], fh);
          unpack8_h(cin.raw[2 + q], fl);
        } else {
          unpack8(cin.raw[q], fh);
          unpack8(cin.raw[2 + q], fl);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * q + e] = __fmaf_rn(g.beta, __fadd_rn(fh[e], fl[e]), v[8 * q + e]);
      }
      if (ch + 1 < c_hi) cin16_fetch(g, i, col0 + CW, cin);
    }
    const int dc = i - col0;  // diagonal column within the chunk
    if (dc >= 0 && dc < CW) {
#pragma unroll
      for (int c = 0; c < CW; ++c)
        if (c == dc) v[c] = __fadd_rn(v[c], g.gamma);
    }
    uint4 h0, l0, h1, l1;
    if (OUT_H) {
      split8_h(v, h0, l0);
      split8_h(v + 8, h1, l1);
    } else {
      split8(v, h0, l0);
      split8(v + 8, h1, l1);
    }
    // direct row stores: every row of an upper chunk; in a diagonal chunk
    // the rows above its diagonal 16 x 16 block and inside it (the block's
    // lower half is rewritten by the mirror)
    const bool tri = col0 < tri_end;
    const uint32_t off = (uint32_t)i * g.ld + (uint32_t)col0;
    if (!tri || i < col0 + CW) {
      uint4* dh = reinterpret_cast<uint4*>(g.out_hi + off);
      dh[0] = h0;
      dh[1] = h1;
      if (g.out_lo) {
        uint4* dl = reinterpret_cast<uint4*>(g.out_lo + off);
        dl[0] = l0;
        dl[1] = l1;
      }
    }
    if (tri) {
      tri_mirror_part(g.out_hi, g.ld, row_lo, col0, lane, h0, h1, scr);
      if (g.out_lo) tri_mirror_part(g.out_lo, g.ld, row_lo, col0, lane, l0, l1, scr);
    }
  }
}

// GramTile of a warp's part of a tile: the specialised epilogue only when
// all of the warp's chunks are whole.
__device__ __forceinline__ GramTile gram_tile_for(const GemmProblem& pr, int mat, int row_lo, int col_end) {
  GramTile g = gram_tile(pr, mat);
  if (col_end > pr.N || row_lo + 32 > pr.M) g.kind = GRAM_GENERAL;
  return g;
}

// One CW-column chunk of the final O = P X0 tile, fused with the update.
// Row i of the tile is row i of O (m x n); element (i, j) lives at W[i][j]
// for a wide matrix and at W[j][i] for a tall one (w_transposed).  All W
// loads of the chunk are issued before any store, so they overlap instead
// of serialising behind stores the compiler cannot prove independent.
__device__ __forceinline__ void epi_update_chunk(const GemmProblem& pr, int mat, int i, int col0,
                                                 const uint32_t (&r)[CW]) {
  const int M = pr.M, N = pr.N;
  if (i >= M) return;
  const float s = pr.inv[pr.inv_base + mat];
  const float cw = pr.alpha * s;  // -lr * scale / (||M|| + eps)
  float o[CW];
#pragma unroll
  for (int c = 0; c < CW; ++c) o[c] = __uint_as_float(r[c]);
  void* wp = pr.w_ptrs ? pr.w_ptrs[pr.ptr_base + mat] : nullptr;
  float* op = pr.o_ptrs ? pr.o_ptrs[pr.ptr_base + mat] : nullptr;
  const long long wc = pr.w_cols;
  const bool full = (col0 + CW <= N);
  if (!pr.w_transposed) {
    const long long rowoff = (long long)i * wc;
    if (wp) {
      if (!pr.w_f32) {
        __nv_bfloat16* w = reinterpret_cast<__nv_bfloat16*>(wp);
        const bool vec = full && ((wc & 7) == 0) && ((reinterpret_cast<uintptr_t>(w) & 15) == 0);
        if (vec) {
          uint4* pw = reinterpret_cast<uint4*>(w + rowoff + col0);
          uint4 wv[CW / 8];
#pragma unroll
          for (int q = 0; q < CW / 8; ++q) wv[q] = ld_row16(pw + q);
#pragma unroll
          for (int q = 0; q < CW / 8; ++q) {
            float f[8];
            unpack8(wv[q], f);
            uint4 h;
            __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&h);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              hh[e] = __floats2bfloat162_rn(f[2 * e] + cw * o[8 * q + 2 * e],
                                            f[2 * e + 1] + cw * o[8 * q + 2 * e + 1]);
            pw[q] = h;
          }
        } else {
          float wv[CW];
#pragma unroll
          for (int c = 0; c < CW; ++c) wv[c] = (col0 + c < N) ? bf2f(w[rowoff + col0 + c]) : 0.f;
#pragma unroll
          for (int c = 0; c < CW; ++c)
            if (col0 + c < N) w[rowoff + col0 + c] = __float2bfloat16_rn(wv[c] + cw * o[c]);
        }
      } else {
        float* w = reinterpret_cast<float*>(wp);
        float wv[CW];
#pragma unroll
        for (int c = 0; c < CW; ++c) wv[c] = (col0 + c < N) ? w[rowoff + col0 + c] : 0.f;
#pragma unroll
        for (int c = 0; c < CW; ++c)
          if (col0 + c < N) w[rowoff + col0 + c] = wv[c] + cw * o[c];
      }
    }
    if (op) {
#pragma unroll
      for (int c = 0; c < CW; ++c)
        if (col0 + c < N) op[rowoff + col0 + c] = s * o[c];
    }
  } else {
    // W is n x m (rows = N here, cols = M); element (i, j) -> W[j][i]; each
    // store instruction of the warp covers 32 consecutive columns of a row.
    if (wp) {
      if (!pr.w_f32) {
        __nv_bfloat16* w = reinterpret_cast<__nv_bfloat16*>(wp);
        float wv[CW];
#pragma unroll
        for (int c = 0; c < CW; ++c) wv[c] = (col0 + c < N) ? bf2f(w[(long long)(col0 + c) * wc + i]) : 0.f;
#pragma unroll
        for (int c = 0; c < CW; ++c)
          if (col0 + c < N) w[(long long)(col0 + c) * wc + i] = __float2bfloat16_rn(wv[c] + cw * o[c]);
      } else {
        float* w = reinterpret_cast<float*>(wp);
        float wv[CW];
#pragma unroll
        for (int c = 0; c < CW; ++c) wv[c] = (col0 + c < N) ? w[(long long)(col0 + c) * wc + i] : 0.f;
#pragma unroll
        for (int c = 0; c < CW; ++c)
          if (col0 + c < N) w[(long long)(col0 + c) * wc + i] = wv[c] + cw * o[c];
      }
    }
    if (op) {
#pragma unroll
      for (int c = 0; c < CW; ++c)
        if (col0 + c < N) op[(long long)(col0 + c) * wc + i] = s * o[c];
    }
  }
}

// ------------------------------------------------------------- kernel
template <int NA, int NB, int KIND, int TBN>
__global__ void __launch_bounds__(GEMM_THREADS, 1) k_gemm_tc(const __grid_constant__ GemmParams p) {
  using Cfg = TcCfg<NA, NB, TBN>;
  constexpr int BKE = KIND == KIND_TF32 ? 32 : 64;  // elements per 128-byte K-block row
  constexpr int OPFMT = KIND == KIND_TF32 ? 2 : (KIND == KIND_F16 ? 0 : 1);  // idesc A/B format code
  constexpr int S = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t ring = base;
  const uint32_t bars = base + S * Cfg::STAGE_BYTES;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (S + s); };
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * S + b); };
  auto tempty_bar = [&](int b) { return bars + 8u * (2 * S + 2 + b); };
  const uint32_t drain_bar = bars + 8u * (2 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S * Cfg::STAGE_BYTES + 8 * (2 * S + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), EPI_WARPS);
    }
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    for (int pi = 0; pi < p.nprob; ++pi) {
      ptx::prefetch_tmap(&p.maps[p.prob[pi].a_map]);
      ptx::prefetch_tmap(&p.maps[p.prob[pi].b_map]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t issued_mask = 0, issued_par = 0;  // per stage: a load was issued, its phase parity
      for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x) {
        const TileCoord tc = decode_tile<BM, TBN>(p, t);
        const GemmProblem& pr = p.prob[tc.pi];
        // Per-tile operand parameters, read from the parameter space once.
        const CUtensorMap* am = &p.maps[pr.a_map];
        const CUtensorMap* bm = &p.maps[pr.b_map];
        const CUtensorMap* am_t = pr.half_a ? &p.maps[pr.a_map_t] : am;
        const CUtensorMap* bm_t = pr.half_b ? &p.maps[pr.b_map_t] : bm;
        const int na = (NA > 1 && (pr.terms & TERM_LH)) ? 2 : 1;
        const int nb = (NB > 1 && (pr.terms & TERM_HL)) ? 2 : 1;
        const uint32_t bytes = na * A_PART_BYTES + nb * Cfg::B_PART;
        const int nk = (pr.K + BKE - 1) / BKE;
        const int arow = tc.bi * BM, brow = tc.bj * TBN;
        const int thr_a = pr.half_a ? arow / HALF_BLOCK : 0, thr_b = pr.half_b ? brow / HALF_BLOCK : 0;
        const bool a_mn = pr.a_mn != 0, b_mn = pr.b_mn != 0;
        const int za0 = pr.a_z[0] + tc.mat, za1 = pr.a_z[1] + tc.mat;
        const int zb0 = pr.b_z[0] + tc.mat, zb1 = pr.b_z[1] + tc.mat;
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_bar(empty_bar(stage), phase ^ 1u, abort_flag, p)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(stage);
          ptx::mbar_arrive_expect_tx(fb, bytes);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          const int k0 = kb * BKE;
          const uint32_t sa = ring + stage * Cfg::STAGE_BYTES;
          const uint32_t sb = sa + NA * A_PART_BYTES;
          const int ktile = k0 / HALF_BLOCK;
          const bool a_t = ktile < thr_a;  // read the transposed block
          const bool b_t = ktile < thr_b;
          const CUtensorMap* am_k = a_t ? am_t : am;
          const CUtensorMap* bm_k = b_t ? bm_t : bm;
          for (int part = 0; part < na; ++part) {
            const uint32_t dst = sa + part * A_PART_BYTES;
            const int z = part ? za1 : za0;
            if (!a_mn && !a_t) {
              ptx::tma_load_3d(dst, am_k, fb, k0, arow, z);
            } else {
              ptx::tma_load_3d(dst, am_k, fb, arow, k0, z);
              ptx::tma_load_3d(dst + 8192, am_k, fb, arow + 64, k0, z);
            }
          }
          for (int part = 0; part < nb; ++part) {
            const uint32_t dst = sb + part * Cfg::B_PART;
            const int z = part ? zb1 : zb0;
            if (!b_mn && !b_t) {
#pragma unroll
              for (int c = 0; c < TBN / 128; ++c) ptx::tma_load_3d(dst + 16384 * c, bm_k, fb, k0, brow + 128 * c, z);
            } else {
#pragma unroll
              for (int c = 0; c < TBN / 64; ++c) ptx::tma_load_3d(dst + 8192 * c, bm_k, fb, brow + 64 * c, k0, z);
            }
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Before the CTA may exit, every bulk copy it issued must have landed
      // (normally already true: the MMA warp consumed them).
      for (int s2 = 0; s2 < S; ++s2) {
        if (!(issued_mask & (1u << s2))) continue;
        const uint32_t par = (issued_par >> s2) & 1u;
        const uint64_t t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait(full_bar(s2), par)) {
          if ((long long)(ptx::globaltimer() - t0) > p.timeout_ns) {
            atomicOr(p.status, DMU_FLAG_TIMEOUT);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued = false;
      for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x) {
        const TileCoord tc = decode_tile<BM, TBN>(p, t);
        const GemmProblem& pr = p.prob[tc.pi];
        const int nk = (pr.K + BKE - 1) / BKE;
        if (!wait_bar(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TBN);
        // Per-tile MMA parameters in registers: the K loop issues MMAs from
        // precomputed descriptor halves only.
        const int terms = pr.terms, pr_a_mn = pr.a_mn, pr_b_mn = pr.b_mn;
        const int thr_a = pr.half_a ? (tc.bi * BM) / HALF_BLOCK : 0;
        const int thr_b = pr.half_b ? (tc.bj * TBN) / HALF_BLOCK : 0;
        const uint32_t idesc0 = ptx::make_idesc(BM, TBN, 0, 0, OPFMT);
        const uint64_t hi_k = ptx::make_sw128_desc(0u, 16u, 1024u), hi_mn = ptx::make_sw128_desc(0u, 8192u, 1024u);
        uint32_t accumulate = 0;
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_bar(full_bar(stage), phase, abort_flag, p)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const int ktile = (kb * BKE) / HALF_BLOCK;
          const uint32_t a_mn = (uint32_t)(pr_a_mn | (ktile < thr_a ? 1 : 0));
          const uint32_t b_mn = (uint32_t)(pr_b_mn | (ktile < thr_b ? 1 : 0));
          const uint32_t idesc = idesc0 | (a_mn << 15) | (b_mn << 16);
          const uint64_t a_hi = a_mn ? hi_mn : hi_k, b_hi = b_mn ? hi_mn : hi_k;
          const uint32_t a_ks = a_mn ? 2048u : 32u, b_ks = b_mn ? 2048u : 32u;
          const uint32_t sa = ring + stage * Cfg::STAGE_BYTES;
          const uint32_t sb = sa + NA * A_PART_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 4 MMAs x 32 bytes of K per 128-byte row
#pragma unroll
            for (int term = 0; term < 3; ++term) {
              if (term == 1 && NB < 2) continue;
              if (term == 2 && NA < 2) continue;
              if (!(terms & (1 << term))) continue;
              const uint32_t pa = sa + (term == 2 ? A_PART_BYTES : 0) + kk * a_ks;
              const uint32_t pb = sb + (term == 1 ? Cfg::B_PART : 0) + kk * b_ks;
              const uint64_t ad = a_hi | (uint64_t)((pa >> 4) & 0x3FFFu);
              const uint64_t bd = b_hi | (uint64_t)((pb >> 4) & 0x3FFFu);
              if (KIND == KIND_TF32)
                ptx::mma_tf32(d_tmem, ad, bd, idesc, accumulate);
              else
                ptx::mma_bf16(d_tmem, ad, bd, idesc, accumulate);
              accumulate = 1;
            }
          }
          issued = true;
          ptx::mma_commit(empty_bar(stage));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && issued) {
        // wind down: wait (bounded) for the MMAs already issued
        ptx::mma_commit(drain_bar);
        const uint64_t t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait(drain_bar, 0)) {
          if ((long long)(ptx::globaltimer() - t0) > p.timeout_ns) break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;                        // TMEM lane quarter this warp may access
    const uint32_t scr = bars + Cfg::BAR_BYTES + (uint32_t)(warp - 2) * TRI_SCRATCH;
    const int ch_begin = ((warp - 2) >> 2) * (TBN / 2 / CW);  // column half of the tile
    const int ch_end = ch_begin + TBN / 2 / CW;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
      const TileCoord tc = decode_tile<BM, TBN>(p, t);
      const GemmProblem& pr = p.prob[tc.pi];
      const int row_lo = tc.bi * BM + q * 32;
      const bool tri = pr.sym && (!pr.half_out || (tc.bi * BM) / HALF_BLOCK == (tc.bj * TBN) / HALF_BLOCK);
      const int i = row_lo + lane;
      // this warp's chunks of the tile, [c_lo, c_hi): inside the matrix and,
      // in symmetric diagonal tiles, not strictly below the diagonal
      int c_lo = ch_begin, c_hi = ch_end;
      const int c_in = (pr.N - tc.bj * TBN + CW - 1) / CW;
      if (c_hi > c_in) c_hi = c_in;
      if (row_lo >= pr.M) c_hi = c_lo;
      while (tri && c_lo < c_hi && tc.bj * TBN + c_lo * CW + CW - 1 < row_lo) ++c_lo;
      const bool gram = pr.epi == EPI_GRAM;
      const int col_base = tc.bj * TBN;
      GramTile gt;
      gt.kind = GRAM_GENERAL;
      if (gram) gt = gram_tile_for(pr, tc.mat, row_lo, col_base + c_hi * CW);
      CinRow cin;
      cin.ok = false;
      if (gram && c_lo < c_hi) {  // the first chunk's input: overlaps the main loop
        if (gt.kind != GRAM_GENERAL)
          cin16_fetch(gt, i, col_base + c_lo * CW, cin);
        else
          cin_fetch(pr, tc.mat, i, col_base + c_lo * CW, cin);
      }
      int ok = 1;
      if (lane == 0) ok = wait_bar(tfull_bar(acc), acc_phase, abort_flag, p) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t tacc = tmem_base + (uint32_t)(acc * TBN) + ((uint32_t)(q * 32) << 16);
      const int tri_end = tri ? INT_MAX : INT_MIN;
      if (gt.kind == GRAM_BB) {
        gram_tile16<false, false>(gt, tacc, col_base, c_lo, c_hi, row_lo, lane, tri_end, scr, cin);
      } else if (gt.kind == GRAM_HH) {
        gram_tile16<true, true>(gt, tacc, col_base, c_lo, c_hi, row_lo, lane, tri_end, scr, cin);
      } else if (gt.kind == GRAM_BH) {
        gram_tile16<false, true>(gt, tacc, col_base, c_lo, c_hi, row_lo, lane, tri_end, scr, cin);
      } else {
        for (int ch = c_lo; ch < c_hi; ++ch) {
          const int col0 = col_base + ch * CW;
          uint32_t r[CW];
          ptx::tmem_ld16(tacc + (uint32_t)(ch * CW), r);
          ptx::tmem_wait_ld();
          if (gram) {
            epi_gram_chunk(pr, tc.mat, i, col0, r, tri, scr, cin);
            if (ch + 1 < c_hi) cin_fetch(pr, tc.mat, i, col0 + CW, cin);  // overlaps the next accumulator load
          } else {
            epi_update_chunk(pr, tc.mat, i, col0, r);
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------- CTA-pair kernel
// Same problems and epilogues, computed by CTA pairs (a cluster of 2) on
// 256 x 256 output tiles with tcgen05.mma.cta_group::2 (M = 256, N = 256):
// CTA r of the pair TMA-loads rows [128 r, 128 r + 128) of the tile's A
// block and of its B block into its own shared memory and holds rows
// [128 r, 128 r + 128) of the accumulator in its own TMEM.  Per SM this
// halves the B operand bytes of the 128 x 256 single-CTA tile (64 instead
// of 96 bytes per MMA clock), and one K-block stage is only 32 KB, so six
// stages fit.  The leader (rank 0) arms the stage barrier with both CTAs'
// bytes and issues the MMAs; its commits arrive on both CTAs' barriers;
// both epilogues arrive on the leader's TMEM-empty barrier.  No load uses
// cluster multicast: every byte a CTA reads comes from its own TMA loads.
// With TN = 512 the pair's tile is 256 x 512: two N = 256 MMAs per K slice
// share the A operand (a quarter fewer operand bytes per MMA), and the
// 512-column accumulator fills TMEM, so the epilogue of a tile does not
// overlap the next tile's main loop.
constexpr int BM2 = 256;
constexpr int HALF_BYTES = 128 * 128;  // 128 rows x 128-byte K row

// K atoms (128-byte rows) per stage.  By default the one-MMA-per-slice
// configurations take three atoms (12 MMAs, two 96 KB stages) per stage, to
// amortise the fixed cost of a stage boundary (commit, barrier wait, fence);
// the split configurations already issue 8-12 MMAs per atom.  KATV > 0
// overrides the default: fewer atoms per stage mean more stages, so more
// bytes are in flight while the tensor cores work on one stage (2 atoms:
// three 64 KB stages; 1 atom: six 32 KB stages).  The schedule cache picks
// among them per Gram class.
template <int NA, int NB, int KATV = 0, int TN = 256>
struct Tc2Cfg {
  // TN = 512: the pair's tile is 256 x 512 (two N = 256 MMAs per K slice
  // share the A operand), one 512-column accumulator per CTA
  static constexpr int NH = TN == 512 ? 2 : 1;  // B halves per part
  static constexpr int NACC = TN == 512 ? 1 : 2;  // TMEM accumulators
  static constexpr int KAT = KATV > 0 ? KATV : (TN == 512 ? 1 : ((NA + NB <= 2) ? 3 : 1));
  static constexpr int STAGE_BYTES = (NA + NB * NH) * HALF_BYTES * KAT;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256 + EPI_SCRATCH_BYTES;
  static_assert(STAGES >= 2 && STAGES <= 8, "stage count");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(TN == 256 || TN == 512, "pair tile width");
  static_assert(NACC * TN == TMEM_COLS, "accumulators fill TMEM");
};

__device__ __forceinline__ bool wait_bar_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                 const GemmParams& p) {
  if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (;;) {
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if ((long long)(ptx::globaltimer() - t0) > p.timeout_ns) {
      *abort_flag = 1;
      atomicOr(p.status, DMU_FLAG_TIMEOUT);
      return false;
    }
  }
}

template <int NA, int NB, int KIND, int KATV, int TN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    k_gemm_tc2(const __grid_constant__ GemmParams p) {
  using Cfg = Tc2Cfg<NA, NB, KATV, TN>;
  constexpr int NH = Cfg::NH;
  constexpr int NACC = Cfg::NACC;
  constexpr int S = Cfg::STAGES;
  constexpr int KATOMS = Cfg::KAT;
  constexpr int ATOM_E = KIND == KIND_TF32 ? 32 : 64;  // elements per 128-byte K row
  constexpr int BKE = ATOM_E * KATOMS;                 // K elements per stage
  constexpr int OPFMT = KIND == KIND_TF32 ? 2 : (KIND == KIND_F16 ? 0 : 1);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t ring = base;
  const uint32_t bars = base + S * Cfg::STAGE_BYTES;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (S + s); };
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * S + b); };
  auto tempty_bar = [&](int b) { return bars + 8u * (2 * S + 2 + b); };
  const uint32_t drain_bar = bars + 8u * (2 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S * Cfg::STAGE_BYTES + 8 * (2 * S + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), 2 * EPI_WARPS);
    }
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    for (int pi = 0; pi < p.nprob; ++pi) {
      ptx::prefetch_tmap(&p.maps[p.prob[pi].a_map]);
      ptx::prefetch_tmap(&p.maps[p.prob[pi].b_map]);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc2(ptx::smem_u32(tmem_slot), TMEM_COLS);
    ptx::tmem_relinquish2();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // both CTAs' barriers exist before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t issued_mask = 0, issued_par = 0;
      for (int t = pair; ok && t < p.total_tiles; t += npairs) {
        const TileCoord tc = decode_tile<BM2, TN>(p, t);
        const GemmProblem& pr = p.prob[tc.pi];
        // Per-tile operand parameters, read from the parameter space once:
        // the K loop below issues only TMA copies and barrier operations.
        const CUtensorMap* am = &p.maps[pr.a_map];
        const CUtensorMap* bm = &p.maps[pr.b_map];
        const CUtensorMap* am_t = pr.half_a ? &p.maps[pr.a_map_t] : am;
        const CUtensorMap* bm_t = pr.half_b ? &p.maps[pr.b_map_t] : bm;
        // half-stored operands: row block r, K block c < r reads the stored
        // transpose (thresholds in HALF_BLOCK units; B half h is block NH bj + h)
        const int thr_a = pr.half_a ? tc.bi : 0;
        const int thr_b0 = pr.half_b ? NH * tc.bj : 0, thr_b1 = pr.half_b ? NH * tc.bj + 1 : 0;
        const bool a_mn = pr.a_mn != 0, b_mn = pr.b_mn != 0;
        const int za0 = pr.a_z[0] + tc.mat, za1 = pr.a_z[1] + tc.mat;
        const int zb0 = pr.b_z[0] + tc.mat, zb1 = pr.b_z[1] + tc.mat;
        const int na = (NA > 1 && (pr.terms & TERM_LH)) ? 2 : 1;
        const int nb = (NB > 1 && (pr.terms & TERM_HL)) ? 2 : 1;
        const uint32_t bytes_pair = 2u * (uint32_t)(na + nb * NH) * HALF_BYTES * KATOMS;
        const int nk = (pr.K + BKE - 1) / BKE;
        const int arow = tc.bi * BM2 + (int)rank * 128, brow0 = tc.bj * TN + (int)rank * 128;
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_bar(empty_bar(stage), phase ^ 1u, abort_flag, p)) {
            ok = false;
            break;
          }
          const uint32_t fb_leader = ptx::mapa_shared(full_bar(stage), 0);
          if (leader) {
            ptx::mbar_arrive_expect_tx(full_bar(stage), bytes_pair);
            issued_mask |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          }
          // stage layout: [A parts][B parts], each part KATOMS 16 KB atoms
          const uint32_t sa = ring + stage * Cfg::STAGE_BYTES;
          const uint32_t sb = sa + NA * KATOMS * HALF_BYTES;
#pragma unroll
          for (int at = 0; at < KATOMS; ++at) {
            const int k0 = kb * BKE + at * ATOM_E;
            const int ktile = k0 / HALF_BLOCK;
            const bool a_t = ktile < thr_a;  // rows of block bi, K in an earlier block
            const CUtensorMap* am_k = a_t ? am_t : am;
            for (int part = 0; part < na; ++part) {
              const uint32_t dst = sa + (part * KATOMS + at) * HALF_BYTES;
              const int z = part ? za1 : za0;
              if (!a_mn && !a_t) {
                ptx::tma_load_3d_pair(dst, am_k, fb_leader, k0, arow, z);
              } else {
                ptx::tma_load_3d_pair(dst, am_k, fb_leader, arow, k0, z);
                ptx::tma_load_3d_pair(dst + 8192, am_k, fb_leader, arow + 64, k0, z);
              }
            }
            // B layout: [part][half][atom], 16 KB each
#pragma unroll
            for (int h = 0; h < NH; ++h) {
              const bool b_t = ktile < (h ? thr_b1 : thr_b0);
              const CUtensorMap* bm_k = b_t ? bm_t : bm;
              const int brow = brow0 + h * 256;
              for (int part = 0; part < nb; ++part) {
                const uint32_t dst = sb + ((part * NH + h) * KATOMS + at) * HALF_BYTES;
                const int z = part ? zb1 : zb0;
                if (!b_mn && !b_t) {
                  ptx::tma_load_3d_pair(dst, bm_k, fb_leader, k0, brow, z);
                } else {
                  ptx::tma_load_3d_pair(dst, bm_k, fb_leader, brow, k0, z);
                  ptx::tma_load_3d_pair(dst + 8192, bm_k, fb_leader, brow + 64, k0, z);
                }
              }
            }
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // The leader's stage barriers count both CTAs' bytes: wait until every
      // phase it armed has landed before the pair may exit.
      for (int s2 = 0; s2 < S; ++s2) {
        if (!(issued_mask & (1u << s2))) continue;
        const uint32_t par = (issued_par >> s2) & 1u;
        const uint64_t t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait_cluster(full_bar(s2), par)) {
          if ((long long)(ptx::globaltimer() - t0) > p.timeout_ns) {
            atomicOr(p.status, DMU_FLAG_TIMEOUT);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader only)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued = false;
      for (int t = pair; ok && t < p.total_tiles; t += npairs) {
        const TileCoord tc = decode_tile<BM2, TN>(p, t);
        const GemmProblem& pr = p.prob[tc.pi];
        const int nk = (pr.K + BKE - 1) / BKE;
        if (!wait_bar_cluster(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TN);
        uint32_t accumulate[2] = {0u, 0u};  // per N = 256 half of the accumulator
        const int terms = pr.terms, pr_a_mn = pr.a_mn, pr_b_mn = pr.b_mn;
        const int thr_a = pr.half_a ? tc.bi : 0;
        const int thr_b0 = pr.half_b ? NH * tc.bj : 0, thr_b1 = pr.half_b ? NH * tc.bj + 1 : 0;
        const uint32_t idesc0 = ptx::make_idesc(BM2, BN, 0, 0, OPFMT);
        const uint64_t hi_k = ptx::make_sw128_desc(0u, 16u, 1024u), hi_mn = ptx::make_sw128_desc(0u, 8192u, 1024u);
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_bar(full_bar(stage), phase, abort_flag, p)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          // Descriptors: the start address (bits 0-13, bytes / 16) sits in
          // the low word and never carries out of its field (shared
          // addresses are below 256 KB), so each MMA's descriptor is an atom
          // base plus a constant, one 32-bit add.
          const uint32_t sa = ring + stage * Cfg::STAGE_BYTES;
          const uint32_t sb = sa + NA * KATOMS * HALF_BYTES;
#pragma unroll
          for (int at = 0; at < KATOMS; ++at) {
            const int ktile = (kb * BKE + at * ATOM_E) / HALF_BLOCK;
            const uint32_t a_mn = (uint32_t)(pr_a_mn | (ktile < thr_a ? 1 : 0));
            const uint64_t a_hi = a_mn ? hi_mn : hi_k;
            const uint32_t a_up = (uint32_t)(a_hi >> 32), a_dk = a_mn ? 2048u / 16u : 32u / 16u;
            const uint32_t a_lo0 = (uint32_t)a_hi | ((sa + at * HALF_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // the NH halves of the tile share this K slice's A operand
#pragma unroll
              for (int h = 0; h < NH; ++h) {
                const uint32_t b_mn = (uint32_t)(pr_b_mn | (ktile < (h ? thr_b1 : thr_b0) ? 1 : 0));
                const uint32_t idesc = idesc0 | (a_mn << 15) | (b_mn << 16);
                const uint64_t b_hi = b_mn ? hi_mn : hi_k;
                const uint32_t b_up = (uint32_t)(b_hi >> 32), b_dk = b_mn ? 2048u / 16u : 32u / 16u;
                const uint32_t b_lo0 = (uint32_t)b_hi | ((sb + (h * KATOMS + at) * HALF_BYTES) >> 4);
#pragma unroll
                for (int term = 0; term < 3; ++term) {
                  if (term == 1 && NB < 2) continue;
                  if (term == 2 && NA < 2) continue;
                  if (!(terms & (1 << term))) continue;
                  const uint32_t a_lo = a_lo0 + kk * a_dk + (term == 2 ? KATOMS * HALF_BYTES / 16 : 0);
                  const uint32_t b_lo = b_lo0 + kk * b_dk + (term == 1 ? NH * KATOMS * HALF_BYTES / 16 : 0);
                  const uint64_t ad = ((uint64_t)a_up << 32) | a_lo;
                  const uint64_t bd = ((uint64_t)b_up << 32) | b_lo;
                  if (KIND == KIND_TF32)
                    ptx::mma2_tf32(d_tmem + (uint32_t)(h * 256), ad, bd, idesc, accumulate[h]);
                  else
                    ptx::mma2_f16(d_tmem + (uint32_t)(h * 256), ad, bd, idesc, accumulate[h]);
                  accumulate[h] = 1;
                }
              }
            }
          }
          issued = true;
          ptx::mma2_commit_both(empty_bar(stage));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma2_commit_both(tfull_bar(acc));
        if (++acc == NACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok && issued) {
        ptx::mma2_commit_both(drain_bar);
        const uint64_t t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait_cluster(drain_bar, 0)) {
          if ((long long)(ptx::globaltimer() - t0) > p.timeout_ns) break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (both CTAs, warps 2..9)
    const int q = warp & 3;
    const uint32_t scr = bars + 256u + (uint32_t)(warp - 2) * TRI_SCRATCH;
    const int ch_begin = ((warp - 2) >> 2) * (TN / 2 / CW);
    const int ch_end = ch_begin + TN / 2 / CW;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < p.total_tiles; t += npairs) {
      const TileCoord tc = decode_tile<BM2, TN>(p, t);
      const GemmProblem& pr = p.prob[tc.pi];
      const int row_lo = tc.bi * BM2 + (int)rank * 128 + q * 32;
      const int i = row_lo + lane;
      // half-stored outputs: lower blocks are never written, the diagonal
      // block is mirrored, upper blocks are written whole
      auto chunk_tri = [&](int col0) { return pr.sym && (!pr.half_out || col0 / HALF_BLOCK == tc.bi); };
      // this warp's chunks of the tile, [c_lo, c_hi): inside the matrix, not
      // in a lower block, not strictly below the diagonal (the skipped
      // chunks of a tile are always its leftmost ones)
      int c_lo = ch_begin, c_hi = ch_end;
      const int c_in = (pr.N - tc.bj * TN + CW - 1) / CW;
      if (c_hi > c_in) c_hi = c_in;
      if (row_lo >= pr.M) c_hi = c_lo;
      while (c_lo < c_hi) {
        const int col0 = tc.bj * TN + c_lo * CW;
        if (pr.sym && pr.half_out && col0 / HALF_BLOCK < tc.bi) { ++c_lo; continue; }
        if (chunk_tri(col0) && col0 + CW - 1 < row_lo) { ++c_lo; continue; }
        break;
      }
      const bool gram = pr.epi == EPI_GRAM;
      const int col_base = tc.bj * TN;
      GramTile gt;
      gt.kind = GRAM_GENERAL;
      if (gram) gt = gram_tile_for(pr, tc.mat, row_lo, col_base + c_hi * CW);
      CinRow cin;
      cin.ok = false;
      if (gram && c_lo < c_hi) {  // the first chunk's input: overlaps the main loop
        if (gt.kind != GRAM_GENERAL)
          cin16_fetch(gt, i, col_base + c_lo * CW, cin);
        else
          cin_fetch(pr, tc.mat, i, col_base + c_lo * CW, cin);
      }
      int ok = 1;
      if (lane == 0) ok = wait_bar_cluster(tfull_bar(acc), acc_phase, abort_flag, p) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t tacc = tmem_base + (uint32_t)(acc * TN) + ((uint32_t)(q * 32) << 16);
      // symmetric chunks: all (not half-stored) or those of the diagonal block
      const int tri_end = !pr.sym ? INT_MIN : (!pr.half_out ? INT_MAX : (tc.bi + 1) * HALF_BLOCK);
      if (gt.kind == GRAM_BB) {
        gram_tile16<false, false>(gt, tacc, col_base, c_lo, c_hi, row_lo, lane, tri_end, scr, cin);
      } else if (gt.kind == GRAM_HH) {
        gram_tile16<true, true>(gt, tacc, col_base, c_lo, c_hi, row_lo, lane, tri_end, scr, cin);
      } else if (gt.kind == GRAM_BH) {
        gram_tile16<false, true>(gt, tacc, col_base, c_lo, c_hi, row_lo, lane, tri_end, scr, cin);
      } else {
        for (int ch = c_lo; ch < c_hi; ++ch) {
          const int col0 = col_base + ch * CW;
          uint32_t r[CW];
          ptx::tmem_ld16(tacc + (uint32_t)(ch * CW), r);
          ptx::tmem_wait_ld();
          if (gram) {
            epi_gram_chunk(pr, tc.mat, i, col0, r, chunk_tri(col0), scr, cin);
            if (ch + 1 < c_hi) cin_fetch(pr, tc.mat, i, col0 + CW, cin);  // overlaps the next accumulator load
          } else {
            epi_update_chunk(pr, tc.mat, i, col0, r);
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(tempty_bar(acc), 0));
      if (++acc == NACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  ptx::cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc2(tmem_base, TMEM_COLS);
  }
}

// Bounded-wait self-test: one thread waits on an mbarrier that nothing
// arrives on; the wait gives up after timeout_ns and sets DMU_FLAG_TIMEOUT.
__global__ void k_wait_selftest(unsigned int* status, long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&bar), 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = ptx::globaltimer();
    for (;;) {
      if (ptx::mbar_try_wait(ptx::smem_u32(&bar), 0)) break;
      if ((long long)(ptx::globaltimer() - t0) > timeout_ns) {
        atomicOr(status, DMU_FLAG_TIMEOUT);
        break;
      }
    }
  }
}

cudaError_t launch_wait_selftest(unsigned int* status, long long timeout_ns, cudaStream_t s) {
  k_wait_selftest<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

template <int NA, int NB, int KIND, int TBN>
static cudaError_t configure_one() {
  return cudaFuncSetAttribute(k_gemm_tc<NA, NB, KIND, TBN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              TcCfg<NA, NB, TBN>::SMEM_BYTES);
}

template <int NA, int NB, int KIND, int KATV = 0, int TN = 256>
static cudaError_t configure_two() {
  return cudaFuncSetAttribute(k_gemm_tc2<NA, NB, KIND, KATV, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Tc2Cfg<NA, NB, KATV, TN>::SMEM_BYTES);
}

cudaError_t gemm_tc_configure() {
  cudaError_t e;
  if ((e = configure_one<1, 1, KIND_BF16, 256>()) != cudaSuccess) return e;
  if ((e = configure_one<1, 1, KIND_BF16, 128>()) != cudaSuccess) return e;
  if ((e = configure_one<2, 1, KIND_BF16, 256>()) != cudaSuccess) return e;
  if ((e = configure_one<2, 1, KIND_BF16, 128>()) != cudaSuccess) return e;
  if ((e = configure_one<2, 2, KIND_BF16, 256>()) != cudaSuccess) return e;
  if ((e = configure_one<2, 2, KIND_BF16, 128>()) != cudaSuccess) return e;
  if ((e = configure_one<1, 1, KIND_TF32, 256>()) != cudaSuccess) return e;
  if ((e = configure_one<1, 1, KIND_TF32, 128>()) != cudaSuccess) return e;
  if ((e = configure_one<1, 1, KIND_F16, 256>()) != cudaSuccess) return e;
  if ((e = configure_one<1, 1, KIND_F16, 128>()) != cudaSuccess) return e;
  if ((e = configure_one<2, 1, KIND_F16, 256>()) != cudaSuccess) return e;
  if ((e = configure_one<2, 1, KIND_F16, 128>()) != cudaSuccess) return e;
  if ((e = configure_two<1, 1, KIND_BF16>()) != cudaSuccess) return e;
  if ((e = configure_two<2, 1, KIND_BF16>()) != cudaSuccess) return e;
  if ((e = configure_two<2, 2, KIND_BF16>()) != cudaSuccess) return e;
  if ((e = configure_two<1, 1, KIND_TF32>()) != cudaSuccess) return e;
  if ((e = configure_two<1, 1, KIND_F16>()) != cudaSuccess) return e;
  if ((e = configure_two<1, 1, KIND_F16, 2>()) != cudaSuccess) return e;
  if ((e = configure_two<1, 1, KIND_F16, 1>()) != cudaSuccess) return e;
  if ((e = configure_two<2, 1, KIND_F16>()) != cudaSuccess) return e;
  if ((e = configure_two<1, 1, KIND_F16, 0, 512>()) != cudaSuccess) return e;
  if ((e = configure_two<2, 1, KIND_F16, 0, 512>()) != cudaSuccess) return e;
  return cudaSuccess;
}

int gemm_tc_stages(int na, int nb) {
  if (na == 1 && nb == 1) return TcCfg<1, 1>::STAGES;
  if (na == 2 && nb == 1) return TcCfg<2, 1>::STAGES;
  if (na == 2 && nb == 2) return TcCfg<2, 2>::STAGES;
  return 0;
}

template <int NA, int NB, int KIND>
static cudaError_t launch_one(const GemmParams& p, int num_sms, int tbn, cudaStream_t s) {
  const int grid = p.total_tiles < num_sms ? p.total_tiles : num_sms;
  if (grid <= 0) return cudaSuccess;
  if (tbn == 128)
    k_gemm_tc<NA, NB, KIND, 128><<<grid, GEMM_THREADS, TcCfg<NA, NB, 128>::SMEM_BYTES, s>>>(p);
  else
    k_gemm_tc<NA, NB, KIND, 256><<<grid, GEMM_THREADS, TcCfg<NA, NB, 256>::SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

template <int NA, int NB, int KIND, int KATV = 0, int TN = 256>
static cudaError_t launch_two(const GemmParams& p, int num_sms, cudaStream_t s) {
  int pairs = num_sms / 2;
  if (p.total_tiles < pairs) pairs = p.total_tiles;
  if (pairs <= 0) return cudaSuccess;
  k_gemm_tc2<NA, NB, KIND, KATV, TN><<<2 * pairs, GEMM_THREADS, Tc2Cfg<NA, NB, KATV, TN>::SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc2(const GemmParams& p, int na, int nb, int kind, int num_sms, int kat, int tn,
                            cudaStream_t s) {
  if (tn == 512) {  // 256 x 512 pair tiles: scaled-fp16 operands only
    if (kind != KIND_F16) return cudaErrorInvalidValue;
    if (na == 1 && nb == 1) return launch_two<1, 1, KIND_F16, 0, 512>(p, num_sms, s);
    if (na == 2 && nb == 1) return launch_two<2, 1, KIND_F16, 0, 512>(p, num_sms, s);
    return cudaErrorInvalidValue;
  }
  if (tn != 256) return cudaErrorInvalidValue;
  if (kind == KIND_TF32) {
    if (na == 1 && nb == 1) return launch_two<1, 1, KIND_TF32>(p, num_sms, s);
    return cudaErrorInvalidValue;
  }
  if (kind == KIND_F16) {
    if (na == 1 && nb == 1) {
      if (kat == 1) return launch_two<1, 1, KIND_F16, 1>(p, num_sms, s);
      if (kat == 2) return launch_two<1, 1, KIND_F16, 2>(p, num_sms, s);
      return launch_two<1, 1, KIND_F16>(p, num_sms, s);
    }
    if (na == 2 && nb == 1) return launch_two<2, 1, KIND_F16>(p, num_sms, s);
    return cudaErrorInvalidValue;
  }
  if (na == 1 && nb == 1) return launch_two<1, 1, KIND_BF16>(p, num_sms, s);
  if (na == 2 && nb == 1) return launch_two<2, 1, KIND_BF16>(p, num_sms, s);
  if (na == 2 && nb == 2) return launch_two<2, 2, KIND_BF16>(p, num_sms, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_tc(const GemmParams& p, int na, int nb, int kind, int num_sms, int tbn,
                           cudaStream_t s) {
  if (tbn != 128 && tbn != 256) return cudaErrorInvalidValue;
  if (kind == KIND_TF32) {
    if (na == 1 && nb == 1) return launch_one<1, 1, KIND_TF32>(p, num_sms, tbn, s);
    return cudaErrorInvalidValue;
  }
  if (kind == KIND_F16) {
    if (na == 1 && nb == 1) return launch_one<1, 1, KIND_F16>(p, num_sms, tbn, s);
    if (na == 2 && nb == 1) return launch_one<2, 1, KIND_F16>(p, num_sms, tbn, s);
    return cudaErrorInvalidValue;
  }
  if (na == 1 && nb == 1) return launch_one<1, 1, KIND_BF16>(p, num_sms, tbn, s);
  if (na == 2 && nb == 1) return launch_one<2, 1, KIND_BF16>(p, num_sms, tbn, s);
  if (na == 2 && nb == 2) return launch_one<2, 2, KIND_BF16>(p, num_sms, tbn, s);
  return cudaErrorInvalidValue;
}

}  // namespace dmu
