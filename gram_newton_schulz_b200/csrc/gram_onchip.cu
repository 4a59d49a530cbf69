// The whole Gram Newton-Schulz recursion of one small matrix (m <= 128) in
// one CTA, sm_100a.
//
// DMuon page, section 2.2: the recursion runs in the m x m Gram space
// G = X X^T and matrices of similar shape are batched.  For m <= 128 a
// Gram-space matrix is a single 128 x 128 tile, so the staged path (one
// grouped launch per product, every product reading and writing HBM)
// spends its time on launch gaps and epilogue memory traffic rather than on
// the tensor cores.  Here every matrix stays on chip from the Gram matrix
// to the final P:
//
//   SYRK    G0 = s^2 X X^T                    (X streamed from the image by TMA)
//   step k  R = b G + c (G G)                 (k = 0 also P1 = a I + R)
//           T = a G + R G          (k < K-1)
//           P' = a P + R P         (k >= 1)
//           G' = a T + T R         (k < K-1)
//   only P_K leaves the SM: an fp16 hi/lo pair in the class's final-P area,
//   where the final O = P X0 GEMM (fused with the weight update) reads it.
// X is the fp16 image 2^e M (scale folded into `inv`), so the Gram matrix
// is one kind::f16 MMA per K slice on fp16 operands.
//
// Precision is the split-bf16 class of the staged path (three MMAs per
// product: hi*hi + hi*lo + lo*hi), with the same K order, the same epilogue
// arithmetic and the same mirrored upper-triangle stores, so both paths give
// bitwise-equal results.
//
// Shared memory (224 KB): three 64 KB buffers, each a 128 x 128 bf16 hi/lo
// pair in the tcgen05 K-major 128-byte-swizzled operand layout (2 K-atoms of
// 128 rows x 64 columns per part).  Symmetric matrices serve as either
// operand.  Buffer G holds G and, in turn, T (T = aG + RG is the last reader
// of G; G' = aT + TR overwrites T in place); buffer R holds R; buffer P
// holds P.  Rows and columns >= m stay zero.  While the Gram matrix is
// formed, buffers R and P are the TMA staging ring (8 stages of 16 KB).
//
// TMEM: 4 accumulators of 128 columns (SYRK / G', R, T, P').
// Warps: 0 TMA producer, 1 MMA issuer (one thread), 2-17 epilogue (four per
// TMEM lane quarter, each on a quarter of the columns, in 8-column chunks:
// an epilogue is a long dependent chain per warp, so more warps with
// shorter chains finish it sooner).  Every mbarrier wait is
// bounded by the plan's time limit; on expiry the CTA sets
// DMU_FLAG_TIMEOUT and winds down.
#include "dmu_internal.h"
#include "ptx.cuh"

namespace dmu {
namespace {

constexpr int OC_EPI_WARPS = 16;        // four per TMEM lane quarter
constexpr int OC_THREADS = 64 + 32 * OC_EPI_WARPS;
constexpr int OC_ATOM = 16384;            // 128 rows x 128 bytes
constexpr int OC_PART = 2 * OC_ATOM;      // 128 x 128 bf16
constexpr int OC_BUF = 2 * OC_PART;       // hi + lo
constexpr int OC_STAGES = 8;              // SYRK staging in buffers R and P
constexpr int OC_SMEM = 1024 + 3 * OC_BUF + 512;
constexpr int OC_CW = 8;                  // epilogue chunk width (columns): one 16-byte swizzle chunk
constexpr int OC_SLICE = 128 / (OC_EPI_WARPS / 4);  // columns per epilogue warp
enum { BUF_G = 0, BUF_R = 1, BUF_P = 2 };

static_assert(OC_STAGES * OC_ATOM == 2 * OC_BUF, "staging ring covers buffers R and P");
static_assert(OC_SMEM <= 232448, "shared memory per CTA");

// Byte offset of element (i, j) inside one part (hi or lo) of a buffer.
__device__ __forceinline__ uint32_t oc_off(int i, int j) {
  return (uint32_t)((j >> 6) * OC_ATOM + i * 128 + ((((j >> 3) & 7) ^ (i & 7)) << 4) + (j & 7) * 2);
}

__device__ __forceinline__ float bf(__nv_bfloat16 x) { return __bfloat162float(x); }

struct Bars {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t empty(int s) const { return base + 8u * (OC_STAGES + s); }
  __device__ uint32_t acc(int a) const { return base + 8u * (2 * OC_STAGES + a); }
  __device__ uint32_t epi_g() const { return base + 8u * (2 * OC_STAGES + 4); }
  __device__ uint32_t epi_r() const { return base + 8u * (2 * OC_STAGES + 5); }
  __device__ uint32_t epi_p() const { return base + 8u * (2 * OC_STAGES + 6); }
  __device__ uint32_t mat_done() const { return base + 8u * (2 * OC_STAGES + 7); }
  __device__ uint32_t drain() const { return base + 8u * (2 * OC_STAGES + 8); }
};
constexpr int OC_NBARS = 2 * OC_STAGES + 9;

// Bounded wait on an mbarrier phase; false when the CTA is winding down.
__device__ __forceinline__ bool oc_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        const OnchipParams& p) {
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

__device__ __forceinline__ int find_prob(const OnchipParams& p, int t) {
  int pi = 0;
  while (pi + 1 < p.nprob && t >= p.prob[pi + 1].mat_begin) ++pi;
  return pi;
}

// ------------------------------------------------------------- epilogue
// One product's epilogue, as in the staged path's Gram epilogue:
//   v = coef * acc + beta * Cin;  v[i][i] += 0;  out = v;  out2 = v + gamma2 I
// Cin, out and out2 are shared-memory buffers (byte offsets from the
// buffer base) or, for the final P, global hi/lo pairs.  Every rounding
// step is explicit (__fmul_rn, __fadd_rn, __fmaf_rn), as in the staged
// epilogue, so the compiler's choice of fused multiply-adds cannot make the
// two differ.  Only the upper
// triangle (j >= i) is computed and stored; element (j, i) receives a
// mirrored copy, so every stored matrix is exactly symmetric.
struct EpiArgs {
  float coef, beta, gamma2;
  int cin;        // buffer or -1
  int out;        // buffer, or -1 for the global P slot
  int out2;       // buffer, -1 none, -2 the global P slot
  __half* g_hi;  // global P of this matrix, fp16 pair (out == -1 or out2 == -2)
  __half* g_lo;
  long long ld;
};

// hi = RN(v), lo = RN(v - hi) (v - hi is exact), two values per packed
// conversion.
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

__device__ __forceinline__ void st_pair_h(__half* hi, __half* lo, long long o, float v) {
  const __half h = __float2half_rn(v);
  hi[o] = h;
  lo[o] = __float2half_rn(v - __half2float(h));
}


// Row stores of one chunk (row i, columns col0 .. col0 + 7, only i, j < m)
// as a bf16 hi/lo pair: rows above the chunk's diagonal 8 x 8 block and rows
// inside it store all eight values (inside the block, the values left of
// the diagonal are then replaced by mirror_chunk); rows below store nothing.
__device__ __forceinline__ void store_chunk_rows(uint8_t* buf, int m, int i, int col0, const float (&v)[OC_CW]) {
  if (i >= m || i >= col0 + OC_CW) return;
  uint32_t hi[OC_CW / 2], lo[OC_CW / 2];  // packed pairs of columns
#pragma unroll
  for (int c = 0; c < OC_CW; c += 2) {
    // hi = RN(v), lo = RN(v - hi) (exact difference), two per conversion
    const __nv_bfloat162 hq = __floats2bfloat162_rn(v[c], v[c + 1]);
    const float2 f = __bfloat1622float2(hq);
    const __nv_bfloat162 lq = __floats2bfloat162_rn(__fsub_rn(v[c], f.x), __fsub_rn(v[c + 1], f.y));
    hi[c / 2] = *reinterpret_cast<const uint32_t*>(&hq);
    lo[c / 2] = *reinterpret_cast<const uint32_t*>(&lq);
  }
  if (col0 + OC_CW <= m) {
    const uint32_t o = oc_off(i, col0);
    *reinterpret_cast<uint4*>(buf + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(buf + OC_PART + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  } else {
#pragma unroll
    for (int c = 0; c < OC_CW; ++c) {
      if (col0 + c < m) {
        const uint32_t o = oc_off(i, col0 + c);
        *reinterpret_cast<uint16_t*>(buf + o) = (uint16_t)(hi[c / 2] >> (16 * (c & 1)));
        *reinterpret_cast<uint16_t*>(buf + OC_PART + o) = (uint16_t)(lo[c / 2] >> (16 * (c & 1)));
      }
    }
  }
}

// A fragment register holding destination elements (row, col) (low half)
// and (row, col + 1) (high half), with the halves in the padding (row or
// column >= m) cleared.
__device__ __forceinline__ uint32_t pad_clear(uint32_t x, int row, int col, int m) {
  if (row >= m || col >= m) return 0u;
  return col + 1 < m ? x : (x & 0x0000FFFFu);
}

// The mirror images (j, i), i < j, of one chunk's upper elements (rows of
// lane quarter q, columns col0 .. col0 + 7, as store_chunk_rows left them),
// moved as 8 x 8 blocks: each block of 8 rows above the chunk's diagonal
// block is loaded transposed and stored into rows col0 .. col0 + 7; the
// diagonal block keeps its upper half and takes the transpose of that as its
// lower half.  Destination elements in the padding are written as zero, so
// this never meets the padding clear with a different value.  Warp-collective;
// the warp's row stores must be ordered before it (__syncwarp).
__device__ __forceinline__ void mirror_chunk(uint32_t buf, int m, int q, int lane, int col0) {
  const int rq = q * 32;
  const bool ragged = col0 + OC_CW > m || rq + 32 > m;
  const int fr = lane >> 2, fc = 2 * (lane & 3);  // fragment elements (fr, fc) and (fr, fc + 1)
  if (col0 >= rq + 32) {
    // all four blocks lie above the chunk's columns
    uint32_t h[4], l[4];
    const uint32_t src = buf + oc_off(rq + lane, col0);
    ptx::ldsm_x4_trans(src, h);
    ptx::ldsm_x4_trans(src + OC_PART, l);
    if (ragged) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        h[k] = pad_clear(h[k], col0 + fr, rq + 8 * k + fc, m);
        l[k] = pad_clear(l[k], col0 + fr, rq + 8 * k + fc, m);
      }
    }
    const uint32_t dst = buf + oc_off(col0 + (lane & 7), rq + 8 * (lane >> 3));
    ptx::stsm_x4(dst, h);
    ptx::stsm_x4(dst + OC_PART, l);
    return;
  }
  // the chunk holds the diagonal of this quarter: blocks 0 .. kd - 1 lie above
  const int kd = (col0 - rq) >> 3;
  const uint32_t part = (lane & 8) ? (uint32_t)OC_PART : 0u;  // matrix 0: hi, matrix 1: lo
  for (int k = 0; k < kd; ++k) {
    uint32_t a, b;
    ptx::ldsm_x2_trans(buf + oc_off(rq + 8 * k + (lane & 7), col0) + part, a, b);
    if (ragged) {
      a = pad_clear(a, col0 + fr, rq + 8 * k + fc, m);
      b = pad_clear(b, col0 + fr, rq + 8 * k + fc, m);
    }
    ptx::stsm_x2(buf + oc_off(col0 + (lane & 7), rq + 8 * k) + part, a, b);
  }
  const uint32_t d = buf + oc_off(col0 + (lane & 7), col0) + part;
  uint32_t a, b, at, bt;
  ptx::ldsm_x2(d, a, b);
  ptx::ldsm_x2_trans(d, at, bt);
  const uint32_t sel = (fr > fc ? 0x0000FFFFu : 0u) | (fr > fc + 1 ? 0xFFFF0000u : 0u);
  a = (a & ~sel) | (at & sel);
  b = (b & ~sel) | (bt & sel);
  if (ragged) {
    a = pad_clear(a, col0 + fr, col0 + fc, m);
    b = pad_clear(b, col0 + fr, col0 + fc, m);
  }
  ptx::stsm_x2(d, a, b);
}

// Global stores of one chunk of the final P (row i, columns col0 .. col0 +
// 7, only j < m) as an fp16 hi/lo pair (row stride ld): the upper elements
// and their mirror images, as the staged path writes them.
__device__ __forceinline__ void store_chunk_global(__half* ghi, __half* glo, long long ld, int m, int i, int col0,
                                                   const float (&v)[OC_CW]) {
  if (col0 + OC_CW <= m && i <= col0) {
#pragma unroll
    for (int q = 0; q < OC_CW / 8; ++q) {
      uint4 h, l;
      split8_h(v + 8 * q, h, l);
      *reinterpret_cast<uint4*>(ghi + i * ld + col0 + 8 * q) = h;
      *reinterpret_cast<uint4*>(glo + i * ld + col0 + 8 * q) = l;
    }
  } else {
#pragma unroll
    for (int c = 0; c < OC_CW; ++c) {
      const int j = col0 + c;
      if (j < m && i <= j) st_pair_h(ghi, glo, i * ld + j, v[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < OC_CW; ++c) {
    const int j = col0 + c;
    if (j < m && i < j) st_pair_h(ghi, glo, j * ld + i, v[c]);
  }
}

__device__ __forceinline__ void epilogue(uint8_t* smem, uint32_t sbase, uint32_t tacc, int q, int half, int lane,
                                         int m, const EpiArgs& e) {
  const int row_lo = q * 32;
  const int i = row_lo + lane;
  for (int ch = 0; ch < OC_SLICE / OC_CW; ++ch) {
    const int col0 = half * OC_SLICE + ch * OC_CW;
    if (col0 >= m) break;
    if (col0 + OC_CW - 1 < row_lo) continue;  // chunk strictly below the diagonal
    if (row_lo >= m) break;
    uint32_t r[OC_CW];
    ptx::tmem_ld8(tacc + (uint32_t)col0 + ((uint32_t)(q * 32) << 16), r);
    ptx::tmem_wait_ld();
    // rows >= m go through the arithmetic too (their values are never
    // stored): the block moves below are warp-collective
    float v[OC_CW];
#pragma unroll
    for (int c = 0; c < OC_CW; ++c) v[c] = __fmul_rn(e.coef, __uint_as_float(r[c]));
    if (e.cin >= 0) {
      const uint8_t* cb = smem + e.cin * OC_BUF;
      if (col0 + OC_CW <= m) {
#pragma unroll
        for (int qq = 0; qq < OC_CW / 8; ++qq) {
          const uint32_t o = oc_off(i, col0 + 8 * qq);
          const uint4 uh = *reinterpret_cast<const uint4*>(cb + o);
          const uint4 ul = *reinterpret_cast<const uint4*>(cb + OC_PART + o);
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&uh);
          const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&ul);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 fh = __bfloat1622float2(h2[t]);
            const float2 fl = __bfloat1622float2(l2[t]);
            v[8 * qq + 2 * t] = __fmaf_rn(e.beta, __fadd_rn(fh.x, fl.x), v[8 * qq + 2 * t]);
            v[8 * qq + 2 * t + 1] = __fmaf_rn(e.beta, __fadd_rn(fh.y, fl.y), v[8 * qq + 2 * t + 1]);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < OC_CW; ++c) {
          if (col0 + c < m) {
            const uint32_t o = oc_off(i, col0 + c);
            float x = bf(*reinterpret_cast<const __nv_bfloat16*>(cb + o));
            x = __fadd_rn(x, bf(*reinterpret_cast<const __nv_bfloat16*>(cb + OC_PART + o)));
            v[c] = __fmaf_rn(e.beta, x, v[c]);
          }
        }
      }
    }
    const int dc = i - col0;
#pragma unroll
    for (int c = 0; c < OC_CW; ++c)
      if (c == dc) v[c] = __fadd_rn(v[c], 0.f);
    if (e.out >= 0)
      store_chunk_rows(smem + e.out * OC_BUF, m, i, col0, v);
    else if (i < m)
      store_chunk_global(e.g_hi, e.g_lo, e.ld, m, i, col0, v);
    if (e.out2 != -1) {
#pragma unroll
      for (int c = 0; c < OC_CW; ++c) v[c] = __fmaf_rn(v[c], 1.f, c == dc ? e.gamma2 : 0.f);
      if (e.out2 >= 0)
        store_chunk_rows(smem + e.out2 * OC_BUF, m, i, col0, v);
      else if (i < m)
        store_chunk_global(e.g_hi, e.g_lo, e.ld, m, i, col0, v);
    }
    if (e.out >= 0 || e.out2 >= 0) {
      __syncwarp();
      if (e.out >= 0) mirror_chunk(sbase + e.out * OC_BUF, m, q, lane, col0);
      if (e.out2 >= 0) mirror_chunk(sbase + e.out2 * OC_BUF, m, q, lane, col0);
    }
  }
}

// Generic-proxy shared-memory writes of this thread become visible to the
// tensor cores (async proxy) once the consumer has waited on the barrier
// that follows.
__device__ __forceinline__ void epi_done(uint32_t bar, int lane) {
  ptx::tc_fence_before();
  ptx::fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) ptx::mbar_arrive(bar);
}

// ------------------------------------------------------------- MMA helpers
// One symmetric product D = A B over K = m (K atoms of 64 in order), three
// bf16 terms per K slice (hi*hi, hi*lo, lo*hi) in the staged path's order.
__device__ __forceinline__ void issue_product(uint32_t d_tmem, uint32_t a_buf, uint32_t b_buf, int m) {
  const uint32_t idesc = ptx::make_idesc(128, 128, 0, 0, 1);
  const uint64_t hi_k = ptx::make_sw128_desc(0u, 16u, 1024u);
  const int nk = (m + 63) / 64;
  uint32_t accumulate = 0;
  for (int kb = 0; kb < nk; ++kb) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        const uint32_t pa = a_buf + (term == 2 ? OC_PART : 0) + kb * OC_ATOM + kk * 32;
        const uint32_t pb = b_buf + (term == 1 ? OC_PART : 0) + kb * OC_ATOM + kk * 32;
        ptx::mma_bf16(d_tmem, hi_k | (uint64_t)((pa >> 4) & 0x3FFFu), hi_k | (uint64_t)((pb >> 4) & 0x3FFFu),
                      idesc, accumulate);
        accumulate = 1;
      }
    }
  }
}

__global__ void __launch_bounds__(OC_THREADS, 1) k_gram_onchip(const __grid_constant__ OnchipParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const Bars bars{base + 3 * OC_BUF};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 3 * OC_BUF + 8 * OC_NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t buf_addr[3] = {base, base + OC_BUF, base + 2 * OC_BUF};
  const uint32_t ring = base + OC_BUF;  // staging stage s at ring + s * OC_ATOM

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = p.steps;

  if (threadIdx.x == 0) {
    for (int s = 0; s < OC_STAGES; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.empty(s), 1);
    }
    for (int a = 0; a < 4; ++a) ptx::mbar_init(bars.acc(a), 1);
    ptx::mbar_init(bars.epi_g(), OC_EPI_WARPS);
    ptx::mbar_init(bars.epi_r(), OC_EPI_WARPS);
    ptx::mbar_init(bars.epi_p(), OC_EPI_WARPS);
    ptx::mbar_init(bars.mat_done(), OC_EPI_WARPS);
    ptx::mbar_init(bars.drain(), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0)
    for (int pi = 0; pi < p.nprob; ++pi) ptx::prefetch_tmap(&p.maps[p.prob[pi].map]);
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer: the image of X
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t issued_mask = 0, issued_par = 0;
      int local = 0;
      for (int t = blockIdx.x; ok && t < p.total; t += gridDim.x, ++local) {
        const OnchipProblem& pr = p.prob[find_prob(p, t)];
        const CUtensorMap* map = &p.maps[pr.map];
        const int z = t - pr.mat_begin;
        // the staging ring lives in buffers R and P: wait until the previous
        // matrix's last epilogue has finished with them
        if (local > 0 && !oc_wait(bars.mat_done(), (uint32_t)((local - 1) & 1), abort_flag, p)) {
          ok = false;
          break;
        }
        const int nk = (pr.n + 63) / 64;
        for (int kb = 0; kb < nk; ++kb) {
          if (!oc_wait(bars.empty(stage), phase ^ 1u, abort_flag, p)) {
            ok = false;
            break;
          }
          const uint32_t fb = bars.full(stage);
          ptx::mbar_arrive_expect_tx(fb, OC_ATOM);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          const uint32_t dst = ring + stage * OC_ATOM;
          if (!pr.tall) {
            ptx::tma_load_3d(dst, map, fb, kb * 64, 0, z);
          } else {
            ptx::tma_load_3d(dst, map, fb, 0, kb * 64, z);
            ptx::tma_load_3d(dst + 8192, map, fb, 64, kb * 64, z);
          }
          if (++stage == OC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      for (int s2 = 0; s2 < OC_STAGES; ++s2) {  // every issued copy has landed before exit
        if (!(issued_mask & (1u << s2))) continue;
        const uint32_t par = (issued_par >> s2) & 1u;
        const uint64_t t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait(bars.full(s2), par)) {
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
      uint32_t n_g = 0, n_r = 0, n_p = 0;  // epilogue completions waited for
      bool ok = true, issued = false;
      for (int t = blockIdx.x; ok && t < p.total; t += gridDim.x) {
        const OnchipProblem& pr = p.prob[find_prob(p, t)];
        // SYRK into accumulator 0 (the previous matrix's last use of it was
        // G' of step K-2, whose epilogue was waited for before step K-1)
        const int nk = (pr.n + 63) / 64;
        const uint32_t mn = pr.tall ? 1u : 0u;
        const uint32_t idesc = ptx::make_idesc(128, 128, mn, mn, 0);  // fp16 image operands
        const uint64_t hi_d = mn ? ptx::make_sw128_desc(0u, 8192u, 1024u) : ptx::make_sw128_desc(0u, 16u, 1024u);
        const uint32_t ks = mn ? 2048u : 32u;
        uint32_t accumulate = 0;
        for (int kb = 0; kb < nk; ++kb) {
          if (!oc_wait(bars.full(stage), phase, abort_flag, p)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = ring + stage * OC_ATOM;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t d = hi_d | (uint64_t)(((sa + kk * ks) >> 4) & 0x3FFFu);
            ptx::mma_bf16(tmem_base, d, d, idesc, accumulate);
            accumulate = 1;
          }
          issued = true;
          ptx::mma_commit(bars.empty(stage));
          if (++stage == OC_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::mma_commit(bars.acc(0));
        // G0 in buffer G
        if (!oc_wait(bars.epi_g(), n_g++ & 1u, abort_flag, p)) { ok = false; break; }
        for (int k = 0; ok && k < K; ++k) {
          const bool last = k == K - 1;
          ptx::tc_fence_after();
          issue_product(tmem_base + 128, buf_addr[BUF_G], buf_addr[BUF_G], pr.m);  // R: G G
          ptx::mma_commit(bars.acc(1));
          if (!oc_wait(bars.epi_r(), n_r++ & 1u, abort_flag, p)) { ok = false; break; }
          ptx::tc_fence_after();
          if (!last) {
            issue_product(tmem_base + 256, buf_addr[BUF_R], buf_addr[BUF_G], pr.m);  // T: R G
            ptx::mma_commit(bars.acc(2));
          }
          if (k >= 1) {
            issue_product(tmem_base + 384, buf_addr[BUF_R], buf_addr[BUF_P], pr.m);  // P': R P
            ptx::mma_commit(bars.acc(3));
          }
          if (!last) {
            if (!oc_wait(bars.epi_g(), n_g++ & 1u, abort_flag, p)) { ok = false; break; }  // T in buffer G
            ptx::tc_fence_after();
            issue_product(tmem_base, buf_addr[BUF_G], buf_addr[BUF_R], pr.m);  // G': T R
            ptx::mma_commit(bars.acc(0));
          }
          // P (read by the next step's P' MMAs) and G' (the next R) settle
          // before the next step issues
          if (k >= 1 && !oc_wait(bars.epi_p(), n_p++ & 1u, abort_flag, p)) { ok = false; break; }
          if (!last && !oc_wait(bars.epi_g(), n_g++ & 1u, abort_flag, p)) { ok = false; break; }
        }
      }
      if (!ok && issued) {
        ptx::mma_commit(bars.drain());
        const uint64_t t0 = ptx::globaltimer();
        while (!ptx::mbar_try_wait(bars.drain(), 0)) {
          if ((long long)(ptx::globaltimer() - t0) > p.timeout_ns) break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;              // the TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;    // its column slice (OC_SLICE columns)
    uint32_t acc_n[4] = {0, 0, 0, 0};
    const int ethr = threadIdx.x - 64;  // 0 .. 32 * OC_EPI_WARPS - 1
    bool ok = true;
    auto wait_acc = [&](int a) -> bool {
      int w = 1;
      if (lane == 0) w = oc_wait(bars.acc(a), acc_n[a] & 1u, abort_flag, p) ? 1 : 0;
      w = __shfl_sync(0xffffffffu, w, 0);
      ++acc_n[a];
      if (w) ptx::tc_fence_after();
      return w != 0;
    };
    for (int t = blockIdx.x; ok && t < p.total; t += gridDim.x) {
      const OnchipProblem& pr = p.prob[find_prob(p, t)];
      const int mat = t - pr.mat_begin;
      const int m = pr.m;
      __half* g_hi = pr.p_hi + mat * pr.mat_stride;
      __half* g_lo = pr.p_lo + mat * pr.mat_stride;
      const float s = p.inv[pr.inv_base + mat];
      // ---- G0 = s^2 X X^T
      if (!wait_acc(0)) break;
      if (m < ONCHIP_MAX_M) {
        // rows and columns >= m of every buffer must read as zero (a
        // previous matrix may have been larger, and buffers R and P held the
        // staging ring).  Only padding elements are cleared, so these stores
        // never meet the epilogues' stores of elements < m and need no
        // ordering with them; the barrier after this phase orders both
        // before the next MMAs.
        for (int cidx = ethr; cidx < 6 * 128 * 16; cidx += 32 * OC_EPI_WARPS) {
          const int part = cidx >> 11, i = (cidx >> 4) & 127, j0 = (cidx & 15) * 8;
          uint8_t* pb = smem + (part >> 1) * OC_BUF + (part & 1) * OC_PART;
          if (i >= m || j0 >= m) {
            *reinterpret_cast<uint4*>(pb + oc_off(i, j0)) = make_uint4(0u, 0u, 0u, 0u);
          } else if (j0 + 8 > m) {
            for (int j = m; j < j0 + 8; ++j) *reinterpret_cast<uint16_t*>(pb + oc_off(i, j)) = 0;
          }
        }
      }
      {
        float coef = 1.f;
        coef *= s * s;
        EpiArgs e{coef, 0.f, 0.f, -1, BUF_G, -1, nullptr, nullptr, 0};
        epilogue(smem, base, tmem_base, q, half, lane, m, e);
      }
      epi_done(bars.epi_g(), lane);
      for (int k = 0; k < K; ++k) {
        const bool last = k == K - 1;
        // ---- R = b G + c (G G); at k = 0 also P1 = a I + R
        if (!wait_acc(1)) { ok = false; break; }
        {
          EpiArgs e{p.c, p.b, p.a, BUF_G, BUF_R, k == 0 ? (last ? -2 : BUF_P) : -1, g_hi, g_lo, pr.ld};
          epilogue(smem, base, tmem_base + 128, q, half, lane, m, e);
        }
        epi_done(bars.epi_r(), lane);
        if (!last) {
          // ---- T = a G + R G, into buffer G
          if (!wait_acc(2)) { ok = false; break; }
          EpiArgs e{1.f, p.a, 0.f, BUF_G, BUF_G, -1, nullptr, nullptr, 0};
          epilogue(smem, base, tmem_base + 256, q, half, lane, m, e);
          epi_done(bars.epi_g(), lane);
        }
        if (k >= 1) {
          // ---- P' = a P + R P, in place (the last one to global)
          if (!wait_acc(3)) { ok = false; break; }
          EpiArgs e{1.f, p.a, 0.f, BUF_P, last ? -1 : BUF_P, -1, g_hi, g_lo, pr.ld};
          epilogue(smem, base, tmem_base + 384, q, half, lane, m, e);
          epi_done(bars.epi_p(), lane);
        }
        if (!last) {
          // ---- G' = a T + T R, in place
          if (!wait_acc(0)) { ok = false; break; }
          EpiArgs e{1.f, p.a, 0.f, BUF_G, BUF_G, -1, nullptr, nullptr, 0};
          epilogue(smem, base, tmem_base, q, half, lane, m, e);
          epi_done(bars.epi_g(), lane);
        }
      }
      if (!ok) break;
      // this matrix no longer needs buffers R and P: the producer may stage
      // the next matrix's image there
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bars.mat_done());
    }
  }

  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace

cudaError_t onchip_configure() {
  return cudaFuncSetAttribute(k_gram_onchip, cudaFuncAttributeMaxDynamicSharedMemorySize, OC_SMEM);
}

cudaError_t launch_gram_onchip(const OnchipParams& p, int num_sms, cudaStream_t s) {
  int grid = p.total < num_sms ? p.total : num_sms;
  if (grid <= 0) return cudaSuccess;
  k_gram_onchip<<<grid, OC_THREADS, OC_SMEM, s>>>(p);
  return cudaGetLastError();
}

}  // namespace dmu
