// HBM-bound and fp32 kernels of the Muon update:
//   * k_momentum: M <- beta M + G (fp32, in place), the bf16 (or fp32)
//     image of M for the tensor-core path, and per-chunk partial sums of
//     M^2 (DMuon page, section 1: NS runs on the momentum-accumulated
//     gradient); 16-byte vector loads/stores, persistent grid;
//   * k_norm_finalize: fixed-order fp64 sum of the partials per matrix ->
//     1/(||M||_F + eps), deterministic; non-finite norms set a status bit;
//   * k_simt_gemm: the fp32 FFMA path (exact fp32 products) with the same
//     epilogues as the tensor-core kernel, used for fp32 plans;
//   * small helpers: identity P, hi/lo -> fp32 conversion for test hooks.
#include <cuda_fp16.h>

#include "dmu_internal.h"
#include "ptx.cuh"

namespace dmu {

// ------------------------------------------------------------- momentum
__device__ __forceinline__ void load8_grad(const void* g, int f32, long long idx, float* out) {
  if (f32) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(g) + idx);
    float4 a = __ldg(p), b = __ldg(p + 1);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  } else {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(g) + idx));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 t = __bfloat1622float2(h[q]);
      out[2 * q] = t.x;
      out[2 * q + 1] = t.y;
    }
  }
}

// fp16 image entries: 2^e v rounded to fp16 (sc = 2^e)
__device__ __forceinline__ void store8_image_h(void* __restrict__ mb, long long o, const float* v, float sc) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int q = 0; q < 4; ++q) h[q] = __floats2half2_rn(v[2 * q] * sc, v[2 * q + 1] * sc);
  __stcs(reinterpret_cast<uint4*>(reinterpret_cast<__half*>(mb) + o), u);
}

__device__ __forceinline__ void store8_image(void* __restrict__ mb, int mb_f32, long long o, const float* v) {
  if (mb_f32) {
    float4* d = reinterpret_cast<float4*>(reinterpret_cast<float*>(mb) + o);
    d[0] = make_float4(v[0], v[1], v[2], v[3]);
    d[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(mb) + o) = u;
  }
}

// M <- beta M + gscale G over one 16384-element chunk per CTA iteration.
// Each warp owns a fixed 2048-element slice of the chunk and writes its own
// partial sum of M^2 (partial[chunk * 8 + warp]), so no block-wide barrier
// stalls the stream at chunk ends, and the partials -- hence the norm --
// do not depend on the grid size.  Vector path: every thread issues the
// loads of four 8-element vectors (G, M; two for fp32 gradients) before any
// arithmetic or store.  G, M and the image are distinct buffers (restrict).
// bf16 plans on the vector path use k_momentum_bulk below, which computes
// the same values from shared memory.
constexpr int MOM_WARPS = 8;
constexpr int MOM_SLICE = MOM_CHUNK / MOM_WARPS;  // 2048 elements per warp
constexpr int MOM_VEC = 4;                        // vectors in flight per thread
static_assert(MOM_WARPS == MOM_PARTIALS_PER_CHUNK, "partial sums per chunk");

// Raw 8-element gradient vector: one 16-byte load (bf16) or two (fp32);
// converted to fp32 only when it is used, so the loads in flight hold 4
// (bf16) registers per vector.
template <bool F32> struct GradVec;
template <> struct GradVec<false> {
  uint4 u;
  __device__ __forceinline__ void load(const void* g, long long idx) {
    // streamed once: evict-first, so the pass does not churn L2
    u = __ldcs(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(g) + idx));
  }
  __device__ __forceinline__ void get(float* out) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 t = __bfloat1622float2(h[q]);
      out[2 * q] = t.x;
      out[2 * q + 1] = t.y;
    }
  }
};
template <> struct GradVec<true> {
  float4 a, b;
  __device__ __forceinline__ void load(const void* g, long long idx) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(g) + idx);
    a = __ldg(p);
    b = __ldg(p + 1);
  }
  __device__ __forceinline__ void get(float* out) const {
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  }
};

// Image: fp32 plans write M itself; bf16 plans write fp16(2^e M) with the
// scale 2^e the previous call chose for this matrix (iscale), or nothing
// when there is none yet -- k_norm_finalize then flags the matrix and
// k_image_fix writes its image.
template <bool F32>
__global__ void __launch_bounds__(256, 3) k_momentum(const MomChunk* __restrict__ chunks, int nchunks,
                                                  const MomMat* __restrict__ mats,
                                                  const void* const* __restrict__ grads,
                                                  float* const* __restrict__ momenta,
                                                  void* __restrict__ mb, float beta, float gscale,
                                                  const float* __restrict__ iscale, int* __restrict__ fix_count,
                                                  float* __restrict__ partial, int vec) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // k_norm_finalize counts the matrices whose image needs rewriting; the
  // previous call's fix-up pass has finished reading the count (stream order)
  if (fix_count && blockIdx.x == 0 && threadIdx.x == 0) *fix_count = 0;
  // a chunk's descriptor and its matrix's pointers form a chain of dependent
  // loads: the next chunk's are fetched while this chunk streams
  struct Meta {
    MomChunk ch;
    long long mb_off;
    float sc;
    const void* g;
    float* mom;
  };
  auto fetch = [&](int c) {
    Meta m;
    m.ch = chunks[c];
    m.mb_off = mats[m.ch.slot].mb_off;
    m.sc = F32 ? 1.f : iscale[m.ch.slot];
    m.g = grads[m.ch.slot];
    m.mom = momenta ? momenta[m.ch.slot] : nullptr;
    return m;
  };
  Meta next = blockIdx.x < nchunks ? fetch(blockIdx.x) : Meta{};
  for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const Meta cur = next;
    if (c + (int)gridDim.x < nchunks) next = fetch(c + gridDim.x);
    const MomChunk ch = cur.ch;
    const long long mb_off = cur.mb_off;
    const float sc = cur.sc;
    const void* __restrict__ g = cur.g;
    float* __restrict__ mom = cur.mom;
    const int s0 = warp * MOM_SLICE;
    const int s1 = min(ch.len, s0 + MOM_SLICE);
    float ss = 0.f;
    // fp32 gradients hold twice the registers per vector in flight
    constexpr int VEC = F32 ? MOM_VEC / 2 : MOM_VEC;
    if (vec) {
      for (int e = s0 + lane * 8; e < s1; e += 32 * 8 * VEC) {
        GradVec<F32> gv[VEC];
        float4 ma[VEC], mc[VEC];
#pragma unroll
        for (int u = 0; u < VEC; ++u) {
          const int eu = e + u * 256;
          if (eu < s1) {
            gv[u].load(g, ch.start + eu);
            if (mom) {
              const float4* pm = reinterpret_cast<const float4*>(mom + ch.start + eu);
              ma[u] = __ldcs(pm);
              mc[u] = __ldcs(pm + 1);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < VEC; ++u) {
          const int eu = e + u * 256;
          if (eu < s1) {
            const long long i0 = ch.start + eu;
            float v[8];
            gv[u].get(v);
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = __fmul_rn(v[q], gscale);
            if (mom) {  // M = round(beta M + round(s G)), no other contraction
              v[0] = __fmaf_rn(beta, ma[u].x, v[0]); v[1] = __fmaf_rn(beta, ma[u].y, v[1]);
              v[2] = __fmaf_rn(beta, ma[u].z, v[2]); v[3] = __fmaf_rn(beta, ma[u].w, v[3]);
              v[4] = __fmaf_rn(beta, mc[u].x, v[4]); v[5] = __fmaf_rn(beta, mc[u].y, v[5]);
              v[6] = __fmaf_rn(beta, mc[u].z, v[6]); v[7] = __fmaf_rn(beta, mc[u].w, v[7]);
              float4* q0 = reinterpret_cast<float4*>(mom + i0);
              __stcs(q0, make_float4(v[0], v[1], v[2], v[3]));
              __stcs(q0 + 1, make_float4(v[4], v[5], v[6], v[7]));
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) ss = __fmaf_rn(v[q], v[q], ss);
            if (F32)
              store8_image(mb, 1, mb_off + i0, v);  // ldc == cols on the vector path
            else if (sc > 0.f)
              store8_image_h(mb, mb_off + i0, v, sc);
          }
        }
      }
    } else {
      const MomMat mm = mats[ch.slot];
      for (int e = s0 + lane; e < s1; e += 32) {
        const long long idx = ch.start + e;
        float v = F32 ? reinterpret_cast<const float*>(g)[idx]
                      : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(g)[idx]);
        v = __fmul_rn(v, gscale);
        if (mom) {
          v = __fmaf_rn(beta, mom[idx], v);
          mom[idx] = v;
        }
        ss = __fmaf_rn(v, v, ss);
        const long long row = idx / mm.cols, col = idx - row * mm.cols;
        const long long o = mm.mb_off + row * mm.ldc + col;
        if (F32)
          reinterpret_cast<float*>(mb)[o] = v;
        else if (sc > 0.f)
          reinterpret_cast<__half*>(mb)[o] = __float2half_rn(v * sc);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) partial[(long long)c * MOM_WARPS + warp] = ss;
  }
}

// Momentum pass of bf16 plans on the vector path, fed by bulk copies
// (cp.async.bulk): one producer thread streams each chunk's G and M into
// shared memory MB_STAGES chunks ahead, so the bytes in flight are bounded
// by shared memory (192 KB per SM) rather than by registers.  The eight
// consumer warps take the same elements, arithmetic and partial sums as
// k_momentum (bitwise-equal M, image and partials) from shared memory and
// write M and the fp16 image with 16-byte streaming stores.  Every wait is
// bounded; on expiry the CTA sets DMU_FLAG_TIMEOUT and winds down.
constexpr int MB_STAGES = 2;
constexpr int MB_G = MOM_CHUNK * 2;  // bf16 G of one chunk
constexpr int MB_M = MOM_CHUNK * 4;  // fp32 M of one chunk
constexpr int MB_STAGE = MB_G + MB_M;
constexpr int MB_THREADS = 32 * (MOM_WARPS + 1);
constexpr int MB_SMEM = MB_STAGES * MB_STAGE + 16 * MB_STAGES;
static_assert(MB_SMEM <= 232448, "shared memory per CTA");

__device__ __forceinline__ bool mb_wait(uint32_t bar, uint32_t parity, long long timeout_ns, unsigned int* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if ((long long)(ptx::globaltimer() - t0) > timeout_ns) {
      atomicOr(status, DMU_FLAG_TIMEOUT);
      return false;
    }
  }
  return true;
}

__global__ void __launch_bounds__(MB_THREADS, 1)
    k_momentum_bulk(const MomChunk* __restrict__ chunks, int nchunks, const MomMat* __restrict__ mats,
                    const void* const* __restrict__ grads, float* const* __restrict__ momenta, void* __restrict__ mb,
                    float beta, float gscale, const float* __restrict__ iscale, int* __restrict__ fix_count,
                    float* __restrict__ partial, long long timeout_ns, unsigned int* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bars = sbase + MB_STAGES * MB_STAGE;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (MB_STAGES + s); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // k_norm_finalize counts the matrices whose image needs rewriting; the
  // previous call's fix-up pass has finished reading the count (stream order)
  if (fix_count && blockIdx.x == 0 && threadIdx.x == 0) *fix_count = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < MB_STAGES; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), MOM_WARPS);
    }
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == MOM_WARPS) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, par = 0;
      for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
        if (!mb_wait(empty(stage), phase ^ 1u, timeout_ns, status)) break;
        const MomChunk ch = chunks[c];
        const float* mom = momenta ? momenta[ch.slot] : nullptr;
        const uint32_t gbytes = (uint32_t)ch.len * 2u, mbytes = mom ? (uint32_t)ch.len * 4u : 0u;
        ptx::mbar_arrive_expect_tx(full(stage), gbytes + mbytes);
        ptx::bulk_g2s(sbase + stage * MB_STAGE,
                      reinterpret_cast<const __nv_bfloat16*>(grads[ch.slot]) + ch.start, gbytes, full(stage));
        if (mom) ptx::bulk_g2s(sbase + stage * MB_STAGE + MB_G, mom + ch.start, mbytes, full(stage));
        issued |= 1u << stage;
        par = (par & ~(1u << stage)) | (phase << stage);
        if (++stage == MB_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // every issued copy has landed before the CTA exits
      for (int s = 0; s < MB_STAGES; ++s)
        if (issued & (1u << s)) mb_wait(full(s), (par >> s) & 1u, timeout_ns, status);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  int stage = 0;
  uint32_t phase = 0;
  for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const MomChunk ch = chunks[c];
    const long long mb_off = mats[ch.slot].mb_off;
    const float sc = iscale[ch.slot];
    float* __restrict__ mom = momenta ? momenta[ch.slot] : nullptr;
    int ok = 1;
    if (lane == 0) ok = mb_wait(full(stage), phase, timeout_ns, status) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    const uint8_t* sg = smem + stage * MB_STAGE;
    const float* sm = reinterpret_cast<const float*>(smem + stage * MB_STAGE + MB_G);
    const int s0 = warp * MOM_SLICE;
    const int s1 = min(ch.len, s0 + MOM_SLICE);
    float ss = 0.f;
    for (int e = s0 + lane * 8; e < s1; e += 256) {
      const uint4 u = *reinterpret_cast<const uint4*>(sg + 2 * e);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
      float v[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 t = __bfloat1622float2(h[q]);
        v[2 * q] = t.x;
        v[2 * q + 1] = t.y;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = __fmul_rn(v[q], gscale);
      const long long i0 = ch.start + e;
      if (mom) {  // M = round(beta M + round(s G)), no other contraction
        const float4 a = *reinterpret_cast<const float4*>(sm + e);
        const float4 b = *reinterpret_cast<const float4*>(sm + e + 4);
        v[0] = __fmaf_rn(beta, a.x, v[0]); v[1] = __fmaf_rn(beta, a.y, v[1]);
        v[2] = __fmaf_rn(beta, a.z, v[2]); v[3] = __fmaf_rn(beta, a.w, v[3]);
        v[4] = __fmaf_rn(beta, b.x, v[4]); v[5] = __fmaf_rn(beta, b.y, v[5]);
        v[6] = __fmaf_rn(beta, b.z, v[6]); v[7] = __fmaf_rn(beta, b.w, v[7]);
        float4* q0 = reinterpret_cast<float4*>(mom + i0);
        __stcs(q0, make_float4(v[0], v[1], v[2], v[3]));
        __stcs(q0 + 1, make_float4(v[4], v[5], v[6], v[7]));
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) ss = __fmaf_rn(v[q], v[q], ss);
      if (sc > 0.f) store8_image_h(mb, mb_off + i0, v, sc);  // ldc == cols on the vector path
    }
    // this warp is done with the stage: the producer may refill it
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(empty(stage));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) partial[(long long)c * MOM_WARPS + warp] = ss;
    if (++stage == MB_STAGES) {
      stage = 0;
      phase ^= 1u;
    }
  }
}

// bf16 plans also keep the power-of-two scale 2^e of each matrix's fp16
// image (iscale): the previous call's scale stays while 2^e ||M||_F lies in
// (2^9, 2^15] -- every entry of 2^e M is then below fp16's largest finite
// value, and entries down to ||M||_F 2^-23 stay in fp16's normal range --
// so a steady run writes the image in the momentum pass alone.  Otherwise
// (first call, or the norm moved 8x) a new scale with 2^e ||M||_F in
// (2^11, 2^12] is chosen and the matrix is flagged for k_image_fix.
// inv_img = inv 2^-e reads the image back as X0.
__global__ void k_norm_finalize(const MomMat* __restrict__ mats, int nmats,
                                const float* __restrict__ partial, float eps, float* __restrict__ inv,
                                float* __restrict__ iscale, float* __restrict__ inv_img, int* __restrict__ fix,
                                int* __restrict__ fix_count, unsigned int* status) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= nmats) return;
  const MomMat mm = mats[warp];
  double s = 0.0;
  for (long long c = (long long)mm.chunk_begin * MOM_WARPS + lane; c < (long long)mm.chunk_end * MOM_WARPS; c += 32)
    s += (double)partial[c];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    const double nrm = sqrt(s);
    if (!isfinite(s)) atomicOr(status, DMU_FLAG_NONFINITE);
    const float iv = (float)(1.0 / (nrm + (double)eps));
    inv[warp] = iv;
    if (iscale) {
      const float prev = iscale[warp];
      const double scaled = (double)prev * nrm;
      const bool keep = prev > 0.f && isfinite(nrm) && scaled > 512.0 && scaled <= 32768.0;
      float sc = prev;
      if (!keep) {
        int e = 0;
        if (nrm > 0.0 && isfinite(nrm)) e = 12 - (int)ceil(log2(nrm));
        e = max(-100, min(100, e));
        sc = ldexpf(1.f, e);
        iscale[warp] = sc;
      }
      fix[warp] = keep ? 0 : 1;
      if (!keep) atomicAdd(fix_count, 1);
      inv_img[warp] = iv / sc;  // exact: sc is a power of two
    }
  }
}

// The fp16 image 2^e M of the matrices k_norm_finalize flagged, recomputed
// from their source: M as the momentum pass left it, or, without momentum
// state, gscale * G exactly as the momentum pass formed it.  When no matrix
// is flagged (a steady run) every CTA returns after one load; otherwise
// chunks of matrices that keep their scale are skipped.
__global__ void __launch_bounds__(256) k_image_fix(const MomChunk* __restrict__ chunks, int nchunks,
                                                   const MomMat* __restrict__ mats,
                                                   const void* const* __restrict__ grads,
                                                   float* const* __restrict__ momenta, float gscale,
                                                   void* __restrict__ mb, const float* __restrict__ iscale,
                                                   const int* __restrict__ fix, const int* __restrict__ fix_count,
                                                   int vec) {
  if (*fix_count == 0) return;
  for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const MomChunk ch = chunks[c];
    if (!fix[ch.slot]) continue;
    const MomMat mm = mats[ch.slot];
    const float sc = iscale[ch.slot];
    const __nv_bfloat16* g = reinterpret_cast<const __nv_bfloat16*>(grads[ch.slot]);
    const float* mom = momenta ? momenta[ch.slot] : nullptr;
    if (vec) {
      for (int e = threadIdx.x * 8; e < ch.len; e += blockDim.x * 8) {
        const long long i0 = ch.start + e;
        float v[8];
        if (mom) {
          const float4* pm = reinterpret_cast<const float4*>(mom + i0);
          const float4 a = pm[0], b = pm[1];
          v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
          v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        } else {
          GradVec<false> gv;
          gv.load(g, i0);
          gv.get(v);
#pragma unroll
          for (int q = 0; q < 8; ++q) v[q] = __fmul_rn(v[q], gscale);
        }
        store8_image_h(mb, mm.mb_off + i0, v, sc);  // ldc == cols on the vector path
      }
    } else {
      for (int e = threadIdx.x; e < ch.len; e += blockDim.x) {
        const long long idx = ch.start + e;
        const float v = mom ? mom[idx] : __fmul_rn(__bfloat162float(g[idx]), gscale);
        const long long row = idx / mm.cols, col = idx - row * mm.cols;
        reinterpret_cast<__half*>(mb)[mm.mb_off + row * mm.ldc + col] = __float2half_rn(v * sc);
      }
    }
  }
}

cudaError_t launch_image_fix(const MomChunk* chunks, int nchunks, const MomMat* mats, const void* const* grads,
                             float* const* momenta, float gscale, void* mb, const float* iscale, const int* fix,
                             const int* fix_count, int vec_ok, int num_sms, cudaStream_t s) {
  if (nchunks <= 0) return cudaSuccess;
  int grid = num_sms * 8;
  if (grid > nchunks) grid = nchunks;
  k_image_fix<<<grid, 256, 0, s>>>(chunks, nchunks, mats, grads, momenta, gscale, mb, iscale, fix, fix_count,
                                   vec_ok);
  return cudaGetLastError();
}

cudaError_t momentum_configure() {
  return cudaFuncSetAttribute(k_momentum_bulk, cudaFuncAttributeMaxDynamicSharedMemorySize, MB_SMEM);
}

cudaError_t launch_momentum(const MomChunk* chunks, int nchunks, const MomMat* mats,
                            const void* const* grads, float* const* momenta, int grad_f32, void* mb,
                            int mb_f32, float beta, float gscale, const float* iscale, int* fix_count,
                            float* partial, int vec_ok, int num_sms, long long timeout_ns, unsigned int* status,
                            cudaStream_t s) {
  if (nchunks <= 0) return cudaSuccess;
  if (!grad_f32 && !mb_f32 && vec_ok) {
    const int grid = nchunks < num_sms ? nchunks : num_sms;
    k_momentum_bulk<<<grid, MB_THREADS, MB_SMEM, s>>>(chunks, nchunks, mats, grads, momenta, mb, beta, gscale,
                                                       iscale, fix_count, partial, timeout_ns, status);
    return cudaGetLastError();
  }
  int grid = num_sms * 3;  // the resident CTAs per SM of the launch bounds
  if (grid > nchunks) grid = nchunks;
  // the image has the gradients' element type for fp32 plans (fp32 -> fp32);
  // bf16 plans write fp16 at the kept scale
  if (grad_f32 != mb_f32) return cudaErrorInvalidValue;
  if (grad_f32)
    k_momentum<true><<<grid, 256, 0, s>>>(chunks, nchunks, mats, grads, momenta, mb, beta, gscale, nullptr, nullptr,
                                          partial, vec_ok);
  else
    k_momentum<false><<<grid, 256, 0, s>>>(chunks, nchunks, mats, grads, momenta, mb, beta, gscale, iscale,
                                           fix_count, partial, vec_ok);
  return cudaGetLastError();
}

cudaError_t launch_norm_finalize(const MomMat* mats, int nmats, const float* partial, float eps,
                                 float* inv, float* iscale, float* inv_img, int* fix, int* fix_count,
                                 unsigned int* status, cudaStream_t s) {
  if (nmats <= 0) return cudaSuccess;
  const int threads = 256, per = threads / 32;
  k_norm_finalize<<<(nmats + per - 1) / per, threads, 0, s>>>(mats, nmats, partial, eps, inv, iscale, inv_img,
                                                             fix, fix_count, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------- helpers
// Identity as a 16-bit hi/lo pair; `one` is the bit pattern of 1.0 in the
// pair's format (0x3F80 bf16, 0x3C00 fp16).
// One block per row (grid-stride over the count * m rows), so a thread's
// index arithmetic is a 32-bit division per row rather than 64-bit
// divisions per element.
__global__ void k_identity16(uint16_t* hi, uint16_t* lo, int count, int m, long long ld, long long mat_stride,
                             uint16_t one) {
  const int rows = count * m;
  for (int row = blockIdx.x; row < rows; row += gridDim.x) {
    const int mat = row / m, r = row - mat * m;
    const long long o = (long long)mat * mat_stride + (long long)r * ld;
    for (int c = threadIdx.x; c < m; c += blockDim.x) {
      hi[o + c] = c == r ? one : (uint16_t)0;
      lo[o + c] = 0;
    }
  }
}

__global__ void k_identity_f32(float* p, int count, int m, long long ld, long long mat_stride) {
  const long long total = (long long)count * m * m;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long mat = e / ((long long)m * m);
    const long long r = (e / m) % m, c = e % m;
    p[mat * mat_stride + r * ld + c] = (r == c) ? 1.f : 0.f;
  }
}

__device__ __forceinline__ long long half_offset(long long r, long long c, long long ld, int half) {
  if (half && (r / HALF_BLOCK) > (c / HALF_BLOCK)) return c * ld + r;
  return r * ld + c;
}

__global__ void k_pair_to_f32(const __nv_bfloat16* hi, const __nv_bfloat16* lo, long long rows,
                              long long cols, long long ld, float* out, int half) {
  const long long total = rows * cols;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / cols, c = e % cols;
    const long long o = half_offset(r, c, ld, half);
    float v = __bfloat162float(hi[o]);
    if (lo) v += __bfloat162float(lo[o]);
    out[e] = v;
  }
}

__global__ void k_pair_h_to_f32(const __half* hi, const __half* lo, long long rows, long long cols,
                                long long ld, float scale, float* out, int half) {
  const long long total = rows * cols;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / cols, c = e % cols;
    const long long o = half_offset(r, c, ld, half);
    out[e] = (__half2float(hi[o]) + (lo ? __half2float(lo[o]) : 0.f)) * scale;
  }
}

__global__ void k_f32_copy2d(const float* src, long long rows, long long cols, long long ld, float* out) {
  const long long total = rows * cols;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / cols, c = e % cols;
    out[e] = src[r * ld + c];
  }
}

static int grid_for(long long total) {
  long long g = (total + 255) / 256;
  if (g > 4096) g = 4096;
  if (g < 1) g = 1;
  return (int)g;
}

cudaError_t launch_identity16(void* hi, void* lo, int count, int m, long long ld, long long mat_stride, int f16,
                              cudaStream_t s) {
  if ((long long)count * m > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int rows = count * m;
  if (rows <= 0) return cudaSuccess;
  k_identity16<<<rows < 8192 ? rows : 8192, 256, 0, s>>>(
      reinterpret_cast<uint16_t*>(hi), reinterpret_cast<uint16_t*>(lo), count, m, ld, mat_stride,
      f16 ? (uint16_t)0x3C00 : (uint16_t)0x3F80);
  return cudaGetLastError();
}
cudaError_t launch_identity_f32(float* p, int count, int m, long long ld, long long mat_stride,
                                cudaStream_t s) {
  k_identity_f32<<<grid_for((long long)count * m * m), 256, 0, s>>>(p, count, m, ld, mat_stride);
  return cudaGetLastError();
}
cudaError_t launch_pair_to_f32(const __nv_bfloat16* hi, const __nv_bfloat16* lo, long long rows,
                               long long cols, long long ld, float* out, cudaStream_t s, int half) {
  k_pair_to_f32<<<grid_for(rows * cols), 256, 0, s>>>(hi, lo, rows, cols, ld, out, half);
  return cudaGetLastError();
}
cudaError_t launch_pair_h_to_f32(const void* hi, const void* lo, long long rows, long long cols, long long ld,
                                 float scale, float* out, cudaStream_t s, int half) {
  k_pair_h_to_f32<<<grid_for(rows * cols), 256, 0, s>>>(reinterpret_cast<const __half*>(hi),
                                                        reinterpret_cast<const __half*>(lo), rows, cols, ld, scale,
                                                        out, half);
  return cudaGetLastError();
}
cudaError_t launch_f32_copy2d(const float* src, long long rows, long long cols, long long ld, float* out,
                              cudaStream_t s) {
  k_f32_copy2d<<<grid_for(rows * cols), 256, 0, s>>>(src, rows, cols, ld, out);
  return cudaGetLastError();
}

// ------------------------------------------------------------- fp32 path
// 64 x 64 output tile per block, 256 threads, 4 x 4 outputs per thread,
// K slabs of 16 through shared memory; exact fp32 FFMA.
constexpr int ST = 64, SK = 16;

__global__ void __launch_bounds__(256) k_simt_gemm(const SimtProblem p) {
  const int tiles_m = (p.M + ST - 1) / ST;
  const int bi = blockIdx.x % tiles_m, bj = blockIdx.x / tiles_m;
  const int mat = blockIdx.y;
  if (p.sym && bi > bj) return;
  __shared__ float As[SK][ST + 4];
  __shared__ float Bs[SK][ST + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* A = p.a + (long long)mat * p.a_ms;
  const float* B = p.b + (long long)mat * p.b_ms;
  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
  for (int k0 = 0; k0 < p.K; k0 += SK) {
    for (int e = threadIdx.x; e < ST * SK; e += 256) {
      int kk, ii;
      if (p.a_sk == 1) { kk = e % SK; ii = e / SK; } else { ii = e % ST; kk = e / ST; }
      const int gi = bi * ST + ii, gk = k0 + kk;
      As[kk][ii] = (gi < p.M && gk < p.K) ? A[(long long)gi * p.a_si + (long long)gk * p.a_sk] : 0.f;
      int kb, jj;
      if (p.b_sk == 1) { kb = e % SK; jj = e / SK; } else { jj = e % ST; kb = e / ST; }
      const int gj = bj * ST + jj, gk2 = k0 + kb;
      Bs[kb][jj] = (gj < p.N && gk2 < p.K) ? B[(long long)gj * p.b_si + (long long)gk2 * p.b_sk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = As[kk][ty * 4 + r];
#pragma unroll
      for (int c = 0; c < 4; ++c) b[c] = Bs[kk][tx * 4 + c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
    __syncthreads();
  }
  float coef = p.alpha;
  float s = 1.f;
  if (p.alpha_mode != ALPHA_CONST) s = p.inv[p.inv_base + mat];
  if (p.alpha_mode == ALPHA_INV2) coef *= s * s;
  if (p.alpha_mode == ALPHA_INV) coef *= s;
  const long long mb = (long long)mat * p.mat_stride;
  void* wp = (p.epi == EPI_UPDATE && p.w_ptrs) ? p.w_ptrs[p.ptr_base + mat] : nullptr;
  float* op = (p.epi == EPI_UPDATE && p.o_ptrs) ? p.o_ptrs[p.ptr_base + mat] : nullptr;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = bi * ST + ty * 4 + r;
    if (i >= p.M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = bj * ST + tx * 4 + c;
      if (j >= p.N) continue;
      if (p.epi == EPI_GRAM) {
        if (p.sym && i > j) continue;
        float v = coef * acc[r][c];
        if (p.cin) v += p.beta * p.cin[mb + (long long)i * p.ld + j];
        if (i == j) v += p.gamma;
        p.out[mb + (long long)i * p.ld + j] = v;
        if (p.sym && i < j) p.out[mb + (long long)j * p.ld + i] = v;
        if (p.out2) {
          const float v2 = v + (i == j ? p.gamma2 : 0.f);
          p.out2[mb + (long long)i * p.ld + j] = v2;
          if (p.sym && i < j) p.out2[mb + (long long)j * p.ld + i] = v2;
        }
      } else {
        const float o = acc[r][c];
        const long long off = p.w_transposed ? (long long)j * p.w_cols + i : (long long)i * p.w_cols + j;
        if (wp) {
          if (p.w_f32) {
            reinterpret_cast<float*>(wp)[off] += p.alpha * s * o;
          } else {
            __nv_bfloat16* w = reinterpret_cast<__nv_bfloat16*>(wp);
            w[off] = __float2bfloat16_rn(__bfloat162float(w[off]) + p.alpha * s * o);
          }
        }
        if (op) op[off] = s * o;
      }
    }
  }
}

cudaError_t launch_simt_gemm(const SimtProblem& p, cudaStream_t s) {
  const int tiles = ((p.M + ST - 1) / ST) * ((p.N + ST - 1) / ST);
  if (tiles <= 0 || p.count <= 0) return cudaSuccess;
  dim3 grid(tiles, p.count);
  k_simt_gemm<<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace dmu
