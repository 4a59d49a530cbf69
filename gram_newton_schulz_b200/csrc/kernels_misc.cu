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

// Vector path: each thread takes two 8-element vectors per iteration and
// issues every load (G, M) before any store, so two vectors' loads are in
// flight per thread; G, M and the image are distinct buffers (restrict).
__global__ void __launch_bounds__(256, 6) k_momentum(const MomChunk* __restrict__ chunks, int nchunks,
                                                  const MomMat* __restrict__ mats,
                                                  const void* const* __restrict__ grads,
                                                  float* const* __restrict__ momenta, int grad_f32,
                                                  void* __restrict__ mb, int mb_f32, float beta,
                                                  float* __restrict__ partial, int vec) {
  __shared__ float red[8];
  for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const MomChunk ch = chunks[c];
    const MomMat mm = mats[ch.slot];
    const void* __restrict__ g = grads[ch.slot];
    float* __restrict__ mom = momenta ? momenta[ch.slot] : nullptr;
    float ss = 0.f;
    if (vec) {
      const int stride = blockDim.x * 8;
      for (int e = threadIdx.x * 8; e < ch.len; e += 2 * stride) {
        const long long i0 = ch.start + e, i1 = i0 + stride;
        const bool has1 = e + stride < ch.len;
        float v0[8], v1[8];
        float4 m0a, m0b, m1a, m1b;
        load8_grad(g, grad_f32, i0, v0);
        if (has1) load8_grad(g, grad_f32, i1, v1);
        if (mom) {
          const float4* p0 = reinterpret_cast<const float4*>(mom + i0);
          m0a = p0[0];
          m0b = p0[1];
          if (has1) {
            const float4* p1 = reinterpret_cast<const float4*>(mom + i1);
            m1a = p1[0];
            m1b = p1[1];
          }
          v0[0] += beta * m0a.x; v0[1] += beta * m0a.y; v0[2] += beta * m0a.z; v0[3] += beta * m0a.w;
          v0[4] += beta * m0b.x; v0[5] += beta * m0b.y; v0[6] += beta * m0b.z; v0[7] += beta * m0b.w;
          float4* q0 = reinterpret_cast<float4*>(mom + i0);
          q0[0] = make_float4(v0[0], v0[1], v0[2], v0[3]);
          q0[1] = make_float4(v0[4], v0[5], v0[6], v0[7]);
          if (has1) {
            v1[0] += beta * m1a.x; v1[1] += beta * m1a.y; v1[2] += beta * m1a.z; v1[3] += beta * m1a.w;
            v1[4] += beta * m1b.x; v1[5] += beta * m1b.y; v1[6] += beta * m1b.z; v1[7] += beta * m1b.w;
            float4* q1 = reinterpret_cast<float4*>(mom + i1);
            q1[0] = make_float4(v1[0], v1[1], v1[2], v1[3]);
            q1[1] = make_float4(v1[4], v1[5], v1[6], v1[7]);
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) ss += v0[q] * v0[q];
        store8_image(mb, mb_f32, mm.mb_off + i0, v0);  // ldc == cols on the vector path
        if (has1) {
#pragma unroll
          for (int q = 0; q < 8; ++q) ss += v1[q] * v1[q];
          store8_image(mb, mb_f32, mm.mb_off + i1, v1);
        }
      }
    } else {
      for (int e = threadIdx.x; e < ch.len; e += blockDim.x) {
        const long long idx = ch.start + e;
        float v = grad_f32 ? reinterpret_cast<const float*>(g)[idx]
                           : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(g)[idx]);
        if (mom) {
          v += beta * mom[idx];
          mom[idx] = v;
        }
        ss += v * v;
        const long long row = idx / mm.cols, col = idx - row * mm.cols;
        const long long o = mm.mb_off + row * mm.ldc + col;
        if (mb_f32)
          reinterpret_cast<float*>(mb)[o] = v;
        else
          reinterpret_cast<__nv_bfloat16*>(mb)[o] = __float2bfloat16_rn(v);
      }
    }
    // block reduction in a fixed order
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
      float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      if (threadIdx.x == 0) partial[c] = t;
    }
    __syncthreads();
  }
}

__global__ void k_norm_finalize(const MomMat* __restrict__ mats, int nmats,
                                const float* __restrict__ partial, float eps, float* __restrict__ inv,
                                unsigned int* status) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= nmats) return;
  const MomMat mm = mats[warp];
  double s = 0.0;
  for (int c = mm.chunk_begin + lane; c < mm.chunk_end; c += 32) s += (double)partial[c];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    const double nrm = sqrt(s);
    if (!isfinite(s)) atomicOr(status, DMU_FLAG_NONFINITE);
    inv[warp] = (float)(1.0 / (nrm + (double)eps));
  }
}

cudaError_t launch_momentum(const MomChunk* chunks, int nchunks, const MomMat* mats,
                            const void* const* grads, float* const* momenta, int grad_f32, void* mb,
                            int mb_f32, float beta, float* partial, int vec_ok, int num_sms,
                            cudaStream_t s) {
  if (nchunks <= 0) return cudaSuccess;
  int grid = num_sms * 6;
  if (grid > nchunks) grid = nchunks;
  k_momentum<<<grid, 256, 0, s>>>(chunks, nchunks, mats, grads, momenta, grad_f32, mb, mb_f32, beta,
                                  partial, vec_ok);
  return cudaGetLastError();
}

cudaError_t launch_norm_finalize(const MomMat* mats, int nmats, const float* partial, float eps,
                                 float* inv, unsigned int* status, cudaStream_t s) {
  if (nmats <= 0) return cudaSuccess;
  const int threads = 256, per = threads / 32;
  k_norm_finalize<<<(nmats + per - 1) / per, threads, 0, s>>>(mats, nmats, partial, eps, inv, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------- helpers
__global__ void k_identity_bf16(__nv_bfloat16* hi, __nv_bfloat16* lo, int count, int m, long long ld,
                                long long mat_stride) {
  const long long total = (long long)count * m * m;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long mat = e / ((long long)m * m);
    const long long r = (e / m) % m, c = e % m;
    const long long o = mat * mat_stride + r * ld + c;
    hi[o] = __float2bfloat16_rn(r == c ? 1.f : 0.f);
    lo[o] = __float2bfloat16_rn(0.f);
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

cudaError_t launch_identity_bf16(__nv_bfloat16* hi, __nv_bfloat16* lo, int count, int m, long long ld,
                                 long long mat_stride, cudaStream_t s) {
  k_identity_bf16<<<grid_for((long long)count * m * m), 256, 0, s>>>(hi, lo, count, m, ld, mat_stride);
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
