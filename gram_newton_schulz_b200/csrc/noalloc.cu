// dmu_momentum_norm_static: the momentum + Frobenius-norm pass for one
// matrix, for callers that must not allocate device memory.
//
// The plan-based path keeps its per-chunk partial sums in the workspace the
// caller allocates with cudaMalloc (through torch).  Some callers cannot do
// that: a host process whose device memory is owned by another framework's
// pool, which must see every byte it hands out; a plugin or embedded runtime
// that is forbidden to call the CUDA allocator; or a latency-critical loop in
// which cudaMalloc/cudaFree would synchronise the device.  This entry point
// keeps its only scratch -- one fp32 partial sum per 16384-element chunk -- in
// a file-scope __device__ array of fixed size, so the caller passes its
// inputs and outputs and nothing else is allocated.
//
// Every GPU that loads the library holds the 64 KB array until the process
// exits.  In host code the array's name is only a host-side stand-in, so its
// device address is looked up with cudaGetSymbolAddress on every call, with
// the caller's device current: the lookup allocates nothing, and a fresh
// lookup stays right when the device's context was reset and the module
// loaded again at another address.  The first call on a device may load the
// module, so it belongs before any stream capture.

#include "dmu_internal.h"

namespace dmu {
void set_last_error(const char* msg);
}

namespace {

constexpr int SCR_CHUNK = 16384;        // elements per partial sum
constexpr int SCR_MAX_CHUNKS = 16384;   // partial sums held by the static scratch
constexpr long long SCR_MAX_ELEMS = (long long)SCR_CHUNK * SCR_MAX_CHUNKS;  // 2^28 elements

// The scratch: written chunk by chunk before it is read in the same call, so
// it never needs clearing; calls that overlap on the GPU race on it.
static __device__ __align__(256) float g_scratch_partial[SCR_MAX_CHUNKS];

__device__ __forceinline__ void grad8(const void* g, int f32, long long idx, float* v) {
  if (f32) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(g) + idx);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(g) + idx);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 t = __bfloat1622float2(h[q]);
      v[2 * q] = t.x;
      v[2 * q + 1] = t.y;
    }
  }
}

// M <- beta M + G over one matrix of n elements; image = bf16 (or fp32) M;
// partial[c] = sum of M^2 over chunk c, reduced in a fixed order.
__global__ void __launch_bounds__(256) k_mom_static(const void* __restrict__ grad, int grad_f32,
                                                    float* __restrict__ mom, void* __restrict__ img,
                                                    long long n, float beta, float* __restrict__ partial,
                                                    int nchunks, int vec) {
  __shared__ float red[8];
  for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
    const long long start = (long long)c * SCR_CHUNK;
    const int len = (int)((n - start) < SCR_CHUNK ? (n - start) : SCR_CHUNK);
    float ss = 0.f;
    if (vec) {
      for (int e = threadIdx.x * 8; e < len; e += blockDim.x * 8) {
        const long long idx = start + e;
        float v[8];
        grad8(grad, grad_f32, idx, v);
        if (mom) {
          float4* pm = reinterpret_cast<float4*>(mom + idx);
          const float4 a = pm[0], b = pm[1];
          // M = round(beta M + G): one fused multiply-add, as in the plan path
          v[0] = __fmaf_rn(beta, a.x, v[0]); v[1] = __fmaf_rn(beta, a.y, v[1]);
          v[2] = __fmaf_rn(beta, a.z, v[2]); v[3] = __fmaf_rn(beta, a.w, v[3]);
          v[4] = __fmaf_rn(beta, b.x, v[4]); v[5] = __fmaf_rn(beta, b.y, v[5]);
          v[6] = __fmaf_rn(beta, b.z, v[6]); v[7] = __fmaf_rn(beta, b.w, v[7]);
          pm[0] = make_float4(v[0], v[1], v[2], v[3]);
          pm[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) ss += v[q] * v[q];
        if (img) {
          if (grad_f32) {
            float4* d = reinterpret_cast<float4*>(reinterpret_cast<float*>(img) + idx);
            d[0] = make_float4(v[0], v[1], v[2], v[3]);
            d[1] = make_float4(v[4], v[5], v[6], v[7]);
          } else {
            uint4 u;
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
            *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(img) + idx) = u;
          }
        }
      }
    } else {
      for (int e = threadIdx.x; e < len; e += blockDim.x) {
        const long long idx = start + e;
        float v = grad_f32 ? reinterpret_cast<const float*>(grad)[idx]
                           : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(grad)[idx]);
        if (mom) {
          v = __fmaf_rn(beta, mom[idx], v);
          mom[idx] = v;
        }
        ss += v * v;
        if (img) {
          if (grad_f32)
            reinterpret_cast<float*>(img)[idx] = v;
          else
            reinterpret_cast<__nv_bfloat16*>(img)[idx] = __float2bfloat16_rn(v);
        }
      }
    }
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

__global__ void k_norm_static(const float* __restrict__ partial, int nchunks, float eps, float* inv_out) {
  const int lane = threadIdx.x & 31;
  double s = 0.0;
  for (int c = lane; c < nchunks; c += 32) s += (double)partial[c];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) inv_out[0] = (float)(1.0 / (sqrt(s) + (double)eps));
}

// Device address of the static scratch in the current device's context
// (cudaGetSymbolAddress allocates nothing).
cudaError_t scratch_address(float** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch_partial);
  if (e != cudaSuccess) return e;
  *out = reinterpret_cast<float*>(p);
  return cudaSuccess;
}

}  // namespace

extern "C" DMU_API dmu_status dmu_momentum_norm_static(const void* grad, float* momentum, void* image_out,
                                                       int64_t rows, int64_t cols, dmu_dtype dtype, float beta,
                                                       float eps, float* inv_norm_out, void* stream) {
  dmu::set_last_error("");
  if (!grad || !inv_norm_out) {
    dmu::set_last_error("grad and inv_norm_out must be device pointers");
    return DMU_ERR_INVALID_ARG;
  }
  if (rows <= 0 || cols <= 0) {
    dmu::set_last_error("rows and cols must be positive");
    return DMU_ERR_INVALID_ARG;
  }
  if (dtype != DMU_BF16 && dtype != DMU_F32) {
    dmu::set_last_error("unknown dtype");
    return DMU_ERR_INVALID_ARG;
  }
  if (!(eps >= 0.f)) {
    dmu::set_last_error("eps must be >= 0");
    return DMU_ERR_INVALID_ARG;
  }
  const long long n = (long long)rows * (long long)cols;
  if (n > SCR_MAX_ELEMS) {
    dmu::set_last_error("matrix too large for the static scratch: at most 268435456 (2^28) elements");
    return DMU_ERR_UNSUPPORTED;
  }
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  float* scratch = nullptr;
  if (e == cudaSuccess) e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    dmu::set_last_error(cudaGetErrorString(e));
    return DMU_ERR_CUDA;
  }
  const int f32 = dtype == DMU_F32 ? 1 : 0;
  const int vec = (n % 8 == 0) && !(reinterpret_cast<uintptr_t>(grad) & 15) &&
                  !(reinterpret_cast<uintptr_t>(momentum) & 15) && !(reinterpret_cast<uintptr_t>(image_out) & 15);
  const int nchunks = (int)((n + SCR_CHUNK - 1) / SCR_CHUNK);
  int grid = sms * 8;
  if (grid > nchunks) grid = nchunks;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  k_mom_static<<<grid, 256, 0, s>>>(grad, f32, momentum, image_out, n, beta, scratch, nchunks, vec);
  k_norm_static<<<1, 32, 0, s>>>(scratch, nchunks, eps, inv_norm_out);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    dmu::set_last_error(cudaGetErrorString(e));
    return DMU_ERR_CUDA;
  }
  return DMU_OK;
}
