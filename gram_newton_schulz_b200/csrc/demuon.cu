// DeMuon: the elementwise steps of decentralised Muon over a communication
// graph of N agents (DeMuon technical summary, "Methodology", 1. DeMuon).
//
// Each agent i holds three sequences per weight matrix: a local momentum
// estimate M_i, a tracked global-gradient estimate V_i and its iterate X_i.
// One iteration with mixing weights w_ij (row i = what agent i receives):
//
//   M_i' = (1 - theta) M_i + theta G_i                  (local momentum, EMA)
//   V_i' = sum_j w_ij V_j + M_i' - M_i                  (gradient tracking)
//   O_j  = msgn(V_j')                                   (Gram Newton-Schulz)
//   X_i' = sum_j w_ij (X_j - eta O_j)                   (mix neighbours' updates)
//
// The page names the three sequences and the three operations, and says
// msgn is applied to the tracked gradient; the exact recursions above are
// the plain gradient-tracking reading.  msgn runs through the batched Gram
// Newton-Schulz path of the plan (one plan over all agents' matrices); the
// two kernels here are the momentum/tracking update and the gossip mixing.
//
// Layout: every agent's state for all its matrices is one flat array of
// `numel` elements (the caller places the matrices in it); the kernels treat
// it as a vector.  Both kernels are HBM-bound: per element and agent, track
// reads G (2 B), M (4 B) and V (4 B) and writes M, V (4 B each) and the bf16
// msgn input (2 B); mix reads X and O (4 B each) and writes X (4 B).  A
// thread handles 4 consecutive elements for every agent, so each agent's V
// (or X - eta O) is read once and feeds all N outputs from registers.
#include <cmath>

#include "dmu_internal.h"

namespace dmu {
void set_last_error(const char* msg);

constexpr int DEMUON_MAX = DMU_DEMUON_MAX_AGENTS;

struct DemuonTrack {
  int n;
  long long numel;
  float theta;
  float mix[DEMUON_MAX][DEMUON_MAX];
  const __nv_bfloat16* g[DEMUON_MAX];
  float* m[DEMUON_MAX];
  const float* v_in[DEMUON_MAX];
  float* v_out[DEMUON_MAX];
  __nv_bfloat16* vb[DEMUON_MAX];
};

struct DemuonMix {
  int n;
  long long numel;
  float eta;
  float mix[DEMUON_MAX][DEMUON_MAX];
  const float* x_in[DEMUON_MAX];
  const float* o[DEMUON_MAX];
  float* x_out[DEMUON_MAX];
};

__device__ __forceinline__ float4 ld4(const float* p, long long e) {
  return *reinterpret_cast<const float4*>(p + e);
}
__device__ __forceinline__ void st4(float* p, long long e, float4 v) { *reinterpret_cast<float4*>(p + e) = v; }

// Weighted sum over agents j = 0..n-1 in that order (fixed, so deterministic).
__device__ __forceinline__ float4 mix_row(const float (&w)[DEMUON_MAX], const float4 (&v)[DEMUON_MAX], int n) {
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < DEMUON_MAX; ++j) {
    if (j < n) {
      s.x = fmaf(w[j], v[j].x, s.x);
      s.y = fmaf(w[j], v[j].y, s.y);
      s.z = fmaf(w[j], v[j].z, s.z);
      s.w = fmaf(w[j], v[j].w, s.w);
    }
  }
  return s;
}

__global__ void __launch_bounds__(256) k_demuon_track(const __grid_constant__ DemuonTrack a) {
  const long long n4 = a.numel / 4;
  const float keep = 1.f - a.theta;
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < n4;
       q += (long long)gridDim.x * blockDim.x) {
    const long long e = 4 * q;
    float4 v[DEMUON_MAX];
#pragma unroll
    for (int j = 0; j < DEMUON_MAX; ++j)
      if (j < a.n) v[j] = ld4(a.v_in[j], e);
#pragma unroll
    for (int i = 0; i < DEMUON_MAX; ++i) {
      if (i >= a.n) break;
      const float4 mo = ld4(a.m[i], e);
      const uint2 gu = *reinterpret_cast<const uint2*>(a.g[i] + e);
      const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gu.x));
      const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gu.y));
      const float4 mn = make_float4(fmaf(a.theta, g01.x, keep * mo.x), fmaf(a.theta, g01.y, keep * mo.y),
                                    fmaf(a.theta, g23.x, keep * mo.z), fmaf(a.theta, g23.y, keep * mo.w));
      const float4 s = mix_row(a.mix[i], v, a.n);
      const float4 vn = make_float4(s.x + (mn.x - mo.x), s.y + (mn.y - mo.y), s.z + (mn.z - mo.z),
                                    s.w + (mn.w - mo.w));
      st4(a.m[i], e, mn);
      st4(a.v_out[i], e, vn);
      __nv_bfloat162 b01 = __floats2bfloat162_rn(vn.x, vn.y), b23 = __floats2bfloat162_rn(vn.z, vn.w);
      uint2 bu;
      bu.x = *reinterpret_cast<uint32_t*>(&b01);
      bu.y = *reinterpret_cast<uint32_t*>(&b23);
      *reinterpret_cast<uint2*>(a.vb[i] + e) = bu;
    }
  }
  // ragged tail (numel % 4 elements): one thread, scalar
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (long long e = 4 * n4; e < a.numel; ++e) {
      float mo[DEMUON_MAX], vj[DEMUON_MAX];
      for (int j = 0; j < a.n; ++j) vj[j] = a.v_in[j][e];
      for (int i = 0; i < a.n; ++i) mo[i] = a.m[i][e];
      for (int i = 0; i < a.n; ++i) {
        const float mn = fmaf(a.theta, __bfloat162float(a.g[i][e]), keep * mo[i]);
        float s = 0.f;
        for (int j = 0; j < a.n; ++j) s = fmaf(a.mix[i][j], vj[j], s);
        const float vn = s + (mn - mo[i]);
        a.m[i][e] = mn;
        a.v_out[i][e] = vn;
        a.vb[i][e] = __float2bfloat16_rn(vn);
      }
    }
  }
}

__global__ void __launch_bounds__(256) k_demuon_mix(const __grid_constant__ DemuonMix a) {
  const long long n4 = a.numel / 4;
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < n4;
       q += (long long)gridDim.x * blockDim.x) {
    const long long e = 4 * q;
    float4 d[DEMUON_MAX];
#pragma unroll
    for (int j = 0; j < DEMUON_MAX; ++j) {
      if (j < a.n) {
        const float4 x = ld4(a.x_in[j], e), o = ld4(a.o[j], e);
        d[j] = make_float4(fmaf(-a.eta, o.x, x.x), fmaf(-a.eta, o.y, x.y), fmaf(-a.eta, o.z, x.z),
                           fmaf(-a.eta, o.w, x.w));
      }
    }
#pragma unroll
    for (int i = 0; i < DEMUON_MAX; ++i) {
      if (i >= a.n) break;
      st4(a.x_out[i], e, mix_row(a.mix[i], d, a.n));
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (long long e = 4 * n4; e < a.numel; ++e) {
      float dj[DEMUON_MAX];
      for (int j = 0; j < a.n; ++j) dj[j] = fmaf(-a.eta, a.o[j][e], a.x_in[j][e]);
      for (int i = 0; i < a.n; ++i) {
        float s = 0.f;
        for (int j = 0; j < a.n; ++j) s = fmaf(a.mix[i][j], dj[j], s);
        a.x_out[i][e] = s;
      }
    }
  }
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

dmu_status check_common(int n, long long numel, const float* mix) {
  if (n < 1 || n > DEMUON_MAX) {
    set_last_error("n_agents must be in [1, DMU_DEMUON_MAX_AGENTS]");
    return DMU_ERR_INVALID_ARG;
  }
  if (numel < 0) {
    set_last_error("numel must be >= 0");
    return DMU_ERR_INVALID_ARG;
  }
  if (!mix) {
    set_last_error("mix must be a host array of n_agents x n_agents weights");
    return DMU_ERR_INVALID_ARG;
  }
  for (int k = 0; k < n * n; ++k) {
    if (!std::isfinite(mix[k])) {
      set_last_error("mixing weights must be finite");
      return DMU_ERR_INVALID_ARG;
    }
  }
  return DMU_OK;
}

int grid_for(long long numel) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (numel / 4 + 255) / 256;
  long long g = want < (long long)sms * 8 ? want : (long long)sms * 8;
  return g < 1 ? 1 : (int)g;
}

}  // namespace
}  // namespace dmu

extern "C" DMU_API dmu_status dmu_demuon_track(int n_agents, int64_t numel, const float* mix, float theta,
                                               const void* const* grads, float* const* momenta,
                                               const float* const* v_in, float* const* v_out,
                                               void* const* v_bf16, void* stream) {
  using namespace dmu;
  set_last_error("");
  dmu_status st = check_common(n_agents, numel, mix);
  if (st != DMU_OK) return st;
  if (!(theta >= 0.f && theta <= 1.f)) {
    set_last_error("theta must be in [0, 1]");
    return DMU_ERR_INVALID_ARG;
  }
  if (!grads || !momenta || !v_in || !v_out || !v_bf16) {
    set_last_error("grads, momenta, v_in, v_out and v_bf16 must be host arrays of n_agents device pointers");
    return DMU_ERR_INVALID_ARG;
  }
  DemuonTrack a;
  a.n = n_agents;
  a.numel = numel;
  a.theta = theta;
  for (int i = 0; i < DEMUON_MAX; ++i)
    for (int j = 0; j < DEMUON_MAX; ++j) a.mix[i][j] = (i < n_agents && j < n_agents) ? mix[i * n_agents + j] : 0.f;
  for (int i = 0; i < n_agents; ++i) {
    a.g[i] = reinterpret_cast<const __nv_bfloat16*>(grads[i]);
    a.m[i] = momenta[i];
    a.v_in[i] = v_in[i];
    a.v_out[i] = v_out[i];
    a.vb[i] = reinterpret_cast<__nv_bfloat16*>(v_bf16[i]);
    if (!a.g[i] || !a.m[i] || !a.v_in[i] || !a.v_out[i] || !a.vb[i]) {
      set_last_error("null device pointer");
      return DMU_ERR_INVALID_ARG;
    }
    if (!aligned16(a.g[i]) || !aligned16(a.m[i]) || !aligned16(a.v_in[i]) || !aligned16(a.v_out[i]) ||
        !aligned16(a.vb[i])) {
      set_last_error("every agent's array must start on a 16-byte boundary");
      return DMU_ERR_INVALID_ARG;
    }
  }
  for (int i = 0; i < n_agents; ++i)
    for (int j = 0; j < n_agents; ++j) {
      if (a.v_out[i] == a.v_in[j]) {
        set_last_error("v_out must not alias v_in: every output reads all agents' v_in");
        return DMU_ERR_INVALID_ARG;
      }
      if (a.v_out[i] == a.m[j] || (const void*)a.vb[i] == (const void*)a.g[j] ||
          (const void*)a.vb[i] == (const void*)a.m[j] || (const void*)a.v_out[i] == (const void*)a.vb[j]) {
        set_last_error("v_out, v_bf16 and momenta must be distinct arrays, and v_bf16 must not alias grads");
        return DMU_ERR_INVALID_ARG;
      }
    }
  for (int i = n_agents; i < DEMUON_MAX; ++i) {
    a.g[i] = nullptr;
    a.m[i] = a.v_out[i] = nullptr;
    a.v_in[i] = nullptr;
    a.vb[i] = nullptr;
  }
  if (numel == 0) return DMU_OK;
  k_demuon_track<<<grid_for(numel), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return DMU_ERR_CUDA;
  }
  return DMU_OK;
}

extern "C" DMU_API dmu_status dmu_demuon_mix(int n_agents, int64_t numel, const float* mix, float eta,
                                             const float* const* x_in, const float* const* o,
                                             float* const* x_out, void* stream) {
  using namespace dmu;
  set_last_error("");
  dmu_status st = check_common(n_agents, numel, mix);
  if (st != DMU_OK) return st;
  if (!std::isfinite(eta)) {
    set_last_error("eta must be finite");
    return DMU_ERR_INVALID_ARG;
  }
  if (!x_in || !o || !x_out) {
    set_last_error("x_in, o and x_out must be host arrays of n_agents device pointers");
    return DMU_ERR_INVALID_ARG;
  }
  DemuonMix a;
  a.n = n_agents;
  a.numel = numel;
  a.eta = eta;
  for (int i = 0; i < DEMUON_MAX; ++i)
    for (int j = 0; j < DEMUON_MAX; ++j) a.mix[i][j] = (i < n_agents && j < n_agents) ? mix[i * n_agents + j] : 0.f;
  for (int i = 0; i < DEMUON_MAX; ++i) {
    a.x_in[i] = i < n_agents ? x_in[i] : nullptr;
    a.o[i] = i < n_agents ? o[i] : nullptr;
    a.x_out[i] = i < n_agents ? x_out[i] : nullptr;
  }
  for (int i = 0; i < n_agents; ++i) {
    if (!a.x_in[i] || !a.o[i] || !a.x_out[i]) {
      set_last_error("null device pointer");
      return DMU_ERR_INVALID_ARG;
    }
    if (!aligned16(a.x_in[i]) || !aligned16(a.o[i]) || !aligned16(a.x_out[i])) {
      set_last_error("every agent's array must start on a 16-byte boundary");
      return DMU_ERR_INVALID_ARG;
    }
  }
  for (int i = 0; i < n_agents; ++i)
    for (int j = 0; j < n_agents; ++j)
      if (a.x_out[i] == a.x_in[j] || a.x_out[i] == a.o[j]) {
        set_last_error("x_out must not alias x_in or o: every output reads all agents' inputs");
        return DMU_ERR_INVALID_ARG;
      }
  if (numel == 0) return DMU_OK;
  k_demuon_mix<<<grid_for(numel), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return DMU_ERR_CUDA;
  }
  return DMU_OK;
}
