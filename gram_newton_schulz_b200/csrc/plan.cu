// Planner and C ABI of libdmu (see include/dmu.h for the contract).
//
// The planner groups matrices into shape buckets (equal rows, cols) and
// Gram classes (equal m = min(rows, cols)); the batched recursion then runs
// one grouped launch per product over all matrices of all classes that
// share a precision (DMuon page, section 2.2: batching of similar-shape
// matrices so the Gram recursion runs jointly and dispatch is amortised).
// Tall matrices are transposed logically: their Gram matrix is Mb^T Mb
// read through an MN-major tensor map, and their update is written into W
// transposed; nothing is copied.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <fstream>
#include <sstream>
#include <map>
#include <string>
#include <utility>
#include <vector>

#include "dmu_internal.h"

using namespace dmu;

namespace {

thread_local std::string g_err;

dmu_status fail(dmu_status s, const std::string& msg) {
  g_err = msg;
  return s;
}

#define CUDA_TRY(x)                                                                   \
  do {                                                                                \
    cudaError_t e_ = (x);                                                             \
    if (e_ != cudaSuccess) return fail(DMU_ERR_CUDA, std::string(#x) + ": " + cudaGetErrorString(e_)); \
  } while (0)

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t round_up64(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

struct Bucket {
  int64_t rows = 0, cols = 0, m = 0, n = 0;
  bool tall = false;
  int count = 0;
  std::vector<int> mats;  // plan indices, in slot order
  int first_slot = 0;
  int cls = 0, cls_off = 0;
  int64_t ldc = 0;
  int64_t mb_off = 0;  // element offset of the bucket's first image
  int map_k = -1, map_mn = -1;
  int fsched = -1;     // tile schedule of this bucket's final GEMM (-1: the plan's)
  int ssched = -1;     // tile schedule of this bucket's SYRK (-1: its class's)
};

struct GClass {
  int64_t m = 0, ldg = 0;
  int count = 0;
  size_t off = 0;     // byte offset in the workspace
  size_t off_pf = 0;  // all but F16 classes: the final P as an fp16 hi/lo pair
  int prec = DMU_PREC_FAST;
  int kind = KIND_BF16;
  int map = -1;       // TMA map over the Gram slots (bf16 pairs or fp32)
  int map_pf = -1;    // all but F16 classes: fp16 map over the final-P pair
  // Half storage (all but TF32 classes): symmetric Gram-space matrices keep
  // only their upper 256 x 256 blocks; lower blocks are read transposed
  // through MN-major maps (64 x 64 boxes).
  bool half = false;
  int map_t = -1, map_pf_t = -1;
  // Tile schedule of this class's Gram recursion: -1 the plan's, a staged
  // tile schedule (TILE_SCHEDS), or SCHED_ONCHIP: the whole recursion in one
  // CTA per matrix
  int sched = -1;
};

// Schedules: 0 single CTAs, 128 x 256 tiles; 1 CTA pairs, 256 x 256 tiles;
// 2 single CTAs, 128 x 128 tiles; 3 on chip (m <= 128); 4 and 5 CTA pairs
// whose one-MMA-per-slice fp16 kernels take 2 and 1 K atoms per stage
// (three and six stages) instead of 3 (two stages); 6 CTA pairs with
// 256 x 512 tiles (two N = 256 MMAs per K slice share A: a quarter fewer
// operand bytes per MMA, one 512-column accumulator, so the epilogue does
// not overlap the next tile), scaled-fp16 launches only (others run 1).
// The Gram products and the final lose more to the exposed epilogue than
// they gain (measured), so schedule 6 is an autotune candidate only for the
// SYRK, whose K is the long side n (with schedules 0 and 4 beside the
// class's own).
constexpr int SCHED_ONCHIP = 3;
constexpr int SCHED_WIDE = 6;
constexpr int TILE_SCHEDS[6] = {0, 1, 2, 4, 5, 6};
bool is_pair(int sched) { return sched == 1 || sched == 4 || sched == 5 || sched == SCHED_WIDE; }
int pair_kat(int sched) { return sched == 4 ? 2 : (sched == 5 ? 1 : 0); }
bool valid_sched(int v) { return v >= 0 && v <= 6; }
int tile_n(int sched) { return sched == 2 ? 128 : (sched == SCHED_WIDE ? 512 : BN); }

bool onchip_eligible(dmu_dtype dtype, const GClass& g) {
  return dtype == DMU_BF16 && g.prec == DMU_PREC_SPLIT3 && g.m <= ONCHIP_MAX_M;
}

enum { TBL_GRADS = 0, TBL_MOMS, TBL_W, TBL_O, TBL_IN, NUM_TBL };

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

struct DevGuard {
  int prev = -1;
  explicit DevGuard(int d) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != d) cudaSetDevice(d);
  }
  ~DevGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

}  // namespace

struct dmu_plan_s {
  int device = 0, num_sms = 0;
  bool has_device = false;
  dmu_dtype dtype = DMU_BF16;
  dmu_prec prec = DMU_PREC_AUTO;
  int count = 0;
  std::vector<dmu_shape> shapes;
  std::vector<Bucket> buckets;
  std::vector<GClass> classes;
  std::vector<int> slot_of;
  std::vector<MomChunk> chunks;
  std::vector<MomMat> mats;
  bool vec_shapes = true;
  size_t esize = 2;
  // workspace layout (bytes)
  size_t off_status = 0, off_inv = 0, off_iscale = 0, off_invimg = 0, off_fix = 0, off_partial = 0,
         off_chunks = 0, off_mats = 0, off_tbl = 0,
         off_mb = 0, off_gram = 0, total = 0;
  char* ws = nullptr;
  size_t ws_bytes = 0;
  std::vector<CUtensorMap> maps;
  std::vector<const void*> tbl_cache[NUM_TBL];
  bool tbl_valid[NUM_TBL] = {};
  void* pinned[NUM_TBL] = {};
  cudaEvent_t tbl_ev[NUM_TBL] = {};
  bool have_mb = false, have_p = false;
  int p_final = 0;  // 0: P buffer A, 1: P buffer B
  float eps = 1e-7f;
  int launches = 0;
  long long timeout_ns = 2000000000LL;
  // tensor-core tile schedule: 1 = CTA pairs (256 x 256 tiles), 0 = single
  // CTAs (128 x 256), 2 = single CTAs (128 x 128, for many small matrices)
  int sched = 1;
  bool half_store = true;  // half-stored symmetric Gram-space matrices
  int tune_class = -1, tune_bucket = -1;  // autotune: run one class / one bucket only
  int tune_syrk = -1;                      // autotune: the SYRK of one bucket only
  int tune_count = 0;                      // autotune: matrices of the tuned bucket's final (0: all)

  int class_sched(int c) const { return classes[c].sched >= 0 ? classes[c].sched : sched; }
  bool onchip(int c) const { return classes[c].sched == SCHED_ONCHIP; }
  int final_sched(const Bucket& b) const { return b.fsched >= 0 ? b.fsched : sched; }

  unsigned int* status_dev() const { return reinterpret_cast<unsigned int*>(ws + off_status); }
  float* inv_dev() const { return reinterpret_cast<float*>(ws + off_inv); }
  // bf16 plans: per-matrix scale 2^e of the fp16 image, and inv * 2^-e
  float* iscale_dev() const { return reinterpret_cast<float*>(ws + off_iscale); }
  float* invimg_dev() const { return reinterpret_cast<float*>(ws + off_invimg); }
  int* fix_dev() const { return reinterpret_cast<int*>(ws + off_fix); }  // image needs rewriting
  int* fix_count_dev() const { return fix_dev() + count; }              // how many are flagged
  // the scale the tensor-core kernels apply to image products
  const float* inv_kernel() const { return dtype == DMU_BF16 ? invimg_dev() : inv_dev(); }
  float* partial_dev() const { return reinterpret_cast<float*>(ws + off_partial); }
  const MomChunk* chunks_dev() const { return reinterpret_cast<const MomChunk*>(ws + off_chunks); }
  const MomMat* mats_dev() const { return reinterpret_cast<const MomMat*>(ws + off_mats); }
  void** tbl_dev(int t) const { return reinterpret_cast<void**>(ws + off_tbl) + (size_t)t * count; }
  char* mb_dev() const { return ws + off_mb; }
  // bf16 Gram slot of class c (first matrix of the class)
  __nv_bfloat16* slot_bf16(int c, int slot) const {
    const GClass& g = classes[c];
    return reinterpret_cast<__nv_bfloat16*>(ws + g.off) + (size_t)slot * g.count * g.m * g.ldg;
  }
  float* slot_f32(int c, int slot) const {
    const GClass& g = classes[c];
    return reinterpret_cast<float*>(ws + g.off) + (size_t)slot * g.count * g.m * g.ldg;
  }
  // final P of non-F16 classes as an fp16 pair: half 0 = hi, 1 = lo
  __nv_bfloat16* pf_bf16(int c, int half) const {  // 16-bit storage; the bits are fp16
    const GClass& g = classes[c];
    return reinterpret_cast<__nv_bfloat16*>(ws + g.off_pf) + (size_t)half * g.count * g.m * g.ldg;
  }
};

namespace {

dmu_status check_plan(dmu_plan p, bool need_ws) {
  if (!p) return fail(DMU_ERR_INVALID_ARG, "plan is NULL");
  if (need_ws && !p->ws) return fail(DMU_ERR_WORKSPACE, "no workspace set (dmu_set_workspace)");
  if (need_ws && !p->has_device) return fail(DMU_ERR_CUDA, "no CUDA device");
  return DMU_OK;
}

dmu_status upload_table(dmu_plan p, int t, const void* const* ptrs, cudaStream_t s, bool allow_null = false) {
  std::vector<const void*> v(p->count);
  for (int i = 0; i < p->count; ++i) {
    if (!ptrs[i] && !allow_null)
      return fail(DMU_ERR_INVALID_ARG, "null device pointer in table, matrix " + std::to_string(i));
    v[p->slot_of[i]] = ptrs[i];
  }
  if (p->tbl_valid[t] && v == p->tbl_cache[t]) return DMU_OK;
  const size_t bytes = sizeof(void*) * (size_t)p->count;
  if (!p->pinned[t]) {
    CUDA_TRY(cudaMallocHost(&p->pinned[t], bytes));
    CUDA_TRY(cudaEventCreateWithFlags(&p->tbl_ev[t], cudaEventDisableTiming));
  } else {
    CUDA_TRY(cudaEventSynchronize(p->tbl_ev[t]));  // previous upload has left the staging buffer
  }
  std::memcpy(p->pinned[t], v.data(), bytes);
  CUDA_TRY(cudaMemcpyAsync(p->tbl_dev(t), p->pinned[t], bytes, cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaEventRecord(p->tbl_ev[t], s));
  p->tbl_cache[t] = std::move(v);
  p->tbl_valid[t] = true;
  return DMU_OK;
}

bool aligned16(const void* const* ptrs, int n) {
  for (int i = 0; i < n; ++i)
    if (reinterpret_cast<uintptr_t>(ptrs[i]) & 15) return false;
  return true;
}

// Tile grid of one problem for row blocks of `bm` (128: one CTA per tile;
// 256: a CTA pair per tile) and column blocks of BN; symmetric problems keep
// only the tiles that touch the upper triangle (same rule as the kernels).
int tiles_for(int M, int N, bool sym, int* tm, int* tn, int bm = BM, int bn = BN) {
  *tm = (M + bm - 1) / bm;
  *tn = (N + bn - 1) / bn;
  if (!sym) return (*tm) * (*tn);
  int t = 0;
  for (int bj = 0; bj < *tn; ++bj) {
    int c = ((bj + 1) * bn - 1) / bm + 1;
    t += c < *tm ? c : *tm;
  }
  return t;
}

// ---------------------------------------------------------------- tc launches
struct Prob {
  GemmProblem g;
  int amap, bmap;      // plan map indices
  int amap_t = -1, bmap_t = -1;  // transposed-read maps of half-stored operands
};

dmu_status run_tc(dmu_plan p, std::vector<Prob>& probs, int na, int nb, int kind, int sched, cudaStream_t s) {
  if (sched == SCHED_WIDE && kind != KIND_F16) sched = 1;  // the wide pair tile is built for fp16 operands
  size_t i = 0;
  while (i < probs.size()) {
    GemmParams gp;
    std::memset(&gp, 0, sizeof(gp));
    std::vector<int> used;
    int nprob = 0, tiles = 0;
    while (i < probs.size() && nprob < MAX_PROBS) {
      std::vector<int> want = {probs[i].amap, probs[i].bmap};
      if (probs[i].amap_t >= 0) want.push_back(probs[i].amap_t);
      if (probs[i].bmap_t >= 0) want.push_back(probs[i].bmap_t);
      int need = 0;
      for (size_t w = 0; w < want.size(); ++w) {
        bool seen = false;
        for (int u : used) seen |= (u == want[w]);
        for (size_t v = 0; v < w; ++v) seen |= (want[v] == want[w]);
        need += seen ? 0 : 1;
      }
      if ((int)used.size() + need > MAX_MAPS) break;
      auto slot = [&](int pm) {
        for (size_t k = 0; k < used.size(); ++k)
          if (used[k] == pm) return (int)k;
        used.push_back(pm);
        return (int)used.size() - 1;
      };
      GemmProblem g = probs[i].g;
      g.a_map = slot(probs[i].amap);
      g.b_map = slot(probs[i].bmap);
      g.a_map_t = probs[i].amap_t >= 0 ? slot(probs[i].amap_t) : g.a_map;
      g.b_map_t = probs[i].bmap_t >= 0 ? slot(probs[i].bmap_t) : g.b_map;
      g.tiles_per_mat = tiles_for(g.M, g.N, g.sym != 0, &g.tiles_m, &g.tiles_n, is_pair(sched) ? 256 : BM,
                                  tile_n(sched));
      g.tile_begin = tiles;
      tiles += g.count * g.tiles_per_mat;
      gp.prob[nprob++] = g;
      ++i;
    }
    for (size_t k = 0; k < used.size(); ++k) gp.maps[k] = p->maps[used[k]];
    gp.nprob = nprob;
    gp.total_tiles = tiles;
    gp.status = p->status_dev();
    gp.timeout_ns = p->timeout_ns;
    if (is_pair(sched))
      CUDA_TRY(launch_gemm_tc2(gp, na, nb, kind, p->num_sms, pair_kat(sched), tile_n(sched), s));
    else
      CUDA_TRY(launch_gemm_tc(gp, na, nb, kind, p->num_sms, sched == 2 ? 128 : 256, s));
    p->launches++;
  }
  return DMU_OK;
}

void prec_shape(int prec, int* na, int* nb, int* terms, int* kind) {
  *kind = KIND_BF16;
  switch (prec) {
    case DMU_PREC_SPLIT2: *na = 2; *nb = 1; *terms = TERM_HH | TERM_LH; break;
    case DMU_PREC_SPLIT3: *na = 2; *nb = 2; *terms = TERM_HH | TERM_HL | TERM_LH; break;
    case DMU_PREC_TF32: *na = 1; *nb = 1; *terms = TERM_HH; *kind = KIND_TF32; break;
    case DMU_PREC_F16: *na = 1; *nb = 1; *terms = TERM_HH; *kind = KIND_F16; break;
    default: *na = 1; *nb = 1; *terms = TERM_HH; break;
  }
}

// Output slot meaning "the final P, as an fp16 hi/lo pair in the class's
// final-P area" (classes other than F16, whose P slots are fp16 already).
constexpr int OUT_PF = -2;

// A Gram-space product over all matrices of class c:
//   out = alpha * (A B) + beta * Cin + gamma * I   [, out2 = out + gamma2 * I]
Prob gram_prob(dmu_plan p, int c, int a_slot, int b_slot, int terms, float alpha, float beta,
               int cin_slot, int out_slot, bool out_lo, int out2_slot, float gamma2) {
  const GClass& gc = p->classes[c];
  Prob pr;
  std::memset(&pr, 0, sizeof(pr));
  GemmProblem& g = pr.g;
  g.count = gc.count;
  g.M = g.N = g.K = (int)gc.m;
  g.sym = 1;
  g.tiles_per_mat = tiles_for(g.M, g.N, true, &g.tiles_m, &g.tiles_n);
  g.a_mn = g.b_mn = 0;
  g.a_z[0] = a_slot * gc.count;
  g.a_z[1] = (a_slot + 1) * gc.count;
  g.b_z[0] = b_slot * gc.count;
  g.b_z[1] = (b_slot + 1) * gc.count;
  g.terms = terms;
  g.epi = EPI_GRAM;
  g.alpha_mode = ALPHA_CONST;
  g.alpha = alpha;
  g.beta = beta;
  g.gamma = 0.f;
  g.gamma2 = gamma2;
  g.scale2 = 1.f;
  if (cin_slot >= 0) {
    g.cin_hi = p->slot_bf16(c, cin_slot);
    g.cin_lo = p->slot_bf16(c, cin_slot + 1);
  }
  if (out_slot == OUT_PF) {
    g.out_fmt = FMT_PAIR_H;
    g.out_hi = p->pf_bf16(c, 0);
    g.out_lo = p->pf_bf16(c, 1);
  } else {
    g.out_hi = p->slot_bf16(c, out_slot);
    g.out_lo = out_lo ? p->slot_bf16(c, out_slot + 1) : nullptr;
  }
  if (out2_slot == OUT_PF) {
    g.out2_fmt = FMT_PAIR_H;
    g.out2_hi = p->pf_bf16(c, 0);
    g.out2_lo = p->pf_bf16(c, 1);
  } else if (out2_slot >= 0) {
    g.out2_hi = p->slot_bf16(c, out2_slot);
    g.out2_lo = p->slot_bf16(c, out2_slot + 1);
  }
  g.ld = gc.ldg;
  g.mat_stride = gc.m * gc.ldg;
  pr.amap = pr.bmap = gc.map;
  if (gc.half) {
    g.half_a = g.half_b = g.half_out = 1;
    pr.amap_t = pr.bmap_t = gc.map_t;
  }
  return pr;
}

// TF32 classes: fp32 slots; out_slot == OUT_PF writes the final P as an
// fp16 hi/lo pair (the operand of the final fp16 GEMM).

void set_f32_out(dmu_plan p, int c, int slot, int* fmt, float** f, __nv_bfloat16** hi, __nv_bfloat16** lo) {
  if (slot == OUT_PF) {
    *fmt = FMT_PAIR_H;
    *hi = p->pf_bf16(c, 0);
    *lo = p->pf_bf16(c, 1);
  } else if (slot >= 0) {
    *fmt = FMT_F32;
    *f = p->slot_f32(c, slot);
  }
}

Prob gram_prob_f32(dmu_plan p, int c, int a_slot, int b_slot, float alpha, float beta, int cin_slot,
                   int out_slot, int out2_slot, float gamma2) {
  const GClass& gc = p->classes[c];
  Prob pr;
  std::memset(&pr, 0, sizeof(pr));
  GemmProblem& g = pr.g;
  g.count = gc.count;
  g.M = g.N = g.K = (int)gc.m;
  g.sym = 1;
  g.tiles_per_mat = tiles_for(g.M, g.N, true, &g.tiles_m, &g.tiles_n);
  g.a_z[0] = g.a_z[1] = a_slot * gc.count;
  g.b_z[0] = g.b_z[1] = b_slot * gc.count;
  g.terms = TERM_HH;
  g.epi = EPI_GRAM;
  g.alpha_mode = ALPHA_CONST;
  g.alpha = alpha;
  g.beta = beta;
  g.gamma2 = gamma2;
  g.scale2 = 1.f;
  g.cin_fmt = FMT_F32;
  if (cin_slot >= 0) g.cin_f = p->slot_f32(c, cin_slot);
  set_f32_out(p, c, out_slot, &g.out_fmt, &g.out_f, &g.out_hi, &g.out_lo);
  set_f32_out(p, c, out2_slot, &g.out2_fmt, &g.out2_f, &g.out2_hi, &g.out2_lo);
  g.ld = gc.ldg;
  g.mat_stride = gc.m * gc.ldg;
  pr.amap = pr.bmap = gc.map;
  return pr;
}

// F16 classes: every Gram-space quantity is stored as an fp16 hi/lo pair
// pre-scaled by a power of two so its entries sit well inside fp16's
// normal range: G, R, T by 2^8 (their entries are O(1/m)), P by 1 (its
// eigenvalues reach ~500).  The scales are folded exactly into the
// epilogue coefficients.  The final P is written as a bf16 pair (unscaled)
// because the final GEMM multiplies it with the bf16 image of M.
float half_slot_scale(int slot) { return slot >= SLOT_PA_HI ? 1.f : 256.f; }

void set_h_out(dmu_plan p, int c, int slot, int* fmt, __nv_bfloat16** hi, __nv_bfloat16** lo, float* scale) {
  if (slot >= 0) {
    *fmt = FMT_PAIR_H;
    *hi = p->slot_bf16(c, slot);  // fp16 bits; same element size as bf16
    *lo = p->slot_bf16(c, slot + 1);
    *scale = half_slot_scale(slot);
  } else {
    *scale = 1.f;
  }
}

Prob gram_prob_h(dmu_plan p, int c, int a_slot, int b_slot, float alpha, float beta, int cin_slot, int out_slot,
                 int out2_slot, float gamma2, bool out_lo = true) {
  const GClass& gc = p->classes[c];
  Prob pr;
  std::memset(&pr, 0, sizeof(pr));
  GemmProblem& g = pr.g;
  g.count = gc.count;
  g.M = g.N = g.K = (int)gc.m;
  g.sym = 1;
  g.tiles_per_mat = tiles_for(g.M, g.N, true, &g.tiles_m, &g.tiles_n);
  g.a_z[0] = a_slot * gc.count;
  g.a_z[1] = (a_slot + 1) * gc.count;
  g.b_z[0] = b_slot * gc.count;
  g.b_z[1] = (b_slot + 1) * gc.count;
  g.terms = TERM_HH;
  g.epi = EPI_GRAM;
  g.alpha_mode = ALPHA_CONST;
  float s_out = 1.f, s_out2 = 1.f;
  set_h_out(p, c, out_slot, &g.out_fmt, &g.out_hi, &g.out_lo, &s_out);
  set_h_out(p, c, out2_slot, &g.out2_fmt, &g.out2_hi, &g.out2_lo, &s_out2);
  if (!out_lo) g.out_lo = nullptr;
  g.alpha = alpha * s_out / (half_slot_scale(a_slot) * half_slot_scale(b_slot));
  g.gamma = 0.f;
  if (cin_slot >= 0) {
    g.cin_fmt = FMT_PAIR_H;
    g.cin_hi = p->slot_bf16(c, cin_slot);
    g.cin_lo = p->slot_bf16(c, cin_slot + 1);
    g.beta = beta * s_out / half_slot_scale(cin_slot);
  }
  g.scale2 = s_out2 / s_out;
  g.gamma2 = gamma2 * s_out2;
  g.ld = gc.ldg;
  g.mat_stride = gc.m * gc.ldg;
  pr.amap = pr.bmap = gc.map;
  if (gc.half) {
    g.half_a = g.half_b = g.half_out = 1;
    pr.amap_t = pr.bmap_t = gc.map_t;
  }
  return pr;
}

enum Product { PROD_R, PROD_T, PROD_P, PROD_G };

// Operands and epilogue of one product of step k for class c (R-form):
//   R = bG + c(GG),  T = aG + RG,  P' = aP + RP (P0 = aI + R),  G' = aT + TR
Prob product(dmu_plan p, int c, Product what, int k, bool last, const float co[3], int p_in, int p_out) {
  const GClass& gc = p->classes[c];
  int na, nb, terms, kind;
  prec_shape(gc.prec, &na, &nb, &terms, &kind);
  if (kind == KIND_F16) {
    const int hin = p_in == 0 ? SLOT_PA_HI : SLOT_PB_HI, hout = p_out == 0 ? SLOT_PA_HI : SLOT_PB_HI;
    switch (what) {
      case PROD_R:
        // R is only ever an MMA operand (hi): its lo half is not stored
        return gram_prob_h(p, c, SLOT_G_HI, SLOT_G_HI, co[2], co[1], SLOT_G_HI, SLOT_R_HI,
                           k == 0 ? SLOT_PA_HI : -1, co[0], false);
      case PROD_T:
        return gram_prob_h(p, c, SLOT_R_HI, SLOT_G_HI, 1.f, co[0], SLOT_G_HI, SLOT_T_HI, -1, 0.f);
      case PROD_P:
        return gram_prob_h(p, c, SLOT_R_HI, hin, 1.f, co[0], hin, hout, -1, 0.f);
      case PROD_G:
      default:
        return gram_prob_h(p, c, SLOT_T_HI, SLOT_R_HI, 1.f, co[0], SLOT_T_HI, SLOT_G_HI, -1, 0.f);
    }
  }
  if (kind == KIND_TF32) {
    const int fin = p_in == 0 ? FSLOT_PA : FSLOT_PB, fout = p_out == 0 ? FSLOT_PA : FSLOT_PB;
    switch (what) {
      case PROD_R:
        return gram_prob_f32(p, c, FSLOT_G, FSLOT_G, co[2], co[1], FSLOT_G, FSLOT_R,
                             k == 0 ? (last ? OUT_PF : FSLOT_PA) : -1, co[0]);
      case PROD_T:
        return gram_prob_f32(p, c, FSLOT_R, FSLOT_G, 1.f, co[0], FSLOT_G, FSLOT_T, -1, 0.f);
      case PROD_P:
        return gram_prob_f32(p, c, FSLOT_R, fin, 1.f, co[0], fin, last ? OUT_PF : fout, -1, 0.f);
      case PROD_G:
      default:
        return gram_prob_f32(p, c, FSLOT_T, FSLOT_R, 1.f, co[0], FSLOT_T, FSLOT_G, -1, 0.f);
    }
  }
  const bool r_lo = gc.prec != DMU_PREC_FAST;
  const int PA = SLOT_PA_HI, PB = SLOT_PB_HI;
  const int pin = p_in == 0 ? PA : PB, pout = p_out == 0 ? PA : PB;
  switch (what) {
    case PROD_R:
      return gram_prob(p, c, SLOT_G_HI, SLOT_G_HI, terms, co[2], co[1], SLOT_G_HI, SLOT_R_HI, r_lo,
                       k == 0 ? (last ? OUT_PF : PA) : -1, co[0]);
    case PROD_T:
      return gram_prob(p, c, SLOT_R_HI, SLOT_G_HI, terms, 1.f, co[0], SLOT_G_HI, SLOT_T_HI, true, -1, 0.f);
    case PROD_P:
      if (gc.prec == DMU_PREC_SPLIT2)
        return gram_prob(p, c, pin, SLOT_R_HI, terms, 1.f, co[0], pin, last ? OUT_PF : pout, true, -1, 0.f);
      return gram_prob(p, c, SLOT_R_HI, pin, terms, 1.f, co[0], pin, last ? OUT_PF : pout, true, -1, 0.f);
    case PROD_G:
    default:
      return gram_prob(p, c, SLOT_T_HI, SLOT_R_HI, terms, 1.f, co[0], SLOT_T_HI, SLOT_G_HI, true, -1, 0.f);
  }
}

// Run one or two kinds of product for every class, one grouped launch per
// precision group.
dmu_status run_products(dmu_plan p, const std::vector<std::pair<Product, bool>>& kinds, int k, bool last,
                        const float co[3], int p_in, int p_out, cudaStream_t s) {
  const int precs[5] = {DMU_PREC_F16, DMU_PREC_TF32, DMU_PREC_FAST, DMU_PREC_SPLIT2, DMU_PREC_SPLIT3};
  for (int pr : precs) {
    for (int sched : TILE_SCHEDS) {
      std::vector<Prob> probs;
      for (size_t c = 0; c < p->classes.size(); ++c) {
        if (p->classes[c].prec != pr || p->class_sched((int)c) != sched) continue;
        if (p->tune_class >= 0 && (int)c != p->tune_class) continue;
        for (auto& kd : kinds)
          if (kd.second) probs.push_back(product(p, (int)c, kd.first, k, last, co, p_in, p_out));
      }
      if (probs.empty()) continue;
      int na, nb, terms, kind;
      prec_shape(pr, &na, &nb, &terms, &kind);
      dmu_status st = run_tc(p, probs, na, nb, kind, sched, s);
      if (st != DMU_OK) return st;
    }
  }
  return DMU_OK;
}

// Classes on the on-chip schedule: one launch (per 8 buckets) runs SYRK and
// the whole recursion with one CTA per matrix and writes the final P into
// the class's P slot, where the staged path would have left it.
dmu_status run_onchip(dmu_plan p, const float co[3], int steps, int p_final, cudaStream_t s) {
  OnchipParams op;
  std::memset(&op, 0, sizeof(op));
  int nmaps = 0;
  auto flush = [&]() -> dmu_status {
    if (op.nprob == 0) return DMU_OK;
    op.inv = p->inv_kernel();
    op.a = co[0];
    op.b = co[1];
    op.c = co[2];
    op.steps = steps;
    op.status = p->status_dev();
    op.timeout_ns = p->timeout_ns;
    CUDA_TRY(launch_gram_onchip(op, p->num_sms, s));
    p->launches++;
    std::memset(&op, 0, sizeof(op));
    nmaps = 0;
    return DMU_OK;
  };
  for (const Bucket& b : p->buckets) {
    if (!p->onchip(b.cls)) continue;
    if (p->tune_class >= 0 && b.cls != p->tune_class) continue;
    if (op.nprob == MAX_PROBS) {
      dmu_status st = flush();
      if (st != DMU_OK) return st;
    }
    const GClass& gc = p->classes[b.cls];
    OnchipProblem& q = op.prob[op.nprob++];
    q.count = b.count;
    q.m = (int)b.m;
    q.n = (int)b.n;
    q.tall = b.tall ? 1 : 0;
    op.maps[nmaps] = p->maps[b.tall ? b.map_mn : b.map_k];
    q.map = nmaps++;
    q.inv_base = b.first_slot;
    q.mat_begin = op.total;
    op.total += b.count;
    const size_t moff = (size_t)b.cls_off * gc.m * gc.ldg;
    (void)p_final;  // the final P goes to the class's fp16 final-P area
    q.p_hi = reinterpret_cast<__half*>(p->pf_bf16(b.cls, 0) + moff);
    q.p_lo = reinterpret_cast<__half*>(p->pf_bf16(b.cls, 1) + moff);
    q.ld = gc.ldg;
    q.mat_stride = gc.m * gc.ldg;
  }
  return flush();
}

dmu_status gram_bf16(dmu_plan p, const float co[3], int steps, cudaStream_t s) {
  // index of the P buffer that holds P_K after `steps` steps (0: A, 1: B)
  const int p_final = steps >= 1 ? (steps - 1) & 1 : 0;
  if (steps >= 1) {
    dmu_status st0 = run_onchip(p, co, steps, p_final, s);
    if (st0 != DMU_OK) return st0;
  }
  // G0 = s^2 X X^T, one problem per shape bucket (SYRK, upper tiles only),
  // launched with its class's tile schedule
  std::vector<Prob> syrk;
  std::vector<int> syrk_sched;
  for (const Bucket& b : p->buckets) {
    const GClass& gc = p->classes[b.cls];
    if (p->tune_class >= 0 && b.cls != p->tune_class) continue;
    if (p->tune_syrk >= 0 && &b != &p->buckets[p->tune_syrk]) continue;
    if (steps >= 1 && p->onchip(b.cls)) continue;
    Prob pr;
    std::memset(&pr, 0, sizeof(pr));
    GemmProblem& g = pr.g;
    g.count = b.count;
    g.M = g.N = (int)b.m;
    g.K = (int)b.n;
    g.sym = 1;
    g.tiles_per_mat = tiles_for(g.M, g.N, true, &g.tiles_m, &g.tiles_n);
    g.a_mn = g.b_mn = b.tall ? 1 : 0;
    g.terms = TERM_HH;
    g.epi = EPI_GRAM;
    g.alpha_mode = ALPHA_INV2;
    g.alpha = 1.f;
    g.inv = p->inv_kernel();
    g.inv_base = b.first_slot;
    const size_t moff = (size_t)b.cls_off * gc.m * gc.ldg;
    if (gc.kind == KIND_TF32) {
      g.out_fmt = FMT_F32;
      g.out_f = p->slot_f32(b.cls, FSLOT_G) + moff;
    } else if (gc.kind == KIND_F16) {
      g.out_fmt = FMT_PAIR_H;
      g.alpha = half_slot_scale(SLOT_G_HI);
      g.out_hi = p->slot_bf16(b.cls, SLOT_G_HI) + moff;
      g.out_lo = p->slot_bf16(b.cls, SLOT_G_LO) + moff;
    } else {
      g.out_hi = p->slot_bf16(b.cls, SLOT_G_HI) + moff;
      g.out_lo = p->slot_bf16(b.cls, SLOT_G_LO) + moff;
    }
    g.ld = gc.ldg;
    g.mat_stride = gc.m * gc.ldg;
    pr.amap = pr.bmap = b.tall ? b.map_mn : b.map_k;
    g.half_out = gc.half ? 1 : 0;
    syrk.push_back(pr);
    syrk_sched.push_back(p->onchip(b.cls) ? p->sched : (b.ssched >= 0 ? b.ssched : p->class_sched(b.cls)));
  }
  dmu_status st = DMU_OK;
  for (int sched : TILE_SCHEDS) {
    std::vector<Prob> group;
    for (size_t i = 0; i < syrk.size(); ++i)
      if (syrk_sched[i] == sched) group.push_back(syrk[i]);
    if (group.empty()) continue;
    st = run_tc(p, group, 1, 1, KIND_F16, sched, s);  // the fp16 image of X
    if (st != DMU_OK) return st;
  }

  if (steps == 0) {
    for (size_t c = 0; c < p->classes.size(); ++c) {
      const GClass& gc = p->classes[c];
      if (p->tune_class >= 0 && (int)c != p->tune_class) continue;
      if (p->tune_syrk >= 0) continue;  // timing one bucket's SYRK alone
      // P_0 = I as an fp16 pair: in P buffer A for F16 classes, in the
      // final-P area for the others
      const bool f16 = gc.kind == KIND_F16;
      CUDA_TRY(launch_identity16(f16 ? p->slot_bf16((int)c, SLOT_PA_HI) : p->pf_bf16((int)c, 0),
                                 f16 ? p->slot_bf16((int)c, SLOT_PA_LO) : p->pf_bf16((int)c, 1),
                                 gc.count, (int)gc.m, gc.ldg, gc.m * gc.ldg, 1, s));
      p->launches++;
    }
    p->p_final = 0;
    return DMU_OK;
  }
  int p_cur = 0;  // P_k lives in buffer p_cur (after step 0: buffer A)
  for (int k = 0; k < steps; ++k) {
    const bool last = (k == steps - 1);
    st = run_products(p, {{PROD_R, true}}, k, last, co, 0, 0, s);
    if (st != DMU_OK) return st;
    const int p_next = (k == 0) ? 0 : 1 - p_cur;
    st = run_products(p, {{PROD_T, !last}, {PROD_P, k >= 1}}, k, last, co, p_cur, p_next, s);
    if (st != DMU_OK) return st;
    p_cur = p_next;
    if (!last) {
      st = run_products(p, {{PROD_G, true}}, k, last, co, 0, 0, s);
      if (st != DMU_OK) return st;
    }
  }
  p->p_final = p_cur;
  return p_cur == p_final ? DMU_OK : fail(DMU_ERR_CUDA, "internal: final P buffer mismatch");
}

// ---------------------------------------------------------------- fp32 path
SimtProblem simt_gram(dmu_plan p, int c, int a_slot, int b_slot, float alpha, float beta, int cin_slot,
                      int out_slot, int out2_slot, float gamma2) {
  const GClass& gc = p->classes[c];
  SimtProblem q;
  std::memset(&q, 0, sizeof(q));
  q.count = gc.count;
  q.M = q.N = q.K = (int)gc.m;
  q.sym = 1;
  q.a = p->slot_f32(c, a_slot);
  q.a_ms = gc.m * gc.ldg;
  q.a_si = gc.ldg;
  q.a_sk = 1;
  q.b = p->slot_f32(c, b_slot);
  q.b_ms = gc.m * gc.ldg;
  q.b_si = gc.ldg;
  q.b_sk = 1;
  q.epi = EPI_GRAM;
  q.alpha_mode = ALPHA_CONST;
  q.alpha = alpha;
  q.beta = beta;
  q.gamma2 = gamma2;
  q.cin = cin_slot >= 0 ? p->slot_f32(c, cin_slot) : nullptr;
  q.out = p->slot_f32(c, out_slot);
  q.out2 = out2_slot >= 0 ? p->slot_f32(c, out2_slot) : nullptr;
  q.ld = gc.ldg;
  q.mat_stride = gc.m * gc.ldg;
  return q;
}

dmu_status gram_f32(dmu_plan p, const float co[3], int steps, cudaStream_t s) {
  for (const Bucket& b : p->buckets) {
    const GClass& gc = p->classes[b.cls];
    SimtProblem q;
    std::memset(&q, 0, sizeof(q));
    q.count = b.count;
    q.M = q.N = (int)b.m;
    q.K = (int)b.n;
    q.sym = 1;
    q.a = reinterpret_cast<const float*>(p->mb_dev()) + b.mb_off;
    q.a_ms = b.rows * b.ldc;
    q.a_si = b.tall ? 1 : b.ldc;
    q.a_sk = b.tall ? b.ldc : 1;
    q.b = q.a;
    q.b_ms = q.a_ms;
    q.b_si = q.a_si;
    q.b_sk = q.a_sk;
    q.epi = EPI_GRAM;
    q.alpha_mode = ALPHA_INV2;
    q.alpha = 1.f;
    q.inv = p->inv_dev();
    q.inv_base = b.first_slot;
    q.out = p->slot_f32(b.cls, FSLOT_G) + (size_t)b.cls_off * gc.m * gc.ldg;
    q.ld = gc.ldg;
    q.mat_stride = gc.m * gc.ldg;
    CUDA_TRY(launch_simt_gemm(q, s));
    p->launches++;
  }
  if (steps == 0) {
    for (size_t c = 0; c < p->classes.size(); ++c) {
      const GClass& gc = p->classes[c];
      CUDA_TRY(launch_identity_f32(p->slot_f32((int)c, FSLOT_PA), gc.count, (int)gc.m, gc.ldg,
                                   gc.m * gc.ldg, s));
      p->launches++;
    }
    p->p_final = 0;
    return DMU_OK;
  }
  int p_cur = 0;
  for (int k = 0; k < steps; ++k) {
    const bool last = (k == steps - 1);
    const int p_next = (k == 0) ? 0 : 1 - p_cur;
    const int pin = p_cur == 0 ? FSLOT_PA : FSLOT_PB, pout = p_next == 0 ? FSLOT_PA : FSLOT_PB;
    for (size_t c = 0; c < p->classes.size(); ++c) {
      const int ci = (int)c;
      std::vector<SimtProblem> qs;
      qs.push_back(simt_gram(p, ci, FSLOT_G, FSLOT_G, co[2], co[1], FSLOT_G, FSLOT_R, k == 0 ? FSLOT_PA : -1, co[0]));
      if (!last) qs.push_back(simt_gram(p, ci, FSLOT_R, FSLOT_G, 1.f, co[0], FSLOT_G, FSLOT_T, -1, 0.f));
      if (k >= 1) qs.push_back(simt_gram(p, ci, FSLOT_R, pin, 1.f, co[0], pin, pout, -1, 0.f));
      if (!last) qs.push_back(simt_gram(p, ci, FSLOT_T, FSLOT_R, 1.f, co[0], FSLOT_T, FSLOT_G, -1, 0.f));
      for (auto& q : qs) {
        CUDA_TRY(launch_simt_gemm(q, s));
        p->launches++;
      }
    }
    p_cur = p_next;
  }
  p->p_final = p_cur;
  return DMU_OK;
}

dmu_status run_normalize(dmu_plan p, int tbl, bool with_mom, float beta, float gscale, float eps, bool vec,
                         cudaStream_t s) {
  const bool f32 = p->dtype == DMU_F32;
  const void* const* src = const_cast<const void* const*>(p->tbl_dev(tbl));
  float* const* moms = with_mom ? reinterpret_cast<float* const*>(p->tbl_dev(TBL_MOMS)) : nullptr;
  // bf16 plans: the image is fp16(2^e M) at the scale the previous call kept
  // for each matrix; matrices whose scale no longer fits (or that have none
  // yet) are rewritten by the fix-up pass, which reads M (or the gradient)
  CUDA_TRY(launch_momentum(p->chunks_dev(), (int)p->chunks.size(), p->mats_dev(), src, moms, f32 ? 1 : 0,
                           p->mb_dev(), f32 ? 1 : 0, beta, gscale, f32 ? nullptr : p->iscale_dev(),
                           f32 ? nullptr : p->fix_count_dev(), p->partial_dev(), vec ? 1 : 0, p->num_sms,
                           p->timeout_ns, p->status_dev(), s));
  CUDA_TRY(launch_norm_finalize(p->mats_dev(), p->count, p->partial_dev(), eps, p->inv_dev(),
                                f32 ? nullptr : p->iscale_dev(), f32 ? nullptr : p->invimg_dev(),
                                f32 ? nullptr : p->fix_dev(), f32 ? nullptr : p->fix_count_dev(), p->status_dev(),
                                s));
  p->launches += 2;
  if (!f32) {
    CUDA_TRY(launch_image_fix(p->chunks_dev(), (int)p->chunks.size(), p->mats_dev(), src, moms, gscale, p->mb_dev(),
                              p->iscale_dev(), p->fix_dev(), p->fix_count_dev(), vec ? 1 : 0, p->num_sms, s));
    p->launches++;
  }
  p->eps = eps;
  p->have_mb = true;
  p->have_p = false;
  return DMU_OK;
}

// Final O = P X0 GEMM fused with the weight update, bf16 path: one problem
// per shape bucket, launched per tile schedule; W and O come from the
// device pointer tables (TBL_W, TBL_O).
dmu_status final_launch(dmu_plan p, bool with_w, bool with_o, float lr, cudaStream_t s) {
  dmu_status st = DMU_OK;
  std::vector<Prob> probs;
  std::vector<int> scheds;
  const int pf_hi = p->p_final == 0 ? SLOT_PA_HI : SLOT_PB_HI;
  for (const Bucket& b : p->buckets) {
    const GClass& gc = p->classes[b.cls];
    if (p->tune_bucket >= 0 && &b != &p->buckets[p->tune_bucket]) continue;
    Prob pr;
    std::memset(&pr, 0, sizeof(pr));
    GemmProblem& g = pr.g;
    g.count = p->tune_count > 0 ? std::min(p->tune_count, b.count) : b.count;
    g.M = (int)b.m;
    g.N = (int)b.n;
    g.K = (int)b.m;
    g.sym = 0;
    g.tiles_per_mat = tiles_for(g.M, g.N, false, &g.tiles_m, &g.tiles_n);
    g.a_mn = 0;
    const bool f16 = gc.kind == KIND_F16;
    if (f16) {  // P in fp16 at scale 1, one MMA per K slice (hi only)
      g.a_z[0] = g.a_z[1] = pf_hi * gc.count + b.cls_off;
      g.terms = TERM_HH;
    } else {    // the fp16 hi/lo pair of the final-P area, two MMAs
      g.a_z[0] = b.cls_off;
      g.a_z[1] = gc.count + b.cls_off;
      g.terms = TERM_HH | TERM_LH;
    }
    g.b_mn = b.tall ? 0 : 1;
    g.epi = EPI_UPDATE;
    g.alpha = -lr * (float)std::sqrt(std::max(1.0, (double)b.rows / (double)b.cols));
    g.inv = p->inv_kernel();
    g.inv_base = b.first_slot;
    g.w_ptrs = with_w ? reinterpret_cast<void* const*>(p->tbl_dev(TBL_W)) : nullptr;
    g.o_ptrs = with_o ? reinterpret_cast<float* const*>(p->tbl_dev(TBL_O)) : nullptr;
    g.ptr_base = b.first_slot;
    g.w_f32 = 0;
    g.w_transposed = b.tall ? 1 : 0;
    g.w_cols = b.cols;
    pr.amap = f16 ? gc.map : gc.map_pf;
    pr.bmap = b.tall ? b.map_k : b.map_mn;
    if (gc.half) {
      g.half_a = 1;
      pr.amap_t = f16 ? gc.map_t : gc.map_pf_t;
    }
    probs.push_back(pr);
    scheds.push_back(p->final_sched(b));
  }
  for (int sched : TILE_SCHEDS) {
    std::vector<Prob> group;
    for (size_t i = 0; i < probs.size(); ++i)
      if (scheds[i] == sched) group.push_back(probs[i]);
    if (group.empty()) continue;
    st = run_tc(p, group, 2, 1, KIND_F16, sched, s);
    if (st != DMU_OK) return st;
  }
  return DMU_OK;
}

dmu_status encode_map(CUtensorMap* map, void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                      uint64_t s2, uint32_t box0, uint32_t box1,
                      CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = get_encode();
  if (!enc) return fail(DMU_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dt, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DMU_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return DMU_OK;
}

}  // namespace

namespace dmu {
// Lets entry points defined in other files report through dmu_last_error.
void set_last_error(const char* msg) { g_err = msg ? msg : ""; }
}  // namespace dmu

// =================================================================== C ABI
extern "C" {

int dmu_version(void) { return DMU_VERSION; }

const char* dmu_last_error(void) { return g_err.c_str(); }

dmu_status dmu_plan_create(const dmu_shape* shapes, int count, dmu_dtype dtype, dmu_prec prec, int device,
                           dmu_plan* out) {
  g_err.clear();
  if (!out) return fail(DMU_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!shapes) return fail(DMU_ERR_INVALID_ARG, "shapes is NULL");
  if (count <= 0) return fail(DMU_ERR_INVALID_ARG, "count must be positive");
  if (dtype != DMU_BF16 && dtype != DMU_F32) return fail(DMU_ERR_INVALID_ARG, "unknown dtype");
  if (prec < DMU_PREC_AUTO || prec > DMU_PREC_F16) return fail(DMU_ERR_INVALID_ARG, "unknown precision");
  for (int i = 0; i < count; ++i) {
    if (shapes[i].rows <= 0 || shapes[i].cols <= 0)
      return fail(DMU_ERR_INVALID_ARG, "non-positive extent at matrix " + std::to_string(i));
    if (shapes[i].rows > (1 << 20) || shapes[i].cols > (1 << 20) ||
        std::min(shapes[i].rows, shapes[i].cols) > 65536)
      return fail(DMU_ERR_UNSUPPORTED, "extent too large at matrix " + std::to_string(i));
  }
  dmu_plan p = new dmu_plan_s();
  p->device = device;
  p->dtype = dtype;
  p->prec = prec;
  p->count = count;
  p->shapes.assign(shapes, shapes + count);
  p->esize = dtype == DMU_BF16 ? 2 : 4;
  if (const char* e = std::getenv("DMU_CTA_PAIR")) p->sched = std::atoi(e) != 0 ? 1 : 0;
  if (const char* e = std::getenv("DMU_SCHEDULE")) {
    const int v = std::atoi(e);
    if (valid_sched(v) && v != SCHED_ONCHIP) p->sched = v;
  }
  if (const char* e = std::getenv("DMU_HALF")) p->half_store = std::atoi(e) != 0;

  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) == cudaSuccess && ndev > 0) {
    if (device < 0 || device >= ndev) {
      delete p;
      return fail(DMU_ERR_INVALID_ARG, "device index out of range");
    }
    int major = 0, minor = 0, sms = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
    if (dtype == DMU_BF16 && !(major == 10 && minor == 0)) {
      delete p;
      return fail(DMU_ERR_UNSUPPORTED, "the bf16 path is built for sm_100a (compute capability 10.0)");
    }
    p->has_device = true;
    p->num_sms = sms;
  } else {
    cudaGetLastError();  // clear "no device"
  }

  // buckets (equal rows, cols) in order of first appearance; classes (equal m)
  std::map<std::pair<int64_t, int64_t>, int> bidx;
  std::map<int64_t, int> cidx;
  for (int i = 0; i < count; ++i) {
    auto key = std::make_pair(shapes[i].rows, shapes[i].cols);
    auto it = bidx.find(key);
    if (it == bidx.end()) {
      Bucket b;
      b.rows = shapes[i].rows;
      b.cols = shapes[i].cols;
      b.tall = b.rows > b.cols;
      b.m = std::min(b.rows, b.cols);
      b.n = std::max(b.rows, b.cols);
      auto ci = cidx.find(b.m);
      if (ci == cidx.end()) {
        GClass g;
        g.m = b.m;
        g.ldg = dtype == DMU_BF16 ? round_up64(b.m, 8) : b.m;
        if (dtype == DMU_BF16) {
          if (prec == DMU_PREC_AUTO)
            g.prec = b.m >= 1024 ? DMU_PREC_F16 : DMU_PREC_SPLIT3;
          else
            g.prec = prec;
          g.kind = g.prec == DMU_PREC_TF32 ? KIND_TF32 : (g.prec == DMU_PREC_F16 ? KIND_F16 : KIND_BF16);
          g.half = g.kind != KIND_TF32 && p->half_store;
        }
        cidx[b.m] = (int)p->classes.size();
        p->classes.push_back(g);
      }
      b.cls = cidx[b.m];
      bidx[key] = (int)p->buckets.size();
      p->buckets.push_back(b);
      it = bidx.find(key);
    }
    p->buckets[it->second].mats.push_back(i);
  }
  // DMU_ONCHIP=1: classes the on-chip recursion covers (split-bf16
  // precision, m <= 128) start on that schedule
  if (const char* e = std::getenv("DMU_ONCHIP")) {
    if (std::atoi(e) != 0)
      for (GClass& g : p->classes)
        if (onchip_eligible(dtype, g)) g.sched = SCHED_ONCHIP;
  }
  p->slot_of.assign(count, 0);
  int slot = 0;
  int64_t mb_elems = 0;
  for (Bucket& b : p->buckets) {
    b.count = (int)b.mats.size();
    b.first_slot = slot;
    for (int k = 0; k < b.count; ++k) p->slot_of[b.mats[k]] = slot + k;
    slot += b.count;
    GClass& g = p->classes[b.cls];
    b.cls_off = g.count;
    g.count += b.count;
    b.ldc = dtype == DMU_BF16 ? round_up64(b.cols, 8) : b.cols;
    if (b.cols % 8) p->vec_shapes = false;
    b.mb_off = mb_elems;
    mb_elems += round_up64((int64_t)b.count * b.rows * b.ldc, 128);
  }
  // momentum chunks and per-slot geometry
  p->mats.resize(count);
  for (const Bucket& b : p->buckets) {
    for (int k = 0; k < b.count; ++k) {
      MomMat mm;
      mm.rows = b.rows;
      mm.cols = b.cols;
      mm.ldc = b.ldc;
      mm.mb_off = b.mb_off + (int64_t)k * b.rows * b.ldc;
      mm.chunk_begin = (int)p->chunks.size();
      const int64_t total = b.rows * b.cols;
      for (int64_t st = 0; st < total; st += MOM_CHUNK) {
        MomChunk ch;
        ch.start = st;
        ch.slot = b.first_slot + k;
        ch.len = (int)std::min<int64_t>(MOM_CHUNK, total - st);
        p->chunks.push_back(ch);
      }
      mm.chunk_end = (int)p->chunks.size();
      p->mats[b.first_slot + k] = mm;
    }
  }
  // workspace layout
  size_t off = 0;
  p->off_status = off;
  off = align_up(off + 16, 256);
  p->off_inv = off;
  off = align_up(off + sizeof(float) * count, 256);
  p->off_iscale = off;
  off = align_up(off + sizeof(float) * count, 256);
  p->off_invimg = off;
  off = align_up(off + sizeof(float) * count, 256);
  p->off_fix = off;
  off = align_up(off + sizeof(int) * (count + 1), 256);
  p->off_partial = off;
  off = align_up(off + sizeof(float) * MOM_PARTIALS_PER_CHUNK * p->chunks.size(), 256);
  p->off_chunks = off;
  off = align_up(off + sizeof(MomChunk) * p->chunks.size(), 256);
  p->off_mats = off;
  off = align_up(off + sizeof(MomMat) * count, 256);
  p->off_tbl = off;
  off = align_up(off + sizeof(void*) * NUM_TBL * (size_t)count, 256);
  p->off_mb = off;
  off = align_up(off + p->esize * (size_t)mb_elems, 1024);
  p->off_gram = off;
  for (GClass& g : p->classes) {
    g.off = off;
    const size_t elems = (size_t)g.count * g.m * g.ldg;
    if (dtype == DMU_F32) {
      off = align_up(off + 4 * (size_t)NUM_FSLOTS * elems, 1024);
    } else if (g.kind == KIND_TF32) {
      off = align_up(off + 4 * (size_t)NUM_FSLOTS * elems, 1024);
      g.off_pf = off;
      off = align_up(off + 2 * 2 * elems, 1024);
    } else if (g.kind == KIND_F16) {  // its final P stays in its fp16 P slots
      off = align_up(off + 2 * (size_t)NUM_SLOTS * elems, 1024);
    } else {
      off = align_up(off + 2 * (size_t)NUM_SLOTS * elems, 1024);
      g.off_pf = off;
      off = align_up(off + 2 * 2 * elems, 1024);
    }
  }
  p->total = off;
  *out = p;
  return DMU_OK;
}

size_t dmu_workspace_bytes(dmu_plan plan) { return plan ? plan->total : 0; }

dmu_status dmu_set_workspace(dmu_plan p, void* dev_ptr, size_t bytes) {
  g_err.clear();
  dmu_status st = check_plan(p, false);
  if (st != DMU_OK) return st;
  if (!p->has_device) return fail(DMU_ERR_CUDA, "no CUDA device");
  if (!dev_ptr) return fail(DMU_ERR_WORKSPACE, "workspace pointer is NULL");
  if (reinterpret_cast<uintptr_t>(dev_ptr) & 255) return fail(DMU_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (bytes < p->total)
    return fail(DMU_ERR_WORKSPACE, "workspace too small: " + std::to_string(bytes) + " < " + std::to_string(p->total));
  DevGuard dg(p->device);
  p->ws = reinterpret_cast<char*>(dev_ptr);
  p->ws_bytes = bytes;
  for (int t = 0; t < NUM_TBL; ++t) p->tbl_valid[t] = false;
  p->have_mb = p->have_p = false;
  CUDA_TRY(cudaMemset(p->ws + p->off_status, 0, 16));
  // no image scale yet: the first momentum call writes every image in its fix-up pass
  CUDA_TRY(cudaMemset(p->ws + p->off_iscale, 0, sizeof(float) * p->count));
  CUDA_TRY(cudaMemcpy(p->ws + p->off_chunks, p->chunks.data(), sizeof(MomChunk) * p->chunks.size(),
                      cudaMemcpyHostToDevice));
  CUDA_TRY(cudaMemcpy(p->ws + p->off_mats, p->mats.data(), sizeof(MomMat) * p->mats.size(),
                      cudaMemcpyHostToDevice));
  p->maps.clear();
  if (p->dtype == DMU_BF16) {
    CUDA_TRY(gemm_tc_configure());
    CUDA_TRY(onchip_configure());
    CUDA_TRY(momentum_configure());
    for (Bucket& b : p->buckets) {
      CUtensorMap mk, mn;
      void* base = p->mb_dev() + 2 * (size_t)b.mb_off;
      const uint64_t s1 = (uint64_t)b.ldc * 2, s2 = (uint64_t)b.rows * b.ldc * 2;
      // the image is read as fp16 (2^e M, converted in place after the norm)
      st = encode_map(&mk, base, (uint64_t)b.cols, (uint64_t)b.rows, (uint64_t)b.count, s1, s2, 64, 128,
                      CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
      if (st != DMU_OK) return st;
      st = encode_map(&mn, base, (uint64_t)b.cols, (uint64_t)b.rows, (uint64_t)b.count, s1, s2, 64, 64,
                      CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
      if (st != DMU_OK) return st;
      b.map_k = (int)p->maps.size();
      p->maps.push_back(mk);
      b.map_mn = (int)p->maps.size();
      p->maps.push_back(mn);
    }
    for (GClass& g : p->classes) {
      CUtensorMap mg;
      if (g.kind == KIND_TF32) {
        const uint64_t s1 = (uint64_t)g.ldg * 4, s2 = (uint64_t)g.m * g.ldg * 4;
        st = encode_map(&mg, p->ws + g.off, (uint64_t)g.m, (uint64_t)g.m, (uint64_t)NUM_FSLOTS * g.count, s1,
                        s2, 32, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
        if (st != DMU_OK) return st;
        g.map = (int)p->maps.size();
        p->maps.push_back(mg);
        CUtensorMap mp;
        const uint64_t t1 = (uint64_t)g.ldg * 2, t2 = (uint64_t)g.m * g.ldg * 2;
        st = encode_map(&mp, p->ws + g.off_pf, (uint64_t)g.m, (uint64_t)g.m, (uint64_t)2 * g.count, t1, t2, 64,
                        128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
        if (st != DMU_OK) return st;
        g.map_pf = (int)p->maps.size();
        p->maps.push_back(mp);
      } else {
        const uint64_t s1 = (uint64_t)g.ldg * 2, s2 = (uint64_t)g.m * g.ldg * 2;
        const CUtensorMapDataType dt =
            g.kind == KIND_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        st = encode_map(&mg, p->ws + g.off, (uint64_t)g.m, (uint64_t)g.m, (uint64_t)NUM_SLOTS * g.count, s1,
                        s2, 64, 128, dt);
        if (st != DMU_OK) return st;
        g.map = (int)p->maps.size();
        p->maps.push_back(mg);
        CUtensorMap mt;  // transposed reads of half-stored blocks
        st = encode_map(&mt, p->ws + g.off, (uint64_t)g.m, (uint64_t)g.m, (uint64_t)NUM_SLOTS * g.count, s1,
                        s2, 64, 64, dt);
        if (st != DMU_OK) return st;
        g.map_t = (int)p->maps.size();
        p->maps.push_back(mt);
        if (g.kind != KIND_F16) {  // the fp16 final-P pair of bf16-pair classes (half-stored)
          CUtensorMap mp, mpt;
          st = encode_map(&mp, p->ws + g.off_pf, (uint64_t)g.m, (uint64_t)g.m, (uint64_t)2 * g.count, s1, s2, 64,
                          128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
          if (st != DMU_OK) return st;
          g.map_pf = (int)p->maps.size();
          p->maps.push_back(mp);
          st = encode_map(&mpt, p->ws + g.off_pf, (uint64_t)g.m, (uint64_t)g.m, (uint64_t)2 * g.count, s1, s2, 64,
                          64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
          if (st != DMU_OK) return st;
          g.map_pf_t = (int)p->maps.size();
          p->maps.push_back(mpt);
        }
      }
    }
  }
  return DMU_OK;
}

dmu_status dmu_momentum_normalize(dmu_plan p, const void* const* grads, float* const* momenta, float beta,
                                  float grad_scale, float eps, void* stream) {
  g_err.clear();
  dmu_status st = check_plan(p, true);
  if (st != DMU_OK) return st;
  if (!grads) return fail(DMU_ERR_INVALID_ARG, "grads is NULL");
  if (!(eps >= 0.f) || !std::isfinite(beta) || !std::isfinite(grad_scale))
    return fail(DMU_ERR_INVALID_ARG, "eps must be >= 0, beta and grad_scale finite");
  DevGuard dg(p->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  p->launches = 0;
  st = upload_table(p, TBL_GRADS, grads, s);
  if (st != DMU_OK) return st;
  bool vec = p->vec_shapes && aligned16(grads, p->count);
  if (momenta) {
    st = upload_table(p, TBL_MOMS, reinterpret_cast<const void* const*>(momenta), s);
    if (st != DMU_OK) return st;
    vec = vec && aligned16(reinterpret_cast<const void* const*>(momenta), p->count);
  }
  return run_normalize(p, TBL_GRADS, momenta != nullptr, beta, grad_scale, eps, vec, s);
}

dmu_status dmu_gram_ns_batched(dmu_plan p, const void* const* ptrs, const dmu_shape* shapes, int count,
                               const float coeffs[3], int steps, void* stream) {
  g_err.clear();
  dmu_status st = check_plan(p, true);
  if (st != DMU_OK) return st;
  if (!shapes || !coeffs) return fail(DMU_ERR_INVALID_ARG, "shapes or coeffs is NULL");
  if (count != p->count) return fail(DMU_ERR_NOT_PLANNED, "count differs from the plan");
  for (int i = 0; i < count; ++i)
    if (shapes[i].rows != p->shapes[i].rows || shapes[i].cols != p->shapes[i].cols)
      return fail(DMU_ERR_NOT_PLANNED, "shape of matrix " + std::to_string(i) + " differs from the plan");
  if (steps < 0 || steps > 64) return fail(DMU_ERR_INVALID_ARG, "steps must be in [0, 64]");
  for (int k = 0; k < 3; ++k)
    if (!std::isfinite(coeffs[k])) return fail(DMU_ERR_INVALID_ARG, "coefficients must be finite");
  DevGuard dg(p->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  p->launches = 0;
  if (ptrs) {
    st = upload_table(p, TBL_IN, ptrs, s);
    if (st != DMU_OK) return st;
    st = run_normalize(p, TBL_IN, false, 0.f, 1.f, p->eps, p->vec_shapes && aligned16(ptrs, p->count), s);
    if (st != DMU_OK) return st;
  } else if (!p->have_mb) {
    return fail(DMU_ERR_NOT_PLANNED, "no input: call dmu_momentum_normalize first or pass ptrs");
  }
  st = p->dtype == DMU_BF16 ? gram_bf16(p, coeffs, steps, s) : gram_f32(p, coeffs, steps, s);
  if (st != DMU_OK) return st;
  p->have_p = true;
  return DMU_OK;
}

dmu_status dmu_apply_update(dmu_plan p, void* const* weights, float lr, float* const* out_o, void* stream) {
  g_err.clear();
  dmu_status st = check_plan(p, true);
  if (st != DMU_OK) return st;
  if (!p->have_p) return fail(DMU_ERR_NOT_PLANNED, "call dmu_gram_ns_batched first");
  if (!std::isfinite(lr)) return fail(DMU_ERR_INVALID_ARG, "lr must be finite");
  DevGuard dg(p->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  p->launches = 0;
  if (weights) {
    st = upload_table(p, TBL_W, reinterpret_cast<const void* const*>(weights), s);
    if (st != DMU_OK) return st;
  }
  if (out_o) {
    st = upload_table(p, TBL_O, reinterpret_cast<const void* const*>(out_o), s, true);
    if (st != DMU_OK) return st;
  }
  if (!weights && !out_o) return DMU_OK;
  if (p->dtype == DMU_BF16) return final_launch(p, weights != nullptr, out_o != nullptr, lr, s);
  const int pf = p->p_final == 0 ? FSLOT_PA : FSLOT_PB;
  for (const Bucket& b : p->buckets) {
    const GClass& gc = p->classes[b.cls];
    SimtProblem q;
    std::memset(&q, 0, sizeof(q));
    q.count = b.count;
    q.M = (int)b.m;
    q.N = (int)b.n;
    q.K = (int)b.m;
    q.a = p->slot_f32(b.cls, pf) + (size_t)b.cls_off * gc.m * gc.ldg;
    q.a_ms = gc.m * gc.ldg;
    q.a_si = gc.ldg;
    q.a_sk = 1;
    q.b = reinterpret_cast<const float*>(p->mb_dev()) + b.mb_off;
    q.b_ms = b.rows * b.ldc;
    q.b_si = b.tall ? b.ldc : 1;
    q.b_sk = b.tall ? 1 : b.ldc;
    q.epi = EPI_UPDATE;
    q.alpha = -lr * (float)std::sqrt(std::max(1.0, (double)b.rows / (double)b.cols));
    q.alpha_mode = ALPHA_INV;
    q.inv = p->inv_dev();
    q.inv_base = b.first_slot;
    q.w_ptrs = weights ? reinterpret_cast<void* const*>(p->tbl_dev(TBL_W)) : nullptr;
    q.o_ptrs = out_o ? reinterpret_cast<float* const*>(p->tbl_dev(TBL_O)) : nullptr;
    q.ptr_base = b.first_slot;
    q.w_f32 = 1;
    q.w_transposed = b.tall ? 1 : 0;
    q.w_cols = b.cols;
    CUDA_TRY(launch_simt_gemm(q, s));
    p->launches++;
  }
  return DMU_OK;
}

dmu_status dmu_read_status(dmu_plan p, uint32_t* flags) {
  g_err.clear();
  dmu_status st = check_plan(p, true);
  if (st != DMU_OK) return st;
  DevGuard dg(p->device);
  unsigned int v = 0;
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(cudaMemcpy(&v, p->status_dev(), sizeof(v), cudaMemcpyDeviceToHost));
  CUDA_TRY(cudaMemset(p->status_dev(), 0, sizeof(v)));
  if (flags) *flags = v;
  if (v & DMU_FLAG_TIMEOUT) return fail(DMU_ERR_TIMEOUT, "a device wait timed out");
  if (v & DMU_FLAG_NONFINITE) return fail(DMU_ERR_NONFINITE, "a momentum norm is not finite");
  return DMU_OK;
}

dmu_status dmu_debug_gram(dmu_plan p, int which, int index, float* out, void* stream) {
  g_err.clear();
  dmu_status st = check_plan(p, true);
  if (st != DMU_OK) return st;
  if (!out) return fail(DMU_ERR_INVALID_ARG, "out is NULL");
  if (which < 0 || which > 9) return fail(DMU_ERR_INVALID_ARG, "which must be in [0, 9]");
  if (which < 6 && (index < 0 || index >= p->count)) return fail(DMU_ERR_INVALID_ARG, "index out of range");
  if (which == 7 && (index < 0 || index >= p->count)) return fail(DMU_ERR_INVALID_ARG, "index out of range");
  DevGuard dg(p->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (which == 8) {
    // bounded-wait self-test: wait `index` microseconds on a barrier nothing completes
    if (index < 1 || index > 1000000) return fail(DMU_ERR_INVALID_ARG, "self-test wait must be 1..1e6 us");
    CUDA_TRY(launch_wait_selftest(p->status_dev(), 1000LL * index, s));
    CUDA_TRY(cudaStreamSynchronize(s));
    return DMU_OK;
  }
  if (which == 6 || which == 9) {
    const float* src = which == 6 ? p->inv_dev() : p->iscale_dev();
    if (which == 9 && p->dtype != DMU_BF16) return fail(DMU_ERR_INVALID_ARG, "fp32 plans keep no image scale");
    CUDA_TRY(cudaMemcpyAsync(out, src, sizeof(float) * p->count, cudaMemcpyDeviceToDevice, s));
    CUDA_TRY(cudaStreamSynchronize(s));
    return DMU_OK;
  }
  const int slot = p->slot_of[index];
  const Bucket* bk = nullptr;
  for (const Bucket& b : p->buckets)
    if (slot >= b.first_slot && slot < b.first_slot + b.count) bk = &b;
  const int local = slot - bk->first_slot;
  if (which == 5) {
    const MomMat& mm = p->mats[slot];
    if (p->dtype == DMU_BF16) {  // the fp16 image 2^e M, scaled back
      float sc = 1.f;
      CUDA_TRY(cudaMemcpyAsync(&sc, p->iscale_dev() + slot, sizeof(float), cudaMemcpyDeviceToHost, s));
      CUDA_TRY(cudaStreamSynchronize(s));
      CUDA_TRY(launch_pair_h_to_f32(reinterpret_cast<const uint16_t*>(p->mb_dev()) + mm.mb_off, nullptr, mm.rows,
                                    mm.cols, mm.ldc, 1.f / sc, out, s));
    } else {
      CUDA_TRY(launch_f32_copy2d(reinterpret_cast<const float*>(p->mb_dev()) + mm.mb_off, mm.rows, mm.cols,
                                 mm.ldc, out, s));
    }
    CUDA_TRY(cudaStreamSynchronize(s));
    return DMU_OK;
  }
  const GClass& gc = p->classes[bk->cls];
  if (which <= 4 && p->onchip(bk->cls))
    return fail(DMU_ERR_NOT_PLANNED, "matrix " + std::to_string(index) +
                                         " runs its recursion on chip: only the final P (which 7) is kept");
  const size_t moff = (size_t)(bk->cls_off + local) * gc.m * gc.ldg;
  int q = which;
  if (which == 7) q = p->p_final == 0 ? 3 : 4;
  const int hf = gc.half ? 1 : 0;
  if (p->dtype == DMU_BF16 && which == 7 && gc.kind != KIND_F16) {
    // the final P of other classes: the fp16 pair in the final-P area
    CUDA_TRY(launch_pair_h_to_f32(p->pf_bf16(bk->cls, 0) + moff, p->pf_bf16(bk->cls, 1) + moff, gc.m, gc.m, gc.ldg,
                                  1.f, out, s, hf));
  } else if (p->dtype == DMU_BF16 && gc.kind == KIND_F16) {
    {
      const int slots[5] = {SLOT_G_HI, SLOT_R_HI, SLOT_T_HI, SLOT_PA_HI, SLOT_PB_HI};
      const int sh = slots[q];
      CUDA_TRY(launch_pair_h_to_f32(p->slot_bf16(bk->cls, sh) + moff,
                                    sh == SLOT_R_HI ? nullptr : p->slot_bf16(bk->cls, sh + 1) + moff, gc.m, gc.m,
                                    gc.ldg, 1.f / half_slot_scale(sh), out, s, hf));
    }
  } else if (p->dtype == DMU_BF16 && gc.kind == KIND_TF32) {
    CUDA_TRY(launch_f32_copy2d(p->slot_f32(bk->cls, q) + moff, gc.m, gc.m, gc.ldg, out, s));
  } else if (p->dtype == DMU_BF16) {
    const int slots[5] = {SLOT_G_HI, SLOT_R_HI, SLOT_T_HI, SLOT_PA_HI, SLOT_PB_HI};
    const int sh = slots[q];
    const bool has_lo = !(sh == SLOT_R_HI && gc.prec == DMU_PREC_FAST);
    CUDA_TRY(launch_pair_to_f32(p->slot_bf16(bk->cls, sh) + moff,
                                has_lo ? p->slot_bf16(bk->cls, sh + 1) + moff : nullptr, gc.m, gc.m, gc.ldg,
                                out, s, hf));
  } else {
    CUDA_TRY(launch_f32_copy2d(p->slot_f32(bk->cls, q) + moff, gc.m, gc.m, gc.ldg, out, s));
  }
  CUDA_TRY(cudaStreamSynchronize(s));
  return DMU_OK;
}

int dmu_last_launch_count(dmu_plan p) { return p ? p->launches : 0; }

// Schedule cache (DMuon page, section 2.4: kernel configurations are tuned
// per shape and cached).  Every Gram class (equal m) and every bucket's
// final GEMM gets its own entry, keyed by the device, the precision and the
// shapes it covers, so plans that share a class or a bucket share the
// entry.
static std::string device_tag(dmu_plan p) {
  cudaDeviceProp prop;
  std::memset(&prop, 0, sizeof(prop));
  cudaGetDeviceProperties(&prop, p->device);
  std::string name = prop.name;
  for (char& c : name)
    if (c == ' ') c = '_';
  std::ostringstream k;
  k << name << "/sm" << prop.multiProcessorCount;
  return k.str();
}

static std::string class_key(dmu_plan p, const std::string& dev, int c) {
  const GClass& g = p->classes[c];
  std::ostringstream k;
  k << dev << "/gram/m" << g.m << "/p" << g.prec << "/n" << g.count << "/";
  for (const Bucket& b : p->buckets)
    if (b.cls == c) k << b.rows << "x" << b.cols << "*" << b.count << ",";
  return k.str();
}

static std::string final_key(dmu_plan p, const std::string& dev, const Bucket& b) {
  std::ostringstream k;
  k << dev << "/final/" << b.rows << "x" << b.cols << "/n" << b.count << "/p" << p->classes[b.cls].prec;
  return k.str();
}

static std::string syrk_key(dmu_plan p, const std::string& dev, const Bucket& b) {
  std::ostringstream k;
  k << dev << "/syrk/" << b.rows << "x" << b.cols << "/n" << b.count << "/p" << p->classes[b.cls].prec;
  return k.str();
}

static std::map<std::string, int> read_cache(const char* path) {
  std::map<std::string, int> out;
  if (!path) return out;
  std::ifstream in(path);
  std::string line;
  while (std::getline(in, line)) {
    std::istringstream ls(line);
    std::string k;
    int v = -1;
    if ((ls >> k >> v) && valid_sched(v)) out[k] = v;
  }
  return out;
}

int dmu_get_schedule(dmu_plan p) { return p ? p->sched : -1; }

int dmu_get_gram_schedule(dmu_plan p, int index) {
  if (!p || index < 0 || index >= p->count) return -1;
  for (const Bucket& b : p->buckets)
    for (int i : b.mats)
      if (i == index) return p->class_sched(b.cls);
  return -1;
}

int dmu_get_final_schedule(dmu_plan p, int index) {
  if (!p || index < 0 || index >= p->count) return -1;
  for (const Bucket& b : p->buckets)
    for (int i : b.mats)
      if (i == index) return p->final_sched(b);
  return -1;
}

int dmu_get_syrk_schedule(dmu_plan p, int index) {
  if (!p || index < 0 || index >= p->count) return -1;
  for (const Bucket& b : p->buckets)
    for (int i : b.mats)
      if (i == index) return p->onchip(b.cls) ? SCHED_ONCHIP : (b.ssched >= 0 ? b.ssched : p->class_sched(b.cls));
  return -1;
}

dmu_status dmu_autotune(dmu_plan p, const char* cache_path, void* stream) {
  g_err.clear();
  dmu_status st = check_plan(p, true);
  if (st != DMU_OK) return st;
  if (!p->have_mb) return fail(DMU_ERR_NOT_PLANNED, "call dmu_momentum_normalize before dmu_autotune");
  if (p->dtype != DMU_BF16) return DMU_OK;  // one schedule on the fp32 path
  DevGuard dg(p->device);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const std::string dev = device_tag(p);
  std::map<std::string, int> cache = read_cache(cache_path);
  std::vector<std::string> lines;
  const float co[3] = {3.4445f, -4.7750f, 2.0315f};
  cudaEvent_t e0, e1;
  CUDA_TRY(cudaEventCreate(&e0));
  CUDA_TRY(cudaEventCreate(&e1));
  // best of three timed runs after one warm-up; a failed run leaves `st` set
  auto time_min = [&](auto&& run) -> float {
    float best = 0.f;
    st = run();
    for (int rep = 0; st == DMU_OK && rep < 3; ++rep) {
      cudaEventRecord(e0, s);
      st = run();
      cudaEventRecord(e1, s);
      if (cudaEventSynchronize(e1) != cudaSuccess) {
        st = fail(DMU_ERR_CUDA, "autotune: event synchronisation failed");
        break;
      }
      float t = 0.f;
      cudaEventElapsedTime(&t, e0, e1);
      best = rep == 0 ? t : std::min(best, t);
    }
    return best;
  };
  const int saved_launches = p->launches;

  // ---- Gram recursion, one class at a time (CTA pairs first: they win ties)
  for (size_t c = 0; st == DMU_OK && c < p->classes.size(); ++c) {
    GClass& g = p->classes[c];
    const std::string key = class_key(p, dev, (int)c);
    auto hit = cache.find(key);
    if (hit != cache.end() && (hit->second != SCHED_ONCHIP || onchip_eligible(p->dtype, g))) {
      g.sched = hit->second;
      continue;
    }
    std::vector<int> cand = {1, 0, 2};
    if (g.kind == KIND_F16) {  // stage-depth variants of the CTA-pair fp16 kernel
      cand.push_back(4);
      cand.push_back(5);
    }
    if (onchip_eligible(p->dtype, g)) cand.push_back(SCHED_ONCHIP);
    std::ostringstream times;
    int best = -1;
    float best_ms = 0.f;
    p->tune_class = (int)c;
    for (int sc : cand) {
      g.sched = sc;
      const float ms = time_min([&] { return gram_bf16(p, co, 5, s); });
      if (st != DMU_OK) break;
      times << " s" << sc << "_ms=" << ms;
      if (best < 0 || ms < best_ms) {
        best = sc;
        best_ms = ms;
      }
    }
    p->tune_class = -1;
    if (st != DMU_OK) break;
    g.sched = best;
    cache[key] = best;
    lines.push_back(key + " " + std::to_string(best) + times.str());
  }
  // ---- SYRK of every bucket off the on-chip schedule: its class's tile
  // schedule, or the 256 x 512 CTA-pair tile, whose epilogue does not
  // overlap the next tile but whose operands cost a quarter less per MMA
  // (the long K of a wide or tall bucket amortises the epilogue)
  for (size_t bi = 0; st == DMU_OK && bi < p->buckets.size(); ++bi) {
    Bucket& b = p->buckets[bi];
    const GClass& g = p->classes[b.cls];
    if (p->onchip(b.cls)) continue;
    const std::string key = syrk_key(p, dev, b);
    auto hit = cache.find(key);
    if (hit != cache.end() && hit->second != SCHED_ONCHIP) {
      b.ssched = hit->second;
      continue;
    }
    std::ostringstream times;
    int best = -1;
    float best_ms = 0.f;
    p->tune_class = b.cls;
    p->tune_syrk = (int)bi;
    // candidates: the class's own schedule first (it wins ties), then the
    // single-CTA tiles, the three-stage CTA pairs and the 256 x 512 pairs
    // (measured alone on long-K SYRKs: 2 K atoms x 3 stages and single CTAs
    // can beat the class's choice, which is tuned for the products' epilogue)
    const int own = p->class_sched(b.cls);
    std::vector<int> cand = {own};
    for (int sc : {0, 4, SCHED_WIDE})
      if (sc != own) cand.push_back(sc);
    for (int sc : cand) {
      b.ssched = sc;
      const float ms = time_min([&] { return gram_bf16(p, co, 0, s); });
      if (st != DMU_OK) break;
      times << " s" << sc << "_ms=" << ms;
      if (best < 0 || ms < best_ms) {
        best = sc;
        best_ms = ms;
      }
    }
    p->tune_class = -1;
    p->tune_syrk = -1;
    if (st != DMU_OK) break;
    (void)g;
    b.ssched = best;
    cache[key] = best;
    lines.push_back(key + " " + std::to_string(best) + times.str());
  }
  // the recursion once more with every class on its schedule: P_K for all
  if (st == DMU_OK) st = gram_bf16(p, co, 5, s);

  // ---- final GEMM + update, one bucket at a time.  Its weight writes go to
  // the class's G, R and T slots (free after the recursion), never to the
  // caller's weights; when they cannot hold the whole bucket, the first
  // matrices that fit are timed.
  for (size_t bi = 0; st == DMU_OK && bi < p->buckets.size(); ++bi) {
    Bucket& b = p->buckets[bi];
    const GClass& g = p->classes[b.cls];
    const std::string key = final_key(p, dev, b);
    auto hit = cache.find(key);
    if (hit != cache.end() && hit->second != SCHED_ONCHIP) {
      b.fsched = hit->second;
      continue;
    }
    const size_t free_bytes = (size_t)12 * g.count * g.m * g.ldg;  // slots G, R, T of the class
    const size_t w_bytes = align_up((size_t)b.rows * b.cols * 2, 256);
    const int n = (int)std::min<size_t>((size_t)b.count, free_bytes / w_bytes);
    if (n == 0) continue;
    std::vector<const void*> wt(p->count, nullptr);
    char* area = p->ws + g.off;
    for (int k = 0; k < n; ++k) wt[b.mats[k]] = area + (size_t)k * w_bytes;
    st = upload_table(p, TBL_W, wt.data(), s, true);
    if (st != DMU_OK) break;
    p->tune_bucket = (int)bi;
    p->tune_count = n;
    std::ostringstream times;
    int best = -1;
    float best_ms = 0.f;
    for (int sc : {1, 0, 2}) {
      b.fsched = sc;
      const float ms = time_min([&] { return final_launch(p, true, false, 0.f, s); });
      if (st != DMU_OK) break;
      times << " s" << sc << "_ms=" << ms;
      if (best < 0 || ms < best_ms) {
        best = sc;
        best_ms = ms;
      }
    }
    p->tune_bucket = -1;
    p->tune_count = 0;
    p->tbl_valid[TBL_W] = false;  // the caller's table is uploaded again by the next update
    if (st != DMU_OK) break;
    b.fsched = best;
    cache[key] = best;
    lines.push_back(key + " " + std::to_string(best) + times.str() + " timed_matrices=" + std::to_string(n));
  }
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  p->launches = saved_launches;
  if (st != DMU_OK) return st;
  p->have_p = true;  // P_K of the quintic K = 5 recursion on every class
  if (cache_path && !lines.empty()) {
    std::ofstream out(cache_path, std::ios::app);
    for (const std::string& l : lines) out << l << "\n";
  }
  return DMU_OK;
}

void dmu_plan_destroy(dmu_plan p) {
  if (!p) return;
  for (int t = 0; t < NUM_TBL; ++t) {
    if (p->tbl_ev[t]) {
      cudaEventSynchronize(p->tbl_ev[t]);
      cudaEventDestroy(p->tbl_ev[t]);
    }
    if (p->pinned[t]) cudaFreeHost(p->pinned[t]);
  }
  delete p;
}

}  // extern "C"
