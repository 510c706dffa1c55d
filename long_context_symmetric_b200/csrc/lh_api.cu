// Host side of the liblh C ABI: sizes, argument validation, launches.
// Every entry point validates everything before it launches anything, never
// allocates, never synchronises (except lh_get_device_error) and reports
// launch failures as LH_ERR_CUDA.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "lh_common.cuh"

#ifndef LH_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

namespace lh {

// NVTX range over one entry point (named like the entry point), so a profiler
// timeline shows each step of the path with the kernels it launched. The
// header-only NVTX costs a branch when no tool is attached; building with
// -DLH_NO_NVTX removes it.
struct NvtxRange {
#ifndef LH_NO_NVTX
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
#else
  explicit NvtxRange(const char*) {}
#endif
};
#define LH_RANGE(name) ::lh::NvtxRange lh_nvtx_range_(name)

// Device error word: [0] = lh_status, [1] = kernel-specific detail. Kernels with
// bounded waits write it (first writer wins) instead of trapping.
__device__ int g_dev_error[2];

static std::atomic<unsigned long long> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((unsigned long long)n); }

cudaError_t launch_attn_fwd_simt(const Geom& g, lh_dtype dt, const void* qs, const void* ks,
                                 const void* vs, float* os, float* lse, cudaStream_t s);
cudaError_t launch_attn_bwd_simt(const Geom& g, lh_dtype dt, const void* qs, const void* ks,
                                 const void* vs, const void* dos, const float* lse,
                                 const float* delta, float* dqs, float* dks, float* dvs,
                                 cudaStream_t s);

cudaError_t launch_attn_fwd_tc(const Geom& g, const void* qs, const void* ks, const void* vs,
                               float* os, float* lse, const int* seg, const uint32_t* scale, int* err,
                               cudaStream_t s);

// bf16 I/O runs on the tcgen05 tensor-core kernels (fp16 operands); fp32 on
// the fp32 SIMT kernels. LH_ATTN_SIMT=1 in the environment routes bf16 I/O
// through the SIMT kernels too (a debugging aid).
static bool force_simt() {
  const char* e = std::getenv("LH_ATTN_SIMT");
  return e && e[0] == '1';
}

cudaError_t launch_attn_fwd(const Geom& g, lh_dtype dt, const void* qs, const void* ks,
                            const void* vs, float* os, float* lse, const uint32_t* scale, int* err,
                            cudaStream_t s) {
  if (dt == LH_BF16 && !force_simt()) return launch_attn_fwd_tc(g, qs, ks, vs, os, lse, nullptr, scale, err, s);
  return launch_attn_fwd_simt(g, dt, qs, ks, vs, os, lse, s);
}

cudaError_t launch_attn_bwd_tc(const Geom& g, const void* qs, const void* ks, const void* vs,
                               const void* dos, const float* lse, const float* delta, float* dqs,
                               float* dks, float* dvs, const int* seg, const uint32_t* amax, int* err,
                               cudaStream_t s);
cudaError_t launch_selftest_wait(long long limit_cycles, int* err, int* gave_up, cudaStream_t s);
cudaError_t launch_selftest_exp2(const float* x, float* y_fma, float* y_sfu, int n, cudaStream_t s);

cudaError_t launch_attn_bwd(const Geom& g, lh_dtype dt, const void* qs, const void* ks,
                            const void* vs, const void* dos, const float* lse, const float* delta,
                            const uint32_t* scale, float* dqs, float* dks, float* dvs, int* err, cudaStream_t s) {
  if (dt == LH_BF16 && !force_simt())
    return launch_attn_bwd_tc(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, nullptr, scale, err, s);
  return launch_attn_bwd_simt(g, dt, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, s);
}

namespace {

constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {nullptr};

// Device address of g_dev_error on the current device (looked up once per device).
int* device_error_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = (int*)p;
  }
  return g_err_ptr[dev];
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

lh_status make_geom(const lh_config* cfg, Geom* g, lh_plan_t* out) {
  if (!cfg) return LH_ERR_NULL;
  if (cfg->dtype != LH_BF16 && cfg->dtype != LH_FP32) return LH_ERR_DTYPE;
  if (cfg->accum != LH_ACC_FP32 && cfg->accum != LH_ACC_FIXED64) return LH_ERR_MODE;
  if ((unsigned)cfg->score > LH_SCORE_MAXPOOL || (unsigned)cfg->ties > LH_TIES_HIGH_FIRST ||
      (unsigned)cfg->order > LH_ORDER_PRE || (unsigned)cfg->weight > LH_WEIGHT_MEAN ||
      (unsigned)cfg->inclusion > LH_INCL_PARTITION)
    return LH_ERR_MODE;
  const int B = cfg->B, H = cfg->H, N = cfg->N, D = cfg->D, p = cfg->p, L = cfg->L, K = cfg->K;
  if (B < 1 || H < 1 || N < 1) return LH_ERR_SHAPE;
  if (D != 64 && D != 128) return LH_ERR_SHAPE;
  if (p < 2 || L < 1 || L > LH_MAX_LEVELS || K < 1 || K > LH_MAX_K) return LH_ERR_SHAPE;
  if (N >= (1 << 28)) return LH_ERR_SHAPE;
  long long pl[LH_MAX_LEVELS];
  pl[0] = 1;
  for (int l = 1; l < LH_MAX_LEVELS; ++l) {
    pl[l] = pl[l - 1] * p;
    if (pl[l] > (1LL << 40)) pl[l] = 1LL << 40;   // only levels < L are used
  }
  if (pl[L - 1] > N || N % pl[L - 1] != 0) return LH_ERR_SHAPE;
  Geom G;
  std::memset(&G, 0, sizeof(G));
  G.B = B; G.H = H; G.N = N; G.D = D; G.p = p; G.L = L; G.K = K;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) G.pl[l] = pl[l];
  for (int l = 0; l < L; ++l) G.n[l] = (int)(N / pl[l]);
  G.cand[L - 1] = G.n[L - 1];
  long long cand = G.n[L - 1];
  for (int l = L - 1; l >= 1; --l) {
    G.k[l] = (int)(cand < K ? cand : K);
    G.cand[l - 1] = p * G.k[l];
    cand = G.cand[l - 1];
  }
  const bool part = cfg->inclusion == LH_INCL_PARTITION;
  long long S = 0, C = 0;
  for (int l = 0; l < L; ++l) {
    G.c[l] = G.cand[l] - (part && l >= 1 ? G.k[l] : 0);
    S += G.c[l];
    C += G.cand[l];
  }
  if (C >= (1LL << 28)) return LH_ERR_SHAPE;
  G.S = (int)S;
  G.C = (int)C;
  int E = 0;
  for (int l = 1; l < L; ++l) {
    G.off[l] = E;
    E += G.n[l];
  }
  G.E = E;
  G.pow2 = (p & (p - 1)) == 0;
  G.accum = cfg->accum;
  G.score = cfg->score;
  G.ties = cfg->ties;
  G.order = cfg->order;
  G.weight = cfg->weight;
  G.incl = cfg->inclusion;
  *g = G;
  if (out) {
    std::memset(out, 0, sizeof(*out));
    out->S = G.S;
    out->E = G.E;
    for (int l = 0; l < LH_MAX_LEVELS; ++l) {
      out->n[l] = G.n[l];
      out->k[l] = G.k[l];
      out->c[l] = G.c[l];
      out->lvl_off[l] = G.off[l];
    }
    out->ws_bytes = L > 1 ? (size_t)B * H * 5 * (size_t)G.C * sizeof(int32_t) : 0;
  }
  return LH_OK;
}

}  // namespace

// sequence-sharded path (k_cp.cu)
cudaError_t launch_cp_assemble_sq(const Geom& g, int world, int rank, const double* gath, double* sq,
                                  cudaStream_t s);
cudaError_t launch_cp_segment(const Geom& g, int world, int rank, const int32_t* map, const int32_t* slot,
                              int32_t* slot_loc, int32_t* seg, cudaStream_t s);
cudaError_t launch_cp_gather(const Geom& g, lh_dtype dt, int world, int rank, const void* q, const void* k,
                             const void* v, const void* pq, const void* pk, const void* pv, const int32_t* map,
                             const int32_t* seg, const uint32_t* scale, void* qs, void* ks, void* vs, int* err,
                             cudaStream_t s);
cudaError_t launch_cp_zero_outside(const Geom& g, int elem_bytes, void* x, const int32_t* seg, cudaStream_t s);
Geom shard_geom(const Geom& g, int world, int rank);

namespace {

// Whole-sequence geometry plus the checks of the sequence-sharded path: L >= 2,
// 0 <= rank < world, N split evenly into shards of whole coarsest blocks.
lh_status make_cp_geom_checked(const lh_config* cfg, int world, int rank, Geom* g, lh_plan_t* pl) {
  lh_status st = make_geom(cfg, g, pl);
  if (st != LH_OK) return st;
  if (world < 1 || rank < 0 || rank >= world || g->L < 2) return LH_ERR_SHAPE;
  if (g->N % world != 0 || (g->N / world) % g->pl[g->L - 1] != 0) return LH_ERR_SHAPE;
  return LH_OK;
}

#define LH_REQ(p) do { if (!(p)) return LH_ERR_NULL; if (!aligned16(p)) return LH_ERR_ALIGN; } while (0)
#define LH_CUDA(call) do { if ((call) != cudaSuccess) return LH_ERR_CUDA; } while (0)

}  // namespace
}  // namespace lh

using namespace lh;

extern "C" {

int lh_version(void) { return 100; }

const char* lh_status_string(lh_status s) {
  switch (s) {
    case LH_OK: return "ok";
    case LH_ERR_NULL: return "null pointer";
    case LH_ERR_SHAPE: return "unsupported sizes";
    case LH_ERR_ALIGN: return "buffer not 16-byte aligned";
    case LH_ERR_DTYPE: return "unknown dtype";
    case LH_ERR_MODE: return "unknown accumulation mode or reading";
    case LH_ERR_WORKSPACE: return "workspace too small";
    case LH_ERR_CUDA: return "CUDA launch or runtime error";
    case LH_ERR_TIMEOUT: return "device-side wait timed out";
    case LH_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

lh_status lh_plan(const lh_config* cfg, lh_plan_t* out) {
  if (!out) return LH_ERR_NULL;
  Geom g;
  return make_geom(cfg, &g, out);
}

lh_status lh_pool(const lh_config* cfg, const void* q, const void* k, const void* v, void* pyr_q,
                  void* pyr_k, void* pyr_v, double* sq, uint32_t* scale, void* stream) {
  LH_RANGE("lh_pool");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(q); LH_REQ(k); LH_REQ(v); LH_REQ(scale);
  if (g.L > 1) { LH_REQ(pyr_q); LH_REQ(pyr_k); LH_REQ(pyr_v); LH_REQ(sq); }
  LH_CUDA(launch_pool(g, cfg->dtype, q, k, v, pyr_q, pyr_k, pyr_v, sq, scale, device_error_ptr(),
                      (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_score_topk(const lh_config* cfg, const double* sq, int32_t* sel, int32_t* map,
                        int32_t* slot, void* ws, size_t ws_bytes, void* stream) {
  LH_RANGE("lh_score_topk");
  Geom g;
  lh_plan_t pl;
  lh_status st = make_geom(cfg, &g, &pl);
  if (st != LH_OK) return st;
  LH_REQ(map);
  if (g.L > 1) {
    LH_REQ(sq); LH_REQ(sel); LH_REQ(slot); LH_REQ(ws);
    if (ws_bytes < pl.ws_bytes) return LH_ERR_WORKSPACE;
  }
  LH_CUDA(launch_select(g, sq, sel, map, slot, (int32_t*)ws, (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_gather(const lh_config* cfg, const void* q, const void* k, const void* v,
                    const void* pyr_q, const void* pyr_k, const void* pyr_v, const int32_t* map,
                    const uint32_t* scale, void* qs, void* ks, void* vs, void* stream) {
  LH_RANGE("lh_gather");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(q); LH_REQ(k); LH_REQ(v); LH_REQ(map); LH_REQ(scale); LH_REQ(qs); LH_REQ(ks); LH_REQ(vs);
  if (g.L > 1) { LH_REQ(pyr_q); LH_REQ(pyr_k); LH_REQ(pyr_v); }
  LH_CUDA(launch_gather(g, cfg->dtype, q, k, v, pyr_q, pyr_k, pyr_v, map, scale, qs, ks, vs,
                        device_error_ptr(), (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_attn_fwd(const lh_config* cfg, const void* qs, const void* ks, const void* vs,
                      const uint32_t* scale, float* os, float* lse, void* stream) {
  LH_RANGE("lh_attn_fwd");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(qs); LH_REQ(ks); LH_REQ(vs); LH_REQ(scale); LH_REQ(os); LH_REQ(lse);
  LH_CUDA(launch_attn_fwd(g, cfg->dtype, qs, ks, vs, os, lse, scale, device_error_ptr(),
                          (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_scatter(const lh_config* cfg, const float* os, const int32_t* slot, void* o,
                     void* stream) {
  LH_RANGE("lh_scatter");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(os); LH_REQ(o);
  if (g.L > 1) LH_REQ(slot);
  LH_CUDA(launch_scatter(g, cfg->dtype, os, slot, o, (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_scatter_bwd(const lh_config* cfg, const void* dout, const float* os,
                         const int32_t* slot, void* dos, float* delta, uint32_t* scale, void* stream) {
  LH_RANGE("lh_scatter_bwd");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(dout); LH_REQ(os); LH_REQ(dos); LH_REQ(delta); LH_REQ(scale);
  if (g.L > 1) LH_REQ(slot);
  LH_CUDA(launch_scatter_bwd(g, cfg->dtype, dout, os, slot, dos, delta, scale, device_error_ptr(),
                             (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_attn_bwd(const lh_config* cfg, const void* qs, const void* ks, const void* vs,
                      const void* dos, const float* lse, const float* delta, const uint32_t* scale,
                      float* dqs, float* dks, float* dvs, void* stream) {
  LH_RANGE("lh_attn_bwd");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(qs); LH_REQ(ks); LH_REQ(vs); LH_REQ(dos); LH_REQ(lse); LH_REQ(delta); LH_REQ(scale);
  LH_REQ(dqs); LH_REQ(dks); LH_REQ(dvs);
  LH_CUDA(launch_attn_bwd(g, cfg->dtype, qs, ks, vs, dos, lse, delta, scale, dqs, dks, dvs,
                          device_error_ptr(), (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_spread(const lh_config* cfg, const float* dqs, const float* dks, const float* dvs,
                    const int32_t* slot, void* dq, void* dk, void* dv, void* stream) {
  LH_RANGE("lh_spread");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(dqs); LH_REQ(dks); LH_REQ(dvs); LH_REQ(dq); LH_REQ(dk); LH_REQ(dv);
  if (g.L > 1) LH_REQ(slot);
  LH_CUDA(launch_spread(g, cfg->dtype, dqs, dks, dvs, slot, dq, dk, dv, (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_forward(const lh_config* cfg, const void* q, const void* k, const void* v, void* o,
                     const lh_buffers* b, void* stream) {
  LH_RANGE("lh_forward");
  if (!b) return LH_ERR_NULL;
  Geom g;
  lh_plan_t pl;
  lh_status st = make_geom(cfg, &g, &pl);
  if (st != LH_OK) return st;
  // validate everything up front so that nothing is launched on error
  LH_REQ(q); LH_REQ(k); LH_REQ(v); LH_REQ(o); LH_REQ(b->map); LH_REQ(b->qs); LH_REQ(b->ks);
  LH_REQ(b->vs); LH_REQ(b->os); LH_REQ(b->lse); LH_REQ(b->scale);
  if (g.L > 1) {
    LH_REQ(b->pyr_q); LH_REQ(b->pyr_k); LH_REQ(b->pyr_v); LH_REQ(b->sq); LH_REQ(b->sel);
    LH_REQ(b->slot); LH_REQ(b->ws);
    if (b->ws_bytes < pl.ws_bytes) return LH_ERR_WORKSPACE;
  }
  if ((st = lh_pool(cfg, q, k, v, b->pyr_q, b->pyr_k, b->pyr_v, b->sq, b->scale, stream)) != LH_OK) return st;
  if ((st = lh_score_topk(cfg, b->sq, b->sel, b->map, b->slot, b->ws, b->ws_bytes, stream)) != LH_OK)
    return st;
  if ((st = lh_gather(cfg, q, k, v, b->pyr_q, b->pyr_k, b->pyr_v, b->map, b->scale, b->qs, b->ks, b->vs,
                      stream)) != LH_OK)
    return st;
  if ((st = lh_attn_fwd(cfg, b->qs, b->ks, b->vs, b->scale, b->os, b->lse, stream)) != LH_OK) return st;
  return lh_scatter(cfg, b->os, b->slot, o, stream);
}

lh_status lh_backward(const lh_config* cfg, const void* dout, void* dq, void* dk, void* dv,
                      const lh_buffers* b, void* stream) {
  LH_RANGE("lh_backward");
  if (!b) return LH_ERR_NULL;
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(dout); LH_REQ(dq); LH_REQ(dk); LH_REQ(dv); LH_REQ(b->os); LH_REQ(b->dos);
  LH_REQ(b->delta); LH_REQ(b->qs); LH_REQ(b->ks); LH_REQ(b->vs); LH_REQ(b->lse);
  LH_REQ(b->dqs); LH_REQ(b->dks); LH_REQ(b->dvs); LH_REQ(b->scale);
  if (g.L > 1) LH_REQ(b->slot);
  if ((st = lh_scatter_bwd(cfg, dout, b->os, b->slot, b->dos, b->delta, b->scale, stream)) != LH_OK) return st;
  if ((st = lh_attn_bwd(cfg, b->qs, b->ks, b->vs, b->dos, b->lse, b->delta, b->scale, b->dqs, b->dks, b->dvs,
                        stream)) != LH_OK)
    return st;
  return lh_spread(cfg, b->dqs, b->dks, b->dvs, b->slot, dq, dk, dv, stream);
}

// ---------------------------------------------------------------- token ranges (fusion with projections)

namespace {
lh_status check_range(const Geom& g, int t0, int nt) {
  if (g.L < 2) return LH_ERR_SHAPE;
  const long long P = g.pl[g.L - 1];
  if (t0 < 0 || nt < 0 || (long long)t0 + nt > g.N || t0 % P != 0 || nt % P != 0) return LH_ERR_SHAPE;
  return LH_OK;
}
}  // namespace

lh_status lh_pool_range(const lh_config* cfg, int t0, int nt, const void* q, const void* k, const void* v,
                        void* pyr_q, void* pyr_k, void* pyr_v, double* sq, uint32_t* scale, void* stream) {
  LH_RANGE("lh_pool_range");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  if ((st = check_range(g, t0, nt)) != LH_OK) return st;
  LH_REQ(q); LH_REQ(k); LH_REQ(v); LH_REQ(pyr_q); LH_REQ(pyr_k); LH_REQ(pyr_v); LH_REQ(sq); LH_REQ(scale);
  const int P = (int)g.pl[g.L - 1];
  LH_CUDA(launch_pool_range(g, cfg->dtype, t0 / P, nt / P, q, k, v, pyr_q, pyr_k, pyr_v, sq, scale,
                            device_error_ptr(), (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_scatter_range(const lh_config* cfg, int t0, int nt, const float* os, const int32_t* slot, void* o,
                           void* stream) {
  LH_RANGE("lh_scatter_range");
  Geom g;
  lh_status st = make_geom(cfg, &g, nullptr);
  if (st != LH_OK) return st;
  if ((st = check_range(g, t0, nt)) != LH_OK) return st;
  LH_REQ(os); LH_REQ(slot); LH_REQ(o);
  const int P = (int)g.pl[g.L - 1];
  LH_CUDA(launch_scatter_range(g, cfg->dtype, t0 / P, nt / P, os, slot, o, (cudaStream_t)stream));
  return LH_OK;
}

// ---------------------------------------------------------------- sequence-sharded path

lh_status lh_cp_plan(const lh_config* cfg, int world, int rank, lh_cp_plan_t* out) {
  if (!out) return LH_ERR_NULL;
  Geom g;
  lh_plan_t pl;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, &pl);
  if (st != LH_OK) return st;
  const Geom s = shard_geom(g, world, rank);
  std::memset(out, 0, sizeof(*out));
  out->world = world;
  out->rank = rank;
  out->n_loc = s.N;
  out->E_loc = s.E;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) out->lvl_off_loc[l] = l < g.L ? s.off[l] : 0;
  out->global = pl;
  return LH_OK;
}

lh_status lh_cp_pool(const lh_config* cfg, int world, int rank, const void* q, const void* k, const void* v,
                     void* pyr_q, void* pyr_k, void* pyr_v, double* sq_loc, uint32_t* scale, void* stream) {
  LH_RANGE("lh_cp_pool");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(q); LH_REQ(k); LH_REQ(v); LH_REQ(pyr_q); LH_REQ(pyr_k); LH_REQ(pyr_v); LH_REQ(sq_loc); LH_REQ(scale);
  LH_CUDA(launch_pool(shard_geom(g, world, rank), cfg->dtype, q, k, v, pyr_q, pyr_k, pyr_v, sq_loc, scale,
                      device_error_ptr(), (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_cp_assemble_sq(const lh_config* cfg, int world, const double* sq_gathered, double* sq,
                            void* stream) {
  LH_RANGE("lh_cp_assemble_sq");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, 0, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(sq_gathered); LH_REQ(sq);
  LH_CUDA(launch_cp_assemble_sq(g, world, 0, sq_gathered, sq, (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_cp_segment(const lh_config* cfg, int world, int rank, const int32_t* map, const int32_t* slot,
                        int32_t* slot_loc, int32_t* seg, void* stream) {
  LH_RANGE("lh_cp_segment");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(map); LH_REQ(slot); LH_REQ(slot_loc); LH_REQ(seg);
  LH_CUDA(launch_cp_segment(g, world, rank, map, slot, slot_loc, seg, (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_cp_gather(const lh_config* cfg, int world, int rank, const void* q, const void* k, const void* v,
                       const void* pyr_q, const void* pyr_k, const void* pyr_v, const int32_t* map,
                       const int32_t* seg, const uint32_t* scale, void* qs, void* ks, void* vs, void* stream) {
  LH_RANGE("lh_cp_gather");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(q); LH_REQ(k); LH_REQ(v); LH_REQ(pyr_q); LH_REQ(pyr_k); LH_REQ(pyr_v); LH_REQ(map); LH_REQ(seg);
  LH_REQ(scale); LH_REQ(qs); LH_REQ(ks); LH_REQ(vs);
  LH_CUDA(launch_cp_gather(g, cfg->dtype, world, rank, q, k, v, pyr_q, pyr_k, pyr_v, map, seg, scale, qs, ks, vs,
                           device_error_ptr(), (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_cp_attn_fwd(const lh_config* cfg, int world, int rank, const int32_t* seg, const void* qs,
                         const void* ks, const void* vs, const uint32_t* scale, float* os, float* lse,
                         void* stream) {
  LH_RANGE("lh_cp_attn_fwd");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, nullptr);
  if (st != LH_OK) return st;
  if (cfg->dtype != LH_BF16) return LH_ERR_DTYPE;
  LH_REQ(seg); LH_REQ(qs); LH_REQ(ks); LH_REQ(vs); LH_REQ(scale); LH_REQ(os); LH_REQ(lse);
  LH_CUDA(launch_attn_fwd_tc(g, qs, ks, vs, os, lse, seg, scale, device_error_ptr(), (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_cp_scatter(const lh_config* cfg, int world, int rank, const float* os, const int32_t* slot_loc,
                        void* o, void* stream) {
  LH_RANGE("lh_cp_scatter");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(os); LH_REQ(slot_loc); LH_REQ(o);
  LH_CUDA(launch_scatter(shard_geom(g, world, rank), cfg->dtype, os, slot_loc, o, (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_cp_scatter_bwd(const lh_config* cfg, int world, int rank, const void* dout, const float* os,
                            const int32_t* slot_loc, const int32_t* seg, void* dos, float* delta, uint32_t* scale,
                            void* stream) {
  LH_RANGE("lh_cp_scatter_bwd");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, nullptr);
  if (st != LH_OK) return st;
  if (cfg->dtype != LH_BF16) return LH_ERR_DTYPE;
  LH_REQ(dout); LH_REQ(os); LH_REQ(slot_loc); LH_REQ(seg); LH_REQ(dos); LH_REQ(delta); LH_REQ(scale);
  LH_CUDA(launch_cp_zero_outside(g, 2, dos, seg, (cudaStream_t)stream));
  LH_CUDA(launch_scatter_bwd(shard_geom(g, world, rank), cfg->dtype, dout, os, slot_loc, dos, delta, scale,
                             device_error_ptr(), (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_cp_attn_bwd(const lh_config* cfg, int world, int rank, const int32_t* seg, const void* qs,
                         const void* ks, const void* vs, const void* dos, const float* lse, const float* delta,
                         const uint32_t* scale, float* dqs, float* dks, float* dvs, void* stream) {
  LH_RANGE("lh_cp_attn_bwd");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, nullptr);
  if (st != LH_OK) return st;
  if (cfg->dtype != LH_BF16) return LH_ERR_DTYPE;
  LH_REQ(seg); LH_REQ(qs); LH_REQ(ks); LH_REQ(vs); LH_REQ(dos); LH_REQ(lse); LH_REQ(delta); LH_REQ(scale);
  LH_REQ(dqs); LH_REQ(dks); LH_REQ(dvs);
  LH_CUDA(launch_attn_bwd_tc(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, seg, scale, device_error_ptr(),
                             (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_cp_spread(const lh_config* cfg, int world, int rank, const float* dqs, const float* dks,
                       const float* dvs, const int32_t* slot_loc, void* dq, void* dk, void* dv, void* stream) {
  LH_RANGE("lh_cp_spread");
  Geom g;
  lh_status st = make_cp_geom_checked(cfg, world, rank, &g, nullptr);
  if (st != LH_OK) return st;
  LH_REQ(dqs); LH_REQ(dks); LH_REQ(dvs); LH_REQ(slot_loc); LH_REQ(dq); LH_REQ(dk); LH_REQ(dv);
  LH_CUDA(launch_spread(shard_geom(g, world, rank), cfg->dtype, dqs, dks, dvs, slot_loc, dq, dk, dv,
                        (cudaStream_t)stream));
  return LH_OK;
}

lh_status lh_selftest_timeout(long long limit_cycles, int* gave_up, void* stream) {
  if (!gave_up) return LH_ERR_NULL;
  if (limit_cycles < 1 || limit_cycles > 2000000000LL) return LH_ERR_SHAPE;
  int* err = device_error_ptr();
  if (!err) return LH_ERR_CUDA;
  return lh::launch_selftest_wait(limit_cycles, err, gave_up, (cudaStream_t)stream) == cudaSuccess ? LH_OK
                                                                                                  : LH_ERR_CUDA;
}

lh_status lh_selftest_exp2(const float* x, float* y_fma, float* y_sfu, int n, void* stream) {
  if (n < 0) return LH_ERR_SHAPE;
  if (n == 0) return LH_OK;
  if (!x || !y_fma || !y_sfu) return LH_ERR_NULL;
  return lh::launch_selftest_exp2(x, y_fma, y_sfu, n, (cudaStream_t)stream) == cudaSuccess ? LH_OK : LH_ERR_CUDA;
}

lh_status lh_get_device_error(void* stream, int* detail) {
  int h[2] = {0, 0};
  const int zero[2] = {0, 0};
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyFromSymbolAsync(h, g_dev_error, sizeof(h), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return LH_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LH_ERR_CUDA;
  if (h[0] != 0) {
    if (cudaMemcpyToSymbolAsync(g_dev_error, zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return LH_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return LH_ERR_CUDA;
  }
  if (detail) *detail = h[1];
  return (lh_status)h[0];
}

unsigned long long lh_launch_count(void) { return g_launches.load(); }

}  // extern "C"
