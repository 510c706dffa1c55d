// Pyramid pool + squared l2 norms, one pass over Q, K, V.
//
// "Long Context Pre-Training with Lighthouse Attention", §3.1 stage (i) and
// Fig. 2 steps 1-2: Q, K and V are mean-pooled with the same factor p into
// levels l = 1..L-1 (entry i of level l = mean of tokens [i p^l, (i+1) p^l));
// pooled entries are ranked by l2 norm, for queries and keys alike.
//
// Arithmetic (fixed so that the selection downstream is reproducible bit for
// bit): sums are fp64; level l's sum is the left-to-right sum of its p
// children's sums starting from the first child; the mean is sum / p^l (an
// exact scaling when p is a power of two, an IEEE division otherwise) and is
// stored rounded to nearest-even in the I/O dtype. The squared norm of the
// fp64 mean is formed per 8-component chunk left to right from the first
// rounded product (no fused multiply-add), then the D/8 chunk partials are
// combined by a butterfly over the lanes that hold them, which equals the
// stride-halving tree c[j] += c[j + s] for s = D/16, ..., 1.
//
// Thread mapping: one thread owns 8 consecutive components of one head; the
// D/8 lanes of a head are consecutive lanes of one warp. A thread walks the
// p^(L-1) tokens of one coarsest-level block in order, keeping one running fp64
// sum per level (carry chain), and emits each entry when its last child is in.
// HBM traffic: every token row is read once; pyramid rows and norms written once.
#include "lh_common.cuh"

namespace lh {
namespace {

struct PoolArgs {
  Geom g;
  int hg;        // heads per CTA
  int yb;        // coarsest blocks per CTA (blockDim.y)
  int ncoarse;   // coarsest blocks per batch row
};

template <typename T, int LV>
__global__ void __launch_bounds__(256) k_pool(const T* __restrict__ q, const T* __restrict__ k,
                                              const T* __restrict__ v, T* __restrict__ pq,
                                              T* __restrict__ pk, T* __restrict__ pv,
                                              double* __restrict__ sq, PoolArgs a) {
  const Geom& g = a.g;
  const int C8 = g.D >> 3;
  const int tensor = blockIdx.z % 3;
  const int b = blockIdx.z / 3;
  const int head = blockIdx.y * a.hg + threadIdx.x / C8;
  const int chunk = threadIdx.x % C8;
  const int cb = blockIdx.x * a.yb + threadIdx.y;
  const bool live = head < g.H && cb < a.ncoarse;   // whole head groups share liveness
  const T* x = tensor == 0 ? q : (tensor == 1 ? k : v);
  T* pyr = tensor == 0 ? pq : (tensor == 1 ? pk : pv);
  const int p = g.p;
  const long long P = g.pl[LV];
  const size_t tok_stride = (size_t)g.H * g.D;
  const T* src = x + ((size_t)b * g.N + (size_t)cb * P) * tok_stride + (size_t)head * g.D + chunk * 8;
  T* dst_head = pyr + ((size_t)b * g.H + head) * (size_t)g.E * g.D + chunk * 8;
  double* sq_head = (tensor < 2) ? sq + ((size_t)tensor * g.B * g.H + (size_t)b * g.H + head) * g.E
                                 : nullptr;

  double acc[LV][8];   // acc[l-1]: running sum of the open entry of level l
  const long long ngroups = P / p;   // level-1 entries in this block

  for (long long g1 = 0; g1 < ngroups; ++g1) {
    // level 1: p tokens, left to right from the first child
    double s[8];
    for (int c0 = 0; c0 < p; c0 += 8) {
      const int nb = min(8, p - c0);
      typename Vec8<T>::Raw raw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < nb && live) Vec8<T>::load_raw(src + (size_t)(g1 * p + c0 + u) * tok_stride, raw[u]);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (u < nb) {
          double xr[8];
          Vec8<T>::raw_f64(raw[u], xr);
          if (c0 + u == 0) {
#pragma unroll
            for (int d = 0; d < 8; ++d) s[d] = xr[d];
          } else {
#pragma unroll
            for (int d = 0; d < 8; ++d) s[d] = __dadd_rn(s[d], xr[d]);
          }
        }
      }
    }
#pragma unroll
    for (int d = 0; d < 8; ++d) acc[0][d] = s[d];
    // emit level 1, then carry the completed sum upward while levels complete
    long long gi = (long long)cb * (P / p) + g1;   // index of this level-1 entry
#pragma unroll
    for (int l = 1; l <= LV; ++l) {
      if (l > 1) {
        const int pos = (int)(gi % p);   // gi here is the level-(l-1) index
        if (pos == 0) {
#pragma unroll
          for (int d = 0; d < 8; ++d) acc[l - 1][d] = acc[l - 2][d];
        } else {
#pragma unroll
          for (int d = 0; d < 8; ++d) acc[l - 1][d] = __dadd_rn(acc[l - 1][d], acc[l - 2][d]);
        }
        if (pos != p - 1) break;
        gi /= p;
      }
      // entry (l, gi) complete
      double m[8];
      if (g.pow2) {
        const double inv = 1.0 / (double)g.pl[l];   // exact: p^l is a power of two
#pragma unroll
        for (int d = 0; d < 8; ++d) m[d] = __dmul_rn(acc[l - 1][d], inv);
      } else {
        const double den = (double)g.pl[l];
#pragma unroll
        for (int d = 0; d < 8; ++d) m[d] = __ddiv_rn(acc[l - 1][d], den);
      }
      const size_t e = (size_t)g.off[l] + gi;
      if (live) Vec8<T>::store_f64(dst_head + e * g.D, m);
      if (tensor < 2) {
        double part = __dmul_rn(m[0], m[0]);
#pragma unroll
        for (int d = 1; d < 8; ++d) part = __dadd_rn(part, __dmul_rn(m[d], m[d]));
        for (int off = C8 >> 1; off >= 1; off >>= 1)
          part = __dadd_rn(part, __shfl_xor_sync(0xffffffffu, part, off));
        if (live && chunk == 0) sq_head[e] = part;
      }
    }
  }
}

template <typename T>
cudaError_t launch_t(const Geom& g, const void* q, const void* k, const void* v, void* pq,
                     void* pk, void* pv, double* sq, cudaStream_t s) {
  const int LV = g.L - 1;
  if (LV < 1) return cudaSuccess;
  PoolArgs a;
  a.g = g;
  const int C8 = g.D / 8;
  int hg = g.H;
  while (hg * C8 > 256) {   // largest divisor of H that fits 256 threads
    --hg;
    while (g.H % hg) --hg;
  }
  a.hg = hg;
  a.ncoarse = g.n[g.L - 1];
  a.yb = 1;
  while (a.yb * 2 * hg * C8 <= 256 && a.yb * 2 <= a.ncoarse) a.yb *= 2;
  dim3 block(hg * C8, a.yb);
  dim3 grid((a.ncoarse + a.yb - 1) / a.yb, g.H / hg, 3 * g.B);
  const T* tq = (const T*)q; const T* tk = (const T*)k; const T* tv = (const T*)v;
  T* tpq = (T*)pq; T* tpk = (T*)pk; T* tpv = (T*)pv;
  switch (LV) {
#define LH_POOL_CASE(n) \
    case n: k_pool<T, n><<<grid, block, 0, s>>>(tq, tk, tv, tpq, tpk, tpv, sq, a); break;
    LH_POOL_CASE(1) LH_POOL_CASE(2) LH_POOL_CASE(3) LH_POOL_CASE(4)
    LH_POOL_CASE(5) LH_POOL_CASE(6) LH_POOL_CASE(7)
#undef LH_POOL_CASE
    default: return cudaErrorInvalidValue;
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                        void* pq, void* pk, void* pv, double* sq, cudaStream_t s) {
  if (dt == LH_BF16) return launch_t<__nv_bfloat16>(g, q, k, v, pq, pk, pv, sq, s);
  return launch_t<float>(g, q, k, v, pq, pk, pv, sq, s);
}

}  // namespace lh
