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
// Max-pool score reading (MP; Fig. 2 step 2 read as "l2 norm of every token,
// then max-pooled up the levels"): instead of the norms of the means, sq gets,
// for each entry, the largest pinned-order squared norm among its tokens, for
// queries and keys separately (a token's norm is formed exactly as a mean's).
// Taking the max of the two then equals max-pooling the tokens' bidirectional
// scores level by level, since max commutes.
//
// Thread mapping: one thread owns 8 consecutive components of one head; the
// D/8 lanes of a head are consecutive lanes of one warp. A thread walks the
// p^(L-1) tokens of one coarsest-level block in order, keeping one running fp64
// sum per level (carry chain), and emits each entry when its last child is in.
// Rows arrive through a shared-memory ring filled by bulk async copies.
// HBM traffic: every token row is read once; pyramid rows and norms written once.
#include "tc_ptx.cuh"

namespace lh {
namespace {

using tc::mbar_init;
using tc::fence_mbar_init;
using tc::mbar_expect_tx;
using tc::smem_u32;

struct PoolArgs {
  Geom g;
  int hg;          // heads per CTA (a divisor of H)
  int ts;          // tokens per shared-memory stage
  int ns;          // stages in the ring
  int row_bytes;   // bytes of one token row of the head group
  int cb0;         // first coarsest block (a token range pools blocks cb0 .. cb0 + gridDim.x - 1)
};

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// One CTA: one coarsest block of one tensor for one head group. Token rows of
// the head group stream through a ring of shared-memory stages filled by 1-D
// bulk async copies (one copy per stage when the group is the whole row), so
// the loads in flight do not depend on registers; each thread then reads its
// 16 bytes of every row from shared memory.
// PP: the pooling factor p as a compile-time constant when it is one of the
// common values and a stage holds whole level-1 entries (ts % p == 0); then a
// level-1 entry's p token rows are read and widened together, so the widening
// conversions (a quarter-rate pipe) overlap instead of waiting on the add chain.
// PP == 0: any p, one token at a time.
template <typename T, int LV, int PP, bool MP>
__global__ void __launch_bounds__(256, 2) k_pool(const T* __restrict__ q, const T* __restrict__ k,
                                                 const T* __restrict__ v, T* __restrict__ pq,
                                                 T* __restrict__ pk, T* __restrict__ pv,
                                                 double* __restrict__ sq, uint32_t* __restrict__ scale,
                                                 PoolArgs a, int* err) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Geom& g = a.g;
  const int C8 = g.D >> 3;
  const int tensor = blockIdx.z % 3;
  const int b = blockIdx.z / 3;
  const int hg0 = blockIdx.y * a.hg;
  const int head = hg0 + threadIdx.x / C8;
  const int chunk = threadIdx.x % C8;
  const int cb = a.cb0 + (int)blockIdx.x;
  const T* x = tensor == 0 ? q : (tensor == 1 ? k : v);
  T* pyr = tensor == 0 ? pq : (tensor == 1 ? pk : pv);
  const int p = PP ? PP : g.p;
  const long long P = g.pl[LV];
  const size_t tok_stride = (size_t)g.H * g.D;
  const T* src0 = x + ((size_t)b * g.N + (size_t)cb * P) * tok_stride + (size_t)hg0 * g.D;
  T* dst_head = pyr + ((size_t)b * g.H + head) * (size_t)g.E * g.D + chunk * 8;
  double* sq_head = (tensor < 2) ? sq + ((size_t)tensor * g.B * g.H + (size_t)b * g.H + head) * g.E
                                 : nullptr;
  // lanes of this warp that exist (a head group narrower than a warp)
  const int wbase = threadIdx.x & ~31;
  const unsigned wmask = (wbase + 32 <= (int)blockDim.x) ? 0xffffffffu
                                                         : ((1u << (blockDim.x - wbase)) - 1u);

  const int row_bytes = a.row_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)a.ns * a.ts * row_bytes);
  const int nstages = (int)((P + a.ts - 1) / a.ts);
  const bool contiguous = (a.hg == g.H);
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < a.ns; ++s2) mbar_init(&full[s2], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int kk) {
    const int slot = kk % a.ns;
    const long long t0 = (long long)kk * a.ts;
    const int nt = (int)min((long long)a.ts, P - t0);
    uint8_t* dst = smem + (size_t)slot * a.ts * row_bytes;
    mbar_expect_tx(&full[slot], (uint32_t)(nt * row_bytes));
    if (contiguous) {
      bulk_load(dst, src0 + t0 * tok_stride, (uint32_t)(nt * row_bytes), &full[slot]);
    } else {
      for (int u = 0; u < nt; ++u)
        bulk_load(dst + (size_t)u * row_bytes, src0 + (t0 + u) * tok_stride, (uint32_t)row_bytes,
                  &full[slot]);
    }
  };
  if (threadIdx.x == 0)
    for (int kk = 0; kk < a.ns && kk < nstages; ++kk) issue(kk);

  double acc[LV][8];                    // acc[l-1]: running sum of the open entry of level l
  double (&s)[8] = acc[0];
  double mx[MP ? LV : 1];               // MP: mx[l-1] = largest token norm of the open level-l entry
  // MP: pinned-order squared norm of one token's row (the same on every lane of the head)
  auto token_norm = [&](const double (&xr)[8]) -> double {
    double part = __dmul_rn(xr[0], xr[0]);
#pragma unroll
    for (int d = 1; d < 8; ++d) part = __dadd_rn(part, __dmul_rn(xr[d], xr[d]));
    for (int off = C8 >> 1; off >= 1; off >>= 1) part = __dadd_rn(part, __shfl_xor_sync(wmask, part, off));
    return part;
  };
  uint32_t amax = 0;                    // bf16 I/O: largest |x| of this thread's components (fp32 bits)
  long long gi1 = (long long)cb * (P / p);   // index of the open level-1 entry
  int c = 0;                            // position of the next token in its level-1 entry
  tc::Abort none{0};
  for (int kk = 0; kk < nstages; ++kk) {
    const int slot = kk % a.ns;
    const bool ok = tc::mbar_wait(&full[slot], (kk / a.ns) & 1, &none, err, 200);
    if (__syncthreads_or(!ok)) break;   // copies never landed: reported, all threads leave
    const long long t0 = (long long)kk * a.ts;
    const int nt = (int)min((long long)a.ts, P - t0);
    const uint8_t* buf = smem + (size_t)slot * a.ts * row_bytes + (size_t)threadIdx.x * 8 * sizeof(T);
    // level-1 entry gi1 complete (its sum in acc[0]): emit it, then carry
    // upward while levels complete
    auto complete = [&]() {
      long long gi = gi1++;
#pragma unroll
      for (int l = 1; l <= LV; ++l) {
        if (l > 1) {
          const int pos = (int)(gi % p);   // gi here is the level-(l-1) index
          if (pos == 0) {
#pragma unroll
            for (int d = 0; d < 8; ++d) acc[l - 1][d] = acc[l - 2][d];
            if constexpr (MP) mx[l - 1] = mx[l - 2];
          } else {
#pragma unroll
            for (int d = 0; d < 8; ++d) acc[l - 1][d] = __dadd_rn(acc[l - 1][d], acc[l - 2][d]);
            if constexpr (MP) mx[l - 1] = fmax(mx[l - 1], mx[l - 2]);
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
        Vec8<T>::store_f64(dst_head + e * g.D, m);
        if (MP) {
          if (tensor < 2 && chunk == 0) sq_head[e] = mx[l - 1];
        } else if (tensor < 2) {
          double part = __dmul_rn(m[0], m[0]);
#pragma unroll
          for (int d = 1; d < 8; ++d) part = __dadd_rn(part, __dmul_rn(m[d], m[d]));
          for (int off = C8 >> 1; off >= 1; off >>= 1)
            part = __dadd_rn(part, __shfl_xor_sync(wmask, part, off));
          if (chunk == 0) sq_head[e] = part;
        }
      }
    };
    if constexpr (PP > 0) {
      // whole level-1 entries: all PP rows read first, then widened and summed
      // left to right
      for (int u0 = 0; u0 < nt; u0 += PP) {
        typename Vec8<T>::Raw raw[PP > 0 ? PP : 1];
#pragma unroll
        for (int u = 0; u < PP; ++u)
          raw[u] = *reinterpret_cast<const typename Vec8<T>::Raw*>(buf + (size_t)(u0 + u) * row_bytes);
#pragma unroll
        for (int u = 0; u < PP; ++u) {
          if constexpr (sizeof(T) == 2) amax = max(amax, absmax8_bf16(raw[u].a));
          double xr[8];
          Vec8<T>::raw_f64(raw[u], xr);
#pragma unroll
          for (int d = 0; d < 8; ++d) s[d] = u == 0 ? xr[d] : __dadd_rn(s[d], xr[d]);
          if constexpr (MP) {
            if (tensor < 2) {
              const double tn = token_norm(xr);
              mx[0] = u == 0 ? tn : fmax(mx[0], tn);
            }
          }
        }
        complete();
      }
    } else {
      for (int u = 0; u < nt; ++u) {
        typename Vec8<T>::Raw raw = *reinterpret_cast<const typename Vec8<T>::Raw*>(buf + (size_t)u * row_bytes);
        if constexpr (sizeof(T) == 2) amax = max(amax, absmax8_bf16(raw.a));
        double xr[8];
        Vec8<T>::raw_f64(raw, xr);
        if (c == 0) {
#pragma unroll
          for (int d = 0; d < 8; ++d) s[d] = xr[d];
        } else {
#pragma unroll
          for (int d = 0; d < 8; ++d) s[d] = __dadd_rn(s[d], xr[d]);
        }
        if constexpr (MP) {
          if (tensor < 2) {
            const double tn = token_norm(xr);
            mx[0] = c == 0 ? tn : fmax(mx[0], tn);
          }
        }
        if (++c < p) continue;
        c = 0;
        complete();
      }
    }
    __syncthreads();                    // every thread is done with this stage
    if (threadIdx.x == 0 && kk + a.ns < nstages) issue(kk + a.ns);
  }
  if constexpr (sizeof(T) == 2) {
    // the head's largest magnitude (tokens; pooled means are no larger)
    for (int off = C8 >> 1; off >= 1; off >>= 1) amax = max(amax, __shfl_xor_sync(wmask, amax, off));
    if (chunk == 0 && amax) atomicMax(scale + (size_t)tensor * g.B * g.H + (size_t)b * g.H + head, amax);
  }
}

// rows [r0, r0 + nr) of the scale buffer ([kScaleRows][B*H]) set to zero
__global__ void k_scale_zero(uint32_t* __restrict__ scale, int r0, int nr, int bh) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nr * bh; i += gridDim.x * blockDim.x)
    scale[(size_t)r0 * bh + i] = 0u;
}

// L = 1 (no pyramid): the largest |x| of each (b, h) of q, k, v over all tokens.
// grid (token blocks, B*H, 3); each thread walks tokens t = threadIdx.x + ...,
// reading the head's D components of a token (contiguous), then one atomic
// per warp.
__global__ void __launch_bounds__(256) k_absmax_tokens(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                       const uint4* __restrict__ v, uint32_t* __restrict__ scale,
                                                       Geom g) {
  const int tensor = blockIdx.z;
  const uint4* x = tensor == 0 ? q : (tensor == 1 ? k : v);
  const int bh = blockIdx.y, b = bh / g.H, h = bh - b * g.H;
  const int vpr = g.D / 8;                      // 16-byte vectors of one head row
  uint32_t m = 0;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < g.N; t += gridDim.x * blockDim.x) {
    const uint4* row = x + (((size_t)b * g.N + t) * g.H + h) * vpr;
    for (int c = 0; c < vpr; ++c) m = max(m, absmax8_bf16(__ldg(row + c)));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0 && m) atomicMax(scale + (size_t)tensor * g.B * g.H + bh, m);
}

template <typename T>
cudaError_t launch_t(const Geom& g, const void* q, const void* k, const void* v, void* pq,
                     void* pk, void* pv, double* sq, uint32_t* scale, int cb0, int ncb, int* err,
                     cudaStream_t s) {
  const int LV = g.L - 1;
  if (cb0 == 0 && scale) {
    // the maxima accumulate over the calls that start from the sequence's first block
    k_scale_zero<<<1, 256, 0, s>>>(scale, kScaleQ, 3, g.B * g.H);
    count_launch();
  }
  if (LV < 1) {
    if (sizeof(T) == 2 && scale) {
      dim3 grid((unsigned)((g.N + 255) / 256 < 64 ? (g.N + 255) / 256 : 64), (unsigned)(g.B * g.H), 3);
      k_absmax_tokens<<<grid, 256, 0, s>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, scale, g);
      count_launch();
    }
    return cudaGetLastError();
  }
  if (ncb <= 0) return cudaGetLastError();
  PoolArgs a;
  a.g = g;
  a.cb0 = cb0;
  const int C8 = g.D / 8;
  int hg = g.H;
  while (hg * C8 > 256) {   // largest divisor of H that fits 256 threads
    --hg;
    while (g.H % hg) --hg;
  }
  const int stage_bytes = 32768;
  a.hg = hg;
  a.row_bytes = hg * g.D * (int)sizeof(T);
  const long long P = g.pl[LV];
  int ts = 1;
  while (ts * 2 * a.row_bytes <= stage_bytes && ts * 2 <= P) ts *= 2;
  a.ts = ts;
  a.ns = 3;
  const size_t smem = (size_t)a.ns * a.ts * a.row_bytes + a.ns * sizeof(uint64_t);
  cudaError_t e = cudaSuccess;
  // compile-time p when it divides the stage
  const int pp = (a.ts % g.p == 0 && (g.p == 2 || g.p == 4 || g.p == 8)) ? g.p : 0;
  dim3 block(hg * C8);
  dim3 grid(ncb, g.H / hg, 3 * g.B);
  const T* tq = (const T*)q; const T* tk = (const T*)k; const T* tv = (const T*)v;
  T* tpq = (T*)pq; T* tpk = (T*)pk; T* tpv = (T*)pv;
  switch (LV) {
#define LH_POOL_MP(n, P, M)                                                                             \
  e = cudaFuncSetAttribute(k_pool<T, n, P, M>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
  if (e != cudaSuccess) return e;                                                                       \
  k_pool<T, n, P, M><<<grid, block, smem, s>>>(tq, tk, tv, tpq, tpk, tpv, sq, scale, a, err);
#define LH_POOL_PP(n, P)                                                                                \
  if (g.score == LH_SCORE_MAXPOOL) { LH_POOL_MP(n, P, true) } else { LH_POOL_MP(n, P, false) }
#define LH_POOL_CASE(n)                                                                                 \
    case n:                                                                                             \
      if (pp == 8) { LH_POOL_PP(n, 8) } else if (pp == 4) { LH_POOL_PP(n, 4) }                          \
      else if (pp == 2) { LH_POOL_PP(n, 2) } else { LH_POOL_PP(n, 0) }                                  \
      break;
    LH_POOL_CASE(1) LH_POOL_CASE(2) LH_POOL_CASE(3) LH_POOL_CASE(4)
    LH_POOL_CASE(5) LH_POOL_CASE(6) LH_POOL_CASE(7)
#undef LH_POOL_CASE
#undef LH_POOL_PP
#undef LH_POOL_MP
    default: return cudaErrorInvalidValue;
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scale_zero(uint32_t* scale, int r0, int nr, int bh, cudaStream_t s) {
  k_scale_zero<<<1, 256, 0, s>>>(scale, r0, nr, bh);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_pool(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                        void* pq, void* pk, void* pv, double* sq, uint32_t* scale, int* err, cudaStream_t s) {
  return launch_pool_range(g, dt, 0, g.L > 1 ? g.n[g.L - 1] : 0, q, k, v, pq, pk, pv, sq, scale, err, s);
}

// Coarsest blocks [cb0, cb0 + ncb) of every sequence: the tokens
// [cb0 p^(L-1), (cb0 + ncb) p^(L-1)) and the pyramid entries above them.
// scale: [kScaleRows][B][H] (rows q, k, v written; zeroed first when cb0 == 0).
cudaError_t launch_pool_range(const Geom& g, lh_dtype dt, int cb0, int ncb, const void* q, const void* k,
                              const void* v, void* pq, void* pk, void* pv, double* sq, uint32_t* scale, int* err,
                              cudaStream_t s) {
  if (dt == LH_BF16) return launch_t<__nv_bfloat16>(g, q, k, v, pq, pk, pv, sq, scale, cb0, ncb, err, s);
  return launch_t<float>(g, q, k, v, pq, pk, pv, sq, scale, cb0, ncb, err, s);
}

}  // namespace lh
