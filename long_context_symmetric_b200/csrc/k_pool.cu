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
// Two kernel forms with the same arithmetic (bit-identical results):
//  - ring form (k_pool): one thread owns 8 consecutive components of one head;
//    the D/8 lanes of a head are consecutive lanes of one warp. A thread walks
//    the p^(L-1) tokens of one coarsest-level block in order, keeping one
//    running fp64 sum per level (carry chain), and emits each entry when its
//    last child is in. Rows arrive through a shared-memory ring filled by bulk
//    async copies; the last warp done with a stage refills it.
//  - block-parallel form (k_pool_par, bf16): one CTA per (block, head,
//    tensor), a thread per level-1 entry and 8 components, higher levels from
//    shared-memory sums; for short token ranges and few heads.
// For bf16 and p in {2, 4, 8}, a level-1 entry's p values are summed in fp32
// where that chain is provably exact (sum_rows_bf16), else in fp64.
// HBM traffic: every token row is read once; pyramid rows and norms written once.
#include <algorithm>

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

// Sum of PP bf16 token rows (8 components each), as the fp64 chain
// ((x_0 + x_1) + x_2) + ... gives it, and the largest |x| among them (fp32
// bits). When, for every component, the PP values are normal (exponent field
// e in [1, 250]) and their fields differ by at most 16 - log2(PP), the chain is
// exact in fp32 as well, and it is summed there and widened once:
//   a normal bf16 with field e is a multiple of u = 2^(e_min - 134) and below
//   2^(e - 126) in magnitude, so every partial sum is a multiple of u below
//   PP * 2^(e_max - 126) = 2^(e_max - e_min + 8 + log2 PP) * u <= 2^24 u (and
//   below 2^127): each fp32 addition is exact, each fp64 addition of the chain
//   is exact too, and both give the exact sum.
// Otherwise (a zero, subnormal, infinite or NaN value, or a wider spread) the
// rows are widened to fp64 one by one and added in fp64, left to right. The
// result is the same bit pattern either way; the fast form saves the
// per-element fp32 -> fp64 conversions, which run on a narrow pipe.
template <int PP>
__device__ __forceinline__ void sum_rows_bf16(const typename Vec8<__nv_bfloat16>::Raw (&raw)[PP],
                                              double (&s)[8], uint32_t& amax) {
  constexpr uint32_t kMaxSpread = (16 - (PP == 2 ? 1 : PP == 4 ? 2 : 3)) << 7;
  uint32_t mx[4], mn[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) mx[w] = mn[w] = (&raw[0].a.x)[w] & 0x7FFF7FFFu;
#pragma unroll
  for (int u = 1; u < PP; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t a = (&raw[u].a.x)[w] & 0x7FFF7FFFu;
      mx[w] = max_u16x2(mx[w], a);
      mn[w] = min_u16x2(mn[w], a);
    }
  const uint32_t m = max_u16x2(max_u16x2(mx[0], mx[1]), max_u16x2(mx[2], mx[3]));
  amax = max(amax, max(m & 0xFFFFu, m >> 16) << 16);
  bool fast = true;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t ex = mx[w] & 0x7F807F80u, en = mn[w] & 0x7F807F80u;
    const uint32_t ex_lo = ex & 0xFFFFu, ex_hi = ex >> 16, en_lo = en & 0xFFFFu, en_hi = en >> 16;
    fast = fast && en_lo >= 0x80u && en_hi >= 0x80u && ex_lo <= (250u << 7) && ex_hi <= (250u << 7) &&
           ex_lo - en_lo <= kMaxSpread && ex_hi - en_hi <= kMaxSpread;
  }
  if (fast) {
    float f[8];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t x = (&raw[0].a.x)[w];
      f[2 * w] = __uint_as_float(x << 16);
      f[2 * w + 1] = __uint_as_float(x & 0xFFFF0000u);
    }
#pragma unroll
    for (int u = 1; u < PP; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t x = (&raw[u].a.x)[w];
        f[2 * w] = __fadd_rn(f[2 * w], __uint_as_float(x << 16));
        f[2 * w + 1] = __fadd_rn(f[2 * w + 1], __uint_as_float(x & 0xFFFF0000u));
      }
#pragma unroll
    for (int d = 0; d < 8; ++d) s[d] = (double)f[d];
  } else {
#pragma unroll
    for (int u = 0; u < PP; ++u) {
      double xr[8];
      Vec8<__nv_bfloat16>::raw_f64(raw[u], xr);
#pragma unroll
      for (int d = 0; d < 8; ++d) s[d] = u == 0 ? xr[d] : __dadd_rn(s[d], xr[d]);
    }
  }
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
  int* done = reinterpret_cast<int*>(full + a.ns);   // warps done with each stage
  __shared__ tc::Abort ab;
  const int nstages = (int)((P + a.ts - 1) / a.ts);
  const bool contiguous = (a.hg == g.H);
  const int nwarps = (blockDim.x + 31) >> 5;
  if (threadIdx.x == 0) {
    ab.flag = 0;
    for (int s2 = 0; s2 < a.ns; ++s2) {
      mbar_init(&full[s2], 1);
      done[s2] = 0;
    }
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
  for (int kk = 0; kk < nstages; ++kk) {
    const int slot = kk % a.ns;
    const bool ok = tc::mbar_wait(&full[slot], (kk / a.ns) & 1, &ab, err, 200);
    if (!__all_sync(wmask, ok)) break;   // copies never landed: reported, the warp leaves
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
        if constexpr (sizeof(T) == 2 && !MP) {
          sum_rows_bf16<PP>(raw, s, amax);
        } else {
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
    // the last warp to finish with this stage refills it (no CTA-wide barrier:
    // a warp moves on to the next stage as soon as it has landed)
    __syncwarp(wmask);
    if ((threadIdx.x & 31) == 0) {
      __threadfence_block();
      if (atomicAdd(&done[slot], 1) == nwarps - 1) {
        atomicExch(&done[slot], 0);
        __threadfence_block();
        if (kk + a.ns < nstages) issue(kk + a.ns);
      }
    }
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

// Pyramid entry e (its row index in the level-major pyramid) of level l with
// fp64 sum sm over this thread's 8 components: the mean (sum * 2^-l log2 p, or
// sum / p^l) stored to the row, and, for queries and keys, the squared norm
// of the mean in the pinned order (chunk left to right, then the butterfly
// over the C8 lanes of the row, which are aligned lanes of one warp). Every
// lane of the warp calls it (the norm's shuffles); `live` lanes store.
// inv: 1 / p^l (exact when p is a power of two; otherwise unused, the mean is
// an IEEE division by p^l).
template <typename T>
__device__ __forceinline__ void emit_entry(const Geom& g, int l, double inv, size_t e, const double (&sm)[8],
                                           bool live, int c8, int C8, bool norm, T* dst_head, double* sq_head) {
  double m[8];
  if (g.pow2) {
#pragma unroll
    for (int d = 0; d < 8; ++d) m[d] = __dmul_rn(sm[d], inv);
  } else {
    const double den = (double)g.pl[l];
#pragma unroll
    for (int d = 0; d < 8; ++d) m[d] = __ddiv_rn(sm[d], den);
  }
  if (live) Vec8<T>::store_f64(dst_head + e * g.D, m);
  if (norm) {
    double part = __dmul_rn(m[0], m[0]);
#pragma unroll
    for (int d = 1; d < 8; ++d) part = __dadd_rn(part, __dmul_rn(m[d], m[d]));
    for (int off = C8 >> 1; off >= 1; off >>= 1) part = __dadd_rn(part, __shfl_xor_sync(0xffffffffu, part, off));
    if (live && c8 == 0) sq_head[e] = part;
  }
}

// Block-parallel form (bf16 I/O, p a compile-time 2, 4 or 8, the mean-norm
// scores): one CTA per (coarsest block, head, tensor). Thread (i, c8) owns the
// 8 components c8 of level-1 entries i, i + slots, ...: it reads the entry's p
// token rows (16 bytes each, all loads issued together), sums them left to
// right in fp64 and emits the mean and its norm, keeping the fp64 sum in shared
// memory. Each higher level then sums its p children's sums from shared
// memory, left to right, on the threads of its entries. Every sum, mean and
// norm is formed as in k_pool, so the results are bit-identical; the unit of
// parallel work is a level-1 entry instead of a whole coarsest block, so a
// short token range still fills the SMs and no thread holds a carry chain.
// CTAs of one token block's heads are adjacent in the grid, so the token rows
// are read whole across them at about the same time.
// Shared layout of a level: sums[(i * 8 + d) * C8 + c8] (component d of chunk
// c8 of entry i), so the lanes of a warp touch consecutive doubles.
constexpr int kParThreads = 512;

template <typename T, int PP, int LV>
__global__ void __launch_bounds__(kParThreads, 2) k_pool_par(const T* __restrict__ q, const T* __restrict__ k,
                                                             const T* __restrict__ v, T* __restrict__ pq,
                                                             T* __restrict__ pk, T* __restrict__ pv,
                                                             double* __restrict__ sq, uint32_t* __restrict__ scale,
                                                             Geom g, int cb0) {
  extern __shared__ __align__(16) double sums[];   // fp64 sums of levels 1 .. LV-1 of this block
  constexpr int p = PP;
  const int C8 = g.D >> 3;
  const int tensor = blockIdx.z % 3, b = blockIdx.z / 3;
  const int head = (int)(blockIdx.x % (unsigned)g.H);
  const int cb = cb0 + (int)(blockIdx.x / (unsigned)g.H);
  const T* x = tensor == 0 ? q : (tensor == 1 ? k : v);
  T* pyr = tensor == 0 ? pq : (tensor == 1 ? pk : pv);
  const long long P = g.pl[LV];
  const int n1 = (int)(P / p);                   // level-1 entries of the block
  const int c8 = (int)threadIdx.x % C8;
  const int slots = (int)blockDim.x / C8;        // entries handled at once
  const size_t tok_stride = (size_t)g.H * g.D;
  const T* src = x + ((size_t)b * g.N + (size_t)cb * P) * tok_stride + (size_t)head * g.D + c8 * 8;
  T* dst_head = pyr + ((size_t)b * g.H + head) * (size_t)g.E * g.D + c8 * 8;
  double* sq_head = tensor < 2 ? sq + ((size_t)tensor * g.B * g.H + (size_t)b * g.H + head) * g.E : nullptr;
  uint32_t amax = 0;
  int base[LV + 1];                              // offset (doubles) of level l's sums
  {
    int o = 0, ne = n1;
#pragma unroll
    for (int l = 1; l <= LV; ++l) {
      base[l] = o;
      o += ne * g.D;
      ne /= p;
    }
  }
  // entry i of level l (of this block) has fp64 sum sm: store its mean, its norm
  auto finish = [&](int l, int i, const double (&sm)[8], bool live) {
    const size_t e = (size_t)g.off[l] + (size_t)cb * (size_t)(P / g.pl[l]) + i;
    emit_entry<T>(g, l, 1.0 / (double)g.pl[l], e, sm, live, c8, C8, tensor < 2, dst_head, sq_head);
  };
  // level 1 from the token rows (the loop bounds are uniform over the CTA, so
  // every lane takes the norm's shuffles)
  for (int i0 = 0; i0 < n1; i0 += slots) {
    const int i = i0 + (int)threadIdx.x / C8;
    const bool live = i < n1;
    typename Vec8<T>::Raw raw[PP];
#pragma unroll
    for (int u = 0; u < PP; ++u) {
      if (live) Vec8<T>::load_raw(src + (size_t)(i * p + u) * tok_stride, raw[u]);
      else raw[u] = typename Vec8<T>::Raw{};
    }
    double sm[8];
    sum_rows_bf16<PP>(raw, sm, amax);
    if (LV > 1 && live) {
#pragma unroll
      for (int d = 0; d < 8; ++d) sums[base[1] + (i * 8 + d) * C8 + c8] = sm[d];
    }
    finish(1, i, sm, live);
  }
  // levels 2 .. LV from the children's sums
#pragma unroll
  for (int l = 2; l <= LV; ++l) {
    __syncthreads();                             // level l-1 complete
    const int nl = (int)(P / g.pl[l]);
    for (int i0 = 0; i0 < nl; i0 += slots) {
      const int i = i0 + (int)threadIdx.x / C8;
      const bool live = i < nl;
      if (!__any_sync(0xffffffffu, live)) continue;   // warp-uniform
      double sm[8];
#pragma unroll
      for (int d = 0; d < 8; ++d) {
        double acc = 0.0;
        if (live) {
          const double* ch = sums + base[l - 1] + ((size_t)i * p * 8 + d) * C8 + c8;
          acc = ch[0];
#pragma unroll
          for (int u = 1; u < PP; ++u) acc = __dadd_rn(acc, ch[(size_t)u * 8 * C8]);
          if (l < LV) sums[base[l] + (i * 8 + d) * C8 + c8] = acc;
        }
        sm[d] = acc;
      }
      finish(l, i, sm, live);
    }
  }
  if constexpr (sizeof(T) == 2) {
    // the head's largest magnitude (tokens; pooled means are no larger)
    amax = __reduce_max_sync(0xffffffffu, amax);
    if ((threadIdx.x & 31) == 0 && amax) atomicMax(scale + (size_t)tensor * g.B * g.H + (size_t)b * g.H + head, amax);
  }
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
  const int C8 = g.D / 8;
  int hg = g.H;
  while (hg * C8 > 256) {   // ring form: largest divisor of H that fits 256 threads
    --hg;
    while (g.H % hg) --hg;
  }
  // The ring form streams well when its CTAs have at least 4 warps (H * D >=
  // 1024), walk coarsest blocks of at least 64 tokens and fill the SMs at least
  // twice over; a short token range, or few or narrow heads, leaves it with few
  // warps, and the block-parallel form (bf16) takes it.
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const bool ring_fills = hg * C8 >= 128 && g.pl[LV] >= 64 && (long long)ncb * (g.H / hg) * 3 * g.B >= 4LL * nsm;
  if constexpr (sizeof(T) == 2) {
  if (!ring_fills && g.score != LH_SCORE_MAXPOOL && (g.p == 2 || g.p == 4 || g.p == 8)) {
    // block-parallel form (bf16): one CTA per (coarsest block, head, tensor)
    const long long n1 = g.pl[LV] / g.p;
    const int threads = (int)std::min<long long>(kParThreads, ((n1 * C8 + 31) / 32) * 32);
    size_t smem = 0;
    for (int l = 1; l < LV; ++l) smem += (size_t)(g.pl[LV] / g.pl[l]) * g.D * sizeof(double);
    if (threads >= C8 && smem <= 200 * 1024 && (long long)ncb * g.H <= 0x7fffffffLL) {
      dim3 grid((unsigned)ncb * (unsigned)g.H, 1, 3 * g.B);
      const T* tq = (const T*)q; const T* tk = (const T*)k; const T* tv = (const T*)v;
      T* tpq = (T*)pq; T* tpk = (T*)pk; T* tpv = (T*)pv;
      cudaError_t e = cudaSuccess;
      switch (LV * 16 + g.p) {
#define LH_PAR(n, P)                                                                                        \
  case n * 16 + P:                                                                                         \
    e = cudaFuncSetAttribute(k_pool_par<T, P, n>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                                        \
    k_pool_par<T, P, n><<<grid, threads, smem, s>>>(tq, tk, tv, tpq, tpk, tpv, sq, scale, g, cb0);         \
    break;
#define LH_PAR_L(n) LH_PAR(n, 2) LH_PAR(n, 4) LH_PAR(n, 8)
        LH_PAR_L(1) LH_PAR_L(2) LH_PAR_L(3) LH_PAR_L(4) LH_PAR_L(5) LH_PAR_L(6) LH_PAR_L(7)
#undef LH_PAR_L
#undef LH_PAR
        default: return cudaErrorInvalidValue;
      }
      count_launch();
      return cudaGetLastError();
    }
  }
  }
  PoolArgs a;
  a.g = g;
  a.cb0 = cb0;
  const int stage_bytes = 32768;
  a.hg = hg;
  a.row_bytes = hg * g.D * (int)sizeof(T);
  const long long P = g.pl[LV];
  int ts = 1;
  while (ts * 2 * a.row_bytes <= stage_bytes && ts * 2 <= P) ts *= 2;
  a.ts = ts;
  a.ns = 3;
  const size_t smem = (size_t)a.ns * a.ts * a.row_bytes + a.ns * (sizeof(uint64_t) + sizeof(int));
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
