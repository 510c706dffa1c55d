// Scatter back (forward), its adjoint (block sums, backward) and the spread of
// the sub-sequence gradients onto the tokens (backward of gather + mean-pool).
//
// "Long Context Pre-Training with Lighthouse Attention", §3.1 stage (iv):
// every output of the sub-sequence is written back onto the p^l token positions
// its entry stands for; Fig. 1: gradients flow back through the scatter, the
// attention and the gather to the pyramid pool.
//
// B200 design: owner-computes instead of atomics. The entries covering token t
// are the chain of its ancestors (t / p^l at level l) from the coarsest level
// down to the first entry that was not expanded; the slot table written by
// lh_score_topk gives each ancestor's slot and expanded bit (levels >= 1), and a
// token included at level 0 sits p - (t mod p) slots before its level-1
// parent. One thread owns 8 components of one (token, head) row, sums its
// contributions coarse level first in registers and writes the row once:
// every output byte is written exactly once, no read-modify-write, and the
// result does not depend on scheduling. The accumulation arithmetic follows
// lh_accum (fp32, or int64 fixed point with one count = 2^-32).
#include "tc_ptx.cuh"   // lh_common.cuh, mbarrier helpers

namespace lh {
namespace {

constexpr double kTwo32 = 4294967296.0;
constexpr double kTwoM32 = 1.0 / 4294967296.0;

// Accumulator for one thread's 8 components.
template <int FIXED> struct Acc;
template <> struct Acc<0> {
  float v[8];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int d = 0; d < 8; ++d) v[d] = 0.f;
  }
  __device__ __forceinline__ void add(const float (&x)[8], float w, double, double) {
#pragma unroll
    for (int d = 0; d < 8; ++d) v[d] = __fadd_rn(v[d], __fmul_rn(x[d], w));
  }
  __device__ __forceinline__ void value(float (&o)[8]) const {
#pragma unroll
    for (int d = 0; d < 8; ++d) o[d] = v[d];
  }
  __device__ __forceinline__ void value64(double (&o)[8]) const {
#pragma unroll
    for (int d = 0; d < 8; ++d) o[d] = v[d];
  }
};
template <> struct Acc<1> {
  long long v[8];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int d = 0; d < 8; ++d) v[d] = 0;
  }
  // count = round_half_even(x * 2^32 / den), den = p^l (1 for weight 1); the
  // quotient is formed as one IEEE division, or as the (identical) exact
  // scaling by 1/den when den is a power of two (inv != 0)
  __device__ __forceinline__ void add(const float (&x)[8], float, double den, double inv) {
#pragma unroll
    for (int d = 0; d < 8; ++d) {
      const double t = __dmul_rn((double)x[d], kTwo32);
      const double qt = den == 1.0 ? t : (inv != 0.0 ? __dmul_rn(t, inv) : __ddiv_rn(t, den));
      v[d] += __double2ll_rn(qt);
    }
  }
  __device__ __forceinline__ void value64(double (&o)[8]) const {
#pragma unroll
    for (int d = 0; d < 8; ++d) o[d] = __dmul_rn(__ll2double_rn(v[d]), kTwoM32);
  }
};

template <typename T, int FIXED>
__device__ __forceinline__ void store_acc(T* dst, const Acc<FIXED>& a);

template <>
__device__ __forceinline__ void store_acc<__nv_bfloat16, 0>(__nv_bfloat16* dst, const Acc<0>& a) {
  float o[8];
  a.value(o);
  Vec8<__nv_bfloat16>::store_f32(dst, o);
}
template <>
__device__ __forceinline__ void store_acc<float, 0>(float* dst, const Acc<0>& a) {
  float o[8];
  a.value(o);
  Vec8<float>::store_f32(dst, o);
}
template <>
__device__ __forceinline__ void store_acc<__nv_bfloat16, 1>(__nv_bfloat16* dst, const Acc<1>& a) {
  double o[8];
  a.value64(o);
  Vec8<__nv_bfloat16>::store_f64(dst, o);
}
template <>
__device__ __forceinline__ void store_acc<float, 1>(float* dst, const Acc<1>& a) {
  double o[8];
  a.value64(o);
  Vec8<float>::store_f64(dst, o);
}

// Sum, over the entries covering token t of head bh, of w_l * src[slot] (8 components).
template <int FIXED, bool WEIGHTED>
__device__ __forceinline__ void chain_sum(const Geom& g, const float* __restrict__ src,
                                          const int32_t* __restrict__ slot_h, long long bh, int t,
                                          int c8, Acc<FIXED>& acc) {
  acc.zero();
  float x[8];
  if (g.L == 1) {
    load8_f32(src + ((size_t)bh * g.S + t) * g.D + c8 * 8, x);
    acc.add(x, 1.f, 1.0, 1.0);
    return;
  }
  int l = g.L - 1;
  int e = __ldg(slot_h + g.off[l] + (int)(t / g.pl[l]));
  while (true) {
    if (slot_in(e, g)) {          // (partition reading: an expanded entry is not in the sub-sequence)
      load8_f32(src + ((size_t)bh * g.S + (e >> 1)) * g.D + c8 * 8, x);
      const double den = WEIGHTED ? (double)g.pl[l] : 1.0;
      const double inv = g.pow2 ? 1.0 / den : 0.0;     // exact when p is a power of two
      acc.add(x, WEIGHTED ? (float)(1.0 / den) : 1.f, den, inv);
    }
    if (!(e & 1)) break;          // not expanded: no finer entry covers t
    if (l == 1) {                 // expanded level-1 parent: t itself is in the sub-sequence
      const int s0 = slot_tokens(e, g) + (t % g.p);
      load8_f32(src + ((size_t)bh * g.S + s0) * g.D + c8 * 8, x);
      acc.add(x, 1.f, 1.0, 1.0);
      break;
    }
    --l;
    e = __ldg(slot_h + g.off[l] + (int)(t / g.pl[l]));
  }
}

// o[b][t][h][:] = sum of os rows covering t (weights 1, or 1/p^l when
// WEIGHTED), for the tokens t0 .. t0 + nt - 1 of every sequence. One thread per
// 8 output components, each walking its token's chain of covering entries: the
// same sums in the same order as k_scatter_tree, with parallelism over tokens
// (the form a short token range needs).
template <typename T, int FIXED, bool WEIGHTED>
__global__ void __launch_bounds__(256) k_scatter(const float* __restrict__ os,
                                                 const int32_t* __restrict__ slot,
                                                 T* __restrict__ o, Geom g, int t0, int nt) {
  const int C8 = g.D >> 3;
  const long long total = (long long)g.B * nt * g.H * C8;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c8 = (int)(i % C8);
    const long long r = i / C8;                 // (b, t - t0, h) within the range
    const int h = (int)(r % g.H);
    const long long bt = r / g.H;
    const int t = t0 + (int)(bt % nt);
    const long long b = bt / nt;
    const long long bh = b * g.H + h;
    Acc<FIXED> acc;
    chain_sum<FIXED, WEIGHTED>(g, os, slot + bh * g.E, bh, t, c8, acc);
    store_acc<T, FIXED>(o + (((size_t)b * g.N + t) * g.H + h) * g.D + c8 * 8, acc);
  }
}

// dx[b][t][h][:] = sum of dxs rows covering t, weighted 1/p^l; three tensors (grid.y).
template <typename T, int FIXED>
__global__ void __launch_bounds__(256) k_spread(const float* __restrict__ dqs,
                                                const float* __restrict__ dks,
                                                const float* __restrict__ dvs,
                                                const int32_t* __restrict__ slot,
                                                T* __restrict__ dq, T* __restrict__ dk,
                                                T* __restrict__ dv, Geom g) {
  const int C8 = g.D >> 3;
  const long long total = (long long)g.B * g.N * g.H * C8;
  const float* src = blockIdx.y == 0 ? dqs : (blockIdx.y == 1 ? dks : dvs);
  T* dst = blockIdx.y == 0 ? dq : (blockIdx.y == 1 ? dk : dv);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c8 = (int)(i % C8);
    const long long r = i / C8;
    const int h = (int)(r % g.H);
    const long long bt = r / g.H;
    const int t = (int)(bt % g.N);
    const long long b = bt / g.N;
    const long long bh = b * g.H + h;
    Acc<FIXED> acc;
    chain_sum<FIXED, true>(g, src, slot + bh * g.E, bh, t, c8, acc);
    store_acc<T, FIXED>(dst + r * g.D + c8 * 8, acc);
  }
}

// Packed output row chunk: the value written for 8 components of one token.
template <typename T> struct Packed;
template <> struct Packed<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void from(const Acc<0>& a) {
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(a.v[2 * i], a.v[2 * i + 1]);
  }
  __device__ __forceinline__ void from(const Acc<1>& a) {
    double o[8];
    a.value64(o);
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = __double2bfloat16(o[i]);
  }
  __device__ __forceinline__ void store(__nv_bfloat16* p) const { *reinterpret_cast<uint4*>(p) = v; }
};
template <> struct Packed<float> {
  float4 a, b;
  __device__ __forceinline__ void from(const Acc<0>& x) {
    a = make_float4(x.v[0], x.v[1], x.v[2], x.v[3]);
    b = make_float4(x.v[4], x.v[5], x.v[6], x.v[7]);
  }
  __device__ __forceinline__ void from(const Acc<1>& x) {
    double o[8];
    x.value64(o);
    a = make_float4(__double2float_rn(o[0]), __double2float_rn(o[1]), __double2float_rn(o[2]),
                    __double2float_rn(o[3]));
    b = make_float4(__double2float_rn(o[4]), __double2float_rn(o[5]), __double2float_rn(o[6]),
                    __double2float_rn(o[7]));
  }
  __device__ __forceinline__ void store(float* p) const {
    reinterpret_cast<float4*>(p)[0] = a;
    reinterpret_cast<float4*>(p)[1] = b;
  }
};

// Contribution of one level-l row (weight 1/p^l when WEIGHTED and l >= 1, else 1).
template <int FIXED, bool WEIGHTED>
__device__ __forceinline__ void add_level(Acc<FIXED>& acc, const float (&x)[8], const Geom& g, int l) {
  const double den = (WEIGHTED && l >= 1) ? (double)g.pl[l] : 1.0;
  const double inv = g.pow2 ? 1.0 / den : 0.0;
  acc.add(x, (float)(1.0 / den), den, inv);
}

// Scatter / spread walking one coarsest block in token order (L >= 2).
// Every token under a level-l entry shares that entry's contribution, so the
// thread keeps acc[l] = sum of the contributions of levels >= l and refreshes
// it only where a level-l entry starts (integer countdowns, no division). When
// no level-0 row covers the token (its level-1 parent was not expanded), the
// output equals the previous token's and the converted value is stored again.
// Result and summation order (coarse level first) are those of chain_sum.
// One thread: 8 components of one head; CTA: a head group (x) by coarsest
// blocks (y). grid.z = batch x tensors.
template <typename T, int FIXED, bool WEIGHTED, int LV>
__global__ void __launch_bounds__(256) k_scatter_tree(const float* __restrict__ s0,
                                                      const float* __restrict__ s1,
                                                      const float* __restrict__ s2,
                                                      const int32_t* __restrict__ slot,
                                                      T* __restrict__ d0, T* __restrict__ d1,
                                                      T* __restrict__ d2, Geom g, int hg, int yb,
                                                      int ntens, int cb0, int cb_end, int nseg) {
  const int C8 = g.D >> 3;
  const int tensor = blockIdx.z % ntens;
  const int b = blockIdx.z / ntens;
  const int head = blockIdx.y * hg + threadIdx.x / C8;
  const int chunk = threadIdx.x % C8;
  // segment sg of coarsest block cb (nseg equal token segments per block)
  const int cs = cb0 * nseg + (int)blockIdx.x * yb + (int)threadIdx.y;
  if (cs >= cb_end * nseg) return;     // no collectives below: a thread may leave
  const int cb = cs / nseg, sg = cs - cb * nseg;
  const float* src = tensor == 0 ? s0 : (tensor == 1 ? s1 : s2);
  T* dst = tensor == 0 ? d0 : (tensor == 1 ? d1 : d2);
  const long long bh = (long long)b * g.H + head;
  const int32_t* slot_h = slot + bh * g.E;
  const float* srow = src + (size_t)bh * g.S * g.D + chunk * 8;
  const long long P = g.pl[LV];
  const long long seglen = P / nseg;
  const long long t_begin = (long long)sg * seglen;    // first token of the segment within the block
  const size_t tstride = (size_t)g.H * g.D;
  T* out = dst + ((size_t)b * g.N + (size_t)cb * P + (size_t)t_begin) * tstride + (size_t)head * g.D + chunk * 8;

  Acc<FIXED> acc[LV + 1];              // acc[l]: contributions of levels >= l (l >= 1)
  bool expd[LV + 1];                   // entry of level l expanded (its children included)
  int rem[LV + 1];                     // tokens left in the current level-l entry
  int idx[LV + 1];                     // index of the current level-l entry
  float x[8];
  int tok1 = 0, r0 = 0;                // first token slot of the current level-1 entry, offset in it
  {
    const int e = __ldg(slot_h + g.off[LV] + cb);
    acc[LV].zero();
    if (slot_in(e, g)) {
      load8_f32(srow + (size_t)(e >> 1) * g.D, x);
      add_level<FIXED, WEIGHTED>(acc[LV], x, g, LV);
    }
    expd[LV] = e & 1;
    if (LV == 1) tok1 = slot_tokens(e, g);
  }
  // the entries of levels LV-1 .. 1 that cover the segment's first token, as
  // the walk below meets an entry start (a segment starts on a level-1
  // boundary: seglen is a multiple of p)
#pragma unroll
  for (int l = LV - 1; l >= 1; --l) {
    const long long pos = t_begin % g.pl[l];
    rem[l] = (int)(g.pl[l] - pos);
    idx[l] = (int)(((long long)cb * P + t_begin) / g.pl[l]);
    if (expd[l + 1]) {
      const int e = __ldg(slot_h + g.off[l] + idx[l]);
      acc[l] = acc[l + 1];
      if (slot_in(e, g)) {
        load8_f32(srow + (size_t)(e >> 1) * g.D, x);
        add_level<FIXED, WEIGHTED>(acc[l], x, g, l);
      }
      expd[l] = e & 1;
      if (l == 1) tok1 = slot_tokens(e, g);
    } else {
      acc[l] = acc[l + 1];
      expd[l] = false;
    }
  }
  Packed<T> pk;
  bool pk_ok = false;
  for (long long t = 0; t < seglen; ++t) {
#pragma unroll
    for (int l = LV - 1; l >= 1; --l) {
      if (rem[l] == 0) {               // a level-l entry starts here (finer ones too)
        rem[l] = (int)g.pl[l];
        ++idx[l];
        if (expd[l + 1]) {
          const int e = __ldg(slot_h + g.off[l] + idx[l]);
          acc[l] = acc[l + 1];
          if (slot_in(e, g)) {
            load8_f32(srow + (size_t)(e >> 1) * g.D, x);
            add_level<FIXED, WEIGHTED>(acc[l], x, g, l);
          }
          expd[l] = e & 1;
          if (l == 1) tok1 = slot_tokens(e, g);
        } else {
          acc[l] = acc[l + 1];
          expd[l] = false;
        }
        if (l == 1) r0 = 0;
        pk_ok = false;
      }
      --rem[l];
    }
    T* o = out + (size_t)t * tstride;
    if (expd[1]) {                     // the token itself is in the sub-sequence
      // the p tokens of an expanded level-1 entry sit right before it
      // (post-order), right after it (pre-order), or at its run (partition)
      load8_f32(srow + (size_t)(tok1 + r0) * g.D, x);
      Acc<FIXED> a = acc[1];
      add_level<FIXED, WEIGHTED>(a, x, g, 0);
      Packed<T> q;
      q.from(a);
      q.store(o);
    } else {
      if (!pk_ok) {
        pk.from(acc[1]);
        pk_ok = true;
      }
      pk.store(o);
    }
    if (LV == 1 && ++r0 == g.p) r0 = 0;
    else if (LV > 1) ++r0;
  }
}

// Coarsest blocks [cb0, cb0 + ncb) (ncb < 0: all of them).
template <typename T, int FIXED, bool WEIGHTED>
cudaError_t tree_t(const Geom& g, const float* s0, const float* s1, const float* s2,
                   const int32_t* slot, T* d0, T* d1, T* d2, int ntens, cudaStream_t s, int cb0 = 0,
                   int ncb = -1) {
  const int C8 = g.D / 8;
  int hg = g.H;
  while (hg * C8 > 256) {
    --hg;
    while (g.H % hg) --hg;
  }
  const int ncoarse = ncb < 0 ? g.n[g.L - 1] : ncb;
  if (ncoarse <= 0) return cudaSuccess;
  // split a block's token walk into nseg segments (each a multiple of 64 tokens)
  // while there are fewer than 32 CTAs per SM: shorter walks, a smaller tail
  // (512K, fp32 accumulation: scatter 0.47 -> 0.42 ms, spread 1.29 -> 1.27 ms)
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const long long P = g.pl[g.L - 1];
  int nseg = 1;
  if (g.L > 2 && !FIXED)   // (the fixed-point walks, at 2 CTAs per SM, measured slower split)
    while (P / (2 * nseg) >= 64 && (P / (2 * nseg)) % g.p == 0 &&
           (long long)ncoarse * nseg * (g.H / hg) * g.B * ntens < 32LL * nsm)
      nseg *= 2;
  const int nunits = ncoarse * nseg;
  int yb = 1;
  while (yb * 2 * hg * C8 <= 256 && yb * 2 <= nunits) yb *= 2;
  dim3 block(hg * C8, yb);
  dim3 grid((nunits + yb - 1) / yb, g.H / hg, g.B * ntens);
  const int cb_end = cb0 + ncoarse;
  switch (g.L - 1) {
#define LH_TREE_CASE(n) \
    case n: k_scatter_tree<T, FIXED, WEIGHTED, n><<<grid, block, 0, s>>>(s0, s1, s2, slot, d0, d1, d2, g, hg, yb, ntens, cb0, cb_end, nseg); break;
    LH_TREE_CASE(1) LH_TREE_CASE(2) LH_TREE_CASE(3) LH_TREE_CASE(4)
    LH_TREE_CASE(5) LH_TREE_CASE(6) LH_TREE_CASE(7)
#undef LH_TREE_CASE
    default: return cudaErrorInvalidValue;
  }
  count_launch();
  return cudaGetLastError();
}

// Backward of the scatter: dos[j] = sum of dout over the tokens entry j covers,
// delta[j] = <dos[j], os[j]> with dos as stored. dos is stored as the backward's operand
// type TO: for bf16 I/O fp16 (block sums of up to p^(L-1) tokens need more
// significand than bf16 has) of the sum times 2^-e, e the head's power-of-two
// exponent (scale_exp of its largest block-sum magnitude). A first pass
// (REDO = false) stores with e = 0 and records each head's largest magnitude in
// the scale buffer; a second launch (REDO = true) redoes, with their exponent,
// only the heads whose largest magnitude lies outside [4, 256) (its CTAs of
// other heads leave at once). A non-finite block sum is reported as
// LH_ERR_DEVICE, detail 100. A thread owns 8 components of one head and
// walks the tokens of one coarsest block in order; level sums are fp32 and
// formed level by level (each the left-to-right sum of its p children), so
// every token row of dout is read exactly once per pass.
template <typename T, typename TO, int LV, bool REDO>
__global__ void __launch_bounds__(256) k_blocksum(const T* __restrict__ dout,
                                                  const float* __restrict__ os,
                                                  const int32_t* __restrict__ slot,
                                                  TO* __restrict__ dos, float* __restrict__ delta,
                                                  uint32_t* __restrict__ amax, Geom g, int hg, int yb, int* err) {
  const int C8 = g.D >> 3;
  const int b = blockIdx.z;
  const int head = blockIdx.y * hg + threadIdx.x / C8;
  const int chunk = threadIdx.x % C8;
  const int cb = blockIdx.x * yb + threadIdx.y;
  const int ncoarse = g.n[g.L - 1];
  const bool live = head < g.H && cb < ncoarse;
  const int ex = (REDO && sizeof(TO) == 2 && head < g.H)
                     ? scale_exp(amax[(size_t)kScaleDO * g.B * g.H + (size_t)b * g.H + head]) : 0;
  if (REDO && __syncthreads_and(ex == 0)) return;       // nothing of this CTA to redo
  const float mul = pow2f(-ex), unmul = pow2f(ex);
  uint32_t vmax = 0;                                     // largest |block sum| (fp32 bits), first pass
  const int p = g.p;
  const long long P = g.pl[LV];
  const size_t tok_stride = (size_t)g.H * g.D;
  const long long bh = (long long)b * g.H + head;
  const T* src = dout + ((size_t)b * g.N + (size_t)cb * P) * tok_stride + (size_t)head * g.D + chunk * 8;
  const int32_t* slot_h = slot + bh * g.E;

  // one included entry: write its row and its delta
  // scale: the entry's weight in the forward scatter (1, or 1/p^l under LH_WEIGHT_MEAN)
  auto emit = [&](int s, const float (&v0)[8], float scale) {
    float v[8];
#pragma unroll
    for (int d = 0; d < 8; ++d) v[d] = v0[d] * scale;
    float mx = 0.f;
#pragma unroll
    for (int d = 0; d < 8; ++d) mx = fmaxf(mx, fabsf(v[d]));
    if (sizeof(TO) == 2) {
#pragma unroll
      for (int d = 0; d < 8; ++d) v[d] *= mul;         // a power of two: exact
    }
    float part = 0.f;
    float ov[8];
    if (s >= 0 && !LH_BOUNDS(s < g.S, err, 303)) s = -1;
    if (live && s >= 0) {
      load8_f32(os + ((size_t)bh * g.S + s) * g.D + chunk * 8, ov);
      // delta from the stored (rounded) dos: the values the backward's dP uses
#pragma unroll
      for (int d = 0; d < 8; ++d)
        part = fmaf(sizeof(TO) == 2 ? __half2float(__float2half_rn(v[d])) : v[d], ov[d], part);
    }
    for (int off = C8 >> 1; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (live && s >= 0) {
      Vec8<TO>::store_f32(dos + ((size_t)bh * g.S + s) * g.D + chunk * 8, v);
      if (chunk == 0) delta[(size_t)bh * g.S + s] = part * unmul;
      if (sizeof(TO) == 2) {
        if (!(mx < INFINITY)) report_error(err, LH_ERR_DEVICE, 100);
        if (!REDO) vmax = max(vmax, __float_as_uint(mx));
      }
    }
  };

  float acc[LV + 1][8];   // acc[l]: running sum of the open entry of level l (acc[0] unused)
  float wl[LV + 1];        // weight of a level-l entry in the forward scatter
#pragma unroll
  for (int l = 0; l <= LV; ++l) wl[l] = g.weight == LH_WEIGHT_MEAN ? (float)(1.0 / (double)g.pl[l]) : 1.f;
  const long long ngroups = P / p;
  for (long long g1 = 0; g1 < ngroups; ++g1) {
    const long long i1 = (long long)cb * (P / p) + g1;      // level-1 index
    // the group's token rows and its level-1 slot entry, all loads issued together
    const int e1 = live ? __ldg(slot_h + g.off[1] + (int)i1) : -1;
    float s[8];
    for (int c0 = 0; c0 < p; c0 += 8) {
      const int nb = min(8, p - c0);
      typename Vec8<T>::Raw raw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < nb && live) Vec8<T>::load_raw(src + (size_t)(g1 * p + c0 + u) * tok_stride, raw[u]);
      const bool tok_in = e1 >= 0 && (e1 & 1);               // children (tokens) included
      const int tok0 = tok_in ? slot_tokens(e1, g) : -1;
      // tokens are emitted only where some lane of the warp has them included
      const bool any_tok = __any_sync(0xffffffffu, tok_in);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (u < nb) {
          float x[8];
          if (live) Vec8<T>::raw_f32(raw[u], x);
          else {
#pragma unroll
            for (int d = 0; d < 8; ++d) x[d] = 0.f;
          }
          if (c0 + u == 0) {
#pragma unroll
            for (int d = 0; d < 8; ++d) s[d] = x[d];
          } else {
#pragma unroll
            for (int d = 0; d < 8; ++d) s[d] = __fadd_rn(s[d], x[d]);
          }
          if (any_tok) emit(tok_in ? tok0 + c0 + u : -1, x, 1.f);
        }
      }
    }
#pragma unroll
    for (int d = 0; d < 8; ++d) acc[1][d] = s[d];
    const bool in1 = slot_in(e1, g);
    if (__any_sync(0xffffffffu, in1)) emit(in1 ? (e1 >> 1) : -1, s, wl[1]);
    long long gi = i1;
#pragma unroll
    for (int l = 2; l <= LV; ++l) {
      const int pos = (int)(gi % p);
      if (pos == 0) {
#pragma unroll
        for (int d = 0; d < 8; ++d) acc[l][d] = acc[l - 1][d];
      } else {
#pragma unroll
        for (int d = 0; d < 8; ++d) acc[l][d] = __fadd_rn(acc[l][d], acc[l - 1][d]);
      }
      if (pos != p - 1) break;
      gi /= p;
      const int e = live ? __ldg(slot_h + g.off[l] + (int)gi) : -1;
      const bool in = slot_in(e, g);
      if (__any_sync(0xffffffffu, in)) emit(in ? (e >> 1) : -1, acc[l], wl[l]);
    }
  }
  if (!REDO && sizeof(TO) == 2) {
    for (int off = C8 >> 1; off >= 1; off >>= 1) vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
    if (live && chunk == 0 && vmax) atomicMax(amax + (size_t)kScaleDO * g.B * g.H + bh, vmax);
  }
}

// (Token slots: the p tokens of an expanded level-1 entry sit right before its
// slot in post-order, right after it in pre-order, at its run start under the
// partition reading; slot_tokens.)
// Same block sums with the token rows streamed through a shared-memory ring
// filled by 1-D bulk async copies (one CTA per coarsest block and head group;
// hg * D / 8 threads, a multiple of 32). PP = p, a compile-time 2, 4 or 8 that
// divides the stage: a level-1 group's PP rows are read from shared memory
// together. Emission order and arithmetic are those of k_blocksum.
struct RingArgs {
  int hg;          // heads per CTA (a divisor of H)
  int ts;          // tokens per stage
  int ns;          // stages
  int row_bytes;   // bytes of one token row of the head group
};

__device__ __forceinline__ void bs_bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

template <typename T, typename TO, int LV, int PP, bool REDO>
__global__ void __launch_bounds__(256, 2) k_blocksum_ring(const T* __restrict__ dout,
                                                          const float* __restrict__ os,
                                                          const int32_t* __restrict__ slot,
                                                          TO* __restrict__ dos, float* __restrict__ delta,
                                                          uint32_t* __restrict__ amax, Geom g, RingArgs a,
                                                          int* err) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int C8 = g.D >> 3;
  const int b = blockIdx.z;
  const int hg0 = blockIdx.y * a.hg;
  const int head = hg0 + threadIdx.x / C8;
  const int chunk = threadIdx.x % C8;
  const int cb = blockIdx.x;
  constexpr int p = PP;
  const long long P = g.pl[LV];
  const size_t tok_stride = (size_t)g.H * g.D;
  const long long bh = (long long)b * g.H + head;
  const T* src0 = dout + ((size_t)b * g.N + (size_t)cb * P) * tok_stride + (size_t)hg0 * g.D;
  const int32_t* slot_h = slot + bh * g.E;
  // the head's power-of-two exponent (second pass only; see k_blocksum)
  const int ex = (REDO && sizeof(TO) == 2) ? scale_exp(amax[(size_t)kScaleDO * g.B * g.H + bh]) : 0;
  if (REDO && __syncthreads_and(ex == 0)) return;       // nothing of this CTA to redo
  const float mul = pow2f(-ex), unmul = pow2f(ex);
  uint32_t vmax = 0;
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
      tc::mbar_init(&full[s2], 1);
      done[s2] = 0;
    }
    tc::fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int kk) {
    const int si = kk % a.ns;
    const long long t0 = (long long)kk * a.ts;
    const int nt = (int)min((long long)a.ts, P - t0);
    uint8_t* dst = smem + (size_t)si * a.ts * row_bytes;
    tc::mbar_expect_tx(&full[si], (uint32_t)(nt * row_bytes));
    if (contiguous) {
      bs_bulk_load(dst, src0 + t0 * tok_stride, (uint32_t)(nt * row_bytes), &full[si]);
    } else {
      for (int u = 0; u < nt; ++u)
        bs_bulk_load(dst + (size_t)u * row_bytes, src0 + (t0 + u) * tok_stride, (uint32_t)row_bytes, &full[si]);
    }
  };
  if (threadIdx.x == 0)
    for (int kk = 0; kk < a.ns && kk < nstages; ++kk) issue(kk);

  // one included entry: write its row and its delta
  // scale: the entry's weight in the forward scatter (1, or 1/p^l under LH_WEIGHT_MEAN)
  // ov_pre: the entry's os row when already loaded (else it is loaded here)
  auto emit = [&](int s, const float (&v0)[8], float scale, const float* ov_pre) {
    float v[8];
#pragma unroll
    for (int d = 0; d < 8; ++d) v[d] = v0[d] * scale;
    float mx = 0.f;
#pragma unroll
    for (int d = 0; d < 8; ++d) mx = fmaxf(mx, fabsf(v[d]));
    if (sizeof(TO) == 2) {
#pragma unroll
      for (int d = 0; d < 8; ++d) v[d] *= mul;         // a power of two: exact
    }
    float part = 0.f;
    float ov[8];
    if (s >= 0 && !LH_BOUNDS(s < g.S, err, 303)) s = -1;
    if (s >= 0) {
      if (ov_pre) {
#pragma unroll
        for (int d = 0; d < 8; ++d) ov[d] = ov_pre[d];
      } else {
        load8_f32(os + ((size_t)bh * g.S + s) * g.D + chunk * 8, ov);
      }
      // delta from the stored (rounded) dos: the values the backward's dP uses
#pragma unroll
      for (int d = 0; d < 8; ++d)
        part = fmaf(sizeof(TO) == 2 ? __half2float(__float2half_rn(v[d])) : v[d], ov[d], part);
    }
    for (int off = C8 >> 1; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (s >= 0) {
      Vec8<TO>::store_f32(dos + ((size_t)bh * g.S + s) * g.D + chunk * 8, v);
      if (chunk == 0) delta[(size_t)bh * g.S + s] = part * unmul;
      if (sizeof(TO) == 2) {
        if (!(mx < INFINITY)) report_error(err, LH_ERR_DEVICE, 100);
        if (!REDO) vmax = max(vmax, __float_as_uint(mx));
      }
    }
  };

  float acc[LV + 1][8];   // acc[l]: running sum of the open entry of level l (acc[0] unused)
  float wl[LV + 1];        // weight of a level-l entry in the forward scatter
#pragma unroll
  for (int l = 0; l <= LV; ++l) wl[l] = g.weight == LH_WEIGHT_MEAN ? (float)(1.0 / (double)g.pl[l]) : 1.f;
  const long long i1_end = (long long)(cb + 1) * (P / p);
  long long i1 = (long long)cb * (P / p);          // level-1 index of the next group
  int e1n = __ldg(slot_h + g.off[1] + (int)i1);    // its slot entry, fetched one group ahead
  for (int kk = 0; kk < nstages; ++kk) {
    const int si = kk % a.ns;
    const bool ok = tc::mbar_wait(&full[si], (kk / a.ns) & 1, &ab, err, 201);
    if (!__all_sync(0xffffffffu, ok)) break;   // copies never landed: reported, the warp leaves
    const long long t0 = (long long)kk * a.ts;
    const int nt = (int)min((long long)a.ts, P - t0);
    const uint8_t* buf = smem + (size_t)si * a.ts * row_bytes + (size_t)threadIdx.x * 8 * sizeof(T);
    for (int u0 = 0; u0 < nt; u0 += p, ++i1) {
      const int e1 = e1n;
      if (i1 + 1 < i1_end) e1n = __ldg(slot_h + g.off[1] + (int)(i1 + 1));
      // the level-1 entry's os row, loaded now so that its latency overlaps the sums
      float ov1[8];
      const bool in1 = slot_in(e1, g) && LH_BOUNDS((e1 >> 1) < g.S, err, 303);
      if (in1) load8_f32(os + ((size_t)bh * g.S + (e1 >> 1)) * g.D + chunk * 8, ov1);
      typename Vec8<T>::Raw raw[p];
#pragma unroll
      for (int u = 0; u < p; ++u)
        raw[u] = *reinterpret_cast<const typename Vec8<T>::Raw*>(buf + (size_t)(u0 + u) * row_bytes);
      const bool tok_in = e1 >= 0 && (e1 & 1) &&              // children (tokens) included
                          LH_BOUNDS(slot_tokens(e1, g) >= 0 && slot_tokens(e1, g) + p <= g.S, err, 303);
      // tokens are emitted only where some lane of the warp has them included
      const bool any_tok = __any_sync(0xffffffffu, tok_in);
      float sum[8];
      // the tokens' os rows, loaded TB at a time so that their latencies overlap
      // (fp32 rows of dout take twice the registers: smaller batches)
      constexpr int TB = p < 4 ? p : (sizeof(T) == 2 ? 4 : 2);
      const int tok0 = slot_tokens(e1, g);
      float ovt[TB][8];
#pragma unroll
      for (int u = 0; u < p; ++u) {
        if (u % TB == 0 && tok_in) {
#pragma unroll
          for (int w = 0; w < TB; ++w) load8_f32(os + ((size_t)bh * g.S + tok0 + u + w) * g.D + chunk * 8, ovt[w]);
        }
        float x[8];
        Vec8<T>::raw_f32(raw[u], x);
        if (u == 0) {
#pragma unroll
          for (int d = 0; d < 8; ++d) sum[d] = x[d];
        } else {
#pragma unroll
          for (int d = 0; d < 8; ++d) sum[d] = __fadd_rn(sum[d], x[d]);
        }
        if (any_tok) emit(tok_in ? tok0 + u : -1, x, 1.f, ovt[u % TB]);
      }
#pragma unroll
      for (int d = 0; d < 8; ++d) acc[1][d] = sum[d];
      if (__any_sync(0xffffffffu, in1)) emit(in1 ? (e1 >> 1) : -1, sum, wl[1], ov1);
      long long gi = i1;
#pragma unroll
      for (int l = 2; l <= LV; ++l) {
        const int pos = (int)(gi % p);
        if (pos == 0) {
#pragma unroll
          for (int d = 0; d < 8; ++d) acc[l][d] = acc[l - 1][d];
        } else {
#pragma unroll
          for (int d = 0; d < 8; ++d) acc[l][d] = __fadd_rn(acc[l][d], acc[l - 1][d]);
        }
        if (pos != p - 1) break;
        gi /= p;
        const int e = __ldg(slot_h + g.off[l] + (int)gi);
        const bool in = slot_in(e, g);
        if (__any_sync(0xffffffffu, in)) emit(in ? (e >> 1) : -1, acc[l], wl[l], nullptr);
      }
    }
    // the last warp to finish with this stage refills it (no CTA-wide barrier:
    // a warp moves on to the next stage as soon as it has landed)
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
      __threadfence_block();
      if (atomicAdd(&done[si], 1) == nwarps - 1) {
        atomicExch(&done[si], 0);
        __threadfence_block();
        if (kk + a.ns < nstages) issue(kk + a.ns);
      }
    }
  }
  if (!REDO && sizeof(TO) == 2) {
    for (int off = C8 >> 1; off >= 1; off >>= 1) vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
    if (chunk == 0 && vmax) atomicMax(amax + (size_t)kScaleDO * g.B * g.H + bh, vmax);
  }
}

// L == 1: dos = dout transposed to [B][H][N][D] (times the head's 2^-e, two
// passes as k_blocksum); delta = <dout, os>.
template <typename T, typename TO, bool REDO>
__global__ void __launch_bounds__(256) k_blocksum_l1(const T* __restrict__ dout,
                                                     const float* __restrict__ os,
                                                     TO* __restrict__ dos, float* __restrict__ delta,
                                                     uint32_t* __restrict__ amax, Geom g) {
  const int C8 = g.D >> 3;
  const long long total = (long long)g.B * g.H * g.N * C8;
  const size_t row_do = (size_t)kScaleDO * g.B * g.H;
  const long long stride = (long long)gridDim.x * blockDim.x;
  // every lane of a warp takes every iteration (the shuffles below need them
  // all); lanes past the end or with nothing to redo only skip the memory work
  for (long long base = (long long)blockIdx.x * blockDim.x; base < total; base += stride) {
    const long long i = base + threadIdx.x;
    const bool in = i < total;
    const long long ii = in ? i : total - 1;
    const int c8 = (int)(ii % C8);
    const long long r = ii / C8;         // (b, h, t) row of dos
    const int t = (int)(r % g.N);
    const long long bh = r / g.N;
    const int h = (int)(bh % g.H);
    const long long b = bh / g.H;
    const int ex = (REDO && sizeof(TO) == 2) ? scale_exp(amax[row_do + bh]) : 0;
    const bool work = in && !(REDO && ex == 0);
    float x[8], ov[8];
    if (work) {
      Vec8<T>::load_f32(dout + ((b * g.N + t) * g.H + h) * g.D + c8 * 8, x);
      load8_f32(os + r * g.D + c8 * 8, ov);
    } else {
#pragma unroll
      for (int d = 0; d < 8; ++d) x[d] = ov[d] = 0.f;
    }
    float part = 0.f;
#pragma unroll
    for (int d = 0; d < 8; ++d) part = fmaf(x[d], ov[d], part);
    for (int off = C8 >> 1; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (sizeof(TO) == 2 && !REDO) {
      // the row's largest magnitude (its C8 lanes), one atomic per row
      float mx = 0.f;
#pragma unroll
      for (int d = 0; d < 8; ++d) mx = fmaxf(mx, fabsf(x[d]));
      for (int off = C8 >> 1; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (work && c8 == 0 && mx > 0.f) atomicMax(amax + row_do + bh, __float_as_uint(mx));
    }
    if (!work) continue;
    if (sizeof(TO) == 2) {
      const float mul = pow2f(-ex);
#pragma unroll
      for (int d = 0; d < 8; ++d) x[d] *= mul;
    }
    Vec8<TO>::store_f32(dos + r * g.D + c8 * 8, x);
    if (c8 == 0) delta[r] = part;
  }
}

int grid_for(long long total) {
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return (int)blocks;
}

template <typename T>
cudaError_t scatter_t(const Geom& g, const float* os, const int32_t* slot, void* o, cudaStream_t s,
                      int cb0 = 0, int ncb = -1) {
  if (g.L > 1) {
    // weights 1 (the default reading) or 1/p^l (LH_WEIGHT_MEAN)
    if (g.weight == LH_WEIGHT_MEAN)
      return g.accum == LH_ACC_FIXED64
                 ? tree_t<T, 1, true>(g, os, os, os, slot, (T*)o, (T*)o, (T*)o, 1, s, cb0, ncb)
                 : tree_t<T, 0, true>(g, os, os, os, slot, (T*)o, (T*)o, (T*)o, 1, s, cb0, ncb);
    return g.accum == LH_ACC_FIXED64
               ? tree_t<T, 1, false>(g, os, os, os, slot, (T*)o, (T*)o, (T*)o, 1, s, cb0, ncb)
               : tree_t<T, 0, false>(g, os, os, os, slot, (T*)o, (T*)o, (T*)o, 1, s, cb0, ncb);
  }
  const long long total = (long long)g.B * g.N * g.H * (g.D / 8);
  if (g.accum == LH_ACC_FIXED64)
    k_scatter<T, 1, false><<<grid_for(total), 256, 0, s>>>(os, slot, (T*)o, g, 0, g.N);
  else
    k_scatter<T, 0, false><<<grid_for(total), 256, 0, s>>>(os, slot, (T*)o, g, 0, g.N);
  count_launch();
  return cudaGetLastError();
}

// A token range: the per-token chain walk (many threads even for a few
// coarsest blocks), bit-identical to the tree walk of the whole sequence.
template <typename T>
cudaError_t scatter_tokens_t(const Geom& g, const float* os, const int32_t* slot, void* o, int t0, int nt,
                             cudaStream_t s) {
  const long long total = (long long)g.B * nt * g.H * (g.D / 8);
  if (total <= 0) return cudaSuccess;
  const bool w = g.weight == LH_WEIGHT_MEAN;
  if (g.accum == LH_ACC_FIXED64) {
    if (w) k_scatter<T, 1, true><<<grid_for(total), 256, 0, s>>>(os, slot, (T*)o, g, t0, nt);
    else k_scatter<T, 1, false><<<grid_for(total), 256, 0, s>>>(os, slot, (T*)o, g, t0, nt);
  } else {
    if (w) k_scatter<T, 0, true><<<grid_for(total), 256, 0, s>>>(os, slot, (T*)o, g, t0, nt);
    else k_scatter<T, 0, false><<<grid_for(total), 256, 0, s>>>(os, slot, (T*)o, g, t0, nt);
  }
  count_launch();
  return cudaGetLastError();
}

template <typename T>
cudaError_t spread_t(const Geom& g, const float* dqs, const float* dks, const float* dvs,
                     const int32_t* slot, void* dq, void* dk, void* dv, cudaStream_t s) {
  if (g.L > 1)
    return g.accum == LH_ACC_FIXED64
               ? tree_t<T, 1, true>(g, dqs, dks, dvs, slot, (T*)dq, (T*)dk, (T*)dv, 3, s)
               : tree_t<T, 0, true>(g, dqs, dks, dvs, slot, (T*)dq, (T*)dk, (T*)dv, 3, s);
  const long long total = (long long)g.B * g.N * g.H * (g.D / 8);
  dim3 grid(grid_for(total), 3);
  if (g.accum == LH_ACC_FIXED64)
    k_spread<T, 1><<<grid, 256, 0, s>>>(dqs, dks, dvs, slot, (T*)dq, (T*)dk, (T*)dv, g);
  else
    k_spread<T, 0><<<grid, 256, 0, s>>>(dqs, dks, dvs, slot, (T*)dq, (T*)dk, (T*)dv, g);
  count_launch();
  return cudaGetLastError();
}

template <typename T, bool REDO>
cudaError_t blocksum_pass(const Geom& g, const void* dout, const float* os, const int32_t* slot,
                          void* dos, float* delta, uint32_t* amax, int* err, cudaStream_t s) {
  using TO = typename BwdOperand<T>::type;
  if (g.L == 1) {
    const long long total = (long long)g.B * g.H * g.N * (g.D / 8);
    k_blocksum_l1<T, TO, REDO><<<grid_for(total), 256, 0, s>>>((const T*)dout, os, (TO*)dos, delta, amax, g);
    count_launch();
    return cudaGetLastError();
  }
  const int C8 = g.D / 8;
  int hg = g.H;
  while (hg * C8 > 256) {
    --hg;
    while (g.H % hg) --hg;
  }
  const int ncoarse = g.n[g.L - 1];
  if ((hg * C8) % 32 == 0 && (g.p == 2 || g.p == 4 || g.p == 8)) {
    // ring-streamed variant: whole level-1 groups per stage
    RingArgs a;
    a.hg = hg;
    a.row_bytes = hg * g.D * (int)sizeof(T);
    const long long P = g.pl[g.L - 1];
    int ts = 1;
    while (ts * 2 * a.row_bytes <= 32768 && ts * 2 <= P) ts *= 2;
    a.ts = ts;
    a.ns = 3;
    if (ts % g.p == 0) {
      const size_t smem = (size_t)a.ns * a.ts * a.row_bytes + a.ns * (sizeof(uint64_t) + sizeof(int));
      dim3 rgrid(ncoarse, g.H / hg, g.B);
      const T* d = (const T*)dout;
      TO* o = (TO*)dos;
      cudaError_t e = cudaSuccess;
#define LH_BSR(n, P)                                                                                     \
  e = cudaFuncSetAttribute(k_blocksum_ring<T, TO, n, P, REDO>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           (int)smem);                                                                   \
  if (e != cudaSuccess) return e;                                                                        \
  k_blocksum_ring<T, TO, n, P, REDO><<<rgrid, hg * C8, smem, s>>>(d, os, slot, o, delta, amax, g, a, err);
#define LH_BSR_CASE(n)                                                                                   \
    case n:                                                                                              \
      if (g.p == 8) { LH_BSR(n, 8) } else if (g.p == 4) { LH_BSR(n, 4) } else { LH_BSR(n, 2) }          \
      break;
      switch (g.L - 1) {
        LH_BSR_CASE(1) LH_BSR_CASE(2) LH_BSR_CASE(3) LH_BSR_CASE(4)
        LH_BSR_CASE(5) LH_BSR_CASE(6) LH_BSR_CASE(7)
        default: return cudaErrorInvalidValue;
      }
#undef LH_BSR_CASE
#undef LH_BSR
      count_launch();
      return cudaGetLastError();
    }
  }
  int yb = 1;
  while (yb * 2 * hg * C8 <= 256 && yb * 2 <= ncoarse) yb *= 2;
  dim3 block(hg * C8, yb);
  dim3 grid((ncoarse + yb - 1) / yb, g.H / hg, g.B);
  const T* d = (const T*)dout;
  TO* o = (TO*)dos;
  switch (g.L - 1) {
#define LH_BS_CASE(n) \
    case n: k_blocksum<T, TO, n, REDO><<<grid, block, 0, s>>>(d, os, slot, o, delta, amax, g, hg, yb, err); break;
    LH_BS_CASE(1) LH_BS_CASE(2) LH_BS_CASE(3) LH_BS_CASE(4)
    LH_BS_CASE(5) LH_BS_CASE(6) LH_BS_CASE(7)
#undef LH_BS_CASE
    default: return cudaErrorInvalidValue;
  }
  count_launch();
  return cudaGetLastError();
}

// bf16 I/O: the dO row of the scale buffer is zeroed, the first pass stores the
// block sums unscaled and records each head's largest magnitude, the second
// redoes the heads whose magnitude needs a power-of-two exponent. fp32 I/O:
// one pass, no scaling.
template <typename T>
cudaError_t blocksum_t(const Geom& g, const void* dout, const float* os, const int32_t* slot,
                       void* dos, float* delta, uint32_t* amax, int* err, cudaStream_t s) {
  constexpr bool F16 = sizeof(typename BwdOperand<T>::type) == 2;
  if (F16) {
    cudaError_t e = launch_scale_zero(amax, kScaleDO, 1, g.B * g.H, s);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = blocksum_pass<T, false>(g, dout, os, slot, dos, delta, amax, err, s);
  if (e != cudaSuccess || !F16) return e;
  return blocksum_pass<T, true>(g, dout, os, slot, dos, delta, amax, err, s);
}

}  // namespace

cudaError_t launch_scatter(const Geom& g, lh_dtype dt, const float* os, const int32_t* slot,
                           void* o, cudaStream_t s) {
  return dt == LH_BF16 ? scatter_t<__nv_bfloat16>(g, os, slot, o, s)
                       : scatter_t<float>(g, os, slot, o, s);
}

// Tokens of the coarsest blocks [cb0, cb0 + ncb) only (L >= 2). Ranges of
// fewer blocks than the GPU has SMs run the per-token walk; longer ones the
// tree walk of the whole sequence restricted to their blocks.
cudaError_t launch_scatter_range(const Geom& g, lh_dtype dt, int cb0, int ncb, const float* os,
                                 const int32_t* slot, void* o, cudaStream_t s) {
  if (g.L < 2) return cudaErrorInvalidValue;
  // a few coarsest blocks: a walk per token; otherwise the tree walk, split
  // into token segments (8,192-token ranges at 512K: 2.9 ms for the 64 chunks
  // against 3.7 ms per token)
  if (ncb * (long long)g.B < 16) {
    const int P = (int)g.pl[g.L - 1];
    return dt == LH_BF16 ? scatter_tokens_t<__nv_bfloat16>(g, os, slot, o, cb0 * P, ncb * P, s)
                         : scatter_tokens_t<float>(g, os, slot, o, cb0 * P, ncb * P, s);
  }
  return dt == LH_BF16 ? scatter_t<__nv_bfloat16>(g, os, slot, o, s, cb0, ncb)
                       : scatter_t<float>(g, os, slot, o, s, cb0, ncb);
}

cudaError_t launch_spread(const Geom& g, lh_dtype dt, const float* dqs, const float* dks,
                          const float* dvs, const int32_t* slot, void* dq, void* dk, void* dv,
                          cudaStream_t s) {
  return dt == LH_BF16 ? spread_t<__nv_bfloat16>(g, dqs, dks, dvs, slot, dq, dk, dv, s)
                       : spread_t<float>(g, dqs, dks, dvs, slot, dq, dk, dv, s);
}

cudaError_t launch_scatter_bwd(const Geom& g, lh_dtype dt, const void* dout, const float* os,
                               const int32_t* slot, void* dos, float* delta, uint32_t* scale, int* err,
                               cudaStream_t s) {
  return dt == LH_BF16 ? blocksum_t<__nv_bfloat16>(g, dout, os, slot, dos, delta, scale, err, s)
                       : blocksum_t<float>(g, dout, os, slot, dos, delta, scale, err, s);
}

}  // namespace lh
