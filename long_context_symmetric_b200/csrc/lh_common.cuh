// Device-side helpers shared by the liblh kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>

#include "lh.h"

namespace lh {

// Problem geometry, computed once on the host by lh_plan and passed by value.
struct Geom {
  int B, H, N, D, p, L, K, S, E;
  int n[LH_MAX_LEVELS];
  int k[LH_MAX_LEVELS];
  int c[LH_MAX_LEVELS];        // entries of level l in the sub-sequence
  int cand[LH_MAX_LEVELS];     // candidates at level l (the selection's working arrays)
  int C;                       // sum of cand
  int off[LH_MAX_LEVELS];      // start of level l (>= 1) in the per-head E axis
  long long pl[LH_MAX_LEVELS]; // p^l
  int pow2;                    // p is a power of two (division by p^l is exact scaling)
  int accum;                   // lh_accum
  int score, ties, order, weight;   // lh_score, lh_ties, lh_order, lh_weight
  int incl;                         // lh_inclusion
};

// Slot-table entry e of a level >= 1 entry (written by the selection):
//   e < 0         not a candidate (pruned): neither in the sub-sequence nor expanded;
//   e = 2s        in the sub-sequence at slot s, not expanded;
//   e = 2s + 1    expanded; nested reading: in the sub-sequence at slot s;
//                 partition reading: not in it, s = first slot of its descendants' run.
// Every entry a walk from the coarsest level visits is a candidate (e >= 0).
__host__ __device__ __forceinline__ bool slot_in(int e, const Geom& g) { return e >= 0 && !(g.incl && (e & 1)); }
// First slot of the p tokens of an expanded level-1 entry: right before its own
// slot (post-order), right after it (pre-order), or the run start (partition).
__host__ __device__ __forceinline__ int slot_tokens(int e, const Geom& g) {
  const int s = e >> 1;
  return g.incl ? s : (g.order ? s + 1 : s - g.p);
}

// Element I/O: 8 consecutive components of a dtype row.
template <typename T> struct Vec8;

template <> struct Vec8<__nv_bfloat16> {
  struct Raw { uint4 a; };
  static __device__ __forceinline__ void load_raw(const __nv_bfloat16* p, Raw& r) {
    r.a = __ldg(reinterpret_cast<const uint4*>(p));
  }
  static __device__ __forceinline__ void raw_f64(const Raw& r, double (&x)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.a);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = (double)f.x;
      x[2 * i + 1] = (double)f.y;
    }
  }
  static __device__ __forceinline__ void raw_f32(const Raw& r, float (&x)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.a);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void load_f64(const __nv_bfloat16* p, double (&x)[8]) {
    uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = (double)f.x;
      x[2 * i + 1] = (double)f.y;
    }
  }
  static __device__ __forceinline__ void load_f32(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store_f64(__nv_bfloat16* p, const double (&x)[8]) {
    uint4 r;
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(&r);
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = __double2bfloat16(x[i]);   // one rounding, nearest-even
    *reinterpret_cast<uint4*>(p) = r;
  }
  static __device__ __forceinline__ void store_f32(__nv_bfloat16* p, const float (&x)[8]) {
    uint4 r;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = r;
  }
};

template <> struct Vec8<float> {
  struct Raw { float4 a, b; };
  static __device__ __forceinline__ void load_raw(const float* p, Raw& r) {
    r.a = __ldg(reinterpret_cast<const float4*>(p));
    r.b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  static __device__ __forceinline__ void raw_f64(const Raw& r, double (&x)[8]) {
    x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
    x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
  }
  static __device__ __forceinline__ void raw_f32(const Raw& r, float (&x)[8]) {
    x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
    x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
  }
  static __device__ __forceinline__ void load_f64(const float* p, double (&x)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ __forceinline__ void load_f32(const float* p, float (&x)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ __forceinline__ void store_f64(float* p, const double (&x)[8]) {
    float4 a = make_float4(__double2float_rn(x[0]), __double2float_rn(x[1]),
                           __double2float_rn(x[2]), __double2float_rn(x[3]));
    float4 b = make_float4(__double2float_rn(x[4]), __double2float_rn(x[5]),
                           __double2float_rn(x[6]), __double2float_rn(x[7]));
    reinterpret_cast<float4*>(p)[0] = a;
    reinterpret_cast<float4*>(p)[1] = b;
  }
  static __device__ __forceinline__ void store_f32(float* p, const float (&x)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
};

// fp16 rows: the backward's tensor-core operands (11-bit significand; every
// bf16 value with magnitude in [2^-14, 65504] converts exactly).
template <> struct Vec8<__half> {
  static __device__ __forceinline__ void load_f32(const __half* p, float (&x)[8]) {
    uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
    const __half2* h = reinterpret_cast<const __half2*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __half22float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store_f32(__half* p, const float (&x)[8]) {
    uint4 r;
    __half2* h = reinterpret_cast<__half2*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = r;
  }
};

// Attention operand type of the sub-sequence (qs, ks, vs, dos): fp16 for bf16
// I/O, fp32 for fp32 I/O.
template <typename T> struct BwdOperand { using type = float; };
template <> struct BwdOperand<__nv_bfloat16> { using type = __half; };

// Largest finite fp16 value; block sums beyond it are reported, not stored as inf.
constexpr float kHalfMax = 65504.f;

// Power-of-two scaling of the fp16 attention operands (bf16 I/O). The scale
// buffer holds, per (b, h), the largest magnitude (fp32 bit pattern; the
// pattern of a non-negative float orders like the value) of the sub-sequence
// queries, keys, values and of the block sums of dO: [4][B][H] uint32. An
// operand x enters fp16 as x * 2^-e, e = scale_exp(largest magnitude): 0 while
// that magnitude is in [4, 256), otherwise the exponent that puts it in [4, 8).
// A power of two moves no significant bit, so every bf16 value within 2^19 of
// its head's largest stays exact in fp16 (the wider range of bf16, beyond
// fp16's 65504 and below its 2^-14, included), and the products and sums formed
// from the scaled operands are those of the unscaled ones times powers of two
// that the kernels take out again. With every operand below 256 in magnitude a
// dS of 128-term dot products stays inside fp16 for any data of that range.
enum { kScaleQ = 0, kScaleK = 1, kScaleV = 2, kScaleDO = 3, kScaleRows = 4 };
constexpr int kScaleMaxExp = 60;      // |e| beyond this is clamped (magnitudes outside 2^-60 .. 2^60)

__host__ __device__ __forceinline__ int scale_exp(uint32_t amax_bits) {
  const int E = (int)((amax_bits >> 23) & 0xFFu);
  if (E == 0 || E == 255) return 0;   // zero / fp32-subnormal, or inf / NaN (reported where it is used)
  const int ex = E - 127;             // floor(log2(largest magnitude))
  if (ex >= 2 && ex < 8) return 0;
  const int e = ex - 2;
  return e < -kScaleMaxExp ? -kScaleMaxExp : (e > kScaleMaxExp ? kScaleMaxExp : e);
}
// 2^e as fp32 for |e| <= 126 (exact).
__host__ __device__ __forceinline__ float pow2f(int e) {
  const uint32_t b = (uint32_t)(127 + e) << 23;
  float f;
  memcpy(&f, &b, sizeof(f));
  return f;
}
// Lane-wise max / min of two pairs of unsigned 16-bit values, one instruction
// each (PTX max.u16x2 / min.u16x2, sm_90 and later).
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// |x| of eight bf16 (a 16-byte vector) as the fp32 bit pattern of the largest.
__device__ __forceinline__ uint32_t absmax8_bf16(const uint4& r) {
  uint32_t m = max_u16x2(max_u16x2(r.x & 0x7FFF7FFFu, r.y & 0x7FFF7FFFu), max_u16x2(r.z & 0x7FFF7FFFu, r.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16) << 16;
}

__device__ __forceinline__ void report_error(int* err, int code, int detail) {
  if (err && atomicCAS(err, 0, code) == 0) atomicExch(err + 1, detail);
}

// Debug build (-DLH_DEBUG_BOUNDS, liblh_debug.so): the indices the memory
// kernels read from the gather map and the slot table are checked against the
// buffers they address before use; a bad one is reported as LH_ERR_DEVICE with
// the site's detail (301 gather map entry, 302 scatter / spread slot, 303
// block-sum slot) and its access is skipped. The release build compiles the
// checks away.
#ifdef LH_DEBUG_BOUNDS
__device__ __forceinline__ bool lh_bounds_ok(bool ok, int* err, int detail) {
  if (!ok) report_error(err, LH_ERR_DEVICE, detail);
  return ok;
}
#define LH_BOUNDS(cond, err, detail) ::lh::lh_bounds_ok((cond), (err), (detail))
#else
#define LH_BOUNDS(cond, err, detail) true
#endif

__device__ __forceinline__ void load8_f32(const float* p, float (&x)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Map entry packing: (level << 28) | index.
__device__ __forceinline__ int map_level(int e) { return (int)((unsigned)e >> 28); }
__device__ __forceinline__ int map_index(int e) { return e & 0x0FFFFFFF; }

}  // namespace lh

// Host-side launchers (defined next to each kernel, called by lh_api.cu).
namespace lh {
cudaError_t launch_pool(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                        void* pq, void* pk, void* pv, double* sq, uint32_t* scale, int* err, cudaStream_t s);
cudaError_t launch_scale_zero(uint32_t* scale, int r0, int nr, int bh, cudaStream_t s);
cudaError_t launch_pool_range(const Geom& g, lh_dtype dt, int cb0, int ncb, const void* q, const void* k,
                              const void* v, void* pq, void* pk, void* pv, double* sq, uint32_t* scale, int* err,
                              cudaStream_t s);
cudaError_t launch_scatter_range(const Geom& g, lh_dtype dt, int cb0, int ncb, const float* os,
                                 const int32_t* slot, void* o, cudaStream_t s);
cudaError_t launch_select(const Geom& g, const double* sq, int32_t* sel, int32_t* map,
                          int32_t* slot, int32_t* ws, cudaStream_t s);
cudaError_t launch_gather(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                          const void* pq, const void* pk, const void* pv, const int32_t* map,
                          const uint32_t* scale, void* qs, void* ks, void* vs, int* err, cudaStream_t s);
cudaError_t launch_scatter(const Geom& g, lh_dtype dt, const float* os, const int32_t* slot,
                           void* o, cudaStream_t s);
cudaError_t launch_scatter_bwd(const Geom& g, lh_dtype dt, const void* dout, const float* os,
                               const int32_t* slot, void* dos, float* delta, uint32_t* scale, int* err,
                               cudaStream_t s);
cudaError_t launch_spread(const Geom& g, lh_dtype dt, const float* dqs, const float* dks,
                          const float* dvs, const int32_t* slot, void* dq, void* dk, void* dv,
                          cudaStream_t s);
cudaError_t launch_attn_fwd(const Geom& g, lh_dtype dt, const void* qs, const void* ks,
                            const void* vs, float* os, float* lse, const uint32_t* scale, int* err,
                            cudaStream_t s);
cudaError_t launch_attn_bwd(const Geom& g, lh_dtype dt, const void* qs, const void* ks,
                            const void* vs, const void* dos, const float* lse, const float* delta,
                            const uint32_t* scale, float* dqs, float* dks, float* dvs, int* err, cudaStream_t s);
void count_launch(int n = 1);
}  // namespace lh
