// Causal attention on the sub-sequence with fp32 SIMT arithmetic.
//
// "Long Context Pre-Training with Lighthouse Attention", Eq. (1) and §3.1
// stage (iii): softmax(Q K^T / sqrt(d) + M) V with the lower-triangular mask,
// on the gathered sub-sequence. This is the fp32 path (tensor cores cannot
// hold fp32 operands at fp32 precision); with LH_ATTN_SIMT=1 it also serves
// bf16 I/O (whose sub-sequence holds fp16 values, widened to fp32 exactly).
//
// Forward: one CTA per (b, h, 64-row query tile); K/V tiles of 64 rows staged
// in shared memory as fp32 (row stride D+1 so the lane-per-key dot products are
// bank-conflict free); each warp owns 8 query rows; online softmax in the
// exp2 domain. Backward: two deterministic kernels, one per 64-row key tile
// (dK, dV) and one per 64-row query tile (dQ), each recomputing P from lse.
#include "lh_common.cuh"

namespace lh {
namespace {

constexpr int BM = 64;     // rows per CTA tile
constexpr int BN = 64;     // rows per streamed tile
constexpr int NW = 8;      // warps per CTA
constexpr int RPW = BM / NW;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T>
__device__ __forceinline__ float ld1(const T* p);
template <>
__device__ __forceinline__ float ld1<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ld1<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <>
__device__ __forceinline__ float ld1<__half>(const __half* p) {
  return __half2float(*p);
}

// rows [r0, r0+nrows) of a [S][D] matrix into smem (stride ld), zero past S
template <typename T, int D>
__device__ __forceinline__ void stage(float* dst, int ld, const T* src, int r0, int nrows, int S,
                                      float mul) {
  for (int i = threadIdx.x; i < nrows * D; i += blockDim.x) {
    const int r = i / D, d = i % D;
    const int gr = r0 + r;
    dst[r * ld + d] = gr < S ? ld1<T>(src + (size_t)gr * D + d) * mul : 0.f;
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T, int D>
__global__ void __launch_bounds__(NW * 32) k_fwd(const T* __restrict__ qs, const T* __restrict__ ks,
                                                 const T* __restrict__ vs, float* __restrict__ os,
                                                 float* __restrict__ lse, int S, float scale) {
  extern __shared__ float sm[];
  float* Qs = sm;                       // [BM][D]
  float* Ks = Qs + BM * D;              // [BN][D+1]
  float* Vs = Ks + BN * (D + 1);        // [BN][D]
  constexpr int DC = D / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * BM;
  const size_t base = (size_t)blockIdx.y * S * D;
  stage<T, D>(Qs, D, qs + base, r0, BM, S, scale * kLog2e);   // scores in the log2 domain
  float o[RPW][DC], m[RPW], l[RPW];
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int c = 0; c < DC; ++c) o[i][c] = 0.f;
  }
  const int nend = min(r0 + BM, S);
  for (int n0 = 0; n0 < nend; n0 += BN) {
    __syncthreads();
    stage<T, D>(Ks, D + 1, ks + base, n0, BN, S, 1.f);
    stage<T, D>(Vs, D, vs + base, n0, BN, S, 1.f);
    __syncthreads();
#pragma unroll 1
    for (int i = 0; i < RPW; ++i) {
      const int rr = warp * RPW + i;
      const int row = r0 + rr;
      if (row >= S) continue;            // warp-uniform
      float s0 = 0.f, s1 = 0.f;
      const float* qrow = Qs + rr * D;
      const float* k0 = Ks + lane * (D + 1);
      const float* k1 = Ks + (lane + 32) * (D + 1);
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        const float qd = qrow[d];
        s0 = fmaf(qd, k0[d], s0);
        s1 = fmaf(qd, k1[d], s1);
      }
      if (n0 + lane > row) s0 = -INFINITY;
      if (n0 + lane + 32 > row) s1 = -INFINITY;
      const float mnew = fmaxf(m[i], warp_max(fmaxf(s0, s1)));
      const float alpha = exp2f(m[i] - mnew);
      const float p0 = exp2f(s0 - mnew), p1 = exp2f(s1 - mnew);
      l[i] = l[i] * alpha + warp_sum(p0 + p1);
      m[i] = mnew;
#pragma unroll
      for (int c = 0; c < DC; ++c) o[i][c] *= alpha;
#pragma unroll 4
      for (int j = 0; j < 32; ++j) {
        const float pj0 = __shfl_sync(0xffffffffu, p0, j);
        const float pj1 = __shfl_sync(0xffffffffu, p1, j);
#pragma unroll
        for (int c = 0; c < DC; ++c) {
          o[i][c] = fmaf(pj0, Vs[j * D + lane + 32 * c], o[i][c]);
          o[i][c] = fmaf(pj1, Vs[(j + 32) * D + lane + 32 * c], o[i][c]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int row = r0 + warp * RPW + i;
    if (row >= S) continue;
    const float inv = 1.f / l[i];
#pragma unroll
    for (int c = 0; c < DC; ++c) os[base + (size_t)row * D + lane + 32 * c] = o[i][c] * inv;
    if (lane == 0) lse[(size_t)blockIdx.y * S + row] = (m[i] + log2f(l[i])) * kLn2;
  }
}

// dQ = scale * sum_m P (dP - delta) K, per 64-row query tile.
template <typename T, int D>
__global__ void __launch_bounds__(NW * 32) k_bwd_dq(const T* __restrict__ qs, const T* __restrict__ ks,
                                                    const T* __restrict__ vs, const T* __restrict__ dos,
                                                    const float* __restrict__ lse,
                                                    const float* __restrict__ delta,
                                                    float* __restrict__ dqs, int S, float scale) {
  extern __shared__ float sm[];
  float* Qs = sm;                       // [BM][D]   (scaled into the log2 domain)
  float* Gs = Qs + BM * D;              // [BM][D]   dO
  float* Ks = Gs + BM * D;              // [BN][D+1]
  float* Vs = Ks + BN * (D + 1);        // [BN][D+1]
  constexpr int DC = D / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * BM;
  const size_t base = (size_t)blockIdx.y * S * D;
  const size_t rbase = (size_t)blockIdx.y * S;
  stage<T, D>(Qs, D, qs + base, r0, BM, S, scale * kLog2e);
  stage<T, D>(Gs, D, dos + base, r0, BM, S, 1.f);
  float acc[RPW][DC], lse2[RPW], dl[RPW];
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int row = r0 + warp * RPW + i;
    lse2[i] = row < S ? lse[rbase + row] * kLog2e : 0.f;
    dl[i] = row < S ? delta[rbase + row] : 0.f;
#pragma unroll
    for (int c = 0; c < DC; ++c) acc[i][c] = 0.f;
  }
  const int nend = min(r0 + BM, S);
  for (int n0 = 0; n0 < nend; n0 += BN) {
    __syncthreads();
    stage<T, D>(Ks, D + 1, ks + base, n0, BN, S, 1.f);
    stage<T, D>(Vs, D + 1, vs + base, n0, BN, S, 1.f);
    __syncthreads();
#pragma unroll 1
    for (int i = 0; i < RPW; ++i) {
      const int rr = warp * RPW + i;
      const int row = r0 + rr;
      if (row >= S) continue;
      float s0 = 0.f, s1 = 0.f, g0 = 0.f, g1 = 0.f;
      const float* qrow = Qs + rr * D;
      const float* grow = Gs + rr * D;
      const float* k0 = Ks + lane * (D + 1);
      const float* k1 = Ks + (lane + 32) * (D + 1);
      const float* v0 = Vs + lane * (D + 1);
      const float* v1 = Vs + (lane + 32) * (D + 1);
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        const float qd = qrow[d], gd = grow[d];
        s0 = fmaf(qd, k0[d], s0);
        s1 = fmaf(qd, k1[d], s1);
        g0 = fmaf(gd, v0[d], g0);
        g1 = fmaf(gd, v1[d], g1);
      }
      const float p0 = n0 + lane <= row ? exp2f(s0 - lse2[i]) : 0.f;
      const float p1 = n0 + lane + 32 <= row ? exp2f(s1 - lse2[i]) : 0.f;
      const float ds0 = p0 * (g0 - dl[i]);
      const float ds1 = p1 * (g1 - dl[i]);
#pragma unroll 4
      for (int j = 0; j < 32; ++j) {
        const float a0 = __shfl_sync(0xffffffffu, ds0, j);
        const float a1 = __shfl_sync(0xffffffffu, ds1, j);
#pragma unroll
        for (int c = 0; c < DC; ++c) {
          acc[i][c] = fmaf(a0, Ks[j * (D + 1) + lane + 32 * c], acc[i][c]);
          acc[i][c] = fmaf(a1, Ks[(j + 32) * (D + 1) + lane + 32 * c], acc[i][c]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int row = r0 + warp * RPW + i;
    if (row >= S) continue;
#pragma unroll
    for (int c = 0; c < DC; ++c) dqs[base + (size_t)row * D + lane + 32 * c] = acc[i][c] * scale;
  }
}

// dV = sum_j P_j dO_j and dK = scale * sum_j dS_j Q_j, per 64-row key tile.
template <typename T, int D>
__global__ void __launch_bounds__(NW * 32) k_bwd_dkdv(const T* __restrict__ qs, const T* __restrict__ ks,
                                                      const T* __restrict__ vs, const T* __restrict__ dos,
                                                      const float* __restrict__ lse,
                                                      const float* __restrict__ delta,
                                                      float* __restrict__ dks, float* __restrict__ dvs,
                                                      int S, float scale) {
  extern __shared__ float sm[];
  float* Ks = sm;                       // [BN][D]  (this CTA's keys, scaled into log2 domain)
  float* Vs = Ks + BN * D;              // [BN][D]
  float* Qs = Vs + BN * D;              // [BM][D+1]
  float* Gs = Qs + BM * (D + 1);        // [BM][D+1]
  float* Ls = Gs + BM * (D + 1);        // [BM] lse (log2 domain)
  float* Ds = Ls + BM;                  // [BM] delta
  constexpr int DC = D / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n0 = blockIdx.x * BN;
  const size_t base = (size_t)blockIdx.y * S * D;
  const size_t rbase = (size_t)blockIdx.y * S;
  stage<T, D>(Ks, D, ks + base, n0, BN, S, scale * kLog2e);
  stage<T, D>(Vs, D, vs + base, n0, BN, S, 1.f);
  float dk[RPW][DC], dv[RPW][DC];
#pragma unroll
  for (int i = 0; i < RPW; ++i)
#pragma unroll
    for (int c = 0; c < DC; ++c) dk[i][c] = dv[i][c] = 0.f;
  for (int r0 = n0; r0 < S; r0 += BM) {
    __syncthreads();
    stage<T, D>(Qs, D + 1, qs + base, r0, BM, S, 1.f);
    stage<T, D>(Gs, D + 1, dos + base, r0, BM, S, 1.f);
    for (int i = threadIdx.x; i < BM; i += blockDim.x) {
      const int row = r0 + i;
      Ls[i] = row < S ? lse[rbase + row] * kLog2e : 0.f;
      Ds[i] = row < S ? delta[rbase + row] : 0.f;
    }
    __syncthreads();
#pragma unroll 1
    for (int i = 0; i < RPW; ++i) {
      const int kr = warp * RPW + i;
      const int key = n0 + kr;
      if (key >= S) continue;
      float s0 = 0.f, s1 = 0.f, g0 = 0.f, g1 = 0.f;
      const float* krow = Ks + kr * D;
      const float* vrow = Vs + kr * D;
      const float* q0 = Qs + lane * (D + 1);
      const float* q1 = Qs + (lane + 32) * (D + 1);
      const float* d0 = Gs + lane * (D + 1);
      const float* d1 = Gs + (lane + 32) * (D + 1);
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        const float kd = krow[d], vd = vrow[d];
        s0 = fmaf(kd, q0[d], s0);
        s1 = fmaf(kd, q1[d], s1);
        g0 = fmaf(vd, d0[d], g0);
        g1 = fmaf(vd, d1[d], g1);
      }
      const int j0 = r0 + lane, j1 = r0 + lane + 32;
      const float p0 = (j0 < S && j0 >= key) ? exp2f(s0 - Ls[lane]) : 0.f;
      const float p1 = (j1 < S && j1 >= key) ? exp2f(s1 - Ls[lane + 32]) : 0.f;
      const float ds0 = p0 * (g0 - Ds[lane]);
      const float ds1 = p1 * (g1 - Ds[lane + 32]);
#pragma unroll 4
      for (int j = 0; j < 32; ++j) {
        const float a0 = __shfl_sync(0xffffffffu, p0, j);
        const float a1 = __shfl_sync(0xffffffffu, p1, j);
        const float b0 = __shfl_sync(0xffffffffu, ds0, j);
        const float b1 = __shfl_sync(0xffffffffu, ds1, j);
#pragma unroll
        for (int c = 0; c < DC; ++c) {
          const int dd = lane + 32 * c;
          dv[i][c] = fmaf(a0, Gs[j * (D + 1) + dd], dv[i][c]);
          dv[i][c] = fmaf(a1, Gs[(j + 32) * (D + 1) + dd], dv[i][c]);
          dk[i][c] = fmaf(b0, Qs[j * (D + 1) + dd], dk[i][c]);
          dk[i][c] = fmaf(b1, Qs[(j + 32) * (D + 1) + dd], dk[i][c]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int key = n0 + warp * RPW + i;
    if (key >= S) continue;
#pragma unroll
    for (int c = 0; c < DC; ++c) {
      dks[base + (size_t)key * D + lane + 32 * c] = dk[i][c] * scale;
      dvs[base + (size_t)key * D + lane + 32 * c] = dv[i][c];
    }
  }
}

template <typename T, int D>
cudaError_t fwd_t(const Geom& g, const void* qs, const void* ks, const void* vs, float* os,
                  float* lse, cudaStream_t s) {
  const size_t smem = (size_t)(BM * D + BN * (D + 1) + BN * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_fwd<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((g.S + BM - 1) / BM, g.B * g.H);
  k_fwd<T, D><<<grid, NW * 32, smem, s>>>((const T*)qs, (const T*)ks, (const T*)vs, os, lse, g.S,
                                          (float)(1.0 / sqrt((double)g.D)));
  count_launch();
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t bwd_t(const Geom& g, const void* qs, const void* ks, const void* vs, const void* dos,
                  const float* lse, const float* delta, float* dqs, float* dks, float* dvs,
                  cudaStream_t s) {
  const float scale = (float)(1.0 / sqrt((double)g.D));
  const size_t smq = (size_t)(2 * BM * D + 2 * BN * (D + 1)) * sizeof(float);
  const size_t smk = (size_t)(2 * BN * D + 2 * BM * (D + 1) + 2 * BM) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_bwd_dq<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_bwd_dkdv<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smk);
  if (e != cudaSuccess) return e;
  dim3 grid((g.S + BM - 1) / BM, g.B * g.H);
  k_bwd_dq<T, D><<<grid, NW * 32, smq, s>>>((const T*)qs, (const T*)ks, (const T*)vs, (const T*)dos,
                                            lse, delta, dqs, g.S, scale);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_bwd_dkdv<T, D><<<grid, NW * 32, smk, s>>>((const T*)qs, (const T*)ks, (const T*)vs, (const T*)dos,
                                              lse, delta, dks, dvs, g.S, scale);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_simt(const Geom& g, lh_dtype dt, const void* qs, const void* ks,
                                 const void* vs, float* os, float* lse, cudaStream_t s) {
  // bf16 I/O: the sub-sequence holds fp16 values (see lh_gather)
  if (dt == LH_BF16)
    return g.D == 64 ? fwd_t<__half, 64>(g, qs, ks, vs, os, lse, s)
                     : fwd_t<__half, 128>(g, qs, ks, vs, os, lse, s);
  return g.D == 64 ? fwd_t<float, 64>(g, qs, ks, vs, os, lse, s)
                   : fwd_t<float, 128>(g, qs, ks, vs, os, lse, s);
}

cudaError_t launch_attn_bwd_simt(const Geom& g, lh_dtype dt, const void* qs, const void* ks,
                                 const void* vs, const void* dos, const float* lse,
                                 const float* delta, float* dqs, float* dks, float* dvs,
                                 cudaStream_t s) {
  // bf16 I/O: the sub-sequence and dos hold fp16 values
  if (dt == LH_BF16)
    return g.D == 64 ? bwd_t<__half, 64>(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, s)
                     : bwd_t<__half, 128>(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, s);
  return g.D == 64 ? bwd_t<float, 64>(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, s)
                   : bwd_t<float, 128>(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, s);
}

}  // namespace lh
