// Dense gather of the selected entries into the sub-sequence.
//
// "Long Context Pre-Training with Lighthouse Attention", Fig. 1 (the dense
// gather feeds one contiguous causal sequence to the attention); "Lighthouse
// Attention Technique" (the selection is sorted by position, then gathered).
// Row j of qs/ks/vs ([B][H][S][D]) is entry map[j]: a token row of q/k/v
// ([B][N][H][D]) for level 0, a pyramid row ([B][H][E][D]) above, stored in the
// attention operand type: an exact copy for fp32 I/O; for bf16 I/O the fp16
// value of x * 2^-e with the head's power-of-two exponent e (scale_exp of the
// head's largest magnitude, from lh_pool), exact for every bf16 value within
// 2^19 of that largest one; a non-finite value is reported as LH_ERR_DEVICE,
// detail 102. fp16 keeps 11 significant bits for the attention's P and dS
// operands where bf16 keeps 8.
// Reading 16 bytes per thread (8 bf16 -> 8 fp16, or 4 fp32); consecutive
// threads cover a row, so loads of a row and all stores are coalesced.
#include <algorithm>

#include "lh_common.cuh"

namespace lh {
namespace {

// One CTA covers kU * RPB rows of one (b, h) at a time and one of q / k / v
// (grid.y strides over b * H + h, grid.z = tensor). VPR = 2^LG threads per
// row, so each thread moves kU independent 16-byte vectors (all loads in
// flight before the stores) and no per-element index needs a division.
constexpr int kU = 4;

template <bool TO_F16, int LG>
__global__ void __launch_bounds__(256) k_gather(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                const uint4* __restrict__ v, const uint4* __restrict__ pq,
                                                const uint4* __restrict__ pk, const uint4* __restrict__ pv,
                                                const int32_t* __restrict__ map,
                                                const uint32_t* __restrict__ scale, uint4* __restrict__ qs,
                                                uint4* __restrict__ ks, uint4* __restrict__ vs, Geom g,
                                                int* err) {
  constexpr int VPR = 1 << LG, RPB = 256 >> LG;
  const int tensor = blockIdx.z;
  const uint4* x = tensor == 0 ? q : (tensor == 1 ? k : v);
  const uint4* px = tensor == 0 ? pq : (tensor == 1 ? pk : pv);
  uint4* xs = tensor == 0 ? qs : (tensor == 1 ? ks : vs);
  const int c = threadIdx.x & (VPR - 1);
  const int s0 = blockIdx.x * (RPB * kU) + (threadIdx.x >> LG);
  bool big = false;
  for (int bh = blockIdx.y; bh < g.B * g.H; bh += gridDim.y) {
    const int b = bh / g.H, h = bh - b * g.H;
    const int32_t* mrow = map + (size_t)bh * g.S;
    const uint4* xrow = x + ((size_t)b * g.N * g.H + h) * VPR + c;     // + token * H * VPR
    const uint4* prow = px + (size_t)bh * g.E * VPR + c;               // + entry * VPR
    uint4* out = xs + (size_t)bh * g.S * VPR + c;
    const float mul = TO_F16 ? pow2f(-scale_exp(scale[(size_t)tensor * g.B * g.H + bh])) : 1.f;
    int e[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int s = s0 + u * RPB;
      e[u] = s < g.S ? __ldg(mrow + s) : -1;
      if (e[u] >= 0) {
        const int l = map_level(e[u]), idx = map_index(e[u]);
        if (!LH_BOUNDS(l < g.L && idx < (l == 0 ? g.N : g.n[l]), err, 301)) e[u] = -1;
      }
    }
    uint4 val[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (e[u] < 0) continue;
      const int l = map_level(e[u]), idx = map_index(e[u]);
      const uint4* src = l == 0 ? xrow + (size_t)idx * g.H * VPR : prow + (size_t)(g.off[l] + idx) * VPR;
      val[u] = __ldg(src);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (e[u] < 0) continue;
      uint4* o = out + (size_t)(s0 + u * RPB) * VPR;
      if (TO_F16) {
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&val[u]);
        uint4 hv;
        __half2* h2 = reinterpret_cast<__half2*>(&hv);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          float2 f = __bfloat1622float2(b2[w]);
          f.x *= mul;                 // a power of two: exact
          f.y *= mul;
          big |= !(fabsf(f.x) <= kHalfMax) || !(fabsf(f.y) <= kHalfMax);
          h2[w] = __float22half2_rn(f);
        }
        *o = hv;
      } else {
        *o = val[u];
      }
    }
  }
  if (TO_F16 && big) report_error(err, LH_ERR_DEVICE, 102);
}

}  // namespace

cudaError_t launch_gather(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                          const void* pq, const void* pk, const void* pv, const int32_t* map,
                          const uint32_t* scale, void* qs, void* ks, void* vs, int* err, cudaStream_t s) {
  if (g.S == 0 || g.B * g.H == 0) return cudaSuccess;
  const int esz = dt == LH_BF16 ? 2 : 4;
  const int vpr = g.D * esz / 16;                  // 8, 16 or 32 (D = 64 or 128)
  const int lg = vpr == 8 ? 3 : (vpr == 16 ? 4 : 5);
  const int rows_per_cta = (256 / vpr) * kU;
  dim3 grid((unsigned)((g.S + rows_per_cta - 1) / rows_per_cta), (unsigned)std::min(g.B * g.H, 65535), 3);
  const uint4 *q4 = (const uint4*)q, *k4 = (const uint4*)k, *v4 = (const uint4*)v;
  const uint4 *pq4 = (const uint4*)pq, *pk4 = (const uint4*)pk, *pv4 = (const uint4*)pv;
  uint4 *qs4 = (uint4*)qs, *ks4 = (uint4*)ks, *vs4 = (uint4*)vs;
#define LH_GATHER(F16, LG) \
  k_gather<F16, LG><<<grid, 256, 0, s>>>(q4, k4, v4, pq4, pk4, pv4, map, scale, qs4, ks4, vs4, g, err)
  if (dt == LH_BF16) {
    if (lg == 3) LH_GATHER(true, 3); else LH_GATHER(true, 4);
  } else {
    if (lg == 4) LH_GATHER(false, 4); else LH_GATHER(false, 5);
  }
#undef LH_GATHER
  count_launch();
  return cudaGetLastError();
}

}  // namespace lh
