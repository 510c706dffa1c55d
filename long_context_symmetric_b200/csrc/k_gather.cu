// Dense gather of the selected entries into the sub-sequence.
//
// "Long Context Pre-Training with Lighthouse Attention", Fig. 1 (the dense
// gather feeds one contiguous causal sequence to the attention); "Lighthouse
// Attention Technique" (the selection is sorted by position, then gathered).
// Row j of qs/ks/vs ([B][H][S][D]) is entry map[j]: a token row of q/k/v
// ([B][N][H][D]) for level 0, a pyramid row ([B][H][E][D]) above, stored in the
// attention operand type: an exact copy for fp32 I/O; for bf16 I/O the fp16
// value (nearest-even; exact for every bf16 magnitude in [2^-14, 65504], and a
// magnitude above 65504 is reported as LH_ERR_DEVICE, detail 102). fp16 keeps
// 11 significant bits for the attention's P and dS operands where bf16 keeps 8.
// Reading 16 bytes per thread (8 bf16 -> 8 fp16, or 4 fp32); consecutive
// threads cover a row, so stores are fully coalesced.
#include "lh_common.cuh"

namespace lh {
namespace {

template <bool TO_F16>
__global__ void __launch_bounds__(256) k_gather(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                const uint4* __restrict__ v, const uint4* __restrict__ pq,
                                                const uint4* __restrict__ pk, const uint4* __restrict__ pv,
                                                const int32_t* __restrict__ map, uint4* __restrict__ qs,
                                                uint4* __restrict__ ks, uint4* __restrict__ vs, Geom g,
                                                int vpr /* 16-byte vectors per row */, int* err) {
  const long long rows = (long long)g.B * g.H * g.S;
  const long long total = rows * vpr;
  const int tensor = blockIdx.y;
  const uint4* x = tensor == 0 ? q : (tensor == 1 ? k : v);
  const uint4* px = tensor == 0 ? pq : (tensor == 1 ? pk : pv);
  uint4* xs = tensor == 0 ? qs : (tensor == 1 ? ks : vs);
  bool big = false;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / vpr;
    const int c = (int)(i - row * vpr);
    const long long bh = row / g.S;
    const int e = __ldg(map + row);
    const int l = map_level(e), idx = map_index(e);
    const uint4* src;
    if (l == 0) {
      const long long b = bh / g.H, h = bh - b * g.H;
      src = x + ((b * g.N + idx) * g.H + h) * vpr;
    } else {
      src = px + (bh * g.E + g.off[l] + idx) * vpr;
    }
    const uint4 val = __ldg(src + c);
    if (TO_F16) {
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&val);
      uint4 hv;
      __half2* h2 = reinterpret_cast<__half2*>(&hv);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(b2[u]);
        big |= !(fabsf(f.x) <= kHalfMax) || !(fabsf(f.y) <= kHalfMax);
        h2[u] = __float22half2_rn(f);
      }
      xs[i] = hv;
    } else {
      xs[i] = val;
    }
  }
  if (TO_F16 && big) report_error(err, LH_ERR_DEVICE, 102);
}

}  // namespace

cudaError_t launch_gather(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                          const void* pq, const void* pk, const void* pv, const int32_t* map,
                          void* qs, void* ks, void* vs, int* err, cudaStream_t s) {
  const int esz = dt == LH_BF16 ? 2 : 4;
  const int vpr = g.D * esz / 16;
  const long long total = (long long)g.B * g.H * g.S * vpr;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  dim3 grid((unsigned)blocks, 3);
  if (dt == LH_BF16)
    k_gather<true><<<grid, 256, 0, s>>>((const uint4*)q, (const uint4*)k, (const uint4*)v,
                                        (const uint4*)pq, (const uint4*)pk, (const uint4*)pv, map,
                                        (uint4*)qs, (uint4*)ks, (uint4*)vs, g, vpr, err);
  else
    k_gather<false><<<grid, 256, 0, s>>>((const uint4*)q, (const uint4*)k, (const uint4*)v,
                                         (const uint4*)pq, (const uint4*)pk, (const uint4*)pv, map,
                                         (uint4*)qs, (uint4*)ks, (uint4*)vs, g, vpr, err);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lh
