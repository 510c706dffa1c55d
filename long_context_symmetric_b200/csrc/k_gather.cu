// Dense gather of the selected entries into the sub-sequence.
//
// "Long Context Pre-Training with Lighthouse Attention", Fig. 1 (the dense
// gather feeds one contiguous causal sequence to the attention); "Lighthouse
// Attention Technique" (the selection is sorted by position, then gathered).
// Row j of qs/ks/vs ([B][H][S][D]) is a bit-exact copy of entry map[j]: a token
// row of q/k/v ([B][N][H][D]) for level 0, a pyramid row ([B][H][E][D]) above.
// One thread moves 16 bytes; consecutive threads cover a row, so stores are
// fully coalesced and each source row is read as whole 32-byte sectors.
// For bf16 I/O the same pass can also write fp16 copies (qh, kh, vh), the
// operands of the tensor-core backward; the conversion is exact for every bf16
// value of magnitude in [2^-14, 65504].
#include "lh_common.cuh"

namespace lh {
namespace {

__global__ void __launch_bounds__(256) k_gather(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                const uint4* __restrict__ v, const uint4* __restrict__ pq,
                                                const uint4* __restrict__ pk, const uint4* __restrict__ pv,
                                                const int32_t* __restrict__ map, uint4* __restrict__ qs,
                                                uint4* __restrict__ ks, uint4* __restrict__ vs,
                                                uint4* __restrict__ qh, uint4* __restrict__ kh,
                                                uint4* __restrict__ vh, Geom g,
                                                int vpr /* 16-byte vectors per row */) {
  const long long rows = (long long)g.B * g.H * g.S;
  const long long total = rows * vpr;
  const int tensor = blockIdx.y;
  const uint4* x = tensor == 0 ? q : (tensor == 1 ? k : v);
  const uint4* px = tensor == 0 ? pq : (tensor == 1 ? pk : pv);
  uint4* xs = tensor == 0 ? qs : (tensor == 1 ? ks : vs);
  uint4* xh = tensor == 0 ? qh : (tensor == 1 ? kh : vh);
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
    xs[i] = val;
    if (xh) {
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&val);
      uint4 hv;
      __half2* h2 = reinterpret_cast<__half2*>(&hv);
#pragma unroll
      for (int u = 0; u < 4; ++u) h2[u] = __float22half2_rn(__bfloat1622float2(b2[u]));
      xh[i] = hv;
    }
  }
}

}  // namespace

cudaError_t launch_gather(const Geom& g, lh_dtype dt, const void* q, const void* k, const void* v,
                          const void* pq, const void* pk, const void* pv, const int32_t* map,
                          void* qs, void* ks, void* vs, void* qh, void* kh, void* vh, cudaStream_t s) {
  const int esz = dt == LH_BF16 ? 2 : 4;
  const int vpr = g.D * esz / 16;
  const long long total = (long long)g.B * g.H * g.S * vpr;
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  dim3 grid((unsigned)blocks, 3);
  k_gather<<<grid, 256, 0, s>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, (const uint4*)pq,
                                (const uint4*)pk, (const uint4*)pv, map, (uint4*)qs, (uint4*)ks,
                                (uint4*)vs, dt == LH_BF16 ? (uint4*)qh : nullptr,
                                dt == LH_BF16 ? (uint4*)kh : nullptr, dt == LH_BF16 ? (uint4*)vh : nullptr,
                                g, vpr);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lh
