// Sequence-sharded (context-parallel) path: the per-rank steps between the
// collectives.
//
// The pages scale Lighthouse to 1M-token context over 32 B200s with context
// parallelism ("Nous Research's Lighthouse Attention Trains 1.69x Faster on
// Million-Token Contexts", key points; "Lighthouse Attention Technique":
// beyond 100K context the model is scaled with context parallelism). Rank r
// holds tokens [r n, (r+1) n), n a multiple of p^(L-1), so its pyramid entries
// are its own ("Long Context Pre-Training with Lighthouse Attention", Fig. 2
// steps 1-2: pooling and scores are local to an entry's tokens). The kernels
// here, with the collectives the caller runs between them:
//   lh_pool on the shard                     -> local squared norms
//   [all-gather of every rank's norms]
//   k_cp_assemble_sq                         -> the whole sequence's norms, in
//                                               the single-GPU layout
//   lh_score_topk (unchanged, every rank)    -> the same selection, map and
//                                               slot table on every rank
//   k_cp_segment                             -> this rank's slice of the slot
//                                               table; its segment of the map
//   k_cp_gather                              -> the segment's rows of the
//                                               sub-sequence, zero elsewhere
//   [all-reduce (sum) of the sub-sequence keys and values: the segments are
//    disjoint, so the sum is every rank's rows]
//   attention of the segment's queries over the keys before them, scatter,
//   block sums and spread on the shard, and in the backward an all-reduce of
//   the key and value gradients, each rank contributing its queries' part.
// Entries of a rank end inside its shard, and the sub-sequence is sorted by
// position (Fig. 1), so each rank's entries are one contiguous run of slots.
#include "lh_common.cuh"

namespace lh {
namespace {

struct CpGeom {
  int world, rank, nloc;                 // ranks, this rank, tokens per rank
  int nl[LH_MAX_LEVELS];                 // entries of level l per rank
  int offl[LH_MAX_LEVELS];               // start of level l in a rank's entry axis (l >= 1)
  int El;                                // entries of levels >= 1 per rank
};

// sq [2][B][H][E] from the gathered [world][2][B][H][El]: level l entry i of
// the whole sequence is entry i mod nl of rank i / nl.
__global__ void __launch_bounds__(256) k_cp_assemble_sq(const double* __restrict__ gath, double* __restrict__ sq,
                                                        Geom g, CpGeom c) {
  const long long per = (long long)g.B * g.H * g.E;     // one side (query or key norms)
  const long long total = 2 * per;
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
       x += (long long)gridDim.x * blockDim.x) {
    const long long side_bh = x / g.E;                  // side * B * H + bh
    const int e = (int)(x - side_bh * g.E);
    int l = 1;
    while (l + 1 < g.L && e >= g.off[l + 1]) ++l;
    const int i = e - g.off[l];
    const int r = i / c.nl[l], il = i - r * c.nl[l];
    sq[x] = gath[((long long)r * 2 * g.B * g.H + side_bh) * c.El + c.offl[l] + il];
  }
}

// Position of an entry that orders the sub-sequence: last covered token
// (post-order) or first covered token (pre-order). Every entry lies inside one
// shard, so "ordered before rank r's first token" is the same test either way.
__device__ __forceinline__ long long entry_pos(int e, const Geom& g) {
  const int l = map_level(e), i = map_index(e);
  return g.order ? (long long)i * g.pl[l] : ((long long)i + 1) * g.pl[l] - 1;
}

// seg[bh] = (first slot, count) of this rank's entries, by binary search of
// the position-sorted map; one thread per (b, h).
__global__ void k_cp_segment(const int32_t* __restrict__ map, int32_t* __restrict__ seg, Geom g, CpGeom c) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= g.B * g.H) return;
  const int32_t* m = map + (size_t)bh * g.S;
  auto first_at = [&](long long tok) {                 // first slot whose entry lies at or after tok
    int lo = 0, hi = g.S;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (entry_pos(m[mid], g) < tok) lo = mid + 1; else hi = mid;
    }
    return lo;
  };
  const int s0 = first_at((long long)c.rank * c.nloc);
  const int s1 = c.rank + 1 == c.world ? g.S : first_at((long long)(c.rank + 1) * c.nloc);
  seg[2 * bh] = s0;
  seg[2 * bh + 1] = s1 - s0;
}

// slot_loc[bh][offl[l] + i] = slot[bh][off[l] + rank * nl[l] + i]: the slot
// table of this rank's entries (slot values stay slots of the whole sub-sequence).
__global__ void __launch_bounds__(256) k_cp_slot(const int32_t* __restrict__ slot, int32_t* __restrict__ slot_loc,
                                                 Geom g, CpGeom c) {
  const long long total = (long long)g.B * g.H * c.El;
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < total;
       x += (long long)gridDim.x * blockDim.x) {
    const long long bh = x / c.El;
    const int e = (int)(x - bh * c.El);
    int l = 1;
    while (l + 1 < g.L && e >= c.offl[l + 1]) ++l;
    slot_loc[x] = slot[bh * g.E + g.off[l] + (long long)c.rank * c.nl[l] + (e - c.offl[l])];
  }
}

// Rows [0, S) of qs / ks / vs ([B][H][S][D], attention operand type): rows of
// this rank's segment take the stored entry their map entry names (a token row
// of the shard, or a row of the shard's pyramid), every other row is zero.
// Threads cover 16-byte vectors of a row; VPR vectors per row.
template <bool TO_F16>
__global__ void __launch_bounds__(256) k_cp_gather(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                   const uint4* __restrict__ v, const uint4* __restrict__ pq,
                                                   const uint4* __restrict__ pk, const uint4* __restrict__ pv,
                                                   const int32_t* __restrict__ map, const int32_t* __restrict__ seg,
                                                   const uint32_t* __restrict__ scale, uint4* __restrict__ qs,
                                                   uint4* __restrict__ ks,
                                                   uint4* __restrict__ vs, Geom g, CpGeom c, int vin, int vout,
                                                   int* err) {
  const int tensor = blockIdx.z;
  const uint4* x = tensor == 0 ? q : (tensor == 1 ? k : v);
  const uint4* px = tensor == 0 ? pq : (tensor == 1 ? pk : pv);
  uint4* xs = tensor == 0 ? qs : (tensor == 1 ? ks : vs);
  const int bh = blockIdx.y;
  const int b = bh / g.H, h = bh - b * g.H;
  const int s0 = seg[2 * bh], len = seg[2 * bh + 1];
  const float mul = TO_F16 ? pow2f(-scale_exp(scale[(size_t)tensor * g.B * g.H + bh])) : 1.f;
  bool big = false;
  const long long total = (long long)g.S * vout;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const int row = (int)(t / vout), cv = (int)(t - (long long)row * vout);
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (row >= s0 && row < s0 + len) {
      const int e = map[(size_t)bh * g.S + row];
      const int l = map_level(e);
      const int il = map_index(e) - c.rank * (l == 0 ? c.nloc : c.nl[l]);
      if (TO_F16) {
        // bf16 I/O: 8 elements of 16 bytes in, 8 fp16 out (vin == vout)
        const uint4 val = l == 0 ? __ldg(x + (((size_t)b * c.nloc + il) * g.H + h) * vin + cv)
                                 : __ldg(px + ((size_t)bh * c.El + c.offl[l] + il) * vin + cv);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&val);
        __half2* h2 = reinterpret_cast<__half2*>(&out);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          float2 f = __bfloat1622float2(b2[w]);
          f.x *= mul;                 // the head's power-of-two exponent (exact)
          f.y *= mul;
          big |= !(fabsf(f.x) <= kHalfMax) || !(fabsf(f.y) <= kHalfMax);
          h2[w] = __float22half2_rn(f);
        }
      } else {
        out = l == 0 ? __ldg(x + (((size_t)b * c.nloc + il) * g.H + h) * vin + cv)
                     : __ldg(px + ((size_t)bh * c.El + c.offl[l] + il) * vin + cv);
      }
    }
    xs[((size_t)bh * g.S + row) * vout + cv] = out;
  }
  if (TO_F16 && big) report_error(err, LH_ERR_DEVICE, 102);
}

// Rows of x ([B][H][S][vpr] 16-byte vectors) outside this rank's segment set
// to zero: the rows of other ranks' queries that the backward's key-tile loads
// read past the segment's end must be finite (a zero P times a NaN is NaN).
__global__ void __launch_bounds__(256) k_cp_zero_outside(uint4* __restrict__ x, const int32_t* __restrict__ seg,
                                                         int S, int vpr) {
  const int bh = blockIdx.y;
  const int s0 = seg[2 * bh], len = seg[2 * bh + 1];
  const long long total = (long long)S * vpr;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const int row = (int)(t / vpr);
    if (row < s0 || row >= s0 + len) x[(size_t)bh * total + t] = make_uint4(0u, 0u, 0u, 0u);
  }
}

}  // namespace

static CpGeom make_cp_geom(const Geom& g, int world, int rank) {
  CpGeom c{};
  c.world = world;
  c.rank = rank;
  c.nloc = g.N / world;
  int E = 0;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    c.nl[l] = l < g.L ? g.n[l] / world : 0;
    if (l >= 1 && l < g.L) {
      c.offl[l] = E;
      E += c.nl[l];
    }
  }
  c.El = E;
  return c;
}

static int grid_for(long long total) {
  const long long b = (total + 255) / 256;
  return (int)(b < 148 * 16 ? (b > 0 ? b : 1) : 148 * 16);
}

cudaError_t launch_cp_assemble_sq(const Geom& g, int world, int rank, const double* gath, double* sq,
                                  cudaStream_t s) {
  const CpGeom c = make_cp_geom(g, world, rank);
  k_cp_assemble_sq<<<grid_for(2LL * g.B * g.H * g.E), 256, 0, s>>>(gath, sq, g, c);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_cp_segment(const Geom& g, int world, int rank, const int32_t* map, const int32_t* slot,
                              int32_t* slot_loc, int32_t* seg, cudaStream_t s) {
  const CpGeom c = make_cp_geom(g, world, rank);
  k_cp_segment<<<(g.B * g.H + 127) / 128, 128, 0, s>>>(map, seg, g, c);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_cp_slot<<<grid_for((long long)g.B * g.H * c.El), 256, 0, s>>>(slot, slot_loc, g, c);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_cp_gather(const Geom& g, lh_dtype dt, int world, int rank, const void* q, const void* k,
                             const void* v, const void* pq, const void* pk, const void* pv, const int32_t* map,
                             const int32_t* seg, const uint32_t* scale, void* qs, void* ks, void* vs, int* err,
                             cudaStream_t s) {
  const CpGeom c = make_cp_geom(g, world, rank);
  const int esz = dt == LH_BF16 ? 2 : 4;
  const int vin = g.D * esz / 16;                  // 16-byte vectors per input row
  const int vout = dt == LH_BF16 ? g.D * 2 / 16 : vin;
  const long long per = (long long)g.S * vout;
  dim3 grid((unsigned)((per + 255) / 256 < 4096 ? (per + 255) / 256 : 4096), (unsigned)(g.B * g.H), 3);
  if (dt == LH_BF16)
    k_cp_gather<true><<<grid, 256, 0, s>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, (const uint4*)pq,
                                           (const uint4*)pk, (const uint4*)pv, map, seg, scale, (uint4*)qs,
                                           (uint4*)ks, (uint4*)vs, g, c, vin, vout, err);
  else
    k_cp_gather<false><<<grid, 256, 0, s>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, (const uint4*)pq,
                                            (const uint4*)pk, (const uint4*)pv, map, seg, scale, (uint4*)qs,
                                            (uint4*)ks, (uint4*)vs, g, c, vin, vout, err);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_cp_zero_outside(const Geom& g, int elem_bytes, void* x, const int32_t* seg, cudaStream_t s) {
  const int vpr = g.D * elem_bytes / 16;
  const long long per = (long long)g.S * vpr;
  dim3 grid((unsigned)((per + 255) / 256 < 2048 ? (per + 255) / 256 : 2048), (unsigned)(g.B * g.H));
  k_cp_zero_outside<<<grid, 256, 0, s>>>((uint4*)x, seg, g.S, vpr);
  count_launch();
  return cudaGetLastError();
}

// Geometry of rank `rank`'s shard for the token-side kernels (pool, scatter,
// block sums, spread): its tokens and entries, with slot values and sub-sequence
// rows of the whole sequence (S unchanged).
Geom shard_geom(const Geom& g, int world, int rank) {
  const CpGeom c = make_cp_geom(g, world, rank);
  Geom s = g;
  s.N = c.nloc;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    s.n[l] = c.nl[l];
    s.off[l] = c.offl[l];
  }
  s.E = c.El;
  return s;
}

}  // namespace lh
