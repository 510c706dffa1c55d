// Hierarchical top-K descent + post-order of the selection, one CTA per (b, h).
//
// "Long Context Pre-Training with Lighthouse Attention", §3.1 stage (ii) and
// Fig. 2 step 3 (chunked bitonic top-K, parents kept, tree pruned), Fig. 1 (the
// gathered hierarchy is sorted topologically into one causal sequence);
// "Lighthouse Attention Technique" (positions sorted before the gather, no
// holes in the causal sequence).
//
// Per level l = L-1 .. 1 (all entries of level L-1 are the first candidates):
//   score = max(|mean_Q|^2, |mean_K|^2) (fp64, from lh_pool); the other
//   selectable readings: |mean_K|^2, |mean_Q| + |mean_K|, |mean_Q|^2 |mean_K|^2,
//   and the max-pool reading (the same max, of lh_pool's max-pooled token norms)
//   the first k_l candidates in the order (score desc, index asc; or index
//   desc under the other tie reading) are expanded.
//   Only the set matters (the sub-sequence order comes from the tree below),
//   so for up to 8192 candidates it is found by a most-significant-digit
//   radix select on the unique key (score bits, then position reversed): ten
//   8-bit digit passes, each a 256-bin shared-memory histogram of the keys
//   that still match the chosen prefix, give the k_l-th key, and every key at
//   or above it is expanded. Beyond 8192 candidates the pages' chunked bitonic
//   sort is used: a sorting network over shared-memory chunks of 8192
//   (score, position) keys, the current best k_l kept at the head of the chunk
//   and the rest refilled with new candidates, chunk after chunk (k_l <= 4096).
//   the p children of each expanded entry, in index order, are the next
//   level's candidates and sub-sequence entries.
// Post-order: every included entry's subtree (itself plus its included
// descendants) occupies a contiguous run of slots ending at the entry, coarse
// entries in index order. Subtree sizes are formed bottom-up, run starts
// top-down; slot = start + size - 1. This equals sorting the entries by
// (last covered token, level). Pre-order (the other order reading): the run
// starts at the entry, slot = start, children runs from start + 1; this equals
// sorting by (first covered token, coarser level first). Partition reading
// (expanded entries leave the sub-sequence): an expanded entry's run is its
// children's runs alone, the included entries tile the tokens and both orders
// give the same sequence; the slot table keeps the run start of an expanded
// entry (2 * start + 1), which locates the tokens of a level-1 entry.
//
// Per-level working arrays (candidate index, expanded flag, rank among the
// expanded, subtree size, run start) live in the caller's workspace
// (5 int32 per candidate of any level, per (b,h)); the sort keys live in
// shared memory.
#include "lh_common.cuh"

namespace lh {
namespace {

constexpr int kThreads = 1024;
constexpr int kChunk = 8192;   // sort keys per shared-memory chunk (12 bytes each)

struct SelArgs {
  Geom g;
  int lvl_base[LH_MAX_LEVELS];   // start of level l's arrays inside one array of the per-head ws
};

__device__ __forceinline__ bool precedes(unsigned long long sa, unsigned pa, unsigned long long sb,
                                         unsigned pb, bool high_first) {
  return sa > sb || (sa == sb && (high_first ? pa > pb : pa < pb));
}

// Block-wide exclusive scan of in[0..n) into out[0..n); returns the total.
// `in` and `out` may alias. All threads must call it.
__device__ int block_exclusive_scan(const int* in, int* out, int n, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int carry = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + threadIdx.x;
    const int x = i < n ? in[i] : 0;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int t = warp_tot[lane];
      int ti = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, ti, o);
        if (lane >= o) ti += y;
      }
      warp_tot[lane] = ti - t;      // exclusive prefix of warp totals
      if (lane == 31) warp_tot[32] = ti;
    }
    __syncthreads();
    if (i < n) out[i] = carry + warp_tot[warp] + incl - x;
    carry += warp_tot[32];
    __syncthreads();
  }
  return carry;
}

// Bitonic sort of keys[0..n) (n a power of two) so that index 0 comes first
// under `precedes`.
__device__ void bitonic_sort(unsigned long long* sk, unsigned* sp, int n, bool high_first) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (n >> 1); i += kThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const unsigned long long a = sk[lo], b = sk[hi];
        const unsigned pa = sp[lo], pb = sp[hi];
        const bool sw = up ? precedes(b, pb, a, pa, high_first) : precedes(a, pa, b, pb, high_first);
        if (sw) {
          sk[lo] = b; sk[hi] = a;
          sp[lo] = pb; sp[hi] = pa;
        }
      }
      __syncthreads();
    }
  }
}

// Score of entry e as an order-preserving 64-bit key (every score is >= 0, so
// its bit pattern orders like its value). mode: lh_score.
__device__ __forceinline__ unsigned long long score_bits(const double* sqq, const double* sqk,
                                                         int e, int mode) {
  const double a = sqq[e], b = sqk[e];
  double s;
  switch (mode) {
    case 1: s = b; break;                                           // |mean_k|^2
    case 2: s = __dadd_rn(__dsqrt_rn(a), __dsqrt_rn(b)); break;     // |mean_q| + |mean_k|
    case 3: s = __dmul_rn(a, b); break;                             // |mean_q|^2 |mean_k|^2
    default: s = fmax(a, b);   // max of the squared norms (maxpool: of the max-pooled token norms)
  }
  return (unsigned long long)__double_as_longlong(s);
}

// Flags fl[q] = 1 for the k (< c <= kChunk) candidates q first in the order
// (score desc, q asc; q desc if high_first), 0 for the rest. Key of q: hi =
// score bits, lo = c-1-q (q if high_first), compared as (hi, lo) descending;
// keys are unique. hist: 257 ints of shared memory, bc: 3 ints. All threads
// must call it.
__device__ void radix_select_flags(const double* sq_l, const double* sk_l, const int32_t* cl, int c, int k,
                                   int score_mode, bool high_first, int32_t* fl, int* hist, int* bc) {
  constexpr int KPT = kChunk / kThreads;
  const int lane = threadIdx.x & 31;
  unsigned long long hi[KPT];
  unsigned lo[KPT];
  bool valid[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int q = threadIdx.x + j * kThreads;
    valid[j] = q < c;
    hi[j] = valid[j] ? score_bits(sq_l, sk_l, cl[q], score_mode) : 0ull;
    lo[j] = valid[j] ? (unsigned)(high_first ? q : c - 1 - q) : 0u;
  }
  unsigned long long thi = 0ull;   // chosen digits of the threshold key so far
  unsigned tlo = 0u;
  int kk = k;                      // rank of the threshold among keys matching the prefix
  // passes 0..7: hi bits 63..0; passes 8, 9: lo bits 15..0 (c <= kChunk < 2^16)
#pragma unroll 1
  for (int pass = 0; pass < 10; ++pass) {
    for (int i = threadIdx.x; i < 257; i += kThreads) hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      int d = 256;                 // 256: not counted
      if (valid[j]) {
        if (pass < 8) {
          const int sh = 56 - 8 * pass;
          const bool m = pass == 0 || (hi[j] >> (sh + 8)) == (thi >> (sh + 8));
          if (m) d = (int)((hi[j] >> sh) & 0xFF);
        } else {
          const int sh = 8 * (9 - pass);
          const bool m = hi[j] == thi && (pass == 8 || (lo[j] >> (sh + 8)) == (tlo >> (sh + 8)));
          if (m) d = (int)((lo[j] >> sh) & 0xFF);
        }
      }
      // one atomic per distinct digit of the warp
      const unsigned same = __match_any_sync(0xffffffffu, d);
      if (d < 256 && lane == __ffs(same) - 1) atomicAdd(&hist[d], __popc(same));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // bins from the top: lane l sums bins 255-8l .. 248-8l
      int loc[8], sum = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) { loc[u] = hist[255 - 8 * lane - u]; sum += loc[u]; }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int above = incl - sum;      // keys in bins above this lane's first bin
      if (above < kk && kk <= incl) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (above < kk && kk <= above + loc[u]) {
            bc[0] = 255 - 8 * lane - u;
            bc[1] = kk - above;
            bc[2] = loc[u];
          }
          above += loc[u];
        }
      }
    }
    __syncthreads();
    const int b = bc[0];
    kk = bc[1];
    // the threshold is the bin's last key and the bin is taken whole: every key
    // with this prefix is expanded, so the digits below can stay zero (with
    // continuous scores this ends the select after two or three passes)
    const bool whole = bc[2] == kk;
    if (pass < 8) thi |= (unsigned long long)b << (56 - 8 * pass);
    else tlo |= (unsigned)b << (8 * (9 - pass));
    __syncthreads();               // bc is rewritten by the next pass
    if (whole) break;
  }
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int q = threadIdx.x + j * kThreads;
    if (valid[j]) fl[q] = (hi[j] > thi || (hi[j] == thi && lo[j] >= tlo)) ? 1 : 0;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
k_select(const double* __restrict__ sq, int32_t* __restrict__ sel, int32_t* __restrict__ map,
         int32_t* __restrict__ slot, int32_t* __restrict__ ws, SelArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned long long* sk = reinterpret_cast<unsigned long long*>(smem_raw);
  unsigned* sp = reinterpret_cast<unsigned*>(sk + kChunk);
  __shared__ int warp_tot[33];
  __shared__ int hist[257], bcast[3];

  const Geom& g = a.g;
  const int bh = blockIdx.x;
  const int L = g.L, p = g.p, S = g.S, C = g.C;
  const double* sqq = sq + (size_t)bh * g.E;
  const double* sqk = sq + ((size_t)g.B * g.H + bh) * g.E;
  int32_t* cand = ws + (size_t)bh * 5 * C;
  int32_t* flag = cand + C;
  int32_t* rank = flag + C;
  int32_t* size = rank + C;
  int32_t* start = size + C;
  int32_t* slot_h = slot + (size_t)bh * g.E;
  int32_t* sel_h = sel + (size_t)bh * (L - 1) * g.K;
  int32_t* map_h = map + (size_t)bh * S;

  // levels 1..L-2 hold entries that may stay out of the sub-sequence
  for (int l = 1; l <= L - 2; ++l)
    for (int i = threadIdx.x; i < g.n[l]; i += kThreads) slot_h[g.off[l] + i] = -1;
  {
    int32_t* c0 = cand + a.lvl_base[L - 1];
    for (int i = threadIdx.x; i < g.n[L - 1]; i += kThreads) c0[i] = i;
  }
  __syncthreads();

  // ---------------- descent
  for (int l = L - 1; l >= 1; --l) {
    const int c = g.cand[l], k = g.k[l];
    int32_t* cl = cand + a.lvl_base[l];
    int32_t* fl = flag + a.lvl_base[l];
    const double* sq_l = sqq + g.off[l];
    const double* sk_l = sqk + g.off[l];
    if (k >= c) {
      for (int q = threadIdx.x; q < c; q += kThreads) fl[q] = 1;
    } else if (c <= kChunk) {
      radix_select_flags(sq_l, sk_l, cl, c, k, g.score, g.ties != 0, fl, hist, bcast);
    } else {
      for (int q = threadIdx.x; q < c; q += kThreads) fl[q] = 0;
      // chunked top-k: best k stay at the head of the chunk between rounds. With
      // ties broken towards higher positions, positions are stored + 1 so that
      // the sentinel (position 0) sorts after every real candidate.
      const unsigned pos_shift = g.ties ? 1u : 0u;
      int n2 = 1;
      while (n2 < (c < kChunk ? c : kChunk)) n2 <<= 1;
      int next = 0, held = 0;
      while (next < c) {
        const int room = n2 - held;
        const int take = min(room, c - next);
        for (int i = threadIdx.x; i < room; i += kThreads) {
          if (i < take) {
            const int qpos = next + i;
            sk[held + i] = score_bits(sq_l, sk_l, cl[qpos], g.score);
            sp[held + i] = (unsigned)qpos + pos_shift;
          } else {
            sk[held + i] = 0ull;            // sentinel: after every real candidate
            sp[held + i] = g.ties ? 0u : 0xFFFFFFFFu;
          }
        }
        __syncthreads();
        bitonic_sort(sk, sp, n2, g.ties != 0);
        next += take;
        held = k;
      }
      for (int r = threadIdx.x; r < k; r += kThreads) fl[sp[r] - pos_shift] = 1;
    }
    __syncthreads();
    // rank among expanded (exclusive scan), selection output, next candidates
    int32_t* rl = rank + a.lvl_base[l];
    block_exclusive_scan(fl, rl, c, warp_tot);
    int32_t* cn = cand + a.lvl_base[l - 1];
    int32_t* sel_l = sel_h + (size_t)(l - 1) * g.K;
    for (int q = threadIdx.x; q < c; q += kThreads) {
      if (fl[q]) {
        const int r = rl[q];
        const int e = cl[q];
        sel_l[r] = e;
        for (int j = 0; j < p; ++j) cn[r * p + j] = e * p + j;
      }
    }
    for (int r = k + threadIdx.x; r < g.K; r += kThreads) sel_l[r] = -1;
    __syncthreads();
  }

  // ---------------- subtree sizes, bottom-up
  {
    int32_t* f0 = flag + a.lvl_base[0];
    int32_t* s0 = size + a.lvl_base[0];
    for (int q = threadIdx.x; q < g.cand[0]; q += kThreads) { f0[q] = 0; s0[q] = 1; }
  }
  __syncthreads();
  for (int l = 1; l <= L - 1; ++l) {
    const int32_t* fl = flag + a.lvl_base[l];
    const int32_t* rl = rank + a.lvl_base[l];
    int32_t* sl = size + a.lvl_base[l];
    const int32_t* sc = size + a.lvl_base[l - 1];
    for (int q = threadIdx.x; q < g.cand[l]; q += kThreads) {
      int sz = (fl[q] && g.incl) ? 0 : 1;   // partition: an expanded entry is not in its run
      if (fl[q]) {
        const int base = rl[q] * p;
        for (int j = 0; j < p; ++j) sz += sc[base + j];
      }
      sl[q] = sz;
    }
    __syncthreads();
  }

  // ---------------- run starts, top-down
  block_exclusive_scan(size + a.lvl_base[L - 1], start + a.lvl_base[L - 1], g.cand[L - 1], warp_tot);
  __syncthreads();
  for (int l = L - 1; l >= 1; --l) {
    const int32_t* fl = flag + a.lvl_base[l];
    const int32_t* rl = rank + a.lvl_base[l];
    const int32_t* stl = start + a.lvl_base[l];
    const int32_t* sc = size + a.lvl_base[l - 1];
    int32_t* stc = start + a.lvl_base[l - 1];
    for (int q = threadIdx.x; q < g.cand[l]; q += kThreads) {
      if (fl[q]) {
        // pre-order (nested): the entry first, then its children's runs
        int s = stl[q] + (g.order && !g.incl ? 1 : 0);
        const int base = rl[q] * p;
        for (int j = 0; j < p; ++j) {
          stc[base + j] = s;
          s += sc[base + j];
        }
      }
    }
    __syncthreads();
  }

  // ---------------- outputs: gather map and slot table
  for (int l = 0; l <= L - 1; ++l) {
    const int32_t* cl = cand + a.lvl_base[l];
    const int32_t* fl = flag + a.lvl_base[l];
    const int32_t* sl = size + a.lvl_base[l];
    const int32_t* stl = start + a.lvl_base[l];
    for (int q = threadIdx.x; q < g.cand[l]; q += kThreads) {
      const int e = cl[q];
      if (g.incl && fl[q]) {                // partition: expanded, not in the sub-sequence
        slot_h[g.off[l] + e] = 2 * stl[q] + 1;
        continue;
      }
      const int sidx = g.order ? stl[q] : stl[q] + sl[q] - 1;
      map_h[sidx] = (l << 28) | e;
      if (l >= 1) slot_h[g.off[l] + e] = 2 * sidx + (fl[q] ? 1 : 0);
    }
  }
}

// L == 1: the sub-sequence is the token sequence itself.
__global__ void k_identity_map(int32_t* __restrict__ map, long long total, int N) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x)
    map[i] = (int32_t)(i % N);
}

}  // namespace

cudaError_t launch_select(const Geom& g, const double* sq, int32_t* sel, int32_t* map,
                          int32_t* slot, int32_t* ws, cudaStream_t s) {
  if (g.L == 1) {
    const long long total = (long long)g.B * g.H * g.N;
    const int blocks = (int)((total + 255) / 256 < 148 * 8 ? (total + 255) / 256 : 148 * 8);
    k_identity_map<<<blocks, 256, 0, s>>>(map, total, g.N);
    count_launch();
    return cudaGetLastError();
  }
  SelArgs a;
  a.g = g;
  int base = 0;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    a.lvl_base[l] = base;
    if (l < g.L) base += g.cand[l];
  }
  const size_t smem = (size_t)kChunk * (sizeof(unsigned long long) + sizeof(unsigned));
  cudaError_t e = cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_select<<<g.B * g.H, kThreads, smem, s>>>(sq, sel, map, slot, ws, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lh
