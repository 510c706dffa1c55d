// Causal flash attention on the sub-sequence with tcgen05 tensor cores,
// backward pass (fp16 operands, fp32 accumulate, deterministic: no atomics).
//
// "Long Context Pre-Training with Lighthouse Attention", Fig. 1: the gradient
// flows through the attention on the gathered sub-sequence. With P recomputed
// from the forward lse (natural log):
//   P = exp(S / sqrt(d) - lse),  dV = P^T dO,  dP = dO V^T,
//   dS = P o (dP - delta),  dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d).
//
// Operands are fp16 (11-bit significand): dO of a pooled entry is a block sum
// of up to p^(L-1) token gradients, and dS inherits that range, so bf16 operands
// would leave gradient errors several times the stated bound (measured against
// the fp64 oracle at 512K context); q/k/v arrive as exact fp16 copies of the
// bf16 sub-sequence. Two kernels, each one CTA per 128-row tile, heavy tiles
// first:
//  k_bwd_dkdv_tc  per key tile j, over query tiles i >= j:
//      S^T = K_j Q_i^T and dP^T = V_j dO_i^T into TMEM; the compute warps (two
//      per TMEM lane quarter, each on half of the columns) form P^T and dS^T
//      and store them as fp16 back into the same TMEM columns; then
//      dV += P^T dO_i and dK += dS^T Q_i take their A operand from TMEM.
//  k_bwd_dq_tc    per query tile i, over key tiles j <= i:
//      S = Q_i K_j^T and dP = dO_i V_j^T into TMEM; dS split into an fp16 head
//      and an fp16 remainder (dS = hi + lo to about 2^-22 relative) back into
//      TMEM; dQ += hi K_j + lo K_j.
// A dS whose fp16 rounding overflows (or is NaN) is reported as LH_ERR_DEVICE,
// detail 101.
// Q_i/dO_i (dkdv) or K_j/V_j (dq) stream through a 2-stage TMA ring; the
// operands that stay fixed for the CTA are loaded once. Same warp roles and
// bounded waits as the forward kernel.
#include "tc_ptx.cuh"

namespace lh {

bool make_tmap_16(CUtensorMap* m, const void* base, int D, int S, int BH, bool fp16);

namespace {

using namespace tc;

constexpr int kT = 128;              // rows per tile (both directions)
constexpr int kSub = 128 * 64 * 2;   // 128 x 64 bf16 swizzle tile
constexpr int kStages = 2;
// Warp roles: 0 producer, 1 MMA issuer, 2..9 compute. Two compute warps share
// each TMEM lane quarter (warps w and w+4), each taking half of a tile's 128
// columns, so every SM sub-partition has two compute warps to interleave.
constexpr int kComputeThreads = 256;
constexpr int kThreads = 64 + kComputeThreads;

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

template <int D>
struct BwdLayout {
  static constexpr int SUB = D / 64;
  static constexpr int FIX0 = 0;                               // fixed operand 0 (K_j or Q_i)
  static constexpr int FIX1 = FIX0 + SUB * kSub;               // fixed operand 1 (V_j or dO_i)
  static constexpr int RING = FIX1 + SUB * kSub;               // stages of (A, B) streamed tiles
  static constexpr int STAGE = 2 * SUB * kSub;
  static constexpr int VEC = RING + kStages * STAGE;           // lse / delta per query (dkdv)
  static constexpr int BAR = VEC + 2 * 2 * kT * 4;
  static constexpr int BYTES = (BAR + 256 + 1024) > 120 * 1024 ? (BAR + 256 + 1024) : 120 * 1024;
};

struct BwdBars {
  uint64_t fix_full, ring_full[kStages], ring_empty[kStages], s_ready[2], ds_ready[2], done, drain;
  uint32_t tmem_base;
  Abort abort;
};

// Shared prologue: barriers, TMEM allocation (512 columns).
__device__ __forceinline__ void bwd_setup(BwdBars* bars, int warp) {
  if (threadIdx.x == 0) {
    mbar_init(&bars->fix_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->ring_full[s], 1);
      mbar_init(&bars->ring_empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars->s_ready[h], 1);
      mbar_init(&bars->ds_ready[h], kComputeThreads / 2);
    }
    mbar_init(&bars->done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort.flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

__device__ __forceinline__ void bwd_teardown(uint32_t tbase, int warp) {
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tbase, 512);
  }
}

// Producer: the two fixed tiles once, then `n` pairs of streamed tiles at
// rows (first + t) * 128 of maps ma, mb.
template <int D>
__device__ void bwd_produce(uint8_t* sm, BwdBars* bars, const CUtensorMap* f0, const CUtensorMap* f1,
                            int frow, const CUtensorMap* ma, const CUtensorMap* mb, int first, int n,
                            int bh, volatile Abort* ab, int* err) {
  using Lay = BwdLayout<D>;
  constexpr int SUB = Lay::SUB;
  mbar_expect_tx(&bars->fix_full, 2 * SUB * kSub);
  for (int c = 0; c < SUB; ++c) {
    tma_load_3d(sm + Lay::FIX0 + c * kSub, f0, &bars->fix_full, 64 * c, frow * kT, bh);
    tma_load_3d(sm + Lay::FIX1 + c * kSub, f1, &bars->fix_full, 64 * c, frow * kT, bh);
  }
  int issued = 0;
  for (int t = 0; t < n; ++t) {
    const int st = t % kStages;
    if (t >= kStages && !mbar_wait(&bars->ring_empty[st], ((t / kStages) - 1) & 1, ab, err, 11)) break;
    uint8_t* base = sm + Lay::RING + st * Lay::STAGE;
    mbar_expect_tx(&bars->ring_full[st], Lay::STAGE);
    for (int c = 0; c < SUB; ++c) {
      tma_load_3d(base + c * kSub, ma, &bars->ring_full[st], 64 * c, (first + t) * kT, bh);
      tma_load_3d(base + (SUB + c) * kSub, mb, &bars->ring_full[st], 64 * c, (first + t) * kT, bh);
    }
    issued = t + 1;
  }
  if (ab->flag) {
    Abort none{0};
    mbar_wait(&bars->fix_full, 0, &none, nullptr, 0);
    for (int t = issued - kStages < 0 ? 0 : issued - kStages; t < issued; ++t)
      mbar_wait(&bars->ring_full[t % kStages], (t / kStages) & 1, &none, nullptr, 0);
  }
}

// MMA issuer shared by both kernels, pipelined by half tiles. For streamed
// tile t and half h (its rows 64h..64h+63):
//   X_h = F0 * A_t[h]^T (TMEM cols 64h..64h+63), Y_h = F1 * B_t[h]^T (cols 128+64h..)
// and, once compute warpgroup h has turned X_h/Y_h into fp16 operands in place,
//   dkdv (TWO_ACC): acc0 += Xh * B_t[h] (dV += P^T dO),  acc1 += Yh * A_t[h] (dK += dS^T Q)
//   dq:             acc1 += Xh * A_t[h] + Yh * A_t[h]   (dQ += (dS_hi + dS_lo) K)
// Issue order: acc(t-1, 0), X/Y_0(t), acc(t-1, 1), X/Y_1(t), ... so the tensor
// core works on one half while the other half's warps compute. acc(t-1, h)
// reads the fp16 values that X/Y_h(t) then overwrite; MMAs issued by one thread
// execute in issue order, which makes that safe without a wait.
template <int D, bool TWO_ACC>
__device__ void bwd_mma(uint8_t* sm, BwdBars* bars, uint32_t tbase, int n, volatile Abort* ab, int* err) {
  using Lay = BwdLayout<D>;
  constexpr int SUB = Lay::SUB;
  constexpr uint32_t IDX = idesc_f16(kT, 64, false);
  constexpr uint32_t IDACC = idesc_f16(kT, D, true);
  const uint32_t sbase = smem_u32(sm);
  const uint32_t tX = tbase, tY = tbase + 128;
  const uint32_t tAcc0 = tbase + 256, tAcc1 = tbase + 256 + (TWO_ACC ? D : 0);
  auto issue_xy = [&](int t, int h) {
    const uint32_t ring = sbase + Lay::RING + (t % kStages) * Lay::STAGE;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t koff = (kk >> 2) * kSub + (kk & 3) * 32;
      umma_f16(tX + 64 * h, sdesc_sw128(sbase + Lay::FIX0 + koff, 16, 1024),
               sdesc_sw128(ring + koff + 8192 * h, 16, 1024), IDX, kk > 0 ? 1u : 0u);
    }
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t koff = (kk >> 2) * kSub + (kk & 3) * 32;
      umma_f16(tY + 64 * h, sdesc_sw128(sbase + Lay::FIX1 + koff, 16, 1024),
               sdesc_sw128(ring + SUB * kSub + koff + 8192 * h, 16, 1024), IDX, kk > 0 ? 1u : 0u);
    }
    umma_commit(&bars->s_ready[h]);
  };
  auto accumulate = [&](int tt, int h) -> bool {
    if (!mbar_wait(&bars->ds_ready[h], tt & 1, ab, err, 14)) return false;
    tc_fence_after();
    const int st = tt % kStages;
    const uint32_t ring = sbase + Lay::RING + st * Lay::STAGE;
    const uint32_t tileA = ring, tileB = ring + SUB * kSub;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t acol = 64 * h + 8 * kk;        // half h's packed operand columns
      const uint32_t roff = (4 * h + kk) * 2048;     // its 16 rows of the streamed tiles
      const uint32_t first = (tt == 0 && h == 0 && kk == 0) ? 0u : 1u;
      const uint64_t g = sdesc_sw128(tileA + roff, kSub, 1024);
      if (TWO_ACC) {
        const uint64_t b = sdesc_sw128(tileB + roff, kSub, 1024);
        umma_f16_ts(tAcc0, tX + acol, b, IDACC, first);
        umma_f16_ts(tAcc1, tY + acol, g, IDACC, first);
      } else {
        umma_f16_ts(tAcc1, tX + acol, g, IDACC, first);
        umma_f16_ts(tAcc1, tY + acol, g, IDACC, 1u);
      }
    }
    if (h == 1) umma_commit(&bars->ring_empty[st]);
    return true;
  };
  bool ok = mbar_wait(&bars->fix_full, 0, ab, err, 12);
  for (int t = 0; ok && t < n; ++t) {
    const int st = t % kStages;
    if (!mbar_wait(&bars->ring_full[st], (t / kStages) & 1, ab, err, 13)) { ok = false; break; }
    for (int h = 0; h < 2; ++h) {
      if (t >= 1 && !accumulate(t - 1, h)) { ok = false; break; }
      tc_fence_after();
      issue_xy(t, h);
    }
  }
  if (ok && accumulate(n - 1, 0) && accumulate(n - 1, 1)) umma_commit(&bars->done);
  umma_commit(&bars->drain);
  Abort none{0};
  mbar_wait(&bars->drain, 0, &none, nullptr, 0);
}

__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a), __uint_as_float(b));
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// One 32-column chunk of this thread's key row of S^T and dP^T (dK/dV kernel):
// P^T = 2^(S^T c2 - lse2) and dS^T = P^T o (dP^T - delta) as fp16 pairs, two
// columns per packed fp32 instruction. nl2/ndl hold -lse2 and -delta of the
// chunk's 32 query columns (the same for every lane: broadcast reads). MASK:
// columns outside [vlo, vhi] (causal diagonal, rows past S) get P = 0.
template <bool MASK>
__device__ __forceinline__ void dkdv_chunk(const uint32_t (&s)[32], const uint32_t (&dp)[32],
                                           const float* nl2, const float* ndl, float c2, int col0, int vlo,
                                           int vhi, uint32_t (&pk)[16], uint32_t (&dk)[16], __half2& hm) {
  const float2 cc = make_float2(c2, c2);
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 a = *reinterpret_cast<const float4*>(nl2 + e);
    const float4 b = *reinterpret_cast<const float4*>(ndl + e);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float2 x = __ffma2_rn(f2(s[e + u], s[e + u + 1]), cc, u ? make_float2(a.z, a.w) : make_float2(a.x, a.y));
      float p0 = ex2(x.x), p1 = ex2(x.y);
      if (MASK) {
        const int col = col0 + e + u;
        if (col < vlo || col > vhi) p0 = 0.f;
        if (col + 1 < vlo || col + 1 > vhi) p1 = 0.f;
      }
      const float2 d = __fadd2_rn(f2(dp[e + u], dp[e + u + 1]), u ? make_float2(b.z, b.w) : make_float2(b.x, b.y));
      const __half2 ds = __float22half2_rn(__fmul2_rn(make_float2(p0, p1), d));
      hm = __hmax2_nan(hm, __habs2(ds));
      pk[(e + u) >> 1] = pack_f16(p0, p1);
      dk[(e + u) >> 1] = h2_bits(ds);
    }
  }
}

// One 32-column chunk of this thread's query row of S and dP (dQ kernel): dS as
// an fp16 head and an fp16 remainder (hi + lo = dS to about 2^-22 relative).
// nl2 = -lse2, ndl = -delta of the row. MASK: key columns past vhi get P = 0.
template <bool MASK>
__device__ __forceinline__ void dq_chunk(const uint32_t (&s)[32], const uint32_t (&dp)[32], float nl2, float ndl,
                                         float c2, int col0, int vhi, uint32_t (&hi)[16], uint32_t (&lo)[16],
                                         __half2& hm) {
  const float2 cc = make_float2(c2, c2), nl = make_float2(nl2, nl2), nd = make_float2(ndl, ndl);
  const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float2 x = __ffma2_rn(f2(s[e], s[e + 1]), cc, nl);
    float p0 = ex2(x.x), p1 = ex2(x.y);
    if (MASK) {
      if (col0 + e > vhi) p0 = 0.f;
      if (col0 + e + 1 > vhi) p1 = 0.f;
    }
    const float2 ds = __fmul2_rn(make_float2(p0, p1), __fadd2_rn(f2(dp[e], dp[e + 1]), nd));
    const __half2 h = __float22half2_rn(ds);
    hm = __hmax2_nan(hm, __habs2(h));
    const float2 r = __ffma2_rn(__half22float2(h), m1, ds);     // ds - hi, exact
    hi[e >> 1] = h2_bits(h);
    lo[e >> 1] = h2_bits(__float22half2_rn(r));
  }
}

// ---------------------------------------------------------------- dK, dV
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
              const float* __restrict__ lse, const float* __restrict__ delta, float* __restrict__ dks,
              float* __restrict__ dvs, int S, float c2, float scale, int* err) {
  using Lay = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  BwdBars* bars = reinterpret_cast<BwdBars*>(sm + Lay::BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = gridDim.x;
  const int j = blockIdx.x;            // key tile; small j has the most query tiles
  const int bh = blockIdx.y;
  const int n = ntiles - j;            // query tiles i = j .. ntiles-1
  bwd_setup(bars, warp);
  const uint32_t tbase = bars->tmem_base;
  volatile Abort* ab = &bars->abort;

  if (warp == 0) {
    if (lane == 0) bwd_produce<D>(sm, bars, &tk, &tv, j, &tq, &tdo, j, n, bh, ab, err);
  } else if (warp == 1) {
    if (lane == 0) bwd_mma<D, true>(sm, bars, tbase, n, ab, err);
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;                   // which 64 of the 128 columns
    const int m = quarter * 32 + lane;                  // key row within the tile / TMEM lane
    const int ctid = threadIdx.x - 64;                  // 0..255
    const uint32_t la = (uint32_t)(quarter * 32) << 16;
    const int key = j * kT + m;
    float* vec = reinterpret_cast<float*>(sm + Lay::VEC);   // [2][2][128]: -lse2, -delta
    // this thread's share of a query tile's -lse2 / -delta (thread hid of the
    // half: column 64*half + (hid & 63)), fetched one tile ahead
    const int hid = ctid & 127;
    const float* vsrc = (hid < 64 ? lse : delta) + (size_t)bh * S;
    const float vmul = hid < 64 ? -1.4426950408889634f : -1.f;
    auto fetch = [&](int i) -> float {
      const int q = i * kT + 64 * half + (hid & 63);
      return q < S ? vsrc[q] : 0.f;
    };
    float nxt = fetch(j);
    __half2 hm = __float2half2_rn(0.f);
    bool ok = true;
    // every compute thread runs all n iterations (and their named barrier), also
    // after a wind-down, so no warp can be left waiting at the barrier
    for (int t = 0; t < n; ++t) {
      const int i = j + t;
      // this half's 64 query columns, double-buffered by tile parity
      float* nl2 = vec + (t & 1) * 256 + 64 * half;
      float* ndl = nl2 + 128;
      (hid < 64 ? nl2 : ndl)[hid & 63] = nxt * vmul;
      named_bar_sync(1 + half, kComputeThreads / 2);
      if (t + 1 < n) nxt = fetch(i + 1);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_ready[half], t & 1, ab, err, 15));
      if (!ok) continue;
      tc_fence_after();
      const int vlo = i == j ? m : 0;                   // causal: query col >= key row
      const int vhi = min(kT - 1, S - 1 - i * kT);      // last valid query column
      const bool mask = vlo > 0 || vhi < kT - 1 || i == j;
      // chunk c0 = 2*half, then c0 + 1; the second chunk's loads overlap the
      // first chunk's arithmetic
      const int c0 = 2 * half;
      uint32_t s0[32], d0[32], s1[32], d1[32], pk[16], dk[16];
      tmem_ld32(tbase + la + 32 * c0, s0);
      tmem_ld32(tbase + la + 128 + 32 * c0, d0);
      tmem_wait_ld_regs(s0);
      reg_fence32(d0);
      tmem_ld32(tbase + la + 32 * c0 + 32, s1);
      tmem_ld32(tbase + la + 160 + 32 * c0, d1);
      if (mask) dkdv_chunk<true>(s0, d0, nl2, ndl, c2, 32 * c0, vlo, vhi, pk, dk, hm);
      else dkdv_chunk<false>(s0, d0, nl2, ndl, c2, 32 * c0, vlo, vhi, pk, dk, hm);
      // fp16 results go to columns this warp has already read: chunk c's 16
      // packed columns at 16c + 32*half (each half packs inside its own 64)
      tmem_st16(tbase + la + 16 * c0 + 32 * half, pk);
      tmem_st16(tbase + la + 128 + 16 * c0 + 32 * half, dk);
      tmem_wait_ld_regs(s1);
      reg_fence32(d1);
      if (mask) dkdv_chunk<true>(s1, d1, nl2 + 32, ndl + 32, c2, 32 * c0 + 32, vlo, vhi, pk, dk, hm);
      else dkdv_chunk<false>(s1, d1, nl2 + 32, ndl + 32, c2, 32 * c0 + 32, vlo, vhi, pk, dk, hm);
      tmem_st16(tbase + la + 16 * c0 + 16 + 32 * half, pk);
      tmem_st16(tbase + la + 128 + 16 * c0 + 16 + 32 * half, dk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready[half]);
    }
    const float dsmax = __half2float(__hmax_nan(__low2half(hm), __high2half(hm)));
    if (!(dsmax <= kHalfMax)) report_error(err, LH_ERR_DEVICE, 101);
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->done, 0, ab, err, 16))) {
      tc_fence_after();
      float* ddv = dvs + ((size_t)bh * S + key) * D;
      float* ddk = dks + ((size_t)bh * S + key) * D;
#pragma unroll 1
      for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
        // the TMEM loads are warp-collective (.sync.aligned): every lane runs
        // them, rows past S included; only the stores are per-row
        uint32_t a[32], b[32];
        tmem_ld32(tbase + la + 256 + 32 * c, a);
        tmem_ld32(tbase + la + 256 + D + 32 * c, b);
        tmem_wait_ld();
        if (key < S) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            *reinterpret_cast<float4*>(ddv + 32 * c + e) =
                make_float4(__uint_as_float(a[e]), __uint_as_float(a[e + 1]), __uint_as_float(a[e + 2]),
                            __uint_as_float(a[e + 3]));
            *reinterpret_cast<float4*>(ddk + 32 * c + e) =
                make_float4(__uint_as_float(b[e]) * scale, __uint_as_float(b[e + 1]) * scale,
                            __uint_as_float(b[e + 2]) * scale, __uint_as_float(b[e + 3]) * scale);
          }
        }
      }
    }
  }
  bwd_teardown(tbase, warp);
}

// ---------------------------------------------------------------- dQ
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
k_bwd_dq_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
            const float* __restrict__ lse, const float* __restrict__ delta, float* __restrict__ dqs,
            int S, float c2, float scale, int* err) {
  using Lay = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  BwdBars* bars = reinterpret_cast<BwdBars*>(sm + Lay::BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = gridDim.x;
  const int i = ntiles - 1 - (int)blockIdx.x;     // query tile; late tiles have the most key tiles
  const int bh = blockIdx.y;
  const int n = i + 1;                            // key tiles j = 0 .. i
  bwd_setup(bars, warp);
  const uint32_t tbase = bars->tmem_base;
  volatile Abort* ab = &bars->abort;

  if (warp == 0) {
    if (lane == 0) bwd_produce<D>(sm, bars, &tq, &tdo, i, &tk, &tv, 0, n, bh, ab, err);
  } else if (warp == 1) {
    if (lane == 0) bwd_mma<D, false>(sm, bars, tbase, n, ab, err);
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;             // which 64 of the 128 columns
    const int r = quarter * 32 + lane;            // query row within the tile / TMEM lane
    const uint32_t la = (uint32_t)(quarter * 32) << 16;
    const int q = i * kT + r;
    const float nl2 = q < S ? lse[(size_t)bh * S + q] * -1.4426950408889634f : 0.f;
    const float ndl = q < S ? -delta[(size_t)bh * S + q] : 0.f;
    __half2 hm = __float2half2_rn(0.f);
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_ready[half], jj & 1, ab, err, 17))) { ok = false; break; }
      tc_fence_after();
      const int klim = min(jj == i ? r : kT - 1, S - 1 - jj * kT);   // last valid key column
      const bool mask = klim < kT - 1;
      // chunk c0 = 2*half, then c0 + 1 (its loads overlap chunk c0's arithmetic);
      // head into the (consumed) S columns, remainder into the (consumed) dP
      // columns, packed inside this half's own 64 columns
      const int c0 = 2 * half;
      uint32_t s0[32], d0[32], s1[32], d1[32], hi[16], lo[16];
      tmem_ld32(tbase + la + 32 * c0, s0);
      tmem_ld32(tbase + la + 128 + 32 * c0, d0);
      tmem_wait_ld_regs(s0);
      reg_fence32(d0);
      tmem_ld32(tbase + la + 32 * c0 + 32, s1);
      tmem_ld32(tbase + la + 160 + 32 * c0, d1);
      if (mask) dq_chunk<true>(s0, d0, nl2, ndl, c2, 32 * c0, klim, hi, lo, hm);
      else dq_chunk<false>(s0, d0, nl2, ndl, c2, 32 * c0, klim, hi, lo, hm);
      tmem_st16(tbase + la + 16 * c0 + 32 * half, hi);
      tmem_st16(tbase + la + 128 + 16 * c0 + 32 * half, lo);
      tmem_wait_ld_regs(s1);
      reg_fence32(d1);
      if (mask) dq_chunk<true>(s1, d1, nl2, ndl, c2, 32 * c0 + 32, klim, hi, lo, hm);
      else dq_chunk<false>(s1, d1, nl2, ndl, c2, 32 * c0 + 32, klim, hi, lo, hm);
      tmem_st16(tbase + la + 16 * c0 + 16 + 32 * half, hi);
      tmem_st16(tbase + la + 128 + 16 * c0 + 16 + 32 * half, lo);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready[half]);
    }
    const float dsmax = __half2float(__hmax_nan(__low2half(hm), __high2half(hm)));
    if (!(dsmax <= kHalfMax)) report_error(err, LH_ERR_DEVICE, 101);
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->done, 0, ab, err, 18))) {
      tc_fence_after();
      float* dst = dqs + ((size_t)bh * S + q) * D;
#pragma unroll 1
      for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
        uint32_t a[32];
        tmem_ld32(tbase + la + 256 + 32 * c, a);
        tmem_wait_ld();
        if (q < S) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + e) =
                make_float4(__uint_as_float(a[e]) * scale, __uint_as_float(a[e + 1]) * scale,
                            __uint_as_float(a[e + 2]) * scale, __uint_as_float(a[e + 3]) * scale);
        }
      }
    }
  }
  bwd_teardown(tbase, warp);
}

template <int D>
cudaError_t bwd_tc_t(const Geom& g, const void* qs, const void* ks, const void* vs, const void* dos,
                     const float* lse, const float* delta, float* dqs, float* dks, float* dvs, int* err,
                     cudaStream_t s) {
  CUtensorMap tq, tk, tv, tdo;
  const int BH = g.B * g.H;
  if (!make_tmap_16(&tq, qs, D, g.S, BH, true) || !make_tmap_16(&tk, ks, D, g.S, BH, true) ||
      !make_tmap_16(&tv, vs, D, g.S, BH, true) || !make_tmap_16(&tdo, dos, D, g.S, BH, true))
    return cudaErrorInvalidValue;
  const int smem = BwdLayout<D>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(k_bwd_dkdv_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_bwd_dq_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const float scale = (float)(1.0 / sqrt((double)D));
  const float c2 = (float)(1.4426950408889634 / sqrt((double)D));
  dim3 grid((g.S + kT - 1) / kT, BH);
  k_bwd_dkdv_tc<D><<<grid, kThreads, smem, s>>>(tq, tk, tv, tdo, lse, delta, dks, dvs, g.S, c2, scale, err);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_bwd_dq_tc<D><<<grid, kThreads, smem, s>>>(tq, tk, tv, tdo, lse, delta, dqs, g.S, c2, scale, err);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const Geom& g, const void* qs, const void* ks, const void* vs,
                               const void* dos, const float* lse, const float* delta, float* dqs,
                               float* dks, float* dvs, int* err, cudaStream_t s) {
  return g.D == 64 ? bwd_tc_t<64>(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, err, s)
                   : bwd_tc_t<128>(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, err, s);
}

}  // namespace lh
