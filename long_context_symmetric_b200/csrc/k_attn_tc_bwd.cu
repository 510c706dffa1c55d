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
// A dS beyond the fp16 range is reported as LH_ERR_DEVICE, detail 101.
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
    float* vec = reinterpret_cast<float*>(sm + Lay::VEC);   // [2][2][128]: lse2, delta
    float dsmax = 0.f;
    bool ok = true;
    // every compute thread runs all n iterations (and their named barrier), also
    // after a wind-down, so no warp can be left waiting at the barrier
    for (int t = 0; t < n; ++t) {
      const int i = j + t;
      // this half's 64 query columns: lse (log2 units) and delta, double-buffered
      float* lse2 = vec + (t & 1) * 256 + 64 * half;
      float* dl = lse2 + 128;
      {
        const int hid = ctid & 127;                 // thread within the half
        const int q = i * kT + 64 * half + (hid & 63);
        if (hid < 64) lse2[hid] = q < S ? lse[(size_t)bh * S + q] * 1.4426950408889634f : 0.f;
        else dl[hid - 64] = q < S ? delta[(size_t)bh * S + q] : 0.f;
      }
      named_bar_sync(1 + half, kComputeThreads / 2);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_ready[half], t & 1, ab, err, 15));
      if (!ok) continue;
      tc_fence_after();
      const bool diag = (i == j);
      const int qlim = S - 1 - i * kT;                  // last valid query column
#pragma unroll 1
      for (int c = 2 * half; c < 2 * half + 2; ++c) {
        uint32_t s[32], dp[32];
        tmem_ld32(tbase + la + 32 * c, s);
        tmem_ld32(tbase + la + 128 + 32 * c, dp);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pe[2], de[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = 32 * c + e + u;
            const bool valid = col <= qlim && (!diag || col >= m);
            const float p = valid ? ex2(__uint_as_float(s[e + u]) * c2 - lse2[col - 64 * half]) : 0.f;
            pe[u] = p;
            de[u] = p * (__uint_as_float(dp[e + u]) - dl[col - 64 * half]);
            dsmax = fmaxf(dsmax, fabsf(de[u]));
          }
          pk[e >> 1] = pack_f16(pe[0], pe[1]);
          dk[e >> 1] = pack_f16(de[0], de[1]);
        }
        // fp16 results go to columns this warp has already read: chunk c's 16
        // packed columns at 16c + 32*half (each half packs inside its own 64)
        tmem_st16(tbase + la + 16 * c + 32 * half, pk);
        tmem_st16(tbase + la + 128 + 16 * c + 32 * half, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready[half]);
    }
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
    const float lse2 = q < S ? lse[(size_t)bh * S + q] * 1.4426950408889634f : 0.f;
    const float dl = q < S ? delta[(size_t)bh * S + q] : 0.f;
    float dsmax = 0.f;
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_ready[half], jj & 1, ab, err, 17))) { ok = false; break; }
      tc_fence_after();
      const bool diag = (jj == i);
      const int klim = min(diag ? r : kT - 1, S - 1 - jj * kT);   // last valid key column
#pragma unroll 1
      for (int c = 2 * half; c < 2 * half + 2; ++c) {
        uint32_t s[32], dp[32];
        tmem_ld32(tbase + la + 32 * c, s);
        tmem_ld32(tbase + la + 128 + 32 * c, dp);
        tmem_wait_ld();
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float h[2], rl[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = 32 * c + e + u;
            const float p = col <= klim ? ex2(__uint_as_float(s[e + u]) * c2 - lse2) : 0.f;
            const float ds = p * (__uint_as_float(dp[e + u]) - dl);
            dsmax = fmaxf(dsmax, fabsf(ds));
            h[u] = __half2float(__float2half_rn(ds));
            rl[u] = ds - h[u];
          }
          hi[e >> 1] = pack_f16(h[0], h[1]);
          lo[e >> 1] = pack_f16(rl[0], rl[1]);
        }
        // head into the (consumed) S columns, remainder into the (consumed) dP
        // columns, packed inside this half's own 64 columns
        tmem_st16(tbase + la + 16 * c + 32 * half, hi);
        tmem_st16(tbase + la + 128 + 16 * c + 32 * half, lo);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready[half]);
    }
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
