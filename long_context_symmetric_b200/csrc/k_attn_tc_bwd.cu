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
//      X = S^T = K_j Q_i^T and Y = dP^T = V_j dO_i^T (TMEM); the compute warps
//      form P^T and dS^T and store them as fp16 into Y's columns; then
//      dK += dS^T Q_i and dV += P^T dO_i take their A operand from TMEM.
//  k_bwd_dq_tc    per query tile i, over key tiles j <= i:
//      X = S = Q_i K_j^T and Y = dP = dO_i V_j^T, Y in two alternating TMEM
//      buffers; dS is split into an fp16 head and an fp16 remainder
//      (dS = hi + lo to about 2^-22 relative) stored into Y's columns;
//      dQ += hi K_j + lo K_j.
// A dS whose fp16 rounding overflows (or any NaN) makes dK and dQ non-finite
// (an infinite operand times any value, summed in fp32, stays inf or NaN), so
// the epilogues check their fp32 results and report LH_ERR_DEVICE, detail 101.
//
// Pipeline (tensor core order per streamed tile t): dK/dV X(t+1), dV(t),
// dK(t), Y(t+1); dQ X(t+1), Y(t+1), acc(t). The compute warps copy X(t) into
// registers and release it at once, so X(t+1) runs while they exponentiate;
// they read Y(t) and write the fp16 operands of the accumulating MMAs into
// Y's columns. In the dK/dV kernel (whose TMEM holds two accumulators) Y(t+1)
// must follow dK(t) and dV(t); P^T is stored before dS^T is formed and has its
// own barrier, so dV(t) runs during that work and only dK(t) and Y(t+1) lie
// between one tile's dS^T and the next. The dQ kernel has a second Y buffer
// and computes Y(t+1) during the compute warps' work on tile t (tcgen05.mma
// ops issued by one thread execute in order, which orders every reuse of a
// TMEM column). All score MMAs are
// full 128 x 128 tiles: N = 64 halves run at about two thirds of the rate and
// lose more when the compute warps use TMEM at the same time (measured).
// Streamed tiles come through a TMA ring whose two operands have their own
// stages and full/empty barriers, so each is refilled as soon as its last
// reader is done; the operand that X reads gets three stages, as X(t+2) is
// issued right after acc(t), before a two-stage ring could have refilled it.
// Bounded waits as in the forward kernel.
#include "tc_ptx.cuh"

namespace lh {

bool make_tmap_16(CUtensorMap* m, const void* base, int D, int S, int BH, bool fp16, int box_rows);

namespace {

using namespace tc;

constexpr int kT = 128;              // rows per tile (both directions)
constexpr int kSub = 128 * 64 * 2;   // 128 x 64 16-bit swizzle tile
constexpr int kMaxStages = 3;
// TMEM columns: X at 0, Y at 128 (dq: Y buffers at 128 and 256), accumulators
// from 256 (dkdv: dV, then dK) or 384 (dq: dQ)
constexpr uint32_t kColY = 128;
__host__ __device__ constexpr uint32_t col_acc(bool two_acc) { return two_acc ? 256u : 384u; }
// Warp roles: 0 producer, 1 MMA issuer, 2..9 compute. Two compute warps share
// each TMEM lane quarter (warps w and w+4), each taking 64 of a tile's 128
// columns, so every SM sub-partition has two compute warps to interleave.
constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = 32 * kComputeWarps;
constexpr int kThreads = 64 + kComputeThreads;

// Barriers and the lse/delta vector (dkdv) come first, the swizzled tiles from
// the next 1024-byte boundary (TILES bytes, offsets below relative to that
// boundary); BYTES covers the worst-case alignment gap of the dynamic
// shared-memory base.
template <int D>
struct BwdLayout {
  static constexpr int SUB = D / 64;
  static constexpr int OPB = SUB * kSub;                       // one 128-row operand tile
  static constexpr int NSTA = 3;                               // stages of A_t (read by X and acc)
  static constexpr int NSTB = 2;                               // stages of B_t
  static constexpr int FIX0 = 0;                               // fixed operand 0 (K_j / Q_i)
  static constexpr int FIX1 = FIX0 + OPB;                      // fixed operand 1 (V_j / dO_i)
  static constexpr int RA = FIX1 + OPB;                        // A_t stages
  static constexpr int RB = RA + NSTA * OPB;                   // B_t stages
  static constexpr int TILES = RB + NSTB * OPB;
  static constexpr int HEAD = 256 + 2 * kT * 4;                // barriers, then -lse2 / -delta (dkdv)
  static constexpr int BYTES = HEAD + 1024 + TILES;
  static_assert(BYTES <= 227 * 1024, "shared memory");
};

// ring_full/ring_empty[stage][o]: o = 0 the streamed operand A_t (Q_i in dkdv,
// K_j in dq), o = 1 the operand B_t (dO_i in dkdv, V_j in dq).
struct BwdBars {
  uint64_t fix_full, ring_full[kMaxStages][2], ring_empty[kMaxStages][2];
  uint64_t x_full, y_full[2], x_free, p_ready, ds_ready, done, drain;   // y_full[b]: Y buffer b
  uint32_t tmem_base;
  Abort abort;
};
static_assert(sizeof(BwdBars) <= 256, "barrier block");

// Shared prologue: barriers, TMEM allocation (512 columns).
__device__ __forceinline__ void bwd_setup(BwdBars* bars, int warp) {
  if (threadIdx.x == 0) {
    mbar_init(&bars->fix_full, 1);
    for (int s = 0; s < kMaxStages; ++s)
      for (int o = 0; o < 2; ++o) {
        mbar_init(&bars->ring_full[s][o], 1);
        mbar_init(&bars->ring_empty[s][o], 1);
      }
    mbar_init(&bars->x_full, 1);
    mbar_init(&bars->y_full[0], 1);
    mbar_init(&bars->y_full[1], 1);
    mbar_init(&bars->x_free, kComputeWarps);     // one arrival per compute warp
    mbar_init(&bars->p_ready, kComputeWarps);    // dkdv: P^T stored
    mbar_init(&bars->ds_ready, kComputeWarps);
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

// Producer: the two fixed tiles once (rows frow .. frow + 127), then `n`
// streamed tiles of rows row0 + t * 128 of maps ma (operand A_t) and mb (B_t).
template <int D>
__device__ void bwd_produce(uint8_t* sm, BwdBars* bars, const CUtensorMap* f0, const CUtensorMap* f1,
                            int frow, const CUtensorMap* ma, const CUtensorMap* mb, int row0, int n,
                            int bh, volatile Abort* ab, int* err) {
  using Lay = BwdLayout<D>;
  constexpr int SUB = Lay::SUB, NSTA = Lay::NSTA, NSTB = Lay::NSTB;
  mbar_expect_tx(&bars->fix_full, 2 * Lay::OPB);
  for (int c = 0; c < SUB; ++c) {
    tma_load_3d(sm + Lay::FIX0 + c * kSub, f0, &bars->fix_full, 64 * c, frow, bh);
    tma_load_3d(sm + Lay::FIX1 + c * kSub, f1, &bars->fix_full, 64 * c, frow, bh);
  }
  int issued = 0;                        // (tile, operand) loads issued, in order
  for (int t = 0; t < n; ++t) {
    bool go = true;
    for (int o = 0; o < 2; ++o) {
      const int nst = o ? NSTB : NSTA, st = t % nst;
      if (t >= nst && !mbar_wait(&bars->ring_empty[st][o], ((t / nst) - 1) & 1, ab, err, 11)) {
        go = false;
        break;
      }
      uint64_t* full = &bars->ring_full[st][o];
      uint8_t* dst = sm + (o ? Lay::RB : Lay::RA) + st * Lay::OPB;
      mbar_expect_tx(full, Lay::OPB);
      for (int c = 0; c < SUB; ++c)
        tma_load_3d(dst + c * kSub, o ? mb : ma, full, 64 * c, row0 + t * kT, bh);
      issued = 2 * t + o + 1;
    }
    if (!go) break;
  }
  if (ab->flag) {
    // wind-down: let the copies still in flight land before the CTA exits
    Abort none{0};
    mbar_wait(&bars->fix_full, 0, &none, nullptr, 0);
    // the latest load into each stage of each operand
    const int na = (issued + 1) / 2, nb = issued / 2;   // tiles of A_t / B_t issued
    for (int tt = na - NSTA < 0 ? 0 : na - NSTA; tt < na; ++tt)
      mbar_wait(&bars->ring_full[tt % NSTA][0], (tt / NSTA) & 1, &none, nullptr, 0);
    for (int tt = nb - NSTB < 0 ? 0 : nb - NSTB; tt < nb; ++tt)
      mbar_wait(&bars->ring_full[tt % NSTB][1], (tt / NSTB) & 1, &none, nullptr, 0);
  }
}

// MMA issuer shared by both kernels. For streamed tile t:
//   X(t) = F0 * A_t^T -> cols 0..127,  Y(t) = F1 * B_t^T -> Y buffer of t
//   (dkdv: cols 128..255; dq: buffer t & 1 at 128 + 128 (t & 1)),
//   the accumulating MMAs, A operand from that Y buffer (fp16 pairs; chunk
//   c = 32 columns of the tile, its first 16 packed columns hold P^T / dS_hi,
//   the next 16 dS^T / dS_lo):
//     dkdv (TWO_ACC): dV += P^T B_t once P^T is stored (p_ready), then
//                     dK += dS^T A_t once dS^T is (ds_ready)
//     dq:             dQ += dS_hi A_t + dS_lo A_t
// Issue order: X(0), Y(0), then per t: dkdv X(t+1), dV(t), dK(t), Y(t+1);
// dq X(t+1), Y(t+1), acc(t).
// Run by the whole (converged) MMA warp: every lane takes the same waits and
// branches, one elected lane issues the MMAs and commits. Shared-memory
// descriptors are built once per operand and advanced by constant offsets
// (the start address, in 16-byte units, sits in the low 14 bits).
template <int D, bool TWO_ACC>
__device__ void bwd_mma(uint8_t* sm, BwdBars* bars, uint32_t tbase, int n, volatile Abort* ab, int* err) {
  using Lay = BwdLayout<D>;
  constexpr int NSTA = Lay::NSTA, NSTB = Lay::NSTB;
  constexpr uint32_t IDX = idesc_f16(kT, kT, false);      // scores: both operands K-major
  constexpr uint32_t IDACC = idesc_f16(kT, D, true);      // accumulate: B MN-major
  constexpr uint32_t OPB16 = Lay::OPB >> 4;
  const bool leader = elect_one();
  const uint32_t sbase = smem_u32(sm);
  const uint64_t dF0 = sdesc_sw128(sbase + Lay::FIX0, 16, 1024), dF1 = sdesc_sw128(sbase + Lay::FIX1, 16, 1024);
  const uint64_t dA = sdesc_sw128(sbase + Lay::RA, 16, 1024), dB = sdesc_sw128(sbase + Lay::RB, 16, 1024);
  const uint64_t dAm = sdesc_sw128(sbase + Lay::RA, kSub, 1024), dBm = sdesc_sw128(sbase + Lay::RB, kSub, 1024);
  // K slice kk of a K-major tile: 16 columns = 32 bytes within a 64-column slab
  auto kofs = [](int kk) -> uint64_t { return (uint64_t)((kk >> 2) * (kSub >> 4) + (kk & 3) * 2); };
  const uint32_t tX = tbase;
  auto tY = [&](int t) -> uint32_t { return tbase + kColY + (TWO_ACC ? 0u : 128u * (t & 1)); };
  const uint32_t tAcc0 = tbase + col_acc(TWO_ACC), tAcc1 = tAcc0 + (TWO_ACC ? D : 0);
  auto issue_x = [&](int t) {
    const uint64_t b0 = dA + (uint64_t)((t % NSTA) * OPB16);
    if (leader) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) umma_f16(tX, dF0 + kofs(kk), b0 + kofs(kk), IDX, kk > 0 ? 1u : 0u);
      umma_commit(&bars->x_full);
    }
  };
  auto issue_y = [&](int t) {
    const uint64_t b0 = dB + (uint64_t)((t % NSTB) * OPB16);
    const uint32_t y = tY(t);
    if (leader) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) umma_f16(y, dF1 + kofs(kk), b0 + kofs(kk), IDX, kk > 0 ? 1u : 0u);
      umma_commit(&bars->y_full[TWO_ACC ? 0 : (t & 1)]);
      if (!TWO_ACC) umma_commit(&bars->ring_empty[t % NSTB][1]);   // dq: V_j has no other reader
    }
  };
  // accumulating MMAs: 16-row slice kk of the streamed tiles (MN-major
  // descriptor + kk * 2048 bytes) and its packed operand columns in the Y
  // buffer at acol(kk)
  auto acol = [](int kk) -> uint32_t { return 32 * (kk >> 1) + 8 * (kk & 1); };
  auto issue_acc = [&](int t) {
    const uint64_t bA = dAm + (uint64_t)((t % NSTA) * OPB16);
    const uint32_t y = tY(t);
    if (!leader) return;
    if (TWO_ACC) {
      // dK(t); dV(t) went ahead in issue_dv
#pragma unroll
      for (int kk = 0; kk < kT / 16; ++kk)
        umma_f16_ts(tAcc1, y + acol(kk) + 16, bA + kk * 128, IDACC, (t > 0 || kk > 0) ? 1u : 0u);
      umma_commit(&bars->ring_empty[t % NSTA][0]);
    } else {
#pragma unroll
      for (int kk = 0; kk < kT / 16; ++kk) {
        umma_f16_ts(tAcc0, y + acol(kk), bA + kk * 128, IDACC, (t > 0 || kk > 0) ? 1u : 0u);
        umma_f16_ts(tAcc0, y + acol(kk) + 16, bA + kk * 128, IDACC, 1u);
      }
      umma_commit(&bars->ring_empty[t % NSTA][0]);
    }
  };
  auto issue_dv = [&](int t) {
    const uint64_t bB = dBm + (uint64_t)((t % NSTB) * OPB16);
    const uint32_t y = tY(t);
    if (!leader) return;
#pragma unroll
    for (int kk = 0; kk < kT / 16; ++kk)
      umma_f16_ts(tAcc0, y + acol(kk), bB + kk * 128, IDACC, (t > 0 || kk > 0) ? 1u : 0u);
    umma_commit(&bars->ring_empty[t % NSTB][1]);
  };
  auto wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, ab, err, site));
  };
  auto ring_wait = [&](int t, int o) -> bool {
    const int nst = o ? NSTB : NSTA;
    return wait(&bars->ring_full[t % nst][o], (t / nst) & 1, 13);
  };
  bool ok = wait(&bars->fix_full, 0, 12) && ring_wait(0, 0);
  if (ok) {
    tc_fence_after();
    issue_x(0);
    ok = ring_wait(0, 1);
  }
  if (ok) issue_y(0);
  for (int t = 0; ok && t < n; ++t) {
    if (t + 1 < n) {
      if (!ring_wait(t + 1, 0) || !wait(&bars->x_free, t & 1, 14)) { ok = false; break; }
      tc_fence_after();
      issue_x(t + 1);
      if (!TWO_ACC) {
        // dq: Y(t+1) overwrites the buffer that acc(t-1), issued earlier, read
        if (!ring_wait(t + 1, 1)) { ok = false; break; }
        issue_y(t + 1);
      }
    }
    if (TWO_ACC) {
      if (!wait(&bars->p_ready, t & 1, 22)) { ok = false; break; }
      tc_fence_after();
      issue_dv(t);
    }
    if (!wait(&bars->ds_ready, t & 1, 15)) { ok = false; break; }
    tc_fence_after();
    issue_acc(t);
    if (TWO_ACC && t + 1 < n) {
      if (!ring_wait(t + 1, 1)) { ok = false; break; }
      issue_y(t + 1);
    }
  }
  if (leader) {
    if (ok) umma_commit(&bars->done);
    umma_commit(&bars->drain);
  }
  __syncwarp();
  Abort none{0};
  mbar_wait(&bars->drain, 0, &none, nullptr, 0);
}

__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a), __uint_as_float(b));
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// 32 columns of this thread's key row (dK/dV kernel): P^T = 2^(S^T c2 - lse2)
// in place, two columns per packed fp32 instruction. nl2 holds -lse2 of the
// 32 query columns (the same for every lane: broadcast reads). MASK: columns
// outside [vlo, vhi] (causal diagonal, rows past S) get P = 0.
template <bool MASK>
__device__ __forceinline__ void p_chunk_t(uint32_t (&s)[32], const float* nl2, float c2, int col0, int vlo,
                                          int vhi) {
  const float2 cc = make_float2(c2, c2);
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 a = *reinterpret_cast<const float4*>(nl2 + e);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float2 x = __ffma2_rn(f2(s[e + u], s[e + u + 1]), cc, u ? make_float2(a.z, a.w) : make_float2(a.x, a.y));
      float p0 = ex2(x.x), p1 = ex2(x.y);
      if (MASK) {
        const int col = col0 + e + u;
        if (col < vlo || col > vhi) p0 = 0.f;
        if (col + 1 < vlo || col + 1 > vhi) p1 = 0.f;
      }
      s[e + u] = __float_as_uint(p0);
      s[e + u + 1] = __float_as_uint(p1);
    }
  }
}

// P^T of 32 columns as fp16 pairs.
__device__ __forceinline__ void pack_h2(const uint32_t (&p)[32], uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) pk[e >> 1] = h2_bits(__float22half2_rn(f2(p[e], p[e + 1])));
}

// dS^T = P^T o (dP^T - delta) for 32 columns, as fp16 pairs. ndl holds -delta
// of the 32 query columns.
__device__ __forceinline__ void ds_chunk_t(const uint32_t (&p)[32], const uint32_t (&dp)[32], const float* ndl,
                                           uint32_t (&dk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 b = *reinterpret_cast<const float4*>(ndl + e);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float2 pp = f2(p[e + u], p[e + u + 1]);
      const float2 d = __fadd2_rn(f2(dp[e + u], dp[e + u + 1]), u ? make_float2(b.z, b.w) : make_float2(b.x, b.y));
      dk[(e + u) >> 1] = h2_bits(__float22half2_rn(__fmul2_rn(pp, d)));
    }
  }
}

// 32 columns of this thread's query row (dQ kernel): P = 2^(S c2 - lse2) in
// place. nl2 = -lse2 of the row. MASK: key columns past vhi get P = 0.
template <bool MASK>
__device__ __forceinline__ void p_chunk(uint32_t (&s)[32], float nl2, float c2, int col0, int vhi) {
  const float2 cc = make_float2(c2, c2), nl = make_float2(nl2, nl2);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float2 x = __ffma2_rn(f2(s[e], s[e + 1]), cc, nl);
    float p0 = ex2(x.x), p1 = ex2(x.y);
    if (MASK) {
      if (col0 + e > vhi) p0 = 0.f;
      if (col0 + e + 1 > vhi) p1 = 0.f;
    }
    s[e] = __float_as_uint(p0);
    s[e + 1] = __float_as_uint(p1);
  }
}

// dS = P o (dP - delta) for 32 columns, as an fp16 head and an fp16 remainder.
__device__ __forceinline__ void ds_chunk(const uint32_t (&p)[32], const uint32_t (&dp)[32], float ndl,
                                         uint32_t (&hi)[16], uint32_t (&lo)[16]) {
  const float2 nd = make_float2(ndl, ndl), m1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float2 ds = __fmul2_rn(f2(p[e], p[e + 1]), __fadd2_rn(f2(dp[e], dp[e + 1]), nd));
    const __half2 h = __float22half2_rn(ds);
    const float2 r = __ffma2_rn(__half22float2(h), m1, ds);     // ds - hi, exact
    hi[e >> 1] = h2_bits(h);
    lo[e >> 1] = h2_bits(__float22half2_rn(r));
  }
}

// ---------------------------------------------------------------- dK, dV
// SEG: the queries are one per-(b, h) segment of the rows (seg); without it,
// every row is a query (q0 = 0, nq = S at compile time).
template <int D, bool SEG>
__global__ void __launch_bounds__(kThreads, 1)
k_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
              const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
              const float* __restrict__ lse, const float* __restrict__ delta, float* __restrict__ dks,
              float* __restrict__ dvs, int S, float c2, float scale, const int* __restrict__ seg,
              const uint32_t* __restrict__ amax, int* err) {
  using Lay = BwdLayout<D>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem_raw);
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + Lay::HEAD + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x;            // key tile (rows j*128 ..); small j has the most query tiles
  const int bh = blockIdx.y;
  // query rows [q0, q0 + nq) of this (b, h) (all S rows, or one rank's segment)
  const int q0 = SEG ? seg[2 * bh] : 0, nq = SEG ? seg[2 * bh + 1] : S;
  const int ntq = (nq + kT - 1) / kT;
  const int i0 = max(0, j * kT - q0) / kT;   // first query tile with a row at or after key row j*128
  const int n = ntq - i0;                    // query tiles i = i0 .. ntq-1
  // operands q * 2^-eq, k * 2^-ek, v * 2^-ev (lh_gather) and dO * 2^-edo
  // (lh_scatter_bwd): scores carry 2^-(eq+ek), dP and delta 2^-(edo+ev),
  // dV 2^-edo, dK 2^-(edo+ev+eq); each is taken out where it is used
  const int BH = (int)gridDim.y;
  const int eq = scale_exp(amax[kScaleQ * BH + bh]), ek = scale_exp(amax[kScaleK * BH + bh]);
  const int ev = scale_exp(amax[kScaleV * BH + bh]), edo = scale_exp(amax[kScaleDO * BH + bh]);
  c2 *= pow2f(eq + ek);
  if (n <= 0) {
    // no query of this head reaches this key tile: its gradient rows are zero
    const size_t rows = (size_t)min(kT, S - j * kT);
    float4* a = reinterpret_cast<float4*>(dks + ((size_t)bh * S + (size_t)j * kT) * D);
    float4* b = reinterpret_cast<float4*>(dvs + ((size_t)bh * S + (size_t)j * kT) * D);
    for (size_t x = threadIdx.x; x < rows * D / 4; x += blockDim.x) {
      a[x] = make_float4(0.f, 0.f, 0.f, 0.f);
      b[x] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  bwd_setup(bars, warp);
  const uint32_t tbase = bars->tmem_base;
  volatile Abort* ab = &bars->abort;

  if (warp == 0) {
    if (lane == 0) bwd_produce<D>(sm, bars, &tk, &tv, j * kT, &tq, &tdo, q0 + i0 * kT, n, bh, ab, err);
  } else if (warp == 1) {
    bwd_mma<D, true>(sm, bars, tbase, n, ab, err);
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;                   // which 64 of the 128 columns
    const int m = quarter * 32 + lane;                  // key row within the tile / TMEM lane
    const int ctid = threadIdx.x - 64;                  // 0..255
    const uint32_t la = (uint32_t)(quarter * 32) << 16;
    const uint32_t cX = tbase + la + 64 * half, cY = cX + kColY;
    const int key = j * kT + m;
    float* vec = reinterpret_cast<float*>(smem_raw + 256);  // [2][128]: -lse2, -delta
    // this thread's share of a query tile's -lse2 / -delta (thread hid of the
    // half: column 64*half + (hid & 63)), fetched one tile ahead
    const int hid = ctid & 127;
    const float* vsrc = (hid < 64 ? lse : delta) + (size_t)bh * S;
    const float vmul = hid < 64 ? -1.4426950408889634f : -pow2f(-(edo + ev));
    auto fetch = [&](int i) -> float {
      const int q = i * kT + 64 * half + (hid & 63);    // within this head's query rows
      return q < nq ? vsrc[q0 + q] : 0.f;
    };
    float nxt = fetch(i0);
    bool ok = true;
    // this half's 64 query columns
    float* nl2 = vec + 64 * half;
    float* ndl = nl2 + 128;
    // every compute thread runs all n iterations (and their named barriers),
    // also after a wind-down, so no warp can be left waiting at a barrier
    for (int t = 0; t < n; ++t) {
      const int i = i0 + t;
      named_bar_sync(1 + half, kComputeThreads / 2);   // the half is done with tile t-1's vector
      (hid < 64 ? nl2 : ndl)[hid & 63] = nxt * vmul;
      named_bar_sync(1 + half, kComputeThreads / 2);
      if (t + 1 < n) nxt = fetch(i + 1);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->x_full, t & 1, ab, err, 16));
      if (!ok) continue;
      tc_fence_after();
      // S^T: this warp's 64 columns into registers, then X is released
      uint32_t p0[32], p1[32];
      tmem_ld32(cX, p0);
      tmem_ld32(cX + 32, p1);
      tmem_wait_ld_regs(p0);
      reg_fence32(p1);
      tc_fence_before();
      mbar_arrive_warp(&bars->x_free);
      const int vlo = max(0, key - q0 - i * kT);         // causal: query position >= key position
      const int vhi = min(kT - 1, nq - 1 - i * kT);      // last valid query column
      if (vlo > 0 || vhi < kT - 1) {
        p_chunk_t<true>(p0, nl2, c2, 64 * half, vlo, vhi);
        p_chunk_t<true>(p1, nl2 + 32, c2, 64 * half + 32, vlo, vhi);
      } else {
        p_chunk_t<false>(p0, nl2, c2, 0, 0, 0);
        p_chunk_t<false>(p1, nl2 + 32, c2, 0, 0, 0);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->y_full[0], t & 1, ab, err, 17));
      if (!ok) continue;
      tc_fence_after();
      // dP^T: both 32-column chunks, then fp16 pairs into the chunk's own
      // (already read) columns: P^T at +0..15 first, so that dV(t) runs while
      // dS^T is formed, then dS^T at +16..31
      uint32_t d0[32], d1[32], pk[16];
      tmem_ld32(cY, d0);
      tmem_ld32(cY + 32, d1);
      tmem_wait_ld_regs(d0);
      reg_fence32(d1);
      pack_h2(p0, pk);
      tmem_st16(cY, pk);
      pack_h2(p1, pk);
      tmem_st16(cY + 32, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(&bars->p_ready);
      ds_chunk_t(p0, d0, ndl, pk);
      tmem_st16(cY + 16, pk);
      ds_chunk_t(p1, d1, ndl + 32, pk);
      tmem_st16(cY + 48, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(&bars->ds_ready);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->done, 0, ab, err, 18))) {
      tc_fence_after();
      const float mv = pow2f(edo), mk = scale * pow2f(edo + ev + eq);
      float* ddv = dvs + ((size_t)bh * S + key) * D;
      float* ddk = dks + ((size_t)bh * S + key) * D;
#pragma unroll 1
      for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
        // the TMEM loads are warp-collective (.sync.aligned): every lane runs
        // them, rows past S included; only the stores are per-row
        uint32_t a[32], b[32];
        tmem_ld32(tbase + la + col_acc(true) + 32 * c, a);
        tmem_ld32(tbase + la + col_acc(true) + D + 32 * c, b);
        tmem_wait_ld();
        if (key < S) {
          bool fin = true;
#pragma unroll
          for (int e = 0; e < 32; ++e) fin &= fabsf(__uint_as_float(b[e])) < INFINITY;
          if (!fin) report_error(err, LH_ERR_DEVICE, 101);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            *reinterpret_cast<float4*>(ddv + 32 * c + e) =
                make_float4(__uint_as_float(a[e]) * mv, __uint_as_float(a[e + 1]) * mv,
                            __uint_as_float(a[e + 2]) * mv, __uint_as_float(a[e + 3]) * mv);
            *reinterpret_cast<float4*>(ddk + 32 * c + e) =
                make_float4(__uint_as_float(b[e]) * mk, __uint_as_float(b[e + 1]) * mk,
                            __uint_as_float(b[e + 2]) * mk, __uint_as_float(b[e + 3]) * mk);
          }
        }
      }
    }
  }
  bwd_teardown(tbase, warp);
}

// ---------------------------------------------------------------- dQ
template <int D, bool SEG>
__global__ void __launch_bounds__(kThreads, 1)
k_bwd_dq_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
            const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
            const float* __restrict__ lse, const float* __restrict__ delta, float* __restrict__ dqs,
            int S, float c2, float scale, const int* __restrict__ seg, const uint32_t* __restrict__ amax,
            int* err) {
  using Lay = BwdLayout<D>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem_raw);
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + Lay::HEAD + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int q0 = SEG ? seg[2 * bh] : 0, nq = SEG ? seg[2 * bh + 1] : S;
  const int ntq = (nq + kT - 1) / kT;
  const int i = ntq - 1 - (int)blockIdx.x;        // query tile; late tiles have the most key tiles
  if (i < 0) return;                              // whole CTA, before any set-up
  // key tiles up to the one holding the tile's last row, within the keys that exist
  const int n = min((q0 + i * kT + kT - 1) / kT + 1, (q0 + nq + kT - 1) / kT);
  // operand exponents as in the dK/dV kernel: dQ carries 2^-(edo+ev+ek)
  const int BH = (int)gridDim.y;
  const int eq = scale_exp(amax[kScaleQ * BH + bh]), ek = scale_exp(amax[kScaleK * BH + bh]);
  const int ev = scale_exp(amax[kScaleV * BH + bh]), edo = scale_exp(amax[kScaleDO * BH + bh]);
  c2 *= pow2f(eq + ek);
  bwd_setup(bars, warp);
  const uint32_t tbase = bars->tmem_base;
  volatile Abort* ab = &bars->abort;

  if (warp == 0) {
    if (lane == 0) bwd_produce<D>(sm, bars, &tq, &tdo, q0 + i * kT, &tk, &tv, 0, n, bh, ab, err);
  } else if (warp == 1) {
    bwd_mma<D, false>(sm, bars, tbase, n, ab, err);
  } else {
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;             // which 64 of the 128 columns
    const int r = quarter * 32 + lane;            // query row within the tile / TMEM lane
    const uint32_t la = (uint32_t)(quarter * 32) << 16;
    const uint32_t cX = tbase + la + 64 * half;
    const int q = i * kT + r;                      // within this head's query rows
    const float nl2 = q < nq ? lse[(size_t)bh * S + q0 + q] * -1.4426950408889634f : 0.f;
    const float ndl = q < nq ? -delta[(size_t)bh * S + q0 + q] * pow2f(-(edo + ev)) : 0.f;
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->x_full, jj & 1, ab, err, 19))) { ok = false; break; }
      tc_fence_after();
      uint32_t p0[32], p1[32];
      tmem_ld32(cX, p0);
      tmem_ld32(cX + 32, p1);
      tmem_wait_ld_regs(p0);
      reg_fence32(p1);
      tc_fence_before();
      mbar_arrive_warp(&bars->x_free);
      const int klim = min(q0 + q - jj * kT, kT - 1);   // last valid key column (causal)
      if (klim < kT - 1) {
        p_chunk<true>(p0, nl2, c2, 64 * half, klim);
        p_chunk<true>(p1, nl2, c2, 64 * half + 32, klim);
      } else {
        p_chunk<false>(p0, nl2, c2, 0, 0);
        p_chunk<false>(p1, nl2, c2, 0, 0);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->y_full[jj & 1], (jj >> 1) & 1, ab, err, 20))) { ok = false; break; }
      tc_fence_after();
      const uint32_t cY = cX + kColY + 128 * (jj & 1);
      // dP: both chunks, then head / remainder into the chunk's own columns
      uint32_t d0[32], d1[32], hi[16], lo[16];
      tmem_ld32(cY, d0);
      tmem_ld32(cY + 32, d1);
      tmem_wait_ld_regs(d0);
      reg_fence32(d1);
      ds_chunk(p0, d0, ndl, hi, lo);
      tmem_st16(cY, hi);
      tmem_st16(cY + 16, lo);
      ds_chunk(p1, d1, ndl, hi, lo);
      tmem_st16(cY + 32, hi);
      tmem_st16(cY + 48, lo);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(&bars->ds_ready);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->done, 0, ab, err, 21))) {
      tc_fence_after();
      float* dst = dqs + ((size_t)bh * S + q0 + q) * D;
      const float mq = scale * pow2f(edo + ev + ek);
#pragma unroll 1
      for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
        uint32_t a[32];
        tmem_ld32(tbase + la + col_acc(false) + 32 * c, a);
        tmem_wait_ld();
        if (q < nq) {
          bool fin = true;
#pragma unroll
          for (int e = 0; e < 32; ++e) fin &= fabsf(__uint_as_float(a[e])) < INFINITY;
          if (!fin) report_error(err, LH_ERR_DEVICE, 101);
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + e) =
                make_float4(__uint_as_float(a[e]) * mq, __uint_as_float(a[e + 1]) * mq,
                            __uint_as_float(a[e + 2]) * mq, __uint_as_float(a[e + 3]) * mq);
        }
      }
    }
  }
  bwd_teardown(tbase, warp);
}

template <int D>
cudaError_t bwd_tc_t(const Geom& g, const void* qs, const void* ks, const void* vs, const void* dos,
                     const float* lse, const float* delta, float* dqs, float* dks, float* dvs, const int* seg,
                     const uint32_t* amax, int* err, cudaStream_t s) {
  CUtensorMap tq, tk, tv, tdo;
  const int BH = g.B * g.H;
  if (!make_tmap_16(&tq, qs, D, g.S, BH, true, kT) || !make_tmap_16(&tk, ks, D, g.S, BH, true, kT) ||
      !make_tmap_16(&tv, vs, D, g.S, BH, true, kT) || !make_tmap_16(&tdo, dos, D, g.S, BH, true, kT))
    return cudaErrorInvalidValue;
  const int smem = BwdLayout<D>::BYTES, smem_q = smem;
  auto dkdv = seg ? k_bwd_dkdv_tc<D, true> : k_bwd_dkdv_tc<D, false>;
  auto dq = seg ? k_bwd_dq_tc<D, true> : k_bwd_dq_tc<D, false>;
  cudaError_t e = cudaFuncSetAttribute(dkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(dq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
  if (e != cudaSuccess) return e;
  const float scale = (float)(1.0 / sqrt((double)D));
  const float c2 = (float)(1.4426950408889634 / sqrt((double)D));
  dim3 grid((g.S + kT - 1) / kT, BH);
  dkdv<<<grid, kThreads, smem, s>>>(tk, tv, tq, tdo, lse, delta, dks, dvs, g.S, c2, scale, seg, amax, err);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dq<<<grid, kThreads, smem_q, s>>>(tq, tdo, tk, tv, lse, delta, dqs, g.S, c2, scale, seg, amax, err);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

// seg: nullptr (every row of the sub-sequence is a query) or [B*H][2] device
// int32 (first query row, number of query rows) per (b, h); then dks / dvs
// hold every key row's gradient from those queries alone (zero rows where no
// query reaches), and dqs only the segment's rows.
cudaError_t launch_attn_bwd_tc(const Geom& g, const void* qs, const void* ks, const void* vs,
                               const void* dos, const float* lse, const float* delta, float* dqs,
                               float* dks, float* dvs, const int* seg, const uint32_t* amax, int* err,
                               cudaStream_t s) {
  return g.D == 64 ? bwd_tc_t<64>(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, seg, amax, err, s)
                   : bwd_tc_t<128>(g, qs, ks, vs, dos, lse, delta, dqs, dks, dvs, seg, amax, err, s);
}

}  // namespace lh
