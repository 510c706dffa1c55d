// Causal flash attention on the sub-sequence with tcgen05 tensor cores (fp16
// operands, fp32 accumulate), forward pass.
//
// "Long Context Pre-Training with Lighthouse Attention", Eq. (1) and §3.1
// stage (iii): the gathered sub-sequence is a dense causal sequence, so this is
// plain causal attention softmax(Q K^T / sqrt(d) + M) V over S entries. For
// bf16 I/O the sub-sequence arrives as exact fp16 values (lh_gather), and P
// enters the P V product as fp16: 11 significant bits instead of bf16's 8
// keep the output within the stated tolerance (with bf16 P, errors of 1.5e-2
// in the attention output were measured on scaled inputs).
//
// One CTA per (b, h, pair of 128-row query tiles A = 2m, B = 2m+1); heavy
// (late) pairs are scheduled first. Warp roles (320 threads):
//   warp 0    TMA producer: Q_A and Q_B once, then K and V tiles of 128 rows,
//             each through its own 2-stage ring (128-byte swizzle, no
//             multicast): K_j is released once both score MMAs have read it.
//   warp 1    allocates all 512 TMEM columns (S_A, O_A, S_B, O_B, 128 each);
//             lane 0 issues every tcgen05.mma, per key tile j:
//               PV_A(j), S_A(j+1), PV_B(j), S_B(j+1)
//             so one tile's softmax runs while the tensor core works on the
//             other tile (about 1.5 tiles of MMA time for 1 tile of softmax).
//   warps 2-5 softmax of tile A, warps 6-9 of tile B; one thread per query row
//             (= TMEM lane): scores from TMEM, causal mask on the diagonal
//             tile, online softmax in the exp2 domain with a lazily updated
//             running max (O is rescaled in TMEM only when the max grows by
//             more than 2^8); P is split into an fp16 head and an fp16
//             remainder written into the score columns (each 32-column chunk
//             holds its own 16 head and 16 remainder columns), and
//             O += P_hi V + P_lo V as TMEM-operand MMAs, so O carries P to
//             about 2^-22 instead of fp16's 2^-12 (the backward's
//             delta = <dO, O> needs that: at 512K context with outlier tokens
//             the fp16-only O put delta off by 0.07); finally O / l and lse.
// Reuse of TMEM columns is ordered by the MMA stream: S_t(j+1) is issued after
// PV_t(j), and tcgen05.mma ops issued by one thread execute in order, so once
// S_t(j+1) is complete, PV_t(j) has finished reading P_t(j) and O_t is current.
// Every mbarrier wait is bounded (tc::mbar_wait): on timeout the kernel records
// LH_ERR_TIMEOUT, drains its outstanding copies and MMAs, frees TMEM, returns.
#include <cudaTypedefs.h>

#include <cstdlib>

#include "tc_ptx.cuh"

namespace lh {
namespace {

using namespace tc;

constexpr int kBM = 128;       // query rows per tile
constexpr int kBN = 128;       // key rows per tile
constexpr int kSub = 128 * 64 * 2;   // one 128-row x 64-column 16-bit swizzle tile (16 KB)
constexpr float kLn2f = 0.6931471805599453f;
constexpr int kFwdThreads = 320;

// Barriers first, then the swizzled tiles from the next 1024-byte boundary.
template <int D>
struct FwdLayout {
  static constexpr int SUB = D / 64;
  static constexpr int OPB = SUB * kSub;   // one 128-row operand tile
  static constexpr int Q = 0;              // Q_A, Q_B
  static constexpr int K = Q + 2 * OPB;    // 2 stages
  static constexpr int V = K + 2 * OPB;    // 2 stages
  static constexpr int TILES = V + 2 * OPB;
  static constexpr int HEAD = 256;
  static constexpr int BYTES = HEAD + 1024 + TILES;
  static_assert(BYTES <= 227 * 1024, "shared memory");
};

// Per query tile t (0 = A, 1 = B): s_full (score MMA done), p_full (one
// arrival per softmax warp), o_done (P V MMA done).
struct FwdBars {
  uint64_t q_full, k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], o_done[2], drain;
  uint32_t tmem_base;
  Abort abort;
};
static_assert(sizeof(FwdBars) <= 256, "barrier block");

// SEG: the queries are one per-(b, h) segment of the rows (seg); without it,
// every row is a query (q0 = 0, nq = S at compile time).
template <int D, bool SEG>
__global__ void __launch_bounds__(kFwdThreads, 1)
k_attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, float* __restrict__ os, float* __restrict__ lse,
              int S, float c2, const int* __restrict__ seg, const uint32_t* __restrict__ scale, int* err) {
  using Lay = FwdLayout<D>;
  constexpr int SUB = Lay::SUB;
  constexpr uint32_t IDS = idesc_f16(kBM, kBN, false);    // S = Q K^T, both K-major
  constexpr uint32_t IDO = idesc_f16(kBM, D, true);       // O = P V, V MN-major
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem_raw);
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + Lay::HEAD + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(sm);

  // Query rows of this (b, h): rows [q0, q0 + nq) of qs attend to key rows
  // [0, q0 + nq) of ks / vs (the whole sub-sequence, or one rank's segment of
  // it in the sequence-sharded path, `seg` = (q0, nq) per (b, h)).
  const int bh = blockIdx.y;
  const int q0 = SEG ? seg[2 * bh] : 0, nq = SEG ? seg[2 * bh + 1] : S;
  const int ntiles = (nq + kBM - 1) / kBM;
  const int mp = (ntiles + 1) / 2 - 1 - (int)blockIdx.x;     // heavy (late) pairs first
  if (mp < 0) return;                                          // whole CTA, before any set-up
  const int itA = 2 * mp, itB = 2 * mp + 1;
  const bool hasB = itB < ntiles;
  // key tiles up to the one holding the tile's last row, within the keys that exist
  const int nk_end = (q0 + nq + kBN - 1) / kBN;
  const int nkvA = min((q0 + itA * kBM + kBM - 1) / kBN + 1, nk_end);
  const int nkvB = hasB ? min((q0 + itB * kBM + kBM - 1) / kBN + 1, nk_end) : 0;
  const int nkv = hasB ? nkvB : nkvA;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the operands are q * 2^-eq, k * 2^-ek, v * 2^-ev (lh_gather): scores carry
  // 2^-(eq+ek), taken out in the softmax scale, and O carries 2^-ev
  const int BH = (int)gridDim.y;
  const int eq = scale_exp(scale[kScaleQ * BH + bh]), ek = scale_exp(scale[kScaleK * BH + bh]);
  const int ev = scale_exp(scale[kScaleV * BH + bh]);
  c2 *= pow2f(eq + ek);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 4);     // one arrival per softmax warp of the tile
      mbar_init(&bars->o_done[s], 1);
    }
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
  const uint32_t tbase = bars->tmem_base;
  volatile Abort* ab = &bars->abort;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer
      int ik = 0, iv = 0;            // K / V tiles issued
      mbar_expect_tx(&bars->q_full, (hasB ? 2 : 1) * Lay::OPB);
      for (int c = 0; c < SUB; ++c) {
        tma_load_3d(sm + Lay::Q + c * kSub, &tq, &bars->q_full, 64 * c, q0 + itA * kBM, bh);
        if (hasB) tma_load_3d(sm + Lay::Q + Lay::OPB + c * kSub, &tq, &bars->q_full, 64 * c, q0 + itB * kBM, bh);
      }
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(&bars->k_empty[st], ((j >> 1) - 1) & 1, ab, err, 1)) break;
        mbar_expect_tx(&bars->k_full[st], Lay::OPB);
        for (int c = 0; c < SUB; ++c)
          tma_load_3d(sm + Lay::K + st * Lay::OPB + c * kSub, &tk, &bars->k_full[st], 64 * c, j * kBN, bh);
        ik = j + 1;
        if (j >= 2 && !mbar_wait(&bars->v_empty[st], ((j >> 1) - 1) & 1, ab, err, 1)) break;
        mbar_expect_tx(&bars->v_full[st], Lay::OPB);
        for (int c = 0; c < SUB; ++c)
          tma_load_3d(sm + Lay::V + st * Lay::OPB + c * kSub, &tv, &bars->v_full[st], 64 * c, j * kBN, bh);
        iv = j + 1;
      }
      if (ab->flag) {
        // wind-down: let the copies still in flight land before the CTA exits
        Abort none{0};
        mbar_wait(&bars->q_full, 0, &none, nullptr, 0);
        for (int j = ik - 2 < 0 ? 0 : ik - 2; j < ik; ++j)
          mbar_wait(&bars->k_full[j & 1], (j >> 1) & 1, &none, nullptr, 0);
        for (int j = iv - 2 < 0 ? 0 : iv - 2; j < iv; ++j)
          mbar_wait(&bars->v_full[j & 1], (j >> 1) & 1, &none, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole (converged) warp takes the same
    // waits and branches, one elected lane issues; shared-memory descriptors
    // are built once per operand and advanced by constant offsets (the start
    // address, in 16-byte units, sits in the low 14 bits)
    const bool leader = elect_one();
    constexpr uint32_t OPB16 = Lay::OPB >> 4;
    const uint64_t dQ = sdesc_sw128(sbase + Lay::Q, 16, 1024), dK = sdesc_sw128(sbase + Lay::K, 16, 1024);
    const uint64_t dV = sdesc_sw128(sbase + Lay::V, kSub, 1024);
    auto kofs = [](int kk) -> uint64_t { return (uint64_t)((kk >> 2) * (kSub >> 4) + (kk & 3) * 2); };
    auto issue_s = [&](int t, int j) {       // S_t = Q_t K_j^T
      const uint64_t a0 = dQ + (uint64_t)(t * OPB16), b0 = dK + (uint64_t)((j & 1) * OPB16);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16(tbase + 256 * t, a0 + kofs(kk), b0 + kofs(kk), IDS, kk > 0 ? 1u : 0u);
        umma_commit(&bars->s_full[t]);
      }
    };
    auto issue_pv = [&](int t, int j) {      // O_t += P_hi V_j + P_lo V_j
      const uint64_t b0 = dV + (uint64_t)((j & 1) * OPB16);
      const uint32_t tS = tbase + 256 * t, tO = tS + 128;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t acol = 32 * (kk >> 1) + 8 * (kk & 1);
          umma_f16_ts(tO, tS + acol, b0 + kk * 128, IDO, (j > 0 || kk > 0) ? 1u : 0u);
          umma_f16_ts(tO, tS + acol + 16, b0 + kk * 128, IDO, 1u);
        }
        umma_commit(&bars->o_done[t]);
      }
    };
    auto wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, ab, err, site));
    };
    bool ok = wait(&bars->q_full, 0, 2) && wait(&bars->k_full[0], 0, 3);
    if (ok) {
      tc_fence_after();
      issue_s(0, 0);
      if (hasB) issue_s(1, 0);
      if (leader) umma_commit(&bars->k_empty[0]);
    }
    for (int j = 0; ok && j < nkv; ++j) {
      if (!wait(&bars->v_full[j & 1], (j >> 1) & 1, 4)) { ok = false; break; }
      bool kwait = false;
      auto k_next = [&]() -> bool {
        if (kwait) return true;
        kwait = true;
        return wait(&bars->k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, 3);
      };
      if (j < nkvA) {
        if (!wait(&bars->p_full[0], j & 1, 5)) { ok = false; break; }
        tc_fence_after();
        issue_pv(0, j);
        if (j + 1 < nkvA) {
          if (!k_next()) { ok = false; break; }
          tc_fence_after();
          issue_s(0, j + 1);
        }
      }
      if (hasB) {
        if (!wait(&bars->p_full[1], j & 1, 5)) { ok = false; break; }
        tc_fence_after();
        issue_pv(1, j);
        if (j + 1 < nkvB) {
          if (!k_next()) { ok = false; break; }
          tc_fence_after();
          issue_s(1, j + 1);
        }
      }
      if (leader) {
        umma_commit(&bars->v_empty[j & 1]);
        if (j + 1 < nkv) umma_commit(&bars->k_empty[(j + 1) & 1]);
      }
    }
    // wait until every MMA issued here has finished before TMEM is released
    if (leader) umma_commit(&bars->drain);
    __syncwarp();
    Abort none{0};
    mbar_wait(&bars->drain, 0, &none, nullptr, 0);
  } else {
    // ---------------- softmax: one thread per query row / TMEM lane of tile t
    const int t = (warp - 2) >> 2;
    const int it = t ? itB : itA;
    if (t == 0 || hasB) {
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;
      const uint32_t la = (uint32_t)(quarter * 32) << 16;
      const uint32_t cS = tbase + la + 256 * t, cO = cS + 128;
      const int q_row = it * kBM + r;                  // within this head's query rows
      const int nk = t ? nkvB : nkvA;
      float m_run = 0.f, l_run = 0.f;
      bool ok = true;
      for (int j = 0; j < nk; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], j & 1, ab, err, 6))) { ok = false; break; }
        tc_fence_after();
        uint32_t s[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(cS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
        tmem_wait_ld_regs(*reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[64]));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[96]));
        // causal mask where the key tile reaches past this row's position; the
        // running max is taken on the raw scores (c2 > 0, and rounding is
        // monotone, so max(s) c2 = max(s c2)). Key tile 0 always keeps column 0,
        // so a row's running max is finite from its first tile on.
        const int lim = q0 + q_row - j * kBN;            // last valid column of this row
        if (__any_sync(0xffffffffu, lim < kBN - 1)) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim) s[c] = __float_as_uint(-INFINITY);
        }
        float mq[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          mq[g] = __uint_as_float(s[32 * g]);
#pragma unroll
          for (int c = 1; c < 31; c += 2)
            mq[g] = fmax3(mq[g], __uint_as_float(s[32 * g + c]), __uint_as_float(s[32 * g + c + 1]));
          mq[g] = fmaxf(mq[g], __uint_as_float(s[32 * g + 31]));
        }
        const float mx = fmax3(fmaxf(mq[0], mq[1]), mq[2], mq[3]) * c2;
        float m_new = m_run, alpha = 1.f;
        if (j == 0) {
          m_new = mx;
        } else if (mx > m_run + 8.f) {
          m_new = mx;
          alpha = ex2(m_run - m_new);
        }
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          // O_t is current: PV_t(j-1) finished before S_t(j) (same MMA stream)
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(cO + 16 * c, o);
            tmem_wait_ld_regs16(o);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st16(cO + 16 * c, o);
          }
        }
        // P = 2^(s c2 - m): head and remainder of each 32-column chunk into
        // that chunk's own score columns (+0..15 head, +16..31 remainder)
        const float2 cc = make_float2(c2, c2), nm = make_float2(-m_new, -m_new);
        const float2 m1 = make_float2(-1.f, -1.f);
        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {          // 8 columns: 4 head and 4 remainder pairs
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int e = 4 * g + u;
              const float2 x = __ffma2_rn(
                  make_float2(__uint_as_float(s[32 * c + 2 * e]), __uint_as_float(s[32 * c + 2 * e + 1])), cc, nm);
              const float2 pp = make_float2(ex2(x.x), ex2(x.y));
              acc[u & 1] = __fadd2_rn(acc[u & 1], pp);
              const __half2 h = __float22half2_rn(pp);
              const __half2 l = __float22half2_rn(__ffma2_rn(__half22float2(h), m1, pp));   // p - hi, exact
              hi[u] = *reinterpret_cast<const uint32_t*>(&h);
              lo[u] = *reinterpret_cast<const uint32_t*>(&l);
            }
            tmem_st4(cS + 32 * c + 4 * g, hi[0], hi[1], hi[2], hi[3]);
            tmem_st4(cS + 32 * c + 16 + 4 * g, lo[0], lo[1], lo[2], lo[3]);
          }
        }
        const float2 a01 = __fadd2_rn(acc[0], acc[1]);
        l_run = l_run * alpha + (a01.x + a01.y);
        m_run = m_new;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(&bars->p_full[t]);
      }
      // PV_t(nk-2) finished before S_t(nk-1), so o_done's phase nk-1 is the
      // only one left: its parity identifies it
      if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->o_done[t], (nk - 1) & 1, ab, err, 8))) {
        tc_fence_after();
        const float inv = pow2f(ev) / l_run;
        float* dst = os + ((size_t)bh * S + q0 + q_row) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(cO + 32 * c, o);
          tmem_wait_ld_regs(o);
          if (q_row < nq) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + 32 * c + e) =
                  make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                              __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
          }
        }
        if (q_row < nq) lse[(size_t)bh * S + q0 + q_row] = (m_run + log2f(l_run)) * kLn2f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tbase, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

}  // namespace

// [BH][S][D] 16-bit elements (bf16, or fp16 when `fp16`) viewed as a 3-D tensor
// (D, S, BH); boxes of 64 columns x `box_rows` rows, 128-byte swizzle.
bool make_tmap_16(CUtensorMap* m, const void* base, int D, int S, int BH, bool fp16, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static cudaError_t fwd_tc_t(const Geom& g, const void* qs, const void* ks, const void* vs, float* os,
                            float* lse, const int* seg, const uint32_t* scale, int* err, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  const int BH = g.B * g.H;
  if (!make_tmap_16(&tq, qs, D, g.S, BH, true, kBM) || !make_tmap_16(&tk, ks, D, g.S, BH, true, kBN) ||
      !make_tmap_16(&tv, vs, D, g.S, BH, true, kBN))
    return cudaErrorInvalidValue;
  const int smem = FwdLayout<D>::BYTES;
  auto kern = seg ? k_attn_fwd_tc<D, true> : k_attn_fwd_tc<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const float c2 = (float)(1.4426950408889634 / sqrt((double)D));
  const int ntiles = (g.S + kBM - 1) / kBM;
  dim3 grid((ntiles + 1) / 2, BH);
  kern<<<grid, kFwdThreads, smem, s>>>(tq, tk, tv, os, lse, g.S, c2, seg, scale, err);
  count_launch();
  return cudaGetLastError();
}

// seg: nullptr (every row of the sub-sequence is a query) or [B*H][2] device
// int32 (first query row, number of query rows) per (b, h).
// scale: [kScaleRows][B*H] largest magnitudes (the operands' power-of-two exponents).
cudaError_t launch_attn_fwd_tc(const Geom& g, const void* qs, const void* ks, const void* vs,
                               float* os, float* lse, const int* seg, const uint32_t* scale, int* err,
                               cudaStream_t s) {
  return g.D == 64 ? fwd_tc_t<64>(g, qs, ks, vs, os, lse, seg, scale, err, s)
                   : fwd_tc_t<128>(g, qs, ks, vs, os, lse, seg, scale, err, s);
}

}  // namespace lh
