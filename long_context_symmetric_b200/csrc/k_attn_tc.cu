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
// One CTA per (b, h, 128-row query tile); heavy (late) tiles are scheduled
// first. Warp roles (192 threads):
//   warp 0    TMA producer: the Q tile once, then K/V tiles of 128 rows into a
//             2-stage ring (128-byte swizzle, no multicast).
//   warp 1    allocates 512 TMEM columns; lane 0 issues every tcgen05.mma:
//             S_j = Q K_j^T into one of two TMEM score buffers, then
//             O += P_{j-1} V_{j-1} into the TMEM output accumulator, so the
//             tensor core computes S_{j+1} while the softmax warps work on S_j.
//   warps 2-5 softmax, one thread per query row (= TMEM lane): scores from
//             TMEM, causal mask on the diagonal tile, online softmax in the
//             exp2 domain with a lazily updated running max (the output is
//             rescaled in TMEM only when the max grows by more than 2^8); P is
//             split into an fp16 head (to shared memory, in the MMA's K-major
//             swizzled layout) and an fp16 remainder (to spare TMEM columns),
//             and O += P_hi V + P_lo V, so O carries P to about 2^-22 instead
//             of fp16's 2^-12 (the backward's delta = <dO, O> needs that: at
//             512K context with outlier tokens the fp16-only O put delta off
//             by 0.07); finally O / l and lse are written.
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
constexpr int kSub = 128 * 64 * 2;   // one 128-row x 64-column bf16 swizzle tile (16 KB)
constexpr int kStages = 2;
constexpr float kLn2f = 0.6931471805599453f;
constexpr uint32_t kPlo = 384;       // TMEM columns of the fp16 remainder of P (64 columns)

template <int D>
struct FwdLayout {
  static constexpr int SUB = D / 64;
  static constexpr int Q = 0;
  static constexpr int K = Q + SUB * kSub;
  static constexpr int V = K + kStages * SUB * kSub;
  static constexpr int P = V + kStages * SUB * kSub;
  static constexpr int BAR = P + 2 * kSub;
  // barriers + alignment slack; at least 120 KB so that one CTA (and its 512
  // TMEM columns) occupies an SM
  static constexpr int BYTES = (BAR + 256 + 1024) > 120 * 1024 ? (BAR + 256 + 1024) : 120 * 1024;
};

struct FwdBars {
  uint64_t q_full, kv_full[kStages], kv_empty[kStages], s_full[2], s_free[2], p_full, o_done, drain;
  uint32_t tmem_base;
  Abort abort;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
k_attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, float* __restrict__ os, float* __restrict__ lse,
              int S, float c2, int* err) {
  using Lay = FwdLayout<D>;
  constexpr int SUB = Lay::SUB;
  constexpr uint32_t IDS = idesc_f16(kBM, kBN, false);    // S = Q K^T, both K-major
  constexpr uint32_t IDO = idesc_f16(kBM, D, true);       // O = P V, V MN-major
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  FwdBars* bars = reinterpret_cast<FwdBars*>(sm + Lay::BAR);
  const uint32_t sbase = smem_u32(sm);

  const int ntiles = gridDim.x;
  const int it = ntiles - 1 - (int)blockIdx.x;
  const int bh = blockIdx.y;
  const int nkv = it + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], 4);      // one arrival per softmax warp
    }
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->o_done, 1);
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
      int issued = 0;
      mbar_expect_tx(&bars->q_full, SUB * kSub);
      for (int c = 0; c < SUB; ++c)
        tma_load_3d(sm + Lay::Q + c * kSub, &tq, &bars->q_full, 64 * c, it * kBM, bh);
      for (int j = 0; j < nkv; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(&bars->kv_empty[st], ((j / kStages) - 1) & 1, ab, err, 1)) break;
        mbar_expect_tx(&bars->kv_full[st], 2 * SUB * kSub);
        for (int c = 0; c < SUB; ++c)
          tma_load_3d(sm + Lay::K + (st * SUB + c) * kSub, &tk, &bars->kv_full[st], 64 * c, j * kBN, bh);
        for (int c = 0; c < SUB; ++c)
          tma_load_3d(sm + Lay::V + (st * SUB + c) * kSub, &tv, &bars->kv_full[st], 64 * c, j * kBN, bh);
        issued = j + 1;
      }
      if (ab->flag) {
        // wind-down: let the copies still in flight land before the CTA exits
        Abort none{0};
        mbar_wait(&bars->q_full, 0, &none, nullptr, 0);
        for (int j = issued - kStages < 0 ? 0 : issued - kStages; j < issued; ++j)
          mbar_wait(&bars->kv_full[j % kStages], (j / kStages) & 1, &none, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      auto issue_pv = [&](int jj) -> bool {
        if (!mbar_wait(&bars->p_full, jj & 1, ab, err, 5)) return false;
        tc_fence_after();
        const int st = jj % kStages;
        const uint32_t dO = tbase + 256;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t a = sdesc_sw128(sbase + Lay::P + (kk >> 2) * kSub + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(sbase + Lay::V + st * SUB * kSub + kk * 2048, kSub, 1024);
          umma_f16(dO, a, b, IDO, (jj > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t b = sdesc_sw128(sbase + Lay::V + st * SUB * kSub + kk * 2048, kSub, 1024);
          umma_f16_ts(dO, tbase + kPlo + 8 * kk, b, IDO, 1u);
        }
        umma_commit(&bars->o_done);
        umma_commit(&bars->kv_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, ab, err, 2);
      for (int j = 0; ok && j < nkv; ++j) {
        const int st = j % kStages, sb = j & 1;
        if (!mbar_wait(&bars->kv_full[st], (j / kStages) & 1, ab, err, 3)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&bars->s_free[sb], ((j >> 1) - 1) & 1, ab, err, 4)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dS = tbase + sb * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * kSub + (kk & 3) * 32;
          const uint64_t a = sdesc_sw128(sbase + Lay::Q + koff, 16, 1024);
          const uint64_t b = sdesc_sw128(sbase + Lay::K + st * SUB * kSub + koff, 16, 1024);
          umma_f16(dS, a, b, IDS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[sb]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(nkv - 1);
      // wait until every MMA issued here has finished before TMEM is released
      umma_commit(&bars->drain);
      Abort none{0};
      mbar_wait(&bars->drain, 0, &none, nullptr, 0);
    }
  } else {
    // ---------------- softmax: one thread per query row / TMEM lane
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const int q_row = it * kBM + r;
    float m_run = 0.f, l_run = 0.f;
    bool ok = true;
    uint8_t* P0 = sm + Lay::P;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[sb], (j >> 1) & 1, ab, err, 6))) { ok = false; break; }
      tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]);
        tmem_ld32(tbase + lane_addr + sb * 128 + 32 * c, chunk);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive_warp(&bars->s_free[sb]);
      // causal mask on the diagonal tile; the running max is taken on the raw
      // scores (c2 > 0, and rounding is monotone, so max(s) c2 = max(s c2))
      if (j == it) {
        const int lim = min(r, S - 1 - j * kBN);   // last valid column of this row
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
      // P = 2^(s c2 - m), two columns per packed FMA; four partial sums
      const float2 cc = make_float2(c2, c2), nm = make_float2(-m_new, -m_new);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), cc, nm);
        const float2 pc = make_float2(ex2(x.x), ex2(x.y));
        acc[(c >> 1) & 3] = __fadd2_rn(acc[(c >> 1) & 3], pc);
        s[c] = __float_as_uint(pc.x);
        s[c + 1] = __float_as_uint(pc.y);
      }
      const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
      const float sum = (a01.x + a23.x) + (a01.y + a23.y);
      l_run = l_run * alpha + sum;
      m_run = m_new;
      if (j >= 1) {
        // PV_{j-1} done: the P buffer is free and O is current
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done, (j - 1) & 1, ab, err, 7))) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tbase + lane_addr + 256 + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tbase + lane_addr + 256 + 32 * c, o);
          }
          tmem_wait_st();
        }
      }
      // head fp16(P) to shared memory, remainder P - fp16(P) to TMEM (two per column)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 pp = make_float2(__uint_as_float(s[32 * c + 2 * e]), __uint_as_float(s[32 * c + 2 * e + 1]));
          const __half2 h = __float22half2_rn(pp);
          const float2 rem = __ffma2_rn(__half22float2(h), make_float2(-1.f, -1.f), pp);   // p - hi, exact
          const __half2 l = __float22half2_rn(rem);
          hi[e] = *reinterpret_cast<const uint32_t*>(&h);
          lo[e] = *reinterpret_cast<const uint32_t*>(&l);
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int c16 = 4 * c + q4;       // 16-byte chunk (8 columns) of the 128-column row
          *reinterpret_cast<uint4*>(P0 + (c16 >> 3) * kSub + sw128_off(r, c16 & 7)) =
              make_uint4(hi[4 * q4], hi[4 * q4 + 1], hi[4 * q4 + 2], hi[4 * q4 + 3]);
        }
        tmem_st16(tbase + lane_addr + kPlo + 16 * c, lo);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive_warp(&bars->p_full);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bars->o_done, (nkv - 1) & 1, ab, err, 8))) {
      tc_fence_after();
      const float inv = 1.f / l_run;
      float* dst = os + ((size_t)bh * S + q_row) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tbase + lane_addr + 256 + 32 * c, o);
        tmem_wait_ld();
        if (q_row < S) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + e) =
                make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                            __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
        }
      }
      if (q_row < S) lse[(size_t)bh * S + q_row] = (m_run + log2f(l_run)) * kLn2f;
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
                            float* lse, int* err, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  const int BH = g.B * g.H;
  if (!make_tmap_16(&tq, qs, D, g.S, BH, true, kBM) || !make_tmap_16(&tk, ks, D, g.S, BH, true, kBN) ||
      !make_tmap_16(&tv, vs, D, g.S, BH, true, kBN))
    return cudaErrorInvalidValue;
  const int smem = FwdLayout<D>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(k_attn_fwd_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const float c2 = (float)(1.4426950408889634 / sqrt((double)D));
  dim3 grid((g.S + kBM - 1) / kBM, BH);
  k_attn_fwd_tc<D><<<grid, 192, smem, s>>>(tq, tk, tv, os, lse, g.S, c2, err);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_tc(const Geom& g, const void* qs, const void* ks, const void* vs,
                               float* os, float* lse, int* err, cudaStream_t s) {
  return g.D == 64 ? fwd_tc_t<64>(g, qs, ks, vs, os, lse, err, s)
                   : fwd_tc_t<128>(g, qs, ks, vs, os, lse, err, s);
}

}  // namespace lh
