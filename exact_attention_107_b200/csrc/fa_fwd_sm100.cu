// fa_fwd_sm100.cu -- bf16 / fp16 attention forward on the sm_100a tensor cores.
//
// Computes O = softmax(scale * Q K^T [causal]) V and lse = ln(sum_j exp(scale * q.k_j))
// with the tiled, online-softmax scheme of "LLM paper notes #8: FlashAttention"
// (adg.csdn.net), sections "tiling" and "online softmax", and of "CUDA-kernel-level
// optimisation: why Flash Attention is 5-10x faster than native PyTorch"
// (guanweilu.cn), section "three tricks": Q/K/V tiles are staged on chip, each
// query row keeps a running max m and sum l, the output accumulated so far is
// rescaled when m grows, and it is normalised once at the end.  No N x N matrix
// ever reaches device memory.
//
// B200 mapping (one CTA per SM, 384 threads, 2 query tiles of 128 rows per CTA):
//   warp 0      TMA producer: Q tiles once, then K_j / V_j through a shared-memory ring
//   warp 1      MMA issuer (one thread): S_t = Q_t K_j^T into tensor memory, then
//               O_t += P_t V_j with P_t read straight from tensor memory
//   warps 4-7   softmax for query tile 0 (thread r owns query row r = TMEM lane r)
//   warps 8-11  softmax for query tile 1
// The MMA thread interleaves the two tiles (S_0, S_1, PV_0, S_0', PV_1, S_1', ...)
// so one tile's softmax overlaps the other tile's matrix products.
//
// Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D, 256+2D).  P_t (16-bit, two per 32-bit column) overwrites the first 64
// columns of S_t once the scores have been read into registers.  P_t takes the
// element type of the inputs (bf16, or fp16 when F16), as the tensor-core operands
// of one MMA share one type.  It is written and announced in two halves of 64 keys,
// and the MMA thread issues the first half's P V products while the softmax computes
// the second half.
//
// Online-softmax detail: the running max used for the exponentials is only raised
// when a new row max exceeds it by more than 2^8 (in exp2 units).  Numerator and
// denominator then share the same, possibly stale, reference, so the normalised
// result is unchanged while most O rescales (a TMEM round trip) are skipped; the
// un-normalised probabilities stay below 2^8.
#include <cstdint>
#include <math_constants.h>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;            // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;            // keys per tile
constexpr int kThreads = 384;
constexpr float kRescaleThreshold = 8.0f;
// All exponentials of the forward go to the MUFU unit: with two softmax warps per SMSP
// the FMA-pipe polynomial (exp2_poly2) gave no measurable gain here (it does in the
// backward, whose phases run four warps per SMSP).
template <int D>
__device__ __forceinline__ bool poly_pair(int) { return false; }
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct FwdSmem {
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kBox = 128 * 64 * 2;      // 128 rows x 64 16-bit values: one 128-byte swizzle span
  static constexpr int kNBox = D / 64;
  static constexpr int kTile = kBox * kNBox;     // one 128-row tile of Q, K, V (or O staging)
  static constexpr int kOffQ = 0;                // 2 query tiles (reused to stage O)
  static constexpr int kOffK = kOffQ + 2 * kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffBar = kOffV + kStages * kTile;
  static constexpr int kBarQFull = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kStages;
  static constexpr int kBarVFull = kBarKEmpty + kStages;
  static constexpr int kBarVEmpty = kBarVFull + kStages;
  static constexpr int kBarSFull = kBarVEmpty + kStages;  // [2]
  static constexpr int kBarPFull = kBarSFull + 2;         // [half][tile]: P of keys [64h, 64h+64)
  static constexpr int kBarOFull = kBarPFull + 4;         // [2]
  static constexpr int kBarMmaDone = kBarOFull + 2;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;  // TMEM base address, then abort flag
  // + slack for 1024-byte alignment; at least 120 KB so that only one CTA (which
  // holds all 512 tensor-memory columns) is ever resident per SM.
  static constexpr int kBytes = (kOffSlot + 16 + 1024) > 122880 ? (kOffSlot + 16 + 1024) : 122880;
  static_assert(kBytes <= 232448, "shared memory budget");
};

template <int D, bool CAUSAL, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    float* __restrict__ lse, int N, int BH, int nqb, int hg, float scale_log2, int* status) {
  using L = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: 256 query rows (two tiles) of one (batch, head).  Causal work grows
  // with the query index, so the heaviest blocks are handed out first.
  int qblk, bh;
  {
    const WorkItem wi = grouped_order(static_cast<int>(blockIdx.x), BH, nqb, hg);
    bh = wi.bh;
    qblk = CAUSAL ? nqb - 1 - wi.tile : wi.tile;
  }
  const int nkv_all = (N + kBN - 1) / kBN;
  int q0[2], nkv[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    q0[t] = qblk * 2 * kBM + t * kBM;
    nkv[t] = (q0[t] >= N) ? 0 : (CAUSAL ? min(nkv_all, q0[t] / kBN + 1) : nkv_all);
  }
  const int nkv_max = max(nkv[0], nkv[1]);

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarQFull), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kBarKFull + s), 1);
      mbar_init(bar(L::kBarKEmpty + s), 1);
      mbar_init(bar(L::kBarVFull + s), 1);
      mbar_init(bar(L::kBarVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::kBarSFull + t), 1);
      mbar_init(bar(L::kBarPFull + t), kBM);
      mbar_init(bar(L::kBarPFull + 2 + t), kBM);
      mbar_init(bar(L::kBarOFull + t), 1);
    }
    mbar_init(bar(L::kBarMmaDone), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    FA_CONVERGED(status);
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmO);
      uint32_t qbytes = 0;
      for (int t = 0; t < 2; ++t)
        if (nkv[t] > 0) qbytes += L::kTile;
      mbar_arrive_expect_tx(bar(L::kBarQFull), qbytes);
      for (int t = 0; t < 2; ++t)
        if (nkv[t] > 0)
          for (int c = 0; c < L::kNBox; ++c)
            tma_load_3d(sb + L::kOffQ + t * L::kTile + c * L::kBox, &tmQ, bar(L::kBarQFull), c * 64, q0[t], bh);
      int nk = 0, nv = 0;
      bool ok = true;
      for (int j = 0; j < nkv_max; ++j) {
        const int s = j % L::kStages;
        const uint32_t ph = (j / L::kStages) & 1;
        if (!(ok = mbar_wait(bar(L::kBarKEmpty + s), ph ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(L::kBarKFull + s), L::kTile);
        for (int c = 0; c < L::kNBox; ++c)
          tma_load_3d(sb + L::kOffK + s * L::kTile + c * L::kBox, &tmK, bar(L::kBarKFull + s), c * 64, j * kBN, bh);
        ++nk;
        if (!(ok = mbar_wait(bar(L::kBarVEmpty + s), ph ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(L::kBarVFull + s), L::kTile);
        for (int c = 0; c < L::kNBox; ++c)
          tma_load_3d(sb + L::kOffV + s * L::kTile + c * L::kBox, &tmV, bar(L::kBarVFull + s), c * 64, j * kBN, bh);
        ++nv;
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      // Never leave with copies in flight: wait for the last load of every stage.
      mbar_wait_drain(bar(L::kBarQFull), 0);
      for (int j = max(0, nk - L::kStages); j < nk; ++j)
        mbar_wait_drain(bar(L::kBarKFull + j % L::kStages), (j / L::kStages) & 1);
      for (int j = max(0, nv - L::kStages); j < nv; ++j)
        mbar_wait_drain(bar(L::kBarVFull + j % L::kStages), (j / L::kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_16(kBM, kBN, false, false, F16);  // Q, K both K-major
      constexpr uint32_t kIdO = idesc_16(kBM, D, false, true, F16);    // P from TMEM, V MN-major
      // Each 64-column box of Q_t and K_j holds four K-steps of 16 (32 bytes apart).
      auto issue_s = [&](int t, int j) {
        const uint32_t qa = sb + L::kOffQ + t * L::kTile;
        const uint32_t kb = sb + L::kOffK + (j % L::kStages) * L::kTile;
#pragma unroll
        for (int c = 0; c < L::kNBox; ++c)
          mma_ss_x4<2, 4, 6, 2, 4, 6>(tmem + t * 128, sdesc_sw128(qa + c * L::kBox, 16, 1024),
                                      sdesc_sw128(kb + c * L::kBox, 16, 1024), kIdS, c > 0 ? 1u : 0u);
        tc_commit(bar(L::kBarSFull + t));
      };
      // O_t += P_t V_j over keys [64h, 64h+64): K-steps 4h .. 4h+3, each 8 packed P columns
      // and 16 V rows (2048 bytes) further on.
      auto issue_pv = [&](int t, int j, int h) {
        const uint32_t vb = sb + L::kOffV + (j % L::kStages) * L::kTile;
        mma_ts_x4<8, 16, 24, 128, 256, 384>(tmem + 256 + t * D, tmem + t * 128 + 32 * h,
                                            sdesc_sw128(vb + h * 4 * 2048, L::kBox, 1024), kIdO,
                                            (j > 0 || h > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait_spin(bar(L::kBarQFull), 0, abort_flag);
      if (ok && nkv_max > 0) {
        ok = mbar_wait_spin(bar(L::kBarKFull), 0, abort_flag);
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (nkv[t] > 0) issue_s(t, 0);
          tc_commit(bar(L::kBarKEmpty));
        }
      }
      for (int j = 0; ok && j < nkv_max; ++j) {
        const int s = j % L::kStages;
        if (!(ok = mbar_wait_spin(bar(L::kBarVFull + s), (j / L::kStages) & 1, abort_flag))) break;
        tc_fence_after();
        bool k_next = false;
        for (int t = 0; t < 2; ++t) {
          if (j >= nkv[t]) continue;
          // P_t arrives in two halves; the first half's products start while the
          // softmax still computes the second.
          if (!(ok = mbar_wait_spin(bar(L::kBarPFull + t), j & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(t, j, 0);
          if (!(ok = mbar_wait_spin(bar(L::kBarPFull + 2 + t), j & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(t, j, 1);
          if (j == nkv[t] - 1) tc_commit(bar(L::kBarOFull + t));
          if (j + 1 < nkv[t]) {
            if (!k_next) {
              const int jn = j + 1;
              if (!(ok = mbar_wait_spin(bar(L::kBarKFull + jn % L::kStages), (jn / L::kStages) & 1, abort_flag)))
                break;
              tc_fence_after();
              k_next = true;
            }
            issue_s(t, j + 1);
          }
        }
        if (!ok) break;
        tc_commit(bar(L::kBarVEmpty + s));
        if (k_next) tc_commit(bar(L::kBarKEmpty + (j + 1) % L::kStages));
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      // Every MMA this thread issued has finished before tensor memory is released.
      tc_commit(bar(L::kBarMmaDone));
      mbar_wait_drain(bar(L::kBarMmaDone), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;
    const int r = threadIdx.x - kBM * (t + 1);                  // row in tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const int qrow = q0[t] + r;
    float m = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv[t]; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarSFull + t), j & 1, abort_flag));
      if (!ok) break;
      FA_CONVERGED(status);                                     // warp-collective TMEM loads follow
      tc_fence_after();
      uint32_t sr[4][32];
      tmem_ld32(tS, sr[0]);
      tmem_ld32(tS + 32, sr[1]);
      tmem_ld32(tS + 64, sr[2]);
      tmem_ld32(tS + 96, sr[3]);
      tmem_ld_wait();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      reg_fence(sr[2]);
      reg_fence(sr[3]);
      const int kv0 = j * kBN;
      const bool diag = CAUSAL && (kv0 + kBN - 1 > q0[t]);
      if (diag || kv0 + kBN > N) {
        const int lim = min(CAUSAL ? qrow - kv0 : kBN - 1, N - 1 - kv0);   // keep columns c <= lim
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c > lim) sr[c >> 5][c & 31] = 0xff800000u;                  // -inf
      }
      float mx[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
      for (int c = 0; c < kBN; c += 2)
        mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], __uint_as_float(sr[c >> 5][c & 31]),
                                 __uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]));
      const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale_log2;
      const float m_new = fmaxf(m, m_tile);
      const bool need = m_new > m + kRescaleThreshold;                     // always true at j == 0
      const float m_use = need ? m_new : m;
      const float alpha = need ? ex2_approx(m - m_new) : 1.f;
      const float neg = (m_use == -CUDART_INF_F) ? 0.f : -m_use;
      // P = exp2(s * scale * log2 e - m) in two halves of 64 keys; each half is stored as
      // packed 16-bit pairs over the first 32 + 32 columns of S_t (already read) and
      // announced on its own barrier, so the P V products of the first half overlap the
      // exponentials of the second.
      float2 sum[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 sl2 = make_float2(scale_log2, scale_log2), neg2 = make_float2(neg, neg);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // P of keys [64h, 64h+64) as packed pairs, stored 16 pairs at a time (nothing reads
        // them before this half's barrier arrival below), to keep the registers for S.
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[16];
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) {
            const int c = 32 * h + 16 * hh + c2;           // pair index: columns 2c, 2c + 1
            const float2 sv = make_float2(__uint_as_float(sr[(2 * c) >> 5][(2 * c) & 31]),
                                          __uint_as_float(sr[(2 * c + 1) >> 5][(2 * c + 1) & 31]));
            const float2 p = exp2_pair(__ffma2_rn(sv, sl2, neg2), poly_pair<D>(c));
            sum[c & 1] = __fadd2_rn(sum[c & 1], p);
            pk[c2] = pack16<F16>(p.x, p.y);
          }
          tmem_st16(tS + 32 * h + 16 * hh, pk);
        }
        if (h == 0 && j > 0 && __any_sync(0xffffffffu, need)) {
          FA_CONVERGED(status);
          // Rescale O_t before any of this step's P V products lands in it (after the
          // first half's exponentials, whose scores no longer occupy registers).  O_t was
          // finished by the PV MMAs of step j-1: the commit that announced S_t(j) also
          // covers every earlier MMA of this thread, including those.
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_ld_wait();
            reg_fence(o);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])),
                                          make_float2(alpha, alpha));
              o[i] = __float_as_uint(v.x);
              o[i + 1] = __float_as_uint(v.y);
            }
            tmem_st32(tO + cc * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(L::kBarPFull + 2 * h + t));
      }
      l = l * alpha + ((sum[0].x + sum[0].y) + (sum[1].x + sum[1].y));
      m = m_use;
    }
    if (ok && nkv[t] > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarOFull + t), 0, abort_flag));
    if (!ok) {
      raise_error(status, abort_flag, kStatusTimeout);
    } else if (nkv[t] > 0) {
      FA_CONVERGED(status);
      tc_fence_after();
      // Epilogue: O / l -> bf16 / fp16 into this warp's 32 rows of the (now idle) Q_t tile,
      // in the 128-byte-swizzled layout the O tensor map expects, then one TMA store
      // per warp (rows past N are clipped by the hardware).
      const float inv_l = 1.f / l;
      uint8_t* stage = smem + L::kOffQ + t * L::kTile;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_ld_wait();
        reg_fence(o);
        const int box = cc >> 1;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (cc & 1) * 4 + q4;
          uint4 v;
          v.x = pack16<F16>(__uint_as_float(o[8 * q4 + 0]) * inv_l, __uint_as_float(o[8 * q4 + 1]) * inv_l);
          v.y = pack16<F16>(__uint_as_float(o[8 * q4 + 2]) * inv_l, __uint_as_float(o[8 * q4 + 3]) * inv_l);
          v.z = pack16<F16>(__uint_as_float(o[8 * q4 + 4]) * inv_l, __uint_as_float(o[8 * q4 + 5]) * inv_l);
          v.w = pack16<F16>(__uint_as_float(o[8 * q4 + 6]) * inv_l, __uint_as_float(o[8 * q4 + 7]) * inv_l);
          *reinterpret_cast<uint4*>(stage + box * L::kBox + r * 128 + ((chunk ^ (r & 7)) << 4)) = v;
        }
      }
      fence_async_smem();
      __syncwarp();
      const int wrow = (warp & 3) * 32;
      if (lane == 0 && q0[t] + wrow < N) {
        for (int c = 0; c < L::kNBox; ++c)
          tma_store_3d(&tmO, sb + L::kOffQ + t * L::kTile + c * L::kBox + wrow * 128, c * 64, q0[t] + wrow, bh);
        bulk_commit();
        bulk_wait_read0();
      }
      if (qrow < N && FA_BOUNDS(static_cast<size_t>(bh) < static_cast<size_t>(BH), status))
        lse[static_cast<size_t>(bh) * N + qrow] = m * kLn2 + logf(l);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    FA_CONVERGED(status);
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool CAUSAL, bool F16>
cudaError_t launch_impl(const FwdLaunch& a, cudaStream_t stream) {
  using L = FwdSmem<D>;
  auto kern = fwd_kernel<D, CAUSAL, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const int nqb = (a.N + 2 * kBM - 1) / (2 * kBM);
  const unsigned grid = static_cast<unsigned>(nqb) * static_cast<unsigned>(a.BH);
  const float scale_log2 = a.scale * 1.44269504088896340736f;
  kern<<<grid, kThreads, L::kBytes, stream>>>(a.tmQ, a.tmK, a.tmV, a.tmO, a.lse, a.N, a.BH, nqb, a.hg, scale_log2,
                                               a.status);
  return cudaGetLastError();
}

template <bool F16>
cudaError_t launch_typed(const FwdLaunch& a, cudaStream_t stream) {
  // Head dims 32 and 96 run the 64- and 128-column kernels: the tensor maps describe
  // the caller's D, so the TMA fills the missing columns of every loaded tile with
  // zeros (which add nothing to Q K^T and give zero columns of P V) and clips them
  // from every store.
  if (a.D <= 64) return a.causal ? launch_impl<64, true, F16>(a, stream) : launch_impl<64, false, F16>(a, stream);
  return a.causal ? launch_impl<128, true, F16>(a, stream) : launch_impl<128, false, F16>(a, stream);
}

}  // namespace

cudaError_t launch_fwd_16(const FwdLaunch& a, cudaStream_t stream) {
  return a.f16 ? launch_typed<true>(a, stream) : launch_typed<false>(a, stream);
}

}  // namespace fa
