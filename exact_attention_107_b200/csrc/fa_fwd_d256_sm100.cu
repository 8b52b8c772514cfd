// fa_fwd_d256_sm100.cu -- attention forward for head dimension 256 (bf16 / fp16) on the
// sm_100a tensor cores.
//
// The same computation as fa_fwd_sm100.cu (tiling and online softmax of "LLM paper
// notes #8: FlashAttention", adg.csdn.net, sections "tiling" and "online softmax"):
// O = softmax(scale * Q K^T [causal]) V and lse per row, no N x N matrix in memory.
//
// What changes at D = 256 is the on-chip budget.  The fp32 output accumulator of one
// 128-row query tile takes 256 of the 512 tensor-memory columns, so a CTA holds ONE
// query tile (instead of two) and uses the other half for two score buffers:
//   TMEM  S_a [0,128)  S_b [128,256)  O [256,512)
// Scores of key tile j go to buffer j & 1, so the MMA thread computes S_{j+1} before
// O += P_j V_j and the softmax of tile j+1 overlaps the P V product of tile j:
//   MMA order   S_0, S_1, PV_0, S_2, PV_1, S_3, ...
// A 128 x 256 tile of K or V is 64 KB, so shared memory holds Q (64 KB) and a ring of
// eight 16 KB boxes (128 rows x 64 columns each) that the producer fills in exactly
// the order the MMAs read them (K_0, K_1, V_0, K_2, V_1, ...), one box at a time: a
// box is refilled as soon as the MMAs reading it have finished.
//
// Warps: 0 TMA producer, 1 MMA issuer (one thread), 4-7 softmax + epilogue (thread r
// owns query row r = TMEM lane r).  Warps 2-3 have no work.
#include <cstdint>
#include <math_constants.h>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kD = 256;
constexpr int kBM = 128;             // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;             // keys per tile
constexpr int kThreads = 256;
constexpr float kRescaleThreshold = 8.0f;   // lazy rescale, as in the D <= 128 forward
constexpr float kLn2 = 0.69314718055994530942f;

struct Smem {
  static constexpr int kBox = 128 * 128;            // 128 rows x 64 16-bit values (one swizzle span per row)
  static constexpr int kNBox = kD / 64;             // 4 boxes per 128 x 256 tile
  static constexpr int kRing = 8;                   // ring of boxes: two K/V tiles
  static constexpr int kOffQ = 0;                   // Q tile (later: O staging)
  static constexpr int kOffRing = kOffQ + kNBox * kBox;
  static constexpr int kOffBar = kOffRing + kRing * kBox;
  static constexpr int kBarQFull = 0;
  static constexpr int kBarFull = 1;                     // [kRing]
  static constexpr int kBarEmpty = kBarFull + kRing;     // [kRing]
  static constexpr int kBarSFull = kBarEmpty + kRing;    // [2]
  static constexpr int kBarPFull = kBarSFull + 2;        // [2]
  static constexpr int kBarODone = kBarPFull + 2;        // one phase per P V product
  static constexpr int kBarOFull = kBarODone + 1;        // after the last P V product
  static constexpr int kBarMmaDone = kBarOFull + 1;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;   // TMEM base address, then abort flag
  static constexpr int kBytes = kOffSlot + 16 + 1024;       // + slack for 1024-byte alignment
  static_assert(kBytes <= 232448, "shared memory budget");
  static_assert(kBytes > 116 * 1024, "one CTA per SM (it holds all 512 TMEM columns)");
};

// Position of a key tile's K and V in the load / MMA sequence K_0, K_1, V_0, K_2, V_1,
// ..., K_{n-1}, V_{n-2}, V_{n-1} (n key tiles); each entry is 4 consecutive boxes.
__device__ __forceinline__ int seq_k(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int seq_v(int j, int n) { return j < n - 1 ? 2 * j + 2 : 2 * n - 1; }

template <bool CAUSAL, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    float* __restrict__ lse, int N, int BH, int nqt, int hg, float scale_log2, int* status) {
  using L = Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  auto box = [&](int b) -> uint32_t { return sb + L::kOffRing + (b & (L::kRing - 1)) * L::kBox; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: one 128-row query tile of one (batch, head); causal work grows with the
  // query index, so the heaviest tiles are handed out first.
  int qt, bh;
  {
    const WorkItem wi = grouped_order(static_cast<int>(blockIdx.x), BH, nqt, hg);
    bh = wi.bh;
    qt = CAUSAL ? nqt - 1 - wi.tile : wi.tile;
  }
  const int q0 = qt * kBM;
  const int nkv_all = (N + kBN - 1) / kBN;
  const int n = CAUSAL ? min(nkv_all, q0 / kBN + 1) : nkv_all;   // >= 1
  const int nseq = 2 * n;                                          // K/V tile entries in the sequence

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarQFull), 1);
    for (int s = 0; s < L::kRing; ++s) {
      mbar_init(bar(L::kBarFull + s), 1);
      mbar_init(bar(L::kBarEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::kBarSFull + b), 1);
      mbar_init(bar(L::kBarPFull + b), kBM);
    }
    mbar_init(bar(L::kBarODone), 1);
    mbar_init(bar(L::kBarOFull), 1);
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
      mbar_arrive_expect_tx(bar(L::kBarQFull), L::kNBox * L::kBox);
      for (int c = 0; c < L::kNBox; ++c)
        tma_load_3d(sb + L::kOffQ + c * L::kBox, &tmQ, bar(L::kBarQFull), c * 64, q0, bh);
      int nb = 0;                          // boxes issued so far (box b: ring slot b % 8, phase (b / 8) & 1)
      bool ok = true;
      for (int u = 0; ok && u < nseq; ++u) {
        // entry u of the sequence: K_j or V_j
        const bool is_v = (u == nseq - 1) || (u >= 2 && (u & 1) == 0);
        const int j = is_v ? (u == nseq - 1 ? n - 1 : (u - 2) / 2) : (u == 0 ? 0 : (u + 1) / 2);
        const CUtensorMap* tm = is_v ? &tmV : &tmK;
        for (int c = 0; c < L::kNBox; ++c, ++nb) {
          const int s = nb & (L::kRing - 1);
          if (!(ok = mbar_wait(bar(L::kBarEmpty + s), ((nb >> 3) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(bar(L::kBarFull + s), L::kBox);
          tma_load_3d(box(nb), tm, bar(L::kBarFull + s), c * 64, j * kBN, bh);
        }
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      // Never leave with copies in flight: wait for the last load of every ring slot.
      mbar_wait_drain(bar(L::kBarQFull), 0);
      for (int b = max(0, nb - L::kRing); b < nb; ++b)
        mbar_wait_drain(bar(L::kBarFull + (b & (L::kRing - 1))), (b >> 3) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_16(kBM, kBN, false, false, F16);   // Q, K both K-major
      constexpr uint32_t kIdO = idesc_16(kBM, kD, false, true, F16);     // P from TMEM, V MN-major, N = 256
      // S_j = Q K_j^T into buffer j & 1; each K box is released once its 4 K-steps finish.
      auto issue_s = [&](int j) -> bool {
        const int b0 = 4 * seq_k(j);
        for (int c = 0; c < L::kNBox; ++c) {
          const int b = b0 + c;
          if (!mbar_wait_spin(bar(L::kBarFull + (b & (L::kRing - 1))), (b >> 3) & 1, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            mma_ss(tmem + (j & 1) * 128, sdesc_sw128(sb + L::kOffQ + c * L::kBox + k4 * 32, 16, 1024),
                   sdesc_sw128(box(b) + k4 * 32, 16, 1024), kIdS, (c | k4) ? 1u : 0u);
          tc_commit(bar(L::kBarEmpty + (b & (L::kRing - 1))));
        }
        tc_commit(bar(L::kBarSFull + (j & 1)));
        return true;
      };
      // O += P_j V_j, one N = 256 MMA per 16 keys (an N = 256 MMA runs at the full rate,
      // two N = 128 halves would not); the 4 V boxes are consecutive ring slots.
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait_spin(bar(L::kBarPFull + (j & 1)), (j >> 1) & 1, abort_flag)) return false;
        const int b0 = 4 * seq_v(j, n);
        for (int c = 0; c < L::kNBox; ++c) {
          const int b = b0 + c;
          if (!mbar_wait_spin(bar(L::kBarFull + (b & (L::kRing - 1))), (b >> 3) & 1, abort_flag)) return false;
        }
        tc_fence_after();
        const uint32_t vb = box(b0);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(tmem + 256, tmem + (j & 1) * 128 + kk * 8, sdesc_sw128(vb + kk * 2048, L::kBox, 1024), kIdO,
                 (j > 0 || kk > 0) ? 1u : 0u);
        for (int c = 0; c < L::kNBox; ++c) tc_commit(bar(L::kBarEmpty + ((b0 + c) & (L::kRing - 1))));
        tc_commit(bar(L::kBarODone));
        if (j == n - 1) tc_commit(bar(L::kBarOFull));
        return true;
      };
      bool ok = mbar_wait_spin(bar(L::kBarQFull), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n && !(ok = issue_s(j + 1))) break;
        ok = issue_pv(j);
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      // Every MMA this thread issued has finished before tensor memory is released.
      tc_commit(bar(L::kBarMmaDone));
      mbar_wait_drain(bar(L::kBarMmaDone), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int r = threadIdx.x - kBM;                          // row in tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + lane_off + 256;
    const int qrow = q0 + r;
    float m = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const uint32_t tS = tmem + lane_off + (j & 1) * 128;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarSFull + (j & 1)), (j >> 1) & 1, abort_flag));
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
      const bool diag = CAUSAL && (kv0 + kBN - 1 > q0);
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
      uint32_t pk[2][32];
      float2 sum[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 sl2 = make_float2(scale_log2, scale_log2), neg2 = make_float2(neg, neg);
#pragma unroll
      for (int c = 0; c < kBN / 2; ++c) {
        const float2 sv = make_float2(__uint_as_float(sr[(2 * c) >> 5][(2 * c) & 31]),
                                      __uint_as_float(sr[(2 * c + 1) >> 5][(2 * c + 1) & 31]));
        const float2 p = exp2_pair(__ffma2_rn(sv, sl2, neg2), false);
        sum[c & 1] = __fadd2_rn(sum[c & 1], p);
        pk[c >> 5][c & 31] = pack16<F16>(p.x, p.y);
      }
      l = l * alpha + ((sum[0].x + sum[0].y) + (sum[1].x + sum[1].y));
      m = m_use;
      tmem_st32(tS, pk[0]);
      tmem_st32(tS + 32, pk[1]);
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O is rescaled only between P V products: wait for PV_{j-1} (phase j-1 of
        // ODone).  PV_j cannot start before this thread arrives on PFull below.
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarODone), (j - 1) & 1, abort_flag));
        if (!ok) break;
        FA_CONVERGED(status);
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < kD / 32; ++cc) {
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
      mbar_arrive(bar(L::kBarPFull + (j & 1)));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarOFull), 0, abort_flag));
    if (!ok) {
      raise_error(status, abort_flag, kStatusTimeout);
    } else {
      FA_CONVERGED(status);
      tc_fence_after();
      // Epilogue: O / l -> 16-bit into this warp's 32 rows of the (now idle) Q tile, in
      // the 128-byte-swizzled layout of the O tensor map, then one TMA store per box.
      const float inv_l = 1.f / l;
      uint8_t* stage = smem + L::kOffQ;
#pragma unroll
      for (int cc = 0; cc < kD / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_ld_wait();
        reg_fence(o);
        const int bx = cc >> 1;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = (cc & 1) * 4 + q4;
          uint4 v;
          v.x = pack16<F16>(__uint_as_float(o[8 * q4 + 0]) * inv_l, __uint_as_float(o[8 * q4 + 1]) * inv_l);
          v.y = pack16<F16>(__uint_as_float(o[8 * q4 + 2]) * inv_l, __uint_as_float(o[8 * q4 + 3]) * inv_l);
          v.z = pack16<F16>(__uint_as_float(o[8 * q4 + 4]) * inv_l, __uint_as_float(o[8 * q4 + 5]) * inv_l);
          v.w = pack16<F16>(__uint_as_float(o[8 * q4 + 6]) * inv_l, __uint_as_float(o[8 * q4 + 7]) * inv_l);
          *reinterpret_cast<uint4*>(stage + bx * L::kBox + r * 128 + ((chunk ^ (r & 7)) << 4)) = v;
        }
      }
      fence_async_smem();
      __syncwarp();
      const int wrow = (warp & 3) * 32;
      if (lane == 0 && q0 + wrow < N) {
        for (int c = 0; c < L::kNBox; ++c)
          tma_store_3d(&tmO, sb + L::kOffQ + c * L::kBox + wrow * 128, c * 64, q0 + wrow, bh);
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

template <bool CAUSAL, bool F16>
cudaError_t launch_impl(const FwdLaunch& a, cudaStream_t stream) {
  auto kern = fwd_d256_kernel<CAUSAL, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem::kBytes);
  if (e != cudaSuccess) return e;
  const int nqt = (a.N + kBM - 1) / kBM;
  const unsigned grid = static_cast<unsigned>(nqt) * static_cast<unsigned>(a.BH);
  const float scale_log2 = a.scale * 1.44269504088896340736f;
  kern<<<grid, kThreads, Smem::kBytes, stream>>>(a.tmQ, a.tmK, a.tmV, a.tmO, a.lse, a.N, a.BH, nqt, a.hg, scale_log2,
                                                   a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_d256(const FwdLaunch& a, cudaStream_t stream) {
  if (a.f16) return a.causal ? launch_impl<true, true>(a, stream) : launch_impl<false, true>(a, stream);
  return a.causal ? launch_impl<true, false>(a, stream) : launch_impl<false, false>(a, stream);
}

}  // namespace fa
