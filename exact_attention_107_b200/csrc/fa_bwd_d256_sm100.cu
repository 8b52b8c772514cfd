// fa_bwd_d256_sm100.cu -- attention backward for head dimension 256 (bf16 / fp16).
//
// The same computation as fa_bwd_sm100.cu (P recomputed from the saved logsumexp, as
// "LLM paper notes #8: FlashAttention", adg.csdn.net, section "recomputation",
// describes; dV = P^T dO, dS = P * (dP - delta), dQ = scale dS K, dK = scale dS^T Q).
//
// At D = 256 one SM cannot hold what the 128-key (or 128-query) tiling of the smaller
// head dims keeps on chip: S^T, dP^T, dV and dK would need 768 tensor-memory columns,
// and K, V, Q, dO tiles 256 KB of shared memory.  So two CTAs share each tile, one per
// half h of the head dimension: each owns the columns [128h, 128h+128) of dV, dK (or
// dQ) and recomputes the full-depth S and dP products that both halves need.  The
// price is twice the S / dP work; what it buys is a layout that fits:
//   dK/dV CTA  TMEM  S^T [0,128)  dP^T [128,256)  dV_h [256,384)  dK_h [384,512)
//              smem  K_j, V_j (128 KB, resident) + a ring of six 16 KB boxes
//   dQ CTA     TMEM  S [0,128)    dP [128,256)    dQ_h [256,384)
//              smem  Q_i, dO_i (128 KB, resident) + the same ring
// Everything streamed goes through the ring as 128-row x 64-column boxes in exactly the
// order the MMAs consume them, and each box is released right after its last MMA, so
// the ring is a plain FIFO (a box that two products need is simply loaded twice):
//   dK/dV, per query tile i   Q_i (4 boxes), dO_i (4), dO_i half h (2), Q_i half h (2)
//   dQ,    per key tile j     K_j (4 boxes), V_j (4), K_j half h (2)
// Element-wise work (P, dS) is split over four warpgroups of 32 columns, as in the
// D <= 128 kernels.
#include <cstdint>
#include <math_constants.h>
#include <type_traits>

#include "bwd_common.cuh"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kBox = 128 * 128;          // 128 rows x 64 16-bit values
constexpr int kRing = 6;                 // box b of the sequence: slot b % 6, phase (b / 6) & 1

struct DkdvD256Smem {
  static constexpr int kOffK = 0;                          // K_j, 4 boxes (later dK_h staging)
  static constexpr int kOffV = 4 * kBox;                   // V_j, 4 boxes (later dV_h staging)
  static constexpr int kOffRing = 8 * kBox;
  static constexpr int kOffBar = kOffRing + kRing * kBox;  // 224 KB of tiles
  static constexpr int kBarKV = 0;
  static constexpr int kBarFull = 1;                       // [kRing]
  static constexpr int kBarEmpty = kBarFull + kRing;       // [kRing]
  static constexpr int kBarS = kBarEmpty + kRing;
  static constexpr int kBarDP = kBarS + 1;
  static constexpr int kBarP = kBarDP + 1;                 // packed P^T stored (512 threads)
  static constexpr int kBarDS = kBarP + 1;                 // packed dS^T stored (512 threads)
  static constexpr int kBarAcc = kBarDS + 1;
  static constexpr int kBarMmaDone = kBarAcc + 1;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kBytes = kOffSlot + 16 + 1024;
  static_assert(kBytes <= 232448, "shared memory budget");
};

struct DqD256Smem {
  static constexpr int kOffQ = 0;                          // Q_i, 4 boxes (later dQ_h staging)
  static constexpr int kOffdO = 4 * kBox;
  static constexpr int kOffRing = 8 * kBox;
  static constexpr int kOffBar = kOffRing + kRing * kBox;
  static constexpr int kBarQ = 0;
  static constexpr int kBarFull = 1;
  static constexpr int kBarEmpty = kBarFull + kRing;
  static constexpr int kBarS = kBarEmpty + kRing;
  static constexpr int kBarDP = kBarS + 1;
  static constexpr int kBarDS = kBarDP + 1;
  static constexpr int kBarAcc = kBarDS + 1;
  static constexpr int kBarMmaDone = kBarAcc + 1;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kBytes = kOffSlot + 16 + 1024;
  static_assert(kBytes <= 232448, "shared memory budget");
};

// Loads box b of a sequence into its ring slot once the slot's previous box has been
// released.  Returns false when the wait gave up.
__device__ __forceinline__ bool ring_load(uint32_t ring, uint32_t full0, uint32_t empty0, int b, const CUtensorMap* tm,
                                          int x, int y, int z, volatile int* abort_flag) {
  const int s = b % kRing;
  if (!mbar_wait(empty0 + 8 * s, ((b / kRing) & 1) ^ 1, abort_flag)) return false;
  mbar_arrive_expect_tx(full0 + 8 * s, kBox);
  tma_load_3d(ring + s * kBox, tm, full0 + 8 * s, x, y, z);
  return true;
}
// Never leave with copies in flight: waits for the last load of every ring slot.
__device__ __forceinline__ void ring_drain(uint32_t full0, int nb) {
  for (int b = max(0, nb - kRing); b < nb; ++b) mbar_wait_drain(full0 + 8 * (b % kRing), (b / kRing) & 1);
}

// ----------------------------------------------------------------------------- dK, dV
template <bool CAUSAL, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_d256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                         const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                         const float* __restrict__ ws_nl, const float* __restrict__ ws_delta, int N, int Npad,
                         int BH, int nkt, float scale, int* status) {
  using L = DkdvD256Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  auto slot_addr = [&](int b) -> uint32_t { return sb + L::kOffRing + (b % kRing) * kBox; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: half h of key tile kt of head bh.  Causal: low kt meet the most query
  // tiles and go first.
  const int h = static_cast<int>(blockIdx.x & 1);
  const int item = static_cast<int>(blockIdx.x >> 1);
  int kt, bh;
  if (CAUSAL) {
    kt = item / BH;
    bh = item % BH;
  } else {
    kt = item % nkt;
    bh = item / nkt;
  }
  const int kv0 = kt * 128;
  const int it0 = CAUSAL ? kt : 0;
  const int n = nkt - it0;                 // query tiles visited, >= 1

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarKV), 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(bar(L::kBarFull + s), 1);
      mbar_init(bar(L::kBarEmpty + s), 1);
    }
    mbar_init(bar(L::kBarS), 1);
    mbar_init(bar(L::kBarDP), 1);
    mbar_init(bar(L::kBarP), 512);
    mbar_init(bar(L::kBarDS), 512);
    mbar_init(bar(L::kBarAcc), 1);
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
  constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;

  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar(L::kBarKV), 8 * kBox);
      for (int c = 0; c < 4; ++c) {
        tma_load_3d(sb + L::kOffK + c * kBox, &tmK, bar(L::kBarKV), c * 64, kv0, bh);
        tma_load_3d(sb + L::kOffV + c * kBox, &tmV, bar(L::kBarKV), c * 64, kv0, bh);
      }
      int nb = 0;
      bool ok = true;
      for (int i = 0; ok && i < n; ++i) {
        const int q0 = (it0 + i) * 128;
        for (int e = 0; e < 12; ++e, ++nb) {
          const bool is_q = e < 4 || e >= 10;
          const int col = e < 4 ? e : e < 8 ? e - 4 : e < 10 ? 2 * h + e - 8 : 2 * h + e - 10;
          if (!(ok = ring_load(sb + L::kOffRing, bar(L::kBarFull), bar(L::kBarEmpty), nb, is_q ? &tmQ : &tmdO,
                               col * 64, q0, bh, abort_flag)))
            break;
        }
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      mbar_wait_drain(bar(L::kBarKV), 0);
      ring_drain(bar(L::kBarFull), nb);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_16(128, 128, false, false, F16);   // S^T, dP^T: K-major A and B
      constexpr uint32_t kIdAcc = idesc_16(128, 128, false, true, F16);  // dV_h, dK_h: A in TMEM, B MN-major
      auto full = [&](int b) { return bar(L::kBarFull + b % kRing); };
      auto empty = [&](int b) { return bar(L::kBarEmpty + b % kRing); };
      // acc = A_smem (resident tile, 4 boxes) x B^T over the 4 ring boxes starting at b0
      auto issue_full_depth = [&](uint32_t dcol, uint32_t a_tile, int b0) -> bool {
        for (int c = 0; c < 4; ++c) {
          const int b = b0 + c;
          if (!mbar_wait_spin(full(b), (b / kRing) & 1, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            mma_ss(tmem + dcol, sdesc_sw128(a_tile + c * kBox + k4 * 32, 16, 1024),
                   sdesc_sw128(slot_addr(b) + k4 * 32, 16, 1024), kIdS, (c | k4) ? 1u : 0u);
          tc_commit(empty(b));
        }
        return true;
      };
      // acc (+)= A_tmem (packed, 128 queries) x B (the ring pair b, b+1: 128 queries x 128 columns)
      auto issue_half = [&](uint32_t dcol, uint32_t abase, int b, bool first) -> bool {
        if (!mbar_wait_spin(full(b), (b / kRing) & 1, abort_flag)) return false;
        if (!mbar_wait_spin(full(b + 1), ((b + 1) / kRing) & 1, abort_flag)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + dcol, tmem + packed_col(abase, kk), sdesc_sw128(slot_addr(b) + kk * 2048, kBox, 1024), kIdAcc,
                 (!first || kk > 0) ? 1u : 0u);
        tc_commit(empty(b));
        tc_commit(empty(b + 1));
        return true;
      };
      bool ok = mbar_wait_spin(bar(L::kBarKV), 0, abort_flag);
      for (int i = 0; ok && i < n; ++i) {
        const int b0 = 12 * i;
        tc_fence_after();
        if (!(ok = issue_full_depth(kColS, sb + L::kOffK, b0))) break;         // S^T = K_j Q_i^T
        tc_commit(bar(L::kBarS));
        if (!(ok = issue_full_depth(kColDP, sb + L::kOffV, b0 + 4))) break;    // dP^T = V_j dO_i^T
        tc_commit(bar(L::kBarDP));
        if (!(ok = mbar_wait_spin(bar(L::kBarP), i & 1, abort_flag))) break;
        if (!(ok = issue_half(kColDV, kColS, b0 + 8, i == 0))) break;          // dV_h += P^T dO_i[:, h]
        if (!(ok = mbar_wait_spin(bar(L::kBarDS), i & 1, abort_flag))) break;
        if (!(ok = issue_half(kColDK, kColDP, b0 + 10, i == 0))) break;        // dK_h += dS^T Q_i[:, h]
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      tc_commit(bar(L::kBarAcc));
      tc_commit(bar(L::kBarMmaDone));
      mbar_wait_drain(bar(L::kBarMmaDone), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ P^T, dS^T (32 query columns), epilogue
    const int g = (warp - 4) >> 2;                                      // query columns [32g, 32g+32)
    const int r = threadIdx.x - 128 * (1 + g);                           // key row = TMEM lane
    const uint32_t tb = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = kv0 + r;
    const float scale_log2 = scale * kLog2e;
    const float2 sl2 = make_float2(scale_log2, scale_log2);
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int q0 = (it0 + i) * 128;
      // this warpgroup's 32 query statistics in the padded workspace (in bounds, 16-byte aligned)
      const size_t srow = static_cast<size_t>(bh) * Npad + q0 + 32 * g;
      const bool sin = FA_BOUNDS(srow + 32 <= static_cast<size_t>(BH) * Npad, status);
      float4 nl4[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        nl4[q] = sin ? __ldg(reinterpret_cast<const float4*>(ws_nl + srow) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS), i & 1, abort_flag));
      if (!ok) break;
      FA_CONVERGED(status);                                     // warp-collective TMEM loads follow
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tb + kColS + 32 * g, sr);
      tmem_ld_wait();
      reg_fence(sr);
      const int qc0 = q0 + 32 * g;                                       // query of this thread's column 0
      const bool diag = CAUSAL && __any_sync(0xffffffffu, qc0 < key + 32);   // warp-uniform
      uint32_t pk[16];
      auto p_phase = [&](auto masked) {
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) {
          const int c = 2 * c2;
          const float2 nl = (c2 & 1) ? make_float2(nl4[c2 >> 1].z, nl4[c2 >> 1].w)
                                     : make_float2(nl4[c2 >> 1].x, nl4[c2 >> 1].y);
          const float2 sv = make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
          float2 p = exp2_pair(__ffma2_rn(sv, sl2, nl), poly_pair(c2));
          if (decltype(masked)::value) {
            if (key > qc0 + c) p.x = 0.f;
            if (key > qc0 + c + 1) p.y = 0.f;
          }
          pk[c2] = pack16<F16>(p.x, p.y);
        }
      };
      if (diag) p_phase(std::true_type{});
      else p_phase(std::false_type{});
      tmem_st16(tb + kColS + 32 * g, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarP));
      // dS^T = P^T * (dP^T - delta)
      float4 dl4[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        dl4[q] = sin ? __ldg(reinterpret_cast<const float4*>(ws_delta + srow) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP), i & 1, abort_flag));
      if (!ok) break;
      FA_CONVERGED(status);
      tc_fence_after();
      uint32_t dp[32];
      tmem_ld32(tb + kColDP + 32 * g, dp);
      tmem_ld_wait();
      reg_fence(dp);
      uint32_t dsk[16];
#pragma unroll
      for (int c2 = 0; c2 < 16; ++c2) {
        const int c = 2 * c2;
        const float2 dl = (c2 & 1) ? make_float2(dl4[c2 >> 1].z, dl4[c2 >> 1].w) : make_float2(dl4[c2 >> 1].x, dl4[c2 >> 1].y);
        const float2 dpv = make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1]));
        const float2 ds = __fmul2_rn(make_float2(unpack16_lo<F16>(pk[c2]), unpack16_hi<F16>(pk[c2])),
                                     __ffma2_rn(dl, make_float2(-1.f, -1.f), dpv));
        dsk[c2] = pack16<F16>(ds.x, ds.y);
      }
      tmem_st16(tb + kColDP + 32 * g, dsk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarDS));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarAcc), 0, abort_flag));
    if (!ok) {
      raise_error(status, abort_flag, kStatusTimeout);
    } else {
      // One 64-column box per warpgroup: dV_h boxes 0-1 (via the idle V tile), dK_h boxes 0-1
      // (via the idle K tile); global columns 128h + 64c.
      FA_CONVERGED(status);
      tc_fence_after();
      const int wrow = (warp & 3) * 32;
      const bool is_dv = g < 2;
      const int c = g & 1;
      stage_box_16<128, F16>(tb + (is_dv ? kColDV : kColDK), c, is_dv ? 1.f : scale,
                             smem + (is_dv ? L::kOffV : L::kOffK), r);
      store_warp_box_x(is_dv ? &tmdV : &tmdK, sb + (is_dv ? L::kOffV : L::kOffK), c, 2 * h + c, wrow, kv0, bh,
                       lane, N);
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

// ----------------------------------------------------------------------------- dQ
template <bool CAUSAL, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_d256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdQ, const float* __restrict__ ws_nl,
                       const float* __restrict__ ws_delta, int N, int Npad, int BH, int nqt, float scale,
                       int* status) {
  using L = DqD256Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  auto slot_addr = [&](int b) -> uint32_t { return sb + L::kOffRing + (b % kRing) * kBox; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: half h of query tile qt of head bh.  Causal: heaviest first.
  const int h = static_cast<int>(blockIdx.x & 1);
  const int item = static_cast<int>(blockIdx.x >> 1);
  int qt, bh;
  if (CAUSAL) {
    qt = nqt - 1 - item / BH;
    bh = item % BH;
  } else {
    qt = item % nqt;
    bh = item / nqt;
  }
  const int q0 = qt * 128;
  const int nkt = (N + 127) / 128;
  const int n = CAUSAL ? min(nkt, qt + 1) : nkt;           // key tiles visited, >= 1

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarQ), 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(bar(L::kBarFull + s), 1);
      mbar_init(bar(L::kBarEmpty + s), 1);
    }
    mbar_init(bar(L::kBarS), 1);
    mbar_init(bar(L::kBarDP), 1);
    mbar_init(bar(L::kBarDS), 512);
    mbar_init(bar(L::kBarAcc), 1);
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
  constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;

  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar(L::kBarQ), 8 * kBox);
      for (int c = 0; c < 4; ++c) {
        tma_load_3d(sb + L::kOffQ + c * kBox, &tmQ, bar(L::kBarQ), c * 64, q0, bh);
        tma_load_3d(sb + L::kOffdO + c * kBox, &tmdO, bar(L::kBarQ), c * 64, q0, bh);
      }
      int nb = 0;
      bool ok = true;
      for (int j = 0; ok && j < n; ++j) {
        for (int e = 0; e < 10; ++e, ++nb) {
          const bool is_k = e < 4 || e >= 8;
          const int col = e < 4 ? e : e < 8 ? e - 4 : 2 * h + e - 8;
          if (!(ok = ring_load(sb + L::kOffRing, bar(L::kBarFull), bar(L::kBarEmpty), nb, is_k ? &tmK : &tmV,
                               col * 64, j * 128, bh, abort_flag)))
            break;
        }
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      mbar_wait_drain(bar(L::kBarQ), 0);
      ring_drain(bar(L::kBarFull), nb);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_16(128, 128, false, false, F16);   // S, dP: K-major A and B
      constexpr uint32_t kIdAcc = idesc_16(128, 128, false, true, F16);  // dQ_h: A in TMEM, B MN-major
      auto full = [&](int b) { return bar(L::kBarFull + b % kRing); };
      auto empty = [&](int b) { return bar(L::kBarEmpty + b % kRing); };
      auto issue_full_depth = [&](uint32_t dcol, uint32_t a_tile, int b0) -> bool {
        for (int c = 0; c < 4; ++c) {
          const int b = b0 + c;
          if (!mbar_wait_spin(full(b), (b / kRing) & 1, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            mma_ss(tmem + dcol, sdesc_sw128(a_tile + c * kBox + k4 * 32, 16, 1024),
                   sdesc_sw128(slot_addr(b) + k4 * 32, 16, 1024), kIdS, (c | k4) ? 1u : 0u);
          tc_commit(empty(b));
        }
        return true;
      };
      bool ok = mbar_wait_spin(bar(L::kBarQ), 0, abort_flag);
      for (int j = 0; ok && j < n; ++j) {
        const int b0 = 10 * j;
        tc_fence_after();
        if (!(ok = issue_full_depth(kColS, sb + L::kOffQ, b0))) break;         // S = Q K_j^T
        tc_commit(bar(L::kBarS));
        if (!(ok = issue_full_depth(kColDP, sb + L::kOffdO, b0 + 4))) break;   // dP = dO V_j^T
        tc_commit(bar(L::kBarDP));
        if (!(ok = mbar_wait_spin(bar(L::kBarDS), j & 1, abort_flag))) break;
        const int b = b0 + 8;                                                 // K_j columns [128h, 128h+128)
        if (!(ok = mbar_wait_spin(full(b), (b / kRing) & 1, abort_flag))) break;
        if (!(ok = mbar_wait_spin(full(b + 1), ((b + 1) / kRing) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)                                        // dQ_h += dS K_j[:, h]
          mma_ts(tmem + kColDQ, tmem + packed_col(kColDP, kk), sdesc_sw128(slot_addr(b) + kk * 2048, kBox, 1024),
                 kIdAcc, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(empty(b));
        tc_commit(empty(b + 1));
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      tc_commit(bar(L::kBarAcc));
      tc_commit(bar(L::kBarMmaDone));
      mbar_wait_drain(bar(L::kBarMmaDone), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ P, dS (32 key columns), epilogue
    const int w = (warp - 4) >> 2;                                      // key columns [32w, 32w+32)
    const int r = threadIdx.x - 128 * (1 + w);                          // query row = TMEM lane
    const uint32_t tb = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int qrow = q0 + r;
    const size_t prow = static_cast<size_t>(bh) * Npad + qrow;         // < B*H*Npad: q0 < N <= Npad
    const bool pin = FA_BOUNDS(prow < static_cast<size_t>(BH) * Npad, status);
    const float nl = pin ? ws_nl[prow] : -CUDART_INF_F;
    const float dl = pin ? ws_delta[prow] : 0.f;
    const float scale_log2 = scale * kLog2e;
    const float2 sl2 = make_float2(scale_log2, scale_log2), nl2 = make_float2(nl, nl);
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int kc0 = j * 128 + 32 * w;                                 // key of this thread's column 0
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS), j & 1, abort_flag));
      if (!ok) break;
      FA_CONVERGED(status);                                     // warp-collective TMEM loads follow
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tb + kColS + 32 * w, sr);
      tmem_ld_wait();
      reg_fence(sr);
      // keep key columns c <= lim (causal diagonal, keys past N)
      const int lim = min(CAUSAL ? qrow - kc0 : 31, N - 1 - kc0);
      const bool edge = __any_sync(0xffffffffu, lim < 31);              // warp-uniform
      uint32_t pk[16];
      auto p_phase = [&](auto masked) {
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) {
          const int c = 2 * c2;
          const float2 sv = make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
          float2 p = exp2_pair(__ffma2_rn(sv, sl2, nl2), poly_pair(c2));
          if (decltype(masked)::value) {
            if (c > lim) p.x = 0.f;
            if (c + 1 > lim) p.y = 0.f;
          }
          pk[c2] = pack16<F16>(p.x, p.y);
        }
      };
      if (edge) p_phase(std::true_type{});
      else p_phase(std::false_type{});
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP), j & 1, abort_flag));
      if (!ok) break;
      FA_CONVERGED(status);
      tc_fence_after();
      uint32_t dp[32];
      tmem_ld32(tb + kColDP + 32 * w, dp);
      tmem_ld_wait();
      reg_fence(dp);
      uint32_t dsk[16];
#pragma unroll
      for (int c2 = 0; c2 < 16; ++c2) {
        const float2 ds = __fmul2_rn(make_float2(unpack16_lo<F16>(pk[c2]), unpack16_hi<F16>(pk[c2])),
                                     __ffma2_rn(make_float2(dl, dl), make_float2(-1.f, -1.f),
                                                make_float2(__uint_as_float(dp[2 * c2]), __uint_as_float(dp[2 * c2 + 1]))));
        dsk[c2] = pack16<F16>(ds.x, ds.y);
      }
      tmem_st16(tb + kColDP + 32 * w, dsk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarDS));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarAcc), 0, abort_flag));
    if (!ok) {
      raise_error(status, abort_flag, kStatusTimeout);
    } else if (w < 2) {
      // dQ_h box w (64 columns) via the idle Q tile; global columns 128h + 64w
      FA_CONVERGED(status);
      tc_fence_after();
      stage_box_16<128, F16>(tb + kColDQ, w, scale, smem + L::kOffQ, r);
      store_warp_box_x(&tmdQ, sb + L::kOffQ, w, 2 * h + w, (warp & 3) * 32, q0, bh, lane, N);
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
cudaError_t dkdv_impl(const BwdLaunch& a, cudaStream_t stream) {
  auto kern = bwd_dkdv_d256_kernel<CAUSAL, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DkdvD256Smem::kBytes);
  if (e != cudaSuccess) return e;
  const int nkt = (a.N + 127) / 128;
  kern<<<2u * static_cast<unsigned>(nkt) * a.BH, kThreads, DkdvD256Smem::kBytes, stream>>>(
      a.tmQ, a.tmK, a.tmV, a.tmdO, a.tmdK, a.tmdV, a.ws_nl, a.ws_delta, a.N, a.Npad, a.BH, nkt, a.scale, a.status);
  return cudaGetLastError();
}

template <bool CAUSAL, bool F16>
cudaError_t dq_impl(const BwdLaunch& a, cudaStream_t stream) {
  auto kern = bwd_dq_d256_kernel<CAUSAL, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DqD256Smem::kBytes);
  if (e != cudaSuccess) return e;
  const int nqt = (a.N + 127) / 128;
  kern<<<2u * static_cast<unsigned>(nqt) * a.BH, kThreads, DqD256Smem::kBytes, stream>>>(
      a.tmQ, a.tmK, a.tmV, a.tmdO, a.tmdQ, a.ws_nl, a.ws_delta, a.N, a.Npad, a.BH, nqt, a.scale, a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dkdv_d256(const BwdLaunch& a, cudaStream_t stream) {
  if (a.f16) return a.causal ? dkdv_impl<true, true>(a, stream) : dkdv_impl<false, true>(a, stream);
  return a.causal ? dkdv_impl<true, false>(a, stream) : dkdv_impl<false, false>(a, stream);
}

cudaError_t launch_bwd_dq_d256(const BwdLaunch& a, cudaStream_t stream) {
  if (a.f16) return a.causal ? dq_impl<true, true>(a, stream) : dq_impl<false, true>(a, stream);
  return a.causal ? dq_impl<true, false>(a, stream) : dq_impl<false, false>(a, stream);
}

}  // namespace fa
