// fa_bwd_sm100.cu -- bf16 attention backward on the sm_100a tensor cores.
//
// The backward never stores P: it recomputes it from the saved logsumexp, as
// "LLM paper notes #8: FlashAttention" (adg.csdn.net), section "recomputation",
// and "CUDA-kernel-level optimisation: why Flash Attention is 5-10x faster than
// native PyTorch" (guanweilu.cn), section "three tricks", describe.  With scaled
// scores s = scale * q.k, P_ij = exp(s_ij - lse_i), and L a scalar loss:
//     dV = P^T dO,   dP = dO V^T,   delta_i = sum_d dO_id O_id,
//     dS = P * (dP - delta),   dQ = scale * dS K,   dK = scale * dS^T Q.
//
// Three stages, all on the caller's stream:
//   1. preprocess   delta = rowsum(dO * O) in fp32 (bandwidth bound)
//   2. dkdv kernel  one CTA per 128-key tile j walks the query tiles i:
//                     S^T = K_j Q_i^T, dP^T = V_j dO_i^T           (tensor memory)
//                     P^T, dS^T computed by 128 threads, one key row each
//                     dV_j += P^T dO_i, dK_j += dS^T Q_i             (A from tensor memory)
//   3. dq kernel    one CTA per 128-query tile i walks the key tiles j:
//                     S = Q_i K_j^T, dP = dO_i V_j^T, dS, dQ_i += dS K_j
// Every output tile is owned by exactly one CTA, so there are no atomics, no
// fp32 dQ accumulator in device memory and the result is deterministic; the
// price is recomputing S and dP a second time in stage 3.
//
// The probabilities used for dS are the bf16-rounded P that also feeds dV.
#include <cstdint>
#include <math_constants.h>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kTileRows = 128;
constexpr int kThreads = 256;           // warp 0 loads, warp 1 issues MMAs, warps 4-7 compute
constexpr float kLog2e = 1.44269504088896340736f;

// ----------------------------------------------------------------------------- stage 1
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o,
                                                             const __nv_bfloat16* __restrict__ dO,
                                                             float* __restrict__ delta, long long rows) {
  constexpr int kLanesPerRow = D / 8;   // each lane reads 8 bf16 (16 bytes) of O and of dO
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gt / kLanesPerRow;
  const int part = static_cast<int>(gt % kLanesPerRow);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + row * D + part * 8);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(av[i] << 16), __uint_as_float(bv[i] << 16), acc);
      acc = fmaf(__uint_as_float(av[i] & 0xffff0000u), __uint_as_float(bv[i] & 0xffff0000u), acc);
    }
  }
#pragma unroll
  for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && part == 0) delta[row] = acc;
}

// ----------------------------------------------------------------------------- shared helpers
template <int D>
struct Tiles {
  static constexpr int kBox = kTileRows * 64 * 2;   // 16 KB: 128 rows x 64 bf16, 128-byte swizzle
  static constexpr int kNBox = D / 64;
  static constexpr int kTile = kBox * kNBox;
};

// Copies this thread's accumulator row (D fp32 columns of tensor memory, times `mul`)
// as bf16 into row r of a 128-row staging tile in the TMA 128-byte-swizzled layout.
template <int D>
__device__ __forceinline__ void stage_row_bf16(uint32_t tacc, float mul, uint8_t* stage, int r) {
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32(tacc + cc * 32, o);
    tmem_ld_wait();
    reg_fence(o);
    const int box = cc >> 1;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int chunk = (cc & 1) * 4 + q4;
      uint4 v;
      v.x = pack_bf16(__uint_as_float(o[8 * q4 + 0]) * mul, __uint_as_float(o[8 * q4 + 1]) * mul);
      v.y = pack_bf16(__uint_as_float(o[8 * q4 + 2]) * mul, __uint_as_float(o[8 * q4 + 3]) * mul);
      v.z = pack_bf16(__uint_as_float(o[8 * q4 + 4]) * mul, __uint_as_float(o[8 * q4 + 5]) * mul);
      v.w = pack_bf16(__uint_as_float(o[8 * q4 + 6]) * mul, __uint_as_float(o[8 * q4 + 7]) * mul);
      *reinterpret_cast<uint4*>(stage + box * Tiles<D>::kBox + r * 128 + ((chunk ^ (r & 7)) << 4)) = v;
    }
  }
}

// One warp stores its 32 staged rows with the TMA (tensor map box: 64 x 32 x 1).
template <int D>
__device__ __forceinline__ void store_warp_rows(const CUtensorMap* tm, uint32_t stage_s, int wrow, int row0, int bh,
                                                int lane, int n_rows) {
  fence_async_smem();
  __syncwarp();
  if (lane == 0 && row0 + wrow < n_rows) {
    for (int c = 0; c < Tiles<D>::kNBox; ++c)
      tma_store_3d(tm, stage_s + c * Tiles<D>::kBox + wrow * 128, c * 64, row0 + wrow, bh);
    bulk_commit();
    bulk_wait_read0();
  }
  __syncwarp();
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// ----------------------------------------------------------------------------- stage 2: dK, dV
template <int D>
struct DkdvSmem {
  using T = Tiles<D>;
  static constexpr int kStages = 2;
  static constexpr int kOffK = 0;                          // K_j (later dK staging)
  static constexpr int kOffV = kOffK + T::kTile;           // V_j (later dV staging)
  static constexpr int kOffQ = kOffV + T::kTile;           // [stage] Q_i
  static constexpr int kOffdO = kOffQ + kStages * T::kTile;  // [stage] dO_i
  static constexpr int kOffStat = kOffdO + kStages * T::kTile;  // [stage] -lse*log2e[128], delta[128]
  static constexpr int kOffBar = kOffStat + kStages * 2 * kTileRows * 4;
  static constexpr int kBarKV = 0;
  static constexpr int kBarQFull = 1;
  static constexpr int kBarQEmpty = kBarQFull + kStages;
  static constexpr int kBarS = kBarQEmpty + kStages;
  static constexpr int kBarDP = kBarS + 1;
  static constexpr int kBarP = kBarDP + 1;
  static constexpr int kBarDS = kBarP + 1;
  static constexpr int kBarAcc = kBarDS + 1;
  static constexpr int kBarMmaDone = kBarAcc + 1;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kBytes = (kOffSlot + 16 + 1024) > 122880 ? (kOffSlot + 16 + 1024) : 122880;  // 1 CTA / SM
  static_assert(kBytes <= 232448, "shared memory budget");
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                    const float* __restrict__ lse, const float* __restrict__ delta, int N, int BH, int nt,
                    float scale, int* status) {
  using L = DkdvSmem<D>;
  using T = Tiles<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: key tile kt of head bh.  Causal: it meets query tiles kt..nt-1, so low
  // kt are the heaviest and go first.
  int kt, bh;
  if (CAUSAL) {
    kt = static_cast<int>(blockIdx.x / BH);
    bh = blockIdx.x % BH;
  } else {
    kt = blockIdx.x % nt;
    bh = blockIdx.x / nt;
  }
  const int kv0 = kt * kTileRows;
  const int it0 = CAUSAL ? kt : 0;        // first query tile
  const int n = nt - it0;                 // query tiles visited

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarKV), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kBarQFull + s), 2);   // TMA bytes + the warp's statistics
      mbar_init(bar(L::kBarQEmpty + s), 1);
    }
    mbar_init(bar(L::kBarS), 1);
    mbar_init(bar(L::kBarDP), 1);
    mbar_init(bar(L::kBarP), kTileRows);
    mbar_init(bar(L::kBarDS), kTileRows);
    mbar_init(bar(L::kBarAcc), 1);
    mbar_init(bar(L::kBarMmaDone), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  // Tensor memory: S^T / P^T [0,128), dP^T / dS^T [128,256), dV [256,256+D), dK [256+D,256+2D)
  constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;

  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar(L::kBarKV), 2 * T::kTile);
      for (int c = 0; c < T::kNBox; ++c) {
        tma_load_3d(sb + L::kOffK + c * T::kBox, &tmK, bar(L::kBarKV), c * 64, kv0, bh);
        tma_load_3d(sb + L::kOffV + c * T::kBox, &tmV, bar(L::kBarKV), c * 64, kv0, bh);
      }
    }
    int issued = 0;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int s = i % L::kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarQEmpty + s), ((i / L::kStages) & 1) ^ 1, abort_flag));
      if (!ok) break;
      const int q0 = (it0 + i) * kTileRows;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(L::kBarQFull + s), 2 * T::kTile);
        for (int c = 0; c < T::kNBox; ++c) {
          tma_load_3d(sb + L::kOffQ + s * T::kTile + c * T::kBox, &tmQ, bar(L::kBarQFull + s), c * 64, q0, bh);
          tma_load_3d(sb + L::kOffdO + s * T::kTile + c * T::kBox, &tmdO, bar(L::kBarQFull + s), c * 64, q0, bh);
        }
      }
      // Row statistics of this query tile; rows past N get P = 0 (lse = +inf) and delta = 0.
      float* st = reinterpret_cast<float*>(smem + L::kOffStat + s * 2 * kTileRows * 4);
      for (int c = lane; c < kTileRows; c += 32) {
        const int qrow = q0 + c;
        const bool in = qrow < N;
        st[c] = in ? -lse[static_cast<size_t>(bh) * N + qrow] * kLog2e : -CUDART_INF_F;
        st[kTileRows + c] = in ? delta[static_cast<size_t>(bh) * N + qrow] : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(L::kBarQFull + s));
      ++issued;
    }
    if (lane == 0) {
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      mbar_wait_drain(bar(L::kBarKV), 0);
      for (int i = max(0, issued - L::kStages); i < issued; ++i)
        mbar_wait_drain(bar(L::kBarQFull + i % L::kStages), (i / L::kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(kTileRows, kTileRows, false, false);
      constexpr uint32_t kIdAcc = idesc_bf16(kTileRows, D, false, true);
      const uint32_t sK = sb + L::kOffK, sV = sb + L::kOffV;
      // S^T = K_j Q_i^T and dP^T = V_j dO_i^T (both operands K-major)
      auto issue_st = [&](int i) {
        const uint32_t sQ = sb + L::kOffQ + (i % L::kStages) * T::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * T::kBox + (kk & 3) * 32;
          mma_ss(tmem + kColS, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024), kIdS, kk > 0);
        }
        tc_commit(bar(L::kBarS));
      };
      auto issue_dpt = [&](int i) {
        const uint32_t sdO = sb + L::kOffdO + (i % L::kStages) * T::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * T::kBox + (kk & 3) * 32;
          mma_ss(tmem + kColDP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sdO + off, 16, 1024), kIdS, kk > 0);
        }
        tc_commit(bar(L::kBarDP));
      };
      // acc (+)= A_tmem [128 x 128 queries] * B_smem (queries x D, MN-major)
      auto issue_acc = [&](uint32_t dcol, uint32_t acol, uint32_t b_tile, int i) {
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk)
          mma_ts(tmem + dcol, tmem + acol + kk * 8, sdesc_sw128(b_tile + kk * 2048, T::kBox, 1024), kIdAcc,
                 (i > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar(L::kBarKV), 0, abort_flag);
      for (int i = 0; ok && i < n; ++i) {
        const int s = i % L::kStages;
        if (i == 0) {
          if (!(ok = mbar_wait(bar(L::kBarQFull), 0, abort_flag))) break;
          tc_fence_after();
          issue_st(0);
          issue_dpt(0);
        }
        if (!(ok = mbar_wait(bar(L::kBarP), i & 1, abort_flag))) break;
        tc_fence_after();
        issue_acc(kColDV, kColS, sb + L::kOffdO + s * T::kTile, i);          // dV += P^T dO_i
        if (i + 1 < n) {
          const int sn = (i + 1) % L::kStages;
          if (!(ok = mbar_wait(bar(L::kBarQFull + sn), ((i + 1) / L::kStages) & 1, abort_flag))) break;
          tc_fence_after();
          issue_st(i + 1);
        }
        if (!(ok = mbar_wait(bar(L::kBarDS), i & 1, abort_flag))) break;
        tc_fence_after();
        issue_acc(kColDK, kColDP, sb + L::kOffQ + s * T::kTile, i);          // dK += dS^T Q_i
        tc_commit(bar(L::kBarQEmpty + s));
        if (i + 1 < n) issue_dpt(i + 1);
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      tc_commit(bar(L::kBarAcc));
      tc_commit(bar(L::kBarMmaDone));
      mbar_wait_drain(bar(L::kBarMmaDone), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ P^T, dS^T, epilogue
    const int r = threadIdx.x - 128;                                    // key row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tb = tmem + lane_off;
    const int key = kv0 + r;
    const float scale_log2 = scale * kLog2e;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int s = i % L::kStages;
      const int q0 = (it0 + i) * kTileRows;
      const float* st = reinterpret_cast<const float*>(smem + L::kOffStat + s * 2 * kTileRows * 4);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarQFull + s), (i / L::kStages) & 1, abort_flag));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS), i & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
      tmem_ld32(tb + kColS, sr[0]);
      tmem_ld32(tb + kColS + 32, sr[1]);
      tmem_ld32(tb + kColS + 64, sr[2]);
      tmem_ld32(tb + kColS + 96, sr[3]);
      tmem_ld_wait();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      reg_fence(sr[2]);
      reg_fence(sr[3]);
      // P^T[r][c] = exp2(s * scale * log2e - lse_c * log2e); causal: zero where key > query
      const bool diag = CAUSAL && (q0 < kv0 + kTileRows);
      uint32_t pk[2][32];
#pragma unroll
      for (int c2 = 0; c2 < kTileRows / 2; ++c2) {
        const int c = 2 * c2;
        const float4 nl = *reinterpret_cast<const float4*>(st + (c & ~3));
        const float nl0 = (c & 2) ? nl.z : nl.x, nl1 = (c & 2) ? nl.w : nl.y;
        float p0 = ex2_approx(fmaf(__uint_as_float(sr[c >> 5][c & 31]), scale_log2, nl0));
        float p1 = ex2_approx(fmaf(__uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]), scale_log2, nl1));
        if (diag) {
          if (key > q0 + c) p0 = 0.f;
          if (key > q0 + c + 1) p1 = 0.f;
        }
        pk[c2 >> 5][c2 & 31] = pack_bf16(p0, p1);
      }
      tmem_st32(tb + kColS, pk[0]);
      tmem_st32(tb + kColS + 32, pk[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarP));
      // dS^T[r][c] = P^T[r][c] * (dP^T[r][c] - delta_c)
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP), i & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t dsk[2][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t dp[32];
        tmem_ld32(tb + kColDP + cc * 32, dp);
        tmem_ld_wait();
        reg_fence(dp);
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const int c2 = cc * 16 + h;          // packed column
          const int c = 2 * c2;
          const float4 dl = *reinterpret_cast<const float4*>(st + kTileRows + (c & ~3));
          const float d0 = (c & 2) ? dl.z : dl.x, d1 = (c & 2) ? dl.w : dl.y;
          const uint32_t pp = pk[c2 >> 5][c2 & 31];
          const float ds0 = bf16_lo(pp) * (__uint_as_float(dp[2 * h]) - d0);
          const float ds1 = bf16_hi(pp) * (__uint_as_float(dp[2 * h + 1]) - d1);
          dsk[c2 >> 5][c2 & 31] = pack_bf16(ds0, ds1);
        }
      }
      tmem_st32(tb + kColDP, dsk[0]);
      tmem_st32(tb + kColDP + 32, dsk[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarDS));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarAcc), 0, abort_flag));
    if (!ok) {
      raise_error(status, abort_flag, kStatusTimeout);
    } else {
      tc_fence_after();
      const int wrow = (warp & 3) * 32;
      stage_row_bf16<D>(tb + kColDV, 1.f, smem + L::kOffV, r);
      store_warp_rows<D>(&tmdV, sb + L::kOffV, wrow, kv0, bh, lane, N);
      stage_row_bf16<D>(tb + kColDK, scale, smem + L::kOffK, r);
      store_warp_rows<D>(&tmdK, sb + L::kOffK, wrow, kv0, bh, lane, N);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------------------- stage 3: dQ
template <int D>
struct DqSmem {
  using T = Tiles<D>;
  static constexpr int kStages = 2;
  static constexpr int kOffQ = 0;                              // Q_i (later dQ staging)
  static constexpr int kOffdO = kOffQ + T::kTile;
  static constexpr int kOffK = kOffdO + T::kTile;              // [stage] K_j
  static constexpr int kOffV = kOffK + kStages * T::kTile;     // [stage] V_j
  static constexpr int kOffBar = kOffV + kStages * T::kTile;
  static constexpr int kBarQ = 0;
  static constexpr int kBarKVFull = 1;
  static constexpr int kBarKVEmpty = kBarKVFull + kStages;
  static constexpr int kBarS = kBarKVEmpty + kStages;
  static constexpr int kBarDP = kBarS + 1;
  static constexpr int kBarDS = kBarDP + 1;
  static constexpr int kBarAcc = kBarDS + 1;
  static constexpr int kBarMmaDone = kBarAcc + 1;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kBytes = (kOffSlot + 16 + 1024) > 122880 ? (kOffSlot + 16 + 1024) : 122880;  // 1 CTA / SM
  static_assert(kBytes <= 232448, "shared memory budget");
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdQ, const float* __restrict__ lse,
                  const float* __restrict__ delta, int N, int BH, int nt, float scale, int* status) {
  using L = DqSmem<D>;
  using T = Tiles<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: query tile qt of head bh.  Causal: it meets key tiles 0..qt, so high
  // qt are the heaviest and go first.
  int qt, bh;
  if (CAUSAL) {
    qt = nt - 1 - static_cast<int>(blockIdx.x / BH);
    bh = blockIdx.x % BH;
  } else {
    qt = blockIdx.x % nt;
    bh = blockIdx.x / nt;
  }
  const int q0 = qt * kTileRows;
  const int n = CAUSAL ? qt + 1 : nt;     // key tiles visited

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarQ), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kBarKVFull + s), 1);
      mbar_init(bar(L::kBarKVEmpty + s), 1);
    }
    mbar_init(bar(L::kBarS), 1);
    mbar_init(bar(L::kBarDP), 1);
    mbar_init(bar(L::kBarDS), kTileRows);
    mbar_init(bar(L::kBarAcc), 1);
    mbar_init(bar(L::kBarMmaDone), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  // Tensor memory: S / dS [0,128), dP [128,256), dQ [256,256+D)
  constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar(L::kBarQ), 2 * T::kTile);
      for (int c = 0; c < T::kNBox; ++c) {
        tma_load_3d(sb + L::kOffQ + c * T::kBox, &tmQ, bar(L::kBarQ), c * 64, q0, bh);
        tma_load_3d(sb + L::kOffdO + c * T::kBox, &tmdO, bar(L::kBarQ), c * 64, q0, bh);
      }
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        const int s = j % L::kStages;
        if (!(ok = mbar_wait(bar(L::kBarKVEmpty + s), ((j / L::kStages) & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(L::kBarKVFull + s), 2 * T::kTile);
        for (int c = 0; c < T::kNBox; ++c) {
          tma_load_3d(sb + L::kOffK + s * T::kTile + c * T::kBox, &tmK, bar(L::kBarKVFull + s), c * 64,
                      j * kTileRows, bh);
          tma_load_3d(sb + L::kOffV + s * T::kTile + c * T::kBox, &tmV, bar(L::kBarKVFull + s), c * 64,
                      j * kTileRows, bh);
        }
        ++issued;
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      mbar_wait_drain(bar(L::kBarQ), 0);
      for (int j = max(0, issued - L::kStages); j < issued; ++j)
        mbar_wait_drain(bar(L::kBarKVFull + j % L::kStages), (j / L::kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(kTileRows, kTileRows, false, false);
      constexpr uint32_t kIdAcc = idesc_bf16(kTileRows, D, false, true);
      const uint32_t sQ = sb + L::kOffQ, sdO = sb + L::kOffdO;
      auto issue_s_dp = [&](int j) {
        const uint32_t sK = sb + L::kOffK + (j % L::kStages) * T::kTile;
        const uint32_t sV = sb + L::kOffV + (j % L::kStages) * T::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * T::kBox + (kk & 3) * 32;
          mma_ss(tmem + kColS, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024), kIdS, kk > 0);
        }
        tc_commit(bar(L::kBarS));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * T::kBox + (kk & 3) * 32;
          mma_ss(tmem + kColDP, sdesc_sw128(sdO + off, 16, 1024), sdesc_sw128(sV + off, 16, 1024), kIdS, kk > 0);
        }
        tc_commit(bar(L::kBarDP));
      };
      bool ok = mbar_wait(bar(L::kBarQ), 0, abort_flag);
      for (int j = 0; ok && j < n; ++j) {
        const int s = j % L::kStages;
        if (j == 0) {
          if (!(ok = mbar_wait(bar(L::kBarKVFull), 0, abort_flag))) break;
          tc_fence_after();
          issue_s_dp(0);
        }
        if (!(ok = mbar_wait(bar(L::kBarDS), j & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t sK = sb + L::kOffK + s * T::kTile;
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk)                       // dQ += dS K_j
          mma_ts(tmem + kColDQ, tmem + kColS + kk * 8, sdesc_sw128(sK + kk * 2048, T::kBox, 1024), kIdAcc,
                 (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(L::kBarKVEmpty + s));
        if (j + 1 < n) {
          const int sn = (j + 1) % L::kStages;
          if (!(ok = mbar_wait(bar(L::kBarKVFull + sn), ((j + 1) / L::kStages) & 1, abort_flag))) break;
          tc_fence_after();
          issue_s_dp(j + 1);
        }
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      tc_commit(bar(L::kBarAcc));
      tc_commit(bar(L::kBarMmaDone));
      mbar_wait_drain(bar(L::kBarMmaDone), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int r = threadIdx.x - 128;                                    // query row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tb = tmem + lane_off;
    const int qrow = q0 + r;
    const bool row_in = qrow < N;
    const float nlse = row_in ? -lse[static_cast<size_t>(bh) * N + qrow] * kLog2e : -CUDART_INF_F;
    const float dl = row_in ? delta[static_cast<size_t>(bh) * N + qrow] : 0.f;
    const float scale_log2 = scale * kLog2e;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int kv0 = j * kTileRows;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS), j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
      tmem_ld32(tb + kColS, sr[0]);
      tmem_ld32(tb + kColS + 32, sr[1]);
      tmem_ld32(tb + kColS + 64, sr[2]);
      tmem_ld32(tb + kColS + 96, sr[3]);
      tmem_ld_wait();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      reg_fence(sr[2]);
      reg_fence(sr[3]);
      // keep key columns c <= lim (causal diagonal, keys past N)
      const int lim = min(CAUSAL ? qrow - kv0 : kTileRows - 1, N - 1 - kv0);
      const bool edge = (CAUSAL && kv0 + kTileRows - 1 > q0) || (kv0 + kTileRows > N);
      uint32_t pk[2][32];
#pragma unroll
      for (int c2 = 0; c2 < kTileRows / 2; ++c2) {
        const int c = 2 * c2;
        float p0 = ex2_approx(fmaf(__uint_as_float(sr[c >> 5][c & 31]), scale_log2, nlse));
        float p1 = ex2_approx(fmaf(__uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]), scale_log2, nlse));
        if (edge) {
          if (c > lim) p0 = 0.f;
          if (c + 1 > lim) p1 = 0.f;
        }
        pk[c2 >> 5][c2 & 31] = pack_bf16(p0, p1);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP), j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t dsk[2][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t dp[32];
        tmem_ld32(tb + kColDP + cc * 32, dp);
        tmem_ld_wait();
        reg_fence(dp);
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const int c2 = cc * 16 + h;
          const uint32_t pp = pk[c2 >> 5][c2 & 31];
          const float ds0 = bf16_lo(pp) * (__uint_as_float(dp[2 * h]) - dl);
          const float ds1 = bf16_hi(pp) * (__uint_as_float(dp[2 * h + 1]) - dl);
          dsk[c2 >> 5][c2 & 31] = pack_bf16(ds0, ds1);
        }
      }
      tmem_st32(tb + kColS, dsk[0]);
      tmem_st32(tb + kColS + 32, dsk[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarDS));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarAcc), 0, abort_flag));
    if (!ok) {
      raise_error(status, abort_flag, kStatusTimeout);
    } else {
      tc_fence_after();
      stage_row_bf16<D>(tb + kColDQ, scale, smem + L::kOffQ, r);
      store_warp_rows<D>(&tmdQ, sb + L::kOffQ, (warp & 3) * 32, q0, bh, lane, N);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t preprocess_impl(const void* o, const void* dO, float* delta, long long rows, cudaStream_t stream) {
  const long long threads = rows * (D / 8);
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  bwd_preprocess_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), delta, rows);
  return cudaGetLastError();
}

template <int D, bool CAUSAL>
cudaError_t dkdv_impl(const BwdLaunch& a, cudaStream_t stream) {
  using L = DkdvSmem<D>;
  auto kern = bwd_dkdv_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const int nt = (a.N + kTileRows - 1) / kTileRows;
  kern<<<static_cast<unsigned>(nt) * a.BH, kThreads, L::kBytes, stream>>>(
      a.tmQ, a.tmK, a.tmV, a.tmdO, a.tmdK, a.tmdV, a.lse, a.delta, a.N, a.BH, nt, a.scale, a.status);
  return cudaGetLastError();
}

template <int D, bool CAUSAL>
cudaError_t dq_impl(const BwdLaunch& a, cudaStream_t stream) {
  using L = DqSmem<D>;
  auto kern = bwd_dq_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const int nt = (a.N + kTileRows - 1) / kTileRows;
  kern<<<static_cast<unsigned>(nt) * a.BH, kThreads, L::kBytes, stream>>>(
      a.tmQ, a.tmK, a.tmV, a.tmdO, a.tmdQ, a.lse, a.delta, a.N, a.BH, nt, a.scale, a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_preprocess(const void* o, const void* dO, float* delta, long long rows, int D,
                                  cudaStream_t stream) {
  return D == 64 ? preprocess_impl<64>(o, dO, delta, rows, stream) : preprocess_impl<128>(o, dO, delta, rows, stream);
}

cudaError_t launch_bwd_dkdv(const BwdLaunch& a, cudaStream_t stream) {
  if (a.D == 64) return a.causal ? dkdv_impl<64, true>(a, stream) : dkdv_impl<64, false>(a, stream);
  return a.causal ? dkdv_impl<128, true>(a, stream) : dkdv_impl<128, false>(a, stream);
}

cudaError_t launch_bwd_dq(const BwdLaunch& a, cudaStream_t stream) {
  if (a.D == 64) return a.causal ? dq_impl<64, true>(a, stream) : dq_impl<64, false>(a, stream);
  return a.causal ? dq_impl<128, true>(a, stream) : dq_impl<128, false>(a, stream);
}

}  // namespace fa
