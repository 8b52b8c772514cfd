// fa_bwd_sm100.cu -- bf16 / fp16 attention backward on the sm_100a tensor cores.
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
//   1. preprocess   per row: delta = rowsum(dO * O) and nl = -lse * log2(e), both fp32,
//                   into a workspace padded per head to a multiple of 128 rows
//                   (padding rows: nl = -inf so their P is 0, delta = 0)
//   2. dkdv kernel  one CTA per 128-key tile walks the query tiles (128 rows):
//                     S^T = K_j Q_i^T, dP^T = V_j dO_i^T      (M=128 keys, N=128 queries)
//                     P^T, dS^T computed by 512 threads (a key row, a quarter of the queries each)
//                     dV_j += P^T dO_i, dK_j += dS^T Q_i        (A operand read from TMEM)
//                   S^T of the next query tile is computed while dS^T of this one is.
//   3. dq kernel    one CTA per 256 queries (two 128-row tiles) walks the key tiles:
//                     S = Q_i K_j^T, P, dP = dO_i V_j^T (written over S once S is
//                     read), dS, dQ_i += dS K_j
// Every output tile is owned by exactly one CTA: no atomics, no fp32 dQ accumulator
// in device memory, deterministic results; the price is recomputing S and dP in
// stage 3.  The probabilities used for dS are the 16-bit-rounded P that also feed dV.
// All 16-bit operands (inputs, P, dS, outputs) take the inputs' element type: bf16,
// or fp16 when the kernels' F16 parameter is set.
#include <cstdint>
#include <math_constants.h>
#include <type_traits>

#include "bwd_common.cuh"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

// ----------------------------------------------------------------------------- stage 1
// kLanesPerRow lanes per row (a power of two, 8 * kLanesPerRow >= D), each reading 8
// values (16 bytes) of O and of dO; lanes past the row's D columns read nothing.
template <int kLanesPerRow, bool F16>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const uint16_t* __restrict__ o,
                                                             const uint16_t* __restrict__ dO,
                                                             const float* __restrict__ lse,
                                                             float* __restrict__ ws_nl, float* __restrict__ ws_delta,
                                                             float* __restrict__ ws_dq, int N, int Npad, int D, int DK,
                                                             long long padded_rows, int* status) {
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long prow = gt / kLanesPerRow;          // row in the padded (B*H, Npad) layout
  const int part = static_cast<int>(gt % kLanesPerRow);
  const long long bh = prow / Npad;
  const int n = static_cast<int>(prow % Npad);
  const bool real = prow < padded_rows && n < N;
  const long long row = bh * N + n;                  // row in the caller's (B*H, N) layout
  float acc = 0.f;
  const long long rows = padded_rows / Npad * N;       // B*H*N: rows of O, dO and lse
  (void)rows;
  if (real && part * 8 < D && FA_BOUNDS(row < rows && (row * D + part * 8 + 8) <= rows * D, status)) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + row * D + part * 8);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(unpack16_lo<F16>(av[i]), unpack16_lo<F16>(bv[i]), acc);
      acc = fmaf(unpack16_hi<F16>(av[i]), unpack16_hi<F16>(bv[i]), acc);
    }
  }
#pragma unroll
  for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (prow < padded_rows && part == 0) {
    ws_delta[prow] = acc;
    ws_nl[prow] = (real && FA_BOUNDS(row < rows, status)) ? -lse[row] * kLog2e : -CUDART_INF_F;
  }
  // The fused backward adds dQ into an fp32 accumulator of DK floats per padded row: zero
  // this row's share of it (the accumulator's tile layout keeps a row's DK floats
  // contiguous only per tile, but zeroing [prow * DK, prow * DK + DK) over all rows covers it).
  if (ws_dq != nullptr && prow < padded_rows &&
      FA_BOUNDS(prow * DK + (part + 1) * (DK / kLanesPerRow) <= padded_rows * DK, status)) {
    const int per_lane = DK / kLanesPerRow;             // 8 or 16 floats
    float4* z = reinterpret_cast<float4*>(ws_dq + prow * DK + part * per_lane);
    for (int i = 0; i < per_lane / 4; ++i) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ----------------------------------------------------------------------------- stage 2: dK, dV
// One CTA per 128-key tile walks the query tiles (128 rows each).  Every MMA is
// M=128 x N=128 (or N=D): S^T and dP^T (shared-memory operands), dV and dK (A from
// tensor memory).  Four warpgroups split the 128 query columns of S^T / dP^T (32
// each); each writes its 16 columns of packed 16-bit P^T / dS^T into the first half of
// its own (already read) column range, and the K-step addresses of the dV / dK MMAs
// stitch the four quarters back together.
// Q and dO have separate 2-stage rings, each released right after its last use.
template <int D>
struct DkdvSmem {
  using T = Tile<D, 128>;
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kOffK = 0;                                 // K_j (later dK staging)
  static constexpr int kOffV = kOffK + T::kBytes;                 // V_j (later dV staging)
  static constexpr int kOffQ = kOffV + T::kBytes;                 // [stage] Q_i
  static constexpr int kOffdO = kOffQ + kStages * T::kBytes;      // [stage] dO_i
  static constexpr int kOffStat = kOffdO + kStages * T::kBytes;   // [stage] nl[128], delta[128]
  static constexpr int kStatBytes = 2 * 128 * 4;
  static constexpr int kOffBar = kOffStat + kStages * kStatBytes;
  static constexpr int kBarKV = 0;
  static constexpr int kBarQFull = 1;
  static constexpr int kBarQEmpty = kBarQFull + kStages;
  static constexpr int kBarOFull = kBarQEmpty + kStages;
  static constexpr int kBarOEmpty = kBarOFull + kStages;
  static constexpr int kBarS = kBarOEmpty + kStages;
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


template <int D, bool CAUSAL, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                    const float* __restrict__ ws_nl, const float* __restrict__ ws_delta, int N, int Npad, int BH,
                    int nkt, float scale, int* status) {
  using L = DkdvSmem<D>;
  using T = Tile<D, 128>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: key tile kt of head bh.  Causal: it meets query tiles kt..nkt-1, so
  // low kt are the heaviest and go first.
  int kt, bh;
  if (CAUSAL) {
    kt = static_cast<int>(blockIdx.x / BH);
    bh = blockIdx.x % BH;
  } else {
    kt = blockIdx.x % nkt;
    bh = blockIdx.x / nkt;
  }
  const int kv0 = kt * 128;
  const int it0 = CAUSAL ? kt : 0;        // first query tile
  const int n = nkt - it0;                // query tiles visited

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarKV), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bar(L::kBarQFull + s), 1);
      mbar_init(bar(L::kBarQEmpty + s), 1);
      mbar_init(bar(L::kBarOFull + s), 1);
      mbar_init(bar(L::kBarOEmpty + s), 1);
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
  // Tensor memory: S^T / P^T [0,128), dP^T / dS^T [128,256), dV [256,256+D), dK [256+D,256+2D).
  constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;

  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar(L::kBarKV), 2 * T::kBytes);
      for (int c = 0; c < T::kNBox; ++c) {
        tma_load_3d(sb + L::kOffK + c * T::kBox, &tmK, bar(L::kBarKV), c * 64, kv0, bh);
        tma_load_3d(sb + L::kOffV + c * T::kBox, &tmV, bar(L::kBarKV), c * 64, kv0, bh);
      }
      int nq = 0, no = 0;
      bool ok = true;
      // Q_i (with the tile's row statistics) and dO_i, interleaved; each waits for its own ring.
      for (int i = 0; i < n; ++i) {
        const int s = i % L::kStages;
        const uint32_t ph = ((i / L::kStages) & 1) ^ 1;
        const int q0 = (it0 + i) * 128;
        if (!(ok = mbar_wait(bar(L::kBarQEmpty + s), ph, abort_flag))) break;
        const uint32_t qf = bar(L::kBarQFull + s);
        const size_t srow = static_cast<size_t>(bh) * Npad + q0;      // padded rows: always in bounds
        const bool stats_in = FA_BOUNDS(srow + 128 <= static_cast<size_t>(BH) * Npad, status);
        mbar_arrive_expect_tx(qf, T::kBytes + (stats_in ? L::kStatBytes : 0));
        for (int c = 0; c < T::kNBox; ++c)
          tma_load_3d(sb + L::kOffQ + s * T::kBytes + c * T::kBox, &tmQ, qf, c * 64, q0, bh);
        if (stats_in) {
          bulk_load(sb + L::kOffStat + s * L::kStatBytes, ws_nl + srow, 128 * 4, qf);
          bulk_load(sb + L::kOffStat + s * L::kStatBytes + 128 * 4, ws_delta + srow, 128 * 4, qf);
        }
        ++nq;
        if (!(ok = mbar_wait(bar(L::kBarOEmpty + s), ph, abort_flag))) break;
        const uint32_t of = bar(L::kBarOFull + s);
        mbar_arrive_expect_tx(of, T::kBytes);
        for (int c = 0; c < T::kNBox; ++c)
          tma_load_3d(sb + L::kOffdO + s * T::kBytes + c * T::kBox, &tmdO, of, c * 64, q0, bh);
        ++no;
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      mbar_wait_drain(bar(L::kBarKV), 0);
      for (int i = max(0, nq - L::kStages); i < nq; ++i)
        mbar_wait_drain(bar(L::kBarQFull + i % L::kStages), (i / L::kStages) & 1);
      for (int i = max(0, no - L::kStages); i < no; ++i)
        mbar_wait_drain(bar(L::kBarOFull + i % L::kStages), (i / L::kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_16(128, 128, false, false, F16);  // S^T, dP^T: K-major A and B
      constexpr uint32_t kIdAcc = idesc_16(128, D, false, true, F16);   // dV, dK: A in TMEM, B MN-major
      const uint32_t sK = sb + L::kOffK, sV = sb + L::kOffV;
      auto issue_st = [&](int i) {      // S^T = K_j Q_i^T
        const uint32_t sQ = sb + L::kOffQ + (i % L::kStages) * T::kBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + kColS, kmajor_desc(sK, kk, T::kBox), kmajor_desc(sQ, kk, T::kBox), kIdS, kk > 0);
        tc_commit(bar(L::kBarS));
      };
      auto issue_dpt = [&](int i) {     // dP^T = V_j dO_i^T
        const uint32_t sdO = sb + L::kOffdO + (i % L::kStages) * T::kBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + kColDP, kmajor_desc(sV, kk, T::kBox), kmajor_desc(sdO, kk, T::kBox), kIdS, kk > 0);
        tc_commit(bar(L::kBarDP));
      };
      // acc (+)= A_tmem (packed 16-bit, 128 queries) * B_smem (128 queries x D, MN-major)
      auto issue_acc = [&](uint32_t dcol, uint32_t abase, uint32_t b_tile, bool first) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + dcol, tmem + packed_col(abase, kk), mnmajor_desc(b_tile, kk, T::kBox), kIdAcc,
                 (!first || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait_spin(bar(L::kBarKV), 0, abort_flag);
      if (ok && n > 0) {
        ok = mbar_wait_spin(bar(L::kBarQFull), 0, abort_flag) && mbar_wait_spin(bar(L::kBarOFull), 0, abort_flag);
        if (ok) {
          tc_fence_after();
          issue_st(0);
          issue_dpt(0);
        }
      }
      for (int i = 0; ok && i < n; ++i) {
        const int s = i % L::kStages;
        if (!(ok = mbar_wait_spin(bar(L::kBarP), i & 1, abort_flag))) break;
        tc_fence_after();
        issue_acc(kColDV, kColS, sb + L::kOffdO + s * T::kBytes, i == 0);        // dV += P^T dO_i
        tc_commit(bar(L::kBarOEmpty + s));
        if (i + 1 < n) {
          const int sn = (i + 1) % L::kStages;
          if (!(ok = mbar_wait_spin(bar(L::kBarQFull + sn), ((i + 1) / L::kStages) & 1, abort_flag))) break;
          tc_fence_after();
          issue_st(i + 1);                                                       // over P^T_i (read above)
        }
        if (!(ok = mbar_wait_spin(bar(L::kBarDS), i & 1, abort_flag))) break;
        tc_fence_after();
        issue_acc(kColDK, kColDP, sb + L::kOffQ + s * T::kBytes, i == 0);        // dK += dS^T Q_i
        tc_commit(bar(L::kBarQEmpty + s));
        if (i + 1 < n) {
          const int sn = (i + 1) % L::kStages;
          if (!(ok = mbar_wait_spin(bar(L::kBarOFull + sn), ((i + 1) / L::kStages) & 1, abort_flag))) break;
          tc_fence_after();
          issue_dpt(i + 1);                                                      // over dS^T_i (read above)
        }
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
      const int s = i % L::kStages;
      const int q0 = (it0 + i) * 128;
      const float* st = reinterpret_cast<const float*>(smem + L::kOffStat + s * L::kStatBytes) + 32 * g;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarQFull + s), (i / L::kStages) & 1, abort_flag));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS), i & 1, abort_flag));
      if (!ok) break;
      FA_CONVERGED(status);                                     // warp-collective TMEM loads follow
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tb + kColS + 32 * g, sr);
      tmem_ld_wait();
      reg_fence(sr);
      // P^T[r][c] = exp2(s * scale * log2e + nl_c); causal: zero where key > query
      const int qc0 = q0 + 32 * g;                                       // query of this thread's column 0
      // Warp-uniform: whether any lane of this warp has a masked column in this tile.
      const bool diag = CAUSAL && __any_sync(0xffffffffu, qc0 < key + 32);
      // this warpgroup's 32 column statistics, read once (eight 16-byte loads)
      float4 nl4[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) nl4[q] = reinterpret_cast<const float4*>(st)[q];
      uint32_t pk[16];
      // Two copies of the loop so that the common, unmasked tiles carry no mask tests.
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
      // dS^T[r][c] = P^T[r][c] * (dP^T[r][c] - delta_c)
      ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP), i & 1, abort_flag));
      if (!ok) break;
      FA_CONVERGED(status);
      tc_fence_after();
      uint32_t dp[32];
      tmem_ld32(tb + kColDP + 32 * g, dp);
      tmem_ld_wait();
      reg_fence(dp);
      float4 dl4[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) dl4[q] = reinterpret_cast<const float4*>(st + 128)[q];
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
      // One 64-column box per warpgroup: dV boxes into the V tile, dK boxes into the K tile.
      FA_CONVERGED(status);
      tc_fence_after();
      const int wrow = (warp & 3) * 32;
      const int nbox = T::kNBox;                                         // 1 (D=64) or 2 (D=128)
      if (g < 2 * nbox) {
        const bool is_dv = g < nbox;
        const int box = is_dv ? g : g - nbox;
        stage_box_16<D, F16>(tb + (is_dv ? kColDV : kColDK), box, is_dv ? 1.f : scale,
                          smem + (is_dv ? L::kOffV : L::kOffK), r);
        store_warp_box<D>(is_dv ? &tmdV : &tmdK, sb + (is_dv ? L::kOffV : L::kOffK), box, wrow, kv0, bh, lane, N);
      }
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

// ----------------------------------------------------------------------------- stage 3: dQ
template <int D>
struct DqSmem {
  using T = Tile<D, 128>;
  static constexpr int kKStages = 2;
  static constexpr int kVStages = (D == 128) ? 1 : 2;
  static constexpr int kOffQ = 0;                                // Q_0, Q_1 (later dQ staging)
  static constexpr int kOffdO = kOffQ + 2 * T::kBytes;           // dO_0, dO_1
  static constexpr int kOffK = kOffdO + 2 * T::kBytes;           // [K stage]
  static constexpr int kOffV = kOffK + kKStages * T::kBytes;     // [V stage]
  static constexpr int kOffBar = kOffV + kVStages * T::kBytes;
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarS = kBarVEmpty + kVStages;   // [2]
  static constexpr int kBarSC = kBarS + 2;              // [2] S read by the softmax
  static constexpr int kBarDP = kBarSC + 2;             // [2]
  static constexpr int kBarDS = kBarDP + 2;             // [2]
  static constexpr int kBarAcc = kBarDS + 2;            // [2]
  static constexpr int kBarMmaDone = kBarAcc + 2;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  static constexpr int kBytes = (kOffSlot + 16 + 1024) > 122880 ? (kOffSlot + 16 + 1024) : 122880;  // 1 CTA / SM
  static_assert(kBytes <= 232448, "shared memory budget");
};

template <int D, bool CAUSAL, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdQ, const float* __restrict__ ws_nl,
                  const float* __restrict__ ws_delta, int N, int Npad, int BH, int nqb, float scale, int* status) {
  using L = DqSmem<D>;
  using T = Tile<D, 128>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: 256 queries (two 128-row tiles) of head bh.  Causal: heaviest first.
  int qblk, bh;
  if (CAUSAL) {
    qblk = nqb - 1 - static_cast<int>(blockIdx.x / BH);
    bh = blockIdx.x % BH;
  } else {
    qblk = blockIdx.x % nqb;
    bh = blockIdx.x / nqb;
  }
  const int nkt = (N + 127) / 128;
  int q0[2], nk[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    q0[t] = qblk * 256 + t * 128;
    nk[t] = (q0[t] >= N) ? 0 : (CAUSAL ? min(nkt, q0[t] / 128 + 1) : nkt);
  }
  const int nmax = max(nk[0], nk[1]);

  if (threadIdx.x == 0) {
    mbar_init(bar(L::kBarQ), 1);
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(bar(L::kBarKFull + s), 1);
      mbar_init(bar(L::kBarKEmpty + s), 1);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(bar(L::kBarVFull + s), 1);
      mbar_init(bar(L::kBarVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::kBarS + t), 1);
      mbar_init(bar(L::kBarSC + t), 256);
      mbar_init(bar(L::kBarDP + t), 1);
      mbar_init(bar(L::kBarDS + t), 256);
      mbar_init(bar(L::kBarAcc + t), 1);
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
  // Tensor memory: S_t, then dP_t, then dS_t (16-bit, first 64 columns) at 128t; dQ_t at 256 + D t.

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      uint32_t qbytes = 0;
      for (int t = 0; t < 2; ++t)
        if (nk[t] > 0) qbytes += 2 * T::kBytes;
      mbar_arrive_expect_tx(bar(L::kBarQ), qbytes);
      for (int t = 0; t < 2; ++t)
        if (nk[t] > 0)
          for (int c = 0; c < T::kNBox; ++c) {
            tma_load_3d(sb + L::kOffQ + t * T::kBytes + c * T::kBox, &tmQ, bar(L::kBarQ), c * 64, q0[t], bh);
            tma_load_3d(sb + L::kOffdO + t * T::kBytes + c * T::kBox, &tmdO, bar(L::kBarQ), c * 64, q0[t], bh);
          }
      int nkl = 0, nvl = 0;
      bool ok = true;
      for (int j = 0; j < nmax; ++j) {
        const int ks = j % L::kKStages, vs = j % L::kVStages;
        if (!(ok = mbar_wait(bar(L::kBarKEmpty + ks), ((j / L::kKStages) & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(L::kBarKFull + ks), T::kBytes);
        for (int c = 0; c < T::kNBox; ++c)
          tma_load_3d(sb + L::kOffK + ks * T::kBytes + c * T::kBox, &tmK, bar(L::kBarKFull + ks), c * 64, j * 128, bh);
        ++nkl;
        if (!(ok = mbar_wait(bar(L::kBarVEmpty + vs), ((j / L::kVStages) & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(L::kBarVFull + vs), T::kBytes);
        for (int c = 0; c < T::kNBox; ++c)
          tma_load_3d(sb + L::kOffV + vs * T::kBytes + c * T::kBox, &tmV, bar(L::kBarVFull + vs), c * 64, j * 128, bh);
        ++nvl;
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      mbar_wait_drain(bar(L::kBarQ), 0);
      for (int j = max(0, nkl - L::kKStages); j < nkl; ++j)
        mbar_wait_drain(bar(L::kBarKFull + j % L::kKStages), (j / L::kKStages) & 1);
      for (int j = max(0, nvl - L::kVStages); j < nvl; ++j)
        mbar_wait_drain(bar(L::kBarVFull + j % L::kVStages), (j / L::kVStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_16(128, 128, false, false, F16);
      constexpr uint32_t kIdAcc = idesc_16(128, D, false, true, F16);
      // S_t = Q_t K_j^T into region t
      auto issue_s = [&](int t, int j) {
        const uint32_t sQ = sb + L::kOffQ + t * T::kBytes;
        const uint32_t sK = sb + L::kOffK + (j % L::kKStages) * T::kBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 128 * t, kmajor_desc(sQ, kk, T::kBox), kmajor_desc(sK, kk, T::kBox), kIdS, kk > 0);
        tc_commit(bar(L::kBarS + t));
      };
      bool ok = mbar_wait_spin(bar(L::kBarQ), 0, abort_flag);
      if (ok && nmax > 0) {
        ok = mbar_wait_spin(bar(L::kBarKFull), 0, abort_flag);
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (nk[t] > 0) issue_s(t, 0);
        }
      }
      for (int j = 0; ok && j < nmax; ++j) {
        const int ks = j % L::kKStages, vs = j % L::kVStages;
        const uint32_t sV = sb + L::kOffV + vs * T::kBytes;
        const uint32_t sK = sb + L::kOffK + ks * T::kBytes;
        bool v_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {     // dP_t = dO_t V_j^T, over S_t once it has been read
          if (j >= nk[t]) continue;
          if (!(ok = mbar_wait_spin(bar(L::kBarSC + t), j & 1, abort_flag))) break;
          if (!v_ready) {
            if (!(ok = mbar_wait_spin(bar(L::kBarVFull + vs), (j / L::kVStages) & 1, abort_flag))) break;
            v_ready = true;
          }
          tc_fence_after();
          const uint32_t sdO = sb + L::kOffdO + t * T::kBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + 128 * t, kmajor_desc(sdO, kk, T::kBox), kmajor_desc(sV, kk, T::kBox), kIdS, kk > 0);
          tc_commit(bar(L::kBarDP + t));
        }
        if (!ok) break;
        tc_commit(bar(L::kBarVEmpty + vs));
        bool k_next = false;
        for (int t = 0; t < 2 && ok; ++t) {     // dQ_t += dS_t K_j, then S_t for the next key tile
          if (j >= nk[t]) continue;
          if (!(ok = mbar_wait_spin(bar(L::kBarDS + t), j & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)    // dQ += dS K_j; dS half h packed at 64h + [0, 32)
            mma_ts(tmem + 256 + D * t, tmem + 128 * t + 64 * (kk >> 2) + 8 * (kk & 3),
                   mnmajor_desc(sK, kk, T::kBox), kIdAcc, (j > 0 || kk > 0) ? 1u : 0u);
          if (j == nk[t] - 1) tc_commit(bar(L::kBarAcc + t));
          if (j + 1 < nk[t]) {
            if (!k_next) {
              const int jn = j + 1;
              if (!(ok = mbar_wait_spin(bar(L::kBarKFull + jn % L::kKStages), (jn / L::kKStages) & 1, abort_flag)))
                break;
              tc_fence_after();
              k_next = true;
            }
            issue_s(t, j + 1);
          }
        }
        if (!ok) break;
        tc_commit(bar(L::kBarKEmpty + ks));
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      tc_commit(bar(L::kBarMmaDone));
      mbar_wait_drain(bar(L::kBarMmaDone), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // Warpgroup w = 2t + h: query tile t, key columns [64h, 64h+64) of its S / dP region;
    // its packed 16-bit dS goes to columns [64h, 64h+32) of the region.
    const int w = (warp - 4) >> 2, t = w >> 1, h = w & 1;
    const int r = threadIdx.x - 128 * (1 + w);                          // query row = TMEM lane
    const uint32_t tb = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t tR = tb + 128 * t + 64 * h;
    const int qrow = q0[t] + r;
    bool ok = true;
    if (nk[t] > 0) {
      const size_t prow = static_cast<size_t>(bh) * Npad + qrow;       // < B*H*Npad: q0[t] < N <= Npad
      const bool in = FA_BOUNDS(prow < static_cast<size_t>(BH) * Npad, status);
      const float nl = in ? ws_nl[prow] : -CUDART_INF_F;
      const float dl = in ? ws_delta[prow] : 0.f;
      const float scale_log2 = scale * kLog2e;
      for (int j = 0; j < nk[t]; ++j) {
        const int kv0 = j * 128 + 64 * h;                               // key of this thread's column 0
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS + t), j & 1, abort_flag));
        if (!ok) break;
        FA_CONVERGED(status);                                   // warp-collective TMEM loads follow
        tc_fence_after();
        // keep key columns c <= lim (causal diagonal, keys past N)
        const int lim = min(CAUSAL ? qrow - kv0 : 63, N - 1 - kv0);
        // Warp-uniform (the loop below contains warp-collective TMEM loads): whether any
        // lane of this warp has a masked column in this tile.
        const bool edge = __any_sync(0xffffffffu, lim < 63);
        uint32_t pk[32];
        // Two copies of the loop so that the common, unmasked tiles carry no mask tests.
        auto p_phase = [&](auto masked) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t sr[32];
            tmem_ld32(tR + 32 * hh, sr);
            tmem_ld_wait();
            reg_fence(sr);
#pragma unroll
            for (int c2 = 0; c2 < 16; ++c2) {
              const int cl = 2 * c2, c = 32 * hh + cl;
              const float2 sv = make_float2(__uint_as_float(sr[cl]), __uint_as_float(sr[cl + 1]));
              float2 p = exp2_pair(__ffma2_rn(sv, make_float2(scale_log2, scale_log2), make_float2(nl, nl)),
                                   poly_pair(c2));
              if (decltype(masked)::value) {
                if (c > lim) p.x = 0.f;
                if (c + 1 > lim) p.y = 0.f;
              }
              pk[16 * hh + c2] = pack16<F16>(p.x, p.y);
            }
          }
        };
        if (edge) p_phase(std::true_type{});
        else p_phase(std::false_type{});
        tc_fence_before();
        mbar_arrive(bar(L::kBarSC + t));                   // S_t has been read: dP_t may overwrite it
        ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP + t), j & 1, abort_flag));
        if (!ok) break;
        FA_CONVERGED(status);
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t dp[32];
          tmem_ld32(tR + 32 * cc, dp);
          tmem_ld_wait();
          reg_fence(dp);
          uint32_t dsk[16];
#pragma unroll
          for (int h2 = 0; h2 < 16; ++h2) {
            const uint32_t pp = pk[16 * cc + h2];
            const float2 ds = __fmul2_rn(make_float2(unpack16_lo<F16>(pp), unpack16_hi<F16>(pp)),
                                         __ffma2_rn(make_float2(dl, dl), make_float2(-1.f, -1.f),
                                                    make_float2(__uint_as_float(dp[2 * h2]), __uint_as_float(dp[2 * h2 + 1]))));
            dsk[h2] = pack16<F16>(ds.x, ds.y);
          }
          // packed columns [16cc, 16cc+16) of this half lie inside the dP columns already read
          tmem_st16(tR + 16 * cc, dsk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(L::kBarDS + t));
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarAcc + t), 0, abort_flag));
      if (!ok) {
        raise_error(status, abort_flag, kStatusTimeout);
      } else if (h < T::kNBox) {
        // dQ_t box h (64 columns) into the idle Q_t tile, then TMA
        FA_CONVERGED(status);
        tc_fence_after();
        stage_box_16<D, F16>(tb + 256 + D * t, h, scale, smem + L::kOffQ + t * T::kBytes, r);
        store_warp_box<D>(&tmdQ, sb + L::kOffQ + t * T::kBytes, h, (warp & 3) * 32, q0[t], bh, lane, N);
      }
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

template <int kLanesPerRow, bool F16>
cudaError_t preprocess_impl(const BwdLaunch& a, cudaStream_t stream) {
  const long long padded_rows = static_cast<long long>(a.BH) * a.Npad;
  const long long threads = padded_rows * kLanesPerRow;
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  bwd_preprocess_kernel<kLanesPerRow, F16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint16_t*>(a.o), static_cast<const uint16_t*>(a.dO), a.lse, a.ws_nl, a.ws_delta,
      a.ws_dq, a.N, a.Npad, a.D, a.DK, padded_rows, a.status);
  return cudaGetLastError();
}

template <int D, bool CAUSAL, bool F16>
cudaError_t dkdv_impl(const BwdLaunch& a, cudaStream_t stream) {
  using L = DkdvSmem<D>;
  auto kern = bwd_dkdv_kernel<D, CAUSAL, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const int nkt = (a.N + 127) / 128;
  kern<<<static_cast<unsigned>(nkt) * a.BH, kThreads, L::kBytes, stream>>>(
      a.tmQ, a.tmK, a.tmV, a.tmdO, a.tmdK, a.tmdV, a.ws_nl, a.ws_delta, a.N, a.Npad, a.BH, nkt, a.scale, a.status);
  return cudaGetLastError();
}

template <int D, bool CAUSAL, bool F16>
cudaError_t dq_impl(const BwdLaunch& a, cudaStream_t stream) {
  using L = DqSmem<D>;
  auto kern = bwd_dq_kernel<D, CAUSAL, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const int nqb = (a.N + 255) / 256;
  kern<<<static_cast<unsigned>(nqb) * a.BH, kThreads, L::kBytes, stream>>>(
      a.tmQ, a.tmK, a.tmV, a.tmdO, a.tmdQ, a.ws_nl, a.ws_delta, a.N, a.Npad, a.BH, nqb, a.scale, a.status);
  return cudaGetLastError();
}

template <bool F16>
cudaError_t preprocess_typed(const BwdLaunch& a, cudaStream_t stream) {
  if (a.D <= 32) return preprocess_impl<4, F16>(a, stream);
  if (a.D <= 64) return preprocess_impl<8, F16>(a, stream);
  return a.D <= 128 ? preprocess_impl<16, F16>(a, stream) : preprocess_impl<32, F16>(a, stream);
}

template <bool F16>
cudaError_t dkdv_typed(const BwdLaunch& a, cudaStream_t stream) {
  // Head dims 32 and 96 run the 64- and 128-column kernels on zero-filled tile columns
  // (the tensor maps describe the caller's D), as in the forward.
  if (a.D <= 64) return a.causal ? dkdv_impl<64, true, F16>(a, stream) : dkdv_impl<64, false, F16>(a, stream);
  return a.causal ? dkdv_impl<128, true, F16>(a, stream) : dkdv_impl<128, false, F16>(a, stream);
}

template <bool F16>
cudaError_t dq_typed(const BwdLaunch& a, cudaStream_t stream) {
  if (a.D <= 64) return a.causal ? dq_impl<64, true, F16>(a, stream) : dq_impl<64, false, F16>(a, stream);
  return a.causal ? dq_impl<128, true, F16>(a, stream) : dq_impl<128, false, F16>(a, stream);
}

}  // namespace

cudaError_t launch_bwd_preprocess(const BwdLaunch& a, cudaStream_t stream) {
  return a.f16 ? preprocess_typed<true>(a, stream) : preprocess_typed<false>(a, stream);
}

cudaError_t launch_bwd_dkdv(const BwdLaunch& a, cudaStream_t stream) {
  if (a.D == 256) return launch_bwd_dkdv_d256(a, stream);
  return a.f16 ? dkdv_typed<true>(a, stream) : dkdv_typed<false>(a, stream);
}

cudaError_t launch_bwd_dq(const BwdLaunch& a, cudaStream_t stream) {
  if (a.D == 256) return launch_bwd_dq_d256(a, stream);
  return a.f16 ? dq_typed<true>(a, stream) : dq_typed<false>(a, stream);
}

}  // namespace fa
