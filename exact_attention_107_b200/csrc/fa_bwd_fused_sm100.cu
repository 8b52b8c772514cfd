// fa_bwd_fused_sm100.cu -- the attention backward in one pass over the key tiles: dK, dV and dQ.
//
// The backward recomputes P from the saved logsumexp instead of storing it ("LLM paper
// notes #8: FlashAttention", adg.csdn.net, section "recomputation"; "CUDA-kernel-level
// optimisation: why Flash Attention is 5-10x faster than native PyTorch", guanweilu.cn,
// section "three tricks").  With s = scale * q.k and P_ij = exp(s_ij - lse_i):
//     dV = P^T dO,  dP = dO V^T,  dS = P * (dP - delta),  dQ = scale dS K,  dK = scale dS^T Q.
//
// One CTA per 128-key tile j (K_j, V_j resident in shared memory) walks the query tiles i,
// streaming Q_i and dO_i through two rings, and per tile pair issues five tcgen05 GEMMs:
//   S^T  = K_j Q_i^T        dP^T = V_j dO_i^T        (M = 128 keys, N = 128 queries)
//   dV_j += P^T dO_i        dK_j += dS^T Q_i          (A = packed 16-bit P^T / dS^T in tensor memory)
//   dQ_i  = dS_i K_j                                  (A = dS^T staged in shared memory, read MN-major)
// 512 threads (four warpgroups, 32 query columns each) turn S^T into P^T and dP^T into
// dS^T, and drain each dQ_i from tensor memory into an fp32 accumulator in device memory
// with vector reductions performed in L2 (red.global.add.v4.f32).  dq_finish then scales
// the accumulator and rounds it to the 16-bit output.  Against the three-stage path
// (fa_bwd_sm100.cu) this drops the separate dQ pass and its recomputed S and dP: five
// GEMMs per tile pair instead of seven.  The reduction order of dQ varies from run to
// run, so dQ is reproducible to rounding, not bit for bit; dK and dV are deterministic.
//
// Tensor memory (512 columns, lanes = the 128 keys of the tile; lanes = queries for dQ):
//   S^T / P^T [0,128)   dP^T / dS^T [128,256)   dV [256,256+D)   dK [256+D,256+2D)
//   dQ_i: D = 128: [128,256), over dP^T once dS^T has been read (dP^T of the next tile
//         waits until dQ_i has been drained);  D = 64: its own columns [384,448).
// Order of the MMAs per query tile i (each waits only for what it reads or overwrites):
//   dK(i), dQ(i), dV(i+1), dP^T(i+1), S^T(i+2)
// and of the element-wise warps: dS(i), P(i+1), drain dQ(i); so the tensor pipe works on
// dK/dQ while P(i+1) is computed and on dV(i+1) while dQ(i) is drained.
#include <cstdint>
#include <math_constants.h>
#include <type_traits>

#include "bwd_common.cuh"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

template <int D>
struct FusedSmem {
  using T = Tile<D, 128>;
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kOffK = 0;                                 // K_j (later dK staging)
  static constexpr int kOffV = kOffK + T::kBytes;                 // V_j (later dV staging)
  static constexpr int kOffQ = kOffV + T::kBytes;                 // [stage] Q_i
  static constexpr int kOffdO = kOffQ + kStages * T::kBytes;      // [stage] dO_i
  static constexpr int kDSBox = 128 * 128;                        // 128 keys x 64 queries x 2 bytes
  static constexpr int kOffDS = kOffdO + kStages * T::kBytes;     // dS^T: 128 keys x 128 queries, 2 boxes
  static constexpr int kOffStat = kOffDS + 2 * kDSBox;            // [stage] nl[128], delta[128]
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
  static constexpr int kBarDQFull = kBarDS + 1;
  static constexpr int kBarDQEmpty = kBarDQFull + 1;
  static constexpr int kBarAcc = kBarDQEmpty + 1;
  static constexpr int kBarMmaDone = kBarAcc + 1;
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffSlot = kOffBar + 8 * kNumBars;
  // No slack for aligning the base: the kernel checks that the dynamic shared memory starts
  // on a 1024-byte boundary (the 128-byte swizzle atom) and reports FA_ERR_LAUNCH otherwise.
  static constexpr int kBytes = kOffSlot + 16;
  static_assert(kOffDS % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kBytes <= 232448, "shared memory budget");
  static_assert(kBytes > 116 * 1024, "one CTA per SM (each CTA allocates all 512 TMEM columns)");
};

template <int D, bool CAUSAL, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                     const float* __restrict__ ws_nl, const float* __restrict__ ws_delta, float* __restrict__ ws_dq,
                     int N, int Npad, int BH, int nkt, int hg, float scale, int* status) {
  using L = FusedSmem<D>;
  using T = Tile<D, 128>;
  extern __shared__ uint8_t smem[];   // alignment checked below, not assumed
  const uint32_t sb = smem_u32(smem);
  if (sb & 1023u) {   // uniform over the CTA: nothing has been touched yet
    if (threadIdx.x == 0) atomicCAS(status, 0, kStatusLaunch);
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sb + L::kOffBar + 8 * i; };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: key tile kt of head bh (causal: tile 0, which meets every query tile, first).
  const WorkItem wi = grouped_order(static_cast<int>(blockIdx.x), BH, nkt, hg);
  const int bh = wi.bh, kt = wi.tile;
  const int kv0 = kt * 128;
  const int it0 = CAUSAL ? kt : 0;        // first query tile
  const int n = nkt - it0;                // query tiles visited (>= 1)

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
    mbar_init(bar(L::kBarDQFull), 1);
    mbar_init(bar(L::kBarDQEmpty), 512);
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
  constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  constexpr uint32_t kColDQ = (D == 128) ? 128u : 384u;

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
      constexpr uint32_t kIdDQ = idesc_16(128, D, true, true, F16);     // dQ: A (dS) and B (K_j) MN-major
      const uint32_t sK = sb + L::kOffK, sV = sb + L::kOffV, sDS = sb + L::kOffDS;
      auto sQ = [&](int i) { return sb + L::kOffQ + (i % L::kStages) * T::kBytes; };
      auto sdO = [&](int i) { return sb + L::kOffdO + (i % L::kStages) * T::kBytes; };
      auto phase = [&](int i) { return static_cast<uint32_t>((i / L::kStages) & 1); };
      // K-major operands: four K-steps of 16 per 64-column box, 32 bytes apart.  MN-major
      // operands: one K-step per 16 rows (2048 bytes).  Packed 16-bit A operands in tensor
      // memory: K-steps at columns +0, +8, +32, +40 (see packed_col), then the next 64.
      auto issue_st = [&](int i) {      // S^T = K_j Q_i^T
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          mma_ss_x4<2, 4, 6, 2, 4, 6>(tmem + kColS, sdesc_sw128(sK + c * T::kBox, 16, 1024),
                                      sdesc_sw128(sQ(i) + c * T::kBox, 16, 1024), kIdS, c > 0 ? 1u : 0u);
        tc_commit(bar(L::kBarS));
      };
      auto issue_dpt = [&](int i) {     // dP^T = V_j dO_i^T
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          mma_ss_x4<2, 4, 6, 2, 4, 6>(tmem + kColDP, sdesc_sw128(sV + c * T::kBox, 16, 1024),
                                      sdesc_sw128(sdO(i) + c * T::kBox, 16, 1024), kIdS, c > 0 ? 1u : 0u);
        tc_commit(bar(L::kBarDP));
      };
      // acc (+)= A_tmem (packed 16-bit, 128 queries) * B_smem (128 queries x D, MN-major)
      auto issue_acc = [&](uint32_t dcol, uint32_t abase, uint32_t b_tile, bool first) {
#pragma unroll
        for (int g = 0; g < 2; ++g)
          mma_ts_x4<8, 32, 40, 128, 256, 384>(tmem + dcol, tmem + packed_col(abase, 4 * g),
                                              sdesc_sw128(b_tile + g * 4 * 2048, T::kBox, 1024), kIdAcc,
                                              (!first || g > 0) ? 1u : 0u);
      };
      auto issue_dq = [&]() {           // dQ_i = dS_i K_j: 128 queries x D over the 128 keys
#pragma unroll
        for (int g = 0; g < 2; ++g)
          mma_ss_x4<128, 256, 384, 128, 256, 384>(tmem + kColDQ, sdesc_sw128(sDS + g * 4 * 2048, L::kDSBox, 1024),
                                                  sdesc_sw128(sK + g * 4 * 2048, T::kBox, 1024), kIdDQ,
                                                  g > 0 ? 1u : 0u);
        tc_commit(bar(L::kBarDQFull));
      };
      bool ok = mbar_wait_spin(bar(L::kBarKV), 0, abort_flag) &&
                mbar_wait_spin(bar(L::kBarQFull), 0, abort_flag) && mbar_wait_spin(bar(L::kBarOFull), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_st(0);
        issue_dpt(0);
        ok = mbar_wait_spin(bar(L::kBarP), 0, abort_flag);
      }
      if (ok) {
        tc_fence_after();
        issue_acc(kColDV, kColS, sdO(0), true);                                   // dV = P^T dO_0
        tc_commit(bar(L::kBarOEmpty));
        if (n > 1 && (ok = mbar_wait_spin(bar(L::kBarQFull + 1), 0, abort_flag))) {
          tc_fence_after();
          issue_st(1);                                                            // over P^T_0 (read above)
        }
      }
      for (int i = 0; ok && i < n; ++i) {
        if (!(ok = mbar_wait_spin(bar(L::kBarDS), i & 1, abort_flag))) break;
        tc_fence_after();
        issue_acc(kColDK, kColDP, sQ(i), i == 0);                                 // dK += dS^T Q_i
        tc_commit(bar(L::kBarQEmpty + i % L::kStages));
        if (D != 128 && i > 0) {                                                  // own columns: dQ_{i-1} drained
          if (!(ok = mbar_wait_spin(bar(L::kBarDQEmpty), (i - 1) & 1, abort_flag))) break;
          tc_fence_after();
        }
        issue_dq();                                                               // dQ_i = dS_i K_j
        if (i + 1 < n) {
          const int j = i + 1;
          if (!(ok = mbar_wait_spin(bar(L::kBarP), j & 1, abort_flag))) break;
          if (!(ok = mbar_wait_spin(bar(L::kBarOFull + j % L::kStages), phase(j), abort_flag))) break;
          tc_fence_after();
          issue_acc(kColDV, kColS, sdO(j), false);                                // dV += P^T dO_{i+1}
          if (D == 128) {                                                         // dP^T over dQ_i: drained
            if (!(ok = mbar_wait_spin(bar(L::kBarDQEmpty), i & 1, abort_flag))) break;
            tc_fence_after();
          }
          issue_dpt(j);
          tc_commit(bar(L::kBarOEmpty + j % L::kStages));
        }
        if (i + 2 < n) {
          const int j = i + 2;
          if (!(ok = mbar_wait_spin(bar(L::kBarQFull + j % L::kStages), phase(j), abort_flag))) break;
          tc_fence_after();
          issue_st(j);                                                            // over P^T_{i+1} (read above)
        }
      }
      if (!ok) raise_error(status, abort_flag, kStatusTimeout);
      tc_commit(bar(L::kBarAcc));
      tc_commit(bar(L::kBarMmaDone));
      mbar_wait_drain(bar(L::kBarMmaDone), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ P^T, dS^T, dQ drain, epilogue
    const int g = (warp - 4) >> 2;                       // query columns [32g, 32g+32) of S^T / dP^T
    const int r = threadIdx.x - 128 * (1 + g);           // TMEM lane: key row of S^T, query row of dQ
    const uint32_t tb = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int key = kv0 + r;
    const bool key_oob = key >= N;                       // padding rows of the last key tile
    const bool tail = __any_sync(0xffffffffu, key_oob);  // warp-uniform
    const float scale_log2 = scale * kLog2e;
    const float2 sl2 = make_float2(scale_log2, scale_log2);
    // Row r of the dS^T tile (box g/2 holds queries [64(g/2), 64(g/2)+64)); chunk c of a row sits at c ^ (r % 8).
    uint8_t* ds_row = smem + L::kOffDS + (g >> 1) * L::kDSBox + r * 128;
    const int sw = r & 7;
    float* dq_head = ws_dq + static_cast<size_t>(bh) * Npad * D;
    uint32_t pk[16];                                     // packed P^T of the current tile
    // dQ of the previous query tile (this thread: query row r, D/4 columns), held in registers
    // from its drain out of tensor memory until its 16-byte reductions are issued, a few at a
    // time, between the next tile's dS^T and P^T arithmetic.  Each SM can send only about
    // 32 bytes per clock towards L2, so the 64 KB of a tile's dQ take ~2000 clocks to leave:
    // spread over the tile's work they overlap it, issued in one burst they would stall the
    // warps for that long.
    constexpr int kCols = D / 4;
    constexpr int kReds = kCols / 4;                     // reductions per thread per tile: 8 or 4
    uint32_t held[kCols];
    float* held_acc = dq_head + 4 * r;
    const float* const acc_end = ws_dq + static_cast<size_t>(BH) * Npad * D;   // end of the accumulator
    (void)acc_end;
    auto red_held = [&](int q) {
      float* a = held_acc + (kReds * g + q) * 512;
      if (FA_BOUNDS(a >= ws_dq && a + 4 <= acc_end, status)) red_add_f32x4(a, held[4 * q], held[4 * q + 1], held[4 * q + 2], held[4 * q + 3]);
    };

    // P^T[r][c] = exp2(s * scale * log2e + nl_c), zero where key > query or key >= N; with
    // `reds`, issues the held reductions kReds/2 .. kReds-1 along the way.
    auto p_tile = [&](int i, bool reds) -> bool {
      const int s = i % L::kStages;
      bool ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarQFull + s), (i / L::kStages) & 1, abort_flag));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarS), i & 1, abort_flag));
      if (!ok) return false;
      FA_CONVERGED(status);                              // warp-collective TMEM loads follow
      tc_fence_after();
      const float4* st = reinterpret_cast<const float4*>(smem + L::kOffStat + s * L::kStatBytes) + 8 * g;
      const int qc0 = (it0 + i) * 128 + 32 * g;          // query of this thread's column 0
      const bool edge = tail || (CAUSAL && __any_sync(0xffffffffu, qc0 < key + 32));   // warp-uniform
      // two halves of 16 columns (one TMEM load each), to keep the held dQ values in registers
      auto p_phase = [&](auto masked) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t sr[16];
          tmem_ld16(tb + kColS + 32 * g + 16 * hf, sr);
          tmem_ld_wait();
          reg_fence(sr);
#pragma unroll
          for (int c4 = 4 * hf; c4 < 4 * hf + 4; ++c4) {
            const float4 nl = st[c4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int c2 = 2 * c4 + h, c = 2 * c2, cl = c - 16 * hf;
              const float2 nlp = h ? make_float2(nl.z, nl.w) : make_float2(nl.x, nl.y);
              const float2 sv = make_float2(__uint_as_float(sr[cl]), __uint_as_float(sr[cl + 1]));
              float2 p = exp2_pair(__ffma2_rn(sv, sl2, nlp), poly_pair(c2));
              if (decltype(masked)::value) {
                if (key_oob || (CAUSAL && key > qc0 + c)) p.x = 0.f;
                if (key_oob || (CAUSAL && key > qc0 + c + 1)) p.y = 0.f;
              }
              pk[c2] = pack16<F16>(p.x, p.y);
            }
            if (reds && kReds == 8 && (c4 & 1)) red_held(4 + (c4 >> 1));         // reductions 4..7
            if (reds && kReds == 4 && (c4 & 3) == 3) red_held(2 + (c4 >> 2));    // reductions 2, 3
          }
        }
      };
      if (edge) p_phase(std::true_type{});
      else p_phase(std::false_type{});
      tmem_st16(tb + kColS + 32 * g, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarP));
      return true;
    };

    // dS^T[r][c] = P^T[r][c] * (dP^T[r][c] - delta_c), in two halves of 16 columns: packed into
    // tensor memory (for dK) and into the swizzled shared-memory tile (for dQ).
    auto ds_tile = [&](int i) -> bool {
      const int s = i % L::kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::kBarDP), i & 1, abort_flag))) return false;
      FA_CONVERGED(status);
      tc_fence_after();
      const float4* st = reinterpret_cast<const float4*>(smem + L::kOffStat + s * L::kStatBytes + 512) + 8 * g;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t dp[16], dsk[8];
        tmem_ld16(tb + kColDP + 32 * g + 16 * hf, dp);
        tmem_ld_wait();
        reg_fence(dp);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const float4 dl = st[4 * hf + c4];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c2 = 2 * c4 + h, c = 2 * c2;
            const float2 dlp = h ? make_float2(dl.z, dl.w) : make_float2(dl.x, dl.y);
            const float2 dpv = make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1]));
            const uint32_t pp = pk[8 * hf + c2];
            const float2 ds = __fmul2_rn(make_float2(unpack16_lo<F16>(pp), unpack16_hi<F16>(pp)),
                                         __ffma2_rn(dlp, make_float2(-1.f, -1.f), dpv));
            dsk[c2] = pack16<F16>(ds.x, ds.y);
          }
        }
        // packed columns [8 hf, 8 hf + 8) of this warpgroup's range (already read: half 0 read
        // columns [0, 16)) and 16-byte chunks 2 hf, 2 hf + 1 of its 64-byte part of row r
        tmem_st8(tb + kColDP + 32 * g + 8 * hf, dsk);
#pragma unroll
        for (int q = 0; q < 2; ++q)
          if (FA_BOUNDS(ds_row + ((((g & 1) * 4 + 2 * hf + q) ^ sw) << 4) + 16 <= smem + L::kOffDS + 2 * L::kDSBox, status))
          *reinterpret_cast<uint4*>(ds_row + ((((g & 1) * 4 + 2 * hf + q) ^ sw) << 4)) =
              make_uint4(dsk[4 * q], dsk[4 * q + 1], dsk[4 * q + 2], dsk[4 * q + 3]);
      }
      fence_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::kBarDS));
      return true;
    };

    // dQ_i out of tensor memory into `held`; the columns are released at once (the next dP^T
    // may overwrite them) and the first half of the reductions into the accumulator tile of
    // query tile i (laid out [D/4][128 rows][4 floats], so that a warp's reduction covers 512
    // contiguous bytes) is issued while the MMAs compute dV and that dP^T, which the next
    // dS^T waits for; the second half goes out during the next P^T.
    auto drain = [&](int i) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(L::kBarDQFull), i & 1, abort_flag))) return false;
      FA_CONVERGED(status);
      tc_fence_after();
      if constexpr (kCols == 32) tmem_ld32(tb + kColDQ + 32 * g, held);
      else tmem_ld16(tb + kColDQ + 16 * g, held);
      tmem_ld_wait();
      reg_fence(held);
      tc_fence_before();
      mbar_arrive(bar(L::kBarDQEmpty));
      held_acc = dq_head + static_cast<size_t>(it0 + i) * 128 * D + 4 * r;
#pragma unroll
      for (int q = 0; q < kReds / 2; ++q) red_held(q);
      return true;
    };

    bool ok = p_tile(0, false);
    for (int i = 0; ok && i < n; ++i) {
      ok = ds_tile(i);
      if (ok && i + 1 < n) {
        ok = p_tile(i + 1, i > 0);                       // + second half of dQ_{i-1}'s reductions
      } else if (ok && i > 0) {
#pragma unroll
        for (int q = kReds / 2; q < kReds; ++q) red_held(q);
      }
      if (ok) ok = drain(i);                             // + first half of dQ_i's
    }
    if (ok) {
#pragma unroll
      for (int q = kReds / 2; q < kReds; ++q) red_held(q);   // the last tile's second half
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(L::kBarAcc), 0, abort_flag));
    if (!ok) {
      raise_error(status, abort_flag, kStatusTimeout);
    } else {
      // One 64-column box per warpgroup: dV boxes into the V tile, dK boxes into the K tile
      // (the K tile is free: the last dQ product, which reads it, completed before kBarAcc).
      FA_CONVERGED(status);
      tc_fence_after();
      const int wrow = (warp & 3) * 32;
      const int nbox = T::kNBox;                          // 1 (D=64) or 2 (D=128)
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

// dQ = scale * accumulator, rounded to the 16-bit type, for 64 query rows per CTA: the
// tile layout [DK/4][128][4] is read with consecutive threads on consecutive rows, turned
// around in shared memory and written as whole rows of the caller's (B,H,N,D) dQ.
template <int DK, bool F16>
__global__ void __launch_bounds__(256) bwd_dq_finish_kernel(const float* __restrict__ acc, uint16_t* __restrict__ dq,
                                                            int N, int Npad, int D, float scale, int* status) {
  constexpr int kStride = DK / 4 + 1;                     // float4 per staged row (one of padding)
  __shared__ float4 stage[64 * kStride];
  const long long blk = blockIdx.x;
  const int halves = Npad / 64;
  const long long bh = blk / halves;
  const int half = static_cast<int>(blk % halves);
  const int qt = half >> 1, h = half & 1;
  const float4* src = reinterpret_cast<const float4*>(acc + (bh * Npad + static_cast<long long>(qt) * 128) * DK);
  for (int f = threadIdx.x; f < (DK / 4) * 64; f += 256) {
    const int c4 = f >> 6, rr = f & 63;
    const float4* sp = src + c4 * 128 + 64 * h + rr;
    stage[rr * kStride + c4] =
        FA_BOUNDS(sp + 1 <= reinterpret_cast<const float4*>(acc) + static_cast<long long>(gridDim.x) * 64 * DK / 4, status)
            ? *sp : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  const int row0 = qt * 128 + 64 * h;
  const int rows = min(64, N - row0);
  for (int f = threadIdx.x; f < 64 * (DK / 8); f += 256) {
    const int rr = f / (DK / 8), c8 = f % (DK / 8);
    if (rr >= rows || 8 * c8 >= D) continue;
    const float4 a = stage[rr * kStride + 2 * c8], b = stage[rr * kStride + 2 * c8 + 1];
    uint4 o;
    o.x = pack16<F16>(a.x * scale, a.y * scale);
    o.y = pack16<F16>(a.z * scale, a.w * scale);
    o.z = pack16<F16>(b.x * scale, b.y * scale);
    o.w = pack16<F16>(b.z * scale, b.w * scale);
    const long long di = (bh * N + row0 + rr) * D + 8 * c8;
    if (FA_BOUNDS(di + 8 <= static_cast<long long>(gridDim.x) / (Npad / 64) * N * D, status))
      *reinterpret_cast<uint4*>(dq + di) = o;
  }
}

template <int D, bool CAUSAL, bool F16>
cudaError_t fused_impl(const BwdLaunch& a, cudaStream_t stream) {
  using L = FusedSmem<D>;
  auto kern = bwd_fused_kernel<D, CAUSAL, F16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const int nkt = (a.N + 127) / 128;
  kern<<<static_cast<unsigned>(nkt) * a.BH, kThreads, L::kBytes, stream>>>(
      a.tmQ, a.tmK, a.tmV, a.tmdO, a.tmdK, a.tmdV, a.ws_nl, a.ws_delta, a.ws_dq, a.N, a.Npad, a.BH, nkt, a.hg,
      a.scale, a.status);
  return cudaGetLastError();
}

template <bool F16>
cudaError_t fused_typed(const BwdLaunch& a, cudaStream_t stream) {
  // Head dims 32 and 96 run the 64- and 128-column kernels on zero-filled tile columns.
  if (a.DK == 64) return a.causal ? fused_impl<64, true, F16>(a, stream) : fused_impl<64, false, F16>(a, stream);
  return a.causal ? fused_impl<128, true, F16>(a, stream) : fused_impl<128, false, F16>(a, stream);
}

template <int DK, bool F16>
cudaError_t finish_impl(const BwdLaunch& a, void* dq, cudaStream_t stream) {
  const long long blocks = static_cast<long long>(a.BH) * (a.Npad / 64);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  bwd_dq_finish_kernel<DK, F16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      a.ws_dq, static_cast<uint16_t*>(dq), a.N, a.Npad, a.D, a.scale, a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_fused(const BwdLaunch& a, cudaStream_t stream) {
  if (a.DK != 64 && a.DK != 128) return cudaErrorInvalidValue;
  return a.f16 ? fused_typed<true>(a, stream) : fused_typed<false>(a, stream);
}

cudaError_t launch_bwd_dq_finish(const BwdLaunch& a, void* dq, cudaStream_t stream) {
  if (a.DK == 64) return a.f16 ? finish_impl<64, true>(a, dq, stream) : finish_impl<64, false>(a, dq, stream);
  if (a.DK == 128) return a.f16 ? finish_impl<128, true>(a, dq, stream) : finish_impl<128, false>(a, dq, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fa
