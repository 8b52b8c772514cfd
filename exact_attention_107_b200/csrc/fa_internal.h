// fa_internal.h -- launch interfaces between the C ABI (fa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

constexpr int kStatusLaunch = 6;   // FA_ERR_LAUNCH (a kernel found its launch unusable)
constexpr int kStatusTimeout = 7;  // FA_ERR_TIMEOUT

// Order of the CTAs of a (head, tile) grid.  Heads are taken in groups of `hg` whose
// data fits in L2 together; inside a group the order is tile-major (tile 0 of every
// head of the group first, then tile 1, ...), so that with causal masking the heaviest
// tiles of a group start first, and CTAs that run at the same time share their heads'
// K/V (forward) or Q/dO/dQ (backward) through L2 instead of re-reading device memory.
struct WorkItem {
  int bh, tile;
};
__host__ __device__ inline WorkItem grouped_order(int cta, int BH, int ntiles, int hg) {
  const long long per_group = static_cast<long long>(hg) * ntiles;
  const int g = static_cast<int>(cta / per_group);
  const int local = static_cast<int>(cta - g * per_group);
  const int gh = (BH - g * hg) < hg ? (BH - g * hg) : hg;     // the last group may be smaller
  return {g * hg + local % gh, local / gh};
}

// bf16 / fp16 forward (fa_fwd_sm100.cu).  Tensor maps are 3-D (D, N, B*H) of the
// element type with 64 x 128 x 1 boxes (O: 64 x 32 x 1) and 128-byte swizzle.
struct FwdLaunch {
  CUtensorMap tmQ, tmK, tmV, tmO;
  float* lse;
  int BH, N, D;
  float scale;
  int causal;
  int f16;           // element type: 0 = bf16, 1 = fp16
  int hg;            // heads per L2 group (grouped_order)
  int* status;
  int num_sms;
};
cudaError_t launch_fwd_16(const FwdLaunch& a, cudaStream_t stream);
// Head dimension 256 (fa_fwd_d256_sm100.cu): one query tile per CTA, same tensor maps.
cudaError_t launch_fwd_d256(const FwdLaunch& a, cudaStream_t stream);

// fp32 forward (fa_fwd_f32.cu), plain pointers.
cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int BH, int N, int D, float scale, int causal, int* status, cudaStream_t stream);

// Backward stages (fa_bwd_sm100.cu).  The workspace holds, per (b, h) and per row of
// N padded up to a multiple of 128 (Npad): ws_nl = -lse * log2(e) (padding: -inf)
// and ws_delta = rowsum(dO * O) (padding: 0).
struct BwdLaunch {
  CUtensorMap tmQ, tmK, tmV, tmdO;   // loads (query box rows: 64 for dK/dV, 128 for dQ)
  CUtensorMap tmdQ, tmdK, tmdV;      // stores (32-row boxes)
  const void* o;
  const void* dO;
  const float* lse;
  float* ws_nl;
  float* ws_delta;
  float* ws_dq;      // fp32 dQ accumulator of the fused path (B*H*Npad*DK floats), or null
  int BH, N, Npad, D;
  int DK;            // columns of the kernels' tiles: 64 (D <= 64) or 128 (D in {96, 128})
  int hg;            // heads per L2 group (grouped_order)
  float scale;
  int causal;
  int f16;           // element type of q, k, v, o, dO and the gradients: 0 = bf16, 1 = fp16
  int* status;
  int num_sms;
};
cudaError_t launch_bwd_preprocess(const BwdLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd_dkdv(const BwdLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd_dq(const BwdLaunch& a, cudaStream_t stream);
// Fused backward (fa_bwd_fused_sm100.cu), DK in {64, 128}: dK, dV written, dQ added into
// ws_dq (which the preprocess kernel zeroed); then dq_finish writes scale * ws_dq to dq.
cudaError_t launch_bwd_fused(const BwdLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd_dq_finish(const BwdLaunch& a, void* dq, cudaStream_t stream);
// Head dimension 256 (fa_bwd_d256_sm100.cu): two CTAs per tile, one per half of D.
cudaError_t launch_bwd_dkdv_d256(const BwdLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd_dq_d256(const BwdLaunch& a, cudaStream_t stream);

}  // namespace fa
