// fa_internal.h -- launch interfaces between the C ABI (fa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

constexpr int kStatusTimeout = 7;  // FA_ERR_TIMEOUT

// bf16 / fp16 forward (fa_fwd_sm100.cu).  Tensor maps are 3-D (D, N, B*H) of the
// element type with 64 x 128 x 1 boxes (O: 64 x 32 x 1) and 128-byte swizzle.
struct FwdLaunch {
  CUtensorMap tmQ, tmK, tmV, tmO;
  float* lse;
  int BH, N, D;
  float scale;
  int causal;
  int f16;           // element type: 0 = bf16, 1 = fp16
  int* status;
  int num_sms;
};
cudaError_t launch_fwd_16(const FwdLaunch& a, cudaStream_t stream);
// Head dimension 256 (fa_fwd_d256_sm100.cu): one query tile per CTA, same tensor maps.
cudaError_t launch_fwd_d256(const FwdLaunch& a, cudaStream_t stream);

// fp32 forward (fa_fwd_f32.cu), plain pointers.
cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                           int BH, int N, int D, float scale, int causal, cudaStream_t stream);

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
  int BH, N, Npad, D;
  float scale;
  int causal;
  int f16;           // element type of q, k, v, o, dO and the gradients: 0 = bf16, 1 = fp16
  int* status;
  int num_sms;
};
cudaError_t launch_bwd_preprocess(const BwdLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd_dkdv(const BwdLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd_dq(const BwdLaunch& a, cudaStream_t stream);
// Head dimension 256 (fa_bwd_d256_sm100.cu): two CTAs per tile, one per half of D.
cudaError_t launch_bwd_dkdv_d256(const BwdLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd_dq_d256(const BwdLaunch& a, cudaStream_t stream);

}  // namespace fa
