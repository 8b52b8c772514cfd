// fa_fwd_f32.cu -- attention forward in fp32 throughout (FFMA pipe, no tensor cores).
//
// For callers that need the fp32 result to about 1e-6 relative: tf32 tensor-core
// products keep only 10 mantissa bits, so this path multiplies on the FP32 pipe.
// Same tiling and online softmax as the bf16 kernel ("LLM paper notes #8:
// FlashAttention" (adg.csdn.net), sections "tiling" and "online softmax"), with
// exp computed by expf and the running max raised on every tile.
//
// CTA: 64 query rows x D, 256 threads.  Thread (ty = tid / 8, tx = tid % 8) owns
// query rows 2ty and 2ty+1; for the 64 x 32 score tile it owns key columns
// tx + 8c (c < 4), and for the output it owns columns tx + 8c (c < D/8).
#include <cstdint>
#include <math_constants.h>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 64;
constexpr int kBN = 32;
constexpr int kThreads = 256;

template <int D>
struct F32Smem {
  static constexpr int kQStride = D + 1;
  static constexpr int kKStride = D + 1;
  static constexpr int kPStride = kBN + 1;
  static constexpr int kFloats = kBM * kQStride + kBN * kKStride + kBN * D + kBM * kPStride;
  static constexpr int kBytes = kFloats * 4;
};

template <int D>
__global__ void __launch_bounds__(kThreads)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                   float* __restrict__ o, float* __restrict__ lse, int N, float scale, int causal, int* status) {
  using L = F32Smem<D>;
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sK = sQ + kBM * L::kQStride;
  float* sV = sK + kBN * L::kKStride;
  float* sP = sV + kBN * D;

  const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
  const int q0 = blockIdx.x * kBM;
  const size_t base = static_cast<size_t>(blockIdx.y) * N * D;
  const size_t total = static_cast<size_t>(gridDim.y) * N * D;   // elements of each (B,H,N,D) tensor
  (void)total;
  (void)status;

  for (int i = tid; i < kBM * D; i += kThreads) {
    const int r = i / D, d = i % D;
    const size_t gi = base + static_cast<size_t>(q0 + r) * D + d;
    sQ[r * L::kQStride + d] = (q0 + r < N && FA_BOUNDS(gi < total, status)) ? q[gi] : 0.f;
  }

  float acc[2][D / 8];
  float m[2], l[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    m[i] = -CUDART_INF_F;
    l[i] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) acc[i][c] = 0.f;
  }
  const int rows[2] = {q0 + 2 * ty, q0 + 2 * ty + 1};
  const int kv_end = causal ? min(N, q0 + kBM) : N;

  for (int kv0 = 0; kv0 < kv_end; kv0 += kBN) {
    __syncthreads();   // previous tile's sK / sV / sP no longer in use
    for (int i = tid; i < kBN * D; i += kThreads) {
      const int r = i / D, d = i % D;
      const size_t gi = base + static_cast<size_t>(kv0 + r) * D + d;
      const bool in = kv0 + r < N && FA_BOUNDS(gi < total, status);
      sK[r * L::kKStride + d] = in ? k[gi] : 0.f;
      sV[r * D + d] = in ? v[gi] : 0.f;
    }
    __syncthreads();
    float s[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[i][c] = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      const float qa = sQ[(2 * ty) * L::kQStride + d];
      const float qb = sQ[(2 * ty + 1) * L::kQStride + d];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float kv = sK[(tx + 8 * c) * L::kKStride + d];
        s[0][c] = fmaf(qa, kv, s[0][c]);
        s[1][c] = fmaf(qb, kv, s[1][c]);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int key = kv0 + tx + 8 * c;
        const bool masked = key >= N || (causal && key > rows[i]);
        s[i][c] = masked ? -CUDART_INF_F : s[i][c] * scale;
        mx = fmaxf(mx, s[i][c]);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      const float m_new = fmaxf(m[i], mx);
      // m_new is -inf only for a row with no allowed key yet (padding rows past N).
      const float alpha = (m_new == -CUDART_INF_F) ? 1.f : expf(m[i] - m_new);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float p = (m_new == -CUDART_INF_F) ? 0.f : expf(s[i][c] - m_new);
        sP[(2 * ty + i) * L::kPStride + tx + 8 * c] = p;
        rs += p;
      }
      rs += __shfl_xor_sync(0xffffffffu, rs, 1);
      rs += __shfl_xor_sync(0xffffffffu, rs, 2);
      rs += __shfl_xor_sync(0xffffffffu, rs, 4);
      l[i] = l[i] * alpha + rs;
      m[i] = m_new;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) acc[i][c] *= alpha;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kBN; ++kk) {
      const float pa = sP[(2 * ty) * L::kPStride + kk];
      const float pb = sP[(2 * ty + 1) * L::kPStride + kk];
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const float vv = sV[kk * D + tx + 8 * c];
        acc[0][c] = fmaf(pa, vv, acc[0][c]);
        acc[1][c] = fmaf(pb, vv, acc[1][c]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (rows[i] >= N) continue;
    const float inv = 1.f / l[i];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const size_t gi = base + static_cast<size_t>(rows[i]) * D + tx + 8 * c;
      if (FA_BOUNDS(gi < total, status)) o[gi] = acc[i][c] * inv;
    }
    const size_t li = static_cast<size_t>(blockIdx.y) * N + rows[i];
    if (tx == 0 && FA_BOUNDS(li < static_cast<size_t>(gridDim.y) * N, status)) lse[li] = m[i] + logf(l[i]);
  }
}

template <int D>
cudaError_t launch_impl(const float* q, const float* k, const float* v, float* o, float* lse, int BH, int N,
                        float scale, int causal, int* status, cudaStream_t stream) {
  using L = F32Smem<D>;
  cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid((N + kBM - 1) / kBM, BH);
  fwd_f32_kernel<D><<<grid, kThreads, L::kBytes, stream>>>(q, k, v, o, lse, N, scale, causal, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int BH, int N,
                           int D, float scale, int causal, int* status, cudaStream_t stream) {
  switch (D) {
    case 32: return launch_impl<32>(q, k, v, o, lse, BH, N, scale, causal, status, stream);
    case 64: return launch_impl<64>(q, k, v, o, lse, BH, N, scale, causal, status, stream);
    default: return launch_impl<128>(q, k, v, o, lse, BH, N, scale, causal, status, stream);
  }
}

}  // namespace fa
