// fa_fwd_f32.cu -- attention forward in fp32 throughout (FFMA pipe, no tensor cores).
//
// For callers that need the fp32 result to about 1e-6 relative: tf32 tensor-core
// products keep only 10 mantissa bits, so this path multiplies on the FP32 pipe.
// Same tiling and online softmax as the bf16 kernel ("LLM paper notes #8:
// FlashAttention" (adg.csdn.net), sections "tiling" and "online softmax"), with
// exp computed by expf and the running max raised on every key chunk.
//
// The fp32 path serves small problems, so the work is split finely: a CTA of 8 warps
// owns 8 query rows of one (batch, head), one row per warp, and streams the keys in
// chunks of kC through a double-buffered shared-memory ring filled with cp.async (the
// next chunk's copies are in flight while this one is used).  Per chunk and row:
// lane l computes the scores of keys l, l + 32, ... (float4 reads of K rows padded to
// D + 4 floats, so the eight lanes of each 128-byte phase hit distinct banks), the
// warp reduces the chunk's max and sum with shuffles, the probabilities go through a
// per-warp shared-memory row, and lane l accumulates output columns [lane * D/32,
// (lane + 1) * D/32) over the chunk's V rows.
#include <cstdint>
#include <math_constants.h>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kWarps = 8;               // = query rows per CTA
constexpr int kThreads = kWarps * 32;

template <int D>
struct F32Smem {
  static constexpr int kC = (D == 128) ? 32 : 64;       // keys per chunk
  static constexpr int kKStride = D + 4;                // floats per K row
  static constexpr int kKFloats = kC * kKStride;        // one K buffer
  static constexpr int kVFloats = kC * D;               // one V buffer
  static constexpr int kOffK = 0;                       // [2] K buffers
  static constexpr int kOffV = kOffK + 2 * kKFloats;    // [2] V buffers
  static constexpr int kOffQ = kOffV + 2 * kVFloats;    // [kWarps][D]
  static constexpr int kOffP = kOffQ + kWarps * D;      // [kWarps][kC]
  static constexpr int kFloats = kOffP + kWarps * kC;
  static constexpr int kBytes = kFloats * 4;
  static constexpr int kPerLane = D / 32;               // output columns per lane
  static constexpr int kKeysPerLane = kC / 32;
  static_assert(kKStride % 4 == 0 && D % 4 == 0, "16-byte rows");
};

// 16-byte global -> shared copy; `src_bytes` = 0 zero-fills the destination (rows past N).
__device__ __forceinline__ void cp_async16(float* dst, const float* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                   float* __restrict__ o, float* __restrict__ lse, int N, float scale, int causal, int* status) {
  using L = F32Smem<D>;
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q0 = blockIdx.x * kWarps;
  const int row = q0 + warp;
  const bool live = row < N;
  const size_t base = static_cast<size_t>(blockIdx.y) * N * D;
  const size_t total = static_cast<size_t>(gridDim.y) * N * D;   // elements of each (B,H,N,D) tensor
  (void)total;
  (void)status;
  const int kv_end = causal ? min(N, q0 + kWarps) : N;
  const int nchunks = (kv_end + L::kC - 1) / L::kC;

  // Copies of key chunk c into ring slot c & 1 (rows past N are zero-filled).
  auto load_chunk = [&](int c) {
    float* sK = sm + L::kOffK + (c & 1) * L::kKFloats;
    float* sV = sm + L::kOffV + (c & 1) * L::kVFloats;
    for (int i = tid; i < L::kC * (D / 4); i += kThreads) {
      const int r = i / (D / 4), c4 = i % (D / 4);
      const int key = c * L::kC + r;
      const bool in = key < N;
      const size_t gi = base + static_cast<size_t>(in ? key : 0) * D + 4 * c4;
      const bool ok = FA_BOUNDS(gi + 4 <= total, status);
      cp_async16(sK + r * L::kKStride + 4 * c4, k + (ok ? gi : 0), in && ok ? 16u : 0u);
      cp_async16(sV + r * D + 4 * c4, v + (ok ? gi : 0), in && ok ? 16u : 0u);
    }
    cp_async_commit();
  };

  // This CTA's query rows (zeros past N), then the first key chunk.
  for (int i = tid; i < kWarps * (D / 4); i += kThreads) {
    const int r = i / (D / 4), c4 = i % (D / 4);
    const bool in = q0 + r < N;
    const size_t gi = base + static_cast<size_t>(in ? q0 + r : 0) * D + 4 * c4;
    const bool ok = FA_BOUNDS(gi + 4 <= total, status);
    cp_async16(sm + L::kOffQ + r * D + 4 * c4, q + (ok ? gi : 0), in && ok ? 16u : 0u);
  }
  if (nchunks > 0) load_chunk(0);

  const float* sQ = sm + L::kOffQ + warp * D;
  float* sP = sm + L::kOffP + warp * L::kC;
  float acc[L::kPerLane];
#pragma unroll
  for (int c = 0; c < L::kPerLane; ++c) acc[c] = 0.f;
  float m = -CUDART_INF_F, l = 0.f;

  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) {
      load_chunk(c + 1);               // slot (c+1) & 1 was released by the barrier ending step c-1
      cp_async_wait<1>();              // chunk c (and the query rows) have landed
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (live) {
      const float* sK = sm + L::kOffK + (c & 1) * L::kKFloats;
      const float* sV = sm + L::kOffV + (c & 1) * L::kVFloats;
      float s[L::kKeysPerLane];
#pragma unroll
      for (int i = 0; i < L::kKeysPerLane; ++i) s[i] = 0.f;
#pragma unroll 4
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 qv = *reinterpret_cast<const float4*>(sQ + 4 * d4);
#pragma unroll
        for (int i = 0; i < L::kKeysPerLane; ++i) {
          const float4 kv = *reinterpret_cast<const float4*>(sK + (lane + 32 * i) * L::kKStride + 4 * d4);
          s[i] = fmaf(qv.x, kv.x, s[i]);
          s[i] = fmaf(qv.y, kv.y, s[i]);
          s[i] = fmaf(qv.z, kv.z, s[i]);
          s[i] = fmaf(qv.w, kv.w, s[i]);
        }
      }
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int i = 0; i < L::kKeysPerLane; ++i) {
        const int key = c * L::kC + lane + 32 * i;
        const bool masked = key >= N || (causal && key > row);
        s[i] = masked ? -CUDART_INF_F : s[i] * scale;
        mx = fmaxf(mx, s[i]);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m, mx);
      // m_new is -inf only while no allowed key has been seen (cannot happen for a live
      // row after its first chunk, since key 0 is always allowed).
      const float alpha = (m_new == -CUDART_INF_F) ? 1.f : expf(m - m_new);
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < L::kKeysPerLane; ++i) {
        const float p = (m_new == -CUDART_INF_F) ? 0.f : expf(s[i] - m_new);
        sP[lane + 32 * i] = p;
        rs += p;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
      l = l * alpha + rs;
      m = m_new;
#pragma unroll
      for (int cc = 0; cc < L::kPerLane; ++cc) acc[cc] *= alpha;
      __syncwarp();
#pragma unroll 8
      for (int j = 0; j < L::kC; ++j) {
        const float p = sP[j];
        const float* vr = sV + j * D + lane * L::kPerLane;
#pragma unroll
        for (int cc = 0; cc < L::kPerLane; ++cc) acc[cc] = fmaf(p, vr[cc], acc[cc]);
      }
      __syncwarp();
    }
    __syncthreads();                   // every warp is done with slot c & 1
  }
  if (live) {
    const float inv = 1.f / l;
    const size_t gi = base + static_cast<size_t>(row) * D + lane * L::kPerLane;
    if (FA_BOUNDS(gi + L::kPerLane <= total, status)) {
#pragma unroll
      for (int cc = 0; cc < L::kPerLane; ++cc) o[gi + cc] = acc[cc] * inv;
    }
    const size_t li = static_cast<size_t>(blockIdx.y) * N + row;
    if (lane == 0 && FA_BOUNDS(li < static_cast<size_t>(gridDim.y) * N, status)) lse[li] = m + logf(l);
  }
}

template <int D>
cudaError_t launch_impl(const float* q, const float* k, const float* v, float* o, float* lse, int BH, int N,
                        float scale, int causal, int* status, cudaStream_t stream) {
  using L = F32Smem<D>;
  cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid((N + kWarps - 1) / kWarps, BH);
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
