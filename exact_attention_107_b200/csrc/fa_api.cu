// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, TMA tensor
// maps, per-device state, and kernel launches.  No entry point allocates memory,
// synchronises the host (except fa_device_status) or throws.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

// Device status word: kernels record the first device-side failure here
// (FA_ERR_TIMEOUT when a pipeline wait exceeded its limit).
__device__ int g_fa_status;

constexpr int kMaxDevices = 64;

struct DeviceState {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  bool sm100 = false;
  int num_sms = 0;
  int* status = nullptr;
};
DeviceState g_dev[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// Per-device set-up (once per device, with that device current): architecture,
// SM count and the device address of the status word.
int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  DeviceState& s = g_dev[dev];
  std::call_once(s.once, [&s, dev] {
    int major = 0, minor = 0;
    s.err = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (s.err == cudaSuccess) s.err = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (s.err == cudaSuccess) s.err = cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (s.err == cudaSuccess) s.err = cudaGetSymbolAddress(reinterpret_cast<void**>(&s.status), g_fa_status);
    s.sm100 = (major == 10 && minor == 0);
  });
  if (s.err != cudaSuccess) return FA_ERR_CUDA;
  if (!s.sm100) return FA_ERR_UNSUPPORTED_ARCH;
  *out = &s;
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Head dims: 32, 64, 96, 128 and (with_256) 256 on the 16-bit paths (32 and 96 run the
// 64- and 128-column kernels on zero-filled columns); 32, 64, 128 on the fp32 forward.
int check_shape(int B, int H, int N, int D, bool sixteen_bit, bool with_256 = false) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_SHAPE;
  if (D != 32 && D != 64 && D != 128 && !(sixteen_bit && D == 96) && !(with_256 && D == 256))
    return FA_ERR_HEADDIM;
  const long long bh = static_cast<long long>(B) * H;
  if (bh > INT_MAX / 2) return FA_ERR_SHAPE;
  // The largest grid (ceil(N/128) * B*H CTAs, the dK/dV kernel; twice that at D = 256)
  // must fit a 31-bit grid.
  if ((static_cast<long long>(N) + 127) / 128 * bh * (D == 256 ? 2 : 1) > INT_MAX) return FA_ERR_SHAPE;
  return FA_OK;
}

// 3-D (D, N, B*H) bf16 (fp16 when f16) tensor map, box 64 x box_rows x 1, 128-byte swizzle.
int make_tmap(CUtensorMap* map, const void* ptr, int BH, int N, int D, int box_rows, bool f16) {
  auto enc = encode_fn();
  if (!enc) return FA_ERR_LAUNCH;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH; }

bool scale_ok(float scale) { return std::isfinite(scale) && scale > 0.f; }

// Columns of the 16-bit kernels' tiles for head dim D (the fused backward's dQ accumulator
// holds this many floats per row); 0 for D = 256, which has no fused backward.
int tile_cols(int D) { return D <= 64 ? 64 : (D <= 128 ? 128 : 0); }

// Bytes of the backward's row statistics: -lse*log2(e) and delta for B*H*Npad rows.
size_t stats_bytes(int B, int H, int N) {
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  return 2 * static_cast<size_t>(B) * H * npad * sizeof(float);
}

// Heads per L2 group of the grouped CTA order: as many heads as fit their shared data
// (bytes_per_head) into 64 MiB, about half of the B200's 126 MB L2.
int heads_per_group(long long bytes_per_head, int BH) {
  const long long budget = 64LL << 20;
  long long hg = bytes_per_head > 0 ? budget / bytes_per_head : BH;
  if (hg < 1) hg = 1;
  if (hg > BH) hg = BH;
  return static_cast<int>(hg);
}

}  // namespace

extern "C" {

int fa_version(void) { return 20000; }

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_NULL: return "FA_ERR_NULL: a required pointer is NULL";
    case FA_ERR_SHAPE: return "FA_ERR_SHAPE: B, H or N out of range";
    case FA_ERR_HEADDIM: return "FA_ERR_HEADDIM: unsupported head dimension";
    case FA_ERR_ALIGN: return "FA_ERR_ALIGN: pointer not 16-byte aligned";
    case FA_ERR_UNSUPPORTED_ARCH: return "FA_ERR_UNSUPPORTED_ARCH: device is not sm_100";
    case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH: kernel launch or tensor-map encoding failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a device-side wait exceeded its limit";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace missing or too small";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA runtime error";
    case FA_ERR_ARG: return "FA_ERR_ARG: invalid argument";
    case FA_ERR_NOALLOC_CAPACITY: return "FA_ERR_NOALLOC_CAPACITY: problem exceeds the fa_bwd_noalloc scratch size";
    case FA_ERR_DEBUG_CHECK: return "FA_ERR_DEBUG_CHECK: a device-side check of the debug build failed";
    default: return "unknown fa_status";
  }
}

int fa_device_status(int reset) {
  DeviceState* ds = nullptr;
  int st = device_state(&ds);
  if (st != FA_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fa_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  }
  return v;
}

}  // extern "C"

// The 16-bit paths, bf16 or (f16) fp16 operands.
static int fwd16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int D,
                 float scale, int causal, void* stream, bool f16) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  int st = check_shape(B, H, N, D, true, true);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  if (!scale_ok(scale) || (causal != 0 && causal != 1)) return FA_ERR_ARG;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  fa::FwdLaunch a{};
  const int BH = B * H;
  if ((st = make_tmap(&a.tmQ, q, BH, N, D, 128, f16)) != FA_OK) return st;
  if ((st = make_tmap(&a.tmK, k, BH, N, D, 128, f16)) != FA_OK) return st;
  if ((st = make_tmap(&a.tmV, v, BH, N, D, 128, f16)) != FA_OK) return st;
  if ((st = make_tmap(&a.tmO, o, BH, N, D, 32, f16)) != FA_OK) return st;
  a.f16 = f16 ? 1 : 0;
  a.lse = lse;
  a.BH = BH;
  a.N = N;
  a.D = D;
  a.scale = scale;
  a.causal = causal;
  a.status = ds->status;
  a.num_sms = ds->num_sms;
  // The forward's CTAs of one head share that head's K and V tiles.
  a.hg = heads_per_group(4LL * N * D, BH);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_status(D == 256 ? fa::launch_fwd_d256(a, s) : fa::launch_fwd_16(a, s));
}

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int D,
           float scale, int causal, void* stream) {
  return fwd16(q, k, v, o, lse, B, H, N, D, scale, causal, stream, false);
}

int fa_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int D,
               float scale, int causal, void* stream) {
  return fwd16(q, k, v, o, lse, B, H, N, D, scale, causal, stream, true);
}

int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int N, int D,
               float scale, int causal, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  int st = check_shape(B, H, N, D, false);
  if (st != FA_OK) return st;
  if (static_cast<long long>(B) * H > 65535) return FA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  if (!scale_ok(scale) || (causal != 0 && causal != 1)) return FA_ERR_ARG;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  return launch_status(
      fa::launch_fwd_f32(q, k, v, o, lse, B * H, N, D, scale, causal, ds->status, static_cast<cudaStream_t>(stream)));
}

size_t fa_bwd_workspace_size(int B, int H, int N, int D) {
  if (check_shape(B, H, N, D, true, true) != FA_OK) return 0;
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  const size_t rows = static_cast<size_t>(B) * H * npad;
  return rows * (2 + static_cast<size_t>(tile_cols(D))) * sizeof(float);   // a multiple of 1024 bytes
}

}  // extern "C"

// Workspace views: ws_nl = [0, R) floats, ws_delta = [R, 2R) with R = B*H*Npad, and (with_acc,
// head dims up to 128) the fused path's dQ accumulator ws_dq = [2R, 2R + R*DK).
static int workspace_views(void* ws, size_t ws_bytes, int B, int H, int N, int D, bool with_acc, fa::BwdLaunch* a) {
  const size_t need = with_acc ? fa_bwd_workspace_size(B, H, N, D) : stats_bytes(B, H, N);
  if (!ws || ws_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned16(ws)) return FA_ERR_ALIGN;
  a->Npad = (N + 127) / 128 * 128;
  const size_t rows = static_cast<size_t>(B) * H * a->Npad;
  a->ws_nl = static_cast<float*>(ws);
  a->ws_delta = a->ws_nl + rows;
  a->DK = tile_cols(D);
  a->ws_dq = (with_acc && a->DK > 0) ? a->ws_delta + rows : nullptr;
  return FA_OK;
}

static int preprocess16(const void* o, const void* dO, const float* lse, void* workspace, size_t workspace_bytes,
                        int B, int H, int N, int D, bool with_acc, void* stream, bool f16) {
  if (!o || !dO || !lse) return FA_ERR_NULL;
  int st = check_shape(B, H, N, D, true, true);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(dO) || !aligned16(lse)) return FA_ERR_ALIGN;
  fa::BwdLaunch a{};
  if ((st = workspace_views(workspace, workspace_bytes, B, H, N, D, with_acc, &a)) != FA_OK) return st;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  a.f16 = f16 ? 1 : 0;
  a.status = ds->status;
  a.o = o;
  a.dO = dO;
  a.lse = lse;
  a.BH = B * H;
  a.N = N;
  a.D = D;
  return launch_status(fa::launch_bwd_preprocess(a, static_cast<cudaStream_t>(stream)));
}

static int bwd_common(const void* q, const void* k, const void* v, const void* dO, const void* workspace,
                      size_t workspace_bytes, int B, int H, int N, int D, float scale, int causal, bool with_acc,
                      bool f16, fa::BwdLaunch* a) {
  if (!q || !k || !v || !dO) return FA_ERR_NULL;
  int st = check_shape(B, H, N, D, true, true);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO)) return FA_ERR_ALIGN;
  if ((st = workspace_views(const_cast<void*>(workspace), workspace_bytes, B, H, N, D, with_acc, a)) != FA_OK)
    return st;
  if (!scale_ok(scale) || (causal != 0 && causal != 1)) return FA_ERR_ARG;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  const int BH = B * H;
  if ((st = make_tmap(&a->tmQ, q, BH, N, D, 128, f16)) != FA_OK) return st;
  if ((st = make_tmap(&a->tmK, k, BH, N, D, 128, f16)) != FA_OK) return st;
  if ((st = make_tmap(&a->tmV, v, BH, N, D, 128, f16)) != FA_OK) return st;
  if ((st = make_tmap(&a->tmdO, dO, BH, N, D, 128, f16)) != FA_OK) return st;
  a->f16 = f16 ? 1 : 0;
  a->BH = BH;
  a->N = N;
  a->D = D;
  a->scale = scale;
  a->causal = causal;
  a->status = ds->status;
  a->num_sms = ds->num_sms;
  // The fused kernel's CTAs of one head share that head's Q and dO tiles and dQ accumulator.
  a->hg = heads_per_group(static_cast<long long>(a->Npad) * (4LL * D + 4LL * a->DK), BH);
  return FA_OK;
}

static int dkdv16(const void* q, const void* k, const void* v, const void* dO, const void* workspace,
                  size_t workspace_bytes, void* dk, void* dv, int B, int H, int N, int D, float scale, int causal,
                  void* stream, bool f16) {
  if (!dk || !dv) return FA_ERR_NULL;
  if (!aligned16(dk) || !aligned16(dv)) return FA_ERR_ALIGN;
  fa::BwdLaunch a{};
  int st = bwd_common(q, k, v, dO, workspace, workspace_bytes, B, H, N, D, scale, causal, false, f16, &a);
  if (st != FA_OK) return st;
  if ((st = make_tmap(&a.tmdK, dk, a.BH, N, D, 32, f16)) != FA_OK) return st;
  if ((st = make_tmap(&a.tmdV, dv, a.BH, N, D, 32, f16)) != FA_OK) return st;
  return launch_status(fa::launch_bwd_dkdv(a, static_cast<cudaStream_t>(stream)));
}

static int dq16(const void* q, const void* k, const void* v, const void* dO, const void* workspace,
                size_t workspace_bytes, void* dq, int B, int H, int N, int D, float scale, int causal, void* stream,
                bool f16) {
  if (!dq) return FA_ERR_NULL;
  if (!aligned16(dq)) return FA_ERR_ALIGN;
  fa::BwdLaunch a{};
  int st = bwd_common(q, k, v, dO, workspace, workspace_bytes, B, H, N, D, scale, causal, false, f16, &a);
  if (st != FA_OK) return st;
  if ((st = make_tmap(&a.tmdQ, dq, a.BH, N, D, 32, f16)) != FA_OK) return st;
  return launch_status(fa::launch_bwd_dq(a, static_cast<cudaStream_t>(stream)));
}

static int dkdvdq16(const void* q, const void* k, const void* v, const void* dO, void* workspace,
                    size_t workspace_bytes, void* dk, void* dv, int B, int H, int N, int D, float scale, int causal,
                    void* stream, bool f16) {
  if (!dk || !dv) return FA_ERR_NULL;
  if (!aligned16(dk) || !aligned16(dv)) return FA_ERR_ALIGN;
  if (D > 128) return check_shape(B, H, N, D, true, false);     // no fused kernel for D = 256
  fa::BwdLaunch a{};
  int st = bwd_common(q, k, v, dO, workspace, workspace_bytes, B, H, N, D, scale, causal, true, f16, &a);
  if (st != FA_OK) return st;
  if ((st = make_tmap(&a.tmdK, dk, a.BH, N, D, 32, f16)) != FA_OK) return st;
  if ((st = make_tmap(&a.tmdV, dv, a.BH, N, D, 32, f16)) != FA_OK) return st;
  return launch_status(fa::launch_bwd_fused(a, static_cast<cudaStream_t>(stream)));
}

static int dq_finish16(const void* workspace, size_t workspace_bytes, void* dq, int B, int H, int N, int D,
                       float scale, void* stream, bool f16) {
  if (!dq) return FA_ERR_NULL;
  int st = check_shape(B, H, N, D, true, false);
  if (st != FA_OK) return st;
  if (!aligned16(dq)) return FA_ERR_ALIGN;
  if (!scale_ok(scale)) return FA_ERR_ARG;
  fa::BwdLaunch a{};
  if ((st = workspace_views(const_cast<void*>(workspace), workspace_bytes, B, H, N, D, true, &a)) != FA_OK) return st;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  a.f16 = f16 ? 1 : 0;
  a.status = ds->status;
  a.BH = B * H;
  a.N = N;
  a.D = D;
  a.scale = scale;
  return launch_status(fa::launch_bwd_dq_finish(a, dq, static_cast<cudaStream_t>(stream)));
}

// Validation shared by the two complete backward entry points, so that an error launches nothing.
static int bwd_validate(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                        void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, size_t ws_need,
                        int B, int H, int N, int D, float scale, int causal) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_NULL;
  int st = check_shape(B, H, N, D, true, true);
  if (st != FA_OK) return st;
  if (!workspace || workspace_bytes < ws_need) return FA_ERR_WORKSPACE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return FA_ERR_ALIGN;
  if (!scale_ok(scale) || (causal != 0 && causal != 1)) return FA_ERR_ARG;
  return FA_OK;
}

// fa_bwd / fa_bwd_f16: the fused kernel for head dims up to 128 (preprocess, which also
// zeroes the dQ accumulator; dK/dV/dQ kernel; dQ finish), the two-CTA three-stage path at 256.
static int bwd16(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int D,
                 float scale, int causal, void* stream, bool f16) {
  int st = bwd_validate(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes,
                        fa_bwd_workspace_size(B, H, N, D), B, H, N, D, scale, causal);
  if (st != FA_OK) return st;
  const bool fused = tile_cols(D) > 0;
  if ((st = preprocess16(o, dO, lse, workspace, workspace_bytes, B, H, N, D, fused, stream, f16)) != FA_OK) return st;
  if (!fused) {
    if ((st = dkdv16(q, k, v, dO, workspace, workspace_bytes, dk, dv, B, H, N, D, scale, causal, stream, f16)) !=
        FA_OK)
      return st;
    return dq16(q, k, v, dO, workspace, workspace_bytes, dq, B, H, N, D, scale, causal, stream, f16);
  }
  if ((st = dkdvdq16(q, k, v, dO, workspace, workspace_bytes, dk, dv, B, H, N, D, scale, causal, stream, f16)) !=
      FA_OK)
    return st;
  return dq_finish16(workspace, workspace_bytes, dq, B, H, N, D, scale, stream, f16);
}

// fa_bwd_deterministic: preprocess, the dK/dV kernel and the dQ kernel (no atomics).
static int bwd_det16(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                     void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N,
                     int D, float scale, int causal, void* stream, bool f16) {
  int st = bwd_validate(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, stats_bytes(B, H, N), B, H, N,
                        D, scale, causal);
  if (st != FA_OK) return st;
  if ((st = preprocess16(o, dO, lse, workspace, workspace_bytes, B, H, N, D, false, stream, f16)) != FA_OK) return st;
  if ((st = dkdv16(q, k, v, dO, workspace, workspace_bytes, dk, dv, B, H, N, D, scale, causal, stream, f16)) != FA_OK)
    return st;
  return dq16(q, k, v, dO, workspace, workspace_bytes, dq, B, H, N, D, scale, causal, stream, f16);
}

extern "C" {

size_t fa_bwd_deterministic_workspace_size(int B, int H, int N, int D) {
  if (check_shape(B, H, N, D, true, true) != FA_OK) return 0;
  return stats_bytes(B, H, N);
}

int fa_bwd_preprocess(const void* o, const void* dO, const float* lse, void* workspace, size_t workspace_bytes,
                      int B, int H, int N, int D, void* stream) {
  // The dQ accumulator is zeroed when the workspace holds one (fa_bwd_workspace_size bytes).
  const size_t full = fa_bwd_workspace_size(B, H, N, D);
  const bool with_acc = tile_cols(D) > 0 && full > 0 && workspace_bytes >= full;
  return preprocess16(o, dO, lse, workspace, workspace_bytes, B, H, N, D, with_acc, stream, false);
}

int fa_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO, const void* workspace,
                size_t workspace_bytes, void* dk, void* dv, int B, int H, int N, int D, float scale, int causal,
                void* stream) {
  return dkdv16(q, k, v, dO, workspace, workspace_bytes, dk, dv, B, H, N, D, scale, causal, stream, false);
}

int fa_bwd_dq(const void* q, const void* k, const void* v, const void* dO, const void* workspace,
              size_t workspace_bytes, void* dq, int B, int H, int N, int D, float scale, int causal, void* stream) {
  return dq16(q, k, v, dO, workspace, workspace_bytes, dq, B, H, N, D, scale, causal, stream, false);
}

int fa_bwd_dkdvdq(const void* q, const void* k, const void* v, const void* dO, void* workspace,
                  size_t workspace_bytes, void* dk, void* dv, int B, int H, int N, int D, float scale, int causal,
                  void* stream) {
  return dkdvdq16(q, k, v, dO, workspace, workspace_bytes, dk, dv, B, H, N, D, scale, causal, stream, false);
}

int fa_bwd_dq_finish(const void* workspace, size_t workspace_bytes, void* dq, int B, int H, int N, int D, float scale,
                     void* stream) {
  return dq_finish16(workspace, workspace_bytes, dq, B, H, N, D, scale, stream, false);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
           void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int D, float scale,
           int causal, void* stream) {
  return bwd16(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, B, H, N, D, scale, causal, stream, false);
}

int fa_bwd_f16(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
               void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int D,
               float scale, int causal, void* stream) {
  return bwd16(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, B, H, N, D, scale, causal, stream, true);
}

int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                         int B, int H, int N, int D, float scale, int causal, void* stream) {
  return bwd_det16(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, B, H, N, D, scale, causal, stream,
                   false);
}

}  // extern "C"
