/*
 * fa.h -- C ABI of libfa.so: exact, IO-aware tiled attention for NVIDIA B200 (sm_100a).
 *
 * The operation (all entry points):
 *     S   = scale * Q K^T                (N x N per batch b and head h)
 *     S_ij = -inf for j > i               (only when causal != 0; top-left aligned)
 *     P   = softmax(S) row-wise,  O = P V
 *     lse_i = ln( sum_j exp(S_ij) )       (natural-log logsumexp of the scaled scores)
 * This is the attention of the three-line PyTorch form in "CUDA-kernel-level
 * optimisation: why Flash Attention is 5-10x faster than native PyTorch"
 * (guanweilu.cn, section "three lines of PyTorch"), computed the way its
 * section "three tricks" and "LLM paper notes #8: FlashAttention" (adg.csdn.net,
 * sections "tiling", "online softmax", "recomputation") describe: Q/K/V tiles
 * staged on chip, an online softmax with a running max and sum, no N x N matrix
 * in device memory, and a backward pass that recomputes P from lse.
 *
 * Conventions shared by every entry point
 *   - Layout: every tensor is contiguous (B, H, N, D), head dimension innermost
 *     (the layout of naive_attention in "Flash Attention principles: making
 *     Transformers faster", ijyty.com, section "memory bottleneck").  lse and
 *     delta are contiguous (B, H, N) float32.
 *   - Pointers are DEVICE pointers (cudaMalloc'd or equivalent) on the current
 *     device, 16-byte aligned.  The caller owns and allocates every buffer; the
 *     library never allocates or frees device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Every call is asynchronous on that stream; the library does no
 *     host synchronisation.
 *   - Supported: B, H, N >= 1; D in {32, 64, 96, 128} for bf16 and fp16 (32
 *     and 96 run the 64- and 128-column kernels on zero-filled columns, so
 *     they cost what 64 and 128 cost), and D = 256 (forward: one query tile
 *     per CTA; backward: two CTAs per tile, one per half of D); D in
 *     {32, 64, 128} for fp32; Nq == Nk == N; causal in {0, 1}; ceil(N/256)*B*H < 2^31 (and
 *     B*H <= 65535 for fa_fwd_f32).
 *   - Return value: FA_OK (0) or an fa_status code.  Arguments are validated
 *     before anything is launched; on an error nothing is launched and no
 *     output is touched.  Errors are never thrown across the ABI.
 *   - Device-side failures (a pipeline wait that exceeded its time limit) do
 *     not trap: the kernel records FA_ERR_TIMEOUT in a device status word and
 *     returns; fa_device_status() reads (and optionally clears) that word.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_NULL = 1,             /* a required pointer is NULL                      */
  FA_ERR_SHAPE = 2,            /* B, H or N out of range, or index overflow       */
  FA_ERR_HEADDIM = 3,          /* unsupported head dimension D                    */
  FA_ERR_ALIGN = 4,            /* a pointer is not 16-byte aligned                */
  FA_ERR_UNSUPPORTED_ARCH = 5, /* current device is not sm_100 (B200)             */
  FA_ERR_LAUNCH = 6,           /* cudaLaunch / tensor-map encoding failed         */
  FA_ERR_TIMEOUT = 7,          /* a device-side wait exceeded its limit           */
  FA_ERR_WORKSPACE = 8,        /* workspace NULL or smaller than required         */
  FA_ERR_CUDA = 9,             /* another CUDA runtime error                      */
  FA_ERR_ARG = 10,             /* another invalid argument (scale not finite ...) */
  FA_ERR_NOALLOC_CAPACITY = 11, /* problem too large for fa_bwd_noalloc's scratch  */
  FA_ERR_DEBUG_CHECK = 12      /* a device-side check of the debug build failed   */
} fa_status;

/* Forward, bf16 in / bf16 out, fp32 accumulation (tcgen05 tensor cores).
 * Q/K/V tiles staged on chip and an online softmax with a running max and sum
 * that rescales the partial output ("LLM paper notes #8: FlashAttention",
 * adg.csdn.net, sections "tiling" and "online softmax"); lse is saved for the
 * backward ("recomputation").
 *   q, k, v : (B,H,N,D) bf16, read only.
 *   o       : (B,H,N,D) bf16, written (O = P V, rounded to nearest even).
 *   lse     : (B,H,N) float32, written (natural-log logsumexp of scale*q.k).
 *   scale   : the softmax scale (e.g. 1/sqrt(D)); must be finite and > 0.
 *   causal  : 0 = full attention, 1 = key j allowed for query i iff j <= i. */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int D, float scale, int causal, void* stream);

/* Forward with fp16 (IEEE binary16) q, k, v and o instead of bf16; otherwise
 * identical to fa_fwd (fp32 accumulation and softmax, fp32 lse).  FP16 is the
 * element type in which "CUDA-kernel-level optimisation: why Flash Attention is
 * 5-10x faster than native PyTorch" (guanweilu.cn, section "three lines of
 * PyTorch") and "Flash Attention principles: making Transformers faster"
 * (ijyty.com, section "memory bottleneck") size the N x N matrices.  P is
 * rounded to fp16 for the P V product, so it carries 3 more mantissa bits than
 * on the bf16 path.  Values of O beyond the fp16 range (|x| > 65504) become
 * +-inf. */
int fa_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse,
               int B, int H, int N, int D, float scale, int causal, void* stream);

/* Forward in fp32 throughout (fp32 in, fp32 FFMA arithmetic, fp32 out), for
 * callers that need ~1e-6 relative accuracy.  Same arguments as fa_fwd with
 * float32 tensors.  Computes the same tiled online softmax as fa_fwd ("LLM paper
 * notes #8: FlashAttention", adg.csdn.net, sections "tiling" and "online
 * softmax"), with every product and exponential in fp32. */
int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
               int B, int H, int N, int D, float scale, int causal, void* stream);

/* ---------------------------------------------------------------------------
 * Backward.  The gradients of O = softmax(S) V for a scalar loss, with P
 * recomputed from lse instead of stored ("LLM paper notes #8: FlashAttention",
 * adg.csdn.net, section "recomputation"; guanweilu.cn, section "three tricks"):
 *     dV = P^T dO,  dP = dO V^T,  delta_i = sum_d dO_id O_id,
 *     dS = P * (dP - delta),  dQ = scale dS K,  dK = scale dS^T Q.
 * Workspace layout (device memory owned by the caller, 16-byte aligned), with
 * Npad = N rounded up to a multiple of 128 and R = B*H*Npad rows:
 *   [0, R) floats            nl_i    = -lse_i * log2(e)   (padding rows: -inf)
 *   [R, 2R) floats           delta_i = sum_d dO_id * O_id (padding rows: 0)
 *   [2R, 2R + R*DK) floats   fp32 dQ accumulator of fa_bwd (head dims up to 128;
 *                            DK = 64 for D <= 64, 128 for D in {96, 128}); per
 *                            128-row query tile a block of 128 x DK floats laid
 *                            out [DK/4][128 rows][4].
 * ------------------------------------------------------------------------- */

/* Bytes of device workspace fa_bwd and fa_bwd_f16 need: 4 * R * (2 + DK) for
 * D <= 128 (statistics and dQ accumulator), 8 * R for D = 256 (statistics only).
 * A multiple of 1024.  Returns 0 for an unsupported shape. */
size_t fa_bwd_workspace_size(int B, int H, int N, int D);

/* Bytes of device workspace fa_bwd_deterministic and its stages (fa_bwd_dkdv,
 * fa_bwd_dq) need: the statistics only, 8 * R.  Returns 0 for an unsupported shape. */
size_t fa_bwd_deterministic_workspace_size(int B, int H, int N, int D);

/* Backward, bf16 (recomputes P from lse; never stores an N x N matrix).
 *   q, k, v, o, dO : (B,H,N,D) bf16 inputs; o and lse must be the outputs of
 *                    fa_fwd for the same q, k, v, scale and causal.
 *   lse            : (B,H,N) float32 from fa_fwd.
 *   dq, dk, dv     : (B,H,N,D) bf16, overwritten (not accumulated into).
 *   workspace      : device buffer of at least fa_bwd_workspace_size() bytes;
 *                    contents on entry ignored, clobbered on exit.
 * For D <= 128 one kernel per 128-key tile computes dK, dV and each tile's
 * contribution dS K to dQ, which it adds into the workspace's fp32 accumulator
 * with reductions in L2; equivalent to fa_bwd_preprocess, fa_bwd_dkdvdq and
 * fa_bwd_dq_finish on the same stream.  The order of those fp32 additions varies
 * from run to run, so dQ is reproducible to rounding (not bit for bit); dK and
 * dV are.  For D = 256 it runs the three-stage path of fa_bwd_deterministic. */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
           const float* lse, void* dq, void* dk, void* dv,
           void* workspace, size_t workspace_bytes,
           int B, int H, int N, int D, float scale, int causal, void* stream);

/* Backward with fp16 q, k, v, o, dO, dq, dk, dv (o and lse from fa_fwd_f16);
 * otherwise identical to fa_bwd, with the same workspace.  P and dS are rounded
 * to fp16 for the tensor-core products; gradients beyond the fp16 range become
 * +-inf. */
int fa_bwd_f16(const void* q, const void* k, const void* v, const void* o, const void* dO,
               const float* lse, void* dq, void* dk, void* dv,
               void* workspace, size_t workspace_bytes,
               int B, int H, int N, int D, float scale, int causal, void* stream);

/* Backward, bf16 only, bit-for-bit reproducible: the same formulas as fa_bwd in
 * three stages with no atomics (fa_bwd_preprocess, fa_bwd_dkdv, fa_bwd_dq):
 * every output tile is owned by one CTA, at the price of a second pass that
 * recomputes S and dP for dQ.  Workspace: at least
 * fa_bwd_deterministic_workspace_size() bytes (fa_bwd's workspace also fits). */
int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv,
                         void* workspace, size_t workspace_bytes,
                         int B, int H, int N, int D, float scale, int causal, void* stream);

/* Backward stage 1 (bf16): fills nl and delta from O, dO and lse (delta is the
 * row sum the softmax gradient subtracts, "recomputation", adg.csdn.net).  When
 * the workspace holds the dQ accumulator (workspace_bytes >=
 * fa_bwd_workspace_size and D <= 128) it is zeroed too. */
int fa_bwd_preprocess(const void* o, const void* dO, const float* lse,
                      void* workspace, size_t workspace_bytes,
                      int B, int H, int N, int D, void* stream);

/* Fused backward stage 2 (bf16, D <= 128): dK, dV (overwritten) and the dQ
 * contributions added into the accumulator that fa_bwd_preprocess zeroed.  Each
 * 128-key tile is owned by one CTA that walks the query tiles, recomputing P
 * from lse ("recomputation", adg.csdn.net).  Workspace: fa_bwd_workspace_size(). */
int fa_bwd_dkdvdq(const void* q, const void* k, const void* v, const void* dO,
                  void* workspace, size_t workspace_bytes, void* dk, void* dv,
                  int B, int H, int N, int D, float scale, int causal, void* stream);

/* Fused backward stage 3 (bf16, D <= 128): dq = scale * accumulator, rounded to
 * bf16 (the "dQ finish" of the backward).  Workspace: fa_bwd_workspace_size(). */
int fa_bwd_dq_finish(const void* workspace, size_t workspace_bytes, void* dq,
                     int B, int H, int N, int D, float scale, void* stream);

/* Deterministic stage 2 (bf16): dK, dV (overwritten), reading the statistics that
 * stage 1 filled.  Each 128-key tile is owned by one CTA that walks the query
 * rows, recomputing P from lse ("recomputation", adg.csdn.net), so dK and dV
 * need no atomics.  Workspace: fa_bwd_deterministic_workspace_size(). */
int fa_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO,
                const void* workspace, size_t workspace_bytes, void* dk, void* dv,
                int B, int H, int N, int D, float scale, int causal, void* stream);

/* Deterministic stage 3 (bf16): dQ (overwritten), reading the statistics that
 * stage 1 filled.  Each 256-query block is owned by one CTA that walks the key
 * tiles and recomputes S, P and dP for them, so dQ needs no atomics.
 * Workspace: fa_bwd_deterministic_workspace_size(). */
int fa_bwd_dq(const void* q, const void* k, const void* v, const void* dO,
              const void* workspace, size_t workspace_bytes, void* dq,
              int B, int H, int N, int D, float scale, int causal, void* stream);

/* Size of the fixed device scratch array that fa_bwd_noalloc uses (8 MiB). */
#define FA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)

/* Backward that allocates nothing and takes no workspace (bf16 only).  The paper
 * has no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory -- code that a host framework hands only its input and
 * output buffers, with all device memory planned up front and no workspace or
 * allocator available to the operator.
 *   Same arguments, layout and errors as fa_bwd_deterministic minus the workspace,
 *     and the same results bit for bit (it runs the same three kernels).
 *   Scratch: a fixed FA_NOALLOC_SCRATCH_BYTES array in the library's own device
 *     memory (held by every GPU that loads the library until the process exits).
 *     Limit: fa_bwd_deterministic_workspace_size(B, H, N, D) <= FA_NOALLOC_SCRATCH_BYTES,
 *     i.e. B*H*ceil(N/128)*128 <= 1,048,576 rows; larger problems return
 *     FA_ERR_NOALLOC_CAPACITY before anything is launched.
 *   Set-up: the first call on a device looks up the array's device address
 *     (with that device current); make that first call before any stream capture.
 *     A failed lookup is not remembered: the next call on that device tries again.
 *   Sharing: every call uses the same array; nothing in it needs to start at zero
 *     (each call rewrites what it reads), but calls whose work overlaps on the GPU
 *     (unordered streams) race on it. */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                   const float* lse, void* dq, void* dk, void* dv,
                   int B, int H, int N, int D, float scale, int causal, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(int status);

/* Reads the device status word of the current device (synchronises the
 * device first).  Returns FA_OK or the first FA_ERR_* a kernel recorded;
 * if reset != 0 the word is cleared afterwards.  Kernels record
 * FA_ERR_TIMEOUT (a pipeline wait ran out) and FA_ERR_LAUNCH (a launch they
 * cannot use); the debug build of the library (libfa_debug.so, compiled with
 * FA_DEBUG_CHECKS) also records FA_ERR_DEBUG_CHECK when a computed index falls
 * outside its buffer or a warp reaches a warp-collective tensor-memory
 * operation diverged, and skips that access instead of performing it. */
int fa_device_status(int reset);

/* Library version, major*10000 + minor*100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
