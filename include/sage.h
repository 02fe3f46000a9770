/*
 * sage.h -- C ABI of an INT8-QK / FP8-PV quantized attention library for
 * NVIDIA B200 (sm_100a).
 *
 * The operation is scaled-dot-product attention
 *     out = softmax(Q K^T * sm_scale [+ causal mask]) V
 * computed the SageAttention way (SageAttention README, "Current Features"):
 * K is smoothed by subtracting its per-channel token mean, Q and K are
 * quantized to INT8 with one fp32 scale per 128-token block, Q K^T runs as an
 * INT8 tensor-core product, the scores go through an online softmax, P is
 * requantized to FP8 E4M3 and P V runs as an FP8 tensor-core product with
 * fp32 accumulation or with the two-level fp16+fp32 accumulation.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never keeps a pointer after the call returns; work is queued on `stream`
 *    (a cudaStream_t; NULL = the legacy default stream) and may still be
 *    running when the call returns.
 *  - Q, K, V and out are dense and contiguous in the given layout
 *    (SageAttention README, "How to Use", tensor_layout):
 *        SAGE_HND: (B, H, N, d)      SAGE_NHD: (B, N, H, d)
 *    with H = Hq for Q and out, H = Hkv for K and V.
 *  - Inputs are fp16 or bf16 (fp32 is rejected with SAGE_ERR_UNSUPPORTED, as the
 *    reference API only accepts 16-bit inputs); out has the input dtype.
 *  - GQA: Hq must be a multiple of Hkv; query head h reads kv head
 *    h / (Hq / Hkv) (qwbw.cn article, pitfalls section).
 *  - head dim 1 <= d <= 256; internally it is zero-padded to dp = 64, 128 or
 *    256, the smallest that holds d (same section, pad_qkv).
 *  - Causal masking keeps key j for query i iff j <= i (Nq = Nk = N).
 *  - Errors: argument checks run first and return without touching the GPU or
 *    writing any output.  A CUDA launch or allocation failure returns
 *    SAGE_ERR_CUDA / SAGE_ERR_OOM.  Kernel-side timeouts (every wait inside the
 *    kernels is bounded) are reported later by sage_check_status().
 *  - A device other than compute capability 10.0 (B200) returns SAGE_ERR_ARCH.
 */
#ifndef SAGE_B200_H_
#define SAGE_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,
  SAGE_ERR_UNSUPPORTED = 2,
  SAGE_ERR_ARCH = 3,
  SAGE_ERR_CUDA = 4,
  SAGE_ERR_OOM = 5,
  SAGE_ERR_TIMEOUT = 6,
  SAGE_ERR_BOUNDS = 7
} sage_status;

typedef enum { SAGE_HND = 0, SAGE_NHD = 1 } sage_layout;
typedef enum { SAGE_FP16 = 0, SAGE_BF16 = 1, SAGE_FP32 = 2 } sage_dtype;

/* P.V operands and accumulation (SageAttention README, "Current Features": FP8
 * PV, FP16 accumulator for FP8 PV and two-level accumulation; "Available APIs":
 * the INT8-QK / FP16-PV CUDA kernel; qwbw.cn article, pitfalls: pv_accum_dtype
 * = "fp32" | "fp16+fp32").
 *   SAGE_PV_FP32        FP8 (E4M3) P and V; P8.V8 accumulates in fp32 across
 *                       all key tiles.
 *   SAGE_PV_FP16_FP32   FP8 P and V; each 128-key tile's P8.V8 goes to a fresh
 *                       fp16 accumulator, which is then added into an fp32 O.
 *                       V codes then span [-1, 1] (instead of [-448, 448]) so
 *                       one tile's fp16 partial (<= 128*448*1) cannot overflow.
 *   SAGE_PV16_FP32      FP16 P and V (V codes = fp16(v / amax_channel), in
 *                       [-1, 1]); fp32 accumulation.  Key tiles of 64.
 *   SAGE_PV16_FP16_FP32 FP16 P and V; each 64-key tile's P.V in a fresh fp16
 *                       accumulator (|partial| <= 64 * 4 * 1), added into fp32 O.
 *   SAGE_PV16_FP16      FP16 P and V accumulated in fp16 across all key tiles
 *                       (pitfalls section: pv_accum_dtype "fp16", the fastest and
 *                       least overflow-safe option on the GPUs the pages target).
 *                       Not offered: every entry point returns
 *                       SAGE_ERR_UNSUPPORTED.  On sm_100a a tcgen05.mma issues at the
 *                       same rate with an F16 as with an F32 accumulator, so the
 *                       mode would only add rounding error and overflow risk.
 * Bit 0 of the value selects fp16+fp32 accumulation, bit 1 FP16 operands, bit 2
 * pure fp16 accumulation. */
typedef enum {
  SAGE_PV_FP32 = 0,
  SAGE_PV_FP16_FP32 = 1,
  SAGE_PV16_FP32 = 2,
  SAGE_PV16_FP16_FP32 = 3,
  SAGE_PV16_FP16 = 6
} sage_pv_mode;

/* Optional quantization settings (SageAttention README, "Current Features":
 * INT8 quantization for Q K^T with varying granularities; news of 2024-12-20:
 * per-thread quantization; the SageAttention2 title's outlier smoothing).
 *   q_gran    query tokens per Q scale: 128 (per block, the default), 32 (per
 *             warp: the rows one warp of the fused kernel owns) or 1 (per
 *             thread: one thread of the fused kernel owns one query row);
 *             0 selects 128.  K keeps one scale per 128-token block.
 *   smooth_v  1: code V - mean_tokens(V) (the mean summed in the same fixed
 *             order as K's) and add the mean back to the output (rows that
 *             see no key stay 0).  0: code V itself.
 * A NULL sage_opts pointer means {128, 0}. */
typedef struct {
  int q_gran;
  int smooth_v;
} sage_opts;

/* Quantized attention, end to end: quantize/smooth pass, then the fused
 * attention kernel.  q: (B,Hq,N,d), k and v: (B,Hkv,N,d), out: (B,Hq,N,d), all
 * in `layout`, dtype `dtype`.  sm_scale <= 0 or NaN selects 1/sqrt(d) (the
 * original d).  The quantized copies of Q/K/V live in a workspace taken
 * stream-ordered on `stream` from a per-device memory pool that the library
 * creates on first use and that keeps its memory for later calls (it holds as
 * much device memory as the largest workspace in flight, until the process
 * exits); the workspace is released stream-ordered before return.
 * SAGE_ERR_OOM if it cannot be allocated.  out must not overlap q, k or v.
 * The call may be captured in a CUDA graph (the workspace then becomes the
 * graph's allocation nodes); the finalize / pass-2 / attention kernels are
 * launched as programmatic dependents of the kernel before them. */
sage_status sage_attn(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv, int N, int d,
                      sage_dtype dtype, sage_layout layout, int is_causal, float sm_scale, sage_pv_mode pv_mode,
                      void* stream);

/* sage_attn with different query and key lengths (SageAttention README news,
 * 2024-11-11: different sequence lengths between q and k, v).  q, out:
 * (B,Hq,Nq,d), k and v: (B,Hkv,Nk,d), in `layout`.  Under is_causal the mask is
 * aligned bottom-right: query i sees keys j <= i + (Nk - Nq), so the last query
 * sees every key; a query that sees no key (Nq > Nk) gets zeros.  Nq = Nk is
 * exactly sage_attn (with opts NULL).  opts: see sage_opts.  Workspace, errors
 * and ownership as sage_attn. */
sage_status sage_attn_ex(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv, int Nq,
                         int Nk, int d, sage_dtype dtype, sage_layout layout, int is_causal, float sm_scale,
                         sage_pv_mode pv_mode, const sage_opts* opts, void* stream);

/* Packed batch of sequences of different lengths (SageAttention README,
 * "Available APIs": sageattn_varlen).  q, out: (total_q, Hq, d); k, v:
 * (total_k, Hkv, d), tokens of all sequences one after the other (contiguous).
 * cu_seqlens_q / cu_seqlens_k: DEVICE int32 arrays of B + 1 non-decreasing
 * offsets; sequence b owns query tokens cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 * and key tokens cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1.  Every sequence is
 * quantized on its own (K mean, 128-token blocks and V scales per sequence) and
 * attends only to its own keys, with the causal mask aligned bottom-right per
 * sequence; queries that see no key (including sequences with no keys) get
 * zeros.  max_seqlen_q >= 1 and max_seqlen_k >= 0 bound every sequence's
 * lengths; cu_seqlens_*[B] must not exceed total_q / total_k.  The table is
 * checked on the device: a violation is reported by sage_check_status as
 * SAGE_ERR_INVALID_ARG, and then no output is written.  Workspace, other errors
 * and ownership as sage_attn. */
sage_status sage_attn_varlen(const void* q, const void* k, const void* v, void* out, const int32_t* cu_seqlens_q,
                             const int32_t* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k,
                             long long total_q, long long total_k, int Hq, int Hkv, int d, sage_dtype dtype,
                             int is_causal, float sm_scale, sage_pv_mode pv_mode, const sage_opts* opts,
                             void* stream);

/* Bytes of workspace sage_attn takes for these sizes, the largest over the P.V
 * modes (0 on invalid sizes). */
size_t sage_workspace_bytes(int B, int Hq, int Hkv, int N, int d);

/* The quantize/smooth pass alone (K token mean, INT8 Q and K - mean(K) codes with
 * per-128-token-block scales, E4M3 or fp16 V codes with per-channel scales).
 * Outputs, with Np = 128 * ceil(N / 128) and dp the padded head dim, all device
 * memory:
 *   q8  int8   [B][Hq][Np][dp]     qs  fp32 [B][Hq][Np/128]
 *   k8  int8   [B][Hkv][Np][dp]    ks  fp32 [B][Hkv][Np/128]    km fp32 [B][Hkv][dp]
 *   v8t        [B][Hkv][dp][Np]    V codes, transposed (keys contiguous): E4M3
 *                                  bytes (SAGE_PV_FP32, SAGE_PV_FP16_FP32) or
 *                                  fp16 values, 2 bytes each (SAGE_PV16_*)
 *   vs  fp32   [B][Hkv][dp]
 *   vm  fp32   [B][Hkv][dp]         V's token mean (zeros unless opts->smooth_v)
 * qs holds Np / q_gran scales per (b, head) (opts->q_gran, 128 by default).
 * Padded tokens and channels hold code 0 (and km 0, vs 0, vm 0).  Codes and scales
 * follow: amax over the block's real tokens and channels, inv = 127 / amax,
 * code = clamp(rint_even(x * inv), -127, 127), scale = amax / 127 (0 when amax
 * is 0); K is smoothed as x = k - km, km summed in fp32 in this order: each
 * 128-token block is split into 8 groups of 16 consecutive tokens, each group is
 * summed token by token from +0.0 (tokens >= N skipped), the block's partial is
 * the pairwise tree ((g0 + g1) + (g2 + g3)) + ((g4 + g5) + (g6 + g7)), the block
 * partials are added one by one in block order from +0.0, and the total is
 * divided by (float)N with one IEEE division (every add and the division round
 * to nearest even); the order is part of the bit-exact contract;
 * V: inv = VMAX / amax_channel, code = E4M3_rne_satfinite(v * inv) (FP8 modes)
 * or fp16_rne(v * inv) (FP16 modes), vs = amax / VMAX with VMAX = 448
 * (SAGE_PV_FP32) or 1 (the other modes); with smooth_v, v - vm in place of v
 * (vm summed like km).  vm may be NULL when smooth_v is off.
 * Its own small scratch comes from the same per-device pool as sage_attn's. */
sage_status sage_quantize(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int N, int d,
                          sage_dtype dtype, sage_layout layout, sage_pv_mode pv_mode, const sage_opts* opts,
                          int8_t* q8, float* qs, int8_t* k8, float* ks, float* km, uint8_t* v8t, float* vs,
                          float* vm, void* stream);

/* The fused attention kernel alone, on buffers in the layouts sage_quantize
 * writes with the same opts.  out: (B,Hq,N,d) in `out_layout`, dtype
 * `out_dtype`.  vm is added to the output when opts->smooth_v (NULL allowed
 * otherwise).  Allocates nothing. */
sage_status sage_attn_quantized(const int8_t* q8, const float* qs, const int8_t* k8, const float* ks,
                                const uint8_t* v8t, const float* vs, const float* vm, void* out, int B, int Hq,
                                int Hkv, int N, int d, sage_dtype out_dtype, sage_layout out_layout, int is_causal,
                                float sm_scale, sage_pv_mode pv_mode, const sage_opts* opts, void* stream);

/* Diagnostic: the exact int32 scores S = Q8 . K8^T of selected 128x128 tiles,
 * computed by the same TMA + tcgen05 kind::i8 path as the fused kernel.
 * tiles: DEVICE int32 array of n_tiles records {b, hq, q_tile, k_tile};
 * s_out: DEVICE int32 [n_tiles][128][128], row = query, column = key.  q8/k8
 * as written by sage_quantize.  Out-of-range records are skipped and flagged
 * (sage_check_status returns SAGE_ERR_INVALID_ARG).  Allocates nothing. */
sage_status sage_qk_int32(const int8_t* q8, const int8_t* k8, int B, int Hq, int Hkv, int N, int d,
                          const int32_t* tiles, int n_tiles, int32_t* s_out, void* stream);

/* Diagnostic for the failure path (no counterpart on the pages): launches one
 * block whose bounded wait, the same wait every pipeline stage of the kernels
 * uses, is on a barrier that nothing completes; it gives up after about
 * budget_us microseconds (1 .. 100000) at the GPU's base clock, records the
 * timeout and returns.  sage_check_status then reports SAGE_ERR_TIMEOUT, and
 * the context stays usable.  SAGE_ERR_INVALID_ARG for a budget out of range. */
sage_status sage_selftest_wait_timeout(int budget_us, void* stream);

/* Diagnostic (no counterpart on the pages): measures nothing itself, but launches
 * one CTA per SM whose single thread issues `iters` x 4 back-to-back tcgen05.mma of
 * M = 128, N = 256 and 32 bytes of K per operand row (kind 0: kind::i8, K = 32;
 * kind 1: kind::f8f6f4 with E4M3 operands, K = 32; kind 2: kind::f16, K = 16) into
 * one tensor-memory accumulator, and waits for them.  *ops receives the
 * operations the launch performs (SMs x iters x 4 x 2 x 128 x 256 x K); the caller
 * times the launch on `stream` (CUDA events) to get the GPU's tensor-core rate for
 * that kind.  SAGE_ERR_INVALID_ARG for a kind outside 0..2, iters outside
 * 1..1000000 or a NULL ops. */
sage_status sage_mma_probe(int kind, int iters, double* ops, void* stream);

/* Synchronizes `stream`, then reports (and clears) the device-side error word:
 * SAGE_ERR_TIMEOUT if a kernel gave up on a bounded wait, SAGE_ERR_BOUNDS if a
 * kernel of the checked build skipped a store outside its buffer (see
 * sage_checked_build), SAGE_ERR_INVALID_ARG for a flagged tile record or
 * cu_seqlens table, SAGE_ERR_CUDA for a pending CUDA error.  The error word is one per device, not per stream: it collects the
 * flags of every call on the current device since it was last read, whatever
 * stream they ran on, and the first sage_check_status to read it (on any stream)
 * reports and clears them.  Only `stream` is synchronized, so a call still
 * running on another stream may flag an error after the read. */
sage_status sage_check_status(void* stream);

/* Static description of a status code. */
const char* sage_status_string(sage_status s);

/* 1 if the current CUDA device can run this library (compute capability 10.0). */
int sage_device_supported(void);

/* Test hook for the failure paths (no counterpart on the pages): host-side
 * injection, with no GPU fault and no device call.  fake_cc > 0: the device check
 * reports that compute capability (major * 10 + minor) instead of querying the
 * device -- 100 passes as a B200, anything else gives SAGE_ERR_ARCH; 0 restores the
 * real query.  fail_allocs > 0: that many of the following workspace allocations
 * fail with SAGE_ERR_OOM before touching the device (0 clears it).  Process-wide;
 * not for use outside tests. */
void sage_test_inject(int fake_cc, int fail_allocs);

/* 1 for the checked build of this library (compiled with -DSAGE_CHECKED, shipped
 * beside the normal one as libsage_b200_checked.so), else 0.  In the checked build
 * every global-memory store of the quantize kernels and of the fused attention
 * kernel first tests that its bytes lie inside the buffer they belong to (sized as
 * this header states: out, the sage_quantize outputs, the workspace's parts); a
 * store outside is skipped, never made, and sage_check_status reports
 * SAGE_ERR_BOUNDS.  (The per-sequence table of packed batches and the tiles of
 * sage_qk_int32 are written at indices that their launch bounds: not checked.)
 * Results are bit-identical to the normal build's; the normal build compiles the
 * tests out. */
int sage_checked_build(void);

/* Test hook for the checked build (no counterpart on the pages): bytes > 0
 * narrows the extent the kernels take for `out` to its first `bytes` bytes, so a
 * call's stores past them are skipped and reported (SAGE_ERR_BOUNDS); 0 restores
 * the full size.  No effect on the normal build.  Process-wide; not for use
 * outside tests. */
void sage_test_out_limit(long long bytes);

/* Largest workspace sage_attn_noalloc can hold: 64 MiB (for example B=2, H=24,
 * N=4096, d=64 with pv_mode SAGE_PV_FP32 needs about 38 MiB). */
#define SAGE_NOALLOC_MAX_BYTES (64u << 20)

/* sage_attn without any device allocation.  The paper has no counterpart: this
 * entry point exists for callers that cannot call cudaMalloc/cudaMallocAsync at
 * call time -- for example a host framework or server that reserves all device
 * memory up front and treats any other allocation as an error, a runtime whose
 * allocations are forbidden after initialisation, or a GPU/driver setup without
 * stream-ordered memory pools.  Same arguments, checks and result as sage_attn.
 *
 * Its workspace is one static device array of SAGE_NOALLOC_MAX_BYTES inside this
 * library: every GPU that loads the library holds that memory until the process
 * exits.  A call whose own workspace -- the quantized Q, K, V, their scales and
 * the quantize pass's partial sums for these sizes and this pv_mode, default
 * options -- exceeds the maximum is rejected with SAGE_ERR_INVALID_ARG before any
 * GPU work.  sage_workspace_bytes() is an upper bound of that figure (it takes the
 * largest P.V mode and options), so sizes it keeps within the maximum are always
 * accepted.  The first call on each
 * device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.  All calls
 * share the one array and it keeps the previous call's contents (every byte a call
 * reads is written by the same call first), so calls that can overlap on the GPU --
 * on different streams, or from different host threads -- race with each other:
 * order them on one stream or synchronise between them.  It allocates nothing: no
 * cudaMalloc, cudaFree or allocating library routine is called. */
sage_status sage_attn_noalloc(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv, int N,
                              int d, sage_dtype dtype, sage_layout layout, int is_causal, float sm_scale,
                              sage_pv_mode pv_mode, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_B200_H_ */
