// Internal parameter blocks and launchers shared by the C ABI and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sage.h"

namespace sage {

// A buffer the kernels write: [base, base + bytes).  In the checked build (-DSAGE_CHECKED) every
// global store is tested against the extent of the buffer it targets; a store outside it is
// skipped and recorded in the kernel's device error word (SAGE_DEVERR_BOUNDS), never made.
struct Extent {
  unsigned char* base;
  unsigned long long bytes;
};
enum : int { SAGE_DEVERR_BOUNDS = 4 };

#ifdef SAGE_CHECKED
__device__ __forceinline__ bool store_in_extent(const Extent& x, const void* ptr, unsigned long long n, int* err) {
  const unsigned char* q = static_cast<const unsigned char*>(ptr);
  const bool ok = x.base != nullptr && q >= x.base && q + n <= x.base + x.bytes;
  if (!ok) atomicOr(err, SAGE_DEVERR_BOUNDS);
  return ok;
}
#define SAGE_STORE_OK(x, ptr, n, err) ::sage::store_in_extent((x), (ptr), (n), (err))
#else
#define SAGE_STORE_OK(x, ptr, n, err) true
#endif

// One sequence of a packed (varlen) batch, as the planning kernel lays it out.
struct SeqDesc {
  int nq, nk;              // query / key tokens
  int q_row, k_row;        // first row of the sequence inside one head's range of q8 / k8 rows (multiple of 128)
  long long q_tok, k_tok;  // first token of the sequence in the packed caller tensors
};

// Where the sequences of a batch live, in the caller's tensors and in the quantized buffers.
//   dense batch (seqs == nullptr): every sequence has Nq queries and Nk keys; inputs in `layout`;
//     q8 rows [B][Hq][Npq], k8 rows [B][Hkv][Npk], V^T [B][Hkv][dp][Npk]  (Np = 128 * ceil(N / 128));
//   packed batch: per-sequence table; inputs (total, H, d);
//     q8 rows [Hq][Tq], k8 rows [Hkv][Tk], V^T [Hkv][dp][Tk], sequence b at rows / columns
//     q_row / k_row of each head's range.
// In both, row (sequence b, head h, token t) of q8 is q_row0(b) + h * q_head_rows + t, the scale of
// its 128-token block is entry row / 128 of qs, and likewise for k8 / ks; V^T rows have pitch
// k_head_rows codes.
struct SeqMap {
  const SeqDesc* seqs;
  int B, Hq, Hkv, d, dp;
  int Nq, Nk;                          // dense lengths (packed: the longest sequence's)
  long long q_head_rows, k_head_rows;  // dense: Npq, Npk; packed: Tq, Tk
  int layout;                          // dense input / output layout (sage_layout)
};

struct SeqView {
  int nq, nk;
  long long q_row0, k_row0;  // q8 / k8 row of (this sequence, head 0, token 0)
  long long v_row0, v_col0;  // V^T row of (this sequence, kv head 0, channel 0), column of token 0
  long long q_in, k_in;      // element offset of (this sequence, token 0, head 0) in q (and out) / in k and v
  long long q_tok, q_head;   // element strides of q (and out) between tokens / heads
  long long k_tok, k_head;   // element strides of k and v
};

// PACKED: 1 = the table, 0 = the dense formulas (lengths then stay kernel parameters), -1 = decide
// at run time by m.seqs.
template <int PACKED = -1>
__host__ __device__ inline SeqView seq_view(const SeqMap& m, int b) {
  SeqView v;
  if (PACKED == 1 || (PACKED == -1 && m.seqs)) {
    const SeqDesc s = m.seqs[b];
    v.nq = s.nq, v.nk = s.nk;
    v.q_row0 = s.q_row, v.k_row0 = s.k_row;
    v.v_row0 = 0, v.v_col0 = s.k_row;
    v.q_tok = (long long)m.Hq * m.d, v.q_head = m.d;
    v.k_tok = (long long)m.Hkv * m.d, v.k_head = m.d;
    v.q_in = s.q_tok * v.q_tok, v.k_in = s.k_tok * v.k_tok;
  } else {
    v.nq = m.Nq, v.nk = m.Nk;
    v.q_row0 = (long long)b * m.Hq * m.q_head_rows;
    v.k_row0 = (long long)b * m.Hkv * m.k_head_rows;
    v.v_row0 = (long long)b * m.Hkv * m.dp, v.v_col0 = 0;
    if (m.layout == SAGE_HND) {
      v.q_tok = m.d, v.q_head = (long long)m.Nq * m.d;
      v.k_tok = m.d, v.k_head = (long long)m.Nk * m.d;
    } else {
      v.q_tok = (long long)m.Hq * m.d, v.q_head = m.d;
      v.k_tok = (long long)m.Hkv * m.d, v.k_head = m.d;
    }
    v.q_in = (long long)b * m.Hq * m.Nq * m.d;
    v.k_in = (long long)b * m.Hkv * m.Nk * m.d;
  }
  return v;
}

struct QuantParams {
  const void* q;
  const void* k;
  const void* v;
  SeqMap m;
  int nblk_q, nblk_k;  // 128-token blocks of the longest query / key sequence (grid extents)
  int dtype;           // sage_dtype
  bool vec_q, vec_k, vec_v;  // 16-byte vector loads allowed (d % 8 == 0 and 16-byte aligned base)
  int8_t* q8;
  float* qs;
  int8_t* k8;
  float* ks;
  float* km;
  uint8_t* v8t;
  float* vs;
  // scratch
  float* ksum_part;  // [k rows / 128][dp]: per 128-token block of K
  float* vmax_part;  // [k rows / 128][dp]
  float* vinv;       // [B][Hkv][dp]
  float* vsum_part;  // [k rows / 128][dp] (V smoothing only)
  float* vmin_part;  // [k rows / 128][dp] (V smoothing only; vmax_part then holds max v, not max |v|)
  float* vm;         // [B][Hkv][dp] V's token mean (nullptr allowed when smooth_v is 0)
  int smooth_v;      // code V - vm instead of V
  int q_gran_log2;   // query tokens per Q scale: 7 (128), 5 (32) or 0 (1)
  int bpc;           // 128-token blocks per CTA of the two passes (grid x = ceil(blocks / bpc))
  int prefetch;      // stream the next block into shared memory while one is processed (dp <= 128)
  float vmax_code;   // 448 (FP8 P.V, fp32 accumulation) or 1 (the other P.V modes)
  int v_fp16;        // V codes are fp16 (FP16 P.V) instead of E4M3; v8t then holds 2 bytes per code
  int fold;          // pass 2 computes the K mean and V scales itself (no finalize launch)
  // extents of the buffers above (store checks of the checked build)
  Extent x_q8, x_qs, x_k8, x_ks, x_km, x_v8t, x_vs, x_vm, x_vinv, x_ksum, x_vmax, x_vsum, x_vmin;
};

struct FwdParams {
  const float* qs;
  const float* ks;
  const float* vs;
  const float* vm;  // V's token mean, added to the output (nullptr: V not smoothed)
  void* out;
  SeqMap m;
  int q_gran_log2;  // query tokens per Q scale = 1 << q_gran_log2
  int nblk_q;     // 128-row query tiles of the longest sequence (grid x)
  int G;          // query heads per kv head
  int vec_out;    // 16-byte output stores allowed (d % 8 == 0 and 16-byte aligned out)
  float scale_log2;  // sm_scale * log2(e)
  Extent x_out;      // the output tensor (store checks of the checked build)
};

struct QkDumpParams {
  const int32_t* tiles;  // n_tiles x {b, hq, q_tile, k_tile}
  int n_tiles;
  int32_t* out;  // n_tiles x 128 x 128
  int B, Hq, Hkv, Np, nblk, G;
};

cudaError_t launch_quantize(const QuantParams& p, cudaStream_t st);
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int dtype, int causal, int pv_mode, cudaStream_t st);
// Packed batches: per-sequence table from the caller's cumulative lengths (validated on the device;
// a bad table flags SAGE_ERR_INVALID_ARG and leaves every sequence empty).
cudaError_t launch_seq_plan(const int32_t* cu_q, const int32_t* cu_k, int B, int max_q, int max_k,
                            long long total_q, long long total_k, SeqDesc* seqs, cudaStream_t st);
cudaError_t read_clear_device_error(int* value);
cudaError_t read_clear_quant_error(int* value);  // the quantize kernels' error word (quant.cu)
cudaError_t launch_wait_probe(long long budget_cycles, cudaStream_t st);
// tcgen05.mma issue-rate probe: kind 0 = kind::i8, 1 = kind::f8f6f4, 2 = kind::f16; one CTA per SM.
cudaError_t launch_mma_probe(int kind, int iters, int n_sm, cudaStream_t st);
cudaError_t launch_qk_dump(const CUtensorMap& tq, const CUtensorMap& tk, const QkDumpParams& p, int dp,
                           cudaStream_t st);

}  // namespace sage
