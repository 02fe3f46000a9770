// Internal parameter blocks and launchers shared by the C ABI and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sage.h"

namespace sage {

struct QuantParams {
  const void* q;
  const void* k;
  const void* v;
  int B, Hq, Hkv, N, d, dp, Np, nblk;
  int layout;  // sage_layout
  int dtype;   // sage_dtype
  bool vec_q, vec_k, vec_v;  // 16-byte vector loads allowed (d % 8 == 0 and 16-byte aligned base)
  int8_t* q8;
  float* qs;
  int8_t* k8;
  float* ks;
  float* km;
  uint8_t* v8t;
  float* vs;
  // scratch
  float* ksum_part;  // [B][Hkv][nblk][dp]
  float* vmax_part;  // [B][Hkv][nblk][dp]
  float* vinv;       // [B][Hkv][dp]
  float vmax_code;   // 448 (FP8 P.V, fp32 accumulation) or 1 (the other P.V modes)
  int v_fp16;        // V codes are fp16 (FP16 P.V) instead of E4M3; v8t then holds 2 bytes per code
};

struct FwdParams {
  const float* qs;
  const float* ks;
  const float* vs;
  void* out;
  int B, Hq, Hkv, N, Np, nblk, d, dp, G;
  int layout;     // output layout (sage_layout)
  int n_vhalves;  // output column halves handled by separate CTAs (2 when dp = 256)
  int vec_out;    // 16-byte output stores allowed (d % 8 == 0 and 16-byte aligned out)
  float scale_log2;  // sm_scale * log2(e)
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
cudaError_t read_clear_device_error(int* value);
cudaError_t launch_qk_dump(const CUtensorMap& tq, const CUtensorMap& tk, const QkDumpParams& p, int dp,
                           cudaStream_t st);

}  // namespace sage
