// Quantize / smooth pass (one read of Q, two of K and V):
//
//   pass 1  per (batch, head, 128-token block):
//             Q -> INT8 codes + per-block scale (final);
//             K -> per-block partial column sums (for the token mean);
//             V -> per-block partial column max |v| (for the per-channel scale).
//   finalize per (batch, kv-head): k_mean = (sum of partials in block order) / N,
//             v_scale = amax / VMAX, v_inv = VMAX / amax.
//   pass 2  per (batch, kv-head, block):
//             K - k_mean -> INT8 codes + per-block scale;
//             V -> E4M3 codes, written transposed (keys contiguous) for the P.V MMA.
//
// Method: INT8 quantization with smoothing for Q K^T and FP8 quantization for
// P V (SageAttention README, "Current Features").  The block size, the
// symmetric rounding, the order of the K-mean sum and the V code range are
// this library's readings of what the pages leave open; every float operation
// below is an explicit IEEE round-to-nearest operation (__fadd_rn, __fmul_rn,
// __fdiv_rn) so the results are reproducible bit for bit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sage_internal.h"

namespace sage {

__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Copy rows [n0, n0 + rows) of one head into a zero-padded shared tile
// tile[128][dp] (16-bit elements, row stride dp).
template <typename T>
__device__ void load_tile(T* tile, const T* __restrict__ x, int b, int h, int H, int N, int d, int dp, int n0,
                          int rows, int layout, bool vec) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  // zero the whole tile first (padding rows and channels)
  uint4* t4 = reinterpret_cast<uint4*>(tile);
  const int n16 = 128 * dp * (int)sizeof(T) / 16;
  for (int i = tid; i < n16; i += nthr) t4[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  auto row_ptr = [&](int n) -> const T* {
    const size_t off = (layout == SAGE_HND) ? ((size_t)(b * H + h) * N + n) * d : ((size_t)(b * N + n) * H + h) * d;
    return x + off;
  };
  if (vec) {
    const int vpr = d / 8;  // 16-byte vectors per row
    for (int i = tid; i < rows * vpr; i += nthr) {
      const int r = i / vpr, cv = i - r * vpr;
      const uint4 val = __ldg(reinterpret_cast<const uint4*>(row_ptr(n0 + r)) + cv);
      *reinterpret_cast<uint4*>(tile + r * dp + cv * 8) = val;
    }
  } else {
    for (int i = tid; i < rows * d; i += nthr) {
      const int r = i / d, c = i - r * d;
      tile[r * dp + c] = row_ptr(n0 + r)[c];
    }
  }
  __syncthreads();
}

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < nw; ++i) r = fmaxf(r, red[i]);
  return r;
}

// INT8 codes of a 128 x dp tile: x(r, c) is given by `val`, which must return 0
// for padding.  Writes 128*dp bytes contiguously at `dst`.
template <typename F>
__device__ void write_int8_codes(int8_t* __restrict__ dst, int dp, float inv, F val) {
  const int nchunk = 128 * dp / 16;
  for (int o = threadIdx.x; o < nchunk; o += blockDim.x) {
    const int r = (o * 16) / dp, c0 = (o * 16) - r * dp;
    uint32_t w[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int code = __float2int_rn(__fmul_rn(val(r, c0 + g * 4 + e), inv));  // rint: ties to even
        code = max(-127, min(127, code));
        packed |= (uint32_t)(code & 0xFF) << (8 * e);
      }
      w[g] = packed;
    }
    *reinterpret_cast<uint4*>(dst + (size_t)o * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) quant_pass1_kernel(QuantParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* tile = reinterpret_cast<T*>(smem_raw);
  __shared__ float red[8];
  const int blk = blockIdx.x, y = blockIdx.y, b = blockIdx.z;
  const int n0 = blk * 128, rows = min(128, p.N - n0);
  const int dp = p.dp, d = p.d;
  if (y < p.Hq) {  // ---- Q: final INT8 codes and per-block scale
    const int h = y;
    load_tile<T>(tile, static_cast<const T*>(p.q), b, h, p.Hq, p.N, d, dp, n0, rows, p.layout, p.vec_q);
    float am = 0.f;
    for (int i = threadIdx.x; i < rows * dp; i += blockDim.x) am = fmaxf(am, fabsf(to_f32(tile[i])));
    am = block_max(am, red);
    const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
    const size_t bh = (size_t)b * p.Hq + h;
    write_int8_codes(p.q8 + (bh * p.Np + n0) * dp, dp, inv, [&](int r, int c) { return to_f32(tile[r * dp + c]); });
    if (threadIdx.x == 0) p.qs[bh * p.nblk + blk] = __fdiv_rn(am, 127.f);
  } else if (y < p.Hq + p.Hkv) {  // ---- K: per-block partial column sums, token by token
    const int h = y - p.Hq;
    load_tile<T>(tile, static_cast<const T*>(p.k), b, h, p.Hkv, p.N, d, dp, n0, rows, p.layout, p.vec_k);
    const size_t base = (((size_t)b * p.Hkv + h) * p.nblk + blk) * dp;
    for (int c = threadIdx.x; c < dp; c += blockDim.x) {
      float acc = 0.f;
      for (int r = 0; r < rows; ++r) acc = __fadd_rn(acc, to_f32(tile[r * dp + c]));
      p.ksum_part[base + c] = acc;
    }
  } else {  // ---- V: per-block partial column amax
    const int h = y - p.Hq - p.Hkv;
    load_tile<T>(tile, static_cast<const T*>(p.v), b, h, p.Hkv, p.N, d, dp, n0, rows, p.layout, p.vec_v);
    const size_t base = (((size_t)b * p.Hkv + h) * p.nblk + blk) * dp;
    for (int c = threadIdx.x; c < dp; c += blockDim.x) {
      float am = 0.f;
      for (int r = 0; r < rows; ++r) am = fmaxf(am, fabsf(to_f32(tile[r * dp + c])));
      p.vmax_part[base + c] = am;
    }
  }
}

__global__ void quant_finalize_kernel(QuantParams p) {
  const int bh = blockIdx.x;
  for (int c = threadIdx.x; c < p.dp; c += blockDim.x) {
    const float* ks = p.ksum_part + (size_t)bh * p.nblk * p.dp + c;
    const float* vm = p.vmax_part + (size_t)bh * p.nblk * p.dp + c;
    float acc = 0.f, am = 0.f;
    for (int i = 0; i < p.nblk; ++i) {
      acc = __fadd_rn(acc, ks[(size_t)i * p.dp]);
      am = fmaxf(am, vm[(size_t)i * p.dp]);
    }
    p.km[(size_t)bh * p.dp + c] = c < p.d ? __fdiv_rn(acc, (float)p.N) : 0.f;
    p.vs[(size_t)bh * p.dp + c] = __fdiv_rn(am, p.vmax_code);
    p.vinv[(size_t)bh * p.dp + c] = am > 0.f ? __fdiv_rn(p.vmax_code, am) : 0.f;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) quant_pass2_kernel(QuantParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* tile = reinterpret_cast<T*>(smem_raw);
  __shared__ float red[8];
  __shared__ float cvec[256];  // k_mean or v_inv of this head
  const int blk = blockIdx.x, y = blockIdx.y, b = blockIdx.z;
  const int n0 = blk * 128, rows = min(128, p.N - n0);
  const int dp = p.dp, d = p.d;
  if (y < p.Hkv) {  // ---- K - mean(K): INT8 codes and per-block scale
    const int h = y;
    const size_t bh = (size_t)b * p.Hkv + h;
    for (int c = threadIdx.x; c < dp; c += blockDim.x) cvec[c] = p.km[bh * dp + c];
    load_tile<T>(tile, static_cast<const T*>(p.k), b, h, p.Hkv, p.N, d, dp, n0, rows, p.layout, p.vec_k);
    auto x = [&](int r, int c) -> float {
      return (r < rows && c < d) ? __fsub_rn(to_f32(tile[r * dp + c]), cvec[c]) : 0.f;
    };
    float am = 0.f;
    for (int i = threadIdx.x; i < rows * dp; i += blockDim.x) am = fmaxf(am, fabsf(x(i / dp, i % dp)));
    am = block_max(am, red);
    const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
    write_int8_codes(p.k8 + (bh * p.Np + n0) * dp, dp, inv, x);
    if (threadIdx.x == 0) p.ks[bh * p.nblk + blk] = __fdiv_rn(am, 127.f);
  } else {  // ---- V: E4M3 codes, transposed to [channel][token]
    const int h = y - p.Hkv;
    const size_t bh = (size_t)b * p.Hkv + h;
    for (int c = threadIdx.x; c < dp; c += blockDim.x) cvec[c] = p.vinv[bh * dp + c];
    load_tile<T>(tile, static_cast<const T*>(p.v), b, h, p.Hkv, p.N, d, dp, n0, rows, p.layout, p.vec_v);
    const int nchunk = dp * 128 / 16;
    for (int o = threadIdx.x; o < nchunk; o += blockDim.x) {
      const int c = o % dp, r0 = (o / dp) * 16;
      const float inv = cvec[c];
      uint32_t w[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float a0 = __fmul_rn(to_f32(tile[(r0 + 4 * g + 0) * dp + c]), inv);
        const float a1 = __fmul_rn(to_f32(tile[(r0 + 4 * g + 1) * dp + c]), inv);
        const float a2 = __fmul_rn(to_f32(tile[(r0 + 4 * g + 2) * dp + c]), inv);
        const float a3 = __fmul_rn(to_f32(tile[(r0 + 4 * g + 3) * dp + c]), inv);
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a0, a1), __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(a2, a3), __NV_SATFINITE, __NV_E4M3);
        w[g] = (lo & 0xFFFF) | (hi << 16);
      }
      *reinterpret_cast<uint4*>(p.v8t + (bh * dp + c) * p.Np + n0 + r0) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <typename T>
static cudaError_t launch_quant_t(const QuantParams& p, cudaStream_t st) {
  const size_t smem = (size_t)128 * p.dp * sizeof(T);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(quant_pass1_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return e;
  if ((e = cudaFuncSetAttribute(quant_pass2_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return e;
  quant_pass1_kernel<T><<<dim3(p.nblk, p.Hq + 2 * p.Hkv, p.B), 256, smem, st>>>(p);
  quant_finalize_kernel<<<p.B * p.Hkv, 256, 0, st>>>(p);
  quant_pass2_kernel<T><<<dim3(p.nblk, 2 * p.Hkv, p.B), 256, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantParams& p, cudaStream_t st) {
  return p.dtype == SAGE_BF16 ? launch_quant_t<__nv_bfloat16>(p, st) : launch_quant_t<__half>(p, st);
}

}  // namespace sage
