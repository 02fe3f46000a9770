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
//             V -> E4M3 codes (FP8 P.V) or fp16 codes of v / amax (FP16 P.V), written
//             transposed (keys contiguous) for the P.V MMA.
//
// Method: INT8 quantization with smoothing for Q K^T and FP8 quantization for
// P V (SageAttention README, "Current Features").  The block size, the
// symmetric rounding, the order of the K-mean sum and the V code range are
// this library's readings of what the pages leave open; every float operation
// below is an explicit IEEE round-to-nearest operation (__fadd_rn, __fmul_rn,
// __fdiv_rn) so the results are reproducible bit for bit.
//
// Thread layout: a CTA of dp threads covers one 128-token block; thread t owns
// the register tile "group g = t / (dp/8) (tokens 16g .. 16g+15) x channel
// vector cv = t % (dp/8) (channels 8cv .. 8cv+7)", loaded as sixteen 16-byte
// vectors.  The K token sum of a block is the pairwise tree over its 8 group
// sums, each group summed token by token.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sage_internal.h"

namespace sage {

// Error word of the quantize kernels (store checks of the checked build), read and cleared by
// sage_check_status() together with the attention kernels' word.
__device__ int g_quant_error = 0;

cudaError_t read_clear_quant_error(int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_quant_error, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_quant_error, &zero, sizeof(int));
}

// Programmatic dependent launch: the finalize and pass-2 grids are launched while their
// predecessor still runs; they wait here for it to complete (and its writes to be visible)
// before reading what it wrote.
__device__ __forceinline__ void wait_for_previous_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_next_grid() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Element e (0..7) of a 16-byte vector of 16-bit values, widened exactly to float.
template <typename T>
__device__ __forceinline__ float elem(const uint4& v, int e) {
  const uint32_t w = (&v.x)[e >> 1];
  const unsigned short h = (e & 1) ? (unsigned short)(w >> 16) : (unsigned short)(w & 0xFFFF);
  T t;
  *reinterpret_cast<unsigned short*>(&t) = h;
  return to_f32(t);
}

// Packed pairs of 16-bit floats.
template <typename T>
struct Pair2;
template <>
struct Pair2<__half> {
  using type = __half2;
};
template <>
struct Pair2<__nv_bfloat16> {
  using type = __nv_bfloat162;
};

// Running max of |x| over packed 16-bit floats, on their bit patterns: with the sign bit
// cleared, the bit-pattern order of finite 16-bit floats is their magnitude order.
__device__ __forceinline__ uint32_t absmax_bits(uint32_t acc, uint32_t w) { return __vmaxu2(acc, w & 0x7FFF7FFFu); }

template <typename T>
__device__ __forceinline__ float bits_to_f32(uint32_t h16) {
  T t;
  *reinterpret_cast<unsigned short*>(&t) = (unsigned short)h16;
  return to_f32(t);
}

// max |x| of this thread's register tile (padding reads as zero and cannot raise it)
template <typename T>
__device__ __forceinline__ float tile_absmax(const uint4 (&v)[16]) {
  uint32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    a0 = absmax_bits(a0, v[r].x);
    a1 = absmax_bits(a1, v[r].y);
    a2 = absmax_bits(a2, v[r].z);
    a3 = absmax_bits(a3, v[r].w);
  }
  const uint32_t a = __vmaxu2(__vmaxu2(a0, a1), __vmaxu2(a2, a3));
  return bits_to_f32<T>(max(a & 0xFFFFu, a >> 16));
}

struct TileCoord {
  int g, cv, c0;  // token group, channel vector, first channel
};

__device__ __forceinline__ TileCoord tile_coord_at(int dp, int tid) {
  const int nv = dp / 8;
  return TileCoord{tid / nv, tid % nv, (tid % nv) * 8};
}
__device__ __forceinline__ TileCoord tile_coord(int dp) { return tile_coord_at(dp, (int)threadIdx.x); }

// Load this thread's 16 x 8 register tile of one head: tokens 16g+r (r < 16) of the block that
// starts at x0 (tokens tok_stride elements apart), channels c0..c0+7.  Tokens >= rows and
// channels >= d read as zero.
template <typename T>
__device__ __forceinline__ void load_tile(uint4 (&v)[16], const T* __restrict__ x0, long long tok_stride, int d,
                                          int rows, bool vec, const TileCoord& tc) {
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int n = tc.g * 16 + r;
    v[r] = make_uint4(0, 0, 0, 0);
    if (n < rows && tc.c0 < d) {
      const T* src = x0 + (size_t)n * tok_stride + tc.c0;
      if (vec) {
        v[r] = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        unsigned short e[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) e[k] = (tc.c0 + k < d) ? *reinterpret_cast<const unsigned short*>(src + k) : 0;
        v[r] = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16), e[6] | (e[7] << 16));
      }
    }
  }
}

// Prefetch of the next block's tile (vector path only): the same 16 x 16-byte loads as load_tile,
// issued as asynchronous copies into this thread's slots of `stage` (slot r of thread t at
// stage[r * blockDim.x + t]); tokens past `rows` and channels past d are zero-filled.
__device__ __forceinline__ void prefetch_tile(uint4* stage, const void* x0, long long tok_stride_bytes, int d,
                                              int rows, const TileCoord& tc) {
  const unsigned char* base = static_cast<const unsigned char*>(x0);
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int n = tc.g * 16 + r;
    const bool valid = n < rows && tc.c0 < d;
    const unsigned char* src = valid ? base + (size_t)n * tok_stride_bytes + tc.c0 * 2 : base;
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(stage + r * blockDim.x + threadIdx.x));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void take_prefetched(uint4 (&v)[16], const uint4* stage) {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
  for (int r = 0; r < 16; ++r) v[r] = stage[r * blockDim.x + threadIdx.x];
}

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < nw; ++i) r = fmaxf(r, red[i]);
  return r;
}

// INT8 codes of this thread's tile, x(r, k) given by `val` and row r's 127 / amax by `inv_of`;
// rows at or beyond `rows` (tokens past N) get code 0 whatever `val` returns for them.
template <typename F, typename G>
__device__ __forceinline__ void store_int8_tile_rows(int8_t* __restrict__ dst, int dp, const TileCoord& tc, G inv_of,
                                                     int rows, F val, const Extent& x) {
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const bool valid = tc.g * 16 + r < rows;
    const float inv = inv_of(r);
    uint32_t w[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int code = __float2int_rn(__fmul_rn(val(r, half * 4 + e), inv));  // rint: ties to even
        code = max(-127, min(127, code));
        packed |= (uint32_t)(code & 0xFF) << (8 * e);
      }
      w[half] = valid ? packed : 0u;
    }
    int8_t* const q = dst + (size_t)(tc.g * 16 + r) * dp + tc.c0;
    if (SAGE_STORE_OK(x, q, 8, &g_quant_error)) *reinterpret_cast<uint2*>(q) = make_uint2(w[0], w[1]);
  }
}

// The same with one 127 / amax for the whole tile.
template <typename F>
__device__ __forceinline__ void store_int8_tile(int8_t* __restrict__ dst, int dp, const TileCoord& tc, float inv, int rows,
                                                F val, const Extent& x) {
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const bool valid = tc.g * 16 + r < rows;
    uint32_t w[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int code = __float2int_rn(__fmul_rn(val(r, half * 4 + e), inv));  // rint: ties to even
        code = max(-127, min(127, code));
        packed |= (uint32_t)(code & 0xFF) << (8 * e);
      }
      w[half] = valid ? packed : 0u;
    }
    int8_t* const q = dst + (size_t)(tc.g * 16 + r) * dp + tc.c0;
    if (SAGE_STORE_OK(x, q, 8, &g_quant_error)) *reinterpret_cast<uint2*>(q) = make_uint2(w[0], w[1]);
  }
}

// Column reduction over the 8 groups of a block: part[g][c] in shared memory -> channel c = threadIdx.x.
__device__ __forceinline__ float tree8_sum(const float* part, int dp, int c) {
  const float* p = part + c;
  return __fadd_rn(__fadd_rn(__fadd_rn(p[0], p[dp]), __fadd_rn(p[2 * dp], p[3 * dp])),
                   __fadd_rn(__fadd_rn(p[4 * dp], p[5 * dp]), __fadd_rn(p[6 * dp], p[7 * dp])));
}
__device__ __forceinline__ float tree8_max(const float* part, int dp, int c) {
  const float* p = part + c;
  float m = p[0];
#pragma unroll
  for (int g = 1; g < 8; ++g) m = fmaxf(m, p[g * dp]);
  return m;
}
__device__ __forceinline__ float tree8_min(const float* part, int dp, int c) {
  const float* p = part + c;
  float m = p[0];
#pragma unroll
  for (int g = 1; g < 8; ++g) m = fminf(m, p[g * dp]);
  return m;
}

// FINE_Q: Q scales per token or per 32 tokens (else per 128-token block); SMOOTH_V: V's token
// mean is subtracted before coding (pass 1 then gathers V's column sums, max and min).  Separate
// instances keep the default path's register count (and occupancy) as low as before.
// Each CTA handles up to p.bpc consecutive 128-token blocks of one head; with p.prefetch the next
// block's tile streams into shared memory (cp.async) while the current one is processed.
template <typename T, bool FINE_Q, bool SMOOTH_V>
__global__ void __launch_bounds__(256, 2) quant_pass1_kernel(QuantParams p) {
  allow_next_grid();
  extern __shared__ uint4 stage[];  // p.prefetch: 16 slots per thread
  __shared__ float red[8];
  __shared__ float part[8 * 256];
  const int y = blockIdx.y, b = blockIdx.z;
  const SeqView sv = seq_view(p.m, b);
  const int dp = p.m.dp, d = p.m.d;
  const TileCoord tc = tile_coord(dp);
  // this CTA's head: its tokens in the caller's tensor
  const T* src;
  long long tstride;
  int ntok;
  bool vec;
  if (y < p.m.Hq) {
    src = static_cast<const T*>(p.q) + sv.q_in + y * sv.q_head, tstride = sv.q_tok, ntok = sv.nq, vec = p.vec_q;
  } else if (y < p.m.Hq + p.m.Hkv) {
    src = static_cast<const T*>(p.k) + sv.k_in + (y - p.m.Hq) * sv.k_head, tstride = sv.k_tok, ntok = sv.nk;
    vec = p.vec_k;
  } else {
    src = static_cast<const T*>(p.v) + sv.k_in + (y - p.m.Hq - p.m.Hkv) * sv.k_head, tstride = sv.k_tok;
    ntok = sv.nk, vec = p.vec_v;
  }
  const int blk0 = blockIdx.x * p.bpc, blk1 = min((ntok + 127) / 128, blk0 + p.bpc);
  if (blk0 >= blk1) return;  // past the end of this sequence (the whole CTA leaves)
  uint4 v[16];
  load_tile<T>(v, src + (long long)blk0 * 128 * tstride, tstride, d, min(128, ntok - blk0 * 128), vec, tc);
  for (int blk = blk0; blk < blk1; ++blk) {
  const int n0 = blk * 128, rows = min(128, ntok - n0);
  const bool pref = p.prefetch && vec && blk + 1 < blk1;
  if (pref) prefetch_tile(stage, src + (long long)(n0 + 128) * tstride, tstride * 2, d, min(128, ntok - n0 - 128), tc);
  if (y < p.m.Hq) {  // ---- Q: final INT8 codes and per-block scale
    const int h = y;
    const long long row = sv.q_row0 + h * p.m.q_head_rows + n0;
    if (!FINE_Q) {  // one scale for the 128-token block
      const float am = block_max(tile_absmax<T>(v), red);
      const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
      store_int8_tile(p.q8 + row * dp, dp, tc, inv, rows, [&](int r, int e) { return elem<T>(v[r], e); }, p.x_q8);
      if (threadIdx.x == 0 && SAGE_STORE_OK(p.x_qs, p.qs + row / 128, 4, &g_quant_error))
        p.qs[row / 128] = __fdiv_rn(am, 127.f);
    } else {  // one scale per token (q_gran 1) or per 32 tokens (q_gran 32)
      // max |q| of each of this thread's 16 tokens over its 8 channels, then over the dp/8
      // consecutive threads that hold the token's other channels
      float ta[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const uint32_t a = __vmaxu2(__vmaxu2(v[r].x & 0x7FFF7FFFu, v[r].y & 0x7FFF7FFFu),
                                    __vmaxu2(v[r].z & 0x7FFF7FFFu, v[r].w & 0x7FFF7FFFu));
        ta[r] = bits_to_f32<T>(max(a & 0xFFFFu, a >> 16));
      }
      for (int o = 1; o < dp / 8; o <<= 1)
#pragma unroll
        for (int r = 0; r < 16; ++r) ta[r] = fmaxf(ta[r], __shfl_xor_sync(0xffffffffu, ta[r], o));
      if (p.q_gran_log2 == 5) {  // tokens 32k..32k+31 = token groups 2k and 2k+1
        float gm = ta[0];
#pragma unroll
        for (int r = 1; r < 16; ++r) gm = fmaxf(gm, ta[r]);
        if (tc.cv == 0) red[tc.g] = gm;
        __syncthreads();
        gm = fmaxf(red[tc.g & ~1], red[tc.g | 1]);
#pragma unroll
        for (int r = 0; r < 16; ++r) ta[r] = gm;
        if (tc.cv == 0 && (tc.g & 1) == 0 && SAGE_STORE_OK(p.x_qs, p.qs + (row + tc.g * 16) / 32, 4, &g_quant_error))
          p.qs[(row + tc.g * 16) / 32] = __fdiv_rn(gm, 127.f);
      } else if (tc.cv == 0) {
#pragma unroll
        for (int r = 0; r < 16; ++r)
          if (SAGE_STORE_OK(p.x_qs, p.qs + row + tc.g * 16 + r, 4, &g_quant_error))
            p.qs[row + tc.g * 16 + r] = __fdiv_rn(ta[r], 127.f);
      }
      store_int8_tile_rows(p.q8 + row * dp, dp, tc, [&](int r) { return ta[r] > 0.f ? __fdiv_rn(127.f, ta[r]) : 0.f; },
                           rows, [&](int r, int e) { return elem<T>(v[r], e); }, p.x_q8);
    }
  } else if (y < p.m.Hq + p.m.Hkv) {  // ---- K: per-block partial column sums
    const int h = y - p.m.Hq;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (tc.g * 16 + r < rows)  // tokens beyond N are skipped, not added as zeros
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], elem<T>(v[r], e));
#pragma unroll
    for (int e = 0; e < 8; ++e) part[tc.g * dp + tc.c0 + e] = acc[e];
    __syncthreads();
    const long long base = (sv.k_row0 + h * p.m.k_head_rows + n0) / 128 * dp;
    if (SAGE_STORE_OK(p.x_ksum, p.ksum_part + base + threadIdx.x, 4, &g_quant_error))
      p.ksum_part[base + threadIdx.x] = tree8_sum(part, dp, threadIdx.x);
  } else if (SMOOTH_V) {  // ---- V, smoothed: per-block partial column sums, max and min
    const int h = y - p.m.Hq - p.m.Hkv;
    float acc[8], hi[8], lo[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f, hi[e] = -INFINITY, lo[e] = INFINITY;
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (tc.g * 16 + r < rows)  // tokens beyond N are skipped
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float x = elem<T>(v[r], e);
          acc[e] = __fadd_rn(acc[e], x);
          hi[e] = fmaxf(hi[e], x);
          lo[e] = fminf(lo[e], x);
        }
    const long long base = (sv.k_row0 + h * p.m.k_head_rows + n0) / 128 * dp;
#pragma unroll
    for (int e = 0; e < 8; ++e) part[tc.g * dp + tc.c0 + e] = acc[e];
    __syncthreads();
    if (SAGE_STORE_OK(p.x_vsum, p.vsum_part + base + threadIdx.x, 4, &g_quant_error))
      p.vsum_part[base + threadIdx.x] = tree8_sum(part, dp, threadIdx.x);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) part[tc.g * dp + tc.c0 + e] = hi[e];
    __syncthreads();
    if (SAGE_STORE_OK(p.x_vmax, p.vmax_part + base + threadIdx.x, 4, &g_quant_error))
      p.vmax_part[base + threadIdx.x] = tree8_max(part, dp, threadIdx.x);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) part[tc.g * dp + tc.c0 + e] = lo[e];
    __syncthreads();
    if (SAGE_STORE_OK(p.x_vmin, p.vmin_part + base + threadIdx.x, 4, &g_quant_error))
      p.vmin_part[base + threadIdx.x] = tree8_min(part, dp, threadIdx.x);
  } else {  // ---- V: per-block partial column amax
    const int h = y - p.m.Hq - p.m.Hkv;
    uint32_t a[4] = {0, 0, 0, 0};  // channels (2e, 2e+1), |x| as bit patterns
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      a[0] = absmax_bits(a[0], v[r].x);
      a[1] = absmax_bits(a[1], v[r].y);
      a[2] = absmax_bits(a[2], v[r].z);
      a[3] = absmax_bits(a[3], v[r].w);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      part[tc.g * dp + tc.c0 + 2 * e] = bits_to_f32<T>(a[e] & 0xFFFFu);
      part[tc.g * dp + tc.c0 + 2 * e + 1] = bits_to_f32<T>(a[e] >> 16);
    }
    __syncthreads();
    const long long base = (sv.k_row0 + h * p.m.k_head_rows + n0) / 128 * dp;
    if (SAGE_STORE_OK(p.x_vmax, p.vmax_part + base + threadIdx.x, 4, &g_quant_error))
      p.vmax_part[base + threadIdx.x] = tree8_max(part, dp, threadIdx.x);
  }
  __syncthreads();  // `part` and `red` are reused by the next block
  if (blk + 1 < blk1) {
    if (pref)
      take_prefetched(v, stage);
    else
      load_tile<T>(v, src + (long long)(n0 + 128) * tstride, tstride, d, min(128, ntok - n0 - 128), vec, tc);
  }
  }
}

// K mean of channel c of one (batch, kv head) from pass 1's per-block partial sums: added one by one
// in block order from +0.0, then one division by the token count (the bit-exact contract's order).
__device__ __forceinline__ float k_mean_of(const QuantParams& p, long long base, int nblk, int nk, int c) {
  const float* ks = p.ksum_part + base + c;
  float acc = 0.f;
#pragma unroll 8
  for (int i = 0; i < nblk; ++i) acc = __fadd_rn(acc, ks[(size_t)i * p.m.dp]);  // the loads overlap
  return (c < p.m.d && nk > 0) ? __fdiv_rn(acc, (float)nk) : 0.f;
}

// V's channel amax (of v, or with smoothing of v - mean: its max |.| is reached at the channel's
// largest or smallest v, since rounding v - mean to float32 is monotonic in v) and token mean.
__device__ __forceinline__ float v_amax_of(const QuantParams& p, long long base, int nblk, int nk, int c, float* mean) {
  const float* vmx = p.vmax_part + base + c;
  if (p.smooth_v) {
    const float* vsum = p.vsum_part + base + c;
    const float* vmin = p.vmin_part + base + c;
    float vacc = 0.f, hi = -INFINITY, lo = INFINITY;
#pragma unroll 8
    for (int i = 0; i < nblk; ++i) {  // sums stay in block order
      vacc = __fadd_rn(vacc, vsum[(size_t)i * p.m.dp]);
      hi = fmaxf(hi, vmx[(size_t)i * p.m.dp]);
      lo = fminf(lo, vmin[(size_t)i * p.m.dp]);
    }
    const float m = (c < p.m.d && nk > 0) ? __fdiv_rn(vacc, (float)nk) : 0.f;
    *mean = m;
    return nk > 0 ? fmaxf(fabsf(__fsub_rn(hi, m)), fabsf(__fsub_rn(lo, m))) : 0.f;
  }
  float am = 0.f;
#pragma unroll 8
  for (int i = 0; i < nblk; ++i) am = fmaxf(am, vmx[(size_t)i * p.m.dp]);
  *mean = 0.f;
  return am;
}

// One CTA per (batch, kv head, 32 channels).  The partials of a chunk of kFinChunk blocks are
// staged in shared memory by all eight warps at once (one 128-byte row per block and array, many
// loads in flight), then warp 0 adds K's sums and warp 1 folds V's statistics, one lane per
// channel, in block order: the same operations in the same order as k_mean_of / v_amax_of, so
// the same bits, without a dependent global load per block.
constexpr int kFinChunk = 64;

__global__ void __launch_bounds__(256) quant_finalize_kernel(QuantParams p) {
  __shared__ float stage[4][kFinChunk][32];  // ksum, vmax, vsum, vmin
  allow_next_grid();
  wait_for_previous_grid();  // pass 1's partial sums
  const int bh = blockIdx.x, b = bh / p.m.Hkv, h = bh - b * p.m.Hkv;
  const SeqView sv = seq_view(p.m, b);
  const int dp = p.m.dp, nblk = (sv.nk + 127) / 128;
  const long long base = (sv.k_row0 + h * p.m.k_head_rows) / 128 * dp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, c = blockIdx.y * 32 + lane;
  const int narr = p.smooth_v ? 4 : 2;
  const float* src[4] = {p.ksum_part, p.vmax_part, p.vsum_part, p.vmin_part};
  float kacc = 0.f, vacc = 0.f, hi = -INFINITY, lo = INFINITY, am = 0.f;
  for (int b0 = 0; b0 < nblk; b0 += kFinChunk) {
    const int nb = min(kFinChunk, nblk - b0);
    // every load of the chunk in flight before the first store (block warp + 8 k of each array)
    float tmp[4][kFinChunk / 8];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int k = 0; k < kFinChunk / 8; ++k) {
        const int i = warp + 8 * k;
        tmp[a][k] = (a < narr && i < nb) ? src[a][base + (long long)(b0 + i) * dp + c] : 0.f;
      }
    __syncthreads();  // the previous chunk has been consumed
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int k = 0; k < kFinChunk / 8; ++k) stage[a][warp + 8 * k][lane] = tmp[a][k];
    __syncthreads();
    if (warp == 0) {
      for (int i = 0; i < nb; ++i) kacc = __fadd_rn(kacc, stage[0][i][lane]);
    } else if (warp == 1) {
      if (p.smooth_v) {
        for (int i = 0; i < nb; ++i) {
          vacc = __fadd_rn(vacc, stage[2][i][lane]);
          hi = fmaxf(hi, stage[1][i][lane]);
          lo = fminf(lo, stage[3][i][lane]);
        }
      } else {
        for (int i = 0; i < nb; ++i) am = fmaxf(am, stage[1][i][lane]);
      }
    }
  }
  const size_t o = (size_t)bh * dp + c;
  if (warp == 0) {
    const float km = (c < p.m.d && sv.nk > 0) ? __fdiv_rn(kacc, (float)sv.nk) : 0.f;
    if (SAGE_STORE_OK(p.x_km, p.km + o, 4, &g_quant_error)) p.km[o] = km;
  } else if (warp == 1) {
    float mean = 0.f;
    if (p.smooth_v) {
      mean = (c < p.m.d && sv.nk > 0) ? __fdiv_rn(vacc, (float)sv.nk) : 0.f;
      am = sv.nk > 0 ? fmaxf(fabsf(__fsub_rn(hi, mean)), fabsf(__fsub_rn(lo, mean))) : 0.f;
    }
    if (p.vm && SAGE_STORE_OK(p.x_vm, p.vm + o, 4, &g_quant_error)) p.vm[o] = mean;
    if (SAGE_STORE_OK(p.x_vs, p.vs + o, 4, &g_quant_error)) p.vs[o] = __fdiv_rn(am, p.vmax_code);
    if (SAGE_STORE_OK(p.x_vinv, p.vinv + o, 4, &g_quant_error)) p.vinv[o] = am > 0.f ? __fdiv_rn(p.vmax_code, am) : 0.f;
  }
}

// Two E4M3 codes (RN, saturating) of a and b, a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3) & 0xFFFFu;
}

// K - mean(K) of one 128-token block in registers: INT8 codes with the block's scale (rows past
// the sequence masked), written at q8-layout row `row`.  max_all reduces a float over every
// thread that holds part of the block; `leader` writes the scale.
template <typename T, typename MaxAll>
__device__ __forceinline__ void code_k_block(const QuantParams& p, const uint4 (&v)[16], const TileCoord& tc, int rows,
                                             const float (&km)[8], long long row, MaxAll max_all, bool leader) {
  const int dp = p.m.dp, d = p.m.d;
  // padded channels read 0 and have mean 0; padded rows are masked by store_int8_tile
  auto x = [&](int r, int e) -> float { return __fsub_rn(elem<T>(v[r], e), km[e]); };
  // max |k - mean| per channel is reached at the channel's largest or smallest k, since
  // rounding k - mean to float32 is monotonic in k: take per-channel extremes on the packed
  // values, then subtract the mean from those two only.
  using P2 = typename Pair2<T>::type;
  P2 hi[4], lo[4];
  bool any = false;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    if (tc.g * 16 + r < rows) {
      const P2* w = reinterpret_cast<const P2*>(&v[r]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hi[e] = any ? __hmax2(hi[e], w[e]) : w[e];
        lo[e] = any ? __hmin2(lo[e], w[e]) : w[e];
      }
      any = true;
    }
  }
  float am = 0.f;
  if (any) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t hb = *reinterpret_cast<const uint32_t*>(&hi[e]);
      const uint32_t lb = *reinterpret_cast<const uint32_t*>(&lo[e]);
      if (tc.c0 + 2 * e < d)
        am = fmaxf(am, fmaxf(fabsf(__fsub_rn(bits_to_f32<T>(hb & 0xFFFFu), km[2 * e])),
                             fabsf(__fsub_rn(bits_to_f32<T>(lb & 0xFFFFu), km[2 * e]))));
      if (tc.c0 + 2 * e + 1 < d)
        am = fmaxf(am, fmaxf(fabsf(__fsub_rn(bits_to_f32<T>(hb >> 16), km[2 * e + 1])),
                             fabsf(__fsub_rn(bits_to_f32<T>(lb >> 16), km[2 * e + 1]))));
    }
  }
  am = max_all(am);
  const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
  store_int8_tile(p.k8 + row * dp, dp, tc, inv, rows, x, p.x_k8);
  if (leader && SAGE_STORE_OK(p.x_ks, p.ks + row / 128, 4, &g_quant_error)) p.ks[row / 128] = __fdiv_rn(am, 127.f);
}

// V of one block in registers: E4M3 or fp16 codes of (v - mean) * inv, transposed to V^T (this
// thread's channels start at V^T row vrow, its 16 tokens at column vcol).
template <typename T, bool SMOOTH_V>
__device__ __forceinline__ void code_v_block(const QuantParams& p, const uint4 (&v)[16], const TileCoord& tc, int rows,
                                             const float (&inv)[8], const float (&mean)[8], long long vrow,
                                             long long vcol) {
  // (v - mean) * inv; tokens past N give 0 (with smoothing the subtraction would not)
  auto vx = [&](int r, int e) -> float {
    if (!SMOOTH_V) return __fmul_rn(elem<T>(v[r], e), inv[e]);  // tokens past N load as 0 -> code 0
    const float x = __fsub_rn(elem<T>(v[r], e), mean[e]);
    return (tc.g * 16 + r < rows) ? __fmul_rn(x, inv[e]) : 0.f;
  };
  const long long pitch = p.m.k_head_rows;
  if (p.v_fp16) {
    // fp16_rne(v * inv): 16 tokens of one channel = 32 bytes (padded tokens and channels read 0)
    uint16_t* vt = reinterpret_cast<uint16_t*>(p.v8t);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      uint32_t w[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const __half2 h2 = __floats2half2_rn(vx(2 * q, e), vx(2 * q + 1, e));
        w[q] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      uint4* dst = reinterpret_cast<uint4*>(vt + (vrow + e) * pitch + vcol);
      if (SAGE_STORE_OK(p.x_v8t, dst, 32, &g_quant_error)) {
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a0 = vx(4 * q + 0, e);
        const float a1 = vx(4 * q + 1, e);
        const float a2 = vx(4 * q + 2, e);
        const float a3 = vx(4 * q + 3, e);
        w[q] = e4m3x2(a0, a1) | (e4m3x2(a2, a3) << 16);
      }
      uint8_t* const dst = p.v8t + (vrow + e) * pitch + vcol;
      if (SAGE_STORE_OK(p.x_v8t, dst, 16, &g_quant_error)) *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <typename T, bool SMOOTH_V>
__global__ void __launch_bounds__(256, 2) quant_pass2_kernel(QuantParams p) {
  extern __shared__ uint4 stage[];  // p.prefetch: 16 slots per thread
  __shared__ float red[8];
  allow_next_grid();
  // Last-read-first: pass 1 read V after K and batch B-1 last, so those are the tiles most likely
  // still in L2 when this pass reads them again.
  const int y = gridDim.y - 1 - blockIdx.y, b = gridDim.z - 1 - blockIdx.z;
  const SeqView sv = seq_view(p.m, b);
  const int dp = p.m.dp, d = p.m.d;
  const TileCoord tc = tile_coord(dp);
  const bool isk = y < p.m.Hkv;
  const T* src = static_cast<const T*>(isk ? p.k : p.v) + sv.k_in + (isk ? y : y - p.m.Hkv) * sv.k_head;
  const long long tstride = sv.k_tok;
  const bool vec = isk ? p.vec_k : p.vec_v;
  const int blk0 = (gridDim.x - 1 - blockIdx.x) * p.bpc, blk1 = min((sv.nk + 127) / 128, blk0 + p.bpc);
  if (blk0 >= blk1) return;  // past the end of this sequence (the whole CTA leaves)
  wait_for_previous_grid();  // pass 1's partials (p.fold), or the finalize kernel's K mean and V scales
  // Short sequences (p.fold): no finalize launch; every CTA computes its head's K mean, or V's
  // scales and mean, from pass 1's partials in the same order, and the head's first CTA writes
  // them out.  Otherwise the finalize kernel has written them.
  __shared__ float hv[2][256];  // K: mean; V: 1 / scale, mean
  const int hh = isk ? y : y - p.m.Hkv;
  const size_t bhh = (size_t)b * p.m.Hkv + hh;
  if (p.fold) {
    const int c = threadIdx.x, nblk = (sv.nk + 127) / 128;
    const long long base = (sv.k_row0 + hh * p.m.k_head_rows) / 128 * dp;
    if (isk) {
      const float km = k_mean_of(p, base, nblk, sv.nk, c);
      hv[0][c] = km;
      if (blk0 == 0 && SAGE_STORE_OK(p.x_km, p.km + bhh * dp + c, 4, &g_quant_error)) p.km[bhh * dp + c] = km;
    } else {
      float mean;
      const float am = v_amax_of(p, base, nblk, sv.nk, c, &mean);
      hv[0][c] = am > 0.f ? __fdiv_rn(p.vmax_code, am) : 0.f;
      hv[1][c] = mean;
      if (blk0 == 0) {
        if (SAGE_STORE_OK(p.x_vs, p.vs + bhh * dp + c, 4, &g_quant_error)) p.vs[bhh * dp + c] = __fdiv_rn(am, p.vmax_code);
        if (p.vm && SAGE_STORE_OK(p.x_vm, p.vm + bhh * dp + c, 4, &g_quant_error)) p.vm[bhh * dp + c] = mean;
      }
    }
    __syncthreads();
  }
  uint4 v[16];
  load_tile<T>(v, src + (long long)blk0 * 128 * tstride, tstride, d, min(128, sv.nk - blk0 * 128), vec, tc);
  for (int blk = blk0; blk < blk1; ++blk) {
  const int n0 = blk * 128, rows = min(128, sv.nk - n0);
  const bool pref = p.prefetch && vec && blk + 1 < blk1;
  if (pref) prefetch_tile(stage, src + (long long)(n0 + 128) * tstride, tstride * 2, d, min(128, sv.nk - n0 - 128), tc);
  if (y < p.m.Hkv) {  // ---- K - mean(K): INT8 codes and per-block scale
    const int h = y;
    const size_t bh = (size_t)b * p.m.Hkv + h;
    float km[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) km[e] = p.fold ? hv[0][tc.c0 + e] : p.km[bh * dp + tc.c0 + e];
    const long long row = sv.k_row0 + h * p.m.k_head_rows + n0;
    code_k_block<T>(p, v, tc, rows, km, row, [&](float a) { return block_max(a, red); }, threadIdx.x == 0);
  } else {  // ---- V: E4M3 or fp16 codes, transposed to [channel][token]
    const int h = y - p.m.Hkv;
    const size_t bh = (size_t)b * p.m.Hkv + h;
    float inv[8], mean[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) inv[e] = p.fold ? hv[0][tc.c0 + e] : p.vinv[bh * dp + tc.c0 + e];
#pragma unroll
    for (int e = 0; e < 8; ++e) mean[e] = SMOOTH_V ? (p.fold ? hv[1][tc.c0 + e] : p.vm[bh * dp + tc.c0 + e]) : 0.f;
    const long long vrow = sv.v_row0 + (long long)h * dp + tc.c0, vcol = sv.v_col0 + n0 + tc.g * 16;
    code_v_block<T, SMOOTH_V>(p, v, tc, rows, inv, mean, vrow, vcol);
  }
  __syncthreads();  // `red` is reused by the next block
  if (blk + 1 < blk1) {
    if (pref)
      take_prefetched(v, stage);
    else
      load_tile<T>(v, src + (long long)(n0 + 128) * tstride, tstride, d, min(128, sv.nk - n0 - 128), vec, tc);
  }
  }
}

// ------------------------------------------------------------------------------------------------
// Single-launch quantize pass for short dense sequences (at most 32 blocks of 128 tokens, dp <= 128,
// per-block Q scales, V not smoothed).  A cluster of ceil(nblk / 4) CTAs covers one head; each CTA
// holds four blocks, one per group of dp threads, in registers.  K and V CTAs exchange their
// per-block statistics through distributed shared memory, so K and V are read once and no
// finalize or second pass is launched; every operation, and its order, is that of the two-pass
// path, so codes, scales and means are the same bits.
// ------------------------------------------------------------------------------------------------
constexpr int kClusterMaxBlocks = 32;
constexpr int kClusterGroupsUsed = 4;  // blocks per CTA: clusters of ceil(nblk / 4) <= 8 CTAs

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// `local` in the shared memory of the cluster's CTA `rank`
__device__ __forceinline__ float ld_cluster(const float* local, int rank) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local));
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}
// max of v over the nthreads threads of group gi (named barrier 1 + gi), as block_max over a CTA
__device__ __forceinline__ float group_max(float v, float* red, int gi, int tid, int nthreads) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((tid & 31) == 0) red[tid >> 5] = v;
  named_bar_sync(1 + gi, nthreads);
  float r = 0.f;
  for (int i = 0; i < (nthreads >> 5); ++i) r = fmaxf(r, red[i]);
  return r;
}

template <typename T, int G>  // G: blocks (thread groups of dp threads) per CTA
__global__ void __launch_bounds__(512, 1) quant_cluster_kernel(QuantParams p) {
  __shared__ float red[G][8];
  __shared__ float part[G][8 * 128];
  __shared__ float bstat[G][128];  // this CTA's per-block statistic (K: column sums, V: column amax)
  __shared__ float hv[128];        // the head's K mean or V 1 / scale
  allow_next_grid();
  const int dp = p.m.dp, d = p.m.d;
  const int gi = threadIdx.x / dp, tid = threadIdx.x - gi * dp;
  const TileCoord tc = tile_coord_at(dp, tid);
  const int rank = blockIdx.x;  // the cluster spans x: the CTA's rank in it
  const int y = blockIdx.y, b = blockIdx.z;
  const SeqView sv = seq_view<0>(p.m, b);
  const T* src;
  long long tstride;
  int ntok;
  bool vec;
  if (y < p.m.Hq) {
    src = static_cast<const T*>(p.q) + sv.q_in + y * sv.q_head, tstride = sv.q_tok, ntok = sv.nq, vec = p.vec_q;
  } else if (y < p.m.Hq + p.m.Hkv) {
    src = static_cast<const T*>(p.k) + sv.k_in + (y - p.m.Hq) * sv.k_head, tstride = sv.k_tok, ntok = sv.nk;
    vec = p.vec_k;
  } else {
    src = static_cast<const T*>(p.v) + sv.k_in + (y - p.m.Hq - p.m.Hkv) * sv.k_head, tstride = sv.k_tok;
    ntok = sv.nk, vec = p.vec_v;
  }
  const int nblk = (ntok + 127) / 128, blk = rank * G + gi;
  const bool has = blk < nblk;
  const int n0 = blk * 128, rows = has ? min(128, ntok - n0) : 0;
  uint4 v[16];
  if (has) load_tile<T>(v, src + (long long)n0 * tstride, tstride, d, rows, vec, tc);
  auto gmax = [&](float a) { return group_max(a, red[gi], gi, tid, dp); };
  if (y < p.m.Hq) {  // ---- Q: codes and per-block scale (a Q cluster takes no cluster barrier)
    if (has) {
      const long long row = sv.q_row0 + y * p.m.q_head_rows + n0;
      const float am = gmax(tile_absmax<T>(v));
      const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
      store_int8_tile(p.q8 + row * dp, dp, tc, inv, rows, [&](int r, int e) { return elem<T>(v[r], e); }, p.x_q8);
      if (tid == 0 && SAGE_STORE_OK(p.x_qs, p.qs + row / 128, 4, &g_quant_error)) p.qs[row / 128] = __fdiv_rn(am, 127.f);
    }
    return;
  }
  const bool isk = y < p.m.Hq + p.m.Hkv;
  const int h = isk ? y - p.m.Hq : y - p.m.Hq - p.m.Hkv;
  const size_t bh = (size_t)b * p.m.Hkv + h;
  if (has) {  // the block's statistic, as pass 1 computes it
    float* pg = part[gi];
    if (isk) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (tc.g * 16 + r < rows)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], elem<T>(v[r], e));
#pragma unroll
      for (int e = 0; e < 8; ++e) pg[tc.g * dp + tc.c0 + e] = acc[e];
      named_bar_sync(1 + gi, dp);
      bstat[gi][tid] = tree8_sum(pg, dp, tid);
    } else {
      uint32_t a[4] = {0, 0, 0, 0};
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        a[0] = absmax_bits(a[0], v[r].x);
        a[1] = absmax_bits(a[1], v[r].y);
        a[2] = absmax_bits(a[2], v[r].z);
        a[3] = absmax_bits(a[3], v[r].w);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        pg[tc.g * dp + tc.c0 + 2 * e] = bits_to_f32<T>(a[e] & 0xFFFFu);
        pg[tc.g * dp + tc.c0 + 2 * e + 1] = bits_to_f32<T>(a[e] >> 16);
      }
      named_bar_sync(1 + gi, dp);
      bstat[gi][tid] = tree8_max(pg, dp, tid);
    }
  }
  cluster_arrive();
  cluster_wait();  // every CTA's bstat is written and visible
  if (gi == 0) {   // the head's statistic, one thread per channel, blocks in order
    float x[kClusterMaxBlocks];
#pragma unroll
    for (int i = 0; i < kClusterMaxBlocks; ++i) x[i] = i < nblk ? ld_cluster(&bstat[i % G][tid], i / G) : 0.f;
    if (isk) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < kClusterMaxBlocks; ++i)
        if (i < nblk) acc = __fadd_rn(acc, x[i]);
      const float km = (tid < d && ntok > 0) ? __fdiv_rn(acc, (float)ntok) : 0.f;
      hv[tid] = km;
      if (rank == 0 && SAGE_STORE_OK(p.x_km, p.km + bh * dp + tid, 4, &g_quant_error)) p.km[bh * dp + tid] = km;
    } else {
      float am = 0.f;
#pragma unroll
      for (int i = 0; i < kClusterMaxBlocks; ++i)
        if (i < nblk) am = fmaxf(am, x[i]);
      hv[tid] = am > 0.f ? __fdiv_rn(p.vmax_code, am) : 0.f;
      if (rank == 0) {
        if (SAGE_STORE_OK(p.x_vs, p.vs + bh * dp + tid, 4, &g_quant_error)) p.vs[bh * dp + tid] = __fdiv_rn(am, p.vmax_code);
        if (p.vm && SAGE_STORE_OK(p.x_vm, p.vm + bh * dp + tid, 4, &g_quant_error)) p.vm[bh * dp + tid] = 0.f;
      }
    }
  }
  cluster_arrive();  // this CTA has read the others' statistics
  __syncthreads();   // hv for every group
  if (has) {
    if (isk) {
      float km[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) km[e] = hv[tc.c0 + e];
      const long long row = sv.k_row0 + h * p.m.k_head_rows + n0;
      code_k_block<T>(p, v, tc, rows, km, row, gmax, tid == 0);
    } else {
      float inv[8], mean[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) inv[e] = hv[tc.c0 + e], mean[e] = 0.f;
      const long long vrow = sv.v_row0 + (long long)h * dp + tc.c0, vcol = sv.v_col0 + n0 + tc.g * 16;
      code_v_block<T, false>(p, v, tc, rows, inv, mean, vrow, vcol);
    }
  }
  cluster_wait();  // no CTA leaves while another may still read its statistics
}

// Launch `kern` so that it may start while the previous kernel in the stream still runs (it
// waits with griddepcontrol.wait before reading that kernel's output).
template <typename K>
static cudaError_t launch_dependent(K kern, dim3 grid, dim3 block, cudaStream_t st, const QuantParams& p,
                                   size_t smem = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <typename T>
static cudaError_t launch_quant_t(const QuantParams& p_in, cudaStream_t st) {
  QuantParams p = p_in;
  const int B = p.m.B, Hq = p.m.Hq, Hkv = p.m.Hkv, dp = p.m.dp;
  const int nblk1 = p.nblk_q > p.nblk_k ? p.nblk_q : p.nblk_k;
  // Blocks per CTA: with more than about four waves of blocks (some 8 CTAs resident per SM), each
  // CTA walks a few consecutive blocks of its head, the next block's tile streaming in behind the
  // current one (measured: 328 -> 305 us on a 604 MB pass); below that, one block per CTA (walking
  // four blocks per CTA made a 113 MB pass slower, 60 -> 64 us).
  // Short dense sequences with the default options: one launch of clusters (see above).
  if (!p.m.seqs && p.q_gran_log2 == 7 && !p.smooth_v && dp <= 128 && nblk1 <= kClusterMaxBlocks) {
    constexpr int G = kClusterGroupsUsed;
    const int cs = (nblk1 + G - 1) / G;
    auto kern = quant_cluster_kernel<T, G>;
    if (cs > 8) {
      const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs, Hq + 2 * Hkv, B);
    cfg.blockDim = dim3(G * dp);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks = (long long)nblk1 * (Hq + 2 * Hkv) * B, slots = (long long)sms * 8;
  p.bpc = (int)std::min<long long>(8, std::max<long long>(1, blocks / (4 * slots)));
  p.prefetch = (dp <= 128 && p.bpc > 1) ? 1 : 0;
  const size_t smem = p.prefetch ? (size_t)dp * 16 * sizeof(uint4) : 0;  // 16 slots per thread
  const dim3 grid1((nblk1 + p.bpc - 1) / p.bpc, Hq + 2 * Hkv, B);
  const bool fine = p.q_gran_log2 != 7;
  if (fine && p.smooth_v) quant_pass1_kernel<T, true, true><<<grid1, dp, smem, st>>>(p);
  else if (fine) quant_pass1_kernel<T, true, false><<<grid1, dp, smem, st>>>(p);
  else if (p.smooth_v) quant_pass1_kernel<T, false, true><<<grid1, dp, smem, st>>>(p);
  else quant_pass1_kernel<T, false, false><<<grid1, dp, smem, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // Up to 64 blocks per sequence pass 2 folds the finalize step in (each of its CTAs reads its head's
  // partials; measured faster than a separate launch there), beyond that a finalize launch.
  p.fold = nblk1 <= 64 ? 1 : 0;
  if (!p.fold) {
    e = launch_dependent(quant_finalize_kernel, dim3(B * Hkv, dp / 32), dim3(256), st, p);
    if (e != cudaSuccess) return e;
  }
  const int nblk2 = p.nblk_k > 0 ? p.nblk_k : 1;
  const dim3 grid2((nblk2 + p.bpc - 1) / p.bpc, 2 * Hkv, B);
  return p.smooth_v ? launch_dependent(quant_pass2_kernel<T, true>, grid2, dim3(dp), st, p, smem)
                    : launch_dependent(quant_pass2_kernel<T, false>, grid2, dim3(dp), st, p, smem);
}

cudaError_t launch_quantize(const QuantParams& p, cudaStream_t st) {
  return p.dtype == SAGE_BF16 ? launch_quant_t<__nv_bfloat16>(p, st) : launch_quant_t<__half>(p, st);
}

}  // namespace sage
