// Fused INT8-QK / FP8-PV (or FP16-PV) attention for sm_100a (tcgen05 + TMA + TMEM).
//
// One CTA computes one 128-row query tile of one (batch, query head), all of its
// output columns (a 256-column O at padded head dim 256).  Six warps:
//
//   warps 0-3  softmax / correction / epilogue; thread t owns query row t
//              (TMEM lane t), so row max and row sum need no shuffles;
//   warp 4     TMA producer: Q once, then K and V^T tiles through an
//              ST-deep ring of shared-memory stages;
//   warp 5     TMEM allocator and UMMA issuer (one elected thread).
//
// Per key tile j of BN keys (the blockwise online softmax of the method):
//   S_j  = Q8 . K8_j^T                    tcgen05.mma kind::i8 -> int32 in TMEM, added to a
//                                         bias that makes each score a float (kSBiasBits)
//   s    = S_j * (qs * ks_j * sm_scale * log2 e), causal / length mask
//   m'   = max(m, rowmax s), p = 2^(s - m'), alpha = 2^(m - m'), l = l alpha + sum p
//   P    = E4M3(p * 448) (FP8 P.V, BN = 128) or fp16(p) (FP16 P.V, BN = 64), written to
//          shared memory as 128-byte rows with the 128B swizzle
//   mode 0 (fp32 accumulation):  O = O * alpha (in TMEM) ; O += P . V_j    (f32 accumulator)
//   mode 1 (fp16+fp32):          T = P . V_j (fresh f16 accumulator) ; O = O * alpha + T
//   out  = O * v_scale / (P scale * l)
// FP8 P.V runs as tcgen05.mma kind::f8f6f4 on E4M3 codes, FP16 P.V as kind::f16 on fp16
// codes (V scaled per channel to [-1, 1]).  The FP16 variant uses 64-key tiles so that its
// twice-as-large P and V tiles still let two CTAs share an SM.
//
// Method: SageAttention README ("Current Features": INT8 QK^T with smoothing,
// FP8 PV, FP16 accumulator for FP8 PV, two-level accumulation; "Available APIs":
// the INT8-QK / FP16-PV kernel) and the qwbw.cn article (pitfalls: pv_accum_dtype
// fp32 / fp16+fp32).  The kernel design (tcgen05, TMEM accumulators, TMA ring,
// warp roles) is this library's own.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <atomic>

#include "sage_internal.h"
#include "sm100.cuh"

namespace sage {
// CTAs that arrived on each SM so far (only the parity is used; see the stagger below).
__device__ unsigned int g_sm_arrivals[256];

template <int DQK, int DV, bool PV16>
struct FwdCfg {
  static constexpr int KSUB = DQK >= 128 ? 128 : 64;  // bytes per row of one Q/K sub-tile (= swizzle span)
  static constexpr int NSUB = DQK / KSUB;
  static constexpr int PB = PV16 ? 2 : 1;  // bytes per P and V element
  // Keys per KV tile.  FP8 P.V: 128 (64-key tiles, which would let three d = 64 CTAs share an
  // SM, measured no faster).  FP16 P.V: 64, so a P row and a V^T row are 128 bytes in both.
  static constexpr int BN = PV16 ? 64 : 128;
  static constexpr int ROWB = BN * PB;  // bytes of one P row / V^T row of a tile = the 128B swizzle span
  static constexpr int Q_BYTES = 128 * DQK;
  static constexpr int K_BYTES = BN * DQK;
  static constexpr int V_BYTES = DV * ROWB;
  static constexpr int P_BYTES = 128 * ROWB;
  static constexpr int ST = PV16 ? (DQK == 64 ? 4 : DQK == 128 ? 3 : 2) : (DQK == 64 ? 5 : 2);  // ring depth
  static constexpr int CTAS_PER_SM = DQK <= 128 ? 2 : 1;  // two CTAs share an SM when they fit (d <= 128)
  // K and V stages freed separately (a K stage after its Q.K^T, a V stage after its P.V), so K tiles
  // run a tile ahead of V tiles.  Measured +16% at d = 256 (one CTA per SM, two stages) and 0.5% to
  // 3% slower at d <= 128, where two CTAs share the SM and the joint ring is kept.
  static constexpr bool SPLIT_RING = DQK == 256;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = 1024 + Q_BYTES + ST * (K_BYTES + V_BYTES) + P_BYTES + BAR_BYTES;
  // TMEM: S (int32 scores, BN columns) and O (fp32, DV columns).  In fp16+fp32 mode the
  // per-tile fp16 accumulator T (DV columns) reuses S's columns (and those up to O) once the
  // scores are in registers.
  static constexpr uint32_t S_COL = 0, T_COL = 0, O_COL = BN > DV ? BN : DV;
  // P (32 columns: 128 E4M3 or 64 fp16 keys per row) in tensor memory for the fp32-accumulation
  // instances where columns are free: between S and O when they fit there, else behind O.  The
  // softmax stores P there with one tcgen05.st and the P.V MMA reads its A operand from tensor
  // memory, so P neither goes through shared memory nor needs an async-proxy fence (the
  // fp16+fp32 instances keep P in shared memory: their T shares S's columns, and they spilled).
  // FP8 P at d = 128 has no free columns (S and O fill 256).
  static constexpr bool P_TMEM = PV16 || DQK == 64 || DQK == 256;
  static constexpr uint32_t P_COL = BN + ROWB / 4 <= O_COL ? BN : O_COL + DV;
  static constexpr uint32_t COLS_USED = (P_TMEM && P_COL + ROWB / 4 > O_COL + DV) ? P_COL + ROWB / 4 : O_COL + DV;
  static constexpr uint32_t TMEM_COLS = COLS_USED <= 128 ? 128 : (COLS_USED <= 256 ? 256 : 512);
  static_assert(!P_TMEM || (P_COL + ROWB / 4 <= TMEM_COLS && (P_COL >= O_COL + DV || P_COL + ROWB / 4 <= O_COL)),
                "P in tensor memory");
  static_assert(ROWB == 128, "P and V^T rows are one 128-byte swizzle span");
  static_assert(O_COL + DV <= TMEM_COLS, "TMEM plan");
  static_assert(ST <= 8, "barrier array size");
  static_assert(SMEM <= 227 * 1024, "shared memory plan");
  static_assert(CTAS_PER_SM * (SMEM + 1024) <= 228 * 1024, "co-resident CTAs must fit in shared memory");
  static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "co-resident CTAs must fit in tensor memory");
};

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[8], v_full[8];
  uint64_t k_empty[8], v_empty[8];  // joint ring: k_empty frees a K and V stage together
  uint64_t s_full, s_free, p_full, pv_done;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

template <typename OutT>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void store_elem(__half* p, float v) { *p = __float2half_rn(v); }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Warp-uniform bounded wait: every lane waits, and the warp proceeds only if all did.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait used only while winding down (ignores the abort flag).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait_suspend(bar, parity, kSuspendHintNs)) {
    if (clock64() - t0 > kWaitBudgetCycles) {
      atomicOr(&g_device_error, SAGE_DEVERR_TIMEOUT);
      return;
    }
  }
}

// Two E4M3 codes (RN, saturating) of a and b, a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3) & 0xFFFFu;
}

// max of three floats in one instruction (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// a0 += low half of t, a1 += high half (fp16 values), each one fp32 add rounded to nearest
__device__ __forceinline__ void add_f16x2_f32(uint32_t t, float& a0, float& a1) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tadd.rn.f32.f16 %0, lo, %0;\n\tadd.rn.f32.f16 %1, hi, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(t));
}

constexpr float kLog2_448 = 8.807354922057604f;  // p * 448 = 2^(log2 p + log2 448)
constexpr float kTau = 2.0f;                       // reference-max slack of the online softmax (log2 units)

// The Q.K^T accumulator is armed with the bit pattern of 1.5 * 2^23 before each tile's MMAs, which
// then add the int32 products to it.  Every score satisfies |S| <= 256 * 127^2 < 2^22, so the sum
// is the bit pattern of the float 1.5 * 2^23 + S: the scores arrive as floats in [2^23, 2^24), where
// float order is integer order (the row max needs no conversion) and S = value - 1.5 * 2^23 is one
// exact subtraction, with no int-to-float conversion.
constexpr uint32_t kSBiasBits = 0x4B400000u;
constexpr float kSBias = 12582912.0f;  // 1.5 * 2^23

template <int DQK, int DV, int MODE, bool CAUSAL, typename OutT, bool PV16, bool PACKED, bool OPTS>
__global__ void __launch_bounds__(192, FwdCfg<DQK, DV, PV16>::CTAS_PER_SM)
    sage_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<DQK, DV, PV16>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sbase = smem_raw + pad;
  unsigned char* sQ = sbase;
  unsigned char* sK = sQ + C::Q_BYTES;
  unsigned char* sV = sK + C::ST * C::K_BYTES;
  unsigned char* sP = sV + C::ST * C::V_BYTES;
  FwdBars* bars = reinterpret_cast<FwdBars*>(sP + C::P_BYTES);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z;
  // Dense batches are a separate instance: their lengths stay kernel parameters in the loop
  // below (measured 12% faster at d = 64 than lengths held in registers).
  const SeqView sv = seq_view<PACKED ? 1 : 0>(p.m, b);
  const int nq = PACKED ? sv.nq : p.m.Nq, nk = PACKED ? sv.nk : p.m.Nk;
  const int nblk_q = (nq + 127) / 128;
  int qt = blockIdx.x;
  if (CAUSAL) qt = nblk_q - 1 - qt;  // longest rows first
  if (qt < 0 || qt >= nblk_q) return;  // past the end of this sequence (the whole CTA leaves)
  const int hq = blockIdx.y;
  const int hkv = hq / p.G;
  // Causal mask, bottom-right aligned: query i sees keys j <= i + (nk - nq).
  const int koff = nk - nq;
  // KV tiles of C::BN keys: up to the last key below nk, and under the causal mask up to the
  // last key the tile's last row sees
  const int n_kv_all = (nk + C::BN - 1) / C::BN;
  const int last_key = qt * 128 + 127 + koff;
  const int n_kv = CAUSAL ? (last_key < 0 ? 0 : min(n_kv_all, last_key / C::BN + 1)) : n_kv_all;
  const int row = threadIdx.x;                 // softmax threads: query row inside the tile, TMEM lane
  const int grow = qt * 128 + row;             // query row in the sequence
  OutT* const out = static_cast<OutT*>(p.out);
  const long long orow = sv.q_in + (long long)grow * sv.q_tok + (long long)hq * sv.q_head;  // output row start
  if (n_kv == 0) {
    // no row of this tile sees a key (nk = 0, or the causal offset leaves the tile empty): zeros
    if (warp < 4 && grow < nq)
      for (int c = 0; c < p.m.d; ++c)
        if (SAGE_STORE_OK(p.x_out, out + orow + c, sizeof(OutT), &g_device_error)) store_elem(out + orow + c, 0.f);
    return;
  }

  // launched as a programmatic dependent of the quantize pass: wait for it to finish (and its
  // codes and scales to be visible) before anything below reads them
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 4);
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int q_row = (int)(sv.q_row0 + (long long)hq * p.m.q_head_rows) + qt * 128;
      const int k_row = (int)(sv.k_row0 + (long long)hkv * p.m.k_head_rows);
      const int v_row = (int)(sv.v_row0 + (long long)hkv * p.m.dp);
      const int v_col = (int)sv.v_col0;
      mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
      for (int s = 0; s < C::NSUB; ++s) tma_load_2d(sQ + s * 128 * C::KSUB, &tmQ, &bars->q_full, s * C::KSUB, q_row);
      auto load_k = [&](int j) {
        const int st = j % C::ST;
        mbar_arrive_expect_tx(&bars->k_full[st], C::K_BYTES);
        for (int s = 0; s < C::NSUB; ++s)
          tma_load_2d(sK + st * C::K_BYTES + s * C::BN * C::KSUB, &tmK, &bars->k_full[st], s * C::KSUB,
                      k_row + j * C::BN);
      };
      auto load_v = [&](int j) {
        const int st = j % C::ST;
        mbar_arrive_expect_tx(&bars->v_full[st], C::V_BYTES);
        tma_load_2d(sV + st * C::V_BYTES, &tmV, &bars->v_full[st], (v_col + j * C::BN) * C::PB, v_row);  // x in bytes
      };
      int k_issued = 0, v_issued = 0;
      if constexpr (C::SPLIT_RING) {
        // K(j) goes out before V(j-1): each waits for its own stage
        for (int j = 0; j <= n_kv; ++j) {
          if (j < n_kv) {
            if (!mbar_wait(&bars->k_empty[j % C::ST], ((j / C::ST) & 1) ^ 1, abort)) break;
            load_k(j);
            k_issued = j + 1;
          }
          if (j > 0) {
            if (!mbar_wait(&bars->v_empty[(j - 1) % C::ST], (((j - 1) / C::ST) & 1) ^ 1, abort)) break;
            load_v(j - 1);
            v_issued = j;
          }
        }
      } else {
        for (int j = 0; j < n_kv; ++j) {
          if (!mbar_wait(&bars->k_empty[j % C::ST], ((j / C::ST) & 1) ^ 1, abort)) break;
          load_k(j);
          load_v(j);
          k_issued = v_issued = j + 1;
        }
      }
      // make sure no copy is still landing in shared memory when the CTA exits
      drain_wait(&bars->q_full, 0);
      for (int j = k_issued - C::ST < 0 ? 0 : k_issued - C::ST; j < k_issued; ++j)
        drain_wait(&bars->k_full[j % C::ST], (j / C::ST) & 1);
      for (int j = v_issued - C::ST < 0 ? 0 : v_issued - C::ST; j < v_issued; ++j)
        drain_wait(&bars->v_full[j % C::ST], (j / C::ST) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ UMMA issuer
    // fp32 mode: QK(j) is issued as soon as S is free (the softmax has it in registers and has
    // re-armed it), ahead of PV(j-1).  fp16+fp32 mode: T(j) lives in S's columns, so QK(j+1)
    // waits until the softmax has taken T(j) into registers, and the order is QK(j), PV(j).
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(2 /*S32*/, 1 /*S8*/, 128, C::BN);
      // A = P, B = V^T, both E4M3 (kind::f8f6f4) or both F16 (kind::f16): format code 0 either way
      constexpr uint32_t idesc_pv = make_idesc(MODE == 0 ? 1 /*F32*/ : 0 /*F16*/, 0, 128, DV);
      const uint32_t pv_dst = tmem + (MODE == 0 ? C::O_COL : C::T_COL);
      const uint32_t pa = smem_u32(sP);
      auto issue_pv = [&](int i) -> bool {
        const int st = i % C::ST;
        if (!mbar_wait(&bars->v_full[st], (i / C::ST) & 1, abort)) return false;
        if (!mbar_wait(&bars->p_full, i & 1, abort)) return false;
        tc_fence_after();
        const uint32_t va = smem_u32(sV + st * C::V_BYTES);
        // one MMA per 32 bytes of the 128-byte rows: K = 32 E4M3 or 16 fp16 keys
#pragma unroll
        for (int k = 0; k < C::ROWB / 32; ++k) {
          const uint32_t acc = MODE == 0 ? (uint32_t)(i > 0 || k > 0) : (uint32_t)(k > 0);
          const uint64_t ad = smem_desc_kmajor(pa + k * 32, C::ROWB), bd = smem_desc_kmajor(va + k * 32, C::ROWB);
          if (C::P_TMEM && MODE == 0) {
            if (PV16)
              umma_f16_ts(pv_dst, tmem + C::P_COL + k * 8, bd, idesc_pv, acc);
            else
              umma_f8_ts(pv_dst, tmem + C::P_COL + k * 8, bd, idesc_pv, acc);
          } else if (PV16) {
            umma_f16(pv_dst, ad, bd, idesc_pv, acc);
          } else {
            umma_f8(pv_dst, ad, bd, idesc_pv, acc);
          }
        }
        umma_commit(C::SPLIT_RING ? &bars->v_empty[st] : &bars->k_empty[st]);  // the V (and K) stage
        umma_commit(&bars->pv_done);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort);
      if (ok) {
        tc_fence_after();
        const uint32_t qa = smem_u32(sQ);
        for (int j = 0; j < n_kv && ok; ++j) {
          const int st = j % C::ST;
          if (!mbar_wait(&bars->k_full[st], (j / C::ST) & 1, abort)) { ok = false; break; }
          // S armed with the score bias (phase j: before tile 0, then after each tile's scores left)
          if (!mbar_wait(&bars->s_free, j & 1, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ka = smem_u32(sK + st * C::K_BYTES);
#pragma unroll
          for (int k = 0; k < DQK / 32; ++k) {
            const int sub = (k * 32) / C::KSUB, off = (k * 32) % C::KSUB;
            umma_i8(tmem + C::S_COL, smem_desc_kmajor(qa + sub * 128 * C::KSUB + off, C::KSUB),
                    smem_desc_kmajor(ka + sub * C::BN * C::KSUB + off, C::KSUB), idesc_qk, 1u);
          }
          if (C::SPLIT_RING) umma_commit(&bars->k_empty[st]);  // the K stage
          umma_commit(&bars->s_full);
          if (MODE == 0) {
            if (j > 0) ok = issue_pv(j - 1);
          } else {
            ok = issue_pv(j);
          }
        }
        if (ok && MODE == 0) issue_pv(n_kv - 1);
      }
      // every UMMA this thread issued has finished before TMEM is released
      umma_commit(&bars->mma_done);
      drain_wait(&bars->mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0-3
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t scol = tmem + lane_base + C::S_COL;
    const uint32_t ocol = tmem + lane_base + C::O_COL;
    // arm S with the score bias, then release it to the first Q.K^T
    auto arm_s = [&]() {
#pragma unroll
      for (int cc = 0; cc < C::BN / 4; ++cc) tmem_fill4(scol + cc * 4, kSBiasBits);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);
    };
    arm_s();
    {
      // Co-resident CTAs share an SM and its MUFU units.  Started together they stay in step,
      // all in their exponential loops at once (each at a fraction of the MUFU rate) and all in
      // their other work at once (MUFU idle).  The CTAs arriving on an SM are therefore started
      // a fraction of a tile apart; measured +2.5% to +6% on the fused kernel.
      __shared__ unsigned int slot;
      if (threadIdx.x == 0) {
        unsigned int smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        slot = atomicAdd(&g_sm_arrivals[smid & 255], 1u) % C::CTAS_PER_SM;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (slot) __nanosleep(slot * (600u / C::CTAS_PER_SM));
    }
    // the Q scale of this row's group (its 128-token block, or with finer scales (OPTS) its 32-token
    // warp group or the row itself).  Instances without the options keep the plain block index:
    // changing it was measured to slow the tile loop's schedule by 2%.
    const float qsv = OPTS ? p.qs[(sv.q_row0 + (long long)hq * p.m.q_head_rows + qt * 128 + row) >> p.q_gran_log2]
                           : p.qs[(sv.q_row0 + (long long)hq * p.m.q_head_rows) / 128 + qt];
    const float* ksp = p.ks + (sv.k_row0 + (long long)hkv * p.m.k_head_rows) / 128;
    unsigned char* prow = sP + row * C::ROWB;
    float m = -INFINITY, l = 0.f;  // m: reference max; l accumulates the stored P values' scale
    // the next key tile's K scale, loaded one tile ahead so that its global-load latency leaves the
    // tile's critical path (measured +2.8% to +3.2% at d = 128 without a causal mask); the causal
    // d >= 128 fp32-accumulation instances load it in the loop, measured faster there
    constexpr bool KS_AHEAD = DQK == 64 || !CAUSAL || MODE == 1;
    float ks_next = KS_AHEAD ? ksp[0] : 0.f;
    bool ok = true;
    for (int i = 0; i < n_kv; ++i) {
      if (!warp_wait(&bars->s_full, i & 1, abort)) { ok = false; break; }
      tc_fence_after();
      constexpr int BN = C::BN;
      // scores as float bit patterns 1.5 * 2^23 + S (see kSBiasBits)
      uint32_t s[BN];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(scol + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[cc * 32]));
      tmem_wait_ld();
      if (MODE == 0) arm_s();  // S is in registers: re-arm it for the next Q.K^T

      // dequantization factor in the log2 domain, with the K scale of the 128-key block (loaded one
      // tile ahead where KS_AHEAD, else here)
      float ksv;
      if constexpr (KS_AHEAD) {
        ksv = ks_next;
        if (i + 1 < n_kv) ks_next = ksp[(i + 1) * BN / 128];
      } else {
        ksv = ksp[i * BN / 128];
      }
      const float f = __fmul_rn(__fmul_rn(qsv, ksv), p.scale_log2);
      const int key0 = i * BN;
      const bool edge = (key0 + BN > nk) || (CAUSAL && key0 + BN - 1 > qt * 128 + koff);
      int lim = BN;  // this row sees the tile's columns c < lim (none if lim <= 0)
      if (edge) {
        lim = min(nk - key0, BN);
        if (CAUSAL) lim = min(lim, grow + koff - key0 + 1);
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c >= lim) s[c] = __float_as_uint(-INFINITY);
      }
      // row max with three-input float maxima on the biased scores (their float order is the
      // scores' order); 1.5 * 2^23 + S - 1.5 * 2^23 recovers S exactly
      float mx4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) mx4[e] = fmaxf(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1]));
#pragma unroll
      for (int c = 8; c < BN; c += 8)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          mx4[e] = fmax3(mx4[e], __uint_as_float(s[c + 2 * e]), __uint_as_float(s[c + 2 * e + 1]));
      const float mx = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]);
      const float mt = (mx == -INFINITY) ? -INFINITY : __fmul_rn(__fsub_rn(mx, kSBias), f);  // the tile's row max, scaled
      // The reference max m moves only when the running max exceeds it by more than kTau,
      // so O is rescaled rarely; p = 2^(s - m) <= 2^kTau is stored as E4M3(p * 448 * 2^-kTau)
      // (FP8 P.V) or as fp16(p) (FP16 P.V).
      const float mc = fmaxf(m, mt);
      const bool upd = mc > __fadd_rn(m, kTau);
      const float m_new = upd ? mc : m;
      const float alpha = upd ? ((m == -INFINITY) ? 0.f : ex2_approx(m - m_new)) : 1.f;
      const float bias = (m_new == -INFINITY) ? 0.f : (PV16 ? 0.f : kLog2_448 - kTau) - m_new;
      const bool rescale = MODE == 0 && i > 0 && __any_sync(0xffffffffu, alpha != 1.f);
      // p * 448 * 2^-kTau = 2^(s*f - m + log2 448 - kTau) -> E4M3, 4 keys per 32-bit word;
      // FP16 P.V: p = 2^(s*f - m) -> fp16, 2 keys per word
      // four scalar partial row sums (packed f32x2 adds measured slower in every instance)
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pw[C::ROWB / 4];
#pragma unroll
      for (int c4 = 0; c4 < BN / 4; ++c4) {
        float pv[4];
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const int c = c4 * 4 + e;
          float x0, x1;
          // the exact score S = (1.5 * 2^23 + S) - 1.5 * 2^23 (same binade: no rounding), then
          // S * f + bias with one rounding, as the scores were integers converted to float
          // packed f32x2 math measured faster only in the causal fp32-accumulation instances
          // (scalar: +13% non-causal at d = 128, +18% at d = 256, -8% causal)
          if (DQK >= 128 && MODE == 0 && CAUSAL) {
            const float2 sc = __fadd2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                         make_float2(-kSBias, -kSBias));
            const float2 x = __ffma2_rn(sc, make_float2(f, f), make_float2(bias, bias));
            x0 = x.x;
            x1 = x.y;
          } else {
            x0 = fmaf(__fsub_rn(__uint_as_float(s[c]), kSBias), f, bias);
            x1 = fmaf(__fsub_rn(__uint_as_float(s[c + 1]), kSBias), f, bias);
          }
          pv[e] = ex2_approx(x0);
          pv[e + 1] = ex2_approx(x1);
          if (edge) {
            pv[e] = (c < lim) ? pv[e] : 0.f;
            pv[e + 1] = (c + 1 < lim) ? pv[e + 1] : 0.f;
          }
          rs[e] += pv[e];
          rs[e + 1] += pv[e + 1];
        }
        if (PV16) {
          pw[2 * c4] = pack2<__half>(pv[0], pv[1]);
          pw[2 * c4 + 1] = pack2<__half>(pv[2], pv[3]);
        } else {
          pw[c4] = e4m3x2(pv[0], pv[1]) | (e4m3x2(pv[2], pv[3]) << 16);
        }
      }
      l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
      m = m_new;
      if (MODE == 0 && i > 0) {
        // P's buffer and O were last used by the P.V MMA of tile i-1 (long done by now)
        if (!warp_wait(&bars->pv_done, (i - 1) & 1, abort)) { ok = false; break; }
        tc_fence_after();
      }
      // 16-byte chunk ch of the 128-byte row goes to chunk ch ^ (row & 7): the 128B swizzle the
      // P.V descriptor expects
      if constexpr (C::P_TMEM && MODE == 0) {
        tmem_st32(tmem + lane_base + C::P_COL, *reinterpret_cast<const uint32_t(*)[32]>(&pw[0]));
        tmem_wait_st();
      } else {
#pragma unroll
        for (int ch = 0; ch < C::ROWB / 16; ++ch) {
          const int sw = row & 7;
          *reinterpret_cast<uint4*>(prow + ((ch ^ sw) << 4)) =
              make_uint4(pw[ch * 4 + 0], pw[ch * 4 + 1], pw[ch * 4 + 2], pw[ch * 4 + 3]);
        }
        fence_proxy_async_smem();
      }
      if (rescale) {
        // O *= alpha (rows whose reference did not move have alpha = 1); 64 columns per batch,
        // every TMEM load of a batch in flight before one wait
#pragma unroll
        for (int hh = 0; hh < DV / 64; ++hh) {
          uint32_t o[64];
          tmem_ld32(ocol + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
          tmem_ld32(ocol + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 64; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(ocol + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
          tmem_st32(ocol + hh * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);

      if (MODE == 1) {
        // O = O * alpha + T(i), T being this tile's fresh fp16 accumulator (in S's columns).  T is
        // taken into registers first, so S is re-armed and released to the next Q.K^T before the
        // merge, which then overlaps that MMA.
        if (!warp_wait(&bars->pv_done, i & 1, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tcol = tmem + lane_base + C::T_COL;
        uint32_t t[DV / 2];
#pragma unroll
        for (int cc = 0; cc < DV / 32; ++cc) tmem_ld16_pack16(tcol + cc * 32, *reinterpret_cast<uint32_t(*)[16]>(&t[cc * 16]));
        tmem_wait_ld();
        arm_s();
        // O = O * alpha + T (tile 0: O = T; rows whose reference did not move have alpha = 1).
        // When no row of the warp moved its reference the multiply is left out: O += T, the same
        // bits (measured +2.8% on the video-DiT shape, +1.7% with FP16 P.V).
        const bool scaled = i == 0 || __any_sync(0xffffffffu, alpha != 1.f);
        const float am = i == 0 ? 0.f : alpha;
        // 64 columns of O per batch, both loads in flight before one wait (the merge waits on
        // tensor-memory loads: measured +1.8% on the video-DiT shape over 32-column batches)
#pragma unroll
        for (int cc = 0; cc < DV / 64; ++cc) {
          uint32_t o[64];
          if (i > 0) {
            tmem_ld32(ocol + cc * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
            tmem_ld32(ocol + cc * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 64; ++e) o[e] = 0u;
          }
          if (scaled) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              float a0 = __uint_as_float(o[2 * e]) * am, a1 = __uint_as_float(o[2 * e + 1]) * am;
              add_f16x2_f32(t[cc * 32 + e], a0, a1);
              o[2 * e] = __float_as_uint(a0);
              o[2 * e + 1] = __float_as_uint(a1);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              float a0 = __uint_as_float(o[2 * e]), a1 = __uint_as_float(o[2 * e + 1]);
              add_f16x2_f32(t[cc * 32 + e], a0, a1);
              o[2 * e] = __float_as_uint(a0);
              o[2 * e + 1] = __float_as_uint(a1);
            }
          }
          tmem_st32(ocol + cc * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
          tmem_st32(ocol + cc * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
        }
        tmem_wait_st();
      }
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && MODE == 0) {
      ok = warp_wait(&bars->pv_done, (n_kv - 1) & 1, abort);
      if (ok) tc_fence_after();
    }
    if (ok) {
      const float inv_l = l > 0.f ? __fdiv_rn(1.f, l) : 0.f;  // a row that saw no key outputs zeros
      const float* vsp = p.vs + ((size_t)b * p.m.Hkv + hkv) * p.m.dp;
      // smoothed V: its token mean goes back on (rows that saw a key)
      const float* vmp =
          (OPTS && p.vm && l > 0.f) ? p.vm + ((size_t)b * p.m.Hkv + hkv) * p.m.dp : nullptr;
#pragma unroll 1
      for (int cc = 0; cc < DV / 32; ++cc) {
        uint32_t o[32];
        float of[32];
        tmem_ld32(ocol + cc * 32, o);
        tmem_wait_ld();
        if (grow < nq) {
          const int c0 = cc * 32;
#pragma unroll
          for (int e = 0; e < 32; ++e) of[e] = __uint_as_float(o[e]) * (vsp[cc * 32 + e] * inv_l);
          if (OPTS && vmp) {
#pragma unroll
            for (int e = 0; e < 32; ++e) of[e] = __fadd_rn(of[e], vmp[cc * 32 + e]);
          }
          if (c0 + 32 <= p.m.d && p.vec_out) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pack2<OutT>(of[2 * e], of[2 * e + 1]);
            uint4* dst = reinterpret_cast<uint4*>(out + orow + c0);
            if (SAGE_STORE_OK(p.x_out, dst, 32 * sizeof(OutT), &g_device_error)) {
#pragma unroll
              for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c0 + e < p.m.d && SAGE_STORE_OK(p.x_out, out + orow + c0 + e, sizeof(OutT), &g_device_error))
                store_elem(out + orow + c0 + e, of[e]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------------
// Diagnostic: int32 S = Q8 . K8^T for a list of (b, hq, q_tile, k_tile) tiles, through the
// same TMA loads, shared-memory descriptors and kind::i8 UMMA as the fused kernel.
// ------------------------------------------------------------------------------------------------
template <int DQK>
struct QkDumpCfg {
  static constexpr int KSUB = DQK >= 128 ? 128 : 64;
  static constexpr int NSUB = DQK / KSUB;
  static constexpr int Q_BYTES = 128 * DQK, K_BYTES = 128 * DQK, BAR_BYTES = 256;
};

template <int DQK>
__global__ void __launch_bounds__(128, 1)
    sage_qk_dump_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const QkDumpParams p) {
  using C = QkDumpCfg<DQK>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* sQ = smem_raw + pad;
  unsigned char* sK = sQ + C::Q_BYTES;
  FwdBars* bars = reinterpret_cast<FwdBars*>(sK + C::K_BYTES);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int b = p.tiles[4 * t], hq = p.tiles[4 * t + 1], qt = p.tiles[4 * t + 2], kt = p.tiles[4 * t + 3];
  const bool valid = b >= 0 && b < p.B && hq >= 0 && hq < p.Hq && qt >= 0 && qt < p.nblk && kt >= 0 && kt < p.nblk;
  if (!valid) {
    if (threadIdx.x == 0) atomicOr(&g_device_error, SAGE_DEVERR_BAD_ARG);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  if (threadIdx.x == 32) {
    const int q_row = (b * p.Hq + hq) * p.Np + qt * 128;
    const int k_row = (b * p.Hkv + hq / p.G) * p.Np + kt * 128;
    mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES + C::K_BYTES);
    for (int s = 0; s < C::NSUB; ++s) {
      tma_load_2d(sQ + s * 128 * C::KSUB, &tmQ, &bars->q_full, s * C::KSUB, q_row);
      tma_load_2d(sK + s * 128 * C::KSUB, &tmK, &bars->q_full, s * C::KSUB, k_row);
    }
    if (mbar_wait(&bars->q_full, 0, abort)) {
      tc_fence_after();
      constexpr uint32_t idesc = make_idesc(2, 1, 128, 128);
#pragma unroll
      for (int k = 0; k < DQK / 32; ++k) {
        const int sub = (k * 32) / C::KSUB, off = (k * 32) % C::KSUB;
        umma_i8(tmem, smem_desc_kmajor(smem_u32(sQ) + sub * 128 * C::KSUB + off, C::KSUB),
                smem_desc_kmajor(smem_u32(sK) + sub * 128 * C::KSUB + off, C::KSUB), idesc, (uint32_t)(k > 0));
      }
    } else {
      drain_wait(&bars->q_full, 0);
    }
    umma_commit(&bars->mma_done);
  }
  if (warp_wait(&bars->mma_done, 0, abort) && !*abort) {
    tc_fence_after();
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int32_t* dst = p.out + ((size_t)t * 128 + warp * 32 + lane) * 128;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_base + cc * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 8; ++e)
        reinterpret_cast<uint4*>(dst + cc * 32)[e] = make_uint4(r[4 * e], r[4 * e + 1], r[4 * e + 2], r[4 * e + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------------------------------------
// Diagnostic: the tcgen05.mma issue rate of this GPU.  One CTA per SM; one thread issues `iters`
// rounds of 4 back-to-back MMAs (M = 128, N = 256, 32 bytes of K per row: K = 32 for kind::i8 and
// kind::f8f6f4, K = 16 for kind::f16) from one zeroed shared-memory tile pair into one TMEM
// accumulator, then waits for them (bounded).  The operand data play no part in the rate.
// ------------------------------------------------------------------------------------------------
template <int KIND>
__global__ void __launch_bounds__(128, 1) sage_mma_probe_kernel(int iters) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char* a = smem_raw + pad;  // 128 rows x 128 bytes
  unsigned char* bt = a + 128 * 128;  // 256 rows x 128 bytes
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (128 + 256) * 128 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(a)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tbase, 256);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    // kind::i8: S32 accumulator, S8 operands; kind::f8f6f4: F32, E4M3; kind::f16: F32, F16
    constexpr uint32_t idesc = make_idesc(KIND == 0 ? 2 : 1, KIND == 0 ? 1 : 0, 128, 256);
    const uint32_t aa = smem_u32(a), bb = smem_u32(bt);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ad = smem_desc_kmajor(aa + k * 32, 128), bd = smem_desc_kmajor(bb + k * 32, 128);
        if (KIND == 0)
          umma_i8(tbase, ad, bd, idesc, 1u);
        else if (KIND == 1)
          umma_f8(tbase, ad, bd, idesc, 1u);
        else
          umma_f16(tbase, ad, bd, idesc, 1u);
      }
    }
    umma_commit(&bar);
    if (!mbar_wait(&bar, 0, &abort_flag)) drain_wait(&bar, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

// ------------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------------
// Sets a kernel's dynamic shared-memory limit once per device (the attribute is per device).
template <typename K>
static cudaError_t ensure_smem_limit(K kern, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

template <int DQK, int DV, int MODE, bool CAUSAL, typename OutT, bool PV16>
static cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const FwdParams& p, cudaStream_t st) {
  using C = FwdCfg<DQK, DV, PV16>;
  const bool opts = p.q_gran_log2 != 7 || p.vm != nullptr;  // finer Q scales or smoothed V
  const int which = (p.m.seqs ? 1 : 0) + (opts ? 2 : 0);
  auto kern = which == 0 ? sage_fwd_kernel<DQK, DV, MODE, CAUSAL, OutT, PV16, false, false>
            : which == 1 ? sage_fwd_kernel<DQK, DV, MODE, CAUSAL, OutT, PV16, true, false>
            : which == 2 ? sage_fwd_kernel<DQK, DV, MODE, CAUSAL, OutT, PV16, false, true>
                         : sage_fwd_kernel<DQK, DV, MODE, CAUSAL, OutT, PV16, true, true>;
  static std::atomic<unsigned long long> attr_done[4] = {{0}, {0}, {0}, {0}};
  cudaError_t e = ensure_smem_limit(kern, C::SMEM, attr_done[which]);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nblk_q, p.m.Hq, p.m.B);
  // a programmatic dependent of whatever ran before on the stream (the quantize pass): the CTAs
  // may start while it finishes and wait for it in griddepcontrol.wait
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p);
}

template <int DQK, int DV, typename OutT, bool PV16>
static cudaError_t launch_fwd_m(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const FwdParams& p, int causal, int accum, cudaStream_t st) {
  if (accum == 0)
    return causal ? launch_fwd_t<DQK, DV, 0, true, OutT, PV16>(tq, tk, tv, p, st)
                  : launch_fwd_t<DQK, DV, 0, false, OutT, PV16>(tq, tk, tv, p, st);
  return causal ? launch_fwd_t<DQK, DV, 1, true, OutT, PV16>(tq, tk, tv, p, st)
                : launch_fwd_t<DQK, DV, 1, false, OutT, PV16>(tq, tk, tv, p, st);
}

// pv_mode: bit 0 = fp16+fp32 accumulation, bit 1 = FP16 P.V operands (sage_pv_mode values)
template <int DQK, int DV, typename OutT>
static cudaError_t launch_fwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const FwdParams& p, int causal, int pv_mode, cudaStream_t st) {
  return (pv_mode & 2) ? launch_fwd_m<DQK, DV, OutT, true>(tq, tk, tv, p, causal, pv_mode & 1, st)
                       : launch_fwd_m<DQK, DV, OutT, false>(tq, tk, tv, p, causal, pv_mode & 1, st);
}

template <typename OutT>
static cudaError_t launch_fwd_o(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const FwdParams& p, int causal, int mode, cudaStream_t st) {
  switch (p.m.dp) {
    case 64: return launch_fwd_d<64, 64, OutT>(tq, tk, tv, p, causal, mode, st);
    case 128: return launch_fwd_d<128, 128, OutT>(tq, tk, tv, p, causal, mode, st);
    case 256: return launch_fwd_d<256, 256, OutT>(tq, tk, tv, p, causal, mode, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                       int dtype, int causal, int pv_mode, cudaStream_t st) {
  return dtype == SAGE_BF16 ? launch_fwd_o<__nv_bfloat16>(tq, tk, tv, p, causal, pv_mode, st)
                            : launch_fwd_o<__half>(tq, tk, tv, p, causal, pv_mode, st);
}

// ------------------------------------------------------------------------------------------------
// Packed (varlen) batches: per-sequence table from the cumulative lengths.  One CTA: each thread
// takes a run of consecutive sequences, a block scan gives every run its first padded row.
// A table that is not non-decreasing from >= 0, exceeds the stated maxima or runs past the
// stated totals flags SAGE_DEVERR_BAD_ARG and leaves every sequence empty, so no later kernel
// reads outside the caller's tensors.
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) seq_plan_kernel(const int32_t* __restrict__ cu_q,
                                                        const int32_t* __restrict__ cu_k, int B, int max_q, int max_k,
                                                        long long total_q, long long total_k, SeqDesc* seqs) {
  __shared__ long long scan_q[1024], scan_k[1024];
  __shared__ int bad;
  const int t = threadIdx.x, per = (B + 1023) / 1024;
  const int b0 = min(B, t * per), b1 = min(B, b0 + per);
  if (t == 0) bad = 0;
  __syncthreads();
  auto pad128 = [](long long n) { return n > 0 ? (n + 127) / 128 * 128 : 0ll; };
  long long run_q = 0, run_k = 0;
  bool my_bad = false;
  for (int b = b0; b < b1; ++b) {
    const long long q0 = cu_q[b], q1 = cu_q[b + 1], k0 = cu_k[b], k1 = cu_k[b + 1];
    if (q0 < 0 || k0 < 0 || q1 < q0 || k1 < k0 || q1 - q0 > max_q || k1 - k0 > max_k || q1 > total_q ||
        k1 > total_k)
      my_bad = true;
    run_q += pad128(q1 - q0);
    run_k += pad128(k1 - k0);
  }
  if (my_bad) atomicOr(&bad, 1);
  scan_q[t] = run_q, scan_k[t] = run_k;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan of the runs' padded lengths
    const long long vq = t >= o ? scan_q[t - o] : 0, vk = t >= o ? scan_k[t - o] : 0;
    __syncthreads();
    scan_q[t] += vq, scan_k[t] += vk;
    __syncthreads();
  }
  const bool any_bad = bad != 0;
  if (t == 0 && any_bad) atomicOr(&g_device_error, SAGE_DEVERR_BAD_ARG);
  long long row_q = scan_q[t] - run_q, row_k = scan_k[t] - run_k;  // first padded row of this run
  for (int b = b0; b < b1; ++b) {
    SeqDesc d{0, 0, 0, 0, 0, 0};
    if (!any_bad) {
      const long long q0 = cu_q[b], k0 = cu_k[b];
      d.nq = (int)(cu_q[b + 1] - q0), d.nk = (int)(cu_k[b + 1] - k0);
      d.q_row = (int)row_q, d.k_row = (int)row_k;
      d.q_tok = q0, d.k_tok = k0;
      row_q += pad128(d.nq), row_k += pad128(d.nk);
    }
    seqs[b] = d;
  }
}

cudaError_t launch_seq_plan(const int32_t* cu_q, const int32_t* cu_k, int B, int max_q, int max_k,
                            long long total_q, long long total_k, SeqDesc* seqs, cudaStream_t st) {
  seq_plan_kernel<<<1, 1024, 0, st>>>(cu_q, cu_k, B, max_q, max_k, total_q, total_k, seqs);
  return cudaGetLastError();
}

// Failure-path check: one thread waits, with the library's bounded wait, on an mbarrier that
// nothing completes.  The wait runs out after `budget_cycles`, records SAGE_DEVERR_TIMEOUT and
// returns, exactly as a stalled pipeline stage of the fused kernel would.
__global__ void sage_wait_probe_kernel(long long budget_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_flag, budget_cycles, 1000u /* re-check every ~1 us */);
  }
}

cudaError_t launch_wait_probe(long long budget_cycles, cudaStream_t st) {
  sage_wait_probe_kernel<<<1, 32, 0, st>>>(budget_cycles);
  return cudaGetLastError();
}

cudaError_t read_clear_device_error(int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

template <int DQK>
static cudaError_t launch_qk_dump_t(const CUtensorMap& tq, const CUtensorMap& tk, const QkDumpParams& p,
                                    cudaStream_t st) {
  using C = QkDumpCfg<DQK>;
  const int smem = 1024 + C::Q_BYTES + C::K_BYTES + C::BAR_BYTES;
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = ensure_smem_limit(sage_qk_dump_kernel<DQK>, smem, attr_done);
  if (e != cudaSuccess) return e;
  sage_qk_dump_kernel<DQK><<<p.n_tiles, 128, smem, st>>>(tq, tk, p);
  return cudaGetLastError();
}

template <int KIND>
static cudaError_t launch_mma_probe_t(int iters, int n_sm, cudaStream_t st) {
  const int smem = 1024 + (128 + 256) * 128;
  static std::atomic<unsigned long long> attr_done{0};
  cudaError_t e = ensure_smem_limit(sage_mma_probe_kernel<KIND>, smem, attr_done);
  if (e != cudaSuccess) return e;
  sage_mma_probe_kernel<KIND><<<n_sm, 128, smem, st>>>(iters);
  return cudaGetLastError();
}

cudaError_t launch_mma_probe(int kind, int iters, int n_sm, cudaStream_t st) {
  switch (kind) {
    case 0: return launch_mma_probe_t<0>(iters, n_sm, st);
    case 1: return launch_mma_probe_t<1>(iters, n_sm, st);
    case 2: return launch_mma_probe_t<2>(iters, n_sm, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_qk_dump(const CUtensorMap& tq, const CUtensorMap& tk, const QkDumpParams& p, int dp,
                           cudaStream_t st) {
  switch (dp) {
    case 64: return launch_qk_dump_t<64>(tq, tk, p, st);
    case 128: return launch_qk_dump_t<128>(tq, tk, p, st);
    case 256: return launch_qk_dump_t<256>(tq, tk, p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sage
