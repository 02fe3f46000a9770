// C ABI: argument checks, workspace, TMA tensor maps and launches.
// The operation and the argument contract are documented in include/sage.h.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "sage_internal.h"

using namespace sage;

namespace {

constexpr size_t kAlign = 1024;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int padded_dim(int d) { return d <= 64 ? 64 : (d <= 128 ? 128 : 256); }

// Sizes of one call.  Dense batches: B sequences of Nq queries and Nk keys.  Packed (varlen)
// batches: B sequences of at most Nq / Nk tokens, total_q / total_k tokens in all.
struct Dims {
  int B, Hq, Hkv, Nq, Nk, d, dp, G;
  int nblk_q, nblk_k;                  // 128-token blocks of the longest query / key sequence
  long long q_head_rows, k_head_rows;  // q8 / k8 rows between heads (dense Npq / Npk; packed Tq / Tk)
  long long q_rows, k_rows;            // q8 / k8 rows in all
  bool packed;
  long long total_q, total_k;
};

long long round128(long long x) { return (x + 127) / 128 * 128; }

sage_status finish_dims(Dims* m) {
  m->dp = padded_dim(m->d);
  m->G = m->Hq / m->Hkv;
  m->nblk_q = (m->Nq + 127) / 128;
  m->nblk_k = (m->Nk + 127) / 128;
  if (m->packed) {
    // every sequence starts a fresh 128-row block: sum of round128(n_b) <= total + 127 B
    m->q_head_rows = round128(m->total_q) + 128LL * m->B;
    m->k_head_rows = round128(m->total_k) + 128LL * m->B;
    m->q_rows = m->q_head_rows * m->Hq;
    m->k_rows = m->k_head_rows * m->Hkv;
  } else {
    m->q_head_rows = round128(m->Nq);
    m->k_head_rows = round128(m->Nk);
    m->q_rows = m->q_head_rows * m->Hq * m->B;
    m->k_rows = m->k_head_rows * m->Hkv * m->B;
  }
  // TMA coordinates are 32-bit signed: rows of q8 / k8 / V^T and the byte column of V^T
  const long long v_rows = m->k_rows / m->k_head_rows * m->dp;
  if (m->q_rows >= (1LL << 31) || m->k_rows >= (1LL << 31) || v_rows >= (1LL << 31) ||
      m->k_head_rows * 2 >= (1LL << 31))
    return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

sage_status check_heads(int B, int Hq, int Hkv, int d) {
  if (B < 1 || Hq < 1 || Hkv < 1 || d < 1) return SAGE_ERR_INVALID_ARG;
  if (d > 256 || Hq % Hkv != 0) return SAGE_ERR_INVALID_ARG;
  if (B > 65535 || 2L * Hq > 65535 || (long)Hq + 2L * Hkv > 65535) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

sage_status check_dims(int B, int Hq, int Hkv, int Nq, int Nk, int d, Dims* out) {
  sage_status s = check_heads(B, Hq, Hkv, d);
  if (s != SAGE_OK) return s;
  if (Nq < 1 || Nk < 1 || Nq > (1 << 30) || Nk > (1 << 30)) return SAGE_ERR_INVALID_ARG;
  Dims m;
  m.B = B, m.Hq = Hq, m.Hkv = Hkv, m.Nq = Nq, m.Nk = Nk, m.d = d;
  m.packed = false;
  m.total_q = (long long)B * Nq, m.total_k = (long long)B * Nk;
  if ((s = finish_dims(&m)) != SAGE_OK) return s;
  *out = m;
  return SAGE_OK;
}

sage_status check_dims_packed(int B, int Hq, int Hkv, int max_q, int max_k, long long total_q, long long total_k,
                              int d, Dims* out) {
  sage_status s = check_heads(B, Hq, Hkv, d);
  if (s != SAGE_OK) return s;
  if (max_q < 1 || max_k < 0 || total_q < 1 || total_k < 0 || max_q > (1 << 30) || max_k > (1 << 30) ||
      total_q > (1LL << 40) || total_k > (1LL << 40))
    return SAGE_ERR_INVALID_ARG;
  Dims m;
  m.B = B, m.Hq = Hq, m.Hkv = Hkv, m.Nq = max_q, m.Nk = max_k, m.d = d;
  m.packed = true;
  m.total_q = total_q, m.total_k = total_k;
  if ((s = finish_dims(&m)) != SAGE_OK) return s;
  *out = m;
  return SAGE_OK;
}

SeqMap seq_map(const Dims& m, int layout, const SeqDesc* seqs) {
  SeqMap s;
  s.seqs = m.packed ? seqs : nullptr;
  s.B = m.B, s.Hq = m.Hq, s.Hkv = m.Hkv, s.d = m.d, s.dp = m.dp;
  s.Nq = m.Nq, s.Nk = m.Nk;
  s.q_head_rows = m.q_head_rows, s.k_head_rows = m.k_head_rows;
  s.layout = m.packed ? SAGE_NHD : layout;
  return s;
}

sage_status check_dtype(int dtype) {
  if (dtype == SAGE_FP32) return SAGE_ERR_UNSUPPORTED;
  if (dtype != SAGE_FP16 && dtype != SAGE_BF16) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + nb && y < x + na;
}

sage_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return SAGE_OK;
  return e == cudaErrorMemoryAllocation ? SAGE_ERR_OOM : SAGE_ERR_CUDA;
}

// Host-side failure injection (sage_test_inject): a compute capability reported instead of the
// device's (0: query the device), and a number of workspace allocations to fail.
std::atomic<int> g_fake_cc{0};
std::atomic<int> g_fail_allocs{0};

sage_status check_device() {
  const int fake = g_fake_cc.load(std::memory_order_relaxed);
  if (fake) return fake == 100 ? SAGE_OK : SAGE_ERR_ARCH;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return SAGE_ERR_CUDA;
  return (major == 10 && minor == 0) ? SAGE_OK : SAGE_ERR_ARCH;
}

float resolve_scale(float sm_scale, int d) {
  if (!(sm_scale > 0.f) || std::isnan(sm_scale)) return 1.0f / std::sqrt((float)d);
  return sm_scale;
}

// ---------------------------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D byte tensor: `inner` bytes per row (contiguous), `rows` rows, box {box_inner, box_rows}.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz = box_inner == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

bool pv_mode_valid(int pv_mode) {
  return pv_mode == SAGE_PV_FP32 || pv_mode == SAGE_PV_FP16_FP32 || pv_mode == SAGE_PV16_FP32 ||
         pv_mode == SAGE_PV16_FP16_FP32;
}
bool pv_mode_fp16_operands(int pv_mode) { return pv_mode == SAGE_PV16_FP32 || pv_mode == SAGE_PV16_FP16_FP32; }

// sage_opts, checked: log2 of the query tokens per Q scale, and V smoothing
struct Opts {
  int q_gran_log2 = 7;
  int smooth_v = 0;
};

sage_status parse_opts(const sage_opts* o, Opts* out) {
  Opts r;
  if (o) {
    switch (o->q_gran) {
      case 0:
      case 128: r.q_gran_log2 = 7; break;
      case 32: r.q_gran_log2 = 5; break;
      case 1: r.q_gran_log2 = 0; break;
      default: return SAGE_ERR_INVALID_ARG;
    }
    if (o->smooth_v != 0 && o->smooth_v != 1) return SAGE_ERR_INVALID_ARG;
    r.smooth_v = o->smooth_v;
  }
  *out = r;
  return SAGE_OK;
}

// Workspace memory: a stream-ordered pool per device, owned by the library, that keeps the
// memory it has handed out (release threshold = unlimited), so that repeated calls reuse
// it instead of mapping fresh device memory each time.
cudaError_t workspace_alloc(void** ptr, size_t bytes, cudaStream_t st) {
  for (int n = g_fail_allocs.load(); n > 0;)  // an injected failure, before any device call
    if (g_fail_allocs.compare_exchange_weak(n, n - 1)) return cudaErrorMemoryAllocation;
  constexpr int kMaxDevices = 128;
  static std::mutex mu;
  static cudaMemPool_t pools[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaMemPool_t pool;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!pools[dev]) {
      cudaMemPoolProps props;
      memset(&props, 0, sizeof(props));
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      cudaMemPool_t p = nullptr;
      if ((e = cudaMemPoolCreate(&p, &props)) != cudaSuccess) return e;
      uint64_t keep = ~0ull;
      if ((e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) return e;
      pools[dev] = p;
    }
    pool = pools[dev];
  }
  return cudaMallocFromPoolAsync(ptr, bytes, pool, st);
}

// Store extents of the checked build (-DSAGE_CHECKED): each buffer's size as the header states it.
Extent extent_of(const void* ptr, size_t bytes) {
  Extent x;
  x.base = static_cast<unsigned char*>(const_cast<void*>(ptr));
  x.bytes = ptr ? bytes : 0;
  return x;
}

std::atomic<long long> g_out_limit{0};  // test hook: narrows the output extent when > 0

Extent out_extent(const Dims& m, const void* out) {
  size_t bytes = (size_t)m.total_q * m.Hq * m.d * 2;  // fp16 / bf16 output
  const long long lim = g_out_limit.load();
  if (lim > 0 && (size_t)lim < bytes) bytes = (size_t)lim;
  return extent_of(out, bytes);
}

struct QuantBufs {
  const SeqDesc* seqs;  // packed batches: the per-sequence table (else nullptr)
  float* vm;            // V's token mean (read only when V is smoothed)
  int8_t* q8;
  float* qs;
  int8_t* k8;
  float* ks;
  float* km;
  uint8_t* v8t;
  float* vs;
};

sage_status run_fwd(const Dims& m, const QuantBufs& qb, void* out, int dtype, int layout, int causal, float sm_scale,
                    int pv_mode, const Opts& o, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  const uint32_t ksub = m.dp >= 128 ? 128 : 64;
  const uint32_t dv = m.dp;  // V^T rows (channels) per tile: all of the padded head dim
  const bool pv16 = pv_mode_fp16_operands(pv_mode);
  const uint32_t bn = pv16 ? 64 : 128;  // keys per KV tile of the fused kernel
  const uint64_t vpitch = (uint64_t)m.k_head_rows * (pv16 ? 2 : 1);  // bytes per V^T row (one channel)
  // V^T tile box: 128 bytes of keys (128 E4M3 or 64 fp16 codes) x dv channels
  if (!make_map(&tq, qb.q8, m.dp, (uint64_t)m.q_rows, ksub, 128) ||
      !make_map(&tk, qb.k8, m.dp, (uint64_t)m.k_rows, ksub, bn) ||
      !make_map(&tv, qb.v8t, vpitch, (uint64_t)(m.k_rows / m.k_head_rows) * m.dp, 128, dv))
    return SAGE_ERR_CUDA;
  FwdParams p;
  p.qs = qb.qs, p.ks = qb.ks, p.vs = qb.vs, p.out = out;
  p.vm = o.smooth_v ? qb.vm : nullptr;
  p.q_gran_log2 = o.q_gran_log2;
  p.m = seq_map(m, layout, qb.seqs);
  p.nblk_q = m.nblk_q;
  p.G = m.G;
  p.vec_out = (m.d % 8 == 0) && aligned16(out);
  p.x_out = out_extent(m, out);
  p.scale_log2 = resolve_scale(sm_scale, m.d) * 1.4426950408889634f;
  return from_cuda(launch_fwd(tq, tk, tv, p, dtype, causal, pv_mode, st));
}

struct WsLayout {
  size_t q8, qs, k8, ks, km, v8t, vs, vm, ksum, vmax, vsum, vmin, vinv, seqs, total;
};

WsLayout ws_layout(const Dims& m, int pv_mode, const Opts& o) {
  WsLayout w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  w.q8 = take((size_t)m.q_rows * m.dp);
  w.qs = take(((size_t)m.q_rows >> o.q_gran_log2) * 4);
  w.k8 = take((size_t)m.k_rows * m.dp);
  w.ks = take((size_t)m.k_rows / 128 * 4);
  w.km = take((size_t)m.B * m.Hkv * m.dp * 4);
  w.v8t = take((size_t)m.k_rows * m.dp * (pv_mode_fp16_operands(pv_mode) ? 2 : 1));
  w.vs = take((size_t)m.B * m.Hkv * m.dp * 4);
  w.vm = take((size_t)m.B * m.Hkv * m.dp * 4);
  w.ksum = take((size_t)m.k_rows / 128 * m.dp * 4);
  w.vmax = take((size_t)m.k_rows / 128 * m.dp * 4);
  w.vsum = take(o.smooth_v ? (size_t)m.k_rows / 128 * m.dp * 4 : 0);
  w.vmin = take(o.smooth_v ? (size_t)m.k_rows / 128 * m.dp * 4 : 0);
  w.vinv = take((size_t)m.B * m.Hkv * m.dp * 4);
  w.seqs = take(m.packed ? (size_t)m.B * sizeof(SeqDesc) : 0);
  w.total = off;
  return w;
}

// Extents of every buffer the quantize kernels write, from the pointers already in p.
void set_quant_extents(QuantParams* p, const Dims& m, int pv_mode, const Opts& o) {
  const size_t per_head = (size_t)m.B * m.Hkv * m.dp * 4;
  const size_t part = (size_t)m.k_rows / 128 * m.dp * 4;
  p->x_q8 = extent_of(p->q8, (size_t)m.q_rows * m.dp);
  p->x_qs = extent_of(p->qs, ((size_t)m.q_rows >> o.q_gran_log2) * 4);
  p->x_k8 = extent_of(p->k8, (size_t)m.k_rows * m.dp);
  p->x_ks = extent_of(p->ks, (size_t)m.k_rows / 128 * 4);
  p->x_km = extent_of(p->km, per_head);
  p->x_v8t = extent_of(p->v8t, (size_t)m.k_rows * m.dp * (pv_mode_fp16_operands(pv_mode) ? 2 : 1));
  p->x_vs = extent_of(p->vs, per_head);
  p->x_vm = extent_of(p->vm, per_head);
  p->x_vinv = extent_of(p->vinv, per_head);
  p->x_ksum = extent_of(p->ksum_part, part);
  p->x_vmax = extent_of(p->vmax_part, part);
  p->x_vsum = extent_of(p->vsum_part, part);
  p->x_vmin = extent_of(p->vmin_part, part);
}

QuantParams quant_params(const Dims& m, const void* q, const void* k, const void* v, int dtype, int layout,
                         int pv_mode, const Opts& o) {
  QuantParams p;
  memset(&p, 0, sizeof(p));
  p.q = q, p.k = k, p.v = v;
  p.m = seq_map(m, layout, nullptr);  // packed batches set p.m.seqs once the table exists
  p.nblk_q = m.nblk_q, p.nblk_k = m.nblk_k;
  p.dtype = dtype;
  p.vec_q = (m.d % 8 == 0) && aligned16(q);
  p.vec_k = (m.d % 8 == 0) && aligned16(k);
  p.vec_v = (m.d % 8 == 0) && aligned16(v);
  p.vmax_code = pv_mode == SAGE_PV_FP32 ? 448.0f : 1.0f;
  p.v_fp16 = pv_mode_fp16_operands(pv_mode) ? 1 : 0;
  p.q_gran_log2 = o.q_gran_log2;
  p.smooth_v = o.smooth_v;
  return p;
}

sage_status check_common(const void* q, const void* k, const void* v, int dtype, int layout, int pv_mode) {
  if (!q || !k || !v) return SAGE_ERR_INVALID_ARG;
  sage_status s = check_dtype(dtype);
  if (s != SAGE_OK) return s;
  if (layout != SAGE_HND && layout != SAGE_NHD) return SAGE_ERR_INVALID_ARG;
  if (pv_mode == SAGE_PV16_FP16) return SAGE_ERR_UNSUPPORTED;
  if (!pv_mode_valid(pv_mode)) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

// out must not overlap q, k or v (2-byte elements)
bool out_overlaps(const Dims& m, const void* q, const void* k, const void* v, const void* out) {
  const size_t qbytes = (size_t)m.total_q * m.Hq * m.d * 2, kvbytes = (size_t)m.total_k * m.Hkv * m.d * 2;
  return overlaps(out, qbytes, q, qbytes) || overlaps(out, qbytes, k, kvbytes) || overlaps(out, qbytes, v, kvbytes);
}

// Quantize pass + fused kernel on a workspace laid out by ws_layout(m, pv_mode, o); packed batches
// first build their per-sequence table from cu_q / cu_k.
sage_status attend_on(const Dims& m, unsigned char* ws, const void* q, const void* k, const void* v, void* out,
                      const int32_t* cu_q, const int32_t* cu_k, int dtype, int layout, int causal, float sm_scale,
                      int pv_mode, const Opts& o, cudaStream_t st) {
  const WsLayout w = ws_layout(m, pv_mode, o);
  SeqDesc* seqs = m.packed ? reinterpret_cast<SeqDesc*>(ws + w.seqs) : nullptr;
  if (m.packed) {
    sage_status s = from_cuda(launch_seq_plan(cu_q, cu_k, m.B, m.Nq, m.Nk, m.total_q, m.total_k, seqs, st));
    if (s != SAGE_OK) return s;
  }
  QuantParams qp = quant_params(m, q, k, v, dtype, layout, pv_mode, o);
  qp.m.seqs = seqs;
  QuantBufs qb{seqs,
               reinterpret_cast<float*>(ws + w.vm),
               reinterpret_cast<int8_t*>(ws + w.q8), reinterpret_cast<float*>(ws + w.qs),
               reinterpret_cast<int8_t*>(ws + w.k8), reinterpret_cast<float*>(ws + w.ks),
               reinterpret_cast<float*>(ws + w.km), ws + w.v8t, reinterpret_cast<float*>(ws + w.vs)};
  qp.q8 = qb.q8, qp.qs = qb.qs, qp.k8 = qb.k8, qp.ks = qb.ks, qp.km = qb.km, qp.v8t = qb.v8t, qp.vs = qb.vs;
  qp.vm = qb.vm;
  qp.ksum_part = reinterpret_cast<float*>(ws + w.ksum);
  qp.vmax_part = reinterpret_cast<float*>(ws + w.vmax);
  qp.vsum_part = reinterpret_cast<float*>(ws + w.vsum);
  qp.vmin_part = reinterpret_cast<float*>(ws + w.vmin);
  qp.vinv = reinterpret_cast<float*>(ws + w.vinv);
  set_quant_extents(&qp, m, pv_mode, o);
  sage_status s = from_cuda(launch_quantize(qp, st));
  if (s == SAGE_OK) s = run_fwd(m, qb, out, dtype, layout, causal, sm_scale, pv_mode, o, st);
  return s;
}

// The same, on a workspace taken from the library's pool and released stream-ordered.
sage_status attend_pooled(const Dims& m, const void* q, const void* k, const void* v, void* out, const int32_t* cu_q,
                          const int32_t* cu_k, int dtype, int layout, int causal, float sm_scale, int pv_mode,
                          const Opts& o, cudaStream_t st) {
  const WsLayout w = ws_layout(m, pv_mode, o);
  unsigned char* ws = nullptr;
  cudaError_t e = workspace_alloc(reinterpret_cast<void**>(&ws), w.total, st);
  if (e != cudaSuccess) return from_cuda(e);
  sage_status s = attend_on(m, ws, q, k, v, out, cu_q, cu_k, dtype, layout, causal, sm_scale, pv_mode, o, st);
  const cudaError_t ef = cudaFreeAsync(ws, st);
  if (s == SAGE_OK && ef != cudaSuccess) s = from_cuda(ef);
  return s;
}

}  // namespace

extern "C" {

size_t sage_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  Dims m;
  if (check_dims(B, Hq, Hkv, N, N, d, &m) != SAGE_OK) return 0;
  Opts largest;
  largest.q_gran_log2 = 0, largest.smooth_v = 1;
  return ws_layout(m, SAGE_PV16_FP32, largest).total;  // the largest over the P.V modes and options
}

sage_status sage_attn_ex(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv, int Nq,
                         int Nk, int d, sage_dtype dtype, sage_layout layout, int is_causal, float sm_scale,
                         sage_pv_mode pv_mode, const sage_opts* opts, void* stream) {
  sage_status s = check_common(q, k, v, dtype, layout, pv_mode);
  if (s != SAGE_OK) return s;
  Opts o;
  if ((s = parse_opts(opts, &o)) != SAGE_OK) return s;
  Dims m;
  if ((s = check_dims(B, Hq, Hkv, Nq, Nk, d, &m)) != SAGE_OK) return s;
  if (!out || out_overlaps(m, q, k, v, out)) return SAGE_ERR_INVALID_ARG;
  if ((s = check_device()) != SAGE_OK) return s;
  return attend_pooled(m, q, k, v, out, nullptr, nullptr, dtype, layout, is_causal ? 1 : 0, sm_scale, pv_mode, o,
                       static_cast<cudaStream_t>(stream));
}

sage_status sage_attn(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv, int N, int d,
                      sage_dtype dtype, sage_layout layout, int is_causal, float sm_scale, sage_pv_mode pv_mode,
                      void* stream) {
  return sage_attn_ex(q, k, v, out, B, Hq, Hkv, N, N, d, dtype, layout, is_causal, sm_scale, pv_mode, nullptr,
                      stream);
}

sage_status sage_attn_varlen(const void* q, const void* k, const void* v, void* out, const int32_t* cu_seqlens_q,
                             const int32_t* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k,
                             long long total_q, long long total_k, int Hq, int Hkv, int d, sage_dtype dtype,
                             int is_causal, float sm_scale, sage_pv_mode pv_mode, const sage_opts* opts,
                             void* stream) {
  sage_status s = check_common(q, k, v, dtype, SAGE_NHD, pv_mode);
  if (s != SAGE_OK) return s;
  Opts o;
  if ((s = parse_opts(opts, &o)) != SAGE_OK) return s;
  if (!cu_seqlens_q || !cu_seqlens_k) return SAGE_ERR_INVALID_ARG;
  Dims m;
  if ((s = check_dims_packed(B, Hq, Hkv, max_seqlen_q, max_seqlen_k, total_q, total_k, d, &m)) != SAGE_OK) return s;
  if (!out || out_overlaps(m, q, k, v, out)) return SAGE_ERR_INVALID_ARG;
  if ((s = check_device()) != SAGE_OK) return s;
  return attend_pooled(m, q, k, v, out, cu_seqlens_q, cu_seqlens_k, dtype, SAGE_NHD, is_causal ? 1 : 0, sm_scale,
                       pv_mode, o, static_cast<cudaStream_t>(stream));
}

sage_status sage_quantize(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int N, int d,
                          sage_dtype dtype, sage_layout layout, sage_pv_mode pv_mode, const sage_opts* opts,
                          int8_t* q8, float* qs, int8_t* k8, float* ks, float* km, uint8_t* v8t, float* vs,
                          float* vm, void* stream) {
  sage_status s = check_common(q, k, v, dtype, layout, pv_mode);
  if (s != SAGE_OK) return s;
  Opts o;
  if ((s = parse_opts(opts, &o)) != SAGE_OK) return s;
  Dims m;
  if ((s = check_dims(B, Hq, Hkv, N, N, d, &m)) != SAGE_OK) return s;
  if (!q8 || !qs || !k8 || !ks || !km || !v8t || !vs || (o.smooth_v && !vm)) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8t)) return SAGE_ERR_INVALID_ARG;
  if ((s = check_device()) != SAGE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t part = align_up((size_t)m.k_rows / 128 * m.dp * 4);
  const size_t vinv = align_up((size_t)m.B * m.Hkv * m.dp * 4);
  const int nparts = o.smooth_v ? 4 : 2;
  unsigned char* scratch = nullptr;
  cudaError_t e = workspace_alloc(reinterpret_cast<void**>(&scratch), nparts * part + vinv, st);
  if (e != cudaSuccess) return from_cuda(e);
  QuantParams qp = quant_params(m, q, k, v, dtype, layout, pv_mode, o);
  qp.q8 = q8, qp.qs = qs, qp.k8 = k8, qp.ks = ks, qp.km = km, qp.v8t = v8t, qp.vs = vs, qp.vm = vm;
  qp.ksum_part = reinterpret_cast<float*>(scratch);
  qp.vmax_part = reinterpret_cast<float*>(scratch + part);
  qp.vsum_part = o.smooth_v ? reinterpret_cast<float*>(scratch + 2 * part) : nullptr;
  qp.vmin_part = o.smooth_v ? reinterpret_cast<float*>(scratch + 3 * part) : nullptr;
  qp.vinv = reinterpret_cast<float*>(scratch + nparts * part);
  set_quant_extents(&qp, m, pv_mode, o);
  s = from_cuda(launch_quantize(qp, st));
  const cudaError_t ef = cudaFreeAsync(scratch, st);
  if (s == SAGE_OK && ef != cudaSuccess) s = from_cuda(ef);
  return s;
}

sage_status sage_attn_quantized(const int8_t* q8, const float* qs, const int8_t* k8, const float* ks,
                                const uint8_t* v8t, const float* vs, const float* vm, void* out, int B, int Hq,
                                int Hkv, int N, int d, sage_dtype out_dtype, sage_layout out_layout, int is_causal,
                                float sm_scale, sage_pv_mode pv_mode, const sage_opts* opts, void* stream) {
  if (!q8 || !qs || !k8 || !ks || !v8t || !vs || !out) return SAGE_ERR_INVALID_ARG;
  sage_status s = check_dtype(out_dtype);
  if (s != SAGE_OK) return s;
  if (out_layout != SAGE_HND && out_layout != SAGE_NHD) return SAGE_ERR_INVALID_ARG;
  if (pv_mode == SAGE_PV16_FP16) return SAGE_ERR_UNSUPPORTED;
  if (!pv_mode_valid(pv_mode)) return SAGE_ERR_INVALID_ARG;
  Opts o;
  if ((s = parse_opts(opts, &o)) != SAGE_OK) return s;
  if (o.smooth_v && !vm) return SAGE_ERR_INVALID_ARG;
  Dims m;
  if ((s = check_dims(B, Hq, Hkv, N, N, d, &m)) != SAGE_OK) return s;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8t)) return SAGE_ERR_INVALID_ARG;
  if ((s = check_device()) != SAGE_OK) return s;
  QuantBufs qb{nullptr, const_cast<float*>(vm), const_cast<int8_t*>(q8), const_cast<float*>(qs),
               const_cast<int8_t*>(k8), const_cast<float*>(ks), nullptr, const_cast<uint8_t*>(v8t),
               const_cast<float*>(vs)};
  return run_fwd(m, qb, out, out_dtype, out_layout, is_causal ? 1 : 0, sm_scale, pv_mode, o,
                 static_cast<cudaStream_t>(stream));
}

sage_status sage_qk_int32(const int8_t* q8, const int8_t* k8, int B, int Hq, int Hkv, int N, int d,
                          const int32_t* tiles, int n_tiles, int32_t* s_out, void* stream) {
  if (!q8 || !k8 || !tiles || !s_out || n_tiles < 0) return SAGE_ERR_INVALID_ARG;
  Dims m;
  sage_status s = check_dims(B, Hq, Hkv, N, N, d, &m);
  if (s != SAGE_OK) return s;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(s_out)) return SAGE_ERR_INVALID_ARG;
  if (n_tiles == 0) return SAGE_OK;
  if ((s = check_device()) != SAGE_OK) return s;
  CUtensorMap tq, tk;
  const uint32_t ksub = m.dp >= 128 ? 128 : 64;
  if (!make_map(&tq, q8, m.dp, (uint64_t)m.q_rows, ksub, 128) || !make_map(&tk, k8, m.dp, (uint64_t)m.k_rows, ksub, 128))
    return SAGE_ERR_CUDA;
  QkDumpParams p;
  p.tiles = tiles, p.n_tiles = n_tiles, p.out = s_out;
  p.B = m.B, p.Hq = m.Hq, p.Hkv = m.Hkv, p.Np = (int)m.q_head_rows, p.nblk = m.nblk_q, p.G = m.G;
  return from_cuda(launch_qk_dump(tq, tk, p, m.dp, static_cast<cudaStream_t>(stream)));
}

sage_status sage_mma_probe(int kind, int iters, double* ops, void* stream) {
  if (kind < 0 || kind > 2 || iters < 1 || iters > 1000000 || !ops) return SAGE_ERR_INVALID_ARG;
  sage_status s = check_device();
  if (s != SAGE_OK) return s;
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0)
    return SAGE_ERR_CUDA;
  const double k = kind == 2 ? 16.0 : 32.0;
  *ops = (double)n_sm * iters * 4.0 * 2.0 * 128.0 * 256.0 * k;
  return from_cuda(launch_mma_probe(kind, iters, n_sm, static_cast<cudaStream_t>(stream)));
}

sage_status sage_selftest_wait_timeout(int budget_us, void* stream) {
  if (budget_us < 1 || budget_us > 100000) return SAGE_ERR_INVALID_ARG;
  sage_status s = check_device();
  if (s != SAGE_OK) return s;
  int dev = 0, khz = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess || khz <= 0) return SAGE_ERR_CUDA;
  return from_cuda(launch_wait_probe((long long)budget_us * (khz / 1000), static_cast<cudaStream_t>(stream)));
}

sage_status sage_check_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return SAGE_ERR_CUDA;
  int flags = 0;
  int qflags = 0;
  if (read_clear_device_error(&flags) != cudaSuccess) return SAGE_ERR_CUDA;
  if (read_clear_quant_error(&qflags) != cudaSuccess) return SAGE_ERR_CUDA;
  flags |= qflags;
  if (flags & 1) return SAGE_ERR_TIMEOUT;
  if (flags & SAGE_DEVERR_BOUNDS) return SAGE_ERR_BOUNDS;
  if (flags & 2) return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

const char* sage_status_string(sage_status s) {
  switch (s) {
    case SAGE_OK: return "ok";
    case SAGE_ERR_INVALID_ARG: return "invalid argument";
    case SAGE_ERR_UNSUPPORTED: return "unsupported (inputs must be fp16 or bf16)";
    case SAGE_ERR_ARCH: return "device is not compute capability 10.0 (B200, sm_100a)";
    case SAGE_ERR_CUDA: return "CUDA error";
    case SAGE_ERR_OOM: return "out of device memory";
    case SAGE_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
    case SAGE_ERR_BOUNDS: return "a kernel skipped a store outside its buffer (checked build)";
  }
  return "unknown status";
}

int sage_device_supported(void) { return check_device() == SAGE_OK ? 1 : 0; }

void sage_test_inject(int fake_cc, int fail_allocs) {
  g_fake_cc.store(fake_cc > 0 ? fake_cc : 0);
  g_fail_allocs.store(fail_allocs > 0 ? fail_allocs : 0);
}

void sage_test_out_limit(long long bytes) { g_out_limit.store(bytes > 0 ? bytes : 0); }

int sage_checked_build(void) {
#ifdef SAGE_CHECKED
  return 1;
#else
  return 0;
#endif
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Allocation-free entry point: the workspace is a static device array in this library.
// ------------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[SAGE_NOALLOC_MAX_BYTES];

namespace {

// The array's device address, looked up once per device with that device current.
cudaError_t noalloc_scratch(int dev, unsigned char** out) {
  constexpr int kMaxDevices = 128;
  static std::mutex mu;
  static unsigned char* addr[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" sage_status sage_attn_noalloc(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                                         int Hkv, int N, int d, sage_dtype dtype, sage_layout layout, int is_causal,
                                         float sm_scale, sage_pv_mode pv_mode, void* stream) {
  sage_status s = check_common(q, k, v, dtype, layout, pv_mode);
  if (s != SAGE_OK) return s;
  Dims m;
  if ((s = check_dims(B, Hq, Hkv, N, N, d, &m)) != SAGE_OK) return s;
  if (!out || out_overlaps(m, q, k, v, out)) return SAGE_ERR_INVALID_ARG;
  const Opts o;  // defaults
  const WsLayout w = ws_layout(m, pv_mode, o);
  if (w.total > (size_t)SAGE_NOALLOC_MAX_BYTES) return SAGE_ERR_INVALID_ARG;
  if ((s = check_device()) != SAGE_OK) return s;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  unsigned char* ws = nullptr;
  if (noalloc_scratch(dev, &ws) != cudaSuccess) return SAGE_ERR_CUDA;
  return attend_on(m, ws, q, k, v, out, nullptr, nullptr, dtype, layout, is_causal ? 1 : 0, sm_scale, pv_mode, o,
                   static_cast<cudaStream_t>(stream));
}
