// nsa_api.cu -- the C ABI of libnsa (include/nsa.h): host-side validation,
// workspace layout, TMA descriptor encoding and kernel launches. No entry
// point allocates device or pinned memory; all buffers belong to the caller.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/nsa.h"
#include "nsa_device.cuh"
#include "nsa_kernels.cuh"

namespace {

thread_local std::string g_last_error;

nsa_status fail(nsa_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

nsa_status cuda_fail(cudaError_t e, const char *where) {
  return fail(NSA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
}

#define NSA_CUDA(call)                                         \
  do {                                                         \
    cudaError_t e_ = (call);                                   \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call);        \
  } while (0)

// One error record per device (word 0: error bits, word 1: site code of the
// first timed-out wait); its device address is looked up per device.
__device__ unsigned int g_nsa_error_word[2] = {0u, 0u};

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  unsigned int *err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

nsa_status device_info(DeviceInfo **out) {
  int dev = 0;
  NSA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(NSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp prop;
    NSA_CUDA(cudaGetDeviceProperties(&prop, dev));
    if (prop.major != 10)
      return fail(NSA_ERR_UNSUPPORTED, "libnsa is built for sm_100a; device %d is sm_%d%d", dev, prop.major,
                  prop.minor);
    d.num_sms = prop.multiProcessorCount;
    void *p = nullptr;
    NSA_CUDA(cudaGetSymbolAddress(&p, g_nsa_error_word));
    d.err = static_cast<unsigned int *>(p);
    d.ready = true;
  }
  *out = &d;
  return NSA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

nsa_status get_encoder(PFN_cuTensorMapEncodeTiled_v12000 *fn) {
  std::call_once(g_encode_once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!g_encode) return fail(NSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  *fn = g_encode;
  return NSA_OK;
}

// bf16 (BH, S, D) viewed as 3-D {D, S, BH}; box {64, rows, 1}, 128-byte swizzle.
// Rows past S read as zero.
nsa_status encode_tokens(CUtensorMap *map, const void *ptr, int D, int S, long long BH, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  nsa_status st = get_encoder(&enc);
  if (st != NSA_OK) return st;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return NSA_OK;
}

// float32 (BH, N, D) viewed as 3-D {D, N, BH}; box {32, rows, 1} (128-byte
// rows), 128-byte swizzle. Rows past N read as zero.
nsa_status encode_f32_rows(CUtensorMap *map, const void *ptr, int D, int N, long long BH, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  nsa_status st = get_encoder(&enc);
  if (st != NSA_OK) return st;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)N * D * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NSA_ERR_CUDA, "cuTensorMapEncodeTiled (float32) failed (%d)", (int)r);
  return NSA_OK;
}

inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Geometry {
  int B, Hq, Hkv, Sq, Skv, D;
  int NQ, NK, Hs;
};

nsa_status check_dims(int B, int Hq, int Hkv, int Sq, int Skv, int D) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || D <= 0)
    return fail(NSA_ERR_INVALID_ARG, "sizes must be positive (B=%d Hq=%d Hkv=%d Sq=%d Skv=%d D=%d)", B, Hq, Hkv,
                Sq, Skv, D);
  if (Hq % Hkv != 0) return fail(NSA_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  if (D != 64 && D != 128) return fail(NSA_ERR_UNSUPPORTED, "head dim %d not supported (64 or 128)", D);
  return NSA_OK;
}

nsa_status check_spec(const nsa_spec *spec) {
  if (!spec) return fail(NSA_ERR_INVALID_ARG, "spec is NULL");
  if (!(spec->budget > 0.f && spec->budget <= 1.f))
    return fail(NSA_ERR_INVALID_ARG, "budget %g outside (0, 1]", (double)spec->budget);
  if (spec->block_q <= 0 || spec->block_kv <= 0)
    return fail(NSA_ERR_INVALID_ARG, "block sizes must be positive (%d, %d)", spec->block_q, spec->block_kv);
  return NSA_OK;
}

nsa_status check_mask(const int8_t *m, const int64_t *s, const char *name) {
  if (m && !s) return fail(NSA_ERR_INVALID_ARG, "%s given without strides", name);
  if (m)
    for (int d = 0; d < 4; ++d)
      if (s[d] < 0) return fail(NSA_ERR_INVALID_ARG, "%s stride %d is negative", name, d);
  return NSA_OK;
}

// workspace layouts
// Tensor-core score scratch of the long-row selection (B, Hs, NQ, NKP)
// float32, NKP = NK rounded up to 128; 0 bytes when the rows take another path.
size_t tc_scores_bytes(int B, int Hs, int NQ, int NK, int D) {
  if (!nsa::select_uses_tc_scores(NK, D, 0)) return 0;
  const size_t nkp = (size_t)((NK + 127) / 128 * 128);
  return (size_t)B * Hs * NQ * nkp * 4;
}
// The tf32 hi and lo parts of the scored keys (Hk kv heads: Hkv, or 1 for
// head-shared scoring), two float32 arrays shaped like them.
size_t tc_split_half(int B, int Hk, int NK, int D) { return (size_t)B * Hk * NK * D * 4; }
size_t tc_split_bytes(int B, int Hk, int NK, int D) {
  if (!nsa::select_uses_tc_scores(NK, D, 0)) return 0;
  return 2 * align256(tc_split_half(B, Hk, NK, D));
}

struct ForwardLayout {
  size_t flags, counters, pq, pk, qm, km, count, index, tc, tcsplit, total;
};
ForwardLayout forward_layout(const Geometry &g, bool head_shared) {
  ForwardLayout L;
  size_t off = 0;
  L.flags = off;
  off += 256;
  L.counters = off;  // per kv group, for the single-kernel selection
  off += align256((size_t)g.B * g.Hkv * 4);
  L.pq = off;
  off += align256((size_t)g.B * g.Hq * g.NQ * g.D * 4);
  L.pk = off;
  off += align256((size_t)g.B * g.Hkv * g.NK * g.D * 4);
  L.qm = off;
  off += head_shared ? align256((size_t)g.B * g.NQ * g.D * 4) : 0;
  L.km = off;
  off += head_shared ? align256((size_t)g.B * g.NK * g.D * 4) : 0;
  L.count = off;
  off += align256((size_t)g.B * g.Hs * g.NQ * 4);
  L.index = off;
  off += align256((size_t)g.B * g.Hs * g.NQ * g.NK * 2);
  L.tc = off;
  off += align256(tc_scores_bytes(g.B, g.Hs, g.NQ, g.NK, g.D));
  L.tcsplit = off;
  off += tc_split_bytes(g.B, head_shared ? 1 : g.Hkv, g.NK, g.D);
  L.total = off;
  return L;
}
// nsa_select: flag word, then the head means when head_shared
struct SelectLayout {
  size_t flags, qm, km, tc, tcsplit, total;
};
SelectLayout select_layout(int B, int Hq, int Hkv, int NQ, int NK, int D, bool head_shared) {
  SelectLayout L;
  L.flags = 0;
  L.qm = 256;
  L.km = L.qm + (head_shared ? align256((size_t)B * NQ * D * 4) : 0);
  L.tc = L.km + (head_shared ? align256((size_t)B * NK * D * 4) : 0);
  L.tcsplit = L.tc + align256(tc_scores_bytes(B, head_shared ? 1 : Hq, NQ, NK, D));
  L.total = L.tcsplit + tc_split_bytes(B, head_shared ? 1 : Hkv, NK, D);
  return L;
}
struct AttnLayout {
  size_t count, index, total;
};
AttnLayout attn_layout(int B, int Hs, int NQ, int NK) {
  AttnLayout L;
  L.count = 256;
  L.index = L.count + align256((size_t)B * Hs * NQ * 4);
  L.total = L.index + align256((size_t)B * Hs * NQ * NK * 2);
  return L;
}

// backward workspace: Dv f32 (B,Hq,Sq) | kv lists (count (B,Hs,NQ) int32,
// index (B,Hs,NQ,NK) uint16) | q lists (count (B,Hs,NK) int32, index
// (B,Hs,NK,NQ) uint16); every region 256-byte aligned
struct BwdLayout {
  size_t dvec, kv_count, kv_index, q_count, q_index, total;
};
BwdLayout bwd_layout(int B, int Hq, int Sq, int Hs, int NQ, int NK) {
  BwdLayout L;
  L.dvec = 0;
  L.kv_count = align256((size_t)B * Hq * Sq * 4);
  L.kv_index = L.kv_count + align256((size_t)B * Hs * NQ * 4);
  L.q_count = L.kv_index + align256((size_t)B * Hs * NQ * NK * 2);
  L.q_index = L.q_count + align256((size_t)B * Hs * NK * 4);
  L.total = L.q_index + align256((size_t)B * Hs * NK * NQ * 2);
  return L;
}

// plan buffer: flag word, tile states (Bp,Hp,NQ,NK) int8, candidate counts
// and budget counts (Bp,Hp,NQ) int32
struct PlanLayout {
  int Bp, Hp;
  size_t state, cnt, kpr, total;
};
PlanLayout plan_layout(int B, int Hs, int NQ, int NK, const int64_t *ps, const int64_t *ds) {
  PlanLayout L;
  L.Bp = ((ps && ps[0] != 0) || (ds && ds[0] != 0)) ? B : 1;
  L.Hp = ((ps && ps[1] != 0) || (ds && ds[1] != 0)) ? Hs : 1;
  const size_t rows = (size_t)L.Bp * L.Hp * NQ;
  L.state = 256;
  L.cnt = L.state + align256(rows * NK);
  L.kpr = L.cnt + align256(rows * 4);
  L.total = L.kpr + align256(rows * 4);
  return L;
}

nsa_status check_attn_geometry(int block_q, int block_kv, int NK) {
  if (block_q != 128 || block_kv != 64)
    return fail(NSA_ERR_UNSUPPORTED, "attention supports block_q=128, block_kv=64 (got %d, %d)", block_q,
                block_kv);
  if (NK > 65535) return fail(NSA_ERR_UNSUPPORTED, "NK=%d exceeds 65535 kv tiles", NK);
  return NSA_OK;
}

nsa_status run_attention(const void *q, const void *k, const void *v, const Geometry &g,
                         const int32_t *count, const uint16_t *index, const unsigned int *dense_if_zero,
                         float scale, void *out, float *lse, DeviceInfo *dev, cudaStream_t stream,
                         const int8_t *kmask = nullptr, const int64_t *kmask_strides = nullptr) {
  CUtensorMap tq, tk, tv;
  nsa_status st;
  if ((st = encode_tokens(&tq, q, g.D, g.Sq, (long long)g.B * g.Hq, 128)) != NSA_OK) return st;
  if ((st = encode_tokens(&tk, k, g.D, g.Skv, (long long)g.B * g.Hkv, 64)) != NSA_OK) return st;
  if ((st = encode_tokens(&tv, v, g.D, g.Skv, (long long)g.B * g.Hkv, 64)) != NSA_OK) return st;
  nsa::AttnArgs a;
  a.B = g.B;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.Sq = g.Sq;
  a.Skv = g.Skv;
  a.NQ = g.NQ;
  a.NK = g.NK;
  a.Hs = g.Hs;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  a.kv_count = count;
  a.kv_index = index;
  a.dense_if_zero = dense_if_zero;
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  a.err = dev->err;
  a.kmask = kmask;
  a.q_first = 0;  // chosen by the launcher
  for (int d = 0; d < 3; ++d) a.ks[d] = 0;
  if (kmask) {
    a.ks[0] = kmask_strides ? kmask_strides[0] : (long long)g.Hkv * g.Skv;
    a.ks[1] = kmask_strides ? kmask_strides[1] : (long long)g.Skv;
    a.ks[2] = kmask_strides ? kmask_strides[2] : 1;
  }
  NSA_CUDA(nsa::launch_attn_fwd(a, g.D, dev->num_sms, tq, tk, tv, stream));
  return NSA_OK;
}

// Long rows: the tf32 split of the pooled keys into `split` (tc_split_bytes),
// then the scores (B, Hq, NQ, NKP) of pq (B, Hq, NQ, D) against pk (B, Hkv,
// NK, D) on the tensor cores into `scores`.
nsa_status run_tc_scores(const float *pq, const float *pk, int B, int Hq, int Hkv, int NQ, int NK, int D,
                         float *scores, char *split, DeviceInfo *dev, cudaStream_t s) {
  float *hi = reinterpret_cast<float *>(split);
  float *lo = reinterpret_cast<float *>(split + align256(tc_split_half(B, Hkv, NK, D)));
  NSA_CUDA(nsa::launch_split_tf32(pk, (long long)B * Hkv * NK * D, hi, lo, dev->num_sms, s));
  CUtensorMap thi, tlo;
  nsa_status st;
  const int rows = nsa::score_tc_chunk(B, Hq, NQ, NK, dev->num_sms);
  if ((st = encode_f32_rows(&thi, hi, D, NK, (long long)B * Hkv, rows)) != NSA_OK) return st;
  if ((st = encode_f32_rows(&tlo, lo, D, NK, (long long)B * Hkv, rows)) != NSA_OK) return st;
  const nsa::ScoreTcArgs a = {pq, pk, B, Hq, Hkv, NQ, NK, (int)cdiv(NK, 128) * 128, D, 1, scores, dev->err};
  NSA_CUDA(nsa::launch_score_tc(a, thi, tlo, dev->num_sms, s));
  return NSA_OK;
}

nsa::SelectArgs select_args(const float *pq, const float *pk, const Geometry &g, const nsa_spec *spec,
                            const int8_t *pins, const int64_t *ps, const int8_t *drops, const int64_t *ds) {
  nsa::SelectArgs a = {};
  a.pq = pq;
  a.pk = pk;
  a.B = g.B;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.NQ = g.NQ;
  a.NK = g.NK;
  a.D = g.D;
  a.Hs = g.Hs;
  a.head_shared = spec->head_shared ? 1 : 0;
  a.block_q = spec->block_q;
  a.block_kv = spec->block_kv;
  a.budget = spec->budget;
  a.pins = pins;
  a.drops = drops;
  for (int d = 0; d < 4; ++d) {
    a.ps[d] = pins ? ps[d] : 0;
    a.ds[d] = drops ? ds[d] : 0;
  }
  return a;
}

std::atomic<unsigned long long> g_launches{0};

}  // namespace

void nsa::set_last_error(const char *msg) { g_last_error = msg; }

void nsa::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

extern "C" {

const char *nsa_last_error(void) { return g_last_error.c_str(); }

const char *nsa_version(void) { return "libnsa 0.1 sm_100a"; }

nsa_status nsa_pool(const void *x, int B, int H, int S, int D, int block, float *pooled, nsa_stream_t stream) {
  g_last_error.clear();
  if (!x || !pooled) return fail(NSA_ERR_INVALID_ARG, "nsa_pool: NULL pointer");
  if (B <= 0 || H <= 0 || S <= 0 || block <= 0) return fail(NSA_ERR_INVALID_ARG, "nsa_pool: sizes must be positive");
  if (D != 64 && D != 128) return fail(NSA_ERR_UNSUPPORTED, "nsa_pool: head dim %d not supported", D);
  if (!aligned(x, 16) || !aligned(pooled, 16)) return fail(NSA_ERR_INVALID_ARG, "nsa_pool: pointers must be 16-byte aligned");
  DeviceInfo *dev;
  nsa_status st = device_info(&dev);
  if (st != NSA_OK) return st;
  nsa::PoolSeg a = {static_cast<const __nv_bfloat16 *>(x), pooled, S, block, (int)cdiv(S, block),
                    (long long)B * H * cdiv(S, block)};
  nsa::PoolSeg none = {nullptr, nullptr, 1, 1, 1, 0};
  NSA_CUDA(nsa::launch_pool(a, none, D, dev->num_sms, nullptr, dev->err, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_score(const float *pq, const float *pk, int B, int Hq, int Hkv, int NQ, int NK, int D,
                     int head_shared, float *scores, nsa_stream_t stream) {
  g_last_error.clear();
  if (!pq || !pk || !scores) return fail(NSA_ERR_INVALID_ARG, "nsa_score: NULL pointer");
  nsa_status st = check_dims(B, Hq, Hkv, NQ, NK, D);
  if (st != NSA_OK) return st;
  if (!aligned(pq, 16) || !aligned(pk, 16)) return fail(NSA_ERR_INVALID_ARG, "nsa_score: pooled inputs must be 16-byte aligned");
  Geometry g = {B, Hq, Hkv, 0, 0, D, NQ, NK, head_shared ? 1 : Hq};
  DeviceInfo *dev;
  if ((st = device_info(&dev)) != NSA_OK) return st;
  if (nsa::select_rows_per_cta(B, g.Hs, NQ, NK, dev->num_sms, D, head_shared) == 0)
    return fail(NSA_ERR_UNSUPPORTED, "nsa_score: NK=%d exceeds 8192", NK);
  nsa_spec spec = {1.0f, 1, 1, head_shared, 1};
  nsa::SelectArgs a = select_args(pq, pk, g, &spec, nullptr, nullptr, nullptr, nullptr);
  a.scores_out = scores;
  NSA_CUDA(nsa::launch_select(a, dev->num_sms, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_score_tc(const float *pq, const float *pk, int B, int Hq, int Hkv, int NQ, int NK, int D,
                        float *scores, void *workspace, size_t workspace_bytes, nsa_stream_t stream) {
  g_last_error.clear();
  if (!pq || !pk || !scores || !workspace) return fail(NSA_ERR_INVALID_ARG, "nsa_score_tc: NULL pointer");
  nsa_status st = check_dims(B, Hq, Hkv, NQ, NK, D);
  if (st != NSA_OK) return st;
  if (!aligned(pq, 16) || !aligned(pk, 16) || !aligned(scores, 16) || !aligned(workspace, 256))
    return fail(NSA_ERR_INVALID_ARG, "nsa_score_tc: pq, pk, scores must be 16-byte aligned, workspace 256");
  const size_t need = 2 * align256(tc_split_half(B, Hkv, NK, D));
  if (workspace_bytes < need)
    return fail(NSA_ERR_INVALID_ARG, "nsa_score_tc: workspace needs %zu bytes (got %zu)", need, workspace_bytes);
  DeviceInfo *dev;
  if ((st = device_info(&dev)) != NSA_OK) return st;
  return run_tc_scores(pq, pk, B, Hq, Hkv, NQ, NK, D, scores, static_cast<char *>(workspace), dev,
                       (cudaStream_t)stream);
}

nsa_status nsa_select(const float *pq, const float *pk, int B, int Hq, int Hkv, int NQ, int NK, int D,
                      const nsa_spec *spec, const int8_t *pins, const int64_t *pin_strides, const int8_t *drops,
                      const int64_t *drop_strides, int8_t *keep, int32_t *kv_count, uint16_t *kv_index,
                      int *is_dense, void *workspace, size_t workspace_bytes, nsa_stream_t stream) {
  g_last_error.clear();
  nsa_status st;
  if ((st = check_spec(spec)) != NSA_OK) return st;
  if (!pq || !pk || !keep || !kv_count || !kv_index || !is_dense || !workspace)
    return fail(NSA_ERR_INVALID_ARG, "nsa_select: NULL pointer");
  if ((st = check_dims(B, Hq, Hkv, NQ, NK, D)) != NSA_OK) return st;
  if ((st = check_mask(pins, pin_strides, "pins")) != NSA_OK) return st;
  if ((st = check_mask(drops, drop_strides, "drops")) != NSA_OK) return st;
  if (!aligned(pq, 16) || !aligned(pk, 16) || !aligned(workspace, 256) || !aligned(kv_count, 4) ||
      !aligned(kv_index, 2))
    return fail(NSA_ERR_INVALID_ARG, "nsa_select: misaligned pointer");
  const SelectLayout L = select_layout(B, Hq, Hkv, NQ, NK, D, spec->head_shared != 0);
  if (workspace_bytes < L.total)
    return fail(NSA_ERR_INVALID_ARG, "nsa_select: workspace needs %zu bytes (got %zu)", L.total, workspace_bytes);
  Geometry g = {B, Hq, Hkv, 0, 0, D, NQ, NK, spec->head_shared ? 1 : Hq};
  DeviceInfo *dev;
  if ((st = device_info(&dev)) != NSA_OK) return st;
  if (nsa::select_rows_per_cta(B, g.Hs, NQ, NK, dev->num_sms, D, 0) == 0)
    return fail(NSA_ERR_UNSUPPORTED, "nsa_select: NK=%d exceeds 8192", NK);
  cudaStream_t s = (cudaStream_t)stream;
  char *ws = static_cast<char *>(workspace);
  unsigned int *flag = reinterpret_cast<unsigned int *>(ws + L.flags);
  NSA_CUDA(cudaMemsetAsync(flag, 0, sizeof(unsigned int), s));
  nsa::SelectArgs a = select_args(pq, pk, g, spec, pins, pin_strides, drops, drop_strides);
  if (spec->head_shared) {
    // score on the head means, computed once
    float *qm = reinterpret_cast<float *>(ws + L.qm);
    float *km = reinterpret_cast<float *>(ws + L.km);
    NSA_CUDA(nsa::launch_head_mean(pq, B, Hq, NQ, D, qm, dev->num_sms, s));
    NSA_CUDA(nsa::launch_head_mean(pk, B, Hkv, NK, D, km, dev->num_sms, s));
    a.pq = qm;
    a.pk = km;
    a.Hq = 1;
    a.Hkv = 1;
    a.head_shared = 0;
  }
  a.keep = keep;
  a.kv_count = kv_count;
  a.kv_index = kv_index;
  a.not_covered = flag;
  a.err = dev->err;
  if (tc_scores_bytes(B, g.Hs, NQ, NK, D) > 0) {
    a.tc_scores = reinterpret_cast<float *>(ws + L.tc);
    if ((st = run_tc_scores(a.pq, a.pk, B, a.Hq, a.Hkv, NQ, NK, D, a.tc_scores, ws + L.tcsplit, dev, s)) != NSA_OK)
      return st;
  }
  NSA_CUDA(nsa::launch_select(a, dev->num_sms, s));
  *is_dense = 0;
  if (!spec->force) {
    // the plan's single readback: does any row keep fewer than all candidates?
    unsigned int host_flag = 1;
    NSA_CUDA(cudaMemcpyAsync(&host_flag, flag, sizeof(host_flag), cudaMemcpyDeviceToHost, s));
    NSA_CUDA(cudaStreamSynchronize(s));
    *is_dense = host_flag == 0u ? 1 : 0;
  }
  return NSA_OK;
}

nsa_status nsa_keep_to_index(const int8_t *keep, int B, int Hs, int NQ, int NK, int32_t *kv_count,
                             uint16_t *kv_index, nsa_stream_t stream) {
  g_last_error.clear();
  if (!keep || !kv_count || !kv_index) return fail(NSA_ERR_INVALID_ARG, "nsa_keep_to_index: NULL pointer");
  if (B <= 0 || Hs <= 0 || NQ <= 0 || NK <= 0) return fail(NSA_ERR_INVALID_ARG, "nsa_keep_to_index: sizes must be positive");
  if (NK > 65535) return fail(NSA_ERR_UNSUPPORTED, "nsa_keep_to_index: NK=%d exceeds 65535", NK);
  if (!aligned(kv_count, 4) || !aligned(kv_index, 2)) return fail(NSA_ERR_INVALID_ARG, "nsa_keep_to_index: misaligned output");
  DeviceInfo *dev;
  nsa_status st = device_info(&dev);
  if (st != NSA_OK) return st;
  NSA_CUDA(nsa::launch_keep_to_index(keep, (long long)B * Hs * NQ, NK, kv_count, kv_index, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_block_sparse_attn_fwd(const void *q, const void *k, const void *v, int B, int Hq, int Hkv, int Sq,
                                     int Skv, int D, const int8_t *keep, int Hs, int block_q, int block_kv,
                                     float scale, void *out, float *lse, void *workspace, size_t workspace_bytes,
                                     nsa_stream_t stream) {
  return nsa_block_sparse_attn_fwd_masked(q, k, v, B, Hq, Hkv, Sq, Skv, D, keep, Hs, block_q, block_kv, nullptr,
                                          nullptr, scale, out, lse, workspace, workspace_bytes, stream);
}

nsa_status nsa_block_sparse_attn_fwd_masked(const void *q, const void *k, const void *v, int B, int Hq, int Hkv,
                                            int Sq, int Skv, int D, const int8_t *keep, int Hs, int block_q,
                                            int block_kv, const int8_t *kmask, const int64_t *kmask_strides,
                                            float scale, void *out, float *lse, void *workspace,
                                            size_t workspace_bytes, nsa_stream_t stream) {
  g_last_error.clear();
  nsa_status st;
  if ((st = check_dims(B, Hq, Hkv, Sq, Skv, D)) != NSA_OK) return st;
  if (!q || !k || !v || !out || !lse) return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_fwd: NULL pointer");
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_fwd: scale must be finite and positive");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_fwd: q, k, v, out must be 16-byte aligned");
  const int NQ = (int)cdiv(Sq, 128), NK = (int)cdiv(Skv, 64);
  if ((st = check_attn_geometry(block_q, block_kv, NK)) != NSA_OK) return st;
  if (keep && Hs != 1 && Hs != Hq) return fail(NSA_ERR_INVALID_ARG, "keep heads Hs=%d must be 1 or Hq=%d", Hs, Hq);
  if (kmask_strides && !kmask) return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_fwd: strides without a key mask");
  if (kmask_strides && (kmask_strides[0] < 0 || kmask_strides[1] < 0 || kmask_strides[2] < 0))
    return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_fwd: key mask strides must be non-negative");
  Geometry g = {B, Hq, Hkv, Sq, Skv, D, NQ, NK, keep ? Hs : 1};
  DeviceInfo *dev;
  if ((st = device_info(&dev)) != NSA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int32_t *count = nullptr;
  const uint16_t *index = nullptr;
  if (keep) {
    AttnLayout L = attn_layout(B, g.Hs, NQ, NK);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.total)
      return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_fwd: workspace needs %zu bytes, 256-byte aligned",
                  L.total);
    char *ws = static_cast<char *>(workspace);
    int32_t *c = reinterpret_cast<int32_t *>(ws + L.count);
    uint16_t *ix = reinterpret_cast<uint16_t *>(ws + L.index);
    NSA_CUDA(nsa::launch_keep_to_index(keep, (long long)B * g.Hs * NQ, NK, c, ix, s));
    count = c;
    index = ix;
  }
  return run_attention(q, k, v, g, count, index, nullptr, scale, out, lse, dev, s, kmask, kmask_strides);
}

}  // extern "C"

namespace {

// A built plan as nsa_forward_plan reads it.
struct PlanView {
  const int8_t *state;
  const int32_t *kpr;
  long long bs, hs;  // row strides per batch / keep head (0 = broadcast)
  bool covers;
};

// The whole path (nsa_forward, nsa_forward_timed, nsa_forward_plan).
nsa_status forward_impl(const void *q, const void *k, const void *v, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                        const nsa_spec *spec, const int8_t *pins, const int64_t *pin_strides, const int8_t *drops,
                        const int64_t *drop_strides, const PlanView *plan, float scale, void *out, float *lse,
                        int8_t *keep_out, void *workspace, size_t workspace_bytes, void *const *events,
                        nsa_stream_t stream) {
  g_last_error.clear();
  nsa_status st;
  if ((st = check_spec(spec)) != NSA_OK) return st;
  if ((st = check_dims(B, Hq, Hkv, Sq, Skv, D)) != NSA_OK) return st;
  if (!q || !k || !v || !out || !lse || !workspace) return fail(NSA_ERR_INVALID_ARG, "nsa_forward: NULL pointer");
  if ((st = check_mask(pins, pin_strides, "pins")) != NSA_OK) return st;
  if ((st = check_mask(drops, drop_strides, "drops")) != NSA_OK) return st;
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(NSA_ERR_INVALID_ARG, "nsa_forward: scale must be finite and positive");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
      !aligned(workspace, 256))
    return fail(NSA_ERR_INVALID_ARG, "nsa_forward: misaligned pointer");
  const int NQ = (int)cdiv(Sq, spec->block_q), NK = (int)cdiv(Skv, spec->block_kv);
  if ((st = check_attn_geometry(spec->block_q, spec->block_kv, NK)) != NSA_OK) return st;
  Geometry g = {B, Hq, Hkv, Sq, Skv, D, NQ, NK, spec->head_shared ? 1 : Hq};
  ForwardLayout L = forward_layout(g, spec->head_shared != 0);
  if (workspace_bytes < L.total)
    return fail(NSA_ERR_INVALID_ARG, "nsa_forward: workspace needs %zu bytes (got %zu)", L.total, workspace_bytes);
  DeviceInfo *dev;
  if ((st = device_info(&dev)) != NSA_OK) return st;
  if (nsa::select_rows_per_cta(B, g.Hs, NQ, NK, dev->num_sms, D, 0) == 0)
    return fail(NSA_ERR_UNSUPPORTED, "nsa_forward: NK=%d exceeds 8192", NK);
  cudaStream_t s = (cudaStream_t)stream;
  char *ws = static_cast<char *>(workspace);
  unsigned int *flag = reinterpret_cast<unsigned int *>(ws + L.flags);
  float *pq = reinterpret_cast<float *>(ws + L.pq);
  float *pk = reinterpret_cast<float *>(ws + L.pk);
  int32_t *count = reinterpret_cast<int32_t *>(ws + L.count);
  uint16_t *index = reinterpret_cast<uint16_t *>(ws + L.index);

  auto mark = [&](int e) -> cudaError_t {
    return (events && events[e]) ? cudaEventRecord(static_cast<cudaEvent_t>(events[e]), s) : cudaSuccess;
  };
  NSA_CUDA(mark(0));
  if (plan && plan->covers && !spec->force) {
    // the plan says every row keeps all its candidates: attend densely with
    // drops ignored (the page's None), no scoring at all
    NSA_CUDA(mark(1));
    NSA_CUDA(mark(2));
    st = run_attention(q, k, v, g, nullptr, nullptr, nullptr, scale, out, lse, dev, s);
    if (st != NSA_OK) return st;
    NSA_CUDA(mark(3));
    return NSA_OK;
  }
  // 1. pooling. Per-head scoring with the pooled keys of a head resident in
  //    shared memory: the select kernel pools its query tiles itself, and,
  //    when its grid fits on the device at once, the kv groups' keys too (one
  //    cooperative kernel for the whole selection; the flag and the group
  //    counters are cleared first). Otherwise pool_kernel pools k (and q),
  //    clearing the flag.
  const bool fuse_q = !spec->head_shared && nsa::select_pools_q(NK, D, 0);
  nsa::SelectArgs a = select_args(pq, pk, g, spec, pins, pin_strides, drops, drop_strides);
  if (fuse_q) {
    a.q_raw = static_cast<const __nv_bfloat16 *>(q);
    a.Sq = Sq;
  }
  const bool fuse_k = fuse_q && nsa::select_pools_k(a, dev->num_sms);
  if (fuse_k) {
    unsigned int *counters = reinterpret_cast<unsigned int *>(ws + L.counters);
    NSA_CUDA(cudaMemsetAsync(ws + L.flags, 0, L.pq - L.flags, s));
    a.k_raw = static_cast<const __nv_bfloat16 *>(k);
    a.Skv = Skv;
    a.pk_out = pk;
    a.group_count = counters;
    a.err = dev->err;
  } else {
    nsa::PoolSeg sq = {static_cast<const __nv_bfloat16 *>(q), pq, Sq, spec->block_q, NQ, (long long)B * Hq * NQ};
    nsa::PoolSeg sk = {static_cast<const __nv_bfloat16 *>(k), pk, Skv, spec->block_kv, NK, (long long)B * Hkv * NK};
    nsa::PoolSeg none = {nullptr, nullptr, 1, 1, 1, 0};
    NSA_CUDA(nsa::launch_pool(fuse_q ? sk : sq, fuse_q ? none : sk, D, dev->num_sms, flag, dev->err, s));
  }
  NSA_CUDA(mark(1));
  // 2. fused score + plan + top-k keep + compacted lists
  if (spec->head_shared) {
    float *qm = reinterpret_cast<float *>(ws + L.qm);
    float *km = reinterpret_cast<float *>(ws + L.km);
    NSA_CUDA(nsa::launch_head_mean(pq, B, Hq, NQ, D, qm, dev->num_sms, s));
    NSA_CUDA(nsa::launch_head_mean(pk, B, Hkv, NK, D, km, dev->num_sms, s));
    a.pq = qm;
    a.pk = km;
    a.Hq = 1;
    a.Hkv = 1;
    a.head_shared = 0;
  }
  if (plan) {
    a.plan_state = plan->state;
    a.plan_k = plan->kpr;
    a.plan_bs = plan->bs;
    a.plan_hs = plan->hs;
    a.pins = nullptr;
    a.drops = nullptr;
  }
  a.keep = keep_out;
  a.kv_count = count;
  a.kv_index = index;
  a.not_covered = plan ? nullptr : flag;
  a.err = dev->err;
  if (tc_scores_bytes(B, g.Hs, NQ, NK, D) > 0) {
    a.tc_scores = reinterpret_cast<float *>(ws + L.tc);
    if ((st = run_tc_scores(a.pq, a.pk, B, a.Hq, a.Hkv, NQ, NK, D, a.tc_scores, ws + L.tcsplit, dev, s)) != NSA_OK)
      return st;
  }
  NSA_CUDA(nsa::launch_select(a, dev->num_sms, s));
  NSA_CUDA(mark(2));
  // 3. attention over kept tiles; without a plan, dense when the device flag
  //    says the selection covered everything and force is off
  st = run_attention(q, k, v, g, count, index, (plan || spec->force) ? nullptr : flag, scale, out, lse, dev, s);
  if (st != NSA_OK) return st;
  NSA_CUDA(mark(3));
  return NSA_OK;
}

}  // namespace

extern "C" {

nsa_status nsa_forward_timed(const void *q, const void *k, const void *v, int B, int Hq, int Hkv, int Sq, int Skv,
                             int D, const nsa_spec *spec, const int8_t *pins, const int64_t *pin_strides,
                             const int8_t *drops, const int64_t *drop_strides, float scale, void *out, float *lse,
                             int8_t *keep_out, void *workspace, size_t workspace_bytes, void *const *events,
                             nsa_stream_t stream) {
  return forward_impl(q, k, v, B, Hq, Hkv, Sq, Skv, D, spec, pins, pin_strides, drops, drop_strides, nullptr, scale,
                      out, lse, keep_out, workspace, workspace_bytes, events, stream);
}

nsa_status nsa_forward(const void *q, const void *k, const void *v, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                       const nsa_spec *spec, const int8_t *pins, const int64_t *pin_strides, const int8_t *drops,
                       const int64_t *drop_strides, float scale, void *out, float *lse, int8_t *keep_out,
                       void *workspace, size_t workspace_bytes, nsa_stream_t stream) {
  return nsa_forward_timed(q, k, v, B, Hq, Hkv, Sq, Skv, D, spec, pins, pin_strides, drops, drop_strides, scale, out,
                           lse, keep_out, workspace, workspace_bytes, nullptr, stream);
}

size_t nsa_workspace_bytes(int B, int Hq, int Hkv, int Sq, int Skv, int D, const nsa_spec *spec) {
  if (!spec || B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || D <= 0 || spec->block_q <= 0 ||
      spec->block_kv <= 0)
    return 0;
  const int NQ = (int)cdiv(Sq, spec->block_q), NK = (int)cdiv(Skv, spec->block_kv);
  const bool hs = spec->head_shared != 0;
  Geometry g = {B, Hq, Hkv, Sq, Skv, D, NQ, NK, hs ? 1 : Hq};
  size_t f = forward_layout(g, hs).total;
  const size_t sel = select_layout(B, Hq, Hkv, NQ, NK, D, hs).total;
  const int NQa = (int)cdiv(Sq, 128), NKa = (int)cdiv(Skv, 64);
  const size_t at = attn_layout(B, Hq, NQa, NKa).total;
  if (sel > f) f = sel;
  return f > at ? f : at;
}

size_t nsa_bwd_workspace_bytes(int B, int Hq, int Hkv, int Sq, int Skv, int D, int Hs) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || D <= 0 || (Hs != 1 && Hs != Hq)) return 0;
  return bwd_layout(B, Hq, Sq, Hs, (int)cdiv(Sq, 128), (int)cdiv(Skv, 64)).total;
}

nsa_status nsa_block_sparse_attn_bwd(const void *q, const void *k, const void *v, const void *out,
                                     const float *lse, const void *dout, int B, int Hq, int Hkv, int Sq, int Skv,
                                     int D, const int8_t *keep, int Hs, int block_q, int block_kv, float scale,
                                     void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                                     nsa_stream_t stream) {
  return nsa_block_sparse_attn_bwd_masked(q, k, v, out, lse, dout, B, Hq, Hkv, Sq, Skv, D, keep, Hs, block_q,
                                          block_kv, nullptr, nullptr, scale, dq, dk, dv, workspace, workspace_bytes,
                                          stream);
}

nsa_status nsa_block_sparse_attn_bwd_masked(const void *q, const void *k, const void *v, const void *out,
                                            const float *lse, const void *dout, int B, int Hq, int Hkv, int Sq,
                                            int Skv, int D, const int8_t *keep, int Hs, int block_q, int block_kv,
                                            const int8_t *kmask, const int64_t *kmask_strides, float scale, void *dq,
                                            void *dk, void *dv, void *workspace, size_t workspace_bytes,
                                            nsa_stream_t stream) {
  g_last_error.clear();
  nsa_status st;
  if ((st = check_dims(B, Hq, Hkv, Sq, Skv, D)) != NSA_OK) return st;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv)
    return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_bwd: NULL pointer");
  if (!std::isfinite(scale) || !(scale > 0.f))
    return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_bwd: scale must be finite and positive");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 2) || !aligned(dv, 2) || !aligned(lse, 4))
    return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_bwd: q, k, v, out, dout, dq must be 16-byte aligned");
  const int NQ = (int)cdiv(Sq, 128), NK = (int)cdiv(Skv, 64);
  if ((st = check_attn_geometry(block_q, block_kv, NK)) != NSA_OK) return st;
  if (NQ > 65535) return fail(NSA_ERR_UNSUPPORTED, "NQ=%d exceeds 65535 query tiles", NQ);
  if (keep && Hs != 1 && Hs != Hq) return fail(NSA_ERR_INVALID_ARG, "keep heads Hs=%d must be 1 or Hq=%d", Hs, Hq);
  if (kmask_strides && !kmask) return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_bwd: strides without a key mask");
  if (kmask_strides && (kmask_strides[0] < 0 || kmask_strides[1] < 0 || kmask_strides[2] < 0))
    return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_bwd: key mask strides must be non-negative");
  const int hs = keep ? Hs : 1;
  const BwdLayout L = bwd_layout(B, Hq, Sq, hs, NQ, NK);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.total)
    return fail(NSA_ERR_INVALID_ARG, "nsa_block_sparse_attn_bwd: workspace needs %zu bytes, 256-byte aligned",
                L.total);
  DeviceInfo *dev;
  if ((st = device_info(&dev)) != NSA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  char *ws = static_cast<char *>(workspace);
  CUtensorMap tq, tdo, tk, tv;
  if ((st = encode_tokens(&tq, q, D, Sq, (long long)B * Hq, 128)) != NSA_OK) return st;
  if ((st = encode_tokens(&tdo, dout, D, Sq, (long long)B * Hq, 128)) != NSA_OK) return st;
  if ((st = encode_tokens(&tk, k, D, Skv, (long long)B * Hkv, 64)) != NSA_OK) return st;
  if ((st = encode_tokens(&tv, v, D, Skv, (long long)B * Hkv, 64)) != NSA_OK) return st;
  nsa::AttnBwdArgs a = {};
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Sq = Sq;
  a.Skv = Skv;
  a.NQ = NQ;
  a.NK = NK;
  a.Hs = hs;
  a.scale = scale;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  a.lse = lse;
  a.dvec = reinterpret_cast<float *>(ws + L.dvec);
  if (keep) {
    int32_t *kc = reinterpret_cast<int32_t *>(ws + L.kv_count);
    uint16_t *ki = reinterpret_cast<uint16_t *>(ws + L.kv_index);
    NSA_CUDA(nsa::launch_keep_to_index(keep, (long long)B * hs * NQ, NK, kc, ki, s));
    a.kv_count = kc;
    a.kv_index = ki;
    a.q_count = reinterpret_cast<int32_t *>(ws + L.q_count);
    a.q_index = reinterpret_cast<uint16_t *>(ws + L.q_index);
  }
  a.dq = static_cast<__nv_bfloat16 *>(dq);
  a.dk = static_cast<__nv_bfloat16 *>(dk);
  a.dv = static_cast<__nv_bfloat16 *>(dv);
  a.err = dev->err;
  a.kmask = kmask;
  if (kmask) {
    a.ks[0] = kmask_strides ? kmask_strides[0] : (long long)Hkv * Skv;
    a.ks[1] = kmask_strides ? kmask_strides[1] : (long long)Skv;
    a.ks[2] = kmask_strides ? kmask_strides[2] : 1;
  }
  NSA_CUDA(nsa::launch_attn_bwd(a, D, static_cast<const __nv_bfloat16 *>(out),
                                static_cast<const __nv_bfloat16 *>(dout), keep, dev->num_sms, tq, tdo, tk, tv, s));
  return NSA_OK;
}

unsigned long long nsa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

nsa_status nsa_selftest_timeout(int which, long long limit_cycles, nsa_stream_t stream) {
  g_last_error.clear();
  if (which != 0 && which != 1) return fail(NSA_ERR_INVALID_ARG, "nsa_selftest_timeout: which must be 0 or 1");
  if (limit_cycles < 1 || limit_cycles > nsa::kWaitLimitCycles)
    return fail(NSA_ERR_INVALID_ARG, "nsa_selftest_timeout: limit_cycles must be in [1, %lld]",
                nsa::kWaitLimitCycles);
  DeviceInfo *dev;
  nsa_status st = device_info(&dev);
  if (st != NSA_OK) return st;
  NSA_CUDA(nsa::launch_selftest_wait(which, limit_cycles, dev->err, (cudaStream_t)stream));
  return NSA_OK;
}

nsa_status nsa_device_status(int clear) {
  g_last_error.clear();
  DeviceInfo *dev;
  nsa_status st = device_info(&dev);
  if (st != NSA_OK) return st;
  NSA_CUDA(cudaDeviceSynchronize());
  unsigned int word[2] = {0u, 0u};
  NSA_CUDA(cudaMemcpy(word, dev->err, sizeof(word), cudaMemcpyDeviceToHost));
  if (clear) NSA_CUDA(cudaMemset(dev->err, 0, sizeof(word)));
  if (word[0] & 1u)
    return fail(NSA_ERR_TIMEOUT, "a device-side bounded wait timed out (error word 0x%x, wait site %u)", word[0],
                word[1]);
  if (word[0]) return fail(NSA_ERR_CUDA, "device error word 0x%x (shared-memory layout check failed)", word[0]);
  return NSA_OK;
}

nsa_status nsa_forward_plan(const void *q, const void *k, const void *v, int B, int Hq, int Hkv, int Sq, int Skv,
                            int D, const nsa_spec *spec, const void *plan, const nsa_plan_info *info, float scale,
                            void *out, float *lse, int8_t *keep_out, void *workspace, size_t workspace_bytes,
                            nsa_stream_t stream) {
  g_last_error.clear();
  nsa_status st;
  if ((st = check_spec(spec)) != NSA_OK) return st;
  if ((st = check_dims(B, Hq, Hkv, Sq, Skv, D)) != NSA_OK) return st;
  if (!plan || !info) return fail(NSA_ERR_INVALID_ARG, "nsa_forward_plan: NULL plan or plan info");
  if (!aligned(plan, 256)) return fail(NSA_ERR_INVALID_ARG, "nsa_forward_plan: plan must be 256-byte aligned");
  const int NQ = (int)cdiv(Sq, spec->block_q), NK = (int)cdiv(Skv, spec->block_kv);
  const int Hs = spec->head_shared ? 1 : Hq;
  if (!(info->batches == 1 || info->batches == B) || !(info->heads == 1 || info->heads == Hs))
    return fail(NSA_ERR_INVALID_ARG, "nsa_forward_plan: plan extents (%d, %d) do not match B=%d, keep heads=%d",
                info->batches, info->heads, B, Hs);
  const int64_t bs_probe[4] = {info->batches > 1 ? 1 : 0, info->heads > 1 ? 1 : 0, 0, 0};
  PlanLayout L = plan_layout(B, Hs, NQ, NK, bs_probe, nullptr);
  const char *base = static_cast<const char *>(plan);
  PlanView pv;
  pv.state = reinterpret_cast<const int8_t *>(base + L.state);
  pv.kpr = reinterpret_cast<const int32_t *>(base + L.kpr);
  pv.bs = info->batches > 1 ? (long long)info->heads * NQ : 0;
  pv.hs = info->heads > 1 ? NQ : 0;
  pv.covers = info->covers_everything != 0;
  return forward_impl(q, k, v, B, Hq, Hkv, Sq, Skv, D, spec, nullptr, nullptr, nullptr, nullptr, &pv, scale, out,
                      lse, keep_out, workspace, workspace_bytes, nullptr, stream);
}

size_t nsa_plan_bytes(int B, int Hq, int Sq, int Skv, const nsa_spec *spec, const int64_t *pin_strides,
                      const int64_t *drop_strides) {
  if (B <= 0 || Hq <= 0 || Sq <= 0 || Skv <= 0 || !spec || spec->block_q <= 0 || spec->block_kv <= 0) return 0;
  const int NQ = (int)cdiv(Sq, spec->block_q), NK = (int)cdiv(Skv, spec->block_kv);
  return plan_layout(B, spec->head_shared ? 1 : Hq, NQ, NK, pin_strides, drop_strides).total;
}

nsa_status nsa_plan_build(int B, int Hq, int Sq, int Skv, const nsa_spec *spec, const int8_t *pins,
                          const int64_t *pin_strides, const int8_t *drops, const int64_t *drop_strides, void *plan,
                          size_t plan_bytes, nsa_plan_info *info, nsa_stream_t stream) {
  g_last_error.clear();
  nsa_status st;
  if ((st = check_spec(spec)) != NSA_OK) return st;
  if (B <= 0 || Hq <= 0 || Sq <= 0 || Skv <= 0)
    return fail(NSA_ERR_INVALID_ARG, "nsa_plan_build: sizes must be positive");
  if (!plan || !info) return fail(NSA_ERR_INVALID_ARG, "nsa_plan_build: NULL plan or plan info");
  if (!aligned(plan, 256)) return fail(NSA_ERR_INVALID_ARG, "nsa_plan_build: plan must be 256-byte aligned");
  if ((st = check_mask(pins, pin_strides, "pins")) != NSA_OK) return st;
  if ((st = check_mask(drops, drop_strides, "drops")) != NSA_OK) return st;
  const int NQ = (int)cdiv(Sq, spec->block_q), NK = (int)cdiv(Skv, spec->block_kv);
  const int Hs = spec->head_shared ? 1 : Hq;
  PlanLayout L = plan_layout(B, Hs, NQ, NK, pins ? pin_strides : nullptr, drops ? drop_strides : nullptr);
  if (plan_bytes < L.total)
    return fail(NSA_ERR_INVALID_ARG, "nsa_plan_build: plan needs %zu bytes (got %zu)", L.total, plan_bytes);
  DeviceInfo *dev;
  if ((st = device_info(&dev)) != NSA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  char *base = static_cast<char *>(plan);
  unsigned int *flag = reinterpret_cast<unsigned int *>(base);
  nsa::PlanArgs p = {};
  p.Bp = L.Bp;
  p.Hp = L.Hp;
  p.NQ = NQ;
  p.NK = NK;
  p.block_q = spec->block_q;
  p.block_kv = spec->block_kv;
  p.budget = spec->budget;
  p.pins = pins;
  p.drops = drops;
  for (int d = 0; d < 4; ++d) {
    p.ps[d] = pins ? pin_strides[d] : 0;
    p.ds[d] = drops ? drop_strides[d] : 0;
  }
  p.state = reinterpret_cast<int8_t *>(base + L.state);
  p.cnt = reinterpret_cast<int32_t *>(base + L.cnt);
  p.kpr = reinterpret_cast<int32_t *>(base + L.kpr);
  p.not_covered = flag;
  NSA_CUDA(cudaMemsetAsync(flag, 0, sizeof(unsigned int), s));
  NSA_CUDA(nsa::launch_plan_build(p, dev->num_sms, s));
  // covers_everything: the page's one readback, amortised over every step
  // that reuses the plan
  unsigned int not_covered = 0;
  NSA_CUDA(cudaMemcpyAsync(&not_covered, flag, sizeof(not_covered), cudaMemcpyDeviceToHost, s));
  NSA_CUDA(cudaStreamSynchronize(s));
  info->batches = L.Bp;
  info->heads = L.Hp;
  info->covers_everything = not_covered ? 0 : 1;
  info->reserved = 0;
  return NSA_OK;
}

nsa_status nsa_schedule(int steps, double budget, double bump, int bump_steps, double *budgets) {
  g_last_error.clear();
  if (steps < 0) return fail(NSA_ERR_INVALID_ARG, "nsa_schedule: steps %d is negative", steps);
  if (steps > 0 && !budgets) return fail(NSA_ERR_INVALID_ARG, "nsa_schedule: budgets is NULL");
  if (!std::isfinite(budget) || !std::isfinite(bump))
    return fail(NSA_ERR_INVALID_ARG, "nsa_schedule: budget and bump must be finite");
  if (bump <= 0 || bump_steps <= 0 || steps <= 0) {
    for (int i = 0; i < steps; ++i) budgets[i] = budget;
    return NSA_OK;
  }
  const double raised = std::fmin(1.0, budget + bump);
  const int half = (steps + 1) / 2;  // ceil(steps / 2)
  const int edge = bump_steps < half ? bump_steps : half;
  for (int i = 0; i < steps; ++i) budgets[i] = (i < edge || i >= steps - edge) ? raised : budget;
  return NSA_OK;
}

nsa_status nsa_radial_blocks(int B, int Sq, int Skv, double density, const nsa_spec *spec, double *width,
                             int8_t *keep, int32_t *kv_count, uint16_t *kv_index, nsa_stream_t stream) {
  g_last_error.clear();
  if (!spec) return fail(NSA_ERR_INVALID_ARG, "nsa_radial_blocks: spec is NULL");
  if (B <= 0 || Sq <= 0 || Skv <= 0 || spec->block_q <= 0 || spec->block_kv <= 0)
    return fail(NSA_ERR_INVALID_ARG, "nsa_radial_blocks: sizes and block sizes must be positive");
  if (!std::isfinite(density)) return fail(NSA_ERR_INVALID_ARG, "nsa_radial_blocks: density must be finite");
  if (!width) return fail(NSA_ERR_INVALID_ARG, "nsa_radial_blocks: width is NULL");
  if (!aligned(width, 8)) return fail(NSA_ERR_INVALID_ARG, "nsa_radial_blocks: width must be 8-byte aligned");
  const long long NQ = cdiv(Sq, spec->block_q), NK = cdiv(Skv, spec->block_kv);
  if (NK > 65535) return fail(NSA_ERR_UNSUPPORTED, "nsa_radial_blocks: NK=%lld exceeds 65535", NK);
  if (NQ * NK >= (1ll << 24))
    return fail(NSA_ERR_UNSUPPORTED, "nsa_radial_blocks: %lld tiles; the float32 fraction is exact below 2^24",
                NQ * NK);
  DeviceInfo *dev;
  nsa_status st;
  if ((st = device_info(&dev)) != NSA_OK) return st;
  nsa::RadialArgs r;
  r.B = B;
  r.Sq = Sq;
  r.Skv = Skv;
  r.NQ = (int)NQ;
  r.NK = (int)NK;
  r.block_q = spec->block_q;
  r.block_kv = spec->block_kv;
  r.density = density;
  r.width = width;
  r.keep = keep;
  r.kv_count = kv_count;
  r.kv_index = kv_index;
  NSA_CUDA(nsa::launch_radial(r, dev->num_sms, (cudaStream_t)stream));
  return NSA_OK;
}

}  // extern "C"
