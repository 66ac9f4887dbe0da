// nsa_kernels.cuh -- internal interface between the C ABI layer (nsa_api.cu)
// and the kernels (pool.cu, select.cu, attn_fwd.cu).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace nsa {

// Counts one kernel launched by the library (nsa_kernel_launches()).
void note_launch();

// Launches `kernel` on `stream` with programmatic stream serialization, so it
// can be scheduled while the previous kernel on the stream drains; the kernel
// calls pdl_wait() before touching its predecessor's outputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) note_launch();
  return e;
}

// One tensor to pool: x (BH, S, D) bf16 -> out (BH, ntiles, D) f32.
struct PoolSeg {
  const __nv_bfloat16 *x;
  float *out;
  int S;
  int block;
  int ntiles;             // ceil(S / block)
  long long total_tiles;  // BH * ntiles (0 = segment unused)
};

// clear_word (nullable): a device word the launch sets to 0 before any later
// kernel on the stream runs. err: the library's device error word (timeouts).
// Every x must be 16-byte aligned (tiles are moved with bulk copies).
cudaError_t launch_pool(const PoolSeg &a, const PoolSeg &b, int D, int num_sms, unsigned int *clear_word,
                        unsigned int *err, cudaStream_t stream);

// Fused score + plan + top-k keep over pooled tensors.
struct SelectArgs {
  const float *pq;  // (B, Hq, NQ, D)
  const float *pk;  // (B, Hkv, NK, D)
  int B, Hq, Hkv, NQ, NK, D;
  int Hs;           // keep heads: 1 if head_shared else Hq
  int head_shared;
  int block_q, block_kv;
  float budget;
  const int8_t *pins;
  long long ps[4];
  const int8_t *drops;
  long long ds[4];
  int8_t *keep;            // (B, Hs, NQ, NK) or null
  int32_t *kv_count;       // (B, Hs, NQ) or null
  uint16_t *kv_index;      // (B, Hs, NQ, NK) or null
  unsigned int *not_covered;  // set to 1 when some row keeps fewer than all its candidates
  float *scores_out;       // when set: write raw scores (B, Hs, NQ, NK) and skip selection
  // when set (per-head scoring with every pooled key row of a head resident
  // in shared memory, select_pools_q): the select kernel pools its query
  // tiles itself from q (B, Hq, Sq, D) bf16 and pq is not read
  const __nv_bfloat16 *q_raw;
  int Sq;
  // when also set (q_raw path, cooperative launch): the select CTAs pool k
  // themselves. The CTAs of a kv group (its query heads x query-tile blocks)
  // split the group's kv tiles, write the pooled rows to pk_out, count
  // themselves in group_count[b * Hkv + hk] (zero before the launch) and wait
  // (bounded) until the whole group has done so.
  const __nv_bfloat16 *k_raw;
  int Skv;
  float *pk_out;
  unsigned int *group_count;
  unsigned int *err;
  // when set (a plan built by launch_plan_build): per-tile state (0 =
  // candidate, 1 = kept, 2 = forbidden) and per-row budget count replace the
  // diagonal, pins, drops and budget; element strides over (batch, keep head)
  // are 0 where the plan is broadcast
  const int8_t *plan_state;
  const int32_t *plan_k;
  long long plan_bs, plan_hs;  // tile-row strides (rows of NK) per batch / head
  // when set (rows whose pooled keys do not fit beside the scoring CTA):
  // the scores were computed on the tensor cores (launch_score_tc) into this
  // scratch, (B, Hs, NQ, NKP) float32 with NKP = NK rounded up to 128, and
  // the top-k reads them from there
  float *tc_scores;
};

// Pooled scores on the tensor cores (score_tc.cu): scores (B, Hq, NQ, NKP)
// = pq (B, Hq, NQ, D) . pk (B, Hkv, NK, D)^T, query head h against kv head
// h / (Hq / Hkv); columns from NK up to NKP hold zeros. The keys come as
// their tf32 hi and lo parts (launch_split_tf32), read through the tensor
// maps thi / tlo: {D, NK, B*Hkv} float32, boxes {32, score_tc_chunk(..), 1},
// 128-byte swizzle.
struct ScoreTcArgs {
  const float *pq;
  const float *pk;
  int B, Hq, Hkv, NQ, NK, NKP, D;
  int nsplit;  // set by the launcher
  float *scores;
  unsigned int *err;
};
cudaError_t launch_score_tc(ScoreTcArgs a, const CUtensorMap &thi, const CUtensorMap &tlo, int num_sms,
                            cudaStream_t stream);
// The kv tiles per chunk (the MMA's N, 256 or 64) launch_score_tc uses for
// these sizes; the tensor maps' boxes must have that many rows.
int score_tc_chunk(int B, int Hq, int NQ, int NK, int num_sms);
size_t score_tc_smem(int D);
// hi = tf32(x), lo = tf32(x - hi) elementwise (n a multiple of 4, 16-byte
// aligned arrays).
cudaError_t launch_split_tf32(const float *x, long long n, float *hi, float *lo, int num_sms, cudaStream_t stream);
// True when launch_select computes the scores of these rows on the tensor
// cores (given a scratch): the pooled keys of a head do not fit in the
// resident path and the row fits the register top-k (NK <= 2048).
bool select_uses_tc_scores(int NK, int D, int head_shared);

// Plan build (selection_plan): rows (Bp, Hp, NQ) of the broadcast extent of
// the pin/drop masks.
struct PlanArgs {
  int Bp, Hp, NQ, NK;
  int block_q, block_kv;
  float budget;
  const int8_t *pins;
  long long ps[4];
  const int8_t *drops;
  long long ds[4];
  int8_t *state;          // (Bp, Hp, NQ, NK)
  int32_t *cnt;           // (Bp, Hp, NQ) candidates
  int32_t *kpr;           // (Bp, Hp, NQ) budget counts
  unsigned int *not_covered;  // set to 1 when some row keeps fewer than all its candidates
};
cudaError_t launch_plan_build(const PlanArgs &p, int num_sms, cudaStream_t stream);

// Radial band control (radial_blocks), written for B batches and one keep head.
struct RadialArgs {
  int B, Sq, Skv, NQ, NK, block_q, block_kv;
  double density;
  double *width;       // device: the band's half width after bisection
  int8_t *keep;        // (B, 1, NQ, NK) or null
  int32_t *kv_count;   // (B, 1, NQ) or null
  uint16_t *kv_index;  // (B, 1, NQ, NK) or null
};
cudaError_t launch_radial(const RadialArgs &r, int num_sms, cudaStream_t stream);

// True when launch_select can pool the query tiles itself (q_raw).
bool select_pools_q(int NK, int D, int head_shared);
// True when, in addition, the select CTAs can pool k (k_raw): the whole grid
// fits on the device at once, so a cooperative launch is possible.
bool select_pools_k(const SelectArgs &a, int num_sms);

// Rows per CTA for the select kernels (4..32); 0 if NK is too large for the
// fused kernel (NK > 8192).
int select_rows_per_cta(int B, int Hs, int NQ, int NK, int num_sms, int D, int head_shared);
cudaError_t launch_select(const SelectArgs &a, int num_sms, cudaStream_t stream);

// out (B, 1, N, D) = mean over H of x (B, H, N, D)
cudaError_t launch_head_mean(const float *x, int B, int H, int N, int D, float *out, int num_sms,
                             cudaStream_t stream);

cudaError_t launch_keep_to_index(const int8_t *keep, long long rows, int NK, int32_t *kv_count,
                                 uint16_t *kv_index, cudaStream_t stream);

// Block-sparse attention forward.
struct AttnArgs {
  int B, Hq, Hkv, Sq, Skv, NQ, NK, Hs;
  float scale_log2;            // softmax scale * log2(e)
  const int32_t *kv_count;     // (B, Hs, NQ); null = dense (every tile)
  const uint16_t *kv_index;    // (B, Hs, NQ, NK)
  const unsigned int *dense_if_zero;  // optional device word: when it reads 0, attend densely
  __nv_bfloat16 *out;          // (B, Hq, Sq, D)
  float *lse;                  // (B, Hq, Sq)
  unsigned int *err;           // device error word
  // optional key-token mask (B, Hkv, Skv), element strides ks; a key token
  // whose byte is 0 takes part in no query row of that kv head (null = none)
  const int8_t *kmask;
  long long ks[3];
  // CTA order: 1 = query tile slowest (set by the launcher from the grid size)
  int q_first;
};

cudaError_t launch_attn_fwd(const AttnArgs &a, int D, int num_sms, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, cudaStream_t stream);
size_t attn_smem_bytes(int D);

// Block-sparse attention backward over kept tiles.
struct AttnBwdArgs {
  int B, Hq, Hkv, Sq, Skv, NQ, NK, Hs;
  float scale;                 // softmax scale (dQ and dK carry it)
  float scale_log2;            // scale * log2(e)
  const float *lse;            // (B, Hq, Sq) from the forward (natural log)
  float *dvec;                 // (B, Hq, Sq) scratch: <dO, O> per row
  const int32_t *kv_count;     // (B, Hs, NQ) kept kv tiles per row; null = dense
  const uint16_t *kv_index;    // (B, Hs, NQ, NK)
  const int32_t *q_count;      // (B, Hs, NK) query tiles keeping each kv tile; null = dense
  const uint16_t *q_index;     // (B, Hs, NK, NQ)
  __nv_bfloat16 *dq;           // (B, Hq, Sq, D)
  __nv_bfloat16 *dk, *dv;      // (B, Hkv, Skv, D)
  unsigned int *err;
  // optional key-token mask (B, Hkv, Skv), element strides ks, as in the
  // forward (null = none)
  const int8_t *kmask;
  long long ks[3];
};
// Runs <dO, O>, the transposed kept lists (from keep, when not null; q_count
// and q_index are written), the dK/dV kernel and the dQ kernel on `stream`.
// tq/tdo: {D, Sq, B*Hq} maps with 128-row boxes; tk/tv: 64-row boxes.
cudaError_t launch_attn_bwd(const AttnBwdArgs &a, int D, const __nv_bfloat16 *out, const __nv_bfloat16 *dout,
                            const int8_t *keep, int num_sms, const CUtensorMap &tq, const CUtensorMap &tdo,
                            const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream);



// A one-CTA kernel whose single bounded wait (which 0: an mbarrier, site
// 0x70; which 1: a counter, site 0x71) runs out after limit_cycles and
// records the timeout in err (selftest.cu).
cudaError_t launch_selftest_wait(int which, long long limit_cycles, unsigned int *err, cudaStream_t stream);

// Sets the calling thread's nsa_last_error() message.
void set_last_error(const char *msg);

}  // namespace nsa
