/*
 * nsa.h -- C ABI of the fixed-budget block-sparse attention library (libnsa).
 *
 * The method: block selection as defined by the page
 * "automatic/modules/attention/sparse/selector.py" (SparseSpec, pool_blocks,
 * diagonal_blocks, score_blocks, selection_plan, select_blocks), followed by a
 * flash-style attention forward pass that visits only the kept kv tiles (the
 * tile skipping of flex-attention's block mask discussed in attention-gym
 * issue #56, "Optimal ordering with block mask").
 *
 * Conventions shared by every entry point
 *  - Tensors are dense, row-major, head-major: q (B,Hq,Sq,D), k and v
 *    (B,Hkv,Skv,D), with the token axis second to last as in pool_blocks.
 *    q, k, v and out are bfloat16; pooled values and LSE are float32.
 *  - Every pointer argument not marked "host" is a device pointer. The caller
 *    owns all memory; the library allocates and frees nothing.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous unless stated. Only nsa_select (when force is
 *    off) and nsa_device_status synchronise, each with one small readback.
 *  - Every call returns an nsa_status. On failure a message is available from
 *    nsa_last_error() on the calling thread; no C++ exception crosses the ABI.
 *    Arguments are validated on the host before anything is enqueued; an
 *    invalid call enqueues nothing.
 *  - Tile counts: NQ = ceil(Sq/block_q), NK = ceil(Skv/block_kv)
 *    (selector.py, block_count). Keep heads Hs = 1 when head_shared, else Hq.
 *  - Pin and drop tile masks are int8 (nonzero = set), addressed as
 *    m[b*s[0] + h*s[1] + i*s[2] + j*s[3]] with element strides s[4] given by
 *    the caller; a stride of 0 broadcasts that axis. h ranges over keep heads.
 *    A NULL mask means none (selection_plan's pins=None / drops=None).
 */
#ifndef NSA_H
#define NSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st *nsa_stream_t;

typedef enum nsa_status {
  NSA_OK = 0,
  NSA_ERR_INVALID_ARG = 1,  /* bad pointer, size, stride, alignment or spec  */
  NSA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. D not 64/128) */
  NSA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed             */
  NSA_ERR_TIMEOUT = 4       /* a device-side bounded wait gave up            */
} nsa_status;

/* selector.py, SparseSpec. budget in (0, 1]: the fraction of each row's
 * candidates (tiles neither forced nor forbidden) that top-k may keep; forced
 * tiles (diagonal and pins) come on top. head_shared: score once for all heads
 * (means over heads), giving one keep head. force: never take the dense short
 * circuit. The page's score_chunk_bytes has no counterpart: the fused kernel
 * never materialises the score tensor. */
typedef struct nsa_spec {
  float budget;
  int32_t block_q;
  int32_t block_kv;
  int32_t head_shared;
  int32_t force;
} nsa_spec;

/* Message describing the last failure on the calling thread ("" if none).
 * The pointer stays valid until the next libnsa call on this thread. */
const char *nsa_last_error(void);

/* Library version string, e.g. "libnsa 0.1 sm_100a". */
const char *nsa_version(void);

/* selector.py, pool_blocks: float32 mean of each run of `block` tokens.
 * x: bf16 (B,H,S,D), 16-byte aligned. pooled: f32 (B,H,ceil(S/block),D).
 * A partial final tile is averaged over its own token count. D in {64,128}
 * (NSA_ERR_UNSUPPORTED otherwise); block >= 1. */
nsa_status nsa_pool(const void *x, int B, int H, int S, int D, int block,
                    float *pooled, nsa_stream_t stream);

/* The tensor-core scores of the long-row selection (debug/test path):
 * scores[b,h,i,j] = <pq[b,h,i,:], pk[b,h/(Hq/Hkv),j,:]> for per-head scoring
 * (Hq % Hkv == 0), from tf32 hi/lo splits of the float32 operands with
 * hi.hi + hi.lo + lo.hi accumulated in f32 (error-compensated 3xTF32).
 * scores: f32 (B,Hq,NQ,NKP) with NKP = NK rounded up to 128; columns NK ..
 * NKP-1 are written as 0. D in {64,128}; pq, pk, scores 16-byte aligned.
 * workspace (device, 256-byte aligned, at least 2 * round_up(B*Hkv*NK*D*4,
 * 256) bytes) receives the tf32 hi and lo parts of pk. nsa_select and
 * nsa_forward use the same kernels for rows whose pooled keys exceed 64 KB
 * (NK * D * 4 > 65536), in their own workspace. */
nsa_status nsa_score_tc(const float *pq, const float *pk, int B, int Hq,
                        int Hkv, int NQ, int NK, int D, float *scores,
                        void *workspace, size_t workspace_bytes,
                        nsa_stream_t stream);

/* selector.py, score_blocks (debug/test path): unscaled pooled affinities
 * scores[b,h,i,j] = <pq'[b,h,i,:], pk'[b,h,j,:]>, f32 (B,Hs,NQ,NK), where
 * pq' / pk' are the pooled tensors after the page's head handling:
 * head_shared averages pq (B,Hq,NQ,D) over Hq and pk (B,Hkv,NK,D) over Hkv;
 * otherwise query head h reads key head h / (Hq/Hkv). Hq % Hkv must be 0.
 * The hot path (nsa_select, nsa_forward) fuses this step and never writes
 * the score tensor. */
nsa_status nsa_score(const float *pq, const float *pk, int B, int Hq, int Hkv,
                     int NQ, int NK, int D, int head_shared, float *scores,
                     nsa_stream_t stream);

/* selector.py, selection_plan + select_blocks, fused with the scoring.
 * Inputs pq (B,Hq,NQ,D) and pk (B,Hkv,NK,D) are pooled f32 (nsa_pool).
 * Per keep row (b,h,i): must = diagonal (nominal token ranges of query tile i
 * and kv tile j overlap) | pins; forbidden = drops; candidates = ~must &
 * ~forbidden; c = number of candidates; k = ceil(f32(c) * f32(budget)) in
 * float32 (as torch evaluates the page's int64 * float); keep = must | (the k
 * candidates ranked highest by score, ties to the lower kv index) with
 * forbidden tiles then cleared.
 * Outputs: keep int8 (B,Hs,NQ,NK) (BlockSelection.keep); kv_count int32
 * (B,Hs,NQ) kept tiles per row; kv_index uint16 (B,Hs,NQ,NK): the first
 * kv_count entries of each row are the kept kv tile indices in ascending
 * order, the rest is untouched. NK <= 8192.
 * is_dense (host out): when force is off, the plan is read back once (one
 * stream synchronisation, as the page's single readback) and *is_dense = 1
 * if every row may keep all its candidates; the caller should then attend
 * densely with drops ignored (the page's `None`) and the keep outputs hold no
 * selection. When force is on nothing is read back and *is_dense = 0.
 * workspace: >= nsa_workspace_bytes(...) bytes, 256-byte aligned. */
nsa_status nsa_select(const float *pq, const float *pk, int B, int Hq, int Hkv,
                      int NQ, int NK, int D, const nsa_spec *spec,
                      const int8_t *pins, const int64_t *pin_strides,
                      const int8_t *drops, const int64_t *drop_strides,
                      int8_t *keep, int32_t *kv_count, uint16_t *kv_index,
                      int *is_dense, void *workspace, size_t workspace_bytes,
                      nsa_stream_t stream);

/* Compacts a keep tensor int8 (B,Hs,NQ,NK) into kv_count int32 (B,Hs,NQ) and
 * ascending kv_index uint16 (B,Hs,NQ,NK), the column-index form the attention
 * kernel reads (flex-attention's block mask, attention-gym issue #56). */
nsa_status nsa_keep_to_index(const int8_t *keep, int B, int Hs, int NQ, int NK,
                             int32_t *kv_count, uint16_t *kv_index,
                             nsa_stream_t stream);

/* Block-sparse flash attention forward over kept tiles.
 * For query token t of head h and key token s < Skv of kv head h/(Hq/Hkv):
 * allowed iff keep[b, Hs==1 ? 0 : h, t/block_q, s/block_kv] != 0;
 * out[t] = softmax(scale * q[t].k[s] over allowed s) . v (bf16),
 * lse[t] = natural log of sum over allowed s of exp(scale * q[t].k[s]) (f32).
 * A row with no allowed key gets out = 0, lse = -inf. keep == NULL means
 * dense (every tile kept). scale must be finite and positive.
 * block_q = 128 and block_kv = 64, D in {64,128}
 * (NSA_ERR_UNSUPPORTED otherwise). q, k, v 16-byte aligned.
 * workspace: >= nsa_workspace_bytes(...) bytes (holds the compacted lists). */
nsa_status nsa_block_sparse_attn_fwd(const void *q, const void *k, const void *v,
                                     int B, int Hq, int Hkv, int Sq, int Skv,
                                     int D, const int8_t *keep, int Hs,
                                     int block_q, int block_kv, float scale,
                                     void *out, float *lse, void *workspace,
                                     size_t workspace_bytes, nsa_stream_t stream);

/* nsa_block_sparse_attn_fwd with a token-level key mask (the qkv_mask of
 * NATTEN issue #124 "Arbitrary masks", read with SDPA's convention that true
 * takes part): kmask int8 (B,Hkv,Skv) on the device, element strides
 * kmask_strides[3] over (batch, kv head, key token) (NULL = contiguous; a 0
 * stride broadcasts). Key token s of kv head hk takes part in query row t of
 * every query head of that kv group iff the tile rule above allows it AND
 * kmask[b, hk, s] != 0. Query rows are not masked: a row whose allowed keys
 * are all masked gets out = 0, lse = -inf. kmask == NULL is the unmasked
 * call. Errors as nsa_block_sparse_attn_fwd; negative strides are
 * NSA_ERR_INVALID_ARG. The mask bytes are read for kept tiles only. */
nsa_status nsa_block_sparse_attn_fwd_masked(
    const void *q, const void *k, const void *v, int B, int Hq, int Hkv, int Sq,
    int Skv, int D, const int8_t *keep, int Hs, int block_q, int block_kv,
    const int8_t *kmask, const int64_t *kmask_strides, float scale, void *out,
    float *lse, void *workspace, size_t workspace_bytes, nsa_stream_t stream);

/* Gradients of nsa_block_sparse_attn_fwd (the backward items -- dv, dk, dq,
 * GQA -- of the native-sparse-attention-pytorch issue #1 todo list). For the
 * loss sum(dout * out), with P the forward's restricted softmax recomputed
 * from lse, dP = dout . v^T, Dv = rowsum(dout * out) and dS = P (dP - Dv):
 *   dv[s] = sum_t P(t,s) dout[t]          (summed over the kv group's heads)
 *   dk[s] = scale sum_t dS(t,s) q[t]      (summed over the kv group's heads)
 *   dq[t] = scale sum_s dS(t,s) k[s]
 * Inputs: q, k, v, keep, Hs, block sizes and scale exactly as given to the
 * forward; out bf16 (B,Hq,Sq,D) and lse f32 (B,Hq,Sq) the forward's outputs;
 * dout bf16 (B,Hq,Sq,D). Outputs (overwritten): dq bf16 (B,Hq,Sq,D), dk and
 * dv bf16 (B,Hkv,Skv,D); kv tiles no row kept get dk = dv = 0, rows with no
 * allowed key get dq = 0. block_q = 128, block_kv = 64, D in {64,128}
 * (NSA_ERR_UNSUPPORTED otherwise). q, k, v, out, dout, dq 16-byte aligned.
 * workspace: >= nsa_bwd_workspace_bytes(...) bytes, 256-byte aligned. */
nsa_status nsa_block_sparse_attn_bwd(
    const void *q, const void *k, const void *v, const void *out,
    const float *lse, const void *dout, int B, int Hq, int Hkv, int Sq,
    int Skv, int D, const int8_t *keep, int Hs, int block_q, int block_kv,
    float scale, void *dq, void *dk, void *dv, void *workspace,
    size_t workspace_bytes, nsa_stream_t stream);

/* nsa_block_sparse_attn_bwd for the key-masked forward
 * (nsa_block_sparse_attn_fwd_masked): kmask and kmask_strides as there (NULL
 * kmask = the unmasked call); masked key columns take no part in P, so they
 * get no dK/dV from any row and give no dQ. out and lse must be that masked
 * forward's. Errors as nsa_block_sparse_attn_bwd; negative strides are
 * NSA_ERR_INVALID_ARG. */
nsa_status nsa_block_sparse_attn_bwd_masked(
    const void *q, const void *k, const void *v, const void *out,
    const float *lse, const void *dout, int B, int Hq, int Hkv, int Sq,
    int Skv, int D, const int8_t *keep, int Hs, int block_q, int block_kv,
    const int8_t *kmask, const int64_t *kmask_strides, float scale, void *dq,
    void *dk, void *dv, void *workspace, size_t workspace_bytes,
    nsa_stream_t stream);

/* Workspace bytes of nsa_block_sparse_attn_bwd (Hs = keep heads, 1 when
 * keep is NULL). Host only; 0 for invalid sizes. */
size_t nsa_bwd_workspace_bytes(int B, int Hq, int Hkv, int Sq, int Skv, int D,
                               int Hs);

/* The whole path in one call: pool q and k, fused score + plan + top-k keep,
 * block-sparse attention over the kept tiles. Nothing is read back: the dense
 * short circuit (every row covers all its candidates and force is off) is
 * decided on the device, and attention then visits every tile with drops
 * ignored, as the page's `None` asks. keep_out (nullable): when given,
 * receives the int8 keep (B,Hs,NQ,NK) of the selection (its contents are the
 * selection even when the dense short circuit is taken).
 * The call allocates nothing and never synchronises with the host, so it can
 * be captured into a CUDA graph; make one call on the device before the
 * capture, which loads the module.
 * workspace: >= nsa_workspace_bytes(...) bytes, 256-byte aligned. */
nsa_status nsa_forward(const void *q, const void *k, const void *v, int B,
                       int Hq, int Hkv, int Sq, int Skv, int D,
                       const nsa_spec *spec, const int8_t *pins,
                       const int64_t *pin_strides, const int8_t *drops,
                       const int64_t *drop_strides, float scale, void *out,
                       float *lse, int8_t *keep_out, void *workspace,
                       size_t workspace_bytes, nsa_stream_t stream);

/* nsa_forward with timing: `events` (nullable) points to 4 cudaEvent_t
 * handles created by the caller (NULL entries are skipped); they are recorded
 * on `stream` before pooling, after pooling, after selection and after
 * attention, so the caller can time each kernel of the path inside a timed
 * loop. Same kernels and results as nsa_forward. The kernels are chained
 * with programmatic dependent launch; an event recorded between two of them
 * serialises that boundary, so time the whole step with the middle entries
 * NULL. */
nsa_status nsa_forward_timed(const void *q, const void *k, const void *v, int B,
                             int Hq, int Hkv, int Sq, int Skv, int D,
                             const nsa_spec *spec, const int8_t *pins,
                             const int64_t *pin_strides, const int8_t *drops,
                             const int64_t *drop_strides, float scale, void *out,
                             float *lse, int8_t *keep_out, void *workspace,
                             size_t workspace_bytes, void *const *events,
                             nsa_stream_t stream);

/* Workspace bytes that nsa_select, nsa_block_sparse_attn_fwd and nsa_forward
 * need for these sizes (the largest of the three). Host only; no CUDA call.
 * Returns 0 for invalid sizes. */
size_t nsa_workspace_bytes(int B, int Hq, int Hkv, int Sq, int Skv, int D,
                           const nsa_spec *spec);

/* nsa_forward without a workspace argument, for callers that may not
 * allocate device memory (no counterpart on the pages: it exists for hosts
 * whose device memory is owned by another allocator, plugins that only get
 * the tensors they compute on, and loops where cudaMalloc's implicit
 * synchronisation is not allowed). The caller still passes inputs and
 * outputs; the scratch comes from one fixed device array of
 * NSA_NOALLOC_SCRATCH_BYTES that the library declares and every GPU that
 * loads it holds until exit. The allocation-free path calls no cudaMalloc,
 * cudaFree or allocating routine.
 *  - Sizes whose workspace (nsa_workspace_bytes) exceeds the array are
 *    rejected with NSA_ERR_INVALID_ARG and a message naming the limit.
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress (with that device current). With lazy module
 *    loading (the CUDA default) that lookup may load the library's device
 *    code on that device, which is when the array is reserved, and it may
 *    synchronise. Make one warm-up call on each device at initialisation
 *    (or set CUDA_MODULE_LOADING=EAGER), and in any case before any stream
 *    capture.
 *  - All calls share the array: calls whose work overlaps on the GPU (on
 *    different streams, or from different threads) race. The array keeps the
 *    last call's contents; nothing in it needs to start at zero. */
#define NSA_NOALLOC_SCRATCH_BYTES (16u << 20)
nsa_status nsa_forward_noalloc(const void *q, const void *k, const void *v,
                               int B, int Hq, int Hkv, int Sq, int Skv, int D,
                               const nsa_spec *spec, const int8_t *pins,
                               const int64_t *pin_strides, const int8_t *drops,
                               const int64_t *drop_strides, float scale,
                               void *out, float *lse, int8_t *keep_out,
                               nsa_stream_t stream);

/* ---------------------------------------------------------------- plans
 * selector.py, selection_plan with its plan_cache: the part of a selection
 * that depends only on the geometry, the spec and the pin/drop layout, built
 * once and reused by every step of a generation that keeps them (the page
 * caches it under a caller key; here the caller keeps the buffer).
 *
 * The plan lives in a caller buffer of nsa_plan_bytes() bytes, 256-byte
 * aligned, laid out as: a 256-byte header (word 0: the build's "some row
 * does not cover all its candidates" flag), then, each section starting at
 * the next multiple of 256 bytes,
 *   state int8  (Bp, Hp, NQ, NK): 0 = candidate, 1 = kept whatever the
 *               scores (diagonal or pinned, and not dropped), 2 = dropped;
 *   cand  int32 (Bp, Hp, NQ): candidates per row, c;
 *   kcnt  int32 (Bp, Hp, NQ): budget count k = ceil(f32(c) * f32(budget)).
 * Bp = B when a mask varies over batches (a non-zero batch stride), else 1;
 * Hp = keep heads when a mask varies over heads, else 1. Rows with a
 * broadcast extent are shared by every batch / head. */
typedef struct nsa_plan_info {
  int32_t batches;           /* Bp */
  int32_t heads;             /* Hp */
  int32_t covers_everything; /* every row may keep all its candidates */
  int32_t reserved;
} nsa_plan_info;

/* Bytes of the plan buffer for these sizes and mask strides (NULL strides =
 * no such mask). Host only; 0 for invalid sizes. */
size_t nsa_plan_bytes(int B, int Hq, int Sq, int Skv, const nsa_spec *spec,
                      const int64_t *pin_strides, const int64_t *drop_strides);

/* Builds the plan on the device (one warp per row) and reads the covers flag
 * back once (one stream synchronisation: the page's single readback,
 * amortised by its cache). pins/drops as in nsa_select; info (host out)
 * receives the plan's extents and covers_everything. */
nsa_status nsa_plan_build(int B, int Hq, int Sq, int Skv, const nsa_spec *spec,
                          const int8_t *pins, const int64_t *pin_strides,
                          const int8_t *drops, const int64_t *drop_strides,
                          void *plan, size_t plan_bytes, nsa_plan_info *info,
                          nsa_stream_t stream);

/* nsa_forward with a built plan in place of pins and drops: the tile states
 * and budget counts come from the plan, and when it covers everything and
 * force is off no scoring is done at all (dense attention, drops ignored,
 * keep_out untouched). The plan must have been built with the same B, Hq,
 * Sq, Skv and spec (as the page's cache keys it) and the masks the caller
 * means; the library does not re-check them. Same results as nsa_forward
 * with those masks. */
nsa_status nsa_forward_plan(const void *q, const void *k, const void *v, int B,
                            int Hq, int Hkv, int Sq, int Skv, int D,
                            const nsa_spec *spec, const void *plan,
                            const nsa_plan_info *info, float scale, void *out,
                            float *lse, int8_t *keep_out, void *workspace,
                            size_t workspace_bytes, nsa_stream_t stream);

/* selector.py, schedule: per-step budgets (host only, into budgets[steps]).
 * Every step gets `budget`; with bump > 0 and bump_steps > 0 the first and
 * last min(bump_steps, ceil(steps/2)) steps get min(1, budget + bump), so
 * there are at most two distinct values (at most two plans). */
nsa_status nsa_schedule(int steps, double budget, double bump, int bump_steps,
                        double *budgets);

/* selector.py, radial_blocks: a fixed band around the diagonal, the baseline
 * a score-based selection should improve on. Tile centres ((i+0.5) block_q, (j+0.5) block_kv); the band keeps
 * tiles whose centre distance is <= w, w the upper end of 40 bisection
 * steps on [0, max(Sq, Skv)] that aim the kept fraction (float32 mean of the
 * 0/1 mask) at `density`. All on the device, nothing read back (the page
 * reads the fraction back at every step). width: device double, receives w.
 * keep int8 (B,1,NQ,NK), kv_count int32 (B,1,NQ) and kv_index uint16
 * (B,1,NQ,NK, first kv_count entries ascending) are each nullable; every
 * batch gets the same band, in the layout nsa_block_sparse_attn_fwd takes
 * with Hs = 1. NK <= 65535 and NQ * NK < 2^24. */
nsa_status nsa_radial_blocks(int B, int Sq, int Skv, double density,
                             const nsa_spec *spec, double *width, int8_t *keep,
                             int32_t *kv_count, uint16_t *kv_index,
                             nsa_stream_t stream);

/* Reads (and with clear != 0 resets) the library's device error word on the
 * current device, synchronising the device first. Returns NSA_ERR_TIMEOUT if
 * a kernel's bounded wait gave up since the last clear, else NSA_OK; the
 * message then names the wait site code of the first wait that gave up. */
nsa_status nsa_device_status(int clear);

/* Failure detection check (no counterpart on the pages): every wait inside
 * the library's kernels is bounded (about one second of SM clock), and a wait
 * that runs out records NSA_ERR_TIMEOUT and its site code in the device error
 * word, drains what its CTA has in flight and returns, leaving the context
 * usable. This call enqueues a one-CTA kernel whose single wait, with a limit
 * of limit_cycles SM clock cycles (1 .. the kernels' own limit), is on a
 * condition nothing satisfies: which = 0 waits on an mbarrier no thread
 * arrives on (site 0x70), which = 1 on a counter no thread increments (site
 * 0x71). The kernel has nothing in flight while it waits. After it,
 * nsa_device_status reports NSA_ERR_TIMEOUT with that site; later calls run
 * normally. NSA_ERR_INVALID_ARG for other values of which or limit_cycles. */
nsa_status nsa_selftest_timeout(int which, long long limit_cycles,
                                nsa_stream_t stream);

/* Number of kernels the library has launched in this process so far, over
 * every device and host thread (memsets and copies are not counted). Host
 * only, no CUDA call. The difference of two readings counts the kernels a
 * span of calls launched. */
unsigned long long nsa_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* NSA_H */
