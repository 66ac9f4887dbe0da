// attn_bwd.cu -- gradients of block-sparse attention over kept tiles on
// tcgen05 tensor cores (dQ, dK, dV; the backward items of the
// native-sparse-attention-pytorch issue #1 todo list: dv, dk, dq, GQA).
//
// For query token t with allowed keys s (the kept tiles of its row, s < Skv),
// P = softmax(scale q k^T) is recomputed from the forward's LSE:
//   P(t,s)  = 2^(scale log2e <q_t,k_s> - log2e LSE_t)
//   dP(t,s) = <dO_t, v_s>,  Dv_t = <dO_t, O_t>,  dS = P (dP - Dv)
//   dV_s += P(t,s) dO_t,  dK_s += scale dS(t,s) q_t,  dQ_t = scale sum_s dS k_s
// Three kernels:
//   bwd_dvec_kernel   Dv_t = <dO_t, O_t> in f32 (streams O and dO once)
//   attn_bwd_dkdv     one CTA per kv tile j of kv head hk: K_j and V_j stay
//                     in shared memory while the (query head, query tile)
//                     pairs that kept j stream through a 3-stage Q ring and
//                     a 2-stage dO ring.
//                     Per pair: S = Q K^T and dP = dO V^T (M=128 query rows,
//                     N=64 keys) into TMEM; four warps form P and dS (bf16)
//                     in shared memory (one tile each); dV^T += dO^T P and dK^T += Q^T dS
//                     (M = head dim, N = 64 keys, K = 128 query rows, both
//                     operands MN-major) accumulate in TMEM over all pairs of
//                     the kv group, so the GQA sum over query heads needs no
//                     atomics.
//   attn_bwd_dq       one CTA per keep row (query head h, query tile i),
//                     two per SM like the forward, visiting its kept kv
//                     tiles: S and dP into TMEM, dS written back over S as
//                     two bf16 parts (hi, and the lo remainder), and
//                     dQ += dS_hi K_j + dS_lo K_j with both read from TMEM.
// Roles in both: lane 0 of warps 0 and 6 issue the TMA loads (two issuing
// threads: one alone moves too few bytes per cycle), lane 0 of warp 1 owns
// TMEM and issues the MMAs, warps 2-5 (one query row per thread, TMEM lane =
// row) compute P and dS and run the epilogue. Every mbarrier wait is bounded
// (nsa_device.cuh); a timeout sets the device error word, and the CTA drains
// its copies and MMAs, frees TMEM and exits.
#include "nsa_device.cuh"
#include "nsa_kernels.cuh"

namespace nsa {

namespace {

constexpr int BQ = 128;
constexpr int BKV = 64;
constexpr int kThreads = 224;  // 7 warps
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ Dv
// Dv[row] = sum_d dO[row, d] * O[row, d]; 16 lanes per row of D=128 (8
// elements per lane), 8 lanes per row of D=64.
template <int D>
__global__ void __launch_bounds__(256) bwd_dvec_kernel(const __nv_bfloat16 *out, const __nv_bfloat16 *dout,
                                                      long long rows, float *dvec) {
  constexpr int LPR = D / 8;  // lanes per row
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;  // a multiple of 32
  const long long total = rows * LPR;
  // every lane of a warp runs the same trip count (the shuffles need all 32)
  const long long padded = (total + 31) / 32 * 32;
  for (long long x = tid; x < padded; x += stride) {
    const bool active = x < total;
    const long long row = x / LPR;
    const int part = (int)(x % LPR);
    float acc = 0.f;
    if (active) {
      const uint4 a = *reinterpret_cast<const uint4 *>(out + row * D + part * 8);
      const uint4 b = *reinterpret_cast<const uint4 *>(dout + row * D + part * 8);
      const __nv_bfloat162 *pa = reinterpret_cast<const __nv_bfloat162 *>(&a);
      const __nv_bfloat162 *pb = reinterpret_cast<const __nv_bfloat162 *>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(pa[e]), fb = __bfloat1622float2(pb[e]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, LPR);
    if (active && part == 0) dvec[row] = acc;
  }
}

// ------------------------------------------------------------ q lists
// keep (rows of NQ x NK per (batch, keep head)) -> per kv tile j the
// ascending list of query tiles i with keep[.., i, j] != 0. One warp per
// (batch, keep head, j).
__global__ void __launch_bounds__(256) keep_to_qindex_kernel(const int8_t *keep, long long bh, int NQ, int NK,
                                                            int32_t *q_count, uint16_t *q_index) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long cols = bh * NK;
  for (long long c = (long long)blockIdx.x * 8 + warp; c < cols; c += (long long)gridDim.x * 8) {
    const long long x = c / NK;
    const int j = (int)(c % NK);
    const int8_t *base = keep + x * NQ * (long long)NK + j;
    uint16_t *dst = q_index + c * NQ;
    int n = 0;
    for (int i0 = 0; i0 < NQ; i0 += 32) {
      const int i = i0 + lane;
      const bool kept = i < NQ && base[(long long)i * NK] != 0;
      const unsigned m = __ballot_sync(0xffffffffu, kept);
      if (kept) dst[n + __popc(m & ((1u << lane) - 1u))] = (uint16_t)i;
      n += __popc(m);
    }
    if (lane == 0) q_count[c] = n;
  }
}

struct Bars {
  uint64_t kv_full;      // dkdv: K_j and V_j; dq: Q and dO
  uint64_t in_full[4];   // dkdv: Q ring; dq: K ring
  uint64_t in_empty[4];
  uint64_t v_full[4];    // dkdv: dO ring; dq: V ring
  uint64_t v_empty[4];
  uint64_t sd_full[2];   // S(n) and dP(n) in TMEM buffer n & 1
  uint64_t ds_full[2];   // the compute warps have consumed S/dP(n) and written P/dS(n)
                         // (dkdv: [0] only, one P/dS tile pair)
  uint64_t ds_empty[2];  // dkdv: [0], the products reading P/dS(n) completed
  uint64_t done;         // every MMA of the CTA completed
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// The key columns of kv tile j that take part, as bits (mlo: columns 0-31,
// mhi: 32-63): inside Skv and, with a key mask, unmasked for kv head hk.
// Called by a whole warp (the bits come from ballots).
__device__ __forceinline__ void tile_colmask(const AttnBwdArgs &a, int b, int hk, int j, uint32_t &mlo,
                                             uint32_t &mhi) {
  const int lane = threadIdx.x & 31;
  const long long s0 = (long long)j * BKV + lane, s1 = s0 + 32;
  bool t0 = s0 < a.Skv, t1 = s1 < a.Skv;
  if (a.kmask != nullptr) {
    const int8_t *mrow = a.kmask + b * a.ks[0] + hk * a.ks[1];
    t0 = t0 && mrow[s0 * a.ks[2]] != 0;
    t1 = t1 && mrow[s1 * a.ks[2]] != 0;
  }
  mlo = __ballot_sync(0xffffffffu, t0);
  mhi = __ballot_sync(0xffffffffu, t1);
}

// P and dS of one query row (thread) for a 64-key tile. s and dp: the raw
// S and dP columns from TMEM. p and ds get bf16 pairs (column 2c in the low
// half). Columns whose bit in mlo/mhi is clear and rows with lse2 = +inf
// give 0.
template <bool WANT_P>
__device__ __forceinline__ void p_and_ds(const uint32_t (&s0)[32], const uint32_t (&s1)[32],
                                         const uint32_t (&d0)[32], const uint32_t (&d1)[32], float sl2,
                                         float lse2, float dv, uint32_t mlo, uint32_t mhi, uint32_t (&p)[32],
                                         uint32_t (&ds)[32]) {
  const uint64_t sc2 = f2_pack(sl2, sl2), nl2 = f2_pack(-lse2, -lse2);
  const bool all_in = (mlo & mhi) == 0xffffffffu;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    float x0, x1, x2, x3;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(s0[2 * c]), __uint_as_float(s0[2 * c + 1])), sc2, nl2), x0, x1);
    f2_unpack(f2_fma(f2_pack(__uint_as_float(s1[2 * c]), __uint_as_float(s1[2 * c + 1])), sc2, nl2), x2, x3);
    float p0 = fast_exp2(x0), p1 = fast_exp2(x1), p2 = fast_exp2(x2), p3 = fast_exp2(x3);
    if (!all_in) {
      if (!((mlo >> (2 * c)) & 1u)) p0 = 0.f;
      if (!((mlo >> (2 * c + 1)) & 1u)) p1 = 0.f;
      if (!((mhi >> (2 * c)) & 1u)) p2 = 0.f;
      if (!((mhi >> (2 * c + 1)) & 1u)) p3 = 0.f;
    }
    const float g0 = p0 * (__uint_as_float(d0[2 * c]) - dv), g1 = p1 * (__uint_as_float(d0[2 * c + 1]) - dv);
    const float g2 = p2 * (__uint_as_float(d1[2 * c]) - dv), g3 = p3 * (__uint_as_float(d1[2 * c + 1]) - dv);
    if (WANT_P) {
      p[c] = pack_bf16x2(p0, p1);
      p[c + 16] = pack_bf16x2(p2, p3);
    }
    ds[c] = pack_bf16x2(g0, g1);
    ds[c + 16] = pack_bf16x2(g2, g3);
  }
}

// Per-row LSE (log2 units) and Dv of query row `row` (global index) of a
// tile; rows past Sq and rows with no allowed key get lse2 = +inf, so every
// P of theirs is 2^-inf = 0.
__device__ __forceinline__ void row_stats(const float *lse, const float *dvec, size_t row, bool in_range,
                                          float &lse2, float &dv) {
  float l = in_range ? lse[row] : -INFINITY;
  const bool ok = l > -INFINITY;
  lse2 = ok ? l * kLog2e : INFINITY;
  dv = ok ? dvec[row] : 0.f;
}

// The (query head, query tile) pairs of one kv tile: for each query head of
// the kv group the ascending list of query tiles that kept tile j (one list
// for all heads when the keep has one head; every tile when q_count is null).
struct Pairs {
  const int32_t *qc;
  const uint16_t *qi;
  int NQ, NK, g, Hs, b, hk, j;
  __device__ __forceinline__ size_t row(int hh) const {
    const int hs = (Hs == 1) ? 0 : hk * g + hh;
    return ((size_t)b * Hs + hs) * NK + j;
  }
  __device__ __forceinline__ int count(int hh) const { return qc ? qc[row(hh)] : NQ; }
  __device__ __forceinline__ int tile(int hh, int pos) const { return qc ? (int)qi[row(hh) * NQ + pos] : pos; }
};

// Walks the pairs in order: head hh, position pos in its list (cnt entries).
struct Cursor {
  int hh, pos, cnt;
  __device__ __forceinline__ void start(const Pairs &P) {
    hh = 0;
    pos = -1;
    cnt = P.count(0);
    next(P);
  }
  __device__ __forceinline__ void next(const Pairs &P) {
    ++pos;
    while (pos >= cnt && hh + 1 < P.g) {
      ++hh;
      pos = 0;
      cnt = P.count(hh);
    }
  }
};

template <int D>
struct DkdvCfg {
  // Q ring 3 stages, dO ring 2 stages, P and dS single tiles: a Q stage is
  // released by dK^T, the last product of its pair, so the third stage lets
  // the Q load of pair n+2 start while pair n's products still run; the dO
  // stage is released earlier (dV^T is issued first) and its load hides
  // behind dK^T(n) and S(n+2)
  static constexpr int QST = 3;
  static constexpr int DST = 2;
  static constexpr int KV_BYTES = BKV * D * 2;
  static constexpr int Q_BYTES = BQ * D * 2;
  static constexpr int PT_BYTES = BQ * BKV * 2;  // one P or dS tile, 128 rows x 128 B
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = KV_BYTES;
  static constexpr int OFF_Q = 2 * KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + QST * Q_BYTES;
  static constexpr int OFF_P = OFF_DO + DST * Q_BYTES;
  static constexpr int OFF_DS = OFF_P + PT_BYTES;
  static constexpr int OFF_BAR = OFF_DS + PT_BYTES;
  static constexpr int TILE_BYTES = OFF_BAR + 256;
  static constexpr int SMEM_BYTES = TILE_BYTES + 1024;  // room to align the base to 1024
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 320;
};
static_assert(DkdvCfg<128>::SMEM_BYTES <= 232448, "dkdv shared memory");

// Barriers of the dK/dV kernel: in_full/in_empty = Q ring, v_full/v_empty =
// dO ring, ds_full[0]/ds_empty[0] = the single P/dS tile pair.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv_kernel(const AttnBwdArgs a, const __grid_constant__ CUtensorMap tq,
                         const __grid_constant__ CUtensorMap tdo, const __grid_constant__ CUtensorMap tk,
                         const __grid_constant__ CUtensorMap tv) {
  using C = DkdvCfg<D>;
  constexpr int QST = C::QST, DST = C::DST;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_u32 & 1023u)) & 1023u;
  uint32_t dyn_size;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_size));
  if (pad + C::TILE_BYTES > dyn_size) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrSmemLayout);
    return;
  }
  unsigned char *smem = smem_raw + pad;
  Bars *bars = reinterpret_cast<Bars *>(smem + C::OFF_BAR);
  volatile int *abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = a.Hq / a.Hkv;

  // work item: kv tile j fastest, so CTAs running together share (b, hk)
  // and their Q/dO tiles stay in L2
  long long x = blockIdx.x;
  const int j = (int)(x % a.NK);
  x /= a.NK;
  const int hk = (int)(x % a.Hkv);
  const int b = (int)(x / a.Hkv);

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars->in_full[s], 1);
      mbar_init(&bars->in_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->sd_full[s], 1);
      mbar_init(&bars->ds_full[s], 4);
      mbar_init(&bars->ds_empty[s], 1);
    }
    mbar_init(&bars->done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  pdl_wait();  // the lists and Dv are the previous kernels' outputs
  const Pairs P = {a.q_count, a.q_index, a.NQ, a.NK, g, a.Hs, b, hk, j};
  int total = 0;
  for (int hh = 0; hh < g; ++hh) total += P.count(hh);

  unsigned char *sK = smem + C::OFF_K;
  unsigned char *sV = smem + C::OFF_V;
  unsigned char *sQ = smem + C::OFF_Q;
  unsigned char *sDO = smem + C::OFF_DO;
  unsigned char *sP = smem + C::OFF_P;
  unsigned char *sDS = smem + C::OFF_DS;

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ producers
    // warp 0: K_j, V_j and the Q ring; warp 6: the dO ring
    if (lane == 0 && total > 0) {
      const bool is_q = (warp == 0);
      const int STAGES = is_q ? QST : DST;
      const CUtensorMap *map = is_q ? &tq : &tdo;
      unsigned char *ring = is_q ? sQ : sDO;
      uint64_t *full = is_q ? bars->in_full : bars->v_full;
      uint64_t *empty = is_q ? bars->in_empty : bars->v_empty;
      tma_prefetch_desc(map);
      if (is_q) {
        tma_prefetch_desc(&tk);
        tma_prefetch_desc(&tv);
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(sK + c * BKV * 128, &tk, &bars->kv_full, c * 64, j * BKV, b * a.Hkv + hk);
          tma_load_3d(sV + c * BKV * 128, &tv, &bars->kv_full, c * 64, j * BKV, b * a.Hkv + hk);
        }
      }
      Cursor cur;
      cur.start(P);
      int issued = 0;
      for (int n = 0; n < total; ++n, cur.next(P)) {
        const int st = n % STAGES;
        const int h = hk * g + cur.hh, i = P.tile(cur.hh, cur.pos);
        if (n >= STAGES && !mbar_wait(&empty[st], ((n / STAGES) - 1) & 1, abort, a.err, 0x40)) break;
        mbar_arrive_expect_tx(&full[st], C::Q_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(ring + st * C::Q_BYTES + c * BQ * 128, map, &full[st], c * 64, i * BQ, b * a.Hq + h);
        issued = n + 1;
      }
      if (*abort) {
        int never = 0;
        if (is_q) mbar_wait(&bars->kv_full, 0, &never, a.err, 0x41);
        for (int n = (issued > STAGES ? issued - STAGES : 0); n < issued; ++n)
          mbar_wait(&full[n % STAGES], (n / STAGES) & 1, &never, a.err, 0x41);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0 && total > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BQ, BKV, 0, 0);   // S, dP: M = query rows, N = keys
      constexpr uint32_t idT = idesc_bf16_f32(128, BKV, 1, 1);  // dV^T, dK^T: M = head dim (128 rows)
      // K-major views for S and dP; MN-major views of Q and dO (M = head
      // dim in 64-element chunks BQ*128 bytes apart; for D=64 the second
      // chunk of M repeats the first, LBO = 0, and lanes 64-127 are unused)
      const uint64_t dQk = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dDOk = smem_desc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dQm = smem_desc_sw128(smem_u32(sQ), D == 128 ? BQ * 128 : 0, 1024);
      const uint64_t dDOm = smem_desc_sw128(smem_u32(sDO), D == 128 ? BQ * 128 : 0, 1024);
      const uint64_t dP = smem_desc_sw128(smem_u32(sP), C::PT_BYTES, 1024);
      const uint64_t dDS = smem_desc_sw128(smem_u32(sDS), C::PT_BYTES, 1024);
      // dV^T(m) (frees the dO stage), then dK^T(m) (frees the Q stage and
      // the P/dS tiles); a stage is committed only when a later pair reuses it
      auto issue_grad = [&](int m) -> bool {
        const int sq = m % QST, sd = m % DST;
        if (!mbar_wait(&bars->ds_full[0], m & 1, abort, a.err, 0x42)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          umma_bf16_ss(tmem + C::COL_DV, dDOm + ((sd * C::Q_BYTES + kk * 2048) >> 4), dP + ((kk * 2048) >> 4), idT,
                       (m > 0 || kk > 0) ? 1u : 0u);
        if (m + DST < total) umma_commit(&bars->v_empty[sd]);
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          umma_bf16_ss(tmem + C::COL_DK, dQm + ((sq * C::Q_BYTES + kk * 2048) >> 4), dDS + ((kk * 2048) >> 4), idT,
                       (m > 0 || kk > 0) ? 1u : 0u);
        if (m + QST < total) umma_commit(&bars->in_empty[sq]);
        if (m + 1 < total) umma_commit(&bars->ds_empty[0]);
        return true;
      };
      bool ok = mbar_wait(&bars->kv_full, 0, abort, a.err, 0x43);
      for (int n = 0; ok && n < total; ++n) {
        const int sq = n % QST, sd = n % DST, bf = n & 1;
        if (!mbar_wait(&bars->in_full[sq], (n / QST) & 1, abort, a.err, 0x44)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_q = sq * C::Q_BYTES + (kk / 4) * (BQ * 128) + (kk % 4) * 32;
          const uint32_t off_k = (kk / 4) * (BKV * 128) + (kk % 4) * 32;
          umma_bf16_ss(tmem + C::COL_S + bf * BKV, dQk + (off_q >> 4), dK + (off_k >> 4), idS, kk > 0);
        }
        if (!mbar_wait(&bars->v_full[sd], (n / DST) & 1, abort, a.err, 0x49)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_o = sd * C::Q_BYTES + (kk / 4) * (BQ * 128) + (kk % 4) * 32;
          const uint32_t off_v = (kk / 4) * (BKV * 128) + (kk % 4) * 32;
          umma_bf16_ss(tmem + C::COL_DP + bf * BKV, dDOk + (off_o >> 4), dV + (off_v >> 4), idS, kk > 0);
        }
        umma_commit(&bars->sd_full[bf]);
        if (n > 0 && !issue_grad(n - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) issue_grad(total - 1);
      umma_commit(&bars->done);
      int never = 0;
      mbar_wait(&bars->done, 0, &never, a.err, 0x45);
    }
    __syncwarp();
  } else {
    // ------------------------------------------ P, dS and the epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int valid = min(BKV, a.Skv - j * BKV);  // key rows of the tile inside Skv
    uint32_t mlo, mhi;  // the same key columns for every pair of this kv tile
    tile_colmask(a, b, hk, j, mlo, mhi);
    bool ok = true;
    Cursor cur;
    cur.start(P);
    for (int n = 0; n < total; ++n, cur.next(P)) {
      const int bf = n & 1;
      const int h = hk * g + cur.hh, i = P.tile(cur.hh, cur.pos);
      const int t = i * BQ + row;
      float lse2, dv;
      row_stats(a.lse, a.dvec, ((size_t)b * a.Hq + h) * a.Sq + t, t < a.Sq, lse2, dv);
      if (!warp_wait(&bars->sd_full[bf], (n >> 1) & 1, abort, a.err, 0x46)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s0[32], s1[32], d0[32], d1[32];
      tmem_ld32(lane_base + C::COL_S + bf * BKV, s0);
      tmem_ld32(lane_base + C::COL_S + bf * BKV + 32, s1);
      tmem_ld32(lane_base + C::COL_DP + bf * BKV, d0);
      tmem_ld32(lane_base + C::COL_DP + bf * BKV + 32, d1);
      tmem_wait_ld();
      uint32_t pp[32], dd[32];
      p_and_ds<true>(s0, s1, d0, d1, a.scale_log2, lse2, dv, mlo, mhi, pp, dd);
      // the P/dS tiles were last read by the products of pair n-1
      if (n >= 1 && !warp_wait(&bars->ds_empty[0], (n - 1) & 1, abort, a.err, 0x47)) {
        ok = false;
        break;
      }
      // row `row` of the 128-byte swizzled tile: 16-byte chunk q (keys
      // 8q..8q+7) at chunk position q ^ (row & 7)
      unsigned char *prow = sP + row * 128;
      unsigned char *drow = sDS + row * 128;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int pos = (q ^ (row & 7)) << 4;
        *reinterpret_cast<uint4 *>(prow + pos) = make_uint4(pp[4 * q], pp[4 * q + 1], pp[4 * q + 2], pp[4 * q + 3]);
        *reinterpret_cast<uint4 *>(drow + pos) = make_uint4(dd[4 * q], dd[4 * q + 1], dd[4 * q + 2], dd[4 * q + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_full[0]);
    }
    if (ok && total > 0 && !warp_wait(&bars->done, 0, abort, a.err, 0x48)) ok = false;
    // dV^T and dK^T: TMEM lane = head dim d, column = key; for D=64 lanes
    // 64-127 repeat 0-63
    if (ok && (D == 128 || quarter < 2)) {
      tc_fence_after();
      const int d = quarter * 32 + lane;
      const size_t kv0 = ((size_t)b * a.Hkv + hk) * a.Skv + (size_t)j * BKV;
      for (int which = 0; which < 2; ++which) {
        uint32_t r0[32], r1[32];
        if (total > 0) {
          const uint32_t col = which == 0 ? C::COL_DV : C::COL_DK;
          tmem_ld32(lane_base + col, r0);
          tmem_ld32(lane_base + col + 32, r1);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) r0[c] = r1[c] = 0u;
        }
        const float mul = which == 0 ? 1.f : a.scale;
        __nv_bfloat16 *dst = (which == 0 ? a.dv : a.dk) + kv0 * D + d;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < valid) dst[(size_t)c * D] = __float2bfloat16_rn(__uint_as_float(r0[c]) * mul);
          if (c + 32 < valid) dst[(size_t)(c + 32) * D] = __float2bfloat16_rn(__uint_as_float(r1[c]) * mul);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D>
struct DqCfg {
  // two CTAs per SM (each with its own MMA issuer, like the forward): at
  // most 256 TMEM columns and about 113 KB of shared memory each, so S and
  // dP are single TMEM buffers and the rings are short (the other CTA's
  // work fills the gaps)
  static constexpr int KST = (D == 64) ? 4 : 2;
  static constexpr int VST = (D == 64) ? 2 : 1;
  static constexpr int KV_BYTES = BKV * D * 2;
  static constexpr int Q_BYTES = BQ * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = Q_BYTES;
  static constexpr int OFF_K = 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
  static constexpr int TILE_BYTES = OFF_BAR + 256;
  static constexpr int SMEM_BYTES = TILE_BYTES;  // the base is checked for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 256;
  // S (then dS as bf16 hi/lo parts), dP, dQ
  static constexpr uint32_t COL_S = 0, COL_DP = 64, COL_DQ = 128;
};
static_assert(2 * (DqCfg<128>::SMEM_BYTES + 1024) <= 233472, "two dQ CTAs per SM");

// dS of one query row for 32 key columns as two bf16 parts: hi = bf16(dS)
// and lo = bf16(dS - hi); hi[c] and lo[c] pack columns 2c and 2c+1. The dQ
// MMA adds hi.K and lo.K. Sum_s dS(t,s) = 0, so dQ = scale sum_s dS(t,s) k_s
// cancels the keys' common part exactly; with dS rounded once to bf16 the
// rounding residue (2^-9 of sum |dS|) times that common part can dwarf dQ
// when the keys are strongly correlated, and the lo part removes it.
__device__ __forceinline__ void ds_split32(const uint32_t (&sv)[32], const uint32_t (&dp)[32], float sl2, float lse2,
                                           float dv, uint32_t m, uint32_t (&hi)[16], uint32_t (&lo)[16]) {
  const uint64_t sc2 = f2_pack(sl2, sl2), nl2 = f2_pack(-lse2, -lse2);
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), sc2, nl2), x0, x1);
    float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
    if (m != 0xffffffffu) {
      if (!((m >> (2 * c)) & 1u)) p0 = 0.f;
      if (!((m >> (2 * c + 1)) & 1u)) p1 = 0.f;
    }
    const float g0 = p0 * (__uint_as_float(dp[2 * c]) - dv), g1 = p1 * (__uint_as_float(dp[2 * c + 1]) - dv);
    const uint32_t h01 = pack_bf16x2(g0, g1);
    hi[c] = h01;
    // a bf16 widened to f32 is its bits shifted into the upper half
    lo[c] = pack_bf16x2(g0 - __uint_as_float(h01 << 16), g1 - __uint_as_float(h01 & 0xffff0000u));
  }
}

template <int D>
__global__ void __launch_bounds__(256, 2)  // 224 threads run; the bound caps registers at 128
    attn_bwd_dq_kernel(const AttnBwdArgs a, const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tdo, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv) {
  using C = DqCfg<D>;
  constexpr int KST = C::KST, VST = C::VST;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_u32 & 1023u)) & 1023u;
  uint32_t dyn_size;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_size));
  if (pad + C::TILE_BYTES > dyn_size) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrSmemLayout);
    return;
  }
  unsigned char *smem = smem_raw + pad;
  Bars *bars = reinterpret_cast<Bars *>(smem + C::OFF_BAR);
  volatile int *abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = a.Hq / a.Hkv;

  // work item as in the forward: consecutive CTAs share a kv head
  long long x = blockIdx.x;
  const int hh = (int)(x % g);
  x /= g;
  const int i = a.NQ - 1 - (int)(x % a.NQ);
  x /= a.NQ;
  const int hk = (int)(x % a.Hkv);
  const int b = (int)(x / a.Hkv);
  const int h = hk * g + hh;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars->in_full[s], 1);
      mbar_init(&bars->in_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->sd_full[0], 1);
    mbar_init(&bars->ds_full[0], 4);
    mbar_init(&bars->done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  pdl_wait();
  const bool dense = (a.kv_count == nullptr);
  const size_t keep_row = ((size_t)b * a.Hs + (a.Hs == 1 ? 0 : h)) * a.NQ + i;
  const int cnt = dense ? a.NK : a.kv_count[keep_row];
  const uint16_t *list = dense ? nullptr : a.kv_index + keep_row * a.NK;

  unsigned char *sQ = smem + C::OFF_Q;
  unsigned char *sDO = smem + C::OFF_DO;
  unsigned char *sK = smem + C::OFF_K;
  unsigned char *sV = smem + C::OFF_V;

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ producers
    // warp 0: Q, dO and the K ring; warp 6: the V ring
    if (lane == 0 && cnt > 0) {
      const bool is_k = (warp == 0);
      const int STAGES = is_k ? KST : VST;
      uint64_t *full = is_k ? bars->in_full : bars->v_full;
      uint64_t *empty = is_k ? bars->in_empty : bars->v_empty;
      unsigned char *ring = is_k ? sK : sV;
      const CUtensorMap *map = is_k ? &tk : &tv;
      tma_prefetch_desc(map);
      if (is_k) {
        tma_prefetch_desc(&tq);
        tma_prefetch_desc(&tdo);
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::Q_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(sQ + c * BQ * 128, &tq, &bars->kv_full, c * 64, i * BQ, b * a.Hq + h);
          tma_load_3d(sDO + c * BQ * 128, &tdo, &bars->kv_full, c * 64, i * BQ, b * a.Hq + h);
        }
      }
      int issued = 0;
      int j_next = dense ? 0 : (int)list[0];
      for (int n = 0; n < cnt; ++n) {
        const int st = n % STAGES;
        const int j = j_next;
        if (n + 1 < cnt) j_next = dense ? n + 1 : (int)list[n + 1];
        if (n >= STAGES && !mbar_wait(&empty[st], ((n / STAGES) - 1) & 1, abort, a.err, is_k ? 0x50 : 0x51)) break;
        mbar_arrive_expect_tx(&full[st], C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(ring + st * C::KV_BYTES + c * BKV * 128, map, &full[st], c * 64, j * BKV, b * a.Hkv + hk);
        issued = n + 1;
      }
      if (*abort) {
        int never = 0;
        if (is_k) mbar_wait(&bars->kv_full, 0, &never, a.err, 0x52);
        for (int n = (issued > STAGES ? issued - STAGES : 0); n < issued; ++n)
          mbar_wait(&full[n % STAGES], (n / STAGES) & 1, &never, a.err, 0x52);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    // per kept tile: S and dP, then (once the compute warps have written dS
    // over S) dQ += dS_hi K + dS_lo K; a ring stage is committed only when a
    // later tile reuses it
    if (lane == 0 && cnt > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BQ, BKV, 0, 0);
      constexpr uint32_t idQ = idesc_bf16_f32(BQ, D, 0, 1);  // dQ += dS K: B = K_j MN-major
      const uint64_t dQk = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dDOk = smem_desc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dKm = smem_desc_sw128(smem_u32(sK), BKV * 128, 1024);
      bool ok = mbar_wait(&bars->kv_full, 0, abort, a.err, 0x53);
      for (int n = 0; ok && n < cnt; ++n) {
        const int sk = n % KST, sv = n % VST;
        if (!mbar_wait(&bars->in_full[sk], (n / KST) & 1, abort, a.err, 0x54) ||
            !mbar_wait(&bars->v_full[sv], (n / VST) & 1, abort, a.err, 0x55))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_q = (kk / 4) * (BQ * 128) + (kk % 4) * 32;
          const uint32_t off_k = sk * C::KV_BYTES + (kk / 4) * (BKV * 128) + (kk % 4) * 32;
          umma_bf16_ss(tmem + C::COL_S, dQk + (off_q >> 4), dK + (off_k >> 4), idS, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_q = (kk / 4) * (BQ * 128) + (kk % 4) * 32;
          const uint32_t off_v = sv * C::KV_BYTES + (kk / 4) * (BKV * 128) + (kk % 4) * 32;
          umma_bf16_ss(tmem + C::COL_DP, dDOk + (off_q >> 4), dV + (off_v >> 4), idS, kk > 0);
        }
        umma_commit(&bars->sd_full[0]);
        if (n + VST < cnt) umma_commit(&bars->v_empty[sv]);
        if (!mbar_wait(&bars->ds_full[0], n & 1, abort, a.err, 0x56)) break;
        tc_fence_after();
        // dS of keys 32h..32h+31: hi parts in S columns [32h, 32h+16), lo
        // parts in [32h+16, 32h+32); k-step kk covers keys 16kk..16kk+15
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t bk = dKm + ((sk * C::KV_BYTES + kk * 2048) >> 4);
          const uint32_t a_hi = tmem + C::COL_S + (uint32_t)((kk / 2) * 32 + (kk % 2) * 8);
          umma_bf16_ts(tmem + C::COL_DQ, a_hi, bk, idQ, (n > 0 || kk > 0) ? 1u : 0u);
          umma_bf16_ts(tmem + C::COL_DQ, a_hi + 16, bk, idQ, 1u);
        }
        if (n + KST < cnt) umma_commit(&bars->in_empty[sk]);
      }
      umma_commit(&bars->done);
      int never = 0;
      mbar_wait(&bars->done, 0, &never, a.err, 0x57);
    }
    __syncwarp();
  } else {
    // ------------------------------------------ dS and the epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int t = i * BQ + row;
    const size_t grow = ((size_t)b * a.Hq + h) * a.Sq + t;
    float lse2, dv;
    row_stats(a.lse, a.dvec, grow, t < a.Sq, lse2, dv);
    bool ok = true;
    int j_next = (cnt > 0) ? (dense ? 0 : (int)list[0]) : 0;
    for (int n = 0; n < cnt; ++n) {
      const int j = j_next;
      if (n + 1 < cnt) j_next = dense ? n + 1 : (int)list[n + 1];
      uint32_t mcol[2];  // key columns of tile j that take part (loads hidden by the wait)
      tile_colmask(a, b, hk, j, mcol[0], mcol[1]);
      if (!warp_wait(&bars->sd_full[0], n & 1, abort, a.err, 0x58)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // two halves of 32 keys; each half's dS parts go over that half's S
      // columns (already read)
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t sv[32], dp[32];
        tmem_ld32(lane_base + C::COL_S + half * 32, sv);
        tmem_ld32(lane_base + C::COL_DP + half * 32, dp);
        tmem_wait_ld();
        uint32_t dh[16], dl[16];
        ds_split32(sv, dp, a.scale_log2, lse2, dv, mcol[half], dh, dl);
        tmem_st16(lane_base + C::COL_S + half * 32, dh);
        tmem_st16(lane_base + C::COL_S + half * 32 + 16, dl);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_full[0]);
    }
    if (ok && cnt > 0 && !warp_wait(&bars->done, 0, abort, a.err, 0x59)) ok = false;
    if (ok) {
      tc_fence_after();
      __nv_bfloat16 *dst_row = a.dq + grow * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (cnt > 0) {
          tmem_ld32(lane_base + C::COL_DQ + c0, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        if (t < a.Sq) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * a.scale, __uint_as_float(o[2 * c + 1]) * a.scale);
          uint4 *dst = reinterpret_cast<uint4 *>(dst_row + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D>
cudaError_t launch_bwd_t(const AttnBwdArgs &a, const __nv_bfloat16 *out, const __nv_bfloat16 *dout,
                         const int8_t *keep, int num_sms, const CUtensorMap &tq, const CUtensorMap &tdo,
                         const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream) {
  cudaError_t e;
  // Dv
  const long long rows = (long long)a.B * a.Hq * a.Sq;
  if (rows > 0) {
    long long blocks = (rows * (D / 8) + 255) / 256;
    if (blocks > (long long)num_sms * 16) blocks = (long long)num_sms * 16;
    bwd_dvec_kernel<D><<<(int)blocks, 256, 0, stream>>>(out, dout, rows, a.dvec);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // per kv tile the query tiles that kept it
  if (keep) {
    const long long cols = (long long)a.B * a.Hs * a.NK;
    long long blocks = (cols + 7) / 8;
    if (blocks > (long long)num_sms * 8) blocks = (long long)num_sms * 8;
    if (blocks > 0) {
      keep_to_qindex_kernel<<<(int)blocks, 256, 0, stream>>>(keep, (long long)a.B * a.Hs, a.NQ, a.NK,
                                                            const_cast<int32_t *>(a.q_count),
                                                            const_cast<uint16_t *>(a.q_index));
      note_launch();
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  if ((e = set_smem(attn_bwd_dkdv_kernel<D>, DkdvCfg<D>::SMEM_BYTES)) != cudaSuccess) return e;
  if ((e = set_smem(attn_bwd_dq_kernel<D>, DqCfg<D>::SMEM_BYTES)) != cudaSuccess) return e;
  const long long kv_ctas = (long long)a.B * a.Hkv * a.NK;
  if (kv_ctas > 0) {
    e = launch_pdl(attn_bwd_dkdv_kernel<D>, dim3((unsigned)kv_ctas), dim3(kThreads), (size_t)DkdvCfg<D>::SMEM_BYTES,
                   stream, a, tq, tdo, tk, tv);
    if (e != cudaSuccess) return e;
  }
  const long long q_ctas = (long long)a.B * a.Hq * a.NQ;
  if (q_ctas > 0) {
    e = launch_pdl(attn_bwd_dq_kernel<D>, dim3((unsigned)q_ctas), dim3(kThreads), (size_t)DqCfg<D>::SMEM_BYTES,
                   stream, a, tq, tdo, tk, tv);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnBwdArgs &a, int D, const __nv_bfloat16 *out, const __nv_bfloat16 *dout,
                            const int8_t *keep, int num_sms, const CUtensorMap &tq, const CUtensorMap &tdo,
                            const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t stream) {
  if (D == 64) return launch_bwd_t<64>(a, out, dout, keep, num_sms, tq, tdo, tk, tv, stream);
  return launch_bwd_t<128>(a, out, dout, keep, num_sms, tq, tdo, tk, tv, stream);
}

}  // namespace nsa
