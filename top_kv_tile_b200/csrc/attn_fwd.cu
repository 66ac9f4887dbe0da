// attn_fwd.cu -- block-sparse flash attention forward on tcgen05 tensor cores.
//
// One CTA computes one keep row: query tile i (128 tokens) of query head h,
// visiting only the kv tiles listed for that row (ascending, from the fused
// selection or nsa_keep_to_index), as a block-sparse consumer of the
// selector's BlockSelection skips unselected tiles (flex-attention's block
// mask, attention-gym issue #56). Per kept tile j:
//   S = Q K_j^T           tcgen05.mma, M=128 N=64 K=D, bf16 -> f32 in TMEM
//   online softmax        4 warps, one query row per thread (tcgen05.ld)
//   O += P V_j            tcgen05.mma, M=128 N=D K=64, P bf16 read from TMEM
// Warp roles: lane 0 of warp 0 issues the TMA loads of Q (once) and the K
// ring, lane 0 of warp 6 those of the V ring (kv tiles addressed by the kept
// index, no multicast); a K stage is refilled as soon as its S MMA completes,
// a V stage after its PV MMA. Warp 1 owns TMEM and issues the MMAs from one
// thread, warps 2-5 run the softmax and the epilogue.
// S is double-buffered in TMEM so S(n+1) runs on the tensor core while the
// softmax of tile n runs. P(n) is written back (bf16, tcgen05.st) over the
// S(n) buffer it came from and PV(n) reads it there as its A operand, so the
// softmax never waits for the previous PV: the next S into that buffer is
// issued by the same thread after PV(n), and tcgen05.mma from one thread run
// in order. Two CTAs share an SM so one CTA's softmax overlaps the other's
// MMAs.
// The running maximum is rescaled lazily: O and l are only rescaled when the
// row maximum grows by more than 8 (log2 units), which keeps P <= 2^8 and is
// exact after the final division by l because O and l always share the same
// reference maximum.
// Optional key-token mask (the qkv_mask asked for in NATTEN issue #124
// "Arbitrary masks", with SDPA's convention that a true byte takes part): a
// second instantiation reads the 64 mask bytes of each kept tile for its kv
// head and treats a masked column like one past Skv (left out of the
// maximum, P = 0). A row whose kept keys are all masked gets O = 0 and
// lse = -inf.
// Every mbarrier wait is bounded (nsa_device.cuh); a timeout sets the
// library's device error word and the CTA drains its copies and MMAs, frees
// TMEM and exits.
#include "nsa_device.cuh"
#include "nsa_kernels.cuh"

namespace nsa {

namespace {

constexpr int BQ = 128;
constexpr int BKV = 64;
constexpr int MAX_STAGES = 4;
constexpr int kThreads = 224;  // 7 warps

template <int D>
struct Cfg {
  // ring depths that fit the 112 KB which lets two CTAs share an SM
  static constexpr int KST = (D == 64) ? 4 : 3;
  static constexpr int VST = (D == 64) ? 4 : 2;
  static constexpr int Q_BYTES = BQ * D * 2;
  static constexpr int KV_BYTES = BKV * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int TILE_BYTES = OFF_BAR + BAR_BYTES;
  static constexpr int SMEM_BYTES = TILE_BYTES;
  static constexpr uint32_t TMEM_COLS = 256;  // S/P 0 [0,64), S/P 1 [64,128), O [128,128+D)
  static constexpr uint32_t COL_O = 128;
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[MAX_STAGES];
  uint64_t k_empty[MAX_STAGES];
  uint64_t v_full[MAX_STAGES];
  uint64_t v_empty[MAX_STAGES];
  uint64_t s_full[2];
  // Tile n's P arrives on p_full[n & 1]: the softmax may finish tiles n and
  // n+1 before the MMA thread waits for P(n) (S(n+1) is issued first), never
  // n+2, so alternating barriers keep the parity waits unambiguous.
  uint64_t p_full[2];
  // PV(n) completes o_done[n & 1]. The softmax waits on these only to
  // rescale O and in the epilogue; by then PV(n-2) is known complete (S(n)
  // completing implies every earlier MMA of the issuing thread completed), so
  // two alternating barriers keep each parity wait unambiguous.
  uint64_t o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

template <int D, bool KMASK>
__global__ void __launch_bounds__(kThreads, 2)
    attn_fwd_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tq,
                    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
  using C = Cfg<D>;
  constexpr int KST = C::KST, VST = C::VST;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 128-byte swizzled operand tiles need 1024-byte aligned bases
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

  // work item: query tiles in descending order, so that where the kept
  // count grows with the tile index (a drop rule forbidding the future) the
  // long rows start first. Consecutive CTAs are the query heads of one kv
  // group. With q_first the query tile is the slowest index: the longest
  // rows of every head and batch start in the first wave and the short
  // ones fill the last (grids of few waves, where the tail counts).
  // Otherwise the query tile comes next after the head in the group, so
  // the resident CTAs share one kv head's K and V in L2.
  long long x = blockIdx.x;
  const int hh = (int)(x % g);
  x /= g;
  int i, hk, b;
  if (a.q_first) {
    hk = (int)(x % a.Hkv);
    x /= a.Hkv;
    b = (int)(x % a.B);
    i = a.NQ - 1 - (int)(x / a.B);
  } else {
    i = a.NQ - 1 - (int)(x % a.NQ);
    x /= a.NQ;
    hk = (int)(x % a.Hkv);
    b = (int)(x / a.Hkv);
  }
  const int h = hk * g + hh;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < MAX_STAGES; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full[0], 1);
    mbar_init(&bars->s_full[1], 1);
    mbar_init(&bars->p_full[0], 4);  // one elected arrive per softmax warp
    mbar_init(&bars->p_full[1], 4);
    mbar_init(&bars->o_done[0], 1);
    mbar_init(&bars->o_done[1], 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // everything above overlaps the previous kernel's tail; the kept lists and
  // the dense flag are that kernel's outputs
  pdl_wait();
  bool dense = (a.kv_count == nullptr);
  if (!dense && a.dense_if_zero != nullptr && *a.dense_if_zero == 0u) dense = true;
  const size_t keep_row = ((size_t)b * a.Hs + (a.Hs == 1 ? 0 : h)) * a.NQ + i;
  const int cnt = dense ? a.NK : a.kv_count[keep_row];
  const uint16_t *list = dense ? nullptr : a.kv_index + keep_row * a.NK;


  unsigned char *sQ = smem + C::OFF_Q;
  unsigned char *sK = smem + C::OFF_K;
  unsigned char *sV = smem + C::OFF_V;

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ producers
    // warp 0 streams Q and the K ring, warp 6 the V ring: a K stage is
    // refilled as soon as its S MMA has completed, a V stage after its PV MMA
    if (lane == 0 && cnt > 0) {
      const bool is_k = (warp == 0);
      const int STAGES = is_k ? KST : VST;
      uint64_t *full = is_k ? bars->k_full : bars->v_full;
      uint64_t *empty = is_k ? bars->k_empty : bars->v_empty;
      unsigned char *ring = is_k ? sK : sV;
      const CUtensorMap *map = is_k ? &tk : &tv;
      tma_prefetch_desc(map);
      if (is_k) {
        tma_prefetch_desc(&tq);
        mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sQ + c * BQ * 128, &tq, &bars->q_full, c * 64, i * BQ, b * a.Hq + h);
      }
      int issued = 0;
      int j_next = dense ? 0 : (int)list[0];
      for (int n = 0; n < cnt; ++n) {
        const int st = n % STAGES;
        const int j = j_next;
        // next index read ahead, its latency hidden behind the ring wait
        if (n + 1 < cnt) j_next = dense ? n + 1 : (int)list[n + 1];
        if (n >= STAGES && !mbar_wait(&empty[st], ((n / STAGES) - 1) & 1, abort, a.err, is_k ? 2 : 3)) break;
        mbar_arrive_expect_tx(&full[st], C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(ring + st * C::KV_BYTES + c * BKV * 128, map, &full[st], c * 64, j * BKV, b * a.Hkv + hk);
        issued = n + 1;
      }
      if (*abort) {
        // wait (bounded, ignoring the abort flag) for copies still in flight
        int never = 0;
        if (is_k) mbar_wait(&bars->q_full, 0, &never, a.err, 4);
        for (int n = (issued > STAGES ? issued - STAGES : 0); n < issued; ++n)
          mbar_wait(&full[n % STAGES], (n / STAGES) & 1, &never, a.err, 4);
      }
    }
    // lanes 1-31 wait here for lane 0, so the whole warp reaches the final
    // CTA barrier together (bar.sync is warp-aligned)
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0 && cnt > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BQ, BKV, 0, 0);
      constexpr uint32_t idPV = idesc_bf16_f32(BQ, D, 0, 1);
      // descriptors of the tile bases; a byte offset o is added as o >> 4 to
      // the 14-bit start-address field (shared addresses stay below 256 KB)
      const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = smem_desc_sw128(smem_u32(sV), BKV * 128, 1024);
      auto issue_s = [&](int n) {
        const int st = n % KST;
        const uint32_t d_tmem = tmem + (uint32_t)((n & 1) * BKV);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off_q = (kk / 4) * (BQ * 128) + (kk % 4) * 32;
          const uint32_t off_k = st * C::KV_BYTES + (kk / 4) * (BKV * 128) + (kk % 4) * 32;
          umma_bf16_ss(d_tmem, dq + (off_q >> 4), dk + (off_k >> 4), idS, kk > 0);
        }
        umma_commit(&bars->s_full[n & 1]);
        umma_commit(&bars->k_empty[st]);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort, a.err, 5) && mbar_wait(&bars->k_full[0], 0, abort, a.err, 8);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        for (int n = 0; n < cnt; ++n) {
          if (n + 1 < cnt) {
            const int st1 = (n + 1) % KST;
            if (!mbar_wait(&bars->k_full[st1], ((n + 1) / KST) & 1, abort, a.err, 8)) break;
            tc_fence_after();
            issue_s(n + 1);
          }
          const int st = n % VST;
          if (!mbar_wait(&bars->p_full[n & 1], (n >> 1) & 1, abort, a.err, 7)) break;
          if (!mbar_wait(&bars->v_full[st], (n / VST) & 1, abort, a.err, 9)) break;
          tc_fence_after();
          // A = P(n) in TMEM over the S(n) buffer, B = V_j (MN-major)
          const uint32_t p_tmem = tmem + (uint32_t)((n & 1) * BKV);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            umma_bf16_ts(tmem + C::COL_O, p_tmem + kk * 8, dv + ((st * C::KV_BYTES + kk * 2048) >> 4), idPV,
                         (n > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->v_empty[st]);
          umma_commit(&bars->o_done[n & 1]);
        }
      }
      // every MMA this thread issued has completed before TMEM is released
      umma_commit(&bars->drain);
      int never = 0;
      mbar_wait(&bars->drain, 0, &never, a.err, 10);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------- softmax and epilogue
    // (warps 2-5; warps 0, 1 and 6 are taken above)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // TMEM lane == query row in the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int tok = i * BQ + row;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    int j_next = (cnt > 0) ? (dense ? 0 : (int)list[0]) : 0;
    const int8_t *mrow = KMASK ? a.kmask + b * a.ks[0] + hk * a.ks[1] : nullptr;
    for (int n = 0; n < cnt; ++n) {
      const int buf = n & 1;
      const int j = j_next;
      if (n + 1 < cnt) j_next = dense ? n + 1 : (int)list[n + 1];
      // key-token mask of tile j: lane c reads the bytes of columns c and
      // c + 32 (issued before the S wait, which hides their latency)
      bool t0 = true, t1 = true;
      if constexpr (KMASK) {
        const long long s0 = (long long)j * BKV + lane, s1 = s0 + 32;
        t0 = s0 < a.Skv && mrow[s0 * a.ks[2]] != 0;
        t1 = s1 < a.Skv && mrow[s1 * a.ks[2]] != 0;
      }
      if (!warp_wait(&bars->s_full[buf], (n >> 1) & 1, abort, a.err, 11)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(lane_base + buf * BKV, r0);
      tmem_ld32(lane_base + buf * BKV + 32, r1);
      tmem_wait_ld();
      const int valid = min(BKV, a.Skv - j * BKV);  // < 64 only on a partial last kv tile
      // with a key mask: bit c of mlo / mhi = column c / c + 32 takes part
      // (inside Skv and unmasked); the same for every row of the tile
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      bool all_in = valid >= BKV;
      if constexpr (KMASK) {
        mlo = __ballot_sync(0xffffffffu, t0);
        mhi = __ballot_sync(0xffffffffu, t1);
        all_in = (mlo & mhi) == 0xffffffffu;
      }
      // row max of the raw scores (scale_log2 > 0, so the scaled max is the
      // max times the scale), as an 8-way tree
      float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (all_in) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          mp[c & 3] = fmax3(mp[c & 3], __uint_as_float(r0[c]), __uint_as_float(r1[c]));
      } else if (KMASK) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if ((mlo >> c) & 1u) mp[c & 3] = fmaxf(mp[c & 3], __uint_as_float(r0[c]));
          if ((mhi >> c) & 1u) mp[c & 3] = fmaxf(mp[c & 3], __uint_as_float(r1[c]));
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < valid) mp[c & 3] = fmaxf(mp[c & 3], __uint_as_float(r0[c]));
          if (c + 32 < valid) mp[c & 3] = fmaxf(mp[c & 3], __uint_as_float(r1[c]));
        }
      }
      const float mraw = fmaxf(fmax3(mp[0], mp[1], mp[2]), mp[3]);
      const float mx = mraw * a.scale_log2;
      // new reference maximum; the rescale decision is warp-uniform because
      // tcgen05.ld/st are warp-collective
      // (the first tile's maximum is -inf only when a key mask removes every
      // column; m then stays -inf, P and O stay 0, and the first tile with a
      // column taking part rescales O and l by 2^-inf = 0)
      float m_new = m;
      bool rescale = false;
      if (n == 0) {
        m_new = mx;
      } else if (__any_sync(0xffffffffu, mx > m + 8.0f)) {
        m_new = fmaxf(m, mx);
        rescale = true;
      }
      const float neg_m = (m_new == -INFINITY) ? 0.f : -m_new;
      // x = s * scale_log2 - m in f32x2 pairs, then p = 2^x
      const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), nm2 = f2_pack(neg_m, neg_m);
      uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float x0, x1, x2, x3;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(r0[2 * c]), __uint_as_float(r0[2 * c + 1])), sc2, nm2), x0, x1);
        f2_unpack(f2_fma(f2_pack(__uint_as_float(r1[2 * c]), __uint_as_float(r1[2 * c + 1])), sc2, nm2), x2, x3);
        float p0 = fast_exp2(x0), p1 = fast_exp2(x1), p2 = fast_exp2(x2), p3 = fast_exp2(x3);
        if (!all_in) {
          if constexpr (KMASK) {
            if (!((mlo >> (2 * c)) & 1u)) p0 = 0.f;
            if (!((mlo >> (2 * c + 1)) & 1u)) p1 = 0.f;
            if (!((mhi >> (2 * c)) & 1u)) p2 = 0.f;
            if (!((mhi >> (2 * c + 1)) & 1u)) p3 = 0.f;
          } else {
            if (2 * c >= valid) p0 = 0.f;
            if (2 * c + 1 >= valid) p1 = 0.f;
            if (2 * c + 32 >= valid) p2 = 0.f;
            if (2 * c + 33 >= valid) p3 = 0.f;
          }
        }
        acc0 = f2_add(acc0, f2_pack(p0, p1));
        acc1 = f2_add(acc1, f2_pack(p2, p3));
        pk[c] = pack_bf16x2(p0, p1);
        pk[c + 16] = pack_bf16x2(p2, p3);
      }
      float s0, s1, s2, s3;
      f2_unpack(acc0, s0, s1);
      f2_unpack(acc1, s2, s3);
      const float rs = (s0 + s1) + (s2 + s3);
      if (rescale) {
        // O may only be rescaled once PV(n-1) has completed
        if (!warp_wait(&bars->o_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort, a.err, 12)) {
          ok = false;
          break;
        }
        const float alpha = fast_exp2(m - m_new);
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + C::COL_O + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(lane_base + C::COL_O + c0, o);
        }
        l *= alpha;
      }
      m = m_new;
      l += rs;
      // P(n) over the first 32 columns of its own S buffer (already read)
      tmem_st32(lane_base + buf * BKV, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[n & 1]);
    }
    // epilogue
    if (ok && cnt > 0 && !warp_wait(&bars->o_done[(cnt - 1) & 1], ((cnt - 1) >> 1) & 1, abort, a.err, 13)) ok = false;
    if (ok) {
      tc_fence_after();
      const size_t orow = ((size_t)b * a.Hq + h) * a.Sq + tok;
      if (cnt == 0) {
        if (tok < a.Sq) {
          uint4 z = make_uint4(0, 0, 0, 0);
          uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * D);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dst[c] = z;
          a.lse[orow] = -INFINITY;
        }
      } else {
        // l == 0: every kept key of the row masked out (O = 0, lse = -inf)
        const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + C::COL_O + c0, o);
          tmem_wait_ld();
          if (tok < a.Sq) {
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
              w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
            uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * D + c0);
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
          }
        }
        if (tok < a.Sq) a.lse[orow] = (l > 0.f) ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, bool KMASK>
cudaError_t launch_t(const AttnArgs &a, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     cudaStream_t stream) {
  const int smem = Cfg<D>::SMEM_BYTES;
  cudaError_t e =
      cudaFuncSetAttribute(attn_fwd_kernel<D, KMASK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long ctas = (long long)a.B * a.Hq * a.NQ;
  if (ctas == 0) return cudaSuccess;
  return launch_pdl(attn_fwd_kernel<D, KMASK>, dim3((unsigned)ctas), dim3(kThreads), (size_t)smem, stream, a, tq,
                    tk, tv);
}

}  // namespace

size_t attn_smem_bytes(int D) { return D == 64 ? Cfg<64>::SMEM_BYTES : Cfg<128>::SMEM_BYTES; }

cudaError_t launch_attn_fwd(const AttnArgs &a, int D, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, cudaStream_t stream) {
  if (a.kmask) return D == 64 ? launch_t<64, true>(a, tq, tk, tv, stream) : launch_t<128, true>(a, tq, tk, tv, stream);
  return D == 64 ? launch_t<64, false>(a, tq, tk, tv, stream) : launch_t<128, false>(a, tq, tk, tv, stream);
}

cudaError_t launch_attn_fwd(const AttnArgs &a, int D, int num_sms, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, cudaStream_t stream) {
  // query-tile-first order for grids of at most 16 waves (two CTAs per SM)
  AttnArgs b = a;
  const long long ctas = (long long)a.B * a.Hq * a.NQ;
  b.q_first = ctas <= 16LL * 2 * num_sms ? 1 : 0;
  return launch_attn_fwd(b, D, tq, tk, tv, stream);
}

}  // namespace nsa
