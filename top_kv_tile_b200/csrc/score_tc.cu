// score_tc.cu -- the unscaled pooled scores S = pq . pk^T (score_blocks in
// automatic/modules/attention/sparse/selector.py) on tcgen05 tensor cores,
// for rows too long to keep the pooled keys resident next to the scoring
// CTA (the Large-2D workload: 2048 kv tiles, 34 GFLOP per step).
//
// The operands are float32; the tensor cores multiply tf32 (10 explicit
// mantissa bits). Each operand is split as x = hi + lo with hi = tf32(x) and
// lo = tf32(x - hi), and S = hi_q.hi_k + hi_q.lo_k + lo_q.hi_k is accumulated
// in f32 (the error-compensated split of Ootomo & Yokota, "Recovering single
// precision accuracy from Tensor Cores while surpassing the FP32 theoretical
// peak performance", 2022); the dropped lo.lo term and the roundings leave a
// relative error near 2^-21 per product, the size of float32 FMA rounding.
//
// The pooled keys of every kv head are split once (split_tf32_kernel) into
// two float32 arrays laid out like pk. One CTA then takes 128 pooled query
// rows (M) of one keep head: its epilogue warps split those rows and store
// hi and lo in TMEM, where they are the A operand of every MMA, so the
// whole shared memory holds key tiles. The keys stream in by TMA in chunks
// of 256 kv tiles (N = 256: one MMA instruction does four times the work of
// an N = 64 one, and issuing MMAs, not executing them, is what bounds a
// single issuing thread; chunks of 64 when 256-wide ones would leave SMs
// idle), one 32-element segment of the head dimension (hi and lo) per ring
// stage. Per segment 4 K-steps x 3 products go into an N-column f32
// accumulator in TMEM; the epilogue warps (one query row
// per thread) copy each finished chunk to the score scratch and free the
// accumulator for the next chunk. Every wait is bounded.
#include <algorithm>

#include "nsa_device.cuh"
#include "nsa_kernels.cuh"

namespace nsa {

namespace {

constexpr int TM = 128;   // query rows per CTA (the MMA's M)
constexpr int KSEG = 32;  // f32 elements of D per 128-byte row
constexpr int KST = 3;    // ring stages
constexpr int kTcThreads = 192;  // 6 warps
constexpr uint32_t COL_QHI = 0, COL_QLO = 128, COL_ACC = 256, TMEM_COLS = 512;

// TN kv tiles per chunk (the MMA's N): 256 normally; 64 when the grid would
// otherwise not cover the SMs (a few row blocks and short rows).
template <int TN>
struct TcCfg {
  static constexpr int SEG_BYTES = TN * 128;         // one D segment of a chunk, hi or lo
  static constexpr int STAGE_BYTES = 2 * SEG_BYTES;  // hi, then lo
  static constexpr int OFF_BAR = KST * STAGE_BYTES;
  static constexpr int TILE_BYTES = OFF_BAR + 256;
};

struct TcBars {
  uint64_t full[KST];
  uint64_t empty[KST];
  uint64_t q_ready;    // the epilogue warps stored the split query rows (4 arrivals)
  uint64_t acc_full;   // a chunk's products completed
  uint64_t acc_empty;  // the epilogue copied the chunk out (4 arrivals)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__global__ void split_tf32_kernel(const float4 *x, long long n4, float4 *hi, float4 *lo) {
  pdl_wait();  // the pooled keys come from the previous kernel
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 v = x[i];
    float4 h, l;
    h.x = __uint_as_float(to_tf32(v.x));
    h.y = __uint_as_float(to_tf32(v.y));
    h.z = __uint_as_float(to_tf32(v.z));
    h.w = __uint_as_float(to_tf32(v.w));
    l.x = __uint_as_float(to_tf32(v.x - h.x));
    l.y = __uint_as_float(to_tf32(v.y - h.y));
    l.z = __uint_as_float(to_tf32(v.z - h.z));
    l.w = __uint_as_float(to_tf32(v.w - h.w));
    hi[i] = h;
    lo[i] = l;
  }
}

template <int D, int TN>
__global__ void __launch_bounds__(kTcThreads, 1)
    score_tc_kernel(const ScoreTcArgs a, const __grid_constant__ CUtensorMap thi,
                    const __grid_constant__ CUtensorMap tlo) {
  constexpr int NSEG = D / KSEG;
  constexpr int SEG_BYTES = TcCfg<TN>::SEG_BYTES, STAGE_BYTES = TcCfg<TN>::STAGE_BYTES;
  constexpr int OFF_BAR = TcCfg<TN>::OFF_BAR, TILE_BYTES = TcCfg<TN>::TILE_BYTES;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_u32 & 1023u)) & 1023u;
  uint32_t dyn_size;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_size));
  if (pad + TILE_BYTES > dyn_size) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrSmemLayout);
    return;
  }
  unsigned char *smem = smem_raw + pad;
  TcBars *bars = reinterpret_cast<TcBars *>(smem + OFF_BAR);
  volatile int *abort = &bars->abort;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const int rb = blockIdx.x, hs = blockIdx.y;
  const int b = blockIdx.z / a.nsplit, sp = blockIdx.z % a.nsplit;
  const int hk = hs / (a.Hq / a.Hkv);
  const int nchunks = (a.NK + TN - 1) / TN;
  const int per = (nchunks + a.nsplit - 1) / a.nsplit;
  const int c0 = sp * per, c1 = min(nchunks, c0 + per);

  if (threadIdx.x == 0) {
    for (int s = 0; s < KST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->q_ready, 4);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 4);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  pdl_wait();  // the pooled vectors and their split come from the previous kernels

  if (warp == 0) {
    // ----------------------------------------------------------- producer
    if (lane == 0 && c0 < c1) {
      tma_prefetch_desc(&thi);
      tma_prefetch_desc(&tlo);
      int it = 0;
      for (int c = c0; c < c1 && !*abort; ++c) {
        for (int sg = 0; sg < NSEG; ++sg, ++it) {
          const int st = it % KST;
          if (it >= KST && !mbar_wait(&bars->empty[st], ((it / KST) - 1) & 1, abort, a.err, 0x60)) break;
          mbar_arrive_expect_tx(&bars->full[st], STAGE_BYTES);
          unsigned char *dst = smem + st * STAGE_BYTES;
          tma_load_3d(dst, &thi, &bars->full[st], sg * KSEG, c * TN, b * a.Hkv + hk);
          tma_load_3d(dst + SEG_BYTES, &tlo, &bars->full[st], sg * KSEG, c * TN, b * a.Hkv + hk);
        }
      }
      if (*abort) {
        // wait (bounded, ignoring the abort flag) for copies still in flight
        int never = 0;
        for (int m = (it > KST ? it - KST : 0); m < it; ++m)
          mbar_wait(&bars->full[m % KST], (m / KST) & 1, &never, a.err, 0x61);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0 && c0 < c1) {
      constexpr uint32_t idesc = idesc_tf32_f32(TM, TN);
      const uint64_t dk = smem_desc_sw128(smem_u32(smem), 16, 1024);
      bool ok = mbar_wait(&bars->q_ready, 0, abort, a.err, 0x62);
      int it = 0;
      for (int c = c0; ok && c < c1; ++c) {
        if (c > c0 && !mbar_wait(&bars->acc_empty, (c - c0 - 1) & 1, abort, a.err, 0x63)) {
          ok = false;
          break;
        }
        for (int sg = 0; sg < NSEG; ++sg, ++it) {
          const int st = it % KST;
          if (!mbar_wait(&bars->full[st], (it / KST) & 1, abort, a.err, 0x64)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dhi = dk + ((uint64_t)(st * STAGE_BYTES) >> 4);
          const uint64_t dlo = dhi + ((uint64_t)SEG_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < KSEG / 8; ++kk) {
            const uint32_t qc = (uint32_t)(sg * KSEG + kk * 8);
            const uint64_t ko = (uint64_t)((kk * 32) >> 4);
            umma_tf32_ts(tmem + COL_ACC, tmem + COL_QHI + qc, dhi + ko, idesc, (sg > 0 || kk > 0) ? 1u : 0u);
            umma_tf32_ts(tmem + COL_ACC, tmem + COL_QHI + qc, dlo + ko, idesc, 1u);
            umma_tf32_ts(tmem + COL_ACC, tmem + COL_QLO + qc, dhi + ko, idesc, 1u);
          }
          umma_commit(&bars->empty[st]);
        }
        if (!ok) break;
        umma_commit(&bars->acc_full);
      }
      // every product has completed before TMEM is released
      umma_commit(&bars->drain);
      int never = 0;
      mbar_wait(&bars->drain, 0, &never, a.err, 0x65);
    }
    __syncwarp();
  } else {
    // ------------------------------------- query split and score epilogue
    // (warps 2-5: TMEM lane quarter warp & 3, one query row per thread)
    const int quarter = warp & 3, row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int i = rb * TM + row;
    const float *qrow = a.pq + (((size_t)b * a.Hq + hs) * a.NQ + (i < a.NQ ? i : 0)) * D;
#pragma unroll
    for (int s0 = 0; s0 < D; s0 += 32) {
      uint32_t h[32], l[32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 v = i < a.NQ ? *reinterpret_cast<const float4 *>(qrow + s0 + 4 * u)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          h[4 * u + e] = to_tf32(vv[e]);
          l[4 * u + e] = to_tf32(vv[e] - __uint_as_float(h[4 * u + e]));
        }
      }
      tmem_st32(lane_base + COL_QHI + s0, h);
      tmem_st32(lane_base + COL_QLO + s0, l);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->q_ready);
    for (int c = c0; c < c1; ++c) {
      if (!warp_wait(&bars->acc_full, (c - c0) & 1, abort, a.err, 0x66)) break;
      tc_fence_after();
      float *dst = a.scores + (((size_t)b * a.Hq + hs) * a.NQ + i) * a.NKP;
#pragma unroll 2
      for (int part = 0; part < TN / 32; ++part) {
        uint32_t r[32];
        tmem_ld32(lane_base + COL_ACC + part * 32, r);
        tmem_wait_ld();
        const int col = c * TN + part * 32;
        if (i < a.NQ && col < a.NKP) {
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + col);
#pragma unroll
          for (int q = 0; q < 8; ++q) d4[q] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace

size_t score_tc_smem(int D) {
  (void)D;
  return (size_t)TcCfg<256>::TILE_BYTES;
}

cudaError_t launch_split_tf32(const float *x, long long n, float *hi, float *lo, int num_sms, cudaStream_t stream) {
  const long long n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  long long blocks = (n4 + 255) / 256;
  if (blocks > (long long)num_sms * 8) blocks = (long long)num_sms * 8;
  return launch_pdl(split_tf32_kernel, dim3((unsigned)blocks), dim3(256), 0, stream,
                    reinterpret_cast<const float4 *>(x), n4, reinterpret_cast<float4 *>(hi),
                    reinterpret_cast<float4 *>(lo));
}

namespace {

template <int D, int TN>
cudaError_t launch_tc_t(ScoreTcArgs a, const CUtensorMap &thi, const CUtensorMap &tlo, int num_sms,
                        cudaStream_t stream) {
  const int nchunks = (a.NK + TN - 1) / TN;
  const long long blocks = (long long)((a.NQ + TM - 1) / TM) * a.Hq * a.B;
  if (blocks == 0 || nchunks == 0) return cudaSuccess;
  // few row blocks: split the kv range so the grid covers the device
  a.nsplit = (int)std::min<long long>(nchunks, std::max<long long>(1, (num_sms + blocks - 1) / blocks));
  const dim3 grid((unsigned)((a.NQ + TM - 1) / TM), (unsigned)a.Hq, (unsigned)(a.B * a.nsplit));
  const int smem = TcCfg<TN>::TILE_BYTES;
  cudaError_t e =
      cudaFuncSetAttribute(score_tc_kernel<D, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(score_tc_kernel<D, TN>, grid, dim3(kTcThreads), (size_t)smem, stream, a, thi, tlo);
}

}  // namespace

int score_tc_chunk(int B, int Hq, int NQ, int NK, int num_sms) {
  // N = 256 when row blocks x 256-wide chunks cover the SMs, else N = 64
  const long long blocks = (long long)((NQ + TM - 1) / TM) * Hq * B;
  return blocks * ((NK + 255) / 256) >= num_sms ? 256 : 64;
}

cudaError_t launch_score_tc(ScoreTcArgs a, const CUtensorMap &thi, const CUtensorMap &tlo, int num_sms,
                            cudaStream_t stream) {
  const bool wide = score_tc_chunk(a.B, a.Hq, a.NQ, a.NK, num_sms) == 256;
  if (a.D == 64)
    return wide ? launch_tc_t<64, 256>(a, thi, tlo, num_sms, stream) : launch_tc_t<64, 64>(a, thi, tlo, num_sms, stream);
  return wide ? launch_tc_t<128, 256>(a, thi, tlo, num_sms, stream)
              : launch_tc_t<128, 64>(a, thi, tlo, num_sms, stream);
}

}  // namespace nsa
