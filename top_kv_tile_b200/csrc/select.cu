// select.cu -- fused pooled scoring, selection plan and fixed-budget top-k
// (selector.py: score_blocks, selection_plan, select_blocks), the head mean
// of pooled tensors for head-shared scoring, and the keep -> compacted index
// list kernel.
//
// One CTA owns R consecutive query tiles (rows) of one (batch, keep head).
//  1. Scores: S[r, j] = <pq'[r], pk'[j]> in float32 FMA over the pooled
//     vectors (GQA: query head h reads key head h / group). The R x NK score
//     rows stay in shared memory: the (B,Hs,NQ,NK) score tensor is never
//     written to HBM. Key rows sit in shared memory with their 16-byte chunks
//     XOR-swizzled by (row / 4) mod 8. A warp computes a 4-row x 32-column
//     tile: lane 8 dq + cl holds the 4 x 4 block of columns 4 cl .. 4 cl + 3
//     over the feature chunks congruent to dq mod 4, so each loaded key value
//     feeds four rows and each query value four columns; the four partial
//     sums are added across lanes at the end. Two staging schemes:
//       - "resident" (NK*D*4 <= 64 KB): every pooled key row of the head is
//         copied into shared memory in one cp.async round;
//       - "chunked" (larger NK, up to 8192): 32 KB chunks of key rows pass
//         through a double-buffered cp.async ring, the next chunk loading
//         while the current one is scored.
//     Head-shared scoring (means over heads) runs on pre-averaged tensors
//     (head_mean_kernel); the chunked path can also average while staging
//     (the raw-score entry point, which has no workspace).
//  2. Plan per row: must = diagonal | pin, forbidden = drop, candidate =
//     ~must & ~forbidden, c = #candidates, k = ceil(f32(c) * f32(budget))
//     evaluated in float32 (round-to-nearest multiply), as torch evaluates the
//     page's int64 tensor times a Python float.
//  3. Top-k: candidate scores become order-preserving 32-bit keys (larger
//     float -> larger key, -0 == +0, every finite candidate key >= 1, non
//     candidates 0). One warp per row finds the k-th largest key T (rows
//     of up to 256 tiles: a bitonic sort of the keys across the warp;
//     longer rows: repeated 256-bin bucketing of the keys' range), then keeps every
//     key > T and the lowest-index keys == T up to k: exactly the stable
//     descending argsort's first k, ties to the lower kv index. Rows of up to 2048 tiles keep
//     their keys in registers; longer rows keep them in shared memory.
//  4. keep = (must & ~forbidden) | selected, written as int8, plus the
//     ascending compacted index list and its count.
#include <algorithm>

#include "nsa_device.cuh"
#include "nsa_kernels.cuh"

namespace nsa {

namespace {

constexpr int kThreads = 256;
constexpr int kResidentBytes = 64 * 1024;
constexpr int kChunkBytes = 32 * 1024;

__device__ __forceinline__ uint32_t order_key(float s) {
  if (s == 0.0f) s = 0.0f;  // -0 and +0 tie, as in a float comparison sort
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int warp_excl_scan(int v, int lane, int *total) {
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  *total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// a[e] += the 8 bf16 values packed in v (in order), in float32
__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4 &v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    a[2 * e] += __uint_as_float(w[e] << 16);
    a[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

// The plan of one row (selection_plan): must = nominal-range overlap of the
// query tile and kv tile (no clamp to Sq / Skv) or a pin; forbidden = a drop.
struct RowPlan {
  long long jd0, jd1;  // the diagonal: kv tiles whose nominal range meets the query tile's
  const int8_t *prow, *drow, *srow;
  long long pstride, dstride;
  __device__ __forceinline__ RowPlan(const SelectArgs &a, int b, int hs, int i) {
    // j * bkv < (i + 1) * bq and i * bq < (j + 1) * bkv, in exact integers:
    // floor(i bq / bkv) <= j <= floor(((i + 1) bq - 1) / bkv)
    jd0 = (long long)i * a.block_q / a.block_kv;
    jd1 = ((long long)(i + 1) * a.block_q - 1) / a.block_kv;
    prow = a.pins ? a.pins + b * a.ps[0] + hs * a.ps[1] + i * a.ps[2] : nullptr;
    drow = a.drops ? a.drops + b * a.ds[0] + hs * a.ds[1] + i * a.ds[2] : nullptr;
    srow = a.plan_state ? a.plan_state + (b * a.plan_bs + hs * a.plan_hs + i) * (long long)a.NK : nullptr;
    pstride = a.ps[3];
    dstride = a.ds[3];
  }
  __device__ __forceinline__ bool must(int j) const {
    if (srow) return srow[j] == 1;
    return (j >= jd0 && j <= jd1) || (prow && prow[(long long)j * pstride] != 0);
  }
  __device__ __forceinline__ bool forbidden(int j) const {
    if (srow) return srow[j] == 2;
    return drow && drow[(long long)j * dstride] != 0;
  }
};

// The k-th largest (1 <= k <= 32 N) of the 32 N keys a warp holds, N per
// lane, by a bitonic sort of all of them into ascending order (element
// index lane * N + e; partners at distances below N are in the same lane,
// the others one shuffle away). The stages are unrolled at compile time
// (every array index a constant, so the keys stay in registers). Every lane
// returns the same value.
template <int N, int SIZE, int D>
struct BitonicStage {
  static __device__ __forceinline__ void run(uint32_t (&x)[N], int lane) {
    if constexpr (D >= N) {
      constexpr int ld = D / N;  // partner lane distance
      const bool lower = (lane & ld) == 0;
#pragma unroll
      for (int e = 0; e < N; ++e) {
        const bool up = ((lane * N + e) & SIZE) == 0;  // this block sorts ascending
        const uint32_t o = __shfl_xor_sync(0xffffffffu, x[e], ld);
        x[e] = (lower == up) ? min(x[e], o) : max(x[e], o);
      }
    } else {
#pragma unroll
      for (int e = 0; e < N; ++e) {
        if ((e ^ D) > e) {
          const bool up = ((lane * N + e) & SIZE) == 0;
          const uint32_t lo = min(x[e], x[e ^ D]), hi = max(x[e], x[e ^ D]);
          x[e] = up ? lo : hi;
          x[e ^ D] = up ? hi : lo;
        }
      }
    }
    if constexpr (D > 1) BitonicStage<N, SIZE, D / 2>::run(x, lane);
  }
};

template <int N, int SIZE>
__device__ __forceinline__ void bitonic_from(uint32_t (&x)[N], int lane) {
  BitonicStage<N, SIZE, SIZE / 2>::run(x, lane);
  if constexpr (SIZE < 32 * N) bitonic_from<N, SIZE * 2>(x, lane);
}

template <int N>
__device__ __forceinline__ uint32_t warp_kth_largest(uint32_t (&x)[N], int k) {
  const int lane = threadIdx.x & 31;
  bitonic_from<N, 2>(x, lane);
  // ascending order: the k-th largest sits at index 32 N - k
  const int pos = 32 * N - k;
  uint32_t v = x[0];
#pragma unroll
  for (int e = 1; e < N; ++e)
    if ((pos % N) == e) v = x[e];
  return __shfl_sync(0xffffffffu, v, pos / N);
}

// The k-th largest (1 <= k <= number of nonzero keys) of the nonzero keys a
// warp holds (4 G per lane; a key of 0 marks a tile that is not a candidate).
// Each pass divides the current key interval [lo, hi] into at most 256
// equal-width bins, counts the keys of the interval per bin (a histogram in
// the warp's slice of shared memory) and keeps the bin that holds the k-th
// largest; a bin one key wide is the exact key. The first interval is the
// keys' own range, from their minimum to their maximum: a row's scores share
// their leading bits, so bins cut from the top bits of the key would pile
// nearly every key into one bin (and its counter). Once the bin that holds
// the k-th largest has at most 32 keys, those keys are gathered and sorted
// across the warp instead of cutting the bin further. Every lane returns
// the same value.
template <int G>
__device__ __forceinline__ uint32_t warp_kth_interval(const uint32_t (&kk)[G][4], int kr, uint32_t lo, uint32_t hi) {
  __shared__ __align__(16) int hist_all[kThreads / 32][256];
  int *hist = hist_all[threadIdx.x / 32];
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  while (lo < hi) {
    // bin width 2^shift with (hi - lo) >> shift < 256
    const int shift = max(0, 24 - __clz(hi - lo));
    for (int q = lane; q < 256; q += 32) hist[q] = 0;
    __syncwarp();
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t key = kk[g][e];
        if (key >= lo && key <= hi) atomicAdd(&hist[(key - lo) >> shift], 1);
      }
    __syncwarp();
    // lane l holds bins 255 - 8 l down to 248 - 8 l (descending), read as two
    // 16-byte vectors (bins 248 - 8 l .. 255 - 8 l)
    int c8[8], sum = 0;
    {
      const int4 b0 = *reinterpret_cast<const int4 *>(hist + 248 - 8 * lane);
      const int4 b1 = *reinterpret_cast<const int4 *>(hist + 252 - 8 * lane);
      c8[0] = b1.w;
      c8[1] = b1.z;
      c8[2] = b1.y;
      c8[3] = b1.x;
      c8[4] = b0.w;
      c8[5] = b0.z;
      c8[6] = b0.y;
      c8[7] = b0.x;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) sum += c8[q];
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int excl = incl - sum;  // keys of the interval in higher bins than this lane's
    const bool mine = excl < kr && kr <= incl;
    int bin = 0, above = excl, cb = 0;
    if (mine) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (above + c8[q] >= kr) {
          bin = 255 - (lane * 8 + q);
          cb = c8[q];
          break;
        }
        above += c8[q];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    bin = __shfl_sync(0xffffffffu, bin, src);
    above = __shfl_sync(0xffffffffu, above, src);
    cb = __shfl_sync(0xffffffffu, cb, src);
    kr -= above;
    const uint32_t nlo = lo + ((uint32_t)bin << shift);
    const uint32_t width = (1u << shift) - 1u;
    hi = (hi - nlo < width) ? hi : nlo + width;
    lo = nlo;
    __syncwarp();  // every lane has read the histogram before it is reused
    if (cb <= 32 && lo < hi) {
      // the bin's keys (at most 32) into the histogram's space, one per lane,
      // then the kr-th largest of them (the zero padding sorts below them)
      int n_in = 0;
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) n_in += (kk[g][e] >= lo && kk[g][e] <= hi) ? 1 : 0;
      int tot;
      int pos = warp_excl_scan(n_in, lane, &tot);
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (kk[g][e] >= lo && kk[g][e] <= hi) hist[pos++] = (int)kk[g][e];
      __syncwarp();
      uint32_t x[1] = {lane < tot ? (uint32_t)hist[lane] : 0u};
      __syncwarp();  // every lane has read its key before the histogram is reused
      return warp_kth_largest<1>(x, kr);
    }
  }
  return lo;
}

// The kr-th largest key in [lo, hi] is the answer; the first interval is the
// keys' own range.
template <int G>
__device__ __forceinline__ uint32_t warp_kth_radix(const uint32_t (&kk)[G][4], int k) {
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (kk[g][e] != 0u) {
        lo = min(lo, kk[g][e]);
        hi = max(hi, kk[g][e]);
      }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  return warp_kth_interval<G>(kk, k, lo, hi);
}


// The row's budget count: the plan's, else ceil(f32(c) * f32(budget)).
__device__ __forceinline__ int row_budget(const SelectArgs &a, int b, int hs, int i, int c) {
  if (a.plan_k) return a.plan_k[b * a.plan_bs + hs * a.plan_hs + i];
  return (int)ceilf(__fmul_rn((float)c, a.budget));
}

// Plan + top-k + outputs with the row's keys held in registers (NKP <= 32 *
// KPL). Lane `lane` owns kv tiles j = 128 g + 4 lane + e (g < KPL / 4,
// e < 4), so a group g of the warp covers 128 consecutive tiles in lane-major
// order. Short rows count with ballots (no shared-memory traffic and no
// reduction latency in the search loop); long rows with one warp reduction
// per step.
template <int R, int KPL>
__device__ __forceinline__ void select_rows_regs(const SelectArgs &a, const float *ss, int NKP, int i0, int hs,
                                                 int b) {
  static_assert(KPL % 4 == 0 && KPL <= 64, "keys per lane");
  constexpr int G = KPL / 4;
  const int NK = a.NK, NQ = a.NQ;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r = warp; r < R; r += kThreads / 32) {
    const int i = i0 + r;
    if (i >= NQ) break;
    const RowPlan pl(a, b, hs, i);

    uint32_t kk[G][4];
    uint64_t forced = 0;  // bit 4g+e: must and not forbidden
    int c_lane = 0;
    // every load of the row first, so that they are in flight together
    float4 svs[G];
#pragma unroll
    for (int g = 0; g < G; ++g)
      // groups past the row stride NKP (a multiple of 128) hold no tiles
      svs[g] = g * 128 < NKP ? *reinterpret_cast<const float4 *>(ss + (size_t)r * NKP + g * 128 + lane * 4)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int jb = g * 128 + lane * 4;
      const float4 sv = svs[g];
      const float sa[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = jb + e;
        kk[g][e] = 0u;
        if (j < NK) {
          const bool must = pl.must(j), forb = pl.forbidden(j);
          if (must && !forb) forced |= 1ull << (4 * g + e);
          if (!must && !forb) {
            kk[g][e] = order_key(sa[e]);
            ++c_lane;
          }
        }
      }
    }
    const int c = __reduce_add_sync(0xffffffffu, c_lane);
    const int k = row_budget(a, b, hs, i, c);
    // (the flag is read first: once set, no row needs to touch it again)
    if (lane == 0 && k < c && a.not_covered && *reinterpret_cast<volatile unsigned int *>(a.not_covered) == 0u)
      atomicOr(a.not_covered, 1u);

    uint32_t T;
    int take;
    if (k <= 0) {
      T = 0xFFFFFFFFu;
      take = 0;
    } else if (k >= c) {
      T = 0u;
      take = 0;
    } else {
      // k-th largest key: the largest T with #{key >= T} >= k
      if (G <= 2) {
        // short rows: sort a copy of the keys across the warp
        uint32_t y[4 * G];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e) y[4 * g + e] = kk[g][e];
        T = warp_kth_largest<4 * G>(y, k);
      } else {
        // long rows: repeated bucketing of the key range
        T = warp_kth_radix<G>(kk, k);
      }
      int above = 0;
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) above += kk[g][e] > T ? 1 : 0;
      take = k - __reduce_add_sync(0xffffffffu, above);
    }

    // keep row, compacted list (ascending j), count
    const size_t row = ((size_t)b * a.Hs + hs) * NQ + i;
    int8_t *krow = a.keep ? a.keep + row * NK : nullptr;
    uint16_t *irow = a.kv_index ? a.kv_index + row * NK : nullptr;
    int tie_base = 0, kept_base = 0;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (g * 128 >= NKP) break;
      const int jb = g * 128 + lane * 4;
      uint32_t tb[4];
      int tie_lo = 0, tie_tot = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        tb[e] = __ballot_sync(0xffffffffu, take > 0 && kk[g][e] == T);
        tie_lo += __popc(tb[e] & lt_mask);
        tie_tot += __popc(tb[e]);
      }
      int tie_rank = tie_base + tie_lo;
      int kp[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bool sel = kk[g][e] > T && kk[g][e] != 0u;
        if ((tb[e] >> lane) & 1u) {
          sel = tie_rank < take;
          ++tie_rank;
        }
        kp[e] = (sel || ((forced >> (4 * g + e)) & 1ull)) ? 1 : 0;
      }
      int pos = kept_base, kept_tot = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t kb = __ballot_sync(0xffffffffu, kp[e] != 0);
        pos += __popc(kb & lt_mask);
        kept_tot += __popc(kb);
      }
      if (krow && (NK & 3) == 0 && (reinterpret_cast<uintptr_t>(a.keep) & 3u) == 0 && jb + 3 < NK) {
        // the lane's four keep bytes in one 4-byte store (the keep tensor is
        // 4-byte aligned and its rows, NK bytes apart, are too)
        *reinterpret_cast<uint32_t *>(krow + jb) =
            (uint32_t)kp[0] | ((uint32_t)kp[1] << 8) | ((uint32_t)kp[2] << 16) | ((uint32_t)kp[3] << 24);
      } else if (krow) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (jb + e < NK) krow[jb + e] = (int8_t)kp[e];
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = jb + e;
        if (j < NK && kp[e]) {
          if (irow) irow[pos] = (uint16_t)j;
          ++pos;
        }
      }
      tie_base += tie_tot;
      kept_base += kept_tot;
    }
    if (lane == 0 && a.kv_count) a.kv_count[row] = kept_base;
  }
}

// The same for rows longer than the register path holds: the keys replace
// the scores in shared memory (row stride NKP) and the plan bits are
// evaluated again in the output pass.
template <int R>
__device__ __forceinline__ void select_rows_smem(const SelectArgs &a, float *ss, int NKP, int i0, int hs, int b) {
  const int NK = a.NK, NQ = a.NQ;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int r = warp; r < R; r += kThreads / 32) {
    const int i = i0 + r;
    if (i >= NQ) break;
    uint32_t *key = reinterpret_cast<uint32_t *>(ss + (size_t)r * NKP);
    const RowPlan pl(a, b, hs, i);

    int c_lane = 0;
    for (int j = lane; j < NKP; j += 32) {
      uint32_t kk = 0;
      if (j < NK && !pl.must(j) && !pl.forbidden(j)) {
        kk = order_key(ss[(size_t)r * NKP + j]);
        ++c_lane;
      }
      key[j] = kk;
    }
    const int c = __reduce_add_sync(0xffffffffu, c_lane);
    const int k = row_budget(a, b, hs, i, c);
    // (the flag is read first: once set, no row needs to touch it again)
    if (lane == 0 && k < c && a.not_covered && *reinterpret_cast<volatile unsigned int *>(a.not_covered) == 0u)
      atomicOr(a.not_covered, 1u);
    __syncwarp();

    uint32_t T;
    int take;
    if (k <= 0) {
      T = 0xFFFFFFFFu;
      take = 0;
    } else if (k >= c) {
      T = 0u;
      take = 0;
    } else {
      T = 0u;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t t = T | (1u << bit);
        int cnt = 0;
        for (int j = lane * 4; j < NKP; j += 128) {
          const uint4 kv = *reinterpret_cast<const uint4 *>(&key[j]);
          cnt += (kv.x >= t) + (kv.y >= t) + (kv.z >= t) + (kv.w >= t);
        }
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        if (cnt >= k) T = t;
      }
      int above = 0;
      for (int j = lane * 4; j < NKP; j += 128) {
        const uint4 kv = *reinterpret_cast<const uint4 *>(&key[j]);
        above += (kv.x > T) + (kv.y > T) + (kv.z > T) + (kv.w > T);
      }
      take = k - __reduce_add_sync(0xffffffffu, above);
    }

    const size_t row = ((size_t)b * a.Hs + hs) * NQ + i;
    int8_t *krow = a.keep ? a.keep + row * NK : nullptr;
    uint16_t *irow = a.kv_index ? a.kv_index + row * NK : nullptr;
    int tie_base = 0, kept_base = 0;
    for (int j0 = 0; j0 < NKP; j0 += 128) {
      const int jb = j0 + lane * 4;
      const uint4 kv = *reinterpret_cast<const uint4 *>(&key[jb]);
      const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
      int tie[4], ntie = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        tie[u] = (take > 0 && kk[u] == T) ? 1 : 0;
        ntie += tie[u];
      }
      int tie_tot;
      int tie_rank = tie_base + warp_excl_scan(ntie, lane, &tie_tot);
      int kp[4], nkept = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = jb + u;
        bool sel = kk[u] > T && kk[u] != 0u;
        if (tie[u]) {
          sel = tie_rank < take;
          ++tie_rank;
        }
        const bool forced = j < NK && pl.must(j) && !pl.forbidden(j);
        kp[u] = (sel || forced) ? 1 : 0;
        nkept += kp[u];
      }
      int kept_tot;
      int pos = kept_base + warp_excl_scan(nkept, lane, &kept_tot);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = jb + u;
        if (j < NK) {
          if (krow) krow[j] = (int8_t)kp[u];
          if (kp[u]) {
            if (irow) irow[pos] = (uint16_t)j;
            ++pos;
          }
        }
      }
      tie_base += tie_tot;
      kept_base += kept_tot;
    }
    if (lane == 0 && a.kv_count) a.kv_count[row] = kept_base;
  }
}

// Selection for the CTA's rows, by row length: keys in registers for up to
// 32 * MAXKPL tiles, else in shared memory.
template <int R, int MAXKPL>
__device__ __forceinline__ void select_rows(const SelectArgs &a, float *ss, int NKP, int i0, int hs, int b) {
  if (NKP <= 128) return select_rows_regs<R, 4>(a, ss, NKP, i0, hs, b);
  if (MAXKPL >= 8 && NKP <= 256) return select_rows_regs<R, (MAXKPL >= 8 ? 8 : 4)>(a, ss, NKP, i0, hs, b);
  if (MAXKPL >= 16 && NKP <= 512) return select_rows_regs<R, (MAXKPL >= 16 ? 16 : 4)>(a, ss, NKP, i0, hs, b);
  if (MAXKPL >= 32 && NKP <= 1024) return select_rows_regs<R, (MAXKPL >= 32 ? 32 : 4)>(a, ss, NKP, i0, hs, b);
  if (MAXKPL >= 64 && NKP <= 2048) return select_rows_regs<R, (MAXKPL >= 64 ? 64 : 4)>(a, ss, NKP, i0, hs, b);
  select_rows_smem<R>(a, ss, NKP, i0, hs, b);
}

// Scores of R rows (sq, [R][D]) against `ncols` key rows (sk, [ncols][D],
// swizzled; ncols a multiple of 32), written to ss[r * NKP + col_base + c].
template <int D, int R>
__device__ __forceinline__ void score_tiles(const float *sk, const float *sq, float *ss, int NKP, int col_base,
                                            int ncols) {
  constexpr int QCH = D / 4;  // 16-byte chunks per row
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int dq = lane >> 3, cl = lane & 7;
  const int ncg = ncols / 32;
  for (int wt = warp; wt < (R / 4) * ncg; wt += kThreads / 32) {
    const int rg = wt % (R / 4), cg = wt / (R / 4);
    const int col0 = cg * 32 + cl * 4;  // (col0 + c) / 4 mod 8 == cl: the row swizzle
    float acc[4][4];
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[t][c] = 0.f;
#pragma unroll 2
    for (int qq = 0; qq < QCH / 4; ++qq) {
      const int ch = qq * 4 + dq;
      float4 kb[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) kb[c] = *reinterpret_cast<const float4 *>(sk + (col0 + c) * D + 4 * (ch ^ cl));
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float4 qa = *reinterpret_cast<const float4 *>(sq + (rg * 4 + t) * D + 4 * ch);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v = acc[t][c];
          v = fmaf(qa.x, kb[c].x, v);
          v = fmaf(qa.y, kb[c].y, v);
          v = fmaf(qa.z, kb[c].z, v);
          v = fmaf(qa.w, kb[c].w, v);
          acc[t][c] = v;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[t][c] += __shfl_xor_sync(0xffffffffu, acc[t][c], 8);
        acc[t][c] += __shfl_xor_sync(0xffffffffu, acc[t][c], 16);
      }
    // lane dq writes row rg*4 + dq
    float4 o = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
#pragma unroll
    for (int t = 1; t < 4; ++t)
      if (dq == t) o = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
    *reinterpret_cast<float4 *>(ss + (size_t)(rg * 4 + dq) * NKP + col_base + col0) = o;
  }
}

template <int R>
__device__ __forceinline__ void write_scores(const SelectArgs &a, const float *ss, int NKP, int i0, int hs, int b) {
  for (int r = 0; r < R; ++r) {
    const int i = i0 + r;
    if (i >= a.NQ) break;
    float *dst = a.scores_out + (((size_t)b * a.Hs + hs) * a.NQ + i) * a.NK;
    for (int j = threadIdx.x; j < a.NK; j += kThreads) dst[j] = ss[(size_t)r * NKP + j];
  }
}

// ---------------------------------------------------------------- resident
// All NK pooled key rows of the head sit in shared memory at once.
template <int D, int R>
__global__ void __launch_bounds__(kThreads) select_resident_kernel(SelectArgs a) {
  pdl_wait();  // pooled inputs come from the previous kernel
  pdl_trigger();
  constexpr int NC = kResidentBytes / (D * 4);  // key rows that fit
  constexpr int QCH = D / 4;                     // 16-byte chunks per row
  static_assert(NC % 128 == 0 && R % 4 == 0, "tiles");

  extern __shared__ __align__(16) unsigned char smem[];
  const int NK = a.NK;
  const int NKP = round_up(NK, 128);
  float *sk = reinterpret_cast<float *>(smem);  // [NC][D], chunks swizzled by (row/4) & 7
  float *sq = sk + NC * D;                       // [R][D]
  float *ss = sq + R * D;                        // [R][NKP]

  const int tid = threadIdx.x;
  const int i0 = blockIdx.x * R;
  const int hs = blockIdx.y;
  const int b = blockIdx.z;
  const int hk = hs / (a.Hq / a.Hkv);
  const float *qbase = a.pq + ((size_t)b * a.Hq + hs) * a.NQ * D;
  const float *kbase = a.pk + ((size_t)b * a.Hkv + hk) * (size_t)NK * D;

  for (int idx = tid; idx < R * QCH; idx += kThreads) {
    const int r = idx / QCH, qq = idx % QCH;
    const bool ok = i0 + r < a.NQ;
    cp_async16(sq + r * D + 4 * qq, ok ? qbase + (size_t)(i0 + r) * D + 4 * qq : a.pq, ok);
  }
  const int nrows = min(NK, NC);
  // rows up to the next multiple of 32 are zero-filled (the score tiles
  // are 32 columns wide; the extra columns are never selected)
  for (int idx = tid; idx < round_up(nrows, 32) * QCH; idx += kThreads) {
    const int c = idx / QCH, qq = idx % QCH;
    const bool ok = c < NK;
    cp_async16(sk + c * D + 4 * (qq ^ ((c >> 2) & 7)), ok ? kbase + (size_t)c * D + 4 * qq : a.pk, ok);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  score_tiles<D, R>(sk, sq, ss, NKP, 0, round_up(nrows, 32));
  __syncthreads();
  if (a.scores_out != nullptr) {
    write_scores<R>(a, ss, NKP, i0, hs, b);
    return;
  }
  select_rows<R, NC / 32>(a, ss, NKP, i0, hs, b);
}

// ------------------------------------------------------- resident, pools q
// Pooling of a tile's token rows (rows of D bf16) by one warp: 16 bytes per
// lane per row, per column a float32 sum over the lane's rows in order, then
// the lanes holding a column added (pool_blocks' mean of a possibly partial
// tile, divided by its row count at the end).
template <int D>
struct WarpPool {
  static constexpr int TPR = D / 8;     // lanes per token row (16 bytes each)
  static constexpr int RPP = 32 / TPR;  // token rows per warp-wide load
  static constexpr int U = 16;          // loads in flight per lane
  static constexpr int STEP = U * RPP;  // rows per round of loads
  float acc[8];

  __device__ __forceinline__ WarpPool() {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  }
  // rows [r_begin, r_end) of the tile at `base`; a split at a multiple of
  // STEP keeps every lane's summation order that of one call over all rows.
  // The loop is warp-uniform (a lane past the end adds zeros); `hook` runs
  // once, warp-uniformly, while the first round of loads is in flight.
  template <class Hook>
  __device__ __forceinline__ void rows(const __nv_bfloat16 *base, int r_begin, int r_end, Hook &&hook) {
    const int lane = threadIdx.x % 32;
    base += (lane % TPR) * 8;
    bool first = true;
    for (int rb = r_begin; rb < r_end; rb += STEP) {
      const int r = rb + lane / TPR;
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        v[u] = (r + u * RPP < r_end) ? ld_stream16(base + (size_t)(r + u * RPP) * D) : make_uint4(0, 0, 0, 0);
      if (first) {
        hook();
        first = false;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) acc_bf16x8(acc, v[u]);
    }
  }
  __device__ __forceinline__ void rows(const __nv_bfloat16 *base, int r_begin, int r_end) {
    rows(base, r_begin, r_end, [] {});
  }
  // column sums over the warp; lanes < TPR then hold columns 8 lane .. 8 lane + 7
  __device__ __forceinline__ void reduce() {
#pragma unroll
    for (int off = TPR; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
  }
  // after reduce(): out[0, D) = sums / n (lanes < TPR write)
  __device__ __forceinline__ void store_mean(float *out, int n) const {
    const int lane = threadIdx.x % 32;
    if (lane < TPR) {
      const float nf = (float)(n > 0 ? n : 1);
      float4 *o = reinterpret_cast<float4 *>(out + lane * 8);
      o[0] = make_float4(acc[0] / nf, acc[1] / nf, acc[2] / nf, acc[3] / nf);
      o[1] = make_float4(acc[4] / nf, acc[5] / nf, acc[6] / nf, acc[7] / nf);
    }
  }
};

// As the resident kernel, but the CTA first pools its own R = 8 query tiles
// from q (one tile per warp): the pooled query vectors never go through HBM.
// With k_raw set (a cooperative launch: every CTA is resident) the CTAs of a
// kv group also pool the group's k: each takes an equal share of the kv
// tiles (one warp per tile), writes the pooled rows to pk_out and counts
// itself in the group's counter, and scoring starts once the counter shows
// the whole group (a bounded wait; on a timeout the library's error word is
// set and the CTA stops). Each warp first looks at the counter halfway
// through its query tile and, when the group is complete by then, fetches
// its share of the pooled keys while the second half of the tile streams
// in. Otherwise the pooled keys come from the previous kernel, and the query
// pooling, which reads nothing that kernel writes, runs before the
// programmatic-dependency wait.
template <int D>
__global__ void __launch_bounds__(kThreads) select_fusedq_kernel(SelectArgs a) {
  constexpr int R = 8;  // one query tile per warp
  constexpr int NC = kResidentBytes / (D * 4);
  constexpr int QCH = D / 4;
  static_assert(NC % 128 == 0 && kThreads == 32 * R, "tiles");

  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int s_stop;
  const int NK = a.NK;
  const int NKP = round_up(NK, 128);
  float *sk = reinterpret_cast<float *>(smem);  // [NC][D], chunks swizzled by (row/4) & 7
  float *sq = sk + NC * D;                       // [R][D]
  float *ss = sq + R * D;                        // [R][NKP]

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int i0 = blockIdx.x * R;
  const int hs = blockIdx.y;
  const int b = blockIdx.z;
  const int g = a.Hq / a.Hkv;
  const int hk = hs / g;
  const int n_group = g * (int)gridDim.x;  // CTAs of this kv group

  const float *kbase = a.pk + ((size_t)b * a.Hkv + hk) * (size_t)NK * D;
  const int nrows = min(NK, NC);
  // this thread's share of the pooled key rows into shared memory (cp.async,
  // waited for before scoring); rows up to the next multiple of 32 are
  // zero-filled (the score tiles are 32 columns wide; the extra columns are
  // never selected)
  auto load_keys = [&]() {
    for (int idx = tid; idx < round_up(nrows, 32) * QCH; idx += kThreads) {
      const int cc = idx / QCH, qq = idx % QCH;
      const bool ok = cc < NK;
      cp_async16(sk + cc * D + 4 * (qq ^ ((cc >> 2) & 7)), ok ? kbase + (size_t)cc * D + 4 * qq : a.pk, ok);
    }
    cp_async_commit();
  };
  unsigned int *ctr = a.group_count ? a.group_count + b * a.Hkv + hk : nullptr;

  if (a.k_raw != nullptr) {
    // ---- this CTA's share of the group's kv tiles, one warp per tile
    const int rank = (hs % g) * (int)gridDim.x + blockIdx.x;
    const int t0 = (int)((long long)NK * rank / n_group), t1 = (int)((long long)NK * (rank + 1) / n_group);
    const __nv_bfloat16 *kb = a.k_raw + ((size_t)b * a.Hkv + hk) * a.Skv * D;
    float *pko = a.pk_out + ((size_t)b * a.Hkv + hk) * (size_t)NK * D;
    for (int t = t0 + warp; t < t1; t += R) {
      const int lo = t * a.block_kv, n = min(a.block_kv, a.Skv - lo);
      WarpPool<D> wp;
      wp.rows(kb + (size_t)lo * D, 0, n);
      wp.reduce();
      wp.store_mean(pko + (size_t)t * D, n);
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();  // the pooled rows before the count
      atomicAdd(ctr, 1u);
    }
  }

  // ---- pool query tile i0 + warp of head hs. With the keys pooled by the
  // group, each warp looks at the group's counter while the first loads of
  // the tile's second half are in flight, and when the group is complete it
  // fetches its share of the pooled keys at once, so that they arrive while
  // the rest of the query rows stream in.
  const int iq = i0 + warp;
  const int qlo = iq * a.block_q, qn = iq < a.NQ ? min(a.block_q, a.Sq - qlo) : 0;
  const __nv_bfloat16 *qb = a.q_raw + (((size_t)b * a.Hq + hs) * a.Sq + (iq < a.NQ ? qlo : 0)) * D;
  constexpr int QSPLIT = 64;
  static_assert(QSPLIT % WarpPool<D>::STEP == 0, "the split keeps the summation order");
  bool issued = false;
  auto early_keys = [&]() {
    if (a.k_raw == nullptr) return;
    unsigned int c = 0;
    if (lane == 0) {
      c = atomicAdd(ctr, 0u);
      __threadfence();  // the group's pooled rows after the count
    }
    __syncwarp();
    c = __shfl_sync(0xffffffffu, c, 0);
    if (c >= (unsigned int)n_group) {
      load_keys();
      issued = true;
    }
  };
  WarpPool<D> pq;
  pq.rows(qb, 0, min(qn, QSPLIT));
  pq.rows(qb, QSPLIT, qn, early_keys);
  pq.reduce();
  if (iq < a.NQ) {
    pq.store_mean(sq + warp * D, qn);
  } else if (lane < QCH) {
    reinterpret_cast<float4 *>(sq + warp * D)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  if (a.k_raw != nullptr) {
    // the warps that found the group incomplete: wait for it (bounded)
    if (!__syncthreads_and(issued)) {
      // (the fence in counter_wait orders the group's pooled rows after the count)
      if (tid == 0) s_stop = counter_wait(ctr, (unsigned int)n_group, a.err, 0x30u) ? 0 : 1;
      __syncthreads();
      if (s_stop) {
        cp_async_wait<0>();  // key copies a warp issued early land before the CTA exits
        return;
      }
      if (!issued) load_keys();
    }
  } else {
    pdl_wait();  // pooled keys come from the previous kernel
    load_keys();
  }
  pdl_trigger();
  cp_async_wait<0>();
  __syncthreads();
  score_tiles<D, R>(sk, sq, ss, NKP, 0, round_up(nrows, 32));
  __syncthreads();
  if (a.scores_out != nullptr) {
    write_scores<R>(a, ss, NKP, i0, hs, b);
    return;
  }
  select_rows<R, NC / 32>(a, ss, NKP, i0, hs, b);
}

// ------------------------------------------------- from tensor-core scores
// Plan + top-k + outputs for rows whose scores score_tc_kernel wrote to the
// scratch (row stride NKP <= 2048): one warp per keep row, four rows per
// CTA at a time, the row's candidate keys in the warp's slice of shared
// memory (tile order; few registers, so many warps per SM hide the long
// dependent chains of a row). Lane l handles the tiles j = l + 32 m: each
// load and shared-memory access of the warp covers 32 consecutive tiles,
// and one lane's tiles lie 32 apart.
// The k-th largest candidate key T: the k-th largest of the warp's group
// maxima (each lane's tiles in four groups) is a key L with at least k keys
// >= L (distinct tiles), so T is the k-th largest of the keys >= L. Those,
// usually a little more than k, are gathered and sorted across the warp
// (bitonic); when more than 256 keys are >= L (or k > 128), the keys are
// bucketed by range instead (warp_kth_radix). Ties at T go to the lowest
// tile indices. Lane l writes the outputs of tiles 64 l .. 64 l + 63.
constexpr int kSelWarps = 4;
constexpr int kSelBuf = 256;

// warp_kth_radix for keys held in shared memory (n keys, nonzero = a
// candidate; lane l reads entries l, l + 32, ...): the same bucketing of
// the key range, with the counts in the warp's 256-entry scratch `hist`.
__device__ __noinline__ uint32_t warp_kth_range_smem(const uint32_t *key, int n, int k, uint32_t *hist) {
  const int lane = threadIdx.x & 31;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int q = lane; q < n; q += 32)
    if (key[q] != 0u) {
      lo = min(lo, key[q]);
      hi = max(hi, key[q]);
    }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  int kr = k;
  while (lo < hi) {
    const int shift = max(0, 24 - __clz(hi - lo));
    for (int q = lane; q < 256; q += 32) hist[q] = 0u;
    __syncwarp();
    for (int q = lane; q < n; q += 32) {
      const uint32_t kv = key[q];
      if (kv != 0u && kv >= lo && kv <= hi) atomicAdd(&hist[(kv - lo) >> shift], 1u);
    }
    __syncwarp();
    int c8[8], sum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c8[q] = (int)hist[255 - (lane * 8 + q)];
      sum += c8[q];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    const int excl = incl - sum;
    const bool mine = excl < kr && kr <= incl;
    int bin = 0, above = excl;
    if (mine) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (above + c8[q] >= kr) {
          bin = 255 - (lane * 8 + q);
          break;
        }
        above += c8[q];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    bin = __shfl_sync(0xffffffffu, bin, src);
    above = __shfl_sync(0xffffffffu, above, src);
    kr -= above;
    const uint32_t nlo = lo + ((uint32_t)bin << shift);
    const uint32_t width = (1u << shift) - 1u;
    hi = (hi - nlo < width) ? hi : nlo + width;
    lo = nlo;
    __syncwarp();
  }
  return lo;
}

template <int KPL>
__global__ void __launch_bounds__(kSelWarps * 32, 6) select_scores_kernel(SelectArgs a) {
  __shared__ __align__(16) uint32_t skey[kSelWarps][32 * KPL];
  __shared__ __align__(16) uint32_t sbuf[kSelWarps][kSelBuf];
  pdl_wait();  // the scores come from the previous kernel
  const int NK = a.NK, NQ = a.NQ;
  const int NKP = round_up(NK, 128);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  uint32_t *key = skey[warp];
  uint32_t *buf = sbuf[warp];
  const long long rows = (long long)a.B * a.Hs * NQ;
  constexpr int GPL = 4;                      // group maxima per lane (128 per warp)
  constexpr int MPG = KPL / GPL > 0 ? KPL / GPL : 1;  // tiles per group
  // keep rows written 16 bytes at a time: the tensor is 16-byte aligned and
  // rows, NK bytes apart, stay aligned
  const bool keep16 = a.keep && (NK & 15) == 0 && (reinterpret_cast<uintptr_t>(a.keep) & 15u) == 0;
  for (long long row = (long long)blockIdx.x * kSelWarps + warp; row < rows; row += (long long)gridDim.x * kSelWarps) {
    const int i = (int)(row % NQ);
    const int hs = (int)((row / NQ) % a.Hs);
    const int b = (int)(row / ((long long)NQ * a.Hs));
    const RowPlan pl(a, b, hs, i);
    // rows with no pins, drops or plan: the forced tiles are the diagonal
    // run [d0, d1] (int compares only)
    const bool diag_only = !pl.prow && !pl.drow && !pl.srow;
    const int d0 = (int)pl.jd0, d1 = (int)pl.jd1;
    auto is_cand = [&](int j) {
      return diag_only ? (j < d0 || j > d1) : (!pl.must(j) && !pl.forbidden(j));
    };
    auto is_forced = [&](int j) { return diag_only ? (j >= d0 && j <= d1) : (pl.must(j) && !pl.forbidden(j)); };
    const float *ss = a.tc_scores + row * NKP;
    // keys: 0 for tiles that are not candidates (and past NK)
    uint32_t gm[GPL] = {0u, 0u, 0u, 0u};
    int c_lane = 0;
#pragma unroll
    for (int g = 0; g < GPL; ++g) {
      float v[MPG];
#pragma unroll
      for (int u = 0; u < MPG; ++u) {
        const int j = lane + 32 * (g * MPG + u);
        v[u] = (g * MPG + u < KPL && j < NKP) ? ss[j] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < MPG; ++u) {
        const int m = g * MPG + u;
        if (m >= KPL) break;
        const int j = lane + 32 * m;
        uint32_t kv = 0u;
        if (j < NK && is_cand(j)) {
          kv = order_key(v[u]);
          ++c_lane;
        }
        key[32 * m + lane] = kv;
        gm[g] = max(gm[g], kv);
      }
    }
    __syncwarp();
    const int c = __reduce_add_sync(0xffffffffu, c_lane);
    const int k = row_budget(a, b, hs, i, c);
    if (lane == 0 && k < c && a.not_covered && *reinterpret_cast<volatile unsigned int *>(a.not_covered) == 0u)
      atomicOr(a.not_covered, 1u);
    uint32_t T = 0xFFFFFFFFu;
    int take = 0;
    if (k >= c) {
      T = 0u;
    } else if (k > 0) {
      bool done = false;
      if (k <= 32 * GPL) {
        const uint32_t L = warp_kth_largest<GPL>(gm, k);
        int n = 0;
#pragma unroll 8
        for (int m = 0; m < KPL; ++m) {
          const uint32_t kv = key[32 * m + lane];
          n += (kv != 0u && kv >= L) ? 1 : 0;
        }
        int cnt;
        int pos = warp_excl_scan(n, lane, &cnt);
        if (cnt <= kSelBuf) {
#pragma unroll 8
          for (int m = 0; m < KPL; ++m) {
            const uint32_t kv = key[32 * m + lane];
            if (kv != 0u && kv >= L) buf[pos++] = kv;
          }
          __syncwarp();
          // lane l takes entries N l .. N l + N - 1 as 16-byte loads (no
          // bank conflicts); entries past cnt count as 0
          if (cnt <= 128) {
            uint32_t y[4];
            const uint4 v = *reinterpret_cast<const uint4 *>(buf + lane * 4);
            y[0] = v.x;
            y[1] = v.y;
            y[2] = v.z;
            y[3] = v.w;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (lane * 4 + e >= cnt) y[e] = 0u;
            __syncwarp();
            T = warp_kth_largest<4>(y, k);
          } else {
            constexpr int NB = kSelBuf / 32;
            uint32_t y[NB];
#pragma unroll
            for (int e4 = 0; e4 < NB / 4; ++e4) {
              const uint4 v = *reinterpret_cast<const uint4 *>(buf + lane * NB + 4 * e4);
              y[4 * e4] = v.x;
              y[4 * e4 + 1] = v.y;
              y[4 * e4 + 2] = v.z;
              y[4 * e4 + 3] = v.w;
            }
#pragma unroll
            for (int e = 0; e < NB; ++e)
              if (lane * NB + e >= cnt) y[e] = 0u;
            __syncwarp();
            T = warp_kth_largest<NB>(y, k);
          }
          done = true;
        }
      }
      if (!done) T = warp_kth_range_smem(key, 32 * KPL, k, buf);
      int above = 0;
#pragma unroll 8
      for (int m = 0; m < KPL; ++m) {
        const uint32_t kv = key[32 * m + lane];
        above += (kv != 0u && kv > T) ? 1 : 0;
      }
      take = k - __reduce_add_sync(0xffffffffu, above);
    }
    // lane l's span: tiles 64 l .. 64 l + 63, as two flag words (> T or
    // every candidate, or forced; ties). The flags are read in the key
    // layout (tile 32 m + lane, conflict-free) and the ballot over column
    // block m is the flag word of tiles 32 m .. 32 m + 31: word m & 1 of
    // lane m / 2's span
    const int span0 = 64 * lane;
    uint32_t gt[2] = {0u, 0u}, tw[2] = {0u, 0u};
#pragma unroll 4
    for (int m2 = 0; m2 < KPL / 2; ++m2) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 64 * m2 + 32 * h + lane;
        const uint32_t kv = key[j];
        const bool forced = j < NK && is_forced(j);
        const uint32_t bg = __ballot_sync(0xffffffffu, (kv != 0u && (kv > T || k >= c)) || forced);
        const uint32_t bt = __ballot_sync(0xffffffffu, take > 0 && kv != 0u && kv == T);
        if (lane == m2) {
          gt[h] = bg;
          tw[h] = bt;
        }
      }
    }
    __syncwarp();  // every lane has read the keys before the warp's next row
    // the first `take` ties in tile order join the keep
    int tie_tot;
    const int tie_before = warp_excl_scan(__popc(tw[0]) + __popc(tw[1]), lane, &tie_tot);
    int room = take - tie_before;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t w = tw[h];
      while (w != 0u && room > 0) {
        const uint32_t bit = w & (0u - w);
        gt[h] |= bit;
        w ^= bit;
        --room;
      }
    }
    int kept_tot;
    int pos = warp_excl_scan(__popc(gt[0]) + __popc(gt[1]), lane, &kept_tot);
    int8_t *krow = a.keep ? a.keep + row * NK : nullptr;
    uint16_t *irow = a.kv_index ? a.kv_index + row * NK : nullptr;
    if (krow && span0 < NK) {
      if (keep16 && span0 + 64 <= NK) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            uint32_t wd[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint32_t nib = (gt[h] >> (16 * qq + 4 * u)) & 0xFu;
              wd[u] = (nib & 1u) | ((nib >> 1) & 1u) << 8 | ((nib >> 2) & 1u) << 16 | ((nib >> 3) & 1u) << 24;
            }
            *reinterpret_cast<uint4 *>(krow + span0 + 32 * h + 16 * qq) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          }
      } else {
        for (int r = 0; r < 64 && span0 + r < NK; ++r) krow[span0 + r] = (int8_t)((gt[r >> 5] >> (r & 31)) & 1u);
      }
    }
    if (irow) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t w = gt[h];
        while (w != 0u) {
          const int r = __ffs(w) - 1;
          w &= w - 1u;
          irow[pos++] = (uint16_t)(span0 + 32 * h + r);
        }
      }
    }
    if (lane == 0 && a.kv_count) a.kv_count[row] = kept_tot;
  }
}

// ----------------------------------------------------------------- chunked
// Key rows stream through two 32 KB shared-memory chunks.
template <int D, int R>
__global__ void __launch_bounds__(kThreads) select_chunked_kernel(SelectArgs a) {
  pdl_wait();  // pooled inputs come from the previous kernel
  pdl_trigger();
  constexpr int NCH = kChunkBytes / (D * 4);  // key rows per chunk (64 or 128)
  constexpr int QCH = D / 4;
  static_assert(NCH % 32 == 0 && R % 4 == 0, "tiles");

  extern __shared__ __align__(16) unsigned char smem[];
  const int NK = a.NK;
  const int NKP = round_up(NK, 128);
  float *sk = reinterpret_cast<float *>(smem);  // [2][NCH][D], swizzled
  float *sq = sk + 2 * NCH * D;                  // [R][D]
  float *ss = sq + R * D;                        // [R][NKP]

  const int tid = threadIdx.x;
  const int i0 = blockIdx.x * R;
  const int hs = blockIdx.y;
  const int b = blockIdx.z;
  const int NQ = a.NQ;
  const int hk = a.head_shared ? 0 : hs / (a.Hq / a.Hkv);
  const float *qbase = a.pq + ((size_t)b * a.Hq + hs) * NQ * D;
  const float *kbase = a.pk + ((size_t)b * a.Hkv + hk) * (size_t)NK * D;

  // query rows (head_shared: the mean over the Hq heads, in head order)
  for (int idx = tid; idx < R * QCH; idx += kThreads) {
    const int r = idx / QCH, qq = idx % QCH;
    const bool ok = i0 + r < NQ;
    if (!a.head_shared) {
      cp_async16(sq + r * D + 4 * qq, ok ? qbase + (size_t)(i0 + r) * D + 4 * qq : a.pq, ok);
    } else {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ok) {
        for (int h = 0; h < a.Hq; ++h) {
          const float4 w =
              *reinterpret_cast<const float4 *>(a.pq + (((size_t)b * a.Hq + h) * NQ + i0 + r) * D + 4 * qq);
          v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
        }
        const float hf = (float)a.Hq;
        v.x /= hf; v.y /= hf; v.z /= hf; v.w /= hf;
      }
      *reinterpret_cast<float4 *>(sq + r * D + 4 * qq) = v;
    }
  }
  auto load_chunk = [&](int ci) {
    float *dst = sk + (ci & 1) * NCH * D;
    for (int idx = tid; idx < NCH * QCH; idx += kThreads) {
      const int c = idx / QCH, qq = idx % QCH;
      const int j = ci * NCH + c;
      const bool ok = j < NK;
      float *d = dst + c * D + 4 * (qq ^ ((c >> 2) & 7));
      if (!a.head_shared) {
        cp_async16(d, ok ? kbase + (size_t)j * D + 4 * qq : a.pk, ok);
      } else {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ok) {
          for (int h = 0; h < a.Hkv; ++h) {
            const float4 w =
                *reinterpret_cast<const float4 *>(a.pk + (((size_t)b * a.Hkv + h) * NK + j) * D + 4 * qq);
            v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
          }
          const float hf = (float)a.Hkv;
          v.x /= hf; v.y /= hf; v.z /= hf; v.w /= hf;
        }
        *reinterpret_cast<float4 *>(d) = v;
      }
    }
    cp_async_commit();
  };

  const int nch = (NK + NCH - 1) / NCH;
  load_chunk(0);
  for (int ci = 0; ci < nch; ++ci) {
    if (ci + 1 < nch) {
      load_chunk(ci + 1);  // its buffer was last read before the barrier ending step ci - 1
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    score_tiles<D, R>(sk + (ci & 1) * NCH * D, sq, ss, NKP, ci * NCH, NCH);
    __syncthreads();
  }

  if (a.scores_out != nullptr) {
    write_scores<R>(a, ss, NKP, i0, hs, b);
    return;
  }
  select_rows<R, 64>(a, ss, NKP, i0, hs, b);
}

// mean over the head axis: x (B, H, N, D) -> out (B, 1, N, D); summation in
// head order, then one division.
__global__ void __launch_bounds__(256) head_mean_kernel(const float *x, int B, int H, int N, int D, float *out) {
  pdl_wait();
  pdl_trigger();
  const long long total = (long long)B * N * D;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long b = t / ((long long)N * D);
    const long long rem = t - b * N * D;
    float s = 0.f;
    for (int h = 0; h < H; ++h) s += x[(b * H + h) * (long long)N * D + rem];
    out[t] = s / (float)H;
  }
}

__global__ void __launch_bounds__(256) keep_to_index_kernel(const int8_t *keep, long long rows, int NK,
                                                             int32_t *kv_count, uint16_t *kv_index) {
  const int lane = threadIdx.x % 32;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) / 32;
  for (long long row = warp; row < rows; row += nwarps) {
    const int8_t *krow = keep + row * NK;
    uint16_t *irow = kv_index + row * NK;
    int base = 0;
    for (int j0 = 0; j0 < NK; j0 += 128) {
      int kp[4], n = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + lane * 4 + u;
        kp[u] = (j < NK && krow[j] != 0) ? 1 : 0;
        n += kp[u];
      }
      int tot;
      int pos = base + warp_excl_scan(n, lane, &tot);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (kp[u]) irow[pos++] = (uint16_t)(j0 + lane * 4 + u);
      base += tot;
    }
    if (lane == 0) kv_count[row] = base;
  }
}

bool resident_fits(int NK, int D, int head_shared) { return !head_shared && (size_t)NK * D * 4 <= kResidentBytes; }

size_t fusedq_smem(int NK, int D) {
  const size_t nkp = (size_t)round_up(NK, 128);
  return (size_t)kResidentBytes + (size_t)8 * D * 4 + (size_t)8 * nkp * 4;
}

size_t resident_smem(int R, int NK, int D) {
  const size_t nkp = (size_t)round_up(NK, 128);
  return (size_t)kResidentBytes + (size_t)R * D * 4 + (size_t)R * nkp * 4;
}

size_t chunked_smem(int R, int NK, int D) {
  const size_t nkp = (size_t)round_up(NK, 128);
  return 2 * (size_t)kChunkBytes + (size_t)R * D * 4 + (size_t)R * nkp * 4;
}

template <typename K>
cudaError_t launch_k(K kernel, dim3 grid, size_t smem, const SelectArgs &a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kernel, grid, dim3(kThreads), smem, stream, a);
}

template <typename K>
cudaError_t launch_sel(K kernel, dim3 grid, const SelectArgs &a, cudaStream_t stream) {
  return launch_pdl(kernel, grid, dim3(kSelWarps * 32), 0, stream, a);
}

// Cooperative launch: every CTA of the grid is resident at once (the launch
// fails otherwise), which the in-kernel group wait relies on.
template <typename K>
cudaError_t launch_coop(K kernel, dim3 grid, size_t smem, const SelectArgs &a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, a);
  if (e == cudaSuccess) note_launch();
  return e;
}

template <typename K>
bool grid_fits(K kernel, long long ctas, size_t smem, int num_sms) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return false;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem) != cudaSuccess) return false;
  return ctas <= (long long)per_sm * num_sms;
}

}  // namespace

bool select_pools_k(const SelectArgs &a, int num_sms) {
  if (!select_pools_q(a.NK, a.D, a.head_shared)) return false;
  const long long ctas = (long long)((a.NQ + 7) / 8) * a.Hs * a.B;
  const size_t smem = fusedq_smem(a.NK, a.D);
  return a.D == 64 ? grid_fits(select_fusedq_kernel<64>, ctas, smem, num_sms)
                   : grid_fits(select_fusedq_kernel<128>, ctas, smem, num_sms);
}

// Rows per CTA: the largest R whose grid still covers the SMs (else the
// smallest), within the shared-memory budget of the chosen path.
int select_rows_per_cta(int B, int Hs, int NQ, int NK, int num_sms, int D, int head_shared) {
  if (NK > 8192) return 0;
  const bool res = resident_fits(NK, D, head_shared);
  const int maxR = res ? 32 : 16;
  int best = 0;
  for (int R = maxR; R >= 4; R /= 2) {
    const size_t smem = res ? resident_smem(R, NK, D) : chunked_smem(R, NK, D);
    if (smem > 200 * 1024) continue;
    best = R;
    if ((long long)B * Hs * ((NQ + R - 1) / R) >= num_sms) break;
  }
  return best;
}

bool select_pools_q(int NK, int D, int head_shared) { return resident_fits(NK, D, head_shared); }

bool select_uses_tc_scores(int NK, int D, int head_shared) {
  return !resident_fits(NK, D, head_shared) && round_up(NK, 128) <= 2048;
}

cudaError_t launch_select(const SelectArgs &a, int num_sms, cudaStream_t stream) {
  if (a.q_raw != nullptr) {
    if (!select_pools_q(a.NK, a.D, a.head_shared)) return cudaErrorInvalidValue;
    const dim3 grid((a.NQ + 7) / 8, a.Hs, a.B);
    const size_t smem = fusedq_smem(a.NK, a.D);
    if (a.k_raw != nullptr) {
      if (!select_pools_k(a, num_sms)) return cudaErrorInvalidValue;
      return a.D == 64 ? launch_coop(select_fusedq_kernel<64>, grid, smem, a, stream)
                       : launch_coop(select_fusedq_kernel<128>, grid, smem, a, stream);
    }
    return a.D == 64 ? launch_k(select_fusedq_kernel<64>, grid, smem, a, stream)
                     : launch_k(select_fusedq_kernel<128>, grid, smem, a, stream);
  }
  if (a.tc_scores != nullptr && a.scores_out == nullptr && select_uses_tc_scores(a.NK, a.D, a.head_shared)) {
    // the scores are in the scratch (launch_score_tc ran before): top-k
    const int nkp = round_up(a.NK, 128);
    const long long rows = (long long)a.B * a.Hs * a.NQ;
    // one warp per row, rows taken in turn by the resident CTAs
    const dim3 g1((unsigned)std::min<long long>((rows + kSelWarps - 1) / kSelWarps, (long long)num_sms * 12));
    if (nkp <= 128) return launch_sel(select_scores_kernel<4>, g1, a, stream);
    if (nkp <= 256) return launch_sel(select_scores_kernel<8>, g1, a, stream);
    if (nkp <= 512) return launch_sel(select_scores_kernel<16>, g1, a, stream);
    if (nkp <= 1024) return launch_sel(select_scores_kernel<32>, g1, a, stream);
    return launch_sel(select_scores_kernel<64>, g1, a, stream);
  }
  const int R = select_rows_per_cta(a.B, a.Hs, a.NQ, a.NK, num_sms, a.D, a.head_shared);
  if (R == 0) return cudaErrorInvalidValue;
  const dim3 grid((a.NQ + R - 1) / R, a.Hs, a.B);
  if (resident_fits(a.NK, a.D, a.head_shared)) {
    const size_t smem = resident_smem(R, a.NK, a.D);
#define NSA_RES(DD, RR) \
  if (a.D == DD && R == RR) return launch_k(select_resident_kernel<DD, RR>, grid, smem, a, stream);
    NSA_RES(128, 32) NSA_RES(128, 16) NSA_RES(128, 8) NSA_RES(128, 4)
    NSA_RES(64, 32) NSA_RES(64, 16) NSA_RES(64, 8) NSA_RES(64, 4)
#undef NSA_RES
    return cudaErrorInvalidValue;
  }
  const size_t smem = chunked_smem(R, a.NK, a.D);
#define NSA_CHK(DD, RR) \
  if (a.D == DD && R == RR) return launch_k(select_chunked_kernel<DD, RR>, grid, smem, a, stream);
  NSA_CHK(128, 16) NSA_CHK(128, 8) NSA_CHK(128, 4)
  NSA_CHK(64, 16) NSA_CHK(64, 8) NSA_CHK(64, 4)
#undef NSA_CHK
  return cudaErrorInvalidValue;
}

cudaError_t launch_head_mean(const float *x, int B, int H, int N, int D, float *out, int num_sms,
                             cudaStream_t stream) {
  const long long total = (long long)B * N * D;
  long long blocks = (total + 255) / 256;
  if (blocks > (long long)num_sms * 8) blocks = (long long)num_sms * 8;
  return launch_pdl(head_mean_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, x, B, H, N, D, out);
}

cudaError_t launch_keep_to_index(const int8_t *keep, long long rows, int NK, int32_t *kv_count,
                                 uint16_t *kv_index, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  long long blocks = (rows + 7) / 8;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  keep_to_index_kernel<<<(int)blocks, 256, 0, stream>>>(keep, rows, NK, kv_count, kv_index);
  note_launch();
  return cudaGetLastError();
}

}  // namespace nsa
