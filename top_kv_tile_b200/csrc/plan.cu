// plan.cu -- the selection plan kept in a caller buffer, and the radial band
// control, both on the device.
//
// Plan (selector.py, selection_plan and its plan_cache): the part of a
// selection that depends only on the geometry, the spec and the pin/drop
// layout. Per tile a state (0 = candidate, 1 = kept whatever the scores:
// diagonal or pinned and not dropped, 2 = forbidden: dropped), per keep row
// the candidate count c and the budget count k = ceil(f32(c) * f32(budget)),
// and whether every row may keep all its candidates (covers_everything). The
// tile and row arrays have the broadcast extent of the pin/drop masks over
// batches and keep heads (1 where neither mask varies along that axis).
//
// Radial band (selector.py, radial_blocks): tile centres ((i+0.5) block_q,
// (j+0.5) block_kv); the band keeps the tiles whose centre distance is at
// most w, with w the upper end of 40 bisection steps on [0, max(Sq, Skv)]
// that aim the kept fraction at `density`. The fraction is the float32 mean
// of the 0/1 mask, as the page evaluates it; the bisection runs in one CTA on
// the device (the page reads the fraction back 40 times). Row i keeps one
// contiguous run of kv tiles, found by binary search with the exact float64
// distance test on each side of the row's nearest tile.
#include "nsa_device.cuh"
#include "nsa_kernels.cuh"

namespace nsa {

namespace {

__global__ void __launch_bounds__(256) plan_build_kernel(PlanArgs p) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long rows = (long long)p.Bp * p.Hp * p.NQ;
  const long long nwarps = (long long)gridDim.x * (blockDim.x / 32);
  for (long long row = (long long)blockIdx.x * (blockDim.x / 32) + warp; row < rows; row += nwarps) {
    const int i = (int)(row % p.NQ);
    const long long bh = row / p.NQ;
    const int h = (int)(bh % p.Hp), b = (int)(bh / p.Hp);
    const long long qlo = (long long)i * p.block_q, qhi = (long long)(i + 1) * p.block_q;
    const int8_t *prow = p.pins ? p.pins + b * p.ps[0] + h * p.ps[1] + i * p.ps[2] : nullptr;
    const int8_t *drow = p.drops ? p.drops + b * p.ds[0] + h * p.ds[1] + i * p.ds[2] : nullptr;
    int8_t *srow = p.state + row * p.NK;
    int c = 0;
    for (int j = lane; j < p.NK; j += 32) {
      const long long klo = (long long)j * p.block_kv, khi = (long long)(j + 1) * p.block_kv;
      // diagonal_blocks: nominal token ranges overlap (no clamp, no scaling)
      const bool must = ((qlo < khi) && (klo < qhi)) || (prow && prow[(long long)j * p.ps[3]] != 0);
      const bool forb = drow && drow[(long long)j * p.ds[3]] != 0;
      const int8_t st = forb ? 2 : (must ? 1 : 0);
      srow[j] = st;
      c += (st == 0) ? 1 : 0;
    }
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) {
      const int k = (int)ceilf(__fmul_rn((float)c, p.budget));
      p.cnt[row] = c;
      p.kpr[row] = k;
      if (k < c) atomicOr(p.not_covered, 1u);
    }
  }
}

// Exact distance test of tile (i, j): |(i+0.5) bq - (j+0.5) bkv| <= w in
// float64 (the centres are multiples of 0.5 and exact).
__device__ __forceinline__ bool in_band(double qc, int j, int bkv, double w) {
  return fabs(qc - ((double)j + 0.5) * (double)bkv) <= w;
}

// The kv tiles of row i inside the band: [lo, hi] (empty when lo > hi).
__device__ __forceinline__ void band_run(int i, const RadialArgs &r, double w, int &lo, int &hi) {
  const double qc = ((double)i + 0.5) * (double)r.block_q;
  // nearest tile to the row centre (the distance falls, then rises, in j)
  long long jn = (long long)floor(qc / (double)r.block_kv);
  if (jn < 0) jn = 0;
  if (jn > r.NK - 1) jn = r.NK - 1;
  int jc = (int)jn;
  if (jc + 1 < r.NK && fabs(qc - ((double)jc + 1.5) * r.block_kv) < fabs(qc - ((double)jc + 0.5) * r.block_kv)) ++jc;
  if (!in_band(qc, jc, r.block_kv, w)) {
    lo = 1;
    hi = 0;
    return;
  }
  // lowest j <= jc in the band (distance non-increasing up to jc)
  int a = 0, b = jc;
  while (a < b) {
    const int m = (a + b) / 2;
    if (in_band(qc, m, r.block_kv, w)) b = m; else a = m + 1;
  }
  lo = a;
  // highest j >= jc in the band
  a = jc;
  b = r.NK - 1;
  while (a < b) {
    const int m = (a + b + 1) / 2;
    if (in_band(qc, m, r.block_kv, w)) a = m; else b = m - 1;
  }
  hi = a;
}

constexpr int kRadialThreads = 1024;

// One CTA: 40 bisection steps, each counting the band's tiles row by row.
__global__ void __launch_bounds__(kRadialThreads) radial_width_kernel(RadialArgs r) {
  __shared__ unsigned long long part[kRadialThreads / 32];
  __shared__ int go_low;
  double low = 0.0, high = (double)max(r.Sq, r.Skv);
  const float total = (float)((long long)r.NQ * r.NK);
  for (int step = 0; step < 40; ++step) {
    const double mid = (low + high) / 2;
    unsigned long long cnt = 0;
    for (int i = threadIdx.x; i < r.NQ; i += blockDim.x) {
      int lo, hi;
      band_run(i, r, mid, lo, hi);
      if (hi >= lo) cnt += (unsigned long long)(hi - lo + 1);
    }
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x / 32] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long all = 0;
      for (int w = 0; w < (int)(blockDim.x / 32); ++w) all += part[w];
      // float32 mean of the 0/1 mask: an exact count (below 2^24 tiles)
      // divided by the tile count, rounded once
      const float frac = __fdiv_rn((float)all, total);
      go_low = ((double)frac < r.density) ? 1 : 0;
    }
    __syncthreads();
    if (go_low)
      low = mid;
    else
      high = mid;
    __syncthreads();
  }
  if (threadIdx.x == 0) *r.width = high;
}

// keep (B, 1, NQ, NK), kv_count (B, 1, NQ), kv_index (B, 1, NQ, NK): the same
// band for every batch. One warp per (batch, row).
__global__ void __launch_bounds__(256) radial_write_kernel(RadialArgs r) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const double w = *r.width;
  const long long rows = (long long)r.B * r.NQ;
  const long long nwarps = (long long)gridDim.x * (blockDim.x / 32);
  for (long long row = (long long)blockIdx.x * (blockDim.x / 32) + warp; row < rows; row += nwarps) {
    const int i = (int)(row % r.NQ);
    int lo, hi;
    band_run(i, r, w, lo, hi);
    const int n = hi >= lo ? hi - lo + 1 : 0;
    if (r.keep) {
      int8_t *krow = r.keep + row * r.NK;
      for (int j = lane; j < r.NK; j += 32) krow[j] = (j >= lo && j <= hi) ? 1 : 0;
    }
    if (r.kv_index) {
      uint16_t *irow = r.kv_index + row * r.NK;
      for (int e = lane; e < n; e += 32) irow[e] = (uint16_t)(lo + e);
    }
    if (r.kv_count && lane == 0) r.kv_count[row] = n;
  }
}

}  // namespace

cudaError_t launch_plan_build(const PlanArgs &p, int num_sms, cudaStream_t stream) {
  const long long rows = (long long)p.Bp * p.Hp * p.NQ;
  if (rows == 0) return cudaSuccess;
  long long blocks = (rows + 7) / 8;
  if (blocks > (long long)num_sms * 8) blocks = (long long)num_sms * 8;
  plan_build_kernel<<<(int)blocks, 256, 0, stream>>>(p);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_radial(const RadialArgs &r, int num_sms, cudaStream_t stream) {
  radial_width_kernel<<<1, kRadialThreads, 0, stream>>>(r);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long rows = (long long)r.B * r.NQ;
  if (rows == 0) return cudaSuccess;
  long long blocks = (rows + 7) / 8;
  if (blocks > (long long)num_sms * 8) blocks = (long long)num_sms * 8;
  radial_write_kernel<<<(int)blocks, 256, 0, stream>>>(r);
  note_launch();
  return cudaGetLastError();
}

}  // namespace nsa
