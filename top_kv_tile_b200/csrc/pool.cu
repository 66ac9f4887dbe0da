// pool.cu -- tile mean pooling (selector.py, pool_blocks).
//
// pooled[bh, i, :] = (1/n_i) * sum_{t in tile i} x[bh, t, :], float32, with
// n_i = min(block, S - i*block): a partial final tile is averaged over its own
// token count. HBM-bound: every input byte is read exactly once.
//
// Persistent kernel, one CTA of eight warps per SM. A tile of `block` token
// rows is one contiguous run of block * D bf16 values. Every warp works alone
// on its own tiles: lane 0 streams the tile, in 8 KB pieces, into the warp's
// private ring of three shared-memory stages with bulk asynchronous copies
// (cp.async.bulk, completion counted in bytes on an mbarrier); the lanes add
// the rows up in float32 from shared memory, refill the stage they just
// read, and at the end of a tile combine their partial sums with shuffles.
// No CTA-wide barrier: 24 pieces (192 KB) per SM stay in flight, so the copy
// engine, not the consumers' latency, sets the pace. One launch can pool two
// tensors (q with block_q and k with block_kv).
//
// Waits are bounded (mbar_wait); on a timeout the error word is set, the
// warp stops, and lane 0 waits (bounded) for the copies it still has in
// flight before the warp exits.
#include "nsa_device.cuh"
#include "nsa_kernels.cuh"

namespace nsa {

namespace {

constexpr int kWarps = 8;  // warps per CTA
constexpr int kWarpStages = 3;
constexpr int kPieceBytes = 8 * 1024;

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4 &v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    // bf16 -> f32 is exact: the bf16 bits are the top half of the f32 bits
    a[2 * e] += __uint_as_float(w[e] << 16);
    a[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

struct TileRef {
  const __nv_bfloat16 *src;  // first row of the tile
  float *dst;                // pooled row
  int n;                     // token rows in the tile
};

__device__ __forceinline__ TileRef tile_ref(const PoolSeg &s0, const PoolSeg &s1, long long t, int D) {
  const bool first = t < s0.total_tiles;
  const PoolSeg &s = first ? s0 : s1;
  const long long tt = first ? t : t - s0.total_tiles;
  const long long bh = tt / s.ntiles;
  const int i = (int)(tt - bh * s.ntiles);
  const int lo = i * s.block;
  TileRef r;
  r.n = min(s.block, s.S - lo);
  r.src = s.x + ((size_t)bh * s.S + lo) * D;
  r.dst = s.out + (size_t)tt * D;
  return r;
}

// The pieces of one warp, in order: its tiles t = gw, gw + nw, ... and each
// tile's rows in runs of at most PR.
template <int D>
struct PieceIter {
  static constexpr int PR = kPieceBytes / (D * 2);  // token rows per piece
  PoolSeg s0, s1;
  long long t, total, stride;
  TileRef tr;
  int p0;  // first row of the current piece in the tile
  __device__ __forceinline__ PieceIter(const PoolSeg &a, const PoolSeg &b, long long t0, long long nw)
      : s0(a), s1(b), t(t0), total(a.total_tiles + b.total_tiles), stride(nw), p0(0) {
    if (t < total) tr = tile_ref(s0, s1, t, D);
  }
  __device__ __forceinline__ bool valid() const { return t < total; }
  __device__ __forceinline__ int rows() const { return min(PR, tr.n - p0); }
  __device__ __forceinline__ void next() {
    p0 += PR;
    if (p0 >= tr.n) {
      p0 = 0;
      t += stride;
      if (t < total) tr = tile_ref(s0, s1, t, D);
    }
  }
};

template <int D, int W>
__global__ void __launch_bounds__(W * 32, 1)
    pool_kernel(PoolSeg s0, PoolSeg s1, unsigned int *clear_word, unsigned int *err) {
  constexpr int TPR = D / 8;    // lanes per token row (16 bytes each)
  constexpr int RPP = 32 / TPR;  // token rows per warp-wide pass
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  unsigned char *ring = smem + (size_t)warp * kWarpStages * kPieceBytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)W * kWarpStages * kPieceBytes) +
                   warp * kWarpStages;
  int *abort_word = reinterpret_cast<int *>(smem + (size_t)W * kWarpStages * kPieceBytes +
                                            sizeof(uint64_t) * W * kWarpStages) + warp;
  volatile int *abort = abort_word;

  if (clear_word != nullptr && blockIdx.x == 0 && tid == 0) *clear_word = 0u;
  if (lane == 0) {
    for (int s = 0; s < kWarpStages; ++s) mbar_init(&full[s], 1);
    *abort_word = 0;
    fence_mbar_init();
  }
  __syncwarp();
  // the next kernel may be scheduled now; it waits for this grid to finish
  pdl_trigger();

  const long long gw = (long long)blockIdx.x * W + warp;
  const long long nw = (long long)gridDim.x * W;
  PieceIter<D> prod(s0, s1, gw, nw);  // lane 0's copy cursor
  PieceIter<D> cons(s0, s1, gw, nw);  // the warp's read cursor
  long long issued = 0;
  if (lane == 0) {
    for (; issued < kWarpStages && prod.valid(); ++issued, prod.next()) {
      const uint32_t bytes = (uint32_t)(prod.rows() * D * 2);
      mbar_arrive_expect_tx(&full[issued], bytes);
      bulk_load(ring + (size_t)issued * kPieceBytes, prod.tr.src + (size_t)prod.p0 * D, bytes, &full[issued]);
    }
  }

  const int c = lane % TPR;
  const int r0 = lane / TPR;
  float a[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) a[e] = 0.f;
  long long g = 0;  // pieces consumed
  bool ok = true;
  for (; cons.valid(); cons.next(), ++g) {
    const int st = (int)(g % kWarpStages);
    const uint32_t par = (uint32_t)(g / kWarpStages) & 1u;
    int w = 1;
    if (lane == 0) w = mbar_wait(&full[st], par, abort, err, 0x20) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, w, 0)) {
      ok = false;
      break;
    }
    mbar_try_wait(&full[st], par);  // every lane observes the completed phase
    const unsigned char *stage = ring + (size_t)st * kPieceBytes;
    const int rows = cons.rows();
    for (int r = r0; r < rows; r += 4 * RPP) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = (r + u * RPP < rows) ? *reinterpret_cast<const uint4 *>(stage + (size_t)(r + u * RPP) * D * 2 + c * 16)
                                    : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < 4; ++u) acc_bf16x8(a, v[u]);
    }
    __syncwarp();
    // refill the stage just read with the piece kWarpStages ahead
    if (lane == 0 && prod.valid()) {
      fence_proxy_async_smem();
      const uint32_t bytes = (uint32_t)(prod.rows() * D * 2);
      mbar_arrive_expect_tx(&full[st], bytes);
      bulk_load(ring + (size_t)st * kPieceBytes, prod.tr.src + (size_t)prod.p0 * D, bytes, &full[st]);
      ++issued;
      prod.next();
    }
    if (cons.p0 + PieceIter<D>::PR >= cons.tr.n) {
      // last piece of the tile: lanes holding the same columns are
      // lane ^ TPR, lane ^ 2 TPR, ...
#pragma unroll
      for (int off = TPR; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] += __shfl_xor_sync(0xffffffffu, a[e], off);
      }
      if (lane < TPR) {
        const float nf = (float)cons.tr.n;
        float4 *o = reinterpret_cast<float4 *>(cons.tr.dst + c * 8);
        o[0] = make_float4(a[0] / nf, a[1] / nf, a[2] / nf, a[3] / nf);
        o[1] = make_float4(a[4] / nf, a[5] / nf, a[6] / nf, a[7] / nf);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] = 0.f;
    }
  }
  if (!ok && lane == 0) {
    // wait (bounded, ignoring the abort flag) for copies still in flight
    int never = 0;
    for (long long n = (issued > kWarpStages ? issued - kWarpStages : 0); n < issued; ++n)
      mbar_wait(&full[n % kWarpStages], (uint32_t)(n / kWarpStages) & 1u, &never, err, 0x22);
  }
  __syncwarp();
}

template <int D, int W>
cudaError_t launch_pool_d(const PoolSeg &a, const PoolSeg &b, int grid, unsigned int *clear_word,
                          unsigned int *err, cudaStream_t stream) {
  constexpr size_t smem = (size_t)W * kWarpStages * (kPieceBytes + sizeof(uint64_t)) + W * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(pool_kernel<D, W>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  pool_kernel<D, W><<<grid, W * 32, smem, stream>>>(a, b, clear_word, err);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const PoolSeg &a, const PoolSeg &b, int D, int num_sms, unsigned int *clear_word,
                        unsigned int *err, cudaStream_t stream) {
  const long long total = a.total_tiles + b.total_tiles;
  if (total == 0 && clear_word == nullptr) return cudaSuccess;
  const long long want = (total + kWarps - 1) / kWarps;  // one tile per warp at least
  const int grid = total == 0 ? 1 : (int)(want < num_sms ? want : num_sms);
  return D == 64 ? launch_pool_d<64, kWarps>(a, b, grid, clear_word, err, stream)
                 : launch_pool_d<128, kWarps>(a, b, grid, clear_word, err, stream);
}

}  // namespace nsa
