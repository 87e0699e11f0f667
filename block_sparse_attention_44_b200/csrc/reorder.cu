// Video-aware block organisation: natural (t, y, x) raster order <-> 3D-tile-major
// order ("FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for Video
// Generation", abstract and §3.1 overview; tiles are raster-numbered boxes).
//
// One CTA moves one tile of one (b, h): S rows of d bf16.  The tile numbered b is
// raster tile b, or tile order[b] when a numbering table is given (Hilbert
// numbering).  On the natural side a tile is tt*ty runs of tx consecutive tokens
// (tx*d*2 contiguous bytes each), on the tile-major side it is one contiguous
// S*d*2-byte block, so both sides stream whole 32-byte sectors with 16-byte vector
// accesses.  Pure HBM copy: 2*S*d*2 bytes of traffic per CTA.  reorder_pool_kernel
// also writes the tile's float64 mean (the routing pool step riding on the same pass:
// no second read of Q or K).
#include "fva_common.cuh"
#include "fva_internal.h"

namespace fva {
namespace {

constexpr int kReorderThreads = 256;

template <int D>
__global__ void __launch_bounds__(kReorderThreads) reorder_kernel(const uint4* __restrict__ src,
                                                                  uint4* __restrict__ dst, int N, int Y, int X,
                                                                  int tt, int ty, int tx, int nY, int nX, int S,
                                                                  int Nb, int inverse, const int32_t* __restrict__ order,
                                                                  int* dev_err) {
  constexpr int CPR = D * 2 / 16;   // 16-byte chunks per token row
  constexpr int U = 8;              // chunks in flight per thread
  extern __shared__ int nat_row[];  // natural token index of tile row r
  const long long blk = blockIdx.x;
  const long long bh = blk / Nb;
  const int b = static_cast<int>(blk - bh * Nb);
  const int tr = order ? order[b] : b;   // raster index of the tile numbered b
  if (tr < 0 || tr >= Nb) {
    if (threadIdx.x == 0) set_device_error(dev_err, kDevErrBadIndex);
    return;
  }
  const int bt = tr / (nY * nX);
  const int rem = tr - bt * nY * nX;
  const int by = rem / nX;
  const int bx = rem - by * nX;
  const int tyx = ty * tx;
  for (int r = threadIdx.x; r < S; r += blockDim.x) {
    const int lt = r / tyx;
    const int rr = r - lt * tyx;
    const int ly = rr / tx;
    const int lx = rr - ly * tx;
    nat_row[r] = ((bt * tt + lt) * Y + by * ty + ly) * X + bx * tx + lx;
  }
  __syncthreads();
  const long long base = bh * static_cast<long long>(N);
  const long long tile0 = base + static_cast<long long>(b) * S;
  const int total = S * CPR;
  for (int c0 = threadIdx.x; c0 < total; c0 += blockDim.x * U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * blockDim.x;
      if (c < total) {
        const int r = c / CPR;
        const int col = c - r * CPR;
        const long long srow = inverse ? (tile0 + r) : (base + nat_row[r]);
        v[u] = __ldg(src + srow * CPR + col);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * blockDim.x;
      if (c < total) {
        const int r = c / CPR;
        const int col = c - r * CPR;
        const long long drow = inverse ? (base + nat_row[r]) : (tile0 + r);
        __stcs(dst + drow * CPR + col, v[u]);
      }
    }
  }
}

// reorder_kernel (forward) that also writes the float64 mean of the tile's rows to
// pooled[blk] ([B*H*Nb, D]).  Thread t holds column chunk t % CPR of rows
// t / CPR + RG * u, so it sums those rows in ascending order and the RG row groups are
// then added in order: the same sums, in the same order, as the routing pool kernel.
template <int D>
__global__ void __launch_bounds__(kReorderThreads) reorder_pool_kernel(const uint4* __restrict__ src,
                                                                       uint4* __restrict__ dst,
                                                                       double* __restrict__ pooled, int N, int Y,
                                                                       int X, int tt, int ty, int tx, int nY, int nX,
                                                                       int S, int Nb, const int32_t* __restrict__ order,
                                                                       int* dev_err) {
  constexpr int CPR = D * 2 / 16;            // 16-byte chunks per token row
  constexpr int RG = kReorderThreads / CPR;  // row groups
  constexpr int U = 8;                       // rows in flight per thread
  extern __shared__ int nat_row[];           // natural token index of tile row r
  __shared__ double part[RG][D];
  const long long blk = blockIdx.x;
  const long long bh = blk / Nb;
  const int b = static_cast<int>(blk - bh * Nb);
  const int tr = order ? order[b] : b;   // raster index of the tile numbered b
  if (tr < 0 || tr >= Nb) {
    if (threadIdx.x == 0) set_device_error(dev_err, kDevErrBadIndex);
    return;
  }
  const int bt = tr / (nY * nX);
  const int rem = tr - bt * nY * nX;
  const int by = rem / nX;
  const int bx = rem - by * nX;
  const int tyx = ty * tx;
  for (int r = threadIdx.x; r < S; r += blockDim.x) {
    const int lt = r / tyx;
    const int rr = r - lt * tyx;
    const int ly = rr / tx;
    const int lx = rr - ly * tx;
    nat_row[r] = ((bt * tt + lt) * Y + by * ty + ly) * X + bx * tx + lx;
  }
  __syncthreads();
  const long long base = bh * static_cast<long long>(N);
  const long long tile0 = base + static_cast<long long>(b) * S;
  const int col = threadIdx.x % CPR;
  const int rg = threadIdx.x / CPR;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int r0 = rg; r0 < S; r0 += RG * U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * RG;
      if (r < S) v[u] = __ldg(src + (base + nat_row[r]) * CPR + col);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u * RG;
      if (r < S) {
        __stcs(dst + (tile0 + r) * CPR + col, v[u]);
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] += static_cast<double>(__uint_as_float(w[q] << 16));
          acc[2 * q + 1] += static_cast<double>(__uint_as_float(w[q] & 0xFFFF0000u));
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][col * 8 + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kReorderThreads) {
    double sum = 0.0;
#pragma unroll 8
    for (int g2 = 0; g2 < RG; ++g2) sum += part[g2][c];
    pooled[blk * D + c] = sum / static_cast<double>(S);
  }
}

}  // namespace

cudaError_t launch_reorder_pool(const void* src, void* dst, double* pooled, const fva_geom& g, const Dims& D,
                                int* dev_err, cudaStream_t s, int* launches) {
  const dim3 grid(static_cast<unsigned>(D.rows()));
  const size_t smem = static_cast<size_t>(D.S) * sizeof(int);
  if (D.d == 128)
    reorder_pool_kernel<128><<<grid, kReorderThreads, smem, s>>>(static_cast<const uint4*>(src),
                                                                 static_cast<uint4*>(dst), pooled, D.N, g.Y, g.X,
                                                                 g.tt, g.ty, g.tx, D.nY, D.nX, D.S, D.Nb, D.order,
                                                                 dev_err);
  else
    reorder_pool_kernel<64><<<grid, kReorderThreads, smem, s>>>(static_cast<const uint4*>(src),
                                                                static_cast<uint4*>(dst), pooled, D.N, g.Y, g.X,
                                                                g.tt, g.ty, g.tx, D.nY, D.nX, D.S, D.Nb, D.order,
                                                                dev_err);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_reorder(const void* src, void* dst, const fva_geom& g, const Dims& D, bool inverse,
                           int* dev_err, cudaStream_t s, int* launches) {
  const dim3 grid(static_cast<unsigned>(D.rows()));
  const size_t smem = static_cast<size_t>(D.S) * sizeof(int);
  if (D.d == 128) {
    reorder_kernel<128><<<grid, kReorderThreads, smem, s>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), D.N, g.Y, g.X, g.tt, g.ty, g.tx, D.nY, D.nX, D.S,
        D.Nb, inverse ? 1 : 0, D.order, dev_err);
  } else {
    reorder_kernel<64><<<grid, kReorderThreads, smem, s>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), D.N, g.Y, g.X, g.tt, g.ty, g.tx, D.nY, D.nX, D.S,
        D.Nb, inverse ? 1 : 0, D.order, dev_err);
  }
  ++*launches;
  return cudaGetLastError();
}

}  // namespace fva
