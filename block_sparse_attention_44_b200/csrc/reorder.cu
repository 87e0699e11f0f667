// Video-aware block organisation: natural (t, y, x) raster order <-> 3D-tile-major
// order ("FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for Video
// Generation", abstract and §3.1 overview; tiles are raster-numbered boxes).
//
// One CTA moves one tile of one (b, h): S rows of d bf16.  On the natural side a
// tile is tt*ty runs of tx consecutive tokens (tx*d*2 contiguous bytes each), on
// the tile-major side it is one contiguous S*d*2-byte block, so both sides stream
// whole 32-byte sectors with 16-byte vector accesses.  Pure HBM copy: 2*S*d*2
// bytes of traffic per CTA.
#include "fva_common.cuh"
#include "fva_internal.h"

namespace fva {
namespace {

constexpr int kReorderThreads = 256;

template <int D>
__global__ void __launch_bounds__(kReorderThreads) reorder_kernel(const uint4* __restrict__ src,
                                                                  uint4* __restrict__ dst, int N, int Y, int X,
                                                                  int tt, int ty, int tx, int nY, int nX, int S,
                                                                  int Nb, int inverse) {
  constexpr int CPR = D * 2 / 16;   // 16-byte chunks per token row
  constexpr int U = 8;              // chunks in flight per thread
  extern __shared__ int nat_row[];  // natural token index of tile row r
  const long long blk = blockIdx.x;
  const long long bh = blk / Nb;
  const int b = static_cast<int>(blk - bh * Nb);
  const int bt = b / (nY * nX);
  const int rem = b - bt * nY * nX;
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

}  // namespace

cudaError_t launch_reorder(const void* src, void* dst, const fva_geom& g, const Dims& D, bool inverse,
                           cudaStream_t s, int* launches) {
  const dim3 grid(static_cast<unsigned>(D.rows()));
  const size_t smem = static_cast<size_t>(D.S) * sizeof(int);
  if (D.d == 128) {
    reorder_kernel<128><<<grid, kReorderThreads, smem, s>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), D.N, g.Y, g.X, g.tt, g.ty, g.tx, D.nY, D.nX, D.S,
        D.Nb, inverse ? 1 : 0);
  } else {
    reorder_kernel<64><<<grid, kReorderThreads, smem, s>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), D.N, g.Y, g.X, g.tt, g.ty, g.tx, D.nY, D.nX, D.S,
        D.Nb, inverse ? 1 : 0);
  }
  ++*launches;
  return cudaGetLastError();
}

}  // namespace fva
