// Latent order <-> cube-major padded order (VSA page, "Cube Partitioning and Token
// Re-Indexing"; VSA2 page, section 2.2 "Permutation").  Pure data movement: one
// 16-byte vector per thread, rows of D * elem_bytes bytes (a multiple of 16).
#include "geometry.cuh"
#include "kernels.h"

namespace sa {

__global__ void tile_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, Geom g, long long rows_out,
                            int vec_per_row, int to_tiled) {
  const long long tid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long total = rows_out * vec_per_row;
  if (tid >= total) return;
  const long long row = tid / vec_per_row;  // row in the tiled tensor: bh * Npad + slot
  const int v = static_cast<int>(tid - row * vec_per_row);
  const long long bh = row / g.Npad;
  const int p = static_cast<int>(row - bh * g.Npad);
  const int c = p >> 6, s = p & 63;
  const int ct = c / (g.Nh * g.Nw), ch = (c / g.Nw) % g.Nh, cw = c % g.Nw;
  const int t = 4 * ct + (s >> 4), h = 4 * ch + ((s >> 2) & 3), w = 4 * cw + (s & 3);
  const bool valid = t < g.lat_t && h < g.lat_h && w < g.lat_w;
  const long long L = (long long)g.lat_t * g.lat_h * g.lat_w;
  const long long lat_row = bh * L + ((long long)t * g.lat_h + h) * g.lat_w + w;
  if (to_tiled) {
    dst[row * vec_per_row + v] = valid ? src[lat_row * vec_per_row + v] : make_uint4(0, 0, 0, 0);
  } else if (valid) {
    dst[lat_row * vec_per_row + v] = src[row * vec_per_row + v];
  }
}

cudaError_t launch_tile(const void* src, void* dst, const Geom& g, int BH, int row_bytes, bool to_tiled,
                        cudaStream_t stream) {
  const int vec_per_row = row_bytes / 16;
  const long long rows = (long long)BH * g.Npad;
  const long long total = rows * vec_per_row;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  tile_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), g, rows, vec_per_row, to_tiled ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace sa
