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

namespace sa {

// ------------------------------------------------------------------------ tile + 3-D RoPE
// VSA2 page, section 2.2 "Permutation": the permutation to cube-major order is applied once,
// at the start of the transformer, with a matching permutation of the RoPE embeddings
// (RoFormer: channel pair (x_2i, x_2i+1) of a token at position m is rotated by m * theta_i).
// Here the rotation is fused into the permutation: each token is rotated by its own (t, h, w)
// while it moves to (or, for the inverse, from) its cube-major slot.  The head dimension is
// split into three even sections (dt, dh, dw) rotated by t, h and w; the cosines and sines come
// from caller tables: lat_t rows of dt/2 entries, then lat_h rows of dh/2, then lat_w rows of
// dw/2.  One thread per 16-byte vector of a tiled row (4 bf16 or 2 fp32 channel pairs).
struct RopeArgs {
  int dt, dh, dw;
  int off_h, off_w;  // first table row of the h and w blocks
  const float* cs;
  const float* sn;
};

template <int ESZ, bool TO_TILED>
__global__ void tile_rope_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, Geom g, long long rows_out,
                                 int vec_per_row, RopeArgs r) {
  constexpr int EPV = 16 / ESZ;  // elements per vector
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
  if (!valid) {
    if (TO_TILED) dst[row * vec_per_row + v] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4 in = TO_TILED ? src[lat_row * vec_per_row + v] : src[row * vec_per_row + v];
  uint32_t wv[4] = {in.x, in.y, in.z, in.w};
  float x[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) {
    if constexpr (ESZ == 2)
      x[e] = __uint_as_float((e & 1) ? (wv[e >> 1] & 0xffff0000u) : (wv[e >> 1] << 16));
    else
      x[e] = __uint_as_float(wv[e]);
  }
#pragma unroll
  for (int q = 0; q < EPV / 2; ++q) {
    const int chn = v * EPV + 2 * q;  // first channel of the pair
    int trow;
    if (chn < r.dt)
      trow = t * (r.dt >> 1) + (chn >> 1);
    else if (chn < r.dt + r.dh)
      trow = r.off_h + h * (r.dh >> 1) + ((chn - r.dt) >> 1);
    else
      trow = r.off_w + w * (r.dw >> 1) + ((chn - r.dt - r.dh) >> 1);
    const float cs = __ldg(r.cs + trow), sn = TO_TILED ? __ldg(r.sn + trow) : -__ldg(r.sn + trow);
    const float a = x[2 * q], b = x[2 * q + 1];
    x[2 * q] = fmaf(a, cs, -b * sn);
    x[2 * q + 1] = fmaf(a, sn, b * cs);
  }
  uint4 out;
  if constexpr (ESZ == 2) {
    out = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                     pack_bf16x2(x[6], x[7]));
  } else {
    out = make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
  }
  if (TO_TILED)
    dst[row * vec_per_row + v] = out;
  else
    dst[lat_row * vec_per_row + v] = out;
}

cudaError_t launch_tile_rope(const void* src, void* dst, const Geom& g, int BH, int D, int elem_bytes, bool to_tiled,
                             int dt, int dh, int dw, const float* cs, const float* sn, cudaStream_t stream) {
  RopeArgs r;
  r.dt = dt;
  r.dh = dh;
  r.dw = dw;
  r.off_h = g.lat_t * (dt / 2);
  r.off_w = r.off_h + g.lat_h * (dh / 2);
  r.cs = cs;
  r.sn = sn;
  const int vec_per_row = D * elem_bytes / 16;
  const long long rows = (long long)BH * g.Npad;
  const long long total = rows * vec_per_row;
  const unsigned blocks = static_cast<unsigned>((total + 255) / 256);
  auto s = static_cast<const uint4*>(src);
  auto d = static_cast<uint4*>(dst);
  if (elem_bytes == 2) {
    if (to_tiled)
      tile_rope_kernel<2, true><<<blocks, 256, 0, stream>>>(s, d, g, rows, vec_per_row, r);
    else
      tile_rope_kernel<2, false><<<blocks, 256, 0, stream>>>(s, d, g, rows, vec_per_row, r);
  } else {
    if (to_tiled)
      tile_rope_kernel<4, true><<<blocks, 256, 0, stream>>>(s, d, g, rows, vec_per_row, r);
    else
      tile_rope_kernel<4, false><<<blocks, 256, 0, stream>>>(s, d, g, rows, vec_per_row, r);
  }
  return cudaGetLastError();
}

}  // namespace sa
