// Router with 128-token query blocks and 64-token key blocks (SpargeAttention2 page,
// "Block-Pooled Attention for Efficient Mask Construction": b_q = 128, b_kv = 64 in all its
// experiments), on the cube layout: query block i is cubes 2i and 2i + 1 (the last block is one
// cube when T is odd), pooled over the valid tokens of both; keys stay per cube.  Scores, row
// softmax and the hybrid Top-k / Top-p selection are the cube router's, over a ceil(T/2) x T
// matrix; each block's list is then written for both of its cubes, so the fine kernels (which
// walk cube pairs) see one list per pair and no union waste.
//
//   pair_mean_kernel    Qbar of each block from the router's fp64 cube means, weighted by the
//                       cubes' valid-token counts (the mean over the block's valid tokens)
//   pair_score_kernel   S[bh][i][j] = scale * Qbar_block[i] . Kbar[j], fp64, 64 x 64 tiles
//   expand_lists_kernel block lists -> cube lists (the first count entries of each row)
#include "geometry.cuh"
#include "kernels.h"

namespace sa {
namespace {

__global__ void __launch_bounds__(256) pair_mean_kernel(const double* __restrict__ qbar, double* __restrict__ qpair,
                                                        Geom g, int BH, int D, int M) {
  const long long u = blockIdx.x * 256LL + threadIdx.x;
  if (u >= static_cast<long long>(BH) * M * D) return;
  const int d = static_cast<int>(u % D);
  const long long r = u / D;
  const int i = static_cast<int>(r % M);
  const long long bh = r / M;
  const int ca = 2 * i, cb = 2 * i + 1;
  const double na = cube_valid_count(g, ca);
  const double nb = cb < g.T ? static_cast<double>(cube_valid_count(g, cb)) : 0.0;
  const double a = qbar[(bh * g.T + ca) * D + d];
  const double b = cb < g.T ? qbar[(bh * g.T + cb) * D + d] : 0.0;
  qpair[u] = (na * a + nb * b) / (na + nb);
}

// One 64 x 64 tile of S per block, 4 x 4 per thread, D in 16-deep slices through shared memory.
__global__ void __launch_bounds__(256) pair_score_kernel(const double* __restrict__ qpair,
                                                         const double* __restrict__ kbar, double* __restrict__ S,
                                                         int M, int T, int D, double scale) {
  __shared__ double Qs[16][65], Ks[16][65];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const long long bh = blockIdx.z;
  const double* Q = qpair + bh * M * D;
  const double* K = kbar + bh * T * D;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  for (int k0 = 0; k0 < D; k0 += 16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + 256 * i, r = idx >> 4, k = idx & 15;
      Qs[k][r] = m0 + r < M ? Q[static_cast<long long>(m0 + r) * D + k0 + k] : 0.0;
      Ks[k][r] = n0 + r < T ? K[static_cast<long long>(n0 + r) * D + k0 + k] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      double a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Qs[k][ty * 4 + i], b[i] = Ks[k][tx * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  double* out = S + bh * M * T;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < T) out[static_cast<long long>(m) * T + n] = acc[i][j] * scale;
    }
  }
}

// One thread per (bh, cube, entry): cube c takes block c / 2's list and count.
__global__ void __launch_bounds__(256) expand_lists_kernel(const int32_t* __restrict__ blk_index,
                                                           const int32_t* __restrict__ blk_count,
                                                           int32_t* __restrict__ kv_index, int32_t* __restrict__ kv_count,
                                                           int BH, int T, int M, int cap) {
  const long long u = blockIdx.x * 256LL + threadIdx.x;
  if (u >= static_cast<long long>(BH) * T * cap) return;
  const int e = static_cast<int>(u % cap);
  const long long r = u / cap;
  const int c = static_cast<int>(r % T);
  const long long bh = r / T;
  const long long src = bh * M + c / 2;
  const int n = blk_count[src];
  if (e == 0) kv_count[r] = n;
  if (e < n) kv_index[u] = blk_index[src * cap + e];
}

}  // namespace

cudaError_t launch_plan_bq128(const void* q, const void* k, const Geom& g, int BH, int D, double scale, int top_k,
                              float top_p, int cap, int32_t* kv_index, int32_t* kv_count, double* qbar, double* kbar,
                              double* qpair, double* S, int32_t* blk_index, int32_t* blk_count, DevStatus* st,
                              cudaStream_t stream, int* launches) {
  const int M = (g.T + 1) / 2;
  cudaError_t e = launch_pool(q, k, g, BH, D, qbar, kbar, stream);
  if (e != cudaSuccess) return e;
  const long long pm = static_cast<long long>(BH) * M * D;
  pair_mean_kernel<<<static_cast<unsigned>((pm + 255) / 256), 256, 0, stream>>>(qbar, qpair, g, BH, D, M);
  const dim3 sg(static_cast<unsigned>((g.T + 63) / 64), static_cast<unsigned>((M + 63) / 64),
                static_cast<unsigned>(BH));
  pair_score_kernel<<<sg, 256, 0, stream>>>(qpair, kbar, S, M, g.T, D, scale);
  e = launch_select(S, blk_index, blk_count, BH * M, g.T, top_k, top_p, cap, st, stream);
  if (e != cudaSuccess) return e;
  const long long ex = static_cast<long long>(BH) * g.T * cap;
  expand_lists_kernel<<<static_cast<unsigned>((ex + 255) / 256), 256, 0, stream>>>(blk_index, blk_count, kv_index,
                                                                                    kv_count, BH, g.T, M, cap);
  *launches = 5;
  return cudaGetLastError();
}

}  // namespace sa
