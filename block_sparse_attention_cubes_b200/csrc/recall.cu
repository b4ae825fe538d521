// Router recall: the share of each query's true attention mass that its kept blocks hold.
//
// SpargeAttention2 page, equation 8: tau = sum_j p_j m_j for the token-level softmax p and the
// block mask m; VSA page, "Kernel Implementation" (Top-32 keeps 50-90% of the mass).  With lse
// the natural log of a row's softmax normaliser, tau = exp(lse over the kept keys - lse over all
// keys), so two calls of the fine forward (with the router's lists and with every block) give
// it without materialising p.  One warp per (bh, cube): tau per valid row and its mean over the
// cube's valid rows; padding rows get 0.
#include <cmath>

#include "geometry.cuh"
#include "kernels.h"

namespace sa {
namespace {

__global__ void __launch_bounds__(256) recall_kernel(const float* __restrict__ lse_kept,
                                                     const float* __restrict__ lse_all, float* __restrict__ recall,
                                                     float* __restrict__ cube_recall, Geom g, int BH) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long cube = blockIdx.x * 8LL + warp;
  if (cube >= static_cast<long long>(BH) * g.T) return;
  int vt, vh, vw;
  cube_extent(g, static_cast<int>(cube % g.T), vt, vh, vw);
  float sum = 0.0f;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int s = lane + 32 * u;
    const long long row = cube * 64 + s;
    float r = 0.0f;
    if (slot_valid(vt, vh, vw, s)) r = expf(lse_kept[row] - lse_all[row]);
    if (recall) recall[row] = r;
    sum += r;
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane == 0 && cube_recall) cube_recall[cube] = sum / static_cast<float>(vt * vh * vw);
}

}  // namespace

cudaError_t launch_recall(const float* lse_kept, const float* lse_all, float* recall, float* cube_recall,
                          const Geom& g, int BH, cudaStream_t stream) {
  const long long cubes = static_cast<long long>(BH) * g.T;
  recall_kernel<<<static_cast<unsigned>((cubes + 7) / 8), 256, 0, stream>>>(lse_kept, lse_all, recall, cube_recall,
                                                                             g, BH);
  return cudaGetLastError();
}

}  // namespace sa
