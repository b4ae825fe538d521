// Pair lists for the M = 128 fine-stage kernels.
//
// The tensor cores run at full rate with 128-row operands, but a cube holds 64 tokens.
// The forward and dQ kernels therefore process two adjacent query cubes (2p, 2p+1) of one
// head together and walk the union of their two KV index lists; every union entry carries
// two membership bits telling which of the two cubes selected that key cube, and the
// rows of the other cube are masked for it.  The dK/dV kernel does the same for two
// adjacent key cubes over the union of their transposed (query-cube) lists.
//
// Entry encoding: (block id << 2) | (1 if in the first list) | (2 if in the second list).
// Lists are ascending, so the merge keeps ascending block ids.
#include "kernels.h"

namespace sa {

// Query-cube pairs: union of kv_index rows 2p and 2p+1 of each (b, h).
// u_list: [BH, P, ucap] with ucap = min(2*cap, T), u_cnt: [BH, P], P = ceil(T/2).  Entries outside [0, T) or
// counts outside [0, cap] are dropped (and reported as index errors).  One warp per pair: both
// lists are scattered into two bit rows in shared memory (order-independent), then read out in
// ascending block order with a warp prefix sum placing each word's entries.
constexpr int QPU_WARPS = 8;
__global__ void __launch_bounds__(QPU_WARPS * 32)
    query_pair_union_kernel(const int32_t* __restrict__ kv_index, const int32_t* __restrict__ kv_count,
                            int32_t* __restrict__ u_list, int32_t* __restrict__ u_cnt, int BH, int T, int cap,
                            int ucap, DevStatus* st) {
  extern __shared__ uint32_t qpu_bits[];  // [QPU_WARPS][2][W]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = (T + 1) >> 1, W = (T + 31) >> 5;
  const long long id = blockIdx.x * static_cast<long long>(QPU_WARPS) + warp;
  if (id >= static_cast<long long>(BH) * P) return;
  const int bh = static_cast<int>(id / P), p = static_cast<int>(id % P);
  uint32_t* ba = qpu_bits + static_cast<size_t>(warp) * 2 * W;
  uint32_t* bb = ba + W;
  for (int w = lane; w < 2 * W; w += 32) ba[w] = 0u;
  __syncwarp();
  for (int u = 0; u < 2; ++u) {
    const int i = 2 * p + u;
    if (i >= T) continue;
    const size_t r = static_cast<size_t>(bh) * T + i;
    int c = kv_count[r];
    if (c < 0 || c > cap) {
      if (lane == 0) flag_error(st, DEVERR_INDEX, 0);
      c = c < 0 ? 0 : cap;
    }
    const int32_t* src = kv_index + r * cap;
    uint32_t* dst = u ? bb : ba;
    for (int t = lane; t < c; t += 32) {
      const int j = src[t];
      if (j < 0 || j >= T) {
        flag_error(st, DEVERR_INDEX, 0);
        continue;
      }
      atomicOr(dst + (j >> 5), 1u << (j & 31));
    }
  }
  __syncwarp();
  int32_t* out = u_list + id * static_cast<long long>(ucap);
  int base = 0;
  for (int w0 = 0; w0 < W; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t a = w < W ? ba[w] : 0u, b = w < W ? bb[w] : 0u;
    uint32_t u = a | b;
    const int cnt = __popc(u);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int k = base + incl - cnt;
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1u;
      if (k < ucap)
        out[k] = ((w * 32 + bit) << 2) | static_cast<int>((a >> bit) & 1u) | (static_cast<int>((b >> bit) & 1u) << 1);
      ++k;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) u_cnt[id] = base < ucap ? base : ucap;
}

// ---------------------------------------------------------------- key-cube pairs
// The selection as a bit matrix: bit i of bits[bh][j] (words of 32 query cubes) is set when
// query cube i selected key cube j.  atomicOr makes the result independent of the order of
// the writes.  One warp per query row (bh, i).
__global__ void selection_bits_kernel(const int32_t* __restrict__ kv_index, const int32_t* __restrict__ kv_count,
                                      uint32_t* __restrict__ bits, int BH, int T, int cap, int W, DevStatus* st) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x * 8LL + warp;
  if (row >= static_cast<long long>(BH) * T) return;
  const int bh = static_cast<int>(row / T), i = static_cast<int>(row % T);
  int n = kv_count[row];
  if (n < 0 || n > cap) {
    if (lane == 0) flag_error(st, DEVERR_INDEX, 0);
    n = n < 0 ? 0 : cap;
  }
  const int32_t* lst = kv_index + row * cap;
  uint32_t* col0 = bits + static_cast<size_t>(bh) * T * W;
  for (int t = lane; t < n; t += 32) {
    const int j = lst[t];
    if (j < 0 || j >= T) {
      flag_error(st, DEVERR_INDEX, 0);
      continue;
    }
    atomicOr(col0 + static_cast<size_t>(j) * W + (i >> 5), 1u << (i & 31));
  }
}

// Key-cube pairs: union of the query cubes that selected key cube 2p or 2p+1, ascending, as
// entries (query cube << 2) | (1 if it selected 2p) | (2 if it selected 2p+1); row stride T.
// One warp per pair: lane w takes words w, w+32, ...; a warp prefix sum places each word's
// entries.
__global__ void key_pair_union_kernel(const uint32_t* __restrict__ bits, int32_t* __restrict__ u_list,
                                      int32_t* __restrict__ u_cnt, int BH, int T, int W) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = (T + 1) >> 1;
  const long long id = blockIdx.x * 8LL + warp;
  if (id >= static_cast<long long>(BH) * P) return;
  const int bh = static_cast<int>(id / P), p = static_cast<int>(id % P);
  const uint32_t* c0 = bits + (static_cast<size_t>(bh) * T + 2 * p) * W;
  const uint32_t* c1 = (2 * p + 1 < T) ? c0 + W : nullptr;
  int32_t* out = u_list + id * static_cast<long long>(T);
  int base = 0;
  for (int w0 = 0; w0 < W; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t a = w < W ? c0[w] : 0u;
    const uint32_t b = (w < W && c1) ? c1[w] : 0u;
    uint32_t u = a | b;
    const int cnt = __popc(u);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int k = base + incl - cnt;
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1u;
      out[k++] = ((w * 32 + bit) << 2) | static_cast<int>((a >> bit) & 1u) | (static_cast<int>((b >> bit) & 1u) << 1);
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) u_cnt[id] = base;
}

cudaError_t launch_query_pair_union(const int32_t* kv_index, const int32_t* kv_count, int32_t* u_list,
                                    int32_t* u_cnt, int BH, int T, int cap, DevStatus* st, cudaStream_t stream) {
  const long long n = static_cast<long long>(BH) * ((T + 1) >> 1);
  const int ucap = 2 * cap < T ? 2 * cap : T;
  const size_t smem = sizeof(uint32_t) * QPU_WARPS * 2 * ((T + 31) / 32);  // 16 KB at T = 8192
  query_pair_union_kernel<<<static_cast<unsigned>((n + QPU_WARPS - 1) / QPU_WARPS), QPU_WARPS * 32, smem, stream>>>(
      kv_index, kv_count, u_list, u_cnt, BH, T, cap, ucap, st);
  return cudaGetLastError();
}

cudaError_t launch_key_pair_union(const int32_t* kv_index, const int32_t* kv_count, uint32_t* bits, int32_t* u_list,
                                  int32_t* u_cnt, int BH, int T, int cap, DevStatus* st, cudaStream_t stream) {
  const int W = (T + 31) / 32;
  cudaError_t e = cudaMemsetAsync(bits, 0, sizeof(uint32_t) * static_cast<size_t>(BH) * T * W, stream);
  if (e != cudaSuccess) return e;
  const long long rows = static_cast<long long>(BH) * T;
  selection_bits_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(kv_index, kv_count, bits, BH, T,
                                                                                   cap, W, st);
  const long long pairs = static_cast<long long>(BH) * ((T + 1) >> 1);
  key_pair_union_kernel<<<static_cast<unsigned>((pairs + 7) / 8), 256, 0, stream>>>(bits, u_list, u_cnt, BH, T, W);
  return cudaGetLastError();
}

}  // namespace sa
