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

// One thread per pair: merge two ascending lists of length n0, n1 (second may be absent).
__device__ __forceinline__ int merge_two(const int32_t* a, int n0, const int32_t* b, int n1, int32_t* out) {
  int x = 0, y = 0, k = 0;
  while (x < n0 || y < n1) {
    const int va = x < n0 ? a[x] : 0x7fffffff;
    const int vb = y < n1 ? b[y] : 0x7fffffff;
    if (va == vb) {
      out[k++] = (va << 2) | 3;
      ++x;
      ++y;
    } else if (va < vb) {
      out[k++] = (va << 2) | 1;
      ++x;
    } else {
      out[k++] = (vb << 2) | 2;
      ++y;
    }
  }
  return k;
}

// Query-cube pairs: union of kv_index rows 2p and 2p+1 of each (b, h).
// u_list: [BH, P, ucap] with ucap = min(2*cap, T), u_cnt: [BH, P], P = ceil(T/2).  Entries outside [0, T) or
// counts outside [0, cap] are dropped (and reported as index errors).
__global__ void query_pair_union_kernel(const int32_t* __restrict__ kv_index, const int32_t* __restrict__ kv_count,
                                        int32_t* __restrict__ u_list, int32_t* __restrict__ u_cnt, int BH, int T,
                                        int cap, int ucap, DevStatus* st) {
  const int P = (T + 1) >> 1;
  const long long id = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (id >= static_cast<long long>(BH) * P) return;
  const int bh = static_cast<int>(id / P), p = static_cast<int>(id % P);
  const int i0 = 2 * p, i1 = 2 * p + 1;
  int n[2] = {0, 0};
  const int32_t* src[2] = {nullptr, nullptr};
  for (int u = 0; u < 2; ++u) {
    const int i = u ? i1 : i0;
    if (i >= T) continue;
    const size_t r = static_cast<size_t>(bh) * T + i;
    int c = kv_count[r];
    if (c < 0 || c > cap) {
      flag_error(st, DEVERR_INDEX, 0);
      c = c < 0 ? 0 : cap;
    }
    n[u] = c;
    src[u] = kv_index + r * cap;
  }
  int32_t* out = u_list + id * static_cast<long long>(ucap);
  // drop out-of-range entries while merging: copy valid prefixes through local filtering
  int x = 0, y = 0, k = 0;
  while (x < n[0] || y < n[1]) {
    int va = 0x7fffffff, vb = 0x7fffffff;
    if (x < n[0]) {
      va = src[0][x];
      if (va < 0 || va >= T) {
        flag_error(st, DEVERR_INDEX, 0);
        ++x;
        continue;
      }
    }
    if (y < n[1]) {
      vb = src[1][y];
      if (vb < 0 || vb >= T) {
        flag_error(st, DEVERR_INDEX, 0);
        ++y;
        continue;
      }
    }
    if (va == vb) {
      out[k++] = (va << 2) | 3;
      ++x;
      ++y;
    } else if (va < vb) {
      out[k++] = (va << 2) | 1;
      ++x;
    } else {
      out[k++] = (vb << 2) | 2;
      ++y;
    }
  }
  u_cnt[id] = k;
}

// Key-cube pairs: union of the transposed lists (CSR q_off/q_idx) of cubes 2p and 2p+1
// (row stride T: a union of query cubes has at most T entries).
__global__ void key_pair_union_kernel(const int32_t* __restrict__ q_off, const int32_t* __restrict__ q_idx,
                                      int32_t* __restrict__ u_list, int32_t* __restrict__ u_cnt, int BH, int T,
                                      int cap) {
  const int P = (T + 1) >> 1;
  const long long id = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (id >= static_cast<long long>(BH) * P) return;
  const int bh = static_cast<int>(id / P), p = static_cast<int>(id % P);
  const int j0 = 2 * p, j1 = 2 * p + 1;
  const int32_t* off = q_off + static_cast<size_t>(bh) * (T + 1);
  const int b0 = off[j0], n0 = off[j0 + 1] - b0;
  int b1 = 0, n1 = 0;
  if (j1 < T) {
    b1 = off[j1];
    n1 = off[j1 + 1] - b1;
  }
  u_cnt[id] = merge_two(q_idx + b0, n0, q_idx + b1, n1, u_list + id * static_cast<long long>(T));
}

cudaError_t launch_query_pair_union(const int32_t* kv_index, const int32_t* kv_count, int32_t* u_list,
                                    int32_t* u_cnt, int BH, int T, int cap, DevStatus* st, cudaStream_t stream) {
  const long long n = static_cast<long long>(BH) * ((T + 1) >> 1);
  const int ucap = 2 * cap < T ? 2 * cap : T;
  query_pair_union_kernel<<<static_cast<unsigned>((n + 127) / 128), 128, 0, stream>>>(kv_index, kv_count, u_list,
                                                                                       u_cnt, BH, T, cap, ucap, st);
  return cudaGetLastError();
}

cudaError_t launch_key_pair_union(const int32_t* q_off, const int32_t* q_idx, int32_t* u_list, int32_t* u_cnt,
                                  int BH, int T, int cap, cudaStream_t stream) {
  const long long n = static_cast<long long>(BH) * ((T + 1) >> 1);
  key_pair_union_kernel<<<static_cast<unsigned>((n + 127) / 128), 128, 0, stream>>>(q_off, q_idx, u_list, u_cnt, BH,
                                                                                     T, cap);
  return cudaGetLastError();
}

}  // namespace sa
