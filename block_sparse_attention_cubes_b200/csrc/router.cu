// Router: cube mean pooling -> block scores -> row softmax -> hybrid Top-k U Top-p ->
// ascending KV index lists.
//
//  * pooling ........ SpargeAttention2 page, "Block-Pooled Attention for Efficient Mask
//                     Construction", step 2 (mean pooling); VSA page, "The Coarse Stage"
//  * scores ......... same section, step 3: S = Qbar Kbar^T / sqrt(d)
//  * selection ...... "The Hybrid Top-k+Top-p Masking Rule", equation 9 and "Definition of
//                     the two component selectors" (Top-k: the ceil(k% T_n) largest; Top-p:
//                     the shortest descending prefix whose sum reaches p of the total)
//  * index lists .... VSA page, "Kernel Implementation": contiguous arrays of block indices
//
// Precision: the selection is an integer decision taken from floating-point scores, so
// the pooled means and the scores are carried in fp64 (the means are exact sums of the
// bf16/e4m3 inputs), and the softmax masses are summed as 64-bit fixed-point integers
// (exp(s - max) * 2^50, truncated), which makes every sum exact and order-independent.
// The softmax normalisation itself is never materialised: Top-p compares prefix sums of
// exp(s - max) with p times their total, which is the same test on P = exp(s - max) / Z.
#include <cfloat>
#include <cmath>

#include "geometry.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace sa {

// ------------------------------------------------------------------------ pooling
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  // 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is subnormal.
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = (e == 0u) ? static_cast<float>(m) * (1.0f / 512.0f)
                      : __uint_as_float(((e + 120u) << 23) | (m << 20));
  if (e == 15u && m == 7u) v = __uint_as_float(0x7fc00000u);
  return (b & 0x80u) ? -v : v;
}

// grid (ceil(T/4), BH, 2); 256 threads = 4 groups of 64, one cube per group.
// ESZ = bytes per element (2: bf16, 1: e4m3).
template <int ESZ>
__global__ void __launch_bounds__(256) pool_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ k,
                                                   const float* __restrict__ q_scale,
                                                   const float* __restrict__ k_scale, double* __restrict__ qbar,
                                                   double* __restrict__ kbar, Geom g, int D) {
  constexpr int EPT = 16 / ESZ;  // elements per 16-byte vector
  __shared__ double red[4][64][EPT];
  const int grp = threadIdx.x >> 6, t64 = threadIdx.x & 63;
  const int c = blockIdx.x * 4 + grp;
  const int bh = blockIdx.y;
  const bool is_k = blockIdx.z == 1;
  const uint8_t* src = is_k ? k : q;
  const int tpr = D * ESZ / 16;  // threads per token row
  const int rows_per_iter = 64 / tpr;
  const int chunk = t64 % tpr, roff = t64 / tpr;
  double acc[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) acc[e] = 0.0;
  int vt = 0, vh = 0, vw = 0;
  if (c < g.T) {
    cube_extent(g, c, vt, vh, vw);
    const size_t row_bytes = static_cast<size_t>(D) * ESZ;
    const uint8_t* base = src + (static_cast<size_t>(bh) * g.Npad + static_cast<size_t>(c) * 64) * row_bytes;
    // four rows' loads in flight per thread before any of them is accumulated
    for (int r0 = roff; r0 < 64; r0 += 4 * rows_per_iter) {
      uint4 v[4];
      bool ok[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = r0 + u * rows_per_iter;
        ok[u] = r < 64 && slot_valid(vt, vh, vw, r);
        v[u] = ok[u] ? __ldg(reinterpret_cast<const uint4*>(base + r * row_bytes) + chunk) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (!ok[u]) continue;
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
          float f;
          if constexpr (ESZ == 2) {
            f = __uint_as_float((e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16));
          } else {
            f = e4m3_value((w[e >> 2] >> (8 * (e & 3))) & 0xffu);
          }
          acc[e] += static_cast<double>(f);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPT; ++e) red[grp][t64][e] = acc[e];
  __syncthreads();
  if (c < g.T && t64 < tpr) {
    const int n = vt * vh * vw;
    double scale = 1.0;
    if constexpr (ESZ == 1) {
      const float* sc = is_k ? k_scale : q_scale;
      scale = static_cast<double>(sc[static_cast<size_t>(bh) * g.T + c]);
    }
    double* dst = (is_k ? kbar : qbar) + (static_cast<size_t>(bh) * g.T + c) * D + chunk * EPT;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      double s = 0.0;
      for (int r = 0; r < rows_per_iter; ++r) s += red[grp][t64 + r * tpr][e];
      dst[e] = s * scale / static_cast<double>(n);
    }
  }
}

// ------------------------------------------------------------------------ block scores
// S[bh][i][j] = scale * sum_d Qbar[bh][i][d] * Kbar[bh][j][d], fp64.  One 128x128 tile per
// CTA, 16-deep slices of Qbar and Kbar staged in shared memory; each of the 256 threads
// accumulates an 8x8 block of rows ty + 16u and columns tx + 16v (u, v < 8), so a warp's
// Qbar reads are two broadcast addresses and its Kbar reads 16 consecutive doubles.
constexpr int SC_TILE = 128, SC_K = 16, SC_PAD = SC_TILE + 2;
__global__ void __launch_bounds__(256) score_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar,
                                                    double* __restrict__ S, int T, int D, double scale) {
  __shared__ double As[SC_K][SC_PAD];
  __shared__ double Bs[SC_K][SC_PAD];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * SC_TILE, j0 = blockIdx.x * SC_TILE;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const double* Q = qbar + static_cast<size_t>(bh) * T * D;
  const double* K = kbar + static_cast<size_t>(bh) * T * D;
  double acc[8][8];
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[u][v] = 0.0;
  for (int d0 = 0; d0 < D; d0 += SC_K) {
    // 128 rows x 16 doubles of each operand: thread e takes row e / 16 + 16 w, column e % 16
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const int r = (threadIdx.x >> 4) + 16 * w, dd = threadIdx.x & 15;
      As[dd][r] = (i0 + r < T) ? Q[static_cast<size_t>(i0 + r) * D + d0 + dd] : 0.0;
      Bs[dd][r] = (j0 + r < T) ? K[static_cast<size_t>(j0 + r) * D + d0 + dd] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int dd = 0; dd < SC_K; ++dd) {
      double a[8], b[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        a[u] = As[dd][ty + 16 * u];
        b[u] = Bs[dd][tx + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
  double* out = S + static_cast<size_t>(bh) * T * T;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int i = i0 + ty + 16 * u;
    if (i >= T) continue;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int j = j0 + tx + 16 * v;
      if (j < T) out[static_cast<size_t>(i) * T + j] = acc[u][v] * scale;
    }
  }
}

// ------------------------------------------------------------------------ selection
// Order key: ascending key == descending score (ties then broken by the smaller block id).
__device__ __forceinline__ uint64_t desc_key(double x) {
  x = x + 0.0;  // -0 -> +0 so that equal scores share one key
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  const uint64_t asc = (u >> 63) ? ~u : (u | 0x8000000000000000ull);
  return ~asc;
}

constexpr double kMassOne = 1125899906842624.0;  // 2^50: fixed-point unit of exp(s - max)

__device__ __forceinline__ uint64_t mass_fx(double x, double m) {
  return static_cast<uint64_t>(__double2ull_rz(exp(x - m) * kMassOne));
}

// One warp per query-block row.  Finds the boundary element of the descending order:
// the first position n-1 such that n >= max(k, 1) and the first n masses reach p * Z,
// by an 8-bit radix descent over the 64-bit order keys in which every bucket carries
// its count and its exact fixed-point mass.  Then writes the kept ids in ascending order.
__global__ void __launch_bounds__(256) select_kernel(const double* __restrict__ S, int32_t* __restrict__ kv_index,
                                                     int32_t* __restrict__ kv_count, int rows, int T, int top_k,
                                                     float top_p, int cap, DevStatus* st) {
  __shared__ uint32_t cnt_s[8][256];
  __shared__ unsigned long long mass_s[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const double* s = S + static_cast<size_t>(row) * T;
  uint32_t* cnt = cnt_s[warp];
  unsigned long long* mass = mass_s[warp];

  double m = -DBL_MAX;
#pragma unroll 4
  for (int j = lane; j < T; j += 32) m = fmax(m, s[j]);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));

  const int nk = max(1, min(top_k, T));
  const bool keep_all = (top_p >= 1.0f) || nk >= T;
  uint64_t kb = ~0ull;  // boundary key
  int jb = T;           // boundary id (elements with key == kb and id <= jb are kept)
  if (!keep_all) {
    uint64_t prefix = 0, cnt_above = 0, mass_above = 0;
    double target = -1.0;  // p <= 0: the mass test always passes
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int d = lane; d < 256; d += 32) {
        cnt[d] = 0;
        mass[d] = 0ull;
      }
      __syncwarp();
      // Keys of one binade share their top bytes, so in the first passes most lanes of a warp
      // fall in the same bucket: then the warp adds its count and (exact, fixed-point) mass
      // once instead of 32 colliding shared-memory atomics.
      // The chunks of 32 scores carry warp collectives, so the loads of four chunks are issued
      // before any of them is processed (otherwise every chunk waits out a full L2 round trip).
      for (int j0 = 0; j0 < T; j0 += 128) {
        double xs[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + 32 * u + lane;
          xs[u] = j < T ? s[j] : 0.0;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (j0 + 32 * u >= T) break;
          const int j = j0 + 32 * u + lane;
          bool part = false;
          int d = 0;
          unsigned long long mj = 0ull;
          if (j < T) {
            const double x = xs[u];
            const uint64_t kj = desc_key(x);
            if (shift == 56 || (kj >> (shift + 8)) == (prefix >> (shift + 8))) {
              part = true;
              d = static_cast<int>((kj >> shift) & 255u);
              mj = static_cast<unsigned long long>(mass_fx(x, m));
            }
          }
          const uint32_t act = __ballot_sync(0xffffffffu, part);
          if (act == 0u) continue;
          const int dl = __shfl_sync(0xffffffffu, d, __ffs(act) - 1);
          if (__all_sync(0xffffffffu, !part || d == dl)) {
            unsigned long long ms = mj;
#pragma unroll
            for (int o = 16; o; o >>= 1) ms += __shfl_xor_sync(0xffffffffu, ms, o);
            if (lane == 0) {
              atomicAdd(&cnt[dl], static_cast<uint32_t>(__popc(act)));
              atomicAdd(&mass[dl], ms);
            }
          } else if (part) {
            atomicAdd(&cnt[d], 1u);
            atomicAdd(&mass[d], mj);
          }
        }
      }
      __syncwarp();
      uint32_t lc = 0;
      unsigned long long lm = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        lc += cnt[lane * 8 + u];
        lm += mass[lane * 8 + u];
      }
      uint32_t ic = lc;
      unsigned long long im = lm;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t oc = __shfl_up_sync(0xffffffffu, ic, o);
        const unsigned long long om = __shfl_up_sync(0xffffffffu, im, o);
        if (lane >= o) {
          ic += oc;
          im += om;
        }
      }
      if (shift == 56) {
        const unsigned long long Z = __shfl_sync(0xffffffffu, im, 31);
        if (top_p > 0.0f) target = static_cast<double>(top_p) * static_cast<double>(Z);
      }
      uint64_t c_run = cnt_above + (ic - lc), m_run = mass_above + (im - lm);
      int hit = -1;
      uint64_t c_before = 0, m_before = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t cu = cnt[lane * 8 + u];
        const unsigned long long mu = mass[lane * 8 + u];
        if (hit < 0 && cu > 0 && c_run + cu >= static_cast<uint64_t>(nk) &&
            static_cast<double>(m_run + mu) >= target) {
          hit = lane * 8 + u;
          c_before = c_run;
          m_before = m_run;
        }
        c_run += cu;
        m_run += mu;
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, hit >= 0);
      const int src = __ffs(bal) - 1;  // the invariant guarantees a hit
      const int dstar = __shfl_sync(0xffffffffu, hit, src);
      cnt_above = __shfl_sync(0xffffffffu, c_before, src);
      mass_above = __shfl_sync(0xffffffffu, m_before, src);
      prefix |= static_cast<uint64_t>(dstar) << shift;
      const uint32_t bucket = cnt[dstar];
      __syncwarp();
      if (bucket == 1u || shift == 0) {
        // Remaining candidates: keys with this prefix.  Walk them in ascending id and stop
        // at the first position where both conditions hold.
        uint64_t c_acc = cnt_above, m_acc = mass_above;
        const uint64_t mask = (shift == 0) ? ~0ull : ~((1ull << shift) - 1ull);
        bool done = false;
        for (int j1 = 0; j1 < T && !done; j1 += 128) {
          double xs[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = j1 + 32 * u + lane;
            xs[u] = j < T ? s[j] : 0.0;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j0 = j1 + 32 * u;
            if (done || j0 >= T) break;
            const int j = j0 + lane;
            uint64_t kj = 0, mj = 0;
            bool cand = false;
            if (j < T) {
              const double x = xs[u];
              kj = desc_key(x);
              cand = (kj & mask) == prefix;
              if (cand) mj = mass_fx(x, m);
            }
            // candidates share one key when shift == 0; a single candidate otherwise
            const uint32_t cb = __ballot_sync(0xffffffffu, cand);
            unsigned long long pm = cand ? mj : 0ull;
            uint32_t pc = cand ? 1u : 0u;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const unsigned long long t1 = __shfl_up_sync(0xffffffffu, pm, o);
              const uint32_t t2 = __shfl_up_sync(0xffffffffu, pc, o);
              if (lane >= o) {
                pm += t1;
                pc += t2;
              }
            }
            const bool ok = cand && (c_acc + pc >= static_cast<uint64_t>(nk)) &&
                            (static_cast<double>(m_acc + pm) >= target);
            const uint32_t okb = __ballot_sync(0xffffffffu, ok);
            if (okb) {
              const int L = __ffs(okb) - 1;
              jb = j0 + L;
              kb = __shfl_sync(0xffffffffu, kj, L);
              done = true;
            } else if (cb) {
              c_acc += __shfl_sync(0xffffffffu, pc, 31);
              m_acc += __shfl_sync(0xffffffffu, pm, 31);
            }
          }
        }
        break;
      }
    }
  }
  // emit the kept ids in ascending order
  int n = 0;
  int32_t* out = kv_index + static_cast<size_t>(row) * cap;
  for (int j0 = 0; j0 < T; j0 += 128) {
    double xs[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + 32 * u + lane;
      xs[u] = j < T ? s[j] : 0.0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + 32 * u + lane;
      bool sel = false;
      if (j < T) {
        const uint64_t kj = desc_key(xs[u]);
        sel = kj < kb || (kj == kb && j <= jb);
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, sel);
      const int pos = n + __popc(bal & ((1u << lane) - 1u));
      if (sel && pos < cap) out[pos] = j;
      n += __popc(bal);
    }
  }
  if (lane == 0) {
    if (n > cap) flag_error(st, DEVERR_CAPACITY, 0);
    kv_count[row] = min(n, cap);
  }
}

// ------------------------------------------------------------------------ launch
cudaError_t launch_plan(const void* q, const void* k, const float* q_scale, const float* k_scale, const Geom& g,
                        int BH, int D, bool fp8, double scale, int top_k, float top_p, int cap, int32_t* kv_index,
                        int32_t* kv_count, double* qbar, double* kbar, double* S, DevStatus* st,
                        cudaStream_t stream, int* launches) {
  dim3 pg((g.T + 3) / 4, BH, 2);
  if (fp8)
    pool_kernel<1><<<pg, 256, 0, stream>>>(static_cast<const uint8_t*>(q), static_cast<const uint8_t*>(k), q_scale,
                                           k_scale, qbar, kbar, g, D);
  else
    pool_kernel<2><<<pg, 256, 0, stream>>>(static_cast<const uint8_t*>(q), static_cast<const uint8_t*>(k), q_scale,
                                           k_scale, qbar, kbar, g, D);
  dim3 sg((g.T + SC_TILE - 1) / SC_TILE, (g.T + SC_TILE - 1) / SC_TILE, BH);
  score_kernel<<<sg, 256, 0, stream>>>(qbar, kbar, S, g.T, D, scale);
  const int rows = BH * g.T;
  select_kernel<<<(rows + 7) / 8, 256, 0, stream>>>(S, kv_index, kv_count, rows, g.T, top_k, top_p, cap, st);
  *launches = 3;
  return cudaGetLastError();
}

// The pooling and selection passes on their own, for routers that score a different matrix
// (bf16 Q and K; the same kernels and launch shapes as launch_plan).
cudaError_t launch_pool(const void* q, const void* k, const Geom& g, int BH, int D, double* qbar, double* kbar,
                        cudaStream_t stream) {
  dim3 pg((g.T + 3) / 4, BH, 2);
  pool_kernel<2><<<pg, 256, 0, stream>>>(static_cast<const uint8_t*>(q), static_cast<const uint8_t*>(k), nullptr,
                                         nullptr, qbar, kbar, g, D);
  return cudaGetLastError();
}

cudaError_t launch_select(const double* S, int32_t* kv_index, int32_t* kv_count, int rows, int T, int top_k,
                          float top_p, int cap, DevStatus* st, cudaStream_t stream) {
  select_kernel<<<(rows + 7) / 8, 256, 0, stream>>>(S, kv_index, kv_count, rows, T, top_k, top_p, cap, st);
  return cudaGetLastError();
}

}  // namespace sa
