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
#include "router_common.cuh"

namespace sa {

// ------------------------------------------------------------------------ pooling

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
// `s` is the row's T scores, `cnt` / `mass` a 256-entry scratch histogram of this warp; the
// kept ids go to `out` (at most cap) and their number to *count.  `mrow`, when given, holds
// every score's mass mass_fx(s_j, max) already (else each pass computes the masses it needs).
// Called by a whole warp.
__device__ void select_row_fp64(const double* __restrict__ s, int T, int top_k, float top_p, int cap,
                                int32_t* __restrict__ out, int32_t* __restrict__ count, DevStatus* st,
                                uint32_t* cnt, unsigned long long* mass,
                                const unsigned long long* __restrict__ mrow = nullptr) {
  const int lane = threadIdx.x & 31;

  double m = -DBL_MAX, mn = DBL_MAX;
#pragma unroll 4
  for (int j = lane; j < T; j += 32) {
    m = fmax(m, s[j]);
    mn = fmin(mn, s[j]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }

  const int nk = max(1, min(top_k, T));
  const bool keep_all = (top_p >= 1.0f) || nk >= T;
  uint64_t kb = ~0ull;  // boundary key
  int jb = T;           // boundary id (elements with key == kb and id <= jb are kept)
  if (!keep_all) {
    // every key of the row lies between those of its maximum and minimum, so the bytes above the
    // highest bit in which those two differ are common to all: the descent starts below them
    const uint64_t kmx = desc_key(m), kdiff = kmx ^ desc_key(mn);
    const int shift0 = kdiff ? ((63 - __clzll(static_cast<long long>(kdiff))) & ~7) : 0;
    uint64_t prefix = shift0 >= 56 ? 0ull : (kmx & ~((1ull << (shift0 + 8)) - 1ull));
    uint64_t cnt_above = 0, mass_above = 0;
    double target = -1.0;  // p <= 0: the mass test always passes
    for (int shift = shift0; shift >= 0; shift -= 8) {
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
            if (shift == 56 || (kj >> (shift + 8)) == (prefix >> (shift + 8))) {  // all keys at shift0
              part = true;
              d = static_cast<int>((kj >> shift) & 255u);
              mj = mrow ? mrow[j] : static_cast<unsigned long long>(mass_fx(x, m));
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
      if (shift == shift0) {  // the first pass counts every key: the row's total mass
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
              if (cand) mj = mrow ? mrow[j] : mass_fx(x, m);
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
    *count = min(n, cap);
  }
}

__global__ void __launch_bounds__(256) select_kernel(const double* __restrict__ S, int32_t* __restrict__ kv_index,
                                                     int32_t* __restrict__ kv_count, int rows, int T, int top_k,
                                                     float top_p, int cap, DevStatus* st) {
  __shared__ uint32_t cnt_s[8][256];
  __shared__ unsigned long long mass_s[8][256];
  const int warp = threadIdx.x >> 5;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  select_row_fp64(S + static_cast<size_t>(row) * T, T, top_k, top_p, cap, kv_index + static_cast<size_t>(row) * cap,
                  kv_count + row, st, cnt_s[warp], mass_s[warp]);
}

// ======================================================================== fast router
// The same decisions as the fp64 path above, at tensor-core speed.
//
//  * pooling .... as above, and each pooled row x (D values, fp64) is also written as an
//                 exact fixed-point integer X = rint(x * 2^(30-E)) (E: the row's binary
//                 exponent, |x_d| < 2^E) split into four signed 8-bit limbs,
//                 X = d0 256^3 + d1 256^2 + d2 256 + d3 (d0 in [-64, 64], others [-128, 127]).
//  * scores ..... Qbar Kbar^T from limb products on the tensor cores (tcgen05 kind::i8,
//                 exact s32 accumulation): the products of limb pairs (a, b) with a + b = w
//                 accumulate into level w (w = 0..3, ten products), and
//                 v = L0 2^24 + L1 2^16 + L2 2^8 + L3 is the dot product in units of
//                 2^(Eq + Ek - 36).  Dropping the levels w >= 4 and rounding the rows to 30
//                 bits bound the error of a raw score by 4.03 * 2^-23 * 2^(Eq + Ek).
//                 Each score is written as a 32-bit fixed-point key, key = rint(raw / 2^f_i),
//                 with f_i chosen from a bound on the row (|raw| <= |Qbar_i|_1 2^Ekmax) so that
//                 |key| <= 2^30.
//  * selection .. one warp per row: radix descent on u = max_key - key (ascending u is
//                 descending score), every bucket carrying its count and its fixed-point mass
//                 exp(s - max) * 2^50 (exponential from ex2.approx on the fractional part,
//                 relative error below 2^-21); the last bucket's few candidates are sorted
//                 exactly (u, then id).  A row is accepted only if its decision cannot change
//                 within the error bounds: the boundary key is more than twice the score bound
//                 from the next key, and the Top-p crossing is farther from p * Z than the
//                 masses' relative error.  Other rows (exact ties among them) are queued and
//                 decided again by the fp64 path, so every row ends with the fp64 decision.

struct RowMeta {
  double cunit;    // log2 units of exp(s - max) per key unit: 2^f * scale * log2(e)
  double eps_key;  // bound on a key's error, in key units
  double eps_s;    // bound on a score's error, natural units (scaled)
  double pad;
};


// Pooling for the tensor-core router.  Persistent CTAs, one per SM; items are (head, cube, Q or
// K), dealt round-robin so the CTAs stream neighbouring cubes together.  The last warp (one
// lane) brings each item's rows (up to the cube's last valid slot: one contiguous range) into a
// 12-stage shared-memory ring with 1-D bulk copies; the kConsumers warps before it take the items
// in turn, each lane summing D/32 columns over the cube's valid rows in fp64, and write the mean,
// its limbs, the row's binary exponent and (Q) its 1-norm.  Measured at 720p (sa_plan alone):
// ten consumers 1.24 ms, eight 1.26, twelve (one stage each, no lookahead) 1.26; half-cube
// stages with twelve consumers were slower still (0.63 against 0.50 ms for the pooling).
namespace rpl {
constexpr int kConsumers = 10;
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kStages = 12;
// A consumer's next stage is kConsumers stages past its last one.  A parity wait tells apart
// only the current phase of a barrier and the one before it, so the previous fill of that
// stage must already have landed: kStages >= kConsumers guarantees it (the consumer has seen
// the producer pass its last stage).
static_assert(kStages >= kConsumers, "a full-barrier wait could pass on a fill two phases old");
constexpr uint32_t kStageBytes = 16384;  // one cube of 64 rows x 256 bytes (bf16, D = 128)
constexpr uint32_t OFF_BAR = kStages * kStageBytes;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 2 * kStages * 8 + 1024;
}  // namespace rpl

struct PoolArgs {
  const uint8_t* q;
  const uint8_t* k;
  const float* q_scale;
  const float* k_scale;
  double* qbar;
  double* kbar;
  int8_t* qlimb;
  int8_t* klimb;
  int* qexp;
  int* kexp;
  double* ql1;
  unsigned* kexp_max;
  int* rkmax;
  int* rkmin;
  DevStatus* st;
  Geom g;
  int BH, D, Tk;
  unsigned long long timeout_ns;
};

// ESZ = bytes per element (2: bf16, 1: e4m3); EPL = D / 32 elements per lane.
template <int ESZ, int EPL>
__global__ void __launch_bounds__(rpl::kThreads, 1) pool_limbs_kernel(const PoolArgs a) {
  using namespace rpl;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + kStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const int D = a.D;
  const size_t row_bytes = static_cast<size_t>(D) * ESZ;
  const long long n_items = 2LL * a.BH * g.T;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (aborted(a.st)) return;
  if (warp == kConsumers) {
    if (lane == 0) {
      long long i = 0;  // item j of this CTA fills stage j % kStages
      bool ok = true;
      for (long long it = blockIdx.x; ok && it < n_items; it += gridDim.x, ++i) {
        const int which = static_cast<int>(it & 1);
        const long long cube = it >> 1;  // bh * T + c
        const int c = static_cast<int>(cube % g.T);
        int vt, vh, vw;
        cube_extent(g, c, vt, vh, vw);
        const uint32_t nrows = static_cast<uint32_t>(16 * (vt - 1) + 4 * (vh - 1) + vw);  // through the last valid slot
        const uint8_t* src = (which ? a.k : a.q) + (static_cast<size_t>(cube / g.T) * g.Npad + static_cast<size_t>(c) * 64) *
                                                       row_bytes;
        const int stage = static_cast<int>(i % kStages);
        if (i >= kStages && !mbar_wait(&empty[stage], ((i / kStages) + 1) & 1, a.st, a.timeout_ns, 131)) {
          ok = false;
          break;
        }
        const uint32_t bytes = nrows * static_cast<uint32_t>(row_bytes);
        mbar_arrive_expect_tx(&full[stage], bytes);
        bulk_load(smem + stage * kStageBytes, src, bytes, &full[stage]);
      }
      // drain: the copies still in flight land before the CTA exits
      const long long issued = i;
      for (long long d = (issued > kStages ? issued - kStages : 0); d < issued; ++d)
        mbar_wait_drain(&full[d % kStages], (d / kStages) & 1, a.st, a.timeout_ns, 132);
    }
    return;
  }
  long long j = warp;  // this CTA's item counter
  for (long long it = blockIdx.x + static_cast<long long>(warp) * gridDim.x; it < n_items;
       it += static_cast<long long>(kConsumers) * gridDim.x, j += kConsumers) {
    const int which = static_cast<int>(it & 1);
    const long long cube = it >> 1;
    const int bh = static_cast<int>(cube / g.T), c = static_cast<int>(cube % g.T);
    int vt, vh, vw;
    cube_extent(g, c, vt, vh, vw);
    // four accumulator sets (slot d0 of each row of 4) keep independent fp64 chains in flight
    double acc4[4][EPL];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc4[u][e] = 0.0;
    {
      const int stage = static_cast<int>(j % kStages);
      if (!mbar_wait_warp(&full[stage], (j / kStages) & 1, a.st, a.timeout_ns, 133)) break;
      const uint8_t* tile = smem + stage * kStageBytes + lane * EPL * ESZ;
      // this lane's EPL elements of one row: loaded from shared memory as NW words, then
      // widened to fp64 and added
      constexpr int NW = ESZ == 2 ? EPL / 2 : 1;
      auto load_row = [&](const uint8_t* rp, uint32_t (&wv)[NW]) {
        if constexpr (ESZ == 2 && EPL == 4) {
          const uint2 t2 = *reinterpret_cast<const uint2*>(rp);
          wv[0] = t2.x;
          wv[1] = t2.y;
        } else if constexpr (ESZ == 1 && EPL == 2) {
          wv[0] = *reinterpret_cast<const uint16_t*>(rp);
        } else {
          wv[0] = *reinterpret_cast<const uint32_t*>(rp);
        }
      };
      auto add_words = [&](double* acc, const uint32_t (&wv)[NW]) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          if constexpr (ESZ == 2)
            acc[e] += static_cast<double>(
                __uint_as_float((e & 1) ? (wv[e >> 1] & 0xffff0000u) : (wv[e >> 1] << 16)));
          else
            acc[e] += static_cast<double>(e4m3_value((wv[0] >> (8 * e)) & 0xffu));
        }
      };
      if (vt == 4 && vh == 4 && vw == 4) {
        // a whole cube: 64 consecutive rows, sixteen at a time with every load of the group
        // issued before its arithmetic (one shared-memory round trip per sixteen rows)
#pragma unroll 1
        for (int r0 = 0; r0 < 64; r0 += 16) {
          uint32_t w16[16][NW];
#pragma unroll
          for (int u = 0; u < 16; ++u) load_row(tile + (r0 + u) * row_bytes, w16[u]);
#pragma unroll
          for (int u = 0; u < 16; ++u) add_words(acc4[u & 3], w16[u]);
        }
      } else {
        for (int a0 = 0; a0 < vt; ++a0)
          for (int b0 = 0; b0 < vh; ++b0)
#pragma unroll
            for (int d0 = 0; d0 < 4; ++d0) {
              if (d0 >= vw) break;
              uint32_t wv[NW];
              load_row(tile + (a0 * 16 + b0 * 4 + d0) * row_bytes, wv);
              add_words(acc4[d0], wv);
            }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);  // the cube's rows have been read
    }
    double acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = (acc4[0][e] + acc4[1][e]) + (acc4[2][e] + acc4[3][e]);
    const int n = vt * vh * vw;
    double scale = 1.0;
    if constexpr (ESZ == 1) scale = static_cast<double>((which ? a.k_scale : a.q_scale)[cube]);
    double x[EPL];
    double amax = 0.0, l1 = 0.0;
    double* dst = (which ? a.kbar : a.qbar) + static_cast<size_t>(cube) * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      x[e] = acc[e] * scale / static_cast<double>(n);
      dst[e] = x[e];
      amax = fmax(amax, fabs(x[e]));
      l1 += fabs(x[e]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    int E = kExpZero;
    if (amax > 0.0) frexp(amax, &E);  // amax = m 2^E, m in [0.5, 1): every |x_d| < 2^E
    const double up = amax > 0.0 ? ldexp(1.0, 30 - E) : 0.0;
    uint32_t limb[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int e = 0; e < EPL; ++e) limb_digits(x[e], up, e, limb);
    int8_t* lb = which ? a.klimb : a.qlimb;
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      int8_t* rowp = lb + ((static_cast<size_t>(bh) * 4 + l) * g.T + c) * kLimbRow;
      if constexpr (EPL == 4) {
        reinterpret_cast<uint32_t*>(rowp)[lane] = limb[l];
      } else {  // D = 64: 64 bytes of limbs, then 64 zero bytes
        reinterpret_cast<uint16_t*>(rowp)[lane] = static_cast<uint16_t>(limb[l]);
        reinterpret_cast<uint16_t*>(rowp + 64)[lane] = 0;
      }
    }
    if (lane == 0) {
      if (which) {
        a.kexp[static_cast<size_t>(bh) * a.Tk + c] = E;  // rows of Tk entries: 16-byte aligned per head
        atomicMax(a.kexp_max + bh, static_cast<unsigned>(E + kExpBias));
      } else {
        a.qexp[cube] = E;
        a.ql1[cube] = l1;
        a.rkmax[cube] = INT_MIN;  // the score kernel's per-row key extrema start here
        a.rkmin[cube] = INT_MAX;
      }
    }
  }
}

// ------------------------------------------------------------------------ exact scores
namespace rsc {
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 TMEM owner + MMA, warps 2-9 epilogue
constexpr uint32_t OFF_Q = 0;                      // 4 limbs x [128 rows][128 B]
constexpr uint32_t OFF_K = 65536;                  // 2 stages x 4 limbs x [128 keys][128 B]
constexpr uint32_t OFF_STG = OFF_K + 2 * 65536;   // 8 epilogue warps x [32 rows][128 B] key staging
constexpr uint32_t OFF_BAR = OFF_STG + 8 * 4096;
constexpr uint32_t OFF_SLOT = OFF_BAR + 128;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;                // level w at columns 128w
enum { B_QF = 0, B_QE = 1, B_KF = 2, B_KE = 4, B_TF = 6, B_TE = 7, B_FIN = 8, NBAR = 9 };
}  // namespace rsc

struct ScoreArgs {
  const int* qexp;
  const int* kexp;
  const double* ql1;
  const unsigned* kexp_max;
  int* keys;        // [BH*T, Tk]
  int* rkmax;       // [BH*T] largest and smallest key of each row (atomics)
  int* rkmin;
  RowMeta* meta;    // [BH*T]
  float* s32;       // optional [BH*T, T]: the scaled scores in fp32
  DevStatus* st;
  int T, Tk, BH;    // kexp rows have Tk entries per head
  double scale;
  unsigned long long timeout_ns;
};

// KS = D / 32 k-steps of 32 int8 per product.  S32: also write every scaled score in fp32 (a.s32).
// Work item = one 128 x 128 tile of (query cubes, key cubes) of one head; each CTA takes a
// contiguous run of items, so consecutive items share their query rows (loaded once per row block).
template <int KS, bool S32>
__global__ void __launch_bounds__(rsc::kThreads, 1)
    score_keys_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_keys, const ScoreArgs a) {
  using namespace rsc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T;
  const int nrb = (T + 127) >> 7;
  const long long n_items = static_cast<long long>(a.BH) * nrb * nrb;
  const long long t0 = n_items * blockIdx.x / gridDim.x, t1 = n_items * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b) mbar_init(&bars[b], b == B_TE ? 256u : 1u);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip_all = aborted(a.st);

  if (warp == 0) {
    if (lane == 0 && !skip_all) {
      uint32_t ks = 0;
      int qn = 0;
      long long prev = -1;
      bool ok = true;
      for (long long t = t0; ok && t < t1; ++t) {
        const int bh = static_cast<int>(t / (static_cast<long long>(nrb) * nrb));
        const int rem = static_cast<int>(t % (static_cast<long long>(nrb) * nrb));
        const int rb = rem / nrb, cb = rem % nrb;
        const long long rbk = static_cast<long long>(bh) * nrb + rb;
        if (rbk != prev) {
          if (qn >= 1 && !mbar_wait(&bars[B_QE], (qn - 1) & 1, a.st, a.timeout_ns, 101)) break;
          mbar_arrive_expect_tx(&bars[B_QF], 65536);
#pragma unroll
          for (int l = 0; l < 4; ++l) tma_load_3d(smem + OFF_Q + l * 16384, &tm_q, &bars[B_QF], 0, rb * 128, bh * 4 + l);
          ++qn;
          prev = rbk;
        }
        const uint32_t st = ks & 1u;
        if (ks >= 2 && !mbar_wait(&bars[B_KE + st], ((ks >> 1) + 1) & 1, a.st, a.timeout_ns, 102)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars[B_KF + st], 65536);
#pragma unroll
        for (int l = 0; l < 4; ++l)
          tma_load_3d(smem + OFF_K + st * 65536 + l * 16384, &tm_k, &bars[B_KF + st], 0, cb * 128, bh * 4 + l);
        ++ks;
      }
      // drain: never leave the CTA with copies in flight
      if (qn > 0) mbar_wait_drain(&bars[B_QF], (qn - 1) & 1, a.st, a.timeout_ns, 103);
      for (uint32_t s = (ks > 2 ? ks - 2 : 0); s < ks; ++s)
        mbar_wait_drain(&bars[B_KF + (s & 1u)], (s >> 1) & 1, a.st, a.timeout_ns, 104);
    }
  } else if (warp == 1) {
    if (!skip_all) {
      uint32_t ks = 0, tile = 0;
      int qn = 0;
      long long prev = -1;
      bool ok = true;
      for (long long t = t0; ok && t < t1; ++t) {
        const int bh = static_cast<int>(t / (static_cast<long long>(nrb) * nrb));
        const int rem = static_cast<int>(t % (static_cast<long long>(nrb) * nrb));
        const int rb = rem / nrb;
        const long long rbk = static_cast<long long>(bh) * nrb + rb;
        if (rbk != prev) {
          if (!mbar_wait_warp(&bars[B_QF], qn & 1, a.st, a.timeout_ns, 111)) break;
          ++qn;
          prev = rbk;
        }
        const long long tn = t + 1;
        const bool last_of_rb =
            tn >= t1 || (tn / (static_cast<long long>(nrb) * nrb)) * nrb +
                                (tn % (static_cast<long long>(nrb) * nrb)) / nrb != rbk;
        if (tile >= 1 && !mbar_wait_warp(&bars[B_TE], (tile - 1) & 1, a.st, a.timeout_ns, 112)) break;
        const uint32_t st = ks & 1u;
        if (!mbar_wait_warp(&bars[B_KF + st], (ks >> 1) & 1, a.st, a.timeout_ns, 113)) break;
        tc_fence_after();
        const uint32_t kb = sbase + OFF_K + st * 65536;
        if (elect_one()) {
          issue_limb_products<KS>(tmem, sbase + OFF_Q, kb);
          umma_commit(&bars[B_KE + st]);
          umma_commit(&bars[B_TF]);
          if (last_of_rb) umma_commit(&bars[B_QE]);
        }
        __syncwarp();
        ++ks;
        ++tile;
      }
      if (elect_one()) umma_commit(&bars[B_FIN]);
      __syncwarp();
      mbar_wait_drain(&bars[B_FIN], 0, a.st, a.timeout_ns, 114);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t tile = 0;
    bool ok = !skip_all;
    long long prev_rbk = -1;
    int A = 0, f = 0, Eq = 0, Ekm = 0;
    bool nonzero = false;
    for (long long t = t0; ok && t < t1; ++t, ++tile) {
      const int bh = static_cast<int>(t / (static_cast<long long>(nrb) * nrb));
      const int rem = static_cast<int>(t % (static_cast<long long>(nrb) * nrb));
      const int rb = rem / nrb, cb = rem % nrb;
      const int i = rb * 128 + r;
      const bool row_ok = i < T;
      const size_t rowid = static_cast<size_t>(bh) * T + (row_ok ? i : 0);
      const long long rbk = static_cast<long long>(bh) * nrb + rb;
      if (rbk != prev_rbk) {
        // per-row scaling of the keys: |raw| <= |Qbar_i|_1 2^Ekmax < 2^e, keys in units of 2^(e - 30)
        prev_rbk = rbk;
        f = 0;
        Eq = __ldg(a.qexp + rowid);
        Ekm = static_cast<int>(__ldg(a.kexp_max + bh)) - kExpBias;
        const double B = ldexp(__ldg(a.ql1 + rowid), Ekm);
        nonzero = Eq != kExpZero && Ekm != kExpZero && B > 0.0;
        if (nonzero) {
          int e;
          frexp(B, &e);
          f = e - 30;
        }
        A = 36 + f - Eq;
      }
      if (row_ok && cb == 0 && half == 0) {
        RowMeta m;
        m.cunit = ldexp(a.scale * 1.4426950408889634, f);
        const double eps_raw = nonzero ? 4.03 * ldexp(1.0, Eq + Ekm - 23) : 0.0;
        m.eps_key = eps_raw * ldexp(1.0, -f) + 1.0;
        m.eps_s = (eps_raw + ldexp(1.0, f)) * a.scale;
        m.pad = 0.0;
        a.meta[rowid] = m;
      }
      if (!mbar_wait_warp(&bars[B_TF], tile & 1, a.st, a.timeout_ns, 121)) {  // warp-uniform (warp ops below)
        ok = false;
        break;
      }
      tc_fence_after();
      const int* ekp = a.kexp + static_cast<size_t>(bh) * a.Tk;  // padded rows: 16-byte aligned
      int lmax = INT_MIN, lmin = INT_MAX;
      uint8_t* stg = smem + OFF_STG + (warp - 2) * 4096;
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        const int col0 = 64 * half + 32 * ch;
        // the 32 key exponents of this chunk (entries past T are never stored: any value will do)
        int ekc[32];
        {
          const int jc = cb * 128 + col0;
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4) {
            const int4 e4 = jc + 4 * v4 < a.Tk ? __ldg(reinterpret_cast<const int4*>(ekp + jc) + v4) : make_int4(0, 0, 0, 0);
            ekc[4 * v4] = e4.x;
            ekc[4 * v4 + 1] = e4.y;
            ekc[4 * v4 + 2] = e4.z;
            ekc[4 * v4 + 3] = e4.w;
          }
        }
        uint32_t L0[32], L1[32], L2[32], L3[32];
        tmem_ld32(t_lane + 0 + col0, L0);
        tmem_ld32(t_lane + 128 + col0, L1);
        tmem_ld32(t_lane + 256 + col0, L2);
        tmem_ld32(t_lane + 384 + col0, L3);
        tmem_ld_wait();
        if (ch == 1) {
          tc_fence_before();
          mbar_arrive(&bars[B_TE]);  // this thread's reads of the tile are complete
        }
        const int j0 = cb * 128 + col0;
        // this warp's previous store has read its staging rows
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const int j = j0 + 4 * c4;
          int kv[4];
          float sv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = 4 * c4 + u;
            const long long v = limb_levels(L0[c], L1[c], L2[c], L3[c]);
            if constexpr (S32) {  // v in units of 2^(Eq + Ek - 36), times the softmax scale
              const int e2 = Eq + ekc[c] - 36;  // a zero row (exponent kExpZero) has v = 0
              sv[u] = (v != 0 && e2 > -1000 && e2 < 1000)
                          ? static_cast<float>(static_cast<double>(v) * a.scale * __hiloint2double((1023 + e2) << 20, 0))
                          : 0.0f;
            }
            int sh = A - ekc[c];
            sh = sh < 1 ? 1 : (sh > 62 ? 62 : sh);
            kv[u] = static_cast<int>((v + (1LL << (sh - 1))) >> sh);
            if (row_ok && j + u < T) {
              lmax = max(lmax, kv[u]);
              lmin = min(lmin, kv[u]);
            }
          }
          if (S32 && row_ok) {  // four consecutive scores of this row: one 16-byte store when aligned
            float* dst = a.s32 + rowid * T + j;
            if ((T & 3) == 0 && j + 3 < T) {
              *reinterpret_cast<float4*>(dst) = make_float4(sv[0], sv[1], sv[2], sv[3]);
            } else {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (j + u < T) dst[u] = sv[u];
            }
          }
          // row `lane` of the warp's 32 x 32 staging tile, 16-byte chunk c4, 128-byte swizzle
          st_shared_v4(smem_u32(stg) + sw128_offset(lane, c4), kv[0], kv[1], kv[2], kv[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        // rows and columns past T fall outside the map and are not written
        if (lane == 0) {
          tma_store_3d(&tm_keys, stg, j0, rb * 128 + quarter * 32, bh);
          bulk_commit_group();
        }
      }
      if (row_ok && lmax >= lmin) {
        atomicMax(a.rkmax + rowid, lmax);
        atomicMin(a.rkmin + rowid, lmin);
      }
    }
    if (lane == 0) bulk_wait0();  // the key stores are complete before the CTA leaves
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, rsc::TMEM_COLS);
}

// ------------------------------------------------------------------------ key selection
// 2^36 * 2^(-u c): the fixed-point mass of a score u key units below the row maximum.  A row's
// masses sum to at most T 2^36 < 2^50 (T <= 8192), so a histogram bucket packs its count in
// bits 50-63 and its mass in bits 0-49 of one 64-bit word, and sums of such words (buckets,
// prefixes) stay packed.
constexpr int kMassBits = 36;
constexpr unsigned long long kMassMask = (1ull << 50) - 1ull;
constexpr unsigned long long kCountOne = 1ull << 50;
__device__ __forceinline__ unsigned long long mass_key(uint32_t u, double c) {
  // Two conversion-pipe operations per entry (f64 -> f32 and ex2); the rest is fp64 and integer
  // arithmetic.  u as fp64 exactly: 2^52 + u has u in its low word.
  const double ud = __hiloint2double(0x43300000, static_cast<int>(u)) - 4503599627370496.0;
  const double x = -ud * c;  // log2 of the mass relative to the row maximum, <= 0
  if (x < -60.0) return 0ull;
  // x = n + f with n = round(x) (round-to-nearest through 1.5 * 2^52) and f in [-1/2, 1/2]
  const double t = x + 6755399441055744.0;
  const int n = __double2loint(t);
  const double f = x - (t - 6755399441055744.0);
  const float p2 = ex2_approx(__double2float_rn(f));  // in [2^-1/2, 2^1/2]
  // 2^(36 + n) * p2 as an integer: p2 = m * 2^(e - 23) with m the 24-bit significand
  const uint32_t pb = __float_as_uint(p2);
  const unsigned long long m = static_cast<unsigned long long>((pb & 0x7fffffu) | 0x800000u);
  const int sh = kMassBits + n + static_cast<int>((pb >> 23) & 0xffu) - 127 - 23;
  return sh >= 0 ? (m << sh) : (sh > -64 ? (m >> -sh) : 0ull);
}

constexpr unsigned kDebugRouterFallback = 2u;  // debug flag: every row takes the fp64 path

// Visit a row of keys 128 at a time (int4 of 4 consecutive keys per lane), in order.  Every
// lane calls f for every chunk (the chunk loop is uniform), so f may use warp collectives;
// keys past T arrive as 0 and f must check j + u < T.  The loads of four chunks are issued
// together, so a pass over a row waits for L2 a quarter as often.
template <class F>
__device__ __forceinline__ void for_key_chunks(const int* kr, int T, int lane, F&& f) {
  for (int j0 = 0; j0 < T; j0 += 512) {
    int4 x[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + 128 * c + 4 * lane;
      x[c] = j < T ? *reinterpret_cast<const int4*>(kr + j) : make_int4(0, 0, 0, 0);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (j0 + 128 * c < T) f(j0 + 128 * c + 4 * lane, x[c]);
  }
}

// One warp per row; every pass reads the row from global memory (after the first, from L2).
__global__ void __launch_bounds__(256, 4) select_keys_kernel(const int* __restrict__ keys, int Tk,
                                                                         const int* __restrict__ rkmax,
                                                                         const int* __restrict__ rkmin,
                                                                         const RowMeta* __restrict__ meta, int rows,
                                                                         int T, int top_k, float top_p, int cap,
                                                                         int32_t* __restrict__ kv_index,
                                                                         int32_t* __restrict__ kv_count,
                                                                         int* __restrict__ flist, DevStatus* st,
                                                                         unsigned debug,
                                                                         unsigned long long timeout_ns) {
  __shared__ unsigned long long hist_s[8][256];  // packed (count << 50) + mass per bucket
  __shared__ unsigned long long cand_s[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const int* kr = keys + static_cast<size_t>(row) * Tk;
  unsigned long long* hist = hist_s[warp];
  int32_t* out = kv_index + static_cast<size_t>(row) * cap;
  const int nk = max(1, min(top_k, T));
  if (top_p >= 1.0f || nk >= T) {  // every block
    for (int j = lane; j < T && j < cap; j += 32) out[j] = j;
    if (lane == 0) {
      if (T > cap) flag_error(st, DEVERR_CAPACITY, 0);
      kv_count[row] = min(T, cap);
    }
    return;
  }
  const int kmax = rkmax[row], kmin = rkmin[row];
  const RowMeta m = meta[row];
  const double c = m.cunit;
  // ---- (1) radix descent on u = kmax - key over [lo, hi]
  uint32_t lo = 0, hi = static_cast<uint32_t>(kmax - kmin);
  unsigned long long c_above = 0, m_above = 0, Z = 0;
  double target = -1.0;
  uint32_t bcnt = 0;
  for (int level = 0;; ++level) {
    const uint32_t span = hi - lo;
    const int s = span < 256u ? 0 : (32 - __clz(span)) - 8;  // (hi - lo) >> s < 256
    for (int d = lane; d < 256; d += 32) hist[d] = 0ull;
    __syncwarp();
    for_key_chunks(kr, T, lane, [&](int j, const int4& v) {
      const int vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        const uint32_t uu = static_cast<uint32_t>(kmax - vv[u4]);
        if (j + u4 < T && uu >= lo && uu <= hi) atomicAdd(&hist[(uu - lo) >> s], kCountOne + mass_key(uu, c));
      }
    });
    __syncwarp();
    unsigned long long lw = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) lw += hist[lane * 8 + u];
    unsigned long long iw = lw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long ow = __shfl_up_sync(0xffffffffu, iw, o);
      if (lane >= o) iw += ow;
    }
    if (level == 0) {
      Z = __shfl_sync(0xffffffffu, iw, 31) & kMassMask;
      if (top_p > 0.0f) target = static_cast<double>(top_p) * static_cast<double>(Z);
    }
    const unsigned long long ex = iw - lw;  // packed sums of the buckets before this lane's
    unsigned long long c_run = c_above + (ex >> 50), m_run = m_above + (ex & kMassMask);
    int hit = -1;
    unsigned long long c_before = 0, m_before = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const unsigned long long wu = hist[lane * 8 + u];
      const uint32_t cu = static_cast<uint32_t>(wu >> 50);
      const unsigned long long mu = wu & kMassMask;
      if (hit < 0 && cu > 0 && c_run + cu >= static_cast<unsigned long long>(nk) &&
          static_cast<double>(m_run + mu) >= target) {
        hit = lane * 8 + u;
        c_before = c_run;
        m_before = m_run;
      }
      c_run += cu;
      m_run += mu;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, hit >= 0);
    if (bal == 0u) {  // cannot happen (the totals meet both conditions); decide the row in fp64
      bcnt = 0xffffffffu;
      break;
    }
    const int src = __ffs(bal) - 1;
    const int bstar = __shfl_sync(0xffffffffu, hit, src);
    c_above = __shfl_sync(0xffffffffu, c_before, src);
    m_above = __shfl_sync(0xffffffffu, m_before, src);
    bcnt = static_cast<uint32_t>(hist[bstar] >> 50);
    __syncwarp();
    const unsigned long long nlo = static_cast<unsigned long long>(lo) + (static_cast<unsigned long long>(bstar) << s);
    const unsigned long long nhi = nlo + (1ull << s) - 1ull;
    lo = static_cast<uint32_t>(nlo);
    hi = static_cast<uint32_t>(nhi < hi ? nhi : hi);
    if (bcnt <= 32u || s == 0) break;
  }
  // the provisional list (ids above the bucket and the candidates) must fit the row
  bool certain = bcnt <= 32u && c_above + bcnt <= static_cast<unsigned long long>(cap) &&
                 (debug & kDebugRouterFallback) == 0u;
  uint32_t ub = 0;
  int jb = -1, n = 0;
  unsigned long long cum_at = 0, cum_before = 0;
  uint32_t unext = 0xffffffffu;
  if (certain) {
    // ---- (2) write ids above the bucket and the marked candidates in ascending id order
    int written = 0, nc = 0;
    uint32_t umin_below = 0xffffffffu;
    for_key_chunks(kr, T, lane, [&](int j, const int4& v) {
      const int vv[4] = {v.x, v.y, v.z, v.w};
      int tag[4];
      int nsel = 0;
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        const uint32_t uu = static_cast<uint32_t>(kmax - vv[u4]);
        const bool in = j + u4 < T;
        tag[u4] = !in ? 0 : (uu < lo ? 1 : (uu <= hi ? 2 : 0));  // 1: kept, 2: candidate
        if (in && uu > hi) umin_below = min(umin_below, uu);
        nsel += tag[u4] ? 1 : 0;
        const bool isc = tag[u4] == 2;
        const uint32_t b = __ballot_sync(0xffffffffu, isc);
        if (isc) {
          const int pos = nc + __popc(b & ((1u << lane) - 1u));
          if (pos < 32) cand_s[warp][pos] = (static_cast<unsigned long long>(uu) << 32) | static_cast<uint32_t>(j + u4);
        }
        nc += __popc(b);
      }
      int incl = nsel;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int pos = written + incl - nsel;
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4)
        if (tag[u4]) {
          if (pos < cap) out[pos] = (j + u4) | (tag[u4] == 2 ? static_cast<int>(0x80000000u) : 0);
          ++pos;
        }
      written += __shfl_sync(0xffffffffu, incl, 31);
    });
#pragma unroll
    for (int o = 16; o; o >>= 1) umin_below = min(umin_below, __shfl_xor_sync(0xffffffffu, umin_below, o));
    __syncwarp();
    // ---- (3) the candidates sorted by (u, id): bitonic sort of 32 keys across the warp
    unsigned long long key = lane < static_cast<int>(bcnt) ? cand_s[warp][lane] : ~0ull;
#pragma unroll
    for (int k2 = 2; k2 <= 32; k2 <<= 1) {
#pragma unroll
      for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, j2);
        const bool up = (lane & k2) == 0;
        const bool lower = (lane & j2) == 0;
        key = (lower == up) ? (key < other ? key : other) : (key > other ? key : other);
      }
    }
    const bool valid = lane < static_cast<int>(bcnt);
    const uint32_t uu = static_cast<uint32_t>(key >> 32);
    const unsigned long long ms = valid ? mass_key(uu, c) : 0ull;
    unsigned long long pm = ms;
    uint32_t pc = valid ? 1u : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long t1 = __shfl_up_sync(0xffffffffu, pm, o);
      const uint32_t t2 = __shfl_up_sync(0xffffffffu, pc, o);
      if (lane >= o) {
        pm += t1;
        pc += t2;
      }
    }
    const bool okb = valid && (c_above + pc >= static_cast<unsigned long long>(nk)) &&
                     (static_cast<double>(m_above + pm) >= target);
    const uint32_t okm = __ballot_sync(0xffffffffu, okb);
    if (okm == 0u || written != static_cast<int>(c_above + bcnt)) {
      certain = false;
    } else {
      const int L = __ffs(okm) - 1;
      ub = __shfl_sync(0xffffffffu, uu, L);
      jb = static_cast<int>(__shfl_sync(0xffffffffu, static_cast<uint32_t>(key & 0xffffffffull), L));
      n = static_cast<int>(c_above) + L + 1;
      cum_at = m_above + __shfl_sync(0xffffffffu, pm, L);
      cum_before = cum_at - __shfl_sync(0xffffffffu, ms, L);
      // the next element in order: the next candidate, else the first key below the bucket
      const uint32_t un = __shfl_sync(0xffffffffu, uu, (L + 1) & 31);
      unext = (L + 1 < static_cast<int>(bcnt)) ? un : umin_below;
      // ---- (4) drop the candidates the boundary leaves out, in place (reads stay ahead of writes)
      int wpos = 0;
      for (int r0 = 0; r0 < written; r0 += 32) {
        const int r = r0 + lane;
        int e = r < written ? out[r] : 0;
        bool keep = r < written;
        if (keep && e < 0) {
          const int jj = e & 0x7fffffff;
          const uint32_t uj = static_cast<uint32_t>(kmax - kr[jj]);
          keep = uj < ub || (uj == ub && jj <= jb);
          e = jj;
        }
        const uint32_t kb = __ballot_sync(0xffffffffu, keep);
        __syncwarp();
        if (keep) out[wpos + __popc(kb & ((1u << lane) - 1u))] = e;
        wpos += __popc(kb);
      }
      if (wpos != n) certain = false;
    }
  }
  if (certain) {
    // ---- is the decision certain within the error bounds?
    const double Zd = static_cast<double>(Z);
    // masses: ex2.approx within 2^-21 relative, scores within eps_s, and one fixed-point unit
    // of truncation per element
    const double delta = (2.0 * m.eps_s + 2.0 * 4.76837158203125e-07 + 1e-12) * Zd + static_cast<double>(T);
    const bool gap_ok = unext == 0xffffffffu || static_cast<double>(unext - ub) > 2.0 * m.eps_key;
    bool cross_ok = true;
    if (top_p > 0.0f) {
      if (n > nk)
        cross_ok = fabs(static_cast<double>(cum_at) - target) > delta &&
                   fabs(static_cast<double>(cum_before) - target) > delta;
      else
        cross_ok = static_cast<double>(cum_at) - target > delta;
    }
    certain = gap_ok && cross_ok;
    if (certain && lane == 0) kv_count[row] = n;  // n <= cap (checked above)
  }
  if (!certain && lane == 0) {
    const unsigned k = atomicAdd(&st->router_fallback, 1u);
    flist[k] = row;
  }
}

// The same decision as select_row_fp64, taken by a whole CTA of NWARP warps: the radix levels
// split the row's keys over the warps (one shared histogram), warp 0 scans each level's 256
// buckets and publishes the hit through shared memory, and the two passes in id order (the
// boundary candidate, the emission) give each warp a contiguous range of ids, offset by the
// counts of the warps before it.  `s` and `mrow` (scores and their fixed-point masses against
// the row maximum m) are in shared memory; mn is the row minimum.  Called by every thread.
struct SelCtl {
  unsigned long long cnt_above, mass_above, bmass, kb;
  double target;
  int dstar, cstar, jb;
  uint32_t bucket;
  int wcount[32];
};

template <int NWARP>
__device__ void select_row_fp64_cta(const double* __restrict__ s, const unsigned long long* __restrict__ mrow,
                                    double m, double mn, int T, int top_k, float top_p, int cap,
                                    int32_t* __restrict__ out, int32_t* __restrict__ count, DevStatus* st,
                                    uint32_t* cnt, unsigned long long* mass, SelCtl* ctl) {
  constexpr int NT = NWARP * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk = max(1, min(top_k, T));
  const bool keep_all = (top_p >= 1.0f) || nk >= T;
  // contiguous id range of this warp for the passes in id order (whole chunks of 32)
  const int per = ((T + NT - 1) / NT) * 32;
  const int w_lo = min(T, warp * per), w_hi = min(T, w_lo + per);
  uint64_t kb = ~0ull;  // boundary key; ids with this key up to jb are kept
  int jb = T;
  if (!keep_all) {
    const uint64_t kmx = desc_key(m), kdiff = kmx ^ desc_key(mn);
    const int shift0 = kdiff ? ((63 - __clzll(static_cast<long long>(kdiff))) & ~7) : 0;
    uint64_t prefix = shift0 >= 56 ? 0ull : (kmx & ~((1ull << (shift0 + 8)) - 1ull));
    uint64_t cnt_above = 0, mass_above = 0;
    double target = -1.0;
    for (int shift = shift0; shift >= 0; shift -= 8) {
      for (int d = tid; d < 256; d += NT) {
        cnt[d] = 0;
        mass[d] = 0ull;
      }
      __syncthreads();
      // chunks of 32 keys dealt to the warps in turn; a warp whose keys share one bucket adds
      // its count and mass once
      for (int j0 = warp * 32; j0 < T; j0 += NT) {
        const int j = j0 + lane;
        bool part = false;
        int d = 0;
        unsigned long long mj = 0ull;
        if (j < T) {
          const uint64_t kj = desc_key(s[j]);
          if (shift == 56 || (kj >> (shift + 8)) == (prefix >> (shift + 8))) {
            part = true;
            d = static_cast<int>((kj >> shift) & 255u);
            mj = mrow[j];
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
      __syncthreads();
      if (warp == 0) {
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
        if (shift == shift0) {  // the first level counts every key: the row's total mass
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
        const int src = __ffs(bal) - 1;  // the totals meet both conditions: some bucket hits
        const int dstar = __shfl_sync(0xffffffffu, hit, src);
        const uint64_t ca = __shfl_sync(0xffffffffu, c_before, src);
        const uint64_t ma = __shfl_sync(0xffffffffu, m_before, src);
        if (lane == 0) {
          ctl->dstar = dstar;
          ctl->cnt_above = ca;
          ctl->mass_above = ma;
          ctl->target = target;
          ctl->bucket = cnt[dstar];
          ctl->bmass = mass[dstar];
        }
      }
      __syncthreads();
      const int dstar = ctl->dstar;
      cnt_above = ctl->cnt_above;
      mass_above = ctl->mass_above;
      target = ctl->target;
      const uint32_t bucket = ctl->bucket;
      prefix |= static_cast<uint64_t>(dstar) << shift;
      if (bucket == 1u || shift == 0) {
        // The candidates (keys with this prefix) share one key, hence one mass: the boundary is
        // the c-th of them in id order for the least c meeting both conditions (c = 1 for a
        // single candidate, where the hit guarantees both).
        const uint64_t mask = (shift == 0) ? ~0ull : ~((1ull << shift) - 1ull);
        if (warp == 0) {
          const unsigned long long mj = ctl->bmass / bucket;
          int cs = -1;
          for (uint32_t c0 = 1; c0 <= bucket && cs < 0; c0 += 32) {
            const uint32_t c = c0 + lane;
            const bool ok = c <= bucket && cnt_above + c >= static_cast<uint64_t>(nk) &&
                            static_cast<double>(mass_above + c * mj) >= target;
            const uint32_t okb = __ballot_sync(0xffffffffu, ok);
            if (okb) cs = static_cast<int>(c0) + __ffs(okb) - 1;
          }
          if (lane == 0) {
            ctl->cstar = cs < 0 ? static_cast<int>(bucket) : cs;
            ctl->jb = 0;  // overwritten below by the warp holding the boundary candidate
          }
        }
        // this warp's candidates in its id range
        int wc = 0;
        for (int j0 = w_lo; j0 < w_hi; j0 += 32) {
          const int j = j0 + lane;
          const bool cand = j < w_hi && (desc_key(s[j]) & mask) == prefix;
          wc += __popc(__ballot_sync(0xffffffffu, cand));
        }
        if (lane == 0) ctl->wcount[warp] = wc;
        __syncthreads();
        const int cs = ctl->cstar;
        int before = 0;
        for (int w = 0; w < warp; ++w) before += ctl->wcount[w];
        if (cs > before && cs <= before + wc) {  // the boundary candidate is in this warp's range
          int seen = before;
          for (int j0 = w_lo; j0 < w_hi; j0 += 32) {
            const int j = j0 + lane;
            const bool cand = j < w_hi && (desc_key(s[j]) & mask) == prefix;
            const uint32_t cb = __ballot_sync(0xffffffffu, cand);
            if (seen + __popc(cb) >= cs) {
              // the (cs - seen)-th set bit of cb
              uint32_t bits = cb;
              for (int r = cs - seen; r > 1; --r) bits &= bits - 1u;
              if (lane == 0) ctl->jb = j0 + __ffs(bits) - 1;
              break;
            }
            seen += __popc(cb);
          }
        }
        __syncthreads();
        jb = ctl->jb;
        kb = desc_key(s[jb]);  // the boundary's whole key (below `shift`, a lone candidate's own bits)
        break;
      }
    }
  }
  // emit the kept ids in ascending order: count per warp range, then write at the offsets
  int wn = 0;
  for (int j0 = w_lo; j0 < w_hi; j0 += 32) {
    const int j = j0 + lane;
    bool sel = false;
    if (j < w_hi) {
      const uint64_t kj = desc_key(s[j]);
      sel = kj < kb || (kj == kb && j <= jb);
    }
    wn += __popc(__ballot_sync(0xffffffffu, sel));
  }
  if (lane == 0) ctl->wcount[warp] = wn;
  __syncthreads();
  int n = 0, pos0 = 0;
  for (int w = 0; w < NWARP; ++w) {
    const int c = ctl->wcount[w];
    if (w < warp) pos0 += c;
    n += c;
  }
  for (int j0 = w_lo; j0 < w_hi; j0 += 32) {
    const int j = j0 + lane;
    bool sel = false;
    if (j < w_hi) {
      const uint64_t kj = desc_key(s[j]);
      sel = kj < kb || (kj == kb && j <= jb);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, sel);
    const int pos = pos0 + __popc(bal & ((1u << lane) - 1u));
    if (sel && pos < cap) out[pos] = j;
    pos0 += __popc(bal);
  }
  if (tid == 0) {
    if (n > cap) flag_error(st, DEVERR_CAPACITY, 0);
    *count = min(n, cap);
  }
  __syncthreads();  // the control block and histogram are reused by the CTA's next row
}

// The fp64 path for the rows the key selection queued: one CTA per row (grid-stride over the
// queue).  Its eight warps compute the row's scores Qbar_i . Kbar_j * scale in fp64 into shared
// memory, lanes splitting each dot product over D (coalesced reads of every Kbar row, then a
// shuffle reduction), then every score's fixed-point mass once (the selection's passes would
// otherwise evaluate the fp64 exponential again in each pass), and the whole CTA selects from
// there (select_row_fp64_cta: the decision of select_row_fp64, with the work of each pass
// split over the warps instead of one warp walking the row while the others wait).
constexpr int kFallbackThreads = 256;  // 8 warps: each key's dot product is one warp's, 8 keys per round
__global__ void __launch_bounds__(kFallbackThreads) router_fallback_kernel(const double* __restrict__ qbar,
                                                              const double* __restrict__ kbar, int D, int T,
                                                              double scale, const int* __restrict__ flist, int top_k,
                                                              float top_p, int cap, int32_t* __restrict__ kv_index,
                                                              int32_t* __restrict__ kv_count, DevStatus* st) {
  extern __shared__ double srow[];  // [T] scores, then [T] masses
  __shared__ uint32_t cnt_s[256];
  __shared__ unsigned long long mass_s[256];
  __shared__ double wmax[kFallbackThreads / 32], wmin[kFallbackThreads / 32];
  __shared__ SelCtl ctl;
  unsigned long long* mrow = reinterpret_cast<unsigned long long*>(srow + T);
  constexpr int kWarps = kFallbackThreads / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nf = static_cast<int>(*reinterpret_cast<const volatile unsigned*>(&st->router_fallback));
  const int per = D >> 5;  // doubles per lane (2 or 4)
  for (int k = blockIdx.x; k < nf; k += gridDim.x) {
    const int row = flist[k];
    const size_t bh = static_cast<size_t>(row) / T;
    double qv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) qv[e] = e < per ? qbar[static_cast<size_t>(row) * D + lane * per + e] : 0.0;
    // eight keys per warp per round, every load issued before the arithmetic
    for (int j0 = warp * 8; j0 < T; j0 += 8 * kWarps) {
      double kv[8][4];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u < T ? j0 + u : T - 1;
        const double* kj = kbar + (bh * T + j) * D + lane * per;
#pragma unroll
        for (int e = 0; e < 4; ++e) kv[u][e] = e < per ? kj[e] : 0.0;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        double acc = 0.0;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc = fma(qv[e], kv[u][e], acc);
#pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0 && j0 + u < T) srow[j0 + u] = acc * scale;
      }
    }
    __syncthreads();
    double mx = -DBL_MAX, mn = DBL_MAX;
    for (int j = threadIdx.x; j < T; j += kFallbackThreads) {
      mx = fmax(mx, srow[j]);
      mn = fmin(mn, srow[j]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if (lane == 0) {
      wmax[warp] = mx;
      wmin[warp] = mn;
    }
    __syncthreads();
    mx = wmax[0];
    mn = wmin[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      mx = fmax(mx, wmax[w]);
      mn = fmin(mn, wmin[w]);
    }
    for (int j = threadIdx.x; j < T; j += kFallbackThreads) mrow[j] = mass_fx(srow[j], mx);
    __syncthreads();
    select_row_fp64_cta<kWarps>(srow, mrow, mx, mn, T, top_k, top_p, cap, kv_index + static_cast<size_t>(row) * cap,
                                kv_count + row, st, cnt_s, mass_s, &ctl);
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

// fixed (not the device's SM count): one row per CTA, grid-stride over the queue (4 CTAs per SM)
int plan_fallback_ctas() { return 592; }

cudaError_t launch_plan_fast(const void* q, const void* k, const float* q_scale, const float* k_scale,
                             const CUtensorMap& tm_qlimb, const CUtensorMap& tm_klimb, const CUtensorMap& tm_keys,
                             const Geom& g, int BH, int D,
                             bool fp8, double scale, int top_k, float top_p, int cap, unsigned debug,
                             unsigned long long timeout_ns, const PlanFastWs& w, int32_t* kv_index, int32_t* kv_count,
                             DevStatus* st, cudaStream_t stream, int* launches) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaSuccess;
    for (auto fn : {score_keys_kernel<4, false>, score_keys_kernel<2, false>, score_keys_kernel<4, true>,
                    score_keys_kernel<2, true>})
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, rsc::SMEM_BYTES);
    if (e == cudaSuccess)  // one fp64 score row and its masses, up to 8192 cubes
      e = cudaFuncSetAttribute(router_fallback_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 8192 * 16);
    for (auto fn : {pool_limbs_kernel<2, 4>, pool_limbs_kernel<2, 2>, pool_limbs_kernel<1, 4>, pool_limbs_kernel<1, 2>})
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, rpl::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  // the per-head maxima of the key exponents start at 0 (below every biased exponent)
  if (cudaMemsetAsync(w.kexp_max, 0, static_cast<size_t>(BH) * sizeof(unsigned), stream) != cudaSuccess)
    return cudaErrorUnknown;
  PoolArgs pa;
  pa.q = static_cast<const uint8_t*>(q);
  pa.k = static_cast<const uint8_t*>(k);
  pa.q_scale = q_scale;
  pa.k_scale = k_scale;
  pa.qbar = w.qbar;
  pa.kbar = w.kbar;
  pa.qlimb = w.qlimb;
  pa.klimb = w.klimb;
  pa.qexp = w.qexp;
  pa.kexp = w.kexp;
  pa.ql1 = w.ql1;
  pa.kexp_max = w.kexp_max;
  pa.rkmax = w.rkmax;
  pa.rkmin = w.rkmin;
  pa.st = st;
  pa.g = g;
  pa.BH = BH;
  pa.D = D;
  pa.Tk = w.Tk;
  pa.timeout_ns = timeout_ns;
  const long long pitems = 2LL * BH * g.T;
  const int pgrid = static_cast<int>(pitems < num_sms() ? pitems : num_sms());
  if (fp8) {
    if (D == 128)
      pool_limbs_kernel<1, 4><<<pgrid, rpl::kThreads, rpl::SMEM_BYTES, stream>>>(pa);
    else
      pool_limbs_kernel<1, 2><<<pgrid, rpl::kThreads, rpl::SMEM_BYTES, stream>>>(pa);
  } else {
    if (D == 128)
      pool_limbs_kernel<2, 4><<<pgrid, rpl::kThreads, rpl::SMEM_BYTES, stream>>>(pa);
    else
      pool_limbs_kernel<2, 2><<<pgrid, rpl::kThreads, rpl::SMEM_BYTES, stream>>>(pa);
  }
  ScoreArgs sa_;
  sa_.qexp = w.qexp;
  sa_.kexp = w.kexp;
  sa_.ql1 = w.ql1;
  sa_.kexp_max = w.kexp_max;
  sa_.keys = w.keys;
  sa_.rkmax = w.rkmax;
  sa_.rkmin = w.rkmin;
  sa_.meta = reinterpret_cast<RowMeta*>(w.meta);
  sa_.s32 = w.s32;
  sa_.st = st;
  sa_.T = g.T;
  sa_.Tk = w.Tk;
  sa_.BH = BH;
  sa_.scale = scale;
  sa_.timeout_ns = timeout_ns;
  const int nrb = (g.T + 127) / 128;
  const long long items = static_cast<long long>(BH) * nrb * nrb;
  const int grid = static_cast<int>(items < num_sms() ? items : num_sms());
  auto kern = D == 64 ? (w.s32 ? score_keys_kernel<2, true> : score_keys_kernel<2, false>)
                      : (w.s32 ? score_keys_kernel<4, true> : score_keys_kernel<4, false>);
  kern<<<grid, rsc::kThreads, rsc::SMEM_BYTES, stream>>>(tm_qlimb, tm_klimb, tm_keys, sa_);
  const int rows = BH * g.T;
  select_keys_kernel<<<(rows + 7) / 8, 256, 0, stream>>>(
        w.keys, w.Tk, w.rkmax, w.rkmin, reinterpret_cast<const RowMeta*>(w.meta), rows, g.T, top_k, top_p, cap,
        kv_index, kv_count, w.flist, st, debug, timeout_ns);
  router_fallback_kernel<<<plan_fallback_ctas(), kFallbackThreads, static_cast<size_t>(g.T) * 16, stream>>>(
      w.qbar, w.kbar, D, g.T, scale, w.flist, top_k, top_p, cap, kv_index, kv_count, st);
  *launches = 5;
  return cudaGetLastError();
}

}  // namespace sa
