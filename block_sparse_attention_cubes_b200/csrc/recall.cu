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

namespace sa {

// ------------------------------------------------------------------------ oracle block scores
// P_oracle (VSA2 page, section 2.2: MeanPool over the B x B tiles of the token-level softmax P,
// the reference the router approximates): for every (query cube i, key cube j), the softmax
// mass the valid query tokens of cube i put on the valid keys of cube j, averaged over cube i's
// valid tokens.  With lse_r the natural log of row r's softmax normaliser over every valid key
// (sa_forward on lists holding every block), P_rc = exp(s_rc * scale - lse_r), so one dense
// pass of S = Q K^T gives it without a second softmax pass.
//
// Work item = two adjacent query cubes (128 rows) against every key cube, two key cubes (128
// keys) per step: S = Q2 [K_2s; K_2s+1]^T on the tensor cores (tcgen05, TMEM accumulator,
// double-buffered), then thread r of group g takes row r and the 64 keys of cube 2s + g:
// exponentials, row sum, a warp sum over 32 rows and a shared-memory sum over the two warps of
// each query cube.  Warp roles as in the forward kernel: warp 0 TMA, warp 1 TMEM owner and
// MMA issuer, warps 2-9 the exponentials.
namespace bm {
constexpr int kThreads = 320;
constexpr int KST = 3;
constexpr uint32_t OFF_Q = 0;                    // Q2: [2 halves][128 rows][128 B]
constexpr uint32_t OFF_K = 32768;                // KST x [2 halves][128 keys][128 B]
constexpr uint32_t OFF_BAR = OFF_K + KST * 32768;
constexpr uint32_t OFF_SLOT = OFF_BAR + 256;
constexpr uint32_t OFF_ABORT = OFF_BAR + 264;
constexpr uint32_t OFF_PART = OFF_BAR + 512;     // [2 S buffers][2 groups][4 warps] float
constexpr uint32_t SMEM_BYTES = OFF_PART + 256 + 1024;
constexpr uint32_t TMEM_COLS = 256;              // S[b] at 128 b
enum { B_QF = 0, B_QE = 1, B_KF = 2, B_KE = 5, B_SF = 8, B_SE = 10, B_FIN = 12, NBAR = 13 };
}  // namespace bm

struct MassArgs {
  const float* lse;                     // [BH, Npad]
  const unsigned long long* cube_mask;  // [T]
  float* pblock;                        // [BH, T, T]
  DevStatus* st;
  Geom g;
  int BH, rows_total;
  float scale_log2;
  unsigned long long timeout_ns;
};

template <int KS>
__global__ void __launch_bounds__(bm::kThreads, 1)
    block_mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const MassArgs a) {
  using namespace bm;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  float* part = reinterpret_cast<float*>(smem + OFF_PART);
  volatile int* sm_abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const int npairs = (g.T + 1) >> 1;
  const int n_items = a.BH * npairs;
  const int nsteps = (g.T + 1) >> 1;  // every key cube, two per step

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b) mbar_init(&bars[b], (b == B_SE || b == B_SE + 1) ? 256u : 1u);
    *sm_abort = aborted(a.st) ? 1 : 0;
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
  const bool skip_all = *sm_abort != 0;

  if (warp == 0) {
    if (lane == 0 && !skip_all) {
      uint32_t gs = 0;
      int issued_q = 0;
      bool ok = true;
      for (int it = blockIdx.x, n = 0; ok && it < n_items; it += gridDim.x, ++n) {
        const int bh = it / npairs, pr = it % npairs;
        if (n >= 1 && !mbar_wait(&bars[B_QE], (n - 1) & 1, a.st, a.timeout_ns, 141)) break;
        const int r0 = bh * g.Npad + (2 * pr) * 64;
        const int r1 = (2 * pr + 1 < g.T) ? r0 + 64 : a.rows_total;
        mbar_arrive_expect_tx(&bars[B_QF], 32768);
        tma_load_2d(smem + OFF_Q, &tm_q, &bars[B_QF], 0, r0);
        tma_load_2d(smem + OFF_Q + 8192, &tm_q, &bars[B_QF], 0, r1);
        tma_load_2d(smem + OFF_Q + 16384, &tm_q, &bars[B_QF], 64, r0);
        tma_load_2d(smem + OFF_Q + 24576, &tm_q, &bars[B_QF], 64, r1);
        ++issued_q;
        for (int s = 0; s < nsteps; ++s) {
          const uint32_t st = gs % KST;
          if (gs >= KST && !mbar_wait(&bars[B_KE + st], ((gs / KST) + 1) & 1, a.st, a.timeout_ns, 142)) {
            ok = false;
            break;
          }
          const int y0 = bh * g.Npad + (2 * s) * 64;
          const int y1 = (2 * s + 1 < g.T) ? y0 + 64 : a.rows_total;
          uint8_t* dst = smem + OFF_K + st * 32768;
          mbar_arrive_expect_tx(&bars[B_KF + st], 32768);
          tma_load_2d(dst, &tm_k, &bars[B_KF + st], 0, y0);
          tma_load_2d(dst + 8192, &tm_k, &bars[B_KF + st], 0, y1);
          tma_load_2d(dst + 16384, &tm_k, &bars[B_KF + st], 64, y0);
          tma_load_2d(dst + 24576, &tm_k, &bars[B_KF + st], 64, y1);
          ++gs;
        }
      }
      if (issued_q > 0) mbar_wait_drain(&bars[B_QF], (issued_q - 1) & 1, a.st, a.timeout_ns, 143);
      for (uint32_t s = (gs > KST ? gs - KST : 0); s < gs; ++s)
        mbar_wait_drain(&bars[B_KF + s % KST], (s / KST) & 1, a.st, a.timeout_ns, 144);
    }
  } else if (warp == 1) {
    if (!skip_all) {
      const uint32_t idesc = make_idesc(128, 128, FMT_BF16, false, false);
      uint32_t gs = 0;
      bool ok = true;
      for (int it = blockIdx.x, n = 0; ok && it < n_items; it += gridDim.x, ++n) {
        if (!mbar_wait_warp(&bars[B_QF], n & 1, a.st, a.timeout_ns, 151)) break;
        for (int s = 0; s < nsteps; ++s, ++gs) {
          const uint32_t kst_i = gs % KST, sb = gs & 1;
          // S buffer sb was last read by the exponentials of step gs - 2
          if (gs >= 2 && !mbar_wait_warp(&bars[B_SE + sb], ((gs >> 1) + 1) & 1, a.st, a.timeout_ns, 152)) {
            ok = false;
            break;
          }
          if (!mbar_wait_warp(&bars[B_KF + kst_i], (gs / KST) & 1, a.st, a.timeout_ns, 153)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kst = sbase + OFF_K + kst_i * 32768;
          if (elect_one()) {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
              umma_f16_ss(tmem + sb * 128, sw128_desc(sbase + OFF_Q + off, 16, 1024), sw128_desc(kst + off, 16, 1024),
                          idesc, ks > 0 ? 1u : 0u);
            }
            umma_commit(&bars[B_SF + sb]);
            umma_commit(&bars[B_KE + kst_i]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) umma_commit(&bars[B_QE]);  // every product reading Q2 has been issued
        __syncwarp();
      }
      if (elect_one()) umma_commit(&bars[B_FIN]);
      __syncwarp();
      mbar_wait_drain(&bars[B_FIN], 0, a.st, a.timeout_ns, 154);
    }
  } else {
    const int grp = (warp - 2) >> 2;    // key cube 2s + grp of each step
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row of the pair == TMEM lane
    const int half = r >> 6;            // which query cube of the pair
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t gs = 0;
    bool ok = !skip_all;
    for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      const int bh = it / npairs, pr = it % npairs;
      const int icube = 2 * pr + half;
      const bool row_exists = icube < g.T;
      const bool row_valid = row_exists && ((a.cube_mask[icube] >> (r & 63)) & 1ull);
      const float nlse2 =
          row_valid ? -a.lse[static_cast<size_t>(bh) * g.Npad + static_cast<size_t>(icube) * 64 + (r & 63)] *
                          1.4426950408889634f
                    : 0.0f;
      const float ninv = row_exists ? 1.0f / static_cast<float>(__popcll(a.cube_mask[icube])) : 0.0f;
      for (int s = 0; s < nsteps; ++s, ++gs) {
        const uint32_t b = gs & 1;
        const int jc = 2 * s + grp;  // key cube of this thread's 64 columns
        const unsigned long long km = jc < g.T ? a.cube_mask[jc] : 0ull;
        // a wait that gives up raises the CTA's abort flag, read by the group after its barrier
        if (!mbar_wait(&bars[B_SF + b], (gs >> 1) & 1, a.st, a.timeout_ns, 161)) *sm_abort = 1;
        tc_fence_after();
        uint32_t s0[32], s1[32];
        tmem_ld32(t_lane + b * 128 + grp * 64, s0);
        tmem_ld32(t_lane + b * 128 + grp * 64 + 32, s1);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bars[B_SE + b]);  // S[b] may take the next product
        float sum = 0.0f;
        if (row_valid) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(s0[c]), a.scale_log2, nlse2));
            const float p1 = ex2_approx(fmaf(__uint_as_float(s1[c]), a.scale_log2, nlse2));
            acc[c & 3] += ((km >> c) & 1ull) ? p0 : 0.0f;
            acc[(c + 2) & 3] += ((km >> (c + 32)) & 1ull) ? p1 : 0.0f;
          }
          sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        float* pp = part + (b * 2 + grp) * 4;
        if (lane == 0) pp[quarter] = sum;
        named_bar_sync(1 + grp, 128);  // the four warps of this group
        if (*sm_abort) {
          ok = false;
          break;
        }
        if ((quarter & 1) == 0 && lane == 0 && row_exists && jc < g.T) {
          const float m = (pp[quarter] + pp[quarter + 1]) * ninv;
          a.pblock[(static_cast<size_t>(bh) * g.T + icube) * g.T + jc] = m;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, bm::TMEM_COLS);
}

// ------------------------------------------------------------------------ best recall
// Sum of the n largest entries of each row of pblock (n = kv_count of the row, clamped to
// [0, T]): the best recall any selection of n blocks could reach under P_oracle.  One warp per
// row: a radix descent over the (non-negative) fp32 bit patterns finds the n-th largest value
// v; the sum is that of the entries above v plus (n - their count) times v, in fp64.
__global__ void __launch_bounds__(256) best_recall_kernel(const float* __restrict__ pblock,
                                                          const int32_t* __restrict__ kv_count, float* __restrict__ best,
                                                          int rows, int T) {
  __shared__ uint32_t hist_s[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const uint32_t* x = reinterpret_cast<const uint32_t*>(pblock + static_cast<size_t>(row) * T);
  uint32_t* hist = hist_s[warp];
  const int n = min(max(kv_count[row], 0), T);
  double total = 0.0;
  if (n > 0) {
    uint32_t prefix = 0;   // the n-th largest bit pattern, built from the top byte down
    int need = n;          // rank still to find inside the current prefix
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int d = lane; d < 256; d += 32) hist[d] = 0;
      __syncwarp();
      const uint32_t hmask = shift == 24 ? 0u : ~((1u << (shift + 8)) - 1u);
      for (int j = lane; j < T; j += 32) {
        const uint32_t v = x[j];
        if ((v & hmask) == (prefix & hmask)) atomicAdd(&hist[(v >> shift) & 255u], 1u);
      }
      __syncwarp();
      // the bucket holding rank `need`, counted from the largest value down
      uint32_t c8[8], lc = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        c8[u] = hist[255 - (lane * 8 + u)];
        lc += c8[u];
      }
      uint32_t ic = lc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, ic, o);
        if (lane >= o) ic += t;
      }
      int hit = -1, above = 0;
      uint32_t run = ic - lc;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (hit < 0 && run + c8[u] >= static_cast<uint32_t>(need)) {
          hit = 255 - (lane * 8 + u);
          above = static_cast<int>(run);
        }
        run += c8[u];
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, hit >= 0);
      const int src = __ffs(bal) - 1;
      const int d = __shfl_sync(0xffffffffu, hit, src);
      need -= __shfl_sync(0xffffffffu, above, src);
      prefix |= static_cast<uint32_t>(d) << shift;
      __syncwarp();
    }
    // entries strictly above the n-th largest, then `need` copies of it
    double s = 0.0;
    int c_above = 0;
    for (int j = lane; j < T; j += 32) {
      const uint32_t v = x[j];
      if (v > prefix) {
        s += static_cast<double>(__uint_as_float(v));
        ++c_above;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      s += __shfl_xor_sync(0xffffffffu, s, o);
      c_above += __shfl_xor_sync(0xffffffffu, c_above, o);
    }
    total = s + static_cast<double>(n - c_above) * static_cast<double>(__uint_as_float(prefix));
  }
  if (lane == 0) best[row] = static_cast<float>(total);
}

cudaError_t launch_block_mass(const CUtensorMap& tq, const CUtensorMap& tk, const float* lse,
                              const unsigned long long* cube_mask, float* pblock, const Geom& g, int BH, int D,
                              float scale_log2, DevStatus* st, unsigned long long timeout_ns, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(block_mass_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         bm::SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(block_mass_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, bm::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  MassArgs a;
  a.lse = lse;
  a.cube_mask = cube_mask;
  a.pblock = pblock;
  a.st = st;
  a.g = g;
  a.BH = BH;
  a.rows_total = BH * g.Npad;
  a.scale_log2 = scale_log2;
  a.timeout_ns = timeout_ns;
  const int items = BH * ((g.T + 1) >> 1);
  const int sms = num_sms();
  const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  if (D == 64)
    block_mass_kernel<4><<<grid, bm::kThreads, bm::SMEM_BYTES, stream>>>(tq, tk, a);
  else
    block_mass_kernel<8><<<grid, bm::kThreads, bm::SMEM_BYTES, stream>>>(tq, tk, a);
  return cudaGetLastError();
}

cudaError_t launch_best_recall(const float* pblock, const int32_t* kv_count, float* best, int rows, int T,
                               cudaStream_t stream) {
  best_recall_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(pblock, kv_count, best, rows, T);
  return cudaGetLastError();
}

}  // namespace sa
