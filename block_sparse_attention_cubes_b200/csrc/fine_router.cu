// VSA2's fine-grained router with per-sequence Top-K (VSA2 page, section 2.2, router equations):
//   Q_r, K_r = MeanPool_R([Q, K])          each cube split into G = 64 / |R| groups of R tokens
//   P^_r = softmax(Q_r K_r^T / sqrt(D))    over every key group of the sequence, per query group
//   P_r = the G x G aggregation of P^_r    one score per (query cube, key cube)
//   per-sequence Top-K                     min(K N, N^2) largest entries of P_r per (batch, head)
//
// Readings (where the page leaves a step open): a group is the R_t x R_h x R_w box of a cube's
// (t, h, w) offsets and is pooled over its valid tokens; a group without valid tokens takes no
// part (no query row, probability 0 as a key); P_r[i, j] is the mass a query group of cube i
// puts on the key groups of cube j, averaged over cube i's valid query groups; Top-K ties are
// broken by the smaller row-major index; a query cube may keep no block.
//
// Kernels:
//   fine_pool_kernel     group means (fp64 sums over the valid tokens), their int8 limbs and
//                        binary exponents, validity flags (a TMA ring of whole cubes, as the
//                        cube router's pooling)
//   fine_score_kernel    the group-level scores on the tensor cores from exact limb products
//                        (tcgen05 kind::i8), one CTA per block of 128 query groups walking every
//                        key group; pass 1 keeps each row's running maximum and sum of
//                        exponentials (log2 units) and writes its lse, pass 2 recomputes the
//                        scores, sums exp(s - lse) per key cube in the epilogue and over the
//                        query groups of each query cube with warp shuffles, and writes P_r
//   seq_topk_kernel      one CTA per (batch, head): radix selection of the budget over the
//                        fp32 bit patterns of P_r (non-negative), then every row's kept ids in
//                        ascending order
// Scores are exact up to the limb error bound; exponentials use ex2.approx on fp32 arguments,
// so P_r carries a relative error of a few 1e-6 and the selection is that of the fp32 P_r.
#include <cfloat>
#include <climits>
#include <cmath>

#include "geometry.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "router_common.cuh"

namespace sa {

// ------------------------------------------------------------------------ group pooling
namespace fpl {
constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kStages = 12;
// A consumer's next stage is kConsumers stages past its last one; a parity wait tells apart only
// a barrier's current phase and the one before, so the previous fill of that stage must have
// landed already: kStages >= kConsumers guarantees it.
static_assert(kStages >= kConsumers, "a full-barrier wait could pass on a fill two phases old");
constexpr uint32_t kStageBytes = 16384;  // one cube of 64 rows x 256 bytes (bf16, D = 128)
constexpr uint32_t OFF_BAR = kStages * kStageBytes;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 2 * kStages * 8 + 1024;
}  // namespace fpl

// EPL = D / 32 values per lane (bf16).  Items (head, cube, Q or K) are dealt round-robin; warp
// 8 streams the cubes into the ring, warps 0-7 take them in turn and write, for each of the G
// groups, the mean, its limbs, its exponent and validity (and for Q the 1-norm).
template <int EPL>
__global__ void __launch_bounds__(fpl::kThreads, 1) fine_pool_kernel(const FinePoolArgs a) {
  using namespace fpl;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + kStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const int D = EPL * 32;
  const size_t row_bytes = static_cast<size_t>(D) * 2;
  const long long n_items = 2LL * a.BH * g.T;
  const int G = 64 / (a.rt * a.rh * a.rw);
  const int TG = g.T * G;
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
      long long i = 0;
      for (long long it = blockIdx.x; it < n_items; it += gridDim.x, ++i) {
        const int stage = static_cast<int>(i % kStages);
        if (i >= kStages && !mbar_wait(&empty[stage], ((i / kStages) + 1) & 1, a.st, a.timeout_ns, 171)) break;
        const long long cube = it >> 1;
        const int c = static_cast<int>(cube % g.T);
        int vt, vh, vw;
        cube_extent(g, c, vt, vh, vw);
        const uint32_t nrows = static_cast<uint32_t>(16 * (vt - 1) + 4 * (vh - 1) + vw);
        const uint8_t* src = ((it & 1) ? a.k : a.q) +
                             (static_cast<size_t>(cube / g.T) * g.Npad + static_cast<size_t>(c) * 64) * row_bytes;
        const uint32_t bytes = nrows * static_cast<uint32_t>(row_bytes);
        mbar_arrive_expect_tx(&full[stage], bytes);
        bulk_load(smem + stage * kStageBytes, src, bytes, &full[stage]);
      }
      const long long issued = i;
      for (long long d = (issued > kStages ? issued - kStages : 0); d < issued; ++d)
        mbar_wait_drain(&full[d % kStages], (d / kStages) & 1, a.st, a.timeout_ns, 172);
    }
    return;
  }
  long long i = warp;
  for (long long it = blockIdx.x + static_cast<long long>(warp) * gridDim.x; it < n_items;
       it += static_cast<long long>(kConsumers) * gridDim.x, i += kConsumers) {
    const int stage = static_cast<int>(i % kStages);
    if (!mbar_wait_warp(&full[stage], (i / kStages) & 1, a.st, a.timeout_ns, 173)) break;
    const int which = static_cast<int>(it & 1);
    const long long cube = it >> 1;
    const int bh = static_cast<int>(cube / g.T), c = static_cast<int>(cube % g.T);
    int vt, vh, vw;
    cube_extent(g, c, vt, vh, vw);
    const uint8_t* tile = smem + stage * kStageBytes + lane * EPL * 2;
    int8_t* lb = which ? a.klimb : a.qlimb;
    for (int gi = 0; gi < G; ++gi) {
      // the group's box: rows a0 in [ta, ta + rt), b0 in [tb, tb + rh), d0 in [td, td + rw)
      const int ng_h = 4 / a.rh, ng_w = 4 / a.rw;
      const int ta = (gi / (ng_h * ng_w)) * a.rt, tb = ((gi / ng_w) % ng_h) * a.rh, td = (gi % ng_w) * a.rw;
      double acc[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] = 0.0;
      int n = 0;
      for (int a0 = ta; a0 < ta + a.rt; ++a0)
        for (int b0 = tb; b0 < tb + a.rh; ++b0)
          for (int d0 = td; d0 < td + a.rw; ++d0) {
            if (a0 >= vt || b0 >= vh || d0 >= vw) continue;
            ++n;
            const uint8_t* rp = tile + (a0 * 16 + b0 * 4 + d0) * row_bytes;
            uint32_t wv[EPL / 2];
            if constexpr (EPL == 4) {
              const uint2 t2 = *reinterpret_cast<const uint2*>(rp);
              wv[0] = t2.x;
              wv[1] = t2.y;
            } else {
              wv[0] = *reinterpret_cast<const uint32_t*>(rp);
            }
#pragma unroll
            for (int e = 0; e < EPL; ++e)
              acc[e] += static_cast<double>(__uint_as_float((e & 1) ? (wv[e >> 1] & 0xffff0000u) : (wv[e >> 1] << 16)));
          }
      const long long grow = static_cast<long long>(bh) * TG + static_cast<long long>(c) * G + gi;  // group row
      double x[EPL], amax = 0.0, l1 = 0.0;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        x[e] = n > 0 ? acc[e] / static_cast<double>(n) : 0.0;
        amax = fmax(amax, fabs(x[e]));
        l1 += fabs(x[e]);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
      int E = kExpZero;
      if (amax > 0.0) frexp(amax, &E);
      const double up = amax > 0.0 ? ldexp(1.0, 30 - E) : 0.0;
      uint32_t limb[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int e = 0; e < EPL; ++e) limb_digits(x[e], up, e, limb);
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        int8_t* rowp = lb + ((static_cast<size_t>(bh) * 4 + l) * TG + static_cast<size_t>(c) * G + gi) * kLimbRow;
        if constexpr (EPL == 4) {
          reinterpret_cast<uint32_t*>(rowp)[lane] = limb[l];
        } else {
          reinterpret_cast<uint16_t*>(rowp)[lane] = static_cast<uint16_t>(limb[l]);
          reinterpret_cast<uint16_t*>(rowp + 64)[lane] = 0;
        }
      }
      if (lane == 0) {
        const size_t prow = static_cast<size_t>(bh) * a.TGp + static_cast<size_t>(c) * G + gi;  // padded rows
        if (which) {
          a.kexp[prow] = E;
          a.kvalid[prow] = n > 0 ? 1 : 0;
          if (n > 0) atomicMax(a.kexp_max + bh, static_cast<unsigned>(E + kExpBias));
        } else {
          a.qexp[grow] = E;
          a.qvalid[grow] = n > 0 ? 1 : 0;
          a.ql1[grow] = l1;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);  // every group of the cube has been read
  }
}

// ------------------------------------------------------------------------ group scores
namespace fsc {
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 TMEM owner + MMA, warps 2-9 epilogue
constexpr uint32_t OFF_Q = 0;              // 4 limbs x [128 rows][128 B]
constexpr uint32_t OFF_K = 65536;          // 2 stages x 4 limbs x [128 key groups][128 B]
constexpr uint32_t OFF_BAR = OFF_K + 2 * 65536;
constexpr uint32_t OFF_SLOT = OFF_BAR + 128;
constexpr uint32_t OFF_ABORT = OFF_BAR + 136;
constexpr uint32_t OFF_RED = OFF_BAR + 256;  // [2 halves][128 rows] float x 2 (max, sum)
constexpr uint32_t SMEM_BYTES = OFF_RED + 2048 + 1024;
constexpr uint32_t TMEM_COLS = 512;
enum { B_QF = 0, B_QE = 1, B_KF = 2, B_KE = 4, B_TF = 6, B_TE = 7, B_FIN = 8, NBAR = 9 };
}  // namespace fsc

// PASS 1: lse of every query group (log2 units, over its valid key groups).  PASS 2: P_r.
// Work item = (head, block of 128 query groups) over every key group, one CTA at a time.
// G = groups per cube (4, 8 or 16): the G key groups of a key cube are G consecutive columns of
// a 32-column chunk and the G query groups of a query cube G consecutive lanes of a warp.
template <int KS, int PASS, int G>
__global__ void __launch_bounds__(fsc::kThreads, 1)
    fine_score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const FineScoreArgs a) {
  using namespace fsc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);
  volatile int* sm_abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int TG = a.TG;
  const int nrb = (TG + 127) >> 7;
  const int n_items = a.BH * nrb;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b) mbar_init(&bars[b], b == B_TE ? 256u : 1u);
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
      uint32_t ks = 0;
      int qn = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        const int bh = it / nrb, rb = it % nrb;
        if (qn >= 1 && !mbar_wait(&bars[B_QE], (qn - 1) & 1, a.st, a.timeout_ns, 181)) break;
        mbar_arrive_expect_tx(&bars[B_QF], 65536);
#pragma unroll
        for (int l = 0; l < 4; ++l) tma_load_3d(smem + OFF_Q + l * 16384, &tm_q, &bars[B_QF], 0, rb * 128, bh * 4 + l);
        ++qn;
        for (int cb = 0; cb < nrb; ++cb) {
          const uint32_t st = ks & 1u;
          if (ks >= 2 && !mbar_wait(&bars[B_KE + st], ((ks >> 1) + 1) & 1, a.st, a.timeout_ns, 182)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars[B_KF + st], 65536);
#pragma unroll
          for (int l = 0; l < 4; ++l)
            tma_load_3d(smem + OFF_K + st * 65536 + l * 16384, &tm_k, &bars[B_KF + st], 0, cb * 128, bh * 4 + l);
          ++ks;
        }
      }
      if (qn > 0) mbar_wait_drain(&bars[B_QF], (qn - 1) & 1, a.st, a.timeout_ns, 183);
      for (uint32_t s = (ks > 2 ? ks - 2 : 0); s < ks; ++s)
        mbar_wait_drain(&bars[B_KF + (s & 1u)], (s >> 1) & 1, a.st, a.timeout_ns, 184);
    }
  } else if (warp == 1) {
    if (!skip_all) {
      uint32_t ks = 0, tile = 0;
      int qn = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        if (!mbar_wait_warp(&bars[B_QF], qn & 1, a.st, a.timeout_ns, 191)) break;
        ++qn;
        for (int cb = 0; cb < nrb; ++cb, ++ks, ++tile) {
          if (tile >= 1 && !mbar_wait_warp(&bars[B_TE], (tile - 1) & 1, a.st, a.timeout_ns, 192)) {
            ok = false;
            break;
          }
          const uint32_t st = ks & 1u;
          if (!mbar_wait_warp(&bars[B_KF + st], (ks >> 1) & 1, a.st, a.timeout_ns, 193)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            issue_limb_products<KS>(tmem, sbase + OFF_Q, sbase + OFF_K + st * 65536);
            umma_commit(&bars[B_KE + st]);
            umma_commit(&bars[B_TF]);
            if (cb + 1 == nrb) umma_commit(&bars[B_QE]);
          }
          __syncwarp();
        }
      }
      if (elect_one()) umma_commit(&bars[B_FIN]);
      __syncwarp();
      mbar_wait_drain(&bars[B_FIN], 0, a.st, a.timeout_ns, 194);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;  // query group row of the block == TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t tile = 0;
    bool ok = !skip_all;
    for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      const int bh = it / nrb, rb = it % nrb;
      const int row = rb * 128 + r;  // query group within the head
      const bool row_in = row < TG;
      const size_t grow = static_cast<size_t>(bh) * TG + (row_in ? row : 0);
      const bool qv = row_in && a.qvalid[grow] != 0;
      const int Eq = a.qexp[grow];
      // s * log2(e) = v * 2^(Eq + Ek - 36) * scale * log2(e): the row factor here, 2^Ek per column
      const float rowf = qv && Eq != kExpZero ? static_cast<float>(ldexp(a.scale_log2, Eq - 36)) : 0.0f;
      float m_run = -FLT_MAX, l_run = 0.0f;   // pass 1: running maximum and sum (log2 units)
      const float lse2 = PASS == 2 && qv ? a.lse2[grow] : 0.0f;
      const int* kexp = a.kexp + static_cast<size_t>(bh) * a.TGp;
      const int* kval = a.kvalid + static_cast<size_t>(bh) * a.TGp;
      for (int cb = 0; cb < nrb; ++cb, ++tile) {
        // warp-uniform: a warp that gives up leaves together (shuffles below), and raises the
        // CTA's abort flag, which the whole epilogue reads after its barrier (pass 1)
        if (!mbar_wait_warp(&bars[B_TF], tile & 1, a.st, a.timeout_ns, 201)) {
          ok = false;
          *sm_abort = 1;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          const int col0 = 64 * half + 32 * ch;
          const int jc = cb * 128 + col0;  // first key group of the chunk
          float colf[32];                  // 2^Ek of each key group, 0 when it has no valid token
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4) {
            const int4 e4 = jc + 4 * v4 < a.TGp ? __ldg(reinterpret_cast<const int4*>(kexp + jc) + v4) : make_int4(0, 0, 0, 0);
            const int4 f4 = jc + 4 * v4 < a.TGp ? __ldg(reinterpret_cast<const int4*>(kval + jc) + v4) : make_int4(0, 0, 0, 0);
            const int ee[4] = {e4.x, e4.y, e4.z, e4.w}, ff[4] = {f4.x, f4.y, f4.z, f4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = jc + 4 * v4 + u;
              const bool kv = j < TG && ff[u] != 0;
              colf[4 * v4 + u] = kv ? (ee[u] == kExpZero ? -1.0f : exp2f(static_cast<float>(ee[u]))) : -2.0f;
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
          // colf: > 0 a valid key group (2^Ek), -1 a valid group with a zero mean (score 0),
          // -2 no key (past TG or no valid token)
          float s2[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float v = static_cast<float>(limb_levels(L0[c], L1[c], L2[c], L3[c]));
            s2[c] = colf[c] > 0.0f ? v * rowf * colf[c] : (colf[c] == -1.0f ? 0.0f : -FLT_MAX);
          }
          if (PASS == 1) {
            if (!qv) continue;
            float cm = -FLT_MAX;
#pragma unroll
            for (int c = 0; c < 32; ++c) cm = fmaxf(cm, s2[c]);
            if (cm > m_run) {
              l_run *= ex2_approx(m_run - cm);
              m_run = cm;
            }
            float acc = 0.0f;
#pragma unroll
            for (int c = 0; c < 32; ++c) acc += s2[c] > -FLT_MAX ? ex2_approx(s2[c] - m_run) : 0.0f;
            l_run += acc;
          } else {
            // exp(s - lse) per key group (0 without a key or a query row), summed per key cube
            float cs[32 / G];
#pragma unroll
            for (int q = 0; q < 32 / G; ++q) {
              float sum = 0.0f;
#pragma unroll
              for (int u = 0; u < G; ++u) {
                const float sv = s2[q * G + u];
                sum += (qv && sv > -FLT_MAX) ? ex2_approx(sv - lse2) : 0.0f;
              }
              cs[q] = sum;
            }
            // and over the G query groups of each query cube (G consecutive lanes)
            int nq = qv ? 1 : 0;
#pragma unroll
            for (int o = 1; o < G; o <<= 1) {
              nq += __shfl_xor_sync(0xffffffffu, nq, o);
#pragma unroll
              for (int q = 0; q < 32 / G; ++q) cs[q] += __shfl_xor_sync(0xffffffffu, cs[q], o);
            }
            if ((lane & (G - 1)) == 0 && row_in && nq > 0) {
              const int icube = row / G;
              float* prow = a.pr + (static_cast<size_t>(bh) * a.T + icube) * a.T;
              const float inv = 1.0f / static_cast<float>(nq);
#pragma unroll
              for (int q = 0; q < 32 / G; ++q) {
                const int j = jc + q * G;
                if (j < TG) prow[j / G] = cs[q] * inv;
              }
            }
          }
        }
      }
      if (PASS == 1) {
        red[half * 128 + r] = m_run;
        red[256 + half * 128 + r] = l_run;
        named_bar_sync(1, 256);
        if (*sm_abort) break;
        if (half == 0 && row_in) {
          const float m2 = red[128 + r], l2 = red[384 + r];
          const float m = fmaxf(m_run, m2);
          const float l = l_run * ex2_approx(m_run - m) + l2 * ex2_approx(m2 - m);
          a.lse2[grow] = qv && l > 0.0f ? m + log2f(l) : 0.0f;
        }
        named_bar_sync(1, 256);
      } else if (!ok) {
        break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, fsc::TMEM_COLS);
}

// ------------------------------------------------------------------------ per-sequence Top-K
// One CTA (1024 threads) per (batch, head): the budget n = min(K T, T^2) largest entries of
// P_r [T, T], ties broken by the smaller row-major index.  A radix descent over the fp32 bit
// patterns (non-negative values) finds the n-th largest value v and how many entries equal to v
// are kept; per-row counts of the entries above and equal to v, a prefix over rows of the equal
// ones, and every row's kept ids are written in ascending order.
__global__ void __launch_bounds__(1024) seq_topk_kernel(const float* __restrict__ pr, int T, int K, int cap,
                                                        int32_t* __restrict__ kv_index, int32_t* __restrict__ kv_count,
                                                        DevStatus* st) {
  extern __shared__ int rowc[];  // [T] entries above v, then [T] entries equal to v, then [T] prefix
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_need;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const uint32_t* x = reinterpret_cast<const uint32_t*>(pr + static_cast<size_t>(bh) * T * T);
  const long long N = static_cast<long long>(T) * T;
  const long long budget = min(static_cast<long long>(K) * T, N);
  int* gt = rowc;
  int* eq = rowc + T;
  int* eqb = rowc + 2 * T;
  if (tid == 0) {
    s_prefix = 0u;
    s_need = static_cast<uint32_t>(budget);
  }
  __syncthreads();
  if (budget > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (tid < 256) hist[tid] = 0u;
      __syncthreads();
      const uint32_t prefix = s_prefix;
      const uint32_t hmask = shift == 24 ? 0u : ~((1u << (shift + 8)) - 1u);
      for (long long idx = tid; idx < N; idx += 1024) {
        const uint32_t v = x[idx];
        if ((v & hmask) == (prefix & hmask)) atomicAdd(&hist[(v >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // buckets from the largest value down: lane l takes buckets 255 - 8l - u
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
        const uint32_t need = s_need;
        int hit = -1;
        uint32_t above = 0, run = ic - lc;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (hit < 0 && run + c8[u] >= need) {
            hit = 255 - (lane * 8 + u);
            above = run;
          }
          run += c8[u];
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, hit >= 0);
        const int src = __ffs(bal) - 1;  // the budget does not exceed the count, so a bucket is hit
        const int d = __shfl_sync(0xffffffffu, hit, src);
        const uint32_t ab = __shfl_sync(0xffffffffu, above, src);
        if (lane == 0) {
          s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
          s_need = need - ab;
        }
      }
      __syncthreads();
    }
  }
  const uint32_t vt = s_prefix;                   // the n-th largest bit pattern
  const int need = budget > 0 ? static_cast<int>(s_need) : 0;  // entries equal to it that are kept
  // per-row counts above and equal to v
  for (int row = warp; row < T; row += 32) {
    int cg = 0, ce = 0;
    if (budget > 0)
      for (int j = lane; j < T; j += 32) {
        const uint32_t v = x[static_cast<size_t>(row) * T + j];
        cg += v > vt ? 1 : 0;
        ce += v == vt ? 1 : 0;
      }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      cg += __shfl_xor_sync(0xffffffffu, cg, o);
      ce += __shfl_xor_sync(0xffffffffu, ce, o);
    }
    if (lane == 0) {
      gt[row] = cg;
      eq[row] = ce;
    }
  }
  __syncthreads();
  if (warp == 0) {  // equal entries in the rows before each row
    int run = 0;
    for (int r0 = 0; r0 < T; r0 += 32) {
      const int r = r0 + lane;
      const int e = r < T ? eq[r] : 0;
      int incl = e;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (r < T) eqb[r] = run + incl - e;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncthreads();
  for (int row = warp; row < T; row += 32) {
    const int keq = budget > 0 ? max(0, min(need - eqb[row], eq[row])) : 0;  // equal entries kept in this row
    const int n = budget > 0 ? gt[row] + keq : 0;
    int32_t* out = kv_index + (static_cast<size_t>(bh) * T + row) * cap;
    int written = 0, eq_seen = 0;
    if (n > 0)
      for (int j0 = 0; j0 < T; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t v = j < T ? x[static_cast<size_t>(row) * T + j] : 0u;
        const bool isg = j < T && v > vt, ise = j < T && v == vt;
        const uint32_t eb = __ballot_sync(0xffffffffu, ise);
        const int erank = eq_seen + __popc(eb & ((1u << lane) - 1u));
        const bool sel = isg || (ise && erank < keq);
        const uint32_t sb = __ballot_sync(0xffffffffu, sel);
        const int pos = written + __popc(sb & ((1u << lane) - 1u));
        if (sel && pos < cap) out[pos] = j;
        written += __popc(sb);
        eq_seen += __popc(eb);
      }
    if (lane == 0) {
      if (n > cap) flag_error(st, DEVERR_CAPACITY, 0);
      kv_count[static_cast<size_t>(bh) * T + row] = min(n, cap);
    }
  }
}

cudaError_t launch_plan_fine(const void* q, const void* k, const CUtensorMap& tm_qlimb, const CUtensorMap& tm_klimb,
                             const Geom& g, int BH, int D, int rt, int rh, int rw, double scale, int K, int cap,
                             const FineWs& w, int32_t* kv_index, int32_t* kv_count, DevStatus* st,
                             unsigned long long timeout_ns, cudaStream_t stream, int* launches) {
  const int G = 64 / (rt * rh * rw);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaSuccess;
    for (auto fn : {fine_pool_kernel<4>, fine_pool_kernel<2>})
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, fpl::SMEM_BYTES);
    for (auto fn : {fine_score_kernel<4, 1, 4>, fine_score_kernel<4, 2, 4>, fine_score_kernel<4, 1, 8>,
                    fine_score_kernel<4, 2, 8>, fine_score_kernel<4, 1, 16>, fine_score_kernel<4, 2, 16>,
                    fine_score_kernel<2, 1, 4>, fine_score_kernel<2, 2, 4>, fine_score_kernel<2, 1, 8>,
                    fine_score_kernel<2, 2, 8>, fine_score_kernel<2, 1, 16>, fine_score_kernel<2, 2, 16>})
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, fsc::SMEM_BYTES);
    if (e == cudaSuccess)  // three int counts per row, up to 8192 rows
      e = cudaFuncSetAttribute(seq_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 3 * 8192 * 4);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  FinePoolArgs pa;
  pa.q = static_cast<const uint8_t*>(q);
  pa.k = static_cast<const uint8_t*>(k);
  pa.qlimb = w.qlimb;
  pa.klimb = w.klimb;
  pa.qexp = w.qexp;
  pa.qvalid = w.qvalid;
  pa.ql1 = w.ql1;
  pa.kexp = w.kexp;
  pa.kvalid = w.kvalid;
  pa.kexp_max = w.kexp_max;
  pa.st = st;
  pa.g = g;
  pa.BH = BH;
  pa.rt = rt;
  pa.rh = rh;
  pa.rw = rw;
  pa.TGp = w.TGp;
  pa.timeout_ns = timeout_ns;
  if (cudaMemsetAsync(w.kexp_max, 0, static_cast<size_t>(BH) * sizeof(unsigned), stream) != cudaSuccess)
    return cudaErrorUnknown;
  const long long pitems = 2LL * BH * g.T;
  const int pgrid = static_cast<int>(pitems < num_sms() ? pitems : num_sms());
  if (D == 128)
    fine_pool_kernel<4><<<pgrid, fpl::kThreads, fpl::SMEM_BYTES, stream>>>(pa);
  else
    fine_pool_kernel<2><<<pgrid, fpl::kThreads, fpl::SMEM_BYTES, stream>>>(pa);
  FineScoreArgs sa_;
  sa_.qexp = w.qexp;
  sa_.qvalid = w.qvalid;
  sa_.kexp = w.kexp;
  sa_.kvalid = w.kvalid;
  sa_.lse2 = w.lse2;
  sa_.pr = w.pr;
  sa_.st = st;
  sa_.T = g.T;
  sa_.TG = g.T * G;
  sa_.TGp = w.TGp;
  sa_.BH = BH;
  sa_.scale_log2 = scale * 1.4426950408889634;
  sa_.timeout_ns = timeout_ns;
  const int nrb = (sa_.TG + 127) / 128;
  const int items = BH * nrb;
  const int grid = items < num_sms() ? items : num_sms();
  using KFn = void (*)(CUtensorMap, CUtensorMap, FineScoreArgs);
  KFn p1 = nullptr, p2 = nullptr;
  if (D == 128) {
    if (G == 4) { p1 = fine_score_kernel<4, 1, 4>; p2 = fine_score_kernel<4, 2, 4>; }
    if (G == 8) { p1 = fine_score_kernel<4, 1, 8>; p2 = fine_score_kernel<4, 2, 8>; }
    if (G == 16) { p1 = fine_score_kernel<4, 1, 16>; p2 = fine_score_kernel<4, 2, 16>; }
  } else {
    if (G == 4) { p1 = fine_score_kernel<2, 1, 4>; p2 = fine_score_kernel<2, 2, 4>; }
    if (G == 8) { p1 = fine_score_kernel<2, 1, 8>; p2 = fine_score_kernel<2, 2, 8>; }
    if (G == 16) { p1 = fine_score_kernel<2, 1, 16>; p2 = fine_score_kernel<2, 2, 16>; }
  }
  if (!p1) return cudaErrorInvalidValue;
  p1<<<grid, fsc::kThreads, fsc::SMEM_BYTES, stream>>>(tm_qlimb, tm_klimb, sa_);
  p2<<<grid, fsc::kThreads, fsc::SMEM_BYTES, stream>>>(tm_qlimb, tm_klimb, sa_);
  seq_topk_kernel<<<BH, 1024, static_cast<size_t>(3) * g.T * sizeof(int), stream>>>(w.pr, g.T, K, cap, kv_index,
                                                                                     kv_count, st);
  *launches = 5;
  return cudaGetLastError();
}

}  // namespace sa
