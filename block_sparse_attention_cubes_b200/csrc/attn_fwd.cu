// Fine-stage forward: online-softmax attention of each 64-token query cube over the key
// cubes in its index list (SpargeAttention2 page, "Kernel Implementation of the
// Hybrid-Masked Block-Sparse Attention": per selected block pair, S = Q_i K_j^T / sqrt(d),
// running max and running sum, O rescaled and accumulated, divided by the sum at the end;
// unselected pairs are skipped entirely.  VSA page, "The Fine Stage", same contract with a
// list of block indices; VSA2 page, "Kernel Implementation", padding keys masked out).
//
// sm_100a design.  A query cube has 64 rows but tcgen05 runs at full rate with M = 128, so
// the kernel works transposed: two selected key tiles are stacked into one 128-row operand,
//     S^T[128 keys x 64 queries]  = [K_j0; K_j1] . Q_i^T         (M=128, N=64, K=D)
//     O^T[D x 64 queries]        += [V_j0; V_j1]^T . P^T          (M=D,   N=64, K=128)
// with both accumulators in TMEM.  Persistent CTAs (one per SM) walk the query cubes
// round-robin; the K and V rings, the S^T buffers and the step counters run on across
// cubes, and O^T is double-buffered so that one cube's epilogue overlaps the next cube's
// products.  K tiles live in a 3-stage ring released as soon as their S^T product is
// done, V tiles in a 2-stage ring released after PV, so K loads run well ahead of the MMA.
// Warp roles (320 threads):
//   warp 0      TMA producers: lane 0 loads Q and K tile pairs, lane 1 loads V tile pairs
//   warp 1      TMEM owner and the single MMA-issuing thread
//   warps 2-9   two groups of four warps; group g owns query columns 32g..32g+31 and
//               thread r of a group owns key r of the pair (TMEM lane r).
// Online softmax with lazy rescaling: a group keeps one running maximum per query column
// and recomputes it (a cross-lane reduction and an O^T rescale) only when some score
// exceeds it by more than 2^8; otherwise a step costs one vote and one named barrier.
#include <cmath>

#include "attn_common.cuh"
#include "kernels.h"

namespace sa {

namespace fwd {
constexpr int kThreads = 320;
constexpr float kTau = 8.0f;       // log2 headroom before a running maximum is raised
constexpr float kNegBig = -1e30f;  // finite "minus infinity" for running maxima
constexpr int KST = 3;                 // K ring stages
constexpr int VST = 2;                 // V ring stages
constexpr uint32_t OFF_Q = 0;          // [2 halves][64 rows][128 B]
constexpr uint32_t OFF_K = 16384;      // KST stages x [2 halves][128 rows][128 B]
constexpr uint32_t OFF_V = OFF_K + KST * 32768;  // VST stages, same shape
constexpr uint32_t OFF_P = OFF_V + VST * 32768;  // {hi, lo} x [128 keys][64 queries] bf16
constexpr uint32_t OFF_BAR = OFF_P + 32768;
constexpr uint32_t OFF_SLOT = OFF_BAR + 256;
constexpr uint32_t OFF_FLAG = OFF_BAR + 264;  // [2] per-group abort flags
constexpr uint32_t OFF_VOTE = OFF_BAR + 272;  // [2 step parities][2 groups][4 warps] "new maximum" votes
constexpr uint32_t OFF_RED = OFF_BAR + 512;   // [2][4][32] float
constexpr uint32_t OFF_M = OFF_RED + 1024;    // [2][32] running maxima (log2 units)
constexpr uint32_t OFF_ALPHA = OFF_M + 256;   // [2][32] rescale factors
constexpr uint32_t OFF_L = OFF_ALPHA + 256;   // [2][32] 1/l for the epilogue
constexpr uint32_t SMEM_BYTES = OFF_L + 256 + 1024;
constexpr uint32_t TMEM_COLS = 256;  // S^T[b] at 64b (b = 0,1), O^T[ob] at 128 + 64ob
enum {
  B_QF = 0, B_QE = 1, B_KF = 2, B_KE = 5, B_VF = 8, B_VE = 10, B_SF = 12, B_PF = 14, B_PFREE = 15, B_OR = 16,
  B_OFREE = 18, B_FIN = 20, NBAR = 21
};
}  // namespace fwd

__global__ void __launch_bounds__(fwd::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using namespace fwd;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  volatile int* grp_abort = reinterpret_cast<volatile int*>(smem + OFF_FLAG);
  volatile int* votes = reinterpret_cast<volatile int*>(smem + OFF_VOTE);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);
  float* m_sh = reinterpret_cast<float*>(smem + OFF_M);
  float* alpha_sh = reinterpret_cast<float*>(smem + OFF_ALPHA);
  float* linv_sh = reinterpret_cast<float*>(smem + OFF_L);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const int n_items = a.BH * g.T;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b) {
      uint32_t cnt = 1;
      if (b == B_PF) cnt = 256;
      if (b == B_OFREE || b == B_OFREE + 1) cnt = 8;
      mbar_init(&bars[b], cnt);
    }
    grp_abort[0] = grp_abort[1] = aborted(a.st) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip_all = grp_abort[0] != 0;
  // When the caller keeps the fp32 output (for the backward's Delta), P enters the PV
  // product as bf16 hi + lo so that O is exact to ~2^-16 instead of bf16's 2^-9.
  const bool split_pv = a.out_f32 != nullptr;

  if (warp == 0) {
    // ------------------------------------------------------------------ producers
    if (lane < 2 && !skip_all && !(a.debug & 1u)) {
      const bool kq = lane == 0;  // lane 0: Q and K tiles; lane 1: V tiles
      const CUtensorMap* tmap = kq ? &tm_k : &tm_v;
      uint32_t gs = 0;            // global step counter
      int issued_q = 0;
      bool ok = true;
      for (int it = blockIdx.x, n = 0; ok && it < n_items; it += gridDim.x, ++n) {
        const int bh = it / g.T, i = it % g.T;
        const int cnt = list_count(a, bh, i, kq);
        if (kq) {
          if (n >= 1 && !mbar_wait(&bars[B_QE], (n - 1) & 1, a.st, a.timeout_ns, 11)) break;
          const int row0 = bh * g.Npad + i * 64;
          mbar_arrive_expect_tx(&bars[B_QF], 16384);
          tma_load_2d(smem + OFF_Q, &tm_q, &bars[B_QF], 0, row0);
          tma_load_2d(smem + OFF_Q + 8192, &tm_q, &bars[B_QF], 64, row0);
          ++issued_q;
        }
        const int nsteps = (cnt + 1) >> 1;
        for (int s = 0; s < nsteps; ++s) {
          uint32_t st, full;
          if (kq) {
            st = gs % KST;
            if (gs >= KST && !mbar_wait(&bars[B_KE + st], ((gs / KST) + 1) & 1, a.st, a.timeout_ns, 12)) {
              ok = false;
              break;
            }
            full = B_KF + st;
          } else {
            st = gs % VST;
            if (gs >= VST && !mbar_wait(&bars[B_VE + st], ((gs / VST) + 1) & 1, a.st, a.timeout_ns, 12)) {
              ok = false;
              break;
            }
            full = B_VF + st;
          }
          const int j0 = list_entry(a, bh, i, cnt, 2 * s, kq);
          const int j1 = list_entry(a, bh, i, cnt, 2 * s + 1, kq);
          const int y0 = j0 >= 0 ? bh * g.Npad + j0 * 64 : a.rows_total;
          const int y1 = j1 >= 0 ? bh * g.Npad + j1 * 64 : a.rows_total;
          uint8_t* dst = smem + (kq ? OFF_K : OFF_V) + st * 32768;
          mbar_arrive_expect_tx(&bars[full], 32768);
          tma_load_2d(dst, tmap, &bars[full], 0, y0);
          tma_load_2d(dst + 8192, tmap, &bars[full], 0, y1);
          tma_load_2d(dst + 16384, tmap, &bars[full], 64, y0);
          tma_load_2d(dst + 24576, tmap, &bars[full], 64, y1);
          ++gs;
        }
      }
      // drain: never leave the CTA with copies in flight
      if (kq && issued_q > 0) mbar_wait(&bars[B_QF], (issued_q - 1) & 1, a.st, a.timeout_ns, 13);
      const uint32_t nst = kq ? KST : VST;
      for (uint32_t s = (gs > nst ? gs - nst : 0); s < gs; ++s)
        mbar_wait(&bars[(kq ? B_KF : B_VF) + s % nst], (s / nst) & 1, a.st, a.timeout_ns, 14);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && !skip_all) {
      const uint32_t idesc_s = make_idesc(128, 64, FMT_BF16, false, false);
      const uint32_t idesc_o = make_idesc(128, 64, FMT_BF16, true, true);
      const int ksteps = a.D / 16;
      const int nk_pv = split_pv ? 16 : 8;
      uint32_t gs_s = 0, gs_o = 0;  // global steps whose S (resp. PV) product was issued
      bool ok = true;
      // S^T for the next global step.  Its S buffer (gs_s & 1) was
      // last read by the softmax of step gs_s - 2, whose P_FULL arrival this thread has
      // already waited for before issuing PV(gs_s - 2).
      auto issue_s = [&]() -> bool {
        const uint32_t kst_i = gs_s % KST, sb = gs_s & 1;
        if (!mbar_wait(&bars[B_KF + kst_i], (gs_s / KST) & 1, a.st, a.timeout_ns, 21)) return false;
        tc_fence_after();
        const uint32_t kst = sbase + OFF_K + kst_i * 32768;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t qoff = (ks >> 2) * 8192 + (ks & 3) * 32;
          umma_f16_ss(tmem + sb * 64, sw128_desc(kst + off, 16, 1024), sw128_desc(sbase + OFF_Q + qoff, 16, 1024),
                      idesc_s, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars[B_SF + sb]);
        umma_commit(&bars[B_KE + kst_i]);  // the K stage is free once this product completes
        ++gs_s;
        return true;
      };
      for (int it = blockIdx.x, n = 0; ok && it < n_items; it += gridDim.x, ++n) {
        const int bh = it / g.T, i = it % g.T;
        const int nsteps = (list_count(a, bh, i, false) + 1) >> 1;
        const int ob = n & 1;
        if (!mbar_wait(&bars[B_QF], n & 1, a.st, a.timeout_ns, 22)) break;
        for (int s = 0; ok && s < nsteps && s < 2; ++s) ok = issue_s();
        if (ok && n >= 2 && nsteps > 0)
          ok = mbar_wait(&bars[B_OFREE + ob], ((n >> 1) + 1) & 1, a.st, a.timeout_ns, 23);
        for (int s = 0; ok && s < nsteps; ++s) {
          const uint32_t st = gs_o % VST;
          ok = mbar_wait(&bars[B_PF], gs_o & 1, a.st, a.timeout_ns, 24) &&
               mbar_wait(&bars[B_VF + st], (gs_o / VST) & 1, a.st, a.timeout_ns, 25);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vst = sbase + OFF_V + st * 32768;
#pragma unroll 1
          for (int ks = 0; ks < nk_pv; ++ks) {  // 8 k-steps over P (or P_hi), then 8 over P_lo
            const uint32_t kk = ks & 7, part = ks >> 3;
            umma_f16_ss(tmem + 128 + ob * 64, sw128_desc(vst + kk * 2048, 16384, 1024),
                        sw128_desc(sbase + OFF_P + part * 16384 + kk * 2048, 8192, 1024), idesc_o,
                        (s > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars[B_VE + st]);
          umma_commit(&bars[B_PFREE]);
          ++gs_o;
          if (s + 2 < nsteps) ok = issue_s();
        }
        if (!ok) break;
        umma_commit(&bars[B_QE]);       // every product reading Q has been issued
        umma_commit(&bars[B_OR + ob]);  // O^T of this cube is final once these complete
      }
      // every issued product must complete before TMEM is freed
      umma_commit(&bars[B_FIN]);
      mbar_wait(&bars[B_FIN], 0, a.st, a.timeout_ns, 26);
    }
  } else {
    // ------------------------------------------------------------------ softmax groups
    const int grp = (warp - 2) >> 2;      // 0: query columns 0..31, 1: 32..63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;    // key row of the pair == TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t bar_id = 1 + grp;
    uint32_t gs = 0;  // global step counter
    bool ok = !skip_all;
    for (int it = blockIdx.x, n = 0; ok && it < n_items; it += gridDim.x, ++n) {
      const int bh = it / g.T, i = it % g.T;
      const int cnt = list_count(a, bh, i, false);
      const int nsteps = (cnt + 1) >> 1;
      const int ob = n & 1;
      const int row0 = bh * g.Npad + i * 64;
      float qs = 1.0f;
      if (a.q_scale) qs = a.q_scale[static_cast<size_t>(bh) * g.T + i];
      float m_run[32], l_part[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        m_run[c] = kNegBig;
        l_part[c] = 0.0f;
      }
      for (int s = 0; s < nsteps; ++s, ++gs) {
        const uint32_t b = gs & 1;
        const int tile = list_entry(a, bh, i, cnt, 2 * s + (r >> 6), false);
        const bool kvalid = tile >= 0 && ((a.cube_mask[tile] >> (r & 63)) & 1ull);
        float sc = a.scale_log2 * qs;
        if (a.k_scale && tile >= 0) sc *= a.k_scale[static_cast<size_t>(bh) * g.T + tile];
        if (!mbar_wait(&bars[B_SF + b], (gs >> 1) & 1, a.st, a.timeout_ns, 31)) grp_abort[grp] = 1;
        tc_fence_after();
        float x[32];
        {
          uint32_t raw[32];
          tmem_ld32(t_lane + b * 64 + grp * 32, raw);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = kvalid ? __uint_as_float(raw[c]) * sc : -INFINITY;
        }
        // a column needs a new maximum when one of its keys exceeds the current one by > kTau
        float dmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) dmax = fmaxf(dmax, x[c] - m_run[c]);
        const bool exceed = __any_sync(0xffffffffu, dmax > kTau);
        // double-buffered by step parity: a warp may write the next step's vote while a
        // slower warp of its group still reads this one
        volatile int* vt = votes + (gs & 1) * 8 + grp * 4;
        if (lane == 0) vt[quarter] = exceed ? 1 : 0;
        named_bar_sync(bar_id, 128);
        if (grp_abort[grp]) {
          ok = false;
          break;
        }
        const bool any_exceed = (vt[0] | vt[1] | vt[2] | vt[3]) != 0;
        bool rescale_o = false;
        float alpha[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) alpha[c] = 1.0f;
        if (any_exceed) {
          // exact column maxima over the 128 keys of the pair
          float w[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) w[c] = x[c];
          const int c0 = warp_colreduce32(w, lane, OpMax());
          red[(grp * 4 + quarter) * 32 + c0] = w[0];
          named_bar_sync(bar_id, 128);
          if (quarter == 0) {
            const int c = lane;
            const float mx = fmaxf(fmaxf(red[(grp * 4 + 0) * 32 + c], red[(grp * 4 + 1) * 32 + c]),
                                   fmaxf(red[(grp * 4 + 2) * 32 + c], red[(grp * 4 + 3) * 32 + c]));
            const float mo = (s == 0) ? kNegBig : m_sh[grp * 32 + c];
            const float mn = fmaxf(mo, mx);
            m_sh[grp * 32 + c] = mn;
            alpha_sh[grp * 32 + c] = ex2_approx(mo - mn);
          }
          named_bar_sync(bar_id, 128);
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 mv = *reinterpret_cast<const float4*>(m_sh + grp * 32 + c);
            const float4 av = *reinterpret_cast<const float4*>(alpha_sh + grp * 32 + c);
            m_run[c] = mv.x;
            m_run[c + 1] = mv.y;
            m_run[c + 2] = mv.z;
            m_run[c + 3] = mv.w;
            alpha[c] = av.x;
            alpha[c + 1] = av.y;
            alpha[c + 2] = av.z;
            alpha[c + 3] = av.w;
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            l_part[c] *= alpha[c];
            rescale_o |= alpha[c] != 1.0f;
          }
          rescale_o = rescale_o && s > 0;
        }
        float p[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          p[c] = ex2_approx(x[c] - m_run[c]);
          l_part[c] += p[c];
        }
        // P is single-buffered and O^T may be rescaled: the previous PV product must be done
        if (gs > 0 && !mbar_wait(&bars[B_PFREE], (gs - 1) & 1, a.st, a.timeout_ns, 32)) grp_abort[grp] = 1;
        if (rescale_o) {
          tc_fence_after();
          uint32_t raw[32];
          tmem_ld32(t_lane + 128 + ob * 64 + grp * 32, raw);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) raw[c] = __float_as_uint(__uint_as_float(raw[c]) * alpha[c]);
          tmem_st32(t_lane + 128 + ob * 64 + grp * 32, raw);
          tmem_st_wait();
        }
        if (split_pv)
          store_half_row_bf16x2_sw128(sbase + OFF_P, sbase + OFF_P + 16384, r, grp, p);
        else
          store_half_row_bf16_sw128(sbase + OFF_P, r, grp, p);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[B_PF]);
      }
      if (!ok) break;
      // -------------------------------------------------------------- epilogue
      {
        float w[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) w[c] = l_part[c];
        const int c0 = warp_colreduce32(w, lane, OpSum());
        red[(grp * 4 + quarter) * 32 + c0] = w[0];
      }
      named_bar_sync(bar_id, 128);
      if (quarter == 0) {
        const int c = lane, q = grp * 32 + lane;
        const float l = red[(grp * 4 + 0) * 32 + c] + red[(grp * 4 + 1) * 32 + c] + red[(grp * 4 + 2) * 32 + c] +
                        red[(grp * 4 + 3) * 32 + c];
        const bool qv = (a.cube_mask[i] >> q) & 1ull;
        const bool has = nsteps > 0 && l > 0.0f;
        linv_sh[grp * 32 + c] = (qv && has) ? 1.0f / l : 0.0f;
        float lse = 0.0f;
        if (qv) lse = has ? (m_sh[grp * 32 + c] + log2f(l)) * 0.69314718055994531f : -INFINITY;
        a.lse[row0 + q] = lse;
      }
      named_bar_sync(bar_id, 128);
      float o[32];
      if (nsteps > 0) {
        if (!mbar_wait(&bars[B_OR + ob], (n >> 1) & 1, a.st, a.timeout_ns, 33)) grp_abort[grp] = 1;
        tc_fence_after();
        uint32_t raw[32];
        tmem_ld32(t_lane + 128 + ob * 64 + grp * 32, raw);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(raw[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0.0f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_OFREE + ob]);
      if (r < a.D) {
        __nv_bfloat16* outp = a.out + static_cast<size_t>(row0 + grp * 32) * a.D + r;
        float* outf = a.out_f32 ? a.out_f32 + static_cast<size_t>(row0 + grp * 32) * a.D + r : nullptr;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float val = o[c] * linv_sh[grp * 32 + c];
          outp[static_cast<size_t>(c) * a.D] = __float2bfloat16_rn(val);
          if (outf) outf[static_cast<size_t>(c) * a.D] = val;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// 64-bit mask of the valid token slots of every cube (bit s = slot s holds a real token).
__global__ void cube_mask_kernel(Geom g, unsigned long long* mask) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= g.T) return;
  int vt, vh, vw;
  cube_extent(g, c, vt, vh, vw);
  unsigned long long m = 0;
  for (int s = 0; s < 64; ++s)
    if (slot_valid(vt, vh, vw, s)) m |= 1ull << s;
  mask[c] = m;
}

cudaError_t launch_cube_mask(const Geom& g, unsigned long long* mask, cudaStream_t stream) {
  cube_mask_kernel<<<(g.T + 255) / 256, 256, 0, stream>>>(g, mask);
  return cudaGetLastError();
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

cudaError_t launch_forward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                           cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         fwd::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int items = a.BH * a.g.T;
  const int sms = num_sms();
  const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  attn_fwd_kernel<<<grid, fwd::kThreads, fwd::SMEM_BYTES, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace sa
