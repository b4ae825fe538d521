// Fine-stage forward: online-softmax attention of one 64-token query cube over the key
// cubes in its index list (SpargeAttention2 page, "Kernel Implementation of the
// Hybrid-Masked Block-Sparse Attention": per selected block pair, S = Q_i K_j^T / sqrt(d),
// running max and running sum, O rescaled and accumulated, divided by the sum at the end;
// unselected pairs are skipped entirely.  VSA page, "The Fine Stage", same contract with a
// list of block indices; VSA2 page, "Kernel Implementation", padding keys masked out).
//
// sm_100a design.  The query cube has 64 rows, but tcgen05 runs at full rate with M = 128,
// so the kernel works transposed: two selected key tiles are stacked into one 128-row
// operand and
//     S^T[128 keys x 64 queries]  = [K_j0; K_j1] . Q_i^T         (M=128, N=64, K=D)
//     O^T[D x 64 queries]        += [V_j0; V_j1]^T . P^T          (M=D,   N=64, K=128)
// with both accumulators in TMEM.  One CTA per (batch*head, query cube):
//   warp 0      TMA producer (Q once, then K/V tile pairs, 2-stage ring)
//   warp 1      TMEM allocation and the single MMA-issuing thread
//   warps 2-5   softmax group: thread r owns key r of the pair (TMEM lane r) and holds
//               its 64 scores; column (query) maxima and sums are reduced across the
//               group, P^T goes to shared memory as the MN-major B operand, O^T is
//               rescaled in TMEM when a running maximum grows, and the epilogue
//               normalises O^T and writes O and lse.
#include <cmath>

#include "attn_common.cuh"
#include "kernels.h"

namespace sa {

namespace fwd {
constexpr int kThreads = 192;
constexpr uint32_t OFF_Q = 0;            // 2 halves x [64 rows][128 B]
constexpr uint32_t OFF_K = 16384;        // 2 stages x 2 halves x [128 rows][128 B]
constexpr uint32_t OFF_V = 81920;        // same
constexpr uint32_t OFF_P = 147456;       // 2 buffers x {hi, lo} x [128 keys][64 queries] bf16
constexpr uint32_t OFF_BAR = 212992;
constexpr uint32_t OFF_SLOT = OFF_BAR + 128;
constexpr uint32_t OFF_FLAG = OFF_BAR + 136;
constexpr uint32_t OFF_RED = OFF_BAR + 256;  // [4][64] float
constexpr uint32_t OFF_M = OFF_RED + 1024;   // [64] running max (log2 units)
constexpr uint32_t OFF_ALPHA = OFF_M + 256;  // [64] rescale factors
constexpr uint32_t OFF_L = OFF_ALPHA + 256;  // [64] final sums
constexpr uint32_t SMEM_BYTES = OFF_L + 256 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 256;          // S^T x2 (cols 0, 64), O^T (col 128)
enum { B_Q = 0, B_KF = 1, B_VF = 3, B_EMPTY = 5, B_SF = 7, B_PF = 9, B_OD = 11, B_FIN = 12, NBAR = 13 };
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
  float* red = reinterpret_cast<float*>(smem + OFF_RED);
  float* m_sh = reinterpret_cast<float*>(smem + OFF_M);
  float* alpha_sh = reinterpret_cast<float*>(smem + OFF_ALPHA);
  float* l_sh = reinterpret_cast<float*>(smem + OFF_L);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x % a.g.T;
  const int bh = blockIdx.x / a.g.T;
  const Geom& g = a.g;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b) mbar_init(&bars[b], (b == B_PF || b == B_PF + 1) ? 128u : 1u);
    *grp_abort = aborted(a.st) ? 1 : 0;
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
  const bool skip_all = *grp_abort != 0;
  const int n = list_count(a, bh, i, threadIdx.x == 0);
  const int nsteps = skip_all ? 0 : (n + 1) >> 1;
  const int row0 = bh * g.Npad + i * 64;
  // When the caller keeps the fp32 output (for the backward's Delta), P enters the PV
  // product as bf16 hi + lo so that O is exact to ~2^-16 instead of bf16's 2^-9.
  const bool split_pv = a.out_f32 != nullptr;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0 && nsteps > 0 && !(a.debug & 1u)) {
      mbar_arrive_expect_tx(&bars[B_Q], 16384);
      tma_load_2d(smem + OFF_Q, &tm_q, &bars[B_Q], 0, row0);
      tma_load_2d(smem + OFF_Q + 8192, &tm_q, &bars[B_Q], 64, row0);
      int issued = 0;
      for (int s = 0; s < nsteps; ++s) {
        const int st = s & 1;
        if (s >= 2 && !mbar_wait(&bars[B_EMPTY + st], ((s >> 1) + 1) & 1, a.st, a.timeout_ns, 11)) break;
        const int j0 = list_entry(a, bh, i, n, 2 * s, true);
        const int j1 = list_entry(a, bh, i, n, 2 * s + 1, true);
        const int y0 = j0 >= 0 ? bh * g.Npad + j0 * 64 : a.rows_total;
        const int y1 = j1 >= 0 ? bh * g.Npad + j1 * 64 : a.rows_total;
        uint8_t* kst = smem + OFF_K + st * 32768;
        uint8_t* vst = smem + OFF_V + st * 32768;
        mbar_arrive_expect_tx(&bars[B_KF + st], 32768);
        tma_load_2d(kst, &tm_k, &bars[B_KF + st], 0, y0);
        tma_load_2d(kst + 8192, &tm_k, &bars[B_KF + st], 0, y1);
        tma_load_2d(kst + 16384, &tm_k, &bars[B_KF + st], 64, y0);
        tma_load_2d(kst + 24576, &tm_k, &bars[B_KF + st], 64, y1);
        mbar_arrive_expect_tx(&bars[B_VF + st], 32768);
        tma_load_2d(vst, &tm_v, &bars[B_VF + st], 0, y0);
        tma_load_2d(vst + 8192, &tm_v, &bars[B_VF + st], 0, y1);
        tma_load_2d(vst + 16384, &tm_v, &bars[B_VF + st], 64, y0);
        tma_load_2d(vst + 24576, &tm_v, &bars[B_VF + st], 64, y1);
        ++issued;
      }
      // drain: never leave the CTA with copies in flight
      mbar_wait(&bars[B_Q], 0, a.st, a.timeout_ns, 12);
      for (int s = (issued > 2 ? issued - 2 : 0); s < issued; ++s) {
        mbar_wait(&bars[B_KF + (s & 1)], (s >> 1) & 1, a.st, a.timeout_ns, 13);
        mbar_wait(&bars[B_VF + (s & 1)], (s >> 1) & 1, a.st, a.timeout_ns, 14);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && nsteps > 0) {
      const uint32_t idesc_s = make_idesc(128, 64, FMT_BF16, false, false);
      const uint32_t idesc_o = make_idesc(128, 64, FMT_BF16, true, true);
      const int ksteps = a.D / 16;
      const int nk_pv = split_pv ? 16 : 8;
      auto issue_s = [&](int s) {
        const uint32_t kst = sbase + OFF_K + (s & 1) * 32768;
        const uint32_t d_tmem = tmem + (s & 1) * 64;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t qoff = (ks >> 2) * 8192 + (ks & 3) * 32;
          umma_f16_ss(d_tmem, sw128_desc(kst + off, 16, 1024), sw128_desc(sbase + OFF_Q + qoff, 16, 1024),
                      idesc_s, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars[B_SF + (s & 1)]);
      };
      bool ok = mbar_wait(&bars[B_Q], 0, a.st, a.timeout_ns, 21);
      for (int s = 0; ok && s < 2 && s < nsteps; ++s) {
        ok = mbar_wait(&bars[B_KF + s], 0, a.st, a.timeout_ns, 22);
        if (ok) {
          tc_fence_after();
          issue_s(s);
        }
      }
      for (int s = 0; ok && s < nsteps; ++s) {
        const int st = s & 1;
        ok = mbar_wait(&bars[B_PF + st], (s >> 1) & 1, a.st, a.timeout_ns, 23) &&
             mbar_wait(&bars[B_VF + st], (s >> 1) & 1, a.st, a.timeout_ns, 24);
        if (!ok) break;
        tc_fence_after();
        const uint32_t vst = sbase + OFF_V + st * 32768;
        const uint32_t pb = sbase + OFF_P + st * 32768;
#pragma unroll 1
        for (int ks = 0; ks < nk_pv; ++ks) {  // 8 k-steps over P (or P_hi), then 8 over P_lo
          const uint32_t kk = ks & 7, part = ks >> 3;
          umma_f16_ss(tmem + 128, sw128_desc(vst + kk * 2048, 16384, 1024),
                      sw128_desc(pb + part * 16384 + kk * 2048, 8192, 1024), idesc_o, (s > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&bars[B_EMPTY + st]);
        umma_commit(&bars[B_OD]);
        if (s + 2 < nsteps) {
          ok = mbar_wait(&bars[B_KF + st], ((s + 2) >> 1) & 1, a.st, a.timeout_ns, 25);
          if (!ok) break;
          tc_fence_after();
          issue_s(s + 2);
        }
      }
      umma_commit(&bars[B_FIN]);
      mbar_wait(&bars[B_FIN], 0, a.st, a.timeout_ns, 26);
    }
  } else {
    // ------------------------------------------------------------------ softmax group
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row of the pair == TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float l_part[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) l_part[c] = 0.0f;
    if (r < 64) m_sh[r] = -INFINITY;
    named_bar_sync(1, 128);
    float qs = 1.0f;
    if (a.q_scale) qs = a.q_scale[static_cast<size_t>(bh) * g.T + i];
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      const int b = s & 1;
      if (!mbar_wait(&bars[B_SF + b], (s >> 1) & 1, a.st, a.timeout_ns, 31)) *grp_abort = 1;
      tc_fence_after();
      float v[64];
      tmem_ld64(t_lane + b * 64, v);
      const int tile = list_entry(a, bh, i, n, 2 * s + (r >> 6), false);
      const bool valid = tile >= 0 && token_valid(g, tile, r & 63);
      float sc = a.scale_log2 * qs;
      if (a.k_scale && tile >= 0) sc *= a.k_scale[static_cast<size_t>(bh) * g.T + tile];
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = valid ? v[c] * sc : -INFINITY;
      float w[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) w[c] = v[c];
      const int c0 = warp_colreduce64(w, lane, OpMax());
      red[quarter * 64 + c0] = w[0];
      red[quarter * 64 + c0 + 1] = w[1];
      named_bar_sync(1, 128);
      if (r < 64) {
        const float mx = fmaxf(fmaxf(red[r], red[64 + r]), fmaxf(red[128 + r], red[192 + r]));
        const float mo = m_sh[r];
        const float mn = fmaxf(mo, mx);
        alpha_sh[r] = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
        m_sh[r] = mn;
      }
      named_bar_sync(1, 128);
      if (*grp_abort) {
        ok = false;
        break;
      }
      bool rescale = false;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float al = alpha_sh[c];
        const float mc = m_sh[c];
        const float p = (mc == -INFINITY) ? 0.0f : exp2f(v[c] - mc);
        l_part[c] = l_part[c] * al + p;
        v[c] = p;
        rescale |= (al != 1.0f);
      }
      if (s >= 1 && !mbar_wait(&bars[B_OD], (s - 1) & 1, a.st, a.timeout_ns, 32)) *grp_abort = 1;
      if (split_pv)
        store_row_bf16x2_sw128(sbase + OFF_P + b * 32768, sbase + OFF_P + b * 32768 + 16384, r, v);
      else
        store_row_bf16_sw128(sbase + OFF_P + b * 32768, r, v);
      if (rescale && s >= 1) {
        tc_fence_after();
        float o[64];
        tmem_ld64(t_lane + 128, o);
#pragma unroll
        for (int c = 0; c < 64; ++c) o[c] *= alpha_sh[c];
        tmem_st64(t_lane + 128, o);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_PF + b]);
    }
    if (ok && nsteps > 0 && !mbar_wait(&bars[B_OD], (nsteps - 1) & 1, a.st, a.timeout_ns, 33)) ok = false;
    // final column sums of the running denominators
    const int c0 = warp_colreduce64(l_part, lane, OpSum());
    red[quarter * 64 + c0] = l_part[0];
    red[quarter * 64 + c0 + 1] = l_part[1];
    named_bar_sync(1, 128);
    if (r < 64) l_sh[r] = red[r] + red[64 + r] + red[128 + r] + red[192 + r];
    named_bar_sync(1, 128);
    // epilogue: thread r holds row d = r of O^T
    tc_fence_after();
    float o[64];
    if (nsteps > 0) {
      tmem_ld64(t_lane + 128, o);
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) o[c] = 0.0f;
    }
    if (r < a.D) {
      __nv_bfloat16* outp = a.out + static_cast<size_t>(row0) * a.D + r;
      float* outf = a.out_f32 ? a.out_f32 + static_cast<size_t>(row0) * a.D + r : nullptr;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float l = l_sh[c];
        const bool qv = token_valid(g, i, c);
        const float val = (qv && ok && nsteps > 0 && l > 0.0f) ? o[c] / l : 0.0f;
        outp[static_cast<size_t>(c) * a.D] = __float2bfloat16_rn(val);
        if (outf) outf[static_cast<size_t>(c) * a.D] = val;
      }
    }
    if (r < 64) {
      const bool qv = token_valid(g, i, r);
      const float l = l_sh[r];
      float lse = 0.0f;
      if (qv) lse = (nsteps > 0 && l > 0.0f) ? (m_sh[r] + log2f(l)) * 0.69314718055994531f : -INFINITY;
      a.lse[row0 + r] = lse;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
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
  const unsigned grid = static_cast<unsigned>(a.BH) * a.g.T;
  attn_fwd_kernel<<<grid, fwd::kThreads, fwd::SMEM_BYTES, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace sa
