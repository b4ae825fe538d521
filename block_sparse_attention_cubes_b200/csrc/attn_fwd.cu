// Fine-stage forward: online-softmax attention of each 64-token query cube over the key
// cubes in its index list (SpargeAttention2 page, "Kernel Implementation of the
// Hybrid-Masked Block-Sparse Attention": per selected block pair, S = Q_i K_j^T / sqrt(d),
// running max and running sum, O rescaled and accumulated, divided by the sum at the end;
// unselected pairs are skipped.  VSA page, "The Fine Stage", same contract with a list of
// block indices; VSA2 page, "Kernel Implementation", padding keys masked out).
//
// sm_100a design.  tcgen05 runs at full rate only with 128-row, >=128-column products, so
// one work item is a pair of adjacent query cubes (128 query rows) walking the union of
// their two KV lists, two key tiles (128 keys) per step:
//     S[128 q x 128 keys]  = Q2 . [K_t0; K_t1]^T        (SS, M=128, N=128, K=D)
//     O_g[128 q x D]      += P_g . V_tg   (g = 0, 1)   (TS: P_g read from TMEM, N=128, K=64)
// P_g overwrites group g's S columns in TMEM (fp16 or bf16 pairs), so it never goes through
// shared memory.  A tile that only one cube of the pair selected is masked for the other
// cube's rows (its products are spent, its exponentials are skipped).  Persistent CTAs take
// the pairs in order from a shared counter.
// Warp roles (320 threads):
//   warp 0      TMA producers: lane 0 loads Q2 and K tile pairs (3-stage ring, released when
//               S is done), lane 1 loads V tile pairs (2-stage ring, released after PV)
//   warp 1      TMEM owner and MMA warp: the whole warp runs the issue loop and one elected
//               lane issues every tcgen05.mma / commit
//   warps 2-9   two groups of 128 threads; thread r of group g owns query row r and the 64
//               key columns of tile t_g, with its own running maximum, sum and accumulator
//               O_g (split-key online softmax), so the groups never wait on each other
//               within a pair; the running maximum is raised (and that row of O_g rescaled in
//               TMEM) only when a score exceeds it by more than 2^15.  At the end of a pair
//               the two partial results of each row are combined once:
//               O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)).
#include <type_traits>
#include <cmath>

#include "attn_common.cuh"
#include "kernels.h"

namespace sa {

namespace fwd {
constexpr int kThreads = 320;
constexpr float kTau = 15.0f;      // log2 headroom before a running maximum is raised (P <= 2^15: fp16 holds it)
constexpr float kNegBig = -1e30f;  // finite "minus infinity" for running maxima
constexpr int KST = 3, VST = 2;    // K and V ring depths
constexpr uint32_t OFF_Q = 0;                    // Q2: [2 halves][128 rows][128 B]
constexpr uint32_t OFF_K = 32768;                // KST x [2 halves][128 keys][128 B]
constexpr uint32_t OFF_V = OFF_K + KST * 32768;  // VST x same
constexpr uint32_t OFF_BAR = OFF_V + VST * 32768;
constexpr uint32_t OFF_SLOT = OFF_BAR + 256;
constexpr uint32_t OFF_ABORT = OFF_BAR + 264;
constexpr uint32_t OFF_RING = OFF_BAR + 272;     // kItemRing item ids
constexpr uint32_t OFF_XMAX = OFF_BAR + 512;     // [2 groups][128 rows] float: running maxima at the item's end
constexpr uint32_t OFF_XL = OFF_XMAX + 1024;     // [2 groups][128 rows] float: partial sums
constexpr uint32_t SMEM_BYTES = OFF_XL + 1024 + 1024;
// S/P[b] at 128b (b = 0,1): group g's 64 key columns at 128b + 64g, its P over them; O_g at 256 + 128g
constexpr uint32_t TMEM_COLS = 512;
// P-full is one barrier per (S buffer, group): the softmax of step s+1 can start before the MMA
// thread has observed P(s) (S(s+1) is issued ahead of PV(s)), so a single barrier per group
// could complete two phases unobserved.  The softmax of step s+2 needs S(s+2), issued only
// after PV(s).  PV-done is one barrier per group (its rescales wait for its previous PV).
enum {
  B_QF = 0, B_QE = 1, B_KF = 2, B_KE = 5, B_VF = 8, B_VE = 10, B_SF = 12, B_PF = 14, B_PFREE = 18, B_OR = 20,
  B_OFREE = 21, B_FIN = 22, B_IF = 23, B_IE = 27, NBAR = 31
};
}  // namespace fwd

// KS = D / 16 k-steps per S product.  Every MMA loop below has a compile-time trip count and
// is unrolled: a single issuing thread running a counted loop spends far more than the
// tensor core's 64 cycles per 128x128x16 product on the loop itself.
// FP8: Q and K are e4m3 bytes (one 128-byte row per token at D = 128) and S comes from a
// kind::f8f6f4 product (K = 32 per instruction, 4 k-steps); the per-cube scales enter in
// the softmax.  V and the PV product stay bf16.
template <int KS, bool FP8>
__global__ void __launch_bounds__(fwd::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_v16,
                    const AttnArgs a) {
  using namespace fwd;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  volatile int* sm_abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  float* xmax = reinterpret_cast<float*>(smem + OFF_XMAX);
  float* xl = reinterpret_cast<float*>(smem + OFF_XL);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const int npairs = (g.T + 1) >> 1;
  const int n_items = a.BH * npairs;
  const int ucap = a.ucap;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b) {
      uint32_t cnt = 1;
      if (b >= B_PF && b < B_PF + 4) cnt = 128;
      if (b == B_OFREE) cnt = 8;
      if (b >= B_IE && b < B_IE + kItemRing) cnt = kRingReaders;
      mbar_init(&bars[b], cnt);
    }
    *sm_abort = aborted(a.st) ? 1 : 0;
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
  const bool skip_all = *sm_abort != 0;
  const ItemRing ring{reinterpret_cast<volatile int*>(smem + OFF_RING), &bars[B_IF], &bars[B_IE]};
  const unsigned long long t_start = (threadIdx.x == 0 && a.cta_clock) ? globaltimer_ns() : 0ull;
  int rec_items = 0;
  uint32_t rec_steps = 0;
  // With the fp32 output kept (for the backward's Delta), P must enter P V to ~2^-11 or better: as one fp16 product against
  // the fp16 copy of V when V fits fp16 (a flag the conversion pass left in device memory, the
  // same for every thread of the launch), else as bf16 hi + lo against V.
  const bool keep32 = a.out_f32 != nullptr;
  const bool use16 = keep32 && a.f16_bad != nullptr && *reinterpret_cast<const volatile unsigned*>(a.f16_bad) == 0u;
  const bool split_pv = keep32 && !use16;

  if (warp == 0) {
    // ------------------------------------------------------------------ producers
    if (lane < 2 && !skip_all) {
      const bool kq = lane == 0;  // lane 0: item ids, Q2 and K tiles; lane 1: V (or its fp16 copy) tiles
      const CUtensorMap* tmap = kq ? &tm_k : (use16 ? &tm_v16 : &tm_v);
      uint32_t gs = 0;
      int issued_q = 0;
      bool ok = true;
      int n = 0;
      for (; ok; ++n) {
        const int it = kq ? ring_publish(ring, n, n_items, a, a.item_next + 0, 15, ok) : ring_read(ring, n, a, 16, ok);
        if (it < 0) break;
        if (a.debug & 1u) break;  // SA_DEBUG_SKIP_LOADS: the item is published, nothing is loaded
        const int bh = it / npairs, pr = it % npairs;
        const int nu = a.u_cnt[it];
        const int32_t* ul = a.u_list + static_cast<size_t>(it) * ucap;
        if (kq) {
          if (n >= 1 && !mbar_wait(&bars[B_QE], (n - 1) & 1, a.st, a.timeout_ns, 11)) break;
          const int r0 = bh * g.Npad + (2 * pr) * 64;
          const int r1 = (2 * pr + 1 < g.T) ? r0 + 64 : a.rows_total;
          mbar_arrive_expect_tx(&bars[B_QF], FP8 ? 16384 : 32768);
          tma_load_2d(smem + OFF_Q, &tm_q, &bars[B_QF], 0, r0);
          tma_load_2d(smem + OFF_Q + 8192, &tm_q, &bars[B_QF], 0, r1);
          if (!FP8) {
            tma_load_2d(smem + OFF_Q + 16384, &tm_q, &bars[B_QF], 64, r0);
            tma_load_2d(smem + OFF_Q + 24576, &tm_q, &bars[B_QF], 64, r1);
          }
          ++issued_q;
        }
        const int nsteps = (nu + 1) >> 1;
        for (int s = 0; s < nsteps; ++s) {
          const uint32_t nst = kq ? KST : VST;
          const uint32_t st = gs % nst;
          if (gs >= nst &&
              !mbar_wait(&bars[(kq ? B_KE : B_VE) + st], ((gs / nst) + 1) & 1, a.st, a.timeout_ns, 12)) {
            ok = false;
            break;
          }
          const int t0 = ul[2 * s] >> 2;
          const int t1 = (2 * s + 1 < nu) ? (ul[2 * s + 1] >> 2) : -1;
          const int y0 = bh * g.Npad + t0 * 64;
          const int y1 = t1 >= 0 ? bh * g.Npad + t1 * 64 : a.rows_total;
          const uint32_t full = (kq ? B_KF : B_VF) + st;
          uint8_t* dst = smem + (kq ? OFF_K : OFF_V) + st * 32768;
          const bool one_box = FP8 && kq;  // an e4m3 K row is a single 128-byte box
          mbar_arrive_expect_tx(&bars[full], one_box ? 16384 : 32768);
          tma_load_2d(dst, tmap, &bars[full], 0, y0);
          tma_load_2d(dst + 8192, tmap, &bars[full], 0, y1);
          if (!one_box) {
            tma_load_2d(dst + 16384, tmap, &bars[full], 64, y0);
            tma_load_2d(dst + 24576, tmap, &bars[full], 64, y1);
          }
          ++gs;
        }
      }
      if (kq) {
        rec_items = n;
        rec_steps = gs;
      }
      // drain: never leave the CTA with copies in flight
      if (kq && issued_q > 0) mbar_wait_drain(&bars[B_QF], (issued_q - 1) & 1, a.st, a.timeout_ns, 13);
      const uint32_t nst = kq ? KST : VST;
      for (uint32_t s = (gs > nst ? gs - nst : 0); s < gs; ++s)
        mbar_wait_drain(&bars[(kq ? B_KF : B_VF) + s % nst], (s / nst) & 1, a.st, a.timeout_ns, 14);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (!skip_all) {
      const uint32_t idesc_s = make_idesc(128, 128, FMT_BF16, false, false);
      const uint32_t idesc_s8 = make_idesc(128, 128, FMT_E4M3, false, false);
      const uint32_t idesc_o = make_idesc(128, 128, use16 ? FMT_F16 : FMT_BF16, false, true);
      uint32_t gs_s = 0, gs_o = 0;
      bool ok = true;
      // S for the next global step into S buffer gs_s & 1.  That buffer last held P of step
      // gs_s - 2, read by PV(gs_s - 2), which this thread issued earlier; the tcgen05.mma
      // operations of one thread execute in issue order.
      auto issue_s = [&]() -> bool {
        const uint32_t kst_i = gs_s % KST, sb = gs_s & 1;
        if (!mbar_wait_warp(&bars[B_KF + kst_i], (gs_s / KST) & 1, a.st, a.timeout_ns, 21)) return false;
        tc_fence_after();
        const uint32_t kst = sbase + OFF_K + kst_i * 32768;
        if (elect_one()) {
          if (FP8) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)  // 32 e4m3 elements = 32 bytes per k-step
              umma_f8_ss(tmem + sb * 128, sw128_desc(sbase + OFF_Q + ks * 32, 16, 1024),
                         sw128_desc(kst + ks * 32, 16, 1024), idesc_s8, ks > 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
              umma_f16_ss(tmem + sb * 128, sw128_desc(sbase + OFF_Q + off, 16, 1024),
                          sw128_desc(kst + off, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
            }
          }
          umma_commit(&bars[B_SF + sb]);
          umma_commit(&bars[B_KE + kst_i]);
        }
        __syncwarp();
        ++gs_s;
        return true;
      };
      for (int n = 0; ok; ++n) {
        const int it = ring_read_warp(ring, n, a, 27, ok);
        if (it < 0) break;
        const int nsteps = (a.u_cnt[it] + 1) >> 1;
        if (!mbar_wait_warp(&bars[B_QF], n & 1, a.st, a.timeout_ns, 22)) break;
        for (int s = 0; ok && s < nsteps && s < 2; ++s) ok = issue_s();
        // O_0 and O_1 of the previous pair must have been read out before this pair's first PV
        if (ok && n >= 1) ok = mbar_wait_warp(&bars[B_OFREE], (n - 1) & 1, a.st, a.timeout_ns, 23);
        for (int s = 0; ok && s < nsteps; ++s) {
          const uint32_t vs = gs_o % VST, pb = gs_o & 1;
          if (!mbar_wait_warp(&bars[B_VF + vs], (gs_o / VST) & 1, a.st, a.timeout_ns, 25)) {
            ok = false;
            break;
          }
          const uint32_t vst = sbase + OFF_V + vs * 32768;
#pragma unroll
          for (int gq = 0; gq < 2; ++gq) {
            // O_g += P_g V_g as soon as group g's P is written: keys 64g.. of the step, K = 64
            if (!mbar_wait_warp(&bars[B_PF + 2 * pb + gq], (gs_o >> 1) & 1, a.st, a.timeout_ns, 24)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t o_acc = tmem + 256 + gq * 128, p_col = tmem + pb * 128 + gq * 64;
            if (elect_one()) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)  // 4 k-steps over P (or P_hi) ...
                umma_f16_ts(o_acc, p_col + kk * 8, sw128_desc(vst + (4 * gq + kk) * 2048, 16384, 1024), idesc_o,
                            (s > 0 || kk > 0) ? 1u : 0u);
              if (split_pv) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // ... then 4 over P_lo
                  umma_f16_ts(o_acc, p_col + 32 + kk * 8, sw128_desc(vst + (4 * gq + kk) * 2048, 16384, 1024),
                              idesc_o, 1u);
              }
              umma_commit(&bars[B_PFREE + gq]);
              if (gq == 1) umma_commit(&bars[B_VE + vs]);
            }
            __syncwarp();
          }
          if (!ok) break;
          ++gs_o;
          if (s + 2 < nsteps) ok = issue_s();
        }
        if (!ok) break;
        if (elect_one()) {
          umma_commit(&bars[B_QE]);  // every product reading Q2 has been issued
          umma_commit(&bars[B_OR]);  // O_0 and O_1 of this pair are final once these complete
        }
        __syncwarp();
      }
      if (elect_one()) umma_commit(&bars[B_FIN]);
      __syncwarp();
      mbar_wait_drain(&bars[B_FIN], 0, a.st, a.timeout_ns, 26);
    }
  } else {
    // ------------------------------------------------------------------ softmax groups
    const int grp = (warp - 2) >> 2;      // key tile t_grp of each step, output columns 64grp..
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;    // query row of the pair == TMEM lane
    const int half = r >> 6;              // which cube of the pair
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t gs = 0;
    bool ok = !skip_all;
    for (int n = 0; ok; ++n) {
      const int it = ring_read_group(ring, n, a, 34, sm_abort, ok);
      if (it < 0) break;
      const int bh = it / npairs, pr = it % npairs;
      const int icube = 2 * pr + half;
      const bool row_exists = icube < g.T;
      const bool row_valid = row_exists && ((a.cube_mask[icube] >> (r & 63)) & 1ull);
      const int nu = a.u_cnt[it];
      const int32_t* ul = a.u_list + static_cast<size_t>(it) * ucap;
      const int nsteps = (nu + 1) >> 1;
      float qs = 1.0f;
      if (a.q_scale && row_exists) qs = a.q_scale[static_cast<size_t>(bh) * g.T + icube];
      float m_run = kNegBig, l_part = 0.0f;
      // this step's and the next step's list entries and key masks are loaded one step ahead
      int e = (grp < nu) ? ul[grp] : 0;
      unsigned long long km = a.cube_mask[e >> 2];
      for (int s = 0; s < nsteps; ++s, ++gs) {
        const uint32_t b = gs & 1;
        const int e_next = (2 * s + 2 + grp < nu) ? ul[2 * s + 2 + grp] : 0;
        const int tile = e >> 2;
        const bool active = ((e >> half) & 1) && row_exists;  // uniform over each warp
        float sc = a.scale_log2 * qs;
        if (a.k_scale && active) sc *= a.k_scale[static_cast<size_t>(bh) * g.T + tile];
        if (!mbar_wait(&bars[B_SF + b], (gs >> 1) & 1, a.st, a.timeout_ns, 31)) *sm_abort = 1;
        tc_fence_after();
        float x[64];
        float pmax = -INFINITY;
        if (active) {
          uint32_t r0[32], r1[32];
          tmem_ld32(t_lane + b * 128 + grp * 64, r0);
          tmem_ld32(t_lane + b * 128 + grp * 64 + 32, r1);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = __uint_as_float(r0[c]);
            x[c + 32] = __uint_as_float(r1[c]);
          }
          if (km != ~0ull) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (!((km >> c) & 1ull)) x[c] = -INFINITY;
          }
          float m8[8];  // eight independent chains of eight
#pragma unroll
          for (int u = 0; u < 8; ++u) m8[u] = x[u];
#pragma unroll
          for (int c = 8; c < 64; ++c) m8[c & 7] = fmaxf(m8[c & 7], x[c]);
          pmax = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * sc;
        }
        // each group keeps its own running maximum, sum and O_g (combined once per pair at the
        // end), so the groups never wait on each other within a pair; P_g overwrites the
        // group's own S columns
        const float rmax = pmax;
        bool rescale = false;
        float alpha = 1.0f;
        if (rmax > m_run + kTau) {
          alpha = ex2_approx(m_run - rmax);
          m_run = rmax;
          l_part *= alpha;
          rescale = s > 0;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          // O_g is read-modified here: the group's previous PV product must have finished
          if (!mbar_wait(&bars[B_PFREE + grp], (gs - 1) & 1, a.st, a.timeout_ns, 32)) *sm_abort = 1;
          tc_fence_after();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {  // the row's 128 accumulator columns, 32 at a time
            uint32_t o0[32];
            const uint32_t oc = t_lane + 256 + grp * 128 + q4 * 32;
            tmem_ld32(oc, o0);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 32; ++c) o0[c] = __float_as_uint(__uint_as_float(o0[c]) * alpha);
            tmem_st32(oc, o0);
          }
          tmem_st_wait();
        }
        // one body per P format, each with its own registers: 0 = bf16, 1 = bf16 hi + lo (the fp32
        // output's P V), 2 = fp16
        auto emit_p = [&](auto mode_tag) {
          constexpr int M = decltype(mode_tag)::value;
          uint32_t ph[32], pl[M == 1 ? 32 : 1];
          if (active) {
            const uint64_t sc2 = pk2(sc, sc), nm2 = pk2(-m_run, -m_run);
            uint64_t l2[4] = {pk2(0.0f, 0.0f), pk2(0.0f, 0.0f), pk2(0.0f, 0.0f), pk2(0.0f, 0.0f)};  // 4 chains
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              float d0, d1;
              upk2(fma2(pk2(x[2 * c], x[2 * c + 1]), sc2, nm2), d0, d1);
              const float p0 = ex2_approx(d0), p1 = ex2_approx(d1);
              const uint64_t pp = pk2(p0, p1);
              l2[c & 3] = add2(l2[c & 3], pp);
              if constexpr (M == 2) {
                ph[c] = pack_f16x2(p0, p1);
              } else {
                ph[c] = pack_bf16x2(p0, p1);
                if constexpr (M == 1) {
                  float r0, r1;
                  upk2(sub2(pp, pk2(__uint_as_float(ph[c] << 16), __uint_as_float(ph[c] & 0xffff0000u))), r0, r1);
                  pl[c] = pack_bf16x2(r0, r1);
                }
              }
            }
            float la, lb;
            upk2(add2(add2(l2[0], l2[1]), add2(l2[2], l2[3])), la, lb);
            l_part += la + lb;
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) ph[c] = 0u;
            if constexpr (M == 1) {
#pragma unroll
              for (int c = 0; c < 32; ++c) pl[c] = 0u;
            }
          }
          tmem_st32(t_lane + b * 128 + grp * 64, ph);
          if constexpr (M == 1) tmem_st32(t_lane + b * 128 + grp * 64 + 32, pl);
        };
        if (use16)
          emit_p(std::integral_constant<int, 2>{});
        else if (split_pv)
          emit_p(std::integral_constant<int, 1>{});
        else
          emit_p(std::integral_constant<int, 0>{});
        e = e_next;
        km = a.cube_mask[e >> 2];
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[B_PF + 2 * b + grp]);
      }
      // -------------------------------------------------------------- epilogue
      // the two groups' partial results of each row: O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / l
      xmax[grp * 128 + r] = m_run;
      xl[grp * 128 + r] = l_part;
      named_bar_sync(1, 256);
      if (*sm_abort) break;
      const float m_oth = xmax[(grp ^ 1) * 128 + r];
      const float m_all = fmaxf(m_run, m_oth);
      const float a_self = ex2_approx(m_run - m_all), a_oth = ex2_approx(m_oth - m_all);
      const float l = l_part * a_self + xl[(grp ^ 1) * 128 + r] * a_oth;
      const bool has = nsteps > 0 && l > 0.0f;
      const float linv = (row_valid && has) ? 1.0f / l : 0.0f;
      const size_t qrow = static_cast<size_t>(bh) * g.Npad + static_cast<size_t>(icube) * 64 + (r & 63);
      if (grp == 0 && row_exists)
        a.lse[qrow] = row_valid ? (has ? (m_all + log2f(l)) * 0.69314718055994531f : -INFINITY) : 0.0f;
      if (!mbar_wait(&bars[B_OR], n & 1, a.st, a.timeout_ns, 33)) *sm_abort = 1;  // every item
      tc_fence_after();
      // output columns 64grp + 32h.. from O_0 (TMEM 256 + 64grp) and O_1 (384 + 64grp), 32 at a time
      const float f0 = (grp == 0 ? a_self : a_oth) * linv, f1 = (grp == 0 ? a_oth : a_self) * linv;
      const bool writes = row_exists && grp * 64 < a.D;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float o[32];
        if (nsteps > 0) {
          uint32_t u0[32], u1[32];
          tmem_ld32(t_lane + 256 + grp * 64 + h * 32, u0);
          tmem_ld32(t_lane + 384 + grp * 64 + h * 32, u1);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = fmaf(__uint_as_float(u0[c]), f0, __uint_as_float(u1[c]) * f1);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0.0f;
        }
        if (h == 1) {  // both accumulators have been read: the next pair's PV may overwrite them
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[B_OFREE]);
        }
        if (writes) {
          const int col = grp * 64 + h * 32;
          if (a.gate && row_valid) {  // the gated combination, with the coarse branch's row of this cube
            const float gv = a.gate[qrow];
            const float4* ocp =
                reinterpret_cast<const float4*>(a.oc + (static_cast<size_t>(bh) * g.T + icube) * a.D + col);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 t = __ldg(ocp + c);
              o[4 * c] = fmaf(gv, t.x, o[4 * c]);
              o[4 * c + 1] = fmaf(gv, t.y, o[4 * c + 1]);
              o[4 * c + 2] = fmaf(gv, t.z, o[4 * c + 2]);
              o[4 * c + 3] = fmaf(gv, t.w, o[4 * c + 3]);
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(a.out + qrow * a.D + col);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            dst[c] = make_uint4(pack_bf16x2(o[8 * c], o[8 * c + 1]), pack_bf16x2(o[8 * c + 2], o[8 * c + 3]),
                                pack_bf16x2(o[8 * c + 4], o[8 * c + 5]), pack_bf16x2(o[8 * c + 6], o[8 * c + 7]));
          if (a.out_f32) {
            float4* df = reinterpret_cast<float4*>(a.out_f32 + qrow * a.D + col);
#pragma unroll
            for (int c = 0; c < 8; ++c) df[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
  if (threadIdx.x == 0) cta_clock_record(a, 0, t_start, rec_items, rec_steps);
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

// bf16 -> fp16 copy of a tensor (n16 = elements / 8 vectors of 16 bytes); any value an fp16
// cannot hold (|x| > 65504, or not finite) sets *bad.  Values below fp16's normal range
// become fp16 subnormals (absolute error at most 2^-25).
// With maxbits set, the largest |x| (fp32 bits, a non-negative float orders as its bits) is
// also recorded there.
__global__ void __launch_bounds__(512) to_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                     long long n16, unsigned int* bad, unsigned int* maxbits) {
  // grid-stride, four 16-byte loads in flight per thread; the range flag and the maximum are
  // reduced over the block, so one atomic per block reaches each status word
  __shared__ float s_mx[16];
  __shared__ int s_out[16];
  bool out = false;
  float mx = 0.0f;
  auto cvt = [&](const uint4 v) -> uint4 {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float a = __uint_as_float(w[u] << 16), b = __uint_as_float(w[u] & 0xffff0000u);
      out |= !(fabsf(a) <= 65504.0f) || !(fabsf(b) <= 65504.0f);
      mx = fmaxf(mx, fmaxf(fabsf(a), fabsf(b)));
      o[u] = pack_f16x2(a, b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  };
  const long long stride = static_cast<long long>(gridDim.x) * 512;
  long long i = static_cast<long long>(blockIdx.x) * 512 + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldcs(src + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) __stcs(dst + i + u * stride, cvt(v[u]));
  }
  for (; i < n16; i += stride) __stcs(dst + i, cvt(__ldcs(src + i)));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const bool wout = __any_sync(0xffffffffu, out);
  if (lane == 0) {
    s_mx[warp] = mx;
    s_out[warp] = wout ? 1 : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
    int o = 0;
    for (int w = 0; w < 16; ++w) {
      m = fmaxf(m, s_mx[w]);
      o |= s_out[w];
    }
    if (o) atomicOr(bad, 1u);
    if (maxbits) atomicMax(maxbits, __float_as_uint(m));
  }
}

cudaError_t launch_to_f16(const void* src, void* dst, long long elems, unsigned int* bad, cudaStream_t stream,
                          unsigned int* maxbits) {
  const long long n16 = elems / 8;
  long long blocks = (n16 + 511) / 512;
  const long long cap = 4LL * num_sms();  // persistent: a few blocks per SM stream the whole tensor
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  to_f16_kernel<<<static_cast<unsigned>(blocks), 512, 0, stream>>>(static_cast<const uint4*>(src),
                                                                   static_cast<uint4*>(dst), n16, bad, maxbits);
  return cudaGetLastError();
}

// The backward's single-product decision: every converted tensor fit fp16, and the bound
// |dS| <= |dP| + |Delta| <= 2 D max|dO| max|V| leaves fp16 (and the forward's P) headroom.
__global__ void f16_decide_kernel(DevStatus* st, int D) {
  const float mdo = __uint_as_float(st->f16_max[0]), mv = __uint_as_float(st->f16_max[1]);
  st->f16_single = (st->f16_out_of_range == 0u && 2.0f * static_cast<float>(D) * mdo * mv <= 32768.0f) ? 1u : 0u;
}

cudaError_t launch_f16_decide(DevStatus* st, int D, cudaStream_t stream) {
  f16_decide_kernel<<<1, 1, 0, stream>>>(st, D);
  return cudaGetLastError();
}

cudaError_t launch_forward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& tv16, const AttnArgs& a, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaSuccess;
    for (auto fn : {attn_fwd_kernel<4, false>, attn_fwd_kernel<8, false>, attn_fwd_kernel<8, true>})
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, fwd::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int items = a.BH * ((a.g.T + 1) >> 1);
  const int sms = num_sms();
  const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  // e4m3 Q/K is built for D = 128 only (the host rejects other head sizes)
  auto fn = a.qk_fp8 ? attn_fwd_kernel<8, true> : (a.D == 64 ? attn_fwd_kernel<4, false> : attn_fwd_kernel<8, false>);
  fn<<<grid, fwd::kThreads, fwd::SMEM_BYTES, stream>>>(tq, tk, tv, tv16, a);
  return cudaGetLastError();
}

}  // namespace sa
