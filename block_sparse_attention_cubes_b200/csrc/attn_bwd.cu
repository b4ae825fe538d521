// Fine-stage backward with the block mask held constant (VSA2 page, section 2.1: the
// router's output carries no gradient; SpargeAttention2 page, "Why this implementation is
// trainable": gradients flow only through the un-masked computations).  With
// S = scale * Q K^T + M, P = softmax(S) recomputed from lse,
//     dV = P^T dO,  dP = dO V^T,  Delta = rowsum(dO * O),  dS = P * (dP - Delta),
//     dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Kernels:
//   delta_kernel      Delta and -lse * log2(e) per query row (one warp per row).
//   pair unions       (pairs.cu) query-cube pairs over their KV lists; key-cube pairs over
//                     the transposed selection, read from a bit matrix that the lists are
//                     scattered into with atomicOr (deterministic, ascending query cubes).
//   attn_dq_kernel    row form over query-cube pairs (M = 128 rows, N = 128 keys).
//   attn_dkdv_kernel  transposed form over key-cube pairs (M = 128 keys, N = 128 queries).
// All products are full-rate 128 x 128 tcgen05 MMAs with accumulators in TMEM; P and dS
// enter the dV, dK and dQ products as bf16 hi + lo pairs read from TMEM.
#include <cmath>
#include <type_traits>

#include "attn_common.cuh"
#include "kernels.h"

namespace sa {

// ------------------------------------------------------------------------ Delta
// O is read from its fp32 copy when there is one, else from the bf16 output.  The same pass
// writes -lse * log2(e) per row, the form in which the dK/dV kernel's exponentials use it.
// One warp per 4 consecutive rows, all loads issued before any arithmetic (padding rows are
// read too and zeroed afterwards), so each warp keeps 4 rows of O and dO in flight.
constexpr int DELTA_ROWS = 4;
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                    const float* __restrict__ o32,
                                                    const __nv_bfloat16* __restrict__ dout,
                                                    const float* __restrict__ lse, float* __restrict__ delta,
                                                    float* __restrict__ nlse2, Geom g, int BH, int D) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(BH) * g.Npad;
  const long long row0 = (blockIdx.x * 8LL + warp) * DELTA_ROWS;
  if (row0 >= rows) return;
  // D is 64 or 128: lane c holds elements 4c..4c+3 of a row (lanes >= D/4 idle)
  const int c = lane;
  const bool on = c < D / 4;
  uint2 y[DELTA_ROWS];
  float4 x[DELTA_ROWS];
#pragma unroll
  for (int u = 0; u < DELTA_ROWS; ++u) {
    const long long row = row0 + u;
    y[u] = make_uint2(0u, 0u);
    x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (on && row < rows) {
      y[u] = reinterpret_cast<const uint2*>(dout + row * D)[c];
      if (o32) {
        x[u] = reinterpret_cast<const float4*>(o32 + row * D)[c];
      } else {
        const uint2 b = reinterpret_cast<const uint2*>(o + row * D)[c];
        x[u] = make_float4(__uint_as_float(b.x << 16), __uint_as_float(b.x & 0xffff0000u),
                           __uint_as_float(b.y << 16), __uint_as_float(b.y & 0xffff0000u));
      }
    }
  }
  float acc[DELTA_ROWS];
#pragma unroll
  for (int u = 0; u < DELTA_ROWS; ++u) {
    acc[u] = x[u].x * __uint_as_float(y[u].x << 16);
    acc[u] += x[u].y * __uint_as_float(y[u].x & 0xffff0000u);
    acc[u] += x[u].z * __uint_as_float(y[u].y << 16);
    acc[u] += x[u].w * __uint_as_float(y[u].y & 0xffff0000u);
  }
#pragma unroll
  for (int u = 0; u < DELTA_ROWS; ++u) {
#pragma unroll
    for (int off = 16; off; off >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
  }
  if (lane < DELTA_ROWS) {
    float a = acc[0];
#pragma unroll
    for (int u = 1; u < DELTA_ROWS; ++u)
      if (lane == u) a = acc[u];
    const long long row = row0 + lane;
    if (row < rows) {
      const int p = static_cast<int>(row % g.Npad);
      delta[row] = token_valid(g, p >> 6, p & 63) ? a : 0.0f;
      nlse2[row] = -lse[row] * 1.4426950408889634f;
    }
  }
}

// ------------------------------------------------------------------------ dQ
// One item = two adjacent query cubes (128 rows) over the union of their KV lists, two key
// tiles per step:  S = Q2 K2^T,  dP = dO2 V2^T  (SS, N=128),  P = exp(S*scale - lse),
// dS = P (dP - Delta) written as bf16 hi + lo into this step's S columns of TMEM, and
// dQ += dS K2 as a TS product (N = D).  Thread r of group g owns row r and the 64 keys of
// tile t_g, and writes its dS over its own S columns, so the groups never wait on each
// other.  S is double-buffered; dQ(s) overlaps the elementwise work of step s + 1.
namespace dqk {
constexpr int kThreads = 320;
constexpr int KST = 3, VST = 2;
constexpr uint32_t OFF_Q = 0;       // Q2  [2 halves][128 rows][128 B]
constexpr uint32_t OFF_DO = 32768;  // dO2 same
constexpr uint32_t OFF_K = 65536;   // KST x [2 halves][128 keys][128 B]
constexpr uint32_t OFF_V = OFF_K + KST * 32768;
constexpr uint32_t OFF_BAR = OFF_V + VST * 32768;
constexpr uint32_t OFF_SLOT = OFF_BAR + 256;
constexpr uint32_t OFF_ABORT = OFF_BAR + 264;
constexpr uint32_t OFF_RING = OFF_BAR + 272;  // kItemRing item ids
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;
constexpr uint32_t TMEM_COLS = 512;  // S/dS[b] at 128b, dP at 256, dQ at 384
enum {
  B_QF = 0, B_QE = 1, B_KF = 2, B_KE = 5, B_VF = 8, B_VE = 10, B_SF = 12, B_DPF = 14, B_PF = 15, B_DQR = 16,
  B_DQFREE = 17, B_FIN = 18, B_IF = 19, B_IE = 23, NBAR = 27
};
}  // namespace dqk

template <int KS>  // D / 16; MMA loops unrolled (a counted loop costs more than the MMA)
__global__ void __launch_bounds__(dqk::kThreads, 1)
    attn_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_q16, const __grid_constant__ CUtensorMap tm_k16,
                   const AttnArgs a, const CoarseAdd add) {
  using namespace dqk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  volatile int* sm_abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const int npairs = (g.T + 1) >> 1;
  const int n_items = a.BH * npairs;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b)
      mbar_init(&bars[b], b == B_PF ? 256u : (b == B_DQFREE ? 8u : ((b >= B_IE && b < B_IE + kItemRing) ? kRingReaders : 1u)));
    *sm_abort = aborted(a.st) ? 1 : 0;
    fence_barrier_init();
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
  // fp16 single products (Q and K from their fp16 copies, dS as one fp16 value) when the
  // conversion pass found every operand and the dS bound within fp16; else bf16, dS as hi + lo
  const bool use16 = a.f16_single != nullptr && *reinterpret_cast<const volatile unsigned*>(a.f16_single) == 1u;
  const CUtensorMap* mq = use16 ? &tm_q16 : &tm_q;

  if (warp == 0) {
    if (lane < 2 && !skip_all) {
      const bool kq = lane == 0;  // lane 0: item ids, Q2, dO2 and K tiles; lane 1: V tiles
      const CUtensorMap* tmap = kq ? (use16 ? &tm_k16 : &tm_k) : &tm_v;
      uint32_t gs = 0;
      int issued_q = 0;
      bool ok = true;
      int n = 0;
      for (; ok; ++n) {
        const int it = kq ? ring_publish(ring, n, n_items, a, a.item_next + 1, 45, ok) : ring_read(ring, n, a, 46, ok);
        if (it < 0) break;
        const int bh = it / npairs, pr = it % npairs;
        const int nu = a.u_cnt[it];
        const int32_t* ul = a.u_list + static_cast<size_t>(it) * a.ucap;
        if (kq) {
          if (n >= 1 && !mbar_wait(&bars[B_QE], (n - 1) & 1, a.st, a.timeout_ns, 41)) break;
          const int r0 = bh * g.Npad + (2 * pr) * 64;
          const int r1 = (2 * pr + 1 < g.T) ? r0 + 64 : a.rows_total;
          mbar_arrive_expect_tx(&bars[B_QF], 65536);
          tma_load_2d(smem + OFF_Q, mq, &bars[B_QF], 0, r0);
          tma_load_2d(smem + OFF_Q + 8192, mq, &bars[B_QF], 0, r1);
          tma_load_2d(smem + OFF_Q + 16384, mq, &bars[B_QF], 64, r0);
          tma_load_2d(smem + OFF_Q + 24576, mq, &bars[B_QF], 64, r1);
          tma_load_2d(smem + OFF_DO, &tm_do, &bars[B_QF], 0, r0);
          tma_load_2d(smem + OFF_DO + 8192, &tm_do, &bars[B_QF], 0, r1);
          tma_load_2d(smem + OFF_DO + 16384, &tm_do, &bars[B_QF], 64, r0);
          tma_load_2d(smem + OFF_DO + 24576, &tm_do, &bars[B_QF], 64, r1);
          ++issued_q;
        }
        const int nsteps = (nu + 1) >> 1;
        for (int s = 0; s < nsteps; ++s) {
          const uint32_t nst = kq ? KST : VST;
          const uint32_t st = gs % nst;
          if (gs >= nst &&
              !mbar_wait(&bars[(kq ? B_KE : B_VE) + st], ((gs / nst) + 1) & 1, a.st, a.timeout_ns, 42)) {
            ok = false;
            break;
          }
          const int t0 = ul[2 * s] >> 2;
          const int t1 = (2 * s + 1 < nu) ? (ul[2 * s + 1] >> 2) : -1;
          const int y0 = bh * g.Npad + t0 * 64;
          const int y1 = t1 >= 0 ? bh * g.Npad + t1 * 64 : a.rows_total;
          const uint32_t full = (kq ? B_KF : B_VF) + st;
          uint8_t* dst = smem + (kq ? OFF_K : OFF_V) + st * 32768;
          mbar_arrive_expect_tx(&bars[full], 32768);
          tma_load_2d(dst, tmap, &bars[full], 0, y0);
          tma_load_2d(dst + 8192, tmap, &bars[full], 0, y1);
          tma_load_2d(dst + 16384, tmap, &bars[full], 64, y0);
          tma_load_2d(dst + 24576, tmap, &bars[full], 64, y1);
          ++gs;
        }
      }
      if (kq) {
        rec_items = n;
        rec_steps = gs;
      }
      if (kq && issued_q > 0) mbar_wait_drain(&bars[B_QF], (issued_q - 1) & 1, a.st, a.timeout_ns, 43);
      const uint32_t nst = kq ? KST : VST;
      for (uint32_t s = (gs > nst ? gs - nst : 0); s < gs; ++s)
        mbar_wait_drain(&bars[(kq ? B_KF : B_VF) + s % nst], (s / nst) & 1, a.st, a.timeout_ns, 44);
    }
  } else if (warp == 1) {
    // the whole warp runs the loop; one elected lane issues (see elect_one)
    if (!skip_all) {
      const uint32_t idesc_kk = make_idesc(128, 128, FMT_BF16, false, false);  // dP: bf16 dO, V
      const uint32_t idesc_s = make_idesc(128, 128, use16 ? FMT_F16 : FMT_BF16, false, false);
      const uint32_t idesc_q = make_idesc(128, 128, use16 ? FMT_F16 : FMT_BF16, false, true);
      uint32_t gs_s = 0, gs_p = 0, gs_q = 0;  // global steps whose S, dP, dQ products were issued
      bool ok = true;
      auto issue_s = [&]() -> bool {
        const uint32_t ks_i = gs_s % KST, sb = gs_s & 1;
        if (!mbar_wait_warp(&bars[B_KF + ks_i], (gs_s / KST) & 1, a.st, a.timeout_ns, 51)) return false;
        tc_fence_after();
        const uint32_t kst = sbase + OFF_K + ks_i * 32768;
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
            umma_f16_ss(tmem + sb * 128, sw128_desc(sbase + OFF_Q + off, 16, 1024), sw128_desc(kst + off, 16, 1024),
                        idesc_s, ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars[B_SF + sb]);
        }
        __syncwarp();
        ++gs_s;
        return true;
      };
      auto issue_dp = [&]() -> bool {
        const uint32_t vs = gs_p % VST;
        if (!mbar_wait_warp(&bars[B_VF + vs], (gs_p / VST) & 1, a.st, a.timeout_ns, 52)) return false;
        tc_fence_after();
        const uint32_t vst = sbase + OFF_V + vs * 32768;
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
            umma_f16_ss(tmem + 256, sw128_desc(sbase + OFF_DO + off, 16, 1024), sw128_desc(vst + off, 16, 1024),
                        idesc_kk, ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars[B_DPF]);
          umma_commit(&bars[B_VE + vs]);
        }
        __syncwarp();
        ++gs_p;
        return true;
      };
      for (int n = 0; ok; ++n) {
        const int it = ring_read_warp(ring, n, a, 57, ok);
        if (it < 0) break;
        const int nsteps = (a.u_cnt[it] + 1) >> 1;
        if (!mbar_wait_warp(&bars[B_QF], n & 1, a.st, a.timeout_ns, 53)) break;
        if (nsteps > 0) ok = issue_s() && issue_dp();
        // dQ of the previous item must have been read out before this item's dQ (or, for an
        // empty item, its ready signal): one phase of DQR / DQFREE per item, never two unobserved
        if (ok && n >= 1) ok = mbar_wait_warp(&bars[B_DQFREE], (n - 1) & 1, a.st, a.timeout_ns, 54);
        for (int s = 0; ok && s < nsteps; ++s) {
          // S(s+1) goes to the other S buffer, whose dS(s-1) was read by the earlier dQ(s-1)
          if (s + 1 < nsteps) ok = issue_s();
          if (!ok || !mbar_wait_warp(&bars[B_PF], gs_q & 1, a.st, a.timeout_ns, 55)) {
            ok = false;
            break;
          }
          // dP(s) has been read: its buffer takes dP(s+1), issued ahead of dQ(s)
          if (s + 1 < nsteps && !issue_dp()) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ks_i = gs_q % KST, sb = gs_q & 1;
          const uint32_t kst = sbase + OFF_K + ks_i * 32768;
          if (elect_one()) {
            if (use16) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {  // 8 k-steps over dS (fp16)
                const uint32_t acol = sb * 128 + (kk >> 2) * 64 + (kk & 3) * 8;
                umma_f16_ts(tmem + 384, tmem + acol, sw128_desc(kst + kk * 2048, 16384, 1024), idesc_q,
                            (s > 0 || kk > 0) ? 1u : 0u);
              }
            } else {
#pragma unroll
              for (int ks = 0; ks < 16; ++ks) {  // 8 k-steps over dS_hi, then 8 over dS_lo
                const uint32_t kk = ks & 7, part = ks >> 3;
                const uint32_t acol = sb * 128 + (kk >> 2) * 64 + part * 32 + (kk & 3) * 8;
                umma_f16_ts(tmem + 384, tmem + acol, sw128_desc(kst + kk * 2048, 16384, 1024), idesc_q,
                            (s > 0 || ks > 0) ? 1u : 0u);
              }
            }
            umma_commit(&bars[B_KE + ks_i]);  // K(s) was read by S(s) and dQ(s)
          }
          __syncwarp();
          ++gs_q;
        }
        if (!ok) break;
        if (elect_one()) {
          umma_commit(&bars[B_QE]);
          umma_commit(&bars[B_DQR]);
        }
        __syncwarp();
      }
      if (elect_one()) umma_commit(&bars[B_FIN]);
      __syncwarp();
      mbar_wait_drain(&bars[B_FIN], 0, a.st, a.timeout_ns, 56);
    }
  } else {
    const int grp = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int half = r >> 6;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t gs = 0;
    bool ok = !skip_all;
    for (int n = 0; ok; ++n) {
      const int it = ring_read_group(ring, n, a, 64, sm_abort, ok);
      if (it < 0) break;
      const int bh = it / npairs, pr = it % npairs;
      const int icube = 2 * pr + half;
      const bool row_exists = icube < g.T;
      const bool row_valid = row_exists && ((a.cube_mask[icube] >> (r & 63)) & 1ull);
      const size_t qrow = static_cast<size_t>(bh) * g.Npad + static_cast<size_t>(icube) * 64 + (r & 63);
      const float lse2 = row_valid ? a.lse[qrow] * 1.4426950408889634f : 0.0f;
      const float dlt = row_valid ? a.delta[qrow] : 0.0f;
      const int nu = a.u_cnt[it];
      const int32_t* ul = a.u_list + static_cast<size_t>(it) * a.ucap;
      const int nsteps = (nu + 1) >> 1;
      int e = (grp < nu) ? ul[grp] : 0;
      unsigned long long km_cur = a.cube_mask[e >> 2];
      for (int s = 0; s < nsteps; ++s, ++gs) {
        const uint32_t b = gs & 1;
        const int e_next = (2 * s + 2 + grp < nu) ? ul[2 * s + 2 + grp] : 0;
        const bool active = ((e >> half) & 1) && row_valid;
        const bool w_active = __any_sync(0xffffffffu, active);
        // P = exp(S * scale - lse) first: the exponentials overlap the dP product of this step,
        // which the MMA warp issues only once both groups have read the previous dP
        if (!mbar_wait(&bars[B_SF + b], (gs >> 1) & 1, a.st, a.timeout_ns, 61)) *sm_abort = 1;
        tc_fence_after();
        float pe[64];
        if (w_active) {
          uint32_t s0[32], s1[32];
          tmem_ld32(t_lane + b * 128 + grp * 64, s0);
          tmem_ld32(t_lane + b * 128 + grp * 64 + 32, s1);
          tmem_ld_wait();
          // the key mask is first used here, so its load (issued a step earlier) hides behind the waits
          const unsigned long long km = active ? km_cur : 0ull;
          const uint64_t sc2 = pk2(a.scale_log2, a.scale_log2), nl2 = pk2(-lse2, -lse2);
          const bool full = km == ~0ull;  // uniform over the warp
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int c0 = 2 * c, c1 = 2 * c + 1;
            const uint32_t sa0 = c0 < 32 ? s0[c0] : s1[c0 - 32], sa1 = c1 < 32 ? s0[c1] : s1[c1 - 32];
            float x0, x1;
            upk2(fma2(pk2(__uint_as_float(sa0), __uint_as_float(sa1)), sc2, nl2), x0, x1);
            pe[c0] = ex2_approx(x0);
            pe[c1] = ex2_approx(x1);
            if (!full) {
              if (!((km >> c0) & 1ull)) pe[c0] = 0.0f;
              if (!((km >> c1) & 1ull)) pe[c1] = 0.0f;
            }
          }
        }
        if (!mbar_wait(&bars[B_DPF], gs & 1, a.st, a.timeout_ns, 62)) *sm_abort = 1;
        tc_fence_after();
        // dS = P (dP - Delta), one body per precision (each with its own registers): fp16, or
        // bf16 hi + lo; dP is read and dS written 32 columns (16 packed pairs) at a time, over
        // the group's own S columns (hi at +0, lo at +32)
        auto emit_ds = [&](auto f16_tag) {
          constexpr bool F16 = decltype(f16_tag)::value;
          const uint64_t dl2 = pk2(dlt, dlt);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t hi[16], lo[F16 ? 1 : 16];
            if (w_active) {
              uint32_t pp[32];
              tmem_ld32(t_lane + 256 + grp * 64 + h * 32, pp);
              tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const int cc = 16 * h + c;  // pair of columns 2cc, 2cc + 1
                float d0, d1;
                upk2(mul2(pk2(pe[2 * cc], pe[2 * cc + 1]),
                          sub2(pk2(__uint_as_float(pp[2 * c]), __uint_as_float(pp[2 * c + 1])), dl2)),
                     d0, d1);
                if constexpr (F16)
                  hi[c] = pack_f16x2(d0, d1);
                else
                  split_bf16x2(d0, d1, hi[c], lo[c]);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 16; ++c) hi[c] = 0u;
              if constexpr (!F16) {
#pragma unroll
                for (int c = 0; c < 16; ++c) lo[c] = 0u;
              }
            }
            tmem_st16(t_lane + b * 128 + grp * 64 + 16 * h, hi);
            if constexpr (!F16) tmem_st16(t_lane + b * 128 + grp * 64 + 32 + 16 * h, lo);
          }
        };
        if (use16)
          emit_ds(std::true_type{});
        else
          emit_ds(std::false_type{});
        e = e_next;
        km_cur = a.cube_mask[e >> 2];
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[B_PF]);
      }
      // epilogue: dQ row r, columns 64grp..64grp+63, times the softmax scale
      float o[64];
      if (!mbar_wait(&bars[B_DQR], n & 1, a.st, a.timeout_ns, 63)) *sm_abort = 1;  // every item
      if (nsteps > 0) {
        tc_fence_after();
        uint32_t o0[32], o1[32];
        tmem_ld32(t_lane + 384 + grp * 64, o0);
        tmem_ld32(t_lane + 384 + grp * 64 + 32, o1);
        tmem_ld_wait();
        const float sc = row_valid ? a.scale : 0.0f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          o[c] = __uint_as_float(o0[c]) * sc;
          o[c + 32] = __uint_as_float(o1[c]) * sc;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) o[c] = 0.0f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_DQFREE]);
      if (row_exists && grp * 64 < a.D) {
        float4* dst = reinterpret_cast<float4*>(a.dq + qrow * a.D + grp * 64);
        // the coarse branch's term of this cube (valid rows only), when there is one
        const float4* cq = (add.q && row_valid) ? reinterpret_cast<const float4*>(
                                                      add.q + (static_cast<size_t>(bh) * g.T + icube) * a.D + grp * 64)
                                                : nullptr;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float4 w = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          if (cq) {
            const float4 t = __ldg(cq + c);
            w.x += t.x, w.y += t.y, w.z += t.z, w.w += t.w;
          }
          dst[c] = w;
        }
      }
      // an abort seen by any thread reaches every thread at the item boundary
      named_bar_sync(1, 256);
      if (*sm_abort) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
  if (threadIdx.x == 0) cta_clock_record(a, 1, t_start, rec_items, rec_steps);
}

// ------------------------------------------------------------------------ dK, dV
// One item = two adjacent key cubes (128 keys) over the union of their transposed lists,
// two query cubes per step:  S^T = K2 Q2^T,  dP^T = V2 dO2^T  (SS, M = 128 keys, N = 128
// queries), P^T = exp(S^T*scale - lse_q), dS^T = P^T (dP^T - Delta_q), both written as bf16
// hi + lo over their own TMEM columns, then  dV += P^T dO2  and  dK += dS^T Q2  (TS, N = D).
// Thread r of group g owns key row r and the 64 queries of query cube g of the step; the
// step's lse and Delta arrive with the Q and dO tiles (1-D bulk copies).
namespace dkv {
constexpr int kThreads = 320;
constexpr int QST = 2;              // Q/dO ring depth
constexpr uint32_t OFF_K = 0;       // K2 [2 halves][128 keys][128 B]
constexpr uint32_t OFF_V = 32768;   // V2 same
constexpr uint32_t OFF_Q = 65536;   // QST x Q2  [2 halves][128 q][128 B]
constexpr uint32_t OFF_DO = OFF_Q + QST * 32768;
constexpr uint32_t OFF_LSE = OFF_DO + QST * 32768;  // QST x [128] float
constexpr uint32_t OFF_DLT = OFF_LSE + QST * 512;   // QST x [128] float
constexpr uint32_t OFF_BAR = OFF_DLT + QST * 512;
constexpr uint32_t OFF_SLOT = OFF_BAR + 256;
constexpr uint32_t OFF_ABORT = OFF_BAR + 264;
constexpr uint32_t OFF_RING = OFF_BAR + 272;  // kItemRing item ids
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;
constexpr uint32_t TMEM_COLS = 512;  // S^T/P^T at 0, dP^T/dS^T at 128, dV at 256, dK at 384
enum {
  B_KVF = 0, B_KVE = 1, B_QF = 2, B_QE = 4, B_DF = 6, B_DE = 8, B_SF = 10, B_DPF = 11, B_PF = 12, B_DSF = 13,
  B_DVR = 14, B_DVFREE = 15, B_FIN = 16, B_IF = 17, B_IE = 21, NBAR = 25
};
}  // namespace dkv

template <int KS>  // D / 16; MMA loops unrolled (a counted loop costs more than the MMA)
__global__ void __launch_bounds__(dkv::kThreads, 1)
    attn_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_q16, const __grid_constant__ CUtensorMap tm_k16,
                     const __grid_constant__ CUtensorMap tm_v16, const __grid_constant__ CUtensorMap tm_do16,
                     const AttnArgs a, const CoarseAdd add) {
  using namespace dkv;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  volatile int* sm_abort = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  const float* lse_sh = reinterpret_cast<const float*>(smem + OFF_LSE);
  const float* dlt_sh = reinterpret_cast<const float*>(smem + OFF_DLT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const int npairs = (g.T + 1) >> 1;
  const int n_items = a.BH * npairs;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b)
      mbar_init(&bars[b], (b == B_PF || b == B_DSF)
                              ? 256u
                              : (b == B_DVFREE ? 8u : ((b >= B_IE && b < B_IE + kItemRing) ? kRingReaders : 1u)));
    *sm_abort = aborted(a.st) ? 1 : 0;
    fence_barrier_init();
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
  // fp16 single products (every operand from its fp16 copy, P^T and dS^T as one fp16 value) when
  // the conversion pass found every operand and the dS bound within fp16; else bf16 with P^T and
  // dS^T as hi + lo
  const bool use16 = a.f16_single != nullptr && *reinterpret_cast<const volatile unsigned*>(a.f16_single) == 1u;
  const CUtensorMap* mk = use16 ? &tm_k16 : &tm_k;
  const CUtensorMap* mv = use16 ? &tm_v16 : &tm_v;

  if (warp == 0) {
    if (lane < 2 && !skip_all) {
      const bool qside = lane == 0;  // lane 0: item ids, K2, V2, Q2 + lse; lane 1: dO2 + Delta
      const CUtensorMap* tmap = qside ? (use16 ? &tm_q16 : &tm_q) : (use16 ? &tm_do16 : &tm_do);
      const float* vec = qside ? a.nlse2 : a.delta;
      uint32_t gs = 0;
      int issued_kv = 0;
      bool ok = true;
      int n = 0;
      for (; ok; ++n) {
        const int it = qside ? ring_publish(ring, n, n_items, a, a.item_next + 2, 75, ok) : ring_read(ring, n, a, 76, ok);
        if (it < 0) break;
        const int bh = it / npairs, pr = it % npairs;
        const int nu = a.uk_cnt[it];
        const int32_t* ul = a.uk_list + static_cast<size_t>(it) * g.T;
        if (qside) {
          if (n >= 1 && !mbar_wait(&bars[B_KVE], (n - 1) & 1, a.st, a.timeout_ns, 71)) break;
          const int r0 = bh * g.Npad + (2 * pr) * 64;
          const int r1 = (2 * pr + 1 < g.T) ? r0 + 64 : a.rows_total;
          mbar_arrive_expect_tx(&bars[B_KVF], 65536);
          tma_load_2d(smem + OFF_K, mk, &bars[B_KVF], 0, r0);
          tma_load_2d(smem + OFF_K + 8192, mk, &bars[B_KVF], 0, r1);
          tma_load_2d(smem + OFF_K + 16384, mk, &bars[B_KVF], 64, r0);
          tma_load_2d(smem + OFF_K + 24576, mk, &bars[B_KVF], 64, r1);
          tma_load_2d(smem + OFF_V, mv, &bars[B_KVF], 0, r0);
          tma_load_2d(smem + OFF_V + 8192, mv, &bars[B_KVF], 0, r1);
          tma_load_2d(smem + OFF_V + 16384, mv, &bars[B_KVF], 64, r0);
          tma_load_2d(smem + OFF_V + 24576, mv, &bars[B_KVF], 64, r1);
          ++issued_kv;
        }
        const int nsteps = (nu + 1) >> 1;
        for (int s = 0; s < nsteps; ++s) {
          const uint32_t st = gs % QST;
          const uint32_t empty = (qside ? B_QE : B_DE) + st, full = (qside ? B_QF : B_DF) + st;
          if (gs >= QST && !mbar_wait(&bars[empty], ((gs / QST) + 1) & 1, a.st, a.timeout_ns, 72)) {
            ok = false;
            break;
          }
          const int u0 = ul[2 * s] >> 2;
          const int u1 = (2 * s + 1 < nu) ? (ul[2 * s + 1] >> 2) : -1;
          const int y0 = bh * g.Npad + u0 * 64;
          const int y1 = u1 >= 0 ? bh * g.Npad + u1 * 64 : a.rows_total;
          uint8_t* dst = smem + (qside ? OFF_Q : OFF_DO) + st * 32768;
          uint8_t* vdst = smem + (qside ? OFF_LSE : OFF_DLT) + st * 512;
          mbar_arrive_expect_tx(&bars[full], 32768 + (u1 >= 0 ? 512 : 256));
          tma_load_2d(dst, tmap, &bars[full], 0, y0);
          tma_load_2d(dst + 8192, tmap, &bars[full], 0, y1);
          tma_load_2d(dst + 16384, tmap, &bars[full], 64, y0);
          tma_load_2d(dst + 24576, tmap, &bars[full], 64, y1);
          bulk_load(vdst, vec + y0, 256, &bars[full]);
          if (u1 >= 0) bulk_load(vdst + 256, vec + y1, 256, &bars[full]);
          ++gs;
        }
      }
      if (qside) {
        rec_items = n;
        rec_steps = gs;
      }
      if (qside && issued_kv > 0) mbar_wait_drain(&bars[B_KVF], (issued_kv - 1) & 1, a.st, a.timeout_ns, 73);
      for (uint32_t s = (gs > QST ? gs - QST : 0); s < gs; ++s)
        mbar_wait_drain(&bars[(qside ? B_QF : B_DF) + s % QST], (s / QST) & 1, a.st, a.timeout_ns, 74);
    }
  } else if (warp == 1) {
    // the whole warp runs the loop; one elected lane issues (see elect_one)
    if (!skip_all) {
      const uint32_t idesc_kk = make_idesc(128, 128, use16 ? FMT_F16 : FMT_BF16, false, false);
      const uint32_t idesc_mn = make_idesc(128, 128, use16 ? FMT_F16 : FMT_BF16, false, true);
      uint32_t gs = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int it = ring_read_warp(ring, n, a, 89, ok);
        if (it < 0) break;
        const int nsteps = (a.uk_cnt[it] + 1) >> 1;
        if (!mbar_wait_warp(&bars[B_KVF], n & 1, a.st, a.timeout_ns, 81)) break;
        // one phase of DVR / DVFREE per item, empty items included (see the dQ kernel)
        if (n >= 1 && !mbar_wait_warp(&bars[B_DVFREE], (n - 1) & 1, a.st, a.timeout_ns, 82)) break;
        // Issue order per step s:  dV(s), S^T(s+1), dK(s), dP^T(s+1).  S^T(s+1) overwrites P^T(s),
        // already read by dV(s); dP^T(s+1) overwrites dS^T(s), already read by dK(s) (one lane
        // issues everything, so the products execute in this order).  The exponentials of step
        // s+1 then overlap dK(s), and dS^T(s+1) overlaps dV(s+1).
        auto issue_sdp = [&](uint32_t g, bool want_s) -> bool {
          const uint32_t st = g % QST;
          if (!mbar_wait_warp(want_s ? &bars[B_QF + st] : &bars[B_DF + st], (g / QST) & 1, a.st, a.timeout_ns,
                              want_s ? 83 : 84))
            return false;
          tc_fence_after();
          const uint32_t opnd = sbase + (want_s ? OFF_Q : OFF_DO) + st * 32768;
          const uint32_t kv = sbase + (want_s ? OFF_K : OFF_V);
          if (elect_one()) {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
              umma_f16_ss(tmem + (want_s ? 0 : 128), sw128_desc(kv + off, 16, 1024), sw128_desc(opnd + off, 16, 1024),
                          idesc_kk, ks > 0 ? 1u : 0u);
            }
            umma_commit(&bars[want_s ? B_SF : B_DPF]);
          }
          __syncwarp();
          return true;
        };
        if (nsteps > 0) ok = issue_sdp(gs, true) && issue_sdp(gs, false);
        for (int s = 0; ok && s < nsteps; ++s, ++gs) {
          const uint32_t st = gs % QST;
          const uint32_t qst = sbase + OFF_Q + st * 32768, dst = sbase + OFF_DO + st * 32768;
          if (!mbar_wait_warp(&bars[B_PF], gs & 1, a.st, a.timeout_ns, 85)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            if (use16) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {  // dV += P^T dO2 (fp16), overlapping dS^T
                const uint32_t acol = (kk >> 2) * 64 + (kk & 3) * 8;
                umma_f16_ts(tmem + 256, tmem + acol, sw128_desc(dst + kk * 2048, 16384, 1024), idesc_mn,
                            (s > 0 || kk > 0) ? 1u : 0u);
              }
            } else {
#pragma unroll
              for (int ks = 0; ks < 16; ++ks) {  // dV += P^T dO2 (hi then lo), overlapping dS^T
                const uint32_t kk = ks & 7, part = ks >> 3;
                const uint32_t acol = (kk >> 2) * 64 + part * 32 + (kk & 3) * 8;
                umma_f16_ts(tmem + 256, tmem + acol, sw128_desc(dst + kk * 2048, 16384, 1024), idesc_mn,
                            (s > 0 || ks > 0) ? 1u : 0u);
              }
            }
          }
          __syncwarp();
          if (s + 1 < nsteps && !issue_sdp(gs + 1, true)) {
            ok = false;
            break;
          }
          if (!mbar_wait_warp(&bars[B_DSF], gs & 1, a.st, a.timeout_ns, 87)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            if (use16) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {  // dK += dS^T Q2 (fp16)
                const uint32_t acol = 128 + (kk >> 2) * 64 + (kk & 3) * 8;
                umma_f16_ts(tmem + 384, tmem + acol, sw128_desc(qst + kk * 2048, 16384, 1024), idesc_mn,
                            (s > 0 || kk > 0) ? 1u : 0u);
              }
            } else {
#pragma unroll
              for (int ks = 0; ks < 16; ++ks) {  // dK += dS^T Q2 (hi then lo)
                const uint32_t kk = ks & 7, part = ks >> 3;
                const uint32_t acol = 128 + (kk >> 2) * 64 + part * 32 + (kk & 3) * 8;
                umma_f16_ts(tmem + 384, tmem + acol, sw128_desc(qst + kk * 2048, 16384, 1024), idesc_mn,
                            (s > 0 || ks > 0) ? 1u : 0u);
              }
            }
            // the Q and dO stages (with their lse and Delta, read by the softmax before DSF) are free
            umma_commit(&bars[B_QE + st]);
            umma_commit(&bars[B_DE + st]);
          }
          __syncwarp();
          if (s + 1 < nsteps && !issue_sdp(gs + 1, false)) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        if (elect_one()) {
          umma_commit(&bars[B_KVE]);
          umma_commit(&bars[B_DVR]);
        }
        __syncwarp();
      }
      if (elect_one()) umma_commit(&bars[B_FIN]);
      __syncwarp();
      mbar_wait_drain(&bars[B_FIN], 0, a.st, a.timeout_ns, 86);
    }
  } else {
    const int grp = (warp - 2) >> 2;      // query cube grp of each step
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;    // key row of the pair == TMEM lane
    const int khalf = r >> 6;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t gs = 0;
    bool ok = !skip_all;
    for (int n = 0; ok; ++n) {
      const int it = ring_read_group(ring, n, a, 94, sm_abort, ok);
      if (it < 0) break;
      const int bh = it / npairs, pr = it % npairs;
      const int kcube = 2 * pr + khalf;
      const bool key_exists = kcube < g.T;
      const bool key_valid = key_exists && ((a.cube_mask[kcube] >> (r & 63)) & 1ull);
      const int nu = a.uk_cnt[it];
      const int32_t* ul = a.uk_list + static_cast<size_t>(it) * g.T;
      const int nsteps = (nu + 1) >> 1;
      int e = (grp < nu) ? ul[grp] : 0;
      unsigned long long qm_cur = a.cube_mask[e >> 2];
      for (int s = 0; s < nsteps; ++s, ++gs) {
        const uint32_t st = gs % QST;
        const int e_next = (2 * s + 2 + grp < nu) ? ul[2 * s + 2 + grp] : 0;
        const bool active = ((e >> khalf) & 1) && key_valid;
        const bool w_active = __any_sync(0xffffffffu, active);
        if (!mbar_wait(&bars[B_SF], gs & 1, a.st, a.timeout_ns, 91)) *sm_abort = 1;
        tc_fence_after();
        // P^T = exp(S^T * scale - lse_q): written as soon as it is known so that dV can start
        float pe[64];
        {
          if (w_active) {
            uint32_t s0[32], s1[32];
            tmem_ld32(t_lane + grp * 64, s0);
            tmem_ld32(t_lane + grp * 64 + 32, s1);
            tmem_ld_wait();
            // the query mask is first used here, so its load hides behind the waits
            const unsigned long long qm = active ? qm_cur : 0ull;
            const bool full = qm == ~0ull;  // uniform over the warp
            const float* lq = lse_sh + st * 128 + grp * 64;
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
              const float4 l4 = *reinterpret_cast<const float4*>(lq + 4 * c4);
              const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int c = 4 * c4 + u;
                const uint32_t sv = c < 32 ? s0[c] : s1[c - 32];
                pe[c] = ex2_approx(fmaf(__uint_as_float(sv), a.scale_log2, lv[u]));  // lv = -lse log2(e)
                if (!full && !((qm >> c) & 1ull)) pe[c] = 0.0f;
              }
            }
          } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) pe[c] = 0.0f;
          }
          // P^T over S^T (every S^T read of this thread's own columns is done): one fp16 value,
          // or bf16 hi + lo
          if (use16) {
            uint32_t ph[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) ph[c] = pack_f16x2(pe[2 * c], pe[2 * c + 1]);
            tmem_st32(t_lane + grp * 64, ph);
          } else {
            uint32_t ph[32], pl[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              ph[c] = pack_bf16x2(pe[2 * c], pe[2 * c + 1]);
              pl[c] = pack_bf16x2(pe[2 * c] - __uint_as_float(ph[c] << 16),
                                  pe[2 * c + 1] - __uint_as_float(ph[c] & 0xffff0000u));
            }
            tmem_st32(t_lane + grp * 64, ph);
            tmem_st32(t_lane + grp * 64 + 32, pl);
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&bars[B_PF]);
        }
        // dS^T = P^T (dP^T - Delta_q)
        if (!mbar_wait(&bars[B_DPF], gs & 1, a.st, a.timeout_ns, 93)) *sm_abort = 1;
        tc_fence_after();
        {
          // pe becomes dS^T in place (P^T is no longer needed once packed)
          if (w_active) {
            uint32_t p0[32], p1[32];
            tmem_ld32(t_lane + 128 + grp * 64, p0);
            tmem_ld32(t_lane + 128 + grp * 64 + 32, p1);
            tmem_ld_wait();
            const float* dq_ = dlt_sh + st * 128 + grp * 64;
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
              const float4 d4 = *reinterpret_cast<const float4*>(dq_ + 4 * c4);
              const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int c = 4 * c4 + u;
                const uint32_t pv = c < 32 ? p0[c] : p1[c - 32];
                pe[c] = pe[c] * (__uint_as_float(pv) - dv4[u]);
              }
            }
          }
          if (use16) {
            uint32_t dh[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) dh[c] = pack_f16x2(pe[2 * c], pe[2 * c + 1]);
            tmem_st32(t_lane + 128 + grp * 64, dh);
          } else {
            uint32_t dh[32], dl[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              dh[c] = pack_bf16x2(pe[2 * c], pe[2 * c + 1]);
              dl[c] = pack_bf16x2(pe[2 * c] - __uint_as_float(dh[c] << 16),
                                  pe[2 * c + 1] - __uint_as_float(dh[c] & 0xffff0000u));
            }
            tmem_st32(t_lane + 128 + grp * 64, dh);
            tmem_st32(t_lane + 128 + grp * 64 + 32, dl);
          }
          e = e_next;
          qm_cur = a.cube_mask[e >> 2];
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&bars[B_DSF]);
        }
      }
      // epilogue: key row r, columns 64grp..64grp+63 of dV and dK (dK times the scale)
      float gv[64], gk[64];
      if (!mbar_wait(&bars[B_DVR], n & 1, a.st, a.timeout_ns, 92)) *sm_abort = 1;  // every item
      if (nsteps > 0) {
        tc_fence_after();
        uint32_t v0[32], v1[32], k0[32], k1[32];
        tmem_ld32(t_lane + 256 + grp * 64, v0);
        tmem_ld32(t_lane + 256 + grp * 64 + 32, v1);
        tmem_ld32(t_lane + 384 + grp * 64, k0);
        tmem_ld32(t_lane + 384 + grp * 64 + 32, k1);
        tmem_ld_wait();
        const float vs = key_valid ? 1.0f : 0.0f, ks = key_valid ? a.scale : 0.0f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          gv[c] = __uint_as_float(v0[c]) * vs;
          gv[c + 32] = __uint_as_float(v1[c]) * vs;
          gk[c] = __uint_as_float(k0[c]) * ks;
          gk[c + 32] = __uint_as_float(k1[c]) * ks;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) gv[c] = gk[c] = 0.0f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_DVFREE]);
      if (key_exists && grp * 64 < a.D) {
        const size_t krow = static_cast<size_t>(bh) * g.Npad + static_cast<size_t>(kcube) * 64 + (r & 63);
        float4* pv = reinterpret_cast<float4*>(a.dv + krow * a.D + grp * 64);
        float4* pk = reinterpret_cast<float4*>(a.dk + krow * a.D + grp * 64);
        // the coarse branch's terms of this cube (valid keys only), when there are some
        const size_t co = (static_cast<size_t>(bh) * g.T + kcube) * a.D + grp * 64;
        const bool has_add = add.k && key_valid;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float4 wv = make_float4(gv[4 * c], gv[4 * c + 1], gv[4 * c + 2], gv[4 * c + 3]);
          float4 wk = make_float4(gk[4 * c], gk[4 * c + 1], gk[4 * c + 2], gk[4 * c + 3]);
          if (has_add) {
            const float4 tv = __ldg(reinterpret_cast<const float4*>(add.v + co) + c);
            const float4 tk = __ldg(reinterpret_cast<const float4*>(add.k + co) + c);
            wv.x += tv.x, wv.y += tv.y, wv.z += tv.z, wv.w += tv.w;
            wk.x += tk.x, wk.y += tk.y, wk.z += tk.z, wk.w += tk.w;
          }
          pv[c] = wv;
          pk[c] = wk;
        }
      }
      named_bar_sync(1, 256);
      if (*sm_abort) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
  if (threadIdx.x == 0) cta_clock_record(a, 2, t_start, rec_items, rec_steps);
}

// ------------------------------------------------------------------------ launch
cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap (&t16)[4], const void* out, const float* out_f32,
                            const void* dout,
                            AttnArgs a, uint32_t* bits, float* delta, float* nlse2,
                            int32_t* uq_list,
                            int32_t* uq_cnt, int32_t* uk_list, int32_t* uk_cnt, const CoarseAdd& add,
                            bool delta_ready, cudaStream_t stream, int* launches) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaSuccess;
    for (auto fn : {attn_dq_kernel<4>, attn_dq_kernel<8>})
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dqk::SMEM_BYTES);
    for (auto fn : {attn_dkdv_kernel<4>, attn_dkdv_kernel<8>})
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const Geom& g = a.g;
  const long long rows = static_cast<long long>(a.BH) * g.Npad;
  if (!delta_ready)
    delta_kernel<<<static_cast<unsigned>((rows + 8 * DELTA_ROWS - 1) / (8 * DELTA_ROWS)), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(out), out_f32, static_cast<const __nv_bfloat16*>(dout), a.lse, delta,
        nlse2, g, a.BH, a.D);
  cudaError_t e = launch_query_pair_union(a.kv_index, a.kv_count, uq_list, uq_cnt, a.BH, g.T, a.cap, a.st, stream);
  if (e != cudaSuccess) return e;
  e = launch_key_pair_union(a.kv_index, a.kv_count, bits, uk_list, uk_cnt, a.BH, g.T, a.cap, a.st, stream);
  if (e != cudaSuccess) return e;
  a.delta = delta;
  a.nlse2 = nlse2;
  a.u_list = uq_list;
  a.u_cnt = uq_cnt;
  a.uk_list = uk_list;
  a.uk_cnt = uk_cnt;
  const int sms = num_sms();
  const int items = a.BH * ((g.T + 1) >> 1);
  const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  if (a.D == 64) {
    attn_dq_kernel<4><<<grid, dqk::kThreads, dqk::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, t16[0], t16[1], a, add);
    attn_dkdv_kernel<4><<<grid, dkv::kThreads, dkv::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, t16[0], t16[1], t16[2],
                                                                         t16[3], a, add);
  } else {
    attn_dq_kernel<8><<<grid, dqk::kThreads, dqk::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, t16[0], t16[1], a, add);
    attn_dkdv_kernel<8><<<grid, dkv::kThreads, dkv::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, t16[0], t16[1], t16[2],
                                                                         t16[3], a, add);
  }
  *launches = delta_ready ? 5 : 6;
  return cudaGetLastError();
}

}  // namespace sa
