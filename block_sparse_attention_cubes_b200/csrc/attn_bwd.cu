// Fine-stage backward with the block mask held constant (VSA2 page, section 2.1: the
// router's output carries no gradient; SpargeAttention2 page, "Why this implementation is
// trainable": gradients flow only through the un-masked computations).  With
// S = scale * Q K^T + M, P = softmax(S) recomputed from lse,
//     dV = P^T dO,  dP = dO V^T,  Delta = rowsum(dO * O),  dS = P * (dP - Delta),
//     dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Kernels:
//   delta_kernel      Delta per query row (one warp per row).
//   count/scan/fill   the transposed lists: for each key cube j the ascending query cubes
//                     whose list holds j (CSR, deterministic).
//   attn_dq_kernel    per query cube, transposed like the forward: over pairs of its key
//                     tiles, S^T = K2 Q^T and dP^T = V2 dO^T (M=128), dS^T in shared memory,
//                     dQ^T += K2^T dS^T (M=D).
//   attn_dkdv_kernel  per key cube, over pairs of the query cubes that selected it:
//                     S = Q2 K^T and dP = dO2 V^T (M=128 query rows), P and dS in shared
//                     memory, dV^T += dO2^T P and dK^T += Q2^T dS (M=D).
// Both main kernels keep every accumulator in TMEM and use the same warp roles as the
// forward (TMA producer, MMA issuer, 128-thread elementwise group).
#include <cmath>

#include "attn_common.cuh"
#include "kernels.h"

namespace sa {

// ------------------------------------------------------------------------ Delta
// O is read from its fp32 copy when there is one, else from the bf16 output.
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                    const float* __restrict__ o32,
                                                    const __nv_bfloat16* __restrict__ dout,
                                                    float* __restrict__ delta, Geom g, int BH, int D) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x * 8LL + warp;
  if (row >= static_cast<long long>(BH) * g.Npad) return;
  const int p = static_cast<int>(row % g.Npad);
  float acc = 0.0f;
  if (token_valid(g, p >> 6, p & 63)) {
    const uint2* b = reinterpret_cast<const uint2*>(dout + row * D);
    for (int c = lane; c < D / 4; c += 32) {
      const uint2 y = b[c];
      float ov[4];
      if (o32) {
        const float4 x = reinterpret_cast<const float4*>(o32 + row * D)[c];
        ov[0] = x.x; ov[1] = x.y; ov[2] = x.z; ov[3] = x.w;
      } else {
        const uint2 x = reinterpret_cast<const uint2*>(o + row * D)[c];
        ov[0] = __uint_as_float(x.x << 16); ov[1] = __uint_as_float(x.x & 0xffff0000u);
        ov[2] = __uint_as_float(x.y << 16); ov[3] = __uint_as_float(x.y & 0xffff0000u);
      }
      acc += ov[0] * __uint_as_float(y.x << 16);
      acc += ov[1] * __uint_as_float(y.x & 0xffff0000u);
      acc += ov[2] * __uint_as_float(y.y << 16);
      acc += ov[3] * __uint_as_float(y.y & 0xffff0000u);
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[row] = acc;
}

// ------------------------------------------------------------------------ transposed lists
__global__ void count_kernel(const int32_t* __restrict__ kv_index, const int32_t* __restrict__ kv_count,
                             int32_t* __restrict__ qcnt, int BH, int T, int cap) {
  const long long row = blockIdx.x * (long long)blockDim.y + threadIdx.y;  // (bh, i)
  if (row >= static_cast<long long>(BH) * T) return;
  const int bh = static_cast<int>(row / T);
  int n = kv_count[row];
  n = n < 0 ? 0 : (n > cap ? cap : n);
  for (int t = threadIdx.x; t < n; t += blockDim.x) {
    const int j = kv_index[row * cap + t];
    if (j >= 0 && j < T) atomicAdd(&qcnt[static_cast<size_t>(bh) * T + j], 1);
  }
}

// exclusive scan of qcnt[bh][0..T) into qoff[bh][0..T], one CTA per bh
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ qcnt, int32_t* __restrict__ qoff,
                                                    int T, int cap) {
  __shared__ int32_t part[1024];
  const int bh = blockIdx.x;
  const int per = (T + 1023) / 1024;
  const int beg = threadIdx.x * per;
  int s = 0;
  for (int j = beg; j < beg + per && j < T; ++j) s += qcnt[static_cast<size_t>(bh) * T + j];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  // entries of head bh start at bh * T * cap (an upper bound of its total)
  int run = static_cast<int>(static_cast<size_t>(bh) * T * cap) + (threadIdx.x ? part[threadIdx.x - 1] : 0);
  for (int j = beg; j < beg + per && j < T; ++j) {
    qoff[static_cast<size_t>(bh) * (T + 1) + j] = run;
    run += qcnt[static_cast<size_t>(bh) * T + j];
  }
  if (threadIdx.x == 1023) qoff[static_cast<size_t>(bh) * (T + 1) + T] = run;
}

// One warp per (bh, key cube j): visit query cubes in ascending order and binary-search j in
// each ascending list; append hits in order.
__global__ void __launch_bounds__(256) fill_kernel(const int32_t* __restrict__ kv_index,
                                                   const int32_t* __restrict__ kv_count,
                                                   const int32_t* __restrict__ qoff, int32_t* __restrict__ qidx,
                                                   int BH, int T, int cap) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long col = blockIdx.x * 8LL + warp;
  if (col >= static_cast<long long>(BH) * T) return;
  const int bh = static_cast<int>(col / T), j = static_cast<int>(col % T);
  int pos = qoff[static_cast<size_t>(bh) * (T + 1) + j];
  for (int i0 = 0; i0 < T; i0 += 32) {
    const int i = i0 + lane;
    bool hit = false;
    if (i < T) {
      const size_t r = static_cast<size_t>(bh) * T + i;
      int n = kv_count[r];
      n = n < 0 ? 0 : (n > cap ? cap : n);
      const int32_t* lst = kv_index + r * cap;
      int lo = 0, hi = n;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (lst[mid] < j) lo = mid + 1; else hi = mid;
      }
      hit = lo < n && lst[lo] == j;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, hit);
    if (hit) qidx[pos + __popc(bal & ((1u << lane) - 1u))] = i;
    pos += __popc(bal);
  }
}

// ------------------------------------------------------------------------ dQ
namespace dqk {
constexpr int kThreads = 192;
constexpr uint32_t OFF_Q = 0;          // [2 halves][64][128 B]
constexpr uint32_t OFF_DO = 16384;     // same
constexpr uint32_t OFF_K = 32768;      // 2 stages x [2 halves][128][128 B]
constexpr uint32_t OFF_V = 98304;      // same
constexpr uint32_t OFF_DS = 163840;    // 2 buffers x {hi, lo} x [128 keys][64 q] bf16
constexpr uint32_t OFF_BAR = 229376;
constexpr uint32_t OFF_SLOT = OFF_BAR + 192;
constexpr uint32_t OFF_FLAG = OFF_BAR + 200;
constexpr uint32_t OFF_LSE = OFF_BAR + 256;    // [64] lse * log2(e)
constexpr uint32_t OFF_DELTA = OFF_LSE + 256;  // [64]
constexpr uint32_t SMEM_BYTES = OFF_DELTA + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;  // S^T[b] at 128b, dP^T[b] at 128b+64, dQ^T at 256
enum { B_QD = 0, B_KF = 1, B_VF = 3, B_EMPTY = 5, B_SDP = 7, B_DSF = 9, B_DSFREE = 11, B_FIN = 13, NBAR = 14 };
}  // namespace dqk

__global__ void __launch_bounds__(dqk::kThreads, 1)
    attn_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                   const AttnArgs a) {
  using namespace dqk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  volatile int* grp_abort = reinterpret_cast<volatile int*>(smem + OFF_FLAG);
  float* lse2_sh = reinterpret_cast<float*>(smem + OFF_LSE);
  float* delta_sh = reinterpret_cast<float*>(smem + OFF_DELTA);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x % a.g.T;
  const int bh = blockIdx.x / a.g.T;
  const Geom& g = a.g;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b) mbar_init(&bars[b], (b == B_DSF || b == B_DSF + 1) ? 128u : 1u);
    *grp_abort = aborted(a.st) ? 1 : 0;
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
  const bool skip_all = *grp_abort != 0;
  const int n = list_count(a, bh, i, threadIdx.x == 0);
  const int nsteps = skip_all ? 0 : (n + 1) >> 1;
  const int row0 = bh * g.Npad + i * 64;

  if (warp == 0) {
    if (lane == 0 && nsteps > 0) {
      mbar_arrive_expect_tx(&bars[B_QD], 32768);
      tma_load_2d(smem + OFF_Q, &tm_q, &bars[B_QD], 0, row0);
      tma_load_2d(smem + OFF_Q + 8192, &tm_q, &bars[B_QD], 64, row0);
      tma_load_2d(smem + OFF_DO, &tm_do, &bars[B_QD], 0, row0);
      tma_load_2d(smem + OFF_DO + 8192, &tm_do, &bars[B_QD], 64, row0);
      int issued = 0;
      for (int s = 0; s < nsteps; ++s) {
        const int st = s & 1;
        if (s >= 2 && !mbar_wait(&bars[B_EMPTY + st], ((s >> 1) + 1) & 1, a.st, a.timeout_ns, 41)) break;
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
      mbar_wait(&bars[B_QD], 0, a.st, a.timeout_ns, 42);
      for (int s = (issued > 2 ? issued - 2 : 0); s < issued; ++s) {
        mbar_wait(&bars[B_KF + (s & 1)], (s >> 1) & 1, a.st, a.timeout_ns, 43);
        mbar_wait(&bars[B_VF + (s & 1)], (s >> 1) & 1, a.st, a.timeout_ns, 44);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nsteps > 0) {
      const uint32_t idesc_kk = make_idesc(128, 64, FMT_BF16, false, false);
      const uint32_t idesc_mn = make_idesc(128, 64, FMT_BF16, true, true);
      const int ksteps = a.D / 16;
      auto issue_sdp = [&](int s) {
        const int st = s & 1;
        const uint32_t kst = sbase + OFF_K + st * 32768, vst = sbase + OFF_V + st * 32768;
        const uint32_t d_s = tmem + st * 128, d_dp = tmem + st * 128 + 64;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t qoff = (ks >> 2) * 8192 + (ks & 3) * 32;
          umma_f16_ss(d_s, sw128_desc(kst + off, 16, 1024), sw128_desc(sbase + OFF_Q + qoff, 16, 1024), idesc_kk,
                      ks > 0 ? 1u : 0u);
        }
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t qoff = (ks >> 2) * 8192 + (ks & 3) * 32;
          umma_f16_ss(d_dp, sw128_desc(vst + off, 16, 1024), sw128_desc(sbase + OFF_DO + qoff, 16, 1024),
                      idesc_kk, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars[B_SDP + st]);
      };
      bool ok = mbar_wait(&bars[B_QD], 0, a.st, a.timeout_ns, 51);
      for (int s = 0; ok && s < 2 && s < nsteps; ++s) {
        ok = mbar_wait(&bars[B_KF + s], 0, a.st, a.timeout_ns, 52) &&
             mbar_wait(&bars[B_VF + s], 0, a.st, a.timeout_ns, 53);
        if (ok) {
          tc_fence_after();
          issue_sdp(s);
        }
      }
      for (int s = 0; ok && s < nsteps; ++s) {
        const int st = s & 1;
        if (!mbar_wait(&bars[B_DSF + st], (s >> 1) & 1, a.st, a.timeout_ns, 54)) break;
        tc_fence_after();
        const uint32_t kst = sbase + OFF_K + st * 32768;
        const uint32_t dsb = sbase + OFF_DS + st * 32768;
#pragma unroll 1
        for (int ks = 0; ks < 16; ++ks) {  // 8 k-steps over dS_hi, then 8 over dS_lo
          const uint32_t kk = ks & 7, part = ks >> 3;
          umma_f16_ss(tmem + 256, sw128_desc(kst + kk * 2048, 16384, 1024),
                      sw128_desc(dsb + part * 16384 + kk * 2048, 8192, 1024), idesc_mn, (s > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&bars[B_EMPTY + st]);
        umma_commit(&bars[B_DSFREE + st]);
        if (s + 2 < nsteps) {
          ok = mbar_wait(&bars[B_KF + st], ((s + 2) >> 1) & 1, a.st, a.timeout_ns, 55) &&
               mbar_wait(&bars[B_VF + st], ((s + 2) >> 1) & 1, a.st, a.timeout_ns, 56);
          if (!ok) break;
          tc_fence_after();
          issue_sdp(s + 2);
        }
      }
      umma_commit(&bars[B_FIN]);
      mbar_wait(&bars[B_FIN], 0, a.st, a.timeout_ns, 57);
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    if (r < 64) {
      const bool qv = token_valid(g, i, r);
      lse2_sh[r] = qv ? a.lse[row0 + r] * 1.4426950408889634f : 0.0f;
      delta_sh[r] = qv ? a.delta[row0 + r] : 0.0f;
    }
    named_bar_sync(1, 128);
    uint64_t qmask = 0;  // valid query columns of this cube
    for (int c = 0; c < 64; ++c)
      if (token_valid(g, i, c)) qmask |= 1ull << c;
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      const int b = s & 1;
      if (!mbar_wait(&bars[B_SDP + b], (s >> 1) & 1, a.st, a.timeout_ns, 61)) *grp_abort = 1;
      tc_fence_after();
      float sv[64], dp[64];
      tmem_ld64(t_lane + b * 128, sv);
      tmem_ld64(t_lane + b * 128 + 64, dp);
      const int tile = list_entry(a, bh, i, n, 2 * s + (r >> 6), false);
      const bool kvalid = tile >= 0 && token_valid(g, tile, r & 63);
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const bool on = kvalid && ((qmask >> c) & 1ull);
        const float p = on ? exp2f(sv[c] * a.scale_log2 - lse2_sh[c]) : 0.0f;
        sv[c] = p * (dp[c] - delta_sh[c]);
      }
      if (s >= 2 && !mbar_wait(&bars[B_DSFREE + b], ((s >> 1) + 1) & 1, a.st, a.timeout_ns, 62)) *grp_abort = 1;
      store_row_bf16x2_sw128(sbase + OFF_DS + b * 32768, sbase + OFF_DS + b * 32768 + 16384, r, sv);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_DSF + b]);
      named_bar_sync(1, 128);
      if (*grp_abort) {
        ok = false;
        break;
      }
    }
    if (ok && nsteps > 0) {
      if (!mbar_wait(&bars[B_DSFREE + ((nsteps - 1) & 1)], ((nsteps - 1) >> 1) & 1, a.st, a.timeout_ns, 63))
        ok = false;
    }
    tc_fence_after();
    float o[64];
    if (nsteps > 0 && ok) {
      tmem_ld64(t_lane + 256, o);
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) o[c] = 0.0f;
    }
    if (r < a.D) {
      float* dst = a.dq + static_cast<size_t>(row0) * a.D + r;
#pragma unroll
      for (int c = 0; c < 64; ++c) dst[static_cast<size_t>(c) * a.D] = ((qmask >> c) & 1ull) ? o[c] * a.scale : 0.0f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------------ dK, dV
namespace dkv {
constexpr int kThreads = 192;
constexpr uint32_t OFF_K = 0;          // [2 halves][64][128 B]
constexpr uint32_t OFF_V = 16384;      // same
constexpr uint32_t OFF_Q = 32768;      // 2 stages x [2 halves][128][128 B]
constexpr uint32_t OFF_DO = 98304;     // same
constexpr uint32_t OFF_P = 163840;     // {hi, lo} x [128 q][64 keys] bf16
constexpr uint32_t OFF_DS = 196608;    // same
constexpr uint32_t OFF_BAR = 229376;
constexpr uint32_t OFF_SLOT = OFF_BAR + 192;
constexpr uint32_t OFF_FLAG = OFF_BAR + 200;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;  // S[b] at 128b, dP[b] at 128b+64, dV^T at 256, dK^T at 320
enum { B_KV = 0, B_QF = 1, B_EMPTY = 3, B_SDP = 5, B_PDS = 7, B_PDSFREE = 8, B_FIN = 9, NBAR = 10 };
}  // namespace dkv

__global__ void __launch_bounds__(dkv::kThreads, 1)
    attn_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const AttnArgs a) {
  using namespace dkv;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  volatile int* grp_abort = reinterpret_cast<volatile int*>(smem + OFF_FLAG);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x % a.g.T;
  const int bh = blockIdx.x / a.g.T;
  const Geom& g = a.g;
  const int qbeg = a.q_off[static_cast<size_t>(bh) * (g.T + 1) + j];
  const int nq = a.q_off[static_cast<size_t>(bh) * (g.T + 1) + j + 1] - qbeg;

  if (threadIdx.x == 0) {
    for (int b = 0; b < NBAR; ++b) mbar_init(&bars[b], b == B_PDS ? 128u : 1u);
    *grp_abort = aborted(a.st) ? 1 : 0;
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
  const bool skip_all = *grp_abort != 0;
  const int nsteps = skip_all ? 0 : (nq + 1) >> 1;
  const int krow0 = bh * g.Npad + j * 64;
  auto qcube = [&](int t) -> int { return t < nq ? a.q_idx[qbeg + t] : -1; };

  if (warp == 0) {
    if (lane == 0 && nsteps > 0) {
      mbar_arrive_expect_tx(&bars[B_KV], 32768);
      tma_load_2d(smem + OFF_K, &tm_k, &bars[B_KV], 0, krow0);
      tma_load_2d(smem + OFF_K + 8192, &tm_k, &bars[B_KV], 64, krow0);
      tma_load_2d(smem + OFF_V, &tm_v, &bars[B_KV], 0, krow0);
      tma_load_2d(smem + OFF_V + 8192, &tm_v, &bars[B_KV], 64, krow0);
      int issued = 0;
      for (int s = 0; s < nsteps; ++s) {
        const int st = s & 1;
        if (s >= 2 && !mbar_wait(&bars[B_EMPTY + st], ((s >> 1) + 1) & 1, a.st, a.timeout_ns, 71)) break;
        const int i0 = qcube(2 * s), i1 = qcube(2 * s + 1);
        const int y0 = i0 >= 0 ? bh * g.Npad + i0 * 64 : a.rows_total;
        const int y1 = i1 >= 0 ? bh * g.Npad + i1 * 64 : a.rows_total;
        uint8_t* qst = smem + OFF_Q + st * 32768;
        uint8_t* dst = smem + OFF_DO + st * 32768;
        mbar_arrive_expect_tx(&bars[B_QF + st], 65536);
        tma_load_2d(qst, &tm_q, &bars[B_QF + st], 0, y0);
        tma_load_2d(qst + 8192, &tm_q, &bars[B_QF + st], 0, y1);
        tma_load_2d(qst + 16384, &tm_q, &bars[B_QF + st], 64, y0);
        tma_load_2d(qst + 24576, &tm_q, &bars[B_QF + st], 64, y1);
        tma_load_2d(dst, &tm_do, &bars[B_QF + st], 0, y0);
        tma_load_2d(dst + 8192, &tm_do, &bars[B_QF + st], 0, y1);
        tma_load_2d(dst + 16384, &tm_do, &bars[B_QF + st], 64, y0);
        tma_load_2d(dst + 24576, &tm_do, &bars[B_QF + st], 64, y1);
        ++issued;
      }
      mbar_wait(&bars[B_KV], 0, a.st, a.timeout_ns, 72);
      for (int s = (issued > 2 ? issued - 2 : 0); s < issued; ++s)
        mbar_wait(&bars[B_QF + (s & 1)], (s >> 1) & 1, a.st, a.timeout_ns, 73);
    }
  } else if (warp == 1) {
    if (lane == 0 && nsteps > 0) {
      const uint32_t idesc_kk = make_idesc(128, 64, FMT_BF16, false, false);
      const uint32_t idesc_mn = make_idesc(128, 64, FMT_BF16, true, true);
      const int ksteps = a.D / 16;
      auto issue_sdp = [&](int s) {
        const int st = s & 1;
        const uint32_t qst = sbase + OFF_Q + st * 32768, dst = sbase + OFF_DO + st * 32768;
        const uint32_t d_s = tmem + st * 128, d_dp = tmem + st * 128 + 64;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t koff = (ks >> 2) * 8192 + (ks & 3) * 32;
          umma_f16_ss(d_s, sw128_desc(qst + off, 16, 1024), sw128_desc(sbase + OFF_K + koff, 16, 1024), idesc_kk,
                      ks > 0 ? 1u : 0u);
        }
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          const uint32_t koff = (ks >> 2) * 8192 + (ks & 3) * 32;
          umma_f16_ss(d_dp, sw128_desc(dst + off, 16, 1024), sw128_desc(sbase + OFF_V + koff, 16, 1024), idesc_kk,
                      ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars[B_SDP + st]);
      };
      bool ok = mbar_wait(&bars[B_KV], 0, a.st, a.timeout_ns, 81);
      for (int s = 0; ok && s < 2 && s < nsteps; ++s) {
        ok = mbar_wait(&bars[B_QF + s], 0, a.st, a.timeout_ns, 82);
        if (ok) {
          tc_fence_after();
          issue_sdp(s);
        }
      }
      for (int s = 0; ok && s < nsteps; ++s) {
        const int st = s & 1;
        if (!mbar_wait(&bars[B_PDS], s & 1, a.st, a.timeout_ns, 83)) break;
        tc_fence_after();
        const uint32_t qst = sbase + OFF_Q + st * 32768, dst = sbase + OFF_DO + st * 32768;
#pragma unroll 1
        for (int ks = 0; ks < 16; ++ks) {  // P_hi then P_lo
          const uint32_t kk = ks & 7, part = ks >> 3;
          umma_f16_ss(tmem + 256, sw128_desc(dst + kk * 2048, 16384, 1024),
                      sw128_desc(sbase + OFF_P + part * 16384 + kk * 2048, 8192, 1024), idesc_mn,
                      (s > 0 || ks > 0) ? 1u : 0u);
        }
#pragma unroll 1
        for (int ks = 0; ks < 16; ++ks) {  // dS_hi then dS_lo
          const uint32_t kk = ks & 7, part = ks >> 3;
          umma_f16_ss(tmem + 320, sw128_desc(qst + kk * 2048, 16384, 1024),
                      sw128_desc(sbase + OFF_DS + part * 16384 + kk * 2048, 8192, 1024), idesc_mn,
                      (s > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&bars[B_EMPTY + st]);
        umma_commit(&bars[B_PDSFREE]);
        if (s + 2 < nsteps) {
          ok = mbar_wait(&bars[B_QF + st], ((s + 2) >> 1) & 1, a.st, a.timeout_ns, 84);
          if (!ok) break;
          tc_fence_after();
          issue_sdp(s + 2);
        }
      }
      umma_commit(&bars[B_FIN]);
      mbar_wait(&bars[B_FIN], 0, a.st, a.timeout_ns, 85);
    }
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row of the pair == TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint64_t kmask = 0;  // valid key columns of cube j
    for (int c = 0; c < 64; ++c)
      if (token_valid(g, j, c)) kmask |= 1ull << c;
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      const int b = s & 1;
      const int icube = qcube(2 * s + (r >> 6));
      const bool qv = icube >= 0 && token_valid(g, icube, r & 63);
      const size_t qrow = static_cast<size_t>(bh) * g.Npad + static_cast<size_t>(icube < 0 ? 0 : icube) * 64 + (r & 63);
      const float lse2 = qv ? a.lse[qrow] * 1.4426950408889634f : 0.0f;
      const float dlt = qv ? a.delta[qrow] : 0.0f;
      if (!mbar_wait(&bars[B_SDP + b], (s >> 1) & 1, a.st, a.timeout_ns, 91)) *grp_abort = 1;
      tc_fence_after();
      float sv[64], dp[64];
      tmem_ld64(t_lane + b * 128, sv);
      tmem_ld64(t_lane + b * 128 + 64, dp);
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const bool on = qv && ((kmask >> c) & 1ull);
        const float p = on ? exp2f(sv[c] * a.scale_log2 - lse2) : 0.0f;
        sv[c] = p;
        dp[c] = p * (dp[c] - dlt);
      }
      if (s >= 1 && !mbar_wait(&bars[B_PDSFREE], (s - 1) & 1, a.st, a.timeout_ns, 92)) *grp_abort = 1;
      store_row_bf16x2_sw128(sbase + OFF_P, sbase + OFF_P + 16384, r, sv);
      store_row_bf16x2_sw128(sbase + OFF_DS, sbase + OFF_DS + 16384, r, dp);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_PDS]);
      named_bar_sync(1, 128);
      if (*grp_abort) {
        ok = false;
        break;
      }
    }
    if (ok && nsteps > 0 && !mbar_wait(&bars[B_PDSFREE], (nsteps - 1) & 1, a.st, a.timeout_ns, 93)) ok = false;
    tc_fence_after();
    float gv[64], gk[64];
    if (nsteps > 0 && ok) {
      tmem_ld64(t_lane + 256, gv);
      tmem_ld64(t_lane + 320, gk);
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) gv[c] = gk[c] = 0.0f;
    }
    if (r < a.D) {
      float* pv = a.dv + static_cast<size_t>(krow0) * a.D + r;
      float* pk = a.dk + static_cast<size_t>(krow0) * a.D + r;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const bool kv = (kmask >> c) & 1ull;
        pv[static_cast<size_t>(c) * a.D] = kv ? gv[c] : 0.0f;
        pk[static_cast<size_t>(c) * a.D] = kv ? gk[c] * a.scale : 0.0f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------------ launch
cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const void* out, const float* out_f32, const void* dout,
                            AttnArgs a, int32_t* qcnt,
                            int32_t* qoff, int32_t* qidx, float* delta, cudaStream_t stream, int* launches) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dqk::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const Geom& g = a.g;
  const long long rows = static_cast<long long>(a.BH) * g.Npad;
  delta_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(out), out_f32, static_cast<const __nv_bfloat16*>(dout), delta, g, a.BH,
      a.D);
  cudaError_t e = cudaMemsetAsync(qcnt, 0, sizeof(int32_t) * static_cast<size_t>(a.BH) * g.T, stream);
  if (e != cudaSuccess) return e;
  const long long qrows = static_cast<long long>(a.BH) * g.T;
  count_kernel<<<static_cast<unsigned>((qrows + 7) / 8), dim3(32, 8), 0, stream>>>(a.kv_index, a.kv_count, qcnt,
                                                                                    a.BH, g.T, a.cap);
  scan_kernel<<<a.BH, 1024, 0, stream>>>(qcnt, qoff, g.T, a.cap);
  fill_kernel<<<static_cast<unsigned>((qrows + 7) / 8), 256, 0, stream>>>(a.kv_index, a.kv_count, qoff, qidx, a.BH,
                                                                          g.T, a.cap);
  a.delta = delta;
  a.q_off = qoff;
  a.q_idx = qidx;
  const unsigned grid = static_cast<unsigned>(a.BH) * g.T;
  attn_dq_kernel<<<grid, dqk::kThreads, dqk::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, a);
  attn_dkdv_kernel<<<grid, dkv::kThreads, dkv::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, a);
  *launches = 6;
  return cudaGetLastError();
}

}  // namespace sa
