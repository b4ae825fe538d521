// Coarse branch of the cube-routed attention and its gated combination with the fine output.
//
// VSA page, "Big-Picture Architecture" item 2 and "What the coarse attention output O_c
// provides"; VSA2 page, section 2.2 "Coarse Branch" and the gate equation:
//   [Qc, Kc, Vc] = MeanPool_64([Q, K, V]),  Pc = Softmax(Qc Kc^T * scale),  Oc^ = Pc Vc,
//   O = G (.) Repeat_64(Oc^) + O_f                  (G: one scalar per token and head)
// The router already holds Qc, Kc and the scaled cube scores in fp64; the coarse branch
// reads them from the plan workspace, so Q and K are pooled once for both uses.
//
//   coarse_pool_kernel      Vc (fp32 mean of the valid tokens) and fp32 copies of Qc, Kc
//   coarse_softmax_kernel   Pc rows (fp32) and lse_c from the fp64 scores
//   coarse_mma_kernel       batched products of the cube-level matrices on the tensor cores
//                           (fp32 operands split into bf16 hi + lo), with the epilogues the
//                           branch needs (plain, dS = P (dP - delta), and the mean-pool
//                           adjoint 1/n per cube)
//   coarse_gate_bwd_kernel  one pass over dO: dG, the fine branch's Delta and -lse*log2(e),
//                           dOc^ = sum_t G_t dO_t and delta_c = <dOc^, Oc^> per cube
//
// The cube-level matrices are T x T per head (T = 1440 at the 720p shape), so the six products
// of a forward and backward are about 1/250 of the fine stage's FLOPs at 95% sparsity.  They
// run on the tensor cores with every fp32 operand split into a bf16 pair (three products per
// tile: about 2^-16 relative per term, fp32 accumulation).
#include <cuda_bf16.h>

#include <cmath>

#include "geometry.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace sa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// PER consecutive bf16 of a row (PER = 2 or 4) as floats
template <int PER>
__device__ __forceinline__ void load_bf(const __nv_bfloat16* p, float* x) {
  if constexpr (PER == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    x[0] = bf_lo(w.x), x[1] = bf_hi(w.x), x[2] = bf_lo(w.y), x[3] = bf_hi(w.y);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    x[0] = bf_lo(w), x[1] = bf_hi(w);
  }
}

template <int PER>
__device__ __forceinline__ void load_f(const float* p, float* x) {
  if constexpr (PER == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x, x[1] = v.y, x[2] = v.z, x[3] = v.w;
  } else {
    const float2 v = *reinterpret_cast<const float2*>(p);
    x[0] = v.x, x[1] = v.y;
  }
}

template <int PER>
__device__ __forceinline__ void store_f(float* p, const float* x) {
  if constexpr (PER == 4)
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  else
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
}

// ------------------------------------------------------------------------ pooling
// One warp per (bh, cube); lane l owns columns PER*l .. PER*l + PER - 1 (D = 32 * PER).
// Eight rows' loads are issued before they are accumulated.
template <int PER>
__global__ void __launch_bounds__(256) coarse_pool_kernel(const __nv_bfloat16* __restrict__ v,
                                                          const double* __restrict__ qbar64,
                                                          const double* __restrict__ kbar64,
                                                          float* __restrict__ qbar, float* __restrict__ kbar,
                                                          float* __restrict__ vbar, Geom g, int BH) {
  constexpr int D = 32 * PER;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long cube = blockIdx.x * 8LL + warp;
  if (cube >= static_cast<long long>(BH) * g.T) return;
  int vt, vh, vw;
  cube_extent(g, static_cast<int>(cube % g.T), vt, vh, vw);
  const __nv_bfloat16* base = v + cube * 64 * D + lane * PER;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
  for (int s0 = 0; s0 < 64; s0 += 8) {
    float x[8][PER];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (slot_valid(vt, vh, vw, s0 + u)) {
        load_bf<PER>(base + (s0 + u) * D, x[u]);
      } else {
#pragma unroll
        for (int e = 0; e < PER; ++e) x[u][e] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] += x[u][e];
  }
  const float inv = 1.0f / static_cast<float>(vt * vh * vw);
  const long long o = cube * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    vbar[o + e] = acc[e] * inv;
    qbar[o + e] = static_cast<float>(qbar64[o + e]);
    kbar[o + e] = static_cast<float>(kbar64[o + e]);
  }
}

// ------------------------------------------------------------------------ softmax
// One warp per cube row: max, sum of exp(s - max), then P = exp(s - max) / sum, in place over
// the row's fp32 scores (each lane rewrites only the entries it read).  The row is read three
// times; after the first pass it comes from L1/L2.
__global__ void __launch_bounds__(256) coarse_softmax_kernel(float* __restrict__ SP, float* __restrict__ lse,
                                                             long long rows, int T) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x * 8LL + warp;
  if (row >= rows) return;
  float* s = SP + row * T;
  float m = -INFINITY;
  for (int j = lane; j < T; j += 32) m = fmaxf(m, s[j]);
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float l = 0.0f;
  for (int j = lane; j < T; j += 32) l += expf(s[j] - m);
#pragma unroll
  for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  const float inv = 1.0f / l;
  for (int j = lane; j < T; j += 32) s[j] = expf(s[j] - m) * inv;
  if (lane == 0) lse[row] = m + logf(l);
}

// ------------------------------------------------------------------------ products
// C[b] (M x N) = alpha * op(A[b]) op(B[b]), fp32 in and out, with
// op(A)(m, k) = TA ? A[k * lda + m] : A[m * lda + k];  op(B)(k, n) = TB ? B[n * ldb + k] : B[k * ldb + n].
enum : int { EPI_STORE = 0, EPI_DS = 1, EPI_UNPOOL = 2 };
struct GemmArgs {
  const float* A;
  const float* B;
  float* C;
  long long sA, sB, sC;  // batch strides in elements
  int lda, ldb, ldc;
  int M, N, K;
  float alpha;
  float* aux;            // EPI_DS: scaled scores in, P out (C's layout)
  const float* row_lse;  // EPI_DS: lse_c per row
  const float* row_dlt;  // EPI_DS: delta_c per row
  long long sRow;
  Geom g;                // EPI_UNPOOL: row m is cube m, divided by its valid-token count
  DevStatus* st;         // bounded waits of the tensor-core kernel report here
  unsigned long long timeout_ns;
};

// ------------------------------------------------------------------------ products on the tensor cores
// The same products on tcgen05: each fp32 operand value x enters as the bf16 pair
// hi = bf16(x), lo = bf16(x - hi) (x to about 2^-16 relative), and a product accumulates
// hi*hi + hi*lo + lo*hi in fp32 in tensor memory (the dropped lo*lo term is below 2^-16 of
// |a||b|).  One CTA per 128 x 128 output tile: eight warps load 64-deep k slices of both
// operands from global memory (fp32, coalesced), split them and store them in the 128-byte
// swizzled layouts the MMA reads (K-major when k is the contiguous index of the source,
// MN-major when m or n is), two slices in flight; warp 8 owns tensor memory and issues the
// MMAs; the same eight warps run the epilogue from tensor memory.
namespace cmm {
constexpr int kThreads = 288;
constexpr int BK = 64;                       // k slice
constexpr uint32_t OP_BYTES = 16384;         // one operand part: 128 x 64 bf16
constexpr uint32_t STAGE_BYTES = 4 * OP_BYTES;  // A hi, A lo, B hi, B lo
constexpr uint32_t OFF_BAR = 2 * STAGE_BYTES;
constexpr uint32_t OFF_SLOT = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128 + 1024;
enum { B_FULL = 0, B_EMPTY = 2, B_DONE = 4, NBAR = 5 };
}  // namespace cmm

// bf16 hi and lo of 8 consecutive values as two 16-byte chunks
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
    l[i] = pack_bf16x2(x[2 * i] - __uint_as_float(h[i] << 16), x[2 * i + 1] - __uint_as_float(h[i] & 0xffff0000u));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// 8 consecutive fp32 values of a source row from column c0 (zeros past `ncols`); vec: rows
// 16-byte aligned, so whole float4 loads are legal where they are in range.
__device__ __forceinline__ void load8(const float* row, int c0, int ncols, bool vec, float (&x)[8]) {
  if (vec && c0 + 8 <= ncols) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + c0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(row + c0 + 4));
    x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = c0 + i < ncols ? __ldg(row + c0 + i) : 0.0f;
  }
}

// One operand slice (128 rows of the MMA's M or N by 64 k) into shared memory as hi and lo, in
// two halves so that a caller can issue the loads of both operands before converting either:
// gather_slice loads the thread's four 8-value chunks into registers, store_slice splits and
// stores them.  KMAJ: the source holds row r's k values contiguously (src[r * ld + k]); the
// slice is stored K-major ([128 rows][128 B]).  Otherwise the source holds k row by k row
// (src[k * ld + r]) and the slice is stored MN-major ([2 halves of 64 r][64 k][128 B]).
template <bool KMAJ>
__device__ __forceinline__ void gather_slice(const float* src, int ld, int r0, int rows, int k0, int K, bool vec,
                                             int tid, float (&x)[4][8]) {
#pragma unroll
  for (int it = 0; it < 4; ++it) {  // 256 threads x 4 chunks of 8 values = 128 x 64
    const int u = tid + 256 * it;
    const int outer = KMAJ ? (u >> 3) : (u >> 4);           // row r (K-major) or k row (MN-major)
    const int c0 = KMAJ ? 8 * (u & 7) : 8 * (u & 15);       // first value of the chunk in that row
    const int g_outer = (KMAJ ? r0 : k0) + outer, lim_outer = KMAJ ? rows : K;
    if (g_outer < lim_outer) {
      load8(src + static_cast<long long>(g_outer) * ld, (KMAJ ? k0 : r0) + c0, KMAJ ? K : rows, vec, x[it]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[it][i] = 0.0f;
    }
  }
}

template <bool KMAJ>
__device__ __forceinline__ void store_slice(const float (&x)[4][8], uint32_t s_hi, uint32_t s_lo, int tid) {
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int u = tid + 256 * it;
    const uint32_t off = KMAJ ? sw128_offset(u >> 3, u & 7) : ((u & 15) >> 3) * 8192u + sw128_offset(u >> 4, u & 7);
    uint4 h, l;
    split8(x[it], h, l);
    st_shared_v4(s_hi + off, h.x, h.y, h.z, h.w);
    st_shared_v4(s_lo + off, l.x, l.y, l.z, l.w);
  }
}

// C[b] = alpha * op(A[b]) op(B[b]) with the epilogues of the fp32 kernel; TA / TB as there
// (TA: A is stored k-major by row, i.e. the MMA reads it MN-major).
template <bool TA, bool TB, int EPI>
__global__ void __launch_bounds__(cmm::kThreads, 1) coarse_mma_kernel(GemmArgs p) {
  using namespace cmm;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * 128, n0 = blockIdx.x * 128;
  const long long b = blockIdx.z;
  const float* A = p.A + b * p.sA;
  const float* B = p.B + b * p.sB;
  const int nk = (p.K + BK - 1) / BK;
  if (threadIdx.x == 0) {
    mbar_init(&bars[B_FULL], 256);
    mbar_init(&bars[B_FULL + 1], 256);
    mbar_init(&bars[B_EMPTY], 1);
    mbar_init(&bars[B_EMPTY + 1], 1);
    mbar_init(&bars[B_DONE], 1);
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip_all = aborted(p.st);
  // A is K-major in shared memory unless TA; B (the MMA's N x K operand) is K-major when TB
  const bool vec_a = (p.lda & 3) == 0 && (reinterpret_cast<uintptr_t>(A) & 15) == 0;
  const bool vec_b = (p.ldb & 3) == 0 && (reinterpret_cast<uintptr_t>(B) & 15) == 0;
  if (warp < 8) {
    const int tid = threadIdx.x;
    bool ok = !skip_all;
    for (int c = 0; ok && c < nk; ++c) {
      const int st = c & 1;
      if (c >= 2 && !mbar_wait(&bars[B_EMPTY + st], ((c >> 1) + 1) & 1, p.st, p.timeout_ns, 141)) {
        ok = false;
        break;
      }
      const uint32_t sb = sbase + st * STAGE_BYTES;
      float xa[4][8], xb[4][8];  // both operands' loads in flight before either is converted
      gather_slice<!TA>(A, p.lda, m0, p.M, c * BK, p.K, vec_a, tid, xa);
      gather_slice<TB>(B, p.ldb, n0, p.N, c * BK, p.K, vec_b, tid, xb);
      store_slice<!TA>(xa, sb, sb + OP_BYTES, tid);
      store_slice<TB>(xb, sb + 2 * OP_BYTES, sb + 3 * OP_BYTES, tid);
      fence_proxy_async_smem();  // generic-proxy stores, read next by the tensor cores
      mbar_arrive(&bars[B_FULL + st]);
    }
    // epilogue: warp w reads TMEM lanes 32 (w % 4).. and columns 64 (w / 4)..
    if (ok && mbar_wait(&bars[B_DONE], 0, p.st, p.timeout_ns, 142)) {
      tc_fence_after();
      const int q = warp & 3, ch = warp >> 2;
      const int m = m0 + q * 32 + lane;
      float* C = p.C + b * p.sC;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + ch * 64 + hh * 32, v);
        tmem_ld_wait();
        if (m < p.M) {
          float rs = p.alpha, lse = 0.0f, dlt = 0.0f;
          if (EPI == EPI_UNPOOL) rs = p.alpha / static_cast<float>(cube_valid_count(p.g, m));
          if (EPI == EPI_DS) {
            lse = p.row_lse[b * p.sRow + m];
            dlt = p.row_dlt[b * p.sRow + m];
          }
          const int nb = n0 + ch * 64 + hh * 32;
          const long long o0 = static_cast<long long>(m) * p.ldc + nb;
          float* aux = EPI == EPI_DS ? p.aux + b * p.sC : nullptr;
          if (nb + 32 <= p.N && (p.ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(C) & 15) == 0 &&
              (EPI != EPI_DS || (reinterpret_cast<uintptr_t>(aux) & 15) == 0)) {
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {  // whole float4 rows of 32 columns
              float r[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) r[u] = __uint_as_float(v[4 * j4 + u]);
              if (EPI == EPI_DS) {
                float4* ap = reinterpret_cast<float4*>(aux + o0) + j4;
                const float4 sv = *ap;
                const float pr[4] = {expf(sv.x - lse), expf(sv.y - lse), expf(sv.z - lse), expf(sv.w - lse)};
                *ap = make_float4(pr[0], pr[1], pr[2], pr[3]);
#pragma unroll
                for (int u = 0; u < 4; ++u) r[u] = pr[u] * (r[u] - dlt);
              } else {
#pragma unroll
                for (int u = 0; u < 4; ++u) r[u] *= rs;
              }
              reinterpret_cast<float4*>(C + o0)[j4] = make_float4(r[0], r[1], r[2], r[3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (nb + j >= p.N) break;
              const long long o = o0 + j;
              const float acc = __uint_as_float(v[j]);
              if (EPI == EPI_DS) {
                const float pr = expf(aux[o] - lse);
                aux[o] = pr;
                C[o] = pr * (acc - dlt);
              } else {
                C[o] = acc * rs;
              }
            }
          }
        }
      }
    }
  } else if (!skip_all) {
    // warp 8: the whole warp runs the loop, one elected lane issues
    const uint32_t idesc = make_idesc(128, 128, FMT_BF16, TA, !TB);
    bool ok = true;
    for (int c = 0; c < nk; ++c) {
      const int st = c & 1;
      if (!mbar_wait_warp(&bars[B_FULL + st], (c >> 1) & 1, p.st, p.timeout_ns, 143)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sb = sbase + st * STAGE_BYTES;
      if (elect_one()) {
#pragma unroll
        for (int prod = 0; prod < 3; ++prod) {  // hi*hi, hi*lo, lo*hi
          const uint32_t a_s = sb + (prod == 2 ? OP_BYTES : 0u);
          const uint32_t b_s = sb + 2 * OP_BYTES + (prod == 1 ? OP_BYTES : 0u);
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            // K-major: k step = 32 bytes along the row; MN-major: 16 k rows = 2048 bytes
            const uint64_t ad = TA ? sw128_desc(a_s + ks * 2048, 8192, 1024) : sw128_desc(a_s + ks * 32, 16, 1024);
            const uint64_t bd = TB ? sw128_desc(b_s + ks * 32, 16, 1024) : sw128_desc(b_s + ks * 2048, 8192, 1024);
            umma_f16_ss(tmem, ad, bd, idesc, (c > 0 || prod > 0 || ks > 0) ? 1u : 0u);
          }
        }
        umma_commit(&bars[B_EMPTY + st]);
        if (c == nk - 1) umma_commit(&bars[B_DONE]);
      }
      __syncwarp();
    }
    if (ok) mbar_wait_drain(&bars[B_DONE], 0, p.st, p.timeout_ns, 144);  // every MMA done before TMEM is freed
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) tmem_dealloc(tmem, 128);
}

template <bool TA, bool TB, int EPI>
cudaError_t gemm(const GemmArgs& a, int batch, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    const cudaError_t e =
        cudaFuncSetAttribute(coarse_mma_kernel<TA, TB, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, cmm::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const dim3 grid(static_cast<unsigned>((a.N + 127) / 128), static_cast<unsigned>((a.M + 127) / 128),
                  static_cast<unsigned>(batch));
  coarse_mma_kernel<TA, TB, EPI><<<grid, cmm::kThreads, cmm::SMEM_BYTES, stream>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------ gate backward
// One warp per (bh, cube), four rows per step with all loads issued first.  Per valid row t:
//   dG_t = <dO_t, Oc^>,  Delta_t = <dO_t, O_t> - G_t dG_t  (= <dO_t, O_f,t>),  -lse_t log2(e);
// per cube: dOc^ = sum_t G_t dO_t and delta_c = <dOc^, Oc^>.  Padding rows get dG = Delta = 0.
template <int PER>
__global__ void __launch_bounds__(256) coarse_gate_bwd_kernel(
    const __nv_bfloat16* __restrict__ out, const float* __restrict__ o32, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ gate, const float* __restrict__ oc,
    float* __restrict__ dgate, float* __restrict__ delta, float* __restrict__ nlse2, float* __restrict__ doc,
    float* __restrict__ dltc, Geom g, int BH) {
  constexpr int D = 32 * PER;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long cube = blockIdx.x * 8LL + warp;
  if (cube >= static_cast<long long>(BH) * g.T) return;
  int vt, vh, vw;
  cube_extent(g, static_cast<int>(cube % g.T), vt, vh, vw);
  float ov[PER], acc[PER];
  load_f<PER>(oc + cube * D + lane * PER, ov);
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.0f;
  const long long row0 = cube * 64;
  for (int s0 = 0; s0 < 64; s0 += 4) {
    float y[4][PER], x[4][PER], gt[4];
    bool ok[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long row = row0 + s0 + u;
      ok[u] = slot_valid(vt, vh, vw, s0 + u);
      gt[u] = 0.0f;
#pragma unroll
      for (int e = 0; e < PER; ++e) y[u][e] = x[u][e] = 0.0f;
      if (ok[u]) {
        gt[u] = gate[row];
        load_bf<PER>(dout + row * D + lane * PER, y[u]);
        if (o32) load_f<PER>(o32 + row * D + lane * PER, x[u]);
        else load_bf<PER>(out + row * D + lane * PER, x[u]);
      }
    }
    float dg[4], dd[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dg[u] = dd[u] = 0.0f;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        dg[u] = fmaf(y[u][e], ov[e], dg[u]);
        dd[u] = fmaf(y[u][e], x[u][e], dd[u]);
        acc[e] = fmaf(gt[u], y[u][e], acc[e]);
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        dg[u] += __shfl_xor_sync(0xffffffffu, dg[u], off);
        dd[u] += __shfl_xor_sync(0xffffffffu, dd[u], off);
      }
    if (lane < 4) {
      float a = dg[0], b = dd[0], gg = gt[0];
      bool okk = ok[0];
#pragma unroll
      for (int u = 1; u < 4; ++u)
        if (lane == u) a = dg[u], b = dd[u], gg = gt[u], okk = ok[u];
      const long long row = row0 + s0 + lane;
      dgate[row] = okk ? a : 0.0f;
      delta[row] = okk ? b - gg * a : 0.0f;
      nlse2[row] = -lse[row] * kLog2e;
    }
  }
  store_f<PER>(doc + cube * D + lane * PER, acc);
  float dl = 0.0f;
#pragma unroll
  for (int e = 0; e < PER; ++e) dl = fmaf(acc[e], ov[e], dl);
#pragma unroll
  for (int off = 16; off; off >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, off);
  if (lane == 0) dltc[cube] = dl;
}

}  // namespace

// ------------------------------------------------------------------------ launch
cudaError_t launch_coarse_forward(const void* v, const double* qbar64, const double* kbar64, float* P32,
                                  const CoarseTensors& c, const Geom& g, int BH, int D, DevStatus* st,
                                  unsigned long long timeout_ns, cudaStream_t stream, int* launches) {
  const long long cubes = static_cast<long long>(BH) * g.T;
  const unsigned blocks = static_cast<unsigned>((cubes + 7) / 8);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
  if (D == 128)
    coarse_pool_kernel<4><<<blocks, 256, 0, stream>>>(vb, qbar64, kbar64, c.qbar, c.kbar, c.vbar, g, BH);
  else
    coarse_pool_kernel<2><<<blocks, 256, 0, stream>>>(vb, qbar64, kbar64, c.qbar, c.kbar, c.vbar, g, BH);
  coarse_softmax_kernel<<<blocks, 256, 0, stream>>>(P32, c.lse, cubes, g.T);
  GemmArgs a{};
  a.A = P32, a.B = c.vbar, a.C = c.oc;
  a.sA = static_cast<long long>(g.T) * g.T, a.sB = static_cast<long long>(g.T) * D, a.sC = a.sB;
  a.lda = g.T, a.ldb = D, a.ldc = D;
  a.M = g.T, a.N = D, a.K = g.T;
  a.alpha = 1.0f;
  a.g = g;
  a.st = st;
  a.timeout_ns = timeout_ns;
  cudaError_t e = gemm<false, false, EPI_STORE>(a, BH, stream);
  *launches = 3;
  return e;
}

cudaError_t launch_coarse_backward(const void* out, const float* out_f32, const void* dout, const float* lse,
                                   const float* gate, const CoarseTensors& c, float* dgate, float* delta,
                                   float* nlse2, const CoarseGradWs& w, float scale, const Geom& g, int BH, int D,
                                   DevStatus* st, unsigned long long timeout_ns, cudaStream_t stream, int* launches) {
  const long long cubes = static_cast<long long>(BH) * g.T;
  const unsigned blocks = static_cast<unsigned>((cubes + 7) / 8);
  const __nv_bfloat16* ob = static_cast<const __nv_bfloat16*>(out);
  const __nv_bfloat16* db = static_cast<const __nv_bfloat16*>(dout);
  if (D == 128)
    coarse_gate_bwd_kernel<4><<<blocks, 256, 0, stream>>>(ob, out_f32, db, lse, gate, c.oc, dgate, delta, nlse2,
                                                          w.doc, w.dltc, g, BH);
  else
    coarse_gate_bwd_kernel<2><<<blocks, 256, 0, stream>>>(ob, out_f32, db, lse, gate, c.oc, dgate, delta, nlse2,
                                                          w.doc, w.dltc, g, BH);
  const long long TT = static_cast<long long>(g.T) * g.T, TD = static_cast<long long>(g.T) * D;
  cudaError_t e = cudaGetLastError();
  // S = scale * Qc Kc^T
  GemmArgs a{};
  a.A = c.qbar, a.B = c.kbar, a.C = w.s;
  a.sA = TD, a.sB = TD, a.sC = TT;
  a.lda = D, a.ldb = D, a.ldc = g.T;
  a.M = g.T, a.N = g.T, a.K = D;
  a.alpha = scale;
  a.g = g;
  a.st = st;
  a.timeout_ns = timeout_ns;
  if (e == cudaSuccess) e = gemm<false, true, EPI_STORE>(a, BH, stream);
  // dP = dOc^ Vc^T;  P = exp(S - lse_c) over S;  dS = P (dP - delta_c)
  GemmArgs d = a;
  d.A = w.doc, d.B = c.vbar, d.C = w.ds;
  d.alpha = 1.0f;
  d.aux = w.s, d.row_lse = c.lse, d.row_dlt = w.dltc, d.sRow = g.T;
  if (e == cudaSuccess) e = gemm<false, true, EPI_DS>(d, BH, stream);
  // dQc / n = scale * dS Kc / n
  GemmArgs q{};
  q.A = w.ds, q.B = c.kbar, q.C = w.cq;
  q.sA = TT, q.sB = TD, q.sC = TD;
  q.lda = g.T, q.ldb = D, q.ldc = D;
  q.M = g.T, q.N = D, q.K = g.T;
  q.alpha = scale;
  q.g = g;
  q.st = st;
  q.timeout_ns = timeout_ns;
  if (e == cudaSuccess) e = gemm<false, false, EPI_UNPOOL>(q, BH, stream);
  // dKc / n = scale * dS^T Qc / n
  GemmArgs k = q;
  k.B = c.qbar, k.C = w.ck;
  if (e == cudaSuccess) e = gemm<true, false, EPI_UNPOOL>(k, BH, stream);
  // dVc / n = P^T dOc^ / n
  GemmArgs vv = q;
  vv.A = w.s, vv.B = w.doc, vv.C = w.cv;
  vv.alpha = 1.0f;
  if (e == cudaSuccess) e = gemm<true, false, EPI_UNPOOL>(vv, BH, stream);
  *launches = 6;
  return e;
}

}  // namespace sa
