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
//   coarse_gemm_kernel      batched fp32 products of the cube-level matrices, with the
//                           epilogues the branch needs (plain, dS = P (dP - delta), and
//                           the mean-pool adjoint 1/n per cube)
//   coarse_combine_kernel   O = G * Oc^[cube] + O_f on the valid rows, in place
//   coarse_gate_bwd_kernel  one pass over dO: dG, the fine branch's Delta and -lse*log2(e),
//                           dOc^ = sum_t G_t dO_t and delta_c = <dOc^, Oc^> per cube
//
// The cube-level matrices are T x T per head (T = 1440 at the 720p shape), so the six products
// of a forward and backward are about 1/250 of the fine stage's FLOPs at 95% sparsity; they run
// on the fp32 FMA pipe, which keeps the branch within fp32 rounding of the fp64 definition.
#include <cuda_bf16.h>

#include <cmath>

#include "geometry.cuh"
#include "kernels.h"

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
// One warp per cube row: max, sum of exp(s - max), then P = exp(s - max) / sum.  The row
// (T doubles) is read three times; after the first pass it comes from L1/L2.
__global__ void __launch_bounds__(256) coarse_softmax_kernel(const double* __restrict__ S, float* __restrict__ P,
                                                             float* __restrict__ lse, long long rows, int T) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x * 8LL + warp;
  if (row >= rows) return;
  const double* s = S + row * T;
  double m = -INFINITY;
  for (int j = lane; j < T; j += 32) m = fmax(m, s[j]);
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
  float l = 0.0f;
  for (int j = lane; j < T; j += 32) l += expf(static_cast<float>(s[j] - m));
#pragma unroll
  for (int off = 16; off; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  const float inv = 1.0f / l;
  float* p = P + row * T;
  for (int j = lane; j < T; j += 32) p[j] = expf(static_cast<float>(s[j] - m)) * inv;
  if (lane == 0) lse[row] = static_cast<float>(m) + logf(l);
}

// ------------------------------------------------------------------------ products
// C[b] (M x N) = alpha * op(A[b]) op(B[b]), fp32, 64 x 64 tiles, 16-deep k slices, 4 x 4
// outputs per thread, the next slice loaded into registers while the current one is used.
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
};

constexpr int GBM = 64, GBN = 64, GBK = 16, GPAD = 4;

template <bool TA, bool TB, int EPI>
__global__ void __launch_bounds__(256) coarse_gemm_kernel(GemmArgs p) {
  __shared__ __align__(16) float As[2][GBK][GBM + GPAD];
  __shared__ __align__(16) float Bs[2][GBK][GBN + GPAD];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * GBM, n0 = blockIdx.x * GBN;
  const long long b = blockIdx.z;
  const float* A = p.A + b * p.sA;
  const float* B = p.B + b * p.sB;
  float ra[4], rb[4];
  // element i of this thread's share of the A slice: (m, k) within the tile
  auto a_pos = [&](int i, int& m, int& k) {
    const int idx = tid + 256 * i;
    if (TA) k = idx >> 6, m = idx & 63;
    else m = idx >> 4, k = idx & 15;
  };
  auto b_pos = [&](int i, int& k, int& n) {
    const int idx = tid + 256 * i;
    if (TB) n = idx >> 4, k = idx & 15;
    else k = idx >> 6, n = idx & 63;
  };
  auto load = [&](int k0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int m, k, n, kb;
      a_pos(i, m, k);
      const int gm = m0 + m, gk = k0 + k;
      ra[i] = (gm < p.M && gk < p.K) ? (TA ? A[static_cast<long long>(gk) * p.lda + gm]
                                            : A[static_cast<long long>(gm) * p.lda + gk])
                                     : 0.0f;
      b_pos(i, kb, n);
      const int gn = n0 + n, gkb = k0 + kb;
      rb[i] = (gn < p.N && gkb < p.K) ? (TB ? B[static_cast<long long>(gn) * p.ldb + gkb]
                                             : B[static_cast<long long>(gkb) * p.ldb + gn])
                                      : 0.0f;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int m, k, n, kb;
      a_pos(i, m, k);
      As[buf][k][m] = ra[i];
      b_pos(i, kb, n);
      Bs[buf][kb][n] = rb[i];
    }
  };
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  const int nk = (p.K + GBK - 1) / GBK;
  load(0);
  store(0);
  __syncthreads();
  for (int t = 0; t < nk; ++t) {
    const int cur = t & 1;
    if (t + 1 < nk) load((t + 1) * GBK);
#pragma unroll
    for (int k = 0; k < GBK; ++k) {
      const float4 a4 = *reinterpret_cast<const float4*>(&As[cur][k][ty * 4]);
      const float4 b4 = *reinterpret_cast<const float4*>(&Bs[cur][k][tx * 4]);
      const float a[4] = {a4.x, a4.y, a4.z, a4.w}, bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    // the other buffer was last read before the previous barrier
    if (t + 1 < nk) store(cur ^ 1);
    __syncthreads();
  }
  float* C = p.C + b * p.sC;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= p.M) continue;
    float rs = p.alpha, lse = 0.0f, dlt = 0.0f;
    if (EPI == EPI_UNPOOL) rs = p.alpha / static_cast<float>(cube_valid_count(p.g, m));
    if (EPI == EPI_DS) {
      lse = p.row_lse[b * p.sRow + m];
      dlt = p.row_dlt[b * p.sRow + m];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= p.N) continue;
      const long long o = static_cast<long long>(m) * p.ldc + n;
      if (EPI == EPI_DS) {
        float* aux = p.aux + b * p.sC;
        const float pr = expf(aux[o] - lse);
        aux[o] = pr;
        C[o] = pr * (acc[i][j] - dlt);
      } else {
        C[o] = acc[i][j] * rs;
      }
    }
  }
}

template <bool TA, bool TB, int EPI>
cudaError_t gemm(const GemmArgs& a, int batch, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((a.N + GBN - 1) / GBN), static_cast<unsigned>((a.M + GBM - 1) / GBM),
                  static_cast<unsigned>(batch));
  coarse_gemm_kernel<TA, TB, EPI><<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------ combine
// O = G * Oc^[cube] + O_f on valid rows, in place on the bf16 output and, when present, its
// fp32 copy (then the bf16 value is the rounded fp32 sum; the C ABI always passes the copy).
// One thread per 4 columns of a row.
__global__ void __launch_bounds__(256) coarse_combine_kernel(__nv_bfloat16* __restrict__ out,
                                                             float* __restrict__ o32, const float* __restrict__ gate,
                                                             const float* __restrict__ oc, Geom g, int BH, int D) {
  const int q4 = D >> 2;
  const long long u = blockIdx.x * 256LL + threadIdx.x;
  const long long rows = static_cast<long long>(BH) * g.Npad;
  if (u >= rows * q4) return;
  const long long row = u / q4;
  const int c = static_cast<int>(u % q4) * 4;
  const int bh = static_cast<int>(row / g.Npad), slot = static_cast<int>(row % g.Npad);
  if (!token_valid(g, slot >> 6, slot & 63)) return;  // padding rows stay 0
  const float gv = gate[row];
  const float4 ov = *reinterpret_cast<const float4*>(oc + (static_cast<long long>(bh) * g.T + (slot >> 6)) * D + c);
  float x[4];
  if (o32) {
    load_f<4>(o32 + row * D + c, x);
  } else {
    load_bf<4>(out + row * D + c, x);
  }
  x[0] = fmaf(gv, ov.x, x[0]);
  x[1] = fmaf(gv, ov.y, x[1]);
  x[2] = fmaf(gv, ov.z, x[2]);
  x[3] = fmaf(gv, ov.w, x[3]);
  if (o32) store_f<4>(o32 + row * D + c, x);
  const __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]), hi = __floats2bfloat162_rn(x[2], x[3]);
  uint2 w;
  w.x = *reinterpret_cast<const uint32_t*>(&lo);
  w.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + row * D + c) = w;
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
cudaError_t launch_coarse_forward(const void* v, const double* qbar64, const double* kbar64, const double* S64,
                                  float* P32, const CoarseTensors& c, const Geom& g, int BH, int D,
                                  cudaStream_t stream, int* launches) {
  const long long cubes = static_cast<long long>(BH) * g.T;
  const unsigned blocks = static_cast<unsigned>((cubes + 7) / 8);
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
  if (D == 128)
    coarse_pool_kernel<4><<<blocks, 256, 0, stream>>>(vb, qbar64, kbar64, c.qbar, c.kbar, c.vbar, g, BH);
  else
    coarse_pool_kernel<2><<<blocks, 256, 0, stream>>>(vb, qbar64, kbar64, c.qbar, c.kbar, c.vbar, g, BH);
  coarse_softmax_kernel<<<blocks, 256, 0, stream>>>(S64, P32, c.lse, cubes, g.T);
  GemmArgs a{};
  a.A = P32, a.B = c.vbar, a.C = c.oc;
  a.sA = static_cast<long long>(g.T) * g.T, a.sB = static_cast<long long>(g.T) * D, a.sC = a.sB;
  a.lda = g.T, a.ldb = D, a.ldc = D;
  a.M = g.T, a.N = D, a.K = g.T;
  a.alpha = 1.0f;
  a.g = g;
  cudaError_t e = gemm<false, false, EPI_STORE>(a, BH, stream);
  *launches = 3;
  return e;
}

cudaError_t launch_coarse_combine(void* out, float* out_f32, const float* gate, const float* oc, const Geom& g,
                                  int BH, int D, cudaStream_t stream) {
  const long long units = static_cast<long long>(BH) * g.Npad * (D / 4);
  coarse_combine_kernel<<<static_cast<unsigned>((units + 255) / 256), 256, 0, stream>>>(
      static_cast<__nv_bfloat16*>(out), out_f32, gate, oc, g, BH, D);
  return cudaGetLastError();
}

cudaError_t launch_coarse_backward(const void* out, const float* out_f32, const void* dout, const float* lse,
                                   const float* gate, const CoarseTensors& c, float* dgate, float* delta,
                                   float* nlse2, const CoarseGradWs& w, float scale, const Geom& g, int BH, int D,
                                   cudaStream_t stream, int* launches) {
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
