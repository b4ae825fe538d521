// C ABI of libsa: argument validation, workspace carving, TMA descriptors and launches.
// Every check here runs on the host before anything is launched.
#include <cmath>
#include <cstring>

#include "../../include/sa.h"
#include "attn_common.cuh"
#include "kernels.h"

namespace {

using sa::Geom;

thread_local int g_last_launches = 0;

constexpr size_t kHeader = 256;
// forward / backward: per-CTA clock records of the three attention kernels after the header
constexpr size_t kClockBytes = 3ull * sa::kClockCtas * 4 * sizeof(unsigned long long);

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool make_geom(const sa_params* p, Geom* g) {
  if (!p || p->lat_t < 1 || p->lat_h < 1 || p->lat_w < 1) return false;
  g->lat_t = p->lat_t;
  g->lat_h = p->lat_h;
  g->lat_w = p->lat_w;
  g->Nt = (p->lat_t + 3) / 4;
  g->Nh = (p->lat_h + 3) / 4;
  g->Nw = (p->lat_w + 3) / 4;
  const long long T = static_cast<long long>(g->Nt) * g->Nh * g->Nw;
  if (T > (1 << 20)) return false;
  g->T = static_cast<int>(T);
  g->Npad = g->T * 64;
  return true;
}

// Shape checks common to all ops.
sa_status check_params(const sa_params* p, Geom* g) {
  if (!p) return SA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || !make_geom(p, g)) return SA_ERR_INVALID_ARG;
  if (p->D != 64 && p->D != 128) return SA_ERR_UNSUPPORTED;
  if (g->T > 8192) return SA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(p->B) * p->H;
  if (BH * g->Npad >= (1LL << 31) - 64) return SA_ERR_UNSUPPORTED;
  if (p->top_k < 0 || !std::isfinite(p->top_p)) return SA_ERR_INVALID_ARG;
  if (p->kv_capacity < 1 || p->kv_capacity > g->T) return SA_ERR_INVALID_ARG;
  if (BH * g->T * static_cast<long long>(p->kv_capacity) >= (1LL << 31)) return SA_ERR_UNSUPPORTED;
  if (p->qk_dtype != SA_BF16 && p->qk_dtype != SA_FP8_E4M3) return SA_ERR_INVALID_ARG;
  if (!std::isfinite(p->softmax_scale) || p->softmax_scale < 0.0f) return SA_ERR_INVALID_ARG;
  return SA_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
bool aligned4(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

double softmax_scale(const sa_params* p) {
  return p->softmax_scale > 0.0f ? static_cast<double>(p->softmax_scale) : 1.0 / std::sqrt(static_cast<double>(p->D));
}

int union_cap(const sa_params* p, const Geom& g) { return 2 * p->kv_capacity < g.T ? 2 * p->kv_capacity : g.T; }

struct WsLayout {
  size_t cmask = 0;                                        // forward, backward: [T] cube masks
  size_t ulist = 0, ucnt = 0;                              // forward: query-pair union lists
  size_t v16 = 0;                                          // forward: fp16 copy of V
  size_t qbar = 0, kbar = 0, scores = 0;                   // plan
  size_t delta = 0, nlse2 = 0, bits = 0;                  // backward
  size_t ukcnt = 0, uklist = 0;                            // backward: key-pair unions
  size_t h16[4] = {0, 0, 0, 0};                            // backward: fp16 copies of Q, K, V, dO
  size_t p32 = 0;                                          // plan + coarse: Pc [BH, T, T] fp32
  size_t doc = 0, dltc = 0, s32 = 0, ds32 = 0;             // gated backward: coarse scratch
  size_t cq = 0, ck = 0, cv = 0;
  size_t qpair = 0, blk_index = 0, blk_count = 0;          // plan with 128-token query blocks
  size_t qlimb = 0, klimb = 0, qexp = 0, kexp = 0, ql1 = 0;  // plan on the tensor cores
  size_t kexpmax = 0, meta = 0, keys = 0, flist = 0, rkmax = 0, rkmin = 0;
  int Tk = 0;
  size_t total = 0;
};

// The routers that keep every fp64 score (the coarse branch reads them; the 128-token block
// router scores blocks of two cubes): status, Qbar, Kbar, S [BH, T, T] fp64.
constexpr int kOpPlanFp64 = 100;

WsLayout ws_layout(const sa_params* p, const Geom& g, int op) {
  WsLayout w;
  const size_t BH = static_cast<size_t>(p->B) * p->H;
  if (op == SA_OP_PLAN_BQ128) {
    // the fp64 plan's (the score rows of the first ceil(T/2) blocks are used), then the block means and lists
    w = ws_layout(p, g, kOpPlanFp64);
    const size_t M = static_cast<size_t>((g.T + 1) / 2);
    size_t off = w.total;
    w.qpair = off;
    off = align256(off + BH * M * p->D * sizeof(double));
    w.blk_count = off;
    off = align256(off + BH * M * sizeof(int32_t));
    w.blk_index = off;
    off = align256(off + BH * M * static_cast<size_t>(p->kv_capacity) * sizeof(int32_t));
    w.total = off;
    return w;
  }
  if (op == SA_OP_PLAN_COARSE || op == SA_OP_BACKWARD_GATED) {
    // the plain layout, then the coarse branch's buffers
    w = ws_layout(p, g, op == SA_OP_PLAN_COARSE ? SA_OP_PLAN : SA_OP_BACKWARD);
    const size_t TT = BH * g.T * static_cast<size_t>(g.T) * sizeof(float);
    const size_t TD = BH * g.T * static_cast<size_t>(p->D) * sizeof(float);
    size_t off = w.total;
    if (op == SA_OP_PLAN_COARSE) {
      w.p32 = off;
      off = align256(off + TT);
    } else {
      w.doc = off;
      off = align256(off + TD);
      w.dltc = off;
      off = align256(off + BH * g.T * sizeof(float));
      w.s32 = off;
      off = align256(off + TT);
      w.ds32 = off;
      off = align256(off + TT);
      w.cq = off;
      off = align256(off + TD);
      w.ck = off;
      off = align256(off + TD);
      w.cv = off;
      off = align256(off + TD);
    }
    w.total = off;
    return w;
  }
  size_t off = kHeader;
  if (op == SA_OP_PLAN) {
    const size_t rows = BH * g.T;
    w.qbar = off;
    off = align256(off + rows * p->D * sizeof(double));
    w.kbar = off;
    off = align256(off + rows * p->D * sizeof(double));
    w.qlimb = off;
    off = align256(off + BH * 4 * g.T * 128);
    w.klimb = off;
    off = align256(off + BH * 4 * g.T * 128);
    w.qexp = off;
    off = align256(off + rows * sizeof(int));
    w.kexp = off;
    off = align256(off + BH * static_cast<size_t>((g.T + 3) & ~3) * sizeof(int));
    w.ql1 = off;
    off = align256(off + rows * sizeof(double));
    w.kexpmax = off;
    off = align256(off + BH * sizeof(unsigned));
    w.meta = off;
    off = align256(off + rows * 32);
    w.Tk = (g.T + 3) & ~3;
    w.keys = off;
    off = align256(off + rows * static_cast<size_t>(w.Tk) * sizeof(int));
    w.flist = off;
    off = align256(off + rows * sizeof(int));
    w.rkmax = off;
    off = align256(off + rows * sizeof(int));
    w.rkmin = off;
    off = align256(off + rows * sizeof(int));
  } else if (op == kOpPlanFp64) {
    w.qbar = off;
    off = align256(off + BH * g.T * p->D * sizeof(double));
    w.kbar = off;
    off = align256(off + BH * g.T * p->D * sizeof(double));
    w.scores = off;
    off = align256(off + BH * g.T * static_cast<size_t>(g.T) * sizeof(double));
  } else if (op == SA_OP_BLOCK_MASS) {
    w.cmask = off;
    off = align256(off + static_cast<size_t>(g.T) * sizeof(unsigned long long));
  } else if (op == SA_OP_FORWARD) {
    off += kClockBytes;
    w.cmask = off;
    off = align256(off + static_cast<size_t>(g.T) * sizeof(unsigned long long));
    const size_t P = static_cast<size_t>((g.T + 1) / 2);
    w.ucnt = off;
    off = align256(off + BH * P * sizeof(int32_t));
    w.ulist = off;
    off = align256(off + BH * P * static_cast<size_t>(union_cap(p, g)) * sizeof(int32_t));
    w.v16 = off;  // fp16 copy of V for the single-product P V when the fp32 output is kept
    off = align256(off + BH * g.Npad * static_cast<size_t>(p->D) * 2);
  } else if (op == SA_OP_BACKWARD) {
    off += kClockBytes;
    w.cmask = off;
    off = align256(off + static_cast<size_t>(g.T) * sizeof(unsigned long long));
    w.delta = off;
    off = align256(off + BH * g.Npad * sizeof(float));
    w.nlse2 = off;
    off = align256(off + BH * g.Npad * sizeof(float));
    w.bits = off;  // selection bit matrix [BH, T, ceil(T/32)]
    off = align256(off + BH * g.T * static_cast<size_t>((g.T + 31) / 32) * sizeof(uint32_t));
    const size_t P = static_cast<size_t>((g.T + 1) / 2);
    w.ucnt = off;
    off = align256(off + BH * P * sizeof(int32_t));
    w.ulist = off;
    off = align256(off + BH * P * static_cast<size_t>(union_cap(p, g)) * sizeof(int32_t));
    w.ukcnt = off;
    off = align256(off + BH * P * sizeof(int32_t));
    w.uklist = off;
    off = align256(off + BH * P * static_cast<size_t>(g.T) * sizeof(int32_t));
    for (int t = 0; t < 4; ++t) {  // fp16 copies for the single-product path
      w.h16[t] = off;
      off = align256(off + BH * g.Npad * static_cast<size_t>(p->D) * 2);
    }
  }
  w.total = off;
  return w;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D map over [rows][D] elements with 64-row boxes of 128 bytes, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, long long rows, int D, int esize) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType dt = esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), 64};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over limb rows {128 bytes, T rows, BH*4 slabs}: 128 x 128 boxes, 128-byte swizzle;
// rows past T read as zeros.
bool make_limb_map(CUtensorMap* m, const void* base, int T, long long slabs) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(slabs)};
  cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(T) * 128};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the router's keys {T columns, T rows, BH heads} (int32, row stride Tk): 32 x 32
// boxes with the 128-byte swizzle; rows and columns past T are outside the map.
bool make_keys_map(CUtensorMap* m, void* base, int T, int Tk, int BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(Tk) * 4, static_cast<cuuint64_t>(T) * Tk * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_INT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

sa_status reset_status(void* ws, cudaStream_t s) {
  return cudaMemsetAsync(ws, 0, kHeader, s) == cudaSuccess ? SA_OK : SA_ERR_LAUNCH;
}

unsigned long long timeout_ns_of(const sa_params* p) {
  const unsigned ms = p->timeout_ms ? p->timeout_ms : 2000u;
  return static_cast<unsigned long long>(ms) * 1000000ull;
}

sa::AttnArgs base_args(const sa_params* p, const Geom& g, void* ws) {
  sa::AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.g = g;
  a.BH = p->B * p->H;
  a.D = p->D;
  a.cap = p->kv_capacity;
  a.rows_total = a.BH * g.Npad;
  const double sc = softmax_scale(p);
  a.scale = static_cast<float>(sc);
  a.scale_log2 = static_cast<float>(sc * 1.4426950408889634);
  const unsigned ms = p->timeout_ms ? p->timeout_ms : 2000u;
  a.timeout_ns = static_cast<unsigned long long>(ms) * 1000000ull;
  a.debug = p->debug_flags;
  a.st = static_cast<sa::DevStatus*>(ws);
  a.item_next = a.st->item_next;
  if (p->debug_flags & SA_DEBUG_CTA_CLOCKS) {  // forward and backward workspaces hold the records
    a.cta_clock = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(ws) + kHeader);
    a.clock_grid = a.st->grid;
  }
  return a;
}

}  // namespace

namespace sa {

// the launch count sa_last_launch_count reports, for entry points defined in other files
void set_last_launches(int n) { g_last_launches = n; }

// sa_plan's host-side argument checks (nothing touches the device); *ws_needed receives the
// workspace size the router needs.
sa_status plan_check(const void* q, const void* k, const float* q_scale, const float* k_scale, const sa_params* p,
                     const int32_t* kv_index, const int32_t* kv_count, size_t* ws_needed) {
  Geom g;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!q || !k || !kv_index || !kv_count) return SA_ERR_INVALID_ARG;
  const bool fp8 = p->qk_dtype == SA_FP8_E4M3;
  if (fp8 && (!q_scale || !k_scale)) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned4(kv_index) || !aligned4(kv_count)) return SA_ERR_ALIGNMENT;
  if (fp8 && (!aligned4(q_scale) || !aligned4(k_scale))) return SA_ERR_ALIGNMENT;
  *ws_needed = ws_layout(p, g, SA_OP_PLAN).total;
  return SA_OK;
}

// The same checks, then the workspace carving and launches of sa_plan on the scratch `ws`
// (a caller's workspace, or the fixed array of sa_plan_static); records the launch count.
sa_status plan_on_scratch(const void* q, const void* k, const float* q_scale, const float* k_scale,
                          const sa_params* p, int32_t* kv_index, int32_t* kv_count, void* ws, size_t ws_bytes,
                          cudaStream_t st, float* s32) {
  g_last_launches = 0;
  size_t need = 0;
  sa_status s = plan_check(q, k, q_scale, k_scale, p, kv_index, kv_count, &need);
  if (s != SA_OK) return s;
  Geom g;
  make_geom(p, &g);
  const bool fp8 = p->qk_dtype == SA_FP8_E4M3;
  const WsLayout w = ws_layout(p, g, SA_OP_PLAN);
  if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SA_ERR_ALIGNMENT;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  const int BH = p->B * p->H;
  PlanFastWs f;
  f.qbar = reinterpret_cast<double*>(wb + w.qbar);
  f.kbar = reinterpret_cast<double*>(wb + w.kbar);
  f.qlimb = reinterpret_cast<int8_t*>(wb + w.qlimb);
  f.klimb = reinterpret_cast<int8_t*>(wb + w.klimb);
  f.qexp = reinterpret_cast<int*>(wb + w.qexp);
  f.kexp = reinterpret_cast<int*>(wb + w.kexp);
  f.ql1 = reinterpret_cast<double*>(wb + w.ql1);
  f.kexp_max = reinterpret_cast<unsigned*>(wb + w.kexpmax);
  f.meta = wb + w.meta;
  f.keys = reinterpret_cast<int*>(wb + w.keys);
  f.Tk = w.Tk;
  f.flist = reinterpret_cast<int*>(wb + w.flist);
  f.rkmax = reinterpret_cast<int*>(wb + w.rkmax);
  f.rkmin = reinterpret_cast<int*>(wb + w.rkmin);
  f.s32 = s32;
  CUtensorMap tq, tk, tkeys;
  if (!make_limb_map(&tq, f.qlimb, g.T, 4LL * BH) || !make_limb_map(&tk, f.klimb, g.T, 4LL * BH) ||
      !make_keys_map(&tkeys, f.keys, g.T, f.Tk, BH))
    return SA_ERR_LAUNCH;
  if (reset_status(ws, st) != SA_OK) return SA_ERR_LAUNCH;
  const unsigned ms = p->timeout_ms ? p->timeout_ms : 2000u;
  int launches = 0;
  if (launch_plan_fast(q, k, q_scale, k_scale, tq, tk, tkeys, g, BH, p->D, fp8, softmax_scale(p), p->top_k, p->top_p,
                       p->kv_capacity, p->debug_flags, static_cast<unsigned long long>(ms) * 1000000ull, f, kv_index,
                       kv_count, static_cast<DevStatus*>(ws), st, &launches) != cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = launches;
  return SA_OK;
}

}  // namespace sa

extern "C" {

int sa_padded_tokens(const sa_params* p) {
  Geom g;
  return make_geom(p, &g) ? g.Npad : 0;
}

int sa_num_cubes(const sa_params* p) {
  Geom g;
  return make_geom(p, &g) ? g.T : 0;
}

int sa_topk_from_fraction(double frac, int T) {
  if (!(frac >= 0.0) || T < 0) return 0;
  return static_cast<int>(std::ceil(frac * T - 1e-12));
}

size_t sa_workspace_size(const sa_params* p, int op) {
  Geom g;
  if (check_params(p, &g) != SA_OK || op < SA_OP_PLAN || op > SA_OP_BLOCK_MASS) return 0;
  return ws_layout(p, g, op).total;
}

static sa_status tile_common(const void* src, void* dst, const sa_params* p, int elem_bytes, sa_stream_t stream,
                             bool to_tiled) {
  Geom g;
  g_last_launches = 0;
  if (!p || !src || !dst || p->B < 1 || p->H < 1 || !make_geom(p, &g)) return SA_ERR_INVALID_ARG;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4) return SA_ERR_INVALID_ARG;
  if (p->D < 1) return SA_ERR_INVALID_ARG;
  const int row_bytes = p->D * elem_bytes;
  if (row_bytes % 16 != 0) return SA_ERR_UNSUPPORTED;
  if (!aligned16(src) || !aligned16(dst)) return SA_ERR_ALIGNMENT;
  if (sa::launch_tile(src, dst, g, p->B * p->H, row_bytes, to_tiled, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = 1;
  return SA_OK;
}

static sa_status tile_rope_common(const void* src, void* dst, const sa_params* p, int elem_bytes, int dt, int dh,
                                  int dw, const float* cs, const float* sn, sa_stream_t stream, bool to_tiled) {
  Geom g;
  g_last_launches = 0;
  if (!p || !src || !dst || !cs || !sn || p->B < 1 || p->H < 1 || !make_geom(p, &g)) return SA_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return SA_ERR_INVALID_ARG;
  if (dt < 0 || dh < 0 || dw < 0 || (dt | dh | dw) & 1 || p->D < 2 || dt + dh + dw != p->D) return SA_ERR_INVALID_ARG;
  if ((p->D * elem_bytes) % 16 != 0) return SA_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->B) * p->H * g.Npad * p->D >= (1LL << 40)) return SA_ERR_UNSUPPORTED;
  if (!aligned16(src) || !aligned16(dst) || !aligned4(cs) || !aligned4(sn)) return SA_ERR_ALIGNMENT;
  if (sa::launch_tile_rope(src, dst, g, p->B * p->H, p->D, elem_bytes, to_tiled, dt, dh, dw, cs, sn,
                           reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = 1;
  return SA_OK;
}

sa_status sa_tile_rope(const void* x_latent, void* x_tiled, const sa_params* p, int elem_bytes, int rope_dt,
                       int rope_dh, int rope_dw, const float* rope_cos, const float* rope_sin, sa_stream_t stream) {
  return tile_rope_common(x_latent, x_tiled, p, elem_bytes, rope_dt, rope_dh, rope_dw, rope_cos, rope_sin, stream,
                          true);
}

sa_status sa_untile_rope(const void* x_tiled, void* x_latent, const sa_params* p, int elem_bytes, int rope_dt,
                         int rope_dh, int rope_dw, const float* rope_cos, const float* rope_sin, sa_stream_t stream) {
  return tile_rope_common(x_tiled, x_latent, p, elem_bytes, rope_dt, rope_dh, rope_dw, rope_cos, rope_sin, stream,
                          false);
}

sa_status sa_tile(const void* x_latent, void* x_tiled, const sa_params* p, int elem_bytes, sa_stream_t stream) {
  return tile_common(x_latent, x_tiled, p, elem_bytes, stream, true);
}

sa_status sa_untile(const void* x_tiled, void* x_latent, const sa_params* p, int elem_bytes, sa_stream_t stream) {
  return tile_common(x_tiled, x_latent, p, elem_bytes, stream, false);
}

sa_status sa_plan(const void* q, const void* k, const float* q_scale, const float* k_scale, const sa_params* p,
                  int32_t* kv_index, int32_t* kv_count, void* ws, size_t ws_bytes, sa_stream_t stream) {
  return sa::plan_on_scratch(q, k, q_scale, k_scale, p, kv_index, kv_count, ws, ws_bytes,
                             reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// sa_forward, and with `gate` / `oc` set sa_forward_gated (the combination in the epilogue).
sa_status forward_impl(const void* q, const void* k, const void* v, const float* q_scale, const float* k_scale,
                       const int32_t* kv_index, const int32_t* kv_count, const sa_params* p, void* out, float* lse,
                       float* out_f32, const float* gate, const float* oc, void* ws, size_t ws_bytes,
                       sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!q || !k || !v || !kv_index || !kv_count || !out || !lse) return SA_ERR_INVALID_ARG;
  const bool fp8 = p->qk_dtype == SA_FP8_E4M3;
  if (fp8 && p->D != 128) return SA_ERR_UNSUPPORTED;  // one 128-byte e4m3 row per token
  if (fp8 && (!q_scale || !k_scale)) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(lse) || !aligned4(kv_index) ||
      !aligned4(kv_count) || (out_f32 && !aligned16(out_f32)) || (fp8 && (!aligned4(q_scale) || !aligned4(k_scale))))
    return SA_ERR_ALIGNMENT;
  const WsLayout w = ws_layout(p, g, SA_OP_FORWARD);
  if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SA_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  sa::AttnArgs a = base_args(p, g, ws);
  a.kv_index = kv_index;
  a.kv_count = kv_count;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.out_f32 = out_f32;
  a.lse = lse;
  a.gate = gate;
  a.oc = oc;
  a.qk_fp8 = fp8 ? 1 : 0;
  if (fp8) {
    a.q_scale = q_scale;
    a.k_scale = k_scale;
  }
  const int qk_esize = fp8 ? 1 : 2;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, a.rows_total, p->D, qk_esize) || !make_map(&tk, k, a.rows_total, p->D, qk_esize) ||
      !make_map(&tv, v, a.rows_total, p->D, 2))
    return SA_ERR_LAUNCH;
  if (reset_status(ws, st) != SA_OK) return SA_ERR_LAUNCH;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  a.cube_mask = reinterpret_cast<unsigned long long*>(wb + w.cmask);
  a.u_list = reinterpret_cast<int32_t*>(wb + w.ulist);
  a.u_cnt = reinterpret_cast<int32_t*>(wb + w.ucnt);
  a.ucap = union_cap(p, g);
  if (sa::launch_cube_mask(g, reinterpret_cast<unsigned long long*>(wb + w.cmask), st) != cudaSuccess ||
      sa::launch_query_pair_union(kv_index, kv_count, reinterpret_cast<int32_t*>(wb + w.ulist),
                                  reinterpret_cast<int32_t*>(wb + w.ucnt), a.BH, g.T, p->kv_capacity, a.st,
                                  st) != cudaSuccess)
    return SA_ERR_LAUNCH;
  CUtensorMap tv16 = tv;
  int extra = 0;
  if (out_f32) {
    // fp16 copy of V (and a range flag in the status block) for the single fp16 P V product
    void* v16 = wb + w.v16;
    a.f16_bad = &static_cast<sa::DevStatus*>(ws)->f16_out_of_range;
    if (!make_map(&tv16, v16, a.rows_total, p->D, 2) ||
        sa::launch_to_f16(v, v16, static_cast<long long>(a.rows_total) * p->D,
                          const_cast<unsigned int*>(a.f16_bad), st) != cudaSuccess)
      return SA_ERR_LAUNCH;
    extra = 1;
  }
  if (sa::launch_forward(tq, tk, tv, tv16, a, st) != cudaSuccess) return SA_ERR_LAUNCH;
  g_last_launches = 3 + extra;
  return SA_OK;
}

}  // namespace

sa_status sa_forward(const void* q, const void* k, const void* v, const float* q_scale, const float* k_scale,
                     const int32_t* kv_index, const int32_t* kv_count, const sa_params* p, void* out, float* lse,
                     float* out_f32, void* ws, size_t ws_bytes, sa_stream_t stream) {
  return forward_impl(q, k, v, q_scale, k_scale, kv_index, kv_count, p, out, lse, out_f32, nullptr, nullptr, ws,
                      ws_bytes, stream);
}

}  // extern "C"

namespace {

sa_status check_coarse(const sa_coarse* c) {
  if (!c || !c->qbar || !c->kbar || !c->vbar || !c->oc || !c->lse) return SA_ERR_INVALID_ARG;
  if (!aligned16(c->qbar) || !aligned16(c->kbar) || !aligned16(c->vbar) || !aligned16(c->oc) || !aligned4(c->lse))
    return SA_ERR_ALIGNMENT;
  return SA_OK;
}

sa::CoarseTensors coarse_tensors(const sa_coarse* c) {
  return sa::CoarseTensors{c->qbar, c->kbar, c->vbar, c->oc, c->lse};
}

// sa_backward, and with `coarse` set sa_backward_gated (gate, dgate and the coarse tensors).
sa_status backward_impl(const void* q, const void* k, const void* v, const void* out, const float* out_f32,
                        const float* lse, const void* dout, const float* gate, const int32_t* kv_index,
                        const int32_t* kv_count, const sa_params* p, const sa_coarse* coarse, float* dq, float* dk,
                        float* dv, float* dgate, void* ws, size_t ws_bytes, sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!q || !k || !v || !out || !lse || !dout || !kv_index || !kv_count || !dq || !dk || !dv)
    return SA_ERR_INVALID_ARG;
  if (p->qk_dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned4(lse) || !aligned4(kv_index) || !aligned4(kv_count) ||
      (out_f32 && !aligned16(out_f32)))
    return SA_ERR_ALIGNMENT;
  const bool gated = coarse != nullptr;
  if (gated) {
    // Delta of the fine branch is recovered from the combined output; from its bf16 rounding
    // (2^-9 of |G Oc^ + O_f|) it misses the gradient bounds, so the fp32 copy is required
    if (!gate || !dgate || !out_f32) return SA_ERR_INVALID_ARG;
    if ((s = check_coarse(coarse)) != SA_OK) return s;
    if (!aligned4(gate) || !aligned4(dgate)) return SA_ERR_ALIGNMENT;
    if (p->B * p->H > 65535) return SA_ERR_UNSUPPORTED;  // one grid layer per head
  }
  const WsLayout w = ws_layout(p, g, gated ? SA_OP_BACKWARD_GATED : SA_OP_BACKWARD);
  if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SA_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  sa::AttnArgs a = base_args(p, g, ws);
  a.kv_index = kv_index;
  a.kv_count = kv_count;
  a.lse = const_cast<float*>(lse);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map(&tq, q, a.rows_total, p->D, 2) || !make_map(&tk, k, a.rows_total, p->D, 2) ||
      !make_map(&tv, v, a.rows_total, p->D, 2) || !make_map(&tdo, dout, a.rows_total, p->D, 2))
    return SA_ERR_LAUNCH;
  if (reset_status(ws, st) != SA_OK) return SA_ERR_LAUNCH;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  a.cube_mask = reinterpret_cast<unsigned long long*>(wb + w.cmask);
  if (sa::launch_cube_mask(g, reinterpret_cast<unsigned long long*>(wb + w.cmask), st) != cudaSuccess)
    return SA_ERR_LAUNCH;
  // fp16 copies of Q, K, V and dO with a range flag and max|dO|, max|V|; the decision kernel sets
  // the status block's single-product switch that both backward kernels read
  sa::DevStatus* dst = static_cast<sa::DevStatus*>(ws);
  CUtensorMap t16[4];
  const void* src16[4] = {q, k, v, dout};
  unsigned int* maxbits[4] = {nullptr, nullptr, &dst->f16_max[1], &dst->f16_max[0]};
  for (int t = 0; t < 4; ++t) {
    void* h = wb + w.h16[t];
    if (!make_map(&t16[t], h, a.rows_total, p->D, 2) ||
        sa::launch_to_f16(src16[t], h, static_cast<long long>(a.rows_total) * p->D, &dst->f16_out_of_range, st,
                          maxbits[t]) != cudaSuccess)
      return SA_ERR_LAUNCH;
  }
  if (sa::launch_f16_decide(dst, p->D, st) != cudaSuccess) return SA_ERR_LAUNCH;
  a.f16_single = &dst->f16_single;
  float* delta = reinterpret_cast<float*>(wb + w.delta);
  float* nlse2 = reinterpret_cast<float*>(wb + w.nlse2);
  int coarse_launches = 0;
  sa::CoarseAdd add{};
  if (gated) {
    const sa::CoarseGradWs cw{reinterpret_cast<float*>(wb + w.doc), reinterpret_cast<float*>(wb + w.dltc),
                              reinterpret_cast<float*>(wb + w.s32),  reinterpret_cast<float*>(wb + w.ds32),
                              reinterpret_cast<float*>(wb + w.cq),   reinterpret_cast<float*>(wb + w.ck),
                              reinterpret_cast<float*>(wb + w.cv)};
    if (sa::launch_coarse_backward(out, out_f32, dout, lse, gate, coarse_tensors(coarse), dgate, delta, nlse2, cw,
                                   a.scale, g, a.BH, p->D, a.st, a.timeout_ns, st, &coarse_launches) != cudaSuccess)
      return SA_ERR_LAUNCH;
    add = sa::CoarseAdd{cw.cq, cw.ck, cw.cv};
  }
  int launches = 0;
  a.ucap = union_cap(p, g);
  if (sa::launch_backward(tq, tk, tv, tdo, t16, out, out_f32, dout, a, reinterpret_cast<uint32_t*>(wb + w.bits), delta,
                          nlse2, reinterpret_cast<int32_t*>(wb + w.ulist), reinterpret_cast<int32_t*>(wb + w.ucnt),
                          reinterpret_cast<int32_t*>(wb + w.uklist), reinterpret_cast<int32_t*>(wb + w.ukcnt), add,
                          gated, st, &launches) != cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = 6 + coarse_launches + launches;
  return SA_OK;
}

}  // namespace

extern "C" {

sa_status sa_backward(const void* q, const void* k, const void* v, const void* out, const float* out_f32,
                      const float* lse, const void* dout, const int32_t* kv_index, const int32_t* kv_count, const sa_params* p,
                      float* dq, float* dk, float* dv, void* ws, size_t ws_bytes, sa_stream_t stream) {
  return backward_impl(q, k, v, out, out_f32, lse, dout, nullptr, kv_index, kv_count, p, nullptr, dq, dk, dv, nullptr,
                       ws, ws_bytes, stream);
}

sa_status sa_plan_coarse(const void* q, const void* k, const void* v, const sa_params* p, int32_t* kv_index,
                         int32_t* kv_count, const sa_coarse* coarse, void* ws, size_t ws_bytes, sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!q || !k || !v || !kv_index || !kv_count) return SA_ERR_INVALID_ARG;
  if (p->qk_dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
  if ((s = check_coarse(coarse)) != SA_OK) return s;
  if (p->B * p->H > 65535) return SA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(kv_index) || !aligned4(kv_count))
    return SA_ERR_ALIGNMENT;
  const WsLayout w = ws_layout(p, g, SA_OP_PLAN_COARSE);
  if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SA_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  const int BH = p->B * p->H;
  float* P32 = reinterpret_cast<float*>(wb + w.p32);
  // the router of sa_plan (same kernels, same lists), which also writes every scaled score in
  // fp32 into P32; then the coarse branch from its fp64 means and those scores
  if ((s = sa::plan_on_scratch(q, k, nullptr, nullptr, p, kv_index, kv_count, ws, ws_bytes, st, P32)) != SA_OK)
    return s;
  const int plan_launches = g_last_launches;
  int coarse_launches = 0;
  if (sa::launch_coarse_forward(v, reinterpret_cast<double*>(wb + w.qbar), reinterpret_cast<double*>(wb + w.kbar), P32,
                                coarse_tensors(coarse), g, BH, p->D, static_cast<sa::DevStatus*>(ws), timeout_ns_of(p),
                                st, &coarse_launches) != cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = plan_launches + coarse_launches;
  return SA_OK;
}

sa_status sa_forward_gated(const void* q, const void* k, const void* v, const int32_t* kv_index,
                           const int32_t* kv_count, const sa_params* p, const sa_coarse* coarse, const float* gate,
                           void* out, float* lse, float* out_f32, void* ws, size_t ws_bytes, sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (p->qk_dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
  // the sum is formed from the fine stage's fp32 output: a bf16 O_f rounded again after
  // the sum misses the output error bounds
  if (!gate || !out_f32) return SA_ERR_INVALID_ARG;
  if ((s = check_coarse(coarse)) != SA_OK) return s;
  if (!aligned4(gate)) return SA_ERR_ALIGNMENT;
  // the forward kernel forms O = G Oc^ + O_f in its epilogue (fp32, then the bf16 copy)
  return forward_impl(q, k, v, nullptr, nullptr, kv_index, kv_count, p, out, lse, out_f32, gate, coarse->oc, ws,
                      ws_bytes, stream);
}

sa_status sa_backward_gated(const void* q, const void* k, const void* v, const void* out, const float* out_f32,
                            const float* lse, const void* dout, const float* gate, const int32_t* kv_index,
                            const int32_t* kv_count, const sa_params* p, const sa_coarse* coarse, float* dq, float* dk,
                            float* dv, float* dgate, void* ws, size_t ws_bytes, sa_stream_t stream) {
  if (!coarse) return SA_ERR_INVALID_ARG;
  return backward_impl(q, k, v, out, out_f32, lse, dout, gate, kv_index, kv_count, p, coarse, dq, dk, dv, dgate, ws,
                       ws_bytes, stream);
}

sa_status sa_plan_bq128(const void* q, const void* k, const sa_params* p, int32_t* kv_index, int32_t* kv_count,
                        void* ws, size_t ws_bytes, sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!q || !k || !kv_index || !kv_count) return SA_ERR_INVALID_ARG;
  if (p->qk_dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
  if (p->B * p->H > 65535) return SA_ERR_UNSUPPORTED;  // one grid layer per head
  if (!aligned16(q) || !aligned16(k) || !aligned4(kv_index) || !aligned4(kv_count)) return SA_ERR_ALIGNMENT;
  const WsLayout w = ws_layout(p, g, SA_OP_PLAN_BQ128);
  if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SA_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (reset_status(ws, st) != SA_OK) return SA_ERR_LAUNCH;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  int launches = 0;
  if (sa::launch_plan_bq128(q, k, g, p->B * p->H, p->D, softmax_scale(p), p->top_k, p->top_p, p->kv_capacity,
                            kv_index, kv_count, reinterpret_cast<double*>(wb + w.qbar),
                            reinterpret_cast<double*>(wb + w.kbar), reinterpret_cast<double*>(wb + w.qpair),
                            reinterpret_cast<double*>(wb + w.scores), reinterpret_cast<int32_t*>(wb + w.blk_index),
                            reinterpret_cast<int32_t*>(wb + w.blk_count), static_cast<sa::DevStatus*>(ws), st,
                            &launches) != cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = launches;
  return SA_OK;
}

sa_status sa_recall(const float* lse_kept, const float* lse_all, const sa_params* p, float* recall,
                    float* cube_recall, sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!lse_kept || !lse_all || (!recall && !cube_recall)) return SA_ERR_INVALID_ARG;
  if (!aligned4(lse_kept) || !aligned4(lse_all) || (recall && !aligned4(recall)) ||
      (cube_recall && !aligned4(cube_recall)))
    return SA_ERR_ALIGNMENT;
  if (sa::launch_recall(lse_kept, lse_all, recall, cube_recall, g, p->B * p->H,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = 1;
  return SA_OK;
}

sa_status sa_block_mass(const void* q, const void* k, const float* lse_all, const sa_params* p, float* pblock,
                        void* ws, size_t ws_bytes, sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!q || !k || !lse_all || !pblock) return SA_ERR_INVALID_ARG;
  if (p->qk_dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->B) * p->H * g.T * g.T >= (1LL << 40)) return SA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned4(lse_all) || !aligned4(pblock)) return SA_ERR_ALIGNMENT;
  const WsLayout w = ws_layout(p, g, SA_OP_BLOCK_MASS);
  if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SA_ERR_ALIGNMENT;
  const int BH = p->B * p->H;
  CUtensorMap tq, tk;
  if (!make_map(&tq, q, static_cast<long long>(BH) * g.Npad, p->D, 2) ||
      !make_map(&tk, k, static_cast<long long>(BH) * g.Npad, p->D, 2))
    return SA_ERR_LAUNCH;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (reset_status(ws, st) != SA_OK) return SA_ERR_LAUNCH;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  auto* cmask = reinterpret_cast<unsigned long long*>(wb + w.cmask);
  const unsigned ms = p->timeout_ms ? p->timeout_ms : 2000u;
  const double sc = softmax_scale(p);
  if (sa::launch_cube_mask(g, cmask, st) != cudaSuccess ||
      sa::launch_block_mass(tq, tk, lse_all, cmask, pblock, g, BH, p->D, static_cast<float>(sc * 1.4426950408889634),
                            static_cast<sa::DevStatus*>(ws), static_cast<unsigned long long>(ms) * 1000000ull,
                            st) != cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = 2;
  return SA_OK;
}

sa_status sa_best_recall(const float* pblock, const int32_t* kv_count, const sa_params* p, float* best,
                         sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!pblock || !kv_count || !best) return SA_ERR_INVALID_ARG;
  if (!aligned4(pblock) || !aligned4(kv_count) || !aligned4(best)) return SA_ERR_ALIGNMENT;
  if (sa::launch_best_recall(pblock, kv_count, best, p->B * p->H * g.T, g.T, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = 1;
  return SA_OK;
}

}  // extern "C"

namespace {

struct FineLayout {
  size_t qlimb, klimb, qexp, qvalid, ql1, kexp, kvalid, kexpmax, lse2, pr, total;
  int TG, TGp;
};

bool fine_shape_ok(int rt, int rh, int rw) {
  auto ok = [](int r) { return r == 1 || r == 2 || r == 4; };
  if (!ok(rt) || !ok(rh) || !ok(rw)) return false;
  const int G = 64 / (rt * rh * rw);
  return G == 4 || G == 8 || G == 16;
}

FineLayout fine_layout(const sa_params* p, const Geom& g, int rt, int rh, int rw) {
  FineLayout w;
  const size_t BH = static_cast<size_t>(p->B) * p->H;
  const int G = 64 / (rt * rh * rw);
  w.TG = g.T * G;
  w.TGp = (w.TG + 3) & ~3;
  const size_t TG = static_cast<size_t>(w.TG), TGp = static_cast<size_t>(w.TGp);
  size_t off = kHeader;
  w.qlimb = off;
  off = align256(off + BH * 4 * TG * 128);
  w.klimb = off;
  off = align256(off + BH * 4 * TG * 128);
  w.qexp = off;
  off = align256(off + BH * TG * sizeof(int));
  w.qvalid = off;
  off = align256(off + BH * TG * sizeof(int));
  w.ql1 = off;
  off = align256(off + BH * TG * sizeof(double));
  w.kexp = off;
  off = align256(off + BH * TGp * sizeof(int));
  w.kvalid = off;
  off = align256(off + BH * TGp * sizeof(int));
  w.kexpmax = off;
  off = align256(off + BH * sizeof(unsigned));
  w.lse2 = off;
  off = align256(off + BH * TG * sizeof(float));
  w.pr = off;
  off = align256(off + BH * g.T * static_cast<size_t>(g.T) * sizeof(float));
  w.total = off;
  return w;
}

}  // namespace

extern "C" {

size_t sa_plan_fine_workspace_size(const sa_params* p, int rt, int rh, int rw) {
  Geom g;
  if (check_params(p, &g) != SA_OK || !fine_shape_ok(rt, rh, rw)) return 0;
  return fine_layout(p, g, rt, rh, rw).total;
}

sa_status sa_plan_fine(const void* q, const void* k, const sa_params* p, int rt, int rh, int rw, int32_t* kv_index,
                       int32_t* kv_count, float* p_r, void* ws, size_t ws_bytes, sa_stream_t stream) {
  Geom g;
  g_last_launches = 0;
  sa_status s = check_params(p, &g);
  if (s != SA_OK) return s;
  if (!q || !k || !kv_index || !kv_count) return SA_ERR_INVALID_ARG;
  if (!fine_shape_ok(rt, rh, rw)) return SA_ERR_UNSUPPORTED;
  if (p->qk_dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned4(kv_index) || !aligned4(kv_count) || (p_r && !aligned4(p_r)))
    return SA_ERR_ALIGNMENT;
  const FineLayout w = fine_layout(p, g, rt, rh, rw);
  if (static_cast<long long>(p->B) * p->H * 4 * w.TG >= (1LL << 31)) return SA_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < w.total) return SA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SA_ERR_ALIGNMENT;
  const int BH = p->B * p->H;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  sa::FineWs f;
  f.qlimb = reinterpret_cast<int8_t*>(wb + w.qlimb);
  f.klimb = reinterpret_cast<int8_t*>(wb + w.klimb);
  f.qexp = reinterpret_cast<int*>(wb + w.qexp);
  f.qvalid = reinterpret_cast<int*>(wb + w.qvalid);
  f.ql1 = reinterpret_cast<double*>(wb + w.ql1);
  f.kexp = reinterpret_cast<int*>(wb + w.kexp);
  f.kvalid = reinterpret_cast<int*>(wb + w.kvalid);
  f.kexp_max = reinterpret_cast<unsigned*>(wb + w.kexpmax);
  f.lse2 = reinterpret_cast<float*>(wb + w.lse2);
  f.pr = p_r ? p_r : reinterpret_cast<float*>(wb + w.pr);
  f.TGp = w.TGp;
  CUtensorMap tq, tk;
  if (!make_limb_map(&tq, f.qlimb, w.TG, 4LL * BH) || !make_limb_map(&tk, f.klimb, w.TG, 4LL * BH))
    return SA_ERR_LAUNCH;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (reset_status(ws, st) != SA_OK) return SA_ERR_LAUNCH;
  const unsigned ms = p->timeout_ms ? p->timeout_ms : 2000u;
  int launches = 0;
  if (sa::launch_plan_fine(q, k, tq, tk, g, BH, p->D, rt, rh, rw, softmax_scale(p), p->top_k, p->kv_capacity, f,
                           kv_index, kv_count, static_cast<sa::DevStatus*>(ws),
                           static_cast<unsigned long long>(ms) * 1000000ull, st, &launches) != cudaSuccess)
    return SA_ERR_LAUNCH;
  g_last_launches = launches;
  return SA_OK;
}

sa_status sa_get_device_status(const void* ws, sa_stream_t stream) {
  if (!ws) return SA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SA_ERR_LAUNCH;
  sa::DevStatus h;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return SA_ERR_LAUNCH;
  if (h.error & sa::DEVERR_TIMEOUT) return SA_ERR_DEVICE_TIMEOUT;
  if (h.error & sa::DEVERR_INDEX) return SA_ERR_DEVICE_INDEX;
  if (h.error & sa::DEVERR_CAPACITY) return SA_ERR_CAPACITY;
  return SA_OK;
}

int sa_plan_fallback_rows(const void* ws, sa_stream_t stream) {
  if (!ws) return -1;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return -1;
  sa::DevStatus h;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
  return static_cast<int>(h.router_fallback);
}

sa_status sa_get_cta_clocks(const void* ws, size_t ws_bytes, int kernel, unsigned long long* out, int max_ctas,
                            int* n_ctas, sa_stream_t stream) {
  if (!ws || !out || !n_ctas || kernel < 0 || kernel > 2 || max_ctas < 0 || ws_bytes < kHeader + kClockBytes)
    return SA_ERR_INVALID_ARG;
  *n_ctas = 0;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SA_ERR_LAUNCH;
  sa::DevStatus h;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return SA_ERR_LAUNCH;
  int n = static_cast<int>(h.grid[kernel]);
  n = n < max_ctas ? n : max_ctas;
  n = n < sa::kClockCtas ? n : sa::kClockCtas;
  if (n > 0) {
    const uint8_t* src = static_cast<const uint8_t*>(ws) + kHeader +
                         static_cast<size_t>(kernel) * sa::kClockCtas * 4 * sizeof(unsigned long long);
    if (cudaMemcpy(out, src, static_cast<size_t>(n) * 4 * sizeof(unsigned long long), cudaMemcpyDeviceToHost) !=
        cudaSuccess)
      return SA_ERR_LAUNCH;
  }
  *n_ctas = n;
  return SA_OK;
}

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case SA_ERR_CAPACITY: return "a row selected more blocks than kv_capacity";
    case SA_ERR_WORKSPACE: return "workspace missing or too small";
    case SA_ERR_LAUNCH: return "CUDA launch or driver call failed";
    case SA_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel timed out";
    case SA_ERR_DEVICE_INDEX: return "kv_index entry or kv_count out of range";
  }
  return "unknown status";
}

int sa_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
