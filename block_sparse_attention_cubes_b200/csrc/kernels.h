// Launch functions of the library's kernels (host side, internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/sa.h"
#include "geometry.cuh"
#include "ptx.cuh"

namespace sa {

// sa_plan's host-side argument checks; *ws_needed receives the router's workspace size (api.cu).
sa_status plan_check(const void* q, const void* k, const float* q_scale, const float* k_scale, const sa_params* p,
                     const int32_t* kv_index, const int32_t* kv_count, size_t* ws_needed);
// sa_plan on the scratch `ws` of `ws_bytes` (a caller's workspace or the library's fixed
// array): the host checks, the workspace carving and the launches of sa_plan, and the launch
// count that sa_last_launch_count reports (api.cu).  s32 (optional, [B*H*T, T] fp32) also
// receives every scaled score.
sa_status plan_on_scratch(const void* q, const void* k, const float* q_scale, const float* k_scale,
                          const sa_params* p, int32_t* kv_index, int32_t* kv_count, void* ws, size_t ws_bytes,
                          cudaStream_t stream, float* s32 = nullptr);

struct DevStatus;
struct AttnArgs;

cudaError_t launch_tile(const void* src, void* dst, const Geom& g, int BH, int row_bytes, bool to_tiled,
                        cudaStream_t stream);

// Tile (to_tiled) or untile with the 3-D RoPE rotation of each token (inverse when untiling).
cudaError_t launch_tile_rope(const void* src, void* dst, const Geom& g, int BH, int D, int elem_bytes, bool to_tiled,
                             int dt, int dh, int dw, const float* cs, const float* sn, cudaStream_t stream);

cudaError_t launch_plan(const void* q, const void* k, const float* q_scale, const float* k_scale, const Geom& g,
                        int BH, int D, bool fp8, double scale, int top_k, float top_p, int cap, int32_t* kv_index,
                        int32_t* kv_count, double* qbar, double* kbar, double* S, DevStatus* st,
                        cudaStream_t stream, int* launches);

// Scratch of the tensor-core router (carved from the plan workspace by api.cu).
struct PlanFastWs {
  double* qbar;        // [BH*T, D] fp64 pooled means (also read by the fp64 fallback rows)
  double* kbar;
  int8_t* qlimb;       // [BH, 4, T, 128] int8 limbs of the pooled rows
  int8_t* klimb;
  int* qexp;           // [BH*T] binary exponent of each pooled row
  int* kexp;           // [BH, Tk] (rows padded to Tk entries)
  double* ql1;         // [BH*T] 1-norm of each pooled query row
  unsigned* kexp_max;  // [BH] largest key exponent per head (biased)
  void* meta;          // [BH*T] per-row key scaling and error bounds (32 bytes each)
  int* keys;           // [BH*T, Tk] fixed-point score keys
  int* rkmax;          // [BH*T] largest / smallest key of each row
  int* rkmin;
  int Tk;              // row stride of keys (T rounded up to 4)
  int* flist;          // [BH*T] rows left to the fp64 path
  float* s32 = nullptr;  // optional [BH*T, T]: every scaled score in fp32 (the coarse branch reads them)
};
int plan_fallback_ctas();
// Router on the tensor cores (pool + limbs, exact limb products -> keys, key selection, fp64
// rows): 5 launches and one memset.  tm_qlimb / tm_klimb: 3-D maps {128 B, T, BH*4} over the
// limb buffers with 128 x 128 boxes and the 128-byte swizzle; tm_keys: 3-D map {T, T, BH} (int32,
// row stride Tk) over the keys with 32 x 32 boxes and the 128-byte swizzle, for the key stores.
cudaError_t launch_plan_fast(const void* q, const void* k, const float* q_scale, const float* k_scale,
                             const CUtensorMap& tm_qlimb, const CUtensorMap& tm_klimb, const CUtensorMap& tm_keys,
                             const Geom& g, int BH, int D,
                             bool fp8, double scale, int top_k, float top_p, int cap, unsigned debug,
                             unsigned long long timeout_ns, const PlanFastWs& w, int32_t* kv_index, int32_t* kv_count,
                             DevStatus* st, cudaStream_t stream, int* launches);

// VSA2 fine-grained router (fine_router.cu).
struct FinePoolArgs {
  const uint8_t* q;
  const uint8_t* k;
  int8_t* qlimb;      // [BH, 4, T*G, 128] int8 limbs of the group means
  int8_t* klimb;
  int* qexp;          // [BH * T*G] exponents and validity of the query groups
  int* qvalid;
  double* ql1;        // [BH * T*G] 1-norms of the query group means
  int* kexp;          // [BH, TGp] exponents and validity of the key groups (rows padded to TGp)
  int* kvalid;
  unsigned* kexp_max; // [BH]
  DevStatus* st;
  Geom g;
  int BH, rt, rh, rw, TGp;
  unsigned long long timeout_ns;
};
struct FineScoreArgs {
  const int* qexp;
  const int* qvalid;
  const int* kexp;
  const int* kvalid;
  float* lse2;        // [BH * T*G] lse of each query group, log2 units
  float* pr;          // [BH, T, T] P_r
  DevStatus* st;
  int T, TG, TGp, BH;
  double scale_log2;
  unsigned long long timeout_ns;
};
struct FineWs {
  int8_t* qlimb;
  int8_t* klimb;
  int* qexp;
  int* qvalid;
  double* ql1;
  int* kexp;
  int* kvalid;
  unsigned* kexp_max;
  float* lse2;
  float* pr;
  int TGp;
};
// Group pooling + limbs, two score passes (lse, then P_r) and the per-sequence Top-K: 5 launches
// and one memset.  tm_qlimb / tm_klimb: 3-D maps {128 B, T*G, BH*4} over the group limbs.
cudaError_t launch_plan_fine(const void* q, const void* k, const CUtensorMap& tm_qlimb, const CUtensorMap& tm_klimb,
                             const Geom& g, int BH, int D, int rt, int rh, int rw, double scale, int K, int cap,
                             const FineWs& w, int32_t* kv_index, int32_t* kv_count, DevStatus* st,
                             unsigned long long timeout_ns, cudaStream_t stream, int* launches);

cudaError_t launch_query_pair_union(const int32_t* kv_index, const int32_t* kv_count, int32_t* u_list,
                                    int32_t* u_cnt, int BH, int T, int cap, DevStatus* st, cudaStream_t stream);
// Key-cube pair unions of the transposed selection, through a [BH, T, ceil(T/32)] bit matrix.
cudaError_t launch_key_pair_union(const int32_t* kv_index, const int32_t* kv_count, uint32_t* bits, int32_t* u_list,
                                  int32_t* u_cnt, int BH, int T, int cap, DevStatus* st, cudaStream_t stream);

cudaError_t launch_cube_mask(const Geom& g, unsigned long long* mask, cudaStream_t stream);
int num_sms();

// tv16: map over the fp16 copy of V, read when a.out_f32 is set and *a.f16_bad is 0.
cudaError_t launch_forward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& tv16, const AttnArgs& a, cudaStream_t stream);
// bf16 -> fp16 copy of `elems` values (a multiple of 8, 16-byte aligned); *bad |= 1 when one
// does not fit fp16; with maxbits set, the largest |x| goes there (fp32 bits, atomicMax).
cudaError_t launch_to_f16(const void* src, void* dst, long long elems, unsigned int* bad, cudaStream_t stream,
                          unsigned int* maxbits = nullptr);
// st->f16_single = the backward's single-product decision from the conversions' flags.
cudaError_t launch_f16_decide(DevStatus* st, int D, cudaStream_t stream);

// Per-cube terms the backward kernels add to every valid row of a cube (the coarse branch's
// gradients through the mean pool), [BH, T, D] fp32 each; all NULL for the fine stage alone.
struct CoarseAdd {
  const float* q;
  const float* k;
  const float* v;
};

// With delta_ready, Delta and -lse*log2(e) are already in `delta` / `nlse2` and the Delta
// pass is not launched.
// t16[4]: maps over the fp16 copies of Q, K, V, dO, read when *a.f16_single is 1.
cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap (&t16)[4], const void* out, const float* out_f32,
                            const void* dout,
                            AttnArgs a, uint32_t* bits, float* delta, float* nlse2,
                            int32_t* uq_list,
                            int32_t* uq_cnt, int32_t* uk_list, int32_t* uk_cnt, const CoarseAdd& add,
                            bool delta_ready, cudaStream_t stream, int* launches);

// Coarse branch (cube-level tensors, fp32, [BH, T, D] and lse [BH, T]).
struct CoarseTensors {
  float* qbar;
  float* kbar;
  float* vbar;
  float* oc;
  float* lse;
};

// Backward scratch of the coarse branch.
struct CoarseGradWs {
  float* doc;   // [BH, T, D]  dOc^
  float* dltc;  // [BH, T]     <dOc^, Oc^>
  float* s;     // [BH, T, T]  scaled scores, then P
  float* ds;    // [BH, T, T]  dS
  float* cq;    // [BH, T, D]  dQc / n, dKc / n, dVc / n
  float* ck;
  float* cv;
};

// Vc pooled from v, fp32 copies of the router's fp64 Qc and Kc, Pc from the router's fp32 scores
// (P32 holds them on entry and Pc on return) and Oc^ = Pc Vc (3 launches).
cudaError_t launch_coarse_forward(const void* v, const double* qbar64, const double* kbar64, float* P32,
                                  const CoarseTensors& c, const Geom& g, int BH, int D, DevStatus* st,
                                  unsigned long long timeout_ns, cudaStream_t stream, int* launches);
// dG, the fine branch's Delta and -lse*log2(e), and the coarse branch's per-cube gradient
// terms w.cq, w.ck, w.cv (6 launches).
cudaError_t launch_coarse_backward(const void* out, const float* out_f32, const void* dout, const float* lse,
                                   const float* gate, const CoarseTensors& c, float* dgate, float* delta,
                                   float* nlse2, const CoarseGradWs& w, float scale, const Geom& g, int BH, int D,
                                   DevStatus* st, unsigned long long timeout_ns, cudaStream_t stream, int* launches);

// The cube router's pooling (bf16) and selection passes on their own.
cudaError_t launch_pool(const void* q, const void* k, const Geom& g, int BH, int D, double* qbar, double* kbar,
                        cudaStream_t stream);
cudaError_t launch_select(const double* S, int32_t* kv_index, int32_t* kv_count, int rows, int T, int top_k,
                          float top_p, int cap, DevStatus* st, cudaStream_t stream);
// Router with 128-token query blocks (cube pairs); writes each block's list for both its cubes
// (5 launches).  qpair [BH, ceil(T/2), D] fp64, S [BH, ceil(T/2), T] fp64, blk_* the block lists.
cudaError_t launch_plan_bq128(const void* q, const void* k, const Geom& g, int BH, int D, double scale, int top_k,
                              float top_p, int cap, int32_t* kv_index, int32_t* kv_count, double* qbar, double* kbar,
                              double* qpair, double* S, int32_t* blk_index, int32_t* blk_count, DevStatus* st,
                              cudaStream_t stream, int* launches);

// tau = exp(lse_kept - lse_all) per valid row (0 on padding) into recall, and its mean over each
// cube's valid rows into cube_recall; either output may be NULL.
// P_oracle over every (query cube, key cube) from a dense S = Q K^T pass and the dense lse.
cudaError_t launch_block_mass(const CUtensorMap& tq, const CUtensorMap& tk, const float* lse,
                              const unsigned long long* cube_mask, float* pblock, const Geom& g, int BH, int D,
                              float scale_log2, DevStatus* st, unsigned long long timeout_ns, cudaStream_t stream);
// Sum of the kv_count[row] largest entries of each row of pblock [rows, T].
cudaError_t launch_best_recall(const float* pblock, const int32_t* kv_count, float* best, int rows, int T,
                               cudaStream_t stream);
cudaError_t launch_recall(const float* lse_kept, const float* lse_all, float* recall, float* cube_recall,
                          const Geom& g, int BH, cudaStream_t stream);

}  // namespace sa
