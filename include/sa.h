/*
 * sa.h - C ABI of the cube-routed block-sparse attention library (libsa.so, sm_100a).
 *
 * The method: a coarse router mean-pools Q and K over 4x4x4 cubes of 64 tokens, scores
 * every (query cube, key cube) pair, applies a row softmax and keeps the union of the
 * Top-k and Top-p key cubes of each query cube (SpargeAttention2 page, "Block-Pooled
 * Attention for Efficient Mask Construction" and "The Hybrid Top-k+Top-p Masking Rule",
 * equation 9).  A fine stage then runs softmax attention over only the selected 64x64
 * tiles, forward and backward (SpargeAttention2 page, "Kernel Implementation of the
 * Hybrid-Masked Block-Sparse Attention"; VSA page, "The Fine Stage").
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are DEVICE pointers owned by the caller.  The library never
 *    allocates or frees device memory and never synchronises, except where stated.
 *  - Token tensors are contiguous [B, H, Npad, D] in cube-major padded order (see
 *    sa_tile), Npad = 64 * N_t * N_h * N_w with N_x = ceil(lat_x / 4).  Row pitch is
 *    D elements; base pointers must be 16-byte aligned.
 *  - T = N_t * N_h * N_w is the number of cubes (query blocks = key blocks).
 *  - Every launch is asynchronous on `stream` (a cudaStream_t; NULL = legacy stream).
 *  - Host-side argument errors are returned synchronously before anything is
 *    launched.  Problems found on the device (a bounded wait that timed out, an index
 *    list entry out of range, too many selected blocks for kv_capacity) are recorded in
 *    the status block at the start of the workspace and read with
 *    sa_get_device_status.  Every entry point that takes a workspace clears that block
 *    first, so the status reports the most recent call on that workspace.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SA_API __attribute__((visibility("default")))
#else
#define SA_API
#endif

typedef struct CUstream_st* sa_stream_t; /* identical to cudaStream_t */

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,    /* null pointer, bad shape, k < 0, p not finite, ... */
  SA_ERR_UNSUPPORTED = 2,    /* a valid request outside what is built (e.g. D not in {64,128}) */
  SA_ERR_ALIGNMENT = 3,      /* a pointer not aligned to 16 bytes */
  SA_ERR_CAPACITY = 4,       /* device: a row selected more than kv_capacity blocks */
  SA_ERR_WORKSPACE = 5,      /* ws == NULL or ws_bytes < sa_workspace_size(...) */
  SA_ERR_LAUNCH = 6,         /* a CUDA launch or driver call failed */
  SA_ERR_DEVICE_TIMEOUT = 7, /* device: a bounded wait inside a kernel gave up */
  SA_ERR_DEVICE_INDEX = 8    /* device: a kv_index entry outside [0,T) or a count outside [0,cap] */
} sa_status;

typedef enum { SA_BF16 = 0, SA_FP8_E4M3 = 1 } sa_qk_dtype;

typedef enum {
  SA_OP_PLAN = 0,
  SA_OP_FORWARD = 1,          /* also sa_forward_gated */
  SA_OP_BACKWARD = 2,
  SA_OP_PLAN_COARSE = 3,      /* sa_plan_coarse */
  SA_OP_BACKWARD_GATED = 4,   /* sa_backward_gated */
  SA_OP_PLAN_BQ128 = 5,       /* sa_plan_bq128 */
  SA_OP_BLOCK_MASS = 6        /* sa_block_mass */
} sa_op;

typedef struct {
  int B, H, D;                /* batch, heads, head dim (D in {64, 128}) */
  int lat_t, lat_h, lat_w;    /* valid latent grid, e.g. 21, 45, 80 */
  int top_k;                  /* Top-k block count, >= 0 (clamped to T); see sa_topk_from_fraction */
  float top_p;                /* Top-p mass fraction; >= 1 keeps every block, <= 0 adds none */
  int kv_capacity;            /* row stride of kv_index; 1 <= kv_capacity <= T */
  int qk_dtype;               /* sa_qk_dtype; SA_FP8_E4M3 needs q_scale / k_scale */
  float softmax_scale;        /* 0 -> 1/sqrt(D) */
  unsigned int timeout_ms;    /* bound of every in-kernel wait; 0 -> 2000 ms */
  unsigned int debug_flags;   /* 0 in normal use; SA_DEBUG_* below */
} sa_params;

/* Test hook: the forward kernel's producer issues no loads, so its consumers' bounded
 * waits run out and the call reports SA_ERR_DEVICE_TIMEOUT without faulting. */
#define SA_DEBUG_SKIP_LOADS 1u
/* Test hook: sa_plan decides every row on its fp64 path (normally taken only by the rows
 * whose tensor-core decision is within the error bound of changing). */
#define SA_DEBUG_ROUTER_FALLBACK 2u
/* Measurement hook: sa_forward and sa_backward record, for every CTA of their attention
 * kernels, its start and end time and the work it did (read with sa_get_cta_clocks). */
#define SA_DEBUG_CTA_CLOCKS 4u
/* Measurement hook: the attention kernels take the fixed round-robin share of work items
 * (CTA c: items c, c + grid, ...) instead of fetching them in order from a shared counter. */
#define SA_DEBUG_STATIC_ITEMS 8u

/* Padded token count Npad and cube count T implied by the latent grid (0 on bad input). */
SA_API int sa_padded_tokens(const sa_params* p);
SA_API int sa_num_cubes(const sa_params* p);

/* ceil(frac * T): SpargeAttention2's k% rule ("Definition of the two component
 * selectors": the largest ceil(k% x T_n) entries). */
SA_API int sa_topk_from_fraction(double frac, int T);

/* Bytes of device workspace `op` (sa_op) needs for these parameters; 0 on bad input.
 * Plan: status block + pooled Q and K (fp64, 2*B*H*T*D) + their int8 limbs (8*B*H*T*128) + per-row
 * exponents, norms and key scaling (48*B*H*T) + the fixed-point score keys (int32, B*H*T*Tk, Tk = T
 * rounded up to 4) + the list of rows decided in fp64 (B*H*T).
 * Forward: status block + one 64-bit valid-slot mask per cube (T) + the union lists of
 * adjacent query-cube pairs (int32, B*H*ceil(T/2)*(1 + 2*kv_capacity)).  Backward: status block
 * + cube masks + Delta and -lse*log2(e) (fp32, 2*B*H*Npad) + the selection as a bit matrix
 * (B*H*T*ceil(T/32) words) + the query-pair and key-pair union lists (int32,
 * B*H*ceil(T/2)*(2 + min(2*kv_capacity, T) + T)).  Plan + coarse: the plan's, then the
 * cube-level softmax Pc (fp32, B*H*T*T).  Gated backward: the backward's, then dOc^ and
 * the three per-cube gradient terms (fp32, 4*B*H*T*D), <dOc^, Oc^> (B*H*T) and the
 * cube-level scores and dS (fp32, 2*B*H*T*T). */
SA_API size_t sa_workspace_size(const sa_params* p, int op);

/* Layout helper (VSA page, "Cube Partitioning and Token Re-Indexing"; VSA2 page,
 * section 2.2 "Permutation" and "Kernel Implementation" for padding).
 * x_latent: [B, H, lat_t*lat_h*lat_w, D] row-major (t, h, w) token order.
 * x_tiled:  [B, H, Npad, D] cube-major; token (t,h,w) goes to slot
 *   ((t/4)*N_h*N_w + (h/4)*N_w + w/4)*64 + (t%4)*16 + (h%4)*4 + (w%4); padding slots are 0.
 * elem_bytes is 1, 2 or 4.  sa_untile is the inverse (padding dropped). */
SA_API sa_status sa_tile(const void* x_latent, void* x_tiled, const sa_params* p, int elem_bytes, sa_stream_t stream);
SA_API sa_status sa_untile(const void* x_tiled, void* x_latent, const sa_params* p, int elem_bytes, sa_stream_t stream);

/* The same permutation with the 3-D rotary position embedding fused in (VSA2 page, section 2.2
 * "Permutation": the permutation to cube-major order is applied once at the start of the
 * transformer with a matching permutation of the RoPE embeddings; RoFormer: channel pair
 * (x_2i, x_2i+1) of a token at position m is rotated by m * theta_i).  The head dimension p->D
 * splits into three even sections rope_dt + rope_dh + rope_dw = D, rotated by the token's t, h
 * and w position.  rope_cos / rope_sin (fp32, device, caller-owned) hold the cosines and sines
 * of the angles: lat_t rows of rope_dt/2 entries (axis t, row = position), then lat_h rows of
 * rope_dh/2, then lat_w rows of rope_dw/2.  A pair (a, b) with cosine c and sine s becomes
 * (a c - b s, a s + b c), computed in fp32 and rounded to the element type.
 * sa_tile_rope: x_latent [B,H,L,D] -> x_tiled [B,H,Npad,D], padding slots 0.
 * sa_untile_rope: x_tiled -> x_latent with the inverse rotation (a c + b s, -a s + b c), e.g. for
 * gradients; padding slots are dropped.  elem_bytes: 2 (bf16) or 4 (fp32); D * elem_bytes a
 * multiple of 16.  Errors: SA_ERR_INVALID_ARG (sections, sizes, NULL), SA_ERR_ALIGNMENT (tensors
 * 16-byte, tables 4-byte aligned).  One launch, no workspace. */
SA_API sa_status sa_tile_rope(const void* x_latent, void* x_tiled, const sa_params* p, int elem_bytes, int rope_dt,
                              int rope_dh, int rope_dw, const float* rope_cos, const float* rope_sin,
                              sa_stream_t stream);
SA_API sa_status sa_untile_rope(const void* x_tiled, void* x_latent, const sa_params* p, int elem_bytes, int rope_dt,
                                int rope_dh, int rope_dw, const float* rope_cos, const float* rope_sin,
                                sa_stream_t stream);

/* Router (SpargeAttention2 page, "Block-Pooled Attention", steps 2-4, and equation 9;
 * VSA page, "Kernel Implementation": contiguous arrays of block indices).
 * q, k: [B,H,Npad,D] bf16, or e4m3 bytes when qk_dtype == SA_FP8_E4M3, in which case
 *   q_scale, k_scale are [B,H,T] fp32 (value = code * scale of its cube); else NULL.
 * Pooling averages the valid tokens of each cube; scores are Qbar Kbar^T * scale; the
 * row softmax, Top-k (top_k largest) and Top-p (shortest prefix of the descending order
 * whose mass reaches top_p of the row) are taken in that order, ties broken by the
 * smaller block id, and at least one block is kept.
 * Outputs: kv_count [B,H,T] int32 = number of kept blocks (clipped to kv_capacity, with
 * SA_ERR_CAPACITY recorded when clipping happened); kv_index [B,H,T,kv_capacity] int32
 * holds the kept block ids in ascending order in its first kv_count entries (the rest
 * are left untouched).  Deterministic.
 * How it runs: the pooled rows are split into four exact 8-bit limbs and the scores come from
 * integer tensor-core products (exact accumulation; each score within 4.03 * 2^-23 * 2^(Eq+Ek)
 * * scale of its fp64 value, 2^Eq and 2^Ek bounding the two rows' entries), as 32-bit
 * fixed-point keys; the selection runs on the keys with fixed-point masses, and every row whose
 * decision could change within those error bounds (exact ties among them) is decided again from
 * fp64 scores, so the result is the fp64 decision (sa_plan_fallback_rows counts those rows). */
SA_API sa_status sa_plan(const void* q, const void* k, const float* q_scale, const float* k_scale, const sa_params* p,
                  int32_t* kv_index, int32_t* kv_count, void* ws, size_t ws_bytes, sa_stream_t stream);

/* Fine stage forward (SpargeAttention2 page, "Kernel Implementation", online softmax;
 * VSA2 page 2.1, O = softmax(QK^T/sqrt(D) + M) V with M = 0 on selected 64x64 tiles,
 * -inf elsewhere and on padding keys).
 * q, k: as for sa_plan; v: [B,H,Npad,D] bf16; kv_index/kv_count: as written by sa_plan
 *   (entries must lie in [0,T), counts in [0,kv_capacity]; violations are recorded as
 *   SA_ERR_DEVICE_INDEX and the offending entries skipped).
 * With qk_dtype == SA_FP8_E4M3 (D = 128 only, else SA_ERR_UNSUPPORTED; q_scale and k_scale
 * required, else SA_ERR_INVALID_ARG): S = (Q8 K8^T) * q_scale[i] * k_scale[j] * scale from an
 * e4m3 tensor-core product with fp32 accumulation (SparkDiffusion page, section 4.3, E4M3);
 * P and V stay bf16.
 * out: [B,H,Npad,D] bf16; lse: [B,H,Npad] fp32, natural log of each row's softmax
 * normaliser of the scaled scores.  Padding query rows get out = 0, lse = 0; a row with
 * count 0 gets out = 0, lse = -inf.  out_f32 (may be NULL): [B,H,Npad,D] fp32, the same
 * output before rounding to bf16; pass it on to sa_backward for an exact Delta.
 * Deterministic. */
SA_API sa_status sa_forward(const void* q, const void* k, const void* v, const float* q_scale, const float* k_scale,
                     const int32_t* kv_index, const int32_t* kv_count, const sa_params* p, void* out, float* lse,
                     float* out_f32, void* ws, size_t ws_bytes, sa_stream_t stream);

/* Fine stage backward with the block mask held constant (VSA2 page 2.1: the router's
 * output carries no gradient).  Inputs as for sa_forward plus out, out_f32 and lse from
 * it and dout [B,H,Npad,D] bf16.  Delta = rowsum(dO * O) is taken from out_f32 when it is
 * not NULL, else from the bf16 out; bf16 rounding of O enters dS = P * (dP - Delta) as an
 * absolute error on every selected key and is multiplied by |k| in dQ, which matters for
 * sink keys of large norm, so pass out_f32 when training.
 * Outputs dq, dk, dv: [B,H,Npad,D] fp32:
 *   P = exp(scale*QK^T - lse), dV = P^T dO, dP = dO V^T, Delta = rowsum(dO * O),
 *   dS = P * (dP - Delta), dQ = scale * dS K, dK = scale * dS^T Q.
 * Padding rows of every output are 0; dout of padding rows is ignored.
 * bf16 only (qk_dtype must be SA_BF16).  Deterministic. */
SA_API sa_status sa_backward(const void* q, const void* k, const void* v, const void* out, const float* out_f32,
                      const float* lse, const void* dout, const int32_t* kv_index, const int32_t* kv_count, const sa_params* p,
                      float* dq, float* dk, float* dv, void* ws, size_t ws_bytes, sa_stream_t stream);

/* ---- Coarse branch and gated combination ----
 * VSA page, "Big-Picture Architecture" item 2, "What the coarse attention output O_c
 * provides" and "Gated Combination"; VSA2 page, section 2.2 "Coarse Branch" and the gate
 * equation.  Per head, with Qc, Kc, Vc the means of the valid tokens of each cube:
 *   Pc = softmax(Qc Kc^T * scale)  (dense, T x T),   Oc^ = Pc Vc,
 *   O  = G (.) Repeat_64(Oc^) + O_f,   O_f the fine stage's output (sa_forward).
 * G is one scalar per token and head, the gate VALUE (VSA2's tanh(X W_g); the projection
 * and its tanh belong to the caller's linear layers, and the backward returns dL/dG).
 * VSA's fine gate is taken as 1 (its sparse adaptation removes it).  Padding slots get
 * O = 0 whatever G holds there, and dG = 0.  bf16 only (qk_dtype SA_BF16, else
 * SA_ERR_UNSUPPORTED); B*H <= 65535.  The cube-level tensors are caller-owned fp32 device
 * arrays: qbar, kbar, vbar, oc [B,H,T,D] (16-byte aligned), lse [B,H,T] (natural log of
 * each row's normaliser of the scaled cube scores). */
typedef struct {
  float* qbar;
  float* kbar;
  float* vbar;
  float* oc;
  float* lse;
} sa_coarse;

/* Router and coarse branch in one call: the same kv_index / kv_count as sa_plan (same
 * kernels, bit-identical), and the cube-level tensors of `coarse` (written).  Q and K are
 * pooled once for both (the coarse branch reads the router's fp64 means, and every scaled score, which
 * the router's score kernel also writes in fp32 for this call: the exact limb dot product rounded once).
 * v: [B,H,Npad,D] bf16.  Workspace: sa_workspace_size(p, SA_OP_PLAN_COARSE).
 * Deterministic. */
SA_API sa_status sa_plan_coarse(const void* q, const void* k, const void* v, const sa_params* p, int32_t* kv_index,
                                int32_t* kv_count, const sa_coarse* coarse, void* ws, size_t ws_bytes,
                                sa_stream_t stream);

/* sa_forward (arguments, errors and outputs as there, bf16 only) with the gated combination
 * O = G (.) Repeat_64(coarse->oc) + O_f formed in the forward kernel's epilogue from the fp32
 * O_f of each valid row (one fused multiply-add per value): out_f32 receives the fp32 sum and
 * out its bf16 rounding; padding rows stay 0.  out_f32 is REQUIRED (SA_ERR_INVALID_ARG when
 * NULL): sa_backward_gated recovers the fine branch's Delta from it.
 * gate: [B,H,Npad] fp32.  lse is the fine stage's.  Workspace:
 * sa_workspace_size(p, SA_OP_FORWARD).  Deterministic. */
SA_API sa_status sa_forward_gated(const void* q, const void* k, const void* v, const int32_t* kv_index,
                                  const int32_t* kv_count, const sa_params* p, const sa_coarse* coarse,
                                  const float* gate, void* out, float* lse, float* out_f32, void* ws, size_t ws_bytes,
                                  sa_stream_t stream);

/* Gradients of the gated output, mask held constant: dq, dk, dv [B,H,Npad,D] fp32 are the
 * fine stage's (as sa_backward, with dO_f = dO) plus the coarse branch's,
 *   dG_t = <dO_t, Oc^[i]>,  dOc^[i] = sum_t G_t dO_t  (t over the valid tokens of cube i),
 *   dVc = Pc^T dOc^,  dPc = dOc^ Vc^T,  dSc = Pc (.) (dPc - rowsum(Pc (.) dPc)),
 *   dQc = scale dSc Kc,  dKc = scale dSc^T Qc,
 * each cube-level gradient handed to the n_i valid tokens of its cube as dXc[i] / n_i.
 * out / out_f32: the combined output from sa_forward_gated; out_f32 is REQUIRED here
 * (SA_ERR_INVALID_ARG when NULL): the fine stage's Delta is taken as <dO, O> - G dG, and
 * from the bf16 rounding of the combined O it exceeds the gradient error bounds.  coarse: as written by sa_plan_coarse (read only).  gate: [B,H,Npad]
 * fp32; dgate: [B,H,Npad] fp32 (0 on padding slots).  Workspace:
 * sa_workspace_size(p, SA_OP_BACKWARD_GATED).  Deterministic. */
SA_API sa_status sa_backward_gated(const void* q, const void* k, const void* v, const void* out, const float* out_f32,
                                   const float* lse, const void* dout, const float* gate, const int32_t* kv_index,
                                   const int32_t* kv_count, const sa_params* p, const sa_coarse* coarse, float* dq,
                                   float* dk, float* dv, float* dgate, void* ws, size_t ws_bytes, sa_stream_t stream);

/* Router with 128-token query blocks and 64-token key blocks (SpargeAttention2 page,
 * "Block-Pooled Attention for Efficient Mask Construction" step 1: b_q = 128, b_kv = 64 in all
 * its experiments).  On the cube layout query block i is cubes 2i and 2i+1 (the last block is
 * one cube when T is odd), pooled over the valid tokens of both; keys stay per cube.  Scores,
 * row softmax, Top-k / Top-p and ties as sa_plan, over the ceil(T/2) x T block matrix (top_k
 * counts key cubes).  Output in sa_plan's per-cube layout, kv_index [B,H,T,kv_capacity] and
 * kv_count [B,H,T], with both cubes of a block holding the block's list, so sa_forward and
 * sa_backward take it as is.  bf16 only.  B*H <= 65535.  Workspace:
 * sa_workspace_size(p, SA_OP_PLAN_BQ128).  Deterministic. */
SA_API sa_status sa_plan_bq128(const void* q, const void* k, const sa_params* p, int32_t* kv_index, int32_t* kv_count,
                               void* ws, size_t ws_bytes, sa_stream_t stream);

/* VSA2's fine-grained router with per-sequence Top-K (VSA2 page, section 2.2, router
 * equations): each cube splits into G = 64 / (rt*rh*rw) groups (an rt x rh x rw box of its
 * (t, h, w) offsets), each group is pooled over its valid tokens (Q_r, K_r = MeanPool_R), the
 * group-level scores Q_r K_r^T * scale get a softmax over every key group of the sequence per
 * query group, the G x G aggregation gives one score per (query cube, key cube) (P_r[i, j] = the
 * mass a query group of cube i puts on the key groups of cube j, averaged over cube i's valid
 * query groups), and per-sequence Top-K keeps the min(top_k * T, T^2) largest entries of P_r of
 * each (batch, head), ties by the smaller row-major index (top_p is not used).  A group without
 * valid tokens takes no part.  Each R_x is 1, 2 or 4 with G in {4, 8, 16} (else
 * SA_ERR_UNSUPPORTED); bf16 only.  Outputs: kv_index / kv_count in sa_plan's layout (a row may
 * keep no block; more than kv_capacity records SA_ERR_CAPACITY), and P_r [B,H,T,T] fp32 in p_r when
 * it is not NULL.  The scores are exact integer limb products on the tensor cores (as sa_plan's);
 * the softmax uses fp32 exponentials, so P_r is within a few 1e-6 relative of its fp64 value and
 * the selection is that of this fp32 P_r.  Workspace: sa_plan_fine_workspace_size(p, rt, rh, rw).
 * Deterministic. */
SA_API size_t sa_plan_fine_workspace_size(const sa_params* p, int rt, int rh, int rw);
SA_API sa_status sa_plan_fine(const void* q, const void* k, const sa_params* p, int rt, int rh, int rw,
                              int32_t* kv_index, int32_t* kv_count, float* p_r, void* ws, size_t ws_bytes,
                              sa_stream_t stream);

/* Router recall diagnostic (SpargeAttention2 page, equation 8: tau = sum_j p_j m_j, the share of a
 * query's true softmax mass inside its kept blocks; VSA page, "Kernel Implementation": Top-32
 * keeps 50-90%).  Since lse is the log of a row's softmax normaliser, tau = exp(lse_kept -
 * lse_all), with lse_kept from sa_forward on the router's lists and lse_all from sa_forward on
 * lists holding every block (kv_capacity = T).  lse_kept, lse_all: [B,H,Npad] fp32.
 * recall: [B,H,Npad] fp32, tau per valid row, 0 on padding rows (may be NULL).
 * cube_recall: [B,H,T] fp32, the mean of tau over each cube's valid rows (may be NULL; not both).
 * Asynchronous, one launch, no workspace.  Deterministic. */
SA_API sa_status sa_recall(const float* lse_kept, const float* lse_all, const sa_params* p, float* recall,
                           float* cube_recall, sa_stream_t stream);

/* Oracle block scores P_oracle (VSA2 page, section 2.2: MeanPool over the B x B tiles of the
 * token-level softmax P, the reference the router approximates): pblock[b,h,i,j] = the softmax
 * mass the valid query tokens of cube i put on the valid keys of cube j, averaged over cube i's
 * valid tokens (each row sums to 1).  lse_all: [B,H,Npad] fp32, the lse of sa_forward on lists
 * holding every block; then P_rc = exp(s_rc * scale - lse_r) and one dense tensor-core pass of
 * S = Q K^T gives every entry.  q, k: [B,H,Npad,D] bf16; pblock: [B,H,T,T] fp32.  Workspace:
 * sa_workspace_size(p, SA_OP_BLOCK_MASS) (status block + cube masks); bounded waits report
 * SA_ERR_DEVICE_TIMEOUT through sa_get_device_status.  Cost: a dense S product over every token
 * pair (2 * B*H*Npad^2*D FLOP) plus one exponential per pair: a diagnostic, not the step.
 * Deterministic. */
SA_API sa_status sa_block_mass(const void* q, const void* k, const float* lse_all, const sa_params* p, float* pblock,
                               void* ws, size_t ws_bytes, sa_stream_t stream);

/* Best recall of a selection size (VSA2 page, section 2.2, P_oracle; VSA page, "Kernel
 * Implementation": Top-32 keeps 50-90% of the mass): best[b,h,i] = the sum of the n largest
 * entries of row i of pblock, n = kv_count[b,h,i] clamped to [0, T]: the most recall any choice
 * of n key cubes could reach, beside sa_recall's cube_recall of the router's own choice.
 * pblock: [B,H,T,T] fp32 (non-negative); kv_count: [B,H,T] int32; best: [B,H,T] fp32.  One
 * launch, no workspace.  Deterministic. */
SA_API sa_status sa_best_recall(const float* pblock, const int32_t* kv_count, const sa_params* p, float* best,
                                sa_stream_t stream);

/* sa_plan without a workspace: the same router and the same results, for callers that
 * cannot allocate device memory (code running under a CUDA stream capture, serving
 * processes confined to a pre-reserved memory arena, C callers with no device
 * allocator).  The pages have no counterpart to it; it is a deployment convenience.
 * Scratch lives in one fixed device array of 64 MiB that every GPU loading the library
 * holds until exit; problems needing more (sa_workspace_size(p, SA_OP_PLAN) > 64 MiB,
 * e.g. 12 heads at the 480p shape fit, 40 heads at 720p do not) return SA_ERR_WORKSPACE.
 * kv_capacity must equal T, so no row can be clipped and there is no device status to
 * read.  Outside a stream capture every call looks up the array's device address on the
 * current device; inside a capture the address cached by an earlier call is used, so the first
 * call on a device must come before any stream capture.  All calls share the array: calls that overlap on the GPU race and
 * must be serialised by the caller.  Allocates nothing (no cudaMalloc/cudaFree). */
SA_API sa_status sa_plan_static(const void* q, const void* k, const float* q_scale, const float* k_scale,
                                const sa_params* p, int32_t* kv_index, int32_t* kv_count, sa_stream_t stream);

/* ---- One step from and to host memory ----
 * The whole hot path of one training step on host buffers: the layout of the VSA page
 * ("Cube Partitioning and Token Re-Indexing"), sa_plan, sa_forward (with its fp32 output)
 * and sa_backward as documented above, and the layout back, with the host<->device copies
 * overlapped with the work.  The B*H (batch, head) problems are independent, so the step
 * runs over chunks of chunk_heads consecutive problems of the flattened [B*H] axis (the
 * last chunk may be shorter): chunk c's inputs are copied in while chunk c-1 is computed
 * and chunk c-2's results are copied out (two internal copy streams, two buffer slots in
 * the workspace, events between them).  Results equal those of the device entry points
 * run on the same data.  bf16 only (qk_dtype SA_BF16, else SA_ERR_UNSUPPORTED); B*H <= 65535.
 * q, k, v, dout: HOST [B,H,lat_t*lat_h*lat_w,D] bf16 in latent (t, h, w) order.
 * out: HOST [B,H,L,D] bf16; dq, dk, dv: HOST [B,H,L,D] fp32 (L = lat_t*lat_h*lat_w).
 * Host buffers should be page-locked (cudaHostAlloc, or pinned tensors) for the copies to
 * run asynchronously; pageable memory works but serialises the copies with the host.  The
 * caller keeps every host buffer alive and unmodified until `stream` has been synchronised.
 * ws: device workspace of sa_step_host_workspace_size(p, chunk_heads) bytes, 16-byte
 * aligned; its first 256 bytes gather the device status of every chunk's calls
 * (sa_get_device_status(ws, stream)).  All device work is ordered on `stream`: it starts
 * after the work already queued there, and work queued after the call starts after the
 * last copy-out.  Returns the first host-side error of any chunk's calls (SA_ERR_* as for
 * those entry points); nothing more is issued after it. */
SA_API size_t sa_step_host_workspace_size(const sa_params* p, int chunk_heads);
SA_API sa_status sa_step_host(const void* q, const void* k, const void* v, const void* dout, const sa_params* p,
                              int chunk_heads, void* out, float* dq, float* dk, float* dv, void* ws,
                              size_t ws_bytes, sa_stream_t stream);

/* Synchronises `stream`, then maps the workspace's device status block to a status:
 * SA_OK, SA_ERR_DEVICE_TIMEOUT, SA_ERR_DEVICE_INDEX or SA_ERR_CAPACITY (first that
 * applies, in that order of precedence: timeout, index, capacity). */
SA_API sa_status sa_get_device_status(const void* ws, sa_stream_t stream);

/* Synchronises `stream` and returns how many rows the last sa_plan on this workspace decided
 * on its fp64 path; -1 on error. */
SA_API int sa_plan_fallback_rows(const void* ws, sa_stream_t stream);

/* Per-CTA clock records of the attention kernels, written by the last sa_forward (kernel 0,
 * the forward) or sa_backward / sa_backward_gated (kernel 1, dQ; kernel 2, dK/dV) that ran on
 * this workspace with SA_DEBUG_CTA_CLOCKS in p->debug_flags.  Synchronises `stream`, then
 * copies min(grid, max_ctas, 1024) records into `out` (host memory, 4 values each: start and
 * end in globaltimer nanoseconds, the work items and the pipeline steps the CTA processed) and
 * sets *n_ctas to that number (0 when the call ran without the flag).  The kernels take their
 * work items in order from a shared counter, each CTA the next one when it is free, so the
 * records measure how evenly the dynamic schedule loaded the SMs.
 * ws / ws_bytes: a workspace of sa_workspace_size(p, SA_OP_FORWARD or SA_OP_BACKWARD[_GATED]).
 * Returns SA_ERR_INVALID_ARG for a null pointer, kernel outside 0..2 or a workspace too small
 * to hold the records, SA_ERR_LAUNCH when the copy fails. */
SA_API sa_status sa_get_cta_clocks(const void* ws, size_t ws_bytes, int kernel, unsigned long long* out,
                                   int max_ctas, int* n_ctas, sa_stream_t stream);

SA_API const char* sa_status_string(sa_status s);

/* Number of kernels the most recent call of each entry point launched on this host
 * thread (for launch accounting in benchmarks). */
SA_API int sa_last_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* SA_H_ */
