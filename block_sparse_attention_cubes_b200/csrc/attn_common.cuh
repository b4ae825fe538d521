// Pieces shared by the fine-stage kernels (forward, dQ, dK/dV).
#pragma once
#include <cuda_bf16.h>

#include "geometry.cuh"
#include "ptx.cuh"

namespace sa {

struct AttnArgs {
  const int32_t* kv_index;  // [BH, T, cap]
  const int32_t* kv_count;  // [BH, T]
  const float* q_scale;     // [BH, T] (fp8 only)
  const float* k_scale;
  __nv_bfloat16* out;       // forward output [BH, Npad, D]
  float* out_f32;           // optional fp32 copy of the forward output
  const unsigned int* f16_bad;  // forward with out_f32: nonzero when V did not fit fp16 (then P as bf16 hi + lo)
  const unsigned int* f16_single;  // backward: 1 when Q, K, V, dO and dS fit fp16 (single fp16 products)
  const float* gate;        // gated forward: G per token [BH, Npad] and the coarse output Oc^ [BH, T, D]
  const float* oc;          //   (O = G Oc^[cube] + O_f on the valid rows, formed in the epilogue)
  const unsigned long long* cube_mask;  // [T] valid-slot mask of every cube
  const int32_t* u_list;    // query-pair unions: [BH, ceil(T/2), ucap] (block << 2 | membership bits)
  const int32_t* u_cnt;     // [BH, ceil(T/2)]
  const int32_t* uk_list;   // key-pair unions of the transposed lists: [BH, ceil(T/2), T]
  const int32_t* uk_cnt;
  int ucap;                 // row stride of u_list: min(2 * cap, T)
  float* lse;               // [BH, Npad]
  const float* delta;       // backward: rowsum(dO * O) [BH, Npad]
  const float* nlse2;       // backward: -lse * log2(e) [BH, Npad]
  float* dq;
  float* dk;
  float* dv;
  DevStatus* st;
  Geom g;
  int BH, D, cap;
  int qk_fp8;               // Q and K are e4m3 bytes with per-cube scales q_scale / k_scale
  int rows_total;           // BH * Npad, the first out-of-range row for zero-filled loads
  float scale;              // softmax scale
  float scale_log2;         // softmax scale * log2(e)
  unsigned long long timeout_ns;
  unsigned int debug;
  unsigned int* item_next;        // work-item counters [3] (forward, dQ, dK/dV), zeroed before the launch
  unsigned long long* cta_clock;  // optional per-CTA records [3][kClockCtas][4]: start, end (ns), items, steps
  unsigned int* clock_grid;       // with cta_clock: [3] grid sizes
};
constexpr int kClockCtas = 1024;  // per-CTA clock records kept per kernel

// ------------------------------------------------------------------ dynamic item order
// Work items (pairs of cubes) go, in their natural order, to whichever CTA is free: CTA c
// starts with item c and takes each later one from a per-launch counter.  Neighbouring items
// belong to the same head and share most of their K/V tiles, so the CTAs at work at any
// moment keep reading the same lines of L2, and no CTA is left with a longer static share.
// One thread (the first producer lane) fetches every id into a small shared ring; each of
// the kernel's other roles reads the same sequence from it and signals the slot free.
constexpr int kItemRing = 4;
constexpr unsigned int kDebugStaticItems = 8u;  // debug flag: item n of CTA c is c + n * gridDim.x
constexpr uint32_t kRingReaders = 10;  // the second producer lane, the MMA warp, eight epilogue warps
struct ItemRing {
  volatile int* ids;  // [kItemRing]; -1 once no item is left
  uint64_t* full;     // [kItemRing], one arrival (the fetching thread)
  uint64_t* empty;    // [kItemRing], kRingReaders arrivals
};

// The fetching thread: item n of this CTA, published in slot n % kItemRing.
__device__ __forceinline__ int ring_publish(const ItemRing& r, int n, int n_items, const AttnArgs& a,
                                            unsigned int* counter, unsigned int where, bool& ok) {
  const int slot = n % kItemRing;
  if (n >= kItemRing && !mbar_wait(&r.empty[slot], ((n / kItemRing) + 1) & 1, a.st, a.timeout_ns, where)) {
    ok = false;
    return -1;
  }
  int it;
  if (a.debug & kDebugStaticItems)  // measurement hook: the fixed round-robin share instead
    it = static_cast<int>(blockIdx.x) + n * static_cast<int>(gridDim.x);
  else
    it = n == 0 ? static_cast<int>(blockIdx.x) : static_cast<int>(gridDim.x + atomicAdd(counter, 1u));
  if (it >= n_items) it = -1;
  r.ids[slot] = it;
  mbar_arrive(&r.full[slot]);
  return it;
}

// One reading thread (a producer lane).
__device__ __forceinline__ int ring_read(const ItemRing& r, int n, const AttnArgs& a, unsigned int where, bool& ok) {
  const int slot = n % kItemRing;
  if (!mbar_wait(&r.full[slot], (n / kItemRing) & 1, a.st, a.timeout_ns, where)) {
    ok = false;
    return -1;
  }
  const int it = r.ids[slot];
  mbar_arrive(&r.empty[slot]);
  return it;
}

// A whole converged warp (the MMA warp): one arrival.
__device__ __forceinline__ int ring_read_warp(const ItemRing& r, int n, const AttnArgs& a, unsigned int where,
                                              bool& ok) {
  const int slot = n % kItemRing;
  if (!mbar_wait_warp(&r.full[slot], (n / kItemRing) & 1, a.st, a.timeout_ns, where)) {
    ok = false;
    return -1;
  }
  const int it = r.ids[slot];
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&r.empty[slot]);
  return it;
}

// The epilogue threads (named barrier 1 over `nthreads`): they agree on success through the
// shared abort flag behind the barrier, so they leave their loops together; one arrival per warp.
__device__ __forceinline__ int ring_read_group(const ItemRing& r, int n, const AttnArgs& a, unsigned int where,
                                               volatile int* sm_abort, bool& ok, uint32_t nthreads = 256) {
  const int slot = n % kItemRing;
  if (!mbar_wait(&r.full[slot], (n / kItemRing) & 1, a.st, a.timeout_ns, where)) *sm_abort = 1;
  named_bar_sync(1, nthreads);
  if (*sm_abort) {
    ok = false;
    return -1;
  }
  const int it = r.ids[slot];
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&r.empty[slot]);
  return it;
}

// Per-CTA clock record of kernel `kid` (thread 0, when records were asked for): start and end
// in globaltimer nanoseconds, the items and steps this CTA processed.
__device__ __forceinline__ void cta_clock_record(const AttnArgs& a, int kid, unsigned long long t0, int items,
                                                 uint32_t steps) {
  if (a.cta_clock == nullptr || blockIdx.x >= static_cast<unsigned>(kClockCtas)) return;
  if (blockIdx.x == 0) a.clock_grid[kid] = gridDim.x;
  unsigned long long* c = a.cta_clock + 4ull * (static_cast<unsigned long long>(kid) * kClockCtas + blockIdx.x);
  c[0] = t0;
  c[1] = globaltimer_ns();
  c[2] = static_cast<unsigned long long>(items);
  c[3] = steps;
}

// bf16 pair of (v0, v1) into hi, and with the remainders (v - bf16(v)) as a second bf16 pair
// into lo: hi + lo carries v to about 16 bits.
__device__ __forceinline__ void split_bf16x2(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(v0, v1);
  float r0, r1;
  upk2(sub2(pk2(v0, v1), pk2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u))), r0, r1);
  lo = pack_bf16x2(r0, r1);
}

// Block id t of query block i's list, or -1 when t is past the count or the entry is
// out of range (the latter is recorded as an index error).
__device__ __forceinline__ int list_entry(const AttnArgs& a, int bh, int i, int n, int t, bool report) {
  if (t >= n) return -1;
  const int j = __ldg(a.kv_index + (static_cast<size_t>(bh) * a.g.T + i) * a.cap + t);
  if (j < 0 || j >= a.g.T) {
    if (report) flag_error(a.st, DEVERR_INDEX, 0);
    return -1;
  }
  return j;
}

__device__ __forceinline__ int list_count(const AttnArgs& a, int bh, int i, bool report) {
  int n = __ldg(a.kv_count + static_cast<size_t>(bh) * a.g.T + i);
  if (n < 0 || n > a.cap) {
    if (report) flag_error(a.st, DEVERR_INDEX, 0);
    n = n < 0 ? 0 : a.cap;
  }
  return n;
}

struct OpMax {
  __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct OpSum {
  __device__ __forceinline__ float operator()(float a, float b) const { return a + b; }
};

// Reduce 64 per-thread column values over the 32 lanes of a warp by recursive halving:
// at the end lane l holds columns c0, c0+1 with c0 = 32*b4 + 16*b3 + 8*b2 + 4*b1 + 2*b0
// (b = bits of l) in v[0], v[1].  62 shuffles instead of 64 x 5.
template <class Op>
__device__ __forceinline__ int warp_colreduce64(float (&v)[64], int lane, Op op) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const bool hi = lane & 16;
    const float send = hi ? v[i] : v[i + 32];
    const float keep = hi ? v[i + 32] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const bool hi = lane & 8;
    const float send = hi ? v[i] : v[i + 16];
    const float keep = hi ? v[i + 16] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 4;
    const float send = hi ? v[i] : v[i + 8];
    const float keep = hi ? v[i + 8] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 2;
    const float send = hi ? v[i] : v[i + 4];
    const float keep = hi ? v[i + 4] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 1;
    const float send = hi ? v[i] : v[i + 2];
    const float keep = hi ? v[i + 2] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 1));
  }
  return 32 * ((lane >> 4) & 1) + 16 * ((lane >> 3) & 1) + 8 * ((lane >> 2) & 1) + 4 * ((lane >> 1) & 1) +
         2 * (lane & 1);
}

// Same reduction for 32 column values: lane l ends with column l in v[0] (31 shuffles).
template <class Op>
__device__ __forceinline__ int warp_colreduce32(float (&v)[32], int lane, Op op) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const bool hi = lane & 16;
    const float send = hi ? v[i] : v[i + 16];
    const float keep = hi ? v[i + 16] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 8;
    const float send = hi ? v[i] : v[i + 8];
    const float keep = hi ? v[i + 8] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 4;
    const float send = hi ? v[i] : v[i + 4];
    const float keep = hi ? v[i + 4] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 2;
    const float send = hi ? v[i] : v[i + 2];
    const float keep = hi ? v[i + 2] : v[i];
    v[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  }
  {
    const bool hi = lane & 1;
    const float send = hi ? v[0] : v[1];
    const float keep = hi ? v[1] : v[0];
    v[0] = op(keep, __shfl_xor_sync(0xffffffffu, send, 1));
  }
  return lane;
}

// Store 32 bf16 values as columns 32*half .. 32*half+31 (64 bytes, chunks 4*half..4*half+3)
// of row `row` of a 128-byte-swizzled tile.
__device__ __forceinline__ void store_half_row_bf16_sw128(uint32_t tile_base, uint32_t row, int half,
                                                          const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t a = pack_bf16x2(v[8 * c + 0], v[8 * c + 1]);
    const uint32_t b = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
    const uint32_t cc = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
    const uint32_t d = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
    st_shared_v4(tile_base + sw128_offset(row, 4 * half + c), a, b, cc, d);
  }
}

// hi + lo version of the above (hi = bf16(v), lo = bf16(v - hi))
__device__ __forceinline__ void store_half_row_bf16x2_sw128(uint32_t base_hi, uint32_t base_lo, uint32_t row,
                                                            int half, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float x0 = v[8 * c + 2 * u], x1 = v[8 * c + 2 * u + 1];
      h[u] = pack_bf16x2(x0, x1);
      l[u] = pack_bf16x2(x0 - __uint_as_float(h[u] << 16), x1 - __uint_as_float(h[u] & 0xffff0000u));
    }
    const uint32_t off = sw128_offset(row, 4 * half + c);
    st_shared_v4(base_hi + off, h[0], h[1], h[2], h[3]);
    st_shared_v4(base_lo + off, l[0], l[1], l[2], l[3]);
  }
}

// Store one 64-element bf16 row (128 bytes) of a 128-byte-swizzled tile.
__device__ __forceinline__ void store_row_bf16_sw128(uint32_t tile_base, uint32_t row, const float (&v)[64]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t a = pack_bf16x2(v[8 * c + 0], v[8 * c + 1]);
    const uint32_t b = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
    const uint32_t cc = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
    const uint32_t d = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
    st_shared_v4(tile_base + sw128_offset(row, c), a, b, cc, d);
  }
}

// Store a 64-element row as two bf16 rows hi + lo with hi = bf16(v) and lo = bf16(v - hi),
// so that hi + lo carries v to about 2^-16 relative.  Products that are summed over many
// query rows (dV of a popular key, dK and dQ next to a large sink key) use both halves.
__device__ __forceinline__ void store_row_bf16x2_sw128(uint32_t base_hi, uint32_t base_lo, uint32_t row,
                                                       const float (&v)[64]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float a = v[8 * c + 2 * u], b = v[8 * c + 2 * u + 1];
      h[u] = pack_bf16x2(a, b);
      const float ha = __uint_as_float(h[u] << 16), hb = __uint_as_float(h[u] & 0xffff0000u);
      l[u] = pack_bf16x2(a - ha, b - hb);
    }
    const uint32_t off = sw128_offset(row, c);
    st_shared_v4(base_hi + off, h[0], h[1], h[2], h[3]);
    st_shared_v4(base_lo + off, l[0], l[1], l[2], l[3]);
  }
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r0[32], r1[32];
  tmem_ld32(taddr, r0);
  tmem_ld32(taddr + 32, r1);
  tmem_ld_wait();
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    v[c] = __uint_as_float(r0[c]);
    v[c + 32] = __uint_as_float(r1[c]);
  }
}

__device__ __forceinline__ void tmem_st64(uint32_t taddr, const float (&v)[64]) {
  uint32_t r0[32], r1[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    r0[c] = __float_as_uint(v[c]);
    r1[c] = __float_as_uint(v[c + 32]);
  }
  tmem_st32(taddr, r0);
  tmem_st32(taddr + 32, r1);
  tmem_st_wait();
}

}  // namespace sa
