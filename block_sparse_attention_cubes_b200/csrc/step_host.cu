// sa_step_host: one step of the hot path (layout, router, fine forward, fine backward, layout
// back) from and to host memory, with the host<->device copies overlapped with the work.
//
// The B*H (batch, head) problems are independent (the router, the forward and the backward
// treat every head on its own), so the step runs over chunks of `chunk_heads` consecutive
// heads of the flattened [B*H] axis, each chunk being the problem B = 1, H = chunk size.
// Three streams, two buffer slots:
//   copy-in stream    chunk c's q, k, v, dO: host -> latent slot c % 2 (one cudaMemcpyAsync each)
//   caller's stream   tile, sa_plan, sa_forward, sa_backward, untile into output slot c % 2
//   copy-out stream   output slot c % 2 -> host (out bf16, dq, dk, dv fp32)
// Events order the slots: an input slot is refilled only after the tiling of the chunk two
// back has read it, an output slot is rewritten only after the copy-out of the chunk two back
// has finished, so chunk c's copy-in, chunk c-1's work and chunk c-2's copy-out overlap.
// Every device status of the chunks' calls is folded into the status block at the head of
// the step's workspace (read with sa_get_device_status).
#include <cstring>

#include "../../include/sa.h"
#include "ptx.cuh"

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct StepLayout {
  size_t lat_in[2][4];   // latent inputs q, k, v, dO of each slot (bf16)
  size_t tiled[4];       // cube-major q, k, v, dO (bf16)
  size_t kv_index, kv_count;
  size_t out_t, lse, out32;
  size_t grad_t[3];      // cube-major dq, dk, dv (fp32)
  size_t lat_out[2][4];  // latent out (bf16), dq, dk, dv (fp32) of each slot
  size_t ws_op[3];       // the plan, forward and backward workspaces
  size_t ws_bytes[3];
  size_t total;
};

// The chunk's parameters: the same problem with B = 1 and H = n heads.
sa_params chunk_params(const sa_params* p, int n) {
  sa_params c = *p;
  c.B = 1;
  c.H = n;
  return c;
}

bool step_layout(const sa_params* p, int chunk, StepLayout* L) {
  const int npad = sa_padded_tokens(p), T = sa_num_cubes(p);
  if (npad <= 0 || T <= 0) return false;
  const sa_params c = chunk_params(p, chunk);
  const size_t lat = static_cast<size_t>(p->lat_t) * p->lat_h * p->lat_w;
  const size_t n = static_cast<size_t>(chunk), D = static_cast<size_t>(p->D);
  size_t o = 256;  // the step's status block
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  for (int s = 0; s < 2; ++s)
    for (int t = 0; t < 4; ++t) L->lat_in[s][t] = take(n * lat * D * 2);
  for (int t = 0; t < 4; ++t) L->tiled[t] = take(n * npad * D * 2);
  L->kv_index = take(n * T * static_cast<size_t>(p->kv_capacity) * 4);
  L->kv_count = take(n * T * 4);
  L->out_t = take(n * npad * D * 2);
  L->lse = take(n * npad * 4);
  L->out32 = take(n * npad * D * 4);
  for (int t = 0; t < 3; ++t) L->grad_t[t] = take(n * npad * D * 4);
  for (int s = 0; s < 2; ++s)
    for (int t = 0; t < 4; ++t) L->lat_out[s][t] = take(n * lat * D * (t == 0 ? 2 : 4));
  const int ops[3] = {SA_OP_PLAN, SA_OP_FORWARD, SA_OP_BACKWARD};
  for (int i = 0; i < 3; ++i) {
    L->ws_bytes[i] = sa_workspace_size(&c, ops[i]);
    if (L->ws_bytes[i] == 0) return false;
    L->ws_op[i] = take(L->ws_bytes[i]);
  }
  L->total = o;
  return true;
}

// Fold an operation's device status into the step's: error bits OR-ed, the first timeout's
// wait code kept, fp64 router rows added up.
__global__ void status_fold_kernel(sa::DevStatus* dst, const sa::DevStatus* src) {
  if (threadIdx.x != 0) return;
  if (src->error && !dst->error) dst->where = src->where;
  dst->error |= src->error;
  dst->abort |= src->abort;
  dst->router_fallback += src->router_fallback;
}

}  // namespace

namespace sa {
void set_last_launches(int n);
}

extern "C" {

size_t sa_step_host_workspace_size(const sa_params* p, int chunk_heads) {
  if (!p || p->B < 1 || p->H < 1 || chunk_heads < 1) return 0;
  const long long bh = static_cast<long long>(p->B) * p->H;
  if (bh > 65535) return 0;
  if (sa_workspace_size(p, SA_OP_BACKWARD) == 0) return 0;  // the parameters themselves are valid
  StepLayout L;
  return step_layout(p, static_cast<int>(chunk_heads < bh ? chunk_heads : bh), &L) ? L.total : 0;
}

sa_status sa_step_host(const void* q, const void* k, const void* v, const void* dout, const sa_params* p,
                       int chunk_heads, void* out, float* dq, float* dk, float* dv, void* ws, size_t ws_bytes,
                       sa_stream_t stream) {
  sa::set_last_launches(0);
  if (!p || !q || !k || !v || !dout || !out || !dq || !dk || !dv || chunk_heads < 1) return SA_ERR_INVALID_ARG;
  if (p->qk_dtype != SA_BF16 || (p->D != 64 && p->D != 128)) return SA_ERR_UNSUPPORTED;
  const size_t need = sa_step_host_workspace_size(p, chunk_heads);
  if (need == 0) return SA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < need) return SA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 15u) != 0) return SA_ERR_ALIGNMENT;
  const int BH = p->B * p->H;
  const int chunk = chunk_heads < BH ? chunk_heads : BH;
  StepLayout L;
  step_layout(p, chunk, &L);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  // copy streams and the events that order the two buffer slots
  enum { E_START, E_END_IN, E_END_OUT, E_IN_DONE, E_IN_FREE = E_IN_DONE + 2, E_WORK_DONE = E_IN_FREE + 2,
         E_OUT_FREE = E_WORK_DONE + 2, NEV = E_OUT_FREE + 2 };
  cudaStream_t sin = nullptr, sout = nullptr;
  cudaEvent_t ev[NEV] = {};
  bool setup = cudaStreamCreateWithFlags(&sin, cudaStreamNonBlocking) == cudaSuccess &&
               cudaStreamCreateWithFlags(&sout, cudaStreamNonBlocking) == cudaSuccess;
  for (int i = 0; setup && i < NEV; ++i) setup = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) == cudaSuccess;
  auto release = [&]() {
    for (int i = 0; i < NEV; ++i)
      if (ev[i]) cudaEventDestroy(ev[i]);  // released once the work recorded on them is done
    if (sin) cudaStreamDestroy(sin);
    if (sout) cudaStreamDestroy(sout);
  };
  if (!setup) {
    release();
    return SA_ERR_LAUNCH;
  }
  sa_status rc = SA_OK;
  auto cu = [&](cudaError_t e) {
    if (e != cudaSuccess && rc == SA_OK) rc = SA_ERR_LAUNCH;
    return rc == SA_OK;
  };
  auto sa_ok = [&](sa_status s) {
    if (s != SA_OK && rc == SA_OK) rc = s;
    return rc == SA_OK;
  };
  int launches = 0;
  // the step's status block starts clear; the copy streams start after the caller's earlier work
  if (cu(cudaMemsetAsync(ws, 0, 256, cs)) && cu(cudaEventRecord(ev[E_START], cs))) {
    cu(cudaStreamWaitEvent(sin, ev[E_START], 0));
    cu(cudaStreamWaitEvent(sout, ev[E_START], 0));
  }

  const size_t lat = static_cast<size_t>(p->lat_t) * p->lat_h * p->lat_w;
  const size_t row16 = lat * p->D * 2, row32 = lat * p->D * 4;  // bytes of one head, bf16 / fp32
  const uint8_t* src[4] = {static_cast<const uint8_t*>(q), static_cast<const uint8_t*>(k),
                           static_cast<const uint8_t*>(v), static_cast<const uint8_t*>(dout)};
  uint8_t* dst[4] = {static_cast<uint8_t*>(out), reinterpret_cast<uint8_t*>(dq), reinterpret_cast<uint8_t*>(dk),
                     reinterpret_cast<uint8_t*>(dv)};
  const size_t dst_row[4] = {row16, row32, row32, row32};
  sa::DevStatus* step_st = static_cast<sa::DevStatus*>(ws);
  auto fold = [&](int op) {
    status_fold_kernel<<<1, 32, 0, cs>>>(step_st, reinterpret_cast<const sa::DevStatus*>(wb + L.ws_op[op]));
    ++launches;
    return cu(cudaGetLastError());
  };
  const int nchunks = (BH + chunk - 1) / chunk;
  for (int c = 0; rc == SA_OK && c < nchunks; ++c) {
    const int slot = c & 1, h0 = c * chunk, n = BH - h0 < chunk ? BH - h0 : chunk;
    const sa_params pc = chunk_params(p, n);
    // copy in (the slot's previous contents were tiled two chunks ago)
    if (c >= 2 && !cu(cudaStreamWaitEvent(sin, ev[E_IN_FREE + slot], 0))) break;
    for (int t = 0; t < 4; ++t)
      if (!cu(cudaMemcpyAsync(wb + L.lat_in[slot][t], src[t] + static_cast<size_t>(h0) * row16,
                              static_cast<size_t>(n) * row16, cudaMemcpyHostToDevice, sin)))
        break;
    if (rc != SA_OK || !cu(cudaEventRecord(ev[E_IN_DONE + slot], sin))) break;
    // the work, on the caller's stream
    if (!cu(cudaStreamWaitEvent(cs, ev[E_IN_DONE + slot], 0))) break;
    for (int t = 0; t < 4; ++t) {
      if (!sa_ok(sa_tile(wb + L.lat_in[slot][t], wb + L.tiled[t], &pc, 2, stream))) break;
      ++launches;
    }
    if (rc != SA_OK || !cu(cudaEventRecord(ev[E_IN_FREE + slot], cs))) break;
    void* tq = wb + L.tiled[0];
    void* tk = wb + L.tiled[1];
    void* tv = wb + L.tiled[2];
    void* tdo = wb + L.tiled[3];
    int32_t* kvi = reinterpret_cast<int32_t*>(wb + L.kv_index);
    int32_t* kvc = reinterpret_cast<int32_t*>(wb + L.kv_count);
    float* lse = reinterpret_cast<float*>(wb + L.lse);
    float* o32 = reinterpret_cast<float*>(wb + L.out32);
    float* g[3];
    for (int t = 0; t < 3; ++t) g[t] = reinterpret_cast<float*>(wb + L.grad_t[t]);
    if (!sa_ok(sa_plan(tq, tk, nullptr, nullptr, &pc, kvi, kvc, wb + L.ws_op[0], L.ws_bytes[0], stream))) break;
    launches += sa_last_launch_count();
    if (!fold(0)) break;
    if (!sa_ok(sa_forward(tq, tk, tv, nullptr, nullptr, kvi, kvc, &pc, wb + L.out_t, lse, o32, wb + L.ws_op[1],
                          L.ws_bytes[1], stream)))
      break;
    launches += sa_last_launch_count();
    if (!fold(1)) break;
    if (!sa_ok(sa_backward(tq, tk, tv, wb + L.out_t, o32, lse, tdo, kvi, kvc, &pc, g[0], g[1], g[2], wb + L.ws_op[2],
                           L.ws_bytes[2], stream)))
      break;
    launches += sa_last_launch_count();
    if (!fold(2)) break;
    // layout back into the output slot (its previous contents were copied out two chunks ago)
    if (c >= 2 && !cu(cudaStreamWaitEvent(cs, ev[E_OUT_FREE + slot], 0))) break;
    const void* res[4] = {wb + L.out_t, g[0], g[1], g[2]};
    for (int t = 0; t < 4; ++t) {
      if (!sa_ok(sa_untile(res[t], wb + L.lat_out[slot][t], &pc, t == 0 ? 2 : 4, stream))) break;
      ++launches;
    }
    if (rc != SA_OK || !cu(cudaEventRecord(ev[E_WORK_DONE + slot], cs))) break;
    // copy out
    if (!cu(cudaStreamWaitEvent(sout, ev[E_WORK_DONE + slot], 0))) break;
    for (int t = 0; t < 4; ++t)
      if (!cu(cudaMemcpyAsync(dst[t] + static_cast<size_t>(h0) * dst_row[t], wb + L.lat_out[slot][t],
                              static_cast<size_t>(n) * dst_row[t], cudaMemcpyDeviceToHost, sout)))
        break;
    if (rc != SA_OK || !cu(cudaEventRecord(ev[E_OUT_FREE + slot], sout))) break;
  }
  // whatever was issued, the caller's stream is ordered after all of it
  cudaEventRecord(ev[E_END_IN], sin);
  cudaEventRecord(ev[E_END_OUT], sout);
  cudaStreamWaitEvent(cs, ev[E_END_IN], 0);
  cudaStreamWaitEvent(cs, ev[E_END_OUT], 0);
  release();
  sa::set_last_launches(launches);
  return rc;
}

}  // extern "C"
