// sa_plan_static: the router with its scratch in a fixed device array instead of a
// caller-supplied workspace, for callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not allowed or not wanted — inside a
// CUDA stream capture that a framework records into a graph, in serving processes whose
// device memory is one pre-reserved arena with no headroom for a 50 MB workspace, or from
// C callers that hold no allocator at all.  They pass inputs and outputs; the library
// brings its own scratch.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes (64 MiB).  Every
// GPU that loads this library holds it until the process exits.  In host code the
// array's name is only a host-side stand-in, so its device address is looked up once per
// device with cudaGetSymbolAddress (on the first call made while that device is
// current) and cached; that first call on a device should come before any stream
// capture.  All calls share the array: calls that overlap on the GPU (two streams, or
// two host threads) race on it and must be serialised by the caller.
#include <cmath>
#include <mutex>

#include "../../include/sa.h"
#include "kernels.h"
#include "ptx.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_plan_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Device address of the scratch array on the current device (looked up once per device).
void* scratch_address(sa_status* err) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = SA_ERR_LAUNCH;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_plan_scratch) != cudaSuccess || !ptr) {
      *err = SA_ERR_LAUNCH;
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" sa_status sa_plan_static(const void* q, const void* k, const float* q_scale, const float* k_scale,
                                    const sa_params* p, int32_t* kv_index, int32_t* kv_count, sa_stream_t stream) {
  // sa_workspace_size validates the parameters (0 when they are not accepted)
  const size_t need = sa_workspace_size(p, SA_OP_PLAN);
  if (need == 0) return SA_ERR_INVALID_ARG;
  if (!q || !k || !kv_index || !kv_count) return SA_ERR_INVALID_ARG;
  const bool fp8 = p->qk_dtype == SA_FP8_E4M3;
  if (fp8 && (!q_scale || !k_scale)) return SA_ERR_INVALID_ARG;
  const int T = sa_num_cubes(p);
  if (p->kv_capacity != T) return SA_ERR_INVALID_ARG;  // no clipping, hence no device-side status to report
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k)) & 15u) return SA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(kv_index) | reinterpret_cast<uintptr_t>(kv_count)) & 3u) return SA_ERR_ALIGNMENT;
  if (need > kStaticScratchBytes) return SA_ERR_WORKSPACE;  // more scratch than the fixed array holds

  sa_status err = SA_OK;
  unsigned char* base = static_cast<unsigned char*>(scratch_address(&err));
  if (!base) return err;

  // same carving as the plan workspace: status block, pooled Q, pooled K, block scores
  const size_t BH = static_cast<size_t>(p->B) * p->H;
  const size_t off_q = 256;
  const size_t off_k = round256(off_q + BH * T * p->D * sizeof(double));
  const size_t off_s = round256(off_k + BH * T * p->D * sizeof(double));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the status block must start at zero; everything else is written before it is read
  if (cudaMemsetAsync(base, 0, 256, st) != cudaSuccess) return SA_ERR_LAUNCH;

  sa::Geom g;
  g.lat_t = p->lat_t;
  g.lat_h = p->lat_h;
  g.lat_w = p->lat_w;
  g.Nt = (p->lat_t + 3) / 4;
  g.Nh = (p->lat_h + 3) / 4;
  g.Nw = (p->lat_w + 3) / 4;
  g.T = T;
  g.Npad = 64 * T;
  const double scale = p->softmax_scale > 0.0f ? static_cast<double>(p->softmax_scale)
                                               : 1.0 / std::sqrt(static_cast<double>(p->D));
  int launches = 0;
  if (sa::launch_plan(q, k, q_scale, k_scale, g, p->B * p->H, p->D, fp8, scale, p->top_k, p->top_p, p->kv_capacity,
                      kv_index, kv_count, reinterpret_cast<double*>(base + off_q),
                      reinterpret_cast<double*>(base + off_k), reinterpret_cast<double*>(base + off_s),
                      reinterpret_cast<sa::DevStatus*>(base), st, &launches) != cudaSuccess)
    return SA_ERR_LAUNCH;
  return SA_OK;
}
