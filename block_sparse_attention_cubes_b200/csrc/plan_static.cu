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
// array's name is only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress while the caller's device is current: on every call made outside a
// stream capture (so a context torn down and created again is followed), and taken from
// the per-device cache inside a capture.  The first call on a device must therefore come
// before any stream capture.  All calls share the array: calls that overlap on the GPU
// (two streams, or two host threads) race on it and must be serialised by the caller.
#include <mutex>

#include "../../include/sa.h"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_plan_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.
void* scratch_address(cudaStream_t stream, sa_status* err) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = SA_ERR_LAUNCH;
    return nullptr;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
    *err = SA_ERR_LAUNCH;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (cap == cudaStreamCaptureStatusNone) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_plan_scratch) != cudaSuccess || !ptr) {
      *err = SA_ERR_LAUNCH;
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  } else if (!g_scratch_ptr[dev]) {
    *err = SA_ERR_LAUNCH;  // first call on this device made under a capture
    return nullptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" sa_status sa_plan_static(const void* q, const void* k, const float* q_scale, const float* k_scale,
                                    const sa_params* p, int32_t* kv_index, int32_t* kv_count, sa_stream_t stream) {
  // every host-side check of sa_plan, before the device is touched
  size_t need = 0;
  const sa_status s = sa::plan_check(q, k, q_scale, k_scale, p, kv_index, kv_count, &need);
  if (s != SA_OK) return s;
  if (p->kv_capacity != sa_num_cubes(p)) return SA_ERR_INVALID_ARG;  // no clipping, hence no device status to read
  if (need > kStaticScratchBytes) return SA_ERR_WORKSPACE;            // more scratch than the fixed array holds
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  sa_status err = SA_OK;
  void* base = scratch_address(st, &err);
  if (!base) return err;
  // the same checks, carving (status block first, cleared) and launches as sa_plan
  return sa::plan_on_scratch(q, k, q_scale, k_scale, p, kv_index, kv_count, base, kStaticScratchBytes, st);
}
