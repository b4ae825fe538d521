// Launch functions of the library's kernels (host side, internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "geometry.cuh"
#include "ptx.cuh"

namespace sa {

struct DevStatus;
struct AttnArgs;

cudaError_t launch_tile(const void* src, void* dst, const Geom& g, int BH, int row_bytes, bool to_tiled,
                        cudaStream_t stream);

cudaError_t launch_plan(const void* q, const void* k, const float* q_scale, const float* k_scale, const Geom& g,
                        int BH, int D, bool fp8, double scale, int top_k, float top_p, int cap, int32_t* kv_index,
                        int32_t* kv_count, double* qbar, double* kbar, double* S, DevStatus* st,
                        cudaStream_t stream, int* launches);

cudaError_t launch_query_pair_union(const int32_t* kv_index, const int32_t* kv_count, int32_t* u_list,
                                    int32_t* u_cnt, int BH, int T, int cap, DevStatus* st, cudaStream_t stream);
// Key-cube pair unions of the transposed selection, through a [BH, T, ceil(T/32)] bit matrix.
cudaError_t launch_key_pair_union(const int32_t* kv_index, const int32_t* kv_count, uint32_t* bits, int32_t* u_list,
                                  int32_t* u_cnt, int BH, int T, int cap, DevStatus* st, cudaStream_t stream);

cudaError_t launch_cube_mask(const Geom& g, unsigned long long* mask, cudaStream_t stream);
int num_sms();

cudaError_t launch_forward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                           cudaStream_t stream);

cudaError_t launch_backward(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const void* out, const float* out_f32, const void* dout,
                            AttnArgs a, uint32_t* bits, float* delta, float* nlse2,
                            int32_t* uq_list,
                            int32_t* uq_cnt, int32_t* uk_list, int32_t* uk_cnt, cudaStream_t stream, int* launches);

}  // namespace sa
