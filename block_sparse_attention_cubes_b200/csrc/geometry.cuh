// Cube geometry shared by the kernels: which of the 64 slots of a cube hold real tokens.
//
// Cube-major layout (VSA page, "Cube Partitioning and Token Re-Indexing"; VSA2 page,
// section 2.2): cube c = (c_t, c_h, c_w) with c = c_t*N_h*N_w + c_h*N_w + c_w holds the
// tokens (4c_t + a, 4c_h + b, 4c_w + d), a, b, d in [0,4), at slot a*16 + b*4 + d.
// A slot is padding when its token lies outside the valid latent grid (VSA2 page,
// "Kernel Implementation": pad to multiples of the cube and mask the padding out).
#pragma once
#include <cstdint>

namespace sa {

struct Geom {
  int lat_t, lat_h, lat_w;  // valid latent grid
  int Nt, Nh, Nw;           // cubes per axis
  int T;                    // number of cubes
  int Npad;                 // 64 * T
};

__host__ __device__ inline int imin(int a, int b) { return a < b ? a : b; }

// extents of the valid part of cube c along t, h, w (each in [1,4])
__host__ __device__ inline void cube_extent(const Geom& g, int c, int& vt, int& vh, int& vw) {
  const int ct = c / (g.Nh * g.Nw);
  const int ch = (c / g.Nw) % g.Nh;
  const int cw = c % g.Nw;
  vt = imin(4, g.lat_t - 4 * ct);
  vh = imin(4, g.lat_h - 4 * ch);
  vw = imin(4, g.lat_w - 4 * cw);
}

__host__ __device__ inline bool slot_valid(int vt, int vh, int vw, int s) {
  return (s >> 4) < vt && ((s >> 2) & 3) < vh && (s & 3) < vw;
}

__host__ __device__ inline bool token_valid(const Geom& g, int c, int s) {
  int vt, vh, vw;
  cube_extent(g, c, vt, vh, vw);
  return slot_valid(vt, vh, vw, s);
}

__host__ __device__ inline int cube_valid_count(const Geom& g, int c) {
  int vt, vh, vw;
  cube_extent(g, c, vt, vh, vw);
  return vt * vh * vw;
}

}  // namespace sa
