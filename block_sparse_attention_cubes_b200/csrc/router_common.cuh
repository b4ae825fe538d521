// Pieces shared by the routers that score pooled rows on the tensor cores (the cube router in
// router.cu, the fine-grained group router in fine_router.cu): e4m3 decoding, the exact split
// of a pooled row into four int8 limbs, and the ten limb-pair products.
//
// A pooled row x (D values, fp64) with binary exponent E (every |x_d| < 2^E) becomes the
// integers X_d = rint(x_d 2^(30 - E)), |X_d| <= 2^30, split into four signed 8-bit limbs
// X = d0 256^3 + d1 256^2 + d2 256 + d3 (d0 in [-64, 64], the others in [-128, 127]).  The
// products of limb pairs (a, b) with a + b = w accumulate (exact s32) into level w, w = 0..3,
// and v = L0 2^24 + L1 2^16 + L2 2^8 + L3 is the dot product of two rows in units of
// 2^(Eq + Ek - 36); dropping the levels w >= 4 and the rounding to 30 bits bound its error by
// 4.03 * 2^-23 * 2^(Eq + Ek).
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace sa {

constexpr int kLimbRow = 128;    // bytes per limb row: K = 128 int8 (D = 64 rows are zero-padded)
constexpr int kExpZero = -1100;  // exponent recorded for an all-zero row
constexpr int kExpBias = 2048;   // exponents are kept as E + 2048 > 0 for the per-head atomicMax

__device__ __forceinline__ float e4m3_value(uint32_t b) {
  // 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is subnormal.
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = (e == 0u) ? static_cast<float>(m) * (1.0f / 512.0f)
                      : __uint_as_float(((e + 120u) << 23) | (m << 20));
  if (e == 15u && m == 7u) v = __uint_as_float(0x7fc00000u);
  return (b & 0x80u) ? -v : v;
}

// The limbs of x * up (up = 2^(30 - E)), each byte placed at bit 8 * slot of limb[0..3].
__device__ __forceinline__ void limb_digits(double x, double up, int slot, uint32_t (&limb)[4]) {
  int X = static_cast<int>(rint(x * up));  // |X| <= 2^30
  const int d3 = ((X + 128) & 255) - 128;
  X = (X - d3) >> 8;
  const int d2 = ((X + 128) & 255) - 128;
  X = (X - d2) >> 8;
  const int d1 = ((X + 128) & 255) - 128;
  const int d0 = (X - d1) >> 8;  // in [-64, 64]
  const int sh = 8 * slot;
  limb[0] |= (static_cast<uint32_t>(d0) & 255u) << sh;
  limb[1] |= (static_cast<uint32_t>(d1) & 255u) << sh;
  limb[2] |= (static_cast<uint32_t>(d2) & 255u) << sh;
  limb[3] |= (static_cast<uint32_t>(d3) & 255u) << sh;
}

// The ten limb-pair products of one 128 x 128 tile into four s32 accumulators of 128 columns
// at tmem + 128 w.  qb / kb: shared-memory addresses of the 4 limb tiles of the rows and of the
// columns ([128 rows][128 B] each, 16 KB apart, 128-byte swizzle).  KS = D / 32 k-steps of 32
// int8.  Called by the one lane that issues.
template <int KS>
__device__ __forceinline__ void issue_limb_products(uint32_t tmem, uint32_t qb, uint32_t kb) {
  const uint32_t idesc = make_idesc_s8(128, 128);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
#pragma unroll
    for (int la = 0; la <= w; ++la) {
      const int lb = w - la;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
        umma_i8_ss(tmem + 128 * w, sw128_desc(qb + la * 16384 + kk * 32, 16, 1024),
                   sw128_desc(kb + lb * 16384 + kk * 32, 16, 1024), idesc, (la > 0 || kk > 0) ? 1u : 0u);
    }
  }
}

// v = L0 2^24 + L1 2^16 + L2 2^8 + L3 from the four level accumulators of one column.
__device__ __forceinline__ long long limb_levels(uint32_t l0, uint32_t l1, uint32_t l2, uint32_t l3) {
  const int hiw = static_cast<int>(l0) * 256 + static_cast<int>(l1);  // |.| < 2^28
  const int low = static_cast<int>(l2) * 256 + static_cast<int>(l3);  // |.| < 2^31
  return static_cast<long long>(hiw) * 65536 + low;
}

}  // namespace sa
