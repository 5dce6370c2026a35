// Exact group-256 regular-Hadamard rotation by a team of 16 threads.
//
// H = (J4 - 2 I4)^{(x)4} factors into four radix-4 stages, one per base-4 digit
// of the index inside the 256-block: y_i = S - 2 x_i with S the sum of the four
// values that differ only in that digit.  The stages run in float64 on values
// pre-scaled by 1/16 (exact).  Every partial sum of +-x/16 over bf16 inputs
// whose leading-bit exponents span at most 37 binades needs at most 53
// significant bits, so each stage is exact and the float64 result is the exact
// rotated value; one __double2float_rn then gives the correctly rounded float32.
// (Method: "Krea-2 Turbo -- INT4 tensorwise W4A4 (+ConvRot, mixed int8
// fallback)", header paragraph: group-256 regular-Hadamard rotation.)
//
// Thread layout: thread tau of the team holds the 16 contiguous elements
// 16*tau .. 16*tau+15 (digits j0, j1 in registers, j2 j3 = tau), transforms
// digits j0 and j1, swaps through shared memory so that it holds positions
// tau + 16*i (digits j2, j3 in registers) and transforms those.
#pragma once

#include <cstdint>

namespace rbd {

__device__ __forceinline__ void radix4_regular(double& a, double& b, double& c, double& d) {
  const double s = (a + b) + (c + d);
  a = fma(-2.0, a, s);
  b = fma(-2.0, b, s);
  c = fma(-2.0, c, s);
  d = fma(-2.0, d, s);
}

// 16 bf16 (two 16-byte vectors) -> 16 doubles scaled by 1/16.
__device__ __forceinline__ void load16_scaled(const uint4& lo, const uint4& hi, double (&v)[16]) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float f0 = __uint_as_float(w[i] << 16);
    const float f1 = __uint_as_float(w[i] & 0xFFFF0000u);
    v[2 * i] = static_cast<double>(f0) * 0.0625;
    v[2 * i + 1] = static_cast<double>(f1) * 0.0625;
  }
}

__device__ __forceinline__ void load16_f32(const uint4& lo, const uint4& hi, float (&v)[16]) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Swizzled index into a team's 256-double exchange buffer: conflict-free both
// for "thread tau writes 16*tau + e" and "thread tau reads tau + 16*i".
__device__ __forceinline__ int xchg_idx(int p) { return p ^ ((p >> 4) & 15); }

// Rotate one 256-block.  tb: this team's 256-double shared buffer.  On exit
// xr[i] is the rotated value at position tau + 16*i of the block.
__device__ __forceinline__ void rotate256_team(const uint4& lo, const uint4& hi, int tau, double* tb,
                                               float (&xr)[16]) {
  double v[16];
  load16_scaled(lo, hi, v);
  // digit j0 (e & 3), then digit j1 (e >> 2)
#pragma unroll
  for (int j1 = 0; j1 < 4; ++j1) radix4_regular(v[4 * j1], v[4 * j1 + 1], v[4 * j1 + 2], v[4 * j1 + 3]);
#pragma unroll
  for (int j0 = 0; j0 < 4; ++j0) radix4_regular(v[j0], v[j0 + 4], v[j0 + 8], v[j0 + 12]);
#pragma unroll
  for (int e = 0; e < 16; ++e) tb[xchg_idx(16 * tau + e)] = v[e];
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = tb[xchg_idx(tau + 16 * i)];
  __syncwarp();
  // now v[i] is position tau + 16*i: digit j2 = i & 3, j3 = i >> 2
#pragma unroll
  for (int j3 = 0; j3 < 4; ++j3) radix4_regular(v[4 * j3], v[4 * j3 + 1], v[4 * j3 + 2], v[4 * j3 + 3]);
#pragma unroll
  for (int j2 = 0; j2 < 4; ++j2) radix4_regular(v[j2], v[j2 + 4], v[j2 + 8], v[j2 + 12]);
#pragma unroll
  for (int i = 0; i < 16; ++i) xr[i] = __double2float_rn(v[i]);
}

}  // namespace rbd
