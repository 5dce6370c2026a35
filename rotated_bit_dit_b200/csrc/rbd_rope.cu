// Q/K RMSNorm + RoPE: the per-head normalisation and rotary turn that sit
// between the Q|K|V|gate GEMM and attention, plus the rotary angle tables.
//
// Method: "Krea 2 Turbo OrbitQuant W4A4", "Fused transformer" (each block runs
// a Q/K RMSNorm + RoPE kernel after the grouped Q|K|V|gate GEMM); "lab",
// Study 6 (a head's rotary bands: channels 0-43 time, 44-85 height, 86-127
// width).
//
// Per token t and head h (128 channels):
//   r = 1 / sqrt(sum(x^2) / 128 + eps)          (float64, rounded to float32;
//                                                 r = 0 when the radicand is 0)
//   u = x * r * gamma                            (gamma bf16 [128], optional)
//   (y[2i], y[2i+1]) = (u0 c - u1 s, u0 s + u1 c),  c = cos[t][i], s = sin[t][i]
//   y rounded once to bf16.
// Tables: pair i of a head lies in the band holding channels 2i, 2i+1 and,
// j its index inside that band of width w, turns by pos[t][band] *
// base^(-2j / w); the angles are formed in float64 and their cosine and sine
// rounded to float32.
//
// Thread mapping: a half-warp per (token, head) unit; lane i of the half owns
// channels 8i .. 8i+7 (four pairs): one 16-byte load of x, 16 bytes each of
// cos and sin, one 16-byte store; the loads of a warp's units are all issued
// before its first reduction.  In-place use (y == x) is safe: every element
// is read and written by the same thread.
#include <cuda_bf16.h>

#include "rbd_common.cuh"
#include "rbd_internal.cuh"
#include "rbd_rope.cuh"

namespace rbd {

namespace {

constexpr int kRopeDim = 128;
constexpr int kRopePairs = kRopeDim / 2;
constexpr int kRopeWarps = 8;
constexpr int kRopeSteps = 2;   // units per half-warp

__device__ __forceinline__ void bf16x8_to_float(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

}  // namespace

__global__ void __launch_bounds__(kRopeWarps * 32) qk_norm_rope_kernel(const uint16_t* x, int64_t ldx,
                                                                        int T, int H,
                                                                        const uint16_t* __restrict__ gamma,
                                                                        const float* __restrict__ cos_t,
                                                                        const float* __restrict__ sin_t, float eps,
                                                                        uint16_t* y, int64_t ldy) {
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4, li = lane & 15;
  const int total = T * H;
  const int unit0 = (blockIdx.x * kRopeWarps + (threadIdx.x >> 5)) * (2 * kRopeSteps);
  float g[8];
  if (gamma) {
    bf16x8_to_float(__ldg(reinterpret_cast<const uint4*>(gamma) + li), g);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) g[j] = 1.f;
  }
  // every load of the warp's units (x and the token's cos / sin) is issued
  // before the first reduction, so a unit costs one memory latency
  uint4 xv[kRopeSteps];
  float4 cv[kRopeSteps], sv[kRopeSteps];
  int tok[kRopeSteps];
#pragma unroll
  for (int k = 0; k < kRopeSteps; ++k) {
    const int unit = unit0 + 2 * k + half;
    if (unit < total) {
      const int t = unit / H, h = unit - t * H;
      tok[k] = t;
      xv[k] = *reinterpret_cast<const uint4*>(x + (int64_t)t * ldx + (int64_t)h * kRopeDim + 8 * li);
      cv[k] = __ldg(reinterpret_cast<const float4*>(cos_t + (int64_t)t * kRopePairs) + li);
      sv[k] = __ldg(reinterpret_cast<const float4*>(sin_t + (int64_t)t * kRopePairs) + li);
    } else {
      tok[k] = -1;
      xv[k] = make_uint4(0u, 0u, 0u, 0u);
      cv[k] = sv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int k = 0; k < kRopeSteps; ++k) {
    float f[8];
    bf16x8_to_float(xv[k], f);
    // float64 squares: a bf16 head anywhere in its range neither overflows nor underflows
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss = fma((double)f[j], (double)f[j], ss);
    // sum over the 16 lanes of this half-warp (xor offsets below 16 stay inside the half)
#pragma unroll
    for (int m = 8; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const int t = tok[k];
    if (t < 0) continue;
    const double rad = ss / 128.0 + (double)eps;
    const float r = rad > 0.0 ? (float)(1.0 / sqrt(rad)) : 0.f;   // an all-zero head with eps 0 stays 0
    const int unit = unit0 + 2 * k + half;
    const int h = unit - t * H;
    const float c[4] = {cv[k].x, cv[k].y, cv[k].z, cv[k].w}, s[4] = {sv[k].x, sv[k].y, sv[k].z, sv[k].w};
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float u0 = f[2 * e] * r * g[2 * e], u1 = f[2 * e + 1] * r * g[2 * e + 1];
      const float y0 = fmaf(u0, c[e], -u1 * s[e]);
      const float y1 = fmaf(u0, s[e], u1 * c[e]);
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
      out[e] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(y + (int64_t)t * ldy + (int64_t)h * kRopeDim + 8 * li) =
        make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// One thread per (token, pair).
__global__ void rope_tables_kernel(const int32_t* __restrict__ pos, int T, double base, float* __restrict__ cos_t,
                                   float* __restrict__ sin_t) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)T * kRopePairs) return;
  const int t = static_cast<int>(idx / kRopePairs), i = static_cast<int>(idx % kRopePairs);
  // bands of 44, 42, 42 channels = 22, 21, 21 pairs
  const int band = i < 22 ? 0 : (i < 43 ? 1 : 2);
  const int j = i - (band == 0 ? 0 : (band == 1 ? 22 : 43));
  const double w = band == 0 ? 44.0 : 42.0;
  const double ang = static_cast<double>(pos[(int64_t)t * 3 + band]) * pow(base, -2.0 * j / w);
  double sv, cv;
  sincos(ang, &sv, &cv);
  cos_t[idx] = static_cast<float>(cv);
  sin_t[idx] = static_cast<float>(sv);
}

cudaError_t launch_qk_norm_rope(const uint16_t* x, int64_t ldx, int T, int H, const uint16_t* gamma,
                                const float* cos_t, const float* sin_t, float eps, uint16_t* y, int64_t ldy,
                                cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int64_t per_block = (int64_t)kRopeWarps * 2 * kRopeSteps;
  const dim3 grid(static_cast<unsigned>(((int64_t)T * H + per_block - 1) / per_block));
  qk_norm_rope_kernel<<<grid, kRopeWarps * 32, 0, st>>>(x, ldx, T, H, gamma, cos_t, sin_t, eps, y, ldy);
  return cudaGetLastError();
}

cudaError_t launch_rope_tables(const int32_t* pos, int T, double base, float* cos_t, float* sin_t,
                               cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int64_t n = (int64_t)T * kRopePairs;
  const dim3 grid(static_cast<unsigned>((n + 255) / 256));
  rope_tables_kernel<<<grid, 256, 0, st>>>(pos, T, base, cos_t, sin_t);
  return cudaGetLastError();
}

}  // namespace rbd
