// INT4 KV-cache codec: encode (slice write) and decode (slice read) of a
// key or value cache with one float32 scale per token, head and group, the
// groups lying inside the rotary bands of the head.
//
// Method: "lab", Study 6 ("The cache becomes the model"): four-bit codes, two
// to a byte, with a scale for each (token, head, rotary band); the bands of a
// head are channels 0-43, 44-85 and 86-127; finer scale groups stay inside one
// band; a read unpacks and rescales in a single pass per token and head.
//
// Arithmetic per group (the same IEEE float32 steps as the activation
// quantiser): amax, s = amax / 7, inv = 7 / amax, q = clamp(rint(x * inv), -8, 7);
// an all-zero group gets s = 0.  A band of b channels split into n groups is
// cut into contiguous runs whose sizes differ by at most one, longer runs
// first.  Decode: RN_bf16(q * s).
//
// Layout: the cache is a ring of `capacity` token slots; input token t goes to
// slot (slot0 + t) mod capacity.  codes [capacity][H][64] bytes (channel 2i in
// the low nibble of byte i), scales [capacity][H][3 n] float32.
// Thread mapping: a warp handles a few (token, head) units; lane l owns
// channels 4l .. 4l+3 of each (one 8-byte access).
#include <cuda_bf16.h>

#include "rbd_common.cuh"
#include "rbd_internal.cuh"

namespace rbd {

namespace {

constexpr int kKvDim = 128;
constexpr int kKvWarps = 8;

// Group of channel c when every band is cut into N groups.
template <int N>
__device__ __forceinline__ int kv4_group_of(int c) {
  const int band = c < 44 ? 0 : (c < 86 ? 1 : 2);
  const int start = band == 0 ? 0 : (band == 1 ? 44 : 86);
  const int size = band == 0 ? 44 : 42;
  const int base = size / N, extra = size % N;
  const int o = c - start;
  const int long_span = extra * (base + 1);
  const int g = o < long_span ? o / (base + 1) : extra + (o - long_span) / base;
  return band * N + g;
}

}  // namespace

// Units per warp, and rounds of 32 (unit, group) pairs: pair p = u * G + g
// lives on lane p % 32 in round p / 32, which does that pair's divisions.
__host__ __device__ constexpr int kv4_units(int n) { return n == 1 ? 8 : (n == 2 ? 5 : 4); }
__host__ __device__ constexpr int kv4_rounds(int n) { return (kv4_units(n) * 3 * n + 31) / 32; }

// Value of pair p (held on lane p % 32 in round p / 32), for every lane.
template <int R>
__device__ __forceinline__ float kv4_pair_value(const float (&v)[R], int p) {
  float r = __shfl_sync(0xffffffffu, v[0], p & 31);
#pragma unroll
  for (int k = 1; k < R; ++k) {
    const float o = __shfl_sync(0xffffffffu, v[k], p & 31);
    if ((p >> 5) == k) r = o;
  }
  return r;
}

// A group has at least 10 channels, so the 4 channels of a lane belong to at
// most two groups (ga, and gb = ga or ga + 1).  A warp handles U consecutive
// (token, head) units and issues all their loads first; then the group maxima
// of every unit (one redux.sync per group), one inverse and one scale per
// (unit, group) on its own lane, and the codes with the inverses shuffled in.
template <int N>
__global__ void __launch_bounds__(kKvWarps * 32) kv4_encode_kernel(const uint16_t* __restrict__ x, int T, int H,
                                                                   int64_t ldt, uint8_t* __restrict__ codes,
                                                                   float* __restrict__ scales, int64_t capacity,
                                                                   int64_t slot0) {
  constexpr int G = 3 * N;
  constexpr int U = kv4_units(N);
  const int lane = threadIdx.x & 31;
  const int total = T * H;
  const int unit0 = (blockIdx.x * kKvWarps + (threadIdx.x >> 5)) * U;
  const int ga = kv4_group_of<N>(4 * lane), gb = kv4_group_of<N>(4 * lane + 3);
  bool in_b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) in_b[j] = kv4_group_of<N>(4 * lane + j) != ga;
  uint2 raw[U];
  int64_t dst[U];   // (slot * H + h) of each unit
  {
    int tt = unit0 / H, hh = unit0 - tt * H;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (unit0 + u < total) {
        raw[u] = *reinterpret_cast<const uint2*>(x + (int64_t)tt * ldt + (int64_t)hh * kKvDim + 4 * lane);
        int64_t slot = slot0 + tt;               // < 2 capacity: one wrap at most
        if (slot >= capacity) slot -= capacity;
        dst[u] = slot * H + hh;
      } else {
        raw[u] = make_uint2(0u, 0u);
      }
      if (++hh == H) { hh = 0; ++tt; }
    }
  }
  // group maxima; pair u * G + g keeps that of (unit u, group g).  Float bit
  // patterns of non-negative values order like unsigned integers.
  constexpr int R = kv4_rounds(N);
  uint32_t amax_lane[R];
#pragma unroll
  for (int k = 0; k < R; ++k) amax_lane[k] = 0u;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    uint32_t ma = 0u, mb = 0u;
    const uint32_t w[4] = {raw[u].x << 16, raw[u].x & 0xFFFF0000u, raw[u].y << 16, raw[u].y & 0xFFFF0000u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t a = w[j] & 0x7FFFFFFFu;     // |x|
      if (in_b[j]) mb = max(mb, a); else ma = max(ma, a);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint32_t r = __reduce_max_sync(0xffffffffu, g == ga ? ma : (g == gb ? mb : 0u));
      if (lane == (u * G + g) % 32) amax_lane[(u * G + g) / 32] = r;
    }
  }
  float inv_lane[R], s_lane[R];
#pragma unroll
  for (int k = 0; k < R; ++k) {
    const float fa = __uint_as_float(amax_lane[k]);
    inv_lane[k] = fa > 0.f ? __fdiv_rn(7.f, fa) : 0.f;
    s_lane[k] = __fdiv_rn(fa, 7.f);
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (unit0 + u >= total) break;   // uniform across the warp
    const float inv_a = kv4_pair_value<R>(inv_lane, u * G + ga);
    const float inv_b = kv4_pair_value<R>(inv_lane, u * G + gb);
    const float v[4] = {__uint_as_float(raw[u].x << 16), __uint_as_float(raw[u].x & 0xFFFF0000u),
                        __uint_as_float(raw[u].y << 16), __uint_as_float(raw[u].y & 0xFFFF0000u)};
    // rint to even by adding 1.5 * 2^23 (exact for |x * inv| < 2^22; here
    // |x * inv| <= 7): the low bits of the sum are the two's-complement code
    uint32_t packed = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float p = __fmul_rn(v[j], in_b[j] ? inv_b : inv_a);
      int q = static_cast<int>(__float_as_uint(__fadd_rn(p, 12582912.0f)) - 0x4B400000u);
      q = q > 7 ? 7 : (q < -8 ? -8 : q);
      packed += (static_cast<uint32_t>(q) & 0xFu) << (4 * j);
    }
    *reinterpret_cast<uint16_t*>(codes + dst[u] * (kKvDim / 2) + 2 * lane) = static_cast<uint16_t>(packed);
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int p = lane + 32 * k;   // this lane's pair in round k
      if (p >= u * G && p < u * G + G) scales[dst[u] * G + (p - u * G)] = s_lane[k];
    }
  }
}

// Decode: a half-warp per (token, head) unit, lane i of the half owning
// channels 8i .. 8i+7 (4 bytes of codes in, one 16-byte store out); the 8
// channels touch at most two groups, whose scales lanes i < G of the half
// load and shuffle.  A warp handles 2 * kKvDecSteps units.
constexpr int kKvDecSteps = 4;

template <int N>
__global__ void __launch_bounds__(kKvWarps * 32) kv4_decode_kernel(const uint8_t* __restrict__ codes,
                                                                   const float* __restrict__ scales,
                                                                   int64_t capacity, int64_t slot0, int T, int H,
                                                                   uint16_t* __restrict__ y, int64_t ldt) {
  constexpr int G = 3 * N;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4, li = lane & 15;
  const int total = T * H;
  const int unit0 = (blockIdx.x * kKvWarps + (threadIdx.x >> 5)) * (2 * kKvDecSteps);
  const int ga = kv4_group_of<N>(8 * li), gb = kv4_group_of<N>(8 * li + 7);
  bool in_b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) in_b[j] = kv4_group_of<N>(8 * li + j) != ga;
  uint32_t pk[kKvDecSteps];
  float sc[kKvDecSteps];
  int64_t dst[kKvDecSteps];
#pragma unroll
  for (int k = 0; k < kKvDecSteps; ++k) {
    const int unit = unit0 + 2 * k + half;
    if (unit < total) {
      const int t = unit / H, h = unit - t * H;
      int64_t slot = slot0 + t;                  // < 2 capacity: one wrap at most
      if (slot >= capacity) slot -= capacity;
      const int64_t src = slot * H + h;
      pk[k] = *reinterpret_cast<const uint32_t*>(codes + src * (kKvDim / 2) + 4 * li);
      sc[k] = li < G ? __ldg(scales + src * G + li) : 0.f;
      dst[k] = (int64_t)t * ldt + (int64_t)h * kKvDim;
    } else {
      pk[k] = 0u;
      sc[k] = 0.f;
      dst[k] = -1;
    }
  }
#pragma unroll
  for (int k = 0; k < kKvDecSteps; ++k) {
    const float sa = __shfl_sync(0xffffffffu, sc[k], ga, 16), sb = __shfl_sync(0xffffffffu, sc[k], gb, 16);
    if (dst[k] < 0) continue;
    // q as a float without a conversion: the bits of 1.5 * 2^23 + q, minus 1.5 * 2^23 (exact)
    float f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int q = static_cast<int>(static_cast<int32_t>(pk[k] << (28 - 4 * j)) >> 28);   // sign-extend nibble j
      f[j] = __fmul_rn(__fsub_rn(__uint_as_float(0x4B400000u + static_cast<uint32_t>(q)), 12582912.0f),
                       in_b[j] ? sb : sa);
    }
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
      out[e] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(y + dst[k] + 8 * li) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

cudaError_t launch_kv4_encode(const uint16_t* x, int T, int H, int64_t ldt, int n, uint8_t* codes, float* scales,
                              int64_t capacity, int64_t slot0, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int64_t per_block = (int64_t)kKvWarps * kv4_units(n);
  const dim3 grid(static_cast<unsigned>(((int64_t)T * H + per_block - 1) / per_block));
  switch (n) {
    case 1: kv4_encode_kernel<1><<<grid, kKvWarps * 32, 0, st>>>(x, T, H, ldt, codes, scales, capacity, slot0); break;
    case 2: kv4_encode_kernel<2><<<grid, kKvWarps * 32, 0, st>>>(x, T, H, ldt, codes, scales, capacity, slot0); break;
    case 4: kv4_encode_kernel<4><<<grid, kKvWarps * 32, 0, st>>>(x, T, H, ldt, codes, scales, capacity, slot0); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_kv4_decode(const uint8_t* codes, const float* scales, int64_t capacity, int64_t slot0, int T,
                              int H, int n, uint16_t* y, int64_t ldt, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int64_t per_block = (int64_t)kKvWarps * 2 * kKvDecSteps;
  const dim3 grid(static_cast<unsigned>(((int64_t)T * H + per_block - 1) / per_block));
  switch (n) {
    case 1: kv4_decode_kernel<1><<<grid, kKvWarps * 32, 0, st>>>(codes, scales, capacity, slot0, T, H, y, ldt); break;
    case 2: kv4_decode_kernel<2><<<grid, kKvWarps * 32, 0, st>>>(codes, scales, capacity, slot0, T, H, y, ldt); break;
    case 4: kv4_decode_kernel<4><<<grid, kKvWarps * 32, 0, st>>>(codes, scales, capacity, slot0, T, H, y, ldt); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace rbd
