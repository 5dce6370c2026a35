// INT4 KV-cache codec: encode (slice write) and decode (slice read) of a
// key or value cache with one float32 scale per token, head and group, the
// groups lying inside the rotary bands of the head.
//
// Method: "Krea Realtime 14B on one RTX 4090" essay, Study 6: the cache stores
// int4 packed two values per byte with one scale per token, per head, per
// rotary band; rotary splits the 128 channels of a head into bands of 44, 42
// and 42; finer groups are cut inside the bands, never across them; reading
// unpacks and scales in one pass per token and head.
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
#include "rbd_common.cuh"
#include "rbd_internal.cuh"

namespace rbd {

namespace {

constexpr int kKvDim = 128;
constexpr int kKvWarps = 8;
constexpr int kKvUnits = 4;   // (token, head) units per warp

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

// A group has at least 10 channels, so the 4 channels of a lane belong to at
// most two groups (ga, and gb = ga or ga + 1).  Each warp handles kKvUnits
// consecutive (token, head) units and issues all their loads first.
template <int N>
__global__ void __launch_bounds__(kKvWarps * 32) kv4_encode_kernel(const uint16_t* __restrict__ x, int T, int H,
                                                                   int64_t ldt, uint8_t* __restrict__ codes,
                                                                   float* __restrict__ scales, int64_t capacity,
                                                                   int64_t slot0) {
  constexpr int G = 3 * N;
  const int lane = threadIdx.x & 31;
  const int total = T * H;
  const int unit0 = (blockIdx.x * kKvWarps + (threadIdx.x >> 5)) * kKvUnits;
  const int ga = kv4_group_of<N>(4 * lane), gb = kv4_group_of<N>(4 * lane + 3);
  bool in_b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) in_b[j] = kv4_group_of<N>(4 * lane + j) != ga;
  // the first unit's token and head; later units step through the heads
  int t = unit0 / H, h = unit0 - t * H;
  uint2 raw[kKvUnits];
  int64_t dst[kKvUnits];   // (slot * H + h) of each unit
  {
    int tt = t, hh = h;
#pragma unroll
    for (int u = 0; u < kKvUnits; ++u) {
      if (unit0 + u < total) {
        raw[u] = *reinterpret_cast<const uint2*>(x + (int64_t)tt * ldt + (int64_t)hh * kKvDim + 4 * lane);
        int64_t slot = slot0 + tt;               // < 2 capacity: one wrap at most
        if (slot >= capacity) slot -= capacity;
        dst[u] = slot * H + hh;
      }
      if (++hh == H) { hh = 0; ++tt; }
    }
  }
#pragma unroll
  for (int u = 0; u < kKvUnits; ++u) {
    if (unit0 + u >= total) break;   // uniform across the warp
    const float v[4] = {__uint_as_float(raw[u].x << 16), __uint_as_float(raw[u].x & 0xFFFF0000u),
                        __uint_as_float(raw[u].y << 16), __uint_as_float(raw[u].y & 0xFFFF0000u)};
    // the lane's maxima in its (at most) two groups; float bit patterns of
    // non-negative values order like unsigned integers
    uint32_t ma = 0u, mb = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t a = __float_as_uint(fabsf(v[j]));
      if (in_b[j]) mb = max(mb, a); else ma = max(ma, a);
    }
    uint32_t amax_a = 0u, amax_b = 0u, amax_mine = 0u;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint32_t r = __reduce_max_sync(0xffffffffu, g == ga ? ma : (g == gb ? mb : 0u));
      if (g == ga) amax_a = r;
      if (g == gb) amax_b = r;
      if (g == lane) amax_mine = r;
    }
    const float fa = __uint_as_float(amax_a), fb = __uint_as_float(amax_b);
    const float inv_a = fa > 0.f ? __fdiv_rn(7.f, fa) : 0.f;
    const float inv_b = gb == ga ? inv_a : (fb > 0.f ? __fdiv_rn(7.f, fb) : 0.f);
    uint32_t packed = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int q = __float2int_rn(__fmul_rn(v[j], in_b[j] ? inv_b : inv_a));
      q = q > 7 ? 7 : (q < -8 ? -8 : q);
      packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * j);
    }
    *reinterpret_cast<uint16_t*>(codes + dst[u] * (kKvDim / 2) + 2 * lane) = static_cast<uint16_t>(packed);
    if (lane < G) scales[dst[u] * G + lane] = __fdiv_rn(__uint_as_float(amax_mine), 7.f);
  }
}

template <int N>
__global__ void __launch_bounds__(kKvWarps * 32) kv4_decode_kernel(const uint8_t* __restrict__ codes,
                                                                   const float* __restrict__ scales,
                                                                   int64_t capacity, int64_t slot0, int T, int H,
                                                                   uint16_t* __restrict__ y, int64_t ldt) {
  constexpr int G = 3 * N;
  const int lane = threadIdx.x & 31;
  const int total = T * H;
  const int unit0 = (blockIdx.x * kKvWarps + (threadIdx.x >> 5)) * kKvUnits;
  const int ga = kv4_group_of<N>(4 * lane), gb = kv4_group_of<N>(4 * lane + 3);
  bool in_b[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) in_b[j] = kv4_group_of<N>(4 * lane + j) != ga;
  uint32_t pk[kKvUnits];
  float sc[kKvUnits];
  int64_t dst[kKvUnits];   // output element offset of each unit
  {
    int tt = unit0 / H, hh = unit0 - tt * H;
#pragma unroll
    for (int u = 0; u < kKvUnits; ++u) {
      if (unit0 + u < total) {
        int64_t slot = slot0 + tt;               // < 2 capacity: one wrap at most
        if (slot >= capacity) slot -= capacity;
        const int64_t src = slot * H + hh;
        pk[u] = *reinterpret_cast<const uint16_t*>(codes + src * (kKvDim / 2) + 2 * lane);
        sc[u] = lane < G ? __ldg(scales + src * G + lane) : 0.f;
        dst[u] = (int64_t)tt * ldt + (int64_t)hh * kKvDim;
      }
      if (++hh == H) { hh = 0; ++tt; }
    }
  }
#pragma unroll
  for (int u = 0; u < kKvUnits; ++u) {
    if (unit0 + u >= total) break;   // uniform across the warp
    const float sa = __shfl_sync(0xffffffffu, sc[u], ga), sb = __shfl_sync(0xffffffffu, sc[u], gb);
    uint32_t out[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      uint32_t half[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = 2 * k + e;
        const int q = static_cast<int>(static_cast<int32_t>(pk[u] << (28 - 4 * j)) >> 28);   // sign-extend nibble j
        half[e] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(static_cast<float>(q), in_b[j] ? sb : sa)));
      }
      out[k] = half[0] | (half[1] << 16);
    }
    *reinterpret_cast<uint2*>(y + dst[u] + 4 * lane) = make_uint2(out[0], out[1]);
  }
}

cudaError_t launch_kv4_encode(const uint16_t* x, int T, int H, int64_t ldt, int n, uint8_t* codes, float* scales,
                              int64_t capacity, int64_t slot0, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int64_t per_block = (int64_t)kKvWarps * kKvUnits;
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
  const int64_t per_block = (int64_t)kKvWarps * kKvUnits;
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
