// Activation / weight prologue kernels: group-wise regular-Hadamard rotation,
// dynamic symmetric quantisation, INT4 packing, and the low-rank down product.
//
// Method: "Krea-2 Turbo -- INT4 tensorwise W4A4 (+ConvRot, mixed int8
// fallback)", header paragraph (group-256 regular-Hadamard rotation of the
// activations online, dynamic quantisation inside the kernel, packed signed
// INT4 weights); group-64 scales per "Krea 2 Turbo Nunchaku Lite INT4 r32".
//
// Rotation arithmetic: see rbd_rotate.cuh (exact float64 radix-4 stages).
//
// Thread layout.  16 threads ("a team") own one 256-block: thread tau holds
// the 16 contiguous elements 16*tau .. 16*tau+15 (digits j0, j1 in registers,
// j2 j3 = tau), transforms digits j0 and j1, swaps through shared memory so
// that it holds positions tau + 16*i (digits j2, j3 in registers), transforms
// those, and quantises.  Codes go back through shared memory so each thread
// stores 16 contiguous bytes.
#include <cuda_fp8.h>

#include "rbd_common.cuh"
#include "rbd_internal.cuh"
#include "rbd_rotate.cuh"

namespace rbd {

namespace {

constexpr int kTeam = 16;  // threads per 256-block

__device__ __forceinline__ int quant1(float v, float inv, float qmax) {
  const float t = __fmul_rn(v, inv);
  int q = __float2int_rn(t);
  const int hi = static_cast<int>(qmax);
  q = q > hi ? hi : q;
  q = q < -hi - 1 ? -hi - 1 : q;
  return q;
}

// The byte that holds one activation code: the two's-complement int8, or (E4)
// the E4M3 byte of the same value, exact for every INT4 code.
template <bool E4>
__device__ __forceinline__ uint32_t code_byte(int q) {
  if constexpr (E4) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(static_cast<float>(q), __NV_SATFINITE, __NV_E4M3));
  } else {
    return static_cast<uint32_t>(q) & 0xFFu;
  }
}

}  // namespace

// RMSNorm + modulation ahead of the rotation (NORM variant).  gamma, shift and
// scale are bf16 [K] vectors or null.
struct NormArgs {
  const uint16_t* gamma;
  const uint16_t* shift;
  const uint16_t* scale;
  float eps;
};

// One CTA handles `rows` rows; each row is handled by T = 16 * teams threads;
// team `tm` of a row processes 256-blocks g = tm, tm + teams, ... (at most CMAX).
// OUT_PACKED: write packed INT4 bytes instead of one code per byte.
// E4: each code byte is the E4M3 byte of the code's value (4-bit codes only).
// NORM: the row (all of it is in registers) is first normalised and modulated
// -- "Krea 2 Turbo OrbitQuant W4A4", section "Fused transformer": the norm and
// the modulation are folded into the kernels that quantise activations.  The sum of the
// exact squares is accumulated in float64 and reduced across the row's
// threads; r = 1 / sqrt(sum / K + eps) (float64 IEEE operations) is rounded
// once to float32; then per element, as single float32 operations,
// u = x * r, u *= gamma, u *= (1 + scale), u += shift, rounded once to bf16.
// A row whose mean square plus eps is zero gets r = 0.
template <bool ROT, bool G64, bool OUT_PACKED, int CMAX, bool NORM = false, bool E4 = false>
__global__ void __launch_bounds__(256) rot_quant_kernel(const uint16_t* __restrict__ x, int64_t M, int K,
                                                        int64_t ldx, float qmax, int teams, int rows,
                                                        int8_t* __restrict__ codes, float* __restrict__ scales,
                                                        NormArgs norm) {
  // a linear launched after this kernel may start streaming its weights now
  pdl_launch_dependents();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* xbuf = reinterpret_cast<double*>(smem_raw);        // [teams*rows][256]
  float* red = reinterpret_cast<float*>(smem_raw + (size_t)blockDim.x / kTeam * 256 * sizeof(double));
  double* red64 = reinterpret_cast<double*>(smem_raw + (size_t)blockDim.x / kTeam * 256 * sizeof(double) +
                                            64 * sizeof(float));

  const int T = kTeam * teams;
  const int tid = threadIdx.x;
  const int rloc = tid / T;
  const int t_in_row = tid % T;
  const int team = t_in_row / kTeam;
  const int tau = t_in_row % kTeam;
  const int64_t m = (int64_t)blockIdx.x * rows + rloc;
  const bool row_ok = (rloc < rows) && (m < M);
  const int G = K >> 8;
  double* tb = xbuf + (size_t)(tid / kTeam) * 256;

  // ---- load all chunks of this thread (16 bf16 each)
  uint4 raw[CMAX][2];
#pragma unroll
  for (int c = 0; c < CMAX; ++c) {
    const int g = team + c * teams;
    if (row_ok && g < G) {
      const uint4* src = reinterpret_cast<const uint4*>(x + m * ldx + (int64_t)g * 256 + tau * 16);
      raw[c][0] = __ldg(src);
      raw[c][1] = __ldg(src + 1);
    } else {
      raw[c][0] = make_uint4(0, 0, 0, 0);
      raw[c][1] = make_uint4(0, 0, 0, 0);
    }
  }

  if constexpr (NORM) {
    // the per-channel vectors of a block are fetched after the row reduction
    // (fetching them earlier raises the register count and measured slower)
    auto fetch_vec = [&](const uint16_t* v, int g, uint4 (&d)[2]) {
      if (v) {
        const uint4* p = reinterpret_cast<const uint4*>(v + (int64_t)g * 256 + tau * 16);
        d[0] = __ldg(p);
        d[1] = __ldg(p + 1);
      }
    };
    // ---- sum of squares (exact squares; blocks past the row end hold zeros)
    double ss = 0.0;
#pragma unroll
    for (int c = 0; c < CMAX; ++c) {
      const uint32_t w[8] = {raw[c][0].x, raw[c][0].y, raw[c][0].z, raw[c][0].w,
                             raw[c][1].x, raw[c][1].y, raw[c][1].z, raw[c][1].w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const double lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
        ss = fma(lo, lo, ss);
        ss = fma(hi, hi, ss);
      }
    }
    if (T <= 32) {
      for (int off = T / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    } else {
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const int wpr = T / 32;
      if ((tid & 31) == 0) red64[tid / 32] = ss;
      __syncthreads();
      ss = 0.0;
      for (int w = 0; w < wpr; ++w) ss += red64[rloc * wpr + w];
    }
    const double d = ss / static_cast<double>(K) + static_cast<double>(norm.eps);
    const float r = d > 0.0 ? __double2float_rn(1.0 / sqrt(d)) : 0.f;
    // ---- per element: u = x r, * gamma, * (1 + scale), + shift, one bf16 rounding
#pragma unroll
    for (int c = 0; c < CMAX; ++c) {
      const int g = team + c * teams;
      if (g >= G) continue;   // blocks past the row end stay zero
      uint4 vg[2], vs[2], vc[2];
      fetch_vec(norm.gamma, g, vg);
      fetch_vec(norm.shift, g, vs);
      fetch_vec(norm.scale, g, vc);
      uint32_t* w = reinterpret_cast<uint32_t*>(&raw[c][0]);   // raw[c][0..1] are contiguous
      const uint32_t* wg = reinterpret_cast<const uint32_t*>(&vg[0]);
      const uint32_t* ws = reinterpret_cast<const uint32_t*>(&vs[0]);
      const uint32_t* wc = reinterpret_cast<const uint32_t*>(&vc[0]);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float u0 = __fmul_rn(__uint_as_float(w[j] << 16), r);
        float u1 = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), r);
        if (norm.gamma) {
          u0 = __fmul_rn(u0, __uint_as_float(wg[j] << 16));
          u1 = __fmul_rn(u1, __uint_as_float(wg[j] & 0xFFFF0000u));
        }
        if (norm.scale) {
          u0 = __fmul_rn(u0, __fadd_rn(1.0f, __uint_as_float(wc[j] << 16)));
          u1 = __fmul_rn(u1, __fadd_rn(1.0f, __uint_as_float(wc[j] & 0xFFFF0000u)));
        }
        if (norm.shift) {
          u0 = __fadd_rn(u0, __uint_as_float(ws[j] << 16));
          u1 = __fadd_rn(u1, __uint_as_float(ws[j] & 0xFFFF0000u));
        }
        w[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(u0)) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(u1)) << 16);
      }
    }
  }

  // ---- rotate
  float xr[CMAX][16];
#pragma unroll
  for (int c = 0; c < CMAX; ++c) {
    if constexpr (ROT) {
      rotate256_team(raw[c][0], raw[c][1], tau, tb, xr[c]);
    } else {
      load16_f32(raw[c][0], raw[c][1], xr[c]);
    }
  }

  // ---- scales
  // Position of register i of chunk c inside its 256-block:
  //   ROT: tau + 16*i ; !ROT: 16*tau + i.
  float inv_row = 0.f;
  float inv_g[CMAX][4];
  if constexpr (!G64) {
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < CMAX; ++c)
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(xr[c][i]));
    if (T <= 32) {
      for (int off = T / 2; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    } else {
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const int wpr = T / 32;
      if ((tid & 31) == 0) red[tid / 32] = amax;
      __syncthreads();
      amax = 0.f;
      for (int w = 0; w < wpr; ++w) amax = fmaxf(amax, red[rloc * wpr + w]);
    }
    inv_row = amax > 0.f ? __fdiv_rn(qmax, amax) : 0.f;
    if (row_ok && t_in_row == 0) scales[m] = __fdiv_rn(amax, qmax);
  } else {
#pragma unroll
    for (int c = 0; c < CMAX; ++c) {
      const int g = team + c * teams;
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        float am = 0.f;
        if constexpr (ROT) {
#pragma unroll
          for (int i = 4 * a; i < 4 * a + 4; ++i) am = fmaxf(am, fabsf(xr[c][i]));
          for (int off = 8; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
        } else {
          // 64-block a of this 256-block covers threads 4a .. 4a+3
#pragma unroll
          for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(xr[c][i]));
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
          am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
          am = __shfl_sync(0xffffffffu, am, (tid & ~15) + 4 * a);
        }
        inv_g[c][a] = am > 0.f ? __fdiv_rn(qmax, am) : 0.f;
        if (row_ok && g < G && tau == a) scales[m * (K / 64) + g * 4 + a] = __fdiv_rn(am, qmax);
      }
    }
  }

  // ---- quantise and store
#pragma unroll
  for (int c = 0; c < CMAX; ++c) {
    const int g = team + c * teams;
    uint32_t packed_words[4];
    if constexpr (ROT) {
      unsigned char* cb = reinterpret_cast<unsigned char*>(tb);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float inv = G64 ? inv_g[c][i >> 2] : inv_row;
        cb[tau + 16 * i] = static_cast<unsigned char>(code_byte<E4>(quant1(xr[c][i], inv, qmax)));
      }
      __syncwarp();
      const uint4 q4 = *reinterpret_cast<const uint4*>(cb + 16 * tau);
      __syncwarp();
      packed_words[0] = q4.x; packed_words[1] = q4.y; packed_words[2] = q4.z; packed_words[3] = q4.w;
    } else {
#pragma unroll
      for (int wv = 0; wv < 4; ++wv) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int i = 4 * wv + b;
          const float inv = G64 ? inv_g[c][tau >> 2] : inv_row;
          word |= code_byte<E4>(quant1(xr[c][i], inv, qmax)) << (8 * b);
        }
        packed_words[wv] = word;
      }
    }
    if (row_ok && g < G) {
      const int64_t k0 = (int64_t)g * 256 + tau * 16;
      if constexpr (OUT_PACKED) {
        // 16 codes -> 8 bytes, code k (even) in the low nibble, k+1 in the high nibble
        uint32_t outw[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t acc = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t pair = (h * 2 + j / 2 < 4) ? packed_words[h * 2 + j / 2] : 0u;
            const uint32_t lo = (pair >> (16 * (j & 1))) & 0xFu;
            const uint32_t hi = (pair >> (16 * (j & 1) + 8)) & 0xFu;
            acc |= (lo | (hi << 4)) << (8 * j);
          }
          outw[h] = acc;
        }
        uint8_t* dst = reinterpret_cast<uint8_t*>(codes) + m * (int64_t)(K / 2) + k0 / 2;
        *reinterpret_cast<uint2*>(dst) = make_uint2(outw[0], outw[1]);
      } else {
        *reinterpret_cast<uint4*>(codes + m * (int64_t)K + k0) =
            make_uint4(packed_words[0], packed_words[1], packed_words[2], packed_words[3]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Low-rank down product ld[M, r] = X[M, K] @ L1 (unrotated bf16 input) with L1
// given output-major as l1t[r, K], on the legacy bf16 mma.sync path
// (m16n8k16, fp32 accumulation).  One CTA = 16 tokens; its 8 warps split K
// and reduce through shared memory in a fixed order (deterministic).
// Fragment loads are 32-bit: A pairs come from consecutive k of one token row,
// B pairs from consecutive k of one l1t row.
// ---------------------------------------------------------------------------
constexpr int kLrWarps = 8;

template <int R>
__global__ void __launch_bounds__(kLrWarps * 32) lowrank_down_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                     int K, int64_t ldx,
                                                                     const uint16_t* __restrict__ l1t,
                                                                     uint16_t* __restrict__ ld) {
  constexpr int NT = R / 8;
  __shared__ float part[kLrWarps][16][R + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int64_t m0 = (int64_t)blockIdx.x * 16;
  const int64_t ra = m0 + g, rb = m0 + g + 8;
  const bool va = ra < M, vb = rb < M;
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const int kper = K / kLrWarps;
  const int kbeg = warp * kper, kend = kbeg + kper;
  const uint32_t* xa = reinterpret_cast<const uint32_t*>(x + (va ? ra : 0) * ldx);
  const uint32_t* xb = reinterpret_cast<const uint32_t*>(x + (vb ? rb : 0) * ldx);
#pragma unroll 4
  for (int k = kbeg; k < kend; k += 16) {
    const int kw = k >> 1;   // 32-bit word index of k
    uint32_t a[4];
    a[0] = va ? __ldg(xa + kw + c4) : 0u;
    a[1] = vb ? __ldg(xb + kw + c4) : 0u;
    a[2] = va ? __ldg(xa + kw + c4 + 4) : 0u;
    a[3] = vb ? __ldg(xb + kw + c4 + 4) : 0u;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const uint32_t* lb = reinterpret_cast<const uint32_t*>(l1t + (int64_t)(n * 8 + g) * K) + kw;
      const uint32_t b0 = __ldg(lb + c4);
      const uint32_t b1 = __ldg(lb + c4 + 4);
      asm volatile(
          "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
          "{%0,%1,%2,%3};"
          : "+f"(acc[n][0]), "+f"(acc[n][1]), "+f"(acc[n][2]), "+f"(acc[n][3])
          : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    part[warp][g][n * 8 + 2 * c4] = acc[n][0];
    part[warp][g][n * 8 + 2 * c4 + 1] = acc[n][1];
    part[warp][g + 8][n * 8 + 2 * c4] = acc[n][2];
    part[warp][g + 8][n * 8 + 2 * c4 + 1] = acc[n][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 16 * R; i += blockDim.x) {
    const int rr = i / R, cc = i % R;
    const int64_t mm = m0 + rr;
    if (mm < M) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kLrWarps; ++w) s += part[w][rr][cc];
      ld[mm * R + cc] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
    }
  }
}

// ---------------------------------------------------------------------------
// Single-pass group-scale prologue: rotated group-64 codes and scales plus the
// low-rank down product from one read of X.
//
// One CTA = 16 tokens = 16 teams; the CTA walks the 256-blocks of its rows in
// order.  For block g every team loads its token's 256 bf16 values (thread tau:
// elements 16 tau .. 16 tau + 15, prefetched two blocks ahead), copies them to
// a shared-memory slab [16 tokens][256], and rotates/quantises them exactly as
// rot_quant_kernel does (same float64 rotation, same scale and rounding
// operations, so codes and scales are identical).  After one barrier the eight
// warps run the low-rank MMAs on the slab: warp w owns k-steps 2w and 2w + 1
// of every block (m16n8k16, bf16 in, fp32 accumulate, A fragments by ldmatrix,
// B fragments from l1t), and at the end the eight partial sums are added in a
// fixed order (deterministic) and rounded to bf16 once.
// The slab is double-buffered, so one barrier per block suffices: a warp that
// reaches block g + 1's barrier has finished block g's MMAs.
// ---------------------------------------------------------------------------
constexpr int kFuseTok = 16;     // tokens per CTA (one team each)
constexpr int kSlabPitch = 264;  // bf16 per slab row: 256 + 8 (conflict-free ldmatrix rows)
constexpr size_t kFuseXbufBytes = (size_t)kFuseTok * 256 * sizeof(double);
constexpr size_t kFuseSlabBytes = 2 * (size_t)kFuseTok * kSlabPitch * sizeof(uint16_t);

__host__ __device__ constexpr size_t fuse_smem_bytes(int r) {
  const size_t main = kFuseXbufBytes + kFuseSlabBytes;
  const size_t red = (size_t)kLrWarps * kFuseTok * (r + 1) * sizeof(float);
  return main > red ? main : red;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&a)[4], const uint16_t* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <bool ROT, int R, bool E4 = false>
__global__ void __launch_bounds__(kLrWarps * 32, R <= 32 ? 3 : 2)
    rot_quant_lowrank_kernel(const uint16_t* __restrict__ x, int64_t M, int K, int64_t ldx, float qmax,
                             const uint16_t* __restrict__ l1t, int8_t* __restrict__ codes,
                             float* __restrict__ scales, uint16_t* __restrict__ ld) {
  pdl_launch_dependents();   // as in rot_quant_kernel
  constexpr int NT = R / 8;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* xbuf = reinterpret_cast<double*>(smem_raw);
  uint16_t* slab = reinterpret_cast<uint16_t*>(smem_raw + kFuseXbufBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int team = tid >> 4, tau = tid & 15;
  const int64_t m0 = (int64_t)blockIdx.x * kFuseTok;
  const int64_t m = m0 + team;
  const bool row_ok = m < M;
  const int G = K >> 8;
  double* tb = xbuf + team * 256;
  const uint4* src = reinterpret_cast<const uint4*>(x + (row_ok ? m : 0) * ldx + tau * 16);
  auto fetch = [&](uint4 (&r)[2], int g) {
    if (row_ok) {
      r[0] = __ldg(src + g * 32);
      r[1] = __ldg(src + g * 32 + 1);
    } else {
      r[0] = make_uint4(0, 0, 0, 0);
      r[1] = make_uint4(0, 0, 0, 0);
    }
  };
  const int g4 = lane >> 2, c4 = lane & 3;
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  uint4 cur[2], nxt[2];
  fetch(cur, 0);
  if (G > 1) fetch(nxt, 1);
  for (int g = 0; g < G; ++g) {
    const uint4 lo = cur[0], hi = cur[1];
    cur[0] = nxt[0];
    cur[1] = nxt[1];
    if (g + 2 < G) fetch(nxt, g + 2);
    uint16_t* sb = slab + (g & 1) * kFuseTok * kSlabPitch;
    *reinterpret_cast<uint4*>(sb + team * kSlabPitch + tau * 16) = lo;
    *reinterpret_cast<uint4*>(sb + team * kSlabPitch + tau * 16 + 8) = hi;

    // ---- rotate, group-64 scales, quantise (register i = position tau + 16 i
    // with the rotation, 16 tau + i without)
    float xr[16];
    if constexpr (ROT) {
      rotate256_team(lo, hi, tau, tb, xr);
    } else {
      load16_f32(lo, hi, xr);
    }
    float inv_g[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float am = 0.f;
      if constexpr (ROT) {
#pragma unroll
        for (int i = 4 * a; i < 4 * a + 4; ++i) am = fmaxf(am, fabsf(xr[i]));
        for (int off = 8; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(xr[i]));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
        am = __shfl_sync(0xffffffffu, am, (lane & 16) + 4 * a);
      }
      inv_g[a] = am > 0.f ? __fdiv_rn(qmax, am) : 0.f;
      if (row_ok && tau == a) scales[m * (K / 64) + g * 4 + a] = __fdiv_rn(am, qmax);
    }
    uint32_t w[4];
    if constexpr (ROT) {
      unsigned char* cb = reinterpret_cast<unsigned char*>(tb);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        cb[tau + 16 * i] = static_cast<unsigned char>(code_byte<E4>(quant1(xr[i], inv_g[i >> 2], qmax)));
      __syncwarp();
      const uint4 q4 = *reinterpret_cast<const uint4*>(cb + 16 * tau);
      __syncwarp();
      w[0] = q4.x; w[1] = q4.y; w[2] = q4.z; w[3] = q4.w;
    } else {
#pragma unroll
      for (int wv = 0; wv < 4; ++wv) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          word |= code_byte<E4>(quant1(xr[4 * wv + b], inv_g[tau >> 2], qmax)) << (8 * b);
        w[wv] = word;
      }
    }
    if (row_ok)
      *reinterpret_cast<uint4*>(codes + m * (int64_t)K + (int64_t)g * 256 + tau * 16) =
          make_uint4(w[0], w[1], w[2], w[3]);

    // ---- low-rank MMAs on the slab
    __syncthreads();
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int kk = (2 * warp + s) * 16;
      uint32_t a[4];
      ldmatrix_x4(a, sb + (lane & 15) * kSlabPitch + kk + (lane >> 4) * 8);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const uint32_t* lb =
            reinterpret_cast<const uint32_t*>(l1t + (int64_t)(n * 8 + g4) * K + (int64_t)g * 256 + kk);
        mma_bf16_16816(acc[n], a, __ldg(lb + c4), __ldg(lb + c4 + 4));
      }
    }
  }

  // ---- fixed-order reduction of the eight warps' partial sums
  __syncthreads();
  float* part = reinterpret_cast<float*>(smem_raw);   // [8 warps][16 tokens][R + 1]
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    float* p0 = part + ((size_t)warp * kFuseTok + g4) * (R + 1) + n * 8 + 2 * c4;
    float* p1 = p0 + 8 * (R + 1);
    p0[0] = acc[n][0];
    p0[1] = acc[n][1];
    p1[0] = acc[n][2];
    p1[1] = acc[n][3];
  }
  __syncthreads();
  for (int i = tid; i < kFuseTok * R; i += blockDim.x) {
    const int rr = i / R, cc = i % R;
    const int64_t mm = m0 + rr;
    if (mm < M) {
      float s = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kLrWarps; ++w2) s += part[((size_t)w2 * kFuseTok + rr) * (R + 1) + cc];
      ld[mm * R + cc] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
    }
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
namespace {
struct Geometry {
  int teams, cmax, T, rows, threads;
  size_t smem;
};

Geometry geometry(int64_t K) {
  Geometry gm{};
  const int G = static_cast<int>(K / 256);
  int teams = G < 16 ? G : 16;
  if (teams > 1 && (teams & 1)) teams += 1;   // keep T a multiple of 32 when above 16
  gm.teams = teams;
  gm.cmax = (G + teams - 1) / teams;
  gm.T = kTeam * teams;
  gm.rows = gm.T >= 256 ? 1 : 256 / gm.T;
  gm.threads = gm.T * gm.rows;
  gm.smem = (size_t)(gm.threads / kTeam) * 256 * sizeof(double) + 64 * sizeof(float) + 64 * sizeof(double);
  return gm;
}

template <bool ROT, bool G64, bool PK, bool NORM = false, bool E4 = false>
cudaError_t launch_rq_c(int cmax, dim3 grid, int threads, size_t smem, cudaStream_t st, const uint16_t* x,
                        int64_t M, int K, int64_t ldx, float qmax, int teams, int rows, int8_t* codes,
                        float* scales, NormArgs norm = NormArgs{}) {
  switch (cmax) {
#define RBD_RQ_CASE(C)                                                                                    \
  case C: {                                                                                               \
    auto kern = rot_quant_kernel<ROT, G64, PK, C, NORM, E4>;                                              \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                                       \
    kern<<<grid, threads, smem, st>>>(x, M, K, ldx, qmax, teams, rows, codes, scales, norm);             \
    return cudaGetLastError();                                                                            \
  }
    RBD_RQ_CASE(1)
    RBD_RQ_CASE(2)
    RBD_RQ_CASE(3)
    RBD_RQ_CASE(4)
#undef RBD_RQ_CASE
    default:
      return cudaErrorInvalidValue;
  }
}
}  // namespace

cudaError_t launch_rot_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int bits, bool rot, bool g64,
                             bool packed, bool e4m3, int8_t* codes, float* scales, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const Geometry gm = geometry(K);
  const float qmax = bits == 4 ? 7.f : 127.f;
  const dim3 grid(static_cast<unsigned>((M + gm.rows - 1) / gm.rows));
  const int Ki = static_cast<int>(K);
  if (e4m3) {
    if (packed || bits != 4) return cudaErrorInvalidValue;
#define RBD_RQ_E4(R_, G_)                                                                                \
  return launch_rq_c<R_, G_, false, false, true>(gm.cmax, grid, gm.threads, gm.smem, st, x, M, Ki, ldx, qmax, \
                                                 gm.teams, gm.rows, codes, scales)
    if (rot) {
      if (g64) RBD_RQ_E4(true, true); else RBD_RQ_E4(true, false);
    } else {
      if (g64) RBD_RQ_E4(false, true); else RBD_RQ_E4(false, false);
    }
#undef RBD_RQ_E4
  }
#define RBD_RQ_DISPATCH(R_, G_, P_)                                                                      \
  return launch_rq_c<R_, G_, P_>(gm.cmax, grid, gm.threads, gm.smem, st, x, M, Ki, ldx, qmax, gm.teams, \
                                 gm.rows, codes, scales)
  if (rot) {
    if (g64) {
      if (packed) RBD_RQ_DISPATCH(true, true, true); else RBD_RQ_DISPATCH(true, true, false);
    } else {
      if (packed) RBD_RQ_DISPATCH(true, false, true); else RBD_RQ_DISPATCH(true, false, false);
    }
  } else {
    if (g64) {
      if (packed) RBD_RQ_DISPATCH(false, true, true); else RBD_RQ_DISPATCH(false, true, false);
    } else {
      if (packed) RBD_RQ_DISPATCH(false, false, true); else RBD_RQ_DISPATCH(false, false, false);
    }
  }
#undef RBD_RQ_DISPATCH
}

cudaError_t launch_norm_rot_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int bits, bool rot,
                                  bool g64, bool e4m3, const uint16_t* gamma, const uint16_t* shift,
                                  const uint16_t* scale, float eps, int8_t* codes, float* scales, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const Geometry gm = geometry(K);
  const float qmax = bits == 4 ? 7.f : 127.f;
  const dim3 grid(static_cast<unsigned>((M + gm.rows - 1) / gm.rows));
  const int Ki = static_cast<int>(K);
  const NormArgs norm{gamma, shift, scale, eps};
  if (e4m3 && bits != 4) return cudaErrorInvalidValue;
#define RBD_NRQ(R_, G_)                                                                                      \
  return e4m3 ? launch_rq_c<R_, G_, false, true, true>(gm.cmax, grid, gm.threads, gm.smem, st, x, M, Ki, ldx,  \
                                                       qmax, gm.teams, gm.rows, codes, scales, norm)           \
              : launch_rq_c<R_, G_, false, true, false>(gm.cmax, grid, gm.threads, gm.smem, st, x, M, Ki, ldx, \
                                                        qmax, gm.teams, gm.rows, codes, scales, norm)
  if (rot) {
    if (g64) RBD_NRQ(true, true); else RBD_NRQ(true, false);
  } else {
    if (g64) RBD_NRQ(false, true); else RBD_NRQ(false, false);
  }
#undef RBD_NRQ
}

cudaError_t launch_lowrank_down(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const uint16_t* l1t, int r,
                                uint16_t* ld, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((M + 15) / 16));
  const int Ki = static_cast<int>(K);
  const int threads = kLrWarps * 32;
  switch (r) {
    case 16: lowrank_down_kernel<16><<<grid, threads, 0, st>>>(x, M, Ki, ldx, l1t, ld); break;
    case 32: lowrank_down_kernel<32><<<grid, threads, 0, st>>>(x, M, Ki, ldx, l1t, ld); break;
    case 64: lowrank_down_kernel<64><<<grid, threads, 0, st>>>(x, M, Ki, ldx, l1t, ld); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_rot_quant_lowrank(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int bits, bool rot,
                                     bool e4m3, const uint16_t* l1t, int r, int8_t* codes, float* scales,
                                     uint16_t* ld, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((M + kFuseTok - 1) / kFuseTok));
  const float qmax = bits == 4 ? 7.f : 127.f;
  const int Ki = static_cast<int>(K);
  if (e4m3 && bits != 4) return cudaErrorInvalidValue;
#define RBD_RQL_CASE(ROT_, R_)                                                                          \
  {                                                                                                     \
    auto kern = e4m3 ? rot_quant_lowrank_kernel<ROT_, R_, true> : rot_quant_lowrank_kernel<ROT_, R_, false>; \
    const size_t smem = fuse_smem_bytes(R_);                                                            \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                                     \
    kern<<<grid, kLrWarps * 32, smem, st>>>(x, M, Ki, ldx, qmax, l1t, codes, scales, ld);               \
    return cudaGetLastError();                                                                          \
  }
  if (rot) {
    switch (r) {
      case 16: RBD_RQL_CASE(true, 16)
      case 32: RBD_RQL_CASE(true, 32)
      case 64: RBD_RQL_CASE(true, 64)
      default: return cudaErrorInvalidValue;
    }
  }
  switch (r) {
    case 16: RBD_RQL_CASE(false, 16)
    case 32: RBD_RQL_CASE(false, 32)
    case 64: RBD_RQL_CASE(false, 64)
    default: return cudaErrorInvalidValue;
  }
#undef RBD_RQL_CASE
}

}  // namespace rbd
