// INT8 attention in the SageAttention v1 scheme: Q.K^T on INT8 codes with one
// scale per token and head (keys smoothed by their mean over the tokens first),
// softmax, and P.V with FP16 operands and float32 accumulation.
//
// Method: "Krea 2 Turbo OrbitQuant W4A4", "Fused transformer" (attention takes
// Q.K^T in INT8 and P.V in FP16, as SageAttention v1 does).  The steps the page
// leaves open follow the plainest form of that scheme:
//   - per head and channel, the key mean over all Tk tokens in float64 (the sum
//     of bf16 values is exact in float64 while a column's values span at most
//     31 binades, so the order of summation does not matter), one IEEE division
//     by Tk; the smoothed key k - mean is formed in float64 and rounded once to
//     float32;
//   - Q and the smoothed K quantised per (token, head) over the 128 channels
//     with the activation quantiser's float32 steps: amax, s = amax / 127,
//     inv = 127 / amax (IEEE divisions), q = clamp(rint(x * inv), -128, 127);
//   - S = (q . k) s_q s_k / sqrt(128) from the exact integer dot product;
//   - softmax over the keys; P.V with V converted bf16 -> fp16 (round to
//     nearest) and P rounded to fp16 after subtracting the running row maximum.
//
// Kernels:
//   attn_key_colsum_kernel  partial float64 column sums of K over 256-token chunks;
//   attn_key_mean_kernel    the chunks added in order, divided by Tk;
//   attn_quant_kernel       a warp per (token, head): Q and smoothed-K codes + scales;
//   attn_vt_kernel          V -> fp16, transposed to [head][channel][token];
//   attn_int8_kernel        the attention itself, one CTA per (head, 128 queries).
//
// attn_int8_kernel, per CTA (19 warps):
//   warps 0 and 18: TMA producers (Q once; K codes and key scales of 128-key
//           tiles into a 2-stage ring freed by Q.K^T; V^T tiles into a 2-stage
//           ring freed by P.V);
//   warp 1: TMEM owner and MMA issuer: S_j = Q K_j^T (kind::i8, int32) into one
//           of two 128-column S buffers, O += P_j V_j (kind::f16, fp32) into a
//           third 128-column buffer;
//   warps 2-17: softmax, four threads per query row (TMEM lane), each with 32
//           of the tile's keys: its part of the row of S_j (int32) is loaded once
//           into registers, scaled, the four parts' row maxima exchanged through
//           shared memory, keys past Tk masked, and 2^(logit - m) taken against
//           the row's running maximum m.  m only moves when a tile's maximum exceeds it by more than 8
//           (so P <= 256 stays well inside fp16); O is then rescaled in TMEM
//           first.  P goes to shared memory as fp16 in the 128-byte-swizzled
//           K-major layout the P.V MMA reads.  The P.V MMA is N = 144 wide: 16
//           rows of ones below V^T make its column 128 the row sum of P.
// The tensor core runs QK_{j+1} while the softmax works on tile j, and PV_j
// while it works on tile j + 1.
#include <cuda_fp16.h>

#include <type_traits>

#include "rbd_common.cuh"
#include "rbd_internal.cuh"

namespace rbd {

namespace {

constexpr int kAttnDim = 128;           // channels per head
constexpr int kAttnTile = 128;          // queries per CTA, keys per tile
constexpr int kAttnParts = 4;           // softmax threads per query row
constexpr int kAttnPartKeys = 128 / kAttnParts;   // keys of a tile per softmax thread
constexpr int kAttnSoftmax0 = 2;        // first softmax warp
constexpr int kAttnVWarp = kAttnSoftmax0 + 4 * kAttnParts;   // the V producer (warp 18)
constexpr int kAttnThreads = 32 * (kAttnVWarp + 1);          // 19 warps
constexpr int kColsumChunk = 256;       // tokens per partial column sum
constexpr float kLog2eRsqrtD = 0.12751743082459868f;   // log2(e) / sqrt(128)
constexpr float kLazyRescale = 8.0f;    // base-2 headroom before the running maximum moves

// The P.V MMA runs with N = 144: rows 128..143 of every V^T half hold fp16 ones,
// so O's column 128 accumulates the row sum of exactly the fp16 P that P.V
// multiplies (the softmax denominator), rescaled together with O.
constexpr int kPvN = kAttnDim + 16;
constexpr uint32_t kVHalf = kPvN * 128;                // 144 rows x 128 B (64 keys)

// shared-memory layout of attn_int8_kernel (offsets from a 1024-byte aligned base)
constexpr uint32_t kQOff = 0;                          // Q codes, 128 x 128 B
constexpr uint32_t kKOff = kQOff + 16384;              // K codes, 2 stages x 16 KB
constexpr uint32_t kVOff = kKOff + 2 * 16384;          // V^T (+ ones), 2 stages x 2 halves x 18 KB
constexpr uint32_t kPOff = kVOff + 4 * kVHalf;         // P, 2 buffers x 2 halves x 16 KB
// Key scales ride with the K codes but are read by the softmax, after Q.K^T: they
// get a 4-deep ring.  Slot j % 4 is rewritten for tile j + 4 only after Q.K^T of
// tile j + 2, which waits for the softmax of tile j to release its S buffer, which
// it does after reading the slot.
constexpr uint32_t kSkOff = kPOff + 2 * 32768;         // key scales, 4 slots x 512 B
constexpr uint32_t kRedOff = kSkOff + 4 * 512;         // row-maximum exchange, 2 x kAttnParts x 128 floats
constexpr uint32_t kBarOff = kRedOff + 2 * kAttnParts * 128 * 4;
constexpr uint32_t kAttnSmem = kBarOff + 512 + 1024;   // + alignment slack

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 3D tiled bulk tensor load (c0 innermost).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t c0,
                                            int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 32 lanes x 16 columns register -> TMEM store.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// kind::f16 instruction descriptor with fp16 A and B (format 0), F32 accumulation.
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t m, uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

}  // namespace

// ---------------------------------------------------------------------------
// Preparation kernels
// ---------------------------------------------------------------------------

// partial[chunk][h][c] = sum over the chunk's tokens of k[t][h * 128 + c] (float64)
__global__ void __launch_bounds__(kAttnDim) attn_key_colsum_kernel(const uint16_t* __restrict__ k, int64_t ldk,
                                                                   int Tk, int H, double* __restrict__ partial) {
  const int c = threadIdx.x, h = blockIdx.y, chunk = blockIdx.x;
  const int t0 = chunk * kColsumChunk;
  const int t1 = min(Tk, t0 + kColsumChunk);
  double s0 = 0.0, s1 = 0.0;   // two chains; exact sums, so their order is immaterial
  const uint16_t* p = k + (int64_t)h * kAttnDim + c;
  int t = t0;
  for (; t + 1 < t1; t += 2) {
    s0 += (double)__uint_as_float((uint32_t)__ldg(p + (int64_t)t * ldk) << 16);
    s1 += (double)__uint_as_float((uint32_t)__ldg(p + (int64_t)(t + 1) * ldk) << 16);
  }
  if (t < t1) s0 += (double)__uint_as_float((uint32_t)__ldg(p + (int64_t)t * ldk) << 16);
  partial[((int64_t)chunk * H + h) * kAttnDim + c] = s0 + s1;
}

// mean[h][c] = (sum over chunks, in order) / Tk
__global__ void __launch_bounds__(kAttnDim) attn_key_mean_kernel(const double* __restrict__ partial, int nchunks,
                                                                 int Tk, int H, double* __restrict__ mean) {
  const int c = threadIdx.x, h = blockIdx.x;
  double s = 0.0;
  for (int i = 0; i < nchunks; ++i) s += partial[((int64_t)i * H + h) * kAttnDim + c];
  mean[h * kAttnDim + c] = s / (double)Tk;
}

// A warp per (token, head) unit: units [0, Tq*H) quantise Q, [Tq*H, (Tq+Tk)*H) the
// smoothed K.  Lane l owns channels 4l .. 4l+3.
__global__ void __launch_bounds__(256) attn_quant_kernel(const uint16_t* __restrict__ q, int64_t ldq,
                                                         const uint16_t* __restrict__ k, int64_t ldk, int Tq, int Tk,
                                                         int H, const double* __restrict__ mean,
                                                         int8_t* __restrict__ qc, float* __restrict__ sq,
                                                         int8_t* __restrict__ kc, float* __restrict__ sk,
                                                         int64_t tkp) {
  const int64_t unit = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t nq = (int64_t)Tq * H, nk = (int64_t)Tk * H;
  if (unit >= nq + nk) return;
  const bool is_k = unit >= nq;
  const int64_t u = is_k ? unit - nq : unit;
  const int t = (int)(u / H), h = (int)(u % H);
  const uint16_t* src = (is_k ? k + (int64_t)t * ldk : q + (int64_t)t * ldq) + h * kAttnDim + 4 * lane;
  const uint2 raw = *reinterpret_cast<const uint2*>(src);
  float x[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
  if (is_k) {
    const double* mu = mean + h * kAttnDim + 4 * lane;
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = __double2float_rn((double)x[e] - mu[e]);
  }
  float am = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
  const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    int v = __float2int_rn(__fmul_rn(x[e], inv));
    v = v > 127 ? 127 : (v < -128 ? -128 : v);
    word |= ((uint32_t)v & 0xFFu) << (8 * e);
  }
  int8_t* dst = is_k ? kc + ((int64_t)h * Tk + t) * kAttnDim : qc + ((int64_t)h * Tq + t) * kAttnDim;
  *reinterpret_cast<uint32_t*>(dst + 4 * lane) = word;
  if (lane == 0) {
    const float s = __fdiv_rn(am, 127.f);
    if (is_k) sk[(int64_t)h * tkp + t] = s;
    else sq[(int64_t)h * Tq + t] = s;
  }
}

// V [Tk, ldv] bf16 -> vt [H][128][tkp] fp16 (round to nearest); tokens Tk .. tkp-1
// are written as zeros.  A CTA transposes 64 tokens x 128 channels of one head.
__global__ void __launch_bounds__(256) attn_vt_kernel(const uint16_t* __restrict__ v, int64_t ldv, int Tk, int H,
                                                      __half* __restrict__ vt, int64_t tkp) {
  __shared__ __half tile[kAttnDim][64 + 2];
  const int h = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * 64;
  // load: thread -> (token tt, channel pair cp); 64 tokens x 64 pairs
  for (int i = threadIdx.x; i < 64 * 64; i += blockDim.x) {
    const int tt = i >> 6, cp = i & 63;
    const int64_t t = t0 + tt;
    float a = 0.f, b = 0.f;
    if (t < Tk) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(v + t * ldv + h * kAttnDim + 2 * cp);
      a = __uint_as_float(w << 16);
      b = __uint_as_float(w & 0xFFFF0000u);
    }
    tile[2 * cp][tt] = __float2half_rn(a);
    tile[2 * cp + 1][tt] = __float2half_rn(b);
  }
  __syncthreads();
  // store: thread -> (channel c, token pair tp); each channel row is 64 contiguous tokens
  for (int i = threadIdx.x; i < kAttnDim * 32; i += blockDim.x) {
    const int c = i >> 5, tp = i & 31;
    const int64_t t = t0 + 2 * tp;
    if (t < tkp) {
      __half2 pair = __halves2half2(tile[c][2 * tp], tile[c][2 * tp + 1]);
      *reinterpret_cast<__half2*>(vt + ((int64_t)h * kAttnDim + c) * tkp + t) = pair;
    }
  }
}

// ---------------------------------------------------------------------------
// Attention kernel
// ---------------------------------------------------------------------------
struct AttnArgs {
  const float* sq;   // [H][Tq]
  int Tq, Tk, H;
  uint16_t* o;       // bf16 [Tq, ldo], head h at columns h*128
  int64_t ldo;
};

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_int8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_sk,
                     const AttnArgs args) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023u) & ~uintptr_t(1023u));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;     // [2] K codes and key scales of a stage landed
  uint64_t* k_empty = bars + 3;    // [2] Q.K^T of the stage's tile done
  uint64_t* v_full = bars + 21;    // [2] V^T of a stage landed
  uint64_t* v_empty = bars + 23;   // [2] P.V of the stage's tile done
  uint64_t* s_full = bars + 5;     // [2]
  uint64_t* s_empty = bars + 7;    // [2]
  uint64_t* p_full = bars + 9;     // [2]
  uint64_t* pv_done = bars + 11;   // [2]
  uint64_t* o_done = bars + 13;
  uint64_t* drain = bars + 14;
  uint64_t* red_bar = bars + 32;   // [2][4] the row maxima of a lane quarter's four parts are in shared memory
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 26);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * kAttnTile;
  const int ntiles = (args.Tk + kAttnTile - 1) / kAttnTile;

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&k_full[b], 1);
      mbar_init(&k_empty[b], 1);
      mbar_init(&v_full[b], 1);
      mbar_init(&v_empty[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 4 * kAttnParts);
      mbar_init(&p_full[b], 4 * kAttnParts);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    for (int b = 0; b < 8; ++b) mbar_init(&red_bar[b], kAttnParts);
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_sk);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  // the ones rows (128..143) of the four V^T halves: 4 x 2 KB of fp16 1.0
  for (int i = threadIdx.x; i < 4 * 128; i += kAttnThreads) {
    const int hv = i >> 7, w = i & 127;
    reinterpret_cast<uint4*>(smem + kVOff + hv * kVHalf + 16384)[w] =
        make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
  }
  fence_async_shared();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t t_o = tmem + 2 * kAttnTile;   // O accumulator columns 256..399 (column 384: the row sum)

  if (warp == 0 || warp == kAttnVWarp) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: Q once, then K codes and key scales (a stage is free once its Q.K^T is
    // done); warp 18: V^T (a stage is free once its P.V is done)
    if (lane == 0) {
      const bool kprod = warp == 0;
      bool ok = true;
      if (kprod) {
        mbar_arrive_expect_tx(q_full, 16384);
        tma_load_3d(smem + kQOff, &tm_q, q_full, 0, q0, h);
      }
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1;
        if (kprod) {
          if (!mbar_wait(&k_empty[s], ((j >> 1) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[s], 16384 + 512);
          tma_load_3d(smem + kKOff + s * 16384, &tm_k, &k_full[s], 0, j * kAttnTile, h);
          tma_load_2d(smem + kSkOff + (j & 3) * 512, &tm_sk, &k_full[s], j * kAttnTile, h);
        } else {
          if (!mbar_wait(&v_empty[s], ((j >> 1) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[s], 32768);
          tma_load_3d(smem + kVOff + (2 * s) * kVHalf, &tm_v, &v_full[s], j * kAttnTile, 0, h);
          tma_load_3d(smem + kVOff + (2 * s + 1) * kVHalf, &tm_v, &v_full[s], j * kAttnTile + 64, 0, h);
        }
      }
      if (!ok) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t id_qk = idesc_i8(kAttnTile, kAttnTile);
      const uint32_t id_pv = idesc_f16(kAttnTile, kPvN);
      const uint64_t qdesc = smem_desc_kmajor(smem_u32(smem + kQOff), 128);
      bool ok = mbar_wait(q_full, 0);
      tc_fence_after();
      auto issue_qk = [&](int j) {
        const int s = j & 1;
        if (!mbar_wait(&k_full[s], (j >> 1) & 1)) return false;
        if (j >= 2 && !mbar_wait(&s_empty[s], ((j - 2) >> 1) & 1)) return false;
        tc_fence_after();
        const uint64_t kdesc = smem_desc_kmajor(smem_u32(smem + kKOff + s * 16384), 128);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_i8_ss(tmem + s * kAttnTile, qdesc + 2 * kk, kdesc + 2 * kk, id_qk, kk > 0);
        tc_commit(&s_full[s]);
        tc_commit(&k_empty[s]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && ntiles > 1) ok = issue_qk(1);
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1;
        if (!mbar_wait(&p_full[s], (j >> 1) & 1) || !mbar_wait(&v_full[s], (j >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t pbase = smem_u32(smem + kPOff + s * 32768);
        const uint32_t vbase = smem_u32(smem + kVOff + 2 * s * kVHalf);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ph = (uint32_t)(kk >> 2) * 16384u, vh = (uint32_t)(kk >> 2) * kVHalf;
          const uint32_t off = (uint32_t)(kk & 3) * 32u;
          mma_bf16_ss(t_o, smem_desc_kmajor(pbase + ph + off, 128), smem_desc_kmajor(vbase + vh + off, 128),
                      id_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&pv_done[s]);
        tc_commit(&v_empty[s]);
        if (j + 2 < ntiles && !issue_qk(j + 2)) { ok = false; break; }
      }
      tc_commit(o_done);
      tc_commit(drain);
      mbar_wait(drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp < kAttnVWarp) {
    // ------------------------------------------------------------ softmax warps
    // Warp w (2..17) covers query rows 32 (w & 3) .. +31 (its TMEM lane quarter) and
    // keys 32 part .. +31 of every tile (part = (w - 2) >> 2): four warps per row.
    // The four exchange their row maxima through shared memory once per tile.
    const uint32_t qtr = warp & 3u;
    const int part = ((int)warp - kAttnSoftmax0) >> 2;
    const int row = 32 * (int)qtr + (int)lane;                  // query row inside the tile (TMEM lane)
    const uint32_t lane_addr = (32u * qtr) << 16;
    const int qrow = q0 + row;
    const float cq = qrow < args.Tq ? __ldg(args.sq + (int64_t)h * args.Tq + qrow) * kLog2eRsqrtD : 0.f;
    float* red = reinterpret_cast<float*>(smem + kRedOff);     // [2 tiles][kAttnParts][128 rows]
    // waits whose outcome the whole warp shares: the warp's TMEM accesses are
    // .sync.aligned, so its lanes must never part ways on a timeout
    auto wait_warp = [](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity)) != 0;
    };
    float m_use = -INFINITY;   // running maximum, base-2 logits
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j & 1;
      if (!wait_warp(&s_full[s], (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      uint32_t sreg[kAttnPartKeys];
      tmem_ld32(tmem + lane_addr + s * kAttnTile + kAttnPartKeys * part, sreg);
      tmem_wait_ld();
      // u = acc * s_k (the logit is u * cq, cq = s_q log2(e) / sqrt(128) >= 0, so the row
      // maximum of u gives that of the logits); keys past Tk are left out (last tile only)
      const float4* sk4 = reinterpret_cast<const float4*>(smem + kSkOff + (j & 3) * 512) + (kAttnPartKeys / 4) * part;
      const int nvalid = args.Tk - j * kAttnTile - kAttnPartKeys * part;   // valid keys of this part
      const bool full = nvalid >= kAttnPartKeys;
      float mx[8];   // eight independent max chains
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
      auto logits = [&](auto full_tile) {
#pragma unroll
        for (int c4 = 0; c4 < kAttnPartKeys / 4; ++c4) {
          const float4 kq = sk4[c4];
          const float ks[4] = {kq.x, kq.y, kq.z, kq.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = 4 * c4 + e;
            const float a = __uint_as_float(sreg[col] + 0x4B400000u) - 12582912.0f;   // exact: |acc| < 2^22
            const float u = a * ks[e];
            if (decltype(full_tile)::value || col < nvalid) mx[col & 7] = fmaxf(mx[col & 7], u);
            sreg[col] = __float_as_uint(u);
          }
        }
      };
      if (full) logits(std::true_type{});
      else logits(std::false_type{});
      float mh = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                       fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      // S buffer read and key-scale slot read: release the S buffer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[s]);
      red[(s * kAttnParts + part) * kAttnTile + row] = mh;
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_bar[4 * s + qtr]);   // only the warps of these rows wait on it
      if (!wait_warp(&red_bar[4 * s + qtr], (j >> 1) & 1)) { ok = false; break; }
#pragma unroll
      for (int o = 1; o < kAttnParts; ++o)
        mh = fmaxf(mh, red[(s * kAttnParts + ((part + o) % kAttnParts)) * kAttnTile + row]);
      const float mt = mh * cq;                                  // the tile's row maximum, base 2
      // the P buffer of this tile is free once PV_{j-2} has completed
      if (j >= 2 && !wait_warp(&pv_done[s], ((j - 2) >> 1) & 1)) { ok = false; break; }
      // Each row decides for itself whether its maximum moves (both warps of the pair
      // decide alike), but the TMEM loads and stores of a rescale are warp-wide
      // (.sync.aligned): the warp rescales when any of its rows needs it, the other
      // rows with factor 1.  Part p rescales O columns 32 p .. 32 p + 31, part 0
      // also the row-sum block 128..143.
      const bool move = mt > m_use + kLazyRescale;
      if (j >= 1 && __any_sync(0xffffffffu, move)) {
        // O holds PV_0 .. PV_{j-1}: wait for the last of them, then scale O in TMEM
        if (!wait_warp(&pv_done[s ^ 1], ((j - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const float f = move ? ex2(m_use - mt) : 1.0f;
        {
          uint32_t ov[32];
          tmem_ld32(t_o + lane_addr + 32 * part, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st32(t_o + lane_addr + 32 * part, ov);
        }
        if (part == 0) {
          uint32_t ov[16];   // columns 128..143: the row sum and the unused rest
          tmem_ld16(t_o + lane_addr + kAttnDim, ov);
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
          tmem_st16(t_o + lane_addr + kAttnDim, ov);
        }
        tmem_wait_st();
      }
      if (move) m_use = mt;
      // P = 2^(u cq - m) as fp16 into this part of the tile's P buffer (row = query;
      // keys 0..63 in the first 16 KB half, 64..127 in the second, 128-byte swizzle);
      // masked keys get P = 0; the P.V MMA's ones column sums it
      unsigned char* prow = smem + kPOff + s * 32768 + (part >> 1) * 16384 + row * 128;
      const int c8_0 = (part & 1) * 4;   // first 16-byte chunk of this part in the row
      const float nm = -m_use;
      auto probs = [&](auto full_tile) {
#pragma unroll
        for (int c8 = 0; c8 < kAttnPartKeys / 8; ++c8) {
          uint32_t packed[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const int col = 8 * c8 + 2 * e2;
            float p0 = ex2(fmaf(__uint_as_float(sreg[col]), cq, nm));
            float p1 = ex2(fmaf(__uint_as_float(sreg[col + 1]), cq, nm));
            if (!decltype(full_tile)::value) {
              p0 = col < nvalid ? p0 : 0.f;
              p1 = col + 1 < nvalid ? p1 : 0.f;
            }
            const __half2 hp = __floats2half2_rn(p0, p1);
            packed[e2] = *reinterpret_cast<const uint32_t*>(&hp);
          }
          *reinterpret_cast<uint4*>(prow + (((c8_0 + c8) ^ (row & 7)) << 4)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      };
      if (full) probs(std::true_type{});
      else probs(std::false_type{});
      fence_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[s]);
    }
    // O / l -> bf16: this warp's 32 output channels of its query rows
    if (ok && wait_warp(o_done, 0)) {
      tc_fence_after();
      uint32_t lv[16];
      tmem_ld16(t_o + lane_addr + kAttnDim, lv);
      const float l = __uint_as_float(lv[0]);
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      uint16_t* orow = args.o + (int64_t)qrow * args.ldo + h * kAttnDim + 32 * part;
      {
        const int c = 0;
        uint32_t ov[32];
        tmem_ld32(t_o + lane_addr + 32 * part, ov);
        tmem_wait_ld();
        if (qrow < args.Tq) {
#pragma unroll
          for (int e8 = 0; e8 < 4; ++e8) {
            uint32_t w[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              const int e = 8 * e8 + 2 * e2;
              const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(ov[e]) * inv_l,
                                                             __uint_as_float(ov[e + 1]) * inv_l);
              w[e2] = *reinterpret_cast<const uint32_t*>(&b);
            }
            *reinterpret_cast<uint4*>(orow + 32 * c + 8 * e8) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
int64_t attn_workspace_bytes(int64_t Tk, int64_t H) {
  const int64_t nchunks = (Tk + kColsumChunk - 1) / kColsumChunk;
  return (nchunks + 1) * H * kAttnDim * (int64_t)sizeof(double);
}

cudaError_t launch_attn_quant(const uint16_t* q, int64_t ldq, const uint16_t* k, int64_t ldk, const uint16_t* v,
                              int64_t ldv, int Tq, int Tk, int H, int8_t* qc, float* sq, int8_t* kc, float* sk,
                              void* vt, int64_t tkp, void* work, cudaStream_t st) {
  const int nchunks = (Tk + kColsumChunk - 1) / kColsumChunk;
  double* partial = static_cast<double*>(work);
  double* mean = partial + (int64_t)nchunks * H * kAttnDim;
  attn_key_colsum_kernel<<<dim3(nchunks, H), kAttnDim, 0, st>>>(k, ldk, Tk, H, partial);
  attn_key_mean_kernel<<<H, kAttnDim, 0, st>>>(partial, nchunks, Tk, H, mean);
  const int64_t units = ((int64_t)Tq + Tk) * H;
  attn_quant_kernel<<<(unsigned)((units + 7) / 8), 256, 0, st>>>(q, ldq, k, ldk, Tq, Tk, H, mean, qc, sq, kc, sk,
                                                                 tkp);
  attn_vt_kernel<<<dim3((unsigned)((tkp + 63) / 64), H), 256, 0, st>>>(v, ldv, Tk, H, static_cast<__half*>(vt),
                                                                       tkp);
  return cudaGetLastError();
}

cudaError_t launch_attn_int8(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const CUtensorMap& tm_sk, const float* sq, int Tq, int Tk, int H, uint16_t* o,
                             int64_t ldo, cudaStream_t st) {
  AttnArgs a{sq, Tq, Tk, H, o, ldo};
  cudaError_t e = cudaFuncSetAttribute(attn_int8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmem);
  if (e != cudaSuccess) return e;
  attn_int8_kernel<<<dim3((Tq + kAttnTile - 1) / kAttnTile, H), kAttnThreads, kAttnSmem, st>>>(tm_q, tm_k, tm_v,
                                                                                              tm_sk, a);
  return cudaGetLastError();
}

}  // namespace rbd
