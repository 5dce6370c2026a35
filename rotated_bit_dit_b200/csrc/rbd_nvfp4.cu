// NVFP4 variant of the rotated low-bit linear layer: group-256 rotation, then
// two-level FP4 quantisation (E2M1 values, an E4M3 scale per 16 elements and
// one float32 tensor scale), and a GEMM on the block-scaled FP4 tensor cores
// (tcgen05.mma kind::mxf4nvf4, 16-element scale blocks, float32 accumulation).
//
// Method: "Krea 2 Turbo Nunchaku Lite INT4 r32", Benchmark (the NVFP4 build of
// the same rotated layer on Blackwell block-scaled tensor cores).  The pages
// give the format only as "E4M3 scale per 16 elements"; the float32 tensor
// scale gs = amax(tensor) / (6 * 448) keeps the E4M3 block scales in their
// normal range:
//   bs = E4M3_RN_satfinite(amax(block16) / (6 * gs))
//   q  = E2M1_RN_satfinite(x / (bs * gs))
// with every division and product an IEEE float32 operation.
#include "rbd_common.cuh"
#include "rbd_internal.cuh"
#include "rbd_rotate.cuh"

namespace rbd {

namespace {

constexpr int kNvTeam = 16;   // threads per 256-block

// E4M3 (sign 0) byte -> float, exact.
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0.001953125f;
}

// float -> E4M3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
  uint16_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}" : "=h"(r) : "f"(0.f), "f"(v));
  return r & 0xFFu;
}

// 8 floats -> 8 E2M1 codes packed little-endian (element 0 in the low nibble).
__device__ __forceinline__ uint32_t f32x8_to_e2m1(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

}  // namespace

// Block-scale layout read by the block-scaled MMA ("tile-interleaved"): rows are
// grouped in tiles of 128 and scale columns (one per 16 elements of K) in steps
// of 4 (64 elements); each (row tile, K step) is a 512-byte atom of 32 lines x
// 16 bytes, line r holding the 4 scales of rows r, r+32, r+64, r+96 of the tile.
// This is the layout `tcgen05.cp .32x128b.warpx4` turns into the TMEM scale
// operand; a buffer holds ceil(rows/128)*128 rows.
__host__ __device__ inline int64_t nvfp4_scale_offset(int64_t row, int64_t col, int64_t K) {
  const int64_t mt = row >> 7, rr = row & 127, ks = col >> 2;
  return ((mt * (K / 64) + ks) * 32 + (rr & 31)) * 16 + (rr >> 5) * 4 + (col & 3);
}

namespace {

// Swizzle of a team's 256-float transpose buffer (position p = 16 b + e stored
// at 16 b + (e ^ b)): conflict-free for "thread tau writes tau + 16 i" and for
// "thread tau reads 16 tau + e".
__device__ __forceinline__ int tr_idx(int p) { return (p & ~15) | ((p ^ (p >> 4)) & 15); }

}  // namespace

// PASS 0: rotate, reduce max |x| over the tensor into *amax_bits (the float's
//         bit pattern; atomicMax orders non-negative floats correctly).
// PASS 1: rotate, quantise with the tensor scale derived from *amax_bits.
// One CTA handles `rows` rows; each row uses 16 * teams threads; team `tm`
// processes 256-blocks g = tm, tm + teams, ... (at most CMAX).
template <bool ROT, int PASS, int CMAX>
__global__ void __launch_bounds__(256) nvfp4_quant_kernel(const uint16_t* __restrict__ x, int64_t M, int K,
                                                          int64_t ldx, int teams, int rows, uint32_t* amax_bits,
                                                          uint8_t* __restrict__ codes, uint8_t* __restrict__ bscale,
                                                          float* __restrict__ gscale) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* xbuf = reinterpret_cast<double*>(smem_raw);   // one 256-double buffer per team
  __shared__ float red[8];

  const int T = kNvTeam * teams;
  const int tid = threadIdx.x;
  const int rloc = tid / T;
  const int t_in_row = tid % T;
  const int team = t_in_row / kNvTeam;
  const int tau = t_in_row % kNvTeam;
  const int64_t m = (int64_t)blockIdx.x * rows + rloc;
  const bool row_ok = (rloc < rows) && (m < M);
  const int G = K >> 8;
  double* tb = xbuf + (size_t)(tid / kNvTeam) * 256;
  float* tf = reinterpret_cast<float*>(tb);

  float gs = 0.f, six_gs = 0.f;
  if (PASS == 1) {
    const float amax_t = __uint_as_float(*reinterpret_cast<volatile uint32_t*>(amax_bits));
    gs = __fdiv_rn(amax_t, 2688.0f);            // 6 * 448
    six_gs = __fmul_rn(6.0f, gs);
    if (blockIdx.x == 0 && tid == 0) *gscale = gs;
  }

  float amax_all = 0.f;
#pragma unroll
  for (int c = 0; c < CMAX; ++c) {
    const int g = team + c * teams;
    const bool ok = row_ok && g < G;
    uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
    if (ok) {
      const uint4* src = reinterpret_cast<const uint4*>(x + m * ldx + (int64_t)g * 256 + tau * 16);
      lo = __ldg(src);
      hi = __ldg(src + 1);
    }
    // v: the 16 rotated values of 16-element block `tau` of this 256-block
    float v[16];
    if constexpr (ROT) {
      float xr[16];
      rotate256_team(lo, hi, tau, tb, xr);      // xr[i] = position tau + 16 i
#pragma unroll
      for (int i = 0; i < 16; ++i) tf[tr_idx(tau + 16 * i)] = xr[i];
      __syncwarp();
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = tf[tr_idx(16 * tau + e)];
      __syncwarp();
    } else {
      load16_f32(lo, hi, v);
    }
    float amax_b = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) amax_b = fmaxf(amax_b, fabsf(v[e]));
    if (PASS == 0) {
      amax_all = fmaxf(amax_all, amax_b);
    } else if (ok) {
      const float ratio_b = six_gs > 0.f ? __fdiv_rn(amax_b, six_gs) : 0.f;
      const uint32_t bs = f32_to_e4m3(ratio_b);
      const float denom = __fmul_rn(e4m3_to_f32(bs), gs);
      float r[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = denom > 0.f ? __fdiv_rn(v[e], denom) : 0.f;
      const uint32_t w0 = f32x8_to_e2m1(r), w1 = f32x8_to_e2m1(r + 8);
      *reinterpret_cast<uint2*>(codes + m * (int64_t)(K / 2) + (int64_t)g * 128 + tau * 8) = make_uint2(w0, w1);
      bscale[nvfp4_scale_offset(m, (int64_t)g * 16 + tau, K)] = static_cast<uint8_t>(bs);
    }
  }
  if (PASS == 0) {
    for (int off = 16; off > 0; off >>= 1) amax_all = fmaxf(amax_all, __shfl_xor_sync(0xffffffffu, amax_all, off));
    if ((tid & 31) == 0) red[tid >> 5] = amax_all;
    __syncthreads();
    if (tid == 0) {
      float mx = 0.f;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
      atomicMax(amax_bits, __float_as_uint(mx));
    }
  }
}

// Clears the tensor-amax slot before pass 0.
__global__ void nvfp4_clear_kernel(uint32_t* amax_bits) { *amax_bits = 0u; }

cudaError_t launch_nvfp4_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, bool rot, uint32_t* work,
                               uint8_t* codes, uint8_t* bscale, float* gscale, cudaStream_t st) {
  const int G = static_cast<int>(K / 256);
  int teams = G < 8 ? G : 8;                  // up to 128 threads per row
  while (G % teams) --teams;                  // whole chunks per team
  const int cmax = G / teams;
  const int T = kNvTeam * teams;
  const int rows = 256 / T > 0 ? 256 / T : 1;
  const int threads = rows * T;
  const int64_t blocks = (M + rows - 1) / rows;
  const size_t smem = (size_t)(threads / kNvTeam) * 256 * sizeof(double);
  nvfp4_clear_kernel<<<1, 1, 0, st>>>(work);
#define RBD_NV_CASE(R, C)                                                                                       \
  if (rot == R && cmax == C) {                                                                                  \
    nvfp4_quant_kernel<R, 0, C><<<(unsigned)blocks, threads, smem, st>>>(x, M, (int)K, ldx, teams, rows, work,    \
                                                                      codes, bscale, gscale);                  \
    nvfp4_quant_kernel<R, 1, C><<<(unsigned)blocks, threads, smem, st>>>(x, M, (int)K, ldx, teams, rows, work,    \
                                                                      codes, bscale, gscale);                  \
    return cudaGetLastError();                                                                                  \
  }
  RBD_NV_CASE(true, 1) RBD_NV_CASE(true, 2) RBD_NV_CASE(true, 3) RBD_NV_CASE(true, 4) RBD_NV_CASE(true, 6)
  RBD_NV_CASE(true, 8)
  RBD_NV_CASE(false, 1) RBD_NV_CASE(false, 2) RBD_NV_CASE(false, 3) RBD_NV_CASE(false, 4) RBD_NV_CASE(false, 6)
#undef RBD_NV_CASE
  return cudaErrorInvalidValue;
}


// ---------------------------------------------------------------------------
// Block-scaled FP4 GEMM.  One persistent CTA per SM; tile = 128 output features
// (MMA M, TMEM lanes) x 128 tokens (MMA N, TMEM columns); stages of 256 K (128
// bytes of E2M1 per row, 128-byte swizzled).  Per stage the producer brings the
// two operand tiles by TMA and the two scale tiles (4 atoms of 512 bytes each,
// contiguous in the tile-interleaved layout) by bulk copy; the MMA thread
// copies the scales into TMEM with tcgen05.cp and issues four K = 64 MMAs.  The
// float32 accumulator is double-buffered in TMEM so the epilogue of one tile
// overlaps the MMAs of the next.  Epilogue: y = acc * gs_x * gs_w + bias, then
// the sigmoid gate or the gated residual, one bf16 rounding.
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issuer, 4..11 epilogue.
// ---------------------------------------------------------------------------
namespace {
constexpr int kNvThreads = 384;
constexpr int kNvWarpEpi0 = 4;
constexpr int kNvTile = 128;                  // features and tokens per tile
constexpr int kNvBK = 256;                    // K elements per stage
constexpr uint32_t kNvOpBytes = 128 * 128;    // one operand stage
constexpr uint32_t kNvSfBytes = 4 * 512;      // one scale stage (4 K steps)
// pipeline stages: 4 with the low-rank branch (its tiles take the rest of
// shared memory and its accumulator TMEM columns 384..511), 6 without
__host__ __device__ constexpr int nv_stages(bool lr) { return lr ? 4 : 6; }
constexpr uint32_t kNvStageBytes = 2 * kNvOpBytes + 2 * kNvSfBytes;
constexpr uint32_t kNvLrBytes = 2 * 128 * 128;  // low-rank tiles: l2t [128 x r] and ld [128 x r], r <= 64
__host__ __device__ constexpr uint32_t nv_smem_bytes(bool lr) {
  return nv_stages(lr) * kNvStageBytes + (lr ? kNvLrBytes : 0u) + 1024 + 256;
}
constexpr uint32_t kNvAccCols = 2 * kNvTile;  // two accumulator buffers
constexpr uint32_t kNvLrCol = 384;            // low-rank accumulator (after the scale regions)
}  // namespace

template <bool LR>
__global__ void __launch_bounds__(kNvThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_ld, const __grid_constant__ CUtensorMap tm_l2,
                      const NvArgs args) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023u) & ~uintptr_t(1023u));
  // stage s: A (weights) | B (tokens) | SFA | SFB
  // low-rank tiles after the stages: l2t rows (A side) then ld rows (B side)
  constexpr int kNvStages = nv_stages(LR);
  unsigned char* lr_a = smem + kNvStages * kNvStageBytes;
  unsigned char* lr_b = lr_a + kNvLrBytes / 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kNvStages * kNvStageBytes + (LR ? kNvLrBytes : 0u));
  uint64_t* full = bars;
  uint64_t* empty = bars + kNvStages;
  uint64_t* tfull = bars + 2 * kNvStages;    // [2]
  uint64_t* tempty = tfull + 2;              // [2]
  uint64_t* drain = tempty + 2;
  uint64_t* lrsfull = drain + 1;             // low-rank tiles landed in shared memory
  uint64_t* lrsempty = lrsfull + 1;          // low-rank MMAs done with them
  uint64_t* lrtempty = lrsempty + 1;         // epilogue has read the low-rank accumulator
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(lrtempty + 1);
  const int R = LR ? args.r : 0;
  const uint32_t warp = warp_id(), lane = lane_id();
  const int nks = args.K / kNvBK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kNvStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], (kNvThreads / 32) - kNvWarpEpi0);
    }
    mbar_init(drain, 1);
    mbar_init(lrsfull, 1);
    mbar_init(lrsempty, 1);
    mbar_init(lrtempty, (kNvThreads / 32) - kNvWarpEpi0);
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    if (R) {
      tma_prefetch_desc(&tm_ld);
      tma_prefetch_desc(&tm_l2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, lr_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        const int mt = t % args.num_m_tiles, nt = t / args.num_m_tiles;
        if (R) {
          // the tile's low-rank operands, consumed after its K loop
          if (!mbar_wait(lrsempty, lr_phase ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(lrsfull, 2u * kNvTile * (uint32_t)R * 2u);
          tma_load_2d(lr_a, &tm_l2, lrsfull, 0, nt * kNvTile);
          tma_load_2d(lr_b, &tm_ld, lrsfull, 0, mt * kNvTile);
          lr_phase ^= 1;
        }
        for (int ks = 0; ks < nks; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          unsigned char* st = smem + stage * kNvStageBytes;
          mbar_arrive_expect_tx(&full[stage], kNvStageBytes);
          tma_load_2d(st, &tm_w, &full[stage], ks * (kNvBK / 2), nt * kNvTile);
          tma_load_2d(st + kNvOpBytes, &tm_x, &full[stage], ks * (kNvBK / 2), mt * kNvTile);
          const int64_t atom0 = (int64_t)ks * (kNvBK / 64);
          bulk_load(st + 2 * kNvOpBytes, args.sfw + ((int64_t)nt * (args.K / 64) + atom0) * 512, kNvSfBytes,
                    &full[stage]);
          bulk_load(st + 2 * kNvOpBytes + kNvSfBytes, args.sfx + ((int64_t)mt * (args.K / 64) + atom0) * 512,
                    kNvSfBytes, &full[stage]);
          if (++stage == kNvStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {}
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (elect_one()) {
      const uint32_t idesc = idesc_nvf4(kNvTile, kNvTile);
      const uint32_t idesc_lr = idesc_bf16(kNvTile, kNvTile);
      const uint32_t lr_row_bytes = (uint32_t)R * 2u;
      int stage = 0;
      uint32_t phase = 0, tph = 0, lr_phase = 0;
      int ab = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[ab], ((tph >> ab) & 1u) ^ 1u)) { ok = false; break; }
        tph ^= 1u << ab;
        tc_fence_after();
        const uint32_t d = tmem + ab * kNvTile;
        for (int ks = 0; ks < nks; ++ks) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + stage * kNvStageBytes);
          const uint64_t adesc = smem_desc_kmajor(st, 128);
          const uint64_t bdesc = smem_desc_kmajor(st + kNvOpBytes, 128);
          const uint32_t sfa = tmem + kNvAccCols + 32u * stage, sfb = sfa + 16u;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tmem_cp_32x128b_x4(sfa + 4u * j, smem_desc_rows16(st + 2 * kNvOpBytes + 512u * j));
            tmem_cp_32x128b_x4(sfb + 4u * j, smem_desc_rows16(st + 2 * kNvOpBytes + kNvSfBytes + 512u * j));
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_nvf4_ss(d, adesc + 2 * j, bdesc + 2 * j, idesc, sfa + 4u * j, sfb + 4u * j, (ks | j) ? 1u : 0u);
          tc_commit(&empty[stage]);
          if (++stage == kNvStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (R) {
          // low-rank segment into its own accumulator; the tile's tfull commit
          // below covers these MMAs too
          if (!mbar_wait(lrsfull, lr_phase) || !mbar_wait(lrtempty, lr_phase ^ 1)) { ok = false; break; }
          lr_phase ^= 1;
          tc_fence_after();
          const uint32_t a0 = smem_u32(lr_a), b0 = smem_u32(lr_b);
          for (int kk = 0; kk < R / 16; ++kk)
            mma_bf16_ss(tmem + kNvLrCol, smem_desc_kmajor(a0 + kk * 32, lr_row_bytes),
                        smem_desc_kmajor(b0 + kk * 32, lr_row_bytes), idesc_lr, kk > 0 ? 1u : 0u);
          tc_commit(lrsempty);
        }
        tc_commit(&tfull[ab]);
        ab ^= 1;
      }
      tc_commit(drain);
      mbar_wait(drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp >= kNvWarpEpi0) {
    // ---------------------------------------------------------- epilogue
    const uint32_t q = warp & 3u, h = (warp - kNvWarpEpi0) >> 2;
    const uint32_t lane_base = (32u * q) << 16;
    const float gsc = __fmul_rn(__ldg(args.gsx), __ldg(args.gsw));
    uint32_t tph = 0;
    int ab = 0;
    for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x) {
      const int mt = t % args.num_m_tiles, nt = t / args.num_m_tiles;
      if (!mbar_wait(&tfull[ab], (tph >> ab) & 1u)) break;
      tph ^= 1u << ab;
      tc_fence_after();
      uint32_t v[4][16], vl[4][16];
      const uint32_t tb = tmem + lane_base + ab * kNvTile + 64u * h;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld16_async(tb + 16u * c, v[c]);
      if (R) {
        const uint32_t tl = tmem + lane_base + kNvLrCol + 64u * h;
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld16_async(tl + 16u * c, vl[c]);
      }
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_reg_fence(v[c]);
      if (R) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_reg_fence(vl[c]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[ab]);
        if (R) mbar_arrive(lrtempty);
      }
      ab ^= 1;

      const int n = nt * kNvTile + 32 * (int)q + (int)lane;
      const int64_t mbase = (int64_t)mt * kNvTile + 64 * h;
      const float bias = args.bias ? __uint_as_float((uint32_t)__ldg(args.bias + n) << 16) : 0.f;
      const bool sig = args.gate_mode == 1 && n >= args.gate_c0 && n < args.gate_c1;
      const float gv = args.gate_mode == 2 ? __uint_as_float((uint32_t)__ldg(args.gate + n) << 16) : 0.f;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const int64_t m = mbase + j;
        if (m < args.M) {
          float o = fmaf(__uint_as_float(v[j >> 4][j & 15]), gsc, bias);
          if (R) o += __uint_as_float(vl[j >> 4][j & 15]);
          if (args.gate_mode == 2) {
            // read-only path: each residual element is read once, by the thread that then
            // writes the output there, so the loads may run ahead of the stores
            o = fmaf(gv, o, __uint_as_float((uint32_t)__ldg(args.residual + m * args.ldr + n) << 16));
          } else if (sig) {
            o = __frcp_rn(1.0f + __expf(-o));
          }
          args.y[m * args.ldy + n] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

uint32_t nvfp4_gemm_smem_bytes() { return nv_smem_bytes(true); }

cudaError_t launch_nvfp4_gemm(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const CUtensorMap& tm_ld,
                              const CUtensorMap& tm_l2, const NvArgs& a, int num_sms, cudaStream_t st) {
  const int grid = a.num_tiles < num_sms ? a.num_tiles : num_sms;
  const bool lr = a.r != 0;
  auto kern = lr ? nvfp4_gemm_kernel<true> : nvfp4_gemm_kernel<false>;
  const uint32_t smem = nv_smem_bytes(lr);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kNvThreads, smem, st>>>(tm_x, tm_w, tm_ld, tm_l2, a);
  return cudaGetLastError();
}

}  // namespace rbd
