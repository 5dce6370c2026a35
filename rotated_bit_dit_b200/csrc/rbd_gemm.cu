// Low-bit GEMM with fused dequant / low-rank / gate epilogue on the sm_100a
// tcgen05 tensor cores.
//
// Method: W4A4 (packed INT4 weights x INT4 activation codes) or W8A8 (per-row
// INT8 weights x INT8 codes), int32 accumulation, dequant scales and the
// epilogue of "Krea 2 Turbo OrbitQuant W4A4", section "Fused transformer"
// (sigmoid gate in the grouped Q|K|V|gate GEMM epilogue, gated residual
// updates in the GEMM epilogues), plus the parallel low-rank branch of
// "Krea-2-SVDQuant-ComfyUI", section "LoRA".
//
// Orientation ("swap AB"): the MMA's M side is 128 output features (weights),
// its N side 128 tokens, so TMEM lane = output feature and TMEM column = token.
//   - W4A4: weights are widened from packed nibbles to INT8 in registers by
//     four converter warps and written straight into tensor memory with
//     tcgen05.st; the MMA reads A from TMEM (tcgen05 has no INT4 kind).  A
//     nibble is placed in the high half of its byte (value 16*q, exact), so
//     widening is a shift, two masks and two byte permutes per 8 codes; the
//     accumulator is 16 * acc and the epilogue folds the 1/16 into the scale.
//   - W8A8: weights come by TMA into shared memory; both operands from smem.
//   - Activation codes (int8) always come by TMA (128-byte swizzle).
// Accumulation segments: one segment per tile (row scales) or one per 64-wide
// K block (group scales).  Two 128-column int32 partial buffers in TMEM
// alternate, so the tensor core fills one while the epilogue drains the
// other.  In group mode each partial starts from the bit pattern of
// 12582912.0f (1.5 * 2^23): the int32 result reinterpreted as float is then
// exactly 12582912 + 16*acc, and fma(f, a, -12582912*a) yields the correctly
// rounded 16*acc*a with no int->float conversion.  (a is the weight scale
// rounded to 22 significant bits so that 12582912*a is exact; the relative
// change of the scale is below 2^-22.)
#include "rbd_common.cuh"
#include "rbd_internal.cuh"

namespace rbd {

namespace {

constexpr int kTileF = 128;    // output features per tile (TMEM lanes)
constexpr int kTileT = 128;    // tokens per tile (MMA N)
constexpr int kBK = 128;       // K per pipeline stage (one 128-byte swizzle row of codes)
constexpr int kStages = 4;
constexpr int kThreads = 448;  // 14 warps
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpConv0 = 2, kWarpEpi0 = 6;
constexpr int kEpiThreads = 256;
constexpr uint32_t kMagicBits = 0x4B400000u;  // 12582912.0f
constexpr float kMagicF = 12582912.0f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColP0 = 0, kColA = 256, kColLR = 384;

__device__ __forceinline__ void named_bar_epi() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

}  // namespace

struct SmemLayout {
  uint32_t x_off, w_off, ld_off, l2_off, sx_off, sw_off, bar_off, total;
  int sx_stride, sw_stride;
};

__host__ __device__ inline SmemLayout smem_layout(bool w4, int r, int G) {
  SmemLayout L{};
  uint32_t off = 0;
  L.x_off = off;
  off += kStages * kTileT * kBK;
  L.w_off = off;
  if (!w4) off += kStages * kTileF * kBK;
  L.ld_off = off;
  off += kTileT * r * 2;
  L.l2_off = off;
  off += kTileF * r * 2;
  off = (off + 1023u) & ~1023u;
  L.sx_stride = kTileT + 4;
  L.sx_off = off;
  off += (uint32_t)G * L.sx_stride * 4;
  L.sw_stride = 0;
  L.sw_off = off;
  off = (off + 15u) & ~15u;
  L.bar_off = off;
  off += 32 * 8 + 16;
  L.total = off + 1024;  // slack for 1024-byte alignment of the base
  return L;
}

template <bool W4, bool G64, bool LR, bool DBG>
__global__ void __launch_bounds__(kThreads, 1)
    lowbit_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w8,
                       const __grid_constant__ CUtensorMap tm_ld, const __grid_constant__ CUtensorMap tm_l2,
                       const GemmArgs args) {
  extern __shared__ unsigned char smem_dyn[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023u) & ~uintptr_t(1023u));
  const SmemLayout L = smem_layout(W4, LR ? args.r : 0, args.G);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* full = bars;                 // [kStages]
  uint64_t* empty = bars + kStages;      // [kStages]
  uint64_t* pfull = bars + 2 * kStages;  // [2]
  uint64_t* pempty = pfull + 2;          // [2]
  uint64_t* lrfull = pempty + 2;
  uint64_t* lrempty = lrfull + 1;
  uint64_t* lrsfull = lrempty + 1;
  uint64_t* lrsempty = lrsfull + 1;
  uint64_t* drain = lrsempty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (warp == kWarpProducer && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], W4 ? 1 + 4 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], kEpiThreads / 32);
    }
    mbar_init(lrfull, 1);
    mbar_init(lrempty, kEpiThreads / 32);
    mbar_init(lrsfull, 1);
    mbar_init(lrsempty, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    if (!W4) tma_prefetch_desc(&tm_w8);
    if (LR) {
      tma_prefetch_desc(&tm_ld);
      tma_prefetch_desc(&tm_l2);
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int K = args.K;
  const int nks = K / kBK;
  const uint32_t x_stage_bytes = kTileT * kBK;

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, lr_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        const int mt = t % args.num_m_tiles, nt = t / args.num_m_tiles;
        const int m0 = mt * kTileT, n0 = nt * kTileF;
        if (LR) {
          if (!mbar_wait(lrsempty, lr_phase ^ 1)) { ok = false; break; }
          const uint32_t bytes = (uint32_t)(kTileT + kTileF) * args.r * 2;
          mbar_arrive_expect_tx(lrsfull, bytes);
          tma_load_2d(smem + L.ld_off, &tm_ld, lrsfull, 0, m0);
          tma_load_2d(smem + L.l2_off, &tm_l2, lrsfull, 0, n0);
          lr_phase ^= 1;
        }
        for (int ks = 0; ks < nks; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], W4 ? x_stage_bytes : 2 * x_stage_bytes);
          tma_load_2d(smem + L.x_off + stage * x_stage_bytes, &tm_x, &full[stage], ks * kBK, m0);
          if (!W4) tma_load_2d(smem + L.w_off + stage * x_stage_bytes, &tm_w8, &full[stage], ks * kBK, n0);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // let bulk copies already in flight land before the CTA can exit
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {}
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t idesc = idesc_i8(kTileF, kTileT);
      const uint32_t idesc_lr = idesc_bf16(kTileF, kTileT);
      int stage = 0;
      uint32_t phase = 0, lr_phase = 0;
      uint32_t pb = 0, pph[2] = {0, 0};
      bool ok = true;
      const int seg = args.seg;
      const uint32_t lr_row_bytes = (uint32_t)args.r * 2;
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        if (LR) {
          if (!mbar_wait(lrsfull, lr_phase) || !mbar_wait(lrempty, lr_phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + L.l2_off), b0 = smem_u32(smem + L.ld_off);
          for (int kk = 0; kk < args.r / 16; ++kk) {
            mma_bf16_ss(tmem + kColLR, smem_desc_kmajor(a0 + kk * 32, lr_row_bytes),
                        smem_desc_kmajor(b0 + kk * 32, lr_row_bytes), idesc_lr, kk > 0 ? 1u : 0u);
          }
          tc_commit(lrfull);
          tc_commit(lrsempty);
          lr_phase ^= 1;
        }
        for (int ks = 0; ks < nks && ok; ++ks) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t xs = smem_u32(smem + L.x_off + stage * x_stage_bytes);
          const uint64_t bdesc = smem_desc_kmajor(xs, 128);
          uint64_t adesc = 0;
          if (!W4) adesc = smem_desc_kmajor(smem_u32(smem + L.w_off + stage * x_stage_bytes), 128);
#pragma unroll
          for (int kk = 0; kk < kBK / 32; ++kk) {
            const int kpos = ks * kBK + kk * 32;
            if (kpos % seg == 0) {
              if (!mbar_wait(&pempty[pb], pph[pb])) { ok = false; break; }
              pph[pb] ^= 1;
              tc_fence_after();
            }
            const uint32_t acc = G64 ? 1u : (kpos % seg != 0 ? 1u : 0u);
            const uint32_t d = tmem + kColP0 + pb * 128;
            if (W4) {
              mma_i8_ts(d, tmem + kColA + stage * 32 + kk * 8, bdesc + (uint64_t)(kk * 2), idesc, acc);
            } else {
              mma_i8_ss(d, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), idesc, acc);
            }
            if ((kpos + 32) % seg == 0) {
              tc_commit(&pfull[pb]);
              pb ^= 1;
            }
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
      // make sure every issued MMA has completed before TMEM can be released
      tc_commit(drain);
      mbar_wait(drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp < kWarpEpi0) {
    // ------------------------------------------------------------ INT4 -> INT8 converters
    // Each thread owns one weight row of the tile (its TMEM lane).  Packed bytes
    // are fetched two stages ahead of the stage being widened.
    if (W4) {
      const uint32_t q = warp & 3u;
      const uint32_t lane_base = (32u * q) << 16;
      const int half_k = K / 2;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        const int nt = t / args.num_m_tiles;
        const int n = nt * kTileF + 32 * q + lane;
        const uint4* wrow = reinterpret_cast<const uint4*>(args.w4 + (int64_t)n * half_k);
        uint4 c0[4], c1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) c0[i] = __ldg(wrow + i);
        if (nks > 1) {
#pragma unroll
          for (int i = 0; i < 4; ++i) c1[i] = __ldg(wrow + 4 + i);
        }
        for (int ks = 0; ks < nks; ++ks) {
          uint4 c2[4];
          if (ks + 2 < nks) {
#pragma unroll
            for (int i = 0; i < 4; ++i) c2[i] = __ldg(wrow + (ks + 2) * 4 + i);
          }
          uint32_t outw[32];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t pw[4] = {c0[i].x, c0[i].y, c0[i].z, c0[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t lo = (pw[j] << 4) & 0xF0F0F0F0u;  // even k, as 16*q
              const uint32_t hi = pw[j] & 0xF0F0F0F0u;         // odd k, as 16*q
              outw[8 * i + 2 * j] = __byte_perm(lo, hi, 0x5140);
              outw[8 * i + 2 * j + 1] = __byte_perm(lo, hi, 0x7362);
            }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            c0[i] = c1[i];
            c1[i] = c2[i];
          }
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          tc_fence_after();
          tmem_st32(tmem + lane_base + kColA + stage * 32, outw);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Thread = one output feature (TMEM lane) x 64 tokens (TMEM columns).
    const uint32_t q = warp & 3u;
    const uint32_t h = (warp - kWarpEpi0) >> 2;   // token half of the tile
    const uint32_t lane_base = (32u * q) << 16;
    const int etid = threadIdx.x - kWarpEpi0 * 32;  // 0..255
    const int G = args.G;
    float* sx_s = reinterpret_cast<float*>(smem + L.sx_off);
    const int fr = 32 * q + lane;  // feature row of this thread in the tile

    // partial buffers start released; in group mode they hold the magic pattern
    if (G64) {
      for (int b = 0; b < 2; ++b)
        for (int c = 0; c < 4; ++c) tmem_fill16(tmem + lane_base + kColP0 + b * 128 + 64 * h + 16 * c, kMagicBits);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&pempty[0]);
      mbar_arrive(&pempty[1]);
      if (LR) mbar_arrive(lrempty);
    }

    uint32_t pb = 0, pph[2] = {0, 0}, lr_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x) {
      const int mt = t % args.num_m_tiles, nt = t / args.num_m_tiles;
      const int m0 = mt * kTileT, n0 = nt * kTileF;
      // stage the tile's activation scales in shared memory, group-major
      named_bar_epi();
      for (int e = etid; e < kTileT * G; e += kEpiThreads) {
        const int tk = e / G, g = e % G;
        const int64_t m = (int64_t)m0 + tk;
        sx_s[g * L.sx_stride + tk] = m < args.M ? __ldg(args.sx + m * G + g) : 0.f;
      }
      named_bar_epi();

      const int n = n0 + fr;
      const float* swrow = args.sw + (int64_t)n * G;
      float sw_next = __ldg(swrow);
      float2 y[32];
      const float bias = args.bias ? __uint_as_float((uint32_t)__ldg(args.bias + n) << 16) : 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) y[j] = make_float2(bias, bias);
      if (LR && ok) {
        if (!mbar_wait(lrfull, lr_phase)) ok = false;
        lr_phase ^= 1;
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + kColLR + 64 * h + 32 * c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              y[16 * c + j].x += __uint_as_float(v[2 * j]);
              y[16 * c + j].y += __uint_as_float(v[2 * j + 1]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(lrempty);
        }
      }
      for (int g = 0; g < G && ok; ++g) {
        const float sw_g = sw_next;
        if (g + 1 < G) sw_next = __ldg(swrow + g + 1);
        if (!mbar_wait(&pfull[pb], pph[pb])) { ok = false; break; }
        pph[pb] ^= 1;
        tc_fence_after();
        const float4* sxg = reinterpret_cast<const float4*>(sx_s + g * L.sx_stride + 64 * h);
        float a = sw_g * args.acc_scale;
        float cneg = 0.f;
        if (G64) {
          a = __uint_as_float((__float_as_uint(a) + 2u) & ~3u);   // 22 significant bits
          cneg = -kMagicF * a;                                       // exact
        }
        const float2 a2 = make_float2(a, a);
        const float2 c2 = make_float2(cneg, cneg);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          const uint32_t taddr = tmem + lane_base + kColP0 + pb * 128 + 64 * h + 32 * c;
          tmem_ld32(taddr, v);
          if (DBG) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int64_t m = (int64_t)m0 + 64 * h + 32 * c + j;
              if (m < args.M) {
                const int32_t raw = G64 ? (int32_t)(v[j] - kMagicBits) : (int32_t)v[j];
                const int32_t accv = W4 ? (raw >> 4) : raw;
                const int64_t idx = (G64 ? (int64_t)g * args.M * args.N : 0) + m * args.N + n;
                args.acc_debug[idx] = accv;
              }
            }
          }
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 b4 = sxg[8 * c + j4];
            const float2 blo = make_float2(b4.x, b4.y), bhi = make_float2(b4.z, b4.w);
            float2& y0 = y[16 * c + 2 * j4];
            float2& y1 = y[16 * c + 2 * j4 + 1];
            if (G64) {
              const float2 f0 = make_float2(__uint_as_float(v[4 * j4]), __uint_as_float(v[4 * j4 + 1]));
              const float2 f1 = make_float2(__uint_as_float(v[4 * j4 + 2]), __uint_as_float(v[4 * j4 + 3]));
              y0 = __ffma2_rn(__ffma2_rn(f0, a2, c2), blo, y0);
              y1 = __ffma2_rn(__ffma2_rn(f1, a2, c2), bhi, y1);
            } else {
              const float2 f0 = make_float2((float)(int32_t)v[4 * j4], (float)(int32_t)v[4 * j4 + 1]);
              const float2 f1 = make_float2((float)(int32_t)v[4 * j4 + 2], (float)(int32_t)v[4 * j4 + 3]);
              y0 = __ffma2_rn(f0, __fmul2_rn(a2, blo), y0);
              y1 = __ffma2_rn(f1, __fmul2_rn(a2, bhi), y1);
            }
          }
          if (G64) {
            tmem_fill16(taddr, kMagicBits);
            tmem_fill16(taddr + 16, kMagicBits);
          }
        }
        if (G64) tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[pb]);
        pb ^= 1;
      }
      if (!ok) continue;  // keep the named barriers balanced; stop producing output
      // gate and store: thread (feature n) writes tokens m0 + 64h + j
      const bool sig = args.gate_mode == 1 && n >= args.gate_c0 && n < args.gate_c1;
      const float gv = args.gate_mode == 2 ? __uint_as_float((uint32_t)__ldg(args.gate + n) << 16) : 0.f;
      const int64_t mbase = (int64_t)m0 + 64 * h;
      uint16_t* yp = args.y + mbase * args.ldy + n;
      const uint16_t* rp = args.gate_mode == 2 ? args.residual + mbase * args.ldr + n : nullptr;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        if (mbase + j < args.M) {
          float o = (j & 1) ? y[j >> 1].y : y[j >> 1].x;
          if (sig) {
            o = 1.0f / (1.0f + __expf(-o));
          } else if (args.gate_mode == 2) {
            const float rres = __uint_as_float((uint32_t)rp[(int64_t)j * args.ldr] << 16);
            o = fmaf(gv, o, rres);
          }
          yp[(int64_t)j * args.ldy] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
        }
      }
    }
  }

  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------
cudaError_t launch_lowbit_gemm(bool w4, bool g64, const CUtensorMap& tm_x, const CUtensorMap& tm_w8,
                               const CUtensorMap& tm_ld, const CUtensorMap& tm_l2, const GemmArgs& a, int num_sms,
                               cudaStream_t st) {
  const bool lr = a.r > 0;
  const SmemLayout L = smem_layout(w4, a.r, a.G);
  if (L.total > 227u * 1024u) return cudaErrorInvalidConfiguration;
  const int grid = a.num_tiles < num_sms ? a.num_tiles : num_sms;
  const bool dbg = a.acc_debug != nullptr;
#define RBD_GEMM_CASE(W, G, R, D)                                                                     \
  if (w4 == W && g64 == G && lr == R && dbg == D) {                                                  \
    auto kern = lowbit_gemm_kernel<W, G, R, D>;                                                      \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total); \
    if (e != cudaSuccess) return e;                                                                  \
    kern<<<grid, kThreads, L.total, st>>>(tm_x, tm_w8, tm_ld, tm_l2, a);                            \
    return cudaGetLastError();                                                                       \
  }
#define RBD_GEMM_CASES(W, G, R) RBD_GEMM_CASE(W, G, R, false) RBD_GEMM_CASE(W, G, R, true)
  RBD_GEMM_CASES(true, true, true)
  RBD_GEMM_CASES(true, true, false)
  RBD_GEMM_CASES(true, false, true)
  RBD_GEMM_CASES(true, false, false)
  RBD_GEMM_CASES(false, true, true)
  RBD_GEMM_CASES(false, true, false)
  RBD_GEMM_CASES(false, false, true)
  RBD_GEMM_CASES(false, false, false)
#undef RBD_GEMM_CASES
#undef RBD_GEMM_CASE
  return cudaErrorInvalidValue;
}

uint32_t gemm_smem_bytes(bool w4, int r, int G) { return smem_layout(w4, r, G).total; }

}  // namespace rbd
