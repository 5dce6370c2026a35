// Small-token rotated low-bit linear: the same product and epilogue as the
// tiled tcgen05 kernel (rbd_gemm.cu), for token counts up to kSkinnyMaxM.
//
// With a handful of tokens (a decode-style call, or the last slice of a
// batch) the layer is a stream of the packed weights: 0.5 byte per weight
// against a few bytes of activations, so HBM bandwidth bounds it and the
// tensor-core rate hardly matters.  The tiled kernel spends a 128-token tile,
// a TMEM round trip and a full promotion per 64-wide group there, and only
// N/128 CTAs work.  This kernel instead
//   - gives each CTA 16 output features and splits K across its 8 warps
//     (N/16 CTAs: 192 for N = 3072), so every SM streams weights;
//   - feeds each warp from its own cp.async ring of 64-wide K groups (weights,
//     activation codes and, with group scales, both scale columns), several
//     groups in flight, no block-wide barrier until the end;
//   - contracts each group with two warp-level m16n8k32 MMAs per 8 tokens:
//     s8 x s8 -> s32 (INT4 nibbles widened to 16 q as in the tiled kernel, or
//     INT8 weights), or e4m3 x e4m3 -> f32 for E4M3 activation codes (nibbles
//     widened to their E4M3 bytes; a 64-wide group partial is an integer of
//     magnitude <= 4096, exact in float32);
//   - promotes group partials in float32 per warp (group scales) or keeps
//     int32 (row scales), sums the 8 warps' partials through shared memory
//     and runs the epilogue (scales, bias, low-rank branch, gate) per output.
// The K positions of an MMA are assigned consistently on both operands: thread
// t of a quad holds group offsets 16 t .. 16 t + 15 in the A rows and in the B
// columns, so the contraction covers each group exactly once.
#include "rbd_common.cuh"
#include "rbd_internal.cuh"

namespace rbd {

namespace {

constexpr int kSkWarps = 8;
constexpr int kSkThreads = kSkWarps * 32;
constexpr int kSkRows = 16;   // output features per block (one m16 row block)

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(pred ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool pred) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(pred ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// D += A (16 x 32, row) * B (32 x 8, col), signed 8-bit operands, int32 accumulators.
__device__ __forceinline__ void mma_s8_16832(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// The same shape with E4M3 operands and float32 accumulators.
__device__ __forceinline__ void mma_e4m3_16832(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Eight packed nibbles (code k in bits 4k..4k+3) -> bytes 16 q, codes 0-3 in o0
// and 4-7 in o1, in order (exact int8 values; the product carries a factor 16).
__device__ __forceinline__ void nibbles_to_16q(uint32_t pw, uint32_t& o0, uint32_t& o1) {
  const uint32_t lo = (pw << 4) & 0xF0F0F0F0u;   // even codes
  const uint32_t hi = pw & 0xF0F0F0F0u;          // odd codes
  o0 = prmt(lo, hi, 0x5140u);
  o1 = prmt(lo, hi, 0x7362u);
}

// One ring stage: the 64-wide K group g of the block's 16 weight rows, of the
// MP = 8 MT token rows (zero past M) and, with group scales, their scales.
template <bool W4, bool G64, int MT>
struct SkStage {
  static constexpr int MP = 8 * MT;
  static constexpr int kW = kSkRows * (W4 ? 32 : 64);
  static constexpr int kX = MP * 64;
  static constexpr int kSx = G64 ? MP * 4 : 0;
  static constexpr int kSw = G64 ? kSkRows * 4 : 0;
  static constexpr int bytes = kW + kX + kSx + kSw;   // a multiple of 16
  static constexpr int stages = MT <= 4 ? 4 : 2;
  static constexpr uint32_t smem = kSkWarps * stages * bytes;
};

template <bool W4, bool G64, bool F8, int MT>
__global__ void __launch_bounds__(kSkThreads) skinny_gemm_kernel(const GemmArgs args) {
  using St = SkStage<W4, G64, MT>;
  constexpr int MP = St::MP, S = St::stages;
  constexpr int MPP = MP + 1;   // padded row of the reduction buffer
  extern __shared__ __align__(16) unsigned char sk_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;   // MMA fragment row group and thread in quad
  const int n0 = blockIdx.x * kSkRows;
  const int M = args.M, N = args.N, K = args.K, G = args.G;
  const int NG = K / 64;
  const int gb = warp * NG / kSkWarps, ng = (warp + 1) * NG / kSkWarps - gb;
  unsigned char* ring = sk_smem + warp * S * St::bytes;
  const uint32_t ring_s = smem_u32(ring);
  const bool dbg = args.acc_debug != nullptr;

  // This warp's share of the block's weight rows (one contiguous range per row)
  // goes to L2 at once, before waiting for the preceding kernel: the weights are
  // not its output, and the whole stream is then in flight instead of a ring's
  // worth.  Everything else (codes, scales, outputs) is touched after the wait.
  if (lane < kSkRows && ng > 0) {
    const int64_t row_bytes = W4 ? K / 2 : K;
    const int gbytes = W4 ? 32 : 64;
    const uint8_t* wrow = (W4 ? args.w4 : reinterpret_cast<const uint8_t*>(args.w8)) +
                          (int64_t)(n0 + lane) * row_bytes + (int64_t)gb * gbytes;
    prefetch_l2_bulk(wrow, (uint32_t)(ng * gbytes));
  }
  pdl_wait();
  pdl_launch_dependents();

  // per-output epilogue operands of this thread (feature n0 + tid % 16, tokens
  // tid / 16 + 16 j), loaded now so that their latency hides behind the ring
  const int erow = threadIdx.x & (kSkRows - 1);
  const int en = n0 + erow;
  const float e_bias = args.bias ? __uint_as_float((uint32_t)__ldg(args.bias + en) << 16) : 0.f;
  const float e_gv = args.gate_mode == 2 ? __uint_as_float((uint32_t)__ldg(args.gate + en) << 16) : 0.f;
  const float e_wsc = G64 ? 0.f : __ldg(args.sw + en) * args.acc_scale;
  constexpr int kEpiPasses = (MP + kSkThreads / kSkRows - 1) / (kSkThreads / kSkRows);
  float e_sx[kEpiPasses];
#pragma unroll
  for (int j = 0; j < kEpiPasses; ++j) {
    const int m = threadIdx.x / kSkRows + j * (kSkThreads / kSkRows);
    e_sx[j] = (!G64 && m < M) ? __ldg(args.sx + m) : 0.f;
  }

  auto issue = [&](int g, int s) {
    const uint32_t base = ring_s + s * St::bytes;
    if (W4) {
      const int row = lane >> 1, h = lane & 1;
      cp_async16(base + row * 32 + h * 16, args.w4 + (int64_t)(n0 + row) * (K / 2) + g * 32 + h * 16, true);
    } else {
#pragma unroll
      for (int c = lane; c < kSkRows * 4; c += 32) {
        const int row = c >> 2, q = c & 3;
        cp_async16(base + row * 64 + q * 16, args.w8 + (int64_t)(n0 + row) * K + g * 64 + q * 16, true);
      }
    }
#pragma unroll
    for (int c = lane; c < MP * 4; c += 32) {
      const int m = c >> 2, q = c & 3;
      const bool ok = m < M;
      cp_async16(base + St::kW + m * 64 + q * 16, args.x + (ok ? (int64_t)m * K + g * 64 + q * 16 : 0), ok);
    }
    if (G64) {
#pragma unroll
      for (int m = lane; m < MP; m += 32) {
        const bool ok = m < M;
        cp_async4(base + St::kW + St::kX + m * 4, args.sx + (ok ? (int64_t)m * G + g : 0), ok);
      }
      if (lane < kSkRows)
        cp_async4(base + St::kW + St::kX + St::kSx + lane * 4, args.sw + (int64_t)(n0 + lane) * G + g, true);
    }
  };

  float yf[MT][4];
  int yi[MT][4];
#pragma unroll
  for (int b = 0; b < MT; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      yf[b][j] = 0.f;
      yi[b][j] = 0;
    }

#pragma unroll
  for (int s = 0; s < S - 1; ++s) {
    if (s < ng) issue(gb + s, s);
    cp_async_commit();
  }
  for (int i = 0; i < ng; ++i) {
    if (i + S - 1 < ng) issue(gb + i + S - 1, (i + S - 1) % S);
    cp_async_commit();
    cp_async_wait<S - 1>();   // this thread's copies of group i have landed
    __syncwarp();             // ... and every other lane's
    const unsigned char* st = ring + (i % S) * St::bytes;
    const int g = gb + i;
    // A fragments of the two k32 steps: rows gq and gq + 8, group offsets
    // 16 tq .. 16 tq + 15 (step 0: +0..7, step 1: +8..15)
    uint32_t a0[4], a1[4];
    if (W4) {
      const uint2 p0 = *reinterpret_cast<const uint2*>(st + gq * 32 + 8 * tq);
      const uint2 p1 = *reinterpret_cast<const uint2*>(st + (gq + 8) * 32 + 8 * tq);
      uint32_t r0[4], r1[4];
      if (F8) {
        nibbles_to_e4m3(p0.x, r0[0], r0[1]);
        nibbles_to_e4m3(p0.y, r0[2], r0[3]);
        nibbles_to_e4m3(p1.x, r1[0], r1[1]);
        nibbles_to_e4m3(p1.y, r1[2], r1[3]);
      } else {
        nibbles_to_16q(p0.x, r0[0], r0[1]);
        nibbles_to_16q(p0.y, r0[2], r0[3]);
        nibbles_to_16q(p1.x, r1[0], r1[1]);
        nibbles_to_16q(p1.y, r1[2], r1[3]);
      }
      a0[0] = r0[0]; a0[1] = r1[0]; a0[2] = r0[1]; a0[3] = r1[1];
      a1[0] = r0[2]; a1[1] = r1[2]; a1[2] = r0[3]; a1[3] = r1[3];
    } else {
      const uint4 w0 = *reinterpret_cast<const uint4*>(st + gq * 64 + 16 * tq);
      const uint4 w1 = *reinterpret_cast<const uint4*>(st + (gq + 8) * 64 + 16 * tq);
      a0[0] = w0.x; a0[1] = w1.x; a0[2] = w0.y; a0[3] = w1.y;
      a1[0] = w0.z; a1[1] = w1.z; a1[2] = w0.w; a1[3] = w1.w;
    }
    float s_lo = 0.f, s_hi = 0.f;   // weight scale x acc_scale of rows gq, gq + 8
    const float* sxs = reinterpret_cast<const float*>(st + St::kW + St::kX);
    if (G64) {
      const float* sws = reinterpret_cast<const float*>(st + St::kW + St::kX + St::kSx);
      s_lo = sws[gq] * args.acc_scale;
      s_hi = sws[gq + 8] * args.acc_scale;
    }
#pragma unroll
    for (int b = 0; b < MT; ++b) {
      // B fragment: token 8 b + gq, the same group offsets as the A rows
      const uint4 xb = *reinterpret_cast<const uint4*>(st + St::kW + (8 * b + gq) * 64 + 16 * tq);
      float c[4];
      int ci[4];
      if (F8) {
        c[0] = c[1] = c[2] = c[3] = 0.f;
        mma_e4m3_16832(c, a0, xb.x, xb.y);
        mma_e4m3_16832(c, a1, xb.z, xb.w);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) ci[j] = G64 ? 0 : yi[b][j];
        mma_s8_16832(ci, a0, xb.x, xb.y);
        mma_s8_16832(ci, a1, xb.z, xb.w);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (G64) c[j] = (float)ci[j];   // |partial| <= 16 * 4096: exact
          else yi[b][j] = ci[j];
        }
      }
      if (G64) {
        // fragment element j: row gq + 8 (j >> 1), token 8 b + 2 tq + (j & 1)
        if (dbg) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = 8 * b + 2 * tq + (j & 1);
            const int n = n0 + gq + 8 * (j >> 1);
            if (m < M) {
              const int v = F8 ? __float2int_rn(c[j]) : (W4 ? (ci[j] >> 4) : ci[j]);
              args.acc_debug[((int64_t)g * M + m) * N + n] = v;
            }
          }
        }
        const float2 sb = *reinterpret_cast<const float2*>(sxs + 8 * b + 2 * tq);
        yf[b][0] = fmaf(c[0], s_lo * sb.x, yf[b][0]);
        yf[b][1] = fmaf(c[1], s_lo * sb.y, yf[b][1]);
        yf[b][2] = fmaf(c[2], s_hi * sb.x, yf[b][2]);
        yf[b][3] = fmaf(c[3], s_hi * sb.y, yf[b][3]);
      }
    }
    __syncwarp();   // every lane is done with the stage before it is refilled
  }
  cp_async_wait<0>();

  // ------------------------------------------------------------ reduction over the warps
  __syncthreads();   // the reduction buffer overlays the rings
  uint32_t* red = reinterpret_cast<uint32_t*>(sk_smem);   // [warp][row][MPP]
#pragma unroll
  for (int b = 0; b < MT; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = gq + 8 * (j >> 1), m = 8 * b + 2 * tq + (j & 1);
      red[(warp * kSkRows + row) * MPP + m] = G64 ? __float_as_uint(yf[b][j]) : (uint32_t)yi[b][j];
    }
  __syncthreads();

  // ------------------------------------------------------------ epilogue: thread = (feature, token)
  const int row = erow;
  const int n = en;
  const bool sig = args.gate_mode == 1 && n >= args.gate_c0 && n < args.gate_c1;
#pragma unroll
  for (int j = 0; j < kEpiPasses; ++j) {
    const int m = threadIdx.x / kSkRows + j * (kSkThreads / kSkRows);
    if (m >= M) break;
    float o;
    if (G64) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kSkWarps; ++w) s += __uint_as_float(red[(w * kSkRows + row) * MPP + m]);
      o = s + e_bias;
    } else {
      int s = 0;
#pragma unroll
      for (int w = 0; w < kSkWarps; ++w) s += (int)red[(w * kSkRows + row) * MPP + m];
      if (dbg) args.acc_debug[(int64_t)m * N + n] = W4 ? (s >> 4) : s;
      o = fmaf((float)s, e_wsc * e_sx[j], e_bias);
    }
    if (args.r) {
      // low-rank branch: (ld l2t^T)[m, n], bf16 products accumulated in float32
      const uint4* lp = reinterpret_cast<const uint4*>(args.ld + (int64_t)m * args.r);
      const uint4* wp = reinterpret_cast<const uint4*>(args.l2t + (int64_t)n * args.r);
      float l = 0.f;
      for (int c = 0; c < args.r / 8; ++c) {
        const uint4 la = __ldg(lp + c), wa = __ldg(wp + c);
        const uint32_t lv[4] = {la.x, la.y, la.z, la.w}, wv[4] = {wa.x, wa.y, wa.z, wa.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          l = fmaf(__uint_as_float(lv[j] << 16), __uint_as_float(wv[j] << 16), l);
          l = fmaf(__uint_as_float(lv[j] & 0xFFFF0000u), __uint_as_float(wv[j] & 0xFFFF0000u), l);
        }
      }
      o += l;
    }
    if (sig) o = __frcp_rn(1.0f + __expf(-o));
    if (args.gate_mode == 2) {
      const float rres = __uint_as_float((uint32_t)__ldg(args.residual + (int64_t)m * args.ldr + n) << 16);
      o = fmaf(e_gv, o, rres);
    }
    args.y[(int64_t)m * args.ldy + n] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
  }
}

template <bool W4, bool G64, bool F8, int MT>
cudaError_t launch_skinny(const GemmArgs& a, cudaStream_t st) {
  const uint32_t smem = SkStage<W4, G64, MT>::smem;
  auto kern = skinny_gemm_kernel<W4, G64, F8, MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // programmatic stream serialisation: the kernel may start while the preceding
  // kernel (normally the activation prologue) is still running; it only
  // prefetches weights before waiting for it
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(a.N / kSkRows);
  cfg.blockDim = dim3(kSkThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <bool W4, bool G64, bool F8>
cudaError_t launch_skinny_mt(const GemmArgs& a, cudaStream_t st) {
  if (a.M <= 8) return launch_skinny<W4, G64, F8, 1>(a, st);
  if (a.M <= 16) return launch_skinny<W4, G64, F8, 2>(a, st);
  if (a.M <= 32) return launch_skinny<W4, G64, F8, 4>(a, st);
  return launch_skinny<W4, G64, F8, 8>(a, st);
}

}  // namespace

cudaError_t launch_skinny_gemm(bool w4, bool g64, bool f8, const GemmArgs& a, cudaStream_t st) {
  if (a.M < 1 || a.M > kSkinnyMaxM || a.N % kSkRows != 0 || a.K % 128 != 0) return cudaErrorInvalidValue;
  if (f8 && !(w4 && g64)) return cudaErrorInvalidValue;
  if (w4) {
    if (!g64) return launch_skinny_mt<true, false, false>(a, st);
    return f8 ? launch_skinny_mt<true, true, true>(a, st) : launch_skinny_mt<true, true, false>(a, st);
  }
  return g64 ? launch_skinny_mt<false, true, false>(a, st) : launch_skinny_mt<false, false, false>(a, st);
}

}  // namespace rbd
