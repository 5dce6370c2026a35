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
// Tile and orientation.  One CTA computes 128 output features x TT tokens:
// the MMA's M side is the weights (TMEM lane = output feature), its N side the
// tokens (TMEM column = token).  On B200 one tcgen05.mma kind::i8 instruction
// (M=128, K=32) takes about the same time for any N up to 256, so wide N is
// what reaches the tensor pipe's rate.  Both operands are read from shared
// memory (128-byte swizzled, K-major):
//   - activation codes (int8) arrive by TMA, TT rows x 128 bytes per stage;
//   - W8A8 weights arrive by TMA, 128 rows x 128 bytes per stage;
//   - W4A4 weights are widened from packed nibbles by four converter warps
//     and written into the same swizzled layout.  tcgen05 has no INT4 kind; a
//     nibble is placed in the high half of its byte (value 16*q, exact), so
//     widening is a shift, two masks and two byte permutes per 8 codes, and
//     the epilogue folds the factor 1/16 into the weight scale.
// Accumulation segments.  NB int32 accumulators of TT columns each rotate in
// TMEM: the tensor core fills one while the epilogue drains another.  A
// segment is the whole K range (row scales) or one 64-wide K block (group
// scales); the low-rank branch, when present, is one more segment per tile,
// computed with a bf16 MMA (fp32 result) into the same buffers.
//   - Row scales: TT = 256, NB = 2.  One promotion per tile.
//   - Group scales: TT = 128, NB = 4 (4 x 128 columns fill the 512 of TMEM).
//     Every 64-wide K block needs its own promotion, so the epilogue is the
//     busy side.  The four buffers are handed over in pairs (the two groups
//     of one 128-wide K stage): the tensor core fills one pair while the
//     epilogue drains the other, and the small tile keeps the epilogue's
//     accumulators and in-flight TMEM loads in registers (see the
//     group-scale epilogue below).
// In group mode the epilogue adds the bit pattern of 12582912.0f (1.5 * 2^23)
// to each int32 partial: read as float the sum is exactly 12582912 + 16*acc,
// and fma(f, a, -12582912*a) gives the correctly rounded 16*acc*a without an
// int->float conversion (a is the weight scale rounded to 22 significant bits
// so that 12582912*a is exact; the relative change of the scale is below
// 2^-22).
//
// E4M3 path (F8, W4A4 with group-64 scales and E4M3 activation codes).  Every
// INT4 code in [-8, 7] is an exact E4M3 value, and a 64-wide group partial of
// such products (|sum| <= 4096) is exact in the float32 accumulator, so the
// contraction can run as tcgen05.mma kind::f8f6f4 at the INT8 rate and hand
// the epilogue float32 partials: promotion is then y += (p * a) * b, two
// float32 operations per element and group, with no int -> float step.  The
// converter warps widen each packed nibble into its E4M3 byte through a
// 16-entry byte-permute lookup (three permutes and one select per 4 codes).
//
// Warp roles (16 warps, registers redistributed per warpgroup with setmaxnreg):
//   warpgroup 0: warps 0, 2, 3 TMA producers, warp 1 TMEM allocator + MMA issuer;
//   warpgroup 1: INT4 -> INT8 converters (W4A4 only);
//   warpgroups 2-3: epilogue; thread = one output feature (TMEM lane) x TT/2
//   tokens (128 with row scales, 64 with group scales).
#include "rbd_common.cuh"
#include "rbd_internal.cuh"

namespace rbd {

namespace {

constexpr int kTileF = 128;    // output features per tile (TMEM lanes)
constexpr int kBK = 128;       // K per pipeline stage (one 128-byte swizzle row)
constexpr int kMaxStages = 4;
constexpr int kThreads = 512;  // 16 warps
constexpr int kWarpMma = 1, kWarpConv0 = 4, kWarpEpi0 = 8;
constexpr int kProducers = 3;  // warps 0, 2, 3
constexpr int kEpiThreads = 256;
constexpr uint32_t kMagicBits = 0x4B400000u;  // 12582912.0f
constexpr float kMagicF = 12582912.0f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWStageBytes = kTileF * kBK;   // 16 KB

__host__ __device__ constexpr int tile_tokens(bool g64) { return g64 ? 128 : 256; }
__host__ __device__ constexpr int num_bufs(bool g64) { return g64 ? 4 : 2; }

__device__ __forceinline__ void named_bar_epi() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace

struct SmemLayout {
  uint32_t x_off, w_off, ld_off, l2_off, sx_off, sw_off, out_off, bar_off, total, x_stage;
  int stages, sx_stride;
  bool sw_table;   // group mode: the tile's weight scales are staged in shared memory
};

// Group-scale tiles keep the tile's weight scales in shared memory too, one row
// of 128 features per group; the odd row stride keeps both the staging writes
// (lanes along groups) and the epilogue's reads (lanes along features) free of
// bank conflicts.
constexpr int kSwStride = kTileF + 1;

// Group-scale tiles stage their bf16 output per epilogue warp (32 features x 64
// tokens, row-major by token) for one bulk tensor store.
constexpr uint32_t kOutWarpBytes = 32 * 64 * 2;

__host__ __device__ inline SmemLayout smem_layout(int stages, int r, int G, int tt, bool sw_table) {
  SmemLayout L{};
  L.sw_table = sw_table && tt == tile_tokens(true);
  uint32_t off = 0;
  L.stages = stages;
  L.x_stage = (uint32_t)tt * kBK;
  L.x_off = off;
  off += stages * L.x_stage;
  off = (off + 1023u) & ~1023u;
  L.w_off = off;
  off += stages * kWStageBytes;
  L.ld_off = off;
  off += (uint32_t)tt * r * 2;
  off = (off + 1023u) & ~1023u;
  L.l2_off = off;
  off += kTileF * r * 2;
  off = (off + 1023u) & ~1023u;
  L.sx_stride = tt + 4;
  L.sx_off = off;
  off += (uint32_t)G * L.sx_stride * 4;
  off = (off + 127u) & ~127u;
  L.sw_off = off;
  if (L.sw_table) off += (uint32_t)G * kSwStride * 4;
  off = (off + 127u) & ~127u;
  L.out_off = off;
  if (tt == tile_tokens(true)) off += 8 * kOutWarpBytes;
  off = (off + 15u) & ~15u;
  L.bar_off = off;
  off += 32 * 8 + 16;
  L.total = off + 1024;  // slack for 1024-byte alignment of the base
  return L;
}

// The layout with the most pipeline stages (up to 4, at least 2) that fits,
// with the weight-scale table when it fits; stages == 0 if nothing fits.
__host__ __device__ inline SmemLayout pick_layout(int r, int G, int tt) {
  for (int t = 1; t >= 0; --t)
    for (int s = kMaxStages; s >= 2; --s) {
      const SmemLayout L = smem_layout(s, r, G, tt, t != 0);
      if (L.total <= 227u * 1024u) return L;
    }
  SmemLayout none{};
  return none;
}

// ---------------------------------------------------------------------------
// Group-scale epilogue (128-token tiles, four TMEM buffers).
//
// Thread mapping.  The epilogue warp of lane quarter q and token half h reads
// TMEM with the 32-lane x 32-bit shape (the fastest TMEM -> register path):
// thread = one output feature x 64 token columns.  A segment is read in two
// phases of 32 columns; while one phase is promoted the other is in flight.
// The activation scales of a column are the same for every lane of the warp,
// so they are read as shared-memory broadcasts.
//
// Each segment's first MMA overwrites its buffer, so TMEM is only read.  The
// int32 partial v is turned into a float by adding the bit pattern of
// 12582912.0f (exact: |v| < 2^22) and one fma with -12582912 * a removes the
// bias while applying the weight scale.
// ---------------------------------------------------------------------------
constexpr int kG64Half = 64;   // token columns per epilogue warp

template <int P>
__device__ __forceinline__ void g64_load_phase(uint32_t tcol, uint32_t (&v)[32]) {
  tmem_ld16_async(tcol + 32u * P, *reinterpret_cast<uint32_t(*)[16]>(v));
  tmem_ld16_async(tcol + 32u * P + 16u, *reinterpret_cast<uint32_t(*)[16]>(v + 16));
}

__device__ __forceinline__ void tmem_reg_fence32(uint32_t (&v)[32]) {
  tmem_reg_fence(*reinterpret_cast<uint32_t(*)[16]>(v));
  tmem_reg_fence(*reinterpret_cast<uint32_t(*)[16]>(v + 16));
}

// y[16 P + j2] += (16*acc*a) * b for the 32 columns of phase P; b4 points at the
// scales of the phase's first column (broadcast reads).  F8: the partials are
// float32 already and y += (p * a) * b, two paired float32 operations per two
// columns.
template <int P, bool W4, bool DBG, bool F8>
__device__ __forceinline__ void g64_promote_phase(float2 (&y)[32], const uint32_t (&v)[32], const float4* b4,
                                                  float a, float c, int32_t* dbg, int64_t dbg_m0, int64_t M,
                                                  int64_t N) {
#pragma unroll
  for (int j4 = 0; j4 < 8; ++j4) {
    const float4 bq = b4[j4];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int j = 4 * j4 + 2 * hh;
      const uint32_t u0 = v[j], u1 = v[j + 1];
      if (DBG) {
        const int64_t m = dbg_m0 + 32 * P + j;
        if (F8) {
          if (m < M) dbg[m * N] = __float2int_rn(__uint_as_float(u0));
          if (m + 1 < M) dbg[(m + 1) * N] = __float2int_rn(__uint_as_float(u1));
        } else {
          if (m < M) dbg[m * N] = W4 ? ((int32_t)u0 >> 4) : (int32_t)u0;
          if (m + 1 < M) dbg[(m + 1) * N] = W4 ? ((int32_t)u1 >> 4) : (int32_t)u1;
        }
      }
      const float2 t = F8 ? __fmul2_rn(make_float2(__uint_as_float(u0), __uint_as_float(u1)), make_float2(a, a))
                          : make_float2(fmaf(__uint_as_float(u0 + kMagicBits), a, c),
                                        fmaf(__uint_as_float(u1 + kMagicBits), a, c));
      const float2 b = hh ? make_float2(bq.z, bq.w) : make_float2(bq.x, bq.y);
      float2& yy = y[16 * P + j / 2];
      yy = __ffma2_rn(t, b, yy);
    }
  }
}

// Low-rank segment (fp32 branch result in TMEM): y += v for phase P.
template <int P>
__device__ __forceinline__ void g64_add_phase(float2 (&y)[32], const uint32_t (&v)[32]) {
#pragma unroll
  for (int j2 = 0; j2 < 16; ++j2) {
    y[16 * P + j2].x += __uint_as_float(v[2 * j2]);
    y[16 * P + j2].y += __uint_as_float(v[2 * j2 + 1]);
  }
}

// One 128 x 128 tile of the group-scale epilogue for this thread (feature n,
// token columns col0 .. col0+63 of the tile): optional low-rank segment, G
// promoted segments, gate and store.  tcol = TMEM address of this warp's lane
// quarter at column col0 of buffer 0; sxc = the scale table at column col0.
// The four buffers are handed over in pairs (pb = pair 0 or 1, buffers 2 pb and
// 2 pb + 1): the two groups of one 128-wide K stage share a pair, the low-rank
// segment takes a pair of its own.  Returns false if a wait timed out (nothing
// is stored then).
template <bool W4, bool LR, bool DBG, bool F8>
__device__ __forceinline__ bool g64_tile(const GemmArgs& args, uint32_t tcol, uint64_t* pfull, uint64_t* pempty,
                                         int& pb, uint32_t& pbits, const float* sxc, int sx_stride,
                                         const float* sws, int m0, int n, int col0, uint32_t lane,
                                         const CUtensorMap* tm_y, uint16_t* sout) {
  constexpr int TT = 128;
  const int G = args.G;
  auto release = [&](int b) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&pempty[b]);
  };
  auto acquire = [&](int b) {
    if (!mbar_wait(&pfull[b], (pbits >> b) & 1u)) return false;
    pbits ^= 1u << b;
    tc_fence_after();
    return true;
  };

  float2 y[32];
  {
    const float bv = args.bias ? __uint_as_float((uint32_t)__ldg(args.bias + n) << 16) : 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) y[j] = make_float2(bv, bv);
  }

  if (LR) {
    if (!acquire(pb)) return false;
    const uint32_t tb = tcol + 2 * pb * TT;
    uint32_t v[32];
    g64_load_phase<0>(tb, v); tmem_wait_ld(); tmem_reg_fence32(v); g64_add_phase<0>(y, v);
    g64_load_phase<1>(tb, v); tmem_wait_ld(); tmem_reg_fence32(v); g64_add_phase<1>(y, v);
    release(pb);
    pb ^= 1;
  }

  // weight scale of this thread's feature, one segment ahead: from the tile's
  // table in shared memory, or (when the table did not fit) from global memory
  const float* swp = args.sw + (int64_t)n * G;
  float swn = sws ? sws[0] : __ldg(swp);
  const int64_t dbg_m0 = (int64_t)m0 + col0;
  int32_t* dbg = DBG ? args.acc_debug + n : nullptr;
  uint32_t vX[32], vY[32];
  if (!acquire(pb)) return false;
  g64_load_phase<0>(tcol + 2 * pb * TT, vX);
  bool ok = true;
  for (int g = 0; g < G; ++g) {
    const int odd = g & 1;
    const uint32_t tA = tcol + (2 * pb + odd) * TT;
    // integer partials: weight scale rounded to 22 significant bits so that c is exact;
    // float32 partials (F8): the weight scale itself
    const float a = F8 ? swn * args.acc_scale : __uint_as_float((__float_as_uint(swn * args.acc_scale) + 2u) & ~3u);
    const float c = -kMagicF * a;
    if (g + 1 < G) swn = sws ? sws[(g + 1) * kSwStride] : __ldg(swp + g + 1);
    const float4* b4 = reinterpret_cast<const float4*>(sxc + (int64_t)g * sx_stride);
    int32_t* dg = DBG ? dbg + (int64_t)g * args.M * args.N : nullptr;
    // phase 0 (columns 0-31) while phase 1 is in flight
    tmem_wait_ld();
    tmem_reg_fence32(vX);
    g64_load_phase<1>(tA, vY);
    g64_promote_phase<0, W4, DBG, F8>(y, vX, b4, a, c, dg, dbg_m0, args.M, args.N);
    // phase 1 (columns 32-63) while the next segment's phase 0 is in flight;
    // a pair is free as soon as the last load of its second buffer has landed
    tmem_wait_ld();
    tmem_reg_fence32(vY);
    if (!odd) {
      g64_load_phase<0>(tA + TT, vX);   // second buffer of the same pair
    } else {
      release(pb);
      pb ^= 1;
      if (g + 1 < G) {
        if (!acquire(pb)) ok = false;
        else g64_load_phase<0>(tcol + 2 * pb * TT, vX);
      }
    }
    g64_promote_phase<1, W4, DBG, F8>(y, vY, b4 + 8, a, c, dg, dbg_m0, args.M, args.N);
    if (!ok) return false;
  }

  // gate and store: feature n, tokens m0 + col0 + j (a warp writes 32
  // consecutive features of one token row per store)
  const int64_t mbase = (int64_t)m0 + col0;
  const int64_t rem = (int64_t)args.M - mbase;
  const int jmax = rem >= kG64Half ? kG64Half : (int)rem;
  uint16_t* yp = args.y + mbase * args.ldy + n;
  if (args.gate_mode == 2) {
    const float gv = __uint_as_float((uint32_t)__ldg(args.gate + n) << 16);
    const uint16_t* rp = args.residual + mbase * args.ldr + n;
#pragma unroll
    for (int j = 0; j < kG64Half; ++j) {
      if (j < jmax) {
        const float o = (j & 1) ? y[j >> 1].y : y[j >> 1].x;
        const float rres = __uint_as_float((uint32_t)__ldg(rp) << 16);   // read-only path, as in row mode
        *yp = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(gv, o, rres)));
      }
      yp += args.ldy;
      rp += args.ldr;
    }
  } else {
    // through shared memory and one bulk tensor store per warp: token row j of
    // the warp's block holds its 32 features (64 contiguous bytes); rows past M
    // are clipped by the tensor map.  The previous tile's store must have read
    // the buffer before it is overwritten.
    const bool sig = args.gate_mode == 1 && n >= args.gate_c0 && n < args.gate_c1;
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
#pragma unroll
    for (int j2 = 0; j2 < kG64Half / 2; ++j2) {
      float o0 = y[j2].x, o1 = y[j2].y;
      if (sig) {
        o0 = __frcp_rn(1.0f + __expf(-o0));
        o1 = __frcp_rn(1.0f + __expf(-o1));
      }
      const __nv_bfloat162 ob = __floats2bfloat162_rn(o0, o1);   // one conversion per pair
      sout[(2 * j2) * 32 + lane] = __bfloat16_as_ushort(ob.x);
      sout[(2 * j2 + 1) * 32 + lane] = __bfloat16_as_ushort(ob.y);
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tm_y, sout, n - (int)lane, m0 + col0);
      bulk_commit();
    }
  }
  return true;
}

template <bool W4, bool G64, bool LR, bool DBG, bool F8 = false>
__global__ void __launch_bounds__(kThreads, 1)
    lowbit_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w8,
                       const __grid_constant__ CUtensorMap tm_ld, const __grid_constant__ CUtensorMap tm_l2,
                       const __grid_constant__ CUtensorMap tm_y, const GemmArgs args) {
  constexpr int TT = tile_tokens(G64);
  constexpr int NB = num_bufs(G64);
  constexpr int EC = TT / 2;       // TMEM columns (tokens) per epilogue thread
  constexpr int NCH = EC / 16;     // 16-column chunks per epilogue thread
  extern __shared__ unsigned char smem_dyn[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023u) & ~uintptr_t(1023u));
  const SmemLayout L = pick_layout(LR ? args.r : 0, args.G, TT);
  const int S = L.stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* full = bars;                    // [kMaxStages]
  uint64_t* empty = bars + kMaxStages;      // [kMaxStages]
  uint64_t* pfull = bars + 2 * kMaxStages;  // [NB]
  uint64_t* pempty = pfull + 4;             // [NB]
  uint64_t* lrsfull = pempty + 4;
  uint64_t* lrsempty = lrsfull + 1;
  uint64_t* drain = lrsempty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], W4 ? 1 + 4 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], kEpiThreads / 32);
    }
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
    if (G64) tma_prefetch_desc(&tm_y);
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

  if (warp < 4) {
    setmaxnreg_dec<40>();
    if (warp != kWarpMma) {
      // ---------------------------------------------------------- TMA producers
      // Warps 0, 2 and 3 own the pipeline stages round-robin: bulk tensor
      // loads issued by one thread complete one after another, so several
      // issuing warps keep several stages in flight.  The number of producers
      // never exceeds the number of stages: a producer's previous wait then
      // guarantees that the slot it waits on is at most one phase behind, which
      // is what a parity wait can tell apart.
      const int nprod = S < kProducers ? S : kProducers;
      const int pidx = warp == 0 ? 0 : (int)warp - 1;   // 0, 1, 2
      if (lane == 0 && pidx < nprod) {
        uint32_t lr_phase = 0;
        bool ok = true;
        int turn = 0, stage = 0;   // round-robin position and pipeline slot of the next stage
        uint32_t phase = 0;
        for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
          const int mt = t % args.num_m_tiles, nt = t / args.num_m_tiles;
          const int m0 = mt * TT, n0 = nt * kTileF;
          if (LR && pidx == 0) {
            if (!mbar_wait(lrsempty, lr_phase ^ 1)) { ok = false; break; }
            const uint32_t bytes = (uint32_t)(TT + kTileF) * args.r * 2;
            mbar_arrive_expect_tx(lrsfull, bytes);
            tma_load_2d(smem + L.ld_off, &tm_ld, lrsfull, 0, m0);
            tma_load_2d(smem + L.l2_off, &tm_l2, lrsfull, 0, n0);
            lr_phase ^= 1;
          }
          for (int ks = 0; ks < nks; ++ks) {
            const bool mine = turn == pidx;
            if (++turn == nprod) turn = 0;
            if (mine) {
              if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
              mbar_arrive_expect_tx(&full[stage], W4 ? L.x_stage : L.x_stage + kWStageBytes);
              tma_load_2d(smem + L.x_off + stage * L.x_stage, &tm_x, &full[stage], ks * kBK, m0);
              if (!W4) tma_load_2d(smem + L.w_off + stage * kWStageBytes, &tm_w8, &full[stage], ks * kBK, n0);
            }
            if (++stage == S) { stage = 0; phase ^= 1; }
          }
        }
        if (!ok) {
          // let bulk copies already in flight land before the CTA can exit
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 200000ull) {}
        }
      }
    } else {
      // ---------------------------------------------------------- MMA issuer
      // One thread issues every MMA; the tensor core completes a K=32 step in
      // about 128 cycles at N=256, so the issue loop is kept free of integer
      // division and dynamic indexing (segment boundaries are compile-time:
      // one per tile with row scales, two per stage with group scales).
      if (elect_one()) {
        static_assert(!F8 || (W4 && G64), "the E4M3 path is the W4A4 group-scale path");
        const uint32_t idesc = F8 ? idesc_e4m3(kTileF, TT) : idesc_i8(kTileF, TT);
        const uint32_t idesc_lr = idesc_bf16(kTileF, TT);
        // descriptor address fields are byte offsets >> 4; stage s adds s * stage bytes >> 4
        const uint64_t bdesc0 = smem_desc_kmajor(smem_u32(smem + L.x_off), 128);
        const uint64_t adesc0 = smem_desc_kmajor(smem_u32(smem + L.w_off), 128);
        int stage = 0;
        uint32_t phase = 0, lr_phase = 0;
        uint64_t bdesc = bdesc0, adesc = adesc0;
        int pb = 0;
        uint32_t pbits = 0;   // bit b: parity of the next pempty phase of buffer b
        bool ok = true;
        const uint32_t lr_row_bytes = (uint32_t)args.r * 2;
        auto acquire = [&](int b) {
          if (!mbar_wait(&pempty[b], (pbits >> b) & 1u)) return false;
          pbits ^= 1u << b;
          tc_fence_after();
          return true;
        };
        auto next = [](int b) { return b + 1 == NB ? 0 : b + 1; };
        for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
          if (LR) {
            // group mode: the low-rank segment takes a whole buffer pair (its first buffer)
            if (!mbar_wait(lrsfull, lr_phase) || !acquire(pb)) { ok = false; break; }
            lr_phase ^= 1;
            tc_fence_after();
            const uint32_t dl = tmem + (G64 ? 2 * pb : pb) * TT;
            const uint32_t a0 = smem_u32(smem + L.l2_off), b0 = smem_u32(smem + L.ld_off);
            for (int kk = 0; kk < args.r / 16; ++kk) {
              mma_bf16_ss(dl, smem_desc_kmajor(a0 + kk * 32, lr_row_bytes),
                          smem_desc_kmajor(b0 + kk * 32, lr_row_bytes), idesc_lr, kk > 0 ? 1u : 0u);
            }
            tc_commit(&pfull[pb]);
            tc_commit(lrsempty);
            pb = G64 ? (pb ^ 1) : next(pb);
          }
          if (!G64 && !acquire(pb)) { ok = false; break; }
          for (int ks = 0; ks < nks; ++ks) {
            if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
            tc_fence_after();
            if constexpr (G64) {
              // K columns 0-63 and 64-127 of the stage are two groups; they fill the two
              // buffers of pair pb (buffers 2 pb, 2 pb + 1), handed over together
              if (!acquire(pb)) { ok = false; break; }
#pragma unroll
              for (int hg = 0; hg < 2; ++hg) {
                const uint32_t d = tmem + (2 * pb + hg) * TT;
                if constexpr (F8) {
                  mma_f8_ss(d, adesc + 4 * hg, bdesc + 4 * hg, idesc, 0u);   // overwrite: a new group
                  mma_f8_ss(d, adesc + 4 * hg + 2, bdesc + 4 * hg + 2, idesc, 1u);
                } else {
                  mma_i8_ss(d, adesc + 4 * hg, bdesc + 4 * hg, idesc, 0u);   // overwrite: a new group
                  mma_i8_ss(d, adesc + 4 * hg + 2, bdesc + 4 * hg + 2, idesc, 1u);
                }
              }
              tc_commit(&pfull[pb]);
              pb ^= 1;
            } else {
              const uint32_t d = tmem + pb * TT;
#pragma unroll
              for (int kk = 0; kk < kBK / 32; ++kk)
                mma_i8_ss(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ks | kk) ? 1u : 0u);
            }
            tc_commit(&empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
              bdesc = bdesc0;
              adesc = adesc0;
            } else {
              bdesc += L.x_stage >> 4;
              adesc += kWStageBytes >> 4;
            }
          }
          if (!ok) break;
          if (!G64) {
            tc_commit(&pfull[pb]);
            pb = next(pb);
          }
        }
        // every issued MMA must complete before TMEM can be released
        tc_commit(drain);
        mbar_wait(drain, 0, 100000000ull);
      }
      __syncwarp();
    }
  } else if (warp < kWarpEpi0) {
    setmaxnreg_dec<88>();
    // ------------------------------------------------------------ INT4 -> INT8 converters
    // Thread = one weight row of the tile.  Packed bytes are fetched two
    // stages ahead; widened bytes go to the 128-byte-swizzled A stage.
    if (W4) {
      const uint32_t fr = (warp - kWarpConv0) * 32 + lane;
      const int half_k = K / 2;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        const int nt = t / args.num_m_tiles;
        const int n = nt * kTileF + fr;
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
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          unsigned char* arow = smem + L.w_off + stage * kWStageBytes + fr * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // 16 packed bytes = codes k = 32i .. 32i+31 -> 16-byte chunks 2i and 2i+1
            const uint32_t pw[4] = {c0[i].x, c0[i].y, c0[i].z, c0[i].w};
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if constexpr (F8) {
                nibbles_to_e4m3(pw[j], o[2 * j], o[2 * j + 1]);   // E4M3 bytes of q
              } else {
                const uint32_t lo = (pw[j] << 4) & 0xF0F0F0F0u;  // even k, as 16*q
                const uint32_t hi = pw[j] & 0xF0F0F0F0u;         // odd k, as 16*q
                o[2 * j] = __byte_perm(lo, hi, 0x5140);
                o[2 * j + 1] = __byte_perm(lo, hi, 0x7362);
              }
            }
            const uint32_t ch0 = (2u * i) ^ (fr & 7u), ch1 = (2u * i + 1u) ^ (fr & 7u);
            *reinterpret_cast<uint4*>(arow + ch0 * 16) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4*>(arow + ch1 * 16) = make_uint4(o[4], o[5], o[6], o[7]);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            c0[i] = c1[i];
            c1[i] = c2[i];
          }
        }
      }
    }
  } else {
    setmaxnreg_inc<192>();
    // ------------------------------------------------------------ epilogue
    // Thread = one output feature (TMEM lane) x EC tokens (TMEM columns).
    const uint32_t q = warp & 3u;
    const uint32_t h = (warp - kWarpEpi0) >> 2;   // token half of the tile
    const uint32_t lane_base = (32u * q) << 16;
    const int etid = threadIdx.x - kWarpEpi0 * 32;  // 0..255
    const int G = args.G;
    float* sx_s = reinterpret_cast<float*>(smem + L.sx_off);
    const int fr = 32 * q + lane;  // feature row of this thread in the tile
    const uint32_t col0 = EC * h;

    // every partial buffer starts released
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
      for (int b = 0; b < NB; ++b) mbar_arrive(&pempty[b]);

    int pb = 0;
    uint32_t pbits = 0;   // bit b: parity of the next pfull phase of buffer b
    bool ok = true;
    for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x) {
      const int mt = t % args.num_m_tiles, nt = t / args.num_m_tiles;
      const int m0 = mt * TT, n0 = nt * kTileF;
      // stage the tile's activation scales in shared memory, group-major
      named_bar_epi();
      {
        // warp w stages tokens w + 8 i; lane l covers groups g0 + l.  All loads
        // of a 32-group chunk are issued before the first store, so a chunk
        // costs one memory latency.
        constexpr int kTokPerWarp = TT / (kEpiThreads / 32);
        const int ew = etid >> 5;
        for (int g0 = 0; g0 < G; g0 += 32) {
          const int g = g0 + (int)lane;
          float v[kTokPerWarp];
#pragma unroll
          for (int i = 0; i < kTokPerWarp; ++i) {
            const int64_t m = (int64_t)m0 + ew + 8 * i;
            v[i] = (g < G && m < args.M) ? __ldg(args.sx + m * G + g) : 0.f;
          }
          if (g < G) {
#pragma unroll
            for (int i = 0; i < kTokPerWarp; ++i) sx_s[g * L.sx_stride + ew + 8 * i] = v[i];
          }
        }
        if (G64 && L.sw_table) {
          // the tile's weight scales: warp w stages features w + 8 i, lane l groups g0 + l
          float* sw_s = reinterpret_cast<float*>(smem + L.sw_off);
          for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + (int)lane;
            float v[kTileF / 8];
#pragma unroll
            for (int i = 0; i < kTileF / 8; ++i)
              v[i] = g < G ? __ldg(args.sw + (int64_t)(n0 + ew + 8 * i) * G + g) : 0.f;
            if (g < G) {
#pragma unroll
              for (int i = 0; i < kTileF / 8; ++i) sw_s[g * kSwStride + ew + 8 * i] = v[i];
            }
          }
        }
      }
      named_bar_epi();
      if constexpr (G64) {
        if (ok)
          ok = g64_tile<W4, LR, DBG, F8>(args, tmem + lane_base + col0, pfull, pempty, pb, pbits, sx_s + col0,
                                     L.sx_stride,
                                     L.sw_table ? reinterpret_cast<const float*>(smem + L.sw_off) + fr : nullptr, m0,
                                     n0 + fr, (int)col0, lane, &tm_y,
                                     reinterpret_cast<uint16_t*>(smem + L.out_off) +
                                         (warp - kWarpEpi0) * (kOutWarpBytes / 2));
        continue;
      } else {

      const int n = n0 + fr;
      const float* swrow = args.sw + (int64_t)n * G;
      float sw_next = __ldg(swrow);
      float2 y[EC / 2];
      const float bias = args.bias ? __uint_as_float((uint32_t)__ldg(args.bias + n) << 16) : 0.f;
#pragma unroll
      for (int j = 0; j < EC / 2; ++j) y[j] = make_float2(bias, bias);

      if (LR && ok) {
        // low-rank segment: fp32 branch result, added once
        if (!mbar_wait(&pfull[pb], (pbits >> pb) & 1u)) ok = false;
        if (ok) {
          pbits ^= 1u << pb;
          tc_fence_after();
          const uint32_t tbase = tmem + lane_base + pb * TT + col0;
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            uint32_t v[16];
            tmem_ld16(tbase + 16 * c, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              y[8 * c + j].x += __uint_as_float(v[2 * j]);
              y[8 * c + j].y += __uint_as_float(v[2 * j + 1]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pempty[pb]);
          pb = pb + 1 == NB ? 0 : pb + 1;
        }
      }
      {
        for (int g = 0; g < G && ok; ++g) {
          const float sw_g = sw_next;
          if (g + 1 < G) sw_next = __ldg(swrow + g + 1);
          if (!mbar_wait(&pfull[pb], (pbits >> pb) & 1u)) { ok = false; break; }
          pbits ^= 1u << pb;
          tc_fence_after();
          const uint32_t tbase = tmem + lane_base + pb * TT + col0;
          const float4* sxg = reinterpret_cast<const float4*>(sx_s + g * L.sx_stride + col0);
          const float a = sw_g * args.acc_scale;
          const float2 a2 = make_float2(a, a);
          {
            // row scales: one promotion per tile; TMEM loads pipelined two deep
            uint32_t va[16], vb[16];
            tmem_ld16_async(tbase, va);
            tmem_wait_ld();
            tmem_reg_fence(va);
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
              uint32_t (&v)[16] = (c & 1) ? vb : va;
              uint32_t (&vn)[16] = (c & 1) ? va : vb;
              if (c + 1 < NCH) tmem_ld16_async(tbase + 16 * (c + 1), vn);
              if (DBG) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  const int64_t m = (int64_t)m0 + col0 + 16 * c + j;
                  if (m < args.M) args.acc_debug[m * args.N + n] = W4 ? ((int32_t)v[j] >> 4) : (int32_t)v[j];
                }
              }
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const float4 b4 = sxg[4 * c + j4];
                const float2 f0 = make_float2((float)(int32_t)v[4 * j4], (float)(int32_t)v[4 * j4 + 1]);
                const float2 f1 = make_float2((float)(int32_t)v[4 * j4 + 2], (float)(int32_t)v[4 * j4 + 3]);
                y[8 * c + 2 * j4] = __ffma2_rn(f0, __fmul2_rn(a2, make_float2(b4.x, b4.y)), y[8 * c + 2 * j4]);
                y[8 * c + 2 * j4 + 1] =
                    __ffma2_rn(f1, __fmul2_rn(a2, make_float2(b4.z, b4.w)), y[8 * c + 2 * j4 + 1]);
              }
              if (c + 1 < NCH) {
                tmem_wait_ld();
                tmem_reg_fence(vn);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pempty[pb]);
          pb = pb + 1 == NB ? 0 : pb + 1;
        }
      }
      if (!ok) continue;  // keep the named barriers balanced; stop producing output

      // gate and store: thread (feature n) writes tokens m0 + col0 + j
      const bool sig = args.gate_mode == 1 && n >= args.gate_c0 && n < args.gate_c1;
      const float gv = args.gate_mode == 2 ? __uint_as_float((uint32_t)__ldg(args.gate + n) << 16) : 0.f;
      const int64_t mbase = (int64_t)m0 + col0;
      const int64_t rem = (int64_t)args.M - mbase;
      const int jmax = rem >= EC ? EC : (int)rem;
      uint16_t* yp = args.y + mbase * args.ldy + n;
      const int64_t ystep = args.ldy;
      if (args.gate_mode == 2) {
        // the residual through the read-only path: each element is read once, by the
        // thread that then writes the output there (so even y == residual is safe),
        // and the loads may move ahead of the stores instead of waiting behind them
        const uint16_t* rp = args.residual + mbase * args.ldr + n;
        const int64_t rstep = args.ldr;
#pragma unroll
        for (int j = 0; j < EC; ++j) {
          if (j < jmax) {
            const float o = (j & 1) ? y[j >> 1].y : y[j >> 1].x;
            const float rres = __uint_as_float((uint32_t)__ldg(rp) << 16);
            *yp = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(gv, o, rres)));
          }
          yp += ystep;
          rp += rstep;
        }
      } else {
        // round to bf16 pairs first (halves the live registers), then store
        uint32_t ob[EC / 2];
#pragma unroll
        for (int j2 = 0; j2 < EC / 2; ++j2) {
          float o0 = y[j2].x, o1 = y[j2].y;
          if (sig) {
            o0 = __frcp_rn(1.0f + __expf(-o0));
            o1 = __frcp_rn(1.0f + __expf(-o1));
          }
          ob[j2] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o0)) |
                   ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o1)) << 16);
        }
#pragma unroll
        for (int j = 0; j < EC; ++j) {
          if (j < jmax) *yp = (uint16_t)((j & 1) ? (ob[j >> 1] >> 16) : (ob[j >> 1] & 0xFFFFu));
          yp += ystep;
        }
      }
      }
    }
  }

  // bulk stores still in flight must complete before the CTA (and its shared memory) goes away
  if (G64 && warp >= kWarpEpi0 && lane == 0) bulk_wait_all();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------
uint32_t gemm_smem_bytes(bool g64, int r, int G) {
  const SmemLayout L = pick_layout(r, G, tile_tokens(g64));
  return L.stages ? L.total : 0xFFFFFFFFu;
}

int gemm_tile_tokens(bool g64) { return tile_tokens(g64); }

// The warpgroup register split (40 + 88 + 2 x 192 per thread) adds up to the
// 128 registers per thread the block is launched with; a build that launched
// with fewer would make setmaxnreg.inc wait forever, so refuse to launch it.
static bool regs_ok(const void* kern) {
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
  return fa.numRegs == 128;
}

cudaError_t launch_lowbit_gemm(bool w4, bool g64, bool f8, const CUtensorMap& tm_x, const CUtensorMap& tm_w8,
                               const CUtensorMap& tm_ld, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                               const GemmArgs& a, int num_sms, cudaStream_t st) {
  const bool lr = a.r > 0;
  const uint32_t smem = gemm_smem_bytes(g64, a.r, a.G);
  if (smem > 227u * 1024u) return cudaErrorInvalidConfiguration;
  const int grid = a.num_tiles < num_sms ? a.num_tiles : num_sms;
  const bool dbg = a.acc_debug != nullptr;
  if (f8 && !(w4 && g64)) return cudaErrorInvalidValue;
#define RBD_GEMM_CASE(W, G, R, D, F)                                                                  \
  if (w4 == W && g64 == G && lr == R && dbg == D && f8 == F) {                                       \
    auto kern = lowbit_gemm_kernel<W, G, R, D, F>;                                                   \
    if (!regs_ok(reinterpret_cast<const void*>(kern))) return cudaErrorInvalidConfiguration;         \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);    \
    if (e != cudaSuccess) return e;                                                                  \
    kern<<<grid, kThreads, smem, st>>>(tm_x, tm_w8, tm_ld, tm_l2, tm_y, a);                               \
    return cudaGetLastError();                                                                       \
  }
#define RBD_GEMM_CASES(W, G, R) RBD_GEMM_CASE(W, G, R, false, false) RBD_GEMM_CASE(W, G, R, true, false)
  RBD_GEMM_CASE(true, true, true, false, true)
  RBD_GEMM_CASE(true, true, true, true, true)
  RBD_GEMM_CASE(true, true, false, false, true)
  RBD_GEMM_CASE(true, true, false, true, true)
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

}  // namespace rbd
