// C ABI of the rotated low-bit linear library: argument validation, tensor-map
// construction, launches, and the device status word.  Every entry point
// validates before launching and never falls back to another implementation.
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include <cmath>

#include "rbd_common.cuh"

#include "rbd_internal.cuh"
#include "rbd_rope.cuh"

namespace {

using rbd::GemmArgs;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

rbd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RBD_OK : RBD_ERR_CUDA; }

rbd_status check_qcfg(const rbd_qcfg& c, int64_t K) {
  if (c.bits != 4 && c.bits != 8) return RBD_ERR_INVALID_ARG;
  if (c.code_format != RBD_CODES_INT8 && c.code_format != RBD_CODES_E4M3) return RBD_ERR_INVALID_ARG;
  if (c.code_format == RBD_CODES_E4M3 && c.bits != 4) return RBD_ERR_UNSUPPORTED;
  if (c.rot_group != 0 && c.rot_group != 256) return RBD_ERR_UNSUPPORTED;
  if (c.scale_group != 0 && c.scale_group != 64) return RBD_ERR_UNSUPPORTED;
  if (K <= 0 || K % 256 != 0 || K > 16384) return RBD_ERR_UNSUPPORTED;
  return RBD_OK;
}

// --- driver entry point for tensor-map encoding (no link against libcuda)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major 2D tensor [rows, cols] with row stride `row_bytes`; box = [box_rows, box_cols].
// Swizzle follows the box's inner size (128/64/32 bytes) unless `plain` asks for
// an unswizzled row-major box.
bool make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint32_t elem_bytes, uint64_t cols,
                 uint64_t rows, uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, bool plain = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint32_t inner_bytes = box_cols * elem_bytes;
  CUtensorMapSwizzle sw;
  switch (inner_bytes) {
    case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
    case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
    default: return false;
  }
  if (plain) sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Row-major tensor of rank 2 or 3 (dims innermost first, strides in bytes for
// dims 1..rank-1) with an explicit swizzle; used by the attention maps.
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint32_t rank, const uint64_t* dims,
              const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t b[3], es[3] = {1, 1, 1};
  for (uint32_t i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    if (i + 1 < rank) st[i] = strides[i];
  }
  CUresult r = fn(map, dt, rank, const_cast<void*>(base), d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Library-owned scratch for rbd_nvfp4_quant_noalloc.  Some callers cannot hand
// the library a scratch buffer: plain C hosts with no device allocator of their
// own, and serving loops that must not touch an allocator between steps.  For
// them the NVFP4 quantiser's one scratch word (the running tensor amax between
// its two passes) lives in this fixed file-scope array instead.  Its size is
// fixed at build time; calls that would need more are rejected.  Every call
// clears the word it uses before the first pass, so nothing needs to start at
// zero.  All calls on a device share the array: calls that overlap in time
// (concurrent streams, or host threads on the same device) race on it.
constexpr int kNoallocScratchWords = 64;                    // 256 bytes per device
constexpr int kNvfp4ScratchWords = 1;                       // what one quantiser call needs
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoallocScratchWords];

// Device address of the scratch array for the current device.  The first call
// on a device resolves it with cudaGetSymbolAddress (a runtime call that should
// happen before any stream capture); later calls reuse the cached address, so
// a device reset after the first call on a device is not supported.
rbd_status noalloc_scratch(uint32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RBD_ERR_CUDA;
  static std::mutex mu;
  static uint32_t* cache[64] = {nullptr};
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RBD_ERR_CUDA;
    cache[dev] = static_cast<uint32_t*>(p);
  }
  *out = cache[dev];
  return RBD_OK;
}

int num_sms_current() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cache[dev]) return cache[dev];
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev < 64) cache[dev] = n;
  return n;
}

rbd_status quant_validate(const void* x, int64_t M, int64_t K, int64_t ld, rbd_qcfg cfg, const void* out,
                          const float* scales) {
  if (M < 0) return RBD_ERR_INVALID_ARG;
  rbd_status s = check_qcfg(cfg, K);
  if (s != RBD_OK) return s;
  if (M == 0) return RBD_OK;
  if (!x || !out || !scales) return RBD_ERR_INVALID_ARG;
  if (ld < K) return RBD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out) || (ld % 8) != 0) return RBD_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(scales) & 3u) return RBD_ERR_ALIGNMENT;
  return RBD_OK;
}

rbd_status quant_common(const void* x, int64_t M, int64_t K, int64_t ld, rbd_qcfg cfg, void* out, float* scales,
                        bool packed, void* stream) {
  rbd_status s = quant_validate(x, M, K, ld, cfg, out, scales);
  if (s != RBD_OK || M == 0) return s;
  return cuda_status(rbd::launch_rot_quant(static_cast<const uint16_t*>(x), M, K, ld, cfg.bits, cfg.rot_group != 0,
                                           cfg.scale_group == 64, packed, cfg.code_format == RBD_CODES_E4M3,
                                           static_cast<int8_t*>(out), scales, as_stream(stream)));
}

template <bool W4>
rbd_status linear_common(const int8_t* codes, const float* sx, const void* w, const float* sw, int64_t M,
                         int64_t N, int64_t K, rbd_qcfg cfg, const rbd_epilogue* epi, void* y, int64_t ldy,
                         void* stream) {
  if (cfg.bits != (W4 ? 4 : 8)) return RBD_ERR_INVALID_ARG;
  if (cfg.scale_group != 0 && cfg.scale_group != 64) return RBD_ERR_UNSUPPORTED;
  if (cfg.code_format != RBD_CODES_INT8 && cfg.code_format != RBD_CODES_E4M3) return RBD_ERR_INVALID_ARG;
  // E4M3 codes: 4-bit codes with group-64 scales (a float32 partial per 64-wide group is exact)
  const bool f8 = cfg.code_format == RBD_CODES_E4M3;
  if (f8 && !(W4 && cfg.scale_group == 64)) return RBD_ERR_UNSUPPORTED;
  if (M < 0 || N <= 0 || K <= 0) return RBD_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 128 != 0) return RBD_ERR_UNSUPPORTED;
  if (M > (int64_t)INT32_MAX / 2 || N > (1 << 24) || K > (1 << 20)) return RBD_ERR_UNSUPPORTED;
  if (M == 0) return RBD_OK;
  if (!codes || !sx || !w || !sw || !y) return RBD_ERR_INVALID_ARG;
  if (ldy < N) return RBD_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(w) || !aligned16(y) || (ldy % 8) != 0) return RBD_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(sx) & 3u) || (reinterpret_cast<uintptr_t>(sw) & 3u)) return RBD_ERR_ALIGNMENT;
  const int G = cfg.scale_group ? static_cast<int>(K / 64) : 1;
  if (G > 256) return RBD_ERR_UNSUPPORTED;

  rbd_epilogue e{};
  if (epi) e = *epi;
  if (e.r != 0 && e.r != 16 && e.r != 32 && e.r != 64) return RBD_ERR_UNSUPPORTED;
  if (e.r && (!e.ld || !e.l2t)) return RBD_ERR_INVALID_ARG;
  if (e.r && (!aligned16(e.ld) || !aligned16(e.l2t))) return RBD_ERR_ALIGNMENT;
  if (e.gate_mode < 0 || e.gate_mode > 2) return RBD_ERR_INVALID_ARG;
  if (e.gate_mode == 1 && (e.gate_col0 < 0 || e.gate_col1 < e.gate_col0 || e.gate_col1 > N))
    return RBD_ERR_INVALID_ARG;
  if (e.gate_mode == 2) {
    if (!e.gate || !e.residual) return RBD_ERR_INVALID_ARG;
    if (e.ldr < N) return RBD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(e.residual) & 1u) || (reinterpret_cast<uintptr_t>(e.gate) & 1u))
      return RBD_ERR_ALIGNMENT;
  }
  if (e.bias && (reinterpret_cast<uintptr_t>(e.bias) & 1u)) return RBD_ERR_ALIGNMENT;
  if (e.acc_debug && (reinterpret_cast<uintptr_t>(e.acc_debug) & 3u)) return RBD_ERR_ALIGNMENT;

  const bool g64 = cfg.scale_group == 64;
  GemmArgs a{};
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.seg = cfg.scale_group ? 64 : static_cast<int>(K);
  a.G = G;
  a.sx = sx;
  a.sw = sw;
  a.w4 = W4 ? static_cast<const uint8_t*>(w) : nullptr;
  a.bias = static_cast<const uint16_t*>(e.bias);
  a.r = e.r;
  a.gate_mode = e.gate_mode;
  a.gate_c0 = static_cast<int>(e.gate_col0);
  a.gate_c1 = static_cast<int>(e.gate_col1);
  a.gate = static_cast<const uint16_t*>(e.gate);
  a.residual = static_cast<const uint16_t*>(e.residual);
  a.ldr = e.ldr;
  a.y = static_cast<uint16_t*>(y);
  a.ldy = ldy;
  a.acc_debug = e.acc_debug;
  a.acc_scale = (W4 && !f8) ? 1.0f / 16.0f : 1.0f;   // the INT8 path widens a nibble q to the byte 16 q
  a.x = reinterpret_cast<const uint8_t*>(codes);
  a.w8 = W4 ? nullptr : static_cast<const int8_t*>(w);
  a.ld = static_cast<const uint16_t*>(e.ld);
  a.l2t = static_cast<const uint16_t*>(e.l2t);
  // a few tokens: the weight-streaming kernel
  if (M <= rbd::kSkinnyMaxM) return cuda_status(rbd::launch_skinny_gemm(W4, g64, f8, a, as_stream(stream)));

  if (rbd::gemm_smem_bytes(g64, e.r, G) > 227u * 1024u) return RBD_ERR_UNSUPPORTED;
  const int tt = rbd::gemm_tile_tokens(g64);

  CUtensorMap tm_x{}, tm_w{}, tm_ld{}, tm_l2{};
  if (!make_map_2d(&tm_x, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, K, 128, tt)) return RBD_ERR_CUDA;
  if (!W4 && !make_map_2d(&tm_w, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, K, 128, 128)) return RBD_ERR_CUDA;
  if (e.r) {
    if (!make_map_2d(&tm_ld, e.ld, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, e.r, M, 2 * e.r, e.r, tt))
      return RBD_ERR_CUDA;
    if (!make_map_2d(&tm_l2, e.l2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, e.r, N, 2 * e.r, e.r, 128))
      return RBD_ERR_CUDA;
  }
  CUtensorMap tm_y{};
  if (g64 && !make_map_2d(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, 2 * ldy, 32, 64, true))
    return RBD_ERR_CUDA;
  a.num_m_tiles = static_cast<int>((M + tt - 1) / tt);
  a.num_tiles = a.num_m_tiles * static_cast<int>(N / 128);
  const int sms = num_sms_current();
  if (sms <= 0) return RBD_ERR_CUDA;
  return cuda_status(rbd::launch_lowbit_gemm(W4, cfg.scale_group == 64, f8, tm_x, tm_w, tm_ld, tm_l2, tm_y, a, sms,
                                             as_stream(stream)));
}

__global__ void timeout_probe_kernel(int64_t timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    rbd::mbar_init(&bar, 1);
    rbd::fence_barrier_init();
    // Nothing ever arrives on `bar`: the bounded wait must expire and record a timeout.
    rbd::mbar_wait(&bar, 0, static_cast<uint64_t>(timeout_ns));
  }
}

}  // namespace

namespace {
rbd_status kv4_validate(int64_t T, int64_t H, int64_t ldt, int32_t n, const void* x, const void* codes,
                        const float* scales, int64_t capacity, int64_t slot0) {
  if (n != 1 && n != 2 && n != 4) return RBD_ERR_UNSUPPORTED;
  if (T < 0 || H <= 0 || capacity <= 0) return RBD_ERR_INVALID_ARG;
  // 32-bit unit indices, with room for a warp's units past the end
  if (H > 65536 || T > ((int64_t)INT32_MAX - 64) / H || capacity > (int64_t)INT32_MAX / H) return RBD_ERR_UNSUPPORTED;
  if (T > capacity || slot0 < 0 || slot0 >= capacity) return RBD_ERR_INVALID_ARG;
  if (T == 0) return RBD_OK;
  if (!x || !codes || !scales) return RBD_ERR_INVALID_ARG;
  if (ldt < H * 128) return RBD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || (ldt % 8) != 0 || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return RBD_ERR_ALIGNMENT;
  return RBD_OK;
}
}  // namespace

extern "C" {

rbd_status rbd_rot_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, rbd_qcfg cfg, int8_t* codes,
                             float* scales, void* stream) {
  return quant_common(x, M, K, ldx, cfg, codes, scales, false, stream);
}

rbd_status rbd_norm_rot_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                                  const void* shift, const void* scale, float eps, rbd_qcfg cfg, int8_t* codes,
                                  float* scales, void* stream) {
  if (!(eps >= 0.0f) || !(eps < INFINITY)) return RBD_ERR_INVALID_ARG;   // rejects NaN too
  if ((gamma && !aligned16(gamma)) || (shift && !aligned16(shift)) || (scale && !aligned16(scale)))
    return RBD_ERR_ALIGNMENT;
  rbd_status s = quant_validate(x, M, K, ldx, cfg, codes, scales);
  if (s != RBD_OK || M == 0) return s;
  return cuda_status(rbd::launch_norm_rot_quant(
      static_cast<const uint16_t*>(x), M, K, ldx, cfg.bits, cfg.rot_group != 0, cfg.scale_group == 64,
      cfg.code_format == RBD_CODES_E4M3, static_cast<const uint16_t*>(gamma), static_cast<const uint16_t*>(shift),
      static_cast<const uint16_t*>(scale), eps, codes, scales, as_stream(stream)));
}

rbd_status rbd_lowrank_fused(const void* x, int64_t M, int64_t K, int64_t ldx, rbd_qcfg cfg, int8_t* codes,
                             float* scales, const void* l1t, int32_t r, void* ld, void* stream) {
  if (r != 16 && r != 32 && r != 64) return RBD_ERR_UNSUPPORTED;
  if (M > 0 && (!l1t || !ld)) return RBD_ERR_INVALID_ARG;
  if (M > 0 && (!aligned16(l1t) || !aligned16(ld))) return RBD_ERR_ALIGNMENT;
  rbd_status s = quant_validate(x, M, K, ldx, cfg, codes, scales);
  if (s != RBD_OK || M == 0) return s;
  if (cfg.scale_group == 64) {
    // group scales: one pass over X yields codes, scales and the down product
    return cuda_status(rbd::launch_rot_quant_lowrank(static_cast<const uint16_t*>(x), M, K, ldx, cfg.bits,
                                                     cfg.rot_group != 0, cfg.code_format == RBD_CODES_E4M3,
                                                     static_cast<const uint16_t*>(l1t), r, codes, scales,
                                                     static_cast<uint16_t*>(ld), as_stream(stream)));
  }
  s = quant_common(x, M, K, ldx, cfg, codes, scales, false, stream);
  if (s != RBD_OK) return s;
  return cuda_status(rbd::launch_lowrank_down(static_cast<const uint16_t*>(x), M, K, ldx,
                                              static_cast<const uint16_t*>(l1t), r, static_cast<uint16_t*>(ld),
                                              as_stream(stream)));
}

rbd_status rbd_lowrank_down(const void* x, int64_t M, int64_t K, int64_t ldx, const void* l1t, int32_t r, void* ld,
                            void* stream) {
  if (r != 16 && r != 32 && r != 64) return RBD_ERR_UNSUPPORTED;
  if (M < 0 || K <= 0) return RBD_ERR_INVALID_ARG;
  if (K % 128 != 0 || K > 16384 || M > (int64_t)INT32_MAX / 2) return RBD_ERR_UNSUPPORTED;
  if (M == 0) return RBD_OK;
  if (!x || !l1t || !ld) return RBD_ERR_INVALID_ARG;
  if (ldx < K) return RBD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(l1t) || !aligned16(ld) || (ldx % 8) != 0) return RBD_ERR_ALIGNMENT;
  return cuda_status(rbd::launch_lowrank_down(static_cast<const uint16_t*>(x), M, K, ldx,
                                              static_cast<const uint16_t*>(l1t), r, static_cast<uint16_t*>(ld),
                                              as_stream(stream)));
}

rbd_status rbd_kv4_encode(const void* x, int64_t T, int64_t H, int64_t ldt, int32_t groups_per_band,
                          uint8_t* codes, float* scales, int64_t capacity, int64_t slot0, void* stream) {
  rbd_status s = kv4_validate(T, H, ldt, groups_per_band, x, codes, scales, capacity, slot0);
  if (s != RBD_OK || T == 0) return s;
  return cuda_status(rbd::launch_kv4_encode(static_cast<const uint16_t*>(x), static_cast<int>(T),
                                            static_cast<int>(H), ldt, groups_per_band, codes, scales, capacity,
                                            slot0, as_stream(stream)));
}

rbd_status rbd_kv4_decode(const uint8_t* codes, const float* scales, int64_t capacity, int64_t slot0, int64_t T,
                          int64_t H, int32_t groups_per_band, void* y, int64_t ldt, void* stream) {
  rbd_status s = kv4_validate(T, H, ldt, groups_per_band, y, codes, scales, capacity, slot0);
  if (s != RBD_OK || T == 0) return s;
  return cuda_status(rbd::launch_kv4_decode(codes, scales, capacity, slot0, static_cast<int>(T),
                                            static_cast<int>(H), groups_per_band, static_cast<uint16_t*>(y), ldt,
                                            as_stream(stream)));
}

rbd_status rbd_qk_norm_rope(const void* x, int64_t T, int64_t H, int64_t ldx, const void* gamma,
                            const float* cos_t, const float* sin_t, float eps, void* y, int64_t ldy,
                            void* stream) {
  if (T < 0 || H <= 0) return RBD_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !(eps < INFINITY)) return RBD_ERR_INVALID_ARG;   // rejects NaN too
  if (H > 65536 || T > ((int64_t)INT32_MAX / 2) / H) return RBD_ERR_UNSUPPORTED;   // 32-bit unit indices
  if (T == 0) return RBD_OK;
  if (!x || !y || !cos_t || !sin_t) return RBD_ERR_INVALID_ARG;
  if (ldx < H * 128 || ldy < H * 128) return RBD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(cos_t) || !aligned16(sin_t) || (gamma && !aligned16(gamma)) ||
      (ldx % 8) != 0 || (ldy % 8) != 0)
    return RBD_ERR_ALIGNMENT;
  return cuda_status(rbd::launch_qk_norm_rope(static_cast<const uint16_t*>(x), ldx, static_cast<int>(T),
                                              static_cast<int>(H), static_cast<const uint16_t*>(gamma), cos_t,
                                              sin_t, eps, static_cast<uint16_t*>(y), ldy, as_stream(stream)));
}

rbd_status rbd_rope_tables(const int32_t* pos, int64_t T, double base, float* cos_t, float* sin_t,
                           void* stream) {
  if (T < 0 || !(base > 0.0) || !(base < INFINITY)) return RBD_ERR_INVALID_ARG;
  if (T > (int64_t)INT32_MAX / 64) return RBD_ERR_UNSUPPORTED;
  if (T == 0) return RBD_OK;
  if (!pos || !cos_t || !sin_t) return RBD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(pos) & 3u) || !aligned16(cos_t) || !aligned16(sin_t)) return RBD_ERR_ALIGNMENT;
  return cuda_status(rbd::launch_rope_tables(pos, static_cast<int>(T), base, cos_t, sin_t, as_stream(stream)));
}

int64_t rbd_attn_workspace_bytes(int64_t Tk, int64_t H) {
  if (Tk <= 0 || H <= 0) return -1;
  return rbd::attn_workspace_bytes(Tk, H);
}

namespace {
rbd_status attn_sizes_ok(int64_t Tq, int64_t Tk, int64_t H, int64_t tkp) {
  if (Tq < 0 || Tk < 0 || H <= 0) return RBD_ERR_INVALID_ARG;
  if (tkp < Tk || tkp % 8 != 0) return RBD_ERR_INVALID_ARG;
  if (H > 256 || Tq > (1 << 24) || tkp > (1 << 24)) return RBD_ERR_UNSUPPORTED;
  return RBD_OK;
}
}  // namespace

rbd_status rbd_attn_quant(const void* q, int64_t ldq, const void* k, int64_t ldk, const void* v, int64_t ldv,
                          int64_t Tq, int64_t Tk, int64_t H, int8_t* qc, float* sq, int8_t* kc, float* sk, void* vt,
                          int64_t tkp, void* work, void* stream) {
  rbd_status s = attn_sizes_ok(Tq, Tk, H, tkp);
  if (s != RBD_OK) return s;
  if (Tq == 0 && Tk == 0) return RBD_OK;
  if (Tk == 0) return RBD_ERR_INVALID_ARG;   // queries with no keys have no softmax
  if (!q || !k || !v || !qc || !sq || !kc || !sk || !vt || !work) return RBD_ERR_INVALID_ARG;
  if (ldq < H * 128 || ldk < H * 128 || ldv < H * 128) return RBD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qc) || !aligned16(kc) || !aligned16(vt) ||
      !aligned16(sk) || !aligned16(work) || (ldq % 8) || (ldk % 8) || (ldv % 8) ||
      (reinterpret_cast<uintptr_t>(sq) & 3u))
    return RBD_ERR_ALIGNMENT;
  return cuda_status(rbd::launch_attn_quant(static_cast<const uint16_t*>(q), ldq, static_cast<const uint16_t*>(k),
                                            ldk, static_cast<const uint16_t*>(v), ldv, static_cast<int>(Tq),
                                            static_cast<int>(Tk), static_cast<int>(H), qc, sq, kc, sk, vt, tkp, work,
                                            as_stream(stream)));
}

rbd_status rbd_attn_int8(const int8_t* qc, const float* sq, const int8_t* kc, const float* sk, const void* vt,
                         int64_t Tq, int64_t Tk, int64_t H, int64_t tkp, void* o, int64_t ldo, void* stream) {
  rbd_status s = attn_sizes_ok(Tq, Tk, H, tkp);
  if (s != RBD_OK) return s;
  if (Tq == 0) return RBD_OK;
  if (Tk == 0) return RBD_ERR_INVALID_ARG;
  if (!qc || !sq || !kc || !sk || !vt || !o) return RBD_ERR_INVALID_ARG;
  if (ldo < H * 128) return RBD_ERR_INVALID_ARG;
  if (!aligned16(qc) || !aligned16(kc) || !aligned16(vt) || !aligned16(sk) || !aligned16(o) || (ldo % 8) ||
      (reinterpret_cast<uintptr_t>(sq) & 3u))
    return RBD_ERR_ALIGNMENT;
  CUtensorMap tm_q{}, tm_k{}, tm_v{}, tm_sk{};
  {
    const uint64_t d[3] = {128, (uint64_t)Tq, (uint64_t)H}, st[2] = {128, (uint64_t)Tq * 128};
    const uint32_t b[3] = {128, 128, 1};
    if (!make_map(&tm_q, qc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B))
      return RBD_ERR_CUDA;
  }
  {
    const uint64_t d[3] = {128, (uint64_t)Tk, (uint64_t)H}, st[2] = {128, (uint64_t)Tk * 128};
    const uint32_t b[3] = {128, 128, 1};
    if (!make_map(&tm_k, kc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B))
      return RBD_ERR_CUDA;
  }
  {
    const uint64_t d[3] = {(uint64_t)tkp, 128, (uint64_t)H}, st[2] = {(uint64_t)tkp * 2, (uint64_t)tkp * 256};
    const uint32_t b[3] = {64, 128, 1};
    if (!make_map(&tm_v, vt, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B))
      return RBD_ERR_CUDA;
  }
  {
    const uint64_t d[2] = {(uint64_t)tkp, (uint64_t)H}, st[1] = {(uint64_t)tkp * 4};
    const uint32_t b[2] = {128, 1};
    if (!make_map(&tm_sk, sk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, d, st, b, CU_TENSOR_MAP_SWIZZLE_NONE))
      return RBD_ERR_CUDA;
  }
  return cuda_status(rbd::launch_attn_int8(tm_q, tm_k, tm_v, tm_sk, sq, static_cast<int>(Tq), static_cast<int>(Tk),
                                           static_cast<int>(H), static_cast<uint16_t*>(o), ldo, as_stream(stream)));
}

namespace {
rbd_status svdquant_cfg_ok(int64_t N, int64_t K, rbd_qcfg cfg, int32_t rank, int32_t oversample) {
  rbd_status s = check_qcfg(cfg, K);
  if (s != RBD_OK) return s;
  if (cfg.code_format != RBD_CODES_INT8) return RBD_ERR_UNSUPPORTED;
  if (N <= 0 || rank <= 0 || oversample < 0) return RBD_ERR_INVALID_ARG;
  const int64_t p = (int64_t)rank + oversample;
  if (p > N || p > K || p > 256 || N > (1 << 20)) return RBD_ERR_UNSUPPORTED;
  return RBD_OK;
}
}  // namespace

int64_t rbd_svdquant_workspace_bytes(int64_t N, int64_t K, int32_t rank, int32_t oversample, rbd_qcfg cfg) {
  if (svdquant_cfg_ok(N, K, cfg, rank, oversample) != RBD_OK) return -1;
  return rbd::svdquant_workspace_bytes(N, K, rank, oversample, cfg.bits, cfg.scale_group);
}

rbd_status rbd_svdquant_fit(const void* w, int64_t N, int64_t K, rbd_qcfg cfg, int32_t rank, int32_t oversample,
                            int32_t iters, const double* omegas, const double* act_rms, void* q, float* scales,
                            double* l1, double* l2, double* errs, int32_t* best, void* work, void* stream) {
  rbd_status s = svdquant_cfg_ok(N, K, cfg, rank, oversample);
  if (s != RBD_OK) return s;
  if (iters <= 0) return RBD_ERR_INVALID_ARG;
  if (!w || !omegas || !q || !scales || !l1 || !l2 || !errs || !work) return RBD_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(q) || !aligned16(work) || (reinterpret_cast<uintptr_t>(scales) & 3u))
    return RBD_ERR_ALIGNMENT;
  int b = -1;
  const cudaError_t e = rbd::svdquant_fit(static_cast<const uint16_t*>(w), N, K, cfg.bits, cfg.rot_group != 0,
                                          cfg.scale_group, rank, oversample, iters, omegas, act_rms, q, scales,
                                          l1, l2, errs, &b, work, as_stream(stream));
  if (best) *best = b;
  return cuda_status(e);
}

rbd_status rbd_pack_weights_int4(const void* w, int64_t N, int64_t K, rbd_qcfg cfg, uint8_t* packed, float* scales,
                                 void* stream) {
  if (cfg.bits != 4) return RBD_ERR_INVALID_ARG;
  if (cfg.code_format != RBD_CODES_INT8) return RBD_ERR_UNSUPPORTED;   // packed nibbles are two's complement
  return quant_common(w, N, K, K, cfg, packed, scales, true, stream);
}

rbd_status rbd_pack_weights_int8(const void* w, int64_t N, int64_t K, rbd_qcfg cfg, int8_t* w8, float* scales,
                                 void* stream) {
  if (cfg.bits != 8) return RBD_ERR_INVALID_ARG;
  if (cfg.code_format != RBD_CODES_INT8) return RBD_ERR_UNSUPPORTED;
  return quant_common(w, N, K, K, cfg, w8, scales, false, stream);
}

rbd_status rbd_w4a4_linear(const int8_t* codes, const float* sx, const uint8_t* w_packed, const float* sw,
                           int64_t M, int64_t N, int64_t K, rbd_qcfg cfg, const rbd_epilogue* epi, void* y,
                           int64_t ldy, void* stream) {
  return linear_common<true>(codes, sx, w_packed, sw, M, N, K, cfg, epi, y, ldy, stream);
}

rbd_status rbd_w8a8_linear(const int8_t* codes, const float* sx, const int8_t* w8, const float* sw, int64_t M,
                           int64_t N, int64_t K, rbd_qcfg cfg, const rbd_epilogue* epi, void* y, int64_t ldy,
                           void* stream) {
  return linear_common<false>(codes, sx, w8, sw, M, N, K, cfg, epi, y, ldy, stream);
}

int64_t rbd_nvfp4_scale_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 64 != 0) return -1;
  return (rows + 127) / 128 * 128 * (K / 16);
}

rbd_status rbd_nvfp4_quant(const void* x, int64_t M, int64_t K, int64_t ldx, int32_t rot_group, uint8_t* codes,
                           uint8_t* block_scales, float* tensor_scale, uint32_t* work, void* stream) {
  if (M < 0 || K <= 0) return RBD_ERR_INVALID_ARG;
  if (rot_group != 256 && rot_group != 0) return RBD_ERR_UNSUPPORTED;
  if (K % 256 != 0 || K > 16384 || M > (int64_t)INT32_MAX / 2) return RBD_ERR_UNSUPPORTED;
  if (M == 0) return RBD_OK;
  if (!x || !codes || !block_scales || !tensor_scale || !work) return RBD_ERR_INVALID_ARG;
  if (ldx < K) return RBD_ERR_INVALID_ARG;
  if (!aligned16(x) || (ldx % 8) != 0 || (reinterpret_cast<uintptr_t>(codes) & 7u)) return RBD_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(tensor_scale) & 3u) || (reinterpret_cast<uintptr_t>(work) & 3u))
    return RBD_ERR_ALIGNMENT;
  return cuda_status(rbd::launch_nvfp4_quant(static_cast<const uint16_t*>(x), M, K, ldx, rot_group != 0, work, codes,
                                             block_scales, tensor_scale, as_stream(stream)));
}

rbd_status rbd_nvfp4_quant_noalloc(const void* x, int64_t M, int64_t K, int64_t ldx, int32_t rot_group,
                                   uint8_t* codes, uint8_t* block_scales, float* tensor_scale, void* stream) {
  if (kNvfp4ScratchWords > kNoallocScratchWords) return RBD_ERR_UNSUPPORTED;   // scratch request too large
  if (M <= 0) return rbd_nvfp4_quant(x, M, K, ldx, rot_group, codes, block_scales, tensor_scale, nullptr, stream);
  if (!x || !codes || !block_scales || !tensor_scale) return RBD_ERR_INVALID_ARG;
  uint32_t* work = nullptr;
  const rbd_status s = noalloc_scratch(&work);
  if (s != RBD_OK) return s;
  return rbd_nvfp4_quant(x, M, K, ldx, rot_group, codes, block_scales, tensor_scale, work, stream);
}

rbd_status rbd_nvfp4_linear(const uint8_t* xq, const uint8_t* xbs, const float* xgs, const uint8_t* wq,
                            const uint8_t* wbs, const float* wgs, int64_t M, int64_t N, int64_t K,
                            const rbd_epilogue* epi, void* y, int64_t ldy, void* stream) {
  if (M < 0 || N <= 0 || K <= 0) return RBD_ERR_INVALID_ARG;
  if (K % 256 != 0 || N % 128 != 0) return RBD_ERR_UNSUPPORTED;
  if (M > (int64_t)INT32_MAX / 2 || N > (1 << 24) || K > (1 << 20)) return RBD_ERR_UNSUPPORTED;
  if (M == 0) return RBD_OK;
  if (!xq || !xbs || !xgs || !wq || !wbs || !wgs || !y) return RBD_ERR_INVALID_ARG;
  if (ldy < N) return RBD_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(xbs) || !aligned16(wbs) || !aligned16(y) || (ldy % 8) != 0)
    return RBD_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(xgs) & 3u) || (reinterpret_cast<uintptr_t>(wgs) & 3u)) return RBD_ERR_ALIGNMENT;
  rbd_epilogue e{};
  if (epi) e = *epi;
  if (e.acc_debug) return RBD_ERR_UNSUPPORTED;
  if (e.r != 0 && e.r != 16 && e.r != 32 && e.r != 64) return RBD_ERR_UNSUPPORTED;
  if (e.r && (!e.ld || !e.l2t)) return RBD_ERR_INVALID_ARG;
  if (e.r && (!aligned16(e.ld) || !aligned16(e.l2t))) return RBD_ERR_ALIGNMENT;
  if (e.gate_mode < 0 || e.gate_mode > 2) return RBD_ERR_INVALID_ARG;
  if (e.gate_mode == 1 && (e.gate_col0 < 0 || e.gate_col1 < e.gate_col0 || e.gate_col1 > N))
    return RBD_ERR_INVALID_ARG;
  if (e.gate_mode == 2) {
    if (!e.gate || !e.residual) return RBD_ERR_INVALID_ARG;
    if (e.ldr < N) return RBD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(e.residual) & 1u) || (reinterpret_cast<uintptr_t>(e.gate) & 1u))
      return RBD_ERR_ALIGNMENT;
  }
  if (e.bias && (reinterpret_cast<uintptr_t>(e.bias) & 1u)) return RBD_ERR_ALIGNMENT;
  CUtensorMap tm_x{}, tm_w{}, tm_ld{}, tm_l2{};
  if (!make_map_2d(&tm_x, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, M, K / 2, 128, 128)) return RBD_ERR_CUDA;
  if (!make_map_2d(&tm_w, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, K / 2, 128, 128)) return RBD_ERR_CUDA;
  if (e.r) {
    if (!make_map_2d(&tm_ld, e.ld, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, e.r, M, 2 * e.r, e.r, 128))
      return RBD_ERR_CUDA;
    if (!make_map_2d(&tm_l2, e.l2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, e.r, N, 2 * e.r, e.r, 128))
      return RBD_ERR_CUDA;
  }
  rbd::NvArgs a{};
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.sfx = xbs;
  a.sfw = wbs;
  a.gsx = xgs;
  a.gsw = wgs;
  a.bias = static_cast<const uint16_t*>(e.bias);
  a.gate_mode = e.gate_mode;
  a.gate_c0 = static_cast<int>(e.gate_col0);
  a.gate_c1 = static_cast<int>(e.gate_col1);
  a.gate = static_cast<const uint16_t*>(e.gate);
  a.residual = static_cast<const uint16_t*>(e.residual);
  a.ldr = e.ldr;
  a.y = static_cast<uint16_t*>(y);
  a.ldy = ldy;
  a.num_m_tiles = static_cast<int>((M + 127) / 128);
  a.num_tiles = a.num_m_tiles * static_cast<int>(N / 128);
  a.r = static_cast<int>(e.r);
  const int sms = num_sms_current();
  if (sms <= 0) return RBD_ERR_CUDA;
  return cuda_status(rbd::launch_nvfp4_gemm(tm_x, tm_w, tm_ld, tm_l2, a, sms, as_stream(stream)));
}

rbd_status rbd_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return RBD_ERR_CUDA;
  int st = 0;
  e = cudaMemcpyFromSymbol(&st, rbd::g_device_status, sizeof(int));
  if (e != cudaSuccess) return RBD_ERR_CUDA;
  if (st != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(rbd::g_device_status, &zero, sizeof(int)) != cudaSuccess) return RBD_ERR_CUDA;
    return static_cast<rbd_status>(st);
  }
  return RBD_OK;
}

rbd_status rbd_debug_timeout_probe(int64_t timeout_ns, void* stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000ll) return RBD_ERR_INVALID_ARG;
  timeout_probe_kernel<<<1, 32, 0, as_stream(stream)>>>(timeout_ns);
  return cuda_status(cudaGetLastError());
}

const char* rbd_status_string(rbd_status s) {
  switch (s) {
    case RBD_OK: return "RBD_OK";
    case RBD_ERR_INVALID_ARG: return "RBD_ERR_INVALID_ARG";
    case RBD_ERR_UNSUPPORTED: return "RBD_ERR_UNSUPPORTED";
    case RBD_ERR_ALIGNMENT: return "RBD_ERR_ALIGNMENT";
    case RBD_ERR_CUDA: return "RBD_ERR_CUDA";
    case RBD_ERR_DEVICE_TIMEOUT: return "RBD_ERR_DEVICE_TIMEOUT";
  }
  return "RBD_ERR_UNKNOWN";
}

const char* rbd_version(void) { return "rotated_bit_dit_b200 0.1 (sm_100a)"; }

}  // extern "C"
