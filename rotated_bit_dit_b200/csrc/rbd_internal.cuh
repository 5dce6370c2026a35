// Host-side interfaces between the C ABI layer and the kernel launchers.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace rbd {

// Arguments of the low-bit GEMM kernel (one launch = one linear call).
struct GemmArgs {
  int M, N, K;
  int seg;              // accumulation segment length along K (64, or K for row scales)
  int G;                // segments per tile = K / seg
  const float* sx;      // activation scales [M] or [M, K/64]
  const float* sw;      // weight scales [N] or [N, K/64]
  const uint8_t* w4;    // packed INT4 weights [N, K/2] (W4A4 only)
  const uint16_t* bias; // bf16 [N] or null
  int r;                // low-rank rank, 0 = no branch
  int gate_mode;        // 0 none, 1 sigmoid on [gate_c0, gate_c1), 2 gated residual
  int gate_c0, gate_c1;
  const uint16_t* gate;      // bf16 [N]
  const uint16_t* residual;  // bf16 [M, ldr]
  int64_t ldr;
  uint16_t* y;          // bf16 [M, ldy]
  int64_t ldy;
  int32_t* acc_debug;   // optional exact accumulators
  float acc_scale;      // 1/16 for widened INT4 weights, 1 for INT8
  int num_m_tiles, num_tiles;
  // plain pointers of the operands the tiled kernel reads through tensor maps
  // (the small-token kernel reads them directly)
  const uint8_t* x;     // activation codes [M, K]
  const int8_t* w8;     // INT8 weights [N, K] (W8A8 only)
  const uint16_t* ld;   // bf16 [M, r]
  const uint16_t* l2t;  // bf16 [N, r]
};

// e4m3: write each (4-bit) code as the E4M3 byte of equal value instead of an int8.
cudaError_t launch_rot_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int bits, bool rot, bool g64,
                             bool packed, bool e4m3, int8_t* codes, float* scales, cudaStream_t st);
// RMSNorm + modulation, then rotate/quantise (activation codes, one byte each).
cudaError_t launch_norm_rot_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int bits, bool rot,
                                  bool g64, bool e4m3, const uint16_t* gamma, const uint16_t* shift,
                                  const uint16_t* scale, float eps, int8_t* codes, float* scales, cudaStream_t st);
// Group-scale prologue and low-rank down product in one pass over X.
cudaError_t launch_rot_quant_lowrank(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int bits, bool rot,
                                     bool e4m3, const uint16_t* l1t, int r, int8_t* codes, float* scales,
                                     uint16_t* ld, cudaStream_t st);
cudaError_t launch_lowrank_down(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const uint16_t* l1t, int r,
                                uint16_t* ld, cudaStream_t st);
// tm_y: unswizzled map of Y with 32-feature x 64-token boxes (group-scale tiles store through it)
// f8: E4M3 activation codes and the kind::f8f6f4 contraction (W4A4 with group scales only).
cudaError_t launch_lowbit_gemm(bool w4, bool g64, bool f8, const CUtensorMap& tm_x, const CUtensorMap& tm_w8,
                               const CUtensorMap& tm_ld, const CUtensorMap& tm_l2, const CUtensorMap& tm_y,
                               const GemmArgs& a, int num_sms, cudaStream_t st);

// Token counts up to this run on the small-token kernel (warp mma.sync with K
// split across the warps of a 16-feature block), larger ones on the tiled one.
constexpr int kSkinnyMaxM = 64;
// f8: E4M3 activation codes (W4A4 with group scales only).
cudaError_t launch_skinny_gemm(bool w4, bool g64, bool f8, const GemmArgs& a, cudaStream_t st);

// Arguments of the block-scaled FP4 GEMM.
struct NvArgs {
  int M, N, K;
  const uint8_t* sfx;   // activation E4M3 block scales, tile-interleaved
  const uint8_t* sfw;   // weight E4M3 block scales, tile-interleaved
  const float* gsx;     // activation tensor scale (device scalar)
  const float* gsw;     // weight tensor scale (device scalar)
  const uint16_t* bias;
  int gate_mode, gate_c0, gate_c1;
  const uint16_t* gate;
  const uint16_t* residual;
  int64_t ldr;
  uint16_t* y;
  int64_t ldy;
  int num_m_tiles, num_tiles;
  int r;                // low-rank branch rank (0: none); ld / l2t come by tensor map
};

cudaError_t launch_nvfp4_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, bool rot, uint32_t* work,
                               uint8_t* codes, uint8_t* bscale, float* gscale, cudaStream_t st);
cudaError_t launch_nvfp4_gemm(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const CUtensorMap& tm_ld,
                              const CUtensorMap& tm_l2, const NvArgs& a, int num_sms, cudaStream_t st);
uint32_t nvfp4_gemm_smem_bytes();

// INT4 KV-cache codec (n = groups per rotary band: 1, 2 or 4).
cudaError_t launch_kv4_encode(const uint16_t* x, int T, int H, int64_t ldt, int n, uint8_t* codes, float* scales,
                              int64_t capacity, int64_t slot0, cudaStream_t st);
cudaError_t launch_kv4_decode(const uint8_t* codes, const float* scales, int64_t capacity, int64_t slot0, int T,
                              int H, int n, uint16_t* y, int64_t ldt, cudaStream_t st);

// INT8 attention (SageAttention v1 scheme): preparation and the attention kernel.
int64_t attn_workspace_bytes(int64_t Tk, int64_t H);
cudaError_t launch_attn_quant(const uint16_t* q, int64_t ldq, const uint16_t* k, int64_t ldk, const uint16_t* v,
                              int64_t ldv, int Tq, int Tk, int H, int8_t* qc, float* sq, int8_t* kc, float* sk,
                              void* vt, int64_t tkp, void* work, cudaStream_t st);
cudaError_t launch_attn_int8(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const CUtensorMap& tm_sk, const float* sq, int Tq, int Tk, int H, uint16_t* o,
                             int64_t ldo, cudaStream_t st);

// Offline SVDQuant fit (synchronous; host linear algebra between device steps).
int64_t svdquant_workspace_bytes(int64_t n, int64_t k, int rank, int oversample, int bits, int scale_group);
cudaError_t svdquant_fit(const uint16_t* w, int64_t n, int64_t k, int bits, bool rot, int scale_group, int rank,
                         int oversample, int iters, const double* omegas, const double* act_rms, void* q_out,
                         float* scales_out, double* l1, double* l2, double* errs, int* best_out, void* work,
                         cudaStream_t st);

uint32_t gemm_smem_bytes(bool g64, int r, int G);   // dynamic shared memory of one GEMM CTA
int gemm_tile_tokens(bool g64);                     // tokens per GEMM tile

}  // namespace rbd
