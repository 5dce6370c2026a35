// Offline SVDQuant fit of the low-rank branch: a seeded randomized SVD of the
// (activation-weighted) weight, then alternating refits of the branch to what
// quantisation misses and requantisation of the remainder, keeping the best
// iterate.
//
// Method: "Krea-2-SVDQuant-ComfyUI", "Low-rank refinement, and what the
// objective actually is" (the objective is the Frobenius distance between W
// and the quantised part plus the branch; the first split comes from a
// randomized SVD; each later iterate re-fits the branch to W - deq(Q) and
// requantises the rest; the best iterate wins) and "Activation-aware branch"
// (with activation statistics each input channel's error counts by its RMS
// d, scaled to mean 1 and floored at 0.05).  Open points, as read here:
//   - the randomized SVD takes its Gaussian test matrices as inputs (one per
//     iterate, K x (rank + oversample)) and one power iteration, with QR
//     re-orthonormalisation after every product;
//   - the residual W - low is rounded to bf16 (the packer's input type) and
//     quantised in the layer's own rotated INT4 / INT8 format;
//   - the rank-r product is split evenly: L1 = (V / d) sqrt(S), L2 = sqrt(S) U^T.
//
// Where the work runs: the products with the full weight (A Omega, A^T Y,
// A Z, Q^T A, U S V^T), the residual, the requantisation (the library's own
// weight packer), the dequantisation with its inverse rotation and the error
// reduction run on the GPU in float64; the thin QR factorisations
// (Householder) and the small SVD (one-sided Jacobi on the (r+p) x K
// projection) run on the host in plain C++, also in float64.  The call is
// synchronous: it waits for the device between steps.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <numeric>
#include <vector>

#include "rbd_common.cuh"
#include "rbd_internal.cuh"

namespace rbd {

namespace {

__device__ __forceinline__ double bf16_to_f64(uint16_t b) { return (double)__uint_as_float((uint32_t)b << 16); }

// bf16 bits of x, rounded to nearest with ties to even directly from float64
// (8 significant bits; bf16 subnormals below 2^-126).
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const double a = fabs(x);
  if (!(a > 0.0)) return (uint16_t)(__double_as_longlong(x) < 0 ? 0x8000u : 0u);
  const int e = (int)((__double_as_longlong(a) >> 52) & 0x7FF) - 1023;   // leading-bit exponent
  const double ulp = ldexp(1.0, max(e, -126) - 7);
  double r = rint(a / ulp) * ulp;
  if (r > 3.3895313892515355e38) r = INFINITY;
  const uint32_t f = __float_as_uint((float)r);
  return (uint16_t)((f >> 16) | (x < 0 ? 0x8000u : 0u));
}

// A[i][k] = (W[i][k] - (deq ? deq[i][k] : 0)) * d[k]
__global__ void svq_make_a(const uint16_t* __restrict__ w, const double* __restrict__ deq,
                           const double* __restrict__ d, double* __restrict__ a, int64_t n, int64_t k) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n * k) return;
  double v = bf16_to_f64(w[i]);
  if (deq) v -= deq[i];
  a[i] = v * d[i % k];
}

// C[m][n] = sum_k A(m, k) B(k, n), float64, with A(m, k) = a[m * sam + k * sak] and
// B(k, n) = b[k * sbk + n * sbn]; C row-major with row stride ldc.  32 x 32 output
// tiles, 16-wide K steps through shared memory, a fixed summation order.
__global__ void __launch_bounds__(256) svq_gemm(const double* __restrict__ a, int64_t sam, int64_t sak,
                                                const double* __restrict__ b, int64_t sbk, int64_t sbn,
                                                double* __restrict__ c, int64_t ldc, int M, int N, int K) {
  __shared__ double as[32][17];
  __shared__ double bs[16][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 8 rows of 32 threads
  const int m0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 32 * 16; i += 256) {
      const int r = i >> 4, kk = i & 15;
      const int m = m0 + r, k = k0 + kk;
      as[r][kk] = (m < M && k < K) ? a[(int64_t)m * sam + (int64_t)k * sak] : 0.0;
      const int kb = i >> 5, nn = i & 31;
      const int kq = k0 + kb, n = n0 + nn;
      bs[kb][nn] = (kq < K && n < N) ? b[(int64_t)kq * sbk + (int64_t)n * sbn] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const double bv = bs[kk][tx];
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] = fma(as[ty + 8 * r][kk], bv, acc[r]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int m = m0 + ty + 8 * r, n = n0 + tx;
    if (m < M && n < N) c[(int64_t)m * ldc + n] = acc[r];
  }
}

// low[i][k] /= d[k]
__global__ void svq_div_cols(double* __restrict__ low, const double* __restrict__ d, int64_t n, int64_t k) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n * k) low[i] /= d[i % k];
}

// rb = bf16(W - low), rounded once from float64
__global__ void svq_residual(const uint16_t* __restrict__ w, const double* __restrict__ low,
                             uint16_t* __restrict__ rb, int64_t n, int64_t k) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n * k) rb[i] = f64_to_bf16_rne(bf16_to_f64(w[i]) - low[i]);
}

// deq[row][256 g + i] = (R (codes * scales))[i] for every 256-block of a row (R =
// H / 16 symmetric, so it is its own inverse), or codes * scales without rotation.
// One CTA of 256 threads per (row, block); the four radix-4 stages of H run in
// float64 through shared memory (exact: a block holds code * scale values with at
// most four distinct scales).
__global__ void __launch_bounds__(256) svq_dequant(const uint8_t* __restrict__ q, const float* __restrict__ sc,
                                                   int bits, int scale_group, bool rot, int64_t k,
                                                   double* __restrict__ deq) {
  __shared__ double v[2][256];
  const int64_t row = blockIdx.y;
  const int i = threadIdx.x;
  const int64_t col = (int64_t)blockIdx.x * 256 + i;
  int code;
  if (bits == 4) {
    const uint8_t byte = q[row * (k / 2) + col / 2];
    const int nib = (col & 1) ? (byte >> 4) : (byte & 15);
    code = nib >= 8 ? nib - 16 : nib;
  } else {
    code = (int8_t)q[row * k + col];
  }
  const float s = scale_group ? sc[row * (k / 64) + col / 64] : sc[row];
  double x = (double)code * (double)s;
  if (rot) {
    int cur = 0;
    v[cur][i] = x;
    __syncthreads();
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int stride = 1 << (2 * t);
      const int base = i - ((i / stride) & 3) * stride;
      const double sum = (v[cur][base] + v[cur][base + stride]) + (v[cur][base + 2 * stride] + v[cur][base + 3 * stride]);
      v[cur ^ 1][i] = fma(-2.0, v[cur][i], sum);
      cur ^= 1;
      __syncthreads();
    }
    x = v[cur][i] * 0.0625;
  }
  deq[row * k + col] = x;
}

// part[row] = sum_k ((W - (deq + low)) d)^2 over the row, fixed order
__global__ void __launch_bounds__(256) svq_err_rows(const uint16_t* __restrict__ w, const double* __restrict__ deq,
                                                    const double* __restrict__ low, const double* __restrict__ d,
                                                    int64_t k, double* __restrict__ part) {
  __shared__ double red[256];
  const int64_t row = blockIdx.x;
  double s = 0.0;
  for (int64_t c = threadIdx.x; c < k; c += 256) {
    const int64_t i = row * k + c;
    const double e = (bf16_to_f64(w[i]) - (deq[i] + low[i])) * d[c];
    s = fma(e, e, s);
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int off = 128; off > 0; off >>= 1) {
    if ((int)threadIdx.x < off) red[threadIdx.x] += red[threadIdx.x + off];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[row] = red[0];
}

// ------------------------------------------------------------------ host algebra
// Thin Householder QR of y (m x n, row-major, m >= n): q (m x n) with orthonormal
// columns spanning y's columns.
void householder_q(const std::vector<double>& y, int m, int n, std::vector<double>& q) {
  std::vector<double> a(y);
  std::vector<std::vector<double>> vs(n);
  for (int j = 0; j < n; ++j) {
    double norm = 0.0;
    for (int i = j; i < m; ++i) norm += a[(size_t)i * n + j] * a[(size_t)i * n + j];
    norm = std::sqrt(norm);
    std::vector<double> v(m - j);
    for (int i = j; i < m; ++i) v[i - j] = a[(size_t)i * n + j];
    const double alpha = v[0] >= 0 ? -norm : norm;
    v[0] -= alpha;
    double vn = 0.0;
    for (double t : v) vn += t * t;
    if (vn > 0.0) {
      for (int c = j; c < n; ++c) {
        double dot = 0.0;
        for (int i = j; i < m; ++i) dot += v[i - j] * a[(size_t)i * n + c];
        const double f = 2.0 * dot / vn;
        for (int i = j; i < m; ++i) a[(size_t)i * n + c] -= f * v[i - j];
      }
    }
    vs[j] = std::move(v);
  }
  // Q = H_0 H_1 ... H_{n-1} applied to the first n columns of I
  q.assign((size_t)m * n, 0.0);
  for (int j = 0; j < n; ++j) q[(size_t)j * n + j] = 1.0;
  for (int j = n - 1; j >= 0; --j) {
    const std::vector<double>& v = vs[j];
    double vn = 0.0;
    for (double t : v) vn += t * t;
    if (vn == 0.0) continue;
    for (int c = 0; c < n; ++c) {
      double dot = 0.0;
      for (int i = j; i < m; ++i) dot += v[i - j] * q[(size_t)i * n + c];
      const double f = 2.0 * dot / vn;
      for (int i = j; i < m; ++i) q[(size_t)i * n + c] -= f * v[i - j];
    }
  }
}

// SVD of b (p x k, row-major, p <= k) by one-sided Jacobi on the columns of b^T:
// b = ub diag(s) vt with ub (p x p), s (p, descending), vt (p x k).
void jacobi_svd(const std::vector<double>& b, int p, int k, std::vector<double>& ub, std::vector<double>& s,
                std::vector<double>& vt) {
  std::vector<double> g((size_t)p * k);   // column c of b^T stored contiguously: g[c][.] = b[c][.]
  std::copy(b.begin(), b.end(), g.begin());
  std::vector<double> j((size_t)p * p, 0.0);   // accumulated rotations, column-major j[c][r]
  for (int c = 0; c < p; ++c) j[(size_t)c * p + c] = 1.0;
  for (int sweep = 0; sweep < 60; ++sweep) {
    double off = 0.0;
    for (int a = 0; a < p - 1; ++a)
      for (int c = a + 1; c < p; ++c) {
        double al = 0.0, be = 0.0, ga = 0.0;
        const double* ga_ = &g[(size_t)a * k];
        const double* gc_ = &g[(size_t)c * k];
        for (int t = 0; t < k; ++t) {
          al += ga_[t] * ga_[t];
          be += gc_[t] * gc_[t];
          ga += ga_[t] * gc_[t];
        }
        if (ga == 0.0 || std::fabs(ga) <= 1e-15 * std::sqrt(al * be)) continue;
        off = std::max(off, std::fabs(ga) / std::sqrt(al * be));
        const double zeta = (be - al) / (2.0 * ga);
        const double t = (zeta >= 0 ? 1.0 : -1.0) / (std::fabs(zeta) + std::sqrt(1.0 + zeta * zeta));
        const double cs = 1.0 / std::sqrt(1.0 + t * t), sn = cs * t;
        double* pa = &g[(size_t)a * k];
        double* pc = &g[(size_t)c * k];
        for (int i = 0; i < k; ++i) {
          const double x = pa[i], y = pc[i];
          pa[i] = cs * x - sn * y;
          pc[i] = sn * x + cs * y;
        }
        double* ja = &j[(size_t)a * p];
        double* jc = &j[(size_t)c * p];
        for (int i = 0; i < p; ++i) {
          const double x = ja[i], y = jc[i];
          ja[i] = cs * x - sn * y;
          jc[i] = sn * x + cs * y;
        }
      }
    if (off <= 1e-15) break;
  }
  std::vector<double> sig(p);
  for (int c = 0; c < p; ++c) {
    double n2 = 0.0;
    for (int t = 0; t < k; ++t) n2 += g[(size_t)c * k + t] * g[(size_t)c * k + t];
    sig[c] = std::sqrt(n2);
  }
  std::vector<int> order(p);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return sig[x] > sig[y]; });
  ub.assign((size_t)p * p, 0.0);
  s.assign(p, 0.0);
  vt.assign((size_t)p * k, 0.0);
  for (int o = 0; o < p; ++o) {
    const int c = order[o];
    s[o] = sig[c];
    for (int r = 0; r < p; ++r) ub[(size_t)r * p + o] = j[(size_t)c * p + r];   // b = j diag(s) u_g^T
    if (sig[c] > 0.0)
      for (int t = 0; t < k; ++t) vt[(size_t)o * k + t] = g[(size_t)c * k + t] / sig[c];
  }
}

inline unsigned blocks_for(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

}  // namespace

// Bytes of the device workspace rbd_svdquant_fit takes.
int64_t svdquant_workspace_bytes(int64_t n, int64_t k, int rank, int oversample, int bits, int scale_group) {
  const int64_t p = rank + oversample;
  const int64_t nk = n * k;
  int64_t b = 0;
  auto add = [&](int64_t bytes) { b += (bytes + 255) / 256 * 256; };
  add(nk * 8);                          // A
  add(nk * 8);                          // low
  add(nk * 8);                          // deq
  add(nk * 2);                          // bf16 residual
  add(bits == 4 ? nk / 2 : nk);         // codes of the iterate
  add((scale_group ? nk / 64 : n) * 4); // scales of the iterate
  add(n * p * 8);                       // Y / A Z
  add(k * p * 8);                       // omega, A^T Q, Z
  add(p * k * 8);                       // Q^T A, V^T
  add(n * p * 8);                       // Q (device copy), U S
  add(k * 8);                           // d
  add(n * 8);                           // per-row errors
  return b;
}

cudaError_t svdquant_fit(const uint16_t* w, int64_t n, int64_t k, int bits, bool rot, int scale_group, int rank,
                         int oversample, int iters, const double* omegas, const double* act_rms, void* q_out,
                         float* scales_out, double* l1, double* l2, double* errs, int* best_out, void* work,
                         cudaStream_t st) {
  const int p = rank + oversample;
  const int64_t nk = n * k;
  char* wp = static_cast<char*>(work);
  auto take = [&](int64_t bytes) {
    char* r = wp;
    wp += (bytes + 255) / 256 * 256;
    return r;
  };
  double* dA = reinterpret_cast<double*>(take(nk * 8));
  double* dLow = reinterpret_cast<double*>(take(nk * 8));
  double* dDeq = reinterpret_cast<double*>(take(nk * 8));
  uint16_t* dRes = reinterpret_cast<uint16_t*>(take(nk * 2));
  uint8_t* dQ = reinterpret_cast<uint8_t*>(take(bits == 4 ? nk / 2 : nk));
  const int64_t nsc = scale_group ? nk / 64 : n;
  float* dSc = reinterpret_cast<float*>(take(nsc * 4));
  double* dY = reinterpret_cast<double*>(take(n * p * 8));
  double* dKp = reinterpret_cast<double*>(take(k * p * 8));
  double* dPk = reinterpret_cast<double*>(take((int64_t)p * k * 8));
  double* dNp = reinterpret_cast<double*>(take(n * p * 8));
  double* dD = reinterpret_cast<double*>(take(k * 8));
  double* dPart = reinterpret_cast<double*>(take(n * 8));
  cudaError_t e;
#define RBD_SVQ_TRY(x)                      \
  do {                                      \
    if ((e = (x)) != cudaSuccess) return e; \
  } while (0)

  // channel weights: activation RMS normalised to mean 1, floored at 0.05; ones without statistics
  std::vector<double> d((size_t)k, 1.0);
  if (act_rms) {
    double mean = 0.0;
    for (int64_t c = 0; c < k; ++c) mean += act_rms[c];
    mean /= (double)k;
    for (int64_t c = 0; c < k; ++c) d[c] = std::max(act_rms[c] / mean, 0.05);
  }
  RBD_SVQ_TRY(cudaMemcpyAsync(dD, d.data(), k * 8, cudaMemcpyHostToDevice, st));

  auto gemm = [&](const double* a, int64_t sam, int64_t sak, const double* b, int64_t sbk, int64_t sbn, double* c,
                  int64_t ldc, int M, int N, int K) {
    svq_gemm<<<dim3(blocks_for(N, 32), blocks_for(M, 32)), 256, 0, st>>>(a, sam, sak, b, sbk, sbn, c, ldc, M, N, K);
    return cudaGetLastError();
  };
  std::vector<double> hY((size_t)n * p), hQ, hZ((size_t)k * p), hB((size_t)p * k), ub, s, vt;
  std::vector<double> us((size_t)n * rank);
  double best_err = 0.0;
  int best = -1;
  const unsigned eb = blocks_for(nk, 256);
  for (int it = 0; it < iters; ++it) {
    // A = (W - deq) d  (W d on the first iterate)
    svq_make_a<<<eb, 256, 0, st>>>(w, it ? dDeq : nullptr, dD, dA, n, k);
    RBD_SVQ_TRY(cudaGetLastError());
    // Y = A Omega, Q = orth(Y)
    RBD_SVQ_TRY(cudaMemcpyAsync(dKp, omegas + (size_t)it * k * p, k * p * 8, cudaMemcpyHostToDevice, st));
    RBD_SVQ_TRY(gemm(dA, k, 1, dKp, p, 1, dY, p, (int)n, p, (int)k));
    RBD_SVQ_TRY(cudaMemcpyAsync(hY.data(), dY, n * p * 8, cudaMemcpyDeviceToHost, st));
    RBD_SVQ_TRY(cudaStreamSynchronize(st));
    householder_q(hY, (int)n, p, hQ);
    // one power iteration: Z = orth(A^T Q), Q = orth(A Z)
    RBD_SVQ_TRY(cudaMemcpyAsync(dNp, hQ.data(), n * p * 8, cudaMemcpyHostToDevice, st));
    RBD_SVQ_TRY(gemm(dA, 1, k, dNp, p, 1, dKp, p, (int)k, p, (int)n));
    RBD_SVQ_TRY(cudaMemcpyAsync(hZ.data(), dKp, k * p * 8, cudaMemcpyDeviceToHost, st));
    RBD_SVQ_TRY(cudaStreamSynchronize(st));
    std::vector<double> z;
    householder_q(hZ, (int)k, p, z);
    RBD_SVQ_TRY(cudaMemcpyAsync(dKp, z.data(), k * p * 8, cudaMemcpyHostToDevice, st));
    RBD_SVQ_TRY(gemm(dA, k, 1, dKp, p, 1, dY, p, (int)n, p, (int)k));
    RBD_SVQ_TRY(cudaMemcpyAsync(hY.data(), dY, n * p * 8, cudaMemcpyDeviceToHost, st));
    RBD_SVQ_TRY(cudaStreamSynchronize(st));
    householder_q(hY, (int)n, p, hQ);
    // B = Q^T A (p x k), its SVD on the host
    RBD_SVQ_TRY(cudaMemcpyAsync(dNp, hQ.data(), n * p * 8, cudaMemcpyHostToDevice, st));
    RBD_SVQ_TRY(gemm(dNp, 1, p, dA, k, 1, dPk, k, p, (int)k, (int)n));
    RBD_SVQ_TRY(cudaMemcpyAsync(hB.data(), dPk, (int64_t)p * k * 8, cudaMemcpyDeviceToHost, st));
    RBD_SVQ_TRY(cudaStreamSynchronize(st));
    jacobi_svd(hB, p, (int)k, ub, s, vt);
    // U = Q ub (first rank columns); low = (U S) V^T / d
    for (int64_t i = 0; i < n; ++i)
      for (int c = 0; c < rank; ++c) {
        double acc = 0.0;
        for (int t = 0; t < p; ++t) acc += hQ[(size_t)i * p + t] * ub[(size_t)t * p + c];
        us[(size_t)i * rank + c] = acc * s[c];
      }
    RBD_SVQ_TRY(cudaMemcpyAsync(dNp, us.data(), n * rank * 8, cudaMemcpyHostToDevice, st));
    RBD_SVQ_TRY(cudaMemcpyAsync(dPk, vt.data(), (int64_t)rank * k * 8, cudaMemcpyHostToDevice, st));
    RBD_SVQ_TRY(gemm(dNp, rank, 1, dPk, k, 1, dLow, k, (int)n, (int)k, rank));
    svq_div_cols<<<eb, 256, 0, st>>>(dLow, dD, n, k);
    RBD_SVQ_TRY(cudaGetLastError());
    // Q, scales of bf16(W - low) in the layer's rotated format; their dequantised value
    svq_residual<<<eb, 256, 0, st>>>(w, dLow, dRes, n, k);
    RBD_SVQ_TRY(cudaGetLastError());
    RBD_SVQ_TRY(launch_rot_quant(dRes, n, k, k, bits, rot, scale_group == 64, bits == 4, false,
                                 reinterpret_cast<int8_t*>(dQ), dSc, st));
    svq_dequant<<<dim3((unsigned)(k / 256), (unsigned)n), 256, 0, st>>>(dQ, dSc, bits, scale_group, rot, k, dDeq);
    RBD_SVQ_TRY(cudaGetLastError());
    // error of this iterate
    svq_err_rows<<<(unsigned)n, 256, 0, st>>>(w, dDeq, dLow, dD, k, dPart);
    RBD_SVQ_TRY(cudaGetLastError());
    std::vector<double> part((size_t)n);
    RBD_SVQ_TRY(cudaMemcpyAsync(part.data(), dPart, n * 8, cudaMemcpyDeviceToHost, st));
    RBD_SVQ_TRY(cudaStreamSynchronize(st));
    double err2 = 0.0;
    for (int64_t i = 0; i < n; ++i) err2 += part[i];
    const double err = std::sqrt(err2);
    errs[it] = err;
    if (best < 0 || err < best_err) {
      best = it;
      best_err = err;
      RBD_SVQ_TRY(cudaMemcpyAsync(q_out, dQ, bits == 4 ? nk / 2 : nk, cudaMemcpyDeviceToDevice, st));
      RBD_SVQ_TRY(cudaMemcpyAsync(scales_out, dSc, nsc * 4, cudaMemcpyDeviceToDevice, st));
      // L1 = (V^T / d)^T sqrt(S): [k][rank]; L2 = sqrt(S) U^T: [rank][n]
      for (int64_t c = 0; c < k; ++c)
        for (int r = 0; r < rank; ++r) l1[(size_t)c * rank + r] = vt[(size_t)r * k + c] / d[c] * std::sqrt(s[r]);
      for (int r = 0; r < rank; ++r) {
        const double root = std::sqrt(s[r]);
        for (int64_t i = 0; i < n; ++i) {
          double u = 0.0;
          for (int t = 0; t < p; ++t) u += hQ[(size_t)i * p + t] * ub[(size_t)t * p + r];
          l2[(size_t)r * n + i] = root * u;
        }
      }
    }
  }
  if (best_out) *best_out = best;
  RBD_SVQ_TRY(cudaStreamSynchronize(st));
#undef RBD_SVQ_TRY
  return cudaSuccess;
}

}  // namespace rbd
