// SLiM-LoRA / Naive-LoRA adapter construction (SLiM review summary,
// "SLIM-LoRA"; rebuttal, "Assumptions in Theoretical Derivations").
//
// The adapters L [N][r], R [r][K] minimise ||F(E - L R)||_F, E = W(') - W_C
// the compression error of a packed layer and F(M) = M diag(xbar) with xbar
// the layer's positive average input magnitude (xbar = 1: Naive-LoRA).  By
// Eckart-Young the optimum is the rank-r truncated SVD of F(E), mapped back
// through F^-1; it is computed here by randomized subspace iteration:
//
//   k_lr_cols      per-column weight factor (SLiM^O) and xbar' (the input
//                  the adapters see: xbar, divided by the factor on salient
//                  channels), both from the SALIENT plane
//   k_lr_residual  Es = F(W' - W_C) in fp32, W_C decoded from the packed
//                  planes (codes, 2:4 / bitmap mask, scales or centroids)
//   k_lr_csr       minus the CSR outliers' share
//   k_lr_rand      Omega [K][p], counter-hashed uniform(-1, 1)
//   k_lr_gemm      Y = Es Omega, Z = Es^T Q, Y = Es Z (fp32 tiles)
//   k_lr_gram / k_lr_chol / k_lr_apply
//                  CholeskyQR2 (Gram and triangular factors in fp64; a pivot
//                  that vanishes drops its direction)
//   k_lr_jacobi    eigen-decomposition of the p x p Gram of Z = Es^T Q
//                  (parallel cyclic Jacobi, one CTA, fp64): its eigenvalues
//                  are the squared singular values of Q^T Es
//   k_lr_final_*   L = Q V_r Sigma_r^(1/2),
//                  R = Sigma_r^(-1/2) (Z V_r)^T diag(xbar')^-1
// p = r + 32 rounded up to 32 (at most min(N, K)), 6 subspace iterations.
// Off the forward path: this runs once per layer, before the final pack.
#include "common.cuh"
#include "kernels.h"

namespace cql {
namespace {

constexpr int kLrIters = 6;

CQL_DEV uint32_t row_bits(const uint8_t* plane, uint32_t row, uint32_t row_bytes, uint32_t bitpos, uint32_t nb) {
  const uint32_t b0 = bitpos >> 3;
  uint32_t v = plane[rit32(row, b0, row_bytes)];
  if (b0 + 1 < row_bytes) v |= (uint32_t)plane[rit32(row, b0 + 1, row_bytes)] << 8;
  return (v >> (bitpos & 7)) & ((1u << nb) - 1u);
}

__global__ void k_lr_cols_init(int K, const float* act, float* colf, float* xbarp) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  colf[k] = 1.0f;
  xbarp[k] = act != nullptr ? act[k] : 1.0f;
}

__global__ void k_lr_cols_salient(const uint16_t* list, int m, int log2, bool weighted, float* colf, float* xbarp) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= m) return;
  const int c = list[i];
  colf[c] = ldexpf(1.0f, log2);
  if (weighted) xbarp[c] = ldexpf(xbarp[c], -log2);
}

// grid (N, K / 128), 32 threads: the warp decodes row n, columns
// [128 G, 128 G + 128), lane = 4 consecutive columns (one 2:4 group)
__global__ void k_lr_residual(DecodeParams p, const void* W, int wdt, const float* colf, const float* xbarp,
                              float* Es) {
  const uint32_t n = blockIdx.x, G = blockIdx.y, lane = threadIdx.x;
  const int K = p.d.k_in;
  const uint32_t c0 = 128u * G + 4u * lane;
  const int bits = codec_bits(p.d.codec);
  const bool lut = codec_is_lut(p.d.codec);
  int j[4] = {-1, -1, -1, -1};
  if (p.d.mask == CQL_MASK_2_4) {
    const uint32_t nib = row_bits(p.meta, n, p.rb.meta, c0, 4);
    const uint32_t i0 = nib & 3u, i1 = nib >> 2;
    j[i0] = (int)(c0 / 2);
    j[i1] = (int)(c0 / 2) + 1;
  } else if (p.d.mask == CQL_MASK_BITMAP50) {
    const uint32_t b4 = row_bits(p.meta, n, p.rb.meta, c0, 4);
    const uint32_t cnt = __popc(b4);
    uint32_t incl = cnt;                                  // inclusive warp scan of the kept counts
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if ((int)lane >= o) incl += v;
    }
    uint32_t run = ldg_u16(p.voff + rit32(n, 2u * G, p.rb.voff)) + incl - cnt;
    for (int t = 0; t < 4; ++t)
      if ((b4 >> t) & 1u) j[t] = (int)run++;
  } else {
    for (int t = 0; t < 4; ++t) j[t] = (int)(c0 + t);
  }
  const float sc = lut ? 0.0f : f16_bits_to_f32(ldg_u16(p.scales + rit32(n, 2u * G, p.rb.scales)));
  for (int t = 0; t < 4; ++t) {
    const uint32_t c = c0 + t;
    double wc = 0.0;
    if (j[t] >= 0) {
      const uint32_t u = row_bits(p.values, n, p.rb.values, (uint32_t)(bits * j[t]), (uint32_t)bits);
      wc = lut ? (double)f16_bits_to_f32(ldg_u16(p.scales + rit32(n, 2u * u, p.rb.scales)))
               : (double)((int)u - (1 << (bits - 1))) * (double)sc;
    }
    const uint64_t idx = (uint64_t)n * K + c;
    const double w = (double)(wdt == CQL_DT_BF16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(W)[idx])
                                                 : reinterpret_cast<const float*>(W)[idx]) *
                     (double)colf[c];
    Es[idx] = (float)((w - wc) * (double)xbarp[c]);
  }
}

__global__ void k_lr_csr(DecodeParams p, const float* xbarp, float* Es) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= p.d.n_out) return;
  const int K = p.d.k_in;
  for (int e = p.csr_rowptr[n]; e < p.csr_rowptr[n + 1]; ++e) {
    const int c = p.csr_col[e];
    const uint64_t idx = (uint64_t)n * K + c;
    Es[idx] = (float)((double)Es[idx] - (double)f16_bits_to_f32(p.csr_val[e]) * (double)xbarp[c]);
  }
}

CQL_DEV uint64_t mix64(uint64_t z) {                  // splitmix64 finaliser
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void k_lr_rand(uint64_t count, float* out) {
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = (float)((double)(mix64(i) >> 11) * 0x1.0p-52 - 1.0);
}

// out[rows][p] = A M: A = Es [N][K] (TRANS false: rows = N, inner = K) or
// Es^T (TRANS true: rows = K, inner = N); M [inner][p].  64 x 32 output
// tile per 256-thread block, 32-deep inner steps; rows, inner multiples of
// 64 and 32, p a multiple of 32.
template <bool TRANS>
__global__ void __launch_bounds__(256) k_lr_gemm(const float* Es, int N, int K, const float* M, int p, float* out) {
  __shared__ float As[32][65];                     // [t][i]
  __shared__ float Ms[32][33];                     // [t][j]
  const int tid = threadIdx.x;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 32;
  const int inner = TRANS ? N : K;
  const int ti = tid & 15, tj = tid >> 4;          // 16 x 16 threads, 4 x 2 outputs each
  float acc[4][2] = {};
  for (int t0 = 0; t0 < inner; t0 += 32) {
    for (int e = tid; e < 64 * 32; e += 256) {
      int i, t;
      float v;
      if (TRANS) {                                 // A(i, t) = Es[t0 + t][i0 + i]: coalesced along i
        i = e & 63; t = e >> 6;
        v = Es[(uint64_t)(t0 + t) * K + i0 + i];
      } else {                                     // A(i, t) = Es[i0 + i][t0 + t]: coalesced along t
        t = e & 31; i = e >> 5;
        v = Es[(uint64_t)(i0 + i) * K + t0 + t];
      }
      As[t][i] = v;
    }
    for (int e = tid; e < 32 * 32; e += 256) {
      const int jj = e & 31, t = e >> 5;
      Ms[t][jj] = M[(uint64_t)(t0 + t) * p + j0 + jj];
    }
    __syncthreads();
#pragma unroll 8
    for (int t = 0; t < 32; ++t) {
      float a[4], b[2];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = As[t][ti + 16 * u];
#pragma unroll
      for (int v = 0; v < 2; ++v) b[v] = Ms[t][tj + 16 * v];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 2; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 2; ++v) out[(uint64_t)(i0 + ti + 16 * u) * p + j0 + tj + 16 * v] = acc[u][v];
}

// G[p][p] = X^T X (fp64), X [rows][p]; block (32 x 32 threads) per 32 x 32 tile
__global__ void __launch_bounds__(1024) k_lr_gram(const float* X, int rows, int p, double* G) {
  __shared__ float xi[32][33], xj[32][33];
  const int a = threadIdx.x, b = threadIdx.y;
  const int I = blockIdx.y * 32, J = blockIdx.x * 32;
  double acc = 0.0;
  for (int r0 = 0; r0 < rows; r0 += 32) {
    xi[b][a] = r0 + b < rows ? X[(uint64_t)(r0 + b) * p + I + a] : 0.0f;
    xj[b][a] = r0 + b < rows ? X[(uint64_t)(r0 + b) * p + J + a] : 0.0f;
    __syncthreads();
#pragma unroll 8
    for (int r = 0; r < 32; ++r) acc += (double)xi[r][b] * (double)xj[r][a];
    __syncthreads();
  }
  G[(uint64_t)(I + b) * p + J + a] = acc;
}

// One CTA: upper Cholesky factor U of G (U^T U = G) in place of Ri's upper
// triangle, then Ri = U^-1.  A pivot below tol drops its direction (its row
// of U and of U^-1 are zero).  Scratch: U [p][p] in 'U'.
__global__ void __launch_bounds__(1024) k_lr_chol(const double* G, int p, double* U, double* Ri) {
  __shared__ double red[32];
  __shared__ double piv;
  const int tid = threadIdx.x, nt = blockDim.x;
  double dmax = 0.0;
  for (int i = 0; i < p; ++i) dmax = fmax(dmax, G[(uint64_t)i * p + i]);
  const double tol = 1e-13 * dmax;
  for (int e = tid; e < p * p; e += nt) U[e] = 0.0;
  __syncthreads();
  for (int j = 0; j < p; ++j) {
    double s = 0.0;
    for (int t = tid; t < j; t += nt) s += U[(uint64_t)t * p + j] * U[(uint64_t)t * p + j];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
    if ((tid & 31) == 0) red[tid >> 5] = s;
    __syncthreads();
    if (tid == 0) {
      double tot = 0.0;
      for (int w = 0; w < (nt + 31) / 32; ++w) tot += red[w];
      const double d = G[(uint64_t)j * p + j] - tot;
      piv = d > tol ? sqrt(d) : 0.0;
      U[(uint64_t)j * p + j] = piv;
    }
    __syncthreads();
    const double dj = piv;
    for (int i = j + 1 + tid; i < p; i += nt) {
      double v = 0.0;
      if (dj > 0.0) {
        v = G[(uint64_t)j * p + i];
        for (int t = 0; t < j; ++t) v -= U[(uint64_t)t * p + j] * U[(uint64_t)t * p + i];
        v /= dj;
      }
      U[(uint64_t)j * p + i] = v;
    }
    __syncthreads();
  }
  // Ri = U^-1, column c by back substitution (thread per column)
  for (int c = tid; c < p; c += nt) {
    for (int i = p - 1; i >= 0; --i) {
      double v = 0.0;
      const double uii = U[(uint64_t)i * p + i];
      if (uii > 0.0) {
        v = i == c ? 1.0 : 0.0;
        for (int t = i + 1; t <= c; ++t) v -= U[(uint64_t)i * p + t] * Ri[(uint64_t)t * p + c];
        v /= uii;
      }
      Ri[(uint64_t)i * p + c] = i <= c ? v : 0.0;
    }
  }
}

// Y[r][c] = sum_{i <= c} X[r][i] Ri[i][c]
__global__ void k_lr_apply(const float* X, int rows, int p, const double* Ri, float* Y) {
  const uint64_t e = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (uint64_t)rows * p) return;
  const uint64_t r = e / p;
  const int c = (int)(e % p);
  double v = 0.0;
  for (int i = 0; i <= c; ++i) v += (double)X[r * p + i] * Ri[(uint64_t)i * p + c];
  Y[e] = (float)v;
}

// One CTA: C (p x p, symmetric, fp64, in place) -> diagonal by parallel
// cyclic Jacobi (round-robin pairing, p even); V accumulates the rotations.
// Then the r largest eigenvalues (descending, ties to the lower index):
// ord[i], sig[i] = sqrt(max(lambda, 0)).
__global__ void __launch_bounds__(1024) k_lr_jacobi(double* C, double* V, int p, int r, int* ord, double* sig) {
  __shared__ int perm[512];
  __shared__ double cs[256], sn[256];
  __shared__ double red[32];
  __shared__ int stop;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int h = p / 2;
  for (int e = tid; e < p * p; e += nt) V[e] = (e / p == e % p) ? 1.0 : 0.0;
  for (int i = tid; i < p; i += nt) perm[i] = i;
  if (tid == 0) stop = 0;
  __syncthreads();
  for (int sweep = 0; sweep < 30; ++sweep) {
    // convergence: off-diagonal mass against the diagonal's
    double off = 0.0, dia = 0.0;
    for (int e = tid; e < p * p; e += nt) {
      const double v = C[e];
      if (e / p == e % p) dia += v * v; else off += v * v;
    }
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_down_sync(0xffffffffu, off, o);
      dia += __shfl_down_sync(0xffffffffu, dia, o);
    }
    if ((tid & 31) == 0) red[tid >> 5] = off;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < nt / 32; ++w) t += red[w];
      red[0] = t;
    }
    __syncthreads();
    const double off_tot = red[0];
    __syncthreads();
    if ((tid & 31) == 0) red[tid >> 5] = dia;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < nt / 32; ++w) t += red[w];
      stop = off_tot <= 1e-28 * t;
    }
    __syncthreads();
    if (stop) break;
    for (int step = 0; step < p - 1; ++step) {
      for (int q = tid; q < h; q += nt) {
        const int a = perm[q], b = perm[p - 1 - q];
        const double app = C[(uint64_t)a * p + a], aqq = C[(uint64_t)b * p + b], apq = C[(uint64_t)a * p + b];
        double c = 1.0, s = 0.0;
        if (fabs(apq) > 1e-300) {
          const double th = (aqq - app) / (2.0 * apq);
          const double t = (th >= 0.0 ? 1.0 : -1.0) / (fabs(th) + sqrt(th * th + 1.0));
          c = 1.0 / sqrt(t * t + 1.0);
          s = t * c;
        }
        cs[q] = c;
        sn[q] = s;
      }
      __syncthreads();
      for (int e = tid; e < h * p; e += nt) {        // rows a, b of each pair
        const int q = e / p, col = e % p;
        const int a = perm[q], b = perm[p - 1 - q];
        const double x = C[(uint64_t)a * p + col], y = C[(uint64_t)b * p + col];
        C[(uint64_t)a * p + col] = cs[q] * x - sn[q] * y;
        C[(uint64_t)b * p + col] = sn[q] * x + cs[q] * y;
      }
      __syncthreads();
      for (int e = tid; e < h * p; e += nt) {        // columns a, b (C and V)
        const int q = e / p, row = e % p;
        const int a = perm[q], b = perm[p - 1 - q];
        const double x = C[(uint64_t)row * p + a], y = C[(uint64_t)row * p + b];
        C[(uint64_t)row * p + a] = cs[q] * x - sn[q] * y;
        C[(uint64_t)row * p + b] = sn[q] * x + cs[q] * y;
        const double vx = V[(uint64_t)row * p + a], vy = V[(uint64_t)row * p + b];
        V[(uint64_t)row * p + a] = cs[q] * vx - sn[q] * vy;
        V[(uint64_t)row * p + b] = sn[q] * vx + cs[q] * vy;
      }
      __syncthreads();
      if (tid == 0) {                                // circle method: rotate positions 1..p-1
        const int last = perm[p - 1];
        for (int i = p - 1; i > 1; --i) perm[i] = perm[i - 1];
        perm[1] = last;
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < p; i += nt) perm[i] = 0;         // reused: 1 = already chosen
  __syncthreads();
  if (tid == 0) {
    for (int i = 0; i < r; ++i) {
      int best = -1;
      double bv = 0.0;
      for (int k = 0; k < p; ++k) {
        const double v = C[(uint64_t)k * p + k];
        if (!perm[k] && (best < 0 || v > bv)) { best = k; bv = v; }
      }
      perm[best] = 1;
      ord[i] = best;
      sig[i] = sqrt(fmax(bv, 0.0));
    }
  }
}

// L[n][i] = sqrt(sig_i) sum_j Q[n][j] V[j][ord_i]   (0 when sig_i is negligible)
__global__ void k_lr_final_L(const float* Q, int N, int p, const double* V, const int* ord, const double* sig, int r,
                             float* L) {
  const uint64_t e = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (uint64_t)N * r) return;
  const uint64_t n = e / r;
  const int i = (int)(e % r);
  const double s = sig[i];
  if (!(s > 1e-12 * sig[0])) { L[e] = 0.0f; return; }
  double v = 0.0;
  for (int j = 0; j < p; ++j) v += (double)Q[n * p + j] * V[(uint64_t)j * p + ord[i]];
  L[e] = (float)(v * sqrt(s));
}

// R[i][k] = (sum_j Z[k][j] V[j][ord_i]) / sqrt(sig_i) / xbar'_k
__global__ void k_lr_final_R(const float* Z, int K, int p, const double* V, const int* ord, const double* sig, int r,
                             const float* xbarp, float* R) {
  const uint64_t e = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (uint64_t)K * r) return;
  const int i = (int)(e / K);
  const uint64_t k = e % K;
  const double s = sig[i];
  if (!(s > 1e-12 * sig[0])) { R[e] = 0.0f; return; }
  double v = 0.0;
  for (int j = 0; j < p; ++j) v += (double)Z[k * p + j] * V[(uint64_t)j * p + ord[i]];
  R[e] = (float)(v / sqrt(s) / (double)xbarp[k]);
}

unsigned blocks_for(uint64_t n, int t) { return (unsigned)((n + t - 1) / t); }

}  // namespace

int lora_width(const cql_desc& d) {
  int p = (d.rank + 32 + 31) / 32 * 32;
  const int lim = d.n_out < d.k_in ? d.n_out : d.k_in;
  return p < lim ? p : lim;
}

LoraWorkspace lora_workspace_layout(const cql_desc& d) {
  LoraWorkspace w{};
  const uint64_t N = (uint64_t)d.n_out, K = (uint64_t)d.k_in, p = (uint64_t)lora_width(d);
  uint64_t pos = 0;
  w.es = pos;    pos = align256(pos + N * K * 4);
  w.y = pos;     pos = align256(pos + N * p * 4);
  w.y2 = pos;    pos = align256(pos + N * p * 4);
  w.z = pos;     pos = align256(pos + K * p * 4);
  w.z2 = pos;    pos = align256(pos + K * p * 4);
  w.g = pos;     pos = align256(pos + p * p * 8);
  w.u = pos;     pos = align256(pos + p * p * 8);
  w.ri = pos;    pos = align256(pos + p * p * 8);
  w.v = pos;     pos = align256(pos + p * p * 8);
  w.sig = pos;   pos = align256(pos + p * 8);
  w.ord = pos;   pos = align256(pos + p * 4);
  w.colf = pos;  pos = align256(pos + K * 4);
  w.xbarp = pos; pos = align256(pos + K * 4);
  w.total = pos;
  return w;
}

// X [rows][p] -> orthonormal columns (CholeskyQR, twice), result in X
static cudaError_t orthonormalise(float* X, float* tmp, int rows, int p, double* G, double* U, double* Ri,
                                  cudaStream_t st) {
  for (int round = 0; round < 2; ++round) {
    k_lr_gram<<<dim3(p / 32, p / 32), dim3(32, 32), 0, st>>>(X, rows, p, G);
    k_lr_chol<<<1, 1024, 0, st>>>(G, p, U, Ri);
    k_lr_apply<<<blocks_for((uint64_t)rows * p, 256), 256, 0, st>>>(X, rows, p, Ri, tmp);
    const cudaError_t e = cudaMemcpyAsync(X, tmp, (size_t)rows * p * 4, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_build_adapters(const DecodeParams& p, const void* W, int wdt, const float* act,
                                  const uint16_t* salient, uint8_t* ws, float* L, float* R, cudaStream_t st) {
  const cql_desc& d = p.d;
  const int N = d.n_out, K = d.k_in, r = d.rank, P = lora_width(d);
  const LoraWorkspace lw = lora_workspace_layout(d);
  float* Es = reinterpret_cast<float*>(ws + lw.es);
  float* Y = reinterpret_cast<float*>(ws + lw.y);
  float* Y2 = reinterpret_cast<float*>(ws + lw.y2);
  float* Z = reinterpret_cast<float*>(ws + lw.z);
  float* Z2 = reinterpret_cast<float*>(ws + lw.z2);
  double* G = reinterpret_cast<double*>(ws + lw.g);
  double* U = reinterpret_cast<double*>(ws + lw.u);
  double* Ri = reinterpret_cast<double*>(ws + lw.ri);
  double* V = reinterpret_cast<double*>(ws + lw.v);
  double* sig = reinterpret_cast<double*>(ws + lw.sig);
  int* ord = reinterpret_cast<int*>(ws + lw.ord);
  float* colf = reinterpret_cast<float*>(ws + lw.colf);
  float* xbarp = reinterpret_cast<float*>(ws + lw.xbarp);

  k_lr_cols_init<<<blocks_for(K, 256), 256, 0, st>>>(K, act, colf, xbarp);
  if (d.salient_channels > 0)
    k_lr_cols_salient<<<blocks_for(d.salient_channels, 256), 256, 0, st>>>(salient, d.salient_channels,
                                                                           d.salient_log2, act != nullptr, colf, xbarp);
  k_lr_residual<<<dim3(N, K / 128), 32, 0, st>>>(p, W, wdt, colf, xbarp, Es);
  if (p.csr_rowptr != nullptr) k_lr_csr<<<blocks_for(N, 128), 128, 0, st>>>(p, xbarp, Es);
  k_lr_rand<<<1184, 256, 0, st>>>((uint64_t)K * P, Z);
  // Y = Es Omega; Q = orth(Y)
  k_lr_gemm<false><<<dim3(P / 32, N / 64), 256, 0, st>>>(Es, N, K, Z, P, Y);
  cudaError_t e = orthonormalise(Y, Y2, N, P, G, U, Ri, st);
  for (int it = 0; it < kLrIters && e == cudaSuccess; ++it) {
    k_lr_gemm<true><<<dim3(P / 32, K / 64), 256, 0, st>>>(Es, N, K, Y, P, Z);
    if ((e = orthonormalise(Z, Z2, K, P, G, U, Ri, st)) != cudaSuccess) break;
    k_lr_gemm<false><<<dim3(P / 32, N / 64), 256, 0, st>>>(Es, N, K, Z, P, Y);
    e = orthonormalise(Y, Y2, N, P, G, U, Ri, st);
  }
  if (e != cudaSuccess) return e;
  // Z = Es^T Q (= B^T, B = Q^T Es); C = Z^T Z = B B^T
  k_lr_gemm<true><<<dim3(P / 32, K / 64), 256, 0, st>>>(Es, N, K, Y, P, Z);
  k_lr_gram<<<dim3(P / 32, P / 32), dim3(32, 32), 0, st>>>(Z, K, P, G);
  k_lr_jacobi<<<1, 1024, 0, st>>>(G, V, P, r, ord, sig);
  k_lr_final_L<<<blocks_for((uint64_t)N * r, 256), 256, 0, st>>>(Y, N, P, V, ord, sig, r, L);
  k_lr_final_R<<<blocks_for((uint64_t)K * r, 256), 256, 0, st>>>(Z, K, P, V, ord, sig, r, xbarp, R);
  return cudaGetLastError();
}

}  // namespace cql
