// Output-error variant of SLiM-Quant (SLiM^O; SLiM rebuttal, "Output Error
// Minimization in SLiM-Quant"): the weights of the ~1% most salient input
// channels are scaled up by a factor before compression and the matching
// activations scaled down by it at run time, so W' x' = W x before
// compression while the salient channels get a finer quantisation grid.
//
// Packer side (one-time, off the forward path):
//   k_sal_partial  fp64 sums of |w| over blocks of 64 rows, per column
//   k_sal_total    column sums (block sums in order) times the activation
//                  statistic: the saliency of each channel
//   k_sal_rank     rank of each channel (saliency descending, ties to the
//                  lower index) by counting, flag the first m
//   k_sal_compact  ascending list of the flagged channels -> SALIENT plane
//   k_sal_scale_w  W' = W with the flagged columns times 2^e, fp32 (exact),
//                  which the rest of the packer then encodes
// Forward side:
//   k_salient_x    x' = x with the listed channels times 2^-e, into the
//                  workspace; PDL-chained, it reads x only after the
//                  preceding kernel completed.
// The summation order is the one the format specification fixes, so the
// selection is bit-exact with a CPU restatement of the same definition.
#include "common.cuh"
#include "kernels.h"

namespace cql {
namespace {

constexpr int kSalRows = 64;       // rows per partial sum
constexpr int kRankTile = 2048;    // saliencies staged in shared memory per step

CQL_DEV double w_abs64(const void* W, int wdt, uint64_t idx) {
  const float v = wdt == CQL_DT_BF16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(W)[idx])
                                     : reinterpret_cast<const float*>(W)[idx];
  return fabs((double)v);
}

// grid (ceil(K / 256), N / 64): thread = (row block, column)
__global__ void __launch_bounds__(256) k_sal_partial(const void* W, int wdt, int K, double* partial) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= K) return;
  const uint64_t base = (uint64_t)blockIdx.y * kSalRows * (uint64_t)K + (uint64_t)c;
  double s = 0.0;
#pragma unroll 8
  for (int i = 0; i < kSalRows; ++i) s = __dadd_rn(s, w_abs64(W, wdt, base + (uint64_t)i * K));
  partial[(uint64_t)blockIdx.y * K + c] = s;
}

__global__ void __launch_bounds__(256) k_sal_total(const double* partial, int nblk, int K, const float* act,
                                                   double* sal) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= K) return;
  double s = 0.0;
  for (int b = 0; b < nblk; ++b) s = __dadd_rn(s, partial[(uint64_t)b * K + c]);
  sal[c] = __dmul_rn((double)act[c], s);
}

// flag[c] = 1 when fewer than m channels precede c in the order (saliency
// descending, index ascending)
__global__ void __launch_bounds__(256) k_sal_rank(const double* sal, int K, int m, uint8_t* flag) {
  __shared__ double tile[kRankTile];
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const double me = c < K ? sal[c] : 0.0;
  int before = 0;
  for (int t0 = 0; t0 < K; t0 += kRankTile) {
    const int n = min(kRankTile, K - t0);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) tile[i] = sal[t0 + i];
    __syncthreads();
    for (int i = 0; i < n; ++i) {
      const double v = tile[i];
      before += (v > me || (v == me && t0 + i < c)) ? 1 : 0;
    }
  }
  if (c < K) flag[c] = before < m ? 1 : 0;
}

// one block of 1024 threads: thread t owns columns [t * per, (t + 1) * per)
__global__ void __launch_bounds__(1024) k_sal_compact(const uint8_t* flag, int K, int m, uint16_t* list,
                                                      uint32_t* err) {
  __shared__ int cnt[1024];
  const int per = (K + 1023) / 1024;
  const int c0 = min(K, threadIdx.x * per), c1 = min(K, c0 + per);
  int n = 0;
  for (int c = c0; c < c1; ++c) n += flag[c];
  cnt[threadIdx.x] = n;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {        // inclusive scan (Hillis-Steele)
    const int v = threadIdx.x >= off ? cnt[threadIdx.x - off] : 0;
    __syncthreads();
    cnt[threadIdx.x] += v;
    __syncthreads();
  }
  int pos = cnt[threadIdx.x] - n;
  for (int c = c0; c < c1; ++c)
    if (flag[c]) {
      if (CQL_IN(err, pos, m, 521)) list[pos] = (uint16_t)c;
      ++pos;
    }
}

__global__ void __launch_bounds__(256) k_sal_scale_w(const void* W, int wdt, uint64_t total, int K,
                                                     const uint8_t* flag, float factor, float* out) {
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const float v = wdt == CQL_DT_BF16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(W)[i])
                                       : reinterpret_cast<const float*>(W)[i];
    out[i] = flag[i % (uint64_t)K] ? v * factor : v;
  }
}

// grid (ceil(K / 2048), min(batch, 65535)), 256 threads: thread = 8
// consecutive channels (one 16-byte vector) of activation rows blockIdx.y,
// blockIdx.y + gridDim.y, ...  The list is staged before the dependency wait
// (the packed buffer is not written by the preceding kernel); x only after.
__global__ void __launch_bounds__(256) k_salient_x(const uint16_t* list, int m, int K, int batch, int xdt,
                                                   int log2, const uint16_t* x, uint16_t* xs, uint32_t* err) {
  extern __shared__ uint16_t sl[];
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < m; i += blockDim.x) sl[i] = list[i];
  __syncthreads();
  pdl_wait();
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (8 * v >= K) return;
  // first listed channel >= 8 v (binary search in the ascending list)
  int lo = 0, hi = m;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((int)sl[mid] < 8 * v) lo = mid + 1; else hi = mid;
  }
  const bool any = lo < m && (int)sl[lo] < 8 * v + 8;
  const float inv = ldexpf(1.0f, -log2);
  for (int b = blockIdx.y; b < batch; b += gridDim.y) {
    const uint64_t off = (uint64_t)b * K + 8u * (uint32_t)v;
    if (!CQL_IN(err, off + 7, (uint64_t)batch * K, 401)) continue;
    uint4 q = *reinterpret_cast<const uint4*>(x + off);
    if (any) {
      uint16_t h[8];
      memcpy(h, &q, 16);
      for (int j = lo; j < m && (int)sl[j] < 8 * v + 8; ++j) {
        const int e = sl[j] - 8 * v;
        if (!CQL_IN(err, (uint64_t)e, 8, 402)) continue;
        if (xdt == CQL_DT_BF16) {
          h[e] = __bfloat16_as_ushort(__float2bfloat16_rn(bf16_bits_to_f32(h[e]) * inv));
        } else {
          h[e] = __half_as_ushort(__float2half_rn(f16_bits_to_f32(h[e]) * inv));
        }
      }
      memcpy(&q, h, 16);
    }
    *reinterpret_cast<uint4*>(xs + off) = q;
  }
}

}  // namespace

cudaError_t launch_salient_pack(PackParams& p, cudaStream_t st) {
  const int N = p.d.n_out, K = p.d.k_in, m = p.d.salient_channels;
  const int nblk = N / kSalRows;
  k_sal_partial<<<dim3((K + 255) / 256, nblk), 256, 0, st>>>(p.W, p.wdt, K, p.sal_partial);
  k_sal_total<<<(K + 255) / 256, 256, 0, st>>>(p.sal_partial, nblk, K, p.act_absmean, p.sal);
  k_sal_rank<<<(K + 255) / 256, 256, 0, st>>>(p.sal, K, m, p.sal_flag);
  k_sal_compact<<<1, 1024, 0, st>>>(p.sal_flag, K, m, p.salient, p.err);
  const uint64_t total = (uint64_t)N * K;
  const float factor = ldexpf(1.0f, p.d.salient_log2);
  const uint64_t nb = (total + 255) / 256;
  k_sal_scale_w<<<(unsigned)(nb < 148ull * 16 ? nb : 148ull * 16), 256, 0, st>>>(
      p.W, p.wdt, total, K, p.sal_flag, factor, p.w_scaled);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  p.W = p.w_scaled;
  p.wdt = CQL_DT_F32;
  return cudaSuccess;
}

cudaError_t launch_salient_x(const DecodeParams& p, const uint16_t* list, void* xs, cudaStream_t st) {
  const int K = p.d.k_in, m = p.d.salient_channels;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((K / 8 + 255) / 256), (unsigned)(p.batch < 65535 ? p.batch : 65535));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = (size_t)m * 2;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_salient_x, list, m, K, (int)p.batch, (int)p.xdt, (int)p.d.salient_log2,
                            static_cast<const uint16_t*>(p.x), static_cast<uint16_t*>(xs), p.err);
}

}  // namespace cql
