// Device packer: W (+ L, R) -> packed planes, bit-exact with the CPU oracle.
//
// The encoding follows the rules written in include/cql.h:
//   * outliers: global top-floor(f N K) |w| (SqueezeLLM, "Approach":
//     dense-and-sparse decomposition), found by a 4-pass radix select over
//     the 32-bit |w| patterns with ties ranked by linear index;
//   * masks: 2:4 top-2 per 4 columns, or per-row top-K/2 (SLiM rebuttal,
//     "Unstructured vs. 2:4 Sparsity");
//   * symmetric clipped RTN per 128 columns (SLiM review summary,
//     "SLIM-Quant"), or a per-row LUT from interpolated quantiles;
//   * AbsMax int4 adapters in groups of 128 (SLiM, "Low-rank adapter
//     quantization").
// Every real-valued step uses explicitly rounded fp64 intrinsics (no
// contraction), then the binary16 rounding of common.cuh.  The packer is off
// the timed path; it favours plain, checkable code over speed.
#include "common.cuh"
#include "kernels.h"

namespace cql {

// |w| as the bit pattern of an fp32 (monotone in |w| for finite values).
CQL_DEV uint32_t abs_key(const void* W, int wdt, uint64_t idx) {
  if (wdt == CQL_DT_BF16) return ((uint32_t)reinterpret_cast<const uint16_t*>(W)[idx] & 0x7FFFu) << 16;
  return __float_as_uint(reinterpret_cast<const float*>(W)[idx]) & 0x7FFFFFFFu;
}
CQL_DEV float wval(const void* W, int wdt, uint64_t idx) {
  if (wdt == CQL_DT_BF16) return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(W)[idx]);
  return reinterpret_cast<const float*>(W)[idx];
}
CQL_DEV double f16_to_f64(uint16_t b) { return (double)__half2float(__ushort_as_half(b)); }
CQL_DEV uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}
// Range check of an access of `width` bytes at byte j of row i of a
// row-interleaved packed plane: j inside the row and the byte offset inside
// the plane.  Checked build only (CQL_ERR_RANGE with the site, access
// skipped); the constant true otherwise.
CQL_DEV bool plane_in(const PackParams& p, uint64_t i, uint64_t j, uint64_t row_bytes, uint64_t width, int plane,
                      uint32_t site) {
  return CQL_IN(p.err, j + width - 1, row_bytes, site) &&
         CQL_IN(p.err, rit(i, j, row_bytes) + width - 1, p.plane_len[plane], site);
}
// Symmetric RTN code: clamp(rint(w / s), -qmax, qmax), 0 when s == 0.
CQL_DEV int rtn_code(double w, double s, int qmax) {
  if (!(s > 0.0)) return 0;
  double r = rint(__ddiv_rn(w, s));
  r = fmin(fmax(r, (double)-qmax), (double)qmax);
  return (int)r;
}

// ---------------------------------------------------------------------------
// header
// ---------------------------------------------------------------------------
__global__ void k_write_header(HeaderBytes h, uint8_t* packed) {
  const int t = threadIdx.x;
  if (t < (int)(sizeof(h.b) / 8)) reinterpret_cast<uint64_t*>(packed)[t] = h.b[t];
}

// ---------------------------------------------------------------------------
// global top-k selection (outliers)
// ---------------------------------------------------------------------------
__global__ void k_topk_init(TopkState* st, uint32_t* hist, uint32_t want) {
  hist[threadIdx.x] = 0;
  if (threadIdx.x == 0) { st->prefix = 0; st->mask = 0; st->want = want; }
}

__global__ void __launch_bounds__(256) k_topk_hist(const void* W, int wdt, uint64_t total,
                                                   const TopkState* st, uint32_t* hist, int shift) {
  __shared__ uint32_t h[256];
  h[threadIdx.x] = 0;
  __syncthreads();
  const uint32_t prefix = st->prefix, mask = st->mask;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const uint32_t key = abs_key(W, wdt, i);
    if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
  }
  __syncthreads();
  if (h[threadIdx.x]) atomicAdd(&hist[threadIdx.x], h[threadIdx.x]);
}

// Pick the digit holding the want-th largest key; reset the histogram.
__global__ void k_topk_pick(TopkState* st, uint32_t* hist, int shift) {
  if (threadIdx.x != 0) return;
  uint32_t want = st->want, cum = 0;
  int d = 255;
  for (; d > 0; --d) {
    if (cum + hist[d] >= want) break;
    cum += hist[d];
  }
  st->prefix |= (uint32_t)d << shift;
  st->mask |= 255u << shift;
  st->want = want - cum;
  for (int i = 0; i < 256; ++i) hist[i] = 0;
}

__global__ void __launch_bounds__(256) k_topk_tiecount(const void* W, int wdt, uint64_t total,
                                                       const TopkState* st, uint32_t* tiecnt) {
  __shared__ uint32_t ws[8];
  const uint32_t T = st->prefix;
  const uint64_t base = (uint64_t)blockIdx.x * kTopkChunk;
  const uint64_t end = min(base + kTopkChunk, total);
  uint32_t cnt = 0;
  for (uint64_t i = base + threadIdx.x; i < end; i += blockDim.x) cnt += abs_key(W, wdt, i) == T;
  for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t s = 0;
    for (int w = 0; w < 8; ++w) s += ws[w];
    tiecnt[blockIdx.x] = s;
  }
}

// out[0..n] = exclusive prefix sums of in[0..n) (out[n] = total).  One block.
__global__ void __launch_bounds__(1024) k_scan_excl(const uint32_t* in, uint32_t* out, int n) {
  __shared__ uint32_t sums[1024];
  const int t = threadIdx.x;
  const int per = (n + 1023) / 1024;
  const int a = min(n, t * per), b = min(n, a + per);
  uint32_t s = 0;
  for (int i = a; i < b; ++i) s += in[i];
  sums[t] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    uint32_t v = t >= o ? sums[t - o] : 0u;
    __syncthreads();
    sums[t] += v;
    __syncthreads();
  }
  uint32_t run = sums[t] - s;   // exclusive
  for (int i = a; i < b; ++i) {
    out[i] = run;
    run += in[i];
  }
  if (t == 1023) out[n] = sums[1023];
}

// Exclusive rank of `flag` among the block's threads in thread order, and the
// block total.  256 threads.
CQL_DEV uint32_t block_rank256(bool flag, uint32_t* ws, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) ws[warp] = __popc(bal);
  __syncthreads();
  uint32_t off = 0, tot = 0;
  for (int w = 0; w < 8; ++w) {
    const uint32_t c = ws[w];
    off += (w < warp) ? c : 0u;
    tot += c;
  }
  __syncthreads();
  *total = tot;
  return off + __popc(bal & lanemask_lt());
}

__global__ void __launch_bounds__(256) k_topk_mark(const void* W, int wdt, uint64_t total,
                                                   const TopkState* st, const uint32_t* tieoff,
                                                   uint32_t* out_bits, uint32_t* err) {
  __shared__ uint32_t ws[8];
  const uint32_t T = st->prefix, want = st->want;
  uint32_t running = tieoff[blockIdx.x];
  const uint64_t base = (uint64_t)blockIdx.x * kTopkChunk;
  const uint64_t end = min(base + kTopkChunk, total);
  for (uint64_t chunk = base; chunk < end; chunk += 256) {
    const uint64_t i = chunk + threadIdx.x;
    const uint32_t key = i < end ? abs_key(W, wdt, i) : 0u;
    const bool eq = i < end && key == T;
    const bool gt = i < end && key > T;
    uint32_t tot;
    const uint32_t rank = running + block_rank256(eq, ws, &tot);
    const bool sel = gt || (eq && rank < want);
    const uint32_t word = __ballot_sync(0xffffffffu, sel);
    const uint64_t w0 = chunk + (threadIdx.x & ~31u);
    if ((threadIdx.x & 31) == 0 && w0 < end && CQL_IN(err, w0 >> 5, total / 32, 501)) out_bits[w0 >> 5] = word;
    running += tot;
  }
}

// Outliers per row (warp per row) -> counts.
__global__ void k_row_popcount(const uint32_t* bits, int n_rows, int words_per_row, uint32_t* counts, uint32_t* err) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  uint32_t c = 0;
  for (int w = lane; w < words_per_row; w += 32) {
    const uint64_t i = (uint64_t)warp * words_per_row + w;
    if (CQL_IN(err, i, (uint64_t)n_rows * words_per_row, 502)) c += __popc(bits[i]);
  }
  for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) counts[warp] = c;
}

// ---------------------------------------------------------------------------
// per-row top-K/2 mask (bitmap50): one block per row, radix select in smem
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_mask_bitmap(PackParams p) {
  __shared__ uint32_t h[256];
  __shared__ uint32_t s_prefix, s_mask, s_want;
  __shared__ uint32_t ws[8];
  const int n = blockIdx.x, K = p.d.k_in, t = threadIdx.x;
  const uint64_t base = (uint64_t)n * K;
  if (t == 0) { s_prefix = 0; s_mask = 0; s_want = (uint32_t)(K / 2); }
  for (int shift = 24; shift >= 0; shift -= 8) {
    h[t] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int c = t; c < K; c += 256) {
      const uint32_t key = abs_key(p.W, p.wdt, base + c);
      if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (t == 0) {
      uint32_t want = s_want, cum = 0;
      int d = 255;
      for (; d > 0; --d) {
        if (cum + h[d] >= want) break;
        cum += h[d];
      }
      s_prefix |= (uint32_t)d << shift;
      s_mask |= 255u << shift;
      s_want = want - cum;
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix, want = s_want;
  uint32_t running = 0;
  for (int chunk = 0; chunk < K; chunk += 256) {
    const int c = chunk + t;
    const uint32_t key = c < K ? abs_key(p.W, p.wdt, base + c) : 0u;
    const bool eq = c < K && key == T;
    const bool gt = c < K && key > T;
    uint32_t tot;
    const uint32_t rank = running + block_rank256(eq, ws, &tot);
    const bool keep = gt || (eq && rank < want);
    const uint32_t word = __ballot_sync(0xffffffffu, keep);
    const int c0 = chunk + (t & ~31);
    if ((t & 31) == 0 && c0 < K && plane_in(p, n, (uint64_t)c0 / 8, p.rb.meta, 4, CQL_PLANE_META, 503))
      *reinterpret_cast<uint32_t*>(p.meta + rit(n, (uint64_t)c0 / 8, p.rb.meta)) = word;
    running += tot;
  }
}

// ---------------------------------------------------------------------------
// bit-stream assembly from one code per byte
// ---------------------------------------------------------------------------
template <int BITS>
CQL_DEV uint32_t stream_byte(const uint8_t* codes, uint32_t ncodes, uint32_t j) {
  if (BITS == 4) {
    const uint32_t lo = 2 * j < ncodes ? codes[2 * j] : 0u;
    const uint32_t hi = 2 * j + 1 < ncodes ? codes[2 * j + 1] : 0u;
    return (lo & 15u) | ((hi & 15u) << 4);
  } else {
    const uint32_t h = j / 3;
    uint32_t v = 0;
    for (int i = 0; i < 8; ++i) {
      const uint32_t ci = 8 * h + i;
      if (ci < ncodes) v |= ((uint32_t)codes[ci] & 7u) << (3 * i);
    }
    return (v >> (8 * (j % 3))) & 0xFFu;
  }
}

CQL_DEV bool outlier_bit(const uint32_t* bits, uint64_t idx) {
  return bits != nullptr && ((bits[idx >> 5] >> (idx & 31)) & 1u);
}

// ---------------------------------------------------------------------------
// uniform codecs: one block (128 threads) per row, thread t <-> column 128g+t
// ---------------------------------------------------------------------------
template <int BITS, int MASK>
__global__ void __launch_bounds__(128, 1) k_codec_uniform(PackParams p) {
  extern __shared__ uint8_t sm[];
  uint8_t* codes = sm;                        // K bytes
  uint8_t* nib = sm + p.d.k_in;               // K/4 bytes (2:4 pattern per group)
  __shared__ float s_wmax[4];
  __shared__ uint32_t s_w[4];
  __shared__ uint32_t s_o[4];
  const int n = blockIdx.x, K = p.d.k_in, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  constexpr int qmax = (1 << (BITS - 1)) - 1;
  const bool has_csr = p.out_bits != nullptr;
  const double alpha = p.alpha_dev != nullptr ? (double)*p.alpha_dev : p.alpha;   // searched or given
  uint32_t kept_run = 0, out_run = 0;
  if (has_csr && CQL_IN(p.err, 4ull * n + 3, p.plane_len[CQL_PLANE_CSR_ROWPTR], 511)) out_run = (uint32_t)p.csr_rowptr[n];
  for (int g = 0; g < K / kGroup; ++g) {
    const int c = g * kGroup + t;
    const uint64_t idx = (uint64_t)n * K + c;
    const float wv = wval(p.W, p.wdt, idx);
    const uint32_t key = __float_as_uint(wv) & 0x7FFFFFFFu;
    const bool outl = outlier_bit(p.out_bits, idx);
    bool keep = true;
    int pat = 0;
    if (MASK == CQL_MASK_2_4) {
      const int q0 = lane & ~3, i = lane & 3;
      int rank = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t kj = __shfl_sync(0xffffffffu, key, q0 + j);
        rank += (kj > key) || (kj == key && j < i);
      }
      keep = rank < 2;
      const uint32_t m4 = (__ballot_sync(0xffffffffu, keep) >> q0) & 15u;
      // kept positions i0 < i1 of the group -> META code i0 | (i1 << 2)
      const int i0 = __ffs(m4) - 1, i1 = 31 - __clz(m4);
      pat = i0 | (i1 << 2);
    } else if (MASK == CQL_MASK_BITMAP50) {
      keep = plane_in(p, n, (uint64_t)c / 8, p.rb.meta, 1, CQL_PLANE_META, 504) &&
             ((p.meta[rit(n, (uint64_t)c / 8, p.rb.meta)] >> (c & 7)) & 1u);
    }
    // group amax over non-outliers
    float a = outl ? 0.0f : fabsf(wv);
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) s_wmax[warp] = a;
    __syncthreads();
    const float amax = fmaxf(fmaxf(s_wmax[0], s_wmax[1]), fmaxf(s_wmax[2], s_wmax[3]));
    const uint16_t s16 = f64_to_f16_bits(__ddiv_rn(__dmul_rn(alpha, (double)amax), (double)qmax));
    const double s = f16_to_f64(s16);
    const int q = rtn_code((double)wv, s, qmax);
    // kept index in the row stream
    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
    const uint32_t ob = __ballot_sync(0xffffffffu, outl);
    if (lane == 0) { s_w[warp] = __popc(kb); s_o[warp] = __popc(ob); }
    __syncthreads();
    uint32_t koff = 0, ktot = 0, ooff = 0, otot = 0;
    for (int w = 0; w < 4; ++w) {
      koff += w < warp ? s_w[w] : 0u;
      ktot += s_w[w];
      ooff += w < warp ? s_o[w] : 0u;
      otot += s_o[w];
    }
    const uint32_t kpos = kept_run + koff + __popc(kb & lanemask_lt());
    if (keep && CQL_IN(p.err, kpos, K, 505)) codes[kpos] = (uint8_t)(q + (1 << (BITS - 1)));
    if (MASK == CQL_MASK_2_4 && (lane & 3) == 0 && CQL_IN(p.err, c >> 2, K / 4, 522)) nib[c >> 2] = (uint8_t)pat;
    if (t == 0) {
      if (plane_in(p, n, 2 * g, p.rb.scales, 2, CQL_PLANE_SCALES, 506))
        *reinterpret_cast<uint16_t*>(p.scales + rit(n, 2 * g, p.rb.scales)) = s16;
      if (MASK == CQL_MASK_BITMAP50 && plane_in(p, n, 2 * g, p.rb.voff, 2, CQL_PLANE_VOFF, 507))
        *reinterpret_cast<uint16_t*>(p.voff + rit(n, 2 * g, p.rb.voff)) = (uint16_t)kept_run;
    }
    const uint32_t opos = out_run + ooff + __popc(ob & lanemask_lt());
    if (has_csr && outl && opos < p.nnz_target &&   // the selection marks exactly nnz entries
        CQL_IN(p.err, 2ull * opos + 1, p.plane_len[CQL_PLANE_CSR_COL], 508) &&
        CQL_IN(p.err, 2ull * opos + 1, p.plane_len[CQL_PLANE_CSR_VAL], 508)) {
      const uint32_t pos = opos;
      const double dense = keep ? __dmul_rn((double)q, s) : 0.0;
      p.csr_col[pos] = (uint16_t)c;
      p.csr_val[pos] = f64_to_f16_bits(__dsub_rn((double)wv, dense));
    }
    kept_run += ktot;
    out_run += otot;
    __syncthreads();
  }
  const uint32_t rbv = p.rb.values;
  for (uint32_t j = t; j < rbv; j += 128)
    if (plane_in(p, n, j, rbv, 1, CQL_PLANE_VALUES, 509))
      p.values[rit(n, j, rbv)] = (uint8_t)stream_byte<BITS>(codes, kept_run, j);
  if (MASK == CQL_MASK_2_4) {
    const uint32_t rbm = p.rb.meta;
    for (uint32_t j = t; j < rbm; j += 128)
      if (plane_in(p, n, j, rbm, 1, CQL_PLANE_META, 510) && CQL_IN(p.err, 2 * j + 1, K / 4, 522))
        p.meta[rit(n, j, rbm)] = (uint8_t)((nib[2 * j] & 15u) | ((nib[2 * j + 1] & 15u) << 4));
  }
}

// ---------------------------------------------------------------------------
// SLiM-Quant clip search (SLiM review summary, "SLIM-Quant"): histogram of
// |w| / amax_g over the entries the codec's error reaches (kept by the mask,
// not outliers), then the expected squared error of clipped RTN at the bin
// centres for every candidate alpha; the least one (ties to the smaller) is
// the layer's alpha.  Bin index and objective follow the format's rule
// operation by operation in fp64 (no contraction), so the choice is
// bit-exact.
// ---------------------------------------------------------------------------
constexpr int kAlphaBins = 1024;
constexpr int kAlphaFirst = 30, kAlphaLast = 100;    // candidates i / 100

template <int MASK>
__global__ void __launch_bounds__(128) k_alpha_hist(PackParams p, unsigned long long* hist) {
  __shared__ uint32_t h[kAlphaBins];
  __shared__ float s_wmax[4];
  const int n = blockIdx.x, K = p.d.k_in, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  for (int b = t; b < kAlphaBins; b += 128) h[b] = 0;
  for (int g = 0; g < K / kGroup; ++g) {
    const int c = g * kGroup + t;
    const uint64_t idx = (uint64_t)n * K + c;
    const float wv = wval(p.W, p.wdt, idx);
    const uint32_t key = __float_as_uint(wv) & 0x7FFFFFFFu;
    const bool outl = outlier_bit(p.out_bits, idx);
    bool keep = true;
    if (MASK == CQL_MASK_2_4) {
      const int q0 = lane & ~3, i = lane & 3;
      int rank = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t kj = __shfl_sync(0xffffffffu, key, q0 + j);
        rank += (kj > key) || (kj == key && j < i);
      }
      keep = rank < 2;
    } else if (MASK == CQL_MASK_BITMAP50) {
      keep = plane_in(p, n, (uint64_t)c / 8, p.rb.meta, 1, CQL_PLANE_META, 512) &&
             ((p.meta[rit(n, (uint64_t)c / 8, p.rb.meta)] >> (c & 7)) & 1u);
    }
    float a = outl ? 0.0f : fabsf(wv);
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) s_wmax[warp] = a;
    __syncthreads();
    const float amax = fmaxf(fmaxf(s_wmax[0], s_wmax[1]), fmaxf(s_wmax[2], s_wmax[3]));
    if (keep && !outl && amax > 0.0f) {
      const double b = floor(__dmul_rn(__ddiv_rn((double)fabsf(wv), (double)amax), (double)kAlphaBins));
      atomicAdd(&h[b < kAlphaBins - 1 ? (int)b : kAlphaBins - 1], 1u);
    }
    __syncthreads();
  }
  for (int b = t; b < kAlphaBins; b += 128)
    if (h[b]) atomicAdd(&hist[b], (unsigned long long)h[b]);
}

// one block: thread i evaluates candidate kAlphaFirst + i over the bins in
// order; thread 0 picks the least, writes it to *alpha and into the packed
// header's descriptor copy (clip_alpha at header byte 28)
__global__ void __launch_bounds__(128) k_alpha_search(const unsigned long long* hist, int bits, float* alpha,
                                                      uint8_t* packed) {
  __shared__ double obj[128];
  const int t = threadIdx.x;
  const int ncand = kAlphaLast - kAlphaFirst + 1;
  const double qmax = (double)((1 << (bits - 1)) - 1);
  if (t < ncand) {
    const double al = (double)__double2float_rn(__ddiv_rn((double)(kAlphaFirst + t), 100.0));
    double s = 0.0;
    for (int b = 0; b < kAlphaBins; ++b) {
      const double c = __ddiv_rn(__dadd_rn((double)b, 0.5), (double)kAlphaBins);
      const double q = fmin(rint(__ddiv_rn(__dmul_rn(c, qmax), al)), qmax);
      const double d = __dsub_rn(c, __ddiv_rn(__dmul_rn(q, al), qmax));
      s = __dadd_rn(s, __dmul_rn((double)hist[b], __dmul_rn(d, d)));
    }
    obj[t] = s;
  }
  __syncthreads();
  if (t == 0) {
    int best = 0;
    for (int i = 1; i < ncand; ++i)
      if (obj[i] < obj[best]) best = i;
    const float a = __double2float_rn(__ddiv_rn((double)(kAlphaFirst + best), 100.0));
    *alpha = a;
    *reinterpret_cast<float*>(packed + 28) = a;
  }
}

// ---------------------------------------------------------------------------
// LUT codecs (no mask): one block (256 threads) per row
// ---------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256, 1) k_codec_lut(PackParams p) {
  extern __shared__ uint8_t sm[];
  const int n = blockIdx.x, K = p.d.k_in, t = threadIdx.x;
  int P = 1;
  while (P < K) P <<= 1;
  float* keys = reinterpret_cast<float*>(sm);                 // P floats
  uint8_t* codes = sm + (size_t)P * 4;                        // K bytes
  __shared__ double cent[16];
  __shared__ uint32_t ws[8];
  __shared__ uint32_t s_nout;
  constexpr int NC = 1 << BITS;
  const uint64_t base = (uint64_t)n * K;
  if (t == 0) s_nout = 0;
  __syncthreads();
  uint32_t nout = 0;
  for (int c = t; c < P; c += 256) {
    float v = __int_as_float(0x7f800000);                      // +inf pads and hides outliers
    if (c < K) {
      const bool o = outlier_bit(p.out_bits, base + c);
      nout += o;
      if (!o) v = wval(p.W, p.wdt, base + c);
    }
    keys[c] = v;
  }
  if (nout) atomicAdd(&s_nout, nout);
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = t; i < P; i += 256) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool up = (i & k) == 0;
          const float a = keys[i], b = keys[ixj];
          if ((a > b) == up) { keys[i] = b; keys[ixj] = a; }
        }
      }
      __syncthreads();
    }
  }
  const int nr = K - (int)s_nout;
  if (t < NC) {
    double c = 0.0;
    if (nr > 0) {
      const double pj = ((double)t + 0.5) / (double)NC;
      const double h = (double)(nr - 1) * pj;                 // exact
      const double fl = floor(h);
      int lo = (int)fl;
      lo = lo < 0 ? 0 : (lo > K - 1 ? K - 1 : lo);
      const double frac = h - fl;                             // exact
      const int hi = min(lo + 1, max(nr - 1, 0));
      const double vlo = (double)keys[lo], vhi = (double)keys[hi];
      c = __dadd_rn(vlo, __dmul_rn(frac, __dsub_rn(vhi, vlo)));
    }
    c = __dadd_rn(c, 0.0);                                    // -0 -> +0
    const uint16_t b = f64_to_f16_bits(c);
    cent[t] = f16_to_f64(b);
    if (p.fisher == nullptr && plane_in(p, n, 2 * t, p.rb.scales, 2, CQL_PLANE_SCALES, 513))
      *reinterpret_cast<uint16_t*>(p.scales + rit(n, 2 * t, p.rb.scales)) = b;
  }
  __syncthreads();
  if (p.fisher != nullptr) {
    // SqueezeLLM sensitivity-weighted k-means (Lloyd, from the quantile
    // table): assign every non-outlier value to its nearest centroid (ties to
    // the lower), stop when an assignment repeats, else move each centroid to
    // sum f v / sum f over its members, summed in column order; at most
    // KMEANS iterations; round to fp16 at the end.
    constexpr int kMaxIters = 32;
    uint8_t* prev = codes + K;                                // K more bytes
    for (int it = 0; it < kMaxIters; ++it) {
      bool changed = false;
      for (int c = t; c < K; c += 256) {
        if (outlier_bit(p.out_bits, base + c)) continue;
        const double wv = (double)wval(p.W, p.wdt, base + c);
        uint32_t code = 0;
        double best = fabs(__dsub_rn(wv, cent[0]));
#pragma unroll
        for (int j = 1; j < NC; ++j) {
          const double d = fabs(__dsub_rn(wv, cent[j]));
          if (d < best) { best = d; code = j; }
        }
        if (it > 0 && prev[c] != code) changed = true;
        prev[c] = (uint8_t)code;
      }
      if (it > 0 && !__syncthreads_or(changed)) break;
      __syncthreads();
      if (t < NC) {
        double num = 0.0, den = 0.0;
        for (int c = 0; c < K; ++c) {
          if (prev[c] != t || outlier_bit(p.out_bits, base + c)) continue;
          const double f = (double)p.fisher[base + c];
          num = __dadd_rn(num, __dmul_rn(f, (double)wval(p.W, p.wdt, base + c)));
          den = __dadd_rn(den, f);
        }
        if (den > 0.0) cent[t] = __ddiv_rn(num, den);
      }
      __syncthreads();
    }
    if (t < NC) {
      const uint16_t b = f64_to_f16_bits(__dadd_rn(cent[t], 0.0));
      cent[t] = f16_to_f64(b);
      if (plane_in(p, n, 2 * t, p.rb.scales, 2, CQL_PLANE_SCALES, 513))
        *reinterpret_cast<uint16_t*>(p.scales + rit(n, 2 * t, p.rb.scales)) = b;
    }
    __syncthreads();
  }
  const bool has_csr = p.out_bits != nullptr;
  uint32_t out_run = 0;
  if (has_csr && CQL_IN(p.err, 4ull * n + 3, p.plane_len[CQL_PLANE_CSR_ROWPTR], 511)) out_run = (uint32_t)p.csr_rowptr[n];
  for (int chunk = 0; chunk < K; chunk += 256) {
    const int c = chunk + t;
    uint32_t code = 0;
    double wv = 0.0;
    bool o = false;
    if (c < K) {
      wv = (double)wval(p.W, p.wdt, base + c);
      o = outlier_bit(p.out_bits, base + c);
      double best = fabs(__dsub_rn(wv, cent[0]));
#pragma unroll
      for (int j = 1; j < NC; ++j) {
        const double d = fabs(__dsub_rn(wv, cent[j]));
        if (d < best) { best = d; code = j; }
      }
      codes[c] = (uint8_t)code;
    }
    uint32_t tot;
    const uint32_t r = block_rank256(o, ws, &tot);
    if (has_csr && o && out_run + r < p.nnz_target &&
        CQL_IN(p.err, 2ull * (out_run + r) + 1, p.plane_len[CQL_PLANE_CSR_COL], 514) &&
        CQL_IN(p.err, 2ull * (out_run + r) + 1, p.plane_len[CQL_PLANE_CSR_VAL], 514)) {
      const uint32_t pos = out_run + r;
      p.csr_col[pos] = (uint16_t)c;
      p.csr_val[pos] = f64_to_f16_bits(__dsub_rn(wv, cent[code]));
    }
    out_run += tot;
  }
  __syncthreads();
  const uint32_t rbv = p.rb.values;
  for (uint32_t j = t; j < rbv; j += 256)
    if (plane_in(p, n, j, rbv, 1, CQL_PLANE_VALUES, 515)) p.values[rit(n, j, rbv)] = (uint8_t)stream_byte<BITS>(codes, K, j);
}

// ---------------------------------------------------------------------------
// adapters: AbsMax int4, groups of 128
// ---------------------------------------------------------------------------
// R [r][K]: thread per (row j, group g along K).
__global__ void k_adapter_R(PackParams p) {
  const int K = p.d.k_in, G = K / kGroup;
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= p.d.rank * G) return;
  const int j = id / G, g = id % G;
  const float* v = p.R + (uint64_t)j * K + g * kGroup;
  float amax = 0.0f;
  for (int i = 0; i < kGroup; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint16_t s16 = f64_to_f16_bits(__ddiv_rn((double)amax, 7.0));
  const double s = f16_to_f64(s16);
  for (int i = 0; i < kGroup / 2; ++i) {
    const int q0 = rtn_code((double)v[2 * i], s, 7), q1 = rtn_code((double)v[2 * i + 1], s, 7);
    if (plane_in(p, j, (uint64_t)g * 64 + i, p.rb.r_values, 1, CQL_PLANE_R_VALUES, 517))
      p.r_values[rit(j, (uint64_t)g * 64 + i, p.rb.r_values)] = (uint8_t)((q0 + 8) | ((q1 + 8) << 4));
  }
  if (plane_in(p, j, 2 * g, p.rb.r_scales, 2, CQL_PLANE_R_SCALES, 518))
    *reinterpret_cast<uint16_t*>(p.r_scales + rit(j, 2 * g, p.rb.r_scales)) = s16;
}

// L [N][r]: thread per (row group g along N, column pair jp).
__global__ void k_adapter_L(PackParams p) {
  const int r = p.d.rank, G = p.d.n_out / kGroup, JP = r / 2;
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= G * JP) return;
  const int g = id / JP, jp = id % JP;
  double s[2];
  for (int h = 0; h < 2; ++h) {
    const int j = 2 * jp + h;
    float amax = 0.0f;
    for (int i = 0; i < kGroup; ++i) amax = fmaxf(amax, fabsf(p.L[(uint64_t)(g * kGroup + i) * r + j]));
    const uint16_t s16 = f64_to_f16_bits(__ddiv_rn((double)amax, 7.0));
    if (CQL_IN(p.err, 2 * ((uint64_t)g * r + j) + 1, p.plane_len[CQL_PLANE_L_SCALES], 519))
      p.l_scales[(uint64_t)g * r + j] = s16;
    s[h] = f16_to_f64(s16);
  }
  for (int i = 0; i < kGroup; ++i) {
    const uint64_t row = (uint64_t)g * kGroup + i;
    const int q0 = rtn_code((double)p.L[row * r + 2 * jp], s[0], 7);
    const int q1 = rtn_code((double)p.L[row * r + 2 * jp + 1], s[1], 7);
    if (plane_in(p, row, jp, p.rb.l_values, 1, CQL_PLANE_L_VALUES, 520))
      p.l_values[rit(row, jp, p.rb.l_values)] = (uint8_t)((q0 + 8) | ((q1 + 8) << 4));
  }
}

// ---------------------------------------------------------------------------
// host-side launch sequence
// ---------------------------------------------------------------------------
// Last operation of every pack: an empty kernel launched with an ordinary
// (full) stream dependency.  The forward's first kernel is launched
// programmatically dependent on whatever kernel precedes it and reads the
// packed weights before waiting for that kernel; with this kernel last, every
// byte of the packed buffer was written before that kernel even started.
__global__ void k_pack_done() {}

static cudaError_t set_smem(const void* f, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_pack(const PackParams& p0, const HeaderBytes& hdr, uint64_t total_bytes,
                        cudaStream_t st) {
  PackParams p = p0;
  const int N = p.d.n_out, K = p.d.k_in;
  cudaError_t e = cudaMemsetAsync(p.packed, 0, total_bytes, st);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.err, 0, 8, st)) != cudaSuccess) return e;
  k_write_header<<<1, 64, 0, st>>>(hdr, p.packed);
  if (p.d.salient_channels > 0 && (e = launch_salient_pack(p, st)) != cudaSuccess) return e;

  const uint64_t total = (uint64_t)N * K;
  if (p.nnz_target > 0) {
    k_topk_init<<<1, 256, 0, st>>>(p.topk_state, p.topk_hist, (uint32_t)p.nnz_target);
    for (int shift = 24; shift >= 0; shift -= 8) {
      k_topk_hist<<<1184, 256, 0, st>>>(p.W, p.wdt, total, p.topk_state, p.topk_hist, shift);
      k_topk_pick<<<1, 32, 0, st>>>(p.topk_state, p.topk_hist, shift);
    }
    const int nblk = (int)((total + kTopkChunk - 1) / kTopkChunk);
    k_topk_tiecount<<<nblk, 256, 0, st>>>(p.W, p.wdt, total, p.topk_state, p.topk_tiecnt);
    k_scan_excl<<<1, 1024, 0, st>>>(p.topk_tiecnt, p.topk_tieoff, nblk);
    k_topk_mark<<<nblk, 256, 0, st>>>(p.W, p.wdt, total, p.topk_state, p.topk_tieoff, p.out_bits, p.err);
    k_row_popcount<<<(N * 32 + 255) / 256, 256, 0, st>>>(p.out_bits, N, K / 32, p.row_counts, p.err);
    k_scan_excl<<<1, 1024, 0, st>>>(p.row_counts, reinterpret_cast<uint32_t*>(p.csr_rowptr), N);
  } else {
    p.out_bits = nullptr;
  }
  if (p.d.mask == CQL_MASK_BITMAP50) k_mask_bitmap<<<N, 256, 0, st>>>(p);

  if (codec_is_lut(p.d.codec)) {
    int P = 1;
    while (P < K) P <<= 1;
    const size_t smem = (size_t)P * 4 + K + (p.fisher != nullptr ? K : 0);
    if (p.d.codec == CQL_CODEC_LUT3_ROW) {
      if ((e = set_smem((const void*)k_codec_lut<3>, smem)) != cudaSuccess) return e;
      k_codec_lut<3><<<N, 256, smem, st>>>(p);
    } else {
      if ((e = set_smem((const void*)k_codec_lut<4>, smem)) != cudaSuccess) return e;
      k_codec_lut<4><<<N, 256, smem, st>>>(p);
    }
  } else {
    if (p.alpha_dev != nullptr) {                             // clip_alpha 0: search it
      if ((e = cudaMemsetAsync(p.alpha_hist, 0, kAlphaBins * sizeof(unsigned long long), st)) != cudaSuccess)
        return e;
      if (p.d.mask == CQL_MASK_2_4) k_alpha_hist<CQL_MASK_2_4><<<N, 128, 0, st>>>(p, p.alpha_hist);
      else if (p.d.mask == CQL_MASK_BITMAP50) k_alpha_hist<CQL_MASK_BITMAP50><<<N, 128, 0, st>>>(p, p.alpha_hist);
      else k_alpha_hist<CQL_MASK_NONE><<<N, 128, 0, st>>>(p, p.alpha_hist);
      k_alpha_search<<<1, 128, 0, st>>>(p.alpha_hist, codec_bits(p.d.codec), p.alpha_dev, p.packed);
    }
    const size_t smem = (size_t)K + K / 4;
#define CQL_LAUNCH_UNI(B, M)                                                   \
  do {                                                                         \
    if ((e = set_smem((const void*)k_codec_uniform<B, M>, smem)) != cudaSuccess) return e; \
    k_codec_uniform<B, M><<<N, 128, smem, st>>>(p);                            \
  } while (0)
    const int bits = codec_bits(p.d.codec);
    if (bits == 4) {
      if (p.d.mask == CQL_MASK_2_4) CQL_LAUNCH_UNI(4, CQL_MASK_2_4);
      else if (p.d.mask == CQL_MASK_BITMAP50) CQL_LAUNCH_UNI(4, CQL_MASK_BITMAP50);
      else CQL_LAUNCH_UNI(4, CQL_MASK_NONE);
    } else {
      if (p.d.mask == CQL_MASK_2_4) CQL_LAUNCH_UNI(3, CQL_MASK_2_4);
      else if (p.d.mask == CQL_MASK_BITMAP50) CQL_LAUNCH_UNI(3, CQL_MASK_BITMAP50);
      else CQL_LAUNCH_UNI(3, CQL_MASK_NONE);
    }
#undef CQL_LAUNCH_UNI
  }
  if (p.d.rank > 0) {
    const int nR = p.d.rank * (K / kGroup);
    k_adapter_R<<<(nR + 127) / 128, 128, 0, st>>>(p);
    const int nL = (N / kGroup) * (p.d.rank / 2);
    k_adapter_L<<<(nL + 127) / 128, 128, 0, st>>>(p);
  }
  k_pack_done<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

}  // namespace cql
