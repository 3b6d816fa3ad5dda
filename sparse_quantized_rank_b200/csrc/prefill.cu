// Prefill path (batch > 16): Y = X deq(Q (.) M)^T + X R^T L^T on the 5th-gen
// tensor cores (tcgen05.mma, kind::f16, bf16 operands, fp32 accumulators in
// tensor memory), operands staged by TMA.
//
// Exactness.  A dequantised weight q*s has up to 14 significant bits; rounding
// it to bf16 (8 bits) would cost ~1e-3 of relative error per output, most of
// the 2e-3 budget.  So the GEMM never multiplies by q*s: the tensor cores see
// the integer codes q (exact in bf16) and accumulate one scale group (128
// columns of K) at a time in tensor memory; the epilogue warps multiply each
// group's partial sums by that row's fp32 scale and add them into registers:
//     Y^T[n][t] = sum_g s[n][g] * (sum_{k in g} q[n][k] X[t][k])
// (SLiM-Quant's per-group scale, SLiM review summary "SLIM-Quant").  Weights
// are the MMA's M side (one tensor-memory lane per output row), so the scale
// is a per-thread scalar.  The low-rank term rides as three extra K blocks
// with exact bf16 hi/lo splits, L^ T^T = Lhi Thi + Lhi Tlo + Llo Thi (SLiM
// "Low-rank adapter quantization"; the adapters are AbsMax int4 g128).
//
// Kernels, in stream order:
//   k_pf_dequant_* R (rows padded to 128) as bf16 codes; L^ hi/lo as the
//                  adapter columns; for the layers the sparse GEMM does not
//                  take (int3, no mask) also q as bf16 (zeros where pruned)
//                  [N][K + r3] and fp32 scales [N][K/128]
//   k_pf_gemm      T-pass: T = X R^T (split over K, fp32 atomics)
//   k_pf_tsplit    T -> [Thi | Tlo | Thi] bf16, clears the accumulator
//   main pass      2:4 int4 layers: k_pf_sgemm (prefill_sp.cu, sparse tensor
//                  cores, weights dequantised on chip); others: k_pf_gemm
// Roles inside k_pf_gemm (one CTA per SM, persistent over 128x256 tiles):
//   warp 0        TMA producer (4-stage ring of A 128x64 and B 256x64 tiles)
//   warp 1        tensor-memory allocator and single-thread MMA issuer
//   warps 4..11   epilogue: tcgen05.ld, per-row group scale, stores
// Every mbarrier wait is bounded; on expiry the kernel records
// CQL_ERR_TIMEOUT in the error word and winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace cql {

constexpr int PF_BM = 128;        // weight rows per tile (MMA M, tensor-memory lanes)
constexpr int PF_BN = 256;        // tokens per tile (MMA N)
constexpr int PF_BK = 64;         // K per stage (one 128-byte swizzle row of bf16)
constexpr int PF_STAGES = 4;
constexpr int PF_THREADS = 384;
constexpr int PF_A_BYTES = PF_BM * PF_BK * 2;
constexpr int PF_B_BYTES = PF_BN * PF_BK * 2;

struct PfGemmParams {
  const float* scales;       // [rows][G] fp32
  int rows;                  // weight rows (N, or R rows padded to 128)
  int m;                     // tokens
  int groups;                // K / 128
  int lr_blocks;             // extra K blocks of 64 (main pass), 0 for the T pass
  int k_splits;              // split of the group range (T pass)
  int row_tiles, tok_tiles;
  int mode;                  // 0: store y (out_dt), 1: atomic-add fp32 into out
  void* out;
  int out_dt;
  int ldo;                   // leading dimension of out (elements)
  int valid_rows;            // rows that produce output (N, or rank for the T pass)
  uint32_t idesc;            // tcgen05 instruction descriptor (operand dtype)
  uint32_t* err;
};

// Instruction descriptor: kind::f16, A and B both bf16 (format 1) or both fp16
// (format 0), D = f32, both K-major, M = 128, N = 256.
CQL_HD uint32_t pf_idesc(bool f16) {
  const uint32_t fmt = f16 ? 0u : 1u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(PF_BN >> 3) << 17) | ((uint32_t)(PF_BM >> 4) << 24);
}

// ---------------------------------------------------------------------------
// the GEMM
// ---------------------------------------------------------------------------
struct PfSmem {
  uint8_t a[PF_STAGES][PF_A_BYTES];
  uint8_t b[PF_STAGES][PF_B_BYTES];
  uint64_t full[PF_STAGES], empty[PF_STAGES];
  uint64_t tfull[2], tempty[2];
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(PF_THREADS, 1)
    k_pf_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmT, PfGemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PfSmem& S = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PF_STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.tfull[b], 1);
      mbar_init(&S.tempty[b], 8);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&S.tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  const int n_items = p.row_tiles * p.tok_tiles * p.k_splits;
  const int main_blocks = 2 * p.groups;

  // Register split: the launch gives every thread 168 registers; warpgroup 0
  // (producer, MMA, two idle warps) drops to 40, the two epilogue warpgroups
  // rise to 232: 128 * 40 + 256 * 232 = 384 * 168.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int split = item % p.k_splits, tile = item / p.k_splits;
        const int rt = tile / p.tok_tiles, tt = tile % p.tok_tiles;
        const int g0 = p.groups * split / p.k_splits, g1 = p.groups * (split + 1) / p.k_splits;
        const int nkb = 2 * (g1 - g0) + (split == p.k_splits - 1 ? p.lr_blocks : 0);
        for (int j = 0; j < nkb; ++j, ++it) {
          const int s = it % PF_STAGES;
          if (!mbar_wait(&S.empty[s], ((it / PF_STAGES) & 1) ^ 1)) { ok = false; break; }
          mbar_expect_tx(&S.full[s], PF_A_BYTES + PF_B_BYTES);
          const int kb = 2 * g0 + j;                       // absolute K block (LR blocks follow the main ones)
          tma_load_2d(S.a[s], &tmA, &S.full[s], kb * PF_BK, rt * PF_BM);
          if (kb < main_blocks) {
            tma_load_2d(S.b[s], &tmB, &S.full[s], kb * PF_BK, tt * PF_BN);
          } else {
            tma_load_2d(S.b[s], &tmT, &S.full[s], (kb - main_blocks) * PF_BK, tt * PF_BN);
          }
        }
      }
      if (!ok) set_error(p.err, CQL_ERR_TIMEOUT, 10);
    }
    } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, gc = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int split = item % p.k_splits;
        const int g0 = p.groups * split / p.k_splits, g1 = p.groups * (split + 1) / p.k_splits;
        const int ngroups = (g1 - g0) + (split == p.k_splits - 1 && p.lr_blocks > 0 ? 1 : 0);
        for (int g = 0; g < ngroups && ok; ++g, ++gc) {
          const bool lr = g >= g1 - g0;
          const int nkb = lr ? p.lr_blocks : 2;
          const uint32_t buf = gc & 1;
          if (!mbar_wait(&S.tempty[buf], ((gc >> 1) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + buf * PF_BN;
          for (int j = 0; j < nkb; ++j, ++it) {
            const int s = it % PF_STAGES;
            if (!mbar_wait(&S.full[s], (it / PF_STAGES) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint64_t da = smem_desc_sw128(smem_u32(S.a[s]));
            const uint64_t db = smem_desc_sw128(smem_u32(S.b[s]));
#pragma unroll
            for (int kk = 0; kk < PF_BK / 16; ++kk)
              tc_mma(d, da + 2 * kk, db + 2 * kk, p.idesc, (j > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&S.empty[s]);
          }
          tc_commit(&S.tfull[buf]);
        }
      }
      if (!ok) set_error(p.err, CQL_ERR_TIMEOUT, 11);
    }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 232;");
    // ---------------- epilogue ----------------
    const int q = warp & 3, h = (warp - 4) >> 2;
    uint32_t gc = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int split = item % p.k_splits, tile = item / p.k_splits;
      const int rt = tile / p.tok_tiles, tt = tile % p.tok_tiles;
      const int g0 = p.groups * split / p.k_splits, g1 = p.groups * (split + 1) / p.k_splits;
      const int ngroups = (g1 - g0) + (split == p.k_splits - 1 && p.lr_blocks > 0 ? 1 : 0);
      const int row = rt * PF_BM + 32 * q + lane;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      float s_next = (g0 < g1) ? __ldg(p.scales + (uint64_t)row * p.groups + g0) : 1.0f;
      for (int g = 0; g < ngroups; ++g, ++gc) {
        const float s = s_next;
        const int gn = g0 + g + 1;
        s_next = (g + 1 < g1 - g0) ? __ldg(p.scales + (uint64_t)row * p.groups + gn) : 1.0f;
        const uint32_t buf = gc & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&S.tfull[buf], (gc >> 1) & 1));   // warp-uniform
        if (!ok) break;
        tc_fence_after();
        const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + buf * PF_BN + h * 128;
#pragma unroll
        for (int c = 0; c < 4; c += 2) {
          float v0[32], v1[32];
          tmem_ld32(base + c * 32, v0);
          tmem_ld32(base + (c + 1) * 32, v1);
          tmem_wait_ld(v0);
          reg_after_wait(v1);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            acc[c * 32 + i] = fmaf(s, v0[i], acc[c * 32 + i]);
            acc[(c + 1) * 32 + i] = fmaf(s, v1[i], acc[(c + 1) * 32 + i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.tempty[buf]);
      }
      if (!ok) break;
      if (row < p.valid_rows) {
        const int t0 = tt * PF_BN + h * 128;
        if (p.mode == 0) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (t0 + i < p.m) store_out(p.out, p.out_dt, (uint64_t)(t0 + i) * p.ldo + row, acc[i]);
        } else {
          float* o = reinterpret_cast<float*>(p.out);
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (t0 + i < p.m) atomicAdd(o + (uint64_t)(t0 + i) * p.ldo + row, acc[i]);
        }
      }
    }
    if (!ok && lane == 0) set_error(p.err, CQL_ERR_TIMEOUT, 12);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------------------
// dequantisation to exact bf16 codes (+ scales), adapters as hi/lo splits
// ---------------------------------------------------------------------------
CQL_DEV uint16_t bf16_bits_rn(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }
// 16-bit operand encodings (bf16 unless f16): round to nearest even, and back.
CQL_DEV uint16_t to16(float v, int f16) { return f16 ? __half_as_ushort(__float2half_rn(v)) : bf16_bits_rn(v); }
CQL_DEV float from16(uint16_t b, int f16) { return f16 ? f16_bits_to_f32(b) : bf16_bits_to_f32(b); }
CQL_DEV uint16_t int_to16(int q, int f16) { return to16((float)q, f16); }   // exact for |q| <= 256

// Codes of the layers the sparse GEMM does not take (int3 2:4, no mask) as
// 16-bit integers, zeros where pruned (generic bit extraction).
__global__ void k_pf_dequant_w(DecodeParams p, uint16_t* qbf, int ldq, float* scales, int f16) {
  const int G = p.upr;
  const uint64_t id = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (uint64_t)p.d.n_out * G) return;
  const int g = (int)(id / p.d.n_out), n = (int)(id % p.d.n_out);   // consecutive threads: consecutive rows
  const int bits = codec_bits(p.d.codec);
  const int bias = 1 << (bits - 1);
  const uint32_t mask = (1u << bits) - 1;
  uint16_t outv[128];
  if (p.d.mask == CQL_MASK_2_4) {
    // 64 kept codes (bits each) from bit 64*bits*g of the row stream, 32 pattern nibbles
    const uint64_t bit0 = (uint64_t)64 * bits * g;
    for (int gi = 0; gi < 32; ++gi) {
      const uint32_t mb = p.meta[rit(n, (uint64_t)g * 16 + gi / 2, p.rb.meta)];
      const uint32_t pt = (mb >> (4 * (gi & 1))) & 15u;
      const int i0 = (int)(pt & 3u), i1 = (int)(pt >> 2);
      int qv[2];
      for (int h = 0; h < 2; ++h) {
        const uint64_t bp = bit0 + (uint64_t)bits * (2 * gi + h);
        uint32_t c = 0;
        for (int t = 0; t < bits; ++t) {
          const uint64_t sb = bp + t;
          c |= ((uint32_t)(p.values[rit(n, sb >> 3, p.rb.values)] >> (sb & 7)) & 1u) << t;
        }
        qv[h] = (int)(c & mask) - bias;
      }
      for (int i = 0; i < 4; ++i) outv[4 * gi + i] = 0;
      outv[4 * gi + i0] = int_to16(qv[0], f16);
      outv[4 * gi + i1] = int_to16(qv[1], f16);
    }
  } else {
    const uint64_t bit0 = (uint64_t)128 * bits * g;
    for (int c = 0; c < 128; ++c) {
      const uint64_t bp = bit0 + (uint64_t)bits * c;
      uint32_t code = 0;
      for (int t = 0; t < bits; ++t) {
        const uint64_t sb = bp + t;
        code |= ((uint32_t)(p.values[rit(n, sb >> 3, p.rb.values)] >> (sb & 7)) & 1u) << t;
      }
      outv[c] = int_to16((int)code - bias, f16);
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(qbf + (uint64_t)n * ldq + (uint64_t)g * 128);
  for (int i = 0; i < 16; ++i) {
    uint4 v;
    v.x = outv[8 * i + 0] | ((uint32_t)outv[8 * i + 1] << 16);
    v.y = outv[8 * i + 2] | ((uint32_t)outv[8 * i + 3] << 16);
    v.z = outv[8 * i + 4] | ((uint32_t)outv[8 * i + 5] << 16);
    v.w = outv[8 * i + 6] | ((uint32_t)outv[8 * i + 7] << 16);
    dst[i] = v;
  }
  scales[(uint64_t)n * G + g] = f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(p.scales + rit(n, 2 * g, p.rb.scales)));
}

// L (N x r) as exact bf16 (f16) hi / hi / lo columns [N][r3] (zero padding
// up to r3): a warp per row, lane = column pairs (2j, 2j + 1), each part
// written as one coalesced run of 4-byte pairs.
__global__ void __launch_bounds__(256) k_pf_dequant_l(DecodeParams p, uint16_t* qbf, int ldq, int col0, int r3,
                                                      int f16) {
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (n >= p.d.n_out) return;
  const int r = p.d.rank;
  uint16_t* out = qbf + (uint64_t)n * ldq + col0;
  const uint16_t* sl = p.l_scales + (uint64_t)(n / kGroup) * r;
  for (int j = 2 * lane; j < r; j += 64) {
    const uint32_t byte = p.l_values[rit(n, j / 2, p.rb.l_values)];
    const float l0 = (float)((int)(byte & 15u) - 8) * f16_bits_to_f32(sl[j]);       // exact
    const float l1 = (float)((int)(byte >> 4) - 8) * f16_bits_to_f32(sl[j + 1]);
    const uint32_t h0 = to16(l0, f16), h1 = to16(l1, f16);
    const uint32_t hi = h0 | (h1 << 16);
    const uint32_t lo = (uint32_t)to16(l0 - from16((uint16_t)h0, f16), f16) |
                        ((uint32_t)to16(l1 - from16((uint16_t)h1, f16), f16) << 16);
    *reinterpret_cast<uint32_t*>(out + j) = hi;
    *reinterpret_cast<uint32_t*>(out + r + j) = hi;
    *reinterpret_cast<uint32_t*>(out + 2 * r + j) = lo;
  }
  for (int c = 3 * r + 2 * lane; c < r3; c += 64) *reinterpret_cast<uint32_t*>(out + c) = 0u;
}

// R rows (padded to 128) as bf16 (f16) codes and fp32 scales: a thread per
// 16 codes (8 bytes of a row, one half of a 16-byte piece of the plane).
__global__ void __launch_bounds__(256) k_pf_dequant_r(DecodeParams p, uint16_t* rbf, float* rscales, int rows,
                                                      int f16) {
  const int K = p.d.k_in, G = p.upr;
  const uint64_t id = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (uint64_t)rows * (K / 16)) return;
  const int j = (int)(id / (K / 16)), k0 = (int)(id % (K / 16)) * 16;
  uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  if (j < p.d.rank) {
    const uint2 b8 = *reinterpret_cast<const uint2*>(p.r_values + rit(j, k0 / 2, p.rb.r_values));
    const uint32_t bw[2] = {b8.x, b8.y};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte = (bw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      w[i] = (uint32_t)int_to16((int)(byte & 15u) - 8, f16) | ((uint32_t)int_to16((int)(byte >> 4) - 8, f16) << 16);
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(rbf + (uint64_t)j * K + k0);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  if (k0 % kGroup == 0)
    rscales[(uint64_t)j * G + k0 / kGroup] =
        j < p.d.rank ? f16_bits_to_f32(*reinterpret_cast<const uint16_t*>(p.r_scales + rit(j, 2 * (k0 / kGroup), p.rb.r_scales)))
                     : 0.0f;
}

// T [m][r_pad] fp32 -> [Thi | Tlo | Thi | 0] as bf16 (or fp16) [m][r3]: a
// warp per token row, lane = column pairs.
__global__ void __launch_bounds__(256) k_pf_tsplit(const float* t, int ldt, uint16_t* t3, int r3, int r, int m,
                                                   int f16) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= m) return;
  uint16_t* out = t3 + (uint64_t)row * r3;
  for (int j = 2 * lane; j < r; j += 64) {
    const float2 x = *reinterpret_cast<const float2*>(t + (uint64_t)row * ldt + j);
    const uint32_t h0 = to16(x.x, f16), h1 = to16(x.y, f16);
    const uint32_t hi = h0 | (h1 << 16);
    const uint32_t lo = (uint32_t)to16(x.x - from16((uint16_t)h0, f16), f16) |
                        ((uint32_t)to16(x.y - from16((uint16_t)h1, f16), f16) << 16);
    *reinterpret_cast<uint32_t*>(out + j) = hi;
    *reinterpret_cast<uint32_t*>(out + r + j) = lo;
    *reinterpret_cast<uint32_t*>(out + 2 * r + j) = hi;
  }
  for (int c = 3 * r + 2 * lane; c < r3; c += 64) *reinterpret_cast<uint32_t*>(out + c) = 0u;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PrefillLayout prefill_layout(const cql_desc& d, int m) {
  PrefillLayout L{};
  const uint64_t n = (uint64_t)d.n_out, k = (uint64_t)d.k_in, r = (uint64_t)d.rank;
  L.r3 = r ? (int)((3 * r + 63) / 64 * 64) : 0;
  L.rrows = r ? (int)((r + 127) / 128 * 128) : 0;
  L.r_pad = (int)((r + 31) / 32 * 32);
  L.sparse = d.mask == CQL_MASK_2_4 && (d.codec == CQL_CODEC_INT4_SYM || d.codec == CQL_CODEC_INT3_SYM);
  // the sparse GEMM dequantises the weights on chip: only the adapter
  // columns [N][r3] are staged in memory
  L.ldq = L.sparse ? L.r3 : (int)(k + L.r3);
  uint64_t pos = 0;
  L.qbf = pos;     pos = align256(pos + n * L.ldq * 2);
  L.wsc = pos;     pos = align256(pos + (L.sparse ? 0 : n * (k / 128) * 4));
  L.rbf = pos;     pos = align256(pos + (uint64_t)L.rrows * k * 2);
  L.rsc = pos;     pos = align256(pos + (uint64_t)L.rrows * (k / 128) * 4);
  L.tacc = pos;    pos = align256(pos + (uint64_t)m * L.r_pad * 4);
  L.t3 = pos;      pos = align256(pos + (uint64_t)m * L.r3 * 2);
  L.total = pos;
  return L;
}

static int sm_count_pf() {
  int dev = 0, v = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
  return v > 0 ? v : 148;
}

bool prefill_supported(const cql_desc& d, int x_dt) {
  if (codec_is_lut(d.codec) || d.mask == CQL_MASK_BITMAP50) return false;
  if (d.outlier_frac > 0.0f) return false;
  return x_dt == CQL_DT_BF16 || x_dt == CQL_DT_F16;
}

// The epilogue raises its register budget with setmaxnreg; that only works if
// the kernel was compiled to the full 168 registers per thread of a 384-thread
// block (128 * 40 + 256 * 232 == 384 * 168).  Checked once before launching.
static cudaError_t check_gemm_regs() {
  static int ok = -1;
  if (ok < 0) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, (const void*)k_pf_gemm) != cudaSuccess) return cudaErrorInvalidDeviceFunction;
    ok = a.numRegs == 168 ? 1 : 0;
  }
  return ok ? cudaSuccess : cudaErrorInvalidConfiguration;
}

cudaError_t launch_prefill(const DecodeParams& p, uint8_t* pws, cudaStream_t st) {
  const PrefillLayout L = prefill_layout(p.d, p.batch);
  const int N = p.d.n_out, K = p.d.k_in, r = p.d.rank, m = p.batch, G = p.upr;
  const int f16 = p.xdt == CQL_DT_F16 ? 1 : 0;
  uint16_t* qbf = reinterpret_cast<uint16_t*>(pws + L.qbf);
  float* wsc = reinterpret_cast<float*>(pws + L.wsc);
  uint16_t* rbf = reinterpret_cast<uint16_t*>(pws + L.rbf);
  float* rsc = reinterpret_cast<float*>(pws + L.rsc);
  float* tacc = reinterpret_cast<float*>(pws + L.tacc);
  uint16_t* t3 = reinterpret_cast<uint16_t*>(pws + L.t3);
  const bool lowrank = r > 0 && !(p.flags & CQL_FLAG_NO_LOWRANK);
  const bool main_on = !(p.flags & CQL_FLAG_NO_MAIN);
  cudaError_t e = check_gemm_regs();
  if (e != cudaSuccess) return e;

  static std::atomic<uint64_t> attr_done{0};
  const size_t smem = sizeof(PfSmem) + 1024;
  if ((e = ensure_smem_attr(attr_done, (const void*)k_pf_gemm, (int)smem)) != cudaSuccess) return e;
  const uint64_t nw = (uint64_t)N * G;
  if (!L.sparse) {
    k_pf_dequant_w<<<(unsigned)((nw + 127) / 128), 128, 0, st>>>(p, qbf, L.ldq, wsc, f16);
    if (!main_on) cudaMemsetAsync(wsc, 0, (uint64_t)N * G * 4, st);     // main term off: zero scales
  }
  if (lowrank) {
    k_pf_dequant_l<<<(unsigned)((N + 7) / 8), 256, 0, st>>>(p, qbf, L.ldq, L.sparse ? 0 : K, L.r3, f16);
    const uint64_t nr = (uint64_t)L.rrows * (K / 16);
    k_pf_dequant_r<<<(unsigned)((nr + 255) / 256), 256, 0, st>>>(p, rbf, rsc, L.rrows, f16);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int sms = sm_count_pf();
  const uint32_t idesc = pf_idesc(f16 != 0);
  CUtensorMap mA, mB, mT, mR;
  if (!make_map(&mB, p.x, (uint64_t)m, (uint64_t)K, (uint64_t)K, PF_BN)) return cudaErrorInvalidValue;
  if (lowrank) {
    // T pass: T = X R^T, split over K, fp32 atomics into tacc
    if ((e = cudaMemsetAsync(tacc, 0, (uint64_t)m * L.r_pad * 4, st)) != cudaSuccess) return e;
    if (!make_map(&mR, rbf, (uint64_t)L.rrows, (uint64_t)K, (uint64_t)K, PF_BM)) return cudaErrorInvalidValue;
    PfGemmParams t{};
    t.scales = rsc; t.rows = L.rrows; t.m = m; t.groups = G; t.lr_blocks = 0;
    t.row_tiles = L.rrows / PF_BM; t.tok_tiles = (m + PF_BN - 1) / PF_BN;
    const int tiles = t.row_tiles * t.tok_tiles;
    t.k_splits = max(1, min(G, sms / max(tiles, 1)));
    t.mode = 1; t.out = tacc; t.out_dt = CQL_DT_F32; t.ldo = L.r_pad; t.valid_rows = r; t.idesc = idesc;
    t.err = p.err;
    const int items = tiles * t.k_splits;
    k_pf_gemm<<<min(items, sms), PF_THREADS, smem, st>>>(mR, mB, mB, t);
    k_pf_tsplit<<<(unsigned)((m + 7) / 8), 256, 0, st>>>(tacc, L.r_pad, t3, L.r3, r, m, f16);
    if (!make_map(&mT, t3, (uint64_t)m, (uint64_t)L.r3, (uint64_t)L.r3, PF_BN)) return cudaErrorInvalidValue;
  } else {
    mT = mB;
  }
  if (L.sparse) return launch_pf_sgemm(p, qbf, L.r3, t3, lowrank, st);
  if (!make_map(&mA, qbf, (uint64_t)N, (uint64_t)L.ldq, (uint64_t)L.ldq, PF_BM)) return cudaErrorInvalidValue;
  PfGemmParams g{};
  g.scales = wsc; g.rows = N; g.m = m; g.groups = G; g.lr_blocks = lowrank ? L.r3 / PF_BK : 0;
  g.row_tiles = N / PF_BM; g.tok_tiles = (m + PF_BN - 1) / PF_BN; g.k_splits = 1;
  g.mode = 0; g.out = p.y; g.out_dt = p.ydt; g.ldo = N; g.valid_rows = N; g.idesc = idesc; g.err = p.err;
  const int items = g.row_tiles * g.tok_tiles;
  k_pf_gemm<<<min(items, sms), PF_THREADS, smem, st>>>(mA, mB, mT, g);
  return cudaGetLastError();
}

}  // namespace cql
