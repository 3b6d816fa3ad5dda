// Prefill main GEMM on the sparse tensor cores, 2:4 int4 and int3 layers
// (batch > 16):
//
//   Y^T[n][t] = sum_g s[n][g] * (sum_{k in g} q[n][k] X[t][k])  +  L^ T^T
//
// (SLiM-Quant's per-group scale on a 2:4-pruned matrix, SLiM review summary
// "SLIM-Quant"; the 2:4 pattern is what the sparse tensor cores execute; the
// adapter term rides as dense K blocks of exact bf16 hi/lo parts, SLiM
// "Low-rank adapter quantization").
//
// The weights never go back to HBM dequantised: a converter warpgroup reads
// the packed codes and META codes of a (128-row tile, 128-column group) from
// the row-interleaved planes (cp.async, lane = row), turns the 64 kept codes
// of each row into exact bf16/f16 integers written straight into tensor
// memory (compressed A, 32 columns, lane = row), and the META codes,
// regrouped across lanes, next to them as the sparse metadata.  Four
// tcgen05.mma.sp (M 128, N 208, K 32) per group, with X tiles (the B
// operand) staged by TMA, accumulate into one of two fp32 accumulators in
// tensor memory; the epilogue warps read each group's partial sums back,
// scale them by the row's fp32 group scale (so no dequantised weight is
// rounded to 16 bits) and sum them in registers.  (With A in shared memory
// the MMAs read both operands from it and issued at half the rate.)
//
// N = 208 tokens a tile: two 208-column accumulators, two 32-column A stages
// and two 8-column metadata stages fit the 512 tensor-memory columns (three
// stages fit only at N = 192, whose extra token tile costs more than the
// deeper prefetch gains at 2048 tokens).  A stage holds one K item (a group:
// A in tensor memory, X 2 x 26 KB; or an adapter block: its X tile and its A
// tile in the same 52 KB), with one barrier that fills it and one that frees
// it.  The MMA issuer, which pays on the order of a hundred cycles per
// tcgen05 instruction, issues eight a group (one wait, four MMAs, one
// commit, and the accumulator hand-offs).  The converters turn a group's
// codes into registers before waiting for its stage.
//
// Roles (512 threads, one CTA per SM, persistent over (row tile, token tile)
// items):
//   warp 0        TMA producer (X tiles; the adapter K blocks' A and B tiles)
//   warp 1        tensor-memory allocator and single-thread MMA issuer
//   warps 4..7    converter warpgroup (lane = row of the tile)
//   warps 8..15   epilogue: tcgen05.ld, per-row group scale, stores
// Every mbarrier wait is bounded; on expiry the kernel records
// CQL_ERR_TIMEOUT and winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace cql {
namespace {

constexpr int SP_BM = 128;                       // weight rows per tile (MMA M, tensor-memory lanes)
constexpr int SP_BN = 208;                       // tokens per tile (MMA N)
constexpr int SP_STAGES = 2;                     // K-item stages (a group, or an adapter block)
constexpr int SP_THREADS = 512;
constexpr int SP_A_BYTES = SP_BM * 128;          // an adapter block's A tile: 128 rows x 64 16-bit values
constexpr int SP_B_SLICE = SP_BN * 128;          // 208 tokens x 64 columns of 16-bit X (26 KB)
constexpr int SP_RING = 4;                       // groups of packed codes in flight per converter warp
constexpr int SP_RAW = 1536;                     // one row block of one group: codes 1024, META 512
constexpr uint32_t SP_A_COL = 2 * SP_BN;         // compressed A stage s at SP_A_COL + 32 s
constexpr uint32_t SP_META_COL = SP_A_COL + 32 * SP_STAGES;   // metadata stage s at SP_META_COL + 8 s
static_assert(SP_META_COL + 8 * SP_STAGES <= 512, "tensor-memory columns");
constexpr int SP_EPI_COLS = SP_BN / 2;           // accumulator columns per epilogue thread

struct SpSmem {
  // per stage: X tiles K 0..63 and 64..127 of a group; an adapter block puts
  // its X tile in the first and its A tile (16 KB) in the second
  uint8_t b[SP_STAGES][2][SP_B_SLICE];           // 1024-byte aligned (128-byte swizzle atoms)
  uint8_t raw[4][SP_RING][SP_RAW];               // converter warps' packed codes
  // full[s]: the producer's arrival (with the TMA bytes) and the four
  // converter warps'; done[s]: the MMAs that read stage s completed
  uint64_t full[SP_STAGES], done[SP_STAGES];
  uint64_t dfull[2], dempty[2];
  uint32_t tmem_base;
};

struct SpParams {
  const uint8_t* values;      // packed planes of the layer
  const uint8_t* meta;
  const uint8_t* scales;
  RowBytes rb;
  int rows;                   // N
  int m;                      // tokens
  int groups;                 // G = K / 128
  int main_on;                // the quantised term (else only the adapter blocks)
  int lr_blocks;              // adapter K blocks of 64 (3r rounded up, / 64)
  int row_tiles, tok_tiles;
  void* out;                  // y [m][N]
  int out_dt;
  uint32_t* err;
  uint64_t len_values, len_meta, len_scales;   // plane bytes (the checked build's bounds)
};

// Instruction descriptors (M = 128, N = 208, D f32, A = B = bf16 or f16,
// both K-major): sparse for the quantised term, dense for the adapter blocks.
CQL_HD uint32_t sp_idesc(bool f16, bool sparse) {
  const uint32_t fmt = f16 ? 0u : 1u;
  return (sparse ? (1u << 2) : 0u) | (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(SP_BN >> 3) << 17) |
         ((uint32_t)(SP_BM >> 4) << 24);
}

// One 2:4 group's two codes u as exact 16-bit integers q = u - 8 (the code
// byte at bits 0 and 16 by a byte permute, the exponent of 128 (bf16) or 1024
// (f16) ORed in, the offset removed by one packed subtraction).
template <bool F16>
CQL_DEV uint32_t code_pair(uint32_t lo, uint32_t hi, uint32_t sel) {
  const uint32_t t = prmt(lo, hi, sel);
  uint32_t a;
  constexpr uint32_t magic = F16 ? 0x64006400u : 0x43004300u;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(a) : "r"(t), "r"(0x000F000Fu), "r"(magic));
  uint32_t q;
  if (F16) asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(a), "r"(0x64086408u));
  else asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(a), "r"(0x43084308u));
  return q;
}

// One 2:4 group's two 3-bit codes (bits 0..2 and 3..5 of 'six') as exact
// 16-bit integers q = u - 4: placed under the exponent of 128 (bf16) or 1024
// (f16), then one packed subtraction of 132 (1028).
template <bool F16>
CQL_DEV uint32_t code_pair3(uint32_t six) {
  const uint32_t t = (six & 7u) | ((six & 0x38u) << 13);
  constexpr uint32_t magic = F16 ? 0x64006400u : 0x43004300u;
  const uint32_t a = t | magic;
  uint32_t q;
  if (F16) asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(a), "r"(0x64046404u));
  else asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(a), "r"(0x43044304u));
  return q;
}

template <bool F16, int BITS>
__global__ void __launch_bounds__(SP_THREADS, 1)
    k_pf_sgemm(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmL,
               const __grid_constant__ CUtensorMap tmT, SpParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  SpSmem& S = *reinterpret_cast<SpSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SP_STAGES; ++s) {
      mbar_init(&S.full[s], 5);
      mbar_init(&S.done[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.dfull[b], 1);
      mbar_init(&S.dempty[b], 8);
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

  const int n_items = p.row_tiles * p.tok_tiles;
  const int mg = p.main_on ? p.groups : 0;       // quantised groups per tile
  const int kitems = mg + p.lr_blocks;            // K items per tile, each taking one stage

  // Register split: the launch gives every thread 128 registers; the producer
  // warpgroup drops to 40, the converters to 64, the two epilogue warpgroups
  // rise to 200: 128 * 40 + 128 * 64 + 256 * 200 = 64512 <= 512 * 128.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    if (warp == 0 && lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t ai = 0;                              // K items so far
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int rt = item / p.tok_tiles, tt = item % p.tok_tiles;
        for (int j = 0; j < kitems; ++j, ++ai) {
          const int s = ai % SP_STAGES;
          if (!mbar_wait(&S.done[s], ((ai / SP_STAGES) & 1) ^ 1)) { ok = false; break; }
          if (j < mg) {
            mbar_expect_tx(&S.full[s], 2 * SP_B_SLICE);
            tma_load_2d(S.b[s][0], &tmX, &S.full[s], 128 * j, tt * SP_BN);
            tma_load_2d(S.b[s][1], &tmX, &S.full[s], 128 * j + 64, tt * SP_BN);
          } else {
            const int lb = j - mg;
            mbar_expect_tx(&S.full[s], SP_A_BYTES + SP_B_SLICE);
            tma_load_2d(S.b[s][1], &tmL, &S.full[s], 64 * lb, rt * SP_BM);
            tma_load_2d(S.b[s][0], &tmT, &S.full[s], 64 * lb, tt * SP_BN);
          }
        }
      }
      if (!ok) set_error(p.err, CQL_ERR_TIMEOUT, 30);
    } else if (warp == 1 && lane == 0) {
      // ---------------- MMA issuer ----------------
      uint32_t ai = 0, gc = 0;
      bool ok = true;
      const uint32_t id_sp = sp_idesc(F16, true), id_dn = sp_idesc(F16, false);
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        for (int j = 0; j < kitems; ++j, ++ai) {
          const bool lr = j >= mg;
          const bool first = !lr || j == mg;        // first K item of an accumulator group
          const bool last = !lr || j == kitems - 1;
          const uint32_t buf = gc & 1;
          if (first && !mbar_wait(&S.dempty[buf], ((gc >> 1) & 1) ^ 1)) { ok = false; break; }
          const int s = ai % SP_STAGES;
          if (!mbar_wait(&S.full[s], (ai / SP_STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + buf * SP_BN;
          const uint32_t b0 = smem_u32(S.b[s][0]), b1 = smem_u32(S.b[s][1]);
          if (!lr) {
            // four K-32 steps: compressed A (tensor memory) advances 8 columns
            // a step; X takes K 0..63 from the first tile, 64..127 from the second
            const uint32_t m = tmem + SP_META_COL + 8u * s, at = tmem + SP_A_COL + 32u * s;
            tc_mma_sp_ta(d, at, smem_desc_sw128(b0), m, id_sp, 0u);
            tc_mma_sp_ta(d, at + 8, smem_desc_sw128(b0 + 64), m, id_sp | 1u, 1u);
            tc_mma_sp_ta(d, at + 16, smem_desc_sw128(b1), m + 4, id_sp, 1u);
            tc_mma_sp_ta(d, at + 24, smem_desc_sw128(b1 + 64), m + 4, id_sp | 1u, 1u);
          } else {
            const uint64_t da = smem_desc_sw128(b1), db = smem_desc_sw128(b0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma(d, da + 2 * kk, db + 2 * kk, id_dn, (j > mg || kk > 0) ? 1u : 0u);
          }
          tc_commit(&S.done[s]);
          if (last) {
            tc_commit(&S.dfull[buf]);
            ++gc;
          }
        }
      }
      if (!ok) set_error(p.err, CQL_ERR_TIMEOUT, 31);
    }
  } else if (warp < 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 64;");
    // ---------------- converter warpgroup ----------------
    const int qq = warp & 3;                        // row block of the tile = tensor-memory lane quarter
    const uint32_t lane_base = (uint32_t)(32 * qq) << 16;
    const uint32_t sel_meta = (lane & 8) ? 0x3276u : 0x5410u;
    const uint32_t vstride = (p.rb.values >> 4) * 512u, mstride = (p.rb.meta >> 4) * 512u;
    uint8_t* ring = S.raw[qq][0] + lane * 16;
    // next quantised group to fetch, as (tile number of this CTA, group)
    int f_tile = 0, f_g = 0;
    const int my_tiles = n_items > (int)blockIdx.x ? (n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto fetch = [&](int slot) {
      if (mg == 0 || f_tile >= my_tiles) return;
      const int item = blockIdx.x + f_tile * gridDim.x;
      const uint32_t rbk = 4u * (uint32_t)(item / p.tok_tiles) + qq;
      // int4: a group's codes are two slabs (32 bytes); int3: 24 bytes at
      // byte 24 g, inside the two slabs from (24 g) / 16 on
      const uint32_t slab0 = BITS == 4 ? 2u * (uint32_t)f_g : (24u * (uint32_t)f_g) >> 4;
      const uint32_t ov = rbk * vstride + slab0 * 512u + lane * 16;
      const uint32_t om = rbk * mstride + (uint32_t)f_g * 512u + lane * 16;
      const uint8_t* vsrc = p.values + ov;
      uint8_t* sl = ring + slot * SP_RAW;
      if (CQL_IN(p.err, ov + 512 + 15, p.len_values, 301)) {
        cp_async16(sl, vsrc);
        cp_async16(sl + 512, vsrc + 512);
      }
      if (CQL_IN(p.err, om + 15, p.len_meta, 302)) cp_async16(sl + 1024, p.meta + om);
      if (++f_g == mg) {
        f_g = 0;
        ++f_tile;
      }
    };
#pragma unroll 1
    for (int d = 0; d < SP_RING; ++d) {
      fetch(d);
      cp_async_commit();
    }
    uint32_t ai = 0, gi = 0;                        // K items, quantised groups converted
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      for (int j = 0; j < kitems; ++j, ++ai) {
        const int s = ai % SP_STAGES;
        if (j < mg) {
          const int si = gi % SP_RING;
          uint8_t* sl = ring + si * SP_RAW;
          cp_async_wait<SP_RING - 1>();
          const uint4 va = *reinterpret_cast<const uint4*>(sl);
          const uint4 vb = *reinterpret_cast<const uint4*>(sl + 512);
          const uint4 mm = *reinterpret_cast<const uint4*>(sl + 1024);
          const uint32_t vw[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
          uint32_t q[32];                           // compressed A row: 64 kept values
          if constexpr (BITS == 4) {
#pragma unroll
            for (int wi = 0; wi < 8; ++wi) {
              const uint32_t hi = vw[wi] >> 4;
#pragma unroll
              for (int by = 0; by < 4; ++by)
                q[4 * wi + by] = code_pair<F16>(vw[wi], hi, (uint32_t)(by | (by << 4) | ((4 + by) << 8) | ((4 + by) << 12)));
            }
          } else {
            // the 24 bytes start at byte 0 (even group) or 8 (odd group) of
            // the 32 fetched; pair m is stream bits [6 m, 6 m + 6)
            const bool odd = (j & 1) != 0;            // j: the group of this item
            uint32_t ws[7];
#pragma unroll
            for (int k = 0; k < 6; ++k) ws[k] = odd ? vw[k + 2] : vw[k];
            ws[6] = 0u;
#pragma unroll
            for (int m = 0; m < 32; ++m) {
              const int wi = (6 * m) >> 5, sh = (6 * m) & 31;
              const uint32_t six = sh <= 26 ? (ws[wi] >> sh) : __funnelshift_r(ws[wi], ws[wi + 1], sh);
              q[m] = code_pair3<F16>(six);
            }
          }
          // META: the sparse MMA wants, in lane 16h + i, rows 16h + i and
          // 16h + 8 + i side by side (16 bits each) for groups 0..3 of a K
          // step, and in lane 16h + 8 + i the same two rows for groups 4..7
          const uint32_t mw[4] = {mm.x, mm.y, mm.z, mm.w};
          uint32_t me[4];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t o = __shfl_xor_sync(0xffffffffu, mw[kk], 8);
            me[kk] = prmt(mw[kk], o, sel_meta);
          }
          __syncwarp();                             // the slot is read by all lanes before its refill
          fetch(si);
          cp_async_commit();
          // the stage is free once the MMAs of its previous item completed
          ok = __all_sync(0xffffffffu, mbar_wait(&S.done[s], ((ai / SP_STAGES) & 1) ^ 1));
          if (!ok) break;
          tmem_st32(tmem + lane_base + SP_A_COL + 32u * s, q);
          tmem_st8(tmem + lane_base + SP_META_COL + 8u * s, me[0], me[1], 0u, 0u, me[2], me[3], 0u, 0u);
          tmem_wait_st();
          ++gi;
        } else {
          ok = __all_sync(0xffffffffu, mbar_wait(&S.done[s], ((ai / SP_STAGES) & 1) ^ 1));
          if (!ok) break;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.full[s]);
      }
    }
    cp_async_wait<0>();
    if (!ok && lane == 0) set_error(p.err, CQL_ERR_TIMEOUT, 32);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;");
    // ---------------- epilogue ----------------
    const int q = warp & 3, h = (warp - 8) >> 2;
    uint32_t gc = 0;
    bool ok = true;
    const int ngroups = mg + (p.lr_blocks > 0 ? 1 : 0);
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int rt = item / p.tok_tiles, tt = item % p.tok_tiles;
      const int row = rt * SP_BM + 32 * q + lane;
      float acc[SP_EPI_COLS];
#pragma unroll
      for (int i = 0; i < SP_EPI_COLS; ++i) acc[i] = 0.0f;
      auto scale_of = [&](int g) {
        const uint32_t os = rit32((uint32_t)row, 2u * g, p.rb.scales);
        return g < mg ? (CQL_IN(p.err, os + 1, p.len_scales, 303) ? f16_bits_to_f32(ldg_u16(p.scales + os)) : 0.0f)
                      : 1.0f;
      };
      float s_next = ngroups > 0 ? scale_of(0) : 1.0f;
      for (int g = 0; g < ngroups; ++g, ++gc) {
        const float s = s_next;
        if (g + 1 < ngroups) s_next = scale_of(g + 1);
        const uint32_t buf = gc & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&S.dfull[buf], (gc >> 1) & 1));
        if (!ok) break;
        tc_fence_after();
        const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + buf * SP_BN + h * SP_EPI_COLS;
        // 104 columns: 64, then 32, then 8
        {
          float v0[32], v1[32];
          tmem_ld32(base, v0);
          tmem_ld32(base + 32, v1);
          tmem_wait_ld(v0);
          reg_after_wait(v1);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            acc[i] = fmaf(s, v0[i], acc[i]);
            acc[32 + i] = fmaf(s, v1[i], acc[32 + i]);
          }
        }
        {
          float w0[32];
          tmem_ld32(base + 64, w0);
          tmem_wait_ld(w0);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[64 + i] = fmaf(s, w0[i], acc[64 + i]);
        }
        if constexpr (SP_EPI_COLS > 96) {
          static_assert(SP_EPI_COLS == 104, "epilogue column split");
          float w2[8];
          tmem_ld_wait<8>(base + 96, w2);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[96 + i] = fmaf(s, w2[i], acc[96 + i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.dempty[buf]);
      }
      if (!ok) break;
      const int t0 = tt * SP_BN + h * SP_EPI_COLS;
#pragma unroll
      for (int i = 0; i < SP_EPI_COLS; ++i)
        if (t0 + i < p.m && CQL_IN(p.err, (uint64_t)(t0 + i) * p.rows + row, (uint64_t)p.m * p.rows, 304))
          store_out(p.out, p.out_dt, (uint64_t)(t0 + i) * p.rows + row, acc[i]);
    }
    if (!ok && lane == 0) set_error(p.err, CQL_ERR_TIMEOUT, 33);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

}  // namespace

// The register split above assumes 128 registers a thread at launch.
template <bool F16, int BITS>
static cudaError_t check_sgemm_regs() {
  static int ok = -1;
  if (ok < 0) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, (const void*)k_pf_sgemm<F16, BITS>) != cudaSuccess)
      return cudaErrorInvalidDeviceFunction;
    ok = a.numRegs == 128 ? 1 : 0;
  }
  return ok ? cudaSuccess : cudaErrorInvalidConfiguration;
}

template <bool F16, int BITS>
static cudaError_t launch_sg(const DecodeParams& p, const uint16_t* lbuf, int r3, const uint16_t* t3, bool lowrank,
                             cudaStream_t st) {
  cudaError_t e = check_sgemm_regs<F16, BITS>();
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> attr_done{0};
  const size_t smem = sizeof(SpSmem) + 1024;
  if ((e = ensure_smem_attr(attr_done, (const void*)k_pf_sgemm<F16, BITS>, (int)smem)) != cudaSuccess) return e;
  const int N = p.d.n_out, K = p.d.k_in, m = p.batch;
  CUtensorMap mX, mL, mT;
  if (!make_map(&mX, p.x, (uint64_t)m, (uint64_t)K, (uint64_t)K, SP_BN)) return cudaErrorInvalidValue;
  if (lowrank) {
    if (!make_map(&mL, lbuf, (uint64_t)N, (uint64_t)r3, (uint64_t)r3, SP_BM)) return cudaErrorInvalidValue;
    if (!make_map(&mT, t3, (uint64_t)m, (uint64_t)r3, (uint64_t)r3, SP_BN)) return cudaErrorInvalidValue;
  } else {
    mL = mX;
    mT = mX;
  }
  SpParams s{};
  s.values = p.values;
  s.meta = p.meta;
  s.scales = p.scales;
  s.rb = p.rb;
  s.rows = N;
  s.m = m;
  s.groups = K / 128;
  s.main_on = (p.flags & CQL_FLAG_NO_MAIN) ? 0 : 1;
  s.lr_blocks = lowrank ? r3 / 64 : 0;
  s.row_tiles = N / SP_BM;
  s.tok_tiles = (m + SP_BN - 1) / SP_BN;
  s.out = p.y;
  s.len_values = p.plane_len[CQL_PLANE_VALUES];
  s.len_meta = p.plane_len[CQL_PLANE_META];
  s.len_scales = p.plane_len[CQL_PLANE_SCALES];
  s.out_dt = p.ydt;
  s.err = p.err;
  const int items = s.row_tiles * s.tok_tiles;
  const int grid = items < device_sm_count() ? items : device_sm_count();
  k_pf_sgemm<F16, BITS><<<grid, SP_THREADS, smem, st>>>(mX, mL, mT, s);
  return cudaGetLastError();
}

cudaError_t launch_pf_sgemm(const DecodeParams& p, const uint16_t* lbuf, int r3, const uint16_t* t3, bool lowrank,
                            cudaStream_t st) {
  if (p.d.codec == CQL_CODEC_INT3_SYM)
    return p.xdt == CQL_DT_F16 ? launch_sg<true, 3>(p, lbuf, r3, t3, lowrank, st)
                               : launch_sg<false, 3>(p, lbuf, r3, t3, lowrank, st);
  return p.xdt == CQL_DT_F16 ? launch_sg<true, 4>(p, lbuf, r3, t3, lowrank, st)
                             : launch_sg<false, 4>(p, lbuf, r3, t3, lowrank, st);
}

}  // namespace cql
