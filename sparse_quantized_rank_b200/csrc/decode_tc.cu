// Decode main term on the sparse tensor cores: 2:4 mask, int4 or int3 codes,
// batch 1..16.  y_acc[b][n] += sum_g s[n][g] * sum_{k in g} q[n][k] x[b][k]
// (SLiM-Quant's per-group scale on a 2:4-pruned matrix, SLiM review summary
// "SLIM-Quant"; the 2:4 pattern is what the sparse tensor cores execute).
//
// A tile is 128 weight rows x one scale group (128 columns).  Per tile:
//   * each converter warp fetches its 32-row block's packed bytes (two code
//     slabs and one META slab, 16 bytes per lane each) with cp.async, several
//     tiles ahead; x (the MMA's B operand, batch padded with zeros to the
//     box's 8 or 16 rows) arrives in chunks of 1024 columns, one 3-D TMA box
//     per chunk;
//   * a converter warpgroup (lanes = rows, as the planes are laid out) turns
//     the 64 kept codes of each row (int4: 32 bytes, two slabs; int3: 24
//     bytes inside the two slabs that cover them) into exact bf16/f16
//     integers and writes
//     them straight into tensor memory (compressed A, 32 columns), and writes
//     the META codes, regrouped across lanes into the order the sparse MMA
//     reads them, next to it;
//   * the MMA warp issues four tcgen05.mma.sp (M 128, N 16, K 32) into a
//     fresh fp32 accumulator in tensor memory;
//   * the converter warpgroup reads the accumulator back (lane = row), scales
//     it by the row's fp32 group scale and sums over the tile's row tile;
//     partial row sums go to y_acc with reductions at L2 (split-K across
//     CTAs), where the epilogue kernel adds the adapter term and rounds.
// The scale is applied outside the MMA so that no dequantised weight is ever
// rounded to 16 bits: the tensor cores multiply exact integers.
//
// Launched programmatically dependent on the previous kernel in the stream: the
// weight tiles (inputs nobody writes) stream in before griddepcontrol.wait;
// x, the accumulators and t are touched only after it.
//
// Roles (640 threads, one CTA per SM, persistent over a contiguous tile range):
//   warps 0..3    MMA issuer of converter warpgroup 0..3 (one lane each);
//                 warp 0 also allocates tensor memory and loads the x chunks
//   warps 4..19   converter warpgroups 0..3 (tile k of the range goes to
//                 warpgroup k mod 4); each warp fetches its own row block's
//                 packed bytes with cp.async into a private ring
// Every mbarrier wait is bounded; on expiry the kernel records
// CQL_ERR_TIMEOUT and winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace cql {
namespace {

constexpr int TC_WG = 4;                          // converter warpgroups
constexpr int TC_THREADS = 128 * (1 + TC_WG);     // warps 0..3 MMA issuers, then the warpgroups
constexpr int TC_KC = 8;                          // scale groups per x chunk (1024 columns)
constexpr int TC_RING = 3;                        // tiles in flight per converter warp (cp.async ring)
constexpr int TC_TS = 2;                          // tensor-memory stages per converter warpgroup
constexpr int TC_VAL_BYTES = 1024;                // codes of one 32-row block: 2 slabs
constexpr int TC_META_BYTES = 512;                // META of one 32-row block: 1 slab
constexpr int TC_SLOT_BYTES = TC_VAL_BYTES + TC_META_BYTES + 512;   // one row block of one tile (+ scale slab)
constexpr int TC_XBOX_BYTES = 16 * 64 * 2;        // TMA box: 16 rows x 64 columns of 16-bit x
constexpr int TC_XCHUNK_BYTES = TC_KC * 2 * TC_XBOX_BYTES;
// Up to 8 batch rows the box holds 8 rows (one 1 KB swizzle atom): the MMA
// still reads 16 rows (N = 16), its rows 8..15 falling on the next box, but
// they only reach accumulator columns 8..15, which are never read.
template <int B>
constexpr int tc_xrows() { return B <= 8 ? 8 : 16; }
template <int B>
constexpr int tc_xbox_bytes() { return tc_xrows<B>() * 64 * 2; }
template <int B>
constexpr int tc_xchunk_bytes() { return TC_KC * 2 * tc_xbox_bytes<B>(); }

// Tensor-memory columns of converter warpgroup w (512 allocated, 128 each):
//   A (compressed codes) stage s: 128 w + 32 s          (32 columns)
//   D (fp32 accumulator) stage s: 128 w + 64 + 16 s     (16 columns)
//   META stage s:                 128 w + 96 + 8 s      (8 columns: K steps 0, 1 at
//                                 +0, +1 and 2, 3 at +4, +5)
// The sparse MMA takes its metadata address aligned and the column inside the
// aligned pair from the instruction descriptor's selector bits [0, 2).
CQL_HD uint32_t col_a(int w, int s) { return 128u * w + 32u * s; }
CQL_HD uint32_t col_d(int w, int s) { return 128u * w + 64u + 16u * s; }
CQL_HD uint32_t col_m(int w, int s) { return 128u * w + 96u + 8u * s; }

struct TcSmem {
  uint8_t x[2][TC_XCHUNK_BYTES];                  // x chunks, 1024-byte aligned (128-byte swizzle atoms)
  uint8_t ring[4 * TC_WG][TC_RING][TC_SLOT_BYTES];   // per converter warp: [values 1024][META 512][scales 512]
  int slot_rt[4 * TC_WG][TC_RING];                // row tile and group of each ring slot
  int slot_g[4 * TC_WG][TC_RING];
  float scale[TC_WG][TC_TS][128];                 // group scale of each row of a tensor-memory stage
  int tinfo[TC_WG][TC_TS][4];                     // row tile of a stage (one copy per converter warp)
  uint64_t afull[TC_WG][TC_TS], dfull[TC_WG][TC_TS];
  uint64_t xfull[2], xempty[2];
  uint32_t tmem_base;
};

struct TcGeom {
  int n_rt;          // row tiles (N / 128)
  int G;             // scale groups per row (K / 128)
  int n_chunks;      // ceil(G / TC_KC)
  int n_tiles;       // n_rt * G  (N K <= 2^32 keeps it below 2^18)
};

// Tile order: x chunk, then row tile, then group inside the chunk, so that a
// CTA's contiguous range touches one or two x chunks and runs along K inside
// a row tile.
CQL_DEV void tile_coords(const TcGeom& g, int t, int& c, int& rt, int& grp) {
  const int per_full = g.n_rt * TC_KC;
  const int cc = min(t / per_full, g.n_chunks - 1);
  const int r = t - cc * per_full;
  const int gc = min(TC_KC, g.G - cc * TC_KC);
  c = cc;
  rt = r / gc;
  grp = cc * TC_KC + (r - rt * gc);
}

// Walks the tile order without divisions: (chunk, row tile, group in chunk).
struct TileIter {
  int c, rt, gl, gc, g;
  CQL_DEV void init(const TcGeom& geo, int t) {
    if (t >= geo.n_tiles) t = geo.n_tiles - 1;      // past the end: any valid tile (never used)
    tile_coords(geo, t, c, rt, g);
    gc = min(TC_KC, geo.G - c * TC_KC);
    gl = g - c * TC_KC;
  }
  // advance by 'steps' tiles (steps <= one chunk's tiles)
  CQL_DEV void advance(const TcGeom& geo, int steps) {
    gl += steps;
    while (gl >= gc) {
      gl -= gc;
      if (++rt == geo.n_rt) {
        rt = 0;
        if (c + 1 < geo.n_chunks) ++c;
        gc = min(TC_KC, geo.G - c * TC_KC);
      }
    }
    g = c * TC_KC + gl;
  }
  CQL_DEV void next(const TcGeom& geo) {
    if (++gl == gc) {
      gl = 0;
      if (++rt == geo.n_rt) {
        rt = 0;
        if (c + 1 < geo.n_chunks) ++c;
        gc = min(TC_KC, geo.G - c * TC_KC);
      }
    }
    g = c * TC_KC + gl;
  }
};

// One 2:4 group's two codes u as exact 16-bit integers q = u - 8.  'lo'
// holds the group's byte (low nibble: code of the first kept column), 'hi'
// the same word shifted right by 4.  The byte permute puts the two nibbles at
// bits 0 and 16; the LOP3 masks them and ORs in the exponent of 128 (bf16:
// 0x4300, giving u + 128) or 1024 (f16: 0x6400, u + 1024); one packed
// subtraction of 136 (1032) leaves q.  (Subtracting here costs one
// instruction per pair; removing the offset with a second MMA over the same
// metadata instead doubles the MMAs a tile issues, and MMA issue is the
// scarcer resource.)
template <bool F16>
CQL_DEV uint32_t code_pair(uint32_t lo, uint32_t hi, uint32_t sel) {
  const uint32_t t = prmt(lo, hi, sel);
  uint32_t a;
  constexpr uint32_t magic = F16 ? 0x64006400u : 0x43004300u;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(a) : "r"(t), "r"(0x000F000Fu), "r"(magic));
  uint32_t q;
  if (F16) asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(a), "r"(0x64086408u));    // 1032
  else asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(a), "r"(0x43084308u));      // 136
  return q;
}


// One 2:4 group's two 3-bit codes u (bits 0..2 and 3..5 of 'six') as exact
// 16-bit integers q = u - 4: placed at bits 0 and 16 under the exponent of
// 128 (bf16) or 1024 (f16), then one packed subtraction of 132 (1028).
template <bool F16>
CQL_DEV uint32_t code_pair3(uint32_t six) {
  const uint32_t t = (six & 7u) | ((six & 0x38u) << 13);
  constexpr uint32_t magic = F16 ? 0x64006400u : 0x43004300u;
  const uint32_t a = t | magic;
  uint32_t q;
  if (F16) asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(a), "r"(0x64046404u));    // 1028
  else asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(a), "r"(0x43044304u));      // 132
  return q;
}

// First 16-byte slab (of the two a converter fetches) of group g's codes in
// a row: int4 codes take 32 bytes a group, int3 codes 24 (at byte 24 g).
template <int BITS>
CQL_HD uint32_t tc_code_slab(uint32_t g) { return BITS == 4 ? 2u * g : (24u * g) >> 4; }

// Instruction descriptor: sparse, D f32, A = B = bf16 (or f16), K-major,
// M = 128, N = 16.
CQL_HD uint32_t tc_idesc(bool f16) {
  const uint32_t fmt = f16 ? 0u : 1u;
  return (1u << 2) | (1u << 4) | (fmt << 7) | (fmt << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
}

// Side work of the MMA issuer warps (all lanes), done before their MMA loops:
// their first MMA waits for the first tile conversion anyway (it needs none
// of the kernel's shared or tensor memory):
//  * the CSR outliers (SqueezeLLM "Approach": the sparse part of the
//    dense-and-sparse split) of this CTA's share of the rows, a thread per
//    row, added into y_acc;
//  * a share of t = deq(R_q) x (SLiM "Low-rank adapter quantization"): items
//    of (32 R rows, 32 columns, all batch rows), a warp each, added into t_acc
//    with the R group scale applied.
// R codes and scale of the first R x item of a warp: weights, safe to read
// before griddepcontrol.wait.
struct SideFirst {
  uint4 q4;
  uint32_t sc;
};
// Side workers per CTA: the 4 issuer warps for small batches; for 8 and more
// batch rows the R x items are 8 to 16 times heavier and go to the 16
// converter warps instead (at their first read-back, see the kernel).
template <int B>
constexpr int tc_side_workers() { return B >= 8 ? 4 * TC_WG : TC_WG; }

template <int B>
CQL_DEV SideFirst tc_side_prefetch(const DecodeParams& p, int iw, int lane) {
  SideFirst f{make_uint4(0u, 0u, 0u, 0u), 0u};
  const int K = p.d.k_in;
  const int it = iw * gridDim.x + blockIdx.x;
  if (p.d.rank > 0 && !(p.flags & CQL_FLAG_NO_LOWRANK) && it < (p.r_pad / 32) * (K / 32)) {
    const int s32 = it % (K / 32), rbr = it / (K / 32);
    const uint32_t ov = slab_off32((uint32_t)rbr, (uint32_t)s32, p.rb.r_values) + lane * 16;
    const uint32_t os = rit32((uint32_t)(32 * rbr + lane), 2u * (s32 >> 2), p.rb.r_scales);
    if (CQL_IN(p.err, ov + 15, p.plane_len[CQL_PLANE_R_VALUES], 101)) f.q4 = ldg_stream(p.r_values + ov);
    if (CQL_IN(p.err, os + 1, p.plane_len[CQL_PLANE_R_SCALES], 102)) f.sc = ldg_u16(p.r_scales + os);
  }
  return f;
}

template <int B>
CQL_DEV void tc_side_work(const DecodeParams& p, int iw, int lane, const SideFirst& first) {
  constexpr int NW = tc_side_workers<B>();
  const int N = p.d.n_out, K = p.d.k_in;
  // t of this call accumulates in buffer (calls so far) & 1, which the call
  // before cleared; clear the other one (the previous call's, whose epilogue
  // is complete) for the next call
  const uint32_t par = ld_cg_u32(p.t_counter) & 1u;
  float* t_acc = p.t_final + (size_t)par * B * p.r_pad;
  {
    float* t_old = p.t_final + (size_t)(par ^ 1u) * B * p.r_pad;
    const int tot = B * p.r_pad, per = (tot + gridDim.x - 1) / gridDim.x;
    for (int i = blockIdx.x * per + iw * 32 + lane; i < min(tot, (int)(blockIdx.x + 1) * per); i += NW * 32)
      if (CQL_IN(p.err, (uint64_t)(t_old - p.t_final) + i, p.t_final_elems, 103)) t_old[i] = 0.0f;
    if (blockIdx.x == 0 && iw == 0 && lane == 0) p.t_counter[1] = par;
  }
  if (p.csr_rowptr != nullptr && !(p.flags & CQL_FLAG_NO_CSR)) {
    const int r0 = (int)((uint64_t)N * blockIdx.x / gridDim.x), r1 = (int)((uint64_t)N * (blockIdx.x + 1) / gridDim.x);
    for (int row = r0 + iw * 32 + lane; row < r1; row += NW * 32) {
      if (!CQL_IN(p.err, 4ull * row + 7, p.plane_len[CQL_PLANE_CSR_ROWPTR], 104)) continue;
      int e0 = p.csr_rowptr[row], e1 = p.csr_rowptr[row + 1];
      e0 = max(0, min(e0, (int)p.nnz));
      e1 = max(e0, min(e1, (int)p.nnz));
      if (e1 == e0) continue;
      float acc[B];
#pragma unroll
      for (int b = 0; b < B; ++b) acc[b] = 0.0f;
      for (int e = e0; e < e1; ++e) {
        const int col = p.csr_col[e];
        if (col >= K) continue;
        const float v = f16_bits_to_f32(p.csr_val[e]);
#pragma unroll
        for (int b = 0; b < B; ++b)
          if (b < p.batch && CQL_IN(p.err, (uint64_t)b * K + col, p.x_elems, 105))
            acc[b] = fmaf(v, to_f32_act(p.x, p.xdt, (uint64_t)b * K + col), acc[b]);
      }
#pragma unroll
      for (int b = 0; b < B; ++b)
        if (b < p.batch && CQL_IN(p.err, (uint64_t)b * N + row, p.y_elems, 106))
          atomicAdd(p.y_acc + (uint64_t)b * N + row, acc[b]);
    }
  }
  if (p.d.rank > 0 && !(p.flags & CQL_FLAG_NO_LOWRANK)) {
    // item i goes to issuer warp i / gridDim.x (mod TC_WG) of CTA i % gridDim.x,
    // so that the items spread over all CTAs before any warp gets a second one
    const int items = (p.r_pad / 32) * (K / 32);
    const int nwarps = gridDim.x * NW;
    for (int it = iw * gridDim.x + blockIdx.x; it < items; it += nwarps) {
      const int s32 = it % (K / 32), rbr = it / (K / 32);
      const int j = 32 * rbr + lane, u = s32 >> 2;
      const bool pre = it == iw * (int)gridDim.x + (int)blockIdx.x;   // the prefetched first item
      const uint32_t ov = slab_off32((uint32_t)rbr, (uint32_t)s32, p.rb.r_values) + lane * 16;
      const uint32_t os = rit32((uint32_t)j, 2u * u, p.rb.r_scales);
      const uint4 q4 = pre ? first.q4
                           : (CQL_IN(p.err, ov + 15, p.plane_len[CQL_PLANE_R_VALUES], 107) ? ldg_stream(p.r_values + ov)
                                                                                           : make_uint4(0u, 0u, 0u, 0u));
      const float sc = f16_bits_to_f32(
          pre ? first.sc
              : (CQL_IN(p.err, os + 1, p.plane_len[CQL_PLANE_R_SCALES], 108) ? ldg_u16(p.r_scales + os) : 0u));
      float xv[B];                                  // x[b][32 s32 + lane]
#pragma unroll
      for (int b = 0; b < B; ++b) {
        xv[b] = 0.0f;
        if (b < p.batch && CQL_IN(p.err, (uint64_t)b * K + 32 * s32 + lane, p.x_elems, 109)) {
          const uint32_t xh = static_cast<const uint16_t*>(p.x)[(uint64_t)b * K + 32 * s32 + lane];
          xv[b] = p.xdt == CQL_DT_BF16 ? bf16_bits_to_f32(xh) : f16_bits_to_f32(xh);
        }
      }
      const uint32_t wd[4] = {q4.x, q4.y, q4.z, q4.w};
      float a[B];
#pragma unroll
      for (int b = 0; b < B; ++b) a[b] = 0.0f;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float q = (float)((int)((wd[k >> 3] >> (4 * (k & 7))) & 15u) - 8);
#pragma unroll
        for (int b = 0; b < B; ++b) a[b] = fmaf(q, __shfl_sync(0xffffffffu, xv[b], k), a[b]);
      }
      if (j < p.d.rank) {
#pragma unroll
        for (int b = 0; b < B; ++b)
          if (b < p.batch &&
              CQL_IN(p.err, (uint64_t)(t_acc - p.t_final) + (uint64_t)b * p.r_pad + j, p.t_final_elems, 110))
            atomicAdd(t_acc + (uint64_t)b * p.r_pad + j, sc * a[b]);
      }
    }
  }
}

// 88 registers per thread: 640 x 88 leaves room for one epilogue block (128
// threads) to become resident beside this kernel and prefetch its operands.
template <int B, bool F16, int BITS>
__global__ void __maxnreg__(88)
    k_decode_tc(const __grid_constant__ CUtensorMap tmX, DecodeParams p, TcGeom geo) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  TcSmem& S = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();                          // let the epilogue kernel get resident
  const long long wlim = (p.flags & CQL_FLAG_DEBUG_SKIP_X) ? kTcDebugWaitCycles : kTcWaitCycles;

  const int t0 = (int)((uint64_t)geo.n_tiles * blockIdx.x / gridDim.x);
  const int t1 = (int)((uint64_t)geo.n_tiles * (blockIdx.x + 1) / gridDim.x);
  const int n = t1 - t0;

  if (threadIdx.x == 0) {
    for (int w = 0; w < TC_WG; ++w)
      for (int s = 0; s < TC_TS; ++s) {
        mbar_init(&S.afull[w][s], 4);
        mbar_init(&S.dfull[w][s], 1);
      }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.xfull[b], 1);
      mbar_init(&S.xempty[b], TC_WG);               // one commit from each MMA issuer
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&S.tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp < TC_WG) {
    // ---------------- MMA issuer of warpgroup w (one lane) ----------------
    // A thread pays ~120 cycles per tcgen05.mma it issues; issuers in
    // different warps overlap, so each warpgroup has its own.  Issuer 0 also
    // loads the x chunks (one 3-D TMA box each), one chunk ahead.  x chunk c
    // uses buffer c & 1; the chunks of the range are consecutive, so the
    // phase of a buffer follows from the chunk index.
    TileIter first, last;
    first.init(geo, t0);
    last.init(geo, t1 - 1);
    const int c0 = first.c, c1 = last.c;
    constexpr bool issuer_side = tc_side_workers<B>() == TC_WG;
    const SideFirst side_first = issuer_side ? tc_side_prefetch<B>(p, warp, lane) : SideFirst{};
    // x, the accumulators and t may be written by the kernels before this one
    // (this kernel is launched early, programmatically dependent on them)
    pdl_wait();
    // the header too may have been written by the kernel before this one
    if (blockIdx.x == 0 && threadIdx.x == 0 && !header_ok(p)) set_error(p.err, CQL_ERR_FORMAT, 1);
    if (warp == 0 && lane == 0 && n > 0 && !(p.flags & CQL_FLAG_DEBUG_SKIP_X)) {
      for (int c = c0; c <= min(c0 + 1, c1); ++c) {
        mbar_expect_tx(&S.xfull[c & 1], tc_xchunk_bytes<B>());
        tma_load_3d(S.x[c & 1], &tmX, &S.xfull[c & 1], 0, 0, c * 2 * TC_KC);
      }
    }
    if (issuer_side) tc_side_work<B>(p, warp, lane, side_first);
    __syncwarp();
    if (lane == 0 && n > 0) {
      const int w = warp;
      bool ok = true;
      auto phase = [&](int c) { return (uint32_t)(((c - c0) >> 1) & 1); };   // use index of buffer c & 1
      int cur_c = -1, xc = -1;                      // chunk retired up to / chunk whose x is acquired
      uint32_t xb = 0;
      const uint32_t idesc = tc_idesc(F16);
      TileIter it;
      it.init(geo, t0 + w);
      for (int k = w; ok; k += TC_WG, it.advance(geo, TC_WG)) {
        const int c = k < n ? it.c : c1 + 1;        // past the end: retire every remaining chunk
        for (; cur_c < c && ok;) {
          if (cur_c >= 0) {
            tc_commit(&S.xempty[cur_c & 1]);        // free once this issuer's MMAs on it finish
            if (w == 0 && cur_c + 2 <= c1) {        // chunk cur_c + 2 reuses that buffer
              const int cn = cur_c + 2, b = cn & 1;
              if (!mbar_wait(&S.xempty[b], phase(cn) ^ 1, wlim)) { ok = false; break; }
              mbar_expect_tx(&S.xfull[b], tc_xchunk_bytes<B>());
              tma_load_3d(S.x[b], &tmX, &S.xfull[b], 0, 0, cn * 2 * TC_KC);
            }
          }
          cur_c = cur_c < 0 ? c0 : cur_c + 1;
        }
        if (!ok || k >= n) break;
        if (c != xc) {
          const int b = c & 1;
          if (!mbar_wait(&S.xfull[b], phase(c), wlim)) { ok = false; break; }
          xb = smem_u32(S.x[b]);
          xc = c;
          tc_fence_after();
        }
        const int i = k / TC_WG, ts = i % TC_TS;
        if (!mbar_wait(&S.afull[w][ts], (i / TC_TS) & 1, wlim)) { ok = false; break; }
        tc_fence_after();
        constexpr uint32_t XBOX = tc_xbox_bytes<B>();
        const uint32_t xg = xb + (uint32_t)(2 * it.gl) * XBOX;
        const uint32_t d = tmem + col_d(w, ts), a = tmem + col_a(w, ts), m = tmem + col_m(w, ts);
        const uint64_t b0 = smem_desc_sw128(xg), b1 = smem_desc_sw128(xg + 64);
        const uint64_t b2 = smem_desc_sw128(xg + XBOX), b3 = smem_desc_sw128(xg + XBOX + 64);
        tc_mma_sp_ta(d, a, b0, m, idesc, 0u);
        tc_mma_sp_ta(d, a + 8, b1, m, idesc | 1u, 1u);
        tc_mma_sp_ta(d, a + 16, b2, m + 4, idesc, 1u);
        tc_mma_sp_ta(d, a + 24, b3, m + 4, idesc | 1u, 1u);

        tc_commit(&S.dfull[w][ts]);
      }
      if (!ok) set_error(p.err, CQL_ERR_TIMEOUT, 21);
    }
  } else {
    // ---------------- converter / accumulator warpgroups ----------------
    const int w = (warp >> 2) - 1, qq = warp & 3;   // qq: tensor-memory lane quarter = row block of the tile
    const int cw = warp - 4;                        // converter warp index
    const int nw = (n - w + TC_WG - 1) / TC_WG;     // tiles of this warpgroup: k = TC_WG i + w
    const uint32_t lane_base = (uint32_t)(32 * qq) << 16;
    const uint32_t sel_meta = (lane & 8) ? 0x3276u : 0x5410u;
    const uint32_t srow = 32u * qq + lane;          // row inside the tile
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;
    bool ok = true;
    bool dep_done = false;                          // griddepcontrol.wait passed (before touching y_acc)
    // This warp's ring: lane l copies, and later reads back, only its own row's
    // 16-byte pieces (codes, META, the scale slab piece holding its group's
    // scale), so no cross-lane synchronisation is needed for them.
    uint8_t* ring = S.ring[cw][0] + lane * 16;
    const uint32_t vstride = (p.rb.values >> 4) * 512u, mstride = (p.rb.meta >> 4) * 512u;
    const uint32_t sstride = (p.rb.scales >> 4) * 512u;
    TileIter ld;                                    // next tile to fetch
    ld.init(geo, t0 + w);
    auto fetch = [&](int slot_i) {
      const uint32_t rb = 4u * ld.rt + qq;
      uint8_t* slot = ring + slot_i * TC_SLOT_BYTES;
#ifdef CQL_CHECKED
      const uint32_t ov = rb * vstride + tc_code_slab<BITS>((uint32_t)ld.g) * 512u + lane * 16;
      const uint32_t om = rb * mstride + (uint32_t)ld.g * 512u + lane * 16;
      const uint32_t os = rb * sstride + (uint32_t)(ld.g >> 3) * 512u + lane * 16;
      if (CQL_IN(p.err, ov + 512 + 15, p.plane_len[CQL_PLANE_VALUES], 111)) {
        cp_async16(slot, p.values + ov);
        cp_async16(slot + 512, p.values + ov + 512);
      }
      if (CQL_IN(p.err, om + 15, p.plane_len[CQL_PLANE_META], 112)) cp_async16(slot + 1024, p.meta + om);
      if (CQL_IN(p.err, os + 15, p.plane_len[CQL_PLANE_SCALES], 113)) cp_async16(slot + 1536, p.scales + os);
#else
      const uint8_t* vsrc = p.values + rb * vstride + tc_code_slab<BITS>((uint32_t)ld.g) * 512u + lane * 16;
      cp_async16(slot, vsrc);
      cp_async16(slot + 512, vsrc + 512);
      cp_async16(slot + 1024, p.meta + rb * mstride + (uint32_t)ld.g * 512u + lane * 16);
      cp_async16(slot + 1536, p.scales + rb * sstride + (uint32_t)(ld.g >> 3) * 512u + lane * 16);
#endif
      if (lane == 0) {
        S.slot_rt[cw][slot_i] = ld.rt;
        S.slot_g[cw][slot_i] = ld.g;
      }
      ld.advance(geo, TC_WG);
    };
#pragma unroll 1
    for (int d = 0; d < TC_RING; ++d) {
      if (d < nw) fetch(d);
      cp_async_commit();
    }
    if (B <= 4) {
      // small batches: no conversion before the dependency resolves (the
      // conversions would take issue slots from the previous call's epilogue,
      // which runs beside this kernel on the same SMs); from 8 batch rows on,
      // converting ahead is worth more
      pdl_wait();
      dep_done = true;
    }
    constexpr bool conv_side = tc_side_workers<B>() != TC_WG;
    bool side_done = !conv_side;
    const SideFirst side_first = conv_side ? tc_side_prefetch<B>(p, cw, lane) : SideFirst{};
    for (int i = 0; i < nw + TC_TS && ok; ++i) {
      // read back tile i - TC_TS: its stage is the one tile i writes
      const int j = i - TC_TS;
      if (conv_side && j == 0) {                    // the first MMA results are some way off
        pdl_wait();
        tc_side_work<B>(p, cw, lane, side_first);
        dep_done = true;
        side_done = true;
      }
      if (j >= 0) {
        const int ts = j % TC_TS;
        ok = __all_sync(0xffffffffu, mbar_wait(&S.dfull[w][ts], (j / TC_TS) & 1, wlim));
        if (!ok) break;
        tc_fence_after();
        float d[B];
        tmem_ld_wait<B>(tmem + lane_base + col_d(w, ts), d);
        const float s = S.scale[w][ts][srow];
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = fmaf(s, d[b], acc[b]);
        const int rt = S.tinfo[w][ts][qq];
        const int rt2 = j + 1 < nw ? S.tinfo[w][(j + 1) % TC_TS][qq] : -1;
        if (rt2 != rt) {                            // last tile of this row tile in this warpgroup's range
          const int row = rt * 128 + (int)srow;
          if (!dep_done) {
            pdl_wait();
            dep_done = true;
          }
#pragma unroll
          for (int b = 0; b < B; ++b) {
            if (b < p.batch && CQL_IN(p.err, (uint64_t)b * p.d.n_out + row, p.y_elems, 114))
              atomicAdd(p.y_acc + (uint64_t)b * p.d.n_out + row, acc[b]);
            acc[b] = 0.0f;
          }
        }
      }
      if (i >= nw) continue;
      // convert tile i into tensor-memory stage i % TC_TS
      const int ts = i % TC_TS, si = i % TC_RING;
      uint8_t* slot = ring + si * TC_SLOT_BYTES;
      cp_async_wait<TC_RING - 1>();
      __syncwarp();                                 // lane 0's slot_rt / slot_g stores
      const uint4 va = *reinterpret_cast<const uint4*>(slot);
      const uint4 vb = *reinterpret_cast<const uint4*>(slot + 512);
      const uint4 mm = *reinterpret_cast<const uint4*>(slot + 1024);
      const int g = S.slot_g[cw][si], rt = S.slot_rt[cw][si];
      const uint32_t sc16 = *reinterpret_cast<const uint16_t*>(slot + 1536 + 2 * (g & 7));
      const uint32_t vw[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
      uint32_t a[32];
      if constexpr (BITS == 4) {
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {
          const uint32_t hi = vw[wi] >> 4;
#pragma unroll
          for (int by = 0; by < 4; ++by)
            a[4 * wi + by] = code_pair<F16>(vw[wi], hi, (uint32_t)(by | (by << 4) | ((4 + by) << 8) | ((4 + by) << 12)));
        }
      } else {
        // the group's 24 bytes start at byte 0 or 8 of the 32 fetched
        // (24 g mod 16); pair m (the group's two kept codes) is stream
        // bits [6 m, 6 m + 6)
        const bool odd = (g & 1) != 0;
        uint32_t ws[7];
#pragma unroll
        for (int k = 0; k < 6; ++k) ws[k] = odd ? vw[k + 2] : vw[k];
        ws[6] = 0u;
#pragma unroll
        for (int m = 0; m < 32; ++m) {
          const int wi = (6 * m) >> 5, sh = (6 * m) & 31;
          const uint32_t six = sh <= 26 ? (ws[wi] >> sh) : __funnelshift_r(ws[wi], ws[wi + 1], sh);
          a[m] = code_pair3<F16>(six);
        }
      }
      // META: this row's 32-bit code word of each K step holds groups 0..7 of
      // it; the sparse MMA wants, in lane 16h + i, rows 16h + i and 16h + 8 + i
      // side by side (16 bits each) for groups 0..3, and in lane 16h + 8 + i
      // the same two rows for groups 4..7.
      const uint32_t mw[4] = {mm.x, mm.y, mm.z, mm.w};
      uint32_t me[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t o = __shfl_xor_sync(0xffffffffu, mw[kk], 8);
        me[kk] = prmt(mw[kk], o, sel_meta);
      }
      __syncwarp();                                 // all lanes read the slot's metadata
      // refill the slot with tile i + TC_RING (after its bytes were used above)
      if (i + TC_RING < nw) fetch(si);
      cp_async_commit();
      tmem_st32(tmem + lane_base + col_a(w, ts), a);
      tmem_st8(tmem + lane_base + col_m(w, ts), me[0], me[1], 0u, 0u, me[2], me[3], 0u, 0u);
      S.scale[w][ts][srow] = f16_bits_to_f32((uint16_t)sc16);
      if (lane == 0) S.tinfo[w][ts][qq] = rt;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.afull[w][ts]);
    }
    cp_async_wait<0>();
    if (!side_done) {                               // no tile here, or stopped early: the side work still runs
      pdl_wait();
      tc_side_work<B>(p, cw, lane, side_first);
    }
    if (!ok && lane == 0) set_error(p.err, CQL_ERR_TIMEOUT, 22);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

}  // namespace

// ---------------------------------------------------------------------------
// host launch
// ---------------------------------------------------------------------------
bool decode_tc_eligible(const DecodeParams& p) {
  return p.d.mask == CQL_MASK_2_4 && (p.d.codec == CQL_CODEC_INT4_SYM || p.d.codec == CQL_CODEC_INT3_SYM) &&
         p.batch >= 1 && p.batch <= 16 && (p.xdt == CQL_DT_BF16 || p.xdt == CQL_DT_F16);
}

template <int B, bool F16, int BITS>
static cudaError_t launch_tc(const DecodeParams& p, cudaStream_t st, bool pdl) {
  TcGeom geo;
  geo.n_rt = p.d.n_out / 128;
  geo.G = p.d.k_in / 128;
  geo.n_chunks = (geo.G + TC_KC - 1) / TC_KC;
  geo.n_tiles = geo.n_rt * geo.G;
  CUtensorMap mx;
  if (!make_map_xchunk(&mx, p.x, (uint64_t)p.batch, (uint64_t)p.d.k_in, tc_xrows<B>(), 2 * TC_KC)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(TcSmem) + 1024;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e = ensure_smem_attr(attr_done, (const void*)k_decode_tc<B, F16, BITS>, (int)smem);
  if (e != cudaSuccess) return e;
  uint64_t grid = (uint64_t)device_sm_count();
  if (grid > (uint64_t)geo.n_tiles) grid = (uint64_t)geo.n_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_decode_tc<B, F16, BITS>, mx, p, geo);
}

template <int B>
static cudaError_t launch_tc_b(const DecodeParams& p, cudaStream_t st, bool pdl) {
  if (p.d.codec == CQL_CODEC_INT3_SYM)
    return p.xdt == CQL_DT_F16 ? launch_tc<B, true, 3>(p, st, pdl) : launch_tc<B, false, 3>(p, st, pdl);
  return p.xdt == CQL_DT_F16 ? launch_tc<B, true, 4>(p, st, pdl) : launch_tc<B, false, 4>(p, st, pdl);
}

cudaError_t launch_decode_tc(const DecodeParams& p, int bpad, cudaStream_t st, bool pdl) {
  switch (bpad) {
    case 1: return launch_tc_b<1>(p, st, pdl);
    case 2: return launch_tc_b<2>(p, st, pdl);
    case 4: return launch_tc_b<4>(p, st, pdl);
    case 8: return launch_tc_b<8>(p, st, pdl);
    default: return launch_tc_b<16>(p, st, pdl);
  }
}

}  // namespace cql
