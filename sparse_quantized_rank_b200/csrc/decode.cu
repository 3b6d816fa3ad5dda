// Decode path (batch 1..16): y = deq(Q (.) M) x + S_csr x + deq(L_q)(deq(R_q) x).
//
// Bandwidth-bound CUDA-core GEMV, no tensor cores.  The design choices:
//
//  * lanes = rows.  A warp owns a block of 32 output rows and walks K in
//    units of 128 columns (one scale group).  The packed planes are row
//    interleaved, so at every step the 32 lanes read 16 consecutive bytes
//    each: one fully coalesced 512-byte access per warp per slab, staged into
//    a per-warp ring of shared memory with cp.async, 4 units in flight.
//  * Because all lanes of a warp sit on the same columns, the activations are
//    warp-uniform.  For the 2:4 mask the x pair a kept pair multiplies,
//    (x[4g+i0], x[4g+i1]), is read from a shared-memory table indexed by the
//    group and the META code (the kept positions, i0 | i1 << 2; 6 valid
//    codes): at most 6 distinct addresses per warp access, all in distinct
//    banks, so one wavefront.  The code becomes a table offset with a shift
//    and a mask.
//  * int4 codes are turned into floats two at a time with byte permutes into
//    the 2^23 magic exponent and one packed fp32x2 subtraction; the products
//    are packed fp32x2 FMAs.  The group scale multiplies the group's partial
//    sum once (SLiM-Quant's per-group scale, review summary "SLIM-Quant").
//  * Work is balanced at unit granularity: the (row block, unit) space is cut
//    into one contiguous range per CTA (persistent grid, one CTA per SM), and
//    each warp takes a contiguous part of it.  Partial row sums are added into
//    an fp32 accumulator with reductions at L2, with no fence or counter on the
//    streaming path.
//  * Three kernels per call, chained by programmatic dependent launch:
//      k_pre       t = R_q x partial sums (SLiM "Low-rank adapter
//                  quantization") and the CSR outlier rows added into the
//                  accumulator (SqueezeLLM "Approach": dense-and-sparse);
//      k_decode    the main term, streaming;
//      k_epilogue  y = accumulator + L_q t, rounding, accumulator reset;
//    each later kernel starts early and waits (griddepcontrol.wait) only where
//    it reads the earlier kernel's results.
#include "common.cuh"
#include "kernels.h"

namespace cql {

constexpr int kDecSmem = 220 * 1024;           // shared memory per CTA: tables + ring
constexpr int kEpiThreads = 128;                // epilogue block: four row blocks = one row group of 128

constexpr uint32_t kMagic = 0x4B000000u;       // fp32 bit pattern of 2^23

CQL_DEV float act(const DecodeParams& p, int b, int col) {
  return b < p.batch && CQL_IN(p.err, (uint64_t)b * p.d.k_in + col, p.x_elems, 201)
             ? to_f32_act(p.x, p.xdt, (uint64_t)b * p.d.k_in + col)
             : 0.0f;
}

CQL_DEV uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// Activations x[b][c0, c0 + ncols) -> fp32 xs[c * B + b] in shared memory,
// eight columns per 16-byte load (ncols is a multiple of 128; rows of x are
// 16-byte aligned).  Batch rows beyond p.batch are zero.
template <int B>
CQL_DEV void stage_x(const DecodeParams& p, float* xs, int c0, int ncols) {
  const int chunks = ncols >> 3;
  const uint16_t* xb = static_cast<const uint16_t*>(p.x);
  for (int i = threadIdx.x; i < B * chunks; i += blockDim.x) {
    const int b = i / chunks, ch = i - b * chunks;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (b < p.batch && CQL_IN(p.err, (uint64_t)b * p.d.k_in + c0 + 8 * ch + 7, p.x_elems, 202))
      w = *reinterpret_cast<const uint4*>(xb + (uint64_t)b * p.d.k_in + c0 + 8 * ch);
    const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t h = (wd[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
      xs[(8 * ch + j) * B + b] = p.xdt == CQL_DT_BF16 ? bf16_bits_to_f32(h) : f16_bits_to_f32(h);
    }
  }
}

// Add a warp's partial row sums into the fp32 accumulator (reductions at L2).
template <int B>
CQL_DEV void red_rows(const DecodeParams& p, int rb, const float (&acc)[B], int lane) {
  const int row = rb * 32 + lane;
#pragma unroll
  for (int b = 0; b < B; ++b)
    if (b < p.batch && CQL_IN(p.err, (uint64_t)b * p.d.n_out + row, p.y_elems, 203))
      atomicAdd(p.y_acc + (uint64_t)b * p.d.n_out + row, acc[b]);
}

// ---------------------------------------------------------------------------
// unit: 2:4 mask, int4 / int3 codes
// ---------------------------------------------------------------------------
CQL_DEV void pair_of(int pt, int& i0, int& i1) {
  i0 = pt < 3 ? 0 : (pt < 5 ? 1 : 2);
  i1 = pt == 0 ? 1 : (pt == 1 || pt == 3 ? 2 : 3);
}

template <int BITS, int B>
struct Unit24 {
  // batch 1 needs little register state: 32 warps per CTA, 2 units in flight
  // each; larger batches keep more accumulators: 16 warps, 4 units in flight
  static constexpr int kThreads = 512;
  static constexpr int kDepth = 4;
  static constexpr int NBP = B == 1 ? 1 : B / 2;                     // batch pairs
  static constexpr int kGroupBytes = B == 1 ? 128 : 256 * NBP;       // 16 entries per group (by META code)
  static constexpr int kTableBytes = 32 * kGroupBytes;
  static constexpr int kUnitBytes = kTableBytes + kGroup * B * 4;   // table + staged x
  struct Frag {
    uint32_t v[8];
    uint32_t m[4];
    uint32_t s;
  };

  // Pair table of the K tile: entry (group, META code i0 | i1 << 2) = the x
  // values of columns i0 and i1 (B == 1), or of two batches (B >= 2); only
  // the six valid codes are written.
  static CQL_DEV void build(const DecodeParams& p, uint8_t* smem, int kt) {
    const int c0 = kt * p.ktu * kGroup;
    const int units = min(p.ktu, p.upr - kt * p.ktu);
    const int ngroups = units * (kGroup / 4);
    float* xs = reinterpret_cast<float*>(smem + (size_t)p.ktu * kTableBytes);
    stage_x<B>(p, xs, c0, units * kGroup);
    __syncthreads();
    // one (group, batch pair) per iteration: read its 4 columns once, write
    // the 6 pattern entries with straight-line stores
    for (int i = threadIdx.x; i < ngroups * NBP; i += blockDim.x) {
      const int bp = i % NBP, g = i / NBP;
      const float* xc = xs + (4 * g) * B + 2 * bp;
      if (B == 1) {
        const float4 x4 = *reinterpret_cast<const float4*>(xc);
        uint8_t* e = smem + g * 128;                   // 8 bytes per code
        *reinterpret_cast<float2*>(e + 8 * 0x4) = make_float2(x4.x, x4.y);                 // (0,1)
        *reinterpret_cast<float4*>(e + 8 * 0x8) = make_float4(x4.x, x4.z, x4.y, x4.z);     // (0,2) (1,2)
        *reinterpret_cast<float4*>(e + 8 * 0xC) = make_float4(x4.x, x4.w, x4.y, x4.w);     // (0,3) (1,3)
        *reinterpret_cast<float2*>(e + 8 * 0xE) = make_float2(x4.z, x4.w);                 // (2,3)
      } else {
        const float2 c0v = *reinterpret_cast<const float2*>(xc);          // column 0, batches b, b+1
        const float2 c1v = *reinterpret_cast<const float2*>(xc + B);
        const float2 c2v = *reinterpret_cast<const float2*>(xc + 2 * B);
        const float2 c3v = *reinterpret_cast<const float2*>(xc + 3 * B);
        float4* e = reinterpret_cast<float4*>(smem + (g * NBP + bp) * 256);   // 16 bytes per code
        e[0x4] = make_float4(c0v.x, c1v.x, c0v.y, c1v.y);
        e[0x8] = make_float4(c0v.x, c2v.x, c0v.y, c2v.y);
        e[0xC] = make_float4(c0v.x, c3v.x, c0v.y, c3v.y);
        e[0x9] = make_float4(c1v.x, c2v.x, c1v.y, c2v.y);
        e[0xD] = make_float4(c1v.x, c3v.x, c1v.y, c3v.y);
        e[0xE] = make_float4(c2v.x, c3v.x, c2v.y, c3v.y);
      }
    }
  }
  static CQL_DEV void on_row(const DecodeParams&, uint8_t*, int, int) {}

  // Stage one unit: its code slabs and pattern slab (cp.async into this
  // lane's 16-byte column of the slot); returns the scale (and, for 3-bit
  // codes, whether the unit starts mid-slab).
  static constexpr int kSlabs = 3;
  static CQL_DEV uint32_t issue(const DecodeParams& p, int rb, int uk, int lane, uint8_t* slot) {
    const uint32_t vs = BITS == 4 ? 2u * uk : (24u * uk) >> 4;
    const uint32_t ov = slab_off32(rb, vs, p.rb.values) + lane * 16, om = slab_off32(rb, uk, p.rb.meta) + lane * 16;
    const uint32_t os = rit32((uint32_t)rb * 32 + lane, 2 * uk, p.rb.scales);
    if (CQL_IN(p.err, ov + 512 + 15, p.plane_len[CQL_PLANE_VALUES], 204)) {
      cp_async16(slot, p.values + ov);
      cp_async16(slot + 512, p.values + ov + 512);
    }
    if (CQL_IN(p.err, om + 15, p.plane_len[CQL_PLANE_META], 205)) cp_async16(slot + 1024, p.meta + om);
    const uint32_t sc = CQL_IN(p.err, os + 1, p.plane_len[CQL_PLANE_SCALES], 206) ? ldg_u16(p.scales + os) : 0u;
    return sc | (BITS == 3 && ((24u * uk) & 15u) ? 0x10000u : 0u);
  }
  static CQL_DEV void gather(const uint8_t* slot, uint32_t sc, Frag& f) {
    const uint4 a = lds128(slot), b = lds128(slot + 512), m = lds128(slot + 1024);
    if (BITS == 4) {
      f.v[0] = a.x; f.v[1] = a.y; f.v[2] = a.z; f.v[3] = a.w;
      f.v[4] = b.x; f.v[5] = b.y; f.v[6] = b.z; f.v[7] = b.w;
    } else {
      const bool odd = (sc >> 16) & 1u;             // codes start at bit 64 of the window
      f.v[0] = odd ? a.z : a.x; f.v[1] = odd ? a.w : a.y; f.v[2] = odd ? b.x : a.z; f.v[3] = odd ? b.y : a.w;
      f.v[4] = odd ? b.z : b.x; f.v[5] = odd ? b.w : b.y; f.v[6] = b.z; f.v[7] = b.w;
    }
    f.m[0] = m.x; f.m[1] = m.y; f.m[2] = m.z; f.m[3] = m.w;
    f.s = sc & 0xFFFFu;
  }

  template <int J>
  static CQL_DEV uint32_t code3(const Frag& f) {      // J-th 3-bit code as magic float bits
    constexpr int bit = 3 * J, wi = bit >> 5, sh = bit & 31;
    if (sh <= 29) return ((f.v[wi] >> sh) & 7u) | kMagic;
    return (__funnelshift_r(f.v[wi], f.v[wi + 1], sh) & 7u) | kMagic;
  }

  template <int GI>
  static CQL_DEV void group(const uint8_t* tb, const Frag& f, uint32_t lo, uint32_t hi, uint64_t (&a2)[B]) {
    constexpr int j = GI & 3;
    uint32_t f0, f1;
    if (BITS == 4) {
      f0 = prmt(lo, kMagic, 0x7540u + j);
      f1 = prmt(hi, kMagic, 0x7540u + j);
    } else {
      f0 = code3<2 * GI>(f);
      f1 = code3<2 * GI + 1>(f);
    }
    constexpr float kBias = BITS == 4 ? -8388616.0f : -8388612.0f;   // -(2^23 + 2^(b-1))
    const uint64_t qq = f2_add(((uint64_t)f1 << 32) | f0, f2_pack(kBias, kBias));
    const uint32_t mw = f.m[GI >> 3];
    constexpr int jn = GI & 7;
    if (B == 1) {
      const uint32_t off = jn == 0 ? ((mw << 3) & 0x78u) : ((mw >> (4 * jn - 3)) & 0x78u);
      const uint64_t xp = *reinterpret_cast<const uint64_t*>(tb + GI * 128 + off);
      a2[0] = f2_fma(qq, xp, a2[0]);
    } else {
      const uint32_t off = jn == 0 ? ((mw << 4) & 0xF0u) : ((mw >> (4 * jn - 4)) & 0xF0u);
#pragma unroll
      for (int bp = 0; bp < NBP; ++bp) {
        const ulonglong2 e = *reinterpret_cast<const ulonglong2*>(tb + (GI * NBP + bp) * 256 + off);
        a2[2 * bp] = f2_fma(qq, e.x, a2[2 * bp]);
        a2[2 * bp + 1] = f2_fma(qq, e.y, a2[2 * bp + 1]);
      }
    }
  }

  template <int I>
  static CQL_DEV void word(const uint8_t* tb, const Frag& f, uint64_t (&a2)[B]) {
    const uint32_t lo = f.v[I] & 0x0F0F0F0Fu, hi = (f.v[I] >> 4) & 0x0F0F0F0Fu;
    group<4 * I + 0>(tb, f, lo, hi, a2);
    group<4 * I + 1>(tb, f, lo, hi, a2);
    group<4 * I + 2>(tb, f, lo, hi, a2);
    group<4 * I + 3>(tb, f, lo, hi, a2);
  }

  static CQL_DEV void compute(const DecodeParams& p, const uint8_t* smem, const Frag& f, int ut, int lane,
                              float (&acc)[B]) {
    const uint8_t* tb = smem + (size_t)ut * kTableBytes;
    uint64_t a2[B];
#pragma unroll
    for (int b = 0; b < B; ++b) a2[b] = 0;
    word<0>(tb, f, a2); word<1>(tb, f, a2); word<2>(tb, f, a2); word<3>(tb, f, a2);
    word<4>(tb, f, a2); word<5>(tb, f, a2); word<6>(tb, f, a2); word<7>(tb, f, a2);
    const float s = f16_bits_to_f32(f.s);
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = fmaf(s, f2_lo(a2[b]) + f2_hi(a2[b]), acc[b]);
  }
};

// ---------------------------------------------------------------------------
// unit: no mask (dense codes), uniform int4/int3 or per-row LUT
// ---------------------------------------------------------------------------
template <int BITS, bool LUT, int B>
struct UnitDense {
  static constexpr int kThreads = 512;
  static constexpr int kDepth = 4;
  static constexpr int kUnitBytes = kGroup * B * 4;        // x tile [128][B] fp32
  static constexpr int kWords = BITS * 4;                  // 128 codes = 16 or 12 words
  struct Frag {
    uint32_t v[kWords];
    uint32_t s;
  };
  // per-warp LUT after the x tile region: [warp][16 codes][32 lanes] fp32
  static CQL_DEV float* lut_base(uint8_t* smem, const DecodeParams& p) {
    return reinterpret_cast<float*>(smem + (size_t)p.ktu * kUnitBytes);
  }
  static CQL_DEV void build(const DecodeParams& p, uint8_t* smem, int kt) {
    const int c0 = kt * p.ktu * kGroup;
    const int ncols = min(p.ktu, p.upr - kt * p.ktu) * kGroup;
    stage_x<B>(p, reinterpret_cast<float*>(smem), c0, ncols);
  }
  static CQL_DEV void on_row(const DecodeParams& p, uint8_t* smem, int rb, int lane) {
    if (!LUT) return;
    float* lut = lut_base(smem, p) + (threadIdx.x >> 5) * (16 * 32);
    const uint64_t row = (uint64_t)rb * 32 + lane;
#pragma unroll
    for (int c = 0; c < (1 << BITS); ++c)
      lut[c * 32 + lane] = CQL_IN(p.err, rit(row, 2 * c, p.rb.scales) + 1, p.plane_len[CQL_PLANE_SCALES], 207)
                               ? f16_bits_to_f32(ldg_u16(p.scales + rit(row, 2 * c, p.rb.scales)))
                               : 0.0f;
    __syncwarp();
  }
  static constexpr int kSlabs = BITS;                     // 64 or 48 bytes of codes per unit
  static CQL_DEV uint32_t issue(const DecodeParams& p, int rb, int uk, int lane, uint8_t* slot) {
    const uint32_t ov = slab_off32(rb, (uint32_t)BITS * uk, p.rb.values) + lane * 16;
    if (CQL_IN(p.err, ov + 512 * (BITS - 1) + 15, p.plane_len[CQL_PLANE_VALUES], 208)) {
#pragma unroll
      for (int s = 0; s < BITS; ++s) cp_async16(slot + 512 * s, p.values + ov + 512 * s);
    }
    if (LUT) return 0u;
    const uint32_t os = rit32((uint32_t)rb * 32 + lane, 2 * uk, p.rb.scales);
    return CQL_IN(p.err, os + 1, p.plane_len[CQL_PLANE_SCALES], 209) ? ldg_u16(p.scales + os) : 0u;
  }
  static CQL_DEV void gather(const uint8_t* slot, uint32_t sc, Frag& f) {
#pragma unroll
    for (int s = 0; s < BITS; ++s) {
      const uint4 a = lds128(slot + 512 * s);
      f.v[4 * s + 0] = a.x; f.v[4 * s + 1] = a.y; f.v[4 * s + 2] = a.z; f.v[4 * s + 3] = a.w;
    }
    f.s = sc;
  }
  template <int C>
  static CQL_DEV uint32_t code(const Frag& f) {
    constexpr int bit = BITS * C, wi = bit >> 5, sh = bit & 31;
    constexpr uint32_t mask = (1u << BITS) - 1;
    if (sh <= 32 - BITS) return (f.v[wi] >> sh) & mask;
    return __funnelshift_r(f.v[wi], f.v[wi + 1], sh) & mask;
  }
  template <int C>
  static CQL_DEV void col(const float* xs, const float* lut, const Frag& f, int lane, float (&a)[B]) {
    const uint32_t c = code<C>(f);
    const float w = LUT ? lut[c * 32 + lane] : (float)((int)c - (1 << (BITS - 1)));
#pragma unroll
    for (int b = 0; b < B; ++b) a[b] = fmaf(w, xs[C * B + b], a[b]);
  }
  template <int C0>
  static CQL_DEV void cols8(const float* xs, const float* lut, const Frag& f, int lane, float (&a)[B]) {
    col<C0 + 0>(xs, lut, f, lane, a); col<C0 + 1>(xs, lut, f, lane, a);
    col<C0 + 2>(xs, lut, f, lane, a); col<C0 + 3>(xs, lut, f, lane, a);
    col<C0 + 4>(xs, lut, f, lane, a); col<C0 + 5>(xs, lut, f, lane, a);
    col<C0 + 6>(xs, lut, f, lane, a); col<C0 + 7>(xs, lut, f, lane, a);
  }
  static CQL_DEV void compute(const DecodeParams& p, const uint8_t* smem, const Frag& f, int ut, int lane,
                              float (&acc)[B]) {
    const float* xs = reinterpret_cast<const float*>(smem) + (size_t)ut * kGroup * B;
    const float* lut = lut_base(const_cast<uint8_t*>(smem), p) + (threadIdx.x >> 5) * (16 * 32);
    float a[B];
#pragma unroll
    for (int b = 0; b < B; ++b) a[b] = 0.0f;
    cols8<0>(xs, lut, f, lane, a); cols8<8>(xs, lut, f, lane, a); cols8<16>(xs, lut, f, lane, a);
    cols8<24>(xs, lut, f, lane, a); cols8<32>(xs, lut, f, lane, a); cols8<40>(xs, lut, f, lane, a);
    cols8<48>(xs, lut, f, lane, a); cols8<56>(xs, lut, f, lane, a); cols8<64>(xs, lut, f, lane, a);
    cols8<72>(xs, lut, f, lane, a); cols8<80>(xs, lut, f, lane, a); cols8<88>(xs, lut, f, lane, a);
    cols8<96>(xs, lut, f, lane, a); cols8<104>(xs, lut, f, lane, a); cols8<112>(xs, lut, f, lane, a);
    cols8<120>(xs, lut, f, lane, a);
    const float s = LUT ? 1.0f : f16_bits_to_f32(f.s);
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = fmaf(s, a[b], acc[b]);
  }
};

// ---------------------------------------------------------------------------
// unit: unstructured 50% bitmap, uniform int4/int3
// ---------------------------------------------------------------------------
template <int BITS, int B>
struct UnitBitmap {
  static constexpr int kThreads = 512;
  static constexpr int kDepth = 4;
  static constexpr int kUnitBytes = kGroup * B * 4;        // x tile [128][B] fp32
  // 96-byte code window per lane: a unit's codes (<= 128 * BITS bits) start
  // at most 127 bits into the first slab, and the funnel shift also reads the
  // word after the last code: 127 + 127 * 4 + 4 < 21 * 32.
  static constexpr int kWinWords = 24;
  struct Frag {
    uint32_t bm[4];
    uint32_t voff;
    uint32_t s;
  };
  static CQL_DEV uint32_t* win_base(uint8_t* smem, const DecodeParams& p) {
    return reinterpret_cast<uint32_t*>(smem + (size_t)p.ktu * kUnitBytes);
  }
  static CQL_DEV void build(const DecodeParams& p, uint8_t* smem, int kt) {
    const int c0 = kt * p.ktu * kGroup;
    const int ncols = min(p.ktu, p.upr - kt * p.ktu) * kGroup;
    stage_x<B>(p, reinterpret_cast<float*>(smem), c0, ncols);
  }
  static CQL_DEV void on_row(const DecodeParams&, uint8_t*, int, int) {}
  static constexpr int kSlabs = 1;                        // the unit's bitmap slab
  static CQL_DEV uint32_t issue(const DecodeParams& p, int rb, int uk, int lane, uint8_t* slot) {
    const uint64_t om = slab_off(rb, uk, p.rb.meta) + lane * 16;
    if (CQL_IN(p.err, om + 15, p.plane_len[CQL_PLANE_META], 210)) cp_async16(slot, p.meta + om);
    const uint64_t row = (uint64_t)rb * 32 + lane;
    const uint64_t oo = rit(row, 2 * uk, p.rb.voff), os = rit(row, 2 * uk, p.rb.scales);
    if (!CQL_IN(p.err, oo + 1, p.plane_len[CQL_PLANE_VOFF], 211) ||
        !CQL_IN(p.err, os + 1, p.plane_len[CQL_PLANE_SCALES], 212))
      return 0u;
    return ldg_u16(p.voff + oo) | (ldg_u16(p.scales + os) << 16);
  }
  static CQL_DEV void gather(const uint8_t* slot, uint32_t sc, Frag& f) {
    const uint4 m = lds128(slot);
    f.bm[0] = m.x; f.bm[1] = m.y; f.bm[2] = m.z; f.bm[3] = m.w;
    f.voff = sc & 0xFFFFu;
    f.s = sc >> 16;
  }
  static CQL_DEV void compute(const DecodeParams& p, uint8_t* smem, const Frag& f, int ut, int lane, int rb,
                              float (&acc)[B]) {
    const float* xs = reinterpret_cast<const float*>(smem) + (size_t)ut * kGroup * B;
    uint32_t* win = win_base(smem, p) + (threadIdx.x >> 5) * (kWinWords * 32);
    const uint32_t bitpos = f.voff * BITS;
    const uint32_t bo = bitpos >> 3;
    const uint32_t nslab = p.rb.values >> 4;
    __syncwarp();
#pragma unroll
    for (int s = 0; s < kWinWords / 4; ++s) {
      const uint32_t sl = min((bo >> 4) + s, nslab - 1);
      const uint64_t ov = slab_off(rb, sl, p.rb.values) + lane * 16;
      const uint4 a = CQL_IN(p.err, ov + 15, p.plane_len[CQL_PLANE_VALUES], 213) ? ldg_stream(p.values + ov)
                                                                                 : make_uint4(0u, 0u, 0u, 0u);
      win[(4 * s + 0) * 32 + lane] = a.x; win[(4 * s + 1) * 32 + lane] = a.y;
      win[(4 * s + 2) * 32 + lane] = a.z; win[(4 * s + 3) * 32 + lane] = a.w;
    }
    __syncwarp();
    uint32_t cb = (bo & 15u) * 8u + (bitpos & 7u);
    constexpr int bias = 1 << (BITS - 1);
    float a[B];
#pragma unroll
    for (int b = 0; b < B; ++b) a[b] = 0.0f;
    // Every column in turn (the same column in all lanes: no divergence, x
    // read as a shared-memory broadcast).  Per 8 columns one 32-bit window
    // of the row's code stream holds their <= 8 kept codes; a column's code
    // sits at the window offset advanced by BITS per kept column before it
    // (bit-field extract), and a pruned column contributes 0.
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t word = f.bm[w];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t wi = cb >> 5, sh = cb & 31u;
        const uint32_t win32 = __funnelshift_r(win[wi * 32 + lane], win[(wi + 1) * 32 + lane], sh);
        uint32_t off = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint32_t bit = (word >> (8 * k + t)) & 1u;
          uint32_t c;
          asm("bfe.u32 %0, %1, %2, %3;" : "=r"(c) : "r"(win32), "r"(off), "n"(BITS));
          // exact integer to float: c under the exponent of 2^23, minus 2^23 + bias
          const float q = bit ? __uint_as_float(c | kMagic) - (8388608.0f + (float)bias) : 0.0f;
          const float* xc = xs + (32 * w + 8 * k + t) * B;
#pragma unroll
          for (int b = 0; b < B; ++b) a[b] = fmaf(q, xc[b], a[b]);
          off += bit * BITS;
        }
        cb += __popc((word >> (8 * k)) & 0xFFu) * BITS;
      }
    }
    const float s = f16_bits_to_f32(f.s);
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = fmaf(s, a[b], acc[b]);
  }
};

// Uniform compute signature across unit kinds.
template <class U, int B>
struct Call {
  static CQL_DEV void compute(const DecodeParams& p, uint8_t* smem, const typename U::Frag& f, int ut, int lane,
                              int, float (&acc)[B]) {
    U::compute(p, smem, f, ut, lane, acc);
  }
};
template <int BITS, int B>
struct Call<UnitBitmap<BITS, B>, B> {
  static CQL_DEV void compute(const DecodeParams& p, uint8_t* smem, const typename UnitBitmap<BITS, B>::Frag& f,
                              int ut, int lane, int rb, float (&acc)[B]) {
    UnitBitmap<BITS, B>::compute(p, smem, f, ut, lane, rb, acc);
  }
};

// ---------------------------------------------------------------------------
// the persistent decode kernel
// ---------------------------------------------------------------------------
CQL_DEV uint64_t tile_begin(const DecodeParams& p, int kt) { return (uint64_t)kt * p.n_rb * p.ktu; }
CQL_DEV int tile_size(const DecodeParams& p, int kt) { return min(p.ktu, p.upr - kt * p.ktu); }
CQL_DEV void unit_coords(const DecodeParams& p, uint64_t u, int& kt, int& rb, int& ut) {
  const uint64_t per_full = (uint64_t)p.n_rb * p.ktu;
  const uint64_t q = u / per_full;
  kt = (int)(q < (uint64_t)(p.n_tiles - 1) ? q : (uint64_t)(p.n_tiles - 1));
  const uint64_t r = u - (uint64_t)kt * per_full;
  const int s = tile_size(p, kt);
  rb = (int)(r / s);
  ut = (int)(r % s);
}


template <class U, int B>
__global__ void __launch_bounds__(U::kThreads, 1) k_decode(DecodeParams p, int ring_off) {
  constexpr int kDepth = U::kDepth;
  constexpr int kDecNW = U::kThreads / 32;
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_launch_dependents();                          // let the epilogue kernel get resident
  if (blockIdx.x == 0 && threadIdx.x == 0 && !header_ok(p)) set_error(p.err, CQL_ERR_FORMAT, 1);
  // this warp's ring of kDepth unit slots; lane l owns bytes [16 l, 16 l + 16) of every 512-byte slab
  uint8_t* ring = smem + ring_off + (size_t)warp * (kDepth * U::kSlabs * 512) + lane * 16;
  const uint64_t U_ = p.n_units;
  const uint64_t ubeg = U_ * blockIdx.x / gridDim.x, uend = U_ * (blockIdx.x + 1) / gridDim.x;
  uint64_t u = ubeg;
  while (u < uend) {
    int kt, rb, ut;
    unit_coords(p, u, kt, rb, ut);
    const uint64_t tnext = tile_begin(p, kt + 1);
    const uint64_t tend = uend < tnext ? uend : tnext;
    const uint64_t n = tend - u;
    const uint64_t wb = u + n * warp / kDecNW, we = u + n * (warp + 1) / kDecNW;
    const int ts = tile_size(p, kt);
    const int uk0 = kt * p.ktu;
    int cur_rb = 0, cur_ut = 0;
    if (wb < we) {
      int kt0;
      unit_coords(p, wb, kt0, cur_rb, cur_ut);
    }
    // prologue: start streaming this warp's first kDepth units before the
    // tile's tables are built (the copies do not depend on them)
    int irb = cur_rb, iut = cur_ut;
    uint32_t sc[kDepth];
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
      sc[d] = 0;
      if (wb + d < we) {
        sc[d] = U::issue(p, irb, uk0 + iut, lane, ring + d * (U::kSlabs * 512));
        if (++iut == ts) { iut = 0; ++irb; }
      }
      cp_async_commit();
    }
    __syncthreads();
    U::build(p, smem, kt);
    __syncthreads();
    if (wb < we) {
      U::on_row(p, smem, cur_rb, lane);
      float acc[B];
#pragma unroll
      for (int b = 0; b < B; ++b) acc[b] = 0.0f;
      int slot = 0;
      for (uint64_t i = wb; i < we; ++i) {
        uint8_t* sl = ring + slot * (U::kSlabs * 512);
        cp_async_wait<kDepth - 1>();
        __syncwarp();
        typename U::Frag f;
        U::gather(sl, sc[0], f);
        __syncwarp();                               // slot contents are in registers
#pragma unroll
        for (int d = 0; d + 1 < kDepth; ++d) sc[d] = sc[d + 1];
        if (i + kDepth < we) {
          sc[kDepth - 1] = U::issue(p, irb, uk0 + iut, lane, sl);
          if (++iut == ts) { iut = 0; ++irb; }
        }
        cp_async_commit();
        if (++slot == kDepth) slot = 0;
        Call<U, B>::compute(p, smem, f, cur_ut, lane, cur_rb, acc);
        int nrb = cur_rb, nut = cur_ut + 1;
        if (nut == ts) { nut = 0; ++nrb; }
        const bool more = i + 1 < we;
        if (!more || nrb != cur_rb) {
          red_rows<B>(p, cur_rb, acc, lane);
#pragma unroll
          for (int b = 0; b < B; ++b) acc[b] = 0.0f;
          if (more) U::on_row(p, smem, nrb, lane);
        }
        cur_rb = nrb;
        cur_ut = nut;
      }
    }
    cp_async_wait<0>();
    u = tend;
  }
  // complete only after the pre-kernel: the epilogue, which waits on this
  // grid, then also sees the pre-kernel's CSR sums and adapter partials
  if (p.has_pre && threadIdx.x == 0) pdl_wait();
}

// ---------------------------------------------------------------------------
// epilogue: a warp per row block (lanes = rows).
//   y = accumulator + deq(L_q) t,  t = sum of the pre-kernel's slices,
// rounded to the output dtype; the accumulator is left zeroed.  The packed L
// codes and scales are read before waiting on the previous kernel; the
// accumulator and t only after.
// ---------------------------------------------------------------------------
// At most 64 registers a thread, so that a block fits beside the tensor-core
// decode kernel (640 threads x 88 registers) and prefetches its L codes (with
// cp.async, into shared memory) while that kernel runs.
template <int B>
__global__ void __maxnreg__(64) k_epilogue(DecodeParams p, int kq) {
  // dynamic shared memory: u[b][j] = s_L[g][j] t[b][j] (B x r floats), then the
  // block's L codes, [32-column chunk m][thread] 16 bytes each
  extern __shared__ __align__(16) uint8_t esm[];
  const int lane = threadIdx.x & 31;
  const int rb = blockIdx.x * (kEpiThreads / 32) + (threadIdx.x >> 5);
  const bool lowrank = p.d.rank > 0 && !(p.flags & CQL_FLAG_NO_LOWRANK);
  const int N = p.d.n_out, r = p.d.rank;
  const int row = rb * 32 + lane;
  const int g = (blockIdx.x * kEpiThreads) / kGroup;   // the block's rows lie in one group of 128
  const int nch = (r + 31) / 32;
  pdl_launch_dependents();                          // the next call's main kernel may start streaming
  float* us = reinterpret_cast<float*>(esm);
  uint8_t* lsm = esm + (size_t)B * p.r_pad * 4;
  uint16_t* ssm = reinterpret_cast<uint16_t*>(lsm + (size_t)nch * kEpiThreads * 16);   // s_L[g][0 .. r)
  if (lowrank) {
    for (int m = 0; m < nch; ++m) {
      const uint64_t ol = slab_off(rb, m, p.rb.l_values) + lane * 16;
      if (CQL_IN(p.err, ol + 15, p.plane_len[CQL_PLANE_L_VALUES], 214))
        cp_async16(lsm + ((size_t)m * kEpiThreads + threadIdx.x) * 16, p.l_values + ol);
    }
    for (int i = threadIdx.x; i < r / 2; i += kEpiThreads)   // r is a multiple of 16
      if (CQL_IN(p.err, 2 * ((uint64_t)g * r + 2 * i) + 3, p.plane_len[CQL_PLANE_L_SCALES], 215))
        cp_async4(ssm + 2 * i, p.l_scales + (uint64_t)g * r + 2 * i);
  }
  cp_async_commit();
  pdl_wait();                                       // main term (and pre-kernel) complete
  float acc[B];
#pragma unroll
  for (int b = 0; b < B; ++b) {
    acc[b] = 0.0f;
    if (b < p.batch && CQL_IN(p.err, (uint64_t)b * N + row, p.y_elems, 216)) acc[b] = ld_cg_f32(p.y_acc + (uint64_t)b * N + row);
  }
  if (lowrank) {
    cp_async_wait<0>();
    __syncthreads();                                // the s_L row copied by other threads
    // every (b, j) of t: the accumulated t (slices == 0: the buffer the main
    // kernel named) or the sum of the pre-kernel's K-slice partials, loaded
    // four at a time
    const float* tfin = p.t_final + (kq == 0 ? (size_t)(ld_cg_u32(p.t_counter + 1) & 1u) * B * p.r_pad : 0);
    if (kq == 0 && blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(p.t_counter, 1u);   // next call: other buffer
    if (kq == 0) {
      // a thread's columns j, all batch rows: B loads in flight before any is used
      for (int j = threadIdx.x; j < r; j += kEpiThreads) {
        float v[B];
#pragma unroll
        for (int b = 0; b < B; ++b)
          v[b] = b < p.batch && CQL_IN(p.err, (uint64_t)(tfin - p.t_final) + (uint64_t)b * p.r_pad + j, p.t_final_elems, 217)
                     ? ld_cg_f32(tfin + (uint64_t)b * p.r_pad + j)
                     : 0.0f;
        const float sl = f16_bits_to_f32(ssm[j]);
#pragma unroll
        for (int b = 0; b < B; ++b) us[b * r + j] = sl * v[b];
      }
    }
    for (int i = threadIdx.x; kq > 0 && i < B * r; i += kEpiThreads) {
      const int b = i / r, j = i - b * r;
      float t0 = 0.0f, t1 = 0.0f, t2 = 0.0f, t3 = 0.0f;
      const float* tp = p.t_part + (uint64_t)b * p.r_pad + j;
      const uint64_t st = (uint64_t)B * p.r_pad;
      int k = 0;
      if (!CQL_IN(p.err, (uint64_t)(tp - p.t_part) + (uint64_t)(kq - 1) * st, p.t_part_elems, 218)) k = kq;   // skip
      for (; k + 4 <= kq; k += 4) {
        t0 += ld_cg_f32(tp + (k + 0) * st);
        t1 += ld_cg_f32(tp + (k + 1) * st);
        t2 += ld_cg_f32(tp + (k + 2) * st);
        t3 += ld_cg_f32(tp + (k + 3) * st);
      }
      for (; k < kq; ++k) t0 += ld_cg_f32(tp + k * st);
      us[i] = f16_bits_to_f32(ssm[j]) * ((t0 + t1) + (t2 + t3));
    }
  }
  __syncthreads();
#pragma unroll
  for (int b = 0; b < B; ++b)
    if (b < p.batch && CQL_IN(p.err, (uint64_t)b * N + row, p.y_elems, 219)) p.y_acc[(uint64_t)b * N + row] = 0.0f;
  if (lowrank && B >= 8) {
    cp_async_wait<0>();
    // 8 and more batch rows: every code is converted once per 8 batch rows,
    // each row's sum running in its own accumulator (the 8 chains are
    // independent of one another)
#pragma unroll
    for (int b0 = 0; b0 < B; b0 += 8)
    for (int m = 0; m < nch; ++m) {
      const uint4 l4 = *reinterpret_cast<const uint4*>(lsm + ((size_t)m * kEpiThreads + threadIdx.x) * 16);
      const uint32_t wd[4] = {l4.x, l4.y, l4.z, l4.w};
      const int nj = min(32, r - 32 * m);           // 16 or 32
#pragma unroll
      for (int jj = 0; jj < 32; jj += 4) {
        if (jj >= nj) break;
        const uint32_t wv = wd[jj >> 3] >> (4 * (jj & 7));
        const float q0 = nib_f32(wv), q1 = nib_f32(wv >> 4), q2 = nib_f32(wv >> 8), q3 = nib_f32(wv >> 12);
#pragma unroll
        for (int b = b0; b < b0 + 8; ++b) {
          const float4 u4 = *reinterpret_cast<const float4*>(us + b * r + 32 * m + jj);
          acc[b] = fmaf(q0, u4.x, fmaf(q1, u4.y, fmaf(q2, u4.z, fmaf(q3, u4.w, acc[b]))));
        }
      }
    }
  } else if (lowrank) {
    cp_async_wait<0>();
    // batch rows in groups of up to 4 (bounded live registers), each with
    // independent partial sums (the FMA chain would otherwise run through all
    // r terms one after the other)
    constexpr int BG = B < 4 ? B : 4;
    constexpr int P = B <= 2 ? 4 : 2;
#pragma unroll
    for (int b0 = 0; b0 < B; b0 += BG) {
      float part[BG][P];
#pragma unroll
      for (int bb = 0; bb < BG; ++bb)
#pragma unroll
        for (int k = 0; k < P; ++k) part[bb][k] = 0.0f;
      for (int m = 0; m < nch; ++m) {
        const uint4 l4 = *reinterpret_cast<const uint4*>(lsm + ((size_t)m * kEpiThreads + threadIdx.x) * 16);
        const uint32_t wd[4] = {l4.x, l4.y, l4.z, l4.w};
        const int nj = min(32, r - 32 * m);         // 16 or 32
#pragma unroll
        for (int jj = 0; jj < 32; jj += 4) {
          if (jj >= nj) break;
          const uint32_t wv = wd[jj >> 3] >> (4 * (jj & 7));
          const float q0 = nib_f32(wv), q1 = nib_f32(wv >> 4), q2 = nib_f32(wv >> 8), q3 = nib_f32(wv >> 12);
#pragma unroll
          for (int bb = 0; bb < BG; ++bb) {
            const float4 u4 = *reinterpret_cast<const float4*>(us + (b0 + bb) * r + 32 * m + jj);
            float& a = part[bb][(jj >> 2) % P];
            a = fmaf(q0, u4.x, fmaf(q1, u4.y, fmaf(q2, u4.z, fmaf(q3, u4.w, a))));
          }
        }
      }
#pragma unroll
      for (int bb = 0; bb < BG; ++bb)
#pragma unroll
        for (int k = 0; k < P; ++k) acc[b0 + bb] += part[bb][k];
    }
  }
#pragma unroll
  for (int b = 0; b < B; ++b)
    if (b < p.batch && CQL_IN(p.err, (uint64_t)b * N + row, p.y_elems, 220)) store_out(p.y, p.ydt, (uint64_t)b * N + row, acc[b]);
}

// ---------------------------------------------------------------------------
// pre-kernel, PDL primary of the decode kernel:
//  * blocks [0, n_s1): low-rank stage 1, t = deq(R_q) x.  Block (R row block,
//    K slice of up to 8 units): a warp per unit, partial sums reduced in shared
//    memory, one partial per K slice in t_part; the epilogue sums the slices
//    in a fixed order (deterministic).
//  * blocks [n_s1, ..): the CSR outliers, a thread per output row, added into
//    the fp32 accumulator (SqueezeLLM "Approach": the sparse part of the
//    dense-and-sparse decomposition).
// The epilogue kernel reads these results only after griddepcontrol.wait
// (the main kernel completes only after this grid).
// ---------------------------------------------------------------------------
constexpr int kS1Units = 8;

template <int B>
__global__ void __launch_bounds__(256, 1) k_pre(DecodeParams p, int n_s1) {
  pdl_launch_dependents();
  extern __shared__ __align__(16) float s1[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (blockIdx.x < n_s1) {
    const int KQ = (p.upr + kS1Units - 1) / kS1Units;
    const int rbR = blockIdx.x / KQ, kq = blockIdx.x % KQ;
    const int u0 = kq * kS1Units, u1 = min(p.upr, u0 + kS1Units);
    const int j = 32 * rbR + lane;
    const int u = u0 + warp;                          // one unit per warp (kS1Units == 8 warps)
    uint4 q4[4];
    float sc = 0.0f;
    if (u < u1) {                                     // R codes first: they do not depend on x
      const uint64_t ob = slab_off(rbR, 4 * u, p.rb.r_values) + lane * 16;
      const uint64_t os = rit(j, 2 * u, p.rb.r_scales);
      const bool okv = CQL_IN(p.err, ob + 3 * 512 + 15, p.plane_len[CQL_PLANE_R_VALUES], 221);
#pragma unroll
      for (int s = 0; s < 4; ++s) q4[s] = okv ? ldg_stream(p.r_values + ob + 512 * s) : make_uint4(0u, 0u, 0u, 0u);
      sc = CQL_IN(p.err, os + 1, p.plane_len[CQL_PLANE_R_SCALES], 222) ? f16_bits_to_f32(ldg_u16(p.r_scales + os)) : 0.0f;
    }
    stage_x<B>(p, s1, u0 * kGroup, (u1 - u0) * kGroup);
    __syncthreads();
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;
    if (u < u1) {
      const float* xs = s1 + (u - u0) * kGroup * B;
      float au[B];
#pragma unroll
      for (int b = 0; b < B; ++b) au[b] = 0.0f;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t wd[4] = {q4[s].x, q4[s].y, q4[s].z, q4[s].w};
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float q = (float)((int)((wd[k >> 3] >> (4 * (k & 7))) & 15u) - 8);
#pragma unroll
          for (int b = 0; b < B; ++b) au[b] = fmaf(q, xs[(32 * s + k) * B + b], au[b]);
        }
      }
#pragma unroll
      for (int b = 0; b < B; ++b) acc[b] = sc * au[b];
    }
    __syncthreads();                                   // x no longer needed: reuse for partials
#pragma unroll
    for (int b = 0; b < B; ++b) s1[(warp * B + b) * 32 + lane] = acc[b];
    __syncthreads();
    for (int i = threadIdx.x; i < B * 32; i += blockDim.x) {
      const int b = i >> 5, l = i & 31;
      float t = 0.0f;
#pragma unroll
      for (int w = 0; w < 8; ++w) t += s1[(w * B + b) * 32 + l];
      if (CQL_IN(p.err, ((uint64_t)kq * B + b) * p.r_pad + 32 * rbR + l, p.t_part_elems, 223))
        p.t_part[((uint64_t)kq * B + b) * p.r_pad + 32 * rbR + l] = t;
    }
  } else {
    const int row = (blockIdx.x - n_s1) * blockDim.x + threadIdx.x;
    if (row >= p.d.n_out) return;
    if (!CQL_IN(p.err, 4ull * row + 7, p.plane_len[CQL_PLANE_CSR_ROWPTR], 224)) return;
    int e0 = p.csr_rowptr[row], e1 = p.csr_rowptr[row + 1];
    e0 = max(0, min(e0, (int)p.nnz));
    e1 = max(e0, min(e1, (int)p.nnz));
    if (e1 == e0) return;
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;
    for (int e = e0; e < e1; e += 8) {
      int col[8];
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool ok = e + i < e1;
        col[i] = ok ? (int)p.csr_col[e + i] : 0;
        v[i] = ok ? f16_bits_to_f32(p.csr_val[e + i]) : 0.0f;
        if (col[i] >= p.d.k_in) { col[i] = 0; v[i] = 0.0f; }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = fmaf(v[i], act(p, b, col[i]), acc[b]);
    }
#pragma unroll
    for (int b = 0; b < B; ++b)
      if (b < p.batch && CQL_IN(p.err, (uint64_t)b * p.d.n_out + row, p.y_elems, 225))
        atomicAdd(p.y_acc + (uint64_t)b * p.d.n_out + row, acc[b]);
  }
}

// ---------------------------------------------------------------------------
// host launch
// ---------------------------------------------------------------------------
int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!cache[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = v > 0 ? v : 148;
  }
  return cache[dev];
}

template <class U, int B>
static cudaError_t launch_unit(DecodeParams p, int unit_bytes, int extra_bytes, cudaStream_t st, bool pdl) {
  const int ring = (U::kThreads / 32) * U::kDepth * U::kSlabs * 512;
  int ktu = (kDecSmem - ring - extra_bytes) / unit_bytes;
  ktu = max(1, min(ktu, p.upr));
  p.ktu = ktu;
  p.n_tiles = (p.upr + ktu - 1) / ktu;
  const int ring_off = ktu * unit_bytes + extra_bytes;
  const size_t smem = (size_t)ring_off + ring;
  static std::atomic<uint64_t> attr_done{0};   // per instantiation and device: allow the opt-in maximum
  {
    int dev = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaError_t e = ensure_smem_attr(attr_done, (const void*)k_decode<U, B>, optin > 0 ? optin : (int)smem);
    if (e != cudaSuccess) return e;
  }
  uint64_t grid = (uint64_t)device_sm_count();
  if (grid > p.n_units) grid = p.n_units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(U::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_decode<U, B>, p, ring_off);
}

static cudaError_t launch_pdl(const void* f, void** args, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelExC(&cfg, f, args);
}

template <int B>
static cudaError_t launch_main(const DecodeParams& p, cudaStream_t st, bool pdl) {
  const int bits = codec_bits(p.d.codec);
  if (p.d.mask == CQL_MASK_2_4) {
    if (bits == 4) return launch_unit<Unit24<4, B>, B>(p, Unit24<4, B>::kUnitBytes, 0, st, pdl);
    return launch_unit<Unit24<3, B>, B>(p, Unit24<3, B>::kUnitBytes, 0, st, pdl);
  }
  if (p.d.mask == CQL_MASK_BITMAP50) {
    const int extra = (UnitBitmap<4, B>::kThreads / 32) * UnitBitmap<4, B>::kWinWords * 32 * 4;
    if (bits == 4) return launch_unit<UnitBitmap<4, B>, B>(p, UnitBitmap<4, B>::kUnitBytes, extra, st, pdl);
    return launch_unit<UnitBitmap<3, B>, B>(p, UnitBitmap<3, B>::kUnitBytes, extra, st, pdl);
  }
  const int lut_extra = (UnitDense<3, true, B>::kThreads / 32) * 16 * 32 * 4;
  switch (p.d.codec) {
    case CQL_CODEC_INT4_SYM:
      return launch_unit<UnitDense<4, false, B>, B>(p, UnitDense<4, false, B>::kUnitBytes, 0, st, pdl);
    case CQL_CODEC_INT3_SYM:
      return launch_unit<UnitDense<3, false, B>, B>(p, UnitDense<3, false, B>::kUnitBytes, 0, st, pdl);
    case CQL_CODEC_LUT3_ROW:
      return launch_unit<UnitDense<3, true, B>, B>(p, UnitDense<3, true, B>::kUnitBytes, lut_extra, st, pdl);
    default:
      return launch_unit<UnitDense<4, true, B>, B>(p, UnitDense<4, true, B>::kUnitBytes, lut_extra, st, pdl);
  }
}

template <int B>
static size_t epilogue_smem(const DecodeParams& p) {
  const size_t r = (size_t)p.d.rank;
  return (size_t)B * p.r_pad * 4 + ((r + 31) / 32) * kEpiThreads * 16 + (size_t)p.r_pad * 2;   // u, L codes, s_L
}

// pre (adapter partials, CSR rows) -> main term -> epilogue, each PDL-chained
// to the one before it.
template <int B>
static cudaError_t launch_decode_b(const DecodeParams& p0, cudaStream_t st) {
  DecodeParams p = p0;
  const bool lowrank = p.d.rank > 0 && !(p.flags & CQL_FLAG_NO_LOWRANK);
  const bool csr = p.csr_rowptr != nullptr && !(p.flags & CQL_FLAG_NO_CSR);
  const int kq = (p.upr + kS1Units - 1) / kS1Units;
  const int n_s1 = lowrank ? (p.r_pad / 32) * kq : 0;
  const int n_csr = csr ? (p.d.n_out + 255) / 256 : 0;
  p.has_pre = (n_s1 + n_csr) > 0;
  cudaError_t e;
  const bool main_on = !(p.flags & CQL_FLAG_NO_MAIN);
  if (main_on && decode_tc_eligible(p) && !(p.flags & CQL_FLAG_CUDA_CORE)) {
    // tensor-core path: the main kernel also adds the CSR rows and t = R x
    // (into t_final); the epilogue reads t_final directly (slices = 0)
    p.has_pre = 0;
    if ((e = launch_decode_tc(p, B, st, true)) != cudaSuccess) return e;
    int zero = 0;
    void* args0[2] = {&p, &zero};
    const dim3 grid0((p.n_rb * 32 + kEpiThreads - 1) / kEpiThreads);
    return launch_pdl((const void*)k_epilogue<B>, args0, grid0, dim3(kEpiThreads), epilogue_smem<B>(p), st, true);
  }
  if (p.has_pre) {
    const size_t smem = (size_t)kS1Units * kGroup * B * 4;
    static std::atomic<uint64_t> attr_done{0};
    if ((e = ensure_smem_attr(attr_done, (const void*)k_pre<B>, (int)smem)) != cudaSuccess) return e;
    k_pre<B><<<n_s1 + n_csr, 256, smem, st>>>(p, n_s1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (main_on) {
    if ((e = launch_main<B>(p, st, p.has_pre)) != cudaSuccess) return e;
  }
  int kq_arg = kq;
  void* args[2] = {&p, &kq_arg};
  const dim3 grid((p.n_rb * 32 + kEpiThreads - 1) / kEpiThreads);
  return launch_pdl((const void*)k_epilogue<B>, args, grid, dim3(kEpiThreads), epilogue_smem<B>(p), st,
                    main_on || p.has_pre);
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st) {
  const int b = p.batch;
  if (b <= 1) return launch_decode_b<1>(p, st);
  if (b <= 2) return launch_decode_b<2>(p, st);
  if (b <= 4) return launch_decode_b<4>(p, st);
  if (b <= 8) return launch_decode_b<8>(p, st);
  return launch_decode_b<16>(p, st);
}

}  // namespace cql
