// Decode path (batch 1..16): y = deq(Q (.) M) x + S_csr x + deq(L_q)(deq(R_q) x).
//
// Bandwidth-bound CUDA-core GEMV, no tensor cores.  The design choices:
//
//  * lanes = rows.  A warp owns a block of 32 output rows and walks K in
//    units of 128 columns (one scale group).  The packed planes are row
//    interleaved, so at every step the 32 lanes read 16 consecutive bytes
//    each: one fully coalesced 512-byte access per warp per slab.
//  * Because all lanes of a warp sit on the same columns, the activations are
//    warp-uniform.  For the 2:4 mask the x pair a kept pair multiplies,
//    (x[4g+i0], x[4g+i1]), is read from a shared-memory table indexed by the
//    group and the pattern nibble (6 patterns): at most 6 distinct addresses
//    per warp access, all in distinct banks, so one wavefront.  The metadata
//    nibble becomes a table offset with a shift and a mask.
//  * int4 codes are turned into floats two at a time with byte permutes into
//    the 2^23 magic exponent and one packed fp32x2 subtraction; the products
//    are packed fp32x2 FMAs.  The group scale multiplies the group's partial
//    sum once (SLiM-Quant's per-group scale, review summary "SLIM-Quant").
//  * Work is balanced at unit granularity: the (row block, unit) space is cut
//    into one contiguous range per CTA (persistent grid over all SMs).  Partial
//    row sums are added into an fp32 accumulator with reductions at L2; the
//    warp that completes a row block (arrival counter) runs the epilogue: the
//    CSR outliers of its rows (SqueezeLLM "Approach": dense-and-sparse), the
//    second low-rank stage L_q t (SLiM "Low-rank adapter quantization"), the
//    final rounding, and the reset of the accumulator for the next call.
//  * The first low-rank stage t = R_q x runs in its own small kernel that
//    starts the main kernel at once through programmatic dependent launch; the
//    epilogue waits on it with griddepcontrol.wait, long after it finished.
#include "common.cuh"
#include "kernels.h"

namespace cql {

constexpr int kDecNT = 512;                    // threads per decode CTA
// Batch 1 runs two CTAs per SM (64 registers per thread, <= 100 KB of tables
// each); larger batches need more accumulator registers and run one CTA per
// SM with up to 200 KB of tables.
template <int B> struct DecCfg {
  static constexpr int kMinBlocks = B == 1 ? 2 : 1;
  static constexpr int kSmemBudget = B == 1 ? 100 * 1024 : 200 * 1024;
};
constexpr uint32_t kMagic = 0x4B000000u;       // fp32 bit pattern of 2^23

CQL_DEV float act(const DecodeParams& p, int b, int col) {
  return b < p.batch ? to_f32_act(p.x, p.xdt, (uint64_t)b * p.d.k_in + col) : 0.0f;
}
CQL_DEV uint32_t ldg_u16(const uint8_t* p) { return __ldg(reinterpret_cast<const unsigned short*>(p)); }

// ---------------------------------------------------------------------------
// epilogue for one row block: accumulator + CSR + low rank -> y
// ---------------------------------------------------------------------------
template <int B>
CQL_DEV void finish_rowblock(const DecodeParams& p, int rb, int lane) {
  const int N = p.d.n_out, K = p.d.k_in;
  const int row = rb * 32 + lane;
  float acc[B];
#pragma unroll
  for (int b = 0; b < B; ++b) {
    acc[b] = 0.0f;
    if (b < p.batch) {
      float* a = p.y_acc + (uint64_t)b * N + row;
      acc[b] = ld_cg_f32(a);
      *a = 0.0f;
    }
  }
  if (p.csr_rowptr != nullptr && !(p.flags & CQL_FLAG_NO_CSR)) {
    int e0 = p.csr_rowptr[row], e1 = p.csr_rowptr[row + 1];
    e0 = max(0, min(e0, (int)p.nnz));
    e1 = max(e0, min(e1, (int)p.nnz));
    for (int e = e0; e < e1; ++e) {
      const int col = p.csr_col[e];
      if (col >= K) continue;
      const float v = f16_bits_to_f32(p.csr_val[e]);
#pragma unroll
      for (int b = 0; b < B; ++b) acc[b] = fmaf(v, act(p, b, col), acc[b]);
    }
  }
  if (p.d.rank > 0 && !(p.flags & CQL_FLAG_NO_LOWRANK)) {
    pdl_wait();                                   // stage 1 (t = R_q x) complete
    const int r = p.d.rank, g = row / kGroup;
    for (int m = 0; m * 32 < r; ++m) {
      const int j = 32 * m + lane;
      float u[B];
      const float ls = j < r ? f16_bits_to_f32(p.l_scales[(uint64_t)g * r + j]) : 0.0f;
#pragma unroll
      for (int b = 0; b < B; ++b) u[b] = j < r ? ls * ld_cg_f32(p.t_final + (uint64_t)b * p.r_pad + j) : 0.0f;
      const uint4 w = ldg_stream(p.l_values + slab_off(rb, m, p.rb.l_values) + lane * 16);
      const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        if (32 * m + jj >= r) break;
        const float q = (float)((int)((wd[jj >> 3] >> (4 * (jj & 7))) & 15u) - 8);
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = fmaf(q, __shfl_sync(0xffffffffu, u[b], jj), acc[b]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < B; ++b)
    if (b < p.batch) store_out(p.y, p.ydt, (uint64_t)b * N + row, acc[b]);
  if (lane == 0) p.counters[rb] = 0u;
}

// Add a warp's partial sums of a row block and count its units; the warp
// that completes the row block runs the epilogue.
template <int B>
CQL_DEV void flush_rowblock(const DecodeParams& p, int rb, uint32_t units, const float (&acc)[B], int lane) {
  const int N = p.d.n_out;
  const int row = rb * 32 + lane;
#pragma unroll
  for (int b = 0; b < B; ++b)
    if (b < p.batch) atomicAdd(p.y_acc + (uint64_t)b * N + row, acc[b]);
  __threadfence();
  __syncwarp();
  uint32_t old = 0;
  if (lane == 0) old = atomicAdd(p.counters + rb, units);
  old = __shfl_sync(0xffffffffu, old, 0);
  if (old + units == (uint32_t)p.upr) {
    __threadfence();
    finish_rowblock<B>(p, rb, lane);
  }
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
  static constexpr int NBP = B == 1 ? 1 : B / 2;                     // batch pairs
  static constexpr int kGroupBytes = B == 1 ? 64 : 128 * NBP;        // 8 patterns per group
  static constexpr int kUnitBytes = 32 * kGroupBytes;
  struct Frag {
    uint32_t v[8];
    uint32_t m[4];
    uint32_t s;
  };

  static CQL_DEV void build(const DecodeParams& p, uint8_t* smem, int kt) {
    const int c0 = kt * p.ktu * kGroup;
    const int ngroups = min(p.ktu, p.upr - kt * p.ktu) * (kGroup / 4);
    for (int i = threadIdx.x; i < ngroups * NBP * 6; i += blockDim.x) {
      const int pt = i % 6, t2 = i / 6, bp = t2 % NBP, g = t2 / NBP;
      int i0, i1;
      pair_of(pt, i0, i1);
      const int col = c0 + 4 * g;
      if (B == 1) {
        *reinterpret_cast<float2*>(smem + g * 64 + pt * 8) = make_float2(act(p, 0, col + i0), act(p, 0, col + i1));
      } else {
        const int b = 2 * bp;
        *reinterpret_cast<float4*>(smem + ((g * NBP + bp) * 8 + pt) * 16) =
            make_float4(act(p, b, col + i0), act(p, b, col + i1), act(p, b + 1, col + i0), act(p, b + 1, col + i1));
      }
    }
  }
  static CQL_DEV void on_row(const DecodeParams&, uint8_t*, int, int) {}

  static CQL_DEV void load(const DecodeParams& p, int rb, int uk, int lane, Frag& f) {
    if (BITS == 4) {
      const uint8_t* vb = p.values + slab_off(rb, 2 * uk, p.rb.values) + lane * 16;
      const uint4 a = ldg_stream(vb), b = ldg_stream(vb + 512);
      f.v[0] = a.x; f.v[1] = a.y; f.v[2] = a.z; f.v[3] = a.w;
      f.v[4] = b.x; f.v[5] = b.y; f.v[6] = b.z; f.v[7] = b.w;
    } else {
      const uint32_t byte0 = 24u * uk;
      const uint8_t* vb = p.values + slab_off(rb, byte0 >> 4, p.rb.values) + lane * 16;
      const uint4 a = ldg_stream(vb), b = ldg_stream(vb + 512);
      const bool odd = (byte0 & 15u) != 0;          // codes start at bit 64 of the window
      f.v[0] = odd ? a.z : a.x; f.v[1] = odd ? a.w : a.y; f.v[2] = odd ? b.x : a.z; f.v[3] = odd ? b.y : a.w;
      f.v[4] = odd ? b.z : b.x; f.v[5] = odd ? b.w : b.y; f.v[6] = b.z; f.v[7] = b.w;
    }
    const uint4 m = ldg_stream(p.meta + slab_off(rb, uk, p.rb.meta) + lane * 16);
    f.m[0] = m.x; f.m[1] = m.y; f.m[2] = m.z; f.m[3] = m.w;
    f.s = ldg_u16(p.scales + rit((uint64_t)rb * 32 + lane, 2 * uk, p.rb.scales));
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
      const uint32_t off = jn == 0 ? ((mw << 3) & 0x38u) : ((mw >> (4 * jn - 3)) & 0x38u);
      const uint64_t xp = *reinterpret_cast<const uint64_t*>(tb + GI * 64 + off);
      a2[0] = f2_fma(qq, xp, a2[0]);
    } else {
      const uint32_t off = jn == 0 ? ((mw << 4) & 0x70u) : ((mw >> (4 * jn - 4)) & 0x70u);
#pragma unroll
      for (int bp = 0; bp < NBP; ++bp) {
        const ulonglong2 e = *reinterpret_cast<const ulonglong2*>(tb + (GI * NBP + bp) * 128 + off);
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
    const uint8_t* tb = smem + (size_t)ut * kUnitBytes;
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
    float* xs = reinterpret_cast<float*>(smem);
    for (int i = threadIdx.x; i < ncols * B; i += blockDim.x) xs[i] = act(p, i % B, c0 + i / B);
  }
  static CQL_DEV void on_row(const DecodeParams& p, uint8_t* smem, int rb, int lane) {
    if (!LUT) return;
    float* lut = lut_base(smem, p) + (threadIdx.x >> 5) * (16 * 32);
    const uint64_t row = (uint64_t)rb * 32 + lane;
#pragma unroll
    for (int c = 0; c < (1 << BITS); ++c) lut[c * 32 + lane] = f16_bits_to_f32(ldg_u16(p.scales + rit(row, 2 * c, p.rb.scales)));
    __syncwarp();
  }
  static CQL_DEV void load(const DecodeParams& p, int rb, int uk, int lane, Frag& f) {
    constexpr int slabs = BITS;                            // 64 or 48 bytes per unit
    const uint8_t* vb = p.values + slab_off(rb, (uint64_t)slabs * uk, p.rb.values) + lane * 16;
#pragma unroll
    for (int s = 0; s < slabs; ++s) {
      const uint4 a = ldg_stream(vb + 512 * s);
      f.v[4 * s + 0] = a.x; f.v[4 * s + 1] = a.y; f.v[4 * s + 2] = a.z; f.v[4 * s + 3] = a.w;
    }
    f.s = LUT ? 0u : ldg_u16(p.scales + rit((uint64_t)rb * 32 + lane, 2 * uk, p.rb.scales));
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
    float* xs = reinterpret_cast<float*>(smem);
    for (int i = threadIdx.x; i < ncols * B; i += blockDim.x) xs[i] = act(p, i % B, c0 + i / B);
  }
  static CQL_DEV void on_row(const DecodeParams&, uint8_t*, int, int) {}
  static CQL_DEV void load(const DecodeParams& p, int rb, int uk, int lane, Frag& f) {
    const uint4 m = ldg_stream(p.meta + slab_off(rb, uk, p.rb.meta) + lane * 16);
    f.bm[0] = m.x; f.bm[1] = m.y; f.bm[2] = m.z; f.bm[3] = m.w;
    const uint64_t row = (uint64_t)rb * 32 + lane;
    f.voff = ldg_u16(p.voff + rit(row, 2 * uk, p.rb.voff));
    f.s = ldg_u16(p.scales + rit(row, 2 * uk, p.rb.scales));
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
      const uint4 a = ldg_stream(p.values + slab_off(rb, sl, p.rb.values) + lane * 16);
      win[(4 * s + 0) * 32 + lane] = a.x; win[(4 * s + 1) * 32 + lane] = a.y;
      win[(4 * s + 2) * 32 + lane] = a.z; win[(4 * s + 3) * 32 + lane] = a.w;
    }
    __syncwarp();
    uint32_t cb = (bo & 15u) * 8u + (bitpos & 7u);
    constexpr uint32_t mask = (1u << BITS) - 1;
    constexpr int bias = 1 << (BITS - 1);
    float a[B];
#pragma unroll
    for (int b = 0; b < B; ++b) a[b] = 0.0f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t word = f.bm[w];
      while (word) {
        const int t = __ffs(word) - 1;
        word &= word - 1;
        const uint32_t wi = cb >> 5, sh = cb & 31u;
        const uint32_t c = __funnelshift_r(win[wi * 32 + lane], win[(wi + 1) * 32 + lane], sh) & mask;
        cb += BITS;
        const float q = (float)((int)c - bias);
        const float* xc = xs + (32 * w + t) * B;
#pragma unroll
        for (int b = 0; b < B; ++b) a[b] = fmaf(q, xc[b], a[b]);
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

CQL_DEV bool header_ok(const DecodeParams& p) {
  const uint32_t* h = reinterpret_cast<const uint32_t*>(p.header);
  const int32_t* d = reinterpret_cast<const int32_t*>(p.header + 8);
  return h[0] == 0x314C5143u /* "CQL1" */ && h[1] == CQL_VERSION && d[0] == p.d.n_out && d[1] == p.d.k_in &&
         d[2] == p.d.mask && d[3] == p.d.codec && d[7] == p.d.rank;
}

template <class U, int B>
__global__ void __launch_bounds__(kDecNT, DecCfg<B>::kMinBlocks) k_decode(DecodeParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = kDecNT / 32;
  if (blockIdx.x == 0 && threadIdx.x == 0 && !header_ok(p)) set_error(p.err, CQL_ERR_FORMAT, 1);
  const uint64_t U_ = p.n_units;
  const uint64_t ubeg = U_ * blockIdx.x / gridDim.x, uend = U_ * (blockIdx.x + 1) / gridDim.x;
  uint64_t u = ubeg;
  while (u < uend) {
    int kt, rb, ut;
    unit_coords(p, u, kt, rb, ut);
    const uint64_t tnext = tile_begin(p, kt + 1);
    const uint64_t tend = uend < tnext ? uend : tnext;
    __syncthreads();
    U::build(p, smem, kt);
    __syncthreads();
    const uint64_t n = tend - u;
    const uint64_t wb = u + n * warp / NW, we = u + n * (warp + 1) / NW;
    if (wb < we) {
      int kt0, cur_rb, cur_ut;
      unit_coords(p, wb, kt0, cur_rb, cur_ut);
      const int ts = tile_size(p, kt);
      const int uk0 = kt * p.ktu;
      typename U::Frag cur, nxt;
      U::load(p, cur_rb, uk0 + cur_ut, lane, cur);
      U::on_row(p, smem, cur_rb, lane);
      float acc[B];
#pragma unroll
      for (int b = 0; b < B; ++b) acc[b] = 0.0f;
      uint32_t cnt = 0;
      for (uint64_t i = wb; i < we; ++i) {
        int nrb = cur_rb, nut = cur_ut + 1;
        if (nut == ts) { nut = 0; ++nrb; }
        const bool more = i + 1 < we;
        if (more) U::load(p, nrb, uk0 + nut, lane, nxt);
        Call<U, B>::compute(p, smem, cur, cur_ut, lane, cur_rb, acc);
        ++cnt;
        if (!more || nrb != cur_rb) {
          flush_rowblock<B>(p, cur_rb, cnt, acc, lane);
#pragma unroll
          for (int b = 0; b < B; ++b) acc[b] = 0.0f;
          cnt = 0;
          if (more) U::on_row(p, smem, nrb, lane);
        }
        cur = nxt;
        cur_rb = nrb;
        cur_ut = nut;
      }
    }
    u = tend;
  }
}

// Epilogue only (main term disabled by CQL_FLAG_NO_MAIN): a warp per row block.
template <int B>
__global__ void __launch_bounds__(256, 1) k_finish_only(DecodeParams p) {
  const int lane = threadIdx.x & 31;
  const int rb = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (blockIdx.x == 0 && threadIdx.x == 0 && !header_ok(p)) set_error(p.err, CQL_ERR_FORMAT, 1);
  if (rb >= p.n_rb) return;
  finish_rowblock<B>(p, rb, lane);
}

// ---------------------------------------------------------------------------
// low-rank stage 1: t = deq(R_q) x  (one CTA per 128-column group, a warp per
// 32 adapter rows), deterministic final sum by the last CTA
// ---------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(256, 1) k_lowrank_stage1(DecodeParams p) {
  pdl_launch_dependents();
  __shared__ float xs[B][kGroup];
  __shared__ bool s_last;
  const int g = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < B * kGroup; i += blockDim.x) xs[i / kGroup][i % kGroup] = act(p, i / kGroup, g * kGroup + i % kGroup);
  __syncthreads();
  for (int w = warp; w < p.r_pad / 32; w += blockDim.x / 32) {
    const uint8_t* base = p.r_values + slab_off(w, 4 * g, p.rb.r_values) + lane * 16;
    float acc[B];
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b] = 0.0f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint4 q4 = ldg_stream(base + 512 * s);
      const uint32_t wd[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float q = (float)((int)((wd[k >> 3] >> (4 * (k & 7))) & 15u) - 8);
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = fmaf(q, xs[b][32 * s + k], acc[b]);
      }
    }
    const int j = 32 * w + lane;
    const float sc = f16_bits_to_f32(ldg_u16(p.r_scales + rit(j, 2 * g, p.rb.r_scales)));
#pragma unroll
    for (int b = 0; b < B; ++b) p.t_part[((uint64_t)g * B + b) * p.r_pad + j] = acc[b] * sc;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(p.t_counter, 1u) == gridDim.x - 1;
  __syncthreads();
  if (s_last) {
    __threadfence();
    for (int i = threadIdx.x; i < B * p.r_pad; i += blockDim.x) {
      const int b = i / p.r_pad, j = i % p.r_pad;
      float s = 0.0f;
      for (int gg = 0; gg < (int)gridDim.x; ++gg) s += ld_cg_f32(p.t_part + ((uint64_t)gg * B + b) * p.r_pad + j);
      p.t_final[(uint64_t)b * p.r_pad + j] = s;
    }
    if (threadIdx.x == 0) *p.t_counter = 0u;
  }
}

// ---------------------------------------------------------------------------
// host launch
// ---------------------------------------------------------------------------
static int sm_count() {
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
  int ktu = (DecCfg<B>::kSmemBudget - extra_bytes) / unit_bytes;
  ktu = max(1, min(ktu, p.upr));
  p.ktu = ktu;
  p.n_tiles = (p.upr + ktu - 1) / ktu;
  const size_t smem = (size_t)ktu * unit_bytes + extra_bytes;
  static bool attr_set = false;       // once per instantiation: allow the opt-in maximum
  if (!attr_set) {
    int dev = 0, optin = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaError_t e = cudaFuncSetAttribute((const void*)k_decode<U, B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         optin > 0 ? optin : (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int per_sm = DecCfg<B>::kMinBlocks;
  uint64_t grid = (uint64_t)sm_count() * per_sm;
  if (grid > p.n_units) grid = p.n_units;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kDecNT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_decode<U, B>, p);
}

template <int B>
static cudaError_t launch_decode_b(const DecodeParams& p, cudaStream_t st) {
  const bool lowrank = p.d.rank > 0 && !(p.flags & CQL_FLAG_NO_LOWRANK);
  if (lowrank) {
    k_lowrank_stage1<B><<<p.upr, 256, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.flags & CQL_FLAG_NO_MAIN) {
    const int blocks = (p.n_rb * 32 + 255) / 256;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = lowrank ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_finish_only<B>, p);
  }
  const int bits = codec_bits(p.d.codec);
  if (p.d.mask == CQL_MASK_2_4) {
    if (bits == 4) return launch_unit<Unit24<4, B>, B>(p, Unit24<4, B>::kUnitBytes, 0, st, lowrank);
    return launch_unit<Unit24<3, B>, B>(p, Unit24<3, B>::kUnitBytes, 0, st, lowrank);
  }
  if (p.d.mask == CQL_MASK_BITMAP50) {
    const int extra = (kDecNT / 32) * UnitBitmap<4, B>::kWinWords * 32 * 4;
    if (bits == 4) return launch_unit<UnitBitmap<4, B>, B>(p, UnitBitmap<4, B>::kUnitBytes, extra, st, lowrank);
    return launch_unit<UnitBitmap<3, B>, B>(p, UnitBitmap<3, B>::kUnitBytes, extra, st, lowrank);
  }
  const int lut_extra = (kDecNT / 32) * 16 * 32 * 4;
  switch (p.d.codec) {
    case CQL_CODEC_INT4_SYM:
      return launch_unit<UnitDense<4, false, B>, B>(p, UnitDense<4, false, B>::kUnitBytes, 0, st, lowrank);
    case CQL_CODEC_INT3_SYM:
      return launch_unit<UnitDense<3, false, B>, B>(p, UnitDense<3, false, B>::kUnitBytes, 0, st, lowrank);
    case CQL_CODEC_LUT3_ROW:
      return launch_unit<UnitDense<3, true, B>, B>(p, UnitDense<3, true, B>::kUnitBytes, lut_extra, st, lowrank);
    default:
      return launch_unit<UnitDense<4, true, B>, B>(p, UnitDense<4, true, B>::kUnitBytes, lut_extra, st, lowrank);
  }
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
