// Shared device/host helpers of libcql (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

#include "../../include/cql.h"

#define CQL_DEV __device__ __forceinline__
#define CQL_HD __host__ __device__ __forceinline__

namespace cql {

constexpr int kRowBlk = 32;     // rows per interleaved row block
constexpr int kSlab = 16;       // bytes per row per slab
constexpr int kGroup = 128;     // scale group (columns)

CQL_HD uint64_t pad16(uint64_t x) { return (x + 15) & ~uint64_t(15); }
CQL_HD uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }
CQL_HD int codec_bits(int codec) { return (codec == CQL_CODEC_INT4_SYM || codec == CQL_CODEC_LUT4_ROW) ? 4 : 3; }
CQL_HD bool codec_is_lut(int codec) { return codec == CQL_CODEC_LUT3_ROW || codec == CQL_CODEC_LUT4_ROW; }

// Byte offset of byte j of row i in a row-interleaved plane whose rows are
// row_bytes long (a multiple of 16).
CQL_HD uint64_t rit(uint64_t i, uint64_t j, uint64_t row_bytes) {
  return ((i >> 5) * (row_bytes >> 4) + (j >> 4)) * 512u + (i & 31u) * 16u + (j & 15u);
}
// Offset of slab s of row block rb (the 512-byte run lane l of a warp reads at +16 l).
CQL_HD uint64_t slab_off(uint64_t rb, uint64_t s, uint64_t row_bytes) {
  return (rb * (row_bytes >> 4) + s) * 512u;
}
// Offsets inside one plane fit in 32 bits (N * K <= 2^32 keeps every plane
// below 4 GB), so the per-unit address arithmetic stays 32-bit.
CQL_DEV uint32_t slab_off32(uint32_t rb, uint32_t s, uint32_t row_bytes) { return (rb * (row_bytes >> 4) + s) * 512u; }
CQL_DEV uint32_t rit32(uint32_t i, uint32_t j, uint32_t row_bytes) {
  return ((i >> 5) * (row_bytes >> 4) + (j >> 4)) * 512u + (i & 31u) * 16u + (j & 15u);
}

// Per-plane row bytes of the packed format (see include/cql.h).
struct RowBytes {
  uint32_t values, meta, scales, voff, r_values, r_scales, l_values;
};

CQL_HD RowBytes row_bytes_of(const cql_desc& d) {
  RowBytes rb{};
  const uint64_t k = (uint64_t)d.k_in;
  const int bits = codec_bits(d.codec);
  const uint64_t kept = (d.mask == CQL_MASK_NONE) ? k : k / 2;
  rb.values = (uint32_t)pad16((kept * bits + 7) / 8);
  rb.meta = (d.mask == CQL_MASK_NONE) ? 0u : (uint32_t)(k / 8);
  rb.scales = codec_is_lut(d.codec) ? (uint32_t)(2u << bits) : (uint32_t)pad16(2 * (k / kGroup));
  rb.voff = (d.mask == CQL_MASK_BITMAP50) ? (uint32_t)pad16(2 * (k / kGroup)) : 0u;
  rb.r_values = d.rank ? (uint32_t)(k / 2) : 0u;
  rb.r_scales = d.rank ? (uint32_t)pad16(2 * (k / kGroup)) : 0u;
  rb.l_values = d.rank ? (uint32_t)pad16((uint64_t)d.rank / 2) : 0u;
  return rb;
}

// ---------------------------------------------------------------------------
// device error word (first 8 bytes of every workspace): status, detail
// ---------------------------------------------------------------------------
CQL_DEV void set_error(uint32_t* err, uint32_t status, uint32_t detail) {
  if (atomicCAS(err, 0u, status) == 0u) atomicExch(err + 1, detail);
}

// Range checks of the checked build (compiled with -DCQL_CHECKED, the
// library's stand-in for a memory checker): CQL_IN(err, i, n, site) is true
// when 0 <= i < n; otherwise it records CQL_ERR_RANGE with the site number
// as the detail and the caller skips the access.  In the normal build it is
// the constant true and costs nothing.
CQL_DEV bool in_range(uint32_t* err, uint64_t i, uint64_t n, uint32_t site) {
  if (i < n) return true;
  set_error(err, CQL_ERR_RANGE, site);
  return false;
}
#ifdef CQL_CHECKED
#define CQL_IN(err, i, n, site) ::cql::in_range((err), (uint64_t)(i), (uint64_t)(n), (site))
#else
#define CQL_IN(err, i, n, site) true
#endif

// ---------------------------------------------------------------------------
// exact conversions
// ---------------------------------------------------------------------------
CQL_DEV float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }
CQL_DEV float f16_bits_to_f32(uint32_t b) { return __half2float(__ushort_as_half((unsigned short)b)); }

// Round an fp64 value to binary16, round to nearest, ties to even, in one
// step from the fp64 bits (no intermediate fp32 rounding).  Written from the
// IEEE 754 binary16 definition: 10 fraction bits, exponent bias 15, minimum
// normal exponent -14, subnormal quantum 2^-24.  Overflow gives infinity.
CQL_HD uint16_t f64_to_f16_bits(double x) {
#ifdef __CUDA_ARCH__
  const uint64_t b = (uint64_t)__double_as_longlong(x);
#else
  uint64_t b;
  memcpy(&b, &x, 8);
#endif
  const uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
  const uint64_t a = b & 0x7FFFFFFFFFFFFFFFull;
  if (a == 0) return sign;
  if (a >= 0x7FF0000000000000ull) return (uint16_t)(sign | 0x7C00u);   // inf/nan -> inf
  const int e_raw = (int)(a >> 52);
  if (e_raw == 0) return sign;                       // fp64 subnormal: far below fp16 range
  const int e = e_raw - 1023;                        // value = m * 2^(e-52), m in [2^52, 2^53)
  const uint64_t m = (a & ((1ull << 52) - 1)) | (1ull << 52);
  const int eq = (e < -14 ? -14 : e);                // exponent of the fp16 binade
  const int shift = 42 + (eq - e);                   // m * 2^(e-52) / 2^(eq-10) = m >> shift
  if (shift >= 64) return sign;                      // < 2^-25 (never a tie here): rounds to 0
  uint64_t r = m >> shift;
  const uint64_t rem = m & ((1ull << shift) - 1);
  const uint64_t half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (r & 1))) r += 1;
  uint32_t bits;
  if (e < -14) {
    bits = (uint32_t)r;                              // subnormal (r == 1024 -> min normal)
  } else {
    bits = (uint32_t)(((uint32_t)(e + 15) << 10) + (uint32_t)(r - 1024));   // carry bumps exponent
  }
  if (bits >= 0x7C00u) bits = 0x7C00u;
  return (uint16_t)(sign | bits);
}

CQL_DEV float to_f32_act(const void* x, int dt, uint64_t idx) {
  const uint16_t b = reinterpret_cast<const uint16_t*>(x)[idx];
  return dt == CQL_DT_BF16 ? bf16_bits_to_f32(b) : f16_bits_to_f32(b);
}

CQL_DEV void store_out(void* y, int dt, uint64_t idx, float v) {
  if (dt == CQL_DT_F32) {
    reinterpret_cast<float*>(y)[idx] = v;
  } else if (dt == CQL_DT_F16) {
    reinterpret_cast<__half*>(y)[idx] = __float2half_rn(v);
  } else {
    reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
  }
}

// Byte-permute: result byte i = byte sel_i of {b:a} (a = bytes 0-3, b = 4-7).
CQL_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Packed fp32x2 arithmetic (sm_100): two lanes of fp32 in one instruction.
CQL_DEV uint64_t f2_pack(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
CQL_DEV float f2_lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
CQL_DEV float f2_hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
CQL_DEV uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
CQL_DEV uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 128-bit read-only streaming load (data is read once per call).
CQL_DEV uint4 ldg_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
CQL_DEV uint32_t ldg_u16(const uint8_t* p) { return __ldg(reinterpret_cast<const unsigned short*>(p)); }
CQL_DEV uint32_t ld_cg_u32(const uint32_t* p) {
  uint32_t r;
  asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
CQL_DEV float ld_cg_f32(const float* p) {
  float r;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(r) : "l"(p));
  return r;
}

// Signed int4 code (stored u = q + 8) in bits 0..3 of y as the float q,
// without an integer-to-float conversion: with u in the low mantissa bits of
// 2^23 the float is 2^23 + u exactly.
CQL_DEV float nib_f32(uint32_t y) { return __uint_as_float((y & 0x0Fu) | 0x4B000000u) - 8388616.0f; }

// Programmatic dependent launch controls (no-ops without a PDL edge).
// 16-byte asynchronous global -> shared copies (LSU path), grouped per thread.
CQL_DEV void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}
CQL_DEV void cp_async4(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}
CQL_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
CQL_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

CQL_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
CQL_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace cql
