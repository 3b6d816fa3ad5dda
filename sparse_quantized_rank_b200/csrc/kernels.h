// Parameter blocks and launch entry points shared by the host API and the
// kernel translation units of libcql.
#pragma once
#include <cuda.h>

#include <atomic>

#include "common.cuh"

namespace cql {

constexpr int kTopkChunk = 8192;    // elements per block in the outlier tie pass

struct TopkState {
  uint32_t prefix, mask, want, pad;
};

struct HeaderBytes {
  uint64_t b[CQL_HEADER_BYTES / 8];
};

struct PackParams {
  cql_desc d;
  RowBytes rb;
  const void* W;
  int wdt;
  const float* L;
  const float* R;
  double alpha;                      // clip_alpha widened to fp64
  uint64_t nnz_target;               // floor(f N K)
  uint8_t* packed;
  uint8_t* values;
  uint8_t* meta;
  uint8_t* scales;
  uint8_t* voff;
  int32_t* csr_rowptr;
  uint16_t* csr_col;
  uint16_t* csr_val;
  uint8_t* r_values;
  uint8_t* r_scales;
  uint8_t* l_values;
  uint16_t* l_scales;
  // workspace
  uint32_t* out_bits;                // [N*K/32] outlier bitmask (or null)
  TopkState* topk_state;
  uint32_t* topk_hist;               // [256]
  uint32_t* topk_tiecnt;             // [nblk]
  uint32_t* topk_tieoff;             // [nblk+1]
  uint32_t* row_counts;              // [N]
  // SLiM^O (salient_channels > 0): input statistic, output plane, scratch
  const float* act_absmean;          // [K] mean |x_c|
  uint16_t* salient;                 // SALIENT plane [m]
  float* w_scaled;                   // [N*K] W' (fp32)
  double* sal_partial;               // [N/64][K]
  double* sal;                       // [K]
  uint8_t* sal_flag;                 // [K]
  // SLiM-Quant alpha search (clip_alpha 0) and SqueezeLLM Fisher k-means
  float* alpha_dev;                  // the searched alpha (device), or null: use 'alpha'
  unsigned long long* alpha_hist;    // [1024] histogram
  const float* fisher;               // [N*K] Fisher diagonal (LUT codecs), or null
  // range checks (checked build): error word, plane lengths in bytes
  uint32_t* err;                     // first word of the pack workspace
  uint64_t plane_len[CQL_NPLANES];
};

struct PackWorkspace {
  uint64_t err, out_bits, state, hist, tiecnt, tieoff, row_counts, w_scaled, sal_partial, sal, sal_flag, alpha, total;
};
PackWorkspace pack_workspace_layout(const cql_desc& d);

// SLiM^O packer step: selects the salient channels (SALIENT plane) and
// writes W' into the workspace; on return p.W / p.wdt name W' (fp32).
cudaError_t launch_salient_pack(PackParams& p, cudaStream_t st);

cudaError_t launch_pack(const PackParams& p, const HeaderBytes& hdr, uint64_t total_bytes,
                        cudaStream_t st);

struct DecodeParams {
  cql_desc d;
  RowBytes rb;
  const uint8_t* header;
  const uint8_t* values;
  const uint8_t* meta;
  const uint8_t* scales;
  const uint8_t* voff;
  const int32_t* csr_rowptr;
  const uint16_t* csr_col;
  const uint16_t* csr_val;
  const uint8_t* r_values;
  const uint8_t* r_scales;
  const uint8_t* l_values;
  const uint16_t* l_scales;
  uint64_t nnz;
  uint64_t plane_len[CQL_NPLANES];   // bytes of every plane (the checked build's bounds)
  uint64_t x_elems, y_elems;         // batch * K, batch * N
  uint64_t t_final_elems;            // floats in t_final
  uint64_t t_part_elems;             // floats in t_part
  const void* x;
  int xdt;
  void* y;
  int ydt;
  int batch;
  uint32_t flags;
  // geometry
  int n_rb;          // N / 32
  int upr;           // units (128 columns) per row = K / 128
  int ktu;           // units per K tile
  int n_tiles;
  uint64_t n_units;  // n_rb * upr
  int r_pad;         // rank rounded up to 32
  int has_pre;       // a pre-kernel (adapter stage 1 and/or CSR rows) runs first, PDL-overlapped
  // workspace
  uint32_t* err;         // [2]
  uint32_t* t_counter;   // [2]   tensor-core path: [0] calls so far (bumped by the epilogue), [1] the
                         //       t buffer of the current call (written by the main kernel)
  float* y_acc;          // [batch][N]
  uint32_t* counters;    // [N/32]
  float* t_part;         // [upr][batch][r_pad]
  float* t_final;        // [2][batch][r_pad]  tensor-core path: t = R x, the buffer alternating by call
};

struct ForwardWorkspace {
  uint64_t err, t_counter, y_acc, counters, t_part, t_final, xs, prefill, total;
};
ForwardWorkspace forward_workspace_layout(const cql_desc& d, int batch);

// The packed header matches the descriptor the call was made with.
CQL_DEV bool header_ok(const DecodeParams& p) {
  const uint32_t* h = reinterpret_cast<const uint32_t*>(p.header);
  const int32_t* d = reinterpret_cast<const int32_t*>(p.header + 8);
  return h[0] == 0x314C5143u /* "CQL1" */ && h[1] == CQL_VERSION && d[0] == p.d.n_out && d[1] == p.d.k_in &&
         d[2] == p.d.mask && d[3] == p.d.codec && d[7] == p.d.rank && d[11] == p.d.salient_channels &&
         d[12] == p.d.salient_log2;
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st);

// SLiM-LoRA / Naive-LoRA adapter construction (lora.cu).
struct LoraWorkspace {
  uint64_t es, y, y2, z, z2, g, u, ri, v, sig, ord, colf, xbarp, total;
};
int lora_width(const cql_desc& d);                     // subspace width p
LoraWorkspace lora_workspace_layout(const cql_desc& d);
// p: the layer's planes (as for a forward); act: mean |x_c| or null
// (Naive-LoRA); salient: the SALIENT plane (SLiM^O) or null.
cudaError_t launch_build_adapters(const DecodeParams& p, const void* W, int wdt, const float* act,
                                  const uint16_t* salient, uint8_t* ws, float* L, float* R, cudaStream_t st);

// SLiM^O forward prologue: xs = x with the listed channels divided by
// 2^salient_log2 (same dtype, [batch][K]); PDL-chained to the kernel before.
cudaError_t launch_salient_x(const DecodeParams& p, const uint16_t* list, void* xs, cudaStream_t st);

// Device address of compressed_linear_forward_noalloc's scratch array on the
// current device (nullptr before its first call there).
void* noalloc_scratch_current_device();

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) applies to the device that
// is current when it runs, so the opt-in is made once per (kernel, device):
// 'done' holds one bit per device index (a repeated call is harmless).
inline cudaError_t ensure_smem_attr(std::atomic<uint64_t>& done, const void* f, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Tensor-core decode of the main term (2:4 mask, int4 codes, bf16/f16 x).
bool decode_tc_eligible(const DecodeParams& p);
cudaError_t launch_decode_tc(const DecodeParams& p, int bpad, cudaStream_t st, bool pdl);
int device_sm_count();

// Tensor maps (tma_host.cu); false when the driver rejects the encoding.
// 2-D 16-bit row-major matrix [rows][cols] (ld elements per row): boxes of
// box_rows x 64 columns, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows);
// 16-bit x [batch][k] seen as [k/64 column blocks][batch rows][64 columns]:
// one box of box_blocks x box_rows x 64 lands as box_blocks consecutive
// 128-byte-swizzled [box_rows][64] tiles (rows past the batch read as zero).
bool make_map_xchunk(CUtensorMap* m, const void* x, uint64_t batch, uint64_t k, uint32_t box_rows, uint32_t box_blocks);
// A row-interleaved plane seen as [n_blocks][block_bytes] (8-byte elements, no
// swizzle): one box copies box_bytes from each of box_blocks consecutive row
// blocks.
bool make_map_rowblocks(CUtensorMap* m, const void* plane, uint64_t block_bytes, uint64_t n_blocks,
                        uint32_t box_bytes, uint32_t box_blocks);

// Prefill scratch (inside the forward workspace): byte offsets.
struct PrefillLayout {
  bool sparse;     // 2:4 int4 / int3: the sparse GEMM (weights dequantised on chip)
  int r3;          // adapter extension columns (3 r rounded up to 64)
  int rrows;       // R rows padded to 128
  int r_pad;       // rank rounded up to 32
  int ldq;         // K + r3
  uint64_t qbf, wsc, rbf, rsc, tacc, t3, total;
};
PrefillLayout prefill_layout(const cql_desc& d, int m);
bool prefill_supported(const cql_desc& d, int x_dt);
cudaError_t launch_prefill(const DecodeParams& p, uint8_t* prefill_ws, cudaStream_t st);
// The sparse-tensor-core GEMM of 2:4 int4 layers (prefill_sp.cu): lbuf holds
// the adapter columns [N][r3], t3 the split T = X R^T [m][r3].
cudaError_t launch_pf_sgemm(const DecodeParams& p, const uint16_t* lbuf, int r3, const uint16_t* t3, bool lowrank,
                            cudaStream_t st);

}  // namespace cql
