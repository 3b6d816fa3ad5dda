// Parameter blocks and launch entry points shared by the host API and the
// kernel translation units of libcql.
#pragma once
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
};

struct PackWorkspace {
  uint64_t out_bits, state, hist, tiecnt, tieoff, row_counts, total;
};
PackWorkspace pack_workspace_layout(const cql_desc& d);

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
  uint32_t* t_counter;   // [1]   low-rank stage-1 arrival counter
  float* y_acc;          // [batch][N]
  uint32_t* counters;    // [N/32]
  float* t_part;         // [upr][batch][r_pad]
  float* t_final;        // [batch][r_pad]
};

struct ForwardWorkspace {
  uint64_t err, t_counter, y_acc, counters, t_part, t_final, prefill, total;
};
ForwardWorkspace forward_workspace_layout(const cql_desc& d, int batch);

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st);

// Prefill scratch (inside the forward workspace): byte offsets.
struct PrefillLayout {
  int r3;          // adapter extension columns (3 r rounded up to 64)
  int rrows;       // R rows padded to 128
  int r_pad;       // rank rounded up to 32
  int ldq;         // K + r3
  uint64_t qbf, wsc, rbf, rsc, tacc, t3, total;
};
PrefillLayout prefill_layout(const cql_desc& d, int m);
bool prefill_supported(const cql_desc& d, int x_dt);
cudaError_t launch_prefill(const DecodeParams& p, uint8_t* prefill_ws, cudaStream_t st);

}  // namespace cql
