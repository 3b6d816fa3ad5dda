// libcql host ABI: validation, packed layout, workspace layout, dispatch.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

using namespace cql;

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

cql_status validate_desc(const cql_desc* d) {
  if (d == nullptr) return CQL_ERR_ARG;
  if (d->n_out <= 0 || d->n_out % 128 != 0 || d->n_out > (1 << 20)) return CQL_ERR_ARG;
  if (d->k_in <= 0 || d->k_in % 128 != 0 || d->k_in > 65536) return CQL_ERR_ARG;
  if ((uint64_t)d->n_out * (uint64_t)d->k_in > (1ull << 32)) return CQL_ERR_ARG;
  if (d->mask < CQL_MASK_NONE || d->mask > CQL_MASK_BITMAP50) return CQL_ERR_ARG;
  if (d->codec < CQL_CODEC_INT4_SYM || d->codec > CQL_CODEC_LUT4_ROW) return CQL_ERR_ARG;
  if (d->group != 128 || d->adapter_bits != 4 || d->adapter_group != 128) return CQL_ERR_UNSUPPORTED;
  if (!(d->clip_alpha >= 0.0f && d->clip_alpha <= 1.0f)) return CQL_ERR_ARG;   // 0: search it
  if (!(d->outlier_frac >= 0.0f && d->outlier_frac <= 0.0625f)) return CQL_ERR_ARG;
  if (d->rank < 0 || d->rank > 256 || d->rank % 16 != 0) return CQL_ERR_ARG;
  if (d->salient_channels < 0 || d->salient_channels > d->k_in / 8) return CQL_ERR_ARG;
  if (d->salient_channels > 0 ? (d->salient_log2 < 1 || d->salient_log2 > 8) : d->salient_log2 != 0)
    return CQL_ERR_ARG;
  if (codec_is_lut(d->codec)) {
    if (d->mask != CQL_MASK_NONE) return CQL_ERR_UNSUPPORTED;
    if (d->k_in > 16384) return CQL_ERR_UNSUPPORTED;          // per-row sort lives in shared memory
  }
  return CQL_OK;
}

uint64_t n_outliers(const cql_desc& d) {
  if (!(d.outlier_frac > 0.0f)) return 0;
  return (uint64_t)floor((double)d.outlier_frac * (double)d.n_out * (double)d.k_in);
}

void compute_layout(const cql_desc& d, cql_layout* L) {
  const RowBytes rb = row_bytes_of(d);
  const uint64_t n = (uint64_t)d.n_out, r = (uint64_t)d.rank;
  const uint64_t rpad = (r + 31) / 32 * 32;
  const uint64_t nnz = n_outliers(d);
  uint64_t len[CQL_NPLANES] = {0};
  len[CQL_PLANE_HEADER] = CQL_HEADER_BYTES;
  len[CQL_PLANE_VALUES] = n * rb.values;
  len[CQL_PLANE_META] = n * rb.meta;
  len[CQL_PLANE_SCALES] = n * rb.scales;
  len[CQL_PLANE_VOFF] = n * rb.voff;
  if (d.outlier_frac > 0.0f) {
    len[CQL_PLANE_CSR_ROWPTR] = 4 * (n + 1);
    len[CQL_PLANE_CSR_COL] = 2 * nnz;
    len[CQL_PLANE_CSR_VAL] = 2 * nnz;
  }
  if (r) {
    len[CQL_PLANE_R_VALUES] = rpad * rb.r_values;
    len[CQL_PLANE_R_SCALES] = rpad * rb.r_scales;
    len[CQL_PLANE_L_VALUES] = n * rb.l_values;
    len[CQL_PLANE_L_SCALES] = 2 * (n / 128) * r;
  }
  len[CQL_PLANE_SALIENT] = 2 * (uint64_t)d.salient_channels;
  uint64_t pos = 0;
  for (int i = 0; i < CQL_NPLANES; ++i) {
    pos = align256(pos);
    L->off[i] = pos;
    L->len[i] = len[i];
    pos += len[i];
  }
  L->total_bytes = align256(pos);
  L->nnz = nnz;
}

HeaderBytes make_header(const cql_desc& d, const cql_layout& L) {
  HeaderBytes h;
  memset(&h, 0, sizeof(h));
  uint8_t* b = reinterpret_cast<uint8_t*>(h.b);
  memcpy(b, "CQL1", 4);
  const uint32_t ver = CQL_VERSION;
  memcpy(b + 4, &ver, 4);
  memcpy(b + 8, &d, sizeof(cql_desc));
  memcpy(b + 72, &L.total_bytes, 8);
  memcpy(b + 80, &L.nnz, 8);
  memcpy(b + 88, L.off, 8 * CQL_NPLANES);
  memcpy(b + 88 + 8 * CQL_NPLANES, L.len, 8 * CQL_NPLANES);
  static_assert(88 + 16 * CQL_NPLANES <= CQL_HEADER_BYTES, "header size");
  return h;
}

// The layer's plane pointers and sizes, as every kernel reads them.
DecodeParams planes_of(const cql_desc& d, const void* packed, const cql_layout& lay) {
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.d = d;
  p.rb = row_bytes_of(d);
  p.header = base;
  p.values = base + lay.off[CQL_PLANE_VALUES];
  p.meta = base + lay.off[CQL_PLANE_META];
  p.scales = base + lay.off[CQL_PLANE_SCALES];
  p.voff = base + lay.off[CQL_PLANE_VOFF];
  p.csr_rowptr = d.outlier_frac > 0.0f ? reinterpret_cast<const int32_t*>(base + lay.off[CQL_PLANE_CSR_ROWPTR]) : nullptr;
  p.csr_col = reinterpret_cast<const uint16_t*>(base + lay.off[CQL_PLANE_CSR_COL]);
  p.csr_val = reinterpret_cast<const uint16_t*>(base + lay.off[CQL_PLANE_CSR_VAL]);
  p.r_values = base + lay.off[CQL_PLANE_R_VALUES];
  p.r_scales = base + lay.off[CQL_PLANE_R_SCALES];
  p.l_values = base + lay.off[CQL_PLANE_L_VALUES];
  p.l_scales = reinterpret_cast<const uint16_t*>(base + lay.off[CQL_PLANE_L_SCALES]);
  p.nnz = lay.nnz;
  for (int i = 0; i < CQL_NPLANES; ++i) p.plane_len[i] = lay.len[i];
  return p;
}

int padded_batch(int b) {
  if (b <= 1) return 1;
  if (b <= 2) return 2;
  if (b <= 4) return 4;
  if (b <= 8) return 8;
  return 16;
}

}  // namespace

namespace cql {

PackWorkspace pack_workspace_layout(const cql_desc& d) {
  PackWorkspace w{};
  const uint64_t total = (uint64_t)d.n_out * d.k_in;
  const uint64_t nblk = (total + kTopkChunk - 1) / kTopkChunk;
  uint64_t pos = 0;
  w.err = pos;       pos = align256(pos + 8);       // device error word (read by cql_get_device_status)
  w.out_bits = pos;  pos = align256(pos + (d.outlier_frac > 0.0f ? total / 8 : 0));
  w.state = pos;     pos = align256(pos + sizeof(TopkState));
  w.hist = pos;      pos = align256(pos + 256 * 4);
  w.tiecnt = pos;    pos = align256(pos + nblk * 4);
  w.tieoff = pos;    pos = align256(pos + (nblk + 1) * 4);
  w.row_counts = pos; pos = align256(pos + (uint64_t)d.n_out * 4);
  const bool sal = d.salient_channels > 0;
  w.w_scaled = pos;  pos = align256(pos + (sal ? total * 4 : 0));
  w.sal_partial = pos; pos = align256(pos + (sal ? (uint64_t)(d.n_out / 64) * d.k_in * 8 : 0));
  w.sal = pos;       pos = align256(pos + (sal ? (uint64_t)d.k_in * 8 : 0));
  w.sal_flag = pos;  pos = align256(pos + (sal ? (uint64_t)d.k_in : 0));
  w.alpha = pos;     pos = align256(pos + 1024 * 8 + 16);    // alpha histogram, then the alpha
  w.total = pos;
  return w;
}

ForwardWorkspace forward_workspace_layout(const cql_desc& d, int batch) {
  ForwardWorkspace w{};
  const uint64_t n = (uint64_t)d.n_out;
  const uint64_t upr = (uint64_t)d.k_in / 128;
  const uint64_t rpad = ((uint64_t)d.rank + 31) / 32 * 32;
  const uint64_t bp = batch <= CQL_MAX_DECODE_BATCH ? (uint64_t)padded_batch(batch) : 0;
  uint64_t pos = 0;
  w.err = pos;       pos = align256(pos + 8);
  w.t_counter = pos; pos = align256(pos + 8);    // [0] calls so far (tensor-core path), [1] this call's t buffer
  w.counters = pos;  pos = align256(pos + (n / 32) * 4);
  w.y_acc = pos;     pos = align256(pos + (batch <= CQL_MAX_DECODE_BATCH ? (uint64_t)batch * n * 4 : 0));
  w.t_part = pos;    pos = align256(pos + upr * bp * rpad * 4);
  w.t_final = pos;   pos = align256(pos + 2 * bp * rpad * 4);   // two t buffers, alternating by call
  w.xs = pos;        pos = align256(pos + (d.salient_channels > 0 ? (uint64_t)batch * d.k_in * 2 : 0));
  w.prefill = pos;
  if (batch > CQL_MAX_DECODE_BATCH) pos = align256(pos + prefill_layout(d, batch).total);
  w.total = pos;
  return w;
}

}  // namespace cql

extern "C" {

const char* cql_status_string(cql_status s) {
  switch (s) {
    case CQL_OK: return "CQL_OK";
    case CQL_ERR_ARG: return "CQL_ERR_ARG: invalid argument";
    case CQL_ERR_ALIGN: return "CQL_ERR_ALIGN: pointer not aligned";
    case CQL_ERR_FORMAT: return "CQL_ERR_FORMAT: packed header does not match the descriptor";
    case CQL_ERR_SIZE: return "CQL_ERR_SIZE: buffer or workspace too small";
    case CQL_ERR_UNSUPPORTED: return "CQL_ERR_UNSUPPORTED: combination not implemented";
    case CQL_ERR_CUDA: return "CQL_ERR_CUDA: CUDA runtime error";
    case CQL_ERR_TIMEOUT: return "CQL_ERR_TIMEOUT: bounded device wait ran out";
    case CQL_ERR_RANGE: return "CQL_ERR_RANGE: an index outside its buffer (checked build)";
  }
  return "CQL_ERR_UNKNOWN";
}

int32_t cql_version(void) { return CQL_VERSION; }

cql_status cql_packed_layout(const cql_desc* desc, cql_layout* out) {
  if (out == nullptr) return CQL_ERR_ARG;
  const cql_status s = validate_desc(desc);
  if (s != CQL_OK) return s;
  compute_layout(*desc, out);
  return CQL_OK;
}

cql_status cql_pack_workspace_size(const cql_desc* desc, uint64_t* bytes) {
  if (bytes == nullptr) return CQL_ERR_ARG;
  const cql_status s = validate_desc(desc);
  if (s != CQL_OK) return s;
  *bytes = pack_workspace_layout(*desc).total;
  return CQL_OK;
}

cql_status pack_compressed_weight(const cql_desc* desc, const void* W, cql_dtype w_dt, const float* L,
                                  const float* R, const float* act_absmean, const float* fisher, void* packed, uint64_t packed_bytes, void* workspace,
                                  uint64_t ws_bytes, cql_stream_t stream) {
  cql_status s = validate_desc(desc);
  if (s != CQL_OK) return s;
  const cql_desc& d = *desc;
  if (W == nullptr || packed == nullptr || workspace == nullptr) return CQL_ERR_ARG;
  if (w_dt != CQL_DT_F32 && w_dt != CQL_DT_BF16) return CQL_ERR_ARG;
  if (d.rank > 0 && (L == nullptr || R == nullptr)) return CQL_ERR_ARG;
  if (!aligned(W, 16) || !aligned(packed, 256) || !aligned(workspace, 256)) return CQL_ERR_ALIGN;
  if (d.rank > 0 && (!aligned(L, 16) || !aligned(R, 16))) return CQL_ERR_ALIGN;
  if (d.salient_channels > 0 && act_absmean == nullptr) return CQL_ERR_ARG;
  if (d.salient_channels > 0 && !aligned(act_absmean, 4)) return CQL_ERR_ALIGN;
  if (fisher != nullptr && !aligned(fisher, 4)) return CQL_ERR_ALIGN;
  cql_layout lay;
  compute_layout(d, &lay);
  if (packed_bytes < lay.total_bytes) return CQL_ERR_SIZE;
  const PackWorkspace pw = pack_workspace_layout(d);
  if (ws_bytes < pw.total) return CQL_ERR_SIZE;

  PackParams p;
  memset(&p, 0, sizeof(p));
  p.d = d;
  p.rb = row_bytes_of(d);
  p.W = W;
  p.wdt = (int)w_dt;
  p.L = L;
  p.R = R;
  p.alpha = (double)d.clip_alpha;
  p.nnz_target = lay.nnz;
  uint8_t* base = static_cast<uint8_t*>(packed);
  p.packed = base;
  p.values = base + lay.off[CQL_PLANE_VALUES];
  p.meta = base + lay.off[CQL_PLANE_META];
  p.scales = base + lay.off[CQL_PLANE_SCALES];
  p.voff = base + lay.off[CQL_PLANE_VOFF];
  p.csr_rowptr = reinterpret_cast<int32_t*>(base + lay.off[CQL_PLANE_CSR_ROWPTR]);
  p.csr_col = reinterpret_cast<uint16_t*>(base + lay.off[CQL_PLANE_CSR_COL]);
  p.csr_val = reinterpret_cast<uint16_t*>(base + lay.off[CQL_PLANE_CSR_VAL]);
  p.r_values = base + lay.off[CQL_PLANE_R_VALUES];
  p.r_scales = base + lay.off[CQL_PLANE_R_SCALES];
  p.l_values = base + lay.off[CQL_PLANE_L_VALUES];
  p.l_scales = reinterpret_cast<uint16_t*>(base + lay.off[CQL_PLANE_L_SCALES]);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.err = reinterpret_cast<uint32_t*>(ws + pw.err);
  for (int i = 0; i < CQL_NPLANES; ++i) p.plane_len[i] = lay.len[i];
  p.out_bits = reinterpret_cast<uint32_t*>(ws + pw.out_bits);
  p.topk_state = reinterpret_cast<TopkState*>(ws + pw.state);
  p.topk_hist = reinterpret_cast<uint32_t*>(ws + pw.hist);
  p.topk_tiecnt = reinterpret_cast<uint32_t*>(ws + pw.tiecnt);
  p.topk_tieoff = reinterpret_cast<uint32_t*>(ws + pw.tieoff);
  p.row_counts = reinterpret_cast<uint32_t*>(ws + pw.row_counts);
  p.act_absmean = act_absmean;
  p.salient = reinterpret_cast<uint16_t*>(base + lay.off[CQL_PLANE_SALIENT]);
  p.w_scaled = reinterpret_cast<float*>(ws + pw.w_scaled);
  p.sal_partial = reinterpret_cast<double*>(ws + pw.sal_partial);
  p.sal = reinterpret_cast<double*>(ws + pw.sal);
  p.sal_flag = ws + pw.sal_flag;
  p.alpha_hist = reinterpret_cast<unsigned long long*>(ws + pw.alpha);
  p.alpha_dev = (d.clip_alpha == 0.0f && !codec_is_lut(d.codec)) ? reinterpret_cast<float*>(ws + pw.alpha + 1024 * 8)
                                                                : nullptr;
  p.fisher = codec_is_lut(d.codec) ? fisher : nullptr;
  if (d.outlier_frac <= 0.0f) p.csr_rowptr = nullptr;
  const HeaderBytes h = make_header(d, lay);
  const cudaError_t e = launch_pack(p, h, lay.total_bytes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CQL_OK : CQL_ERR_CUDA;
}

cql_status cql_workspace_size(const cql_desc* desc, int32_t batch, uint64_t* bytes) {
  if (bytes == nullptr) return CQL_ERR_ARG;
  const cql_status s = validate_desc(desc);
  if (s != CQL_OK) return s;
  if (batch < 1 || batch > 65536) return CQL_ERR_ARG;
  *bytes = forward_workspace_layout(*desc, batch).total;
  return CQL_OK;
}

cql_status cql_workspace_init(void* workspace, uint64_t ws_bytes, cql_stream_t stream) {
  if (workspace == nullptr) return CQL_ERR_ARG;
  if (!aligned(workspace, 256)) return CQL_ERR_ALIGN;
  const cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CQL_OK : CQL_ERR_CUDA;
}

cql_status compressed_linear_forward(const cql_desc* desc, const void* packed, const void* x, cql_dtype x_dt,
                                     void* y, cql_dtype y_dt, int32_t batch, void* workspace, uint64_t ws_bytes,
                                     cql_stream_t stream) {
  cql_status s = validate_desc(desc);
  if (s != CQL_OK) return s;
  const cql_desc& d = *desc;
  if (packed == nullptr || x == nullptr || y == nullptr || workspace == nullptr) return CQL_ERR_ARG;
  if (x_dt != CQL_DT_F16 && x_dt != CQL_DT_BF16) return CQL_ERR_ARG;
  if (y_dt != CQL_DT_F32 && y_dt != CQL_DT_F16 && y_dt != CQL_DT_BF16) return CQL_ERR_ARG;
  if (batch < 1 || batch > 65536) return CQL_ERR_ARG;
  if (!aligned(packed, 256) || !aligned(workspace, 256) || !aligned(x, 16) || !aligned(y, 16)) return CQL_ERR_ALIGN;
  const ForwardWorkspace fw = forward_workspace_layout(d, batch);
  if (ws_bytes < fw.total) return CQL_ERR_SIZE;
  if (batch > CQL_MAX_DECODE_BATCH && !prefill_supported(d, x_dt)) return CQL_ERR_UNSUPPORTED;

  cql_layout lay;
  compute_layout(d, &lay);
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams p = planes_of(d, packed, lay);
  p.x = x;
  p.xdt = (int)x_dt;
  p.y = y;
  p.ydt = (int)y_dt;
  p.batch = batch;
  p.flags = d.flags;
  p.n_rb = d.n_out / 32;
  p.upr = d.k_in / 128;
  p.n_units = (uint64_t)p.n_rb * p.upr;
  p.r_pad = (d.rank + 31) / 32 * 32;
  p.err = reinterpret_cast<uint32_t*>(ws + fw.err);
  p.t_counter = reinterpret_cast<uint32_t*>(ws + fw.t_counter);
  p.y_acc = reinterpret_cast<float*>(ws + fw.y_acc);
  p.counters = reinterpret_cast<uint32_t*>(ws + fw.counters);
  p.t_part = reinterpret_cast<float*>(ws + fw.t_part);
  p.t_final = reinterpret_cast<float*>(ws + fw.t_final);
  p.x_elems = (uint64_t)batch * d.k_in;
  p.y_elems = (uint64_t)batch * d.n_out;
  p.t_final_elems = (fw.xs - fw.t_final) / 4;
  p.t_part_elems = (fw.t_final - fw.t_part) / 4;
  if (d.salient_channels > 0) {
    // SLiM^O: every later step reads x' from the workspace
    const cudaError_t e0 = launch_salient_x(p, reinterpret_cast<const uint16_t*>(base + lay.off[CQL_PLANE_SALIENT]),
                                            ws + fw.xs, reinterpret_cast<cudaStream_t>(stream));
    if (e0 != cudaSuccess) return CQL_ERR_CUDA;
    p.x = ws + fw.xs;
  }
  const cudaError_t e = batch > CQL_MAX_DECODE_BATCH
                            ? launch_prefill(p, ws + fw.prefill, reinterpret_cast<cudaStream_t>(stream))
                            : launch_decode(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CQL_OK : CQL_ERR_CUDA;
}

cql_status cql_adapter_workspace_size(const cql_desc* desc, uint64_t* bytes) {
  if (bytes == nullptr) return CQL_ERR_ARG;
  const cql_status s = validate_desc(desc);
  if (s != CQL_OK) return s;
  if (desc->rank <= 0 || desc->rank > desc->n_out || desc->rank > desc->k_in) return CQL_ERR_ARG;
  *bytes = lora_workspace_layout(*desc).total;
  return CQL_OK;
}

cql_status cql_build_adapters(const cql_desc* desc, const void* W, cql_dtype w_dt, const void* packed,
                              const float* act_absmean, float* L, float* R, void* workspace, uint64_t ws_bytes,
                              cql_stream_t stream) {
  uint64_t need = 0;
  const cql_status s = cql_adapter_workspace_size(desc, &need);
  if (s != CQL_OK) return s;
  if (W == nullptr || packed == nullptr || L == nullptr || R == nullptr || workspace == nullptr) return CQL_ERR_ARG;
  if (w_dt != CQL_DT_F32 && w_dt != CQL_DT_BF16) return CQL_ERR_ARG;
  if (!aligned(W, 16) || !aligned(packed, 256) || !aligned(workspace, 256) || !aligned(L, 4) || !aligned(R, 4) ||
      (act_absmean != nullptr && !aligned(act_absmean, 4)))
    return CQL_ERR_ALIGN;
  if (ws_bytes < need) return CQL_ERR_SIZE;
  cql_layout lay;
  compute_layout(*desc, &lay);
  const DecodeParams p = planes_of(*desc, packed, lay);
  const uint16_t* sal = desc->salient_channels > 0
                            ? reinterpret_cast<const uint16_t*>(static_cast<const uint8_t*>(packed) +
                                                                lay.off[CQL_PLANE_SALIENT])
                            : nullptr;
  const cudaError_t e = launch_build_adapters(p, W, (int)w_dt, act_absmean, sal, static_cast<uint8_t*>(workspace),
                                              L, R, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CQL_OK : CQL_ERR_CUDA;
}

cql_status cql_read_header(const void* packed_host, uint64_t bytes, cql_desc* desc_out, cql_layout* layout_out) {
  if (packed_host == nullptr || desc_out == nullptr) return CQL_ERR_ARG;
  if (bytes < CQL_HEADER_BYTES) return CQL_ERR_SIZE;
  const uint8_t* b = static_cast<const uint8_t*>(packed_host);
  uint32_t ver = 0;
  memcpy(&ver, b + 4, 4);
  if (memcmp(b, "CQL1", 4) != 0 || ver != CQL_VERSION) return CQL_ERR_FORMAT;
  cql_desc d;
  memcpy(&d, b + 8, sizeof(cql_desc));
  if (validate_desc(&d) != CQL_OK) return CQL_ERR_FORMAT;
  cql_layout stored, expect;
  memcpy(&stored.total_bytes, b + 72, 8);
  memcpy(&stored.nnz, b + 80, 8);
  memcpy(stored.off, b + 88, 8 * CQL_NPLANES);
  memcpy(stored.len, b + 88 + 8 * CQL_NPLANES, 8 * CQL_NPLANES);
  compute_layout(d, &expect);
  if (stored.total_bytes != expect.total_bytes || stored.nnz != expect.nnz ||
      memcmp(stored.off, expect.off, sizeof(expect.off)) != 0 || memcmp(stored.len, expect.len, sizeof(expect.len)) != 0)
    return CQL_ERR_FORMAT;
  if (bytes < stored.total_bytes) return CQL_ERR_SIZE;
  *desc_out = d;
  if (layout_out != nullptr) *layout_out = stored;
  return CQL_OK;
}

cql_status cql_plane_checksums(const void* packed_host, uint64_t bytes, uint32_t out[CQL_NPLANES]) {
  if (out == nullptr) return CQL_ERR_ARG;
  cql_desc d;
  cql_layout lay;
  const cql_status s = cql_read_header(packed_host, bytes, &d, &lay);
  if (s != CQL_OK) return s;
  // CRC-32, reflected, polynomial 0xEDB88320, initial and final xor ~0
  uint32_t table[256];
  for (uint32_t i = 0; i < 256; ++i) {
    uint32_t c = i;
    for (int k = 0; k < 8; ++k) c = (c & 1u) ? 0xEDB88320u ^ (c >> 1) : c >> 1;
    table[i] = c;
  }
  const uint8_t* b = static_cast<const uint8_t*>(packed_host);
  for (int i = 0; i < CQL_NPLANES; ++i) {
    uint32_t c = 0xFFFFFFFFu;
    for (uint64_t j = 0; j < lay.len[i]; ++j) c = table[(c ^ b[lay.off[i] + j]) & 0xFFu] ^ (c >> 8);
    out[i] = lay.len[i] ? ~c : 0u;
  }
  return CQL_OK;
}

cql_status cql_get_device_status(void* workspace, cql_stream_t stream, cql_status* out) {
  if (out == nullptr) return CQL_ERR_ARG;
  if (workspace == nullptr) {
    // the fixed scratch of the no-workspace entry point on the current device
    workspace = noalloc_scratch_current_device();
    if (workspace == nullptr) {                     // no such call has run here
      *out = CQL_OK;
      return CQL_OK;
    }
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t w[2] = {0, 0};
  if (cudaMemcpyAsync(w, workspace, sizeof(w), cudaMemcpyDeviceToHost, st) != cudaSuccess) return CQL_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return CQL_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(w), st) != cudaSuccess) return CQL_ERR_CUDA;
  *out = (cql_status)w[0];
  return CQL_OK;
}

}  // extern "C"
