/*
 * cql.h -- C ABI of libcql, the B200 (sm_100a) compressed linear layer.
 *
 * The layer computes, for activations x [B][K] and outputs y [B][N],
 *
 *     y = deq(Q (.) M) x  +  S_csr x  +  deq(L_q) (deq(R_q) x)
 *
 * where Q holds low-bit codes of W (symmetric clipped int4/int3 with one fp16
 * scale per 128 columns, as in SLiM-Quant; or a 3/4-bit per-row non-uniform
 * table, as in SqueezeLLM), M is a 2:4 or unstructured-50% sparsity mask,
 * S_csr an optional fp16 CSR matrix of outliers (SqueezeLLM's dense-and-sparse
 * split), and L_q, R_q rank-r adapters quantised AbsMax int4 in groups of 128
 * (SLiM's "Low-rank adapter quantization").
 *
 * Output-error variant (SLiM^O; SLiM rebuttal, "Output Error Minimization in
 * SLiM-Quant"): a layer packed with desc.salient_channels = m > 0 stores the
 * compression of W' = W diag(sigma), where sigma_c = 2^salient_log2 on the m
 * input channels of highest saliency and 1 elsewhere, and computes the
 * formula above on x' = x diag(1/sigma): the forward divides those m
 * activation channels by the factor before anything else reads x.
 *
 * Sources: "SLiM: One-shot Quantization and Sparsity with Low-rank
 * Approximation for LLM Weight Compression" (review summary: SLIM-Quant,
 * Low-rank adapter quantization; rebuttal: Unstructured vs. 2:4 Sparsity,
 * Speedup Comparison without LoRA, Output Error Minimization in SLiM-Quant) and "SqueezeLLM: Dense-and-Sparse
 * Quantization" (Approach; Key results).  The pages fix no API, byte layout,
 * scale dtype, rounding or tie rule; those are defined here.
 *
 * Conventions for every entry point
 *   - All data pointers are DEVICE pointers owned by the caller, except the
 *     descriptor/layout/output-scalar pointers, which are host pointers.
 *   - The library allocates no memory.  Scratch memory comes from the
 *     caller's workspace (the one exception, compressed_linear_forward_noalloc,
 *     uses a fixed scratch array inside the library instead).
 *   - Calls are stream-ordered and asynchronous.  Argument and format errors
 *     are returned synchronously before anything is launched.  Errors found
 *     on the device (a bad header, a bounded wait that ran out) are written to
 *     the error word at the start of the workspace; read it with
 *     cql_get_device_status.
 *   - Nothing crosses the ABI as an exception; the library never exits,
 *     aborts or traps.
 *
 * ------------------------------------------------------------------------
 * PACKED FORMAT (version 2)
 * ------------------------------------------------------------------------
 * A packed weight is one contiguous device buffer: a 512-byte header (plane
 * 0) followed by up to 12 planes (CQL_PLANE_* indices 1-12, in that order).
 * Every plane starts on a 256-byte boundary; an absent plane has length 0
 * and the offset where it would start.  All multi-byte fields are
 * little-endian.
 *
 * Header: "CQL1", uint32 version = 2, cql_desc (64 bytes), then the
 * cql_layout (uint64 total_bytes, uint64 nnz, uint64 off[13], uint64 len[13]);
 * the rest of the 512 bytes is zero.
 *
 * Row-interleaved planes (VALUES, META, SCALES, VOFF, R_VALUES, R_SCALES,
 * L_VALUES).  Each row contributes row_bytes bytes (a multiple of 16, zero
 * padded).  Rows are grouped in blocks of 32; a block is stored as a run of
 * 512-byte slabs, slab s holding bytes [16s, 16s+16) of each of its 32 rows in
 * row order.  Byte j of row i is at
 *     ((i / 32) * (row_bytes / 16) + j / 16) * 512 + (i % 32) * 16 + (j % 16).
 * (32 consecutive lanes reading 16 bytes each read one slab: one coalesced
 * 512-byte access per warp.)
 *
 * Bit streams.  Code c of a row occupies stream bits [b*c, b*c + b) for b-bit
 * codes; stream bit t is bit (t % 8) of row byte t / 8.
 *
 * VALUES  b-bit codes of the kept entries of each row, in column order.
 *         int4/int3: u = q + 2^(b-1), q in [-(2^(b-1)-1), 2^(b-1)-1].
 *         lut3/lut4: index of the row's centroid.
 *         kept per row = K/2 under 2:4 and bitmap50, K without a mask.
 *         row_bytes = pad16(ceil(kept * b / 8)).
 * META    2:4: 4-bit code of column group g (columns 4g..4g+3) at stream
 *         bits [4g, 4g+4): the kept positions themselves, i0 | (i1 << 2),
 *         i0 < i1 (the 2-bit-index form sparse tensor cores read; valid codes
 *         0x4 0x8 0xC 0x9 0xD 0xE).  The kept codes of the group are, in
 *         VALUES, those of columns 4g+i0 then 4g+i1.
 *         bitmap50: bit k of the row stream is 1 when column k is kept.
 *         row_bytes = K/8.  Absent without a mask.
 * SCALES  int4/int3: fp16 scale of columns [128g, 128g+128) at row bytes
 *         [2g, 2g+2); row_bytes = pad16(K/64).
 *         lut3/lut4: the row's 2^b fp16 centroids; row_bytes = 2^(b+1).
 * VOFF    bitmap50 only: uint16 index, in the row's VALUES stream, of the
 *         first kept code of columns [128g, ...) at row bytes [2g, 2g+2);
 *         row_bytes = pad16(K/64).  (Lets a reader start mid-row.)
 * CSR_ROWPTR  int32 [N+1]      present when outlier_frac > 0
 * CSR_COL     uint16 [nnz]     columns ascending within a row
 * CSR_VAL     fp16 [nnz]       value = fp16(w - dense part at that entry)
 * R_VALUES  int4 codes u = q + 8 of R [r][K]; rows padded to a multiple of 32
 *           (padding rows all zero bytes, zero scales); row_bytes = K/2.
 * R_SCALES  fp16 scale of R row j, columns [128g, 128g+128); row_bytes =
 *           pad16(K/64).
 * L_VALUES  int4 codes u = q + 8 of L [N][r]; row_bytes = pad16(r/2).
 * L_SCALES  fp16 [N/128][r], plain row-major: scale of column j over rows
 *           [128g, 128g+128) at index g*r + j.
 * SALIENT   uint16 [m], m = salient_channels: the scaled input channels,
 *           ascending.  Absent when m = 0.
 *
 * Encoding rules (shared by pack_compressed_weight and the CPU oracle; every
 * real-valued step is evaluated in fp64 from exact widenings, then rounded to
 * fp16 round-to-nearest-even, ties in selections go to the lower index):
 *   0. SLiM^O (m > 0 only): saliency of channel c = a_c * sum_n |w[n][c]|,
 *      a_c the caller's float32 mean |x_c| over calibration tokens and the
 *      sum taken in fp64 over consecutive blocks of 64 rows (each block from
 *      its first row on, then the block sums from the first block on); the
 *      m channels of largest saliency have their column multiplied by
 *      2^salient_log2 (exact), and every rule below applies to that W';
 *   1. outliers: the floor(f*N*K) entries of largest |w| over the whole matrix;
 *   2. mask on |w|: 2:4 keeps the two largest of every 4 columns; bitmap50
 *      keeps the K/2 largest of every row;
 *   3. int codecs: s = fp16((alpha * amax) / qmax) with amax over the group's
 *      non-outlier entries, q = clamp(rint(w / s), -qmax, qmax), q = 0 when
 *      s = 0; qmax = 7 (int4) or 3 (int3);
 *      clip_alpha = 0 (SLiM-Quant search): counts h_b, b < 1024, of
 *      b = min(floor((|w| / amax) * 1024), 1023) over the kept non-outlier
 *      entries of groups with amax > 0; for alpha_i = fp32(i / 100),
 *      i = 30..100, E_i = sum_b h_b d_b^2 (b ascending, fp64, no fused
 *      operations) with c = (b + 1/2) / 1024, q = min(rint((c qmax) /
 *      alpha_i), qmax), d = c - (q alpha_i) / qmax; alpha = the alpha_i of
 *      least E_i (ties to the smaller), written into the header's descriptor;
 *      lut codecs: centroid j = linear-interpolated quantile of the row's
 *      sorted non-outlier values at p = (j + 1/2)/2^b, rounded to fp16; with
 *      a Fisher diagonal f (SqueezeLLM sensitivity-weighted k-means) these
 *      start Lloyd iterations instead: each non-outlier value goes to the
 *      nearest centroid (fp64, ties to the lower), an assignment equal to
 *      the previous one stops, else centroid j = (sum f v) / (sum f) over
 *      its members in column order (a centroid without weight stays), at
 *      most 32 updates, then rounded to fp16; every entry takes the nearest
 *      centroid;
 *   4. CSR values as above;
 *   5. adapters: s = fp16(amax / 7), q = clamp(rint(v / s), -7, 7), groups of
 *      128 along K for R and along N for L.
 */
#ifndef CQL_H
#define CQL_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CQL_VERSION 2
#define CQL_HEADER_BYTES 512
#define CQL_NPLANES 13
#define CQL_GROUP 128
#define CQL_MAX_DECODE_BATCH 16

typedef enum {
  CQL_OK = 0,
  CQL_ERR_ARG = 1,          /* null pointer, bad enum, bad size relation    */
  CQL_ERR_ALIGN = 2,        /* pointer not aligned as documented            */
  CQL_ERR_FORMAT = 3,       /* header magic/version/descriptor mismatch     */
  CQL_ERR_SIZE = 4,         /* buffer or workspace too small                */
  CQL_ERR_UNSUPPORTED = 5,  /* valid but not implemented combination        */
  CQL_ERR_CUDA = 6,         /* a CUDA runtime call failed                   */
  CQL_ERR_TIMEOUT = 7,      /* a bounded device wait ran out                */
  CQL_ERR_RANGE = 8         /* checked build only: an index fell outside its
                               buffer; the access was skipped (detail = site) */
} cql_status;

typedef enum { CQL_MASK_NONE = 0, CQL_MASK_2_4 = 1, CQL_MASK_BITMAP50 = 2 } cql_mask;
typedef enum {
  CQL_CODEC_INT4_SYM = 0, CQL_CODEC_INT3_SYM = 1, CQL_CODEC_LUT3_ROW = 2, CQL_CODEC_LUT4_ROW = 3
} cql_codec;
typedef enum { CQL_DT_F32 = 0, CQL_DT_F16 = 1, CQL_DT_BF16 = 2 } cql_dtype;

enum {
  CQL_PLANE_HEADER = 0, CQL_PLANE_VALUES = 1, CQL_PLANE_META = 2, CQL_PLANE_SCALES = 3,
  CQL_PLANE_VOFF = 4, CQL_PLANE_CSR_ROWPTR = 5, CQL_PLANE_CSR_COL = 6, CQL_PLANE_CSR_VAL = 7,
  CQL_PLANE_R_VALUES = 8, CQL_PLANE_R_SCALES = 9, CQL_PLANE_L_VALUES = 10, CQL_PLANE_L_SCALES = 11,
  CQL_PLANE_SALIENT = 12
};

/* Term toggles (cql_desc.flags, read by compressed_linear_forward only; used
 * by the per-term parity tests). */
#define CQL_FLAG_NO_MAIN 0x1u
#define CQL_FLAG_NO_CSR 0x2u
#define CQL_FLAG_NO_LOWRANK 0x4u
/* Test only: the tensor-core decode skips loading x, so that its bounded
 * waits on x run out (after ~10 ms instead of seconds); the call then
 * completes with CQL_ERR_TIMEOUT in the device error word and y undefined.
 * No copy or MMA is left in flight: nothing that waits on x has started any.
 * As after any device error, the workspace must be initialised again
 * (cql_workspace_init) before its next use. */
#define CQL_FLAG_DEBUG_SKIP_X 0x100u
/* Decode on the CUDA cores even where the tensor-core decode applies (2:4
 * int4 and int3 layers); for comparing the two designs on the same layer. */
#define CQL_FLAG_CUDA_CORE 0x200u

/* Layer descriptor, 64 bytes, stored verbatim in the packed header. */
typedef struct cql_desc {
  int32_t n_out;          /* N, rows of W; multiple of 128, <= 2^20          */
  int32_t k_in;           /* K, columns of W; multiple of 128, <= 65536      */
  int32_t mask;           /* cql_mask                                        */
  int32_t codec;          /* cql_codec; lut codecs need CQL_MASK_NONE        */
  int32_t group;          /* weight scale group; must be 128                 */
  float clip_alpha;       /* SLiM-Quant clip alpha in (0, 1]; 0 = search it  */
  float outlier_frac;     /* CSR fraction f in [0, 1/16]; 0 = no CSR         */
  int32_t rank;           /* adapter rank r, multiple of 16, <= 256; 0 = none */
  int32_t adapter_bits;   /* must be 4                                       */
  int32_t adapter_group;  /* must be 128                                     */
  uint32_t flags;         /* CQL_FLAG_* term toggles                         */
  int32_t salient_channels; /* SLiM^O scaled channels m, 0 <= m <= K/8; 0 = off */
  int32_t salient_log2;   /* SLiM^O factor 2^e, e in [1, 8] when m > 0, else 0 */
  int32_t reserved[3];    /* zero                                            */
} cql_desc;

typedef struct cql_layout {
  uint64_t total_bytes;   /* size of the packed buffer                       */
  uint64_t nnz;           /* CSR entries, floor(f * N * K)                   */
  uint64_t off[CQL_NPLANES];
  uint64_t len[CQL_NPLANES];
} cql_layout;

typedef struct CUstream_st* cql_stream_t;   /* == cudaStream_t */

/* Human-readable name of a status code.  Never returns NULL. */
const char* cql_status_string(cql_status s);

/* Library version (CQL_VERSION) and the packed-format version it writes. */
int32_t cql_version(void);

/* Validate a descriptor and compute the packed layout.  Host only: touches no
 * GPU.  Returns CQL_ERR_ARG / CQL_ERR_UNSUPPORTED for descriptors the library
 * cannot pack. */
cql_status cql_packed_layout(const cql_desc* desc, cql_layout* out);

/* Scratch bytes pack_compressed_weight needs.  Host only. */
cql_status cql_pack_workspace_size(const cql_desc* desc, uint64_t* bytes);

/* Encode W (and the adapters) into the packed format (rules above).
 *   W         device, [N][K] row-major, w_dt = CQL_DT_F32 or CQL_DT_BF16,
 *             16-byte aligned.
 *   L         device fp32 [N][r] row-major, or NULL when rank == 0.
 *   R         device fp32 [r][K] row-major, or NULL when rank == 0.  (With
 *             SLiM^O the adapters act on x', the scaled activations.)
 *   act_absmean  device fp32 [K], the mean |x_c| of each input channel over
 *             calibration tokens (finite, >= 0); required when
 *             salient_channels > 0, ignored (may be NULL) otherwise.
 *   fisher    device fp32 [N][K] diagonal Fisher information (finite, >= 0)
 *             for the LUT codecs' weighted k-means, or NULL (quantile
 *             table); ignored by the int codecs.
 *   packed    device, >= cql_layout.total_bytes, 256-byte aligned; every byte
 *             of it is written.
 *   workspace device scratch of >= cql_pack_workspace_size bytes, 256-byte
 *             aligned; its contents on entry do not matter.  Its first 8
 *             bytes are an error word that the pack clears first and that
 *             only the range-checked library (libcql_checked) ever sets:
 *             CQL_ERR_RANGE when a pack kernel's index fell outside its
 *             plane.  Read it with cql_get_device_status(workspace, ...)
 *             before reusing the workspace.
 * The result is bit-exact with the CPU oracle on every byte.  Inputs must be
 * finite. */
cql_status pack_compressed_weight(const cql_desc* desc, const void* W, cql_dtype w_dt,
                                  const float* L, const float* R, const float* act_absmean,
                                  const float* fisher, void* packed,
                                  uint64_t packed_bytes, void* workspace, uint64_t ws_bytes,
                                  cql_stream_t stream);

/* Scratch bytes cql_build_adapters needs (about 4 N K bytes plus
 * O((N + K) r) for the subspace).  Host only.  CQL_ERR_ARG unless
 * 0 < rank <= min(N, K). */
cql_status cql_adapter_workspace_size(const cql_desc* desc, uint64_t* bytes);

/* SLiM-LoRA adapters of a packed layer (SLiM review summary, "SLIM-LoRA";
 * rebuttal, "Assumptions in Theoretical Derivations"): L [N][r] and R [r][K]
 * minimising ||(E - L R) diag(xbar)||_F, E = W' - W_C the compression error
 * (W' the matrix the codec encoded, W_C what the codes and the CSR outliers
 * represent), xbar the input the adapters see: act_absmean, divided by the
 * SLiM^O factor on the salient channels.  act_absmean NULL: Naive-LoRA
 * (xbar = 1, the plain truncated SVD of E).
 *   desc      the layer's descriptor; rank r with 0 < r <= min(N, K).
 *   W         device [N][K], w_dt CQL_DT_F32 or CQL_DT_BF16, 16-byte aligned:
 *             the matrix packed into 'packed'.
 *   packed    device, 256-byte aligned, a buffer pack_compressed_weight
 *             wrote for W under desc (its adapter planes are not read: pack
 *             with zero adapters, build, then pack again with L and R).
 *   act_absmean  device fp32 [K], every entry > 0, or NULL.
 *   L, R      device fp32 outputs, row-major [N][r] and [r][K].
 *   workspace device, >= cql_adapter_workspace_size bytes, 256-byte aligned.
 * Method: randomized subspace iteration on E diag(xbar) (p = r + 32 rounded
 * up to 32 columns, 6 iterations, CholeskyQR2), then a Jacobi
 * eigen-decomposition of the p x p Gram matrix.  The result approaches the
 * exact truncated SVD as the singular-value gap at r grows; the split of
 * the singular values is L = U Sigma^(1/2), R = Sigma^(1/2) V^T diag(xbar)^-1. */
cql_status cql_build_adapters(const cql_desc* desc, const void* W, cql_dtype w_dt, const void* packed,
                              const float* act_absmean, float* L, float* R, void* workspace, uint64_t ws_bytes,
                              cql_stream_t stream);

/* Saving and loading packed layers.  A packed buffer is self-describing:
 * copied to the host (or to a file) and back, it needs no other state.
 *
 * cql_read_header: the descriptor and layout stored in the header of a HOST
 * copy of a packed buffer (at least 512 bytes readable at 'packed_host').
 * Returns CQL_ERR_FORMAT when the magic, the version, the descriptor's
 * validity or the stored layout (recomputed from the descriptor) does not
 * match, CQL_ERR_SIZE when 'bytes' is smaller than the stored total.
 *
 * cql_plane_checksums: CRC-32 (IEEE 802.3 polynomial, the zlib/PNG
 * checksum) of every plane of a HOST copy, out[i] for plane i (0 for an
 * empty plane), after the same checks as cql_read_header; for verifying a
 * layer after saving, copying or loading it.  Host only, both. */
cql_status cql_read_header(const void* packed_host, uint64_t bytes, cql_desc* desc_out, cql_layout* layout_out);
cql_status cql_plane_checksums(const void* packed_host, uint64_t bytes, uint32_t out[CQL_NPLANES]);

/* Workspace bytes compressed_linear_forward needs for this layer and batch.
 * Host only. */
cql_status cql_workspace_size(const cql_desc* desc, int32_t batch, uint64_t* bytes);

/* Reads before the previous kernel completes.  The forward's first kernel is
 * launched programmatically dependent on the kernel that precedes it on the
 * stream and reads the packed weights (never x, y or the workspace) before
 * waiting for that kernel to complete.  So the kernel immediately before a
 * forward must not write the packed buffer; pack_compressed_weight ends with
 * an operation that makes a forward launched right after it safe. */

/* Zero a forward workspace (required once before its first use; the forward
 * leaves the parts it reuses zeroed again when it completes). */
cql_status cql_workspace_init(void* workspace, uint64_t ws_bytes, cql_stream_t stream);

/* y = deq(Q (.) M) x + S_csr x + deq(L_q)(deq(R_q) x)  for a packed layer.
 *   desc      host copy of the descriptor the layer was packed with (its
 *             flags select the terms computed).
 *   packed    device, the packed buffer, 256-byte aligned.
 *   x         device [batch][K], x_dt = CQL_DT_F16 or CQL_DT_BF16, 16-byte
 *             aligned.
 *   y         device [batch][N], y_dt = CQL_DT_F32, F16 or BF16, 16-byte
 *             aligned; fp32 accumulation, one final round to y_dt.
 *   A SLiM^O layer (salient_channels > 0) first runs a small kernel that
 *   writes x' (x with the salient channels divided by 2^salient_log2,
 *   rounded to x_dt, exact unless a value falls into x_dt's subnormal range)
 *   into the workspace; every later step reads x'.
 *   batch     1..16 runs the decode path: sparse tcgen05 MMAs for 2:4 int4
 *             and int3 layers with fp16/bf16 x, a CUDA-core GEMV for the
 *             other codecs and masks; larger batches run the tcgen05
 *             prefill GEMM: on the sparse tensor cores for 2:4 int4 and
 *             int3 layers, dense for int4 / int3 layers without a mask;
 *             LUT codecs, the bitmap mask and CSR outliers give
 *             CQL_ERR_UNSUPPORTED there.
 *   workspace device, >= cql_workspace_size bytes, 256-byte aligned, zeroed
 *             by cql_workspace_init before its first use with a given layer
 *             and batch (the forward leaves it ready for the next call with
 *             the same layer and batch).  Calls sharing one workspace must be
 *             ordered on one stream.
 */
cql_status compressed_linear_forward(const cql_desc* desc, const void* packed, const void* x,
                                     cql_dtype x_dt, void* y, cql_dtype y_dt, int32_t batch,
                                     void* workspace, uint64_t ws_bytes, cql_stream_t stream);

/* Forward pass without a workspace argument, for callers that cannot allocate
 * device memory themselves: e.g. an inference-server plugin whose enqueue path
 * may not allocate, a runtime that budgets every device byte ahead of time, or
 * a binding that can only pass raw input and output pointers.  (This entry
 * point is an addition of this library; the paper has no counterpart.)
 *   Arguments as compressed_linear_forward, minus the workspace.  The scratch
 *   memory is one fixed 4 MiB device array inside the library, held by every
 *   GPU that loads it until the process exits; a call whose workspace
 *   (cql_workspace_size) would exceed 4 MiB returns CQL_ERR_SIZE without
 *   launching anything.  The library never calls cudaMalloc or cudaFree here.
 *   The first call on a device finds the array's address and clears it (with
 *   that device current).
 *   All calls share the array, and each call first clears (memset on its
 *   stream) the part of it that it uses: calls that overlap on the GPU race,
 *   so order them on one stream.  Device errors are recorded in the array's
 *   error word; read them with cql_get_device_status(NULL, stream, &st). */
cql_status compressed_linear_forward_noalloc(const cql_desc* desc, const void* packed, const void* x,
                                             cql_dtype x_dt, void* y, cql_dtype y_dt, int32_t batch,
                                             cql_stream_t stream);

/* Wait for the stream, then read and clear the device error word of a
 * workspace: *out = CQL_OK or the cql_status a kernel recorded.  After an
 * error the rest of the workspace is in an undefined state: initialise it
 * again with cql_workspace_init before the next forward that uses it.
 *   workspace  a forward workspace, a pack workspace (after
 *              pack_compressed_weight: CQL_OK, or CQL_ERR_RANGE from the
 *              range-checked library), or NULL for the fixed scratch array of
 *              compressed_linear_forward_noalloc on the current device (each
 *              no-workspace call clears that word when it starts, so this
 *              reports the most recent such call; CQL_OK if none ran). */
cql_status cql_get_device_status(void* workspace, cql_stream_t stream, cql_status* out);

#ifdef __cplusplus
}
#endif
#endif /* CQL_H */
