/* A plain C99 user of the library's C ABI (no C++, no CUDA headers, no
 * Python): checks that include/cql.h compiles as C and that the host-only
 * entry points behave as the header states when called from C.
 *
 * Usage: abi_consumer <packed file>...
 * For each file (a host copy of a packed layer) it prints one line
 *   file n_out k_in mask codec rank clip_alpha salient_channels salient_log2
 *        total_bytes nnz off[0..12] len[0..12] crc[0..12] pack_ws
 * and exits 0; any call that returns other than documented prints the
 * reason and exits 1.  Argument checks (null pointers, bad descriptors, a
 * truncated copy) are exercised on the first file.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "cql.h"

static int fail(const char* what, cql_status s) {
  fprintf(stderr, "abi_consumer: %s: %s\n", what, cql_status_string(s));
  return 1;
}

static unsigned char* read_file(const char* path, uint64_t* bytes) {
  FILE* f = fopen(path, "rb");
  long n;
  unsigned char* buf;
  if (f == NULL) return NULL;
  if (fseek(f, 0, SEEK_END) != 0 || (n = ftell(f)) < 0 || fseek(f, 0, SEEK_SET) != 0) {
    fclose(f);
    return NULL;
  }
  buf = (unsigned char*)malloc((size_t)n + 1);
  if (buf != NULL && fread(buf, 1, (size_t)n, f) != (size_t)n) {
    free(buf);
    buf = NULL;
  }
  fclose(f);
  *bytes = (uint64_t)n;
  return buf;
}

/* The documented argument errors, all returned before any work. */
static int check_argument_errors(const unsigned char* buf, uint64_t bytes) {
  cql_desc d;
  cql_layout lay;
  uint32_t crc[CQL_NPLANES];
  uint64_t v;
  cql_status s;
  if ((s = cql_read_header(NULL, bytes, &d, &lay)) != CQL_ERR_ARG) return fail("read_header(NULL)", s);
  if ((s = cql_read_header(buf, bytes, NULL, NULL)) != CQL_ERR_ARG) return fail("read_header(no outputs)", s);
  if ((s = cql_read_header(buf, 100, &d, &lay)) != CQL_ERR_SIZE) return fail("read_header(short)", s);
  if ((s = cql_read_header(buf, bytes - 256, &d, &lay)) != CQL_ERR_SIZE) return fail("read_header(truncated)", s);
  if ((s = cql_plane_checksums(NULL, bytes, crc)) != CQL_ERR_ARG) return fail("plane_checksums(NULL)", s);
  if ((s = cql_packed_layout(NULL, &lay)) != CQL_ERR_ARG) return fail("packed_layout(NULL)", s);
  if ((s = cql_read_header(buf, bytes, &d, &lay)) != CQL_OK) return fail("read_header", s);
  d.n_out += 64;                                     /* no longer a multiple of 128 */
  if ((s = cql_packed_layout(&d, &lay)) != CQL_ERR_ARG) return fail("packed_layout(n_out)", s);
  if ((s = cql_pack_workspace_size(&d, &v)) != CQL_ERR_ARG) return fail("pack_workspace_size(n_out)", s);
  d.n_out -= 64;
  d.group = 64;                                      /* valid shape, unsupported group */
  if ((s = cql_packed_layout(&d, &lay)) != CQL_ERR_UNSUPPORTED) return fail("packed_layout(group)", s);
  d.group = 128;
  if ((s = cql_workspace_size(&d, 0, &v)) != CQL_ERR_ARG) return fail("workspace_size(batch 0)", s);
  if ((s = cql_get_device_status(NULL, NULL, NULL)) != CQL_ERR_ARG) return fail("get_device_status(NULL)", s);
  if (cql_status_string((cql_status)12345) == NULL) return fail("status_string(unknown)", CQL_OK);
  return 0;
}

int main(int argc, char** argv) {
  int i, p;
  if (argc < 2) {
    fprintf(stderr, "usage: abi_consumer <packed file>...\n");
    return 2;
  }
  if (cql_version() != 2) return fail("cql_version", CQL_OK);
  for (i = 1; i < argc; ++i) {
    uint64_t bytes = 0, pack_ws = 0;
    unsigned char* buf = read_file(argv[i], &bytes);
    cql_desc d;
    cql_layout lay, lay2;
    uint32_t crc[CQL_NPLANES];
    cql_status s;
    if (buf == NULL) {
      fprintf(stderr, "abi_consumer: cannot read %s\n", argv[i]);
      return 1;
    }
    if (i == 1 && check_argument_errors(buf, bytes) != 0) return 1;
    if ((s = cql_read_header(buf, bytes, &d, &lay)) != CQL_OK) return fail("read_header", s);
    /* the layout the header stores is the one the descriptor gives */
    if ((s = cql_packed_layout(&d, &lay2)) != CQL_OK) return fail("packed_layout", s);
    if (memcmp(&lay, &lay2, sizeof(lay)) != 0) return fail("stored layout differs from computed", CQL_OK);
    if ((s = cql_plane_checksums(buf, bytes, crc)) != CQL_OK) return fail("plane_checksums", s);
    if ((s = cql_pack_workspace_size(&d, &pack_ws)) != CQL_OK) return fail("pack_workspace_size", s);
    printf("%s %d %d %d %d %d %.9g %d %d %llu %llu", argv[i], (int)d.n_out, (int)d.k_in, (int)d.mask,
           (int)d.codec, (int)d.rank, (double)d.clip_alpha, (int)d.salient_channels, (int)d.salient_log2,
           (unsigned long long)lay.total_bytes, (unsigned long long)lay.nnz);
    for (p = 0; p < CQL_NPLANES; ++p) printf(" %llu", (unsigned long long)lay.off[p]);
    for (p = 0; p < CQL_NPLANES; ++p) printf(" %llu", (unsigned long long)lay.len[p]);
    for (p = 0; p < CQL_NPLANES; ++p) printf(" %lu", (unsigned long)crc[p]);
    printf(" %llu\n", (unsigned long long)pack_ws);
    free(buf);
  }
  return 0;
}
