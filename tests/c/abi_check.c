/*
 * The C boundary seen from plain C99: include/sfp8.h compiles as C, every
 * declared entry point links against libsfp8.so, and the entry points that
 * touch no device answer on a machine without one.  Prints "abi ok" and
 * exits 0 when every check holds.
 */
#include <stdio.h>
#include <string.h>

#include "sfp8.h"

typedef void (*any_fn)(void);

int main(void) {
  /* every declaration resolves to a symbol of the library */
  const any_fn fns[] = {
      (any_fn)sfp8_quantize_rowwise, (any_fn)sfp8_quantize_tensorwise_workspace_bytes,
      (any_fn)sfp8_quantize_tensorwise, (any_fn)sfp8_prune_24, (any_fn)sfp8_padded_rows,
      (any_fn)sfp8_compressed_bytes, (any_fn)sfp8_compress_24, (any_fn)sfp8_prepare_weight_24,
      (any_fn)sfp8_decompress_24, (any_fn)sfp8_sparse_linear_workspace_bytes,
      (any_fn)sfp8_workspace_clear, (any_fn)sfp8_sparse_linear,
      (any_fn)sfp8_sparse_linear_algo_count, (any_fn)sfp8_sparse_linear_algo_info,
      (any_fn)sfp8_sparse_linear_plan_count, (any_fn)sfp8_sparse_linear_plan_info,
      (any_fn)sfp8_sparse_linear_algo_workspace_bytes,
      (any_fn)sfp8_sparse_linear_search_workspace_bytes, (any_fn)sfp8_sparse_linear_algo,
      (any_fn)sfp8_sparse_linear_search, (any_fn)sfp8_sparse_linear_set_algo,
      (any_fn)sfp8_sparse_linear_get_algo, (any_fn)sfp8_sparse_linear_quant_workspace_bytes,
      (any_fn)sfp8_sparse_linear_quant, (any_fn)sfp8_sparse_linear_quant_host,
      (any_fn)sfp8_sparse_linear_quant_fused, (any_fn)sfp8_sparse_linear_quant_chained,
      (any_fn)sfp8_sparse_linear_quant_fusable,
      (any_fn)sfp8_sparse_linear_noalloc, (any_fn)sfp8_selftest_timeout,
      (any_fn)sfp8_read_device_status, (any_fn)sfp8_last_device_status,
      (any_fn)sfp8_compressed_values_bytes, (any_fn)sfp8_compressed_meta_bytes,
      (any_fn)sfp8_status_string, (any_fn)sfp8_layout_version};
  for (size_t i = 0; i < sizeof(fns) / sizeof(fns[0]); ++i)
    if (fns[i] == NULL) return 1;

  /* host-only answers */
  if (sfp8_layout_version() != SFP8_LAYOUT_VERSION) return 2;
  if (sfp8_padded_rows(129) != 256 || sfp8_padded_rows(-1) != -1) return 3;
  if (sfp8_compressed_bytes(14336, 4096) != (size_t)36700160) return 4;
  if (sfp8_compressed_values_bytes(14336, 4096) != (size_t)29360128 ||
      sfp8_compressed_meta_bytes(14336, 4096) != (size_t)7340032)
    return 4;
  if (strcmp(sfp8_status_string(SFP8_OK), "ok") != 0) return 5;
  if (strcmp(sfp8_status_string((sfp8_status)99), "unknown status") != 0) return 6;

  /* the decode plan of a 148-SM B200, without a device */
  int64_t info[12];
  if (sfp8_sparse_linear_plan_count(16, 14336, 4096, 148) < 1) return 7;
  if (sfp8_sparse_linear_plan_info(16, 14336, 4096, 148, 0, info) != SFP8_OK) return 8;
  if (info[0] != 0 || info[1] != 16 || info[2] != 4 || info[5] != 1 || info[7] != 112) return 9;

  /* validation before any device is touched */
  if (sfp8_quantize_rowwise(NULL, SFP8_E4M3, 4, 16, 16, NULL, SFP8_E4M3, NULL, NULL) !=
      SFP8_ERR_UNSUPPORTED_DTYPE)
    return 10;
  if (sfp8_quantize_tensorwise_workspace_bytes((sfp8_amax_mode)7) != 0) return 11;
  if (sfp8_sparse_linear_quant_fused(NULL, SFP8_E4M3, 128, SFP8_E4M3, NULL, NULL, 4, NULL,
                                     SFP8_E4M3, NULL, 64, 128, NULL, NULL, NULL, 0, NULL) !=
      SFP8_ERR_UNSUPPORTED_DTYPE)
    return 12;
  if (sfp8_sparse_linear_quant_fusable(16, 14336, 100) != 0) return 13;

  printf("abi ok\n");
  return 0;
}
