"""Row-wise scaled 2:4 sparse FP8 linear for B200 (sm_100a).

The compute path is libsfp8.so (C ABI, include/sfp8.h); this package holds
its build script, a ctypes binding with the same function names, a layer
class on top of it, and the seeded synthetic-input generators.
"""

from .binding import (Sfp8Error, load_library, library_path, new_workspace,
                      sfp8_quantize_rowwise, sfp8_quantize_tensorwise,
                      sfp8_quantize_tensorwise_workspace_bytes, new_tensorwise_workspace,
                      sfp8_prune_24, sfp8_padded_rows,
                      sfp8_compressed_bytes, sfp8_compressed_values_bytes,
                      sfp8_compressed_meta_bytes, sfp8_last_device_status,
                      sfp8_compress_24, sfp8_decompress_24, sfp8_prepare_weight_24,
                      sfp8_sparse_linear_workspace_bytes, sfp8_workspace_clear,
                      sfp8_sparse_linear, sfp8_sparse_linear_noalloc,
                      sfp8_sparse_linear_algo_count, sfp8_sparse_linear_algo_info,
                      sfp8_sparse_linear_algo_workspace_bytes,
                      sfp8_sparse_linear_search_workspace_bytes, sfp8_sparse_linear_algo,
                      sfp8_sparse_linear_search, sfp8_sparse_linear_set_algo,
                      sfp8_sparse_linear_get_algo,
                      sfp8_sparse_linear_quant, sfp8_sparse_linear_quant_workspace_bytes,
                      sfp8_sparse_linear_quant_host, sfp8_sparse_linear_quant_fused,
                      sfp8_sparse_linear_quant_chained, sfp8_sparse_linear_quant_fusable,
                      new_quant_workspace, sfp8_read_device_status, sfp8_selftest_timeout,
                      sfp8_status_string, sfp8_layout_version)
from .layer import HostPipeline, SparseFp8Linear

__all__ = [
    "Sfp8Error", "load_library", "library_path", "new_workspace",
    "sfp8_quantize_rowwise", "sfp8_quantize_tensorwise",
    "sfp8_quantize_tensorwise_workspace_bytes", "new_tensorwise_workspace", "sfp8_prune_24", "sfp8_padded_rows",
    "sfp8_compressed_bytes", "sfp8_compressed_values_bytes", "sfp8_compressed_meta_bytes",
    "sfp8_last_device_status",
    "sfp8_compress_24", "sfp8_decompress_24", "sfp8_prepare_weight_24",
    "sfp8_sparse_linear_workspace_bytes", "sfp8_workspace_clear",
    "sfp8_sparse_linear", "sfp8_sparse_linear_noalloc", "sfp8_sparse_linear_quant",
    "sfp8_sparse_linear_quant_host", "sfp8_sparse_linear_quant_fused",
    "sfp8_sparse_linear_quant_chained", "sfp8_sparse_linear_quant_fusable",
    "sfp8_sparse_linear_algo_count", "sfp8_sparse_linear_algo_info",
    "sfp8_sparse_linear_algo_workspace_bytes", "sfp8_sparse_linear_search_workspace_bytes",
    "sfp8_sparse_linear_algo", "sfp8_sparse_linear_search", "sfp8_sparse_linear_set_algo",
    "sfp8_sparse_linear_get_algo",
    "sfp8_sparse_linear_quant_workspace_bytes", "new_quant_workspace",
    "sfp8_read_device_status", "sfp8_selftest_timeout", "sfp8_status_string",
    "sfp8_layout_version", "SparseFp8Linear", "HostPipeline",
]
