"""CPU oracle for the row-wise scaled 2:4 sparse FP8 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the C-ABI library and
its Python binding) imports, calls or links anything in this package.  Only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` (and its ``--impl reference`` arm) use it.

What it computes (page "Add CUTLASS-based row-wise scaled sparse FP8 kernel",
pytorch/ao pull request 1671, ready-for-review comment):

* item 1 -- a row-wise scaled linear with a 2:4 sparse FP8 weight and an FP8
  activation, plus a converter of FP8 data to the compressed 2:4 format;
* item 3 -- the compressor must treat -0.0 as a zero;
* item 4 -- the activation is quantised dynamically (the
  ``Float8DynamicActivationFloat8SemiSparseWeightConfig`` path), the weight
  once, each with one fp32 scale per row.

The modules are written to be read against those statements and against the
OCP 8-bit floating point specification (OFP8), which defines e4m3 and e5m2:

* :mod:`oracle.fp8`       FP8 decode tables from the bit fields; RNE+satfinite
                          encoder.
* :mod:`oracle.quantize`  per-row amax, scale, divide, encode.
* :mod:`oracle.quantize_tensor`  the same with one amax for the whole tensor
                          (page "[float8nocompile] ...", pytorch/ao pull
                          request 1455).
* :mod:`oracle.prune`     2:4 magnitude prune of a 16/32-bit weight.
* :mod:`oracle.compress`  2:4 compression to kept codes + index nibbles, and
                          its inverse.
* :mod:`oracle.layout`    reader of the library's physical compressed layout
                          (written from the layout's specification).
* :mod:`oracle.linear`    the linear in fp64 and the acceptance bound.

Every function here is a plain restatement.  None of it is shared with the
CUDA path; the two meet only in the tests, which feed both the same seeded
inputs from ``semi_structured_sparse_rowwise_b200.synthetic``.
"""

from .fp8 import (E4M3, E5M2, FORMATS, decode_table, decode, fp8_max,
                  max_code, encode_rne_sat, bf16_bits_to_f32, f16_bits_to_f32,
                  round_to_bf16)
from .quantize import quantize_rowwise, GUARD_AMAX
from .quantize_tensor import quantize_tensorwise
from .prune import prune_24
from .compress import compress_24, decompress_24, NIBBLES_VALID
from .layout import unpack_physical, padded_rows, packed_bytes
from .linear import sparse_linear_ref, acceptance_bound, check_linear

__all__ = [
    "E4M3", "E5M2", "FORMATS", "decode_table", "decode", "fp8_max", "max_code",
    "encode_rne_sat", "bf16_bits_to_f32", "f16_bits_to_f32", "round_to_bf16",
    "quantize_rowwise", "quantize_tensorwise", "GUARD_AMAX", "prune_24", "compress_24",
    "decompress_24", "NIBBLES_VALID", "unpack_physical", "padded_rows",
    "packed_bytes", "sparse_linear_ref", "acceptance_bound",
    "check_linear",
]
