"""CPU oracle for lossless BF16 exponent compression fused with the matmul.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
link this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (``decode_gemm_b200``) and does not import it.

Source of the method: the Cloudflare blog post "Unweight: how we compressed an
LLM 22% without sacrificing quality" (cited below as *Unweight*, with the
section heading the statement sits under).  Where the post leaves a step open,
the reading taken is written next to the code that takes it.

Precision: everything the method does to the weights is integer and exact, so
the oracle is exact; the matmul is accumulated in float64.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test against
something other than itself (round-trip identity, Kraft equality, brute-force
optimal lengths, Huffman cost equality, the RFC 1951 worked example, entropy
bounds, hand-computed bitstreams, brute-force fsum matmul).  No function is
"parity unpinned".
"""
from .bf16 import split_fields, join_fields, exponent_bytes, to_float64
from .palette import (exponent_histogram, build_palette, escape_rows, transcode,
                      pack_nibbles, unpack_nibbles, ROW)
from .huffman import (package_merge_lengths, canonical_codes, encode_bitstream,
                      decode_bitstream, decode_chunk, chunk_offsets, kraft_sum,
                      entropy_bits, average_code_length)
from .container import encode, decode_full, decode_exp, transcode_from_stream, Encoded
from .gemm import gemm_fp64, abs_product_sum, within_tolerance, gemm_entry_fsum, swiglu

__all__ = [
    "split_fields", "join_fields", "exponent_bytes", "to_float64",
    "exponent_histogram", "build_palette", "escape_rows", "transcode", "pack_nibbles",
    "unpack_nibbles", "ROW",
    "package_merge_lengths", "canonical_codes", "encode_bitstream", "decode_bitstream",
    "decode_chunk", "chunk_offsets", "kraft_sum", "entropy_bits", "average_code_length",
    "encode", "decode_full", "decode_exp", "transcode_from_stream", "Encoded",
    "gemm_fp64", "abs_product_sum", "within_tolerance", "gemm_entry_fsum", "swiglu",
]
