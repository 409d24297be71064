"""fp64 CPU oracle for the block-DCT KV codec and coefficient-domain decode
attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
anything under ``oracle/``; only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it. It shares no code with the CUDA path:
no kernels, headers, tables or constant generators. Its only common input with
the CUDA path is the seeded data from ``synth``.

Everything is NumPy float64 and written from the definitions on the
flashcodec-kv 1.0.0 pages:

* ``codec``     -- DCT-II block basis, block compression, the int8
                   per-(block, frequency) quantiser, decompression and storage
                   accounting (README "Math"; ``flashcodec/cache.py``
                   ``_CodecStream._archive``).
* ``attention`` -- decode attention three ways: decompress-then-softmax (the
                   plain definition), the coefficient-domain per-block online
                   softmax (README "Materialization-free decode attention";
                   ``flashcodec/triton_attention.py`` module docstring), and its
                   split-K partials plus combine.
* ``stream``    -- the raw-tail / capacity-doubling archive with append,
                   the reconstructed view, crop, batch gather and reset
                   (``flashcodec/cache.py`` ``_CodecStream``).
* ``png``       -- the PNG-style lossless tier: per-block anchor and fp32
                   first differences, cumulative-sum reconstruction, storage,
                   and decode attention on the stored rows (README "Math").

Every function is pinned by a ``-m "not gpu"`` test against something other
than itself (library DCT, closed forms, brute force, the pages' printed
storage numbers). The one exception is the PSNR band of the README's
reconstruction table, whose random-walk input the pages never define: that
check is a loose ordering sanity test, parity unpinned.
"""

from .codec import (dct_basis, synthesis_basis, split_blocks, compress,
                    quantize, dequantize, decompress, round_to_dtype,
                    storage_bytes_per_block, encode_stream)
from .attention import (decode_attention_reference, coeff_decode_attention,
                        split_partials, combine_partials,
                        splitk_decode_attention, attend_archive)
from .stream import CodecStreamOracle
from .png import (png_filter, png_store, png_reconstruct, png_synthesis,
                  png_rows, png_storage_bytes, png_decode_attention_reference,
                  png_coeff_decode_attention, png_splitk_decode_attention)

__all__ = [
    "dct_basis", "synthesis_basis", "split_blocks", "compress", "quantize",
    "dequantize", "decompress", "round_to_dtype", "storage_bytes_per_block",
    "encode_stream",
    "decode_attention_reference", "coeff_decode_attention", "split_partials",
    "combine_partials", "splitk_decode_attention", "attend_archive",
    "CodecStreamOracle",
    "png_filter", "png_store", "png_reconstruct", "png_synthesis", "png_rows",
    "png_storage_bytes", "png_decode_attention_reference",
    "png_coeff_decode_attention", "png_splitk_decode_attention",
]
