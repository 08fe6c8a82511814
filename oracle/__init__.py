"""fp64 CPU oracle for MLA decode in absorbed latent space.

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline legs of ``bench.py`` may import it.  It shares no code with the
CUDA path (``mla_latent_space_b200``) and never imports it.
"""
from .mla_decode import (absorb, attend, brute, bf16_to_f64, combine, decode, decode_chunk,  # noqa: F401
                         decompress, e4m3_table, gather_rows, mlavar6_decode, new_token_attention, page_rows_f64, round_bf16, sparse_decode,
                         visible_len)
