"""fp64 CPU oracle for latent-cache decode (MLA / MLRA).

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the tests, the smoke check and
the benchmark's CPU-baseline / reference arm may import it.  The CUDA path never
imports, links or calls anything here, and this package imports nothing from the
CUDA path.

Parity status: every function is pinned by ``tests/test_oracle_pins.py`` against
identities and closed forms the pages fix, a library attention routine and hand-worked
fixtures in ``tests/golden/``.  The pages print no worked numeric example of their
own, so no pin compares against a number printed on the pages.
"""
from .reference import (rope_rotate, mlra_decode_expanded, mlra_decode_absorbed, mla_decode, gla_decode,
                        mlra_prefill_expanded,
                        mla_nope_key, mlra_nope_key_blocks, decode_batch, dequantize_int8_blocks,
                        decode_batch_int8, mlra_partial_state, combine_partial_states, upproject_latent)

__all__ = ["rope_rotate", "mlra_decode_expanded", "mlra_decode_absorbed", "mla_decode", "gla_decode", "mlra_prefill_expanded",
           "mla_nope_key", "mlra_nope_key_blocks", "decode_batch", "dequantize_int8_blocks", "decode_batch_int8",
           "mlra_partial_state", "combine_partial_states", "upproject_latent"]
