"""CPU oracle for paged MLA decode, the cache append and the FP8 cache format (test
infrastructure; see mla_decode.py, kv_append.py and fp8_cache.py)."""

from .mla_decode import (  # noqa: F401
    combine,
    decode,
    decode_bruteforce,
    decode_partial,
    gather_tokens,
    visible_tokens,
)
from . import fp8_cache, kv_append  # noqa: F401,E402
