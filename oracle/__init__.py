"""CPU oracle for paged MLA decode and the cache append (test infrastructure; see
mla_decode.py and kv_append.py)."""

from .mla_decode import (  # noqa: F401
    combine,
    decode,
    decode_bruteforce,
    decode_partial,
    gather_tokens,
    visible_tokens,
)
from . import kv_append  # noqa: F401,E402
