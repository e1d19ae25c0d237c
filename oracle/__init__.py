"""CPU oracle for paged MLA decode (test infrastructure; see mla_decode.py)."""

from .mla_decode import (  # noqa: F401
    combine,
    decode,
    decode_bruteforce,
    decode_partial,
    gather_tokens,
    visible_tokens,
)
