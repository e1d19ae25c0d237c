"""CPU oracle for appending new latent rows to the paged cache.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the tests, the package's
`smoke()` check and the benchmark's CPU legs may use it, and it shares no code with the
CUDA path.

What it computes, and where that comes from
-------------------------------------------
FlashMLA keeps the KV cache in fixed-size blocks handed out on demand, which is what
lets it serve sequences of varying length («DeepSeek booste les performances des GPU
NVIDIA Hopper H800…», tomshardware.fr, paragraph on the block-based paging system; the
FlashMLA release article on shoujike.com.cn gives the block size, 64 tokens). Decoding
a token therefore begins by writing that token's cache row into its page. The pages
print no formula for this step; the plain reading, used here:

  for every sequence b and new token j < s_new:
      t = L_b + j                                  (L_b = tokens already cached)
      kcache[block_table[b][t // 64], t % 64, 0, :] = kv_new[b, j, :]   (all 576 dims)

Nothing else in the cache changes. The lengths are not advanced here: the caller owns
them and moves each L_b to L_b + s_new once the rows are in place.

This is a byte copy, so the oracle works on the raw 16-bit patterns and the GPU result
must match it bit for bit.
"""

from __future__ import annotations

import numpy as np

BLOCK_SIZE = 64


def _bits(x) -> np.ndarray:
    """The 16-bit patterns of a bf16 tensor or array (a copy, as uint16)."""
    if hasattr(x, "view") and hasattr(x, "dtype") and "bfloat16" in str(x.dtype):
        import torch
        return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).copy()
    return np.array(x, dtype=np.uint16, copy=True)


def append(kcache, block_table, seqlens, kv_new):
    """The cache after writing kv_new[b, j] at position seqlens[b] + j of sequence b.

    kcache [num_blocks, 64, 1, 576] and kv_new [batch, s_new, 576] are bf16 (torch) or
    uint16 bit patterns; block_table [batch, max_blocks] and seqlens [batch] are ints.
    Returns the new cache as uint16 bit patterns. Raises IndexError when a position is
    past the block table or its block id is outside the pool.
    """
    out = _bits(kcache)
    new = _bits(kv_new)
    bt = np.asarray(block_table, dtype=np.int64)
    lens = np.asarray(seqlens, dtype=np.int64)
    batch, s_new, _ = new.shape
    for b in range(batch):
        for j in range(s_new):
            t = int(lens[b]) + j
            page = t // BLOCK_SIZE
            if page >= bt.shape[1]:
                raise IndexError(f"position {t} of sequence {b} is past its block table")
            blk = int(bt[b, page])
            if not 0 <= blk < out.shape[0]:
                raise IndexError(f"block id {blk} of sequence {b} is outside the pool")
            out[blk, t % BLOCK_SIZE, 0, :] = new[b, j, :]
    return out
