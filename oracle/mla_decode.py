"""CPU oracle for paged MLA decode.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links this
module: only the tests, the package's `smoke()` check and the CPU-baseline leg of the
benchmark may use it. It shares no code with the CUDA path; both sides take their
inputs from the seeded generator, which holds no attention arithmetic.

What it computes, and where that comes from
-------------------------------------------
FlashMLA is a decode kernel for Multi-head Latent Attention over a paged BF16 KV cache
with 64-token blocks, tuned for variable-length sequences («DeepSeek open-sources
FlashMLA» news page, shoujike.com.cn: the paragraphs on the decode kernel, on the
paged kvcache and on dynamic sequence handling). MLA keeps one compressed latent row
per token and every head reads that same row (same page, paragraph on key-value
compression into a latent vector; the DeepSeek-V3 co-design summary on
news.chathome.org gives the resulting ~70 KB per token). The operation decoded here:

  row r = (i, h), i < s_q query tokens, h < h_q heads, one shared latent head
  K_t   = the 576-dim cache row of token t, V_t = its first 512 dims
  n_i   = L - s_q + i + 1 visible tokens if causal, else L
  s_t   = scale * <q[b, i, h, :], K_t>              for t < n_i
  out   = sum_t softmax(s)_t * V_t                  (512 dims)
  lse   = ln sum_t exp(s_t)                         (natural log, scale inside)

The pages print no formula or worked example for this; the formula above is the plain
reading of "attention decode over a latent cache" and is exact attention, not an
approximation. Readings the pages leave open:
  * n_i <= 0 (an empty sequence, or a causal row that sees nothing): out = 0,
    lse = -inf.
  * The oracle never reads a cache slot at t >= n_i, so NaN padding cannot reach it.
  * Arithmetic is fp64 on the bf16 inputs upcast exactly; nothing is rounded back.

Pins (tests/test_oracle.py, run without a GPU) tie each function to something other
than itself: brute-force fsum loops on tiny inputs, a hand-derived worked example in
tests/golden/, the single-token and equal-score closed forms, block-permutation
invariance, NaN padding, the causal reduction to s_q = 1, and the split identity that
defines `combine`. Numeric parity with FlashMLA's own outputs is unpinned: the pages
print no values for it.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK_SIZE = 64
HEAD_DIM_V = 512


def _f64(x) -> np.ndarray:
    """Upcast a numpy array or a (bf16/fp32) torch tensor to float64 exactly."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.is_floating_point():
            x = x.to(dtype=__import__("torch").float64)
        return x.numpy()
    return np.asarray(x, dtype=np.float64)


def _i64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        return x.detach().cpu().numpy().astype(np.int64)
    return np.asarray(x, dtype=np.int64)


def visible_tokens(seqlen: int, s_q: int, i: int, causal: bool) -> int:
    """Tokens query i of a sequence of length `seqlen` may attend to.

    Causal speculative decode appends the s_q query tokens at the end of the sequence,
    so query i (0-based) sees the first L - s_q + i + 1 tokens; non-causal sees all L.
    """
    return seqlen - s_q + i + 1 if causal else seqlen


def gather_tokens(kcache, block_table_row, n: int) -> np.ndarray:
    """Dense fp64 [n, 576] copy of a sequence's first n cache rows through its block table.

    Logical token t lives in physical block block_table_row[t // 64], slot t % 64
    (paged kvcache with block size 64, FlashMLA release article). `kcache` may be a
    numpy array or a torch tensor of any float dtype; only the gathered rows are upcast.
    """
    t = np.arange(n)
    blocks = _i64(block_table_row)[t // BLOCK_SIZE]
    slots = t % BLOCK_SIZE
    if hasattr(kcache, "detach"):
        import torch
        rows = kcache[torch.from_numpy(blocks), torch.from_numpy(slots), 0, :]
        return _f64(rows)
    return np.asarray(kcache, dtype=np.float64)[blocks, slots, 0, :]


def decode(q, kcache, block_table, seqlens, scale: float, causal: bool,
           batch_indices=None):
    """Exact MLA decode attention in fp64.

    q [b, s_q, h_q, 576], kcache [num_blocks, 64, 1, 576], block_table [b, max_blocks],
    seqlens [b]. Returns (out [b', s_q, h_q, 512], lse [b', h_q, s_q]) as float64,
    where b' runs over `batch_indices` (all sequences by default).
    """
    bt = _i64(block_table)
    lens = _i64(seqlens)
    _, s_q, h_q, _ = q.shape
    idx = range(q.shape[0]) if batch_indices is None else list(batch_indices)
    qq = _f64(q[list(idx)] if hasattr(q, "detach") else np.asarray(q)[list(idx)])
    out = np.zeros((len(idx), s_q, h_q, HEAD_DIM_V))
    lse = np.full((len(idx), h_q, s_q), -np.inf)
    for ob, b in enumerate(idx):
        L = int(lens[b])
        n_max = max(visible_tokens(L, s_q, i, causal) for i in range(s_q))
        if n_max <= 0:
            continue
        K = gather_tokens(kcache, bt[b], n_max)      # [n_max, 576]
        V = K[:, :HEAD_DIM_V]                         # V = first 512 dims of the row
        for i in range(s_q):
            n = visible_tokens(L, s_q, i, causal)
            if n <= 0:
                continue
            S = scale * (qq[ob, i] @ K[:n].T)         # [h_q, n]
            m = S.max(axis=1, keepdims=True)
            E = np.exp(S - m)
            l = E.sum(axis=1)
            out[ob, i] = (E @ V[:n]) / l[:, None]
            lse[ob, :, i] = m[:, 0] + np.log(l)
    return out, lse


def decode_partial(q_rows, K_rows, scale: float):
    """Attention of q_rows [R, 576] over an explicit token set K_rows [n, 576].

    Returns (out [R, 512], lse [R]) for that token subset alone; used to state the
    split-KV combine identity. An empty token set gives out = 0, lse = -inf.
    """
    qq = _f64(q_rows)
    K = _f64(K_rows)
    R = qq.shape[0]
    if K.shape[0] == 0:
        return np.zeros((R, HEAD_DIM_V)), np.full(R, -np.inf)
    S = scale * (qq @ K.T)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    l = E.sum(axis=1)
    return (E @ K[:, :HEAD_DIM_V]) / l[:, None], m[:, 0] + np.log(l)


def combine(partial_out, partial_lse):
    """Merge attention over disjoint token subsets.

    partial_out [P, R, 512], partial_lse [P, R] (natural log). The softmax over the
    union of the subsets weighs subset p by exp(lse_p - lse) with
    lse = ln sum_p exp(lse_p); subsets with lse_p = -inf weigh nothing, and if every
    subset is empty the result is out = 0, lse = -inf.
    """
    po = _f64(partial_out)
    pl = _f64(partial_lse)
    m = pl.max(axis=0)                                   # [R]
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.exp(pl - m_safe[None, :])                     # exp(-inf) = 0
    total = w.sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, total, 1.0)), -np.inf)
    coef = np.where(finite[None, :], w / np.where(finite, total, 1.0)[None, :], 0.0)
    out = (coef[:, :, None] * po).sum(axis=0)
    return out, lse


def decode_bruteforce(q, kcache, block_table, seqlens, scale: float, causal: bool):
    """Triple loop with math.fsum and no max subtraction, for tiny inputs only.

    Follows the definition token by token: it looks up block_table[b][t // 64] for each
    token, forms every dot product with fsum, and normalises with fsum of exp(s_t).
    """
    kc = _f64(kcache)
    bt = _i64(block_table)
    lens = _i64(seqlens)
    qq = _f64(q)
    B, s_q, h_q, D = qq.shape
    out = np.zeros((B, s_q, h_q, HEAD_DIM_V))
    lse = np.full((B, h_q, s_q), -np.inf)
    for b in range(B):
        L = int(lens[b])
        for i in range(s_q):
            n = visible_tokens(L, s_q, i, causal)
            for h in range(h_q):
                if n <= 0:
                    continue
                rows = []
                for t in range(n):
                    rows.append(kc[int(bt[b][t // BLOCK_SIZE]), t % BLOCK_SIZE, 0])
                e = []
                for t in range(n):
                    s = scale * math.fsum(float(qq[b, i, h, d]) * float(rows[t][d])
                                          for d in range(D))
                    e.append(math.exp(s))
                z = math.fsum(e)
                for d in range(HEAD_DIM_V):
                    out[b, i, h, d] = math.fsum(e[t] * float(rows[t][d]) for t in range(n)) / z
                lse[b, h, i] = math.log(z)
    return out, lse
