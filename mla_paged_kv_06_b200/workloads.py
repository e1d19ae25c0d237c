"""Seeded synthetic inputs for paged MLA decode.

This module only draws inputs. It holds none of the attention arithmetic, so the
CPU oracle and the CUDA path can share it without sharing any of the method.

Shapes and layout (the paged latent cache of the FlashMLA release article,
«DeepSeek open-sources FlashMLA», shoujike.com.cn: "paged kvcache, BF16, block
size 64"; MLA keeps one compressed latent row per token, shared by every head):

  q            bf16  [batch, s_q, h_q, 576]
  kcache       bf16  [num_blocks, 64, 1, 576]   (one shared latent KV head)
  block_table  int32 [batch, max_blocks]        (physical block id per logical block)
  seqlens      int32 [batch]

Every tensor is drawn on the CPU from a torch.Generator seeded per purpose, so the
same seed gives the same bytes on any machine. q and the cache are N(0, 1) rounded
to bf16 (round-to-nearest-even, torch's conversion).
"""

from __future__ import annotations

import dataclasses
import math

import torch

HEAD_DIM = 576          # latent (512) + rope (64) dims of one cache row
HEAD_DIM_V = 512        # V is the first 512 dims of the same row
BLOCK_SIZE = 64         # tokens per page
DEFAULT_SCALE = 192 ** -0.5


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    s_q: int
    h_q: int
    causal: bool
    seqlen: str            # how the lengths are drawn (see draw_seqlens)
    pool: str              # "exact" (sum of blocks) or "spare:<n>" extra unused blocks
    description: str


# The five decode workloads. Sizes follow DeepSeek-V3 decode shapes: 128 query heads
# without tensor parallelism, one 576-dim latent row per token.
WORKLOADS = {
    "tiny": Workload("tiny", 2, 1, 16, False, "fixed:37,130", "spare:4",
                     "b=2 s_q=1 h_q=16 L={37,130}, 8-block pool, NaN tails and unused blocks"),
    "uniform": Workload("uniform", 64, 1, 16, False, "fixed_all:4096", "exact",
                        "b=64 s_q=1 h_q=16 L=4096, 4096-block pool permuted"),
    "v3": Workload("v3", 128, 1, 128, False, "uniform:1,8192", "exact",
                   "b=128 s_q=1 h_q=128 L~U[1,8192]"),
    "spec": Workload("spec", 128, 2, 128, True, "uniform:512,8192", "exact",
                     "b=128 s_q=2 causal h_q=128 L~U[512,8192]"),
    "skewed": Workload("skewed", 32, 1, 64, False, "lognormal:1024,1.0,4x65536", "exact",
                       "b=32 s_q=1 h_q=64 L~lognormal(median 1024, sigma 1) + 4 x 65536"),
}

# Purpose-specific seed offsets so changing one draw never shifts another.
_SEED_LENS, _SEED_PERM, _SEED_Q, _SEED_CACHE = 11, 23, 37, 41


def _gen(seed: int, purpose: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1_000_003 + purpose)
    return g


def draw_seqlens(spec: str, batch: int, seed: int) -> torch.Tensor:
    """Sequence lengths, int32 [batch]. Integer uniform ranges are inclusive at both ends."""
    kind, _, arg = spec.partition(":")
    g = _gen(seed, _SEED_LENS)
    if kind == "fixed":
        vals = [int(x) for x in arg.split(",")]
        assert len(vals) == batch
        return torch.tensor(vals, dtype=torch.int32)
    if kind == "fixed_all":
        return torch.full((batch,), int(arg), dtype=torch.int32)
    if kind == "uniform":
        lo, hi = (int(x) for x in arg.split(","))
        return torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int64).to(torch.int32)
    if kind == "lognormal":
        median, sigma, forced = arg.split(",")
        n_forced, forced_len = (int(x) for x in forced.split("x"))
        z = torch.randn(batch, generator=g, dtype=torch.float64)
        lens = torch.exp(math.log(float(median)) + float(sigma) * z).round()
        lens = lens.clamp(1, 65536).to(torch.int32)
        idx = torch.randperm(batch, generator=g)[:n_forced]
        lens[idx] = forced_len
        return lens
    raise ValueError(f"unknown seqlen spec {spec!r}")


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor             # bf16 [b, s_q, h_q, 576]
    kcache: torch.Tensor        # bf16 [num_blocks, 64, 1, 576]
    block_table: torch.Tensor   # int32 [b, max_blocks]
    seqlens: torch.Tensor       # int32 [b]
    scale: float
    causal: bool
    workload: str
    seed: int

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def s_q(self) -> int:
        return self.q.shape[1]

    @property
    def h_q(self) -> int:
        return self.q.shape[2]

    @property
    def num_blocks(self) -> int:
        return self.kcache.shape[0]


def blocks_needed(seqlens: torch.Tensor) -> torch.Tensor:
    return (seqlens.to(torch.int64) + BLOCK_SIZE - 1) // BLOCK_SIZE


def make_paged_inputs(seqlens, s_q: int, h_q: int, *, seed: int = 0, causal: bool = False,
                      spare_blocks: int = 0, poison: bool = False,
                      scale: float = DEFAULT_SCALE, workload: str = "custom") -> DecodeInputs:
    """Build q, a paged cache and a block table for the given lengths.

    The pool holds sum(ceil(L/64)) blocks plus `spare_blocks`, in a seeded random
    permutation of physical ids. With `poison`, every cache slot no sequence owns (the
    tail rows of each last block and every spare block) is NaN, and block-table entries
    past a sequence's last block point at spare blocks (or 0 without spares), so a kernel
    that reads past a sequence's end shows NaN in its output.
    """
    seqlens = torch.as_tensor(seqlens, dtype=torch.int32).clone()
    batch = seqlens.numel()
    nblk = blocks_needed(seqlens)
    used = int(nblk.sum())
    num_blocks = max(used + spare_blocks, 1)
    max_blocks = max(int(nblk.max()) if batch else 0, 1)

    perm = torch.randperm(num_blocks, generator=_gen(seed, _SEED_PERM)).to(torch.int32)
    block_table = torch.zeros((batch, max_blocks), dtype=torch.int32)
    spare_ids = perm[used:]
    pos = 0
    for b in range(batch):
        n = int(nblk[b])
        block_table[b, :n] = perm[pos:pos + n]
        pos += n
        if max_blocks > n:
            if spare_ids.numel() > 0:
                fill = spare_ids[torch.arange(max_blocks - n) % spare_ids.numel()]
            else:
                fill = torch.zeros(max_blocks - n, dtype=torch.int32)
            block_table[b, n:] = fill

    q = torch.randn((batch, s_q, h_q, 576), generator=_gen(seed, _SEED_Q),
                    dtype=torch.float32).to(torch.bfloat16)
    kcache = torch.randn((num_blocks, BLOCK_SIZE, 1, 576), generator=_gen(seed, _SEED_CACHE),
                         dtype=torch.float32).to(torch.bfloat16)
    if poison:
        owned = torch.zeros((num_blocks, BLOCK_SIZE), dtype=torch.bool)
        for b in range(batch):
            L = int(seqlens[b])
            for j in range(int(nblk[b])):
                rows = min(BLOCK_SIZE, L - j * BLOCK_SIZE)
                owned[int(block_table[b, j]), :rows] = True
        kcache[~owned] = float("nan")
    return DecodeInputs(q, kcache, block_table, seqlens, scale, causal, workload, seed)


def make_workload(name: str, seed: int = 0, *, poison: bool | None = None) -> DecodeInputs:
    """Inputs for one of the named workloads. `poison` defaults to True for 'tiny' only."""
    w = WORKLOADS[name]
    seqlens = draw_seqlens(w.seqlen, w.batch, seed)
    spare = int(w.pool.split(":")[1]) if w.pool.startswith("spare") else 0
    if poison is None:
        poison = name == "tiny"
    if poison and spare == 0:
        spare = 4
    return make_paged_inputs(seqlens, w.s_q, w.h_q, seed=seed, causal=w.causal,
                             spare_blocks=spare, poison=poison, workload=name)


def algorithmic_work(seqlens, s_q: int, h_q: int, causal: bool):
    """(bytes, flops) of one decode call counted from the operation's definition.

    bytes: every visible KV row once (576 bf16), q, out (512 bf16) and lse (fp32).
    flops: 2*(576 + 512) per (query row, visible token).
    """
    bytes_ = 0
    flops = 0
    for L in (int(x) for x in torch.as_tensor(seqlens).tolist()):
        bytes_ += L * 576 * 2
        for i in range(s_q):
            n = L - s_q + i + 1 if causal else L
            flops += max(n, 0) * h_q * 2 * (576 + 512)
    b = len(torch.as_tensor(seqlens))
    bytes_ += b * s_q * h_q * (576 * 2 + 512 * 2 + 4)
    return bytes_, flops
