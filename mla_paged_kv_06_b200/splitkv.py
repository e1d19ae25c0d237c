"""Split-KV across GPUs: one sequence's pages spread over several ranks.

Batch sharding (`shard.py`) keeps every sequence on one GPU. A sequence whose cache is
too long for one GPU's share, or a batch too small to fill every GPU, can instead have
its pages split across the ranks of a group: rank g holds a contiguous run of pages of
every sequence, decodes all query rows over just those tokens, and the ranks merge
their results with the split-KV identity (the same one the single-GPU combine applies
to chunks; the FlashMLA release article's paragraph on dynamic sequence handling is
where the pages place split-KV scheduling). The pages say nothing about decoding one
sequence on several GPUs, so the partition below is this library's own. Its one rule
comes from the causal mask:

  with causal decode of s_q > 1 query tokens, query i sees tokens t < L - s_q + i + 1.
  A rank that holds the sequence's last token decodes its slice causally (its slice
  length L_g stands in for L, which shifts every n_i by the same offset), and every
  other rank must hold only tokens every query sees, t < L - s_q + 1, so that it can
  decode its slice without a mask. `plan_kv_split` moves the last rank's first page
  back until that holds.

The data path per rank: `mla_get_metadata` + `mla_decode_fwd_partial` on its slice
(fp32 output, natural-log lse), one all-gather of those partials over the group
(`exchange_partials`: batch * s_q * h_q * (512 + 1) * 4 bytes per rank), then
`mla_combine_partials` on the gathered parts. All arithmetic is in the library's
kernels; this module only plans, slices and moves tensors.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from .workloads import BLOCK_SIZE, DecodeInputs


@dataclass
class KvSplitPlan:
    """page_begin[g][b], page_end[g][b]: half-open page range of sequence b on rank g;
    tokens[g][b]: the tokens of that range (the slice length rank g decodes)."""
    world: int
    page_begin: list[list[int]]
    page_end: list[list[int]]
    tokens: list[list[int]]
    causal: bool

    def rank_causal(self, rank: int) -> bool:
        """Whether rank `rank` decodes its slices with the causal mask: only the last
        rank, which holds every sequence's last token."""
        return self.causal and rank == self.world - 1


def plan_kv_split(seqlens, world: int, s_q: int = 1, causal: bool = False) -> KvSplitPlan:
    """Contiguous, balanced page ranges of every sequence over `world` ranks.

    Sequence b with P = ceil(L/64) pages gives rank g the pages
    [floor(g P / world), floor((g+1) P / world)), so the ranks' page counts differ by at
    most one. For causal decode the last rank's first page is moved back to at most
    floor((L - s_q + 1) / 64) (never below 0), and the other ranks' ranges are cut at
    it, so that every token before the last rank's slice is visible to every query.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    if s_q < 1:
        raise ValueError("s_q must be >= 1")
    lens = [int(x) for x in torch.as_tensor(seqlens).tolist()]
    if any(L < 0 for L in lens):
        raise ValueError("negative sequence length")
    pb = [[0] * len(lens) for _ in range(world)]
    pe = [[0] * len(lens) for _ in range(world)]
    tok = [[0] * len(lens) for _ in range(world)]
    for b, L in enumerate(lens):
        P = (L + BLOCK_SIZE - 1) // BLOCK_SIZE
        cuts = [g * P // world for g in range(world + 1)]
        if causal and s_q > 1 and world > 1:
            last_begin = min(cuts[world - 1], max(L - s_q + 1, 0) // BLOCK_SIZE)
            cuts = [min(c, last_begin) for c in cuts[:world]] + [P]
        for g in range(world):
            pb[g][b], pe[g][b] = cuts[g], cuts[g + 1]
            tok[g][b] = max(0, min(cuts[g + 1] * BLOCK_SIZE, L) - cuts[g] * BLOCK_SIZE)
    return KvSplitPlan(world, pb, pe, tok, bool(causal))


def make_kv_slice(x: DecodeInputs, plan: KvSplitPlan, rank: int) -> DecodeInputs:
    """Rank `rank`'s inputs under `plan`: every query row, its page ranges as a compact
    pool (first-use order) with the block table renumbered into it, its slice lengths,
    and its causal flag. Table entries past a slice's last page point at page 0 of the
    pool (the decode never reads them); a rank without pages gets a one-page pool of
    zeros so that every pointer stays valid."""
    batch = x.seqlens.numel()
    counts = [plan.page_end[rank][b] - plan.page_begin[rank][b] for b in range(batch)]
    table = torch.zeros((batch, max(counts + [1])), dtype=torch.int32)
    remap: dict[int, int] = {}
    for b in range(batch):
        for j in range(counts[b]):
            phys = int(x.block_table[b, plan.page_begin[rank][b] + j])
            if phys not in remap:
                remap[phys] = len(remap)
            table[b, j] = remap[phys]
    if remap:
        kcache = x.kcache[list(remap.keys())].clone()
    else:
        kcache = torch.zeros((1,) + tuple(x.kcache.shape[1:]), dtype=x.kcache.dtype)
    seqlens = torch.tensor(plan.tokens[rank], dtype=torch.int32)
    return DecodeInputs(x.q.clone(), kcache, table, seqlens, x.scale, plan.rank_causal(rank),
                        x.workload, x.seed)


def exchange_partials(out_part: torch.Tensor, lse_part: torch.Tensor, group=None):
    """All-gather of every rank's partial over `group` (NCCL for CUDA tensors, gloo for
    CPU ones): returns (o_parts [world, ...], lse_parts [world, ...]) stacked in rank
    order, the layout `mla_combine_partials` reads. Without an initialised process group
    the rank's own partial is the only part."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return out_part.unsqueeze(0).contiguous(), lse_part.unsqueeze(0).contiguous()
    world = dist.get_world_size(group)
    o_parts = torch.empty((world,) + tuple(out_part.shape), dtype=out_part.dtype,
                          device=out_part.device)
    lse_parts = torch.empty((world,) + tuple(lse_part.shape), dtype=lse_part.dtype,
                            device=lse_part.device)
    dist.all_gather(list(o_parts.unbind(0)), out_part.contiguous(), group=group)
    dist.all_gather(list(lse_parts.unbind(0)), lse_part.contiguous(), group=group)
    return o_parts, lse_parts


def split_kv_decode(q, kcache, block_table, seqlens, scale, causal, group=None,
                    num_sms=None, stream=None):
    """Decode of this rank's slice (device tensors from `make_kv_slice`, `causal` its
    rank flag), exchange with the group, merge. Every rank returns the full
    (out bf16 [b,s_q,h_q,512], lse fp32 [b,h_q,s_q])."""
    from . import mla
    batch, s_q, h_q, _ = q.shape
    meta, ns = mla.mla_get_metadata(seqlens, h_q, s_q, num_sms=num_sms, stream=stream)
    o_part, lse_part = mla.mla_decode_fwd_partial(q, kcache, block_table, seqlens, scale,
                                                  causal, meta, ns, stream=stream,
                                                  num_sms=num_sms)
    o_parts, lse_parts = exchange_partials(o_part, lse_part, group)
    return mla.mla_combine_partials(o_parts, lse_parts, stream=stream)
