"""Decode of sequences whose KV cache is split over GPUs by token range.

A very long sequence (e.g. one of a million tokens) can hold its packed cache
on several GPUs: rank r keeps the records of one contiguous token range of every
(sequence, KV head), compressed there by ``tq_compress_kv`` as the tokens arrive.
A decode step is then one partial decode per rank over its own range
(``tq_decode_attention_partial``: the normalized output and the log of the
softmax denominator per query head), ONE exchange step (an all-gather of those
partials, (d + 1) floats per query head, a few KB), and the same log-sum-exp
merge on every rank (``tq_merge_attention``). The merge is an exact identity of
the softmax over the union of the ranges, so the result equals a decode over the
whole cache up to fp32 rounding.

The exchange is NCCL's all-gather through ``torch.distributed``: it moves
rows * (d + 1) floats per rank once per step, far below any bandwidth limit, so
its cost is the collective's launch latency; fusing it into a kernel over peer
memory would save microseconds on a step whose decode reads gigabytes.

Everything runs on torch's current CUDA stream, which the NCCL collective is
ordered with.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib


def token_range(n_tokens: int, world: int, rank: int, block: int = 512) -> tuple[int, int]:
    """[start, end) of the tokens rank ``rank`` of ``world`` holds: the sequence is cut
    into blocks of ``block`` tokens (whole tiles of every decode kernel), and the blocks
    are dealt out in contiguous runs as evenly as they go, earlier ranks taking the
    extra ones. A rank may get an empty range (more ranks than blocks)."""
    if n_tokens < 0 or world < 1 or not 0 <= rank < world or block < 1:
        raise ValueError("token_range: need n_tokens >= 0, world >= 1, 0 <= rank < world, block >= 1")
    n_blocks = -(-n_tokens // block)
    per, extra = divmod(n_blocks, world)
    b0 = rank * per + min(rank, extra)
    b1 = b0 + per + (1 if rank < extra else 0)
    return min(b0 * block, n_tokens), min(b1 * block, n_tokens)


def local_lengths(seq_lens, start: int, end: int):
    """Valid tokens of each sequence inside [start, end): clamp(len - start, 0, end - start)."""
    return (seq_lens - start).clamp(min=0, max=end - start).to(torch.int32)


class SplitSequenceDecoder:
    """Buffers and steps of one decode shape (batch, hq, d) split over the ranks of
    ``group`` (the default process group; a single process when torch.distributed is
    not initialized).

    Each rank's partial lives in one float buffer, output [batch][hq][d] then lse
    [batch][hq] padded to 16 bytes, so the exchange is a single all-gather into a
    [world][part] buffer from which the merge reads every rank's part in place."""

    def __init__(self, batch: int, hq: int, d: int, device=None, group=None):
        self.batch, self.hq, self.d, self.group = batch, hq, d, group
        if dist.is_available() and dist.is_initialized():
            self.world, self.rank = dist.get_world_size(group), dist.get_rank(group)
        else:
            self.world, self.rank = 1, 0
        self.rows = batch * hq
        self.part_floats = self.rows * d + -(-self.rows // 4) * 4
        self.part = torch.zeros(self.part_floats, dtype=torch.float32, device=device)
        self.gathered = (self.part if self.world == 1 else
                         torch.zeros(self.world * self.part_floats, dtype=torch.float32, device=device))
        self.workspace = None

    def local_out(self):
        """This rank's output view [batch, hq, d] inside its part."""
        return self.part[: self.rows * self.d].view(self.batch, self.hq, self.d)

    def local_lse(self):
        """This rank's log-partition view [batch, hq] inside its part."""
        n = self.rows * self.d
        return self.part[n: n + self.rows].view(self.batch, self.hq)

    def exchange(self) -> None:
        """The one exchange step: every rank's part into ``gathered``, in rank order."""
        if self.world > 1:
            dist.all_gather_into_tensor(self.gathered, self.part, group=self.group)

    def gathered_parts(self):
        """Views (outs [world, batch, hq, d], lses [world, batch, hq]) of the gathered parts."""
        g = self.gathered.view(self.world, self.part_floats)
        n = self.rows * self.d
        outs = g[:, :n].view(self.world, self.batch, self.hq, self.d)
        lses = g[:, n: n + self.rows].view(self.world, self.batch, self.hq)
        return outs, lses

    def __call__(self, ctx, q, packed: dict, hkv: int, max_len: int, seq_lens=None,
                 softmax_scale: float = 0.0, out=None):
        """One decode step: q [batch, hq, d] (the same on every rank) against this rank's
        packed token range (``max_len`` slots per (sequence, KV head), ``seq_lens`` the
        valid tokens of this range, e.g. from ``local_lengths``). Returns the attention
        over all ranks' tokens, [batch, hq, d] fp32, on every rank."""
        need = _lib.tq_decode_workspace_bytes(ctx, self.batch, self.hq, hkv, max_len)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
        _lib.tq_decode_attention_partial(ctx, q, packed, self.batch, self.hq, hkv, max_len, seq_lens=seq_lens,
                                         softmax_scale=softmax_scale, out=self.local_out(),
                                         lse=self.local_lse(), workspace=self.workspace)
        self.exchange()
        outs, lses = self.gathered_parts()
        return _lib.tq_merge_attention(outs, lses, out=out)[0]
