"""Vocabulary-parallel decode step: W split by rows over the ranks of a process group.

Rank r holds the contiguous shard W[v0:v1] (``dist.shard_range`` over V) and the same H and
mask as every other rank.  One step:

1. ``masked_partials`` on the shard: compaction, gather, the tensor-core GEMM over the
   shard's vocabulary, and per masked row the softmax partial (max m, sum of exp s, global
   argmax a; plus t and the second max with entropy / margin), written into this rank's
   slot of a packed buffer;
2. one all-gather of the packed partials (12 bytes per row per rank, 20 with entropy /
   margin): the only exchange of the step;
3. ``lse_merge`` of the gathered partials in rank (= vocabulary) order into tok, conf and
   lse over the whole vocabulary;
4. ``select_unmask``.  Every rank ends the step with the same selection.

The merge is the split-vocabulary algebra the GEMM epilogue already applies across its
own vocabulary tiles (Mosaic page, mask-only logits kernel), applied across GPUs.  The
partials are laid out so that one flat collective moves them: ``PartialLayout``.
"""
from __future__ import annotations

import torch

from . import dist as D


class PartialLayout:
    """Packed partials of one rank: fields (m, s, a) -- and (t, m2) in extended mode -- each
    ``n_pad`` entries (n_cap rounded up to 4, so every field starts 16-byte aligned), as one
    float32 buffer [fields, n_pad]; the gathered buffer of ``world`` ranks is
    [world, fields, n_pad], so field f of rank j for row i is at
    (j * fields + f) * n_pad + i, i.e. split stride = fields * n_pad."""

    def __init__(self, n_cap: int, extended: bool):
        self.n_cap = n_cap
        self.n_pad = (n_cap + 3) // 4 * 4
        self.fields = 5 if extended else 3
        self.extended = extended

    @property
    def split_stride(self) -> int:
        return self.fields * self.n_pad

    def empty(self, world: int | None, device) -> torch.Tensor:
        shape = (self.fields, self.n_pad) if world is None else (world, self.fields, self.n_pad)
        return torch.empty(shape, dtype=torch.float32, device=device)

    def fields_of(self, buf: torch.Tensor) -> dict:
        """Views of the fields of a packed buffer (local [fields, n_pad] or gathered [world,
        fields, n_pad]).  A local field is its n_pad entries.  A gathered field starts at
        rank 0's field and runs to the end of the buffer: the merge reads field f of rank j
        at j * split_stride past that start (only the base pointer and the stride are passed
        on), and the view covers every entry it reads."""
        flat = buf.reshape(-1)
        gathered = buf.dim() == 3
        out = {}
        for f, name in enumerate(("m", "s", "a", "t", "m2")[:self.fields]):
            v = flat[f * self.n_pad:] if gathered else flat[f * self.n_pad:(f + 1) * self.n_pad]
            out[name] = v.view(torch.int32) if name == "a" else v
        return out


def exchange_partials(local: torch.Tensor, gathered: torch.Tensor, group=None) -> None:
    """All-gather the packed partials of every rank into ``gathered`` (rank order)."""
    import torch.distributed as dist
    dist.all_gather_into_tensor(gathered.reshape(-1), local.reshape(-1), group=group)


class VocabShardedStep:
    """Buffers and the step of one rank of a vocabulary-parallel decode step.

    ``W_shard`` passed to ``run`` must be rows [v0, v1) of W (``self.v0``, ``self.v1``).
    With world == 1 there is no collective (the local partials are merged directly).
    """

    def __init__(self, B: int, L: int, d: int, V: int, k: int, rank: int = 0, world: int = 1,
                 group=None, stats: int = 0, device="cuda"):
        from . import MAX_K, workspace_bytes
        if k < 1 or k > MAX_K:
            raise ValueError(f"k must be in [1, {MAX_K}]")
        self.B, self.L, self.d, self.V, self.k = B, L, d, V, k
        self.rank, self.world, self.group, self.stats = rank, world, group, stats
        self.v0, self.v1 = D.shard_range(V, rank, world)
        if self.v1 <= self.v0:
            raise ValueError("every rank needs at least one vocabulary row")
        self.device = torch.device(device)
        n = B * L
        i32 = dict(dtype=torch.int32, device=self.device)
        f32 = dict(dtype=torch.float32, device=self.device)
        self.layout = PartialLayout(n, extended=stats != 0)
        self.local = self.layout.empty(None, self.device)
        self.gathered = self.layout.empty(world, self.device) if world > 1 else self.local
        self.tok, self.conf, self.lse = torch.empty(n, **i32), torch.empty(n, **f32), torch.empty(n, **f32)
        self.entropy = torch.empty(n, **f32) if stats & 1 else None
        self.margin = torch.empty(n, **f32) if stats & 2 else None
        self.row_idx, self.seq_off, self.count = torch.empty(n, **i32), torch.empty(B + 1, **i32), torch.empty(4, **i32)
        self.idx, self.n_sel = torch.empty(B, k, **i32), torch.empty(B, **i32)
        self.tok_sel, self.conf_sel = torch.empty(B, k, **i32), torch.empty(B, k, **f32)
        nbytes = workspace_bytes(B, L, d, self.v1 - self.v0)
        if nbytes == 0:
            raise ValueError("invalid shapes (d must be a positive multiple of 64)")
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)

    def run(self, H, M, W_shard, win_lo=None, win_hi=None, stream=None, block_only=False) -> dict:
        from . import lse_merge, masked_partials, select_unmask
        if W_shard.shape[0] != self.v1 - self.v0:
            raise ValueError(f"W_shard must hold rows [{self.v0}, {self.v1}) of W")
        lf = self.layout.fields_of(self.local)
        masked_partials(H, M, W_shard, self.v0, self.stats, lf["m"], lf["s"], lf["a"],
                        lf.get("t"), lf.get("m2"), self.row_idx, self.seq_off, self.count,
                        self.ws, stream, *((win_lo, win_hi) if block_only else (None, None)))
        if self.world > 1:
            s = stream if stream is not None else torch.cuda.current_stream(self.device)
            with torch.cuda.stream(s):
                exchange_partials(self.local, self.gathered, self.group)
        gf = self.layout.fields_of(self.gathered)
        lse_merge(gf["m"], gf["s"], gf["a"], gf.get("t"), gf.get("m2"), self.layout.split_stride,
                  self.world, self.count, self.layout.n_cap, self.stats, self.tok, self.conf,
                  self.lse, self.entropy, self.margin, stream)
        select_unmask(self.conf, self.row_idx, self.seq_off, self.B, self.L, self.k, self.idx,
                      self.n_sel, win_lo, win_hi, self.tok, self.tok_sel, self.conf_sel, stream)
        return dict(tok=self.tok, conf=self.conf, lse=self.lse, entropy=self.entropy,
                    margin=self.margin, row_idx=self.row_idx, seq_off=self.seq_off,
                    count=self.count[:1], idx=self.idx, n_sel=self.n_sel, tok_sel=self.tok_sel,
                    conf_sel=self.conf_sel)
