"""Ulysses sequence parallelism for one streaming session across ranks.

Source: "StreamRender-H3" (molayo1419.me), inference acceleration section:
the model runs on several GPUs with Ulysses context parallelism, i.e. every
rank holds a slice of the sequence for all heads outside attention, and one
all-to-all before attention re-partitions the chunk's Q, K and V by heads
(every rank then sees the whole sequence for its heads), one all-to-all after
it returns O to the sequence partition.  "MiniMax-H3 deep dive" (fiv.co.kr),
transformer config table: 56 heads, i.e. 7 per GPU at 8-way Ulysses; the head
count must be a multiple of the rank count.

Readings (the pages leave them open):
  * the chunk's L tokens are cut into world equal slices of S = ceil(L/world)
    tokens (rank r holds tokens [r*S, min((r+1)*S, L))); the last slice is
    padded with rows that no query or key ever sees (the valid lengths stop
    at L);
  * the persistent window (prompt, sink, tiers, recent) is kept sharded by
    heads, each rank the KV of its own heads, so only the chunk crosses the
    links: the window's history is produced head-sharded by the exchange of
    earlier chunks;
  * head group j of rank r is heads [j*Hn, (j+1)*Hn), Hn = H / world.

Per step, on every rank:
  pack    q, k, v [S, H, D] -> send [world, S, 3, Hn, D]  (slot j: head group j)
  a2a     recv[j] = send_j[r]: tokens of rank j for this rank's heads, so recv
          viewed [world*S, 3, Hn, D] is the whole chunk, token-major
  window  a2 -> a3 -> a4 of ``StreamingWindow`` on the Hn local heads, O into
          the send buffer [world*S, Hn, D]
  a2a     back: recv_o[j] = O of head group j for this rank's tokens
  unpack  recv_o [world, S, Hn, D] -> out [S, H, D]
The pack and unpack are layout copies done by the library's index gather
and scatter (sr_gather_tokens: one launch per tensor; sr_scatter_tokens: one
launch), with a fixed index table: slot (j, t) of the send buffer is token t
of head group j, i.e. row t * world + j of the rank's [n, H, D] tokens viewed
as [n * world, Hn, D].  The exchanges are NCCL all-to-alls over NVLink
(``torch.distributed.all_to_all_single``).  The phases are separate methods
so that a test can run several ranks in one process; ranks on the CPU (the
multi-process tests over gloo) re-lay out with torch copies instead.
"""
from __future__ import annotations

import dataclasses
import math
from types import SimpleNamespace
from typing import Optional

import torch

from .window import StreamingWindow


@dataclasses.dataclass(frozen=True)
class UlyssesPlan:
    """Token and head partition of one session over `world` ranks."""
    n_tokens: int
    n_heads: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.n_heads % self.world:
            raise ValueError(f"{self.n_heads} heads cannot be split over {self.world} ranks")

    @property
    def slice_tokens(self) -> int:           # S
        return max(1, math.ceil(self.n_tokens / self.world))

    @property
    def local_heads(self) -> int:            # Hn
        return self.n_heads // self.world

    def tokens_of(self, rank: int):
        """[lo, hi) of the valid tokens rank `rank` holds (may be empty)."""
        S = self.slice_tokens
        return min(rank * S, self.n_tokens), min((rank + 1) * S, self.n_tokens)

    def heads_of(self, rank: int):
        return rank * self.local_heads, (rank + 1) * self.local_heads


def head_slice(inp, lo: int, hi: int):
    """The window inputs (prompt_k/v, ctx_k/v lists, q, k, v; token-major
    [L, H, D]) restricted to heads [lo, hi)."""
    return SimpleNamespace(prompt_k=inp.prompt_k[:, lo:hi], prompt_v=inp.prompt_v[:, lo:hi],
                           ctx_k=[t[:, lo:hi] for t in inp.ctx_k], ctx_v=[t[:, lo:hi] for t in inp.ctx_v],
                           q=inp.q[:, lo:hi], k=inp.k[:, lo:hi], v=inp.v[:, lo:hi])


class UlyssesAttention:
    """The streaming attention step of one session with its chunk sharded by
    tokens over the ranks of `group` (see the module docstring).

    ``window`` replaces the local head-sharded ``StreamingWindow`` (anything
    with ``load_window``, ``step(q, k, v, out=...)``; used by host-only tests)."""

    def __init__(self, spec, rank: int, world: int, group=None, device="cuda", qk_norm=None, window=None):
        self.spec, self.rank, self.world, self.group = spec, rank, world, group
        self.plan = UlyssesPlan(int(spec.chunk_video_tokens) + int(spec.chunk_audio_tokens),
                                int(spec.n_heads), world)
        self.H, self.D = int(spec.n_heads), int(spec.head_dim)
        self.Hn, self.S = self.plan.local_heads, self.plan.slice_tokens
        self.device = torch.device(device)
        if window is None:
            window = StreamingWindow([dataclasses.replace(spec, n_heads=self.Hn)], device=self.device,
                                     qk_norm=qk_norm)
        self.win = window
        N, S, Hn, D = world, self.S, self.Hn, self.D
        kw = dict(dtype=torch.bfloat16, device=self.device)
        self.send = torch.zeros(N, S, 3, Hn, D, **kw)
        self.recv = torch.zeros(N, S, 3, Hn, D, **kw)
        self.o_send = torch.zeros(N * S, Hn, D, **kw)
        self.o_recv = torch.zeros(N, S, Hn, D, **kw)
        # slot (head group j, token t) <-> row t * world + j of the tokens viewed
        # [n * world, Hn, D]; slots past this rank's n tokens: -1 (zero / skipped)
        lo, hi = self.plan.tokens_of(rank)
        t = torch.arange(S, dtype=torch.int64)
        idx = t[None, :] * N + torch.arange(N, dtype=torch.int64)[:, None]
        idx[:, hi - lo:] = -1
        self.idx = idx.to(torch.int32).contiguous().to(self.device)

    # ------------------------------------------------------------ phases
    def load_window(self, inp) -> None:
        """Window inputs of the session (all heads); this rank keeps its heads."""
        self.win.load_window([head_slice(inp, *self.plan.heads_of(self.rank))])

    def pack(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
        """q, k, v: this rank's tokens [n, H, D] (n <= S; the rest of the
        slice stays zero) -> the send buffer."""
        n = q.shape[0]
        lo, hi = self.plan.tokens_of(self.rank)
        if n != hi - lo:
            raise ValueError(f"rank {self.rank} holds {hi - lo} tokens, got {n}")
        if self.device.type == "cuda":
            from . import capi
            for c, x in enumerate((q, k, v)):
                capi.sr_gather_tokens(self.send[:, :, c], x.reshape(n * self.world, self.Hn, self.D), self.idx)
        else:   # CPU ranks of the multi-process tests
            for c, x in enumerate((q, k, v)):
                self.send[:, :n, c].copy_(x.view(n, self.world, self.Hn, self.D).transpose(0, 1))
        return self.send

    def attend(self, marks=None) -> torch.Tensor:
        """The window step on the received whole chunk (local heads); O lands
        in the send buffer of the return exchange.  `marks`: optional pair of
        CUDA events recorded around the attention launch."""
        L = self.plan.n_tokens
        full = self.recv.view(self.world * self.S, 3, self.Hn, self.D)[:L]
        q, k, v = (full[:, c][None] for c in range(3))
        if marks is None:
            self.win.step(q, k, v, out=self.o_send[:L][None])
        else:
            self.win.step(q, k, v, out=self.o_send[:L][None], marks=marks)
        return self.o_send

    def unpack(self, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """O of this rank's tokens for all heads, [n, H, D]."""
        lo, hi = self.plan.tokens_of(self.rank)
        n = hi - lo
        if out is None:
            out = torch.empty(n, self.H, self.D, dtype=torch.bfloat16, device=self.device)
        if self.device.type == "cuda":
            from . import capi
            capi.sr_scatter_tokens(out.view(n * self.world, self.Hn, self.D), self.o_recv, self.idx)
        else:   # CPU ranks of the multi-process tests
            out.view(n, self.world, self.Hn, self.D).copy_(self.o_recv[:, :n].transpose(0, 1))
        return out

    # ------------------------------------------------------------ the step
    def step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
             marks=None):
        """q, k, v: this rank's chunk tokens [n, H, D] before RoPE -> O [n, H, D]."""
        import torch.distributed as dist
        self.pack(q, k, v)
        dist.all_to_all_single(self.recv, self.send, group=self.group)
        self.attend(marks)
        dist.all_to_all_single(self.o_recv, self.o_send.view(self.world, self.S, self.Hn, self.D),
                               group=self.group)
        return self.unpack(out)


def exchange_in_process(ranks) -> None:
    """The all-to-all of the chunk among rank objects living in one process
    (one device): recv_r[j] = send_j[r].  For tests that run several ranks'
    kernels in sequence on one GPU (no kernel waits on another)."""
    for r, a in enumerate(ranks):
        for j, b in enumerate(ranks):
            a.recv[j].copy_(b.send[r])


def exchange_back_in_process(ranks) -> None:
    for r, a in enumerate(ranks):
        for j, b in enumerate(ranks):
            a.o_recv[j].copy_(b.o_send.view(b.world, b.S, b.Hn, b.D)[r])
