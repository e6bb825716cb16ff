"""A sequence cut along T across the ranks of a process group (one GPU per rank).

Rank r holds tokens [t_r, t_{r+1}) of every sequence of the batch.  The state
crosses each rank boundary forward, S_out of rank r becoming S_in of rank r + 1.
Its gradient crosses backward, dS_in of rank r + 1 becoming dS_out of rank r.
That is the sequence-pipeline hand-off of the StateFlow pages (StateFlow
(newx.sg), Abstract; StateFlow (gptget.net), 方法详解: blocks joined by boundary
states passed from stage to stage) and of Sequence Accumulation across devices
(Sequence Accumulation, Approach), here with point-to-point sends of one
[rows, H, d_k, d_v] float32 state per micro-batch and boundary.

Micro-batches (groups of batch rows) flow through the ranks in order.  A rank
sends a micro-batch's state as soon as it has it and goes on to the next one, so
rank r computes micro-batch m + 1 while rank r + 1 computes m.  With M
micro-batches and N ranks a pass takes M + N - 1 stage times instead of M x N.

Within a rank each micro-batch runs the library's drivers that keep the
forward's intermediates (`layer.forward_keep` / `layer.backward_keep`) on the
rank's slice, cut into pieces as given.  The transport is torch.distributed
send / recv: NCCL over NVLink on GPUs.  Any backend with point-to-point works
for the host logic.
"""
from __future__ import annotations

from dataclasses import dataclass, field


def micro_rows(B: int, micro: int) -> list:
    """Batch-row ranges of `micro` micro-batches as even as possible (none empty)."""
    if not 1 <= micro <= B:
        raise ValueError(f"micro-batches must be in [1, B={B}], got {micro}")
    base, extra = divmod(B, micro)
    out, r0 = [], 0
    for m in range(micro):
        n = base + (1 if m < extra else 0)
        out.append((r0, r0 + n))
        r0 += n
    return out


class KeepRunner:
    """One rank's compute: the CUDA keep drivers on the rank's slice (the product path).

    lens: the cut of the rank's slice into pieces (its lengths must sum to the
    slice's length); or piece: cut the slice into pieces of at most `piece`
    tokens; neither: the slice is one piece.  host_states: the boundary states
    travel through host memory (pinned copies on both sides of a message), for a
    transport that carries host tensors only, such as gloo; NCCL takes the device
    tensors as they are."""

    def __init__(self, lens=None, aux_stream=None, piece=None, host_states=False):
        if lens is not None and piece is not None:
            raise ValueError("give lens or piece, not both")
        self.lens = lens
        self.piece = piece
        self.aux = aux_stream
        self.host_states = host_states

    def _cut(self, T: int):
        if self.piece is not None:
            return [min(self.piece, T - t) for t in range(0, T, self.piece)]
        return self.lens

    def state_buffer(self, rows: int, H: int, dk: int, dv: int, like):
        import torch
        if self.host_states:
            return torch.empty((rows, H, dk, dv), dtype=torch.float32, pin_memory=True)
        return torch.empty((rows, H, dk, dv), dtype=torch.float32, device=like.device)

    def _to_dev(self, s, like):
        return None if s is None else s.to(like.device, non_blocking=True).contiguous()

    def _to_msg(self, s):
        if not self.host_states:
            return s
        import torch
        h = torch.empty(s.shape, dtype=s.dtype, pin_memory=True)
        h.copy_(s)  # synchronous: the message must hold the state before it is sent
        return h

    def fwd(self, q, k, v, g, beta, S_in):
        from . import layer
        lens = self._cut(q.shape[1])
        o, S_out, kept = layer.forward_keep(q, k, v, g, beta, self._to_dev(S_in, q), lens=lens,
                                            aux_stream=self.aux)
        return o, self._to_msg(S_out), (q, k, v, g, beta, kept, lens)

    def bwd(self, ctx, dO, dS_out):
        from . import layer
        q, k, v, g, beta, kept, lens = ctx
        gr = layer.backward_keep(q, k, v, g, beta, dO, kept, dS_out=self._to_dev(dS_out, q), lens=lens,
                                 aux_stream=self.aux)
        gr["dS_in"] = self._to_msg(gr["dS_in"])
        return gr


@dataclass
class ShardContext:
    """What the forward keeps for the backward of one rank's slice."""
    rows: list
    H: int
    dk: int
    dv: int
    ctx: list = field(default_factory=list)


class SeqShard:
    """Rank `rank` of a sequence sharded along T over `group` (torch.distributed)."""

    GRADS = ("dq", "dk", "dv", "dg", "dbeta")

    def __init__(self, runner=None, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.runner = runner or KeepRunner()
        # NCCL matches point-to-point messages of a pair of ranks in issue order and
        # takes no tags; other backends get the micro-batch index as the tag
        self.tagged = dist.get_backend(group) != "nccl"

    def _tag(self, m: int) -> int:
        return m if self.tagged else 0

    def _peer(self, r: int) -> int:
        """Global rank of group rank r (send / recv take global ranks)."""
        return r if self.group is None else self.dist.get_global_rank(self.group, r)

    def forward(self, q, k, v, g=None, beta=None, S_in=None, micro: int = 1):
        """q, k, v: [B, T_r, H, d] on this rank.  S_in ([B, H, dk, dv]) is read on rank 0
        only (None: zero).  Returns (o, S_out, ctx); S_out is the sequence's final state on
        the last rank and None elsewhere."""
        import torch
        B, H, dk, dv = q.shape[0], q.shape[2], q.shape[3], v.shape[3]
        rows = micro_rows(B, micro)
        sc = ShardContext(rows, H, dk, dv)
        outs, finals, sends = [], [], []
        for m, (r0, r1) in enumerate(rows):
            if self.rank == 0:
                s_in = None if S_in is None else S_in[r0:r1].contiguous()
            else:
                s_in = self.runner.state_buffer(r1 - r0, H, dk, dv, q)
                self.dist.recv(s_in, src=self._peer(self.rank - 1), group=self.group, tag=self._tag(m))
            sl = lambda t: None if t is None else t[r0:r1]
            o, s_out, ctx = self.runner.fwd(sl(q), sl(k), sl(v), sl(g), sl(beta), s_in)
            outs.append(o)
            sc.ctx.append(ctx)
            if self.rank < self.world - 1:
                sends.append(self.dist.isend(s_out.contiguous(), dst=self._peer(self.rank + 1),
                                             group=self.group, tag=self._tag(m)))
            else:
                finals.append(s_out)
        for s in sends:
            s.wait()
        o = torch.cat(outs, 0)
        S_out = torch.cat(finals, 0) if finals else None
        return o, S_out, sc

    def backward(self, sc: ShardContext, dO, dS_out=None):
        """dO: [B, T_r, H, dv] on this rank.  dS_out ([B, H, dk, dv]) is read on the last
        rank only (None: zero).  Returns the gradients of this rank's slice; dS_in (the
        gradient of the sequence's initial state) on rank 0, None elsewhere."""
        import torch
        grads = {n: [] for n in self.GRADS}
        firsts, sends = [], []
        for m, (r0, r1) in enumerate(sc.rows):
            if self.rank == self.world - 1:
                ds_out = None if dS_out is None else dS_out[r0:r1].contiguous()
            else:
                ds_out = self.runner.state_buffer(r1 - r0, sc.H, sc.dk, sc.dv, dO)
                self.dist.recv(ds_out, src=self._peer(self.rank + 1), group=self.group, tag=self._tag(m))
            gr = self.runner.bwd(sc.ctx[m], dO[r0:r1], ds_out)
            for n in self.GRADS:
                grads[n].append(gr[n])
            if self.rank > 0:
                sends.append(self.dist.isend(gr["dS_in"].contiguous(), dst=self._peer(self.rank - 1),
                                             group=self.group, tag=self._tag(m)))
            else:
                firsts.append(gr["dS_in"])
        for s in sends:
            s.wait()
        out = {n: (None if v[0] is None else torch.cat(v, 0)) for n, v in grads.items()}
        out["dS_in"] = torch.cat(firsts, 0) if firsts else None
        return out
