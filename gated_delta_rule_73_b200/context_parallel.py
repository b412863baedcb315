"""Context parallelism over T: one long sequence split over the ranks of a process group.

Page "Kimi K3 の KDA(1)", section 2.3 (the algebraic view of the recurrence): a segment of
tokens acts on the state as one affine pair S -> M S + B, and pairs compose in order, so
rank r only needs the pairs of segments 0..r-1 to know the state its own segment starts
from.  Per call, every rank

  1. computes its segment's pair (M_r, B_r) with ``kda_segment_pair``   (one prep pass, two
     scans over its records),
  2. all-gathers the pairs of all ranks                                  (the one exchange),
  3. folds pairs 0..r-1 onto the sequence's start state S0 with ``kda_affine_combine``,
  4. runs ``kda_segment_forward`` over its segment from that state       (a third scan over
     the same records), and
  5. folds all pairs onto S0 for the final state of the whole sequence.

Only step 2 crosses ranks (2 x 64 KiB per head and rank at d = 128, FP32).  The arithmetic
runs in the library's kernels; torch provides the buffers and ``torch.distributed`` the
all-gather (NCCL on GPUs).  ``ops`` can replace the three library calls (the CPU tests of
the exchange pass their own), nothing else changes with it.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The library calls the context-parallel forward is built from.  The segment's workspace
    (its chunk records) is kept from ``segment_pair`` for ``segment_forward``."""

    def __init__(self, **flags):
        self.flags = flags
        self.workspace = None

    def segment_pair(self, q, k, v, g, beta):
        from . import kda
        B, T, H, dk = q.shape
        opts = kda.make_opts(q.dtype, **{n: f for n, f in self.flags.items() if n != "scale"})
        nbytes = kda.kda_segment_pair_workspace_bytes(B, T, H, dk, v.shape[-1], opts)
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
        return kda.segment_pair(q, k, v, g, beta, workspace=self.workspace,
                                **{n: f for n, f in self.flags.items() if n != "scale"})

    def segment_forward(self, q, k, v, g, beta, S0):
        from . import kda
        return kda.segment_forward(q, k, v, g, beta, S0, self.workspace, **self.flags)

    def affine_combine(self, Ms, Bs, n, S0):
        from . import kda
        return kda.affine_combine(Ms, Bs, n, S0)

    def chunk_fwd(self, q, k, v, g, beta, S0):
        from . import kda
        return kda.chunk_fwd(q, k, v, g, beta, S0, **self.flags)


def _all_gather(x, group):
    world = dist.get_world_size(group)
    parts = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.stack(parts)


def chunk_fwd_context_parallel(q, k, v, g, beta, S0=None, *, group=None, ops=None, **flags):
    """Forward over one sequence split over the ranks of ``group``, in rank order.

    Rank r holds tokens [r*T_seg, (r+1)*T_seg) of every sequence as q, k, g [B,T_seg,H,dk],
    v [B,T_seg,H,dv], beta [B,T_seg,H] (segments may differ in length).  ``S0``
    [B,H,dk,dv] FP32 (or None = zero) is the state before the first segment and must be the
    same on every rank.  Returns (out of this rank's segment, the whole sequence's final
    state, the state this segment started from).  ``flags``: the options of ``chunk_fwd``
    (l2norm, complex_gate, unbounded, ...), applied to every step.
    """
    ops = ops or LibraryOps(**flags)
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    M, Bm = ops.segment_pair(q, k, v, g, beta)
    Ms = _all_gather(M, group)                       # [R, B, H, dk, dk]
    Bs = _all_gather(Bm, group)                      # [R, B, H, dk, dv]
    S_start = ops.affine_combine(Ms, Bs, rank, S0)
    out, _ = ops.segment_forward(q, k, v, g, beta, S_start)
    S_T = ops.affine_combine(Ms, Bs, world, S0)
    return out, S_T, S_start
