"""Head-sharded per-layer step: the heads of a layer spread over the ranks of a
process group, one GPU per rank.

Every quantity of the step is per head except the page score of the retrieval,
which sums over heads.  Each rank therefore holds its heads' slices of the pages,
of Q / Kq / Vq, tau and the gate logits (E and F are shared by the heads and
replicated), computes its heads' partial page scores, and the ranks add them with
one all-reduce of NP floats; from there on (top-Kp, gather, block selection, both
branches, merge) every rank works on its own heads with no further exchange.
Argument marshalling and the all-reduce only; the arithmetic runs in the library.
"""
from __future__ import annotations

from . import hkv_page_scores, hkv_select_top
from .step import HkvHsaStep


def sharded_retrieval(partial_scores, all_reduce_sum, select_top):
    """The retrieval of a head-sharded step: this rank's partial page scores (a
    tensor), summed in place over the ranks, then ranked.  In a step the three
    callables are hkv_page_scores, torch.distributed.all_reduce and hkv_select_top."""
    scores = partial_scores()
    all_reduce_sum(scores)
    return select_top(scores)


def head_range(H: int, rank: int, world: int):
    """Heads [h0, h1) of `rank` when H heads are split as evenly as possible."""
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


class HeadShardedStep(HkvHsaStep):
    """HkvHsaStep over this rank's heads, with the page retrieval summed over the
    ranks of `group` (torch.distributed, NCCL on GPUs)."""

    def __init__(self, group, *args, **kw):
        super().__init__(*args, **kw)
        self.group = group

    def _retrieve(self, Q, cand):
        import torch.distributed as dist

        def partial():
            hkv_page_scores(self.kbar_pages, Q, self.scores, self.ws, cand)
            return self.scores

        def select(s):
            hkv_select_top(s, self.Kp, self.sel, self.ws, cand)
            return self.sel

        return sharded_retrieval(partial, lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group),
                                 select)
