"""Data-parallel amax exchange for delayed-scaling rings (torch.distributed).

In data-parallel training every replica quantizes its own micro-batch, so
each ring would see only its rank's amax and the replicas' scales would drift
apart. The exchange keeps them identical: the step's quantizes run with
FP8_QUANTIZE_DEFER_FOLD (each ring keeps the call's amax in its accumulator),
the ranks all-reduce those 4-byte words with MAX, and one fp8_rings_fold
launch folds the group's amax into every ring. Non-negative fp32 values order
like their bit patterns read as integers, so the MAX runs on int32 words and
returns the bits of the largest amax exactly.

The all-reduce is torch.distributed's (NCCL on GPUs, gloo on CPU); this
module only gathers the words and hands them over -- the fold is the
library's kernel.
"""

import torch
import torch.distributed as dist

from . import FP8_RING_BYTES, fp8_rings_fold

RING_WORDS = FP8_RING_BYTES // 4
AMAX_WORD = 18  # int32 index of the accumulator: hist[16], scale, idx, amax_bits, ticket


def allreduce_amax(rings: torch.Tensor, group=None) -> None:
    """rings: int32 [R, 20], R consecutive rings. Replaces each ring's
    accumulated amax by the group's maximum (one all-reduce of R words)."""
    if rings.dtype != torch.int32 or rings.dim() != 2 or rings.shape[1] != RING_WORDS:
        raise ValueError("rings must be an int32 tensor of shape [R, 20]")
    words = rings[:, AMAX_WORD].contiguous()
    dist.all_reduce(words, op=dist.ReduceOp.MAX, group=group)
    rings[:, AMAX_WORD].copy_(words)


def allreduce_amax_and_fold(rings: torch.Tensor, fmts, group=None, stream=None) -> None:
    """The whole exchange after a step's deferred quantizes: all-reduce the
    R amax words, then fold them into the R rings (device tensor)."""
    allreduce_amax(rings, group)
    fp8_rings_fold(rings, rings.shape[0], fmts, stream)
