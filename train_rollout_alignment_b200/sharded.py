"""One tensor's rows split across the ranks of a process group.

The tensor scale needs the whole tensor's amax ("Thinking Machines Lab
releases 4-bit training", forward/backward mismatch paragraph: values that
share a scale are scaled by their group's maximum), so row-sharded
quantization has exactly one exchange:
every rank reduces its own rows' amax on the GPU (nvfp4_tensor_amax), the
group takes the MAX of those scratch words (one 8-byte all-reduce), and each
rank then quantizes its rows with NVFP4_AMAX_PRECOMPUTED.  Every 16-value
block depends only on its own values and that shared amax, so each rank's
codes, scales and hints are bit for bit the rows of the unsharded result.
The train side's guidance and mismatch counters are sums over blocks: a SUM
all-reduce of the counter words gives the whole tensor's counts.

Scratch words: ws[0] holds the FP32 bits of a non-negative amax, which order
like the integers they spell, and ws[1]'s warning bits are 0/1 flags, so an
integer MAX over ws[0:2] is the float max and the OR.

Layers (or experts) split across ranks need none of this; the benchmark's
weak scaling does that.  `lib` defaults to the C-ABI binding; every step runs
in its kernels, the collectives in torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

import torch.distributed as dist


def _lib(lib):
    if lib is not None:
        return lib
    from . import _binding
    return _binding


def _grouped(group) -> bool:
    return dist.is_initialized() and dist.get_world_size(group) > 1


def shared_amax(x_shard, ws, group=None, lib=None) -> None:
    """ws[0] <- bits of max |x| over the whole sharded tensor; ws[1] <- the
    OR of every rank's warning bits."""
    b = _lib(lib)
    b.nvfp4_tensor_amax(x_shard, ws)
    if _grouped(group):
        dist.all_reduce(ws[:2], op=dist.ReduceOp.MAX, group=group)


def quantize_rtn(x_shard, ws, codes, scales, tensor_scale, hints=None, hint_bits=0, group=None,
                 lib=None) -> None:
    """Rollout side on this rank's rows: round-to-nearest NVFP4 with the
    tensor scale of the whole tensor (and the rows' hints when requested)."""
    b = _lib(lib)
    shared_amax(x_shard, ws, group, b)
    b.nvfp4_quantize_rtn(x_shard, ws, codes, scales, tensor_scale, hints, hint_bits,
                         flags=b.NVFP4_AMAX_PRECOMPUTED)


def guided_requant(x_shard, hints, hint_bits, ws, codes, scales, tensor_scale, stats4=None,
                   group=None, lib=None) -> None:
    """Train side on this rank's rows, guided by the same rows' hints.  stats4
    must hold zeros on every rank on entry; on return every rank holds the
    whole tensor's counters (words 0..2)."""
    b = _lib(lib)
    shared_amax(x_shard, ws, group, b)
    b.nvfp4_guided_requant(x_shard, hints, hint_bits, ws, codes, scales, tensor_scale, stats4,
                           flags=b.NVFP4_AMAX_PRECOMPUTED)
    if stats4 is not None and _grouped(group):
        dist.all_reduce(stats4[:3], op=dist.ReduceOp.SUM, group=group)


def mismatch_stats(codes_a, scales_a, ts_a, codes_b, scales_b, ts_b, rows_shard, cols, stats8,
                   group=None, lib=None) -> None:
    """Counters between the two sides' NVFP4 rows of this rank, summed over the
    group.  stats8 must hold zeros on every rank on entry (words 0..6 are
    summed; word 7 is reserved and left alone)."""
    b = _lib(lib)
    b.nvfp4_mismatch_stats(codes_a, scales_a, ts_a, codes_b, scales_b, ts_b, rows_shard, cols, stats8)
    if _grouped(group):
        dist.all_reduce(stats8[:7], op=dist.ReduceOp.SUM, group=group)
