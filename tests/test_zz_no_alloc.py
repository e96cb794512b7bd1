"""The no-allocation SR transpose entry point (nvfp4_sr_transpose_requant_noalloc).

It exists for callers that cannot allocate device memory when they call this
library -- an engine that handed all of HBM to its own pools at start-up, or C
code without an allocator that must not trigger the device synchronisation of
cudaMalloc/cudaFree mid-step -- and therefore cannot pass a scratch buffer.  It
must give exactly what the allocating entry point gives.  This file is
collected last on purpose, and each test also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _lib():
    from train_rollout_alignment_b200 import _binding
    return _binding


def _stack(batch, rows, cols, seed):
    """A quantized [batch, rows, cols] stack made on the GPU by the library's
    own round-to-nearest path (both entry points get the same input)."""
    b = _lib()
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    codes = torch.empty(batch * rows * cols // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(batch * rows * cols // 16, dtype=torch.uint8, device="cuda")
    ts = torch.empty(batch, dtype=torch.float32, device="cuda")
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    n = rows * cols
    for e in range(batch):
        x = (torch.randn(rows, cols, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        b.nvfp4_quantize_rtn(x, ws, codes[e * n // 2:(e + 1) * n // 2],
                             scales[e * n // 16:(e + 1) * n // 16], ts[e:e + 1])
    return codes, scales, ts


def _outputs(batch, rows, cols):
    n = batch * rows * cols
    return (torch.full((n // 2,), 0xAB, dtype=torch.uint8, device="cuda"),
            torch.full((n // 16,), 0xAB, dtype=torch.uint8, device="cuda"),
            torch.full((batch,), -1.0, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("shape", [(3, 64, 192), (9, 80, 48)])
def test_noalloc_matches_allocating_entry_point_twice(shape):
    b = _lib()
    batch, rows, cols = shape
    codes, scales, ts = _stack(batch, rows, cols, seed=batch)
    ws = torch.zeros(batch, dtype=torch.int32, device="cuda")
    for draw in (0, 7):  # two calls in a row: the shared array keeps the last call's words
        ref = _outputs(batch, rows, cols)
        b.nvfp4_sr_transpose_requant(codes, scales, ts, batch, rows, cols, 2, draw, ws, *ref)
        got = _outputs(batch, rows, cols)
        b.nvfp4_sr_transpose_requant_noalloc(codes, scales, ts, batch, rows, cols, 2, draw, *got)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g)


def test_noalloc_at_the_batch_limit_and_beyond():
    b = _lib()
    rows, cols = 16, 16
    batch = b.NVFP4_SR_NOALLOC_MAX_BATCH
    codes, scales, ts = _stack(1, rows, cols, seed=1)
    codes = codes.repeat(batch)
    scales = scales.repeat(batch)
    ts = ts.repeat(batch)
    ws = torch.zeros(batch, dtype=torch.int32, device="cuda")
    ref = _outputs(batch, rows, cols)
    got = _outputs(batch, rows, cols)
    b.nvfp4_sr_transpose_requant(codes, scales, ts, batch, rows, cols, 5, 1, ws, *ref)
    b.nvfp4_sr_transpose_requant_noalloc(codes, scales, ts, batch, rows, cols, 5, 1, *got)
    torch.cuda.synchronize()
    for r, g in zip(ref, got):
        assert torch.equal(r, g)
    over = _outputs(batch + 1, rows, cols)
    with pytest.raises(b.Nvfp4Error) as ei:
        b.nvfp4_sr_transpose_requant_noalloc(torch.cat([codes, codes[:rows * cols // 2]]),
                                             torch.cat([scales, scales[:rows * cols // 16]]),
                                             torch.cat([ts, ts[:1]]), batch + 1, rows, cols, 5, 1, *over)
    assert ei.value.status == b.NVFP4_ERR_SCRATCH_LIMIT
    assert "no-allocation" in str(ei.value)
    torch.cuda.synchronize()
    assert torch.all(over[0] == 0xAB) and torch.all(over[2] == -1.0)
