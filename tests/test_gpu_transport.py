"""Hint transport through the C ABI (nvfp4_hint_pack): the hint streams of
several tensors gathered into one staging buffer and copied to pinned host
memory must be the oracle's hints of each tensor, back to back on 16-byte
boundaries with zero padding (TRACE explainer, guidance-volume and
compaction paragraphs: the back-half layers' low code bits leave the GPU
every step)."""
import numpy as np
import pytest
import torch

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import dev_bf16, lib

pytestmark = pytest.mark.gpu


def _expected(parts):
    out = []
    for p in parts:
        out.append(p)
        pad = (-p.size) % 16
        out.append(np.zeros(pad, np.uint8))
    return np.concatenate(out) if out else np.zeros(0, np.uint8)


def _layers(specs, seed):
    """Device hint streams made by the library's quantizer, and the oracle's."""
    b = lib()
    dev, want = [], []
    for i, (rows, cols, bits) in enumerate(specs):
        x = syn.random_case((rows, cols), seed + i, "heavy")
        codes, scales, ts, ws, hints = b.empty_nvfp4(rows, cols, "cuda", hint_bits=bits)
        b.nvfp4_quantize_rtn(dev_bf16(x), ws, codes, scales, ts, hints, bits)
        dev.append(hints)
        want.append(oracle.quantize_rtn(x, hint_bits=bits)[3])
    return dev, want


@pytest.mark.parametrize("specs", [
    [(3, 16, 2), (64, 256, 1), (37, 528, 2), (128, 1024, 4), (1, 16, 1)],
    [(256, 4096, 2)] * 6,
])
def test_pack_to_pinned_host_matches_oracle_hints(specs):
    b = lib()
    dev, want = _layers(specs, 900)
    total = b.nvfp4_hint_pack_size([t.numel() for t in dev])
    expect = _expected(want)
    assert total == expect.size
    staging = torch.full((total,), 0xAB, dtype=torch.uint8, device="cuda")
    host = torch.full((total,), 0xCD, dtype=torch.uint8).pin_memory()
    b.nvfp4_hint_pack(dev, staging, host)
    torch.cuda.synchronize()
    assert np.array_equal(host.numpy(), expect)
    assert np.array_equal(staging.cpu().numpy(), expect)


def test_pack_more_streams_than_one_launch_takes():
    """300 streams (one launch takes 128), some empty, staging only."""
    b = lib()
    rng = np.random.default_rng(3)
    parts = [rng.integers(0, 256, int(n), dtype=np.uint8) for n in rng.integers(0, 70, 300)]
    dev = [torch.from_numpy(p).cuda() if p.size else torch.empty(0, dtype=torch.uint8, device="cuda")
           for p in parts]
    expect = _expected(parts)
    staging = torch.full((expect.size,), 0xAB, dtype=torch.uint8, device="cuda")
    b.nvfp4_hint_pack(dev, staging)
    torch.cuda.synchronize()
    assert np.array_equal(staging.cpu().numpy(), expect)
    host = torch.empty(expect.size, dtype=torch.uint8).pin_memory()
    b.nvfp4_hint_pack(dev, staging, host)
    torch.cuda.synchronize()
    assert np.array_equal(host.numpy(), expect)


def test_pack_rejects_bad_streams_and_writes_nothing():
    b = lib()
    base = torch.zeros(64, dtype=torch.uint8, device="cuda")
    staging = torch.full((64,), 0xAB, dtype=torch.uint8, device="cuda")
    with pytest.raises(b.Nvfp4Error) as ei:
        b.nvfp4_hint_pack([base[:16], base[8:24]], staging)      # second stream not 16-byte aligned
    assert ei.value.status == 2
    torch.cuda.synchronize()
    assert torch.all(staging == 0xAB)
