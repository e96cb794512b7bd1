"""The seeded input generators (no quantization arithmetic in them): the
device generator of the MoE activation stack has the distribution the host
generator of the parity tests has (Student-t, nu = 4, variance nu / (nu - 2)
= 2; 16 outlier channels x50; rollout copy within 2^-8 relative noise)."""
import numpy as np
import torch

from train_rollout_alignment_b200 import synthetic as syn


def test_moe_stack_device_generator_matches_the_host_distribution():
    xt, xr = syn.cfg1_layer_device(3, "cpu", shape=(2048, 512))
    x = xt.float().numpy()
    col_rms = np.sqrt(np.mean(x * x, axis=0))
    out = np.argsort(col_rms)[-16:]
    rest = np.setdiff1d(np.arange(512), out)
    assert np.min(col_rms[out]) > 20 * np.max(np.median(col_rms[rest]))  # 16 channels x50
    v = x[:, rest]
    assert abs(np.var(v) - 2.0) < 0.25                                   # nu / (nu - 2)
    kurt = np.mean(v ** 4) / np.var(v) ** 2
    assert kurt > 6.0                                                    # heavy tails (normal: 3)
    h = syn.cfg1_layer(3)[0][:2048, :512]
    assert abs(np.var(syn.bf16_to_f32(h)[:, np.setdiff1d(np.arange(512), np.argsort(
        np.sqrt(np.mean(syn.bf16_to_f32(h) ** 2, axis=0)))[-16:])]) - 2.0) < 0.35
    rel = (xr.float() / torch.where(xt.float() == 0, torch.ones_like(xt.float()), xt.float()) - 1).numpy()
    assert abs(np.std(rel[xt.float().numpy() != 0]) - 2.0 ** -8) < 2.0 ** -10
