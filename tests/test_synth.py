"""The seeded input recipe (host only): the properties the workloads are stated to have.

The Llama-2-7B-shaped layer set is fp32 from a bf16 N(0, 0.02) body plus binary32 t(3)
outliers: the body entries are bf16 values, the outliers in general are not.  The other
checks pin the recipe's shapes, fractions and ranges, and that a seed always gives the
same bytes.
"""
import numpy as np
import torch

from post_weight_quantization_rowwise_b200 import synth


def test_same_seed_same_bytes_and_different_seeds_differ():
    a = synth.weight_matrix(16, 256, seed=5)
    assert torch.equal(a, synth.weight_matrix(16, 256, seed=5))
    assert not torch.equal(a, synth.weight_matrix(16, 256, seed=6))
    assert torch.equal(synth.imatrix(256, seed=1), synth.imatrix(256, seed=1))
    assert torch.equal(synth.activations(2, 256, seed=2), synth.activations(2, 256, seed=2))


def test_bf16_body_with_binary32_outliers():
    x = synth.weight_matrix(256, 4096, seed=3000, bf16=True)
    y = synth.weight_matrix(256, 4096, seed=3000, bf16=False)
    out = x != y.to(torch.bfloat16).to(torch.float32)
    # the outliers (0.2 * t(3)) are there, at the same places and with the same binary32
    # values as without the rounding: N(0, 0.02) alone stays far below 0.15
    big = (x.abs() > 0.15).sum().item()
    assert 0.0002 * x.numel() < big < 0.002 * x.numel()
    assert torch.equal(x[out], y[out])
    assert 0.0005 * x.numel() < out.sum().item() < 0.0015 * x.numel()
    # every other entry is a bf16 value; most outliers are not
    body = ~out
    assert torch.equal(x[body].to(torch.bfloat16).to(torch.float32), x[body])
    assert (x[out].to(torch.bfloat16).to(torch.float32) != x[out]).float().mean() > 0.9
    t = synth.llama2_7b_layer_set(1)
    assert [(u.rows, u.cols) for u in t] == [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    assert all(u.bf16 for u in t)


def test_outlier_fraction_and_body():
    x = synth.weight_matrix(512, 4096, seed=11).numpy().astype(np.float64)
    body = x[np.abs(x) < 0.1]
    assert abs(body.std() - 0.02) < 0.001
    # Bernoulli(1e-3) outliers of scale 0.2 * t(3): about 1 in 1000 entries beyond 4 sigma
    assert 0.0004 < np.mean(np.abs(x) > 0.08) < 0.0012


def test_imatrix_log_normal_and_boost():
    qw = synth.imatrix(1 << 16, seed=4).numpy().astype(np.float64)
    assert (qw > 0).all()
    assert abs(np.log(qw).mean()) < 0.02 and abs(np.log(qw).std() - 1.0) < 0.02
    qb = synth.imatrix(1 << 16, seed=4, boost_frac=0.05).numpy()
    boosted = np.sum(~np.isclose(qb, qw.astype(np.float32)))
    assert boosted == round(0.05 * (1 << 16))


def test_activation_spikes_beyond_fp16():
    a = synth.activations(64, 7168, seed=2, spike_frac=1e-3).numpy()
    spikes = np.abs(a) > 6e4
    assert 0.0005 < spikes.mean() < 0.0015
    assert np.abs(a[spikes]).max() <= 2e5 and np.abs(a[~spikes]).max() < 10
    assert (a[spikes] > 0).any() and (a[spikes] < 0).any()
