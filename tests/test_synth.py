"""The seeded generators: determinism, shapes, dtypes and value structure."""
import numpy as np
import torch

import synth


def test_tiny_deterministic_and_shaped():
    cfg = synth.CONFIGS["tiny"]
    a = synth.make_inputs(cfg)
    b = synth.make_inputs(cfg)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    q, k, v, sq, sk = a
    assert q.shape == (1, 2, 128, 64) and q.dtype == torch.float32
    assert sq.shape == (2,) and (sq > 0).all()


def test_vit_offset_biases_signs():
    cfg = synth.CONFIGS["vit"]
    q, k, v, sq, sk = synth.make_inputs(cfg, B=2)
    assert q.dtype == torch.bfloat16 and q.shape == (2, 12, 197, 64)
    frac_pos = (q.float() >= 0).float().mean().item()
    assert 0.59 < frac_pos < 0.65          # P(N(0.3,1) >= 0) ~= 0.618


def test_lowrank_signal_shared_between_q_and_k():
    cfg = synth.CONFIGS["bert"]
    q, k, v, sq, sk = synth.make_inputs(cfg, B=1)
    qf, kf = q.float(), k.float()
    corr = (qf * kf).mean() / (qf.std() * kf.std())
    assert corr > 0.7                       # signal variance 1 vs noise 0.25


def test_sigma_is_population_std_per_head():
    x = torch.randn(3, 4, 10, 64, generator=torch.Generator().manual_seed(0))
    s = synth.per_head_sigma(x)
    for h in range(4):
        ref = np.std(x[:, h].double().numpy())
        assert abs(s[h].item() - ref) < 1e-6


def test_sample_rows_cover_ends():
    cfg = synth.CONFIGS["long"]
    r = synth.sample_rows(cfg, 50)
    assert r[0] == 0 and r[-1] == cfg.rows - 1 and len(np.unique(r)) == len(r)
