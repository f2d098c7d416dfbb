"""The seeded input generator: deterministic, the stated shapes and structure."""
import torch

import synth


def test_deterministic_and_seed_sensitive():
    a = synth.activations(16, 512, seed=0, outliers=[7, 300], factor=20.0)
    b = synth.activations(16, 512, seed=0, outliers=[7, 300], factor=20.0)
    c = synth.activations(16, 512, seed=1, outliers=[7, 300], factor=20.0)
    assert a.dtype == torch.bfloat16 and a.shape == (16, 512)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_outlier_channels_are_scaled():
    base = synth.activations(64, 512, seed=0)
    out = synth.activations(64, 512, seed=0, outliers=[7, 300], factor=20.0)
    f = out.float() / base.float().where(base.float() != 0, torch.ones(()))
    assert torch.allclose(f[:, 7].median(), torch.tensor(20.0), rtol=0.02)
    untouched = torch.ones(512, dtype=torch.bool)
    untouched[[7, 300]] = False
    assert torch.equal(out[:, untouched].view(torch.int16), base[:, untouched].view(torch.int16))


def test_outlier_channel_choice():
    ch = synth.outlier_channels(7168, synth.n_outliers(7168, 0.005), seed=0)
    assert ch.numel() == 36 and ch.unique().numel() == 36 and int(ch.max()) < 7168
    assert synth.n_outliers(8192, 0.01) == 82


def test_weight_std():
    w = synth.weights(512, 512, 0.02, seed=0).float()
    assert abs(w.std().item() - 0.02) < 0.0005


def test_student_t3_is_heavy_tailed():
    x = synth.activations(256, 1024, seed=0, dist="t3").float()
    # t(3) has variance 3 and far more mass beyond 6 sigma than a normal
    assert 2.0 < x.var().item() < 4.5
    assert (x.abs() > 6).float().mean().item() > 1e-3


def test_routing_structure():
    T, E, k = 4096, 256, 8
    row_token, row_expert, off = synth.routing(T, E, k, seed=0)
    assert row_token.numel() == T * k and off[0] == 0 and off[-1] == T * k
    assert (off[1:] >= off[:-1]).all()
    # sorted by expert, then by token within an expert
    assert (row_expert[1:] >= row_expert[:-1]).all()
    for e in [0, 17, 255]:
        seg = row_token[off[e]:off[e + 1]]
        assert (seg[1:] > seg[:-1]).all()
        assert (row_expert[off[e]:off[e + 1]] == e).all()
    # each token appears exactly k times, with k distinct experts
    assert torch.equal(torch.bincount(row_token, minlength=T), torch.full((T,), k))
    pairs = row_token * E + row_expert
    assert pairs.unique().numel() == T * k
    counts = off[1:] - off[:-1]
    assert 90 < counts.float().mean().item() < 170 and int(counts.max()) < 256
    r2 = synth.routing(T, E, k, seed=0)
    assert torch.equal(r2[0], row_token) and torch.equal(r2[2], off)
