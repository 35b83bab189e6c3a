"""The affine fit's checkpoint: (A, b) of a layer's linear stage written to and read from .npz.

Host only: a HybridLayer with CPU buffers (its constructor asks the library for workspace sizes,
which launches nothing), so no GPU is needed.
"""
import numpy as np
import pytest
import torch


def _layer(**kw):
    import linear_hybrid_attention_b200 as zb
    return zb.HybridLayer(2, 256, 64, 2, [0, 2], device="cpu", **kw)


def test_save_then_load_restores_the_fit_bit_for_bit(tmp_path):
    a = _layer()
    g = torch.Generator().manual_seed(3)
    a.A.copy_(torch.randn(a.A.shape, generator=g))
    a.b.copy_(torch.randn(a.b.shape, generator=g))
    path = tmp_path / "fit.npz"
    a.save_fit(path)
    b = _layer()
    b.A.zero_()
    b.b.zero_()
    b.load_fit(path)
    assert torch.equal(a.A, b.A) and torch.equal(a.b, b.b)
    with np.load(path) as f:
        assert int(f["heads"]) == 2 and int(f["head_dim"]) == 64 and not bool(f["centered"])


def test_load_rejects_a_fit_of_another_shape(tmp_path):
    path = tmp_path / "fit.npz"
    np.savez(path, A=np.zeros((3, 64, 64), np.float32), b=np.zeros((3, 64), np.float32),
             heads=3, head_dim=64, centered=False)
    with pytest.raises(ValueError):
        _layer().load_fit(path)


def test_load_rejects_a_fit_of_the_other_variant(tmp_path):
    path = tmp_path / "fit.npz"
    _layer(centered=True).save_fit(path)
    with pytest.raises(ValueError):
        _layer().load_fit(path)


def test_a_name_without_the_suffix_works_both_ways(tmp_path):
    a = _layer()
    a.A.fill_(0.5)
    a.b.fill_(-1.0)
    a.save_fit(tmp_path / "fit")          # numpy writes fit.npz
    b = _layer()
    b.load_fit(tmp_path / "fit")
    assert torch.equal(a.A, b.A) and torch.equal(a.b, b.b)
