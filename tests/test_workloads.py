"""The seeded input generators (tq_workloads.py) on the CPU: shapes, dtype,
determinism and the properties each stress recipe states, so the GPU parity
tests run on the inputs their docstrings describe."""

import os
import sys

import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import tq_workloads as W  # noqa: E402


@pytest.mark.parametrize("kind", W.STRESS_KINDS)
def test_stress_rows_are_seeded_fp16(kind):
    a = W.stress_rows(kind, 257, 64, seed=5, device="cpu")
    b = W.stress_rows(kind, 257, 64, seed=5, device="cpu")
    c = W.stress_rows(kind, 257, 64, seed=6, device="cpu")
    assert a.dtype == torch.float16 and tuple(a.shape) == (257, 64)
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert torch.isfinite(a).all() and a.abs().max().item() <= 60000


def test_stress_recipes():
    n, d = 4000, 128
    sp = W.stress_rows("sparse", n, d, seed=1, device="cpu")
    frac = (sp != 0).float().mean().item()
    assert 0.09 < frac < 0.11  # kept with probability 0.1
    md = W.stress_rows("mean_dominated", n, d, seed=1, device="cpu").float()
    assert abs(md.mean().item() - 3.0) < 1e-3 and 0.009 < md.std().item() < 0.011
    ol = W.stress_rows("outlier_x10", n, d, seed=1, device="cpu").float()
    big = (ol.std(dim=0) > 5.0).nonzero().flatten()
    assert big.numel() == 4  # four channels times 10
    assert 9.0 < ol[:, big].std().item() < 11.0
    dr = W.stress_rows("dynamic_range", n, d, seed=1, device="cpu").float().abs()
    nz = dr[dr > 0]
    assert nz.max().item() / nz.min().item() > 2.0 ** 28  # 2^k, k in [-14, 13], times N(0,1)
    cl = W.stress_rows("channel_lognormal", n, d, seed=1, device="cpu").float()
    s = cl.std(dim=0)
    assert s.max().item() / s.min().item() > 10.0  # per-channel exp(1.5 N(0,1)) scales
    st = W.stress_rows("student3", n, d, seed=1, device="cpu").float()
    g = W.stress_rows("gauss", n, d, seed=1, device="cpu").float()
    assert (st.abs() > 6).float().mean().item() > 20 * max((g.abs() > 6).float().mean().item(), 1e-7)


def test_unknown_stress_kind():
    with pytest.raises(ValueError):
        W.stress_rows("uniform", 4, 64, seed=0, device="cpu")


def test_edge_vectors_cover_the_degenerate_rows():
    e = W.edge_vectors(128)
    assert e.dtype == torch.float16 and e.shape[1] == 128
    f = e.float()
    assert (f.abs().sum(dim=1) == 0).any()  # the zero vector
    assert (f == 65504).all(dim=1).any()  # the fp16 maximum
    assert ((f.abs() > 0) & (f.abs() < 2.0 ** -14)).any()  # subnormals
    spikes = ((f != 0).sum(dim=1) == 1).sum().item()
    assert spikes >= 4
