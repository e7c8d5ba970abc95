"""Pins of the StairFormer nesting pieces (oracle/stairformer.py) against what
the "Fully Nested Transformers" README states: block lower triangular maps and
PrefixRMSNorm make every layer filtration-preserving (output prefixes depend
only on input prefixes), so the top-left corner of the network is the smaller
model and one forward pass of the full model computes every submodel; and
against the base model's plain pieces when there is a single block."""
import numpy as np
import pytest

from oracle import nanochat_fwd as O
from oracle import stairformer as S


def test_readme_d24_blocks():
    # --nested-block-head-counts=6-18 with --head-dim=64 at depth 24: widths 384 + 1152 = 1536
    w = S.head_blocks([6, 18], 64)
    assert w == [384, 1152] and S.block_bounds(w) == [384, 1536]
    C, _ = O.model_dims(24, head_dim=64)
    assert C == 1536


def test_mask_keeps_only_lower_blocks():
    m = S.block_lower_triangular_mask([2, 3, 1], [4, 1, 2])
    assert m.shape == (6, 7)
    assert int(m.sum()) == 2 * 4 + 3 * 5 + 1 * 7
    assert not m[:2, 4:].any() and m[2:5, :5].all() and not m[2:5, 5:].any() and m[5:].all()


def test_single_block_reduces_to_plain_pieces():
    g = np.random.default_rng(0)
    x, w = g.standard_normal((5, 12)), g.standard_normal((7, 12))
    assert np.array_equal(S.btl_linear(x, w, [7], [12]), x @ w.T)
    assert np.allclose(S.prefix_rmsnorm(x, [12]), O.rmsnorm(x), rtol=0, atol=1e-15)
    wu, y = g.standard_normal((50, 12)), g.integers(0, 50, 5)
    y[2] = -1
    (ce,) = S.prefix_ce(x, wu, y, [12])
    ref = O.cross_entropy_per_token(O.softcap(O.rmsnorm(x) @ wu.T), y)
    assert np.allclose(ce, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("widths", [[3, 5], [2, 2, 4], [1, 6, 1]])
def test_layers_preserve_the_filtration(widths):
    """Changing input block b leaves every output block before b unchanged."""
    g = np.random.default_rng(len(widths))
    C = sum(widths)
    x, w = g.standard_normal((4, C)), g.standard_normal((C, C))
    ends = S.block_bounds(widths)
    for b in range(1, len(widths)):
        x2 = x.copy()
        x2[:, ends[b - 1]:ends[b]] += g.standard_normal((4, widths[b]))
        for f in (lambda u: S.btl_linear(u, w, widths, widths), lambda u: S.prefix_rmsnorm(u, widths)):
            y, y2 = f(x), f(x2)
            assert np.array_equal(y[:, :ends[b - 1]], y2[:, :ends[b - 1]])
            assert not np.allclose(y[:, ends[b - 1]:], y2[:, ends[b - 1]:])


def _net(x, layers, widths, hidden_widths):
    """A stack of pre-norm residual ReLU^2 MLPs built from the nesting pieces."""
    for w1, w2 in layers:
        h = np.maximum(S.btl_linear(S.prefix_rmsnorm(x, widths), w1, hidden_widths, widths), 0.0) ** 2
        x = x + S.btl_linear(h, w2, widths, hidden_widths)
    return x


def test_submodel_is_the_top_left_corner():
    """The j-front submodel, built from the top-left corners of the weights
    and run on the prefix of the input, reproduces the prefix of the full
    model's residual stream, and its logits and losses from it."""
    g = np.random.default_rng(7)
    widths, hidden = [4, 8, 4], [16, 32, 16]
    C, Hd = sum(widths), sum(hidden)
    layers = [(g.standard_normal((Hd, C)) / C ** 0.5, g.standard_normal((C, Hd)) / Hd ** 0.5) for _ in range(3)]
    x0 = g.standard_normal((6, C))
    wu, y = g.standard_normal((40, C)) / C ** 0.5, g.integers(0, 40, 6)
    full = _net(x0, layers, widths, hidden)
    ces = S.prefix_ce(full, wu, y, widths)
    ends, hends = S.block_bounds(widths), S.block_bounds(hidden)
    for j in range(1, len(widths) + 1):
        cj, hj = ends[j - 1], hends[j - 1]
        sub_layers = [(w1[:hj, :cj], w2[:cj, :hj]) for w1, w2 in layers]
        sub = _net(x0[:, :cj], sub_layers, widths[:j], hidden[:j])
        assert np.allclose(sub, full[:, :cj], rtol=0, atol=1e-12)
        z_sub = S.prefix_logits(sub, wu[:, :cj], widths[:j], j)
        assert np.allclose(z_sub, S.prefix_logits(full, wu, widths, j), rtol=0, atol=1e-12)
        (ce_last,) = S.prefix_ce(sub, wu[:, :cj], y, widths[:j])[-1:]
        assert np.allclose(ce_last, ces[j - 1], rtol=0, atol=1e-12)
    # the submodels are different models
    assert not np.allclose(ces[0], ces[-1])
