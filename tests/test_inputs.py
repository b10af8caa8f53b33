"""The seeded input recipe: pattern lists and reproducibility."""
import torch

from kronecker_sparse_matrix_b200 import inputs


def test_sweep_has_258_patterns_within_width_limit():
    pats = inputs.sweep_patterns()
    assert len(pats) == 258
    assert len(set(pats)) == 258
    for a, b, c, d in pats:
        assert a * b * d <= 16384 and a * c * d <= 16384
        assert b == c or b == 4 * c


def test_butterfly_chain_widths_match():
    pats = inputs.butterfly_patterns(12)
    assert len(pats) == 12
    for p in pats:
        assert inputs.in_features(p) == inputs.out_features(p) == 4096
    assert pats[0] == (1, 2, 2, 2048) and pats[-1] == (2048, 2, 2, 1)


def test_seeded_draws_repeat_and_bf16_is_rounded_fp32():
    f1 = inputs.factor_inputs((2, 4, 4, 2), 8, seed=3)
    f2 = inputs.factor_inputs((2, 4, 4, 2), 8, seed=3)
    assert torch.equal(f1.X, f2.X) and torch.equal(f1.values, f2.values)
    fb = inputs.factor_inputs((2, 4, 4, 2), 8, seed=3, dtype=torch.bfloat16)
    assert torch.equal(fb.X, f1.X.to(torch.bfloat16))
    assert f1.values.shape == (2, 2, 4, 4)


def test_toy_recipe():
    t = inputs.toy()
    assert t.X.shape == (8, 16) and t.values.shape == (2, 2, 4, 4)
    assert float(t.X.abs().max()) <= 1.0
