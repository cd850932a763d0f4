"""The stress inputs reach the cases they are meant for (checked with the oracle's quantiser, on the CPU)."""
import numpy as np

import oracle
import wq_inputs


def _bf16_exact(v: np.ndarray) -> np.ndarray:
    """True where the binary64 values are exactly representable in bf16 (8 significant bits)."""
    m, e = np.frexp(np.abs(v))
    return (v == 0) | (np.ldexp(m, 8) == np.round(np.ldexp(m, 8)))


def test_offset_group_weight_reaches_zero_points_bf16_cannot_shift():
    """The far-zero-point parity tests need groups whose z is outside [0, 15] and whose 128 + z or q - z is
    not a bf16 value: there a kernel that formed (128 + q) - (128 + z) in bf16 would round."""
    w = wq_inputs.offset_group_weight(640, 2048, 93).numpy()
    codes, s, z = oracle.quantize_int4(w, 128)
    zr = z[::3]  # the banded rows
    assert np.all((zr < 0) | (zr > 15))
    assert np.all((z[1::3] >= 0) & (z[1::3] <= 15))  # the others straddle zero
    not_exact = ~_bf16_exact(128.0 + zr)
    assert not_exact.sum() >= 20, "too few groups where 128 + z rounds in bf16"
    assert (np.abs(zr) > 256).sum() >= 20, "too few groups where q - z can leave bf16's exact integers"
    assert (zr < 0).any() and (zr > 0).any()


def test_positive_activations_have_one_sign():
    x = wq_inputs.positive_activations(4, 1024, 7).float().numpy()
    assert (x > 0).all()


def test_activations_channel_seed_fixes_the_salient_channels():
    """With channel_seed, two draws share their salient channels (inputs of one layer); without it the
    channels follow the seed."""
    import numpy as np
    a = wq_inputs.activations(64, 1024, 1, channel_seed=9).float().abs().mean(0).numpy()
    b = wq_inputs.activations(64, 1024, 2, channel_seed=9).float().abs().mean(0).numpy()
    top_a, top_b = set(np.argsort(a)[-10:]), set(np.argsort(b)[-10:])
    assert top_a == top_b
    c = wq_inputs.activations(64, 1024, 2).float().abs().mean(0).numpy()
    assert set(np.argsort(c)[-10:]) != top_a


def test_generators_are_seeded():
    a = wq_inputs.llm_weight(64, 256, 5)
    assert (a == wq_inputs.llm_weight(64, 256, 5)).all()
    assert not (a == wq_inputs.llm_weight(64, 256, 6)).all()
    x = wq_inputs.activations(4, 256, 5)
    assert (x == wq_inputs.activations(4, 256, 5)).all()


def test_weight_recipes_match_their_description():
    """The recipes the workloads are described with: N(0, 0.02) bodies; a 0.1% fraction of entries x10
    (decode_up, sweep); one x20 entry per 1024 consecutive K of each row (gran); 4 entries of +-1 (tiny)."""
    w = wq_inputs.llm_weight(512, 4096, 2, dtype=__import__("torch").float32).numpy()
    body = np.abs(w) < 0.1
    assert abs(w[body].std() - 0.02) < 0.001
    big = np.abs(w) > 0.1          # 5 sigma of the body: essentially only the x10 entries
    # 0.1% of the entries are multiplied by 10; those drawn above 0.5 sigma (61.7% of them) pass 0.1
    assert 0.55e-3 < big.mean() < 0.68e-3
    g = wq_inputs.block_outlier_weight(64, 8192, 4, dtype=__import__("torch").float32).numpy()
    blocks = np.abs(g).reshape(64, 8, 1024)
    # a x20 entry passes 0.1 (5 sigma of the body) when its draw is above 0.25 sigma: 80% of blocks; a
    # block of 1024 plain draws almost never does, and no block holds two such entries
    over = (blocks > 0.1).sum(-1)
    assert 0.74 < (over >= 1).mean() < 0.86 and over.max() == 1
    t = wq_inputs.tiny_weight().numpy()
    assert t.shape == (512, 256) and (np.abs(t) == 1.0).sum() == 4


def test_activation_recipe_has_one_percent_salient_channels():
    x = wq_inputs.activations(256, 4096, 3).float().numpy()
    m = np.abs(x).mean(0)
    salient = m > 5 * np.median(m)
    assert salient.sum() == round(0.01 * 4096)
    assert abs(np.median(m[salient]) / np.median(m[~salient]) - 20) < 1.5
