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
