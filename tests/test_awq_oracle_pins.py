"""Pins for the AWQ-style scaling oracle (oracle/awq.py), CPU only.

The pages print no numbers for AWQ beyond the worked example's inputs, so these pins check what they do
fix and what the mathematics fixes: alpha = 0 is plain quantisation; the rescaling cancels exactly when
nothing is quantised; scaling the salient channel of the page's example lowers the output error; on
synthetic activations with salient channels the searched scales beat plain quantisation on held-out rows.
A last test plants plausible mistakes in the oracle and checks that these pins catch each one.
"""
import numpy as np
import pytest
import torch

import oracle
import wq_inputs
from golden import read
from oracle import awq


def _deq_asym(g):
    def f(w32):
        codes, s, z = oracle.quantize_int4(w32, g, oracle.STORED)
        return oracle.dequant_int4(codes, s, z, g)
    return f


def _deq_sym(g, mode=oracle.EXACT):
    def f(w32):
        codes, s = oracle.quantize_int4_sym(w32, g, mode)
        return (codes.astype(np.float64) - 8) * np.repeat(s.astype(np.float64), g, axis=1)
    return f


def _toy():
    sc, _ = read("int4_symmetric_examples.txt")
    w = np.array([[float(v) for v in sc["awq_weights"][0]]], dtype=np.float32)
    x = np.array([[float(v) for v in sc["awq_activations"][0]]])
    return w, x


def _llm(seed_w=301, seed_x=302, N=128, K=512, M=48):
    """A layer's weights and M rows of its inputs: 1 % of the channels 20x larger, the same channels for
    every draw of the rows (channel_seed is tied to the layer)."""
    w = wq_inputs.llm_weight(N, K, seed_w, dtype=torch.float32).numpy()
    x = wq_inputs.activations(M, K, seed_x, channel_seed=seed_w).double().numpy()
    return w, x


def test_grid_and_scale_normalisation():
    assert len(awq.GRID) == 21 and awq.GRID[0] == 0.0 and awq.GRID[-1] == 1.0
    mag = np.array([0.5, 2.0, 8.0, 0.0, 1.0])
    for a in (0.0, 0.3, 1.0):
        s = awq.channel_scales(mag, a).astype(np.float64)
        assert np.all(s > 0)
        assert abs(s.max() * s.min() - 1.0) < 1e-6
        if a > 0:  # larger activation magnitude, larger scale; a silent channel gets the smallest
            assert s[2] > s[1] > s[4] > s[0] and s[3] == s[0]
    assert np.all(awq.channel_scales(mag, 0.0) == 1.0)


def test_alpha_zero_is_plain_quantisation():
    w, x = _llm()
    deq = _deq_asym(128)
    s = awq.channel_scales(awq.channel_magnitude(x), 0.0)
    plain = float(np.sum((x @ deq(w).T - x @ w.astype(np.float64).T) ** 2))
    assert awq.output_error(x, w, s, deq) == plain


@pytest.mark.parametrize("alpha", [0.25, 0.5, 1.0])
def test_rescaling_cancels_without_quantisation(alpha):
    """With the quantiser replaced by the identity, (x / s)(w s)^T equals x w^T up to the binary32
    rounding of w s (relative 2^-24 per weight)."""
    w, x = _llm()
    s = awq.channel_scales(awq.channel_magnitude(x), alpha)
    exact = x @ w.astype(np.float64).T
    err = awq.output_error(x, w, s, lambda w32: w32.astype(np.float64))
    assert err <= (2.0 ** -23) ** 2 * float(np.sum(np.abs(x) @ np.abs(w.astype(np.float64)).T) ** 2)
    assert float(np.sum(exact ** 2)) > 1.0


def test_page_example_salient_channel():
    """The page's example: activation 10 on the first channel.  Its scale comes out largest, and the
    searched scales give a smaller output error than plain quantisation."""
    w, x = _toy()
    alpha, s, errors = awq.search(x, w, _deq_sym(w.shape[1]))
    assert alpha > 0 and int(np.argmax(s)) == 0
    assert min(errors) == errors[awq.GRID.index(alpha)] < errors[0]


def test_salient_channels_searched_scales_beat_plain_on_held_out_rows():
    w, x_cal = _llm()
    _, x_test = _llm(seed_x=303)
    deq = _deq_asym(128)
    alpha, s, errors = awq.search(x_cal, w, deq)
    assert alpha > 0 and errors[awq.GRID.index(alpha)] < errors[0]
    plain = awq.output_error(x_test, w, awq.channel_scales(awq.channel_magnitude(x_cal), 0.0), deq)
    assert awq.output_error(x_test, w, s, deq) < plain


MUTANTS = {
    "activations_times_scale": ("quantised_product",
                                lambda x, wh, s: np.asarray(x, np.float64) * np.asarray(s, np.float64)[None, :] @ np.asarray(wh, np.float64).T),
    "weights_divided": ("scaled_weights",
                        lambda w, s: (np.asarray(w, np.float32) / np.asarray(s, np.float32)[None, :]).astype(np.float32)),
    "no_normalisation": ("channel_scales",
                         lambda m, a: (np.where(np.asarray(m) > 0, np.asarray(m, np.float64), 1.0) ** a).astype(np.float32)),
    "magnitude_not_abs": ("channel_magnitude", lambda x: np.mean(np.asarray(x, np.float64), axis=0)),
    "inverted_exponent": ("channel_scales",
                          lambda m, a, f=awq.channel_scales: f(m, -a)),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_mutant(mutant, monkeypatch):
    name, fn = MUTANTS[mutant]
    monkeypatch.setattr(awq, name, fn)
    pins = [test_grid_and_scale_normalisation, test_alpha_zero_is_plain_quantisation,
            lambda: [test_rescaling_cancels_without_quantisation(a) for a in (0.25, 0.5, 1.0)],
            test_page_example_salient_channel, test_salient_channels_searched_scales_beat_plain_on_held_out_rows]
    failures = 0
    for p in pins:
        try:
            p()
        except Exception:
            failures += 1
    assert failures > 0, f"no pin caught {mutant}"
