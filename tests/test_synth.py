"""The seeded input generators: the split-out draws match the full session
recipe, and device-drawn keys follow the same per-channel scales."""
import numpy as np
import torch

import synth


def test_channel_sigma_is_the_sessions_first_draws():
    ses = synth.make_session(3, 2, 4, 1000, 64)
    sigma, outliers = synth.channel_sigma(3, 2)
    assert np.array_equal(ses.sigma, sigma) and np.array_equal(ses.outliers, outliers)
    # 4 outlier channels per KV head at 10x
    assert outliers.shape == (2, synth.N_OUTLIERS)


def test_agent_session_params_match_the_agent_sessions():
    full = synth.make_agent_sessions(3, n_min=1000, n_max=3000)
    params = synth.agent_session_params(3, n_min=1000, n_max=3000)
    for ses, p in zip(full, params):
        assert ses.n_keys == p["n"] and ses.meta["budget"] == p["budget"]
        assert np.array_equal(ses.sigma, p["sigma"])
        assert 1000 <= p["n"] <= 3000 and p["budget"] in (68, 92, 136)


def test_device_keys_are_seeded_and_scaled_per_channel():
    sigma, _ = synth.channel_sigma(0, 2, head_dim=32)
    a = synth.device_keys(torch, sigma, 20000, seed=5, device="cpu")
    b = synth.device_keys(torch, sigma, 20000, seed=5, device="cpu")
    assert a.shape == (2, 20000, 32) and a.dtype == torch.float32
    assert torch.equal(a, b)
    ratio = a.double().std(dim=1).numpy() / sigma
    assert np.all(np.abs(ratio - 1.0) < 0.05)
