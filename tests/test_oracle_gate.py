"""Pins of the oracle's dynamic gate and branch dropping (oracle_gate), each
against a library routine or a closed form: the sigmoid of the bias alone
against scipy's expit, the pooled hidden state through a one-hot weight
against numpy's mean, the timestep path against numpy's dot product, the
dropping threshold at its limits, and head/batch independence."""
import numpy as np
import pytest
from scipy.special import expit

import oracle
import salad_inputs as si


def draw(B=2, N=37, Hh=3, d=16, E=5, seed=3):
    rng = np.random.default_rng(seed)
    q = si.f32_to_bf16_bits(rng.standard_normal((B, N, Hh, d), dtype=np.float32) + 0.3)
    t_emb = rng.standard_normal((B, E))
    w_t = rng.standard_normal((Hh, E)) * 0.5
    w_x = rng.standard_normal((Hh, d)) * 2.0
    beta = rng.standard_normal(Hh)
    return q, t_emb, w_t, w_x, beta


def test_bias_alone_is_its_sigmoid():
    q, t_emb, w_t, w_x, beta = draw()
    s, g = oracle.gate(q, t_emb, np.zeros_like(w_t), np.zeros_like(w_x), beta, 0.0)
    np.testing.assert_allclose(s, np.broadcast_to(expit(beta), s.shape), rtol=0, atol=1e-15)
    np.testing.assert_array_equal(g, s)


def test_one_hot_weight_reads_the_token_mean_of_one_feature():
    q, t_emb, w_t, w_x, beta = draw()
    qf = si.bf16_bits_to_f32(q).astype(np.float64)
    for f in (0, 7, 15):
        w = np.zeros_like(w_x)
        w[:, f] = 1.0
        s, _ = oracle.gate(q, t_emb, np.zeros_like(w_t), w, np.zeros_like(beta), 0.0)
        np.testing.assert_allclose(s, expit(qf[:, :, :, f].mean(axis=1)), rtol=0, atol=1e-14)


def test_timestep_path_is_a_dot_product():
    q, t_emb, w_t, w_x, beta = draw()
    s, _ = oracle.gate(q, t_emb, w_t, np.zeros_like(w_x), np.zeros_like(beta), 0.0)
    np.testing.assert_allclose(s, expit(t_emb @ w_t.T), rtol=0, atol=1e-14)


def test_full_module_is_the_sum_of_its_parts():
    q, t_emb, w_t, w_x, beta = draw()
    qf = si.bf16_bits_to_f32(q).astype(np.float64)
    s, _ = oracle.gate(q, t_emb, w_t, w_x, beta, 0.0)
    pooled = qf.mean(axis=1)                                   # [B, Hh, d]
    logit = t_emb @ w_t.T + np.einsum("bhf,hf->bh", pooled, w_x) + beta
    np.testing.assert_allclose(s, expit(logit), rtol=0, atol=1e-13)


def test_dropping_threshold():
    q, t_emb, w_t, w_x, beta = draw(B=3, Hh=4)
    s, g = oracle.gate(q, t_emb, w_t, w_x, beta, 0.0)
    assert np.all((s > 0) & (s < 1)) and np.array_equal(g, s)        # nothing dropped at 0
    _, g = oracle.gate(q, t_emb, w_t, w_x, beta, 1.0)
    assert np.all(g == 0)                                             # everything dropped at 1
    tau = float(np.median(s))
    _, g = oracle.gate(q, t_emb, w_t, w_x, beta, tau)
    np.testing.assert_array_equal(g, np.where(s < tau, 0.0, s))
    # a gate exactly at the threshold is kept (only gates below it are dropped)
    _, g = oracle.gate(q, t_emb, w_t, w_x, beta, float(s[1, 2]))
    assert g[1, 2] == s[1, 2]


def test_heads_and_batches_are_independent():
    q, t_emb, w_t, w_x, beta = draw()
    s, _ = oracle.gate(q, t_emb, w_t, w_x, beta, 0.0)
    perm = np.array([2, 0, 1])
    sp, _ = oracle.gate(np.ascontiguousarray(q[:, :, perm]), t_emb, w_t[perm], w_x[perm], beta[perm], 0.0)
    np.testing.assert_array_equal(sp, s[:, perm])
    sb, _ = oracle.gate(np.ascontiguousarray(q[::-1]), t_emb[::-1], w_t, w_x, beta, 0.0)
    np.testing.assert_array_equal(sb, s[::-1])


@pytest.mark.parametrize("N", [1, 2, 129])
def test_constant_tokens_pool_to_themselves(N):
    rng = np.random.default_rng(N)
    row = si.f32_to_bf16_bits(rng.standard_normal((1, 1, 2, 8), dtype=np.float32))
    q = np.ascontiguousarray(np.broadcast_to(row, (1, N, 2, 8)))
    w_x = rng.standard_normal((2, 8))
    s, _ = oracle.gate(q, np.zeros((1, 1)), np.zeros((2, 1)), w_x, np.zeros(2), 0.0)
    v = si.bf16_bits_to_f32(row[0, 0]).astype(np.float64)
    np.testing.assert_allclose(s[0], expit(np.sum(w_x * v, axis=1)), rtol=0, atol=1e-15)
