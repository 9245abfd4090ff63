"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these re-types the oracle's formulas: the expected values come from
the pages' worked examples (tests/golden/), closed forms, invariants, brute
force loops, finite differences and torch's independent CPU float64 routine.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import (attention_backward, attention_forward, flash_forward_tiled,
                    merge, running_stats, sum_of_block_outputs)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN2 = math.log(2.0)


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(rng, n, d, scale=1.0):
    return rng.standard_normal((n, d)) * scale


# --------------------------------------------------------------- page examples
def test_scalar_example_full_softmax():
    g = _load("scalar_example.json")
    assert g["values"] == [10.0, 20.0]
    q = np.array([[1.0]])
    k = np.array([[0.0], [LN2]])          # scores [0, ln 2] with scale 1
    v = np.array([[10.0], [20.0]])
    o, lse = attention_forward(np.vstack([q, q]), k, v, scale=1.0)
    assert abs(o[0, 0] - 50.0 / 3.0) < 1e-12
    assert abs(lse[0] - math.log(3.0)) < 1e-12
    # softmax weights [1/3, 2/3]: use one-hot values to read them out
    w, _ = attention_forward(np.vstack([q, q]), k, np.eye(2), scale=1.0)
    assert np.allclose(w[0], [1.0 / 3.0, 2.0 / 3.0], atol=1e-15)


def test_scalar_example_block_merge():
    g = _load("scalar_example.json")
    b1, b2 = g["per_block"]
    m, l, u = merge(np.float64(b1["m"]), np.float64(b1["l"]), np.float64(b1["u"]),
                    np.float64(LN2), np.float64(b2["l"]), np.float64(b2["u"]))
    assert abs(m - LN2) < 1e-15
    assert abs(l - g["merged"]["l"]) < 1e-12
    assert abs(u - g["merged"]["u"]) < 1e-12
    assert abs(u / l - 50.0 / 3.0) < 1e-12
    # the tiled model with one key per block reaches the same output
    q = np.array([[1.0], [1.0]])
    k = np.array([[0.0], [LN2]])
    v = np.array([[10.0], [20.0]])
    o, _ = flash_forward_tiled(q, k, v, br=1, bc=1, scale=1.0)
    assert abs(o[0, 0] - 50.0 / 3.0) < 1e-12
    # negative control: adding the per-block normalised outputs gives 30
    wrong = sum_of_block_outputs([0.0, LN2], [10.0, 20.0], block=1)
    assert abs(wrong - g["sum_of_block_outputs_wrong"]) < 1e-12


def test_running_sum_123():
    g = _load("running_sum_123.json")
    (m1, l1), (m2, l2) = running_stats(g["blocks"])
    e = math.e
    assert m1 == 2.0 and abs(l1 - (e ** -1 + 1.0)) < 1e-15
    assert m2 == 3.0 and abs(l2 - (e ** -1 * (e ** -1 + 1.0) + 1.0)) < 1e-15
    # and the final l equals the plain sum e^{1-3}+e^{2-3}+e^{3-3}
    assert abs(l2 - (e ** -2 + e ** -1 + 1.0)) < 1e-15


def test_scalar_case_embedding_used_on_gpu():
    from exact_attention_117_b200.workloads import scalar_case
    q, k, v, scale = scalar_case(64)
    o, lse = attention_forward(q[0, 0].double().numpy(), k[0, 0].double().numpy(),
                               v[0, 0].double().numpy(), scale=scale)
    assert abs(o[0, 0] - 50.0 / 3.0) < 1e-12
    assert np.all(o[:, 1:] == 0.0)
    assert abs(lse[0] - math.log(3.0)) < 1e-12


# ---------------------------------------------------------- tile-size invariance
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("brc", [(1, 1), (7, 13), (16, 16), (64, 32), (37, 37)])
def test_tiled_equals_naive(causal, brc):
    rng = np.random.default_rng(7)
    n, d = 37, 8
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, d)
    o_ref, lse_ref = attention_forward(q, k, v, causal=causal)
    o, lse = flash_forward_tiled(q, k, v, br=brc[0], bc=brc[1], causal=causal)
    assert np.max(np.abs(o - o_ref)) < 1e-12
    assert np.max(np.abs(lse - lse_ref)) < 1e-12


def test_row_chunking_is_invisible():
    rng = np.random.default_rng(3)
    n, d = 50, 6
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    for causal in (False, True):
        a = attention_forward(q, k, v, causal, row_chunk=7)
        b = attention_forward(q, k, v, causal, row_chunk=1024)
        assert np.max(np.abs(a[0] - b[0])) < 1e-13
        ga = attention_backward(q, k, v, do, causal, row_chunk=7)
        gb = attention_backward(q, k, v, do, causal, row_chunk=1024)
        for x, y in zip(ga, gb):
            assert np.max(np.abs(x - y)) < 1e-12


# ---------------------------------------------------------------- causal masking
def test_causal_row_depends_only_on_prefix():
    rng = np.random.default_rng(11)
    n, d = 40, 8
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, d)
    o, lse = attention_forward(q, k, v, causal=True)
    for i in (0, 5, 19, 38):
        k2, v2 = k.copy(), v.copy()
        k2[i + 1:] = rng.standard_normal(k2[i + 1:].shape) * 10
        v2[i + 1:] = rng.standard_normal(v2[i + 1:].shape) * 10
        o2, lse2 = attention_forward(q, k2, v2, causal=True)
        assert np.array_equal(o[: i + 1], o2[: i + 1])
        assert np.array_equal(lse[: i + 1], lse2[: i + 1])
        assert not np.array_equal(o[i + 1:], o2[i + 1:])


def test_causal_first_row_is_first_value():
    rng = np.random.default_rng(5)
    q, k, v = (_rand(rng, 9, 4) for _ in range(3))
    o, lse = attention_forward(q, k, v, causal=True, scale=0.3)
    assert np.array_equal(o[0], v[0])
    assert abs(lse[0] - 0.3 * q[0] @ k[0]) < 1e-14


# ----------------------------------------------------------------- stability
def test_shift_500_stays_finite_and_equal():
    rng = np.random.default_rng(2)
    n, d = 64, 16
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, d)
    scale = 0.25
    q[:, -1] = 0
    k[:, -1] = 0
    o, lse = attention_forward(q, k, v, scale=scale)
    qs, ks = q.copy(), k.copy()
    qs[:, -1] = 500.0 / scale
    ks[:, -1] = 1.0
    o2, lse2 = attention_forward(qs, ks, v, scale=scale)
    assert np.all(np.isfinite(o2)) and np.all(np.isfinite(lse2))
    assert np.max(np.abs(o2 - o)) < 1e-12
    assert np.max(np.abs(lse2 - lse - 500.0)) < 1e-9
    for causal in (False, True):
        a, _ = flash_forward_tiled(qs, ks, v, 16, 16, causal, scale)
        b, _ = attention_forward(qs, ks, v, causal, scale)
        assert np.max(np.abs(a - b)) < 1e-12


def test_unshifted_float32_softmax_overflows():
    """Page 2, 动手实现 item 3: exp/sum/divide without the max shift overflows."""
    s = (np.arange(8, dtype=np.float32) + np.float32(500.0))
    with np.errstate(over="ignore", invalid="ignore"):
        e = np.exp(s)
        w = e / e.sum()
    assert not np.all(np.isfinite(w))
    o, _ = attention_forward(np.ones((8, 1)), s[:, None].astype(np.float64),
                             np.arange(8.0)[:, None], scale=1.0)
    assert np.all(np.isfinite(o))


# ------------------------------------------------------- closed forms, brute force
def test_single_key_closed_form():
    rng = np.random.default_rng(0)
    q, k, v = _rand(rng, 1, 5), _rand(rng, 1, 5), _rand(rng, 1, 5)
    o, lse = attention_forward(q, k, v, scale=0.7)
    assert np.array_equal(o, v)
    assert abs(lse[0] - 0.7 * float(q[0] @ k[0])) < 1e-14
    dq, dk, dv = attention_backward(q, k, v, np.ones((1, 5)), scale=0.7)
    assert np.allclose(dv, np.ones((1, 5)), atol=0, rtol=0)
    assert np.all(dq == 0) and np.all(dk == 0)


def test_constant_values_and_linearity():
    rng = np.random.default_rng(4)
    q, k = _rand(rng, 20, 6), _rand(rng, 20, 6)
    v1, v2 = _rand(rng, 20, 3), _rand(rng, 20, 3)
    for causal in (False, True):
        o, _ = attention_forward(q, k, np.ones((20, 3)), causal)
        assert np.max(np.abs(o - 1.0)) < 1e-14
        a, _ = attention_forward(q, k, v1 + 2 * v2, causal)
        b1, _ = attention_forward(q, k, v1, causal)
        b2, _ = attention_forward(q, k, v2, causal)
        assert np.max(np.abs(a - (b1 + 2 * b2))) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [1, 2, 5, 16])
def test_brute_force_loops(causal, n):
    rng = np.random.default_rng(n)
    d = 3
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, d)
    scale = 0.9
    o, lse = attention_forward(q, k, v, causal, scale)
    for i in range(n):
        keys = range(i + 1) if causal else range(n)
        sc = [scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in keys]
        z = sum(math.exp(x) for x in sc)
        assert abs(lse[i] - math.log(z)) < 1e-12
        for c in range(d):
            ref = sum(math.exp(x) * v[j][c] for x, j in zip(sc, keys)) / z
            assert abs(o[i][c] - ref) < 1e-12


# ------------------------------------------------------------------ gradients
def _loss(q, k, v, do, causal, scale):
    o, _ = attention_forward(q, k, v, causal, scale)
    return float(np.sum(o * do))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 2), (3, 4), (8, 4), (5, 1)])
def test_backward_finite_differences(causal, n, d):
    rng = np.random.default_rng(100 * n + d)
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    scale = 0.8
    grads = attention_backward(q, k, v, do, causal, scale)
    h = 1e-6
    for which, g in zip(range(3), grads):
        num = np.zeros_like(g)
        for idx in np.ndindex(g.shape):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            up = _loss(*args, do, causal, scale)
            args[which][idx] -= 2 * h
            dn = _loss(*args, do, causal, scale)
            num[idx] = (up - dn) / (2 * h)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-12)
        if np.linalg.norm(num) < 1e-9:
            assert np.max(np.abs(g)) < 1e-8
        else:
            assert err < 1e-6, (which, err)


def test_key_gradients_sum_to_zero():
    """Each softmax row's dS sums to zero, so the sum over keys of dK is 0."""
    rng = np.random.default_rng(9)
    q, k, v, do = (_rand(rng, 30, 5) for _ in range(4))
    for causal in (False, True):
        _, dk, _ = attention_backward(q, k, v, do, causal)
        assert np.max(np.abs(dk.sum(axis=0))) < 1e-12


# ------------------------------------------------- independent library routine
@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_cpu_float64(causal):
    rng = np.random.default_rng(21)
    n, d = 70, 16
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    scale = 1.0 / math.sqrt(d)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(
        tq[None], tk[None], tv[None], is_causal=causal, scale=scale)[0]
    to.backward(torch.tensor(do))
    o, lse = attention_forward(q, k, v, causal, scale)
    assert np.max(np.abs(o - to.detach().numpy())) < 1e-12
    s = scale * torch.tensor(q) @ torch.tensor(k).T
    if causal:
        s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    assert np.max(np.abs(lse - torch.logsumexp(s, dim=1).numpy())) < 1e-12
    dq, dk, dv = attention_backward(q, k, v, do, causal, scale)
    assert np.max(np.abs(dq - tq.grad.numpy())) < 1e-12
    assert np.max(np.abs(dk - tk.grad.numpy())) < 1e-12
    assert np.max(np.abs(dv - tv.grad.numpy())) < 1e-12


def test_d_from_output_identity():
    """sum_j P_ij dP_ij equals sum_c dO_ic O_ic, so forming D from the exact O changes nothing."""
    rng = np.random.default_rng(12)
    q, k, v, do = (_rand(rng, 23, 6) for _ in range(4))
    for causal in (False, True):
        o, _ = attention_forward(q, k, v, causal)
        a = attention_backward(q, k, v, do, causal)
        b = attention_backward(q, k, v, do, causal, o_for_d=o)
        for x, y in zip(a, b):
            assert np.max(np.abs(x - y)) < 1e-12
        # a perturbed O moves dQ and dK but never dV (dV does not involve D)
        c = attention_backward(q, k, v, do, causal, o_for_d=o + 1e-3)
        assert np.array_equal(c[2], a[2])
        assert np.max(np.abs(c[0] - a[0])) > 1e-6


# ------------------------------------------------------------ default scale
# Page "FlashAttention为什么更快更省显存", opening formula: the scores are
# Q K^T / sqrt(d_k).  These pins fix the default that every caller leaving
# ``scale`` out relies on, independently of the oracle's own helper.
def test_default_scale_values():
    from oracle import default_scale
    assert default_scale(64) == 0.125           # 1/sqrt(64), exact in binary
    assert default_scale(16) == 0.25
    assert default_scale(4) == 0.5
    assert abs(default_scale(128) - 0.088388347648318440550) < 3e-17
    assert abs(default_scale(3) * default_scale(3) * 3 - 1.0) < 1e-15


@pytest.mark.parametrize("d", [3, 64])
@pytest.mark.parametrize("causal", [False, True])
def test_default_scale_brute_force(d, causal):
    """scale=None gives the brute-force loops run with 1/sqrt(d) written out."""
    rng = np.random.default_rng(1000 + d)
    n = 6
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, d)
    o, lse = attention_forward(q, k, v, causal)
    for i in range(n):
        keys = range(i + 1) if causal else range(n)
        sc = [sum(q[i][c] * k[j][c] for c in range(d)) / math.sqrt(d) for j in keys]
        z = sum(math.exp(x) for x in sc)
        assert abs(lse[i] - math.log(z)) < 1e-12
        for c in range(d):
            ref = sum(math.exp(x) * v[j][c] for x, j in zip(sc, keys)) / z
            assert abs(o[i][c] - ref) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_default_scale_matches_torch_default(causal):
    """torch's scaled_dot_product_attention defaults to 1/sqrt(E) on its own;
    the oracle's forward and backward with scale left out agree with it."""
    rng = np.random.default_rng(33)
    n, d = 19, 64
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(
        tq[None], tk[None], tv[None], is_causal=causal)[0]
    to.backward(torch.tensor(do))
    o, _ = attention_forward(q, k, v, causal)
    dq, dk, dv = attention_backward(q, k, v, do, causal)
    assert np.max(np.abs(o - to.detach().numpy())) < 1e-12
    for g, t in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.max(np.abs(g - t.grad.numpy())) < 1e-12


def test_workload_and_parity_scales():
    """The seeded workloads and the GPU tests' helper use the same 1/sqrt(d)."""
    from exact_attention_117_b200.workloads import WORKLOADS
    from tests.parity_util import default_scale as parity_default_scale
    assert WORKLOADS["c1"].scale == 0.125 and WORKLOADS["c2"].scale == 0.125
    assert abs(WORKLOADS["c3"].scale - 0.088388347648318440550) < 3e-17
    assert WORKLOADS["c4"].scale == WORKLOADS["c3"].scale
    assert parity_default_scale(64) == 0.125
    assert abs(parity_default_scale(128) - 0.088388347648318440550) < 3e-17
