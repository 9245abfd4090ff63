"""Backward parity on the GPU: dQ, dK, dV from the CUDA path vs the float64 oracle.

The CUDA backward consumes O and LSE from the CUDA forward, as a training
step does; the oracle recomputes everything from Q, K, V, dO alone.
"""
import numpy as np
import pytest
import torch

from exact_attention_117_b200 import fa
from exact_attention_117_b200.workloads import (WORKLOADS, Workload, make_inputs, sample_slices,
                                                scalar_case, sweep_workloads)
from parity_util import (FLOOR_USES, check_grad, floor_report, oracle_bwd_slice,
                         output_rounding_floor, slice_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fwd_bwd(x, causal, scale, workspace=None):
    o, lse = fa.forward(x["q"], x["k"], x["v"], causal=causal, scale=scale)
    grads = fa.backward(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal, scale=scale,
                        workspace=workspace)
    fa.check_device_error()
    return o, lse, grads


def _check(x, grads, causal, scale, slices, floor=False):
    """Stated tolerance; ``floor=True`` (rows shorter than 64 keys only) adds twice the
    bf16-output rounding floor derived by the oracle for the same slice."""
    dq, dk, dv = grads
    for b, h in slices:
        ref = oracle_bwd_slice(x["q"], x["k"], x["v"], x["do"], b, h, causal, scale)
        fl = (output_rounding_floor(x["q"], x["k"], x["v"], x["do"], b, h, causal, scale, ref)
              if floor else (0.0, 0.0, 0.0))
        for name, g, r, f in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref, fl):
            check_grad(slice_np(g, b, h), r, f"{name}[{b},{h}]", floor=2.0 * f)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [1, 2, 127, 128, 129, 300, 1000])
def test_bwd_small_shapes(d, causal, n):
    w = Workload("small", 1, 2, n, d, seed_base=31 + n)
    x = make_inputs(w, DEV)
    _, _, grads = _fwd_bwd(x, causal, w.scale)
    _check(x, grads, causal, w.scale, [(0, 0), (0, 1)], floor=n < 64)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_c1_and_ragged(causal):
    for name in ("c1",):
        w = WORKLOADS[name]
        x = make_inputs(w, DEV)
        _, _, grads = _fwd_bwd(x, causal, w.scale)
        _check(x, grads, causal, w.scale, [(0, 0)])
    w = WORKLOADS["c2r"]
    x = make_inputs(w, DEV)
    _, _, grads = _fwd_bwd(x, causal, w.scale)
    _check(x, grads, causal, w.scale, [(b, h) for b in range(w.B) for h in range(w.H)])


@pytest.mark.parametrize("name", ["c3", "c4"])
def test_bwd_large(name):
    """c3 on every (b, h) slice; c4 on 4 seeded slices."""
    w = WORKLOADS[name]
    x = make_inputs(w, DEV)
    _, _, grads = _fwd_bwd(x, True, w.scale)
    if name == "c3":
        slices = [(b, h) for b in range(w.B) for h in range(w.H)]
    else:
        slices = [(i // w.H, i % w.H) for i in sample_slices(w.B * w.H, 4)]
    _check(x, grads, True, w.scale, slices)


@pytest.mark.parametrize("w", sweep_workloads(), ids=lambda w: w.name)
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_sweep_sampled(w, causal):
    x = make_inputs(w, DEV)
    _, _, grads = _fwd_bwd(x, causal, w.scale)
    idx = sample_slices(w.B * w.H, 2)
    _check(x, grads, causal, w.scale, [(i // w.H, i % w.H) for i in idx])


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_scalar_case(d):
    q, k, v, scale = scalar_case(d, DEV)
    g = torch.Generator(device="cpu").manual_seed(5)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(DEV)
    x = {"q": q, "k": k, "v": v, "do": do}
    _, _, grads = _fwd_bwd(x, False, scale)
    _check(x, grads, False, scale, [(0, 0)], floor=True)


def test_bwd_workspace_contents_do_not_matter():
    w = Workload("ws", 2, 2, 300, 128, seed_base=41)
    x = make_inputs(w, DEV)
    need = fa.workspace_size(2, 2, 300, 128)
    ws = torch.full((need // 4,), float("nan"), dtype=torch.float32, device=DEV)
    _, _, g1 = _fwd_bwd(x, True, w.scale, workspace=ws)
    for t in g1:
        assert torch.isfinite(t.float()).all()
    _check(x, g1, True, w.scale, [(0, 0), (1, 1)])


def test_bwd_dk_dv_deterministic():
    w = Workload("det", 1, 4, 700, 64, seed_base=43)
    x = make_inputs(w, DEV)
    _, _, g1 = _fwd_bwd(x, True, w.scale)
    _, _, g2 = _fwd_bwd(x, True, w.scale)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    # dQ is summed with atomics: equal up to the rounding order of the adds
    assert float((g1[0].float() - g2[0].float()).abs().max()) < 1e-2


def test_bwd_poisoned_outputs_fully_written():
    w = Workload("poison", 1, 3, 333, 128, seed_base=47)
    x = make_inputs(w, DEV)
    o, lse = fa.forward(x["q"], x["k"], x["v"], causal=True)
    dq, dk, dv = (torch.full_like(x["q"], float("nan")) for _ in range(3))
    fa.backward(x["q"], x["k"], x["v"], o, lse, x["do"], causal=True, dq=dq, dk=dk, dv=dv)
    fa.check_device_error()
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("deterministic", [False, True])
def test_bwd_many_items_per_cta(d, deterministic):
    # 4 x 40 heads x 5 key tiles = 800 (head, key tile) work items for the
    # persistent main kernel, several per CTA and of 1 to 5 query tiles each
    # under the causal mask (N = 600: the last key tile is ragged).  Every
    # output element must be written, and the first head, one in the middle
    # and the last (whose items are claimed last) must match the oracle.
    w = Workload("items", 4, 40, 600, d, seed_base=53)
    x = make_inputs(w, DEV)
    o, lse = fa.forward(x["q"], x["k"], x["v"], causal=True)
    dq, dk, dv = (torch.full_like(x["q"], float("nan")) for _ in range(3))
    fa.backward(x["q"], x["k"], x["v"], o, lse, x["do"], causal=True, dq=dq, dk=dk, dv=dv,
                deterministic=deterministic)
    fa.check_device_error()
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    _check(x, (dq, dk, dv), True, w.scale, [(0, 0), (2, 17), (3, 39)])


@pytest.mark.parametrize("scale", [0.0, -0.09])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_any_finite_scale(scale, causal):
    w = Workload("scale", 1, 2, 300, 64, seed_base=14)
    x = make_inputs(w, DEV)
    _, _, grads = _fwd_bwd(x, causal, scale)
    _check(x, grads, causal, scale, [(0, 0), (0, 1)])


def test_bwd_zz_floor_margin_report():
    """Reports the widened gradient bound's worst margin (rows shorter than 64
    keys only); written to $FA_PARITY_REPORT when set.  Runs last in the module."""
    line = floor_report()
    print(line)
    path = __import__("os").environ.get("FA_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(line + "\n")
    assert all(t[2] <= 1.0 for t in FLOOR_USES)
