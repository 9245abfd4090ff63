"""Forward parity on the GPU: CUDA path (through the C ABI) vs the float64 oracle."""
import math

import numpy as np
import pytest
import torch

from exact_attention_117_b200 import fa
from exact_attention_117_b200.workloads import (WORKLOADS, Workload, make_inputs, sample_slices,
                                                scalar_case, shift_copy, sweep_workloads)
from parity_util import (bf16_round, bf16_ulp, check_lse, check_o, oracle_fwd_slice, slice_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_and_check(q, k, v, causal, scale, slices=None):
    o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
    fa.check_device_error()
    B, H = q.shape[:2]
    if slices is None:
        slices = [(b, h) for b in range(B) for h in range(H)]
    for b, h in slices:
        o_ref, lse_ref = oracle_fwd_slice(q, k, v, b, h, causal, scale)
        check_o(slice_np(o, b, h), o_ref, f"O[{b},{h}]")
        check_lse(lse[b, h].double().cpu().numpy(), lse_ref, f"LSE[{b},{h}]")
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [1, 2, 127, 128, 129, 300, 384, 640, 1000])
def test_fwd_small_shapes(d, causal, n):
    w = Workload("small", 1, 2, n, d, seed_base=17 + n)
    x = make_inputs(w, DEV, with_do=False)
    _run_and_check(x["q"], x["k"], x["v"], causal, w.scale)


def test_fwd_c1_full():
    w = WORKLOADS["c1"]
    x = make_inputs(w, DEV, with_do=False)
    _run_and_check(x["q"], x["k"], x["v"], False, w.scale)


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_scalar_case(d):
    q, k, v, scale = scalar_case(d, DEV)
    o, lse = fa.forward(q, k, v, causal=False, scale=scale)
    fa.check_device_error()
    want = 50.0 / 3.0
    got = float(o[0, 0, 0, 0])
    assert abs(got - float(bf16_round(np.array([want]))[0])) <= float(bf16_ulp(np.array([want]))[0])
    assert float(o[0, 0, 0, 1:].abs().max()) == 0.0
    assert abs(float(lse[0, 0, 0]) - math.log(3.0)) <= 1e-3


def test_fwd_shift_500():
    w = WORKLOADS["c1"]
    x = make_inputs(w, DEV, with_do=False)
    (qb, kb), (qs, ks) = shift_copy(x["q"], x["k"], w.scale)
    ob, lb = _run_and_check(qb, kb, x["v"], False, w.scale)
    os_, ls = _run_and_check(qs, ks, x["v"], False, w.scale)
    assert torch.isfinite(os_.float()).all() and torch.isfinite(ls).all()
    assert float((ls - lb - 500.0).abs().max()) <= 1e-3
    assert float((os_.float() - ob.float()).abs().max()) <= 1e-2


@pytest.mark.parametrize("name", ["c2", "c2r"])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_c2(name, causal):
    w = WORKLOADS[name]
    x = make_inputs(w, DEV, with_do=False)
    _run_and_check(x["q"], x["k"], x["v"], causal, w.scale)  # every (b, h) slice


@pytest.mark.parametrize("name", ["c3", "c4"])
def test_fwd_large(name):
    """c3 on every (b, h) slice; c4 on 4 seeded slices (each c4 slice costs the
    float64 oracle seconds of work)."""
    w = WORKLOADS[name]
    x = make_inputs(w, DEV, with_do=False)
    slices = None if name == "c3" else [(i // w.H, i % w.H) for i in sample_slices(w.B * w.H, 4)]
    _run_and_check(x["q"], x["k"], x["v"], True, w.scale, slices)


@pytest.mark.parametrize("w", sweep_workloads(), ids=lambda w: w.name)
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_sweep_sampled(w, causal):
    x = make_inputs(w, DEV, with_do=False)
    idx = sample_slices(w.B * w.H, 2)
    _run_and_check(x["q"], x["k"], x["v"], causal, w.scale, [(i // w.H, i % w.H) for i in idx])


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_deterministic(causal):
    w = Workload("det", 2, 4, 777, 128, seed_base=5)
    x = make_inputs(w, DEV, with_do=False)
    o1, l1 = fa.forward(x["q"], x["k"], x["v"], causal=causal)
    o2, l2 = fa.forward(x["q"], x["k"], x["v"], causal=causal)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_causal_prefix_on_gpu(d):
    w = Workload("prefix", 1, 2, 520, d, seed_base=9)
    x = make_inputs(w, DEV, with_do=False)
    o, lse = fa.forward(x["q"], x["k"], x["v"], causal=True)
    for i in (0, 63, 127, 128, 300, 518):
        k2, v2 = x["k"].clone(), x["v"].clone()
        k2[:, :, i + 1:] = torch.randn_like(k2[:, :, i + 1:].float()).to(torch.bfloat16) * 3
        v2[:, :, i + 1:] = torch.randn_like(v2[:, :, i + 1:].float()).to(torch.bfloat16) * 3
        o2, lse2 = fa.forward(x["q"], k2, v2, causal=True)
        assert torch.equal(o[:, :, : i + 1], o2[:, :, : i + 1])
        assert torch.equal(lse[:, :, : i + 1], lse2[:, :, : i + 1])


def test_fwd_poisoned_outputs_fully_written():
    w = Workload("poison", 2, 3, 333, 64, seed_base=11)
    x = make_inputs(w, DEV, with_do=False)
    o = torch.full_like(x["q"], float("nan"))
    lse = torch.full((2, 3, 333), float("nan"), device=DEV)
    fa.forward(x["q"], x["k"], x["v"], causal=True, out=o, lse=lse)
    fa.check_device_error()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_fwd_writes_nothing_past_the_end():
    """A view into a larger buffer: the rows after N stay untouched."""
    w = Workload("tail", 1, 1, 200, 128, seed_base=12)
    x = make_inputs(w, DEV, with_do=False)
    big = torch.full((1, 1, 256, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    o = big[:, :, :200]
    assert o.is_contiguous()
    lse_big = torch.full((300,), 5.0, device=DEV)
    lse = lse_big[:200].view(1, 1, 200)
    fa.forward(x["q"], x["k"], x["v"], out=o, lse=lse)
    fa.check_device_error()
    assert torch.all(big[:, :, 200:] == 7.0)
    assert torch.all(lse_big[200:] == 5.0)


@pytest.mark.parametrize("scale", [0.0, -0.09, 0.5])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_any_finite_scale(scale, causal):
    """Zero and negative scales are finite values the API accepts."""
    w = Workload("scale", 1, 2, 300, 128, seed_base=13)
    x = make_inputs(w, DEV, with_do=False)
    _run_and_check(x["q"], x["k"], x["v"], causal, scale)


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_many_heads_in_groups(causal):
    """More than 48 heads run in launch groups of 32 with a partial last group
    (B*H = 50): the heads at both ends of each group are right;
    N = 700 (6 Q tiles) and N = 520 (5 Q tiles, so the last pair has a single
    tile) run inside groups."""
    for n in (700, 520):
        w = Workload("groups", 2, 25, n, 64, seed_base=19 + n)
        x = make_inputs(w, DEV, with_do=False)
        heads = [0, 1, 31, 32, 33, 48, 49]
        _run_and_check(x["q"], x["k"], x["v"], causal, w.scale,
                       slices=[(i // 25, i % 25) for i in heads])


def test_fwd_graph_replay_and_concurrent_streams():
    """The persistent forward hands out work from a per-launch counter: a
    captured launch replayed several times, and launches running at the same
    time on several streams, all give the eager single-stream result bit for
    bit (the forward is deterministic)."""
    w = Workload("graph", 2, 8, 1000, 128, seed_base=23)
    x = make_inputs(w, DEV, with_do=False)
    ref_o, ref_lse = fa.forward(x["q"], x["k"], x["v"], causal=True)
    fa.check_device_error()
    o = torch.empty_like(ref_o)
    lse = torch.empty_like(ref_lse)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        fa.forward(x["q"], x["k"], x["v"], causal=True, out=o, lse=lse)
    for _ in range(3):
        o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, ref_o) and torch.equal(lse, ref_lse)
    del g
    streams = [torch.cuda.Stream() for _ in range(4)]
    outs = [(torch.empty_like(ref_o), torch.empty_like(ref_lse)) for _ in streams]
    torch.cuda.synchronize()
    for _ in range(3):
        for s, (oo, ll) in zip(streams, outs):
            with torch.cuda.stream(s):
                oo.fill_(float("nan"))
                fa.forward(x["q"], x["k"], x["v"], causal=True, out=oo, lse=ll)
    torch.cuda.synchronize()
    fa.check_device_error()
    for oo, ll in outs:
        assert torch.equal(oo, ref_o) and torch.equal(ll, ref_lse)
