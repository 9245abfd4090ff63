"""KV-outer (FlashAttention-1 loop order) forward on the GPU: parity with the
float64 oracle at the forward's tolerances, and agreement with fa_fwd."""
import math

import numpy as np
import pytest
import torch

from exact_attention_117_b200 import fa
from exact_attention_117_b200.workloads import (WORKLOADS, Workload, make_inputs, sample_slices,
                                                scalar_case, shift_copy)
from parity_util import bf16_round, bf16_ulp, check_lse, check_o, oracle_fwd_slice, slice_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_and_check(q, k, v, causal, scale, slices=None, workspace=None):
    o, lse = fa.forward_kv_outer(q, k, v, causal=causal, scale=scale, workspace=workspace)
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
@pytest.mark.parametrize("n", [1, 2, 127, 128, 129, 300, 1000])
def test_kv_outer_small_shapes(d, causal, n):
    w = Workload("small", 1, 2, n, d, seed_base=17 + n)
    x = make_inputs(w, DEV, with_do=False)
    _run_and_check(x["q"], x["k"], x["v"], causal, w.scale)


@pytest.mark.parametrize("causal", [False, True])
def test_kv_outer_ragged_and_large(causal):
    w = WORKLOADS["c2r"]
    x = make_inputs(w, DEV, with_do=False)
    idx = sample_slices(w.B * w.H, 3)
    _run_and_check(x["q"], x["k"], x["v"], causal, w.scale, [(i // w.H, i % w.H) for i in idx])
    w = WORKLOADS["c3"]
    x = make_inputs(w, DEV, with_do=False)
    idx = sample_slices(w.B * w.H, 2)
    o, lse = _run_and_check(x["q"], x["k"], x["v"], causal, w.scale,
                            [(i // w.H, i % w.H) for i in idx])
    # same result as the Q-outer kernel up to rounding: each is within the
    # stated O tolerance (1e-2) and LSE tolerance (1e-3) of the oracle
    o2, lse2 = fa.forward(x["q"], x["k"], x["v"], causal=causal, scale=w.scale)
    fa.check_device_error()
    assert float((o.float() - o2.float()).abs().max()) <= 2e-2
    assert float((lse - lse2).abs().max()) <= 2e-3


def test_kv_outer_scalar_shift_and_scales():
    d = 64
    q, k, v, scale = scalar_case(d, DEV)
    o, lse = fa.forward_kv_outer(q, k, v, causal=False, scale=scale)
    fa.check_device_error()
    want = 50.0 / 3.0
    assert abs(float(o[0, 0, 0, 0]) - float(bf16_round(np.array([want]))[0])) <= \
        float(bf16_ulp(np.array([want]))[0])
    assert abs(float(lse[0, 0, 0]) - math.log(3.0)) <= 1e-3
    w = WORKLOADS["c1"]
    x = make_inputs(w, DEV, with_do=False)
    (qb, kb), (qs, ks) = shift_copy(x["q"], x["k"], w.scale)
    ob, lb = _run_and_check(qb, kb, x["v"], False, w.scale)
    os_, ls = _run_and_check(qs, ks, x["v"], False, w.scale)
    assert torch.isfinite(os_.float()).all() and torch.isfinite(ls).all()
    assert float((ls - lb - 500.0).abs().max()) <= 1e-3
    assert float((os_.float() - ob.float()).abs().max()) <= 1e-2
    ws = Workload("scale", 1, 2, 300, 64, seed_base=14)
    xs = make_inputs(ws, DEV, with_do=False)
    for sc in (0.0, -0.09):
        for causal in (False, True):
            _run_and_check(xs["q"], xs["k"], xs["v"], causal, sc)


def test_kv_outer_workspace_contents_do_not_matter():
    w = Workload("ws", 2, 2, 300, 128, seed_base=41)
    x = make_inputs(w, DEV, with_do=False)
    need = fa.kv_outer_workspace_size(2, 2, 300, 128)
    ws = torch.full((need // 4,), float("nan"), dtype=torch.float32, device=DEV)
    _run_and_check(x["q"], x["k"], x["v"], True, w.scale, workspace=ws)
