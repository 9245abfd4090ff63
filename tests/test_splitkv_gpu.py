"""Split-KV forward: key range cut into ranges, merged with the page-3 rule.

Parity against the float64 oracle (the plain definition, no splitting) and
closeness to the single-pass forward, for ragged N, causal masks, and more
splits than key tiles (empty ranges must not disturb the merge).
"""
import numpy as np
import pytest
import torch

from exact_attention_117_b200 import fa
from exact_attention_117_b200.workloads import WORKLOADS, Workload, make_inputs, sample_slices
from parity_util import check_lse, check_o, oracle_fwd_slice, slice_np

P = 0x10000


def test_splitkv_argument_checks():
    from exact_attention_117_b200 import build
    build.build()
    lib = fa.load()
    assert lib.fa_fwd_splitkv_workspace_size(1, 1, 128, 64, 0) == 0
    assert lib.fa_fwd_splitkv_workspace_size(1, 1, 128, 64, 65) == 0
    assert lib.fa_fwd_splitkv_workspace_size(1, 2, 200, 64, 3) == 3 * 2 * 256 * 65 * 4
    ws = lib.fa_fwd_splitkv_workspace_size(1, 1, 128, 64, 2)
    assert lib.fa_fwd_splitkv(P, P, P, P, P, 1, 1, 128, 64, 0, 0.1, 0, P, ws, None) == 2
    assert lib.fa_fwd_splitkv(P, P, P, P, P, 1, 1, 128, 64, 0, 0.1, 2, P, ws - 4, None) == 6
    assert lib.fa_fwd_splitkv(None, P, P, P, P, 1, 1, 128, 64, 0, 0.1, 2, P, ws, None) == 1
    assert lib.fa_fwd_splitkv(P, P, P, P, P, 1, 1, 128, 80, 0, 0.1, 2, P, ws, None) == 3


def _check_vs_oracle(x, o, lse, causal, scale, slices):
    for b, h in slices:
        o_ref, lse_ref = oracle_fwd_slice(x["q"], x["k"], x["v"], b, h, causal, scale)
        check_o(slice_np(o, b, h), o_ref, f"O[{b},{h}]")
        check_lse(lse[b, h].double().cpu().numpy(), lse_ref, f"LSE[{b},{h}]")


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,splits", [(1, 3), (129, 2), (300, 5), (1000, 3), (2048, 4),
                                      (700, 1)])
def test_splitkv_small(d, causal, n, splits):
    w = Workload("split", 1, 2, n, d, seed_base=71 + n)
    x = make_inputs(w, "cuda", with_do=False)
    o, lse = fa.forward_splitkv(x["q"], x["k"], x["v"], causal=causal, num_splits=splits)
    fa.check_device_error()
    _check_vs_oracle(x, o, lse, causal, w.scale, [(0, 0), (0, 1)])
    # and it agrees with the single-pass kernel up to rounding
    o1, lse1 = fa.forward(x["q"], x["k"], x["v"], causal=causal)
    assert float((o1.float() - o.float()).abs().max()) <= 2e-2
    assert float((lse1 - lse).abs().max()) <= 1e-4


@pytest.mark.gpu
@pytest.mark.parametrize("splits", [2, 8])
def test_splitkv_long_context_sampled(splits):
    """The c4 shape (Q * 4, peaky rows), split along the 16384 keys."""
    w = WORKLOADS["c4"]
    x = make_inputs(w, "cuda", with_do=False)
    o, lse = fa.forward_splitkv(x["q"], x["k"], x["v"], causal=True, num_splits=splits)
    fa.check_device_error()
    idx = sample_slices(w.B * w.H, 2)
    _check_vs_oracle(x, o, lse, True, w.scale, [(i // w.H, i % w.H) for i in idx])


@pytest.mark.gpu
def test_splitkv_workspace_contents_do_not_matter():
    w = Workload("splitws", 2, 2, 500, 128, seed_base=79)
    x = make_inputs(w, "cuda", with_do=False)
    need = fa.splitkv_workspace_size(2, 2, 500, 128, 3)
    ws = torch.full((need // 4,), float("nan"), device="cuda")
    o = torch.full_like(x["q"], float("nan"))
    lse = torch.full((2, 2, 500), float("nan"), device="cuda")
    fa.forward_splitkv(x["q"], x["k"], x["v"], causal=True, num_splits=3, out=o, lse=lse,
                       workspace=ws)
    fa.check_device_error()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    _check_vs_oracle(x, o, lse, True, w.scale, [(0, 0), (1, 1)])
