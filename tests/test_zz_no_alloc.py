"""fa_bwd_noalloc: the backward pass with nothing allocated on the call path.

Some callers cannot call cudaMalloc when they run the backward: a host
framework that owns all device memory through its own pool, or a
latency-critical loop that must not allocate or free after start-up (cudaFree
can synchronise the device).  fa_bwd_noalloc serves them with a fixed scratch
array inside the library instead of a caller-provided workspace.  These tests
check that it gives the same gradients as fa_bwd on two calls in a row (the
second call must not see leftovers of the first) and that a problem too large
for the fixed array is refused before anything is launched.

This file is named so that pytest collects it last.
"""
import pytest
import torch

from exact_attention_117_b200 import fa
from exact_attention_117_b200.workloads import Workload, make_inputs
from parity_util import GRAD_REL_L2, rel_l2

P = 0x10000  # fake, never-dereferenced, 16-byte aligned address


def test_noalloc_refuses_problems_larger_than_its_scratch():
    from exact_attention_117_b200 import build
    build.build()
    fa.load()
    # B=1, H=32, N=16384, d=128 needs 256 MiB of scratch: refused, nothing launched
    assert fa.workspace_size(1, 32, 16384, 128) > fa.NOALLOC_SCRATCH_BYTES
    st = fa.bwd_noalloc_raw(P, P, P, P, P, P, P, P, P, 1, 32, 16384, 128, True, 0.088, 0)
    assert st == 6  # FA_ERR_WORKSPACE
    # argument checks come first, exactly as in fa_bwd
    assert fa.bwd_noalloc_raw(None, P, P, P, P, P, P, P, P, 1, 1, 128, 64, 0, 0.1, 0) == 1
    assert fa.bwd_noalloc_raw(P, P, P, P, P, P, P, P, P, 1, 1, 128, 80, 0, 0.1, 0) == 3


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    # the second call's problem fits inside the region the first call wrote, so
    # it runs over the first call's leftovers; the third repeats the first
    # shape over the second call's leftovers
    a = Workload("noalloc_a", 2, 4, 1000, 128, seed_base=61)
    b = Workload("noalloc_b", 1, 3, 700, 64, seed_base=62)
    assert fa.workspace_size(b.B, b.H, b.N, b.d) <= fa.workspace_size(a.B, a.H, a.N, a.d)
    cases = [a, b, Workload("noalloc_a2", 2, 4, 1000, 128, seed_base=63)]
    for w, causal in zip(cases, (True, False, True)):
        assert fa.workspace_size(w.B, w.H, w.N, w.d) <= fa.NOALLOC_SCRATCH_BYTES
        x = make_inputs(w, "cuda")
        o, lse = fa.forward(x["q"], x["k"], x["v"], causal=causal, scale=w.scale)
        ref = fa.backward(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal,
                          scale=w.scale)
        got = [torch.full_like(x["q"], float("nan")) for _ in range(3)]
        fa.backward_noalloc(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal,
                            scale=w.scale, dq=got[0], dk=got[1], dv=got[2])
        fa.check_device_error()
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            assert torch.isfinite(g.float()).all(), name
            err = rel_l2(g.double().cpu().numpy(), r.double().cpu().numpy())
            assert err <= GRAD_REL_L2, f"{w.name} {name}: rel-L2 {err:.3e}"
        # dK and dV have one writer per key tile and no atomics: identical bits
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])
