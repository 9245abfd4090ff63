"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before launching anything (no GPU needed)."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from exact_attention_117_b200 import build, fa
    build.build()
    return fa.load()


def _declared_functions():
    with open(os.path.join(ROOT, "include", "fa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert "fa_fwd" in names and "fa_bwd" in names
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(10):
        s = lib.fa_status_string(code)
        assert s and isinstance(s, bytes)
    assert lib.fa_status_string(0) == b"ok"
    assert lib.fa_version() >= 100


# fake, never-dereferenced device addresses (16-byte aligned)
P = 0x10000


def _fwd(lib, q=P, k=P, v=P, o=P, lse=P, B=1, H=1, N=128, d=64, causal=0, scale=0.125):
    from exact_attention_117_b200 import fa
    return fa.fwd_raw(q, k, v, o, lse, B, H, N, d, causal, scale, 0)


def _bwd(lib, ptrs=None, ws=P, ws_bytes=None, B=1, H=1, N=128, d=64, scale=0.125, raw=None):
    from exact_attention_117_b200 import fa
    p = ptrs or [P] * 9
    if ws_bytes is None:
        ws_bytes = fa.workspace_size(B, H, N, d) if d in (64, 128) and N > 0 else 1 << 20
    return (raw or fa.bwd_raw)(*p[:6], *p[6:9], ws, ws_bytes, B, H, N, d, 0, scale, 0)


def test_fwd_rejects_null(lib):
    for i in range(5):
        args = [P] * 5
        args[i] = None
        assert _fwd(lib, *args) == 1


@pytest.mark.parametrize("B,H,N", [(0, 1, 1), (1, 0, 1), (1, 1, 0), (-1, 1, 1), (1, 1, -5)])
def test_fwd_rejects_shape(lib, B, H, N):
    assert _fwd(lib, B=B, H=H, N=N) == 2


def test_shapes_beyond_the_grid_limits(lib):
    # B*H*ceil(N/128) above 2^31-1 CTAs: refused before any launch, although
    # B*H and N are each within their own limits
    assert _fwd(lib, B=1 << 20, H=1, N=1 << 18) == 2
    assert _bwd(lib, B=1 << 20, H=1, N=1 << 18, ws_bytes=1 << 62) == 2
    # the sequence-length bound: N up to 65535 * 128
    assert _fwd(lib, N=65535 * 128 + 1) == 2


@pytest.mark.parametrize("d", [0, 1, 32, 96, 256])
def test_fwd_rejects_head_dim(lib, d):
    assert _fwd(lib, d=d) == 3


def test_fwd_rejects_misaligned(lib):
    assert _fwd(lib, q=P + 8) == 4
    assert _fwd(lib, o=P + 2) == 4
    assert _fwd(lib, lse=P + 2) == 4


@pytest.mark.parametrize("scale", [math.nan, math.inf, -math.inf])
def test_fwd_rejects_scale(lib, scale):
    assert _fwd(lib, scale=scale) == 5


@pytest.mark.parametrize("entry", ["bwd_raw", "bwd_deterministic_raw"])
def test_bwd_checks(lib, entry):
    from exact_attention_117_b200 import fa
    raw = getattr(fa, entry)
    for i in range(9):
        p = [P] * 9
        p[i] = None
        assert _bwd(lib, ptrs=p, raw=raw) == 1
    assert _bwd(lib, N=0, raw=raw) == 2
    assert _bwd(lib, d=80, raw=raw) == 3
    p = [P] * 9
    p[7] = P + 4
    assert _bwd(lib, ptrs=p, raw=raw) == 4
    assert _bwd(lib, scale=math.nan, raw=raw) == 5
    need = fa.workspace_size(1, 1, 128, 64)
    assert _bwd(lib, ws=None, raw=raw) == 6
    assert _bwd(lib, ws_bytes=need - 1, raw=raw) == 6


def test_workspace_size(lib):
    from exact_attention_117_b200 import fa
    # fp32 dQ accumulator [B,H,Np,d] + two fp32 row vectors, Np = ceil(N/128)*128
    assert fa.workspace_size(1, 1, 128, 64) == 128 * 64 * 4 + 2 * 512
    assert fa.workspace_size(2, 3, 1000, 128) == 6 * 1024 * 128 * 4 + 2 * 6 * 1024 * 4
    assert fa.workspace_size(1, 1, 0, 64) == 0
    assert fa.workspace_size(1, 1, 10, 72) == 0


def test_timing_state_machine(lib):
    assert lib.fa_timing_end(None, None) == 9
    assert lib.fa_timing_begin() == 0
    assert lib.fa_timing_begin() == 9
    from exact_attention_117_b200 import fa
    nk = len(fa.KERNELS)  # FA_KERNEL_COUNT entries
    ms = (ctypes.c_float * nk)()
    cnt = (ctypes.c_int * nk)()
    assert lib.fa_timing_end(ms, cnt) == 0
    assert list(cnt) == [0] * nk


def test_binding_fails_loudly_without_library(monkeypatch):
    from exact_attention_117_b200 import fa
    monkeypatch.setattr(fa, "_lib", None)
    monkeypatch.setattr(fa, "LIB_PATH", "/nonexistent/libfa_b200.so")
    with pytest.raises(RuntimeError, match="not built"):
        fa.load()


def test_binding_kernel_list_matches_header():
    from exact_attention_117_b200 import fa
    with open(os.path.join(ROOT, "include", "fa.h")) as f:
        text = f.read()
    count = int(re.search(r"FA_KERNEL_COUNT\s*=\s*(\d+)", text).group(1))
    assert count == len(fa.KERNELS)


def test_product_path_and_oracle_are_separate():
    """The package never imports the oracle (no CPU fallback can route through
    it), and the oracle never loads the CUDA library."""
    pkg = os.path.join(ROOT, "exact_attention_117_b200")
    for dirpath, _, files in os.walk(pkg):
        for name in files:
            if name.endswith(".py"):
                text = open(os.path.join(dirpath, name)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", text, re.M), name
    for name in os.listdir(os.path.join(ROOT, "oracle")):
        if name.endswith(".py"):
            text = open(os.path.join(ROOT, "oracle", name)).read()
            assert "exact_attention_117_b200" not in text and "libfa_b200" not in text, name
            assert "torch.cuda" not in text and ".cuda(" not in text, name
