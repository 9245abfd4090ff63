"""Pins of the HBM traffic model (oracle/traffic_model.py) against the page's
worked numbers and a brute-force count of simulated kernel traffic."""
import numpy as np
import pytest

from oracle.traffic_model import memory_work, print_traffic_table, traffic_table


def test_page_figures_n4k_d128_fp16():
    # page 2, section 问题背景: N = 4K, d = 128: about 16 M score elements; in
    # FP16 32 MB are read after 32 MB were written
    w = memory_work(4096, 128, elem_bytes=2)
    assert w["s_elements"] == 16_777_216 and abs(w["s_elements"] / 1e6 - 16) < 1
    assert w["s_bytes"] == 32 * 2**20
    assert w["naive_nn_bytes"] >= 2 * w["s_bytes"]  # at least the write and the read


class _Hbm:
    """Counts every element that crosses the HBM boundary."""

    def __init__(self):
        self.mem = {}
        self.read = 0
        self.written = 0

    def store(self, name, arr):
        self.mem[name] = np.array(arr)
        self.written += self.mem[name].size

    def load(self, name, rows=None, cols=None):
        a = self.mem[name]
        if rows is not None:
            a = a[rows]
        if cols is not None:
            a = a[:, cols]
        self.read += a.size
        return np.array(a)


def _naive_pipeline(hbm, n, d):
    # kernel 1: S = Q K^T, stored; kernel 2: softmax reads S, stores P;
    # kernel 3: O = P V reads P and V, stores O
    q, k = hbm.load("Q"), hbm.load("K")
    hbm.store("S", q @ k.T)
    s = hbm.load("S")
    p = np.exp(s - s.max(axis=1, keepdims=True))
    hbm.store("P", p / p.sum(axis=1, keepdims=True))
    p, v = hbm.load("P"), hbm.load("V")
    hbm.store("O", p @ v)


def _tiled_pipeline(hbm, n, d, br, bc, cache_kv):
    # Q tile outer, K/V tile inner; running (m, l, O) stay on chip; K/V tiles
    # are fetched from HBM once when cache_kv (on-chip / L2 reuse), else per Q tile
    fetched = set()
    out = np.zeros((n, d))
    for i0 in range(0, n, br):
        qi = hbm.load("Q", rows=slice(i0, i0 + br))
        m = np.full(qi.shape[0], -np.inf)
        l = np.zeros(qi.shape[0])
        acc = np.zeros((qi.shape[0], d))
        for j0 in range(0, n, bc):
            if cache_kv and j0 in fetched:
                kj, vj = hbm.mem["K"][j0:j0 + bc], hbm.mem["V"][j0:j0 + bc]
            else:
                kj = hbm.load("K", rows=slice(j0, j0 + bc))
                vj = hbm.load("V", rows=slice(j0, j0 + bc))
                fetched.add(j0)
            s = qi @ kj.T
            m_new = np.maximum(m, s.max(axis=1))
            alpha = np.exp(m - m_new)
            p = np.exp(s - m_new[:, None])
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ vj
            m = m_new
        out[i0:i0 + br] = acc / l[:, None]
    hbm.store("O", out)
    return out


@pytest.mark.parametrize("n,d", [(8, 4), (16, 8), (33, 5)])
def test_brute_force_counts_match_model(n, d):
    rng = np.random.default_rng(n)
    for cache_kv in (True, False):
        for which in ("naive", "tiled"):
            hbm = _Hbm()
            for name in ("Q", "K", "V"):
                hbm.store(name, rng.standard_normal((n, d)))
            hbm.read = hbm.written = 0
            if which == "naive":
                _naive_pipeline(hbm, n, d)
            else:
                _tiled_pipeline(hbm, n, d, 4, 4, cache_kv)
            moved = hbm.read + hbm.written
            w = memory_work(n, d, elem_bytes=1)
            if which == "naive":
                assert moved == w["naive_bytes"]
                assert (hbm.read, hbm.written) == (w["naive_read_bytes"], w["naive_write_bytes"])
                assert "S" in hbm.mem and hbm.mem["S"].shape == (n, n)
            elif cache_kv:
                assert moved == w["flash_bytes"]
                assert (hbm.read, hbm.written) == (w["flash_read_bytes"], w["flash_write_bytes"])
                assert not any(a.shape == (n, n) for a in hbm.mem.values())
            else:
                # without on-chip reuse every Q tile re-reads all of K and V
                tiles = -(-n // 4)
                assert moved == w["flash_bytes"] + (tiles - 1) * 2 * n * d


def test_growth_quadratic_vs_linear():
    rows = traffic_table([128, 256, 512, 1024, 2048, 4096], d=128)
    for a, b in zip(rows, rows[1:]):
        assert b["naive_nn_bytes"] == 4 * a["naive_nn_bytes"]
        assert b["flash_bytes"] == 2 * a["flash_bytes"]
        assert b["flash_nn_bytes"] == 0 and b["flash_nn_touches"] == 0


def test_lse_bytes_and_table_text():
    assert memory_work(100, 64, 2, lse_bytes=4)["flash_bytes"] == 4 * 100 * 64 * 2 + 400
    text = print_traffic_table((128, 4096))
    assert "4096" in text and len(text.splitlines()) == 3
    with pytest.raises(ValueError):
        memory_work(-1, 8)


def test_bench_traffic_report_parses_ncu_csv(tmp_path):
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    hdr = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream",'
           '"Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit",'
           '"Metric Value"')
    rows, kid = [hdr], 0

    def add(name, rd_mb, wr_mb):
        nonlocal kid
        for metric, val in (("dram__bytes_read.sum", rd_mb), ("dram__bytes_write.sum", wr_mb)):
            rows.append(f'"{kid}","1","python","h","{name}","1","7","(1, 1, 1)","(1, 1, 1)","0",'
                        f'"10.0","Command line profiler metrics","{metric}","Mbyte","{val}"')
        kid += 1
    add("randn_kernel", 1.0, 1.0)
    for n in bench.TRAFFIC_N:
        add("void fa::fwd_kernel<128, false, false>(...)", 2.0, 0.5)
        for k in range(3):
            add(f"naive_{k}", 10.0, 5.0)
    path = tmp_path / "t.csv"
    path.write_text("==PROF== noise\n" + "\n".join(rows) + "\n")
    text = bench.traffic_report(str(path))
    lines = text.splitlines()
    assert len(lines) == 2 + len(bench.TRAFFIC_N)
    assert lines[2].startswith("| 128 |") and "/ 2.00" in lines[2] and "/ 30.00" in lines[2]


def test_source_digest_ignores_comments_only():
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    a = "int a = 1;  // one\n/* block\n comment */\nint b = a;\n"
    b = "// header\nint a = 1;\n\nint b = a;   \n"
    c = "int a = 2;\nint b = a;\n"
    assert bench._strip_comments(a) == bench._strip_comments(b)
    assert bench._strip_comments(a) != bench._strip_comments(c)


def test_clock_sampler_decodes_nvml_reasons():
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    # NVML samples (ns, SM MHz, max MHz, reason bits) of a GPU at 1800 of 1965 MHz
    # under the power cap (0x4) with the ignored idle bit (0x1); the first and
    # last fall outside the timed region [100, 400].
    raw = [(50, 1965, 1965, 0x1)] + [(t, 1800, 1965, 0x4 | 0x1) for t in (100, 250, 400)] \
        + [(450, 1965, 1965, 0x8)]
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.samples, c.source = [], "nvml"
    c.add_nvml_samples(raw, 100, 400)
    s = c.summary()
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"] and s["source"] == "nvml"


def test_roofline_entry_for_the_dominant_kernel():
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    totals = {"fwd": 3.0, "bwd_main": 8.0, "bwd_pre": 0.6}
    per = {"fwd": 0.15, "bwd_main": 0.4, "bwd_pre": 0.03}
    r = bench.roofline_entry(totals, per, {"fwd": 137.4e9, "bwd_main": 343.6e9},
                             {"bf16_tflops": 1663.5}, "measured", lambda k: 683e6)
    assert r["kernel"] == "bwd_main" and r["bound"] == "tensor" and r["traffic"] == 683e6
    assert abs(r["achieved"] - 343.6e9 / 0.4e-3 / 1e12) < 1e-9
    assert abs(r["frac"] - r["achieved"] / 1663.5) < 1e-12
    assert abs(r["frac_of_nominal"] - r["achieved"] / 2250.0) < 1e-12
    r = bench.roofline_entry({"bwd_pre": 1.0, "fwd": 0.5}, {"bwd_pre": 0.1, "fwd": 0.05},
                             {"fwd": 1e9}, {"hbm_gbs": 6542.4}, "measured", lambda k: None)
    assert r["bound"] == "hbm" and r["frac"] is None


def test_clock_sampler_keeps_nearest_sample_for_a_short_region():
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    raw = [(0, 1900, 1965, 0x0), (1000, 1700, 1965, 0x40)]
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.samples, c.source = [], "nvml"
    c.add_nvml_samples(raw, 700, 800)  # no sample inside: the one at 1000 is nearest
    s = c.summary()
    assert s["samples"] == 1 and s["sm_mhz"] == 1700
    assert s["reasons"] == ["hw_thermal_slowdown"]
