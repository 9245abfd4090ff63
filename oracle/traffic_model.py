"""Analytic HBM traffic model of naive and FlashAttention-style attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/`` and ``bench.py`` (its ``--traffic`` report) use it.  It shares
no code with the CUDA library.

Source: page "从零实现 FlashAttention-2：分块在线 Softmax".

* Section 文件包含 names ``memory_work(N, d)`` -- an analytic HBM traffic
  model counting full N x N matrix touches and total bytes -- and
  ``print_traffic_table(seq_lengths)`` for N = 128 .. 4096.  The pages do not
  print the formula; what follows is the plainest reading of the surrounding
  text, and the reading is the one stated in the design notes.
* Section 为什么 softmax 强迫使用整行 buffer: the naive kernel sequence computes
  S = Q K^T and stores it, reads it back for the softmax, stores P, then reads
  P for P V.  Counted as one-way transfers of a full N x N matrix, that is
  four touches (S write, S read, P write, P read); the page calls the three
  kernel boundaries they cross "three round trips".
* Section 问题背景: for N = 4K, d = 128 the score matrix alone has about 16 M
  elements, and in FP16 the next kernel must read 32 MB after 32 MB were
  written.  This fixes the element size (2 bytes) and one touch of S
  (N^2 * 2 bytes = 32 MiB at N = 4096).
* Section 验证: the naive N x N touches grow quadratically with N, while the
  FlashAttention path touches no N x N matrix in HBM and its bytes grow
  linearly.  The tiled forward reads Q, K, V and writes O (plus, in this
  library, one fp32 log-sum-exp per row); re-reads of K and V by later query
  tiles are assumed to be served on chip (on B200, from the 126 MB L2), which
  is what makes the count linear.

Per (batch, head) slice, with b = bytes per element:

  io_bytes            = 4 N d b           (read Q, K, V; write O)
  naive_nn_touches    = 4                 (S write, S read, P write, P read)
  naive_nn_bytes      = 4 N^2 b
  naive_bytes         = naive_nn_bytes + io_bytes
                        (reads (2 N^2 + 3 N d) b, writes (2 N^2 + N d) b)
  flash_nn_touches    = 0
  flash_bytes         = io_bytes + N * lse_bytes
                        (reads 3 N d b, writes N d b + N lse_bytes)

Pins (tests/test_traffic_model.py): the page's N = 4K, d = 128 FP16 figures
(16.8 M score elements, 32 MiB per touch of S), and a brute-force count of
every element moved by a simulated three-kernel naive pipeline and by a
simulated tiled forward whose on-chip tiles are never written back.
"""
from __future__ import annotations

from typing import Dict, Iterable, List


def memory_work(N: int, d: int, elem_bytes: int = 2, lse_bytes: int = 0) -> Dict[str, int]:
    """HBM traffic of one attention head (page 2, section 文件包含)."""
    if N < 0 or d < 0 or elem_bytes <= 0 or lse_bytes < 0:
        raise ValueError("N, d >= 0, elem_bytes > 0, lse_bytes >= 0 required")
    nn = N * N
    io = 4 * N * d * elem_bytes
    return {
        "N": N,
        "d": d,
        "s_elements": nn,
        "s_bytes": nn * elem_bytes,
        "io_bytes": io,
        "naive_nn_touches": 4,
        "naive_nn_bytes": 4 * nn * elem_bytes,
        "naive_bytes": 4 * nn * elem_bytes + io,
        "naive_read_bytes": (2 * nn + 3 * N * d) * elem_bytes,
        "naive_write_bytes": (2 * nn + N * d) * elem_bytes,
        "flash_nn_touches": 0,
        "flash_nn_bytes": 0,
        "flash_bytes": io + N * lse_bytes,
        "flash_read_bytes": 3 * N * d * elem_bytes,
        "flash_write_bytes": N * d * elem_bytes + N * lse_bytes,
    }


def traffic_table(seq_lengths: Iterable[int], d: int = 128, elem_bytes: int = 2,
                  lse_bytes: int = 0) -> List[Dict[str, int]]:
    """One ``memory_work`` row per sequence length."""
    return [memory_work(n, d, elem_bytes, lse_bytes) for n in seq_lengths]


def print_traffic_table(seq_lengths: Iterable[int] = (128, 256, 512, 1024, 2048, 4096),
                        d: int = 128, elem_bytes: int = 2) -> str:
    """The O(N^2) vs O(N) table of page 2 (section 文件包含), as text."""
    lines = [f"{'N':>6} {'naive NxN touches':>18} {'naive MiB':>10} {'flash NxN':>10} "
             f"{'flash MiB':>10}"]
    for r in traffic_table(seq_lengths, d, elem_bytes):
        lines.append(f"{r['N']:>6} {r['naive_nn_touches'] * r['s_elements']:>18} "
                     f"{r['naive_bytes'] / 2**20:>10.3f} {r['flash_nn_bytes']:>10} "
                     f"{r['flash_bytes'] / 2**20:>10.3f}")
    text = "\n".join(lines)
    print(text)
    return text
