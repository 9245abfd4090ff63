"""CPU model of the tiled online-softmax algebra (float64).

TEST INFRASTRUCTURE ONLY (same import rule as ``oracle.attention``).  It is
not used for GPU parity; it pins the tile algebra the kernels rely on against
the plain definition in ``oracle.attention``.

It follows, step by step:

* page "FlashAttention 为什么能节省显存并提速,是否改变注意力结果?"
  (mianstack.com q-0277), section 难点在于分块后softmax如何归一: each row keeps
  a running max ``m``, exp-sum ``l`` and un-normalised output ``u``; a new
  block contributes its own ``(m_b, l_b, u_b)`` taken relative to ``m_b`` and
  is merged by

      m_new = max(m, m_b)
      l_new = exp(m - m_new) * l + exp(m_b - m_new) * l_b
      u_new = exp(m - m_new) * u + exp(m_b - m_new) * u_b

  and the output is ``u / l`` once all blocks are in;
* page "从零实现 FlashAttention-2：分块在线 Softmax", sections 在线 softmax
  and 从 FlashAttention-1 到 FlashAttention-2: the Q-tile loop is outside, the
  K/V-tile loop inside, causal masking happens inside the tile (section 提示),
  and tiles that lie wholly above the diagonal are skipped (section
  反向传播, last paragraph: only lower-triangular tiles are computed);
* page "FlashAttention为什么更快更省显存", section Softmax 分块后怎么保持结果不变:
  the ``[1, 2, 3]`` running-sum example (``running_stats``).

``sum_of_block_outputs`` is the WRONG method that page 3 warns about (each
block normalised on its own, then added); it exists only as a negative
control for the tests.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["flash_forward_tiled", "running_stats", "merge", "sum_of_block_outputs"]


def _exp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """exp(a - b) with exp(-inf - (-inf)) taken as 0 (an empty block)."""
    with np.errstate(invalid="ignore"):
        x = np.exp(a - b)
    return np.where(np.isneginf(a), 0.0, x)


def merge(m, l, u, m_b, l_b, u_b):
    """One application of the page-3 merge rule; ``u`` may be a vector per row."""
    m_new = np.maximum(m, m_b)
    a = _exp_diff(m, m_new)
    b = _exp_diff(m_b, m_new)
    l_new = a * l + b * l_b
    if np.ndim(u) > np.ndim(l):
        u_new = a[..., None] * u + b[..., None] * u_b
    else:
        u_new = a * u + b * u_b
    return m_new, l_new, u_new


def _block_stats(s: np.ndarray, v: np.ndarray):
    """(m_b, l_b, u_b) of one score block, all relative to the block's own max."""
    m_b = np.max(s, axis=1)
    p = _exp_diff(s, m_b[:, None])
    return m_b, p.sum(axis=1), p @ v


def flash_forward_tiled(q, k, v, br: int, bc: int, causal: bool = False,
                        scale: float | None = None):
    """Tiled forward with the merge rule; returns ``(O, LSE)`` like the oracle."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    n, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.empty((n, v.shape[1]))
    lse = np.empty(n)
    for r0 in range(0, n, br):                     # Q tile: outer loop
        r1 = min(n, r0 + br)
        m = np.full(r1 - r0, -np.inf)
        l = np.zeros(r1 - r0)
        u = np.zeros((r1 - r0, v.shape[1]))
        for c0 in range(0, n, bc):                 # K/V tile: inner loop
            c1 = min(n, c0 + bc)
            if causal and c0 > r1 - 1:             # tile wholly above the diagonal
                break
            s = scale * (q[r0:r1] @ k[c0:c1].T)
            if causal:
                rows = np.arange(r0, r1)[:, None]
                cols = np.arange(c0, c1)[None, :]
                s = np.where(cols > rows, -np.inf, s)
            m, l, u = merge(m, l, u, *_block_stats(s, v[c0:c1]))
        o[r0:r1] = u / l[:, None]
        lse[r0:r1] = m + np.log(l)
    return o, lse


def running_stats(blocks):
    """Running ``(m, l)`` of one score row fed block by block.

    ``blocks`` is a list of 1-D score arrays; returns the state after each.
    """
    m, l = -np.inf, 0.0
    out = []
    for blk in blocks:
        blk = np.asarray(blk, np.float64)
        m_b = float(np.max(blk))
        l_b = float(np.sum(np.exp(blk - m_b)))
        m, l, _ = merge(np.float64(m), np.float64(l), np.float64(0.0),
                        np.float64(m_b), np.float64(l_b), np.float64(0.0))
        m, l = float(m), float(l)
        out.append((m, l))
    return out


def sum_of_block_outputs(scores, values, block: int):
    """Negative control: normalise each block alone and add the block outputs."""
    scores = np.asarray(scores, np.float64)
    values = np.asarray(values, np.float64)
    total = 0.0
    for c0 in range(0, scores.shape[0], block):
        s = scores[c0:c0 + block]
        w = np.exp(s - s.max())
        total = total + (w / w.sum()) @ values[c0:c0 + block]
    return total
