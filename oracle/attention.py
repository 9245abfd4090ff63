"""Plain float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` leg and its ``--impl reference`` arm) may call it.  It shares
no code, tables or helpers with the CUDA library.

What it computes (one (batch, head) slice at a time; inputs are the
bf16-rounded tensors, up-cast exactly to float64):

* Forward -- page "FlashAttention为什么更快更省显存" (hi-bin.com lesson 16),
  opening formula: ``Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V``.  The
  scale is a parameter (default ``1/sqrt(d)``).
* Row-max subtraction before the exponential -- page "从零实现
  FlashAttention-2：分块在线 Softmax", section 动手实现 (the stable naive
  reference subtracts each row's max before exp).
* Causal mask -- same page, section 提示: the key position greater than the
  query position is masked; the diagonal is kept (section 动手实现, item 4:
  row i attends keys 0..i).
* Stored row statistic -- same page, section 反向传播 keeps "each row's max
  and sum"; here they are folded into one natural-log logsumexp of the scaled
  scores, ``LSE_i = m_i + ln sum_j exp(S_ij - m_i)``.
* Backward -- same page, section 反向传播 names the ``dO . P^T`` term (here
  ``dV = P^T dO``); the remaining terms are the exact gradient of the forward
  above by plain calculus: ``dP = dO V^T``, ``D_i = sum_j P_ij dP_ij``,
  ``dS = P * (dP - D)``, ``dQ = scale dS K``, ``dK = scale dS^T Q``.

Rows are processed in chunks of at most ``row_chunk`` queries purely to bound
memory (N=16384 would otherwise need a 2 GiB score matrix per slice); every
row is still the full softmax of that row, with no tiling of the keys.

Pins (tests/test_oracle.py): the default scale 1/sqrt(d) (exact values,
brute-force loops with the factor written out, and torch's own default), the
page-3 scalar example (50/3, LSE = ln 3),
page-1's running sum, tile-size invariance against the tiled model, causal
row dependence, the +500 shift, an N=1 closed form, brute-force loops,
central finite differences for every gradient, and torch's CPU float64
``scaled_dot_product_attention`` / autograd as an independent library check.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["attention_forward", "attention_backward", "default_scale"]


def default_scale(d: int) -> float:
    """``1/sqrt(d_k)`` from the opening formula of page 1."""
    return 1.0 / math.sqrt(d)


def _as_f64(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float64)
    if a.ndim != 2:
        raise ValueError("oracle works on one [N, d] slice at a time")
    return a


def _scaled_scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool,
                   r0: int, r1: int) -> np.ndarray:
    """S = scale * Q[r0:r1] K^T with -inf where key index > query index."""
    s = scale * (q[r0:r1] @ k.T)
    if causal:
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(k.shape[0])[None, :]
        s = np.where(cols > rows, -np.inf, s)
    return s


def _softmax_rows(s: np.ndarray):
    """Row softmax with the row max subtracted first; returns (P, LSE)."""
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=1, keepdims=True)
    p = e / z
    lse = (m + np.log(z))[:, 0]
    return p, lse


def attention_forward(q, k, v, causal: bool = False, scale: float | None = None,
                      row_chunk: int = 1024):
    """Return ``(O, LSE)`` for one slice: O ``[N, dv]`` and LSE ``[N]`` (float64)."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    n, d = q.shape
    if k.shape != (n, d) or v.shape[0] != n:
        raise ValueError("q, k, v must share N (and q, k share d)")
    if scale is None:
        scale = default_scale(d)
    o = np.empty((n, v.shape[1]), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    for r0 in range(0, n, row_chunk):
        r1 = min(n, r0 + row_chunk)
        p, lse[r0:r1] = _softmax_rows(_scaled_scores(q, k, scale, causal, r0, r1))
        o[r0:r1] = p @ v
    return o, lse


def attention_backward(q, k, v, do, causal: bool = False, scale: float | None = None,
                       row_chunk: int = 1024, o_for_d=None):
    """Return ``(dQ, dK, dV)`` of ``L = sum(dO * O)`` for one slice (float64).

    ``D_i`` is ``sum_j P_ij dP_ij`` by default.  If ``o_for_d`` is given, ``D_i``
    is formed as ``sum_c dO_ic O_ic`` from that O instead -- the same number
    when ``o_for_d`` is the exact output (``sum_j P_ij dO_i.v_j = dO_i.O_i``);
    passing a rounded O measures how much the rounding of the stored output
    alone moves the gradients.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    if o_for_d is not None:
        o_for_d = _as_f64(o_for_d)
    n, d = q.shape
    if scale is None:
        scale = default_scale(d)
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for r0 in range(0, n, row_chunk):
        r1 = min(n, r0 + row_chunk)
        p, _ = _softmax_rows(_scaled_scores(q, k, scale, causal, r0, r1))
        dov = do[r0:r1]
        dv += p.T @ dov                      # dV = P^T dO
        dp = dov @ v.T                       # dP = dO V^T
        if o_for_d is None:
            dsum = np.sum(p * dp, axis=1, keepdims=True)   # D_i = sum_j P_ij dP_ij
        else:
            dsum = np.sum(dov * o_for_d[r0:r1], axis=1, keepdims=True)
        ds = p * (dp - dsum)                 # dS = P o (dP - D)
        dq[r0:r1] = scale * (ds @ k)         # dQ = scale dS K
        dk += scale * (ds.T @ q[r0:r1])      # dK = scale dS^T Q
    return dq, dk, dv
