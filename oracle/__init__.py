"""fp64 CPU oracle for the hybrid linear/softmax token mixer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the package's
`smoke()` check and the bench's CPU-baseline / reference legs may import this
package. The CUDA library never calls it, and it imports nothing of the CUDA
path: the only module both sides share is `workloads` (seeded inputs, no
method arithmetic).

What it computes, and where each step comes from. The pages (web summaries of
"SANA-Video 2.0: Hybrid Linear Attention with Attention Residuals for
Efficient Video Generation") fix the structure but print no formula:

* three of every four layers are gated linear attention with a fixed-size
  state and O(N) cost; every fourth layer is a gated softmax "anchor"
  [lode.cx summary, "How It Works"; ai-papers.net summary, section
  "ハイブリッド線形アテンション"; SANA-Video 2.0 abstract on the
  thelatestinai.com listing];
* Block Attention Residuals group 8 consecutive layers into a block and route
  the summaries of completed blocks into later linear layers through a
  shared-query router whose projection is shared across depth
  [ai-papers.net summary, section "ブロックアテンション残差"; lode.cx summary,
  "How It Works"].

The formulas below are the readings this library commits to where the pages
are silent (each is marked "reading"):

  phi(x) = max(x, 0)                                   (feature map, reading)
  S = sum_t phi(K_t)^T V_t,  z = sum_t phi(K_t)          per (batch, head)
  A_t = phi(Q_t) S / (phi(Q_t) . z + eps)               (non-causal, reading)
  A_t = sum_s softmax_s(Q_t . K_s / sqrt(d)) V_s         (non-causal)
  Y = A * sigmoid(G)                                     (per-channel output gate, reading)
  write-gated variant: token t's write into the state of head h is scaled by
     omega_t = sigmoid(W_t) (one logit per token and head, W = u W_w^T):
     S = sum_t omega_t phi(K_t)^T V_t,  z = sum_t omega_t phi(K_t)      (reading)
  [Q | K | V | G] = u W_qkvg^T,  o = Y W_o^T,  h_l = h_{l-1} + o
  router (linear layers of block c >= 2):
     q = h_{l-1} W_r^T
     alpha_{t,b} = softmax_b( q_t . s_b[t] / sqrt(D) ),  b < c
     u = h_{l-1} + sum_b alpha_{t,b} s_b[t]              (additive mix, reading)
  block summary s_c = h_{8c} (residual stream after the block's last layer, reading)

All arithmetic is numpy float64. Inputs are the exact values handed to the GPU
(already rounded to the run dtype), upcast to fp64. Every function here is
pinned by a CPU test against something other than itself (brute force,
closed forms, library routines, invariants); none is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "phi", "split_heads", "merge_heads", "write_weights", "lin_state", "lin_readout", "lin_core",
    "lin_core_bruteforce", "softmax_core", "sigmoid", "gate", "linear_attn",
    "softmax_anchor", "project", "route", "layer_kind", "block_of", "stack",
]


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def phi(x: np.ndarray) -> np.ndarray:
    """Feature map of the linear layers: ReLU (reading; the pages name only a
    fixed-size state [ai-papers.net summary, section "ハイブリッド線形アテンション"])."""
    return np.maximum(_f64(x), 0.0)


def split_heads(x: np.ndarray, H: int) -> np.ndarray:
    """[B, N, H*d] -> [B, H, N, d]; head h owns columns [h*d, (h+1)*d)."""
    B, N, D = x.shape
    assert D % H == 0
    return _f64(x).reshape(B, N, H, D // H).transpose(0, 2, 1, 3)


def merge_heads(a: np.ndarray) -> np.ndarray:
    """[B, H, N, d] -> [B, N, H*d]."""
    B, H, N, d = a.shape
    return a.transpose(0, 2, 1, 3).reshape(B, N, H * d)


# ---------------------------------------------------------------------------
# gated linear attention [ai-papers.net summary, section "ハイブリッド線形アテンション":
# a fixed-size state, O(N) in the number of tokens]
# ---------------------------------------------------------------------------


def write_weights(wgate, H: int) -> np.ndarray:
    """omega [B, H, N, 1] = sigmoid of the write-gate logits [B, N, H].

    The gate sets how much each token writes into the fixed-size state
    [ai-papers.net summary, section "ハイブリッド線形アテンション"]; the reading
    taken here is one logit per token and head, scaling that token's whole
    write (its term in S and in z)."""
    w = _f64(wgate)
    assert w.ndim == 3 and w.shape[2] == H
    return sigmoid(w).transpose(0, 2, 1)[..., None]


def lin_state(k: np.ndarray, v: np.ndarray, H: int, wgate=None) -> Tuple[np.ndarray, np.ndarray]:
    """State of every (batch, head) over all N tokens.

    S[b, h] = sum_t phi(K_t)^T V_t   (d x d),   z[b, h] = sum_t phi(K_t)   (d).
    With write-gate logits wgate [B, N, H] every token's term is scaled by
    omega_t = sigmoid(wgate[b, t, h]) in both sums.
    Returns S [B, H, d, d] and z [B, H, d]. (The sum over tokens is a plain
    matrix product phi(K)^T V.)"""
    fk = phi(split_heads(k, H))
    if wgate is not None:
        fk = fk * write_weights(wgate, H)
    vh = split_heads(v, H)
    S = np.matmul(np.swapaxes(fk, -1, -2), vh)
    z = fk.sum(axis=2)
    return S, z


def lin_readout(q: np.ndarray, S: np.ndarray, z: np.ndarray, H: int, eps: float) -> np.ndarray:
    """A_t = phi(Q_t) S / (phi(Q_t) . z + eps) for every token row of q.

    q may hold any subset of rows; S and z come from `lin_state`."""
    fq = phi(split_heads(q, H))
    num = np.matmul(fq, S)
    den = np.matmul(fq, z[..., None])[..., 0] + eps
    return merge_heads(num / den[..., None])


def lin_core(q, k, v, H: int, eps: float = 1e-6, wgate=None) -> np.ndarray:
    """Normalised non-causal linear attention, associative (state) form."""
    S, z = lin_state(k, v, H, wgate)
    return lin_readout(q, S, z, H, eps)


def lin_core_bruteforce(q, k, v, H: int, eps: float = 1e-6, wgate=None) -> np.ndarray:
    """The same quantity in its O(N^2) pairwise form, with an explicit loop over
    query tokens: A_t = sum_s w_ts V_s / (sum_s w_ts + eps), w_ts = phi(Q_t).phi(K_s),
    times omega_s = sigmoid(wgate[b, s, h]) when write-gate logits are given.
    Used only to pin `lin_core` on small N."""
    fq, fk, vh = phi(split_heads(q, H)), phi(split_heads(k, H)), split_heads(v, H)
    B, _, Nq, d = fq.shape
    Nk = fk.shape[2]
    out = np.zeros((B, H, Nq, vh.shape[-1]))
    for b in range(B):
        for h in range(H):
            om = np.ones(Nk) if wgate is None else np.array(
                [1.0 / (1.0 + math.exp(-float(wgate[b, s, h]))) for s in range(Nk)])
            for t in range(Nq):
                w = (fk[b, h] @ fq[b, h, t]) * om       # w_ts for all s
                out[b, h, t] = (w @ vh[b, h]) / (w.sum() + eps)
    return merge_heads(out)


# ---------------------------------------------------------------------------
# gated softmax anchor [lode.cx summary, "How It Works": every fourth layer is
# gated softmax, which keeps exact token relations]
# ---------------------------------------------------------------------------


def softmax_core(q, k, v, H: int, scale: Optional[float] = None, row_block: int = 256) -> np.ndarray:
    """A_t = sum_s softmax_s(Q_t . K_s * scale) V_s, non-causal, scale = 1/sqrt(d).

    Scores are formed for `row_block` query rows at a time (an N x N fp64 score
    matrix per head would not fit in memory at video lengths); each row block is
    the plain definition: subtract the row max, exponentiate, normalise."""
    qh, kh, vh = split_heads(q, H), split_heads(k, H), split_heads(v, H)
    d = qh.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    B, _, Nq, _ = qh.shape
    out = np.empty((B, H, Nq, vh.shape[-1]))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, Nq, row_block):
                s = (qh[b, h, r0:r0 + row_block] @ kh[b, h].T) * scale
                s -= s.max(axis=1, keepdims=True)
                p = np.exp(s)
                out[b, h, r0:r0 + row_block] = (p @ vh[b, h]) / p.sum(axis=1, keepdims=True)
    return merge_heads(out)


# ---------------------------------------------------------------------------
# output gate [lode.cx summary, "How It Works": both layer kinds are gated]
# ---------------------------------------------------------------------------


def sigmoid(g) -> np.ndarray:
    """1 / (1 + exp(-g)), evaluated without overflow for large |g|."""
    g = _f64(g)
    e = np.exp(-np.abs(g))
    return np.where(g >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def gate(a, g) -> np.ndarray:
    """Y = A * sigmoid(G), per channel (reading: a D-wide output gate)."""
    return _f64(a) * sigmoid(g)


def linear_attn(q, k, v, g, H: int, eps: float = 1e-6, residual=None, wgate=None) -> np.ndarray:
    """Gated linear-attention layer core: Y = lin_core(Q, K, V) * sigmoid(G) (+ residual);
    wgate [B, N, H] (optional) are the write-gate logits of the state."""
    y = gate(lin_core(q, k, v, H, eps, wgate), g)
    return y if residual is None else y + _f64(residual)


def softmax_anchor(q, k, v, g, H: int, scale: Optional[float] = None, residual=None) -> np.ndarray:
    """Gated softmax anchor core: Y = softmax_core(Q, K, V) * sigmoid(G) (+ residual)."""
    y = gate(softmax_core(q, k, v, H, scale), g)
    return y if residual is None else y + _f64(residual)


# ---------------------------------------------------------------------------
# projections and the residual stream
# ---------------------------------------------------------------------------


def project(u, w) -> np.ndarray:
    """y = u W^T with W in the [out, in] layout of a linear layer."""
    return _f64(u) @ _f64(w).T


# ---------------------------------------------------------------------------
# Block Attention Residuals with the shared-query router
# [ai-papers.net summary, section "ブロックアテンション残差": 8-layer blocks,
# completed-block summaries routed into later linear layers, one query
# projection shared across depth]
# ---------------------------------------------------------------------------


def route(h, summaries: Sequence[np.ndarray], w_r) -> Tuple[np.ndarray, np.ndarray]:
    """Router input of a linear layer in a later block.

    q_t = h_t W_r^T; alpha_{t,b} = softmax over the completed blocks b of
    (q_t . s_b[t]) / sqrt(D); u = h + sum_b alpha_{t,b} s_b[t].
    Returns u [B, N, D] and alpha [B, N, n_blocks]."""
    h = _f64(h)
    D = h.shape[-1]
    q = h @ _f64(w_r).T
    logits = np.stack([np.einsum("bnd,bnd->bn", q, _f64(s)) for s in summaries], axis=-1)
    logits /= math.sqrt(D)
    logits -= logits.max(axis=-1, keepdims=True)
    e = np.exp(logits)
    alpha = e / e.sum(axis=-1, keepdims=True)
    r = sum(alpha[..., i:i + 1] * _f64(s) for i, s in enumerate(summaries))
    return h + r, alpha


def layer_kind(l: int, softmax_period: int = 4, all_softmax: bool = False) -> str:
    """'softmax' at every softmax_period-th layer (1-based), else 'linear'
    [lode.cx summary, "How It Works": every fourth layer is gated softmax]."""
    if all_softmax or (softmax_period > 0 and l % softmax_period == 0):
        return "softmax"
    return "linear"


def block_of(l: int, attnres_block: int) -> int:
    """1-based block index of layer l: blocks of `attnres_block` consecutive layers."""
    return (l + attnres_block - 1) // attnres_block


def stack(x, w_qkvg: Sequence[np.ndarray], w_o: Sequence[np.ndarray], w_r, H: int,
          softmax_period: int = 4, attnres_block: int = 8, all_softmax: bool = False,
          eps: float = 1e-6, keep_trace: bool = False, w_wg: Optional[Sequence] = None,
          on_layer: Optional[Callable] = None):
    """The hybrid token mixer: tokens in, mixed tokens out.

    h_0 = x; for l = 1..L: u = routed or plain input, [Q|K|V|G] = u W_qkvg[l]^T,
    Y = gated linear or softmax core, h_l = h_{l-1} + Y W_o[l]^T.
    Summaries s_c = h_{8c} are kept after each completed block; linear layers of
    block c >= 2 read the router output (anchors and block-1 layers read h_{l-1}).
    With w_wg (L weights [H, D]; anchors' entries unused) the linear layers are
    write-gated, the logits being W = u W_wg[l]^T.

    Returns y = h_L and, when keep_trace, a dict of per-layer lists
    u, Y, o (each [B, N, D]) and alpha ([B, N, c-1] or None), plus kinds.
    on_layer, if given, is called after each layer as
    on_layer(l, kind, u, Y, o, alpha) (an observer: it changes nothing), so a
    caller can inspect every layer of a stack too large to keep whole."""
    h = _f64(x).copy()
    D = h.shape[-1]
    L = len(w_qkvg)
    summaries: List[np.ndarray] = []
    trace: Dict[str, list] = {"u": [], "Y": [], "o": [], "alpha": [], "kind": []}
    for l in range(1, L + 1):
        kind = layer_kind(l, softmax_period, all_softmax)
        alpha = None
        if kind == "linear" and attnres_block > 0 and block_of(l, attnres_block) >= 2:
            c = block_of(l, attnres_block)
            u, alpha = route(h, summaries[:c - 1], w_r)
        else:
            u = h
        qkvg = project(u, w_qkvg[l - 1])
        q, k, v, g = (qkvg[..., i * D:(i + 1) * D] for i in range(4))
        if kind == "linear":
            wl = None if w_wg is None else project(u, w_wg[l - 1])
            Y = linear_attn(q, k, v, g, H, eps, wgate=wl)
        else:
            Y = softmax_anchor(q, k, v, g, H)
        o = project(Y, w_o[l - 1])
        h = h + o
        if attnres_block > 0 and l % attnres_block == 0:
            summaries.append(h.copy())
        if on_layer is not None:
            on_layer(l, kind, u, Y, o, alpha)
        if keep_trace:
            trace["u"].append(u)
            trace["Y"].append(Y)
            trace["o"].append(o)
            trace["alpha"].append(alpha)
            trace["kind"].append(kind)
    return (h, trace) if keep_trace else h
