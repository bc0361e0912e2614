"""Oracle parity of whole stacks at full size: the 720p-shaped 24-layer stack
(B = 1, N = 19,320, H = 24, d = 128, D = 3,072; 18 gated linear layers, 6 gated
softmax anchors, 3 AttnRes blocks of 8 with the shared-query router) and the
long-video 4-layer group (N = 37,720, 3 linear + 1 anchor), with the seeded
weights the bench times.

The layer layout follows the lode.cx summary ("How It Works": three gated
linear layers to one gated softmax anchor) and the AttnRes blocks the
ai-papers.net summary (section "ブロックアテンション残差": 8-layer blocks, the
completed blocks' summaries mixed into later layers by a router whose
projection is shared across depth).

The GPU runs the whole stack once with every layer traced (Y_l, o_l, and the
router weights alpha_l of the routed layers). The fp64 oracle then runs the
same stack from the same x and weights, and each of its layers is compared
with the trace as soon as it is computed (the oracle's per-layer observer), so
a full fp64 trace (tens of GB) is never held. After the last layer, the fp32
residual update h_L - x = sum_l o_l and y are compared. The oracle's pass takes
minutes on the host cores."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from tests._util import assert_close, to_host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import softmax_attention_video_gated_b200 as sva  # noqa: E402


class _Fp64Layers:
    """Per-layer weights held on the host in bf16; the oracle gets layer l's
    exact values in fp64 only when it reads that layer."""

    def __init__(self, ts):
        self.ts = ts

    def __len__(self):
        return len(self.ts)

    def __getitem__(self, i):
        return self.ts[i].to(torch.float64).numpy()


def _routed_blocks(w, l):
    """Completed blocks layer l mixes (0 when the layer is not routed)."""
    kind = O.layer_kind(l, w.softmax_period)
    if kind == "linear" and w.attnres_block > 0 and O.block_of(l, w.attnres_block) >= 2:
        return O.block_of(l, w.attnres_block) - 1
    return 0


def _whole_stack_parity(w):
    B, N, D, L = w.B, w.N, w.D, w.L
    std = w.weight_std
    wq = [W.normal_torch((4 * D, D), std, w.seed, W.TAG_WQKVG + l, "bf16") for l in range(1, L + 1)]
    wo = [W.normal_torch((D, D), std, w.seed, W.TAG_WO + l, "bf16") for l in range(1, L + 1)]
    wr = W.normal_torch((D, D), std, w.seed, W.TAG_WR, "bf16")
    x = W.normal_torch((B, N, D), 1.0, w.seed, W.TAG_X, "bf16")
    trace_o = [torch.empty(B * N, D, device="cuda", dtype=torch.float32) for _ in range(L)]
    trace_y = [torch.empty(B * N, D, device="cuda", dtype=torch.bfloat16) for _ in range(L)]
    nb = [_routed_blocks(w, l) for l in range(1, L + 1)]
    trace_alpha = [torch.empty(B * N, n, device="cuda", dtype=torch.float32) if n else None
                   for n in nb]
    st = sva.Stack(wq, wo, wr, B, N, w.H, softmax_period=w.softmax_period,
                   attnres_block=w.attnres_block, trace_o=trace_o, trace_y=trace_y,
                   trace_alpha=trace_alpha)
    y = torch.empty_like(x)
    ws = sva.sva_hybrid_stack_fwd(st, x, y)
    assert sva.sva_check_device_status(ws) == sva.SVA_OK
    del ws
    # the fp32 residual update h_L - x, summed layer by layer in fp64
    update = torch.zeros(B * N, D, device="cuda", dtype=torch.float64)
    for t in trace_o:
        update += t
    update = to_host(update).reshape(B, N, D)

    checked = []
    worst = {"Y": 0.0, "o": 0.0, "alpha": 0.0}

    def on_layer(l, kind, u, Y, o, alpha):
        i = l - 1
        r = assert_close(to_host(trace_y[i]).reshape(Y.shape), Y, "bf16", f"Y_{l} ({kind})")
        worst["Y"] = max(worst["Y"], r)
        r = assert_close(to_host(trace_o[i]).reshape(o.shape), o, "bf16", f"o_{l} ({kind})")
        worst["o"] = max(worst["o"], r)
        if nb[i]:
            assert alpha is not None and alpha.shape[-1] == nb[i]
            r = assert_close(to_host(trace_alpha[i]).reshape(alpha.shape), alpha, "bf16",
                             f"alpha_{l} ({nb[i]} blocks)")
            worst["alpha"] = max(worst["alpha"], r)
        else:
            assert alpha is None
        checked.append((l, kind, nb[i]))

    xh = to_host(x)
    yref = O.stack(xh, _Fp64Layers([t.cpu() for t in wq]), _Fp64Layers([t.cpu() for t in wo]),
                   to_host(wr), w.H, softmax_period=w.softmax_period,
                   attnres_block=w.attnres_block, on_layer=on_layer)
    assert [c[0] for c in checked] == list(range(1, L + 1))
    worst["h_L - x"] = assert_close(update, yref - xh, "bf16", "h_L - x")
    worst["y"] = assert_close(to_host(y), yref, "bf16", "y")
    print(f"{w.name}: worst rel-L2 " + ", ".join(f"{k} {v:.2e}" for k, v in worst.items()))
    return checked


def test_720p_24_layer_stack_whole_against_oracle():
    w = W.STACK720P
    checked = _whole_stack_parity(w)
    # 6 anchors; blocks 2 and 3 route their 6 linear layers each, over 1 and 2 summaries
    assert sum(1 for _, k, _ in checked if k == "softmax") == 6
    assert [n for _, k, n in checked if n] == [1] * 6 + [2] * 6


def test_long_video_4_layer_group_whole_against_oracle():
    w = W.LONG4
    checked = _whole_stack_parity(w)
    assert [k for _, k, _ in checked] == ["linear", "linear", "linear", "softmax"]
