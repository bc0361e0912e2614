"""Host logic of bench.py that sets the numbers on its JSON line: the
algorithmic work each kernel class is credited with (the roofline's numerator),
which layers the router serves, the whole-job rate, and the guard that drops a
profiled DRAM-traffic figure once its kernel's source has changed. No GPU."""
import hashlib
import json
import os

import pytest

import bench

WL = dict(bench.WORKLOAD)


def _tensor_bytes(*shapes_and_sizes):
    total = 0
    for shape, elem in shapes_and_sizes:
        n = 1
        for s in shape:
            n *= s
        total += n * elem
    return total


def test_anchor_flops_are_the_two_products_of_every_head():
    # per head: S = Q K^T is N x N x d multiply-adds, O = P V another N x N x d
    B, N, H, d = WL["B"], WL["N"], WL["H"], WL["d"]
    flops = 0
    for _ in range(B * H):
        flops += 2 * N * N * d  # Q K^T
        flops += 2 * N * N * d  # P V
    bound, work = bench.algorithmic_work("anchor", WL)
    assert bound == "tensor" and work == flops


def test_projection_flops_follow_the_weight_shapes():
    B, N, D = WL["B"], WL["N"], WL["H"] * WL["d"]
    # [Q|K|V|G] = u W^T with W [4D, D]; o = Y W_o^T and k_c = s_c W_r with [D, D]
    assert bench.algorithmic_work("proj_qkvg", WL) == ("tensor", 2 * (B * N) * D * (4 * D))
    assert bench.algorithmic_work("proj_out", WL) == ("tensor", 2 * (B * N) * D * D)
    assert bench.algorithmic_work("keys", WL) == ("tensor", 2 * (B * N) * D * D)


def test_linear_bytes_are_its_tensors_read_and_written_once():
    B, N, D = WL["B"], WL["N"], WL["H"] * WL["d"]
    act = ((B, N, D), 2)  # one bf16 activation
    assert bench.algorithmic_work("linear_state", WL) == ("hbm", _tensor_bytes(act, act))  # K, V
    # Q, G read and Y written
    assert bench.algorithmic_work("linear_readout", WL) == ("hbm", _tensor_bytes(act, act, act))
    # the whole layer: 10 B N D bytes, 593 MB at the 720p shape
    total = bench.algorithmic_work("linear_state", WL)[1] + bench.algorithmic_work("linear_readout", WL)[1]
    assert total == 10 * B * N * D and round(total / 1e6) == 594


def test_write_gated_linear_state_also_reads_one_logit_per_token_and_head():
    wl = dict(WL, write_gate=True)
    B, N, H, D = wl["B"], wl["N"], wl["H"], wl["H"] * wl["d"]
    act = ((B, N, D), 2)
    logits = ((B, N, H), 2)
    assert bench.algorithmic_work("linear_state", wl) == ("hbm", _tensor_bytes(act, act, logits))


@pytest.mark.parametrize("nb", [1, 2, 3])
def test_router_bytes_read_h_once_and_every_key_and_summary(nb):
    B, N, D = WL["B"], WL["N"], WL["H"] * WL["d"]
    h = ((B, N, D), 4)         # the fp32 residual stream
    bf16 = ((B, N, D), 2)
    want = _tensor_bytes(h, *([bf16] * nb), *([bf16] * nb), bf16)  # keys, summaries, u
    assert bench.algorithmic_work("route", WL, nb) == ("hbm", want)


def test_router_serves_the_linear_layers_of_later_blocks():
    # 3 blocks of 8 layers, anchors at 4, 8, ..., 24: block 2's linear layers
    # mix one completed block, block 3's two; block 1 and the anchors none
    assert bench.routed_blocks(WL) == [1] * 6 + [2] * 6
    assert bench.routed_blocks(dict(WL, attnres_block=0)) == []


def test_whole_job_rate_counts_every_rank():
    assert bench.whole_job_rate(1, 19320, 63.0) == pytest.approx(19320 / 0.063)
    assert bench.whole_job_rate(4, 19320, 63.0) == pytest.approx(4 * 19320 / 0.063)


def _fake_tree(tmp_path, src_text):
    csrc = tmp_path / "softmax_attention_video_gated_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "anchor_tc.cu").write_text(src_text)
    (csrc / "common.cuh").write_text("// shared helpers\n")
    h = hashlib.sha256()
    h.update(b"// kernel v1\n")
    h.update(b"// shared helpers\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps({"anchor": {
        "bytes_per_launch": 123.0, "source": "anchor_tc.cu", "source_hash": h.hexdigest()[:16],
        "profile": "profiles/anchor_720p.md"}}))


def test_profiled_traffic_is_used_only_while_the_source_is_unchanged(tmp_path, monkeypatch):
    _fake_tree(tmp_path, "// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("anchor") == (123.0, "profiles/anchor_720p.md")
    assert bench.profiled_traffic("route") == (None, None)  # never captured
    # any edit to the kernel's source (a comment included) voids the figure
    (tmp_path / "softmax_attention_video_gated_b200" / "csrc" / "anchor_tc.cu").write_text(
        "// kernel v2\n")
    assert bench.profiled_traffic("anchor") == (None, None)


def test_profiled_traffic_entries_name_committed_profiles():
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(path) as f:
        entries = json.load(f)
    for kind, e in entries.items():
        assert kind in bench.KINDS
        assert os.path.exists(os.path.join(bench.ROOT, e["profile"])), e["profile"]
        assert os.path.exists(os.path.join(bench.ROOT, "softmax_attention_video_gated_b200", "csrc",
                                           e["source"]))
        assert e["bytes_per_launch"] > 0
