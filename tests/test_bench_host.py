"""Host-side rules of bench.py that need no GPU.

The roofline's `traffic` figure comes from a committed ncu capture; it must be
reported only for the sources the capture was taken from (or for later sources
recorded as leaving the captured kernels unchanged), and only for the workload
that was captured.  The step's FLOP count follows the metric's definition.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from attention_kl_divergence_attn_b200 import inputs  # noqa: E402


def _record(tmp_path, rec):
    (tmp_path / "profiles").mkdir(exist_ok=True)
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))


def test_traffic_only_for_matching_sources_and_workload(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "aaaa")
    kern = {"k": {"workload": "w", "dram_bytes_per_launch": 123}}
    _record(tmp_path, {"source_hash": "aaaa", "kernels": kern})
    assert bench.recorded_traffic("k", "w") == 123
    assert bench.recorded_traffic("k", "other") is None          # another workload
    assert bench.recorded_traffic("missing", "w") is None
    _record(tmp_path, {"source_hash": "bbbb", "kernels": kern})
    assert bench.recorded_traffic("k", "w") is None               # sources changed since the capture
    _record(tmp_path, {"source_hash": "bbbb", "kernels": kern,
                       "unchanged_for": [{"hash": "aaaa", "change": "outside the captured kernels"}]})
    assert bench.recorded_traffic("k", "w") == 123


def test_missing_record_gives_no_traffic(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k", "w") is None


def test_committed_record_names_the_step_kernels():
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        rec = json.load(f)
    w = inputs.WORKLOADS["causal_8k_d128"]
    assert set(rec["kernels"]) == {n for n in bench.kernel_names(w) if n != "streamkl_mean_kernel"}
    for e in rec["kernels"].values():
        assert e["workload"] == "causal_8k_d128" and e["dram_bytes_per_launch"] > 0


def test_step_flops_follow_the_metric():
    # per visible (query, key) pair, 2 d FLOPs per product of two d-vectors: the
    # forward's S_t and S_s, the backward's recomputed S_t and S_s, and dQ_s, dK_s
    # (plus dQ_t, dK_t with teacher gradients); causal counts half the pairs
    w = inputs.WORKLOADS["causal_8k_d128"]
    assert w.causal and w.teacher_grads and w.d_t == w.d_s == 128
    pairs = w.B * w.H * w.N_Q * w.N_K / 2
    assert bench.step_flops(w) == 8 * 2 * 128 * pairs
    assert bench.fwd_flops(w) == 2 * 2 * 128 * pairs
    c = inputs.WORKLOADS["cross_1k_64k"]
    assert not c.causal and not c.teacher_grads
    pairs = c.B * c.H * c.N_Q * c.N_K
    assert bench.step_flops(c) == (2 * 2 * (c.d_t + c.d_s) + 2 * 2 * c.d_s) * pairs


def test_kernel_method_flops_split_the_step():
    # the method's FLOPs of the step are the forward's logits plus, for each of
    # the two backward kernels, its own contraction and half of the recompute;
    # each backward kernel issues one whole recompute, i.e. a quarter more at d = 128
    for name in ("causal_8k_d128", "cross_1k_64k", "causal_2k_d64"):
        w = inputs.WORKLOADS[name]
        km, kf = bench.kernel_method_flops(w), bench.kernel_flops(w)
        fwd, _, dkv, dq = bench.kernel_names(w)
        assert abs(sum(km.values()) - bench.step_flops(w)) <= 1e-9 * bench.step_flops(w)
        assert km[fwd] == kf[fwd]
        pairs = bench.visible_pairs(w) * w.B * w.H
        for k in (dkv, dq):
            assert kf[k] - km[k] == (w.d_t + w.d_s) * pairs
    w = inputs.WORKLOADS["causal_8k_d128"]
    assert bench.kernel_method_flops(w)["streamkl_bwd_dkv_kernel"] == 3 * 256 * bench.visible_pairs(w) * w.H


def test_key_owner_form_follows_the_tensor_memory_budget():
    # the persistent key-owner kernel where the K rows fit in tensor memory
    # (student-only gradients, or heads of 64): every workload but the 8k one
    for name, w in inputs.WORKLOADS.items():
        expect = "streamkl_bwd_dkv_kernel" if name == "causal_8k_d128" else "streamkl_bwd_dkv_persistent_kernel"
        assert bench.key_owner_kernel(w) == expect, name
