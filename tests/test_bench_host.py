"""Host-side accounting of bench.py: parameter count, algorithmic FLOPs per
step, and the rule that the stored ncu traffic is reported only while the GEMM
sources still hash to the ones it was captured on."""
import json
import os

import bench


def test_parameter_counts_and_step_flops():
    # N with the padded vocabulary (tied head: wte counted once)
    assert bench.n_params(bench.WORKLOADS["gpt2-124m"]) == 124_475_904
    assert bench.n_params(bench.WORKLOADS["gpt2-350m"]) == 354_871_296
    w = bench.WORKLOADS["gpt2-124m"]
    step = bench.flops_per_token(w) * w["B"] * w["T"]
    # 6N + 6 L C T per token (causal attention: half the full-matrix count)
    assert step == (6 * 124_475_904 + 6 * 12 * 768 * 1024) * 16 * 1024
    assert abs(step / 1e12 - 13.16) < 0.01


def test_stored_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    """The record is used only while the kernel sources hash to the ones it was
    captured on: a copy of the record stamped with the current sources' hash is
    accepted, the same record stamped with another hash is refused."""
    import hashlib
    assert bench.stored_traffic("gemm", "gpt2-350m", 192) == (None, None)
    rec = json.load(open(os.path.join(bench.ROOT, "profiles",
                                      "gemm_dram_traffic_gpt2_124m_layer_m16384.json")))
    root = tmp_path / "r"
    (root / "profiles").mkdir(parents=True)
    h = hashlib.sha256()
    for f in sorted(rec["kernel_sources"]):
        dst = root / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        data = open(os.path.join(bench.ROOT, f), "rb").read()
        dst.write_bytes(data)
        h.update(data)
    monkeypatch.setattr(bench, "ROOT", str(root))
    path = root / "profiles" / "gemm_dram_traffic_gpt2_124m_layer_m16384.json"
    rec["kernel_sources_sha256"] = h.hexdigest()
    path.write_text(json.dumps(rec))
    per, src = bench.stored_traffic("gemm", "gpt2-124m", 192)
    assert per is not None and per > 1e6 and "per launch" in src
    rec["kernel_sources_sha256"] = "0" * 64
    path.write_text(json.dumps(rec))
    per, why = bench.stored_traffic("gemm", "gpt2-124m", 192)
    assert per is None and "changed" in why


def test_metric_names_the_workload_model():
    assert set(bench.METRICS) == set(bench.WORKLOADS) | set(bench.LMHEAD)
    assert bench.METRICS["gpt2-124m"].startswith("GPT-2 124M training tokens/s")
    assert bench.METRICS["gpt2-124m-accum"] == bench.METRICS["gpt2-124m"]
    assert bench.METRICS["gpt2-350m"].startswith("GPT-2 350M training tokens/s")
    assert "8192x768x50304" in bench.METRICS["lmhead-ce-8192"]
