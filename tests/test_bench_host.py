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
    per, src = bench.stored_traffic("gemm", "gpt2-124m", 192)
    assert per is not None and per > 1e6 and "per launch" in src
    assert bench.stored_traffic("gemm", "gpt2-350m", 192) == (None, None)
    # a record taken on other sources is refused
    rec = json.load(open(os.path.join(bench.ROOT, "profiles",
                                      "gemm_dram_traffic_gpt2_124m_b16_t1024.json")))
    rec["kernel_sources_sha256"] = "0" * 64
    root = tmp_path / "r"
    (root / "profiles").mkdir(parents=True)
    (root / "profiles" / "gemm_dram_traffic_gpt2_124m_b16_t1024.json").write_text(json.dumps(rec))
    for f in rec["kernel_sources"]:
        dst = root / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(bench.ROOT, f), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(root))
    per, why = bench.stored_traffic("gemm", "gpt2-124m", 192)
    assert per is None and "changed" in why
