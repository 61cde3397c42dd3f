"""Host-side pieces of the benchmark, on CPU: the reference arm (the FP64 oracle
timed on the host cores) on the small layer, the oracle's thread count and CPU
model in its result line, and the rule that a committed traffic figure is used
only while the kernel sources it was measured on are unchanged."""
import hashlib
import json
import os

import bench


class _Args:
    steps, warmup, ref_tokens, workload = 1, 3, 4, "tiny"


def test_reference_arm_line_on_the_small_layer():
    res = bench.run_reference(_Args, 1, 0)
    assert res["impl"] == "reference" and res["unit"] == "tok/s" and res["value"] > 0
    assert res["dtype"] == "f64" and res["higher_is_better"] is True
    cb = res["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == res["value"]
    assert cb["cores"] == min(4, os.cpu_count()) and cb["cpu_model"]
    assert res["e2e"] == {"value": res["value"], "unit": "tok/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    assert bench.run_reference(_Args, 2, 1) is None      # ranks other than 0 do no work
    json.dumps(res)


def test_oracle_threads_and_cpu_model():
    n = os.cpu_count()
    assert bench.oracle_threads(1) == 1 and bench.oracle_threads(10 ** 6) == n
    assert bench.oracle_threads(0) == 1
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()


def _profile(tmp_path, src_bytes, recorded):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_bytes(src_bytes)
    rec = {"traffic": {"kern": {"workload": "w", "dram_bytes_per_launch": 1234,
                                "sources": ["k.cu"], "sources_sha256_16": recorded}}}
    (tmp_path / "profiles" / "k.md").write_text("# x\n\n```json\n" + json.dumps(rec) + "\n```\n")


def test_traffic_figure_only_while_sources_unchanged(tmp_path, monkeypatch):
    src = b"__global__ void k() {}\n"
    _profile(tmp_path, src, hashlib.sha256(src).hexdigest()[:16])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("kern", "w") == 1234
    assert bench.profile_traffic("kern", "other") is None
    assert bench.profile_traffic("other", "w") is None
    (tmp_path / "k.cu").write_bytes(src + b"// changed\n")
    assert bench.profile_traffic("kern", "w") is None


def test_oracle_baseline_sample_and_stack_label():
    import synth
    wl = synth.CONFIGS["tiny"]
    seed = synth.workload_seed(wl)
    layer = synth.make_layer(wl.dims, seed)
    T = wl.tokens[0]
    x = synth.make_x_bf16(T, wl.dims.H, seed)
    logits = synth.make_logits(T, wl.dims.E, seed)
    one = bench.oracle_baseline(layer, x, logits, wl.dims.K, T, 0.0)
    assert one["kind"] == "oracle" and one["unit"] == "tok/s" and one["value"] > 0
    assert one["sample"].startswith(f"first 8 of the {T} tokens") and one["cores"] == min(8, os.cpu_count())
    many = bench.oracle_baseline(layer, x, logits, wl.dims.K, T, 0.0, layers=48)
    assert "divided by 48 layers" in many["sample"]
    assert 0 < many["value"] < one["value"]
