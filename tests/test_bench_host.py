"""bench.py's host-side pieces, without a GPU: the kernel-source hashing that gates the
captured DRAM traffic, the CPU sample sizing, and the reference arm's JSON line."""
import contextlib
import io
import json
import os

import pytest

import bench
import synth


def test_every_named_kernel_is_found_and_hashed():
    funcs = bench._device_functions()
    names = {k for k, _ in bench.TRAFFIC} | {
        "k_dispatch_warp", "k_dispatch_elem", "k_dispatch_int8_staged", "k_dispatch_int8",
        "k_combine_v8", "k_combine_scalar", "k_combine_int8_warp", "k_combine_int8_v8",
        "k_combine_int8_scalar", "k_combine_add_rmsnorm_v8", "k_combine_add_rmsnorm_scalar",
        "k_dispatch_int8_smooth_k", "k_dispatch_int8_smooth_scalar", "k_dispatch_int8_smooth_grouped",
        "k_smooth_order",
        "k_expand_warp", "k_expand_bytes"}
    for n in names:
        assert n in funcs, n
        h = bench.kernel_source_hash(n)
        assert len(h) == 16 and h == bench.kernel_source_hash(n)
    assert bench.kernel_source_hash("no_such_kernel") == ""
    assert bench.kernel_source_hash("k_dispatch_warp") != bench.kernel_source_hash("k_combine_v8")


def test_hash_covers_the_helpers_a_kernel_calls():
    """A helper's text is part of the hash of every kernel that calls it: the int8 combine
    calls add_int8_x16, the bf16 combine does not."""
    funcs = bench._device_functions()
    assert "add_int8_x16" in funcs["k_combine_int8_warp"]
    real = bench._device_functions

    def patched():
        f = dict(real())
        f["add_int8_x16"] = f["add_int8_x16"] + "// changed\n"
        return f
    before = {k: bench.kernel_source_hash(k) for k in ("k_combine_int8_warp", "k_combine_v8")}
    bench._device_functions = patched
    try:
        after = {k: bench.kernel_source_hash(k) for k in ("k_combine_int8_warp", "k_combine_v8")}
    finally:
        bench._device_functions = real
    assert after["k_combine_int8_warp"] != before["k_combine_int8_warp"]
    assert after["k_combine_v8"] == before["k_combine_v8"]


@pytest.mark.parametrize("name", ["tiny", "r8", "int8", "skew", "map"])
def test_cpu_sample_sizes(name):
    w = synth.get(name)
    for div in (1, 8):
        S = bench.cpu_sample_S(w, div)
        assert 1 <= S <= w.S
        assert w.R * S * w.K * w.H < (1 << 31)


def test_reference_line_has_the_contract_keys(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    w = synth.scaled(synth.get("tiny"), S=32)
    args = type("A", (), dict(steps=2, warmup=1, gpus=1, ref_div=2))()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, w)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline",
                "e2e", "gpu_launches"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["gpu_launches"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == w.name
