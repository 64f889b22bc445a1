"""Host-side arithmetic of bench.py: the algorithmic bytes and flops behind
every throughput and roofline figure, the layer sets, and the rule that keeps
recorded DRAM traffic only for the sources it was measured on.

The per-layer bytes follow the minimal-traffic definition (x, packed W_d with
its E4M3 scales, L, V, s, bias, y) and are checked against values worked out by
hand for the configs' shapes, so a dropped or doubled term fails here."""
import json
import os

import pytest

import bench
from bit_w4a4_quantised_b200 import workloads

MB = 1e6


def test_layer_bytes_worked_by_hand():
    # 32 x 1024 -> 1024, r = 32: x 65 536 + W_d 589 824 + L 65 536 + V 131 072
    # + s 4 096 + bias 2 048 + y 65 536 = 923 648 bytes
    assert bench.layer_bytes(32, 1024, 1024, 32) == 923_648
    # 4096 x 3072 -> 3072, r = 32: 2 x 25 165 824 (x, y) + 5 308 416 (W_d)
    # + 196 608 (L) + 393 216 (V) + 12 288 (s) + 6 144 (bias)
    assert bench.layer_bytes(4096, 3072, 3072, 32) == 56_248_320
    # r = 0 drops L and V only
    assert bench.layer_bytes(4096, 3072, 3072, 0) == 56_248_320 - 196_608 - 393_216


def test_layer_flops_worked_by_hand():
    M, K, N, r = 4096, 3072, 14336, 32
    gemm = 2 * M * N * K            # FP4 product
    branch = 2 * M * N * r          # u' L^T
    proj = 4 * M * K * r            # u = x~ V and u V^T
    assert bench.layer_flops(M, K, N, r) == gemm + branch + proj
    assert bench.gemm_flops(M, K, N, r) == gemm + branch
    assert bench.prologue_flops(M, K, N, r) == proj
    assert abs(bench.layer_flops(M, K, N, r) / 1e9 - 366.2) < 0.1


def test_kernel_bytes_split_the_layer():
    # the prologue reads x and writes the codes; the GEMM reads the codes back:
    # the two kernels' bytes exceed the layer's by the round trip of the
    # activation codes and of u' plus the prologue's side of V and s
    M, K, N, r = 4096, 3072, 3072, 32
    pro, gem, lay = bench.prologue_bytes(M, K, N, r), bench.gemm_bytes(M, K, N, r), bench.layer_bytes(M, K, N, r)
    codes = 0.5625 * M * K
    assert pro + gem == pytest.approx(lay + 2 * codes + 2 * 2 * M * r)


def test_action_set_readings():
    ctx_specs, ctx = bench.set_layers(bench.SETS["c5action"])
    all_specs, all32 = bench.set_layers(bench.SETS["c5action32"])
    assert len(ctx) == len(all32) == 300
    ctx_m = [ctx_specs[i].M for i in ctx]
    assert ctx_m.count(4096) == 60 and ctx_m.count(32) == 240
    assert all(all_specs[i].M == 32 for i in all32)
    kinds = {(ctx_specs[i].K, ctx_specs[i].N) for i in ctx}
    assert kinds == {(1024, 1024), (1024, 4096), (4096, 1024)}
    # FP4 weights of the set: 30 blocks x (8 x 1024^2 + 2 x 1024 x 4096) x 0.5625 B
    w = sum(0.5625 * ctx_specs[i].K * ctx_specs[i].N for i in ctx)
    assert w == 30 * (8 * 1024 * 1024 + 2 * 1024 * 4096) * 0.5625
    assert all(ctx_specs[i].r == 32 for i in ctx)


def test_action_set_members_are_the_step_specs():
    specs = workloads.c5_layer_specs(cross_kv_context=True)
    _, idx = bench.set_layers(bench.SETS["c5action"])
    assert all(specs[i].name.startswith("action.") for i in idx)
    assert {specs[i].name.split(".")[-1] for i in idx} == {
        "self_q", "self_k", "self_v", "self_o", "cross_q", "cross_k", "cross_v", "cross_o", "ffn0", "ffn2"}


def test_recorded_traffic_needs_the_same_sources(tmp_path, monkeypatch):
    import shutil
    src = os.path.join(bench.ROOT, "bit_w4a4_quantised_b200", "csrc")
    csrc = tmp_path / "bit_w4a4_quantised_b200" / "csrc"
    shutil.copytree(src, csrc)
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pro, gem = bench.traffic_sources("prologue"), bench.traffic_sources("fp4_gemm")
    assert "prologue.cu" in pro and "gemm.cu" not in pro and "api.cu" in pro
    entry = {"bytes_per_launch": 1234, "sources": pro, "sources_sha256": bench.sources_digest(pro)}
    (prof / "traffic.json").write_text(json.dumps({
        "c2:prologue_kernel": entry,
        "c3:prologue_kernel": dict(entry, sources_sha256="0" * 64),
        "c3r0:fp4_gemm_kernel": {"bytes_per_launch": 99, "sources": gem, "sources_sha256": bench.sources_digest(gem)},
        "c4down:prologue_kernel": {"bytes_per_launch": 7, "csrc_sha256": "0" * 64}}))
    assert bench.recorded_traffic("c2", "prologue_kernel") == 1234
    assert bench.recorded_traffic("c3", "prologue_kernel") is None       # other sources
    assert bench.recorded_traffic("c4up", "fp4_gemm_kernel") is None     # not recorded
    assert bench.recorded_traffic("c4down", "prologue_kernel") is None   # no source list
    # a change to the GEMM's file leaves the prologue's figure valid, and not the reverse
    with open(csrc / "gemm.cu", "a") as f:
        f.write("// edited\n")
    assert bench.recorded_traffic("c2", "prologue_kernel") == 1234
    assert bench.recorded_traffic("c3r0", "fp4_gemm_kernel") is None
    # a shared header invalidates both
    with open(csrc / "common.cuh", "a") as f:
        f.write("// edited\n")
    assert bench.recorded_traffic("c2", "prologue_kernel") is None


def test_committed_traffic_entries_name_their_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    for key, e in d.items():
        assert e["bytes_per_launch"] > 0, key
        assert set(bench.SHARED_SOURCES) <= set(e["sources"]), key
        assert len(e["sources_sha256"]) == 64, key


def test_per_unit():
    assert bench.per_unit(2e9, 2.0, "GB/s") == pytest.approx(1.0)
    assert bench.per_unit(3e12, 1.5, "TFLOP/s") == pytest.approx(2.0)


def test_reference_arm_line_on_the_cpu():
    """bench.py --impl reference runs the float64 oracle on the host: its line
    carries the contract's keys and the steps and warm-up it actually ran."""
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "c2", "--steps", "4", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True and line["value"] > 0
    assert (line["steps"], line["warmup"]) == (4, 3)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
