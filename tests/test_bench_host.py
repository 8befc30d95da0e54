"""bench.py's host-side bookkeeping on CPU: the code digest that keys the
committed DRAM-traffic figures, and the lookup that uses it."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = """// a kernel
#include "x.h"
/* block
   comment */ __global__ void k(int* p) {
  const char* s = "not // a comment /* either */";
  p[0] = '/';   // trailing
}
"""


def _write(tmp_path, name, text):
    path = tmp_path / name
    path.write_text(text)
    return str(path)


def test_comments_and_whitespace_do_not_change_the_digest(tmp_path):
    a = bench.code_digest(_write(tmp_path, "a.cu", SRC))
    edited = SRC.replace("// a kernel", "// the same kernel, described again\n// over two lines")
    edited = edited.replace("/* block\n   comment */", "/* another */").replace("  p[0]", "\tp[0]")
    assert bench.code_digest(_write(tmp_path, "b.cu", edited)) == a


def test_code_and_string_literals_change_the_digest(tmp_path):
    a = bench.code_digest(_write(tmp_path, "a.cu", SRC))
    assert bench.code_digest(_write(tmp_path, "b.cu", SRC.replace("p[0] =", "p[1] ="))) != a
    # a "//" inside a string literal is code, not a comment
    assert bench.code_digest(_write(tmp_path, "c.cu", SRC.replace("not // a", "not // b"))) != a
    assert bench.code_digest(_write(tmp_path, "d.cu", SRC.replace("'/'", "'*'"))) != a


def test_traffic_figures_are_used_only_for_the_captured_code():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    for workload, kernels in table.items():
        if workload.startswith("_"):
            continue
        for kernel, ent in kernels.items():
            src = os.path.join(ROOT, ent["source"])
            current = bench.code_digest(src) == ent["code_sha256_16"]
            got = bench.kernel_traffic(workload, kernel)
            assert got == (ent["bytes_per_launch"] if current else None)
            assert ent["bytes_per_launch"] == ent["read"] + ent["write"]
    assert bench.kernel_traffic("no_such_workload", "mega_ffn") is None


def test_workload_overrides():
    from mixture_experts_ffn_token_b200.workloads import WORKLOADS
    base = WORKLOADS["mixtral"]
    wl = bench.apply_overrides(base, ["moe_dim=7168", "has_bias=true", "logits_std=0.5"])
    assert (wl.moe_dim, wl.has_bias, wl.logits_std) == (7168, True, 0.5)
    assert wl.name == "mixtral+moe_dim=7168,has_bias=true,logits_std=0.5"
    # figures recorded for the named workload are not used for a changed one
    assert bench.kernel_traffic(wl.name, "mega_ffn") is None
    assert bench.apply_overrides(base, []) is base
    for bad in (["moe_dim"], ["name=x"], ["no_such_field=1"]):
        try:
            bench.apply_overrides(base, bad)
        except SystemExit:
            continue
        raise AssertionError(f"{bad} accepted")


def test_gpus_must_match_the_started_ranks():
    bench.check_world(1, 1)
    bench.check_world(4, 4)
    for gpus, world in ((2, 1), (1, 2)):
        try:
            bench.check_world(gpus, world)
        except SystemExit as e:
            assert "torch.distributed.run" in str(e)
            continue
        raise AssertionError(f"--gpus {gpus} accepted with {world} rank(s)")


def test_roofline_arithmetic():
    """The dominant kernel's roofline entry: algorithmic FLOPs (or weight
    bytes) over its time, against the peak that bounds it."""
    from mixture_experts_ffn_token_b200.workloads import WORKLOADS
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    mix = WORKLOADS["mixtral"]
    flops = 6 * 8192 * 4096 * 14336
    r = bench.roofline(mix, "mega_ffn", 2.0, peaks, "measured", {"reasons": []}, 8)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1600.0
    assert abs(r["achieved"] - flops / 2e-3 / 1e12) < 1e-9 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / 1600.0) < 1e-12
    assert abs(r["frac_of_nominal"] - r["achieved"] / 2250.0) < 1e-12
    assert abs(r["frac_sustained"] - r["achieved"] / 1400.0) < 1e-12
    # a timed region shorter than a second is compared with the burst figure
    # even under the power cap; a capped region of a second or more with the
    # sustained one
    short = bench.roofline(mix, "mega_ffn", 2.0, peaks, "measured", {"reasons": ["sw_power_cap"]}, 8, region_s=0.05)
    assert short["peak"] == 1600.0 and "burst" in short["peak_kind"]
    long = bench.roofline(mix, "mega_ffn", 2.0, peaks, "measured", {"reasons": ["sw_power_cap"]}, 8, region_s=2.0)
    assert long["peak"] == 1400.0 and "sustained" in long["peak_kind"]
    uncapped = bench.roofline(mix, "mega_ffn", 2.0, peaks, "measured", {"reasons": []}, 8, region_s=2.0)
    assert uncapped["peak"] == 1600.0
    # 64 rows per expert (gptoss): the touched experts' weight bytes bound it
    go = WORKLOADS["gptoss"]
    g = bench.roofline(go, "mega_ffn", 1.0, peaks, "measured", {"reasons": []}, 128)
    wbytes = 3 * 128 * 2880 * 2880 * 2
    assert g["bound"] == "hbm" and g["unit"] == "GB/s"
    assert abs(g["achieved"] - wbytes / 1e-3 / 1e9) < 1e-9 * g["achieved"]
    # the gate_up GEMM alone (two launches): 4 R H D FLOPs
    up = bench.roofline(mix, "gemm_gate_up", 1.0, peaks, "measured", {"reasons": []}, 8)
    assert abs(up["achieved"] - 4 * 8192 * 4096 * 14336 / 1e-3 / 1e12) < 1e-9 * up["achieved"]


def test_dram_frac():
    """Measured DRAM bytes per launch over the live time, against the HBM
    copy peak: 1.7 GB in 0.5 ms is 3.4 TB/s, half of a 6.8 TB/s peak."""
    assert abs(bench.dram_frac(1.7e9, 0.5, {"hbm_gbs": 6800.0}) - 0.5) < 1e-12


def test_launches_per_step():
    from mixture_experts_ffn_token_b200.workloads import WORKLOADS
    W = WORKLOADS
    # small problems: route+CSR in one kernel, gather, single-launch FFN, combine
    assert bench.launches_per_step(W["tiny"], True) == 4
    assert bench.launches_per_step(W["decode"], True, csr_fused=True) == 4
    # router + one CSR kernel + gather + FFN + combine
    assert bench.launches_per_step(W["sink"], True, csr_fused=True) == 5
    assert bench.launches_per_step(W["sink"], True, csr_fused=False) == 7
    assert bench.launches_per_step(W["sink"], False, csr_fused=False) == 8
    # the gate_up GEMM gathering its own rows drops the gather kernel
    assert bench.launches_per_step(W["mixtral"], True, csr_fused=True, fused_gather=True) == 4
    # ... unless the router weight scales the rows first
    assert bench.launches_per_step(W["mixtral_wfirst"], True, csr_fused=True, fused_gather=True) == 5
    # shared experts reading x directly: index kernel + single launch
    assert bench.launches_per_step(W["sink_shared"], True, csr_fused=True) == 7
    assert bench.csr_fused_active(W["sink"], 148) and not bench.csr_fused_active(W["sink"], 16)


def test_per_config_default():
    assert bench.per_config_enabled(None, 1) is True
    assert bench.per_config_enabled(None, 8) is False
    assert bench.per_config_enabled(True, 4) is True
    assert bench.per_config_enabled(False, 1) is False
    assert set(bench.PER_CONFIG) == {"tiny", "gptoss", "sink", "decode"}
