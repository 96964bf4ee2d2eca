"""The bench's algorithmic byte counts (the numerator of every roofline
fraction it reports) against closed forms of the stored formats, and its
count of library launches per forward. CPU only: small expert sets are
generated on the host."""
import pytest

import bench
import moe_inputs as mi


def _experts(wfmt, d=2048, F=512, E=2):
    wl = mi.workload("prefill", E=E, k=2, wfmt=wfmt, d=d, F=F)
    return mi.make_experts(wl, seed=0, device="cpu")


# bytes per expert as multiples of F*d: gate|up holds 2F rows of d inputs,
# down d rows of F inputs; quantised formats add a bf16 scale and a bf16
# bias per group of g elements, i.e. 4/g bytes per element
@pytest.mark.parametrize("wfmt,elem_bytes,group", [
    ("q4", 0.5, 64), ("q4g32", 0.5, 32), ("q4g128", 0.5, 128), ("q8", 1.0, 64),
    ("bf16", 2.0, 0), ("f32", 4.0, 0)])
def test_expert_bytes_closed_form(wfmt, elem_bytes, group):
    d, F = 2048, 512
    ex = _experts(wfmt, d, F)
    per_elem = elem_bytes + (4.0 / group if group else 0.0)
    assert bench.gate_up_bytes(ex) == int(2 * F * d * per_elem)
    assert bench.expert_bytes(ex) == int(3 * F * d * per_elem)


def test_prefill_layer_bytes_match_reported_figure():
    # the prefill layer's algorithmic bytes: every active expert's weights
    # once, x read and y written once (bf16); 501 active experts is the count
    # of the seeded prefill routing
    d, F, T = 2048, 512, 2048
    per_expert = bench.expert_bytes(_experts("q4", d, F))
    assert per_expert == int(1.6875 * F * d)
    assert 501 * per_expert + 2 * T * d * 2 == 903282688


@pytest.mark.parametrize("T,k,tc,fused,launches", [
    (1, 8, False, True, 1),        # the one-launch decode kernel
    (64, 8, False, False, 7),      # single-block sort
    (2048, 10, True, False, 9),    # count, scan and scatter sort kernels
])
def test_kernels_per_forward(T, k, tc, fused, launches):
    assert bench.kernels_per_forward(T, k, tc, fused) == launches


def test_reference_arm_line():
    """`bench.py --impl reference` (the oracle on the host's cores) prints the
    contract's JSON line with the reference keys, on a small workload."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert abs(line["ms_per_step"] - 16 / line["value"] * 1e3) < 1e-9 * line["ms_per_step"] + 1e-12
