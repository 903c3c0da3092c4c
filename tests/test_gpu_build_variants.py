"""The library's diagnostic modes, each in a fresh process.

* The bounds-checked build (``python -m combine_moe_topk_gate_b200.build
  --bounds-check`` -> ``libmoe_bounds_check.so``, loaded with
  ``MOE_LIBRARY``): its kernels also test every receive-row index they derive
  themselves; the parity suite's workload cases must pass on it unchanged
  (so no such index ever falls outside the buffer on them).
* ``MOE_DEBUG=1``: every launch prints its kernel and configuration.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_cases_pass_on_the_bounds_checked_build():
    from combine_moe_topk_gate_b200 import build
    lib = build.build(bounds_check=True)
    env = {**os.environ, "MOE_LIBRARY": lib}
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_parity.py"),
                        os.path.join(ROOT, "tests", "test_gpu_aligned.py"),
                        "-k", "not all_fp32_patterns"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=3000)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_debug_trace_names_every_launch():
    code = ("import torch\n"
            "from combine_moe_topk_gate_b200 import api\n"
            "lg = torch.randn(64, 256, device='cuda')\n"
            "idx, w = api.moe_topk_gate(lg, 8, api.MOE_GATE_SIGMOID_GROUP, 8, 4, 2)\n"
            "L = api.moe_get_layout(idx, 256, 8)\n"
            "torch.cuda.synchronize()\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env={**os.environ, "MOE_DEBUG": "1"},
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stderr.splitlines() if ln.startswith("[moe] launch")]
    assert len(lines) == 2, r.stderr
    assert "topk_gate" in lines[0] and "layout_single" in lines[1]
    assert "grid=(" in lines[0] and "block=(256,1,1)" in lines[0]
    quiet = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env={**os.environ, "MOE_DEBUG": "0"},
                           capture_output=True, text=True, timeout=300)
    assert quiet.returncode == 0 and "[moe] launch" not in quiet.stderr
