"""The single-op cases behind the profile commands run (tiny workload)."""
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

OPS = ["gate", "layout", "dispatch_bf16", "dispatch_fp8", "dispatch_fp8_token", "dispatch_mxfp8",
       "dispatch_nvfp4", "dispatch_e5m6", "dispatch_fp8_ue8m0", "combine", "dispatch_backward", "combine_backward",
       "swiglu_fp8", "quant_fp8_channel"]


@pytest.mark.parametrize("op", OPS)
def test_case_runs(op):
    r = subprocess.run([sys.executable, "-m", "combine_moe_topk_gate_b200.cases", op, "--workload", "tiny",
                        "--reps", "2", "--rows", "256", "--inter", "256"], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "us per launch" in r.stdout

