"""Failure detection without a GPU fault: a launch failure injected on the
host (FD_TEST_FAIL_LAUNCH in the environment) must come back as
FD_ERR_LAUNCH from every compute entry point, leave the outputs untouched,
and leave the device usable. The flag is read once per process, so the
failing calls run in a child process."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

CHILD = r"""
import torch
import decode_attention_07_b200 as fd
from decode_attention_07_b200.configs import Workload
from decode_attention_07_b200.inputs import make_inputs, make_quant
w = Workload("inj", B=2, Hq=8, Hkv=2, D=128, Lmax=500, ragged=False)
x = make_inputs(w, 0, device="cuda")
out = torch.full((2, 8, 128), 7.0, device="cuda")
lse = torch.full((2, 8), 7.0, device="cuda")
S = fd.fd_plan(2, 8, 2, 128, 500)
ws = torch.zeros(fd.fd_workspace_bytes(2, 8, 2, 128, 500, S), dtype=torch.uint8, device="cuda")
codes = []
def expect_launch_error(f):
    try:
        f()
    except fd.FdError as e:
        codes.append(e.code)
        return
    codes.append(0)
expect_launch_error(lambda: fd.fd_decode(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws))
expect_launch_error(lambda: fd.fd_decode_splits(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws, S))
expect_launch_error(lambda: fd.fd_split(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws, S))
expect_launch_error(lambda: fd.fd_combine(2, 8, 2, 128, 500, x.seqlens, out, lse, ws, S))
xq = make_quant(w, "e4m3", 0, device="cuda")
expect_launch_error(lambda: fd.fd_decode_quant(xq.q, xq.k8, xq.v8, xq.k_scale, xq.v_scale, "e4m3", xq.seqlens,
                                               xq.scale, out, lse, ws, S))
expect_launch_error(lambda: fd.fd_merge_partials(out[None], lse[None], torch.empty_like(out), torch.empty_like(lse)))
torch.cuda.synchronize()
untouched = bool((out == 7.0).all() and (lse == 7.0).all())
import json
print("RESULT " + json.dumps({"codes": codes, "untouched": untouched, "status": fd.fd_device_status()}))
"""


def run_child(env_value):
    env = dict(os.environ)
    env.pop("FD_TEST_FAIL_LAUNCH", None)
    if env_value is not None:
        env["FD_TEST_FAIL_LAUNCH"] = env_value
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, cwd=root, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    return json.loads(line[len("RESULT "):])


def test_injected_launch_failure_is_reported():
    assert torch.cuda.is_available()
    res = run_child("1")
    assert res["codes"] == [-9] * 6, res      # FD_ERR_LAUNCH from every entry point
    assert res["untouched"], res              # nothing was launched, nothing written
    assert res["status"] == 0, res            # the device and the library stay usable


def test_without_injection_the_same_calls_run():
    res = run_child("0")
    assert res["codes"] == [0] * 6 and not res["untouched"] and res["status"] == 0, res
