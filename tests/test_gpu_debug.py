"""The debug build (-DFD_DEBUG): device-side bounds checks on every global
access whose index comes from the partition arithmetic, and 50 ms bounded
waits. Run in child processes that load libfdecode_debug.so (FD_DEBUG=1):
  * a set of problems (GQA, MHA, ragged with empty rows, many splits,
    several queries, paged, 8-bit) passes its checks (status 0) and matches
    the release build bitwise;
  * FD_DEBUG_WITHHOLD=n makes block 0 arm its n-th tile without issuing the
    copy: a consumer's bounded wait runs out, the call reports
    FD_ERR_TIMEOUT through fd_device_status, and the next call on the same
    device and stream runs clean."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

CHILD = r"""
import json, os, sys
import torch
import decode_attention_07_b200 as fd
from decode_attention_07_b200.configs import Workload
from decode_attention_07_b200.inputs import make_inputs, make_paged, make_quant
def cases():
    yield "gqa", Workload("d1", B=3, Hq=16, Hkv=2, D=128, Lmax=3000, ragged=False), [3000, 0, 777], None
    yield "mha_many_splits", Workload("d2", B=2, Hq=4, Hkv=4, D=64, Lmax=700, ragged=False), [700, 65], 400
    yield "ragged", Workload("d3", B=5, Hq=8, Hkv=8, D=128, Lmax=2000, ragged=False), [2000, 1, 0, 1999, 64], 37
res = {}
for name, w, lens, S in cases():
    x = make_inputs(w, 1, device="cuda", seqlens=lens)
    o, l = fd.decode(x.q, x.k, x.v, x.seqlens, x.scale, num_splits=S)
    torch.cuda.synchronize()
    res[name] = [fd.fd_device_status(), o.double().sum().item(), l[torch.isfinite(l)].double().sum().item()]
w = Workload("d4", B=2, Hq=8, Hkv=2, D=128, Lmax=1500, ragged=False)
x = make_inputs(w, 2, device="cuda", seqlens=[1500, 3])
g = torch.Generator(device="cuda").manual_seed(3)
q = torch.randn((2, 4, 8, 128), generator=g, device="cuda").to(torch.bfloat16)
o, l = fd.decode_multi(q, x.k, x.v, x.seqlens, x.scale, num_splits=9)
torch.cuda.synchronize()
res["multi"] = [fd.fd_device_status(), o.double().sum().item(), l[torch.isfinite(l)].double().sum().item()]
pg = make_paged(x, 16, "HND", seed=4)
o, l = fd.decode_paged(x.q, pg.k_pages, pg.v_pages, pg.block_table, x.seqlens, x.scale, "HND", num_splits=9)
torch.cuda.synchronize()
res["paged"] = [fd.fd_device_status(), o.double().sum().item(), l[torch.isfinite(l)].double().sum().item()]
wm = Workload("d4m", B=2, Hq=4, Hkv=4, D=128, Lmax=1500, ragged=False)
xm = make_inputs(wm, 7, device="cuda", seqlens=[1500, 37])
pg = make_paged(xm, 8, "NHD", seed=8, unused_entry=987654321)
o, l = fd.decode_paged(xm.q, pg.k_pages, pg.v_pages, pg.block_table, xm.seqlens, xm.scale, "NHD", num_splits=5)
torch.cuda.synchronize()
res["paged_nhd8"] = [fd.fd_device_status(), o.double().sum().item(), l[torch.isfinite(l)].double().sum().item()]
xq = make_quant(w, "e4m3", 5, device="cuda", seqlens=[1500, 700])
o, l = fd.decode_quant(xq.q, xq.k8, xq.v8, xq.k_scale, xq.v_scale, "e4m3", xq.seqlens, xq.scale, num_splits=9)
torch.cuda.synchronize()
res["quant"] = [fd.fd_device_status(), o.double().sum().item(), l[torch.isfinite(l)].double().sum().item()]
if os.environ.get("WITHHOLD_TEST"):
    w = Workload("d5", B=1, Hq=8, Hkv=2, D=128, Lmax=4096, ragged=False)
    x = make_inputs(w, 6, device="cuda")
    os.environ["FD_DEBUG_WITHHOLD"] = "2"
    fd.decode(x.q, x.k, x.v, x.seqlens, x.scale, num_splits=4)
    res["withheld_status"] = fd.fd_device_status()
    del os.environ["FD_DEBUG_WITHHOLD"]
    o, l = fd.decode(x.q, x.k, x.v, x.seqlens, x.scale, num_splits=4)
    torch.cuda.synchronize()
    res["after_status"] = fd.fd_device_status()
    res["after_finite"] = bool(torch.isfinite(o).all())
print("RESULT " + json.dumps(res))
"""


def run_child(debug, withhold=False):
    env = dict(os.environ)
    env["FD_DEBUG"] = "1" if debug else "0"
    env.pop("FD_DEBUG_WITHHOLD", None)
    env.pop("FD_TEST_FAIL_LAUNCH", None)
    if not debug:
        env.pop("FD_DEBUG_SPOIL_GUESS", None)
    if withhold:
        env["WITHHOLD_TEST"] = "1"
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, cwd=root, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1][len("RESULT "):])


@pytest.fixture(scope="module", autouse=True)
def debug_library():
    """The debug build, brought up to date with the sources (no-op when it is)."""
    from decode_attention_07_b200 import build as lib_build
    return lib_build.build(debug=True)


def test_debug_build_checks_pass_and_match_release():
    dbg = run_child(True)
    rel = run_child(False)
    for name, (status, osum, lsum) in dbg.items():
        assert status == 0, f"{name}: device status {status} in the debug build"
        assert rel[name][0] == 0
        assert (osum, lsum) == (rel[name][1], rel[name][2]), f"{name}: debug and release results differ"


def test_a_wrong_start_guess_restarts_the_ring():
    """FD_DEBUG_SPOIL_GUESS=1 makes every block's pre-wait guess of its start
    wrong: the tiles issued from it are drained and the ring restarts one
    phase on. Results must equal the release build's, with no error."""
    os.environ["FD_DEBUG_SPOIL_GUESS"] = "1"
    try:
        dbg = run_child(True)
    finally:
        del os.environ["FD_DEBUG_SPOIL_GUESS"]
    rel = run_child(False)
    for name, (status, osum, lsum) in dbg.items():
        assert status == 0, f"{name}: device status {status} with a spoiled guess"
        assert (osum, lsum) == (rel[name][1], rel[name][2]), f"{name}: results differ after a restart"


def test_a_wait_that_runs_out_is_reported():
    res = run_child(True, withhold=True)
    assert res["withheld_status"] == -10, res      # FD_ERR_TIMEOUT, read (and cleared) by fd_device_status
    assert res["after_status"] == 0 and res["after_finite"], res
