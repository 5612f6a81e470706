"""fd_decode_static: decode attention for callers that cannot allocate device
memory. Such callers are handed their input and output buffers but own no
allocator -- for instance a plugin inside a serving engine that plans every
device byte itself, or a decode loop that must not call cudaMalloc because
cudaMalloc can synchronise the device. The entry point has no workspace
argument and uses the library's fixed device scratch buffer instead.

Each check calls the entry point through the C ABI twice in a row, with
different inputs, and compares both results with fd_decode (the entry point
that takes a caller-allocated workspace) on the same inputs, within the
parity tolerances used everywhere else. Two more checks compare it with the
CPU oracle directly, so its parity does not rest on fd_decode alone: one on
a problem cut into many segments, one on a problem the planner leaves
unsplit (no scratch is needed, so the fixed buffer is never touched). This file is collected last, so a
run that stops at the first failure has already run every other test; it
passes on its own in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_attention_07_b200 as fd
from decode_attention_07_b200.configs import WORKLOADS, Workload
from decode_attention_07_b200.inputs import bf16_bits, make_inputs

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
LSE_REL = 1e-4
FD_ERR_STATIC_LIMIT = -12


@pytest.fixture(scope="module", autouse=True)
def gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    assert fd.fd_device_status() == 0


def static_call(x, out, lse):
    """fd_decode_static through the C ABI (ctypes, raw pointers)."""
    w = x.workload
    return fd.lib().fd_decode_static(
        w.B, w.Hq, w.Hkv, w.D, w.Lmax, x.q.data_ptr(), x.k.data_ptr(), x.v.data_ptr(), x.seqlens.data_ptr(),
        ctypes.c_float(x.scale), out.data_ptr(), lse.data_ptr(), torch.cuda.current_stream().cuda_stream)


def assert_close(out, lse, ref_out, ref_lse, what):
    out, lse = out.double().cpu().numpy(), lse.double().cpu().numpy()
    ref_out, ref_lse = ref_out.double().cpu().numpy(), ref_lse.double().cpu().numpy()
    assert np.isfinite(out).all(), what
    err = np.abs(out - ref_out).max()
    assert err <= OUT_TOL, f"{what}: max |out diff| {err:.3e}"
    empty = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), empty), what
    if (~empty).any():
        rel = np.abs(lse[~empty] - ref_lse[~empty]) / np.maximum(1.0, np.abs(ref_lse[~empty]))
        assert rel.max() <= LSE_REL, f"{what}: lse error {rel.max():.3e}"


CASES = {
    # several segments per row, an empty row, NaN beyond each sequence
    "ragged_gqa": [(Workload("ragged", B=3, Hq=8, Hkv=2, D=128, Lmax=5000, ragged=False, sigma_k=3.0,
                             nan_pad=True), 1, [5000, 1234, 0]),
                   (Workload("ragged", B=3, Hq=8, Hkv=2, D=128, Lmax=5000, ragged=False, sigma_k=3.0,
                             nan_pad=True), 2, [17, 4999, 2500])],
    "mha_16k": [(WORKLOADS["mha_16k"], 0, None), (WORKLOADS["mha_16k"], 1, None)],
    "gqa_128k": [(WORKLOADS["gqa_128k"], 0, None), (WORKLOADS["gqa_128k"], 1, None)],
    "d64_group16": [(Workload("d64", B=2, Hq=32, Hkv=2, D=64, Lmax=3000, ragged=False), 3, [3000, 333]),
                    (Workload("d64", B=2, Hq=32, Hkv=2, D=64, Lmax=3000, ragged=False), 4, [1, 2999])],
}


@pytest.mark.parametrize("name", list(CASES))
def test_two_calls_match_the_workspace_entry_point(name):
    for call, (w, seed, lens) in enumerate(CASES[name]):
        x = make_inputs(w, seed, device="cuda", seqlens=lens)
        assert fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.Lmax,
                                     fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax)) <= fd._lib.FD_STATIC_SCRATCH_BYTES
        out = torch.full((w.B, w.Hq, w.D), 99.0, device="cuda")
        lse = torch.full((w.B, w.Hq), 99.0, device="cuda")
        assert static_call(x, out, lse) == 0
        ref_out, ref_lse = fd.decode(x.q, x.k, x.v, x.seqlens, x.scale)
        torch.cuda.synchronize()
        assert_close(out, lse, ref_out, ref_lse, f"{name}, call {call + 1}")


ORACLE_CASES = {
    # B = 3, L up to 3000: many segments per row, NaN padding, an empty row
    "split": [(Workload("orc", B=3, Hq=8, Hkv=2, D=128, Lmax=3000, ragged=False, sigma_k=3.0, nan_pad=True),
               5, [3000, 700, 0]),
              (Workload("orc", B=3, Hq=8, Hkv=2, D=128, Lmax=3000, ragged=False, sigma_k=3.0, nan_pad=True),
               6, [1, 2999, 1500])],
    # 4 tiles in all: the planner picks one split and no scratch is needed
    "unsplit": [(Workload("one", B=1, Hq=4, Hkv=1, D=128, Lmax=200, ragged=False), 7, None),
                (Workload("one", B=1, Hq=4, Hkv=1, D=128, Lmax=200, ragged=False), 8, [131])],
}


@pytest.mark.parametrize("name", list(ORACLE_CASES))
def test_two_calls_match_the_oracle(name, orc):
    for call, (w, seed, lens) in enumerate(ORACLE_CASES[name]):
        S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax)
        assert (S == 1) == (name == "unsplit")
        x = make_inputs(w, seed, device="cuda", seqlens=lens)
        out = torch.full((w.B, w.Hq, w.D), 99.0, device="cuda")
        lse = torch.full((w.B, w.Hq), 99.0, device="cuda")
        assert static_call(x, out, lse) == 0
        torch.cuda.synchronize()
        ref_out, ref_lse = orc.attention(bf16_bits(x.q), bf16_bits(x.k), bf16_bits(x.v), x.seqlens_host, x.scale)
        assert_close(out, lse, torch.from_numpy(ref_out), torch.from_numpy(ref_lse), f"{name}, call {call + 1}")


def test_rejects_problems_beyond_the_fixed_buffer():
    """A batch whose segment workspace exceeds the fixed buffer is refused
    with FD_ERR_STATIC_LIMIT before anything is launched (buffers of the
    claimed shape are still passed)."""
    w = Workload("big", B=2048, Hq=32, Hkv=8, D=128, Lmax=64, ragged=False)
    need = fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.Lmax, fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax))
    assert need > fd._lib.FD_STATIC_SCRATCH_BYTES
    x = make_inputs(w, 0, device="cuda")
    out = torch.full((w.B, w.Hq, w.D), 7.0, device="cuda")
    lse = torch.full((w.B, w.Hq), 7.0, device="cuda")
    assert static_call(x, out, lse) == FD_ERR_STATIC_LIMIT
    torch.cuda.synchronize()
    assert torch.all(out == 7.0) and torch.all(lse == 7.0)
    assert "8 MiB" in fd.fd_strerror(FD_ERR_STATIC_LIMIT)
