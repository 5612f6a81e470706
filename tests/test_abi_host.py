"""The C-ABI library on the host (no GPU): it loads, exports every symbol the
header declares, rejects bad arguments before any CUDA call, and its host-side
logic (planner, workspace size, where rows are cut) matches the documented
rules, re-derived here independently of the library."""
import ctypes
import os
import re

import numpy as np
import pytest

import decode_attention_07_b200 as fd
from decode_attention_07_b200 import _lib
from decode_attention_07_b200.configs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fd.h")


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^FD_API[^(]*?\b(fd_\w+)\(", text, flags=re.M)))


def test_exports_every_declared_symbol():
    syms = header_symbols()
    assert len(syms) >= 11
    L = fd.lib()
    for s in syms:
        assert hasattr(L, s), f"{s} declared in fd.h but not exported"
    exported = set(re.findall(r" T (fd_\w+)", os.popen(f"nm -D --defined-only {_lib.LIBRARY}").read()))
    assert exported == set(syms), f"exports {exported ^ set(syms)} differ from the header"


def test_constants_match_header():
    text = open(HEADER).read()
    consts = dict(re.findall(r"#define (FD_\w+)\s+(-?\d+)", text))
    assert int(consts["FD_TILE_TOKENS"]) == _lib.FD_TILE_TOKENS
    assert int(consts["FD_MAX_SPLITS"]) == _lib.FD_MAX_SPLITS
    assert int(consts["FD_MAX_GROUP"]) == _lib.FD_MAX_GROUP
    assert int(consts["FD_KV_E4M3"]) == _lib.FD_KV_E4M3 and int(consts["FD_KV_INT8"]) == _lib.FD_KV_INT8
    assert int(consts["FD_KV_HND"]) == _lib.FD_KV_HND and int(consts["FD_KV_NHD"]) == _lib.FD_KV_NHD
    for code, name in _lib.ERRORS.items():
        assert int(consts[name]) == code


def test_strerror_and_version():
    assert fd.fd_version() >= 100
    for code in list(_lib.ERRORS) + [0]:
        assert fd.fd_strerror(code) and fd.fd_strerror(code) != "unknown error code"
    assert fd.fd_strerror(12345) == "unknown error code"


def plan_rule(B, Hq, Hkv, D, Lmax, sms):
    """The documented planner: one split per SM while every split keeps at
    least 4 tiles of 64 tokens per kv head, fewer splits for small batches;
    with at most 16 tiles per SM (and 64 SMs or more) a multiple of 32."""
    tiles = B * Hkv * -(-Lmax // 64)
    want = max(1, min(sms, -(-tiles // 4)))
    if sms >= 64 and tiles <= 16 * sms:
        want = min(want, sms // 32 * 32)
    return want


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_plan_for_workloads(name):
    w = WORKLOADS[name]
    for sms in (148, 132, 108, 1):
        assert fd.fd_plan_for_sms(w.B, w.Hq, w.Hkv, w.D, w.Lmax, sms) == plan_rule(w.B, w.Hq, w.Hkv, w.D, w.Lmax, sms)
    assert fd.fd_plan_for_sms(w.B, w.Hq, w.Hkv, w.D, w.Lmax, 148) == (16 if name == "tiny_mha" else 148)


def test_plan_small_and_edge_shapes():
    assert fd.fd_plan_for_sms(1, 1, 1, 64, 1, 148) == 1
    assert fd.fd_plan_for_sms(1, 1, 1, 64, 0, 148) == 1
    assert fd.fd_plan_for_sms(2, 4, 2, 128, 64 * 4 * 10, 148) == 40   # 2*2*40 tiles / 4
    assert fd.fd_plan_for_sms(1, 64, 8, 128, 8192, 148) == 128      # 1024 tiles: mid-size, a multiple of 32
    assert fd.fd_plan_for_sms(1, 64, 8, 128, 8192 * 3, 148) == 148  # 3072 tiles: one per SM
    assert fd.fd_plan_for_sms(1, 64, 8, 128, 8192, 60) == 60        # too few SMs to round
    L = fd.lib()
    assert L.fd_plan_for_sms(1, 3, 2, 128, 64, 148) == -3      # Hq % Hkv
    assert L.fd_plan_for_sms(1, 34, 2, 128, 64, 148) == -3     # group 17
    assert L.fd_plan_for_sms(1, 4, 4, 96, 64, 148) == -4       # D
    assert L.fd_plan_for_sms(0, 4, 4, 64, 64, 148) == -2
    assert L.fd_plan_for_sms(1, 4, 4, 64, -1, 148) == -2
    assert L.fd_plan_for_sms(1, 4, 4, 64, 64, 0) == -8


def test_workspace_bytes_formula():
    for (B, Hq, Hkv, D, S) in [(1, 32, 32, 128, 148), (1, 64, 8, 128, 148), (64, 32, 8, 128, 148),
                               (32, 32, 8, 128, 148), (1, 4, 4, 64, 16), (3, 12, 4, 64, 5)]:
        slots, g, off, tick = fd.workspace_layout(B, Hq, Hkv, D, S)
        assert off == (slots * g * D * 4 + 255) // 256 * 256
        assert tick == off + (slots * g * 4 + 255) // 256 * 256
        want = tick + ((B * Hkv + slots) * 4 + 255) // 256 * 256   # row counters, then chunk counters
        assert fd.fd_workspace_bytes(B, Hq, Hkv, D, 1000, S) == want
        assert fd.fd_workspace_bytes(B, Hq, Hkv, D, 1000, 1) == 0
    assert fd.fd_workspace_bytes(1, 3, 2, 64, 10, 4) == 0          # invalid shape
    assert fd.fd_workspace_bytes(1, 4, 2, 64, 10, 0) == 0          # invalid splits


def test_bad_arguments_return_codes_without_a_device():
    """Argument checks run before any CUDA call, so on a host without a GPU
    they still return their own code (not FD_ERR_DEVICE)."""
    L = fd.lib()
    buf = (ctypes.c_uint8 * 4096)()
    base = ctypes.addressof(buf)
    a16 = (base + 15) // 16 * 16
    p = ctypes.c_void_p(a16)

    def split(B=1, Hq=4, Hkv=4, D=64, Lmax=64, q=p, k=p, v=p, s=p, out=p, lse=p, ws=p, wsb=4096, S=1):
        return L.fd_decode_splits(B, Hq, Hkv, D, Lmax, q, k, v, s, 0.125, out, lse, ws, wsb, S, None)

    assert split(B=0) == -2
    assert split(Hq=6, Hkv=4) == -3
    assert split(D=80) == -4
    assert split(q=None) == -1 and split(k=None) == -1 and split(out=None) == -1 and split(s=None) == -1
    assert split(k=ctypes.c_void_p(a16 + 8)) == -5
    assert split(out=ctypes.c_void_p(a16 + 2)) == -5
    assert split(out=ctypes.c_void_p(a16 + 4)) == -5      # out needs 16 bytes (vector stores)
    assert split(lse=ctypes.c_void_p(a16 + 4)) != -5      # lse needs 4
    assert split(S=0) == -7 and split(S=70000) == -7
    assert split(S=4, ws=None) == -6
    assert split(S=4, wsb=16) == -6
    assert split(S=4, ws=ctypes.c_void_p(a16 + 4)) == -5
    assert L.fd_combine(1, 4, 4, 64, 64, None, p, p, p, 4096, 4, None) == -1
    assert L.fd_split(1, 4, 4, 64, 64, p, p, p, p, 0.1, p, p, None, 0, 2, None) == -6
    assert L.fd_workspace_init(None, 16, None) == -1
    assert L.fd_workspace_init(None, 0, None) == 0
    # a valid call reaches the device query and fails there on a CPU-only host
    if not os.path.exists("/dev/nvidia0"):
        assert split() == -8
        assert L.fd_decode(1, 4, 4, 64, 64, p, p, p, p, 0.125, p, p, None, 0, None) == -8


def test_paged_argument_errors_without_a_device():
    L = fd.lib()
    buf = (ctypes.c_uint8 * 4096)()
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    p = ctypes.c_void_p(a16)

    def paged(page_size=16, num_pages=8, max_pages=4, layout=0, bt=p, S=1, B=1, Hq=4, Hkv=2, D=128):
        return L.fd_decode_paged(B, Hq, Hkv, D, page_size, num_pages, max_pages, layout, p, p, p, bt, p, 0.1,
                                 p, p, p, 4096, S, None)

    assert paged(page_size=24) == -2 and paged(page_size=4) == -2 and paged(page_size=8192) == -2
    assert paged(max_pages=6) == -2 and paged(max_pages=0) == -2 and paged(num_pages=0) == -2
    assert paged(layout=2) == -2
    assert paged(bt=None) == -1
    assert paged(bt=ctypes.c_void_p(a16 + 4)) == -5
    assert paged(S=-1) == -7
    assert paged(Hq=3) == -3 and paged(D=96) == -4
    if not os.path.exists("/dev/nvidia0"):
        assert paged() == -8


def test_multi_query_argument_errors_without_a_device():
    L = fd.lib()
    buf = (ctypes.c_uint8 * 4096)()
    p = ctypes.c_void_p((ctypes.addressof(buf) + 15) // 16 * 16)

    def multi(q_len=2, Hq=4, Hkv=2, D=128, S=1, B=1):
        return L.fd_decode_multi(B, q_len, Hq, Hkv, D, 64, p, p, p, p, 0.1, p, p, p, 4096, S, None)

    assert multi(q_len=0) == -2 and multi(q_len=17) == -2
    assert multi(q_len=9, Hq=4) == -3          # 9 queries x 2 heads per kv head > 16 columns
    assert multi(q_len=3, Hq=3) == -3 and multi(D=96) == -4 and multi(S=-1) == -7
    if not os.path.exists("/dev/nvidia0"):
        assert multi() == -8 and multi(q_len=8) == -8


def test_quant_argument_errors_without_a_device():
    L = fd.lib()
    buf = (ctypes.c_uint8 * 4096)()
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    p = ctypes.c_void_p(a16)

    def quant(kv_type=1, q_len=1, Hq=4, Hkv=2, D=128, S=1, ks=p, vs=p, kc=p):
        return L.fd_decode_quant(1, q_len, Hq, Hkv, D, 64, kv_type, p, kc, p, ks, vs, p, 0.1, p, p, p, 4096, S,
                                 None)

    assert quant(kv_type=0) == -2 and quant(kv_type=3) == -2 and quant(q_len=0) == -2
    assert quant(q_len=9) == -3 and quant(Hq=3) == -3 and quant(D=96) == -4 and quant(S=-1) == -7
    assert quant(ks=None) == -1 and quant(vs=None) == -1
    assert quant(ks=ctypes.c_void_p(a16 + 2)) == -5 and quant(kc=ctypes.c_void_p(a16 + 8)) == -5
    if not os.path.exists("/dev/nvidia0"):
        assert quant() == -8 and quant(kv_type=2, q_len=2) == -8


def test_merge_partials_argument_errors_without_a_device():
    L = fd.lib()
    buf = (ctypes.c_uint8 * 4096)()
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    p = ctypes.c_void_p(a16)

    def merge(R=2, rows=3, D=128, po=p, out=p, pl=p):
        return L.fd_merge_partials(R, rows, D, po, pl, out, p, None)

    assert merge(R=0) == -2 and merge(rows=-1) == -2
    assert merge(D=6) == -4 and merge(D=0) == -4 and merge(D=8192) == -4
    assert merge(rows=0, po=None) == 0                      # nothing to merge: no pointer read, no CUDA call
    assert merge(po=None) == -1 and merge(pl=None) == -1
    assert merge(out=ctypes.c_void_p(a16 + 4)) == -5 and merge(pl=ctypes.c_void_p(a16 + 2)) == -5
    if not os.path.exists("/dev/nvidia0"):
        assert merge() == -8


def test_read_probe_argument_errors_without_a_device():
    L = fd.lib()
    buf = (ctypes.c_uint8 * 4096)()
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    p = ctypes.c_void_p(a16)
    assert L.fd_read_probe(p, 0, None, None) == 0          # nothing to read: no pointer used, no CUDA call
    assert L.fd_read_probe(None, 64, p, None) == -1 and L.fd_read_probe(p, 64, None, None) == -1
    assert L.fd_read_probe(ctypes.c_void_p(a16 + 4), 64, p, None) == -5
    assert L.fd_read_probe(p, 24, p, None) == -5 and L.fd_read_probe(p, 64, ctypes.c_void_p(a16 + 4), None) == -5
    if not os.path.exists("/dev/nvidia0"):
        assert L.fd_read_probe(p, 64, p, None) == -8


def test_quant_paged_argument_errors_without_a_device():
    L = fd.lib()
    buf = (ctypes.c_uint8 * 4096)()
    a16 = (ctypes.addressof(buf) + 15) // 16 * 16
    p = ctypes.c_void_p(a16)

    def qp(page_size=16, max_pages=4, layout=0, kv_type=1, q_len=1, Hq=4, D=128, bt=p, ks=p, S=1):
        return L.fd_decode_quant_paged(1, q_len, Hq, 2, D, page_size, 8, max_pages, layout, kv_type, p, p, p, ks, p,
                                       bt, p, 0.1, p, p, p, 4096, S, None)

    assert qp(page_size=24) == -2 and qp(max_pages=6) == -2 and qp(layout=2) == -2
    assert qp(kv_type=0) == -2 and qp(q_len=0) == -2
    assert qp(q_len=9) == -3 and qp(Hq=3) == -3 and qp(D=96) == -4 and qp(S=-1) == -7
    assert qp(bt=None) == -1 and qp(ks=None) == -1
    assert qp(bt=ctypes.c_void_p(a16 + 4)) == -5 and qp(ks=ctypes.c_void_p(a16 + 2)) == -5
    if not os.path.exists("/dev/nvidia0"):
        assert qp() == -8


def segments_rule(B, Hkv, Lmax, seqlens, P):
    """Independent statement of the documented partition: rows u = b*Hkv + j
    in order, ceil(L_b/64) tiles each, run i = flat tiles
    [floor(i*N/P), floor((i+1)*N/P)), segment slot = i + u."""
    lens = [min(max(int(x), 0), Lmax) for x in seqlens]
    tiles = [-(-L // 64) for L in lens]
    flat = []                       # (u, tile) in stream order
    for b in range(B):
        for j in range(Hkv):
            flat += [(b * Hkv + j, t) for t in range(tiles[b])]
    N = len(flat)
    segs = {}
    for i in range(P):
        lo, hi = i * N // P, (i + 1) * N // P
        for pos in range(lo, hi):
            u, t = flat[pos]
            segs.setdefault((i, u), []).append(t)
    out = {}
    rows_runs = {}
    for (i, u), ts in segs.items():
        rows_runs.setdefault(u, []).append(i)
    for (i, u), ts in segs.items():
        L = lens[u // Hkv]
        out[i + u] = (u, ts[0] * 64, min((ts[-1] + 1) * 64, L), int(len(rows_runs[u]) == 1))
    return out, N


@pytest.mark.parametrize("case", [
    (1, 4, 1024, [1024], 16), (1, 4, 1024, [1024], 1), (1, 4, 1024, [1024], 4),
    (3, 2, 500, [500, 1, 0], 7), (5, 3, 4096, [4096, 64, 65, 4000, 2], 148),
    (4, 8, 65536, [65536, 1, 30000, 12345], 148), (2, 1, 300, [999, -5], 3),
    (6, 2, 256, [0, 0, 256, 0, 130, 0], 11), (1, 1, 64, [64], 300),
    (3, 2, 5000, [5000, 1234, 3], 400), (2, 3, 640, [640, 300], 61),   # more runs than tiles
])
def test_segments_match_the_documented_partition(case):
    B, Hkv, Lmax, lens, P = case
    seg = fd.fd_segments(B, Hkv, Lmax, np.array(lens, np.int32), P)
    want, N = segments_rule(B, Hkv, Lmax, lens, P)
    assert len(seg["row"]) == P + B * Hkv - 1
    for s in range(len(seg["row"])):
        if s in want:
            u, b0, e0, wh = want[s]
            assert (seg["row"][s], seg["begin"][s], seg["end"][s], seg["whole"][s]) == (u, b0, e0, wh), s
        else:
            assert seg["row"][s] == -1
    # every valid token of every row lies in exactly one segment
    for b in range(B):
        L = min(max(lens[b], 0), Lmax)
        for j in range(Hkv):
            cover = np.zeros(L, np.int32)
            for s in np.nonzero(seg["row"] == b * Hkv + j)[0]:
                cover[seg["begin"][s]:seg["end"][s]] += 1
            assert np.all(cover == 1)


def test_segments_errors():
    L = fd.lib()
    arr = np.zeros(8, np.int32)
    lens = np.array([10, 10], np.int32)
    ptr = arr.ctypes.data
    assert L.fd_segments(2, 2, 10, lens.ctypes.data, 4, ptr, ptr, ptr, ptr, 4) == -11
    assert L.fd_segments(2, 2, 10, lens.ctypes.data, 0, ptr, ptr, ptr, ptr, 8) == -7
    assert L.fd_segments(2, 2, 10, None, 4, ptr, ptr, ptr, ptr, 8) == -1


def test_stale_library_is_reported(tmp_path):
    """A library file older than its sources is named by _newer_sources (the
    binding then warns at load time); one newer than all of them is not."""
    from decode_attention_07_b200.build import DEPS
    shipped = sorted(os.path.basename(d) for d in DEPS if os.path.exists(d))
    lib = tmp_path / "libx.so"
    lib.write_bytes(b"")
    os.utime(lib, (1, 1))
    assert _lib._newer_sources(str(lib)) == shipped
    newest = max(os.path.getmtime(d) for d in DEPS if os.path.exists(d))
    os.utime(lib, (newest + 10, newest + 10))
    assert _lib._newer_sources(str(lib)) == []
