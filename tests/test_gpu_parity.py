"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded bf16 inputs.

Tolerances (from the stated target for bf16 inputs with fp32 accumulation):
max |out - oracle| <= 2e-3 over every element, and
|lse - oracle| <= 1e-4 * max(1, |oracle|) (relative, made absolute near 0,
where a relative bound on a value near 0 means nothing). Rows with no
tokens must give out = 0 and lse = -inf exactly.
"""
import numpy as np
import pytest
import torch

import decode_attention_07_b200 as fd
import oracle
from decode_attention_07_b200.configs import WORKLOADS, Workload
from decode_attention_07_b200.inputs import bf16_bits, make_inputs

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3
LSE_REL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    assert fd.fd_device_status() == 0


def compare(out, lse, ref_out, ref_lse, what, out_tol=OUT_TOL, lse_rel=LSE_REL):
    out = out.detach().double().cpu().numpy() if torch.is_tensor(out) else np.asarray(out, np.float64)
    lse = lse.detach().double().cpu().numpy() if torch.is_tensor(lse) else np.asarray(lse, np.float64)
    assert out.shape == ref_out.shape and lse.shape == ref_lse.shape, what
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref_out).max() if out.size else 0.0
    assert err <= out_tol, f"{what}: max |out - oracle| = {err:.3e}"
    empty = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: -inf lse pattern differs"
    assert np.all(out[empty] == 0.0), f"{what}: empty rows must be 0"
    if (~empty).any():
        rel = np.abs(lse[~empty] - ref_lse[~empty]) / np.maximum(1.0, np.abs(ref_lse[~empty]))
        assert rel.max() <= lse_rel, f"{what}: lse error {rel.max():.3e}"
    return err


def oracle_rows(x, bs=None):
    """Oracle out/lse for sequences `bs` (all by default), reading only the
    valid prefix of each sequence's cache."""
    w = x.workload
    bs = range(w.B) if bs is None else bs
    ref_o = np.zeros((len(bs), w.Hq, w.D))
    ref_l = np.zeros((len(bs), w.Hq))
    for n, b in enumerate(bs):
        L = int(min(max(x.seqlens_host[b], 0), w.Lmax))
        o, l = oracle.attention(bf16_bits(x.q[b:b + 1]), bf16_bits(x.k[b:b + 1, :, :L]),
                                bf16_bits(x.v[b:b + 1, :, :L]), np.array([L], np.int32), x.scale)
        ref_o[n], ref_l[n] = o[0], l[0]
    return ref_o, ref_l


def run(x, num_splits=None, stream=None):
    return fd.decode(x.q, x.k, x.v, x.seqlens, x.scale, num_splits=num_splits, stream=stream)


# ------------------------------------------------------------ the workloads --

@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("name", ["tiny_mha", "mha_16k", "gqa_128k", "batch_4k", "ragged_64k"])
def test_workload_against_oracle(name, seed):
    """Each workload at full size with the planned split count (the launch the
    benchmark times). Seed 0 checks every output; seeds 1 and 2 of the three
    largest workloads check a sample of sequences (all of their heads)."""
    w = WORKLOADS[name]
    x = make_inputs(w, seed, device="cuda")
    out, lse = run(x)
    torch.cuda.synchronize()
    if seed == 0 or name in ("tiny_mha", "mha_16k"):
        bs = list(range(w.B))
    else:
        rng = np.random.default_rng(seed)
        bs = sorted(set(rng.choice(w.B, size=min(w.B, 6), replace=False).tolist()) | {int(np.argmax(x.seqlens_host))})
    ref_o, ref_l = oracle_rows(x, bs)
    compare(out[bs], lse[bs], ref_o, ref_l, f"{name} seed {seed}")


@pytest.mark.parametrize("splits_per_row", [1, 4])
def test_tiny_single_and_four_splits(splits_per_row):
    """The tiny MHA case unsplit and with every row cut into 4 splits
    (4 rows x 4 = 16 runs of 4 tiles)."""
    w = WORKLOADS["tiny_mha"]
    x = make_inputs(w, 0, device="cuda")
    S = 1 if splits_per_row == 1 else 16
    seg = fd.fd_segments(w.B, w.Hkv, w.Lmax, x.seqlens_host, S)
    per_row = np.bincount(seg["row"][seg["row"] >= 0], minlength=w.B * w.Hkv)
    assert np.all(per_row == splits_per_row)
    out, lse = run(x, S)
    ref_o, ref_l = oracle_rows(x)
    compare(out, lse, ref_o, ref_l, f"tiny, {splits_per_row} split(s) per row")


# ---------------------------------------------------- split identity etc. --

def mid_case(g, D, seed=5, B=3, Lmax=5000, lens=(5000, 1234, 3)):
    w = Workload("mid", B=B, Hq=2 * g, Hkv=2, D=D, Lmax=Lmax, ragged=False, sigma_k=2.0, nan_pad=True)
    return make_inputs(w, seed, device="cuda", seqlens=list(lens))


@pytest.mark.parametrize("g,D", [(1, 128), (8, 128), (4, 64), (16, 128)])
def test_split_count_invariance_and_determinism(g, D):
    x = mid_case(g, D)
    ref_o, ref_l = oracle_rows(x)
    results = {}
    for S in (1, 2, 4, 7, 37, fd.fd_plan(*[x.workload.B, x.workload.Hq, x.workload.Hkv, D, x.workload.Lmax]), 148,
              400):
        out, lse = run(x, S)
        compare(out, lse, ref_o, ref_l, f"g={g} D={D} S={S}")
        results[S] = (out.clone(), lse.clone())
        again = run(x, S)
        assert torch.equal(again[0], out) and torch.equal(again[1], lse), f"S={S}: not deterministic"
    base_o, base_l = results[1]
    for S, (o, l) in results.items():
        assert (o - base_o).abs().max().item() <= 2e-5, f"S={S} differs from S=1 beyond fp32 rounding"
        assert (l - base_l).abs().max().item() <= 2e-5


# --------------------------------------------------------------- edge cases --

EDGE = [
    # (B, Hq, Hkv, D, Lmax, seqlens)
    (1, 1, 1, 64, 1, [1]),
    (1, 8, 1, 128, 1, [1]),
    (2, 4, 4, 128, 130, [63, 130]),
    (3, 6, 2, 64, 100, [100, 65, 64]),
    (4, 16, 2, 128, 700, [0, 700, 1, 0]),
    (2, 12, 4, 128, 257, [999, -7]),             # clamped to Lmax and to 0
    (5, 10, 2, 64, 96, [17, 96, 33, 80, 1]),     # g = 5
    (1, 32, 2, 128, 3000, [2999]),               # g = 16
    (40, 8, 8, 128, 200, list(range(0, 200, 5))),
    (2, 3, 1, 128, 64, [64, 32]),                # g = 3
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: f"B{c[0]}-Hq{c[1]}-Hkv{c[2]}-D{c[3]}-L{c[4]}")
def test_edge_shapes(case):
    B, Hq, Hkv, D, Lmax, lens = case
    w = Workload("edge", B=B, Hq=Hq, Hkv=Hkv, D=D, Lmax=Lmax, ragged=False, sigma_k=3.0, nan_pad=True)
    x = make_inputs(w, 11, device="cuda", seqlens=lens)
    ref_o, ref_l = oracle_rows(x)
    for S in (1, 3, fd.fd_plan(B, Hq, Hkv, D, Lmax), 200):
        out, lse = run(x, S)
        compare(out, lse, ref_o, ref_l, f"{case} S={S}")


def test_zero_length_cache():
    """max_len = 0: no token anywhere, every row is (0, -inf)."""
    q = torch.randn(2, 4, 64, device="cuda").to(torch.bfloat16)
    k = torch.empty(2, 2, 0, 64, device="cuda", dtype=torch.bfloat16)
    lens = torch.zeros(2, dtype=torch.int32, device="cuda")
    for S in (1, 5):
        out, lse = fd.decode(q, k, k, lens, 0.125, num_splits=S)
        assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_guard_bands_untouched():
    """Outputs and workspace carved out of larger buffers whose tails hold a
    sentinel: the kernels write nothing past the documented sizes."""
    x = mid_case(8, 128)
    w = x.workload
    S = 37
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.Lmax, S)
    ws = torch.full((nbytes + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    ws[:nbytes].zero_()                      # the row counters start at zero
    out_buf = torch.full((w.B * w.Hq * w.D + 1024,), 12345.0, device="cuda")
    lse_buf = torch.full((w.B * w.Hq + 1024,), 12345.0, device="cuda")
    out = out_buf[:w.B * w.Hq * w.D].view(w.B, w.Hq, w.D)
    lse = lse_buf[:w.B * w.Hq].view(w.B, w.Hq)
    fd.fd_decode_splits(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws[:nbytes], S)
    torch.cuda.synchronize()
    assert torch.all(ws[nbytes:] == 0xA5)
    assert torch.all(out_buf[w.B * w.Hq * w.D:] == 12345.0) and torch.all(lse_buf[w.B * w.Hq:] == 12345.0)
    ref_o, ref_l = oracle_rows(x)
    compare(out, lse, ref_o, ref_l, "guard-band run")


def test_non_default_stream():
    x = mid_case(4, 128)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, lse = run(x, 9, stream=s)
    s.synchronize()
    ref_o, ref_l = oracle_rows(x)
    compare(out, lse, ref_o, ref_l, "side stream")


# ------------------------------------------------ the two stages on their own --

def segment_oracle(x, seg):
    """Oracle (out, lse) of every used workspace slot: attention of each
    query head of the slot's row over the slot's token range."""
    w = x.workload
    res = {}
    for s in np.nonzero(seg["row"] >= 0)[0]:
        u = int(seg["row"][s])
        b, j = divmod(u, w.Hkv)
        t0, t1 = int(seg["begin"][s]), int(seg["end"][s])
        o, l = oracle.attention(bf16_bits(x.q[b:b + 1, j * w.g:(j + 1) * w.g]),
                                bf16_bits(x.k[b:b + 1, j:j + 1, t0:t1]), bf16_bits(x.v[b:b + 1, j:j + 1, t0:t1]),
                                np.array([t1 - t0], np.int32), x.scale)
        res[int(s)] = (o[0], l[0])
    return res


@pytest.mark.parametrize("g,D,S", [(1, 128, 11), (8, 128, 37), (4, 64, 23)])
def test_split_stage_segments_against_oracle(g, D, S):
    """fd_split alone: every segment it writes to the workspace equals the
    oracle's attention over that segment's token range (normalised output and
    log-sum-exp), and rows held whole are final already."""
    x = mid_case(g, D)
    w = x.workload
    seg = fd.fd_segments(w.B, w.Hkv, w.Lmax, x.seqlens_host, S)
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.Lmax, S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.full((w.B, w.Hq, w.D), 777.0, device="cuda")
    lse = torch.full((w.B, w.Hq), 777.0, device="cuda")
    fd.fd_split(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws, S)
    torch.cuda.synchronize()
    slots, gg, off, _ = fd.workspace_layout(w.B, w.Hq, w.Hkv, w.D, S)
    seg_out = ws[:slots * gg * w.D * 4].view(torch.float32).view(slots, gg, w.D).cpu().numpy()
    seg_lse = ws[off:off + slots * gg * 4].view(torch.float32).view(slots, gg).cpu().numpy()
    ref = segment_oracle(x, seg)
    ref_o, ref_l = oracle_rows(x)
    checked = 0
    for s, (o, l) in ref.items():
        u = int(seg["row"][s])
        b, j = divmod(u, w.Hkv)
        if seg["whole"][s]:
            compare(out[b, j * w.g:(j + 1) * w.g], lse[b, j * w.g:(j + 1) * w.g], ref_o[b, j * w.g:(j + 1) * w.g],
                    ref_l[b, j * w.g:(j + 1) * w.g], f"whole row {u}")
        else:
            compare(seg_out[s], seg_lse[s], o, l, f"segment {s} of row {u}")
            checked += 1
    assert checked > 0


@pytest.mark.parametrize("g,D,S", [(8, 128, 37), (1, 64, 13)])
def test_combine_stage_alone_on_oracle_partials(g, D, S):
    """fd_combine alone, fed the oracle's per-segment results (rounded to
    fp32) in the documented workspace layout, against the oracle's own
    reduction of the same partials."""
    x = mid_case(g, D)
    w = x.workload
    seg = fd.fd_segments(w.B, w.Hkv, w.Lmax, x.seqlens_host, S)
    ref = segment_oracle(x, seg)
    slots, gg, off, _ = fd.workspace_layout(w.B, w.Hq, w.Hkv, w.D, S)
    so = np.zeros((slots, gg, w.D), np.float32)
    sl = np.zeros((slots, gg), np.float32)
    for s, (o, l) in ref.items():
        so[s], sl[s] = o, l
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.Lmax, S)
    host = np.zeros(nbytes, np.uint8)
    host[:so.nbytes] = so.view(np.uint8).ravel()
    host[off:off + sl.nbytes] = sl.view(np.uint8).ravel()
    ws = torch.from_numpy(host).cuda()
    out = torch.full((w.B, w.Hq, w.D), 777.0, device="cuda")
    lse = torch.full((w.B, w.Hq), 777.0, device="cuda")
    fd.fd_combine(w.B, w.Hq, w.Hkv, w.D, w.Lmax, x.seqlens, out, lse, ws, S)
    torch.cuda.synchronize()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    multi = 0
    for u in range(w.B * w.Hkv):
        b, j = divmod(u, w.Hkv)
        rows = slice(j * w.g, (j + 1) * w.g)
        mine = [s for s in ref if seg["row"][s] == u]
        if int(min(max(x.seqlens_host[b], 0), w.Lmax)) == 0:
            assert np.all(out[b, rows] == 0) and np.all(np.isneginf(lse[b, rows]))
            continue
        if len(mine) < 2:
            continue
        multi += 1
        po = np.stack([so[s] for s in mine], axis=1).astype(np.float64)       # [g, nseg, D]
        pl = np.stack([sl[s] for s in mine], axis=1).astype(np.float64)       # [g, nseg]
        ro, rl = oracle.combine(po, pl)
        compare(out[b, rows], lse[b, rows], ro, rl, f"combine row {u}", out_tol=1e-5, lse_rel=1e-6)
    assert multi > 0


@pytest.mark.parametrize("g,D,S", [(1, 128, 37), (8, 128, 148), (4, 64, 23), (16, 128, 61)])
def test_fused_equals_two_stages(g, D, S):
    """fd_decode (split with the reduction fused in) gives bitwise the same
    out/lse as fd_split followed by fd_combine."""
    x = mid_case(g, D)
    w = x.workload
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.Lmax, S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    o1 = torch.empty((w.B, w.Hq, w.D), device="cuda")
    l1 = torch.empty((w.B, w.Hq), device="cuda")
    fd.fd_decode_splits(x.q, x.k, x.v, x.seqlens, x.scale, o1, l1, ws, S)
    o2 = torch.full_like(o1, 5.0)
    l2 = torch.full_like(l1, 5.0)
    ws2 = torch.zeros_like(ws)
    fd.fd_split(x.q, x.k, x.v, x.seqlens, x.scale, o2, l2, ws2, S)
    fd.fd_combine(w.B, w.Hq, w.Hkv, w.D, w.Lmax, x.seqlens, o2, l2, ws2, S)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# Shapes that send the rows a block completes down each merge path of the
# fused reduction: at most 8 segments (merged straight from L2); up to 64
# whose outputs fit 160 KB (staged in shared memory, alone or two rows
# together); more, or larger (two levels: chunks of 8 segments, then the
# chunks' partials, direct, staged or from L2); more runs than tiles (empty
# runs and empty chunks). Each is checked against the oracle, and bitwise
# against the standalone combine kernel, which reads every segment from L2.
MERGE_PATHS = [
    # B, Hq, Hkv, D, Lmax, lens, S
    (1, 32, 32, 128, 16384, None, None),        # 4-6 segments per row: direct
    (1, 8, 8, 128, 8192, None, 148),            # ~19 segments, one column: staged
    (1, 64, 8, 128, 8192, None, 148),           # ~19 segments of 8 columns, up to two rows a block
    (1, 4, 4, 64, 16384, None, 148),            # ~37 segments at D = 64: staged
    (1, 32, 4, 128, 16384, None, 148),          # ~37 segments of 8 columns (148 KB): staged
    (1, 24, 3, 128, 16384, None, 148),          # ~49 segments of 8 columns (196 KB): two levels, 7 partials direct
    (1, 32, 2, 128, 8192, None, 60),            # 30 segments of 16 columns (240 KB): two levels, 4 partials
    (1, 8, 1, 128, 65536, None, 148),           # one row of 148 segments: 19 partials, staged
    (1, 16, 1, 64, 32768, None, 148),           # 16 columns at D = 64
    (1, 16, 1, 128, 65536, None, 400),          # 400 segments of 16 columns: 50 partials, from L2
    (1, 8, 1, 128, 6400, None, 148),            # 100 tiles over 148 runs: empty runs and chunks
    (3, 24, 3, 128, 20000, (20000, 9000, 0), 148),   # long and short rows mixed, one sequence empty
]


@pytest.mark.parametrize("case", MERGE_PATHS, ids=lambda c: f"B{c[0]}-Hq{c[1]}-Hkv{c[2]}-D{c[3]}-L{c[4]}")
def test_completed_row_merge_paths(case):
    B, Hq, Hkv, D, Lmax, lens, S = case
    w = Workload("merge", B=B, Hq=Hq, Hkv=Hkv, D=D, Lmax=Lmax, ragged=False, sigma_k=2.0)
    x = make_inputs(w, 11, device="cuda", seqlens=list(lens) if lens else None)
    S = S or fd.fd_plan(B, Hq, Hkv, D, Lmax)
    nbytes = fd.fd_workspace_bytes(B, Hq, Hkv, D, Lmax, S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    o1 = torch.empty((B, Hq, D), device="cuda")
    l1 = torch.empty((B, Hq), device="cuda")
    for _ in range(2):   # the second call reuses the row counters the first one reset
        fd.fd_decode_splits(x.q, x.k, x.v, x.seqlens, x.scale, o1, l1, ws, S)
    o2 = torch.full_like(o1, 5.0)
    l2 = torch.full_like(l1, 5.0)
    ws2 = torch.zeros_like(ws)
    fd.fd_split(x.q, x.k, x.v, x.seqlens, x.scale, o2, l2, ws2, S)
    fd.fd_combine(B, Hq, Hkv, D, Lmax, x.seqlens, o2, l2, ws2, S)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    ref_o, ref_l = oracle_rows(x)
    compare(o1, l1, ref_o, ref_l, f"merge paths {case}")


def test_workspace_reuse_leaves_counters_at_zero():
    """One workspace across calls with different inputs and lengths: every
    call is right, and the row counters are back at zero after each."""
    w = Workload("reuse", B=4, Hq=16, Hkv=4, D=128, Lmax=3000, ragged=False, sigma_k=2.0, nan_pad=True)
    S = 97
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, w.Lmax, S)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    fd.fd_workspace_init(ws)
    slots, _, _, tick = fd.workspace_layout(w.B, w.Hq, w.Hkv, w.D, S)
    out = torch.empty((w.B, w.Hq, w.D), device="cuda")
    lse = torch.empty((w.B, w.Hq), device="cuda")
    for seed, lens in ((1, [3000, 17, 0, 2999]), (2, [64, 3000, 1500, 1]), (3, [0, 0, 0, 700])):
        x = make_inputs(w, seed, device="cuda", seqlens=lens)
        fd.fd_decode_splits(x.q, x.k, x.v, x.seqlens, x.scale, out, lse, ws, S)
        torch.cuda.synchronize()
        ref_o, ref_l = oracle_rows(x)
        compare(out, lse, ref_o, ref_l, f"reuse seed {seed}")
        assert torch.all(ws[tick:tick + 4 * (w.B * w.Hkv + slots)] == 0)
