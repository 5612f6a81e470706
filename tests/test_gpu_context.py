"""Context parallelism on one GPU: the cache is cut into R token ranges,
each range is decoded on its own (as one rank of R would), and
fd_merge_partials reduces the R partials; the result must match the oracle
over the whole cache. The ranks are run one after another (nothing waits on
another rank), and the merge kernel is also checked alone against the
oracle's reduction."""
import numpy as np
import pytest
import torch

import decode_attention_07_b200 as fd
import oracle
from decode_attention_07_b200 import context
from decode_attention_07_b200.configs import WORKLOADS, Workload
from decode_attention_07_b200.inputs import make_inputs
from test_gpu_parity import compare, oracle_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    assert fd.fd_device_status() == 0


@pytest.mark.parametrize("R,D", [(1, 128), (2, 64), (5, 128), (37, 128), (3, 4), (8, 256)])
def test_merge_partials_against_oracle(R, D):
    g = torch.Generator(device="cpu").manual_seed(R * 1000 + D)
    rows = 50
    po = torch.randn((R, rows, D), generator=g) * 3
    pl = torch.randn((R, rows), generator=g) * 20
    pl[torch.rand((R, rows), generator=g) < 0.3] = -float("inf")   # empty parts
    pl[:, 7] = -float("inf")                                          # a row with no tokens at all
    po[pl == -float("inf")] = 0.0
    ref_o, ref_l = oracle.combine(po.permute(1, 0, 2).double().numpy(), pl.permute(1, 0).double().numpy())
    out = torch.empty((rows, D), device="cuda")
    lse = torch.empty((rows,), device="cuda")
    fd.fd_merge_partials(po.cuda().contiguous(), pl.cuda().contiguous(), out, lse)
    torch.cuda.synchronize()
    compare(out, lse, ref_o, ref_l, f"merge R={R} D={D}", out_tol=1e-5)


def sharded_decode(x, R, S=None):
    """Decode each of R token ranges on its own, then merge the partials."""
    w = x.workload
    parts_o, parts_l = [], []
    for r in range(R):
        lo, hi = context.token_range(w.Lmax, r, R)
        k, v = x.k[:, :, lo:hi].contiguous(), x.v[:, :, lo:hi].contiguous()
        o, l = fd.decode(x.q, k, v, context.local_seqlens(x.seqlens, lo), x.scale, num_splits=S)
        parts_o.append(o)
        parts_l.append(l)
    out = torch.empty_like(parts_o[0])
    lse = torch.empty_like(parts_l[0])
    fd.fd_merge_partials(torch.stack(parts_o), torch.stack(parts_l), out, lse)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("R", [2, 3, 8])
@pytest.mark.parametrize("g", [1, 4])
def test_sharded_decode_against_oracle(R, g):
    w = Workload("cp", B=4, Hq=2 * g, Hkv=2, D=128, Lmax=1000, ragged=False, nan_pad=True)
    x = make_inputs(w, 3, device="cuda", seqlens=[1000, 130, 1, 0])   # some ranks hold no token of a row
    ref_o, ref_l = oracle_rows(x)
    for S in (None, 1, 7):
        out, lse = sharded_decode(x, R, S)
        compare(out, lse, ref_o, ref_l, f"R={R} g={g} S={S}")


def test_single_rank_is_plain_decode():
    """With one rank the merge returns the partial unchanged, bitwise."""
    w = Workload("cp", B=2, Hq=8, Hkv=2, D=128, Lmax=3000, ragged=False)
    x = make_inputs(w, 4, device="cuda")
    out, lse = context.cp_decode(x.q, x.k, x.v, x.seqlens, 0, x.scale)
    o2, l2 = fd.decode(x.q, x.k, x.v, x.seqlens, x.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, o2) and torch.equal(lse, l2)


def test_sharded_headline_workload():
    """mha_16k cut into 8 token ranges of 2048 (one per GPU of an 8-GPU node)."""
    x = make_inputs(WORKLOADS["mha_16k"], 0, device="cuda")
    out, lse = sharded_decode(x, 8)
    ref_o, ref_l = oracle_rows(x)
    compare(out, lse, ref_o, ref_l, "mha_16k over 8 token ranges")


def test_read_probe_reads_every_chunk():
    """The bandwidth probe folds the first 32-bit word of every 32 KiB chunk
    with xor: its result must equal that fold computed on the host (sizes
    with a short last chunk, fewer chunks than SMs, many per SM)."""
    import numpy as np
    for n_words in (4, 1000 * 4, (1 << 22) + 12, (1 << 25) + 4):
        g = torch.Generator(device="cpu").manual_seed(n_words)
        host = torch.randint(-2**31, 2**31 - 1, (n_words,), generator=g, dtype=torch.int64).to(torch.int32)
        sink = torch.zeros(1, dtype=torch.int64, device="cuda")
        fd.fd_read_probe(host.cuda(), sink)
        torch.cuda.synchronize()
        words = host.numpy().view(np.uint32)[::32768 // 4]
        want = int(np.bitwise_xor.reduce(words))
        got = int(sink.item())
        assert got >> 32 == 0, "a bounded wait gave up"
        assert got & 0xFFFFFFFF == want
