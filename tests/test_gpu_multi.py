"""Several queries per sequence (fd_decode_multi) on the GPU against the
CPU oracle's multi-query definition: sequence b holds seqlens[b] tokens
including the q_len new ones, and query j sees the first
seqlens[b] - (q_len - 1 - j) of them."""
import numpy as np
import pytest
import torch

import decode_attention_07_b200 as fd
import oracle
from decode_attention_07_b200.configs import WORKLOADS, Workload
from decode_attention_07_b200.inputs import bf16_bits, make_inputs
from test_gpu_parity import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    assert fd.fd_device_status() == 0


def multi_case(w, seed, q_len, lens=None):
    x = make_inputs(w, seed, device="cuda", seqlens=lens)
    g = torch.Generator(device="cuda").manual_seed(1000 + seed)
    q = torch.randn((w.B, q_len, w.Hq, w.D), generator=g, device="cuda").to(torch.bfloat16)
    return x, q


def oracle_multi(x, q, bs=None):
    w = x.workload
    bs = range(w.B) if bs is None else bs
    q_len = q.shape[1]
    ref_o = np.zeros((len(bs), q_len, w.Hq, w.D))
    ref_l = np.zeros((len(bs), q_len, w.Hq))
    for n, b in enumerate(bs):
        L = int(min(max(x.seqlens_host[b], 0), w.Lmax))
        o, l = oracle.attention_multi(bf16_bits(q[b:b + 1]), bf16_bits(x.k[b:b + 1, :, :L]),
                                      bf16_bits(x.v[b:b + 1, :, :L]), np.array([L], np.int32), x.scale)
        ref_o[n], ref_l[n] = o[0], l[0]
    return ref_o, ref_l


@pytest.mark.parametrize("q_len,g,D", [(1, 4, 128), (2, 8, 128), (3, 4, 128), (4, 4, 64), (8, 1, 128),
                                       (2, 1, 64), (5, 3, 128), (16, 1, 128), (4, 2, 64)])
def test_multi_query_against_oracle(q_len, g, D):
    w = Workload("mq", B=4, Hq=2 * g, Hkv=2, D=D, Lmax=3000, ragged=False, sigma_k=3.0, nan_pad=True)
    x, q = multi_case(w, 4, q_len, lens=[3000, q_len, 1777, 70])
    ref_o, ref_l = oracle_multi(x, q)
    for S in (1, fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax), 61):
        out, lse = fd.decode_multi(q, x.k, x.v, x.seqlens, x.scale, num_splits=S)
        torch.cuda.synchronize()
        compare(out, lse, ref_o, ref_l, f"q_len={q_len} g={g} D={D} S={S}")


@pytest.mark.parametrize("q_len,Hq,Hkv,L", [(2, 32, 8, 8192), (2, 64, 8, 8192), (2, 16, 4, 8192),
                                         (2, 8, 1, 16384)])
def test_multi_query_long_rows(q_len, Hq, Hkv, L):
    """Rows of ~19 segments (148 splits over 8 rows) with 8 and 16 columns
    each (q_len * g; staged in shared memory), of ~37 segments of 8 columns
    (staged) and one row of 148 segments of 16 columns (two levels, 19
    partials)."""
    w = Workload("mq_long", B=1, Hq=Hq, Hkv=Hkv, D=128, Lmax=L, ragged=False, sigma_k=2.0)
    x, q = multi_case(w, 6, q_len)
    ref_o, ref_l = oracle_multi(x, q)
    out, lse = fd.decode_multi(q, x.k, x.v, x.seqlens, x.scale, num_splits=148)
    torch.cuda.synchronize()
    compare(out, lse, ref_o, ref_l, f"q_len={q_len} Hq={Hq} Hkv={Hkv}")


def test_queries_before_the_cache_start_are_empty():
    """A sequence shorter than q_len: the first queries see no token and
    give out = 0, lse = -inf."""
    w = Workload("mq", B=2, Hq=4, Hkv=2, D=128, Lmax=64, ragged=False, nan_pad=True)
    x, q = multi_case(w, 5, 4, lens=[2, 64])
    out, lse = fd.decode_multi(q, x.k, x.v, x.seqlens, x.scale, num_splits=3)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_multi(x, q)
    assert np.all(np.isneginf(ref_l[0, :2]))
    compare(out, lse, ref_o, ref_l, "short sequence")


def test_single_query_equals_fd_decode():
    """q_len = 1 gives bitwise the same result as fd_decode_splits."""
    w = Workload("mq", B=3, Hq=16, Hkv=2, D=128, Lmax=5000, ragged=False, nan_pad=True)
    x = make_inputs(w, 6, device="cuda", seqlens=[5000, 4000, 3])
    out1, lse1 = fd.decode_multi(x.q[:, None], x.k, x.v, x.seqlens, x.scale, num_splits=37)
    out2, lse2 = fd.decode(x.q, x.k, x.v, x.seqlens, x.scale, num_splits=37)
    torch.cuda.synchronize()
    assert torch.equal(out1[:, 0], out2) and torch.equal(lse1[:, 0], lse2)


@pytest.mark.parametrize("name,q_len", [("gqa_128k", 2), ("mha_16k", 4)])
def test_multi_query_full_size(name, q_len):
    """Full-size workloads with several queries, in the planned launch."""
    w = WORKLOADS[name]
    x, q = multi_case(w, 0, q_len)
    out, lse = fd.decode_multi(q, x.k, x.v, x.seqlens, x.scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_multi(x, q)
    compare(out, lse, ref_o, ref_l, f"{name} q_len={q_len}")
