"""Paged key/value cache (fd_decode_paged) on the GPU: the same logical
cache scattered into a shuffled pool of pages must give bitwise the same
out/lse as the contiguous path with the same split count, and match the
CPU oracle within the parity tolerances. Unused block-table entries hold
garbage to show they are never used."""
import numpy as np
import pytest
import torch

import decode_attention_07_b200 as fd
from decode_attention_07_b200.configs import WORKLOADS, Workload
from decode_attention_07_b200.inputs import make_inputs, make_paged
from test_gpu_parity import compare, oracle_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    assert fd.fd_device_status() == 0


def paged_vs_contiguous(x, page_size, layout, S, unused_entry=-1, check_oracle=True):
    pg = make_paged(x, page_size, layout, seed=page_size, unused_entry=unused_entry)
    out_p, lse_p = fd.decode_paged(x.q, pg.k_pages, pg.v_pages, pg.block_table, x.seqlens, x.scale, layout=layout,
                                   num_splits=S)
    out_c, lse_c = fd.decode(x.q, x.k, x.v, x.seqlens, x.scale, num_splits=S)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c), f"page {page_size} {layout}: differs from contiguous"
    if check_oracle:
        ref_o, ref_l = oracle_rows(x)
        compare(out_p, lse_p, ref_o, ref_l, f"paged {page_size} {layout}")


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("page_size", [8, 16, 32, 64, 256])
@pytest.mark.parametrize("g,D", [(4, 128), (1, 64), (1, 128), (8, 64), (16, 128)])
def test_paged_equals_contiguous(layout, page_size, g, D):
    w = Workload("paged", B=4, Hq=2 * g, Hkv=2, D=D, Lmax=3000, ragged=False, sigma_k=3.0, nan_pad=True)
    x = make_inputs(w, 9, device="cuda", seqlens=[3000, 1, 1777, 0])
    S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax)
    paged_vs_contiguous(x, page_size, layout, S, check_oracle=(page_size == 16))
    paged_vs_contiguous(x, page_size, layout, 7, unused_entry=987654321, check_oracle=False)


def test_paged_planned_split_count():
    """num_splits = 0 uses the planner on max_pages * page_size."""
    w = Workload("paged", B=3, Hq=8, Hkv=2, D=128, Lmax=2000, ragged=False, nan_pad=True)
    x = make_inputs(w, 3, device="cuda", seqlens=[2000, 999, 64])
    pg = make_paged(x, 32, "HND", seed=5)
    Lp = pg.block_table.shape[1] * 32
    S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, Lp)
    nbytes = fd.fd_workspace_bytes(w.B, w.Hq, w.Hkv, w.D, Lp, S)
    ws = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.B, w.Hq, w.D), device="cuda")
    lse = torch.empty((w.B, w.Hq), device="cuda")
    fd.fd_decode_paged(x.q, pg.k_pages, pg.v_pages, pg.block_table, x.seqlens, x.scale, out, lse, ws, "HND", 0)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_rows(x)
    compare(out, lse, ref_o, ref_l, "paged, planned splits")


@pytest.mark.parametrize("layout,page_size", [("HND", 16), ("NHD", 64)])
def test_paged_ragged_64k_full_size(layout, page_size):
    """The ragged workload at full size from a shuffled page pool, in the
    bench's launch configuration: bitwise equal to the contiguous path, and
    sampled sequences against the oracle."""
    w = WORKLOADS["ragged_64k"]
    x = make_inputs(w, 0, device="cuda")
    S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax)
    pg = make_paged(x, page_size, layout, seed=1)
    out_p, lse_p = fd.decode_paged(x.q, pg.k_pages, pg.v_pages, pg.block_table, x.seqlens, x.scale, layout=layout,
                                   num_splits=S)
    del pg
    out_c, lse_c = fd.decode(x.q, x.k, x.v, x.seqlens, x.scale, num_splits=S)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)
    bs = [int(np.argmax(x.seqlens_host)), int(np.argmin(x.seqlens_host)), 7]
    ref_o, ref_l = oracle_rows(x, bs)
    compare(out_p[bs], lse_p[bs], ref_o, ref_l, "ragged_64k paged")


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("page_size", [8, 16, 64])
@pytest.mark.parametrize("g", [1, 4])
def test_page_outside_the_pool_reads_zeros(layout, page_size, g):
    """A block-table entry past the pool (or negative) on a used page reads a
    page of zeros for K and V instead of faulting: against the oracle on the
    same cache with those tokens set to zero."""
    w = Workload("paged", B=2, Hq=2 * g, Hkv=2, D=128, Lmax=600, ragged=False, nan_pad=True)
    x = make_inputs(w, 11, device="cuda", seqlens=[600, 333])
    pg = make_paged(x, page_size, layout, seed=3)
    num_pages = pg.k_pages.shape[0]
    bad = {(0, 1): num_pages + 5, (1, 2): -3}   # (sequence, logical page) -> out-of-pool index
    for (b, lp), idx in bad.items():
        pg.block_table[b, lp] = idx
    S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax)
    out, lse = fd.decode_paged(x.q, pg.k_pages, pg.v_pages, pg.block_table, x.seqlens, x.scale, layout=layout,
                               num_splits=S)
    torch.cuda.synchronize()
    for (b, lp) in bad:
        x.k[b, :, lp * page_size:(lp + 1) * page_size] = 0
        x.v[b, :, lp * page_size:(lp + 1) * page_size] = 0
    ref_o, ref_l = oracle_rows(x)
    compare(out, lse, ref_o, ref_l, f"out-of-pool pages, {page_size} {layout}")


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("page_size", [8, 16, 32])
@pytest.mark.parametrize("g,D", [(1, 128), (4, 128), (1, 64), (16, 128)])
def test_consecutive_pages_one_box(layout, page_size, g, D):
    """Small pages that are consecutive in the pool are brought by one box per
    tile (a map over runs of pages): an in-order pool, and one where some
    tiles' pages are consecutive and others are not (two logical pages
    swapped, a run ending at the pool's last page), give bitwise the same
    out/lse as the contiguous path."""
    w = Workload("paged", B=3, Hq=2 * g, Hkv=2, D=D, Lmax=2000, ragged=False, sigma_k=3.0, nan_pad=True)
    x = make_inputs(w, 13, device="cuda", seqlens=[2000, 700, 1])
    S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax)
    out_c, lse_c = fd.decode(x.q, x.k, x.v, x.seqlens, x.scale, num_splits=S)
    pg = make_paged(x, page_size, layout, order="inorder", spare_pages=0)
    out_p, lse_p = fd.decode_paged(x.q, pg.k_pages, pg.v_pages, pg.block_table, x.seqlens, x.scale, layout=layout,
                                   num_splits=S)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c), f"in-order pool, page {page_size} {layout}"
    # swap two logical pages of sequence 0 (their tiles are no longer runs), keep the rest in order
    a, b = 3, 17
    bt = pg.block_table
    pa, pb = int(bt[0, a]), int(bt[0, b])
    for pool in (pg.k_pages, pg.v_pages):
        tmp = pool[pa].clone()
        pool[pa] = pool[pb]
        pool[pb] = tmp
    bt[0, a], bt[0, b] = pb, pa
    out_m, lse_m = fd.decode_paged(x.q, pg.k_pages, pg.v_pages, bt, x.seqlens, x.scale, layout=layout, num_splits=S)
    torch.cuda.synchronize()
    assert torch.equal(out_m, out_c) and torch.equal(lse_m, lse_c), f"mixed pool, page {page_size} {layout}"


@pytest.mark.parametrize("kv_type", ["e4m3", "int8"])
@pytest.mark.parametrize("layout", ["HND", "NHD"])
def test_consecutive_pages_one_box_8bit(kv_type, layout):
    """The same for 8-bit page pools (16-token pages): an in-order pool gives
    bitwise the contiguous 8-bit result."""
    from decode_attention_07_b200.inputs import make_quant
    w = Workload("paged", B=2, Hq=8, Hkv=2, D=128, Lmax=1500, ragged=False, nan_pad=True)
    x = make_quant(w, kv_type, 21, device="cuda", seqlens=[1500, 333])
    S = fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax)
    out_c, lse_c = fd.decode_quant(x.q, x.k8, x.v8, x.k_scale, x.v_scale, kv_type, x.seqlens, x.scale, num_splits=S)
    pg = make_paged(x, 16, layout, order="inorder")
    out_p, lse_p = fd.decode_quant_paged(x.q, pg.k_pages, pg.v_pages, x.k_scale, x.v_scale, kv_type, pg.block_table,
                                         x.seqlens, x.scale, layout=layout, num_splits=S)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)
