"""8-bit key/value caches (fd_decode_quant) on the GPU against the CPU
oracle's dequantised definition: k = k_scale[h] * decode(code), likewise v,
then plain attention. The oracle reads the same codes and scales, so the
tolerance is the bf16 path's; the quantisation error belongs to the input."""
import numpy as np
import pytest
import torch

import decode_attention_07_b200 as fd
import oracle
from decode_attention_07_b200.configs import WORKLOADS, Workload
from decode_attention_07_b200.inputs import bf16_bits, make_quant
from test_gpu_parity import compare

pytestmark = pytest.mark.gpu
KV = ["e4m3", "int8"]


@pytest.fixture(scope="module", autouse=True)
def gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    assert fd.fd_device_status() == 0


def oracle_quant(x, q=None, bs=None):
    """Oracle rows for sequences `bs`, reading only each sequence's prefix."""
    w = x.workload
    q = x.q if q is None else q
    bs = range(w.B) if bs is None else bs
    outs, lses = [], []
    for b in bs:
        L = int(min(max(x.seqlens_host[b], 0), w.Lmax))
        o, l = oracle.attention_quant(bf16_bits(q[b:b + 1]), x.k8[b:b + 1, :, :L].cpu().numpy(),
                                      x.v8[b:b + 1, :, :L].cpu().numpy(), x.k_scale.cpu().numpy(),
                                      x.v_scale.cpu().numpy(), np.array([L], np.int32), x.scale, x.kv_type)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


def run(x, q=None, S=None):
    q = x.q if q is None else q
    out, lse = fd.decode_quant(q, x.k8, x.v8, x.k_scale, x.v_scale, x.kv_type, x.seqlens, x.scale, num_splits=S)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("kv_type", KV)
@pytest.mark.parametrize("g,D", [(1, 128), (4, 128), (8, 128), (16, 128), (1, 64), (3, 64), (16, 64)])
def test_quant_against_oracle(kv_type, g, D):
    w = Workload("q8", B=4, Hq=2 * g, Hkv=2, D=D, Lmax=2100, ragged=False, sigma_k=2.0, nan_pad=True)
    x = make_quant(w, kv_type, seed=3, device="cuda", seqlens=[2100, 1, 777, 64])
    ref_o, ref_l = oracle_quant(x)
    for S in (1, fd.fd_plan(w.B, w.Hq, w.Hkv, w.D, w.Lmax), 61):
        out, lse = run(x, S=S)
        compare(out, lse, ref_o, ref_l, f"{kv_type} g={g} D={D} S={S}")


@pytest.mark.parametrize("kv_type", KV)
@pytest.mark.parametrize("q_len,g", [(2, 4), (4, 2), (16, 1), (2, 8)])
def test_quant_multi_query(kv_type, q_len, g):
    w = Workload("q8", B=3, Hq=2 * g, Hkv=2, D=128, Lmax=1500, ragged=False, nan_pad=True)
    x = make_quant(w, kv_type, seed=4, device="cuda", seqlens=[1500, q_len - 1, 300])
    gen = torch.Generator(device="cuda").manual_seed(9)
    q = torch.randn((w.B, q_len, w.Hq, w.D), generator=gen, device="cuda").to(torch.bfloat16)
    ref_o, ref_l = oracle_quant(x, q)
    for S in (1, 37):
        out, lse = run(x, q, S)
        compare(out, lse, ref_o, ref_l, f"{kv_type} q_len={q_len} g={g} S={S}")


@pytest.mark.parametrize("kv_type", KV)
def test_query_magnitudes(kv_type):
    """The per-column power-of-two prescale of q: very large, very small,
    mixed and all-zero query heads in one batch."""
    w = Workload("q8", B=2, Hq=8, Hkv=2, D=128, Lmax=700, ragged=False, nan_pad=True)
    x = make_quant(w, kv_type, seed=5, device="cuda", seqlens=[700, 333])
    q = x.q.float().clone()
    q[:, 0] *= 3e4          # near the top of f16's range before the prescale
    q[:, 1] *= 1e-9         # far below f16's normal range
    q[:, 2] = 0.0
    q[:, 3, ::2] *= 1e-6    # one column with elements of very different sizes
    q = q.to(torch.bfloat16)
    ref_o, ref_l = oracle_quant(x, q)
    out, lse = run(x, q, 5)
    compare(out, lse, ref_o, ref_l, f"{kv_type} query magnitudes")


@pytest.mark.parametrize("kv_type", KV)
def test_split_invariance_and_determinism(kv_type):
    w = Workload("q8", B=2, Hq=8, Hkv=2, D=128, Lmax=5000, ragged=False, nan_pad=True)
    x = make_quant(w, kv_type, seed=6, device="cuda", seqlens=[5000, 2222])
    ref_o, ref_l = oracle_quant(x)
    for S in (1, 2, 7, 148, 400):
        out, lse = run(x, S=S)
        compare(out, lse, ref_o, ref_l, f"{kv_type} S={S}")
        again = run(x, S=S)
        assert torch.equal(out, again[0]) and torch.equal(lse, again[1]), "not deterministic"


@pytest.mark.parametrize("kv_type", KV)
def test_empty_and_clamped(kv_type):
    w = Workload("q8", B=4, Hq=4, Hkv=4, D=64, Lmax=200, ragged=False, nan_pad=True)
    x = make_quant(w, kv_type, seed=7, device="cuda", seqlens=[0, 200, 5, 1])
    x.seqlens = torch.tensor([0, 900, 5, -3], dtype=torch.int32, device="cuda")   # clamped to [0, Lmax]
    x.seqlens_host = np.array([0, 200, 5, 0], np.int32)
    ref_o, ref_l = oracle_quant(x)
    for S in (1, 3, 50):
        out, lse = run(x, S=S)
        compare(out, lse, ref_o, ref_l, f"{kv_type} empty/clamped S={S}")


@pytest.mark.parametrize("name,kv_type", [("mha_16k", "e4m3"), ("mha_16k", "int8"), ("gqa_128k", "e4m3"),
                                          ("ragged_64k", "int8"), ("batch_4k", "e4m3")])
def test_full_size(name, kv_type):
    """Full-size workloads in the planned launch; the oracle checks a sample
    of sequences (all of them when B <= 4)."""
    w = WORKLOADS[name]
    x = make_quant(w, kv_type, seed=0, device="cuda")
    out, lse = run(x)
    bs = list(range(w.B)) if w.B <= 4 else [0, w.B // 2, w.B - 1]
    ref_o, ref_l = oracle_quant(x, bs=bs)
    compare(out[bs], lse[bs], ref_o, ref_l, f"{name} {kv_type}")


def codes_with_profile(x, prof_k):
    """Replace x's key codes by fresh ones whose magnitude follows prof_k[t]
    along the sequence (scales re-derived so the largest value uses the code
    range); value codes are kept."""
    from decode_attention_07_b200.inputs import QUANT_RANGE, _codes
    w = x.workload
    g = torch.Generator(device="cuda").manual_seed(11)
    k = torch.randn((w.B, w.Hkv, w.Lmax, w.D), generator=g, device="cuda") * prof_k[None, None, :, None]
    ks = (k.abs().amax(dim=(0, 2, 3)) / QUANT_RANGE[x.kv_type]).float()
    x.k8 = _codes(k / ks[None, :, None, None], x.kv_type).contiguous()
    x.k_scale = ks.contiguous()
    return x


@pytest.mark.parametrize("kv_type", KV)
@pytest.mark.parametrize("profile", ["rising", "falling"])
def test_lazy_max_fallback(kv_type, profile):
    """Rising logits exceed the reference maximum again and again (the
    rescale fallback runs on many tiles); falling logits put the maximum in
    the first tile (no fallback after it). Both against the oracle."""
    w = Workload("q8", B=2, Hq=8, Hkv=2, D=128, Lmax=4096, ragged=False, nan_pad=False, sigma_q=1.0)
    x = make_quant(w, kv_type, seed=8, device="cuda")
    t = torch.arange(w.Lmax, device="cuda", dtype=torch.float32) / w.Lmax
    prof = 0.2 + 6.0 * t if profile == "rising" else 6.2 - 6.0 * t
    x = codes_with_profile(x, prof)
    ref_o, ref_l = oracle_quant(x)
    for S in (1, 9, 148):
        out, lse = run(x, S=S)
        compare(out, lse, ref_o, ref_l, f"{kv_type} {profile} S={S}")


# ------------------------------------------------------- paged 8-bit pools --

from decode_attention_07_b200.inputs import make_paged  # noqa: E402


@pytest.mark.parametrize("kv_type", KV)
@pytest.mark.parametrize("page,layout,g,D", [(16, "HND", 4, 128), (8, "NHD", 1, 128), (64, "HND", 8, 128),
                                             (256, "NHD", 16, 128), (16, "HND", 4, 64), (32, "NHD", 1, 64)])
def test_paged_quant_equals_contiguous_and_oracle(kv_type, page, layout, g, D):
    w = Workload("q8p", B=3, Hq=2 * g, Hkv=2, D=D, Lmax=1100, ragged=False, nan_pad=True)
    x = make_quant(w, kv_type, seed=12, device="cuda", seqlens=[1100, 17, 530])
    pg = make_paged(x, page, layout, seed=13, unused_entry=10 ** 6)
    ref_o, ref_l = oracle_quant(x)
    for S in (1, 23):
        out, lse = fd.decode_quant_paged(x.q, pg.k_pages, pg.v_pages, x.k_scale, x.v_scale, kv_type, pg.block_table,
                                         x.seqlens, x.scale, layout, num_splits=S)
        o2, l2 = run(x, S=S)
        torch.cuda.synchronize()
        assert torch.equal(out, o2) and torch.equal(lse, l2), f"{kv_type} page {page} {layout} S={S}"
        compare(out, lse, ref_o, ref_l, f"{kv_type} paged {page} {layout} g={g} D={D} S={S}")


@pytest.mark.parametrize("kv_type", KV)
def test_paged_quant_several_queries(kv_type):
    w = Workload("q8p", B=2, Hq=8, Hkv=2, D=128, Lmax=900, ragged=False, nan_pad=True)
    x = make_quant(w, kv_type, seed=14, device="cuda", seqlens=[900, 3])
    g = torch.Generator(device="cuda").manual_seed(15)
    q = torch.randn((w.B, 3, w.Hq, w.D), generator=g, device="cuda").to(torch.bfloat16)
    pg = make_paged(x, 16, "HND", seed=16)
    ref_o, ref_l = oracle_quant(x, q)
    out, lse = fd.decode_quant_paged(q, pg.k_pages, pg.v_pages, x.k_scale, x.v_scale, kv_type, pg.block_table,
                                     x.seqlens, x.scale, "HND", num_splits=11)
    torch.cuda.synchronize()
    compare(out, lse, ref_o, ref_l, f"{kv_type} paged, 3 queries")


def test_paged_quant_full_size():
    """ragged_64k with an E4M3 cache in 16-token pages, planned launch."""
    w = WORKLOADS["ragged_64k"]
    x = make_quant(w, "e4m3", seed=0, device="cuda")
    pg = make_paged(x, 16, "HND", seed=1)
    out, lse = fd.decode_quant_paged(x.q, pg.k_pages, pg.v_pages, x.k_scale, x.v_scale, "e4m3", pg.block_table,
                                     x.seqlens, x.scale, "HND")
    torch.cuda.synchronize()
    bs = [0, w.B // 2, w.B - 1]
    ref_o, ref_l = oracle_quant(x, bs=bs)
    compare(out[bs], lse[bs], ref_o, ref_l, "ragged_64k e4m3 in 16-token pages")
