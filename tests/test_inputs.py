"""The seeded input generator: determinism, the ragged-length recipe, NaN
padding and bf16 rounding (CPU only)."""
import numpy as np
import pytest
import torch

from decode_attention_07_b200.configs import WORKLOADS, ORDER
from decode_attention_07_b200.inputs import make_inputs, draw_seqlens, bf16_bits


def test_workload_table():
    assert ORDER == list(WORKLOADS)
    for w in WORKLOADS.values():
        assert w.Hq % w.Hkv == 0 and w.D in (64, 128)
    assert WORKLOADS["gqa_128k"].g == 8 and WORKLOADS["batch_4k"].g == 4


def test_same_seed_same_bytes():
    w = WORKLOADS["tiny_mha"].with_(Lmax=96)
    a, b = make_inputs(w, 3), make_inputs(w, 3)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v)):
        assert np.array_equal(bf16_bits(x), bf16_bits(y))
    c = make_inputs(w, 4)
    assert not np.array_equal(bf16_bits(a.k), bf16_bits(c.k))


def test_ragged_lengths_and_nan_padding():
    w = WORKLOADS["ragged_64k"].with_(B=5, Hq=4, Hkv=2, Lmax=300)
    x = make_inputs(w, 0)
    lens = x.seqlens_host
    assert lens.dtype == np.int32 and lens.min() >= 1 and lens.max() <= w.Lmax
    assert np.array_equal(lens, draw_seqlens(w, 0))
    for bb in range(w.B):
        L = int(lens[bb])
        assert torch.isnan(x.k[bb, :, L:].float()).all() and torch.isnan(x.v[bb, :, L:].float()).all()
        assert torch.isfinite(x.k[bb, :, :L].float()).all() and torch.isfinite(x.v[bb, :, :L].float()).all()
    # the headline ragged draw for seed 0
    full = WORKLOADS["ragged_64k"]
    assert draw_seqlens(full, 0).shape == (32,)


def test_sigma_and_rounding():
    w = WORKLOADS["ragged_64k"].with_(B=2, Hq=2, Hkv=2, Lmax=4096, nan_pad=False, ragged=False)
    x = make_inputs(w, 1)
    ks, vs = x.k.float().std().item(), x.v.float().std().item()
    assert 3.8 < ks < 4.2 and 0.95 < vs < 1.05
    # bf16 values are exactly what torch's round-to-nearest-even gives
    g = torch.Generator().manual_seed(1)
    q32 = torch.randn((w.B, w.Hq, w.D), generator=g)
    assert torch.equal(q32.to(torch.bfloat16), x.q)


# ------------------------------------------------------ quantised caches --

from decode_attention_07_b200.inputs import QUANT_RANGE, make_quant  # noqa: E402


@pytest.mark.parametrize("kv_type", ["e4m3", "int8"])
def test_quant_inputs_recipe(kv_type):
    w = WORKLOADS["ragged_64k"].with_(B=3, Lmax=200)
    a = make_quant(w, kv_type, seed=5)
    b = make_quant(w, kv_type, seed=5)
    assert torch.equal(a.k8, b.k8) and torch.equal(a.v8, b.v8) and torch.equal(a.q, b.q)
    assert a.k8.dtype == torch.uint8 and a.k8.shape == (w.B, w.Hkv, w.Lmax, w.D)
    assert a.k_scale.shape == (w.Hkv,) and a.k_scale.dtype == torch.float32
    # per-head spread f_h in [1/2, 2]: k_scale / (4 sigma_k / R) is that factor, the same for v
    f_k = a.k_scale.double() / (4 * w.sigma_k / QUANT_RANGE[kv_type])
    f_v = a.v_scale.double() / (4 * w.sigma_v / QUANT_RANGE[kv_type])
    assert torch.allclose(f_k, f_v, rtol=1e-6) and bool((f_k >= 0.5).all() and (f_k <= 2.0).all())
    pad = 0x7F if kv_type == "e4m3" else 0x80
    for bb in range(w.B):
        L = int(a.seqlens_host[bb])
        assert bool((a.k8[bb, :, L:] == pad).all() and (a.v8[bb, :, L:] == pad).all())
        # inside the sequence: dequantised values have the head's sigma * f_h spread
        vals = (a.k8[bb, :, :L].view(torch.float8_e4m3fn).float() if kv_type == "e4m3"
                else a.k8[bb, :, :L].view(torch.int8).float())
        if L >= 100:
            sd = (vals * a.k_scale[:, None, None]).std(dim=(1, 2)) / (w.sigma_k * f_k.float())
            assert bool(((sd > 0.8) & (sd < 1.2)).all())
    assert make_quant(w, kv_type, seed=6).k8.ne(a.k8).any()
