"""Seeded synthetic inputs for decode attention, shared by the CUDA path's
tests and benchmark and by the CPU oracle's tests.

This module holds no arithmetic of the attention method: it only draws
normal variates, scales them by the workload's standard deviation, rounds
them to bf16 (round-to-nearest-even, torch's conversion) and marks padding.

Recipe (for workload w and seed s):
  1. seqlens: all equal to w.Lmax, or, for a ragged workload, drawn with
     ``torch.randint(1, w.Lmax + 1, (w.B,))`` from a CPU generator seeded s.
  2. q, K, V: fp32 ``randn`` from a generator on ``device`` seeded s, in the
     order q, then K one sequence at a time (b = 0..B-1), then V the same
     way; each is multiplied by its sigma and rounded to bf16. Drawing one
     sequence at a time bounds the fp32 temporary to one sequence's cache.
  3. Padding: with w.nan_pad, K and V positions t >= seqlens[b] are set to
     NaN, so any read of them would poison the output.
The same seed gives the same bytes on the same device type; a CPU draw and a
CUDA draw of one seed differ (different generators), so each comparison
draws once and hands the same bytes to both sides.

Quantised caches (make_quant): seqlens and q as above; then per kv head h a
spread factor f_h = 2^u, u ~ U(-1, 1), from a CPU generator seeded s + 1;
scales k_scale[h] = 4 sigma_k f_h / R and v_scale[h] = 4 sigma_v f_h / R with
R = 448 (E4M3) or 127 (int8), so +-4 standard deviations span the code range;
K then V, one sequence at a time, fp32 randn * sigma * f_h, divided by the
head's scale and turned into codes by torch's own conversion (E4M3: clamp to
+-448, then torch.float8_e4m3fn; int8: round half to even, clamp to +-127).
Padding positions hold the NaN code 0x7F (E4M3) or -128 (int8, which has no
NaN) when the workload pads.
"""
from dataclasses import dataclass

import numpy as np
import torch

from .configs import Workload


@dataclass
class DecodeInputs:
    workload: Workload
    seed: int
    q: torch.Tensor          # [B, Hq, D] bf16
    k: torch.Tensor          # [B, Hkv, Lmax, D] bf16
    v: torch.Tensor          # [B, Hkv, Lmax, D] bf16
    seqlens: torch.Tensor    # [B] int32, same device as q
    seqlens_host: np.ndarray  # [B] int32 copy on the host
    scale: float

    def kv_bytes(self) -> int:
        """Bytes of K and V that lie inside the sequences (t < seqlen)."""
        w = self.workload
        return int(self.seqlens_host.astype(np.int64).sum()) * w.Hkv * w.D * 2 * 2


def draw_seqlens(w: Workload, seed: int) -> np.ndarray:
    if not w.ragged:
        return np.full((w.B,), w.Lmax, dtype=np.int32)
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    return torch.randint(1, w.Lmax + 1, (w.B,), generator=g, dtype=torch.int32).numpy()


def make_inputs(w: Workload, seed: int = 0, device="cpu", seqlens=None) -> DecodeInputs:
    """Draw one workload's tensors. ``seqlens`` (host ints) overrides the
    drawn lengths, for edge cases."""
    device = torch.device(device)
    if seqlens is None:
        lens = draw_seqlens(w, seed)
    else:
        lens = np.asarray(seqlens, dtype=np.int32).reshape(w.B)
    g = torch.Generator(device=device).manual_seed(int(seed))
    q = (torch.randn((w.B, w.Hq, w.D), generator=g, device=device) * w.sigma_q).to(torch.bfloat16)
    k = torch.empty((w.B, w.Hkv, w.Lmax, w.D), dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    for dst, sigma in ((k, w.sigma_k), (v, w.sigma_v)):
        for b in range(w.B):
            dst[b] = (torch.randn((w.Hkv, w.Lmax, w.D), generator=g, device=device) * sigma).to(torch.bfloat16)
    if w.nan_pad:
        for b in range(w.B):
            L = int(lens[b])
            if L < w.Lmax:
                k[b, :, max(L, 0):, :] = float("nan")
                v[b, :, max(L, 0):, :] = float("nan")
    seqlens_t = torch.from_numpy(lens.copy()).to(device)
    return DecodeInputs(w, int(seed), q, k, v, seqlens_t, lens.copy(), w.scale)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The bf16 tensor's bit patterns as a host numpy uint16 array."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@dataclass
class PagedInputs:
    """The same logical cache as a DecodeInputs, stored in a pool of pages."""
    k_pages: torch.Tensor        # HND: [num_pages, Hkv, page_size, D]; NHD: [num_pages, page_size, Hkv, D]
    v_pages: torch.Tensor
    block_table: torch.Tensor    # [B, max_pages] int32, same device
    block_table_host: np.ndarray
    page_size: int
    layout: str


def make_paged(x: DecodeInputs, page_size: int, layout: str = "HND", seed: int = 0, spare_pages: int = 3,
               unused_entry: int = -1, order: str = "shuffled") -> PagedInputs:
    """Scatter x's cache into a pool of pages (data movement only).

    Sequence b needs ceil(seqlens[b] / page_size) pages; the pool holds those
    plus `spare_pages` more, in an order drawn from a CPU generator seeded
    `seed` (order "shuffled"), or in sequence order, sequence after sequence
    (order "inorder": consecutive logical pages are consecutive pool pages,
    as an allocator that hands out pages in order produces). Block-table
    entries past a sequence's pages are `unused_entry`;
    pool slots that no sequence position maps to are NaN (for an 8-bit cache,
    QuantInputs: its padding code, and the pools hold codes)."""
    w = x.workload
    quant = hasattr(x, "k8")
    src_k, src_v = (x.k8, x.v8) if quant else (x.k, x.v)
    fill = (0x7F if x.kv_type == "e4m3" else 0x80) if quant else float("nan")
    dev = src_k.device
    lens = np.clip(x.seqlens_host.astype(np.int64), 0, w.Lmax)
    need = [int(-(-int(L) // page_size)) for L in lens]
    max_pages = max(1, -(-w.Lmax // page_size))
    max_pages = (max_pages + 3) // 4 * 4
    total = sum(need) + spare_pages
    if order not in ("shuffled", "inorder"):
        raise ValueError("order must be 'shuffled' or 'inorder'")
    if order == "inorder":
        order = np.arange(total)
    else:
        g = torch.Generator(device="cpu").manual_seed(int(seed))
        order = torch.randperm(total, generator=g).numpy()
    table = np.full((w.B, max_pages), unused_entry, dtype=np.int32)
    shape = (total, w.Hkv, page_size, w.D) if layout == "HND" else (total, page_size, w.Hkv, w.D)
    k_pages = torch.full(shape, fill, dtype=src_k.dtype, device=dev)
    v_pages = torch.full(shape, fill, dtype=src_k.dtype, device=dev)
    nxt = 0
    for b in range(w.B):
        n = need[b]
        if n == 0:
            continue
        ids = order[nxt:nxt + n]
        nxt += n
        table[b, :n] = ids
        span = n * page_size
        for src, dst in ((src_k, k_pages), (src_v, v_pages)):
            part = src[b, :, :min(span, w.Lmax)]                           # [Hkv, tokens, D]
            if part.shape[1] < span:
                pad = torch.full((w.Hkv, span - part.shape[1], w.D), fill, dtype=part.dtype, device=dev)
                part = torch.cat([part, pad], dim=1)
            part = part.reshape(w.Hkv, n, page_size, w.D)
            part = part.permute(1, 0, 2, 3) if layout == "HND" else part.permute(1, 2, 0, 3)
            dst[torch.from_numpy(ids.astype(np.int64)).to(dev)] = part.contiguous()
    return PagedInputs(k_pages, v_pages, torch.from_numpy(table).to(dev), table, page_size, layout)

QUANT_RANGE = {"e4m3": 448.0, "int8": 127.0}


@dataclass
class QuantInputs:
    workload: Workload
    seed: int
    kv_type: str             # "e4m3" or "int8"
    q: torch.Tensor          # [B, Hq, D] bf16
    k8: torch.Tensor         # [B, Hkv, Lmax, D] uint8 codes
    v8: torch.Tensor
    k_scale: torch.Tensor    # [Hkv] float32, same device
    v_scale: torch.Tensor
    seqlens: torch.Tensor
    seqlens_host: np.ndarray
    scale: float

    def kv_bytes(self) -> int:
        """Bytes of K and V codes that lie inside the sequences."""
        w = self.workload
        return int(self.seqlens_host.astype(np.int64).sum()) * w.Hkv * w.D * 2


def _codes(x: torch.Tensor, kv_type: str) -> torch.Tensor:
    if kv_type == "e4m3":
        return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return torch.round(x).clamp(-127.0, 127.0).to(torch.int8).view(torch.uint8)


def make_quant(w: Workload, kv_type: str, seed: int = 0, device="cpu", seqlens=None) -> QuantInputs:
    """Draw a workload with an 8-bit key/value cache (recipe in the module
    docstring)."""
    if kv_type not in QUANT_RANGE:
        raise ValueError("kv_type must be 'e4m3' or 'int8'")
    device = torch.device(device)
    lens = draw_seqlens(w, seed) if seqlens is None else np.asarray(seqlens, dtype=np.int32).reshape(w.B)
    g = torch.Generator(device=device).manual_seed(int(seed))
    q = (torch.randn((w.B, w.Hq, w.D), generator=g, device=device) * w.sigma_q).to(torch.bfloat16)
    gh = torch.Generator(device="cpu").manual_seed(int(seed) + 1)
    f = torch.pow(2.0, torch.rand((w.Hkv,), generator=gh) * 2.0 - 1.0)
    R = QUANT_RANGE[kv_type]
    k_scale = (4.0 * w.sigma_k * f / R).to(torch.float32)
    v_scale = (4.0 * w.sigma_v * f / R).to(torch.float32)
    k8 = torch.empty((w.B, w.Hkv, w.Lmax, w.D), dtype=torch.uint8, device=device)
    v8 = torch.empty_like(k8)
    for dst, sigma, sc in ((k8, w.sigma_k, k_scale), (v8, w.sigma_v, v_scale)):
        spread = (f * sigma).to(device)[:, None, None]
        inv = (1.0 / sc).to(device)[:, None, None]
        for b in range(w.B):
            x = torch.randn((w.Hkv, w.Lmax, w.D), generator=g, device=device) * spread
            dst[b] = _codes(x * inv, kv_type)
    if w.nan_pad:
        pad = 0x7F if kv_type == "e4m3" else 0x80
        for b in range(w.B):
            L = int(lens[b])
            if L < w.Lmax:
                k8[b, :, max(L, 0):, :] = pad
                v8[b, :, max(L, 0):, :] = pad
    return QuantInputs(w, int(seed), kv_type, q, k8, v8, k_scale.to(device), v_scale.to(device),
                       torch.from_numpy(lens.copy()).to(device), lens.copy(), w.scale)
