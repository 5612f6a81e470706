"""ctypes binding over libfdecode.so: the C ABI of include/fd.h with the same
names, taking torch tensors. Argument marshalling only -- every step of the
computation runs in the library's CUDA kernels. There is no fallback: if the
library is missing or a call fails, an exception is raised."""
import ctypes
import os
import warnings

import numpy as np
import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(PKG, "libfdecode.so")
DEBUG_LIBRARY = os.path.join(PKG, "libfdecode_debug.so")   # built with -DFD_DEBUG (device-side bounds checks)

FD_OK = 0
FD_TILE_TOKENS = 64
FD_MAX_SPLITS = 65535
FD_MAX_GROUP = 16
ERRORS = {
    -1: "FD_ERR_NULL_POINTER", -2: "FD_ERR_SHAPE", -3: "FD_ERR_GROUP", -4: "FD_ERR_HEAD_DIM",
    -5: "FD_ERR_ALIGNMENT", -6: "FD_ERR_WORKSPACE", -7: "FD_ERR_SPLITS", -8: "FD_ERR_DEVICE",
    -9: "FD_ERR_LAUNCH", -10: "FD_ERR_TIMEOUT", -11: "FD_ERR_CAPACITY", -12: "FD_ERR_STATIC_LIMIT", -13: "FD_ERR_BOUNDS",
}
FD_STATIC_SCRATCH_BYTES = 8 << 20
FD_KV_HND, FD_KV_NHD = 0, 1
LAYOUTS = {"HND": FD_KV_HND, "NHD": FD_KV_NHD}


class FdError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({fd_strerror(code)})")


_lib = None
_i, _p, _sz, _f = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float


def _newer_sources(path: str) -> list:
    """Sources of the library (decode_attention_07_b200.build.DEPS) modified
    after the library at `path` was built; those not shipped are skipped."""
    from .build import DEPS
    t = os.path.getmtime(path)
    return sorted(os.path.basename(d) for d in DEPS if os.path.exists(d) and os.path.getmtime(d) > t)


def lib() -> ctypes.CDLL:
    """Load libfdecode.so (built in-tree by decode_attention_07_b200.build);
    with FD_DEBUG=1 in the environment, the debug build libfdecode_debug.so."""
    global _lib
    if _lib is None:
        path = DEBUG_LIBRARY if os.environ.get("FD_DEBUG", "0") not in ("", "0") else LIBRARY
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is not built: run `python -c 'import __graft_entry__ as g; g.build()'`")
        stale = _newer_sources(path)
        if stale:
            warnings.warn(f"{os.path.basename(path)} is older than {', '.join(stale)}: the loaded kernels may not be "
                          "the sources' (rebuild with `python -c 'import __graft_entry__ as g; g.build()'`)",
                          RuntimeWarning, stacklevel=2)
        L = ctypes.CDLL(path)
        L.fd_plan.argtypes = [_i] * 5
        L.fd_plan_for_sms.argtypes = [_i] * 6
        L.fd_workspace_bytes.argtypes = [_i] * 6
        L.fd_workspace_bytes.restype = _sz
        compute = [_i] * 5 + [_p, _p, _p, _p, _f, _p, _p, _p, _sz]
        L.fd_decode.argtypes = compute + [_p]
        L.fd_decode_splits.argtypes = compute + [_i, _p]
        L.fd_split.argtypes = compute + [_i, _p]
        L.fd_combine.argtypes = [_i] * 5 + [_p, _p, _p, _p, _sz, _i, _p]
        L.fd_segments.argtypes = [_i, _i, _i, _p, _i, _p, _p, _p, _p, _i]
        L.fd_device_status.argtypes = [_p]
        L.fd_workspace_init.argtypes = [_p, _sz, _p]
        L.fd_decode_static.argtypes = [_i] * 5 + [_p, _p, _p, _p, _f, _p, _p, _p]
        L.fd_decode_paged.argtypes = [_i] * 8 + [_p, _p, _p, _p, _p, _f, _p, _p, _p, _sz, _i, _p]
        L.fd_decode_multi.argtypes = [_i] * 6 + [_p, _p, _p, _p, _f, _p, _p, _p, _sz, _i, _p]
        L.fd_decode_quant.argtypes = [_i] * 7 + [_p, _p, _p, _p, _p, _p, _f, _p, _p, _p, _sz, _i, _p]
        L.fd_merge_partials.argtypes = [_i, _i, _i, _p, _p, _p, _p, _p]
        L.fd_read_probe.argtypes = [_p, _sz, _p, _p]
        L.fd_decode_quant_paged.argtypes = [_i] * 10 + [_p] * 7 + [_f, _p, _p, _p, _sz, _i, _p]
        L.fd_strerror.argtypes = [_i]
        L.fd_strerror.restype = ctypes.c_char_p
        L.fd_version.argtypes = []
        for name in ("fd_plan", "fd_plan_for_sms", "fd_decode", "fd_decode_splits", "fd_split", "fd_combine",
                     "fd_segments", "fd_device_status", "fd_version", "fd_workspace_init", "fd_decode_static",
                     "fd_decode_paged", "fd_decode_multi", "fd_decode_quant", "fd_merge_partials", "fd_read_probe", "fd_decode_quant_paged"):
            getattr(L, name).restype = _i
        _lib = L
    return _lib


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise FdError(rc, what)
    return rc


def _stream(stream, device) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _shapes(q, k_cache, v_cache):
    if q.dim() != 3 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("expected q [B,Hq,D] and k_cache, v_cache [B,Hkv,Lmax,D]")
    B, Hq, D = q.shape
    B2, Hkv, Lmax, D2 = k_cache.shape
    if B2 != B or D2 != D:
        raise ValueError("q and the caches disagree on B or D")
    for t, name in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    return B, Hq, Hkv, D, Lmax


def _outputs(out, lse, B, Hq, D):
    if out.shape != (B, Hq, D) or lse.shape != (B, Hq):
        raise ValueError("out must be [B,Hq,D] and lse [B,Hq]")
    for t, name in ((out, "out"), (lse, "lse")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")


def _seqlens(seqlens, B):
    if seqlens.shape != (B,) or seqlens.dtype != torch.int32 or not seqlens.is_cuda:
        raise ValueError("seqlens must be an int32 CUDA tensor of shape [B]")


def _ws(workspace):
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


# ---------------------------------------------------------------- the ABI --

def fd_plan(B: int, Hq: int, Hkv: int, D: int, max_len: int) -> int:
    return _check(lib().fd_plan(B, Hq, Hkv, D, max_len), "fd_plan")


def fd_plan_for_sms(B: int, Hq: int, Hkv: int, D: int, max_len: int, num_sms: int) -> int:
    return _check(lib().fd_plan_for_sms(B, Hq, Hkv, D, max_len, num_sms), "fd_plan_for_sms")


def fd_workspace_bytes(B: int, Hq: int, Hkv: int, D: int, max_len: int, num_splits: int) -> int:
    return int(lib().fd_workspace_bytes(B, Hq, Hkv, D, max_len, num_splits))


def fd_decode(q, k_cache, v_cache, seqlens, scale, out, lse, workspace=None, stream=None):
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache)
    _outputs(out, lse, B, Hq, D)
    _seqlens(seqlens, B)
    wp, wb = _ws(workspace)
    _check(lib().fd_decode(B, Hq, Hkv, D, Lmax, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                           seqlens.data_ptr(), float(scale), out.data_ptr(), lse.data_ptr(), wp, wb,
                           _stream(stream, q.device)), "fd_decode")


def fd_decode_splits(q, k_cache, v_cache, seqlens, scale, out, lse, workspace, num_splits, stream=None):
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache)
    _outputs(out, lse, B, Hq, D)
    _seqlens(seqlens, B)
    wp, wb = _ws(workspace)
    _check(lib().fd_decode_splits(B, Hq, Hkv, D, Lmax, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                  seqlens.data_ptr(), float(scale), out.data_ptr(), lse.data_ptr(), wp, wb,
                                  int(num_splits), _stream(stream, q.device)), "fd_decode_splits")


def fd_split(q, k_cache, v_cache, seqlens, scale, out, lse, workspace, num_splits, stream=None):
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache)
    _outputs(out, lse, B, Hq, D)
    _seqlens(seqlens, B)
    wp, wb = _ws(workspace)
    _check(lib().fd_split(B, Hq, Hkv, D, Lmax, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                          seqlens.data_ptr(), float(scale), out.data_ptr(), lse.data_ptr(), wp, wb,
                          int(num_splits), _stream(stream, q.device)), "fd_split")


def fd_combine(B, Hq, Hkv, D, max_len, seqlens, out, lse, workspace, num_splits, stream=None):
    _outputs(out, lse, B, Hq, D)
    _seqlens(seqlens, B)
    wp, wb = _ws(workspace)
    _check(lib().fd_combine(B, Hq, Hkv, D, max_len, seqlens.data_ptr(), out.data_ptr(), lse.data_ptr(), wp, wb,
                            int(num_splits), _stream(stream, out.device)), "fd_combine")


def fd_segments(B: int, Hkv: int, max_len: int, seqlens_host, num_splits: int) -> dict:
    """Where the split stage cuts each row (host computation). Returns numpy
    arrays indexed by workspace slot: row (-1 = unused), begin, end, whole."""
    lens = np.ascontiguousarray(np.asarray(seqlens_host, dtype=np.int32).reshape(B))
    cap = num_splits + B * Hkv - 1
    arrs = [np.zeros(cap, np.int32) for _ in range(4)]
    n = _check(lib().fd_segments(B, Hkv, max_len, lens.ctypes.data, int(num_splits),
                                 *(a.ctypes.data for a in arrs), cap), "fd_segments")
    return dict(row=arrs[0][:n], begin=arrs[1][:n], end=arrs[2][:n], whole=arrs[3][:n])


def fd_decode_static(q, k_cache, v_cache, seqlens, scale, out, lse, stream=None):
    """fd_decode without a workspace argument: the library's fixed device
    scratch buffer is used instead (see include/fd.h)."""
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache)
    _outputs(out, lse, B, Hq, D)
    _seqlens(seqlens, B)
    _check(lib().fd_decode_static(B, Hq, Hkv, D, Lmax, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                  seqlens.data_ptr(), float(scale), out.data_ptr(), lse.data_ptr(),
                                  _stream(stream, q.device)), "fd_decode_static")


def fd_decode_multi(q, k_cache, v_cache, seqlens, scale, out, lse, workspace=None, num_splits=0, stream=None):
    """Several queries per sequence: q [B, q_len, Hq, D], out [B, q_len, Hq, D],
    lse [B, q_len, Hq]; query j sees the first seqlens[b] - (q_len-1-j) tokens.
    num_splits 0 lets the library plan the split count."""
    prepare_decode_multi(q, k_cache, v_cache, seqlens, scale, out, lse, workspace, num_splits, stream)()


def decode_multi(q, k_cache, v_cache, seqlens, scale, num_splits=None, stream=None):
    """Allocate out / lse / workspace with torch and run fd_decode_multi."""
    B, q_len, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    S = fd_plan(B, Hq, Hkv, D, Lmax) if num_splits is None else int(num_splits)
    nbytes = fd_workspace_bytes(B, Hq * q_len, Hkv, D, Lmax, S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    out = torch.empty((B, q_len, Hq, D), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, q_len, Hq), dtype=torch.float32, device=q.device)
    fd_decode_multi(q, k_cache, v_cache, seqlens, scale, out, lse, ws, S, stream)
    return out, lse


def _paged_shapes(q, k_pages, v_pages, block_table, layout, pool_dtype=torch.bfloat16):
    if layout not in LAYOUTS:
        raise ValueError("layout must be 'HND' ([pages, Hkv, page_size, D]) or 'NHD' ([pages, page_size, Hkv, D])")
    if q.dim() not in (3, 4) or k_pages.dim() != 4 or v_pages.shape != k_pages.shape or block_table.dim() != 2:
        raise ValueError("expected q [B,Hq,D] (or [B,q_len,Hq,D]), k_pages/v_pages 4-D, block_table [B, max_pages]")
    B, Hq, D = q.shape[0], q.shape[-2], q.shape[-1]
    if layout == "HND":
        num_pages, Hkv, page_size, D2 = k_pages.shape
    else:
        num_pages, page_size, Hkv, D2 = k_pages.shape
    if D2 != D or block_table.shape[0] != B:
        raise ValueError("q, pages and block_table disagree on B or D")
    if q.dtype != torch.bfloat16 or not q.is_cuda or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    for t, name in ((k_pages, "k_pages"), (v_pages, "v_pages")):
        if t.dtype != pool_dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {pool_dtype} CUDA tensor")
    if block_table.dtype != torch.int32 or not block_table.is_cuda or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 CUDA tensor")
    return B, Hq, Hkv, D, page_size, num_pages, block_table.shape[1]


def fd_decode_paged(q, k_pages, v_pages, block_table, seqlens, scale, out, lse, workspace=None, layout="HND",
                    num_splits=0, stream=None):
    B, Hq, Hkv, D, page_size, num_pages, max_pages = _paged_shapes(q, k_pages, v_pages, block_table, layout)
    _outputs(out, lse, B, Hq, D)
    _seqlens(seqlens, B)
    wp, wb = _ws(workspace)
    _check(lib().fd_decode_paged(B, Hq, Hkv, D, page_size, num_pages, max_pages, LAYOUTS[layout], q.data_ptr(),
                                 k_pages.data_ptr(), v_pages.data_ptr(), block_table.data_ptr(), seqlens.data_ptr(),
                                 float(scale), out.data_ptr(), lse.data_ptr(), wp, wb, int(num_splits),
                                 _stream(stream, q.device)), "fd_decode_paged")


def prepare_decode_paged(q, k_pages, v_pages, block_table, seqlens, scale, out, lse, workspace=None, layout="HND",
                         num_splits=0, stream=None):
    """Check and marshal once; return a no-argument callable that enqueues
    fd_decode_paged with those pointers."""
    B, Hq, Hkv, D, page_size, num_pages, max_pages = _paged_shapes(q, k_pages, v_pages, block_table, layout)
    _outputs(out, lse, B, Hq, D)
    _seqlens(seqlens, B)
    wp, wb = _ws(workspace)
    fn = lib().fd_decode_paged
    args = (B, Hq, Hkv, D, page_size, num_pages, max_pages, LAYOUTS[layout], q.data_ptr(), k_pages.data_ptr(),
            v_pages.data_ptr(), block_table.data_ptr(), seqlens.data_ptr(), ctypes.c_float(scale), out.data_ptr(),
            lse.data_ptr(), wp, wb, int(num_splits), _stream(stream, q.device))

    def call():
        rc = fn(*args)
        if rc != 0:
            raise FdError(rc, "fd_decode_paged")

    return call


def prepare_decode_quant_paged(q, k_pages, v_pages, k_scale, v_scale, kv_type, block_table, seqlens, scale, out, lse,
                               workspace=None, layout="HND", num_splits=0, stream=None):
    """prepare_decode for fd_decode_quant_paged: 8-bit page pools (uint8,
    layouts as fd_decode_paged), per-kv-head float32 scales, kv_type "e4m3"
    or "int8"; q [B, Hq, D] or [B, q_len, Hq, D], out / lse shaped to match."""
    if kv_type not in KV_CODES:
        raise ValueError("kv_type must be 'e4m3' or 'int8'")
    B, Hq, Hkv, D, page_size, num_pages, max_pages = _paged_shapes(q, k_pages, v_pages, block_table, layout,
                                                                   torch.uint8)
    q_len = 1 if q.dim() == 3 else q.shape[1]
    for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        if t.shape != (Hkv,) or t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor of shape [Hkv]")
    if out.shape != q.shape or lse.shape != q.shape[:-1]:
        raise ValueError("out must be shaped like q and lse like q without D")
    for t, name in ((out, "out"), (lse, "lse")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")
    _seqlens(seqlens, B)
    wp, wb = _ws(workspace)
    fn = lib().fd_decode_quant_paged
    args = (B, q_len, Hq, Hkv, D, page_size, num_pages, max_pages, LAYOUTS[layout], KV_CODES[kv_type], q.data_ptr(),
            k_pages.data_ptr(), v_pages.data_ptr(), k_scale.data_ptr(), v_scale.data_ptr(), block_table.data_ptr(),
            seqlens.data_ptr(), ctypes.c_float(scale), out.data_ptr(), lse.data_ptr(), wp, wb, int(num_splits),
            _stream(stream, q.device))

    def call():
        rc = fn(*args)
        if rc != 0:
            raise FdError(rc, "fd_decode_quant_paged")

    return call


def decode_quant_paged(q, k_pages, v_pages, k_scale, v_scale, kv_type, block_table, seqlens, scale, layout="HND",
                       num_splits=None, stream=None):
    """Allocate out / lse / workspace with torch and run fd_decode_quant_paged."""
    B, Hq, Hkv, D, page_size, num_pages, max_pages = _paged_shapes(q, k_pages, v_pages, block_table, layout,
                                                                   torch.uint8)
    q_len = 1 if q.dim() == 3 else q.shape[1]
    Lmax = max_pages * page_size
    S = fd_plan(B, Hq, Hkv, D, Lmax) if num_splits is None else int(num_splits)
    nbytes = fd_workspace_bytes(B, Hq * q_len, Hkv, D, Lmax, S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    prepare_decode_quant_paged(q, k_pages, v_pages, k_scale, v_scale, kv_type, block_table, seqlens, scale, out, lse,
                               ws, layout, S, stream)()
    return out, lse


def decode_paged(q, k_pages, v_pages, block_table, seqlens, scale, layout="HND", num_splits=None, stream=None):
    """Allocate out / lse / workspace with torch and run fd_decode_paged."""
    B, Hq, Hkv, D, page_size, num_pages, max_pages = _paged_shapes(q, k_pages, v_pages, block_table, layout)
    Lmax = max_pages * page_size
    S = fd_plan(B, Hq, Hkv, D, Lmax) if num_splits is None else int(num_splits)
    nbytes = fd_workspace_bytes(B, Hq, Hkv, D, Lmax, S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    fd_decode_paged(q, k_pages, v_pages, block_table, seqlens, scale, out, lse, ws, layout, S, stream)
    return out, lse


def fd_workspace_init(workspace, stream=None):
    wp, wb = _ws(workspace)
    if wb:
        _check(lib().fd_workspace_init(wp, wb, _stream(stream, workspace.device)), "fd_workspace_init")


def fd_device_status(stream=None, device=None) -> int:
    return lib().fd_device_status(_stream(stream, device))


def fd_strerror(code: int) -> str:
    return lib().fd_strerror(int(code)).decode()


def fd_version() -> int:
    return lib().fd_version()


# ------------------------------------------------------------ convenience --

def prepare_decode(q, k_cache, v_cache, seqlens, scale, out, lse, workspace=None, num_splits=None, stream=None):
    """Check and marshal the arguments once; return a no-argument callable
    that enqueues fd_decode_splits with those pointers (for decode loops that
    reuse the same buffers). The planned split count is used by default."""
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache)
    _outputs(out, lse, B, Hq, D)
    _seqlens(seqlens, B)
    S = fd_plan(B, Hq, Hkv, D, Lmax) if num_splits is None else int(num_splits)
    wp, wb = _ws(workspace)
    fn = lib().fd_decode_splits
    args = (B, Hq, Hkv, D, Lmax, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(),
            ctypes.c_float(scale), out.data_ptr(), lse.data_ptr(), wp, wb, S, _stream(stream, q.device))

    def call():
        rc = fn(*args)
        if rc != 0:
            raise FdError(rc, "fd_decode_splits")

    call.num_splits = S
    return call


def prepare_decode_multi(q, k_cache, v_cache, seqlens, scale, out, lse, workspace=None, num_splits=None,
                         stream=None):
    """prepare_decode for fd_decode_multi: q [B, q_len, Hq, D], out
    [B, q_len, Hq, D], lse [B, q_len, Hq]."""
    if q.dim() != 4 or not q.is_contiguous():
        raise ValueError("q must be a contiguous [B, q_len, Hq, D] tensor")
    B, q_len, Hq, D = q.shape
    _, _, Hkv, _, Lmax = _shapes(q.view(B, q_len * Hq, D), k_cache, v_cache)
    if out.shape != (B, q_len, Hq, D) or lse.shape != (B, q_len, Hq):
        raise ValueError("out must be [B,q_len,Hq,D] and lse [B,q_len,Hq]")
    for t, name in ((out, "out"), (lse, "lse")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")
    _seqlens(seqlens, B)
    S = fd_plan(B, Hq, Hkv, D, Lmax) if num_splits is None else int(num_splits)
    wp, wb = _ws(workspace)
    fn = lib().fd_decode_multi
    args = (B, q_len, Hq, Hkv, D, Lmax, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(),
            ctypes.c_float(scale), out.data_ptr(), lse.data_ptr(), wp, wb, S, _stream(stream, q.device))

    def call():
        rc = fn(*args)
        if rc != 0:
            raise FdError(rc, "fd_decode_multi")

    call.num_splits = S
    return call


FD_KV_E4M3, FD_KV_INT8 = 1, 2
KV_CODES = {"e4m3": FD_KV_E4M3, "int8": FD_KV_INT8}


def prepare_decode_quant(q, k_codes, v_codes, k_scale, v_scale, kv_type, seqlens, scale, out, lse, workspace=None,
                         num_splits=None, stream=None):
    """prepare_decode for fd_decode_quant: an 8-bit cache (k_codes / v_codes
    uint8 [B, Hkv, Lmax, D], k_scale / v_scale float32 [Hkv], kv_type "e4m3"
    or "int8"); q [B, Hq, D] (one query) or [B, q_len, Hq, D], out / lse
    shaped to match."""
    if kv_type not in KV_CODES:
        raise ValueError("kv_type must be 'e4m3' or 'int8'")
    if q.dim() == 3:
        B, Hq, D = q.shape
        q_len = 1
    elif q.dim() == 4:
        B, q_len, Hq, D = q.shape
    else:
        raise ValueError("q must be [B, Hq, D] or [B, q_len, Hq, D]")
    if q.dtype != torch.bfloat16 or not q.is_cuda or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 CUDA tensor")
    if k_codes.dim() != 4 or v_codes.shape != k_codes.shape or k_codes.shape[0] != B or k_codes.shape[3] != D:
        raise ValueError("k_codes, v_codes must be [B, Hkv, Lmax, D]")
    _, Hkv, Lmax, _ = k_codes.shape
    for t, name in ((k_codes, "k_codes"), (v_codes, "v_codes")):
        if t.dtype != torch.uint8 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous uint8 CUDA tensor")
    for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        if t.shape != (Hkv,) or t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor of shape [Hkv]")
    oshape = q.shape[:-1]
    if out.shape != q.shape or lse.shape != oshape:
        raise ValueError("out must be shaped like q and lse like q without D")
    for t, name in ((out, "out"), (lse, "lse")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")
    _seqlens(seqlens, B)
    S = fd_plan(B, Hq, Hkv, D, Lmax) if num_splits is None else int(num_splits)
    wp, wb = _ws(workspace)
    fn = lib().fd_decode_quant
    args = (B, q_len, Hq, Hkv, D, Lmax, KV_CODES[kv_type], q.data_ptr(), k_codes.data_ptr(), v_codes.data_ptr(),
            k_scale.data_ptr(), v_scale.data_ptr(), seqlens.data_ptr(), ctypes.c_float(scale), out.data_ptr(),
            lse.data_ptr(), wp, wb, S, _stream(stream, q.device))

    def call():
        rc = fn(*args)
        if rc != 0:
            raise FdError(rc, "fd_decode_quant")

    call.num_splits = S
    return call


def fd_decode_quant(q, k_codes, v_codes, k_scale, v_scale, kv_type, seqlens, scale, out, lse, workspace=None,
                    num_splits=0, stream=None):
    """Attention over an 8-bit key/value cache (see prepare_decode_quant);
    num_splits 0 lets the library plan the split count."""
    prepare_decode_quant(q, k_codes, v_codes, k_scale, v_scale, kv_type, seqlens, scale, out, lse, workspace,
                         num_splits, stream)()


def quant_workspace_bytes(q, k_codes, num_splits):
    """Workspace bytes fd_decode_quant needs for these shapes."""
    q_len = 1 if q.dim() == 3 else q.shape[1]
    B, Hq, D = q.shape[0], q.shape[-2], q.shape[-1]
    return fd_workspace_bytes(B, Hq * q_len, k_codes.shape[1], D, k_codes.shape[2], num_splits)


def decode_quant(q, k_codes, v_codes, k_scale, v_scale, kv_type, seqlens, scale, num_splits=None, stream=None):
    """Allocate out / lse / workspace with torch and run fd_decode_quant."""
    B, Hq, D = q.shape[0], q.shape[-2], q.shape[-1]
    Hkv, Lmax = k_codes.shape[1], k_codes.shape[2]
    S = fd_plan(B, Hq, Hkv, D, Lmax) if num_splits is None else int(num_splits)
    nbytes = quant_workspace_bytes(q, k_codes, S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    fd_decode_quant(q, k_codes, v_codes, k_scale, v_scale, kv_type, seqlens, scale, out, lse, ws, S, stream)
    return out, lse


def fd_merge_partials(part_out, part_lse, out, lse, stream=None):
    """Merge R partial results per row: part_out [R, ..., D] and part_lse
    [R, ...] (fp32, contiguous, CUDA) into out [..., D] and lse [...]."""
    if part_out.dim() < 2 or part_lse.shape != part_out.shape[:-1]:
        raise ValueError("part_out must be [R, ..., D] and part_lse [R, ...]")
    R, D = part_out.shape[0], part_out.shape[-1]
    rows = part_lse[0].numel()
    if out.shape != part_out.shape[1:] or lse.shape != part_lse.shape[1:]:
        raise ValueError("out / lse must be shaped like one part")
    for t, name in ((part_out, "part_out"), (part_lse, "part_lse"), (out, "out"), (lse, "lse")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")
    _check(lib().fd_merge_partials(R, rows, D, part_out.data_ptr(), part_lse.data_ptr(), out.data_ptr(),
                                   lse.data_ptr(), _stream(stream, out.device)), "fd_merge_partials")


def fd_read_probe(buf, sink, stream=None):
    """Read every byte of the CUDA tensor `buf` once (HBM read-bandwidth
    probe); `sink` is a one-element int64 CUDA tensor."""
    if not buf.is_cuda or not buf.is_contiguous() or sink.dtype != torch.int64 or not sink.is_cuda:
        raise ValueError("buf must be a contiguous CUDA tensor and sink an int64 CUDA tensor")
    nbytes = buf.numel() * buf.element_size()
    _check(lib().fd_read_probe(buf.data_ptr(), nbytes, sink.data_ptr(), _stream(stream, buf.device)),
           "fd_read_probe")


def workspace_layout(B, Hq, Hkv, D, num_splits):
    """(slots, g, byte offset of seg_lse, byte offset of the counters) of the
    documented workspace layout. The counters are B*Hkv row counters followed
    by `slots` chunk counters, all int32."""
    slots = num_splits + B * Hkv - 1
    g = Hq // Hkv
    off = (slots * g * D * 4 + 255) // 256 * 256
    tick = off + (slots * g * 4 + 255) // 256 * 256
    return slots, g, off, tick


def decode(q, k_cache, v_cache, seqlens, scale, num_splits=None, stream=None):
    """Allocate out / lse / workspace with torch and run fd_decode (or
    fd_decode_splits when num_splits is given). Returns (out, lse)."""
    B, Hq, Hkv, D, Lmax = _shapes(q, k_cache, v_cache)
    S = fd_plan(B, Hq, Hkv, D, Lmax) if num_splits is None else int(num_splits)
    nbytes = fd_workspace_bytes(B, Hq, Hkv, D, Lmax, S)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    fd_decode_splits(q, k_cache, v_cache, seqlens, scale, out, lse, ws, S, stream)
    return out, lse
