"""Python binding of libbsa.so: block-sparse KV attention on a B200 (sm_100a).

Thin ctypes marshalling over the C ABI declared in ``include/bsa.h``: torch
tensors supply device pointers, the current CUDA stream supplies the stream,
and every computation runs in the library's CUDA kernels.  There is no CPU
or PyTorch fallback: importing this package fails when ``libbsa.so`` is
missing, and every call raises :class:`BsaError` when the library reports a
non-OK status.

The functions carry the C names:

* :func:`bsa_gilbert_perm` - host Gilbert order of a T x H x W chunk
* :func:`bsa_kv_append` - scatter a chunk's K/V into the block cache
* :func:`bsa_tokens_to_blocks` / :func:`bsa_blocks_to_tokens` - reorder Q / O
* :func:`bsa_tokens_to_blocks_mean` - reorder Q and pool its blocks in one pass
* :func:`bsa_route` - pooled-score top-K route per query block
* :func:`bsa_route_qmean` - the same route from precomputed query means
* :func:`bsa_attn` - indexed block-sparse attention (O and LSE)
* :func:`bsa_attn_tokens` - the same with O and LSE in raster token order
* :func:`bsa_check_device_error` - read and clear the device error word

Method: "Velox: Spatial Memory Makes World Models Efficient" (Key
Contributions 3; Methodology Steps 4-6).
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional, Tuple

import numpy as np
import torch

BLK = 128
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

STATUS_NAMES = {
    0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_SHAPE", 3: "BSA_ERR_CAPACITY",
    4: "BSA_ERR_UNSUPPORTED", 5: "BSA_ERR_CUDA", 6: "BSA_ERR_DEVICE_FAULT", 7: "BSA_ERR_TIMEOUT",
}
DEV_CODES = {0: "BSA_DEV_OK", 1: "BSA_DEV_BAD_INDEX", 2: "BSA_DEV_BAD_COUNT",
             3: "BSA_DEV_BAD_VALID", 4: "BSA_DEV_BAD_PERM", 5: "BSA_DEV_WAIT_TIMEOUT"}

# Every symbol include/bsa.h declares (checked by the tests).
EXPORTS = ("bsa_abi_version", "bsa_status_string", "bsa_gilbert_perm", "bsa_kv_append",
           "bsa_kv_pool_means",
           "bsa_tokens_to_blocks", "bsa_tokens_to_blocks_mean", "bsa_blocks_to_tokens",
           "bsa_route_workspace_size", "bsa_route", "bsa_route_qmean", "bsa_route_velox",
           "bsa_route_velox_qmean",
           "bsa_route_noalloc", "bsa_attn", "bsa_attn_tokens",
           "bsa_geometry_prior",
           "bsa_check_device_error",
           "bsa_selftest_bounded_wait")


class BsaError(RuntimeError):
    """A libbsa call returned a non-OK status."""

    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        name = STATUS_NAMES.get(status, f"status {status}")
        super().__init__(f"{fn}: {name}{(' - ' + detail) if detail else ''}")


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libbsa.so not found at {LIB_PATH}; build it with "
        "`python -m block_sparse_kv_bsa_b200._build` (there is no fallback path)")

_lib = ctypes.CDLL(LIB_PATH)


class CCache(ctypes.Structure):
    """ctypes mirror of ``bsa_kv_cache``."""
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("block_valid", ctypes.c_void_p),
                ("B", ctypes.c_int32), ("Hh", ctypes.c_int32), ("D", ctypes.c_int32),
                ("max_blocks", ctypes.c_int32), ("n_blocks", ctypes.c_int32),
                ("kmean", ctypes.c_void_p)]


class CVeloxRoute(ctypes.Structure):
    """ctypes mirror of ``bsa_velox_route``."""
    _fields_ = [("coverage", ctypes.c_void_p), ("eta_cov", ctypes.c_float),
                ("tau", ctypes.c_float), ("k_cov", ctypes.c_int32), ("k_unc", ctypes.c_int32),
                ("mass", ctypes.c_float), ("prev_first", ctypes.c_int32),
                ("n_prev", ctypes.c_int32), ("window_half", ctypes.c_int32),
                ("ref_first", ctypes.c_int32), ("n_ref", ctypes.c_int32)]


_i, _p, _f, _sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
_sig = {
    "bsa_abi_version": (ctypes.c_int, []),
    "bsa_status_string": (ctypes.c_char_p, [_i]),
    "bsa_gilbert_perm": (_i, [_i, _i, _i, _p]),
    "bsa_kv_append": (_i, [ctypes.POINTER(CCache), _p, _p, _i, _i, _i, _p, _p, _p]),
    "bsa_kv_pool_means": (_i, [ctypes.POINTER(CCache), _i, _i, _p, _p]),
    "bsa_tokens_to_blocks": (_i, [_p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p]),
    "bsa_tokens_to_blocks_mean": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p]),
    "bsa_blocks_to_tokens": (_i, [_p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p]),
    "bsa_route_workspace_size": (_i, [_i, _i, _i, _i, _i, ctypes.POINTER(_sz)]),
    "bsa_route": (_i, [_p, ctypes.POINTER(CCache), _p, _i, _i, _i, _p, _f, _f, _f, _i,
                       _p, _p, _i, _p, _sz, _p, _p]),
    "bsa_route_qmean": (_i, [_p, ctypes.POINTER(CCache), _i, _i, _i, _p, _f, _f, _f, _i,
                             _p, _p, _i, _p, _sz, _p, _p]),
    "bsa_geometry_prior": (_i, [_p, _i, _f, _f, _f, _f, _p, _p, _i, _p, _p, _i, _i, _i, _p, _p,
                                _p, _i, _p, _p, _p, _p]),
    "bsa_route_velox": (_i, [_p, ctypes.POINTER(CCache), _p, _i, _i, _i, _p, _f, _f, _f,
                             ctypes.POINTER(CVeloxRoute), _p, _p, _i, _p, _sz, _p, _p]),
    "bsa_route_velox_qmean": (_i, [_p, ctypes.POINTER(CCache), _i, _i, _i, _p, _f, _f, _f,
                                   ctypes.POINTER(CVeloxRoute), _p, _p, _i, _p, _sz, _p, _p]),
    "bsa_route_noalloc": (_i, [_p, ctypes.POINTER(CCache), _p, _i, _i, _i, _p, _f, _f, _f, _i,
                               _p, _p, _i, _p, _p]),
    "bsa_attn": (_i, [_p, ctypes.POINTER(CCache), _p, _p, _p, _i, _i, _f, _p, _p, _p, _p]),
    "bsa_attn_tokens": (_i, [_p, ctypes.POINTER(CCache), _p, _p, _p, _i, _f, _i, _i, _i, _p, _p,
                             _p, _p, _p]),
    "bsa_check_device_error": (_i, [_p, _p, ctypes.POINTER(ctypes.c_int32)]),
    "bsa_selftest_bounded_wait": (_i, [_p, ctypes.c_longlong, _p]),
}
for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def lib() -> ctypes.CDLL:
    """The loaded library handle."""
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        raise BsaError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(device) -> torch.device:
    """A device with an explicit index (``cuda`` -> ``cuda:<current>``)."""
    d = torch.device(device)
    if d.type == "cuda" and d.index is None:
        d = torch.device("cuda", torch.cuda.current_device())
    return d


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, device=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != _dev(device):
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


_err_words = {}
_lock = threading.Lock()


def error_word(device) -> torch.Tensor:
    """The per-device int32 word kernels report BSA_DEV_* codes into."""
    device = _dev(device)
    with _lock:
        w = _err_words.get(device)
        if w is None:
            w = torch.zeros(1, dtype=torch.int32, device=device)
            _err_words[device] = w
    return w


def abi_version() -> int:
    return int(_lib.bsa_abi_version())


def status_string(status: int) -> str:
    return _lib.bsa_status_string(int(status)).decode()


def n_blocks_for(T: int, H: int, W: int) -> int:
    return -(-T * H * W // BLK)


# ---------------------------------------------------------------------------
# Gilbert order
# ---------------------------------------------------------------------------

_perm_cache = {}


def bsa_gilbert_perm(T: int, H: int, W: int) -> np.ndarray:
    """perm[i] = curve position of raster token i (host int32 [T*H*W])."""
    n = T * H * W
    out = np.empty(max(n, 1), dtype=np.int32)
    _check("bsa_gilbert_perm", _lib.bsa_gilbert_perm(int(T), int(H), int(W),
                                                      out.ctypes.data_as(ctypes.c_void_p)))
    return out[:n]


def gilbert_perm_device(T: int, H: int, W: int, device) -> torch.Tensor:
    """The Gilbert table of a chunk shape on ``device``, computed once and cached."""
    key = (int(T), int(H), int(W), _dev(device))
    with _lock:
        t = _perm_cache.get(key)
    if t is None:
        t = torch.from_numpy(bsa_gilbert_perm(T, H, W)).to(device)
        with _lock:
            _perm_cache[key] = t
    return t


# ---------------------------------------------------------------------------
# KV cache
# ---------------------------------------------------------------------------

class KVCache:
    """A caller-owned block KV cache: K, V bf16 [B, Hh, max_blocks, 128, D] and
    the valid-row count of every block."""

    def __init__(self, B: int, Hh: int, D: int, max_blocks: int, device="cuda",
                 pooled_keys: bool = False):
        self.B, self.Hh, self.D, self.max_blocks = int(B), int(Hh), int(D), int(max_blocks)
        self.device = _dev(device)
        shape = (self.B, self.Hh, self.max_blocks, BLK, self.D)
        self.k = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        self.v = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        self.block_valid = torch.zeros(self.max_blocks, dtype=torch.int32, device=self.device)
        # Optional pooled-key cache: block means of K, written at append time
        # and read by bsa_route instead of the history keys.
        self.kmean = (torch.zeros((self.B, self.Hh, self.max_blocks, self.D), dtype=torch.float32,
                                  device=self.device) if pooled_keys else None)
        self.n_blocks = 0

    def c_struct(self) -> CCache:
        return CCache(self.k.data_ptr(), self.v.data_ptr(), self.block_valid.data_ptr(),
                      self.B, self.Hh, self.D, self.max_blocks, self.n_blocks,
                      None if self.kmean is None else self.kmean.data_ptr())


def bsa_kv_append(cache: KVCache, k_tok: torch.Tensor, v_tok: torch.Tensor,
                  T: int, H: int, W: int, d_err: Optional[torch.Tensor] = None,
                  table: bool = True) -> int:
    """Append one chunk (bf16 [B, T*H*W, Hh, D] K and V); returns its first block.
    table=False passes no permutation table: the kernels locate the Gilbert
    slots themselves (the same order)."""
    shape = (cache.B, T * H * W, cache.Hh, cache.D)
    _need(k_tok, "k_tok", torch.bfloat16, cache.device, shape)
    _need(v_tok, "v_tok", torch.bfloat16, cache.device, shape)
    perm = gilbert_perm_device(T, H, W, cache.device) if table else None
    err = error_word(cache.device) if d_err is None else d_err
    cs = cache.c_struct()
    first = cache.n_blocks
    _check("bsa_kv_append", _lib.bsa_kv_append(ctypes.byref(cs), _ptr(k_tok), _ptr(v_tok),
                                                int(T), int(H), int(W), _ptr(perm), _ptr(err),
                                                _stream(cache.device)))
    cache.n_blocks = int(cs.n_blocks)
    return first


def bsa_kv_pool_means(cache: KVCache, first: int = 0, count: Optional[int] = None):
    """(Re)compute the pooled-key cache for blocks [first, first + count)."""
    if cache.kmean is None:
        raise ValueError("the cache was created without pooled_keys")
    if count is None:
        count = cache.n_blocks - first
    cs = cache.c_struct()
    _check("bsa_kv_pool_means", _lib.bsa_kv_pool_means(
        ctypes.byref(cs), int(first), int(count), _ptr(error_word(cache.device)),
        _stream(cache.device)))


def bsa_tokens_to_blocks(x_tok: torch.Tensor, T: int, H: int, W: int,
                         out: Optional[torch.Tensor] = None, table: bool = True) -> torch.Tensor:
    """[B, T*H*W, Hh, D] raster tokens -> [B, Hh, nb*128, D] Gilbert blocks (zero pads)."""
    if x_tok.dim() != 4:
        raise ValueError("x_tok must be [B, T*H*W, Hh, D]")
    B, N, Hh, D = x_tok.shape
    _need(x_tok, "x_tok", torch.bfloat16)
    nb = n_blocks_for(T, H, W)
    if out is None:
        out = torch.empty((B, Hh, nb * BLK, D), dtype=torch.bfloat16, device=x_tok.device)
    _need(out, "out", torch.bfloat16, x_tok.device, (B, Hh, nb * BLK, D))
    perm = gilbert_perm_device(T, H, W, x_tok.device) if table else None
    _check("bsa_tokens_to_blocks", _lib.bsa_tokens_to_blocks(
        _ptr(x_tok), _ptr(out), B, Hh, D, int(T), int(H), int(W), _ptr(perm),
        _ptr(error_word(x_tok.device)), _stream(x_tok.device)))
    return out


def bsa_tokens_to_blocks_mean(x_tok: torch.Tensor, T: int, H: int, W: int,
                              out: Optional[torch.Tensor] = None,
                              mean: Optional[torch.Tensor] = None, table: bool = True
                              ) -> Tuple[torch.Tensor, torch.Tensor]:
    """bsa_tokens_to_blocks plus the fp32 mean of every block's valid rows:
    returns (blocks [B, Hh, nb*128, D], means [B, Hh, nb, D])."""
    if x_tok.dim() != 4:
        raise ValueError("x_tok must be [B, T*H*W, Hh, D]")
    B, N, Hh, D = x_tok.shape
    _need(x_tok, "x_tok", torch.bfloat16)
    nb = n_blocks_for(T, H, W)
    if out is None:
        out = torch.empty((B, Hh, nb * BLK, D), dtype=torch.bfloat16, device=x_tok.device)
    if mean is None:
        mean = torch.empty((B, Hh, nb, D), dtype=torch.float32, device=x_tok.device)
    _need(out, "out", torch.bfloat16, x_tok.device, (B, Hh, nb * BLK, D))
    _need(mean, "mean", torch.float32, x_tok.device, (B, Hh, nb, D))
    perm = gilbert_perm_device(T, H, W, x_tok.device) if table else None
    _check("bsa_tokens_to_blocks_mean", _lib.bsa_tokens_to_blocks_mean(
        _ptr(x_tok), _ptr(out), _ptr(mean), B, Hh, D, int(T), int(H), int(W), _ptr(perm),
        _ptr(error_word(x_tok.device)), _stream(x_tok.device)))
    return out, mean


def bsa_blocks_to_tokens(x_blk: torch.Tensor, T: int, H: int, W: int,
                         out: Optional[torch.Tensor] = None, table: bool = True) -> torch.Tensor:
    """[B, Hh, nb*128, D] Gilbert blocks -> [B, T*H*W, Hh, D] raster tokens."""
    if x_blk.dim() != 4:
        raise ValueError("x_blk must be [B, Hh, nb*128, D]")
    B, Hh, R, D = x_blk.shape
    _need(x_blk, "x_blk", torch.bfloat16)
    if R != n_blocks_for(T, H, W) * BLK:
        raise ValueError("x_blk rows do not match the chunk shape")
    if out is None:
        out = torch.empty((B, T * H * W, Hh, D), dtype=torch.bfloat16, device=x_blk.device)
    _need(out, "out", torch.bfloat16, x_blk.device, (B, T * H * W, Hh, D))
    perm = gilbert_perm_device(T, H, W, x_blk.device) if table else None
    _check("bsa_blocks_to_tokens", _lib.bsa_blocks_to_tokens(
        _ptr(x_blk), _ptr(out), B, Hh, D, int(T), int(H), int(W), _ptr(perm),
        _ptr(error_word(x_blk.device)), _stream(x_blk.device)))
    return out


# ---------------------------------------------------------------------------
# Routing and attention
# ---------------------------------------------------------------------------

def bsa_route_workspace_size(B: int, Hh: int, D: int, n_q_blocks: int, n_hist: int) -> int:
    n = ctypes.c_size_t(0)
    _check("bsa_route_workspace_size", _lib.bsa_route_workspace_size(
        int(B), int(Hh), int(D), int(n_q_blocks), int(n_hist), ctypes.byref(n)))
    return int(n.value)


def route_max_sel(top_k: int, n_hist: int, n_own: int) -> int:
    return min(int(top_k), int(n_hist)) + int(n_own)


def bsa_route(q_blk: torch.Tensor, cache: KVCache, n_hist: int, own_first: int, n_own: int,
              top_k: int, g: Optional[torch.Tensor] = None, lam: float = 2.0,
              g_ref: float = 0.2, sm_scale: Optional[float] = None,
              q_valid: Optional[torch.Tensor] = None, max_sel: Optional[int] = None,
              idx: Optional[torch.Tensor] = None, cnt: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Route every (b, h, query block); returns (idx [B,Hh,n_own,max_sel], cnt [B,Hh,n_own])."""
    dev = cache.device
    _need(q_blk, "q_blk", torch.bfloat16, dev, (cache.B, cache.Hh, n_own * BLK, cache.D))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cache.D)
    if max_sel is None:
        max_sel = route_max_sel(top_k, n_hist, n_own)
    if idx is None:
        idx = torch.empty((cache.B, cache.Hh, n_own, max_sel), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((cache.B, cache.Hh, n_own), dtype=torch.int32, device=dev)
    _need(idx, "idx", torch.int32, dev, (cache.B, cache.Hh, n_own, max_sel))
    _need(cnt, "cnt", torch.int32, dev, (cache.B, cache.Hh, n_own))
    if g is not None:
        _need(g, "g", torch.float32, dev, (cache.B, n_own, n_hist))
    if q_valid is not None:
        _need(q_valid, "q_valid", torch.int32, dev, (n_own,))
    ws_bytes = bsa_route_workspace_size(cache.B, cache.Hh, cache.D, n_own, n_hist)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    cs = cache.c_struct()
    _check("bsa_route", _lib.bsa_route(
        _ptr(q_blk), ctypes.byref(cs), _ptr(q_valid), int(n_hist), int(own_first), int(n_own),
        _ptr(g), float(lam), float(g_ref), float(sm_scale), int(top_k), _ptr(idx), _ptr(cnt),
        int(max_sel), _ptr(workspace), workspace.numel(), _ptr(error_word(dev)), _stream(dev)))
    return idx, cnt


def bsa_route_qmean(q_mean: torch.Tensor, cache: KVCache, n_hist: int, own_first: int,
                    n_own: int, top_k: int, g: Optional[torch.Tensor] = None, lam: float = 2.0,
                    g_ref: float = 0.2, sm_scale: Optional[float] = None,
                    max_sel: Optional[int] = None, idx: Optional[torch.Tensor] = None,
                    cnt: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """bsa_route from the query-block means [B, Hh, n_own, D] (fp32), e.g.
    those of bsa_tokens_to_blocks_mean; returns (idx, cnt)."""
    dev = cache.device
    _need(q_mean, "q_mean", torch.float32, dev, (cache.B, cache.Hh, n_own, cache.D))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cache.D)
    if max_sel is None:
        max_sel = route_max_sel(top_k, n_hist, n_own)
    if idx is None:
        idx = torch.empty((cache.B, cache.Hh, n_own, max_sel), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((cache.B, cache.Hh, n_own), dtype=torch.int32, device=dev)
    _need(idx, "idx", torch.int32, dev, (cache.B, cache.Hh, n_own, max_sel))
    _need(cnt, "cnt", torch.int32, dev, (cache.B, cache.Hh, n_own))
    if g is not None:
        _need(g, "g", torch.float32, dev, (cache.B, n_own, n_hist))
    ws_bytes = bsa_route_workspace_size(cache.B, cache.Hh, cache.D, n_own, n_hist)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    cs = cache.c_struct()
    _check("bsa_route_qmean", _lib.bsa_route_qmean(
        _ptr(q_mean), ctypes.byref(cs), int(n_hist), int(own_first), int(n_own), _ptr(g),
        float(lam), float(g_ref), float(sm_scale), int(top_k), _ptr(idx), _ptr(cnt),
        int(max_sel), _ptr(workspace), workspace.numel(), _ptr(error_word(dev)), _stream(dev)))
    return idx, cnt


def velox_max_sel(n_hist: int, n_own: int, k_cov: int = 80, k_unc: int = 150, n_prev: int = 0,
                  window_half: int = 13, n_ref: int = 0) -> int:
    """Smallest max_sel bsa_route_velox accepts."""
    budget = max(k_cov, n_prev, k_unc)
    return min(n_hist, budget + 2 * window_half + 1 + n_ref) + n_own


def bsa_route_velox(q_blk: Optional[torch.Tensor], cache: KVCache, n_hist: int, own_first: int,
                    n_own: int, g: Optional[torch.Tensor] = None,
                    coverage: Optional[torch.Tensor] = None, lam: float = 2.0,
                    g_ref: float = 0.2, sm_scale: Optional[float] = None, tau: float = 0.1,
                    eta_cov: float = 0.9, k_cov: int = 80, k_unc: int = 150, mass: float = 0.9,
                    prev_first: int = 0, n_prev: int = 0, window_half: int = 13,
                    ref_first: int = 0, n_ref: int = 0, q_valid: Optional[torch.Tensor] = None,
                    max_sel: Optional[int] = None, idx: Optional[torch.Tensor] = None,
                    cnt: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None,
                    q_mean: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The page's full route; returns (idx [B,Hh,n_own,max_sel] padded with -1, cnt).
    With ``q_mean`` ([B, Hh, n_own, D] fp32, e.g. from
    bsa_tokens_to_blocks_mean) the query means are taken from it
    (bsa_route_velox_qmean) and ``q_blk`` may be None."""
    dev = cache.device
    if q_mean is not None:
        _need(q_mean, "q_mean", torch.float32, dev, (cache.B, cache.Hh, n_own, cache.D))
    else:
        _need(q_blk, "q_blk", torch.bfloat16, dev, (cache.B, cache.Hh, n_own * BLK, cache.D))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(cache.D)
    if max_sel is None:
        max_sel = velox_max_sel(n_hist, n_own, k_cov, k_unc, n_prev, window_half, n_ref)
    if idx is None:
        idx = torch.empty((cache.B, cache.Hh, n_own, max_sel), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((cache.B, cache.Hh, n_own), dtype=torch.int32, device=dev)
    _need(idx, "idx", torch.int32, dev, (cache.B, cache.Hh, n_own, max_sel))
    _need(cnt, "cnt", torch.int32, dev, (cache.B, cache.Hh, n_own))
    if g is not None:
        _need(g, "g", torch.float32, dev, (cache.B, n_own, n_hist))
    if coverage is not None:
        _need(coverage, "coverage", torch.float32, dev, (cache.B, n_own))
    if q_valid is not None:
        _need(q_valid, "q_valid", torch.int32, dev, (n_own,))
    ws_bytes = bsa_route_workspace_size(cache.B, cache.Hh, cache.D, n_own, n_hist)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    opts = CVeloxRoute(None if coverage is None else coverage.data_ptr(), float(eta_cov),
                       float(tau), int(k_cov), int(k_unc), float(mass), int(prev_first),
                       int(n_prev), int(window_half), int(ref_first), int(n_ref))
    cs = cache.c_struct()
    if q_mean is not None:
        _check("bsa_route_velox_qmean", _lib.bsa_route_velox_qmean(
            _ptr(q_mean), ctypes.byref(cs), int(n_hist), int(own_first), int(n_own), _ptr(g),
            float(lam), float(g_ref), float(sm_scale), ctypes.byref(opts), _ptr(idx), _ptr(cnt),
            int(max_sel), _ptr(workspace), workspace.numel(), _ptr(error_word(dev)),
            _stream(dev)))
        return idx, cnt
    _check("bsa_route_velox", _lib.bsa_route_velox(
        _ptr(q_blk), ctypes.byref(cs), _ptr(q_valid), int(n_hist), int(own_first), int(n_own),
        _ptr(g), float(lam), float(g_ref), float(sm_scale), ctypes.byref(opts), _ptr(idx),
        _ptr(cnt), int(max_sel), _ptr(workspace), workspace.numel(), _ptr(error_word(dev)),
        _stream(dev)))
    return idx, cnt


def bsa_geometry_prior(cams: torch.Tensor, intr, h_cam: torch.Tensor, h_rect: torch.Tensor,
                       q_cam: Optional[torch.Tensor] = None, q_rect: Optional[torch.Tensor] = None,
                       tok_cam: Optional[torch.Tensor] = None,
                       tok_uvd: Optional[torch.Tensor] = None,
                       q_valid: Optional[torch.Tensor] = None, grid_n: int = 8,
                       g: Optional[torch.Tensor] = None, coverage: Optional[torch.Tensor] = None,
                       want_g: bool = True, want_coverage: bool = True):
    """Overlap prior g [B, n_q, n_hist] and coverage [B, n_q] from slabs.

    cams float32 [B, n_cams, 12]; intr = (fx, fy, cx, cy); h_cam int32
    [B, n_hist, S], h_rect float32 [B, n_hist, S, 6]; q_cam/q_rect likewise
    for the query blocks (needed for g); tok_cam int32 [B, n_q, 128] and
    tok_uvd float32 [B, n_q, 128, 3] (needed for coverage).  Returns (g,
    coverage), either None when not requested."""
    dev = _dev(cams.device)
    B, n_cams = cams.shape[0], cams.shape[1]
    _need(cams, "cams", torch.float32, dev, (B, n_cams, 12))
    n_hist, S = h_cam.shape[1], h_cam.shape[2]
    _need(h_cam, "h_cam", torch.int32, dev, (B, n_hist, S))
    _need(h_rect, "h_rect", torch.float32, dev, (B, n_hist, S, 6))
    n_q = (q_cam if q_cam is not None else tok_cam).shape[1]
    if want_g:
        _need(q_cam, "q_cam", torch.int32, dev, (B, n_q, S))
        _need(q_rect, "q_rect", torch.float32, dev, (B, n_q, S, 6))
        if g is None:
            g = torch.empty((B, n_q, n_hist), dtype=torch.float32, device=dev)
        _need(g, "g", torch.float32, dev, (B, n_q, n_hist))
    else:
        g = None
    if want_coverage:
        _need(tok_cam, "tok_cam", torch.int32, dev, (B, n_q, BLK))
        _need(tok_uvd, "tok_uvd", torch.float32, dev, (B, n_q, BLK, 3))
        if coverage is None:
            coverage = torch.empty((B, n_q), dtype=torch.float32, device=dev)
        _need(coverage, "coverage", torch.float32, dev, (B, n_q))
    else:
        coverage = None
    if q_valid is not None:
        _need(q_valid, "q_valid", torch.int32, dev, (n_q,))
    fx, fy, cx, cy = (float(v) for v in intr)
    _check("bsa_geometry_prior", _lib.bsa_geometry_prior(
        _ptr(cams), int(n_cams), fx, fy, cx, cy, _ptr(q_cam), _ptr(q_rect), int(n_q),
        _ptr(h_cam), _ptr(h_rect), int(n_hist), int(S), int(grid_n), _ptr(tok_cam), _ptr(tok_uvd),
        _ptr(q_valid), int(B), _ptr(g), _ptr(coverage), _ptr(error_word(dev)), _stream(dev)))
    return g, coverage


def bsa_attn(q_blk: torch.Tensor, cache: KVCache, idx: torch.Tensor, cnt: torch.Tensor,
             q_valid: Optional[torch.Tensor] = None, sm_scale: Optional[float] = None,
             o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None
             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Indexed block-sparse attention; returns (O bf16 [B,Hh,nQB*128,D], LSE fp32 [B,Hh,nQB*128])."""
    dev = cache.device
    if q_blk.dim() != 4:
        raise ValueError("q_blk must be [B, Hh, nQB*128, D]")
    B, Hh, R, D = q_blk.shape
    if (B, Hh, D) != (cache.B, cache.Hh, cache.D) or R % BLK:
        raise ValueError("q_blk does not match the cache")
    nqb = R // BLK
    _need(q_blk, "q_blk", torch.bfloat16, dev)
    if idx.dim() != 4 or tuple(idx.shape[:3]) != (B, Hh, nqb):
        raise ValueError("idx must be [B, Hh, nQB, max_sel]")
    max_sel = idx.shape[3]
    _need(idx, "idx", torch.int32, dev)
    _need(cnt, "cnt", torch.int32, dev, (B, Hh, nqb))
    if q_valid is not None:
        _need(q_valid, "q_valid", torch.int32, dev, (nqb,))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q_blk)
    if lse is None:
        lse = torch.empty((B, Hh, R), dtype=torch.float32, device=dev)
    _need(o, "o", torch.bfloat16, dev, tuple(q_blk.shape))
    _need(lse, "lse", torch.float32, dev, (B, Hh, R))
    cs = cache.c_struct()
    _check("bsa_attn", _lib.bsa_attn(
        _ptr(q_blk), ctypes.byref(cs), _ptr(q_valid), _ptr(idx), _ptr(cnt), int(nqb),
        int(max_sel), float(sm_scale), _ptr(o), _ptr(lse), _ptr(error_word(dev)), _stream(dev)))
    return o, lse


def bsa_attn_tokens(q_blk: torch.Tensor, cache: KVCache, idx: torch.Tensor, cnt: torch.Tensor,
                    T: int, H: int, W: int, q_valid: Optional[torch.Tensor] = None,
                    sm_scale: Optional[float] = None, o: Optional[torch.Tensor] = None,
                    lse: Optional[torch.Tensor] = None,
                    table: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    """bsa_attn writing O and LSE in raster token order; returns
    (O bf16 [B, T*H*W, Hh, D], LSE fp32 [B, T*H*W, Hh])."""
    dev = cache.device
    if q_blk.dim() != 4:
        raise ValueError("q_blk must be [B, Hh, nQB*128, D]")
    B, Hh, R, D = q_blk.shape
    nqb = n_blocks_for(T, H, W)
    if (B, Hh, D) != (cache.B, cache.Hh, cache.D) or R != nqb * BLK:
        raise ValueError("q_blk does not match the cache and the chunk shape")
    _need(q_blk, "q_blk", torch.bfloat16, dev)
    if idx.dim() != 4 or tuple(idx.shape[:3]) != (B, Hh, nqb):
        raise ValueError("idx must be [B, Hh, nQB, max_sel]")
    max_sel = idx.shape[3]
    _need(idx, "idx", torch.int32, dev)
    _need(cnt, "cnt", torch.int32, dev, (B, Hh, nqb))
    if q_valid is not None:
        _need(q_valid, "q_valid", torch.int32, dev, (nqb,))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    N = T * H * W
    if o is None:
        o = torch.empty((B, N, Hh, D), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, N, Hh), dtype=torch.float32, device=dev)
    _need(o, "o", torch.bfloat16, dev, (B, N, Hh, D))
    _need(lse, "lse", torch.float32, dev, (B, N, Hh))
    perm = gilbert_perm_device(T, H, W, dev) if table else None
    cs = cache.c_struct()
    _check("bsa_attn_tokens", _lib.bsa_attn_tokens(
        _ptr(q_blk), ctypes.byref(cs), _ptr(q_valid), _ptr(idx), _ptr(cnt), int(max_sel),
        float(sm_scale), int(T), int(H), int(W), _ptr(perm), _ptr(o), _ptr(lse),
        _ptr(error_word(dev)), _stream(dev)))
    return o, lse


def bsa_check_device_error(device="cuda", d_err: Optional[torch.Tensor] = None) -> Tuple[int, int]:
    """Synchronise, read and clear the device error word: (status, raw BSA_DEV_* code)."""
    dev = _dev(device)
    err = error_word(dev) if d_err is None else d_err
    code = ctypes.c_int32(0)
    st = _lib.bsa_check_device_error(_ptr(err), _stream(dev), ctypes.byref(code))
    return int(st), int(code.value)


def bsa_selftest_bounded_wait(device="cuda", limit_cycles: int = 2_000_000) -> Tuple[int, int]:
    """Run the bounded-wait self-test; returns bsa_check_device_error's
    (status, code), which should be (BSA_ERR_TIMEOUT, BSA_DEV_WAIT_TIMEOUT)."""
    dev = _dev(device)
    _check("bsa_selftest_bounded_wait", _lib.bsa_selftest_bounded_wait(
        _ptr(error_word(dev)), int(limit_cycles), _stream(dev)))
    return bsa_check_device_error(dev)


def raise_on_device_error(device="cuda"):
    """Raise :class:`BsaError` if a kernel reported a device-side problem."""
    st, code = bsa_check_device_error(device)
    if st != 0:
        raise BsaError("device", st, DEV_CODES.get(code, str(code)))
