"""ctypes binding of libdsa_indexer.so (include/dsa_indexer.h).

Argument marshalling only: torch tensors (device memory) become raw pointers,
every step of the indexer runs in the library's CUDA kernels. The functions
keep the C names. There is no CPU fallback: if the library is missing or no
CUDA device is present, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa_indexer.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "dsa_indexer.h")

DSA_BF16, DSA_FP8_E4M3 = 0, 1
STATUS = {0: "DSA_OK", -1: "DSA_ERR_ARG", -2: "DSA_ERR_UNSUPPORTED", -3: "DSA_ERR_WORKSPACE",
          -4: "DSA_ERR_CUDA", -5: "DSA_ERR_TIMEOUT"}


class DsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


class IndexerArgs(ctypes.Structure):
    """Mirror of dsa_indexer_args."""
    _fields_ = [("batch", ctypes.c_int), ("T", ctypes.c_int), ("L", ctypes.c_int),
                ("H", ctypes.c_int), ("d", ctypes.c_int), ("q_offset", ctypes.c_longlong),
                ("qk_dtype", ctypes.c_int), ("q", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("k", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("w", ctypes.c_void_p)]


_lib = None
_P = ctypes.c_void_p
_SIGS = {
    "dsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "dsa_device_status": (ctypes.c_int, [_P, _P]),
    "dsa_selftest_wait_timeout": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "indexer_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int]),
    "indexer_score_topk": (ctypes.c_int, [_P, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
    "indexer_score_topk_noalloc": (ctypes.c_int, [_P, ctypes.c_int, _P, _P, _P]),
    "dsa_noalloc_status": (ctypes.c_int, [_P]),
    "indexer_lists_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int]),
    "indexer_score_topk_lists": (ctypes.c_int, [_P, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
    "indexer_scores": (ctypes.c_int, [_P, _P, ctypes.c_longlong, _P, ctypes.c_size_t, _P]),
    "indexer_score_gathered": (ctypes.c_int, [_P, _P, ctypes.c_int, ctypes.c_int, _P,
                                              ctypes.c_longlong, _P, ctypes.c_size_t, _P]),
    "indexer_topk_rows": (ctypes.c_int, [_P, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_int,
                                         ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         _P, ctypes.c_int, ctypes.c_int, _P, _P, _P,
                                         ctypes.c_size_t, _P]),
    "dsa_meanpool_keys": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, _P, _P]),
    "misa_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int]),
    "misa_route_score_topk": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "hisa_refine_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int, ctypes.c_int]),
    "hisa_refine_scores": (ctypes.c_int, [_P, _P, ctypes.c_int, ctypes.c_int, _P, ctypes.c_longlong, _P,
                                          ctypes.c_size_t, _P]),
    "dosa_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int, ctypes.c_int]),
    "dosa_score_topk": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "dsa_profile_begin": (ctypes.c_int, []),
    "dsa_profile_end": (ctypes.c_int, [ctypes.c_char_p, ctypes.c_size_t, _P, ctypes.c_int]),
    "indexcache_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int, ctypes.c_char_p, ctypes.c_int]),
    "indexcache_score_topk": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_char_p, ctypes.c_int, _P, _P, _P,
                                             ctypes.c_size_t, _P]),
    "hisa_workspace_size": (ctypes.c_size_t, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "hisa_block_filter_topk": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P,
                                              _P, _P, _P, ctypes.c_size_t, _P]),
    "dsa_pool_keys": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P]),
    "misa_route_score_topk_pooled": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "hisa_block_filter_topk_pooled": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P,
                                                     _P, _P, _P, _P, ctypes.c_size_t, _P]),
}


def header_symbols() -> list:
    """Names of the functions include/dsa_indexer.h exports."""
    with open(HEADER_PATH) as f:
        txt = f.read()
    return re.findall(r"DSA_EXPORT\s+[\w\s\*]+?\b(\w+)\s*\(", txt)


def lib():
    """Load the library (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_attention_token_score_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, st: int):
    if st != 0:
        raise DsaError(fn, st)


def make_args(q: torch.Tensor, k: torch.Tensor, w: torch.Tensor, q_offset: int,
              q_scale: Optional[torch.Tensor] = None, k_scale: Optional[torch.Tensor] = None) -> IndexerArgs:
    """q [batch,T,H,d] bf16 (or uint8 e4m3 bytes), k [batch,L,d], w [batch,T,H] fp32."""
    if q.dim() != 4 or k.dim() != 3 or w.dim() != 3:
        raise ValueError("q [batch,T,H,d], k [batch,L,d], w [batch,T,H] expected")
    fp8 = q.dtype in (torch.uint8, torch.float8_e4m3fn)
    if not fp8 and q.dtype != torch.bfloat16:
        raise ValueError("q must be bf16 or e4m3")
    b, T, H, d = q.shape
    a = IndexerArgs(batch=b, T=T, L=k.shape[1], H=H, d=d, q_offset=int(q_offset),
                    qk_dtype=DSA_FP8_E4M3 if fp8 else DSA_BF16)
    a.q, a.k, a.w = (t.data_ptr() for t in (q, k, w))
    a.q_scale = q_scale.data_ptr() if q_scale is not None else None
    a.k_scale = k_scale.data_ptr() if k_scale is not None else None
    for t in (q, k, w, q_scale, k_scale):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("contiguous device tensors expected")
    return a


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed, 256-byte aligned device buffer of at least nbytes (torch's
    allocator aligns to 512). Zeroing makes the status word of a workspace that
    no call has used yet read as "ok"."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


# ------------------------------------------------------------------ entry points
def indexer_workspace_size(args: IndexerArgs, topk: int) -> int:
    return int(lib().indexer_workspace_size(ctypes.byref(args), topk))


def indexer_score_topk(args: IndexerArgs, topk: int, out_idx: torch.Tensor,
                       out_score: Optional[torch.Tensor], workspace: torch.Tensor, stream=None):
    _check("indexer_score_topk",
           lib().indexer_score_topk(ctypes.byref(args), topk, _ptr(out_idx), _ptr(out_score),
                                    _ptr(workspace), workspace.numel(), _stream_ptr(stream)))


def indexer_score_topk_noalloc(args: IndexerArgs, topk: int, out_idx: torch.Tensor,
                               out_score: Optional[torch.Tensor], stream=None):
    """indexer_score_topk without a workspace (the library's static scratch)."""
    _check("indexer_score_topk_noalloc",
           lib().indexer_score_topk_noalloc(ctypes.byref(args), topk, _ptr(out_idx),
                                            _ptr(out_score), _stream_ptr(stream)))


def indexer_lists_workspace_size(args: IndexerArgs, topk: int) -> int:
    return int(lib().indexer_lists_workspace_size(ctypes.byref(args), topk))


def indexer_score_topk_lists(args: IndexerArgs, topk: int, out_idx: torch.Tensor,
                             out_score: Optional[torch.Tensor], workspace: torch.Tensor, stream=None):
    _check("indexer_score_topk_lists",
           lib().indexer_score_topk_lists(ctypes.byref(args), topk, _ptr(out_idx), _ptr(out_score),
                                          _ptr(workspace), workspace.numel(), _stream_ptr(stream)))


def dsa_noalloc_status(stream=None) -> int:
    """Status word of the static scratch of indexer_score_topk_noalloc (0 = ok)."""
    return int(lib().dsa_noalloc_status(_stream_ptr(stream)))


def indexer_scores(args: IndexerArgs, out_scores: torch.Tensor, ld: int, workspace: torch.Tensor,
                   stream=None):
    _check("indexer_scores",
           lib().indexer_scores(ctypes.byref(args), _ptr(out_scores), ld, _ptr(workspace),
                                workspace.numel(), _stream_ptr(stream)))


def indexer_score_gathered(args: IndexerArgs, cand: torch.Tensor, n_slots: int, blk: int,
                           out: torch.Tensor, ld: int, workspace: torch.Tensor, stream=None):
    _check("indexer_score_gathered",
           lib().indexer_score_gathered(ctypes.byref(args), _ptr(cand), n_slots, blk, _ptr(out), ld,
                                        _ptr(workspace), workspace.numel(), _stream_ptr(stream)))


def indexer_topk_rows(scores: torch.Tensor, rows: int, ld: int, T: int, q_offset: int, pstride: int,
                      row_len: int, topk: int, cand: Optional[torch.Tensor], n_slots: int, blk: int,
                      out_idx: torch.Tensor, out_score: Optional[torch.Tensor],
                      workspace: torch.Tensor, stream=None):
    _check("indexer_topk_rows",
           lib().indexer_topk_rows(_ptr(scores), rows, ld, T, q_offset, pstride, row_len, topk,
                                   _ptr(cand), n_slots, blk, _ptr(out_idx), _ptr(out_score),
                                   _ptr(workspace), workspace.numel(), _stream_ptr(stream)))


def dsa_meanpool_keys(k: torch.Tensor, block: int, kbar: torch.Tensor, stream=None):
    b, L, d = k.shape
    _check("dsa_meanpool_keys",
           lib().dsa_meanpool_keys(_ptr(k), b, L, d, block, _ptr(kbar), _stream_ptr(stream)))


def misa_workspace_size(args: IndexerArgs, block: int, h: int, topk: int, kprime: int) -> int:
    return int(lib().misa_workspace_size(ctypes.byref(args), block, h, topk, kprime))


def misa_route_score_topk(args: IndexerArgs, block: int, h: int, topk: int, kprime: int,
                          out_idx: torch.Tensor, out_score: Optional[torch.Tensor],
                          out_heads: Optional[torch.Tensor], out_cand: Optional[torch.Tensor],
                          workspace: torch.Tensor, stream=None):
    _check("misa_route_score_topk",
           lib().misa_route_score_topk(ctypes.byref(args), block, h, topk, kprime, _ptr(out_idx),
                                       _ptr(out_score), _ptr(out_heads), _ptr(out_cand),
                                       _ptr(workspace), workspace.numel(), _stream_ptr(stream)))


def hisa_workspace_size(args: IndexerArgs, block: int, m: int, topk: int) -> int:
    return int(lib().hisa_workspace_size(ctypes.byref(args), block, m, topk))


def hisa_block_filter_topk(args: IndexerArgs, block: int, m: int, topk: int, out_idx: torch.Tensor,
                           out_score: Optional[torch.Tensor], out_blocks: Optional[torch.Tensor],
                           workspace: torch.Tensor, stream=None):
    _check("hisa_block_filter_topk",
           lib().hisa_block_filter_topk(ctypes.byref(args), block, m, topk, _ptr(out_idx),
                                        _ptr(out_score), _ptr(out_blocks), _ptr(workspace),
                                        workspace.numel(), _stream_ptr(stream)))


def pooled_cache(args: IndexerArgs, block: int, device=None):
    """Empty pooled-key cache buffers for dsa_pool_keys: (kbar, kbar_scale);
    kbar is bf16 [batch, M, d] or, for an FP8 cache, uint8 codes [batch, M, d]
    with fp32 scales [batch, M]."""
    M = -(-args.L // block)
    fp8 = args.qk_dtype == DSA_FP8_E4M3
    kbar = torch.empty((args.batch, M, args.d), dtype=torch.uint8 if fp8 else torch.bfloat16, device=device)
    scale = torch.empty((args.batch, M), dtype=torch.float32, device=device) if fp8 else None
    return kbar, scale


def dsa_pool_keys(args: IndexerArgs, block: int, m0: int, m1: int, kbar: torch.Tensor,
                  kbar_scale: Optional[torch.Tensor], stream=None):
    _check("dsa_pool_keys", lib().dsa_pool_keys(ctypes.byref(args), block, m0, m1, _ptr(kbar), _ptr(kbar_scale),
                                                _stream_ptr(stream)))


def misa_route_score_topk_pooled(args: IndexerArgs, block: int, h: int, topk: int, kprime: int,
                                 kbar: torch.Tensor, kbar_scale: Optional[torch.Tensor], out_idx: torch.Tensor,
                                 out_score: Optional[torch.Tensor], out_heads: Optional[torch.Tensor],
                                 out_cand: Optional[torch.Tensor], workspace: torch.Tensor, stream=None):
    _check("misa_route_score_topk_pooled",
           lib().misa_route_score_topk_pooled(ctypes.byref(args), block, h, topk, kprime, _ptr(kbar),
                                              _ptr(kbar_scale), _ptr(out_idx), _ptr(out_score), _ptr(out_heads),
                                              _ptr(out_cand), _ptr(workspace), workspace.numel(),
                                              _stream_ptr(stream)))


def hisa_block_filter_topk_pooled(args: IndexerArgs, block: int, m: int, topk: int, kbar: torch.Tensor,
                                  kbar_scale: Optional[torch.Tensor], out_idx: torch.Tensor,
                                  out_score: Optional[torch.Tensor], out_blocks: Optional[torch.Tensor],
                                  workspace: torch.Tensor, stream=None):
    _check("hisa_block_filter_topk_pooled",
           lib().hisa_block_filter_topk_pooled(ctypes.byref(args), block, m, topk, _ptr(kbar), _ptr(kbar_scale),
                                               _ptr(out_idx), _ptr(out_score), _ptr(out_blocks), _ptr(workspace),
                                               workspace.numel(), _stream_ptr(stream)))


def hisa_refine_workspace_size(args: IndexerArgs, m: int, blk: int) -> int:
    return int(lib().hisa_refine_workspace_size(ctypes.byref(args), m, blk))


def hisa_refine_scores(args: IndexerArgs, blocks: torch.Tensor, m: int, blk: int, out: torch.Tensor, ld: int,
                       workspace: torch.Tensor, stream=None):
    _check("hisa_refine_scores",
           lib().hisa_refine_scores(ctypes.byref(args), _ptr(blocks), m, blk, _ptr(out), ld, _ptr(workspace),
                                    workspace.numel(), _stream_ptr(stream)))


def dosa_workspace_size(args: IndexerArgs, topk: int, n_screen: int) -> int:
    return int(lib().dosa_workspace_size(ctypes.byref(args), topk, n_screen))


def dosa_score_topk(args: IndexerArgs, topk: int, n_screen: int, out_idx: torch.Tensor,
                    out_score: Optional[torch.Tensor], out_live: Optional[torch.Tensor], workspace: torch.Tensor,
                    stream=None):
    _check("dosa_score_topk",
           lib().dosa_score_topk(ctypes.byref(args), topk, n_screen, _ptr(out_idx), _ptr(out_score), _ptr(out_live),
                                 _ptr(workspace), workspace.numel(), _stream_ptr(stream)))


def dsa_profile_begin():
    _check("dsa_profile_begin", lib().dsa_profile_begin())


def dsa_profile_end(max_entries: int = 4096):
    """Launches recorded since dsa_profile_begin: list of (name, ms)."""
    names = ctypes.create_string_buffer(max_entries * 96)
    ms = (ctypes.c_float * max_entries)()
    n = lib().dsa_profile_end(names, len(names), ctypes.cast(ms, ctypes.c_void_p), max_entries)
    if n < 0:
        raise DsaError("dsa_profile_end", -4)
    out, raw = [], names.raw
    pos = 0
    for i in range(n):
        end = raw.index(b"\0", pos)
        out.append((raw[pos:end].decode(), float(ms[i])))
        pos = end + 1
    return out


def _args_array(layers):
    arr = (IndexerArgs * len(layers))()
    for i, a in enumerate(layers):
        arr[i] = a
    return arr


def indexcache_workspace_size(layers, pattern: str, topk: int) -> int:
    return int(lib().indexcache_workspace_size(_args_array(layers), len(layers), pattern.encode(), topk))


def indexcache_score_topk(layers, pattern: str, topk: int, out_idx, out_score, workspace: torch.Tensor,
                          stream=None):
    """layers: list of IndexerArgs (an S layer's entry needs only batch and T);
    out_idx: list of [batch, T, topk] int32 tensors (an S layer may pass its F
    layer's tensor to share it); out_score: None or a list (entries may be None)."""
    n = len(layers)
    pi = (ctypes.c_void_p * n)(*[t.data_ptr() for t in out_idx])
    ps = None
    if out_score is not None:
        ps = (ctypes.c_void_p * n)(*[t.data_ptr() if t is not None else None for t in out_score])
    _check("indexcache_score_topk",
           lib().indexcache_score_topk(_args_array(layers), n, pattern.encode(), topk, pi, ps,
                                       _ptr(workspace), workspace.numel(), _stream_ptr(stream)))


def dsa_device_status(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().dsa_device_status(_ptr(workspace), _stream_ptr(stream)))


def dsa_selftest_wait_timeout(workspace: torch.Tensor, stream=None):
    _check("dsa_selftest_wait_timeout",
           lib().dsa_selftest_wait_timeout(_ptr(workspace), workspace.numel(), _stream_ptr(stream)))


# ------------------------------------------------------------------ convenience
class Indexer:
    """Holds device inputs of one problem and a workspace; the three methods
    call the C-ABI entry points and return device tensors."""

    def __init__(self, q, k, w, q_offset, q_scale=None, k_scale=None):
        self.q, self.k, self.w, self.q_scale, self.k_scale = q, k, w, q_scale, k_scale
        self.args = make_args(q, k, w, q_offset, q_scale, k_scale)
        self._ws = None

    def workspace(self, nbytes: int) -> torch.Tensor:
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = alloc_workspace(nbytes, self.q.device)
        return self._ws

    def _out(self, topk, with_score):
        a = self.args
        idx = torch.empty((a.batch, a.T, topk), dtype=torch.int32, device=self.q.device)
        sc = torch.empty((a.batch, a.T, topk), dtype=torch.float32, device=self.q.device) if with_score else None
        return idx, sc

    def dense(self, topk: int, with_score: bool = False, stream=None):
        idx, sc = self._out(topk, with_score)
        ws = self.workspace(indexer_workspace_size(self.args, topk))
        indexer_score_topk(self.args, topk, idx, sc, ws, stream)
        return idx, sc

    def misa(self, block: int, h: int, topk: int, kprime: int = 0, with_score: bool = False,
             with_heads: bool = False, with_cand: bool = False, stream=None):
        a = self.args
        idx, sc = self._out(topk, with_score)
        dev = self.q.device
        heads = torch.empty((a.batch, a.T, h), dtype=torch.int32, device=dev) if with_heads else None
        cand = torch.empty((a.batch, a.T, kprime), dtype=torch.int32, device=dev) if (with_cand and kprime) else None
        ws = self.workspace(misa_workspace_size(a, block, h, topk, kprime))
        misa_route_score_topk(a, block, h, topk, kprime, idx, sc, heads, cand, ws, stream)
        return idx, sc, heads, cand

    def hisa(self, block: int, m: int, topk: int, with_score: bool = False, with_blocks: bool = False,
             stream=None):
        a = self.args
        idx, sc = self._out(topk, with_score)
        blocks = torch.empty((a.batch, a.T, m), dtype=torch.int32, device=self.q.device) if with_blocks else None
        ws = self.workspace(hisa_workspace_size(a, block, m, topk))
        hisa_block_filter_topk(a, block, m, topk, idx, sc, blocks, ws, stream)
        return idx, sc, blocks

    def device_status(self, stream=None) -> int:
        return dsa_device_status(self._ws, stream) if self._ws is not None else 0


def to_device(inp, device="cuda"):
    """Copy an IndexerInputs (host numpy buffers) to device tensors:
    returns (q, k, w, q_scale, k_scale)."""
    import numpy as np

    def t(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device).view(dt) if a is not None else None

    if inp.dtype == "bf16":
        q = t(inp.q.view(np.int16), torch.bfloat16)
        k = t(inp.k.view(np.int16), torch.bfloat16)
    else:
        q = t(inp.q, torch.uint8)
        k = t(inp.k, torch.uint8)
    w = t(inp.w, torch.float32)
    return q, k, w, t(inp.q_scale, torch.float32), t(inp.k_scale, torch.float32)
