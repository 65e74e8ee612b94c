"""Thin ctypes binding of libmsa (argument marshalling only).

Every function takes CUDA torch tensors in the C-ABI layouts (see
``include/msa.h``), passes their device pointers and the current CUDA stream
to the library, and raises ``MsaError`` on a non-zero status.  Nothing here
computes any part of the method: when the shared library is missing the
import-time loader raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmsa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "msa.h")

OP_INDEX_SCORES, OP_BLOCK_TOPK, OP_SPARSE_PREFILL, OP_SPARSE_DECODE, OP_FORWARD, \
    OP_DENSE_PREFILL, OP_DENSE_DECODE, OP_FORWARD_ALIGNMENT, OP_FORWARD_PREFILL_PAGED = range(9)

STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_SHAPE", 2: "MSA_ERR_NULL_PTR", 3: "MSA_ERR_MISALIGNED",
          4: "MSA_ERR_WORKSPACE_TOO_SMALL", 5: "MSA_ERR_UNSUPPORTED", 6: "MSA_ERR_CUDA",
          7: "MSA_ERR_DEVICE_TIMEOUT"}


class MsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "batch", "seq_q", "seq_kv", "q_offset", "n_q_heads", "n_kv_heads",
        "head_dim", "index_dim", "block", "topk")]

    @classmethod
    def of(cls, spec) -> "Shape":
        """From any object with the same attribute names (e.g. a WorkloadSpec)."""
        return cls(*[int(getattr(spec, n)) for n, _ in cls._fields_])

    @property
    def nb(self) -> int:
        return (self.seq_kv + self.block - 1) // self.block


_vp = ctypes.c_void_p
_SIGS = {
    "msa_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "msa_workspace_size": ([ctypes.POINTER(Shape), ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)],
                           ctypes.c_int),
    "msa_index_scores": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp], ctypes.c_int),
    "msa_block_topk": ([ctypes.POINTER(Shape), _vp, _vp, _vp], ctypes.c_int),
    "msa_sparse_attn_prefill": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 ctypes.c_size_t, _vp], ctypes.c_int),
    "msa_sparse_attn_decode": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                ctypes.c_size_t, _vp], ctypes.c_int),
    "msa_sparse_attn_decode_static": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp],
                                      ctypes.c_int),
    "msa_forward": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                     ctypes.c_size_t, _vp], ctypes.c_int),
    "msa_forward_alignment": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _vp, _vp, ctypes.c_size_t, _vp], ctypes.c_int),
    "msa_forward_prefill_paged": ([ctypes.POINTER(Shape), ctypes.c_int, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp], ctypes.c_int),
    "msa_forward_decode_paged": ([ctypes.POINTER(Shape), ctypes.c_int, _vp, _vp, _vp, _vp, _vp,
                                  _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp],
                                 ctypes.c_int),
    "msa_forward_decode_ragged": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _vp, ctypes.c_size_t, _vp], ctypes.c_int),
    "msa_dense_attn_prefill": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp,
                                ctypes.c_size_t, _vp], ctypes.c_int),
    "msa_dense_attn_decode": ([ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp,
                               ctypes.c_size_t, _vp], ctypes.c_int),
    "msa_device_status": ([ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
    "msa_set_wait_limit_ns": ([ctypes.c_uint64], ctypes.c_int),
    "msa_profile_enable": ([ctypes.c_int], ctypes.c_int),
    "msa_profile_read": ([ctypes.c_int, ctypes.POINTER(ctypes.c_char_p),
                          ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)],
                         ctypes.c_int),
}

_lib = None


def lib():
    """The loaded libmsa (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmsa is not built ({LIB_PATH} missing); run "
                              "python -m block_sparse_gqa_05_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def header_functions() -> list:
    """Names of the functions ``include/msa.h`` declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_]+)\s*\(", src)))


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmsa takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libmsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _sizes(shape: Shape, pages: int = 0) -> dict:
    """dtype and element count of every array argument, from the C-ABI layouts."""
    B, T, N, H, G = shape.batch, shape.seq_q, shape.seq_kv, shape.n_q_heads, shape.n_kv_heads
    d, di, k, nb = shape.head_dim, shape.index_dim, shape.topk, shape.nb
    bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    return {"q": (bf16, B * T * H * d), "o": (bf16, B * T * H * d),
            "k": (bf16, B * G * N * d), "v": (bf16, B * G * N * d),
            "q_idx": (bf16, B * T * G * di), "k_idx": (bf16, B * N * di),
            "pooled": (f32, B * T * G * nb), "sel": (i32, B * T * G * k),
            "lse": (f32, B * T * H), "kl": (f32, B * T * G), "seq_lens": (i32, B),
            "page_table": (i32, B * nb), "k_pages": (bf16, pages * G * 128 * d),
            "v_pages": (bf16, pages * G * 128 * d), "kidx_pages": (bf16, pages * 128 * di)}


def _args(shape: Shape, pages: int = 0, **tensors) -> dict:
    """Device pointers of the named tensors after checking each one's dtype and
    that it holds at least the elements its layout needs (None stays None)."""
    need = _sizes(shape, pages)
    out = {}
    for name, t in tensors.items():
        if t is not None:
            dtype, n = need[name]
            if t.dtype != dtype:
                raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
            if t.numel() < n:
                raise ValueError(f"{name}: {t.numel()} elements, the shape needs {n}")
        out[name] = _ptr(t)
    return out


def _ws(ws):
    """(pointer, size in bytes) of a workspace tensor."""
    return _ptr(ws), ws.numel() * ws.element_size()


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != 0:
        raise MsaError(status, what)


def workspace_size(shape: Shape, op: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().msa_workspace_size(ctypes.byref(shape), op, ctypes.byref(n)), "msa_workspace_size")
    return int(n.value)


def alloc_workspace(shape: Shape, op: int, device=None) -> torch.Tensor:
    n = workspace_size(shape, op)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def index_scores(shape: Shape, q_idx, k_idx, pooled=None, stream=None):
    if pooled is None:
        pooled = torch.empty((shape.batch, shape.seq_q, shape.n_kv_heads, shape.nb),
                             dtype=torch.float32, device=q_idx.device)
    a = _args(shape, q_idx=q_idx, k_idx=k_idx, pooled=pooled)
    _check(lib().msa_index_scores(ctypes.byref(shape), a["q_idx"], a["k_idx"], a["pooled"],
                                  _stream(stream)), "msa_index_scores")
    return pooled


def block_topk(shape: Shape, pooled, sel=None, stream=None):
    if sel is None:
        sel = torch.empty((shape.batch, shape.seq_q, shape.n_kv_heads, shape.topk),
                          dtype=torch.int32, device=pooled.device)
    a = _args(shape, pooled=pooled, sel=sel)
    _check(lib().msa_block_topk(ctypes.byref(shape), a["pooled"], a["sel"], _stream(stream)),
           "msa_block_topk")
    return sel


def _attn_out(shape, q, o, lse, want_lse):
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((shape.batch, shape.seq_q, shape.n_q_heads), dtype=torch.float32,
                          device=q.device)
    return o, lse


def sparse_attn_prefill(shape: Shape, q, k, v, sel, o=None, lse=None, ws=None, want_lse=True,
                        stream=None):
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    ws = alloc_workspace(shape, OP_SPARSE_PREFILL, q.device) if ws is None else ws
    a = _args(shape, q=q, k=k, v=v, sel=sel, o=o, lse=lse)
    _check(lib().msa_sparse_attn_prefill(ctypes.byref(shape), a["q"], a["k"], a["v"], a["sel"],
                                         a["o"], a["lse"], *_ws(ws), _stream(stream)),
           "msa_sparse_attn_prefill")
    return o, lse


def sparse_attn_decode(shape: Shape, q, k, v, sel, o=None, lse=None, ws=None, want_lse=True,
                       stream=None):
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    ws = alloc_workspace(shape, OP_SPARSE_DECODE, q.device) if ws is None else ws
    a = _args(shape, q=q, k=k, v=v, sel=sel, o=o, lse=lse)
    _check(lib().msa_sparse_attn_decode(ctypes.byref(shape), a["q"], a["k"], a["v"], a["sel"],
                                        a["o"], a["lse"], *_ws(ws), _stream(stream)),
           "msa_sparse_attn_decode")
    return o, lse


def sparse_attn_decode_static(shape: Shape, q, k, v, sel, o=None, lse=None, want_lse=True,
                              stream=None):
    """msa_sparse_attn_decode_static: decode attention whose scratch is the
    library's static device array, so nothing is allocated for it.  Calls
    that may overlap on the GPU share that array and must be serialised."""
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    a = _args(shape, q=q, k=k, v=v, sel=sel, o=o, lse=lse)
    _check(lib().msa_sparse_attn_decode_static(ctypes.byref(shape), a["q"], a["k"], a["v"],
                                               a["sel"], a["o"], a["lse"], _stream(stream)),
           "msa_sparse_attn_decode_static")
    return o, lse


def forward(shape: Shape, q, k, v, q_idx, k_idx, o=None, lse=None, sel=None, ws=None,
            want_lse=True, want_sel=True, stream=None):
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    if sel is None and want_sel:
        sel = torch.empty((shape.batch, shape.seq_q, shape.n_kv_heads, shape.topk),
                          dtype=torch.int32, device=q.device)
    ws = alloc_workspace(shape, OP_FORWARD, q.device) if ws is None else ws
    a = _args(shape, q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx, o=o, lse=lse, sel=sel)
    _check(lib().msa_forward(ctypes.byref(shape), a["q"], a["k"], a["v"], a["q_idx"], a["k_idx"],
                             a["o"], a["lse"], a["sel"], *_ws(ws), _stream(stream)),
           "msa_forward")
    return o, lse, sel


def forward_alignment(shape: Shape, q, k, v, q_idx, k_idx, o=None, lse=None, sel=None,
                      kl=None, ws=None, want_lse=True, want_sel=True, stream=None):
    """msa_forward_alignment: the whole layer plus kl [B, T, G] float32, the
    divergence of the index branch's block distribution from the main
    branch's (forward only).  Returns (o, lse, sel, kl)."""
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    if sel is None and want_sel:
        sel = torch.empty((shape.batch, shape.seq_q, shape.n_kv_heads, shape.topk),
                          dtype=torch.int32, device=q.device)
    if kl is None:
        kl = torch.empty((shape.batch, shape.seq_q, shape.n_kv_heads), dtype=torch.float32,
                         device=q.device)
    ws = alloc_workspace(shape, OP_FORWARD_ALIGNMENT, q.device) if ws is None else ws
    a = _args(shape, q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx, o=o, lse=lse, sel=sel, kl=kl)
    _check(lib().msa_forward_alignment(ctypes.byref(shape), a["q"], a["k"], a["v"], a["q_idx"],
                                       a["k_idx"], a["o"], a["lse"], a["sel"], a["kl"],
                                       *_ws(ws), _stream(stream)),
           "msa_forward_alignment")
    return o, lse, sel, kl


def forward_decode_ragged(shape: Shape, q, k, v, q_idx, k_idx, seq_lens, o=None, lse=None,
                          sel=None, ws=None, want_lse=True, want_sel=True, stream=None):
    """msa_forward_decode_ragged: one decode step over caches of different
    lengths.  seq_lens: int32 CUDA tensor [B], each in [1, shape.seq_kv]
    (shape.seq_kv is the cache capacity)."""
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    if sel is None and want_sel:
        sel = torch.empty((shape.batch, 1, shape.n_kv_heads, shape.topk), dtype=torch.int32,
                          device=q.device)
    ws = alloc_workspace(shape, OP_FORWARD, q.device) if ws is None else ws
    a = _args(shape, seq_lens=seq_lens, q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx, o=o, lse=lse,
              sel=sel)
    _check(lib().msa_forward_decode_ragged(ctypes.byref(shape), a["seq_lens"], a["q"], a["k"],
                                           a["v"], a["q_idx"], a["k_idx"], a["o"], a["lse"],
                                           a["sel"], *_ws(ws), _stream(stream)),
           "msa_forward_decode_ragged")
    return o, lse, sel


def forward_decode_paged(shape: Shape, q, k_pages, v_pages, q_idx, kidx_pages, seq_lens,
                         page_table, o=None, lse=None, sel=None, ws=None, want_lse=True,
                         want_sel=True, stream=None):
    """msa_forward_decode_paged: one decode step over paged caches.
    k_pages / v_pages [P, G, 128, d] bf16, kidx_pages [P, 128, d_i] bf16,
    seq_lens int32 [B], page_table int32 [B, ceil(shape.seq_kv / 128)]."""
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    if sel is None and want_sel:
        sel = torch.empty((shape.batch, 1, shape.n_kv_heads, shape.topk), dtype=torch.int32,
                          device=q.device)
    ws = alloc_workspace(shape, OP_FORWARD, q.device) if ws is None else ws
    P = int(k_pages.shape[0])
    a = _args(shape, P, seq_lens=seq_lens, page_table=page_table, q=q, k_pages=k_pages,
              v_pages=v_pages, q_idx=q_idx, kidx_pages=kidx_pages, o=o, lse=lse, sel=sel)
    _check(lib().msa_forward_decode_paged(ctypes.byref(shape), P, a["seq_lens"], a["page_table"],
                                          a["q"], a["k_pages"], a["v_pages"], a["q_idx"],
                                          a["kidx_pages"], a["o"], a["lse"], a["sel"],
                                          *_ws(ws), _stream(stream)),
           "msa_forward_decode_paged")
    return o, lse, sel


def forward_prefill_paged(shape: Shape, q, k_pages, v_pages, q_idx, kidx_pages, page_table,
                          o=None, lse=None, sel=None, ws=None, want_lse=True, want_sel=True,
                          stream=None):
    """msa_forward_prefill_paged: one chunk of query rows (positions
    shape.q_offset .. + seq_q - 1) over paged caches of seq_kv keys.
    k_pages / v_pages [P, G, 128, d] bf16, kidx_pages [P, 128, d_i] bf16,
    page_table int32 [B, ceil(shape.seq_kv / 128)]."""
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    if sel is None and want_sel:
        sel = torch.empty((shape.batch, shape.seq_q, shape.n_kv_heads, shape.topk),
                          dtype=torch.int32, device=q.device)
    ws = alloc_workspace(shape, OP_FORWARD_PREFILL_PAGED, q.device) if ws is None else ws
    P = int(k_pages.shape[0])
    a = _args(shape, P, page_table=page_table, q=q, k_pages=k_pages, v_pages=v_pages,
              q_idx=q_idx, kidx_pages=kidx_pages, o=o, lse=lse, sel=sel)
    _check(lib().msa_forward_prefill_paged(ctypes.byref(shape), P, a["page_table"], a["q"],
                                           a["k_pages"], a["v_pages"], a["q_idx"],
                                           a["kidx_pages"], a["o"], a["lse"], a["sel"],
                                           *_ws(ws), _stream(stream)),
           "msa_forward_prefill_paged")
    return o, lse, sel


def dense_attn_prefill(shape: Shape, q, k, v, o=None, lse=None, want_lse=True, stream=None):
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    a = _args(shape, q=q, k=k, v=v, o=o, lse=lse)
    _check(lib().msa_dense_attn_prefill(ctypes.byref(shape), a["q"], a["k"], a["v"], a["o"],
                                        a["lse"], None, 0, _stream(stream)),
           "msa_dense_attn_prefill")
    return o, lse


def dense_attn_decode(shape: Shape, q, k, v, o=None, lse=None, ws=None, want_lse=True,
                      stream=None):
    o, lse = _attn_out(shape, q, o, lse, want_lse)
    ws = alloc_workspace(shape, OP_DENSE_DECODE, q.device) if ws is None else ws
    a = _args(shape, q=q, k=k, v=v, o=o, lse=lse)
    _check(lib().msa_dense_attn_decode(ctypes.byref(shape), a["q"], a["k"], a["v"], a["o"],
                                       a["lse"], *_ws(ws), _stream(stream)),
           "msa_dense_attn_decode")
    return o, lse


def profile_enable(on: bool = True):
    """Start (clearing the table) or stop per-kernel CUDA-event timing."""
    _check(lib().msa_profile_enable(1 if on else 0), "msa_profile_enable")


def profile_read() -> dict:
    """{kernel name: (total ms, launches)} of the recorded launches (waits for them)."""
    out = {}
    i = 0
    while True:
        name = ctypes.c_char_p()
        ms = ctypes.c_double()
        n = ctypes.c_longlong()
        st = lib().msa_profile_read(i, ctypes.byref(name), ctypes.byref(ms), ctypes.byref(n))
        if st == 1:
            return out
        _check(st, "msa_profile_read")
        out[name.value.decode()] = (ms.value, n.value)
        i += 1


def device_status() -> int:
    """Raw device error word (bit 0: a bounded wait expired; bit 1: a ragged-decode
    cache length was out of range; bit 2: a page-table entry was out of range;
    bit 3: a prefill selection entry lay past its query's block); clears it."""
    f = ctypes.c_uint32(0)
    st = lib().msa_device_status(ctypes.byref(f))
    if st not in (0, 7):
        raise MsaError(st, "msa_device_status")
    return int(f.value)


def set_wait_limit_ns(ns: int) -> None:
    """Bound of the kernels' waits on the current device, in nanoseconds
    (diagnostics; default 2 s; 0 makes every wait that is not already complete
    expire at once)."""
    _check(lib().msa_set_wait_limit_ns(int(ns)), "msa_set_wait_limit_ns")
