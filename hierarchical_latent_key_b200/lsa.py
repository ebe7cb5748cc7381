"""Thin Python binding of the C ABI in ``include/lsa.h`` (``liblsa.so``).

The ``lsa_*`` functions keep the C names and only marshal arguments: torch
tensors become device pointers and sizes, the current torch stream becomes the
``cudaStream_t``.  Every step of the computation runs in the CUDA library; if the
library cannot be loaded, importing this module raises.  A few helpers below
(``build_tree``, ``select``, ``sparse_attn``, ``sparse_attn_bwd``) allocate
outputs and workspace with torch and then call the same entry points.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

from . import build_ext

LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_SHAPE, LSA_ERR_CUDA, LSA_ERR_TIMEOUT, LSA_ERR_NONFINITE, LSA_ERR_WORKSPACE = range(7)
LSA_F32, LSA_BF16 = 0, 1
MAX_LEVELS = 8
_DTYPE = {torch.float32: LSA_F32, torch.bfloat16: LSA_BF16}


class LsaError(RuntimeError):
    def __init__(self, code: int, what: str, detail: str = ""):
        self.code = code
        super().__init__(f"{what}: {lsa_strerror(code)} ({code}){': ' + detail if detail else ''}")


class lsa_tree_desc(ctypes.Structure):
    _fields_ = [
        ("n_heads", ctypes.c_int32), ("r", ctypes.c_int32), ("levels", ctypes.c_int32),
        ("leaf_size", ctypes.c_int32), ("n_tree", ctypes.c_int64),
        ("branching", ctypes.c_int32 * MAX_LEVELS), ("nodes", ctypes.c_int64 * MAX_LEVELS),
        ("off_centroids", ctypes.c_uint64 * MAX_LEVELS), ("off_min_pos", ctypes.c_uint64 * MAX_LEVELS),
        ("off_leaf_index", ctypes.c_uint64), ("bytes", ctypes.c_uint64),
    ]


def _load():
    path = os.environ.get("LSA_LIBRARY") or build_ext.LIB
    if not os.path.exists(path):
        raise ImportError(f"CUDA library {path} is missing; build it with "
                          f"`python -m hierarchical_latent_key_b200.build_ext`")
    lib = ctypes.CDLL(path)
    P, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    D = ctypes.POINTER(lsa_tree_desc)
    f32 = ctypes.c_float
    sig = {
        "lsa_version": (ctypes.c_int, []),
        "lsa_strerror": (ctypes.c_char_p, [ctypes.c_int]),
        "lsa_last_error": (ctypes.c_char_p, []),
        "lsa_tree_describe": (ctypes.c_int, [i32, i32, P, i32, i32, D]),
        "lsa_build_workspace_bytes": (ctypes.c_int, [D, i32, ctypes.POINTER(sz)]),
        "lsa_build_tree": (ctypes.c_int, [D, P, P, i64, i32, i32, P, i32, u64, P, sz, P, P, P]),
        "lsa_build_tree_pooled": (ctypes.c_int, [D, P, P, i64, i32, i32, P, i32, i32, u64, P, sz, P, P, P]),
        "lsa_tree_append_workspace_bytes": (ctypes.c_int, [D, i32, ctypes.POINTER(ctypes.c_size_t)]),
        "lsa_tree_append": (ctypes.c_int, [D, P, D, P, P, i64, i32, i32, P, i32, u64, P, sz, P, P, P]),
        "lsa_select": (ctypes.c_int, [D, P, P, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P]),
        "lsa_select_batched_workspace_bytes": (ctypes.c_int, [D, i32, P, ctypes.POINTER(sz)]),
        "lsa_select_batched": (ctypes.c_int, [D, P, P, i32, i32, i32, i32, P, P, P, P, P, P, P, P, sz, P, P]),
        "lsa_tree_attn_workspace_bytes": (ctypes.c_int, [D, i32, i32, i32, i32, i32, ctypes.POINTER(sz)]),
        "lsa_tree_attn": (ctypes.c_int, [D, P, P, i32, i32, P, P, i64, i32, i32, P, i32, P, i32, f32, P, P, P, sz,
                                         P, P]),
        "lsa_attn_workspace_bytes": (ctypes.c_int, [i32, i32, i32, i32, i32, i64, ctypes.POINTER(sz)]),
        "lsa_sparse_attn": (ctypes.c_int, [P, i32, i32, P, P, i32, i64, i32, i32, P, i32, P, i32, i64, i64,
                                           f32, P, P, P, sz, P, P]),
        "lsa_sparse_attn_bwd": (ctypes.c_int, [P, i32, i32, P, P, i32, i64, i32, i32, P, P, P, P, i32, P, i32,
                                               i64, i64, f32, P, P, P, P, P]),
        "lsa_sparse_attn_noalloc": (ctypes.c_int, [P, i32, i32, P, P, i32, i64, i32, i32, P, i32, P, i32, i64,
                                                   i64, f32, P, P, P, P]),
        "lsa_select_flat": (ctypes.c_int, [D, P, P, i32, i32, i32, i32, P, i32, P, P, P, P, P, P]),
        "lsa_tree_attn_sw_workspace_bytes": (ctypes.c_int, [D, i32, i32, i32, i32, i32, i32, i32,
                                                            ctypes.POINTER(sz)]),
        "lsa_tree_attn_sw": (ctypes.c_int, [D, P, P, i32, i32, P, P, i64, i32, i32, P, i32, P, i32, i32, f32, P, P,
                                            P, sz, P, P]),
        "lsa_sparse_attn_sw_workspace_bytes": (ctypes.c_int, [i32, i32, i32, i32, i32, i64, i32, i32,
                                                              ctypes.POINTER(sz)]),
        "lsa_sparse_attn_sw": (ctypes.c_int, [P, i32, i32, P, P, i32, i64, i32, i32, P, i32, P, i32, i32, i64, i64,
                                              f32, P, P, P, sz, P, P]),
        "lsa_sparse_attn_sw_bwd": (ctypes.c_int, [P, i32, i32, P, P, i32, i64, i32, i32, P, P, P, P, i32, P, i32,
                                                  i32, i64, i64, f32, P, P, P, P, sz, P, P]),
        "lsa_kv_append": (ctypes.c_int, [P, P, i32, i64, i32, i32, i64, P, P, P]),
        "lsa_project_keys": (ctypes.c_int, [P, i32, i64, i32, i32, P, i32, i64, P, P, P]),
        "lsa_balanced_assign_workspace_bytes": (ctypes.c_int, [i64, i64, i32, ctypes.POINTER(sz)]),
        "lsa_decode_step_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(lsa_tree_desc), i32, i32,
                                                           ctypes.POINTER(i32), i64, ctypes.POINTER(sz)]),
        "lsa_decode_step": (ctypes.c_int, [ctypes.POINTER(lsa_tree_desc), P, P, ctypes.POINTER(i32), P, P, i64,
                                           i32, i32, P, i32, P, P, i64, i64, ctypes.c_float, P, P, P, P, sz,
                                           P, P]),
        "lsa_balanced_assign": (ctypes.c_int, [P, P, i64, i64, i32, i32, i32, P, P, sz, P, P]),
        "lsa_tree_attn_bwd_workspace_bytes": (ctypes.c_int, [D, i32, i32, i32, i32, i32, ctypes.POINTER(sz)]),
        "lsa_tree_attn_bwd": (ctypes.c_int, [D, P, P, i32, i32, P, P, i64, i32, i32, P, P, P, P, i32, P, i32, f32,
                                             P, P, P, P, sz, P, P]),
        "lsa_status_clear": (ctypes.c_int, [P, P]),
        "lsa_status_check": (ctypes.c_int, [P, P, ctypes.POINTER(i32)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
LIBRARY_PATH = _lib._name


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the LSA library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, ref: torch.Tensor | None = None):
    if stream is None:
        dev = ref.device if ref is not None and ref.is_cuda else torch.device("cuda", torch.cuda.current_device())
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    try:
        return _DTYPE[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _raise(rc: int, what: str):
    if rc != LSA_OK:
        raise LsaError(rc, what, _lib.lsa_last_error().decode())


# --- C ABI, same names ------------------------------------------------------------

def lsa_version() -> int:
    return int(_lib.lsa_version())


def lsa_strerror(code: int) -> str:
    return _lib.lsa_strerror(int(code)).decode()


def lsa_tree_describe(n_heads: int, r: int, branching, leaf_size: int) -> lsa_tree_desc:
    br = (ctypes.c_int32 * max(MAX_LEVELS, len(branching)))(*branching)
    out = lsa_tree_desc()
    _raise(_lib.lsa_tree_describe(n_heads, r, ctypes.cast(br, ctypes.c_void_p), len(branching), leaf_size,
                                  ctypes.byref(out)), "lsa_tree_describe")
    return out


def lsa_build_workspace_bytes(desc: lsa_tree_desc, d: int) -> int:
    n = ctypes.c_size_t()
    _raise(_lib.lsa_build_workspace_bytes(ctypes.byref(desc), d, ctypes.byref(n)), "lsa_build_workspace_bytes")
    return int(n.value)


def lsa_build_tree(desc, tree_mem, K, W, iters, seed, workspace, trace=None, status=None, stream=None):
    """K: [n_heads, n_cap, d]; W: [n_heads, d, r]; tree_mem/workspace: uint8 device tensors."""
    _raise(_lib.lsa_build_tree(ctypes.byref(desc), _ptr(tree_mem), _ptr(K), K.shape[1], K.shape[2], _dtype(K),
                               _ptr(W), iters, seed & ((1 << 64) - 1), _ptr(workspace), workspace.numel(),
                               _ptr(trace), _ptr(status), _stream(stream, K)), "lsa_build_tree")


def lsa_build_tree_pooled(desc, tree_mem, K, W, pool, iters, seed, workspace, trace=None, status=None, stream=None):
    """lsa_build_tree over blocks of `pool` consecutive keys (trace by block)."""
    _raise(_lib.lsa_build_tree_pooled(ctypes.byref(desc), _ptr(tree_mem), _ptr(K), K.shape[1], K.shape[2],
                                      _dtype(K), _ptr(W), pool, iters, seed & ((1 << 64) - 1), _ptr(workspace),
                                      workspace.numel(), _ptr(trace), _ptr(status), _stream(stream, K)),
           "lsa_build_tree_pooled")


def lsa_tree_append_workspace_bytes(desc, d):
    n = ctypes.c_size_t()
    _raise(_lib.lsa_tree_append_workspace_bytes(ctypes.byref(desc), d, ctypes.byref(n)),
           "lsa_tree_append_workspace_bytes")
    return int(n.value)


def lsa_tree_append(desc, tree_mem, grown, grown_mem, K, W, iters, seed, workspace, trace=None, status=None,
                    stream=None):
    """Attach a subtree over keys [desc.n_tree, grown.n_tree) of K as top node desc.branching[0]."""
    _raise(_lib.lsa_tree_append(ctypes.byref(desc), _ptr(tree_mem), ctypes.byref(grown), _ptr(grown_mem), _ptr(K),
                                K.shape[1], K.shape[2], _dtype(K), _ptr(W), iters, seed & ((1 << 64) - 1),
                                _ptr(workspace), workspace.numel(), _ptr(trace), _ptr(status), _stream(stream, K)),
           "lsa_tree_append")


def lsa_select(desc, tree_mem, Q, W, beam, q_pos, idx_out, leaves_out=None, qlat_out=None, beam_out=None,
               status=None, stream=None):
    """Q: [T, Hq, d]; beam: host sequence of ints; q_pos: int32 [T] or None."""
    bm = (ctypes.c_int32 * max(MAX_LEVELS, len(beam)))(*beam)
    T, Hq, d = Q.shape
    _raise(_lib.lsa_select(ctypes.byref(desc), _ptr(tree_mem), _ptr(Q), T, Hq, d, _dtype(Q), _ptr(W),
                           ctypes.cast(bm, ctypes.c_void_p), _ptr(q_pos), _ptr(idx_out), _ptr(leaves_out),
                           _ptr(qlat_out), _ptr(beam_out), _ptr(status), _stream(stream, Q)), "lsa_select")


def lsa_select_batched_workspace_bytes(desc, T, beam) -> int:
    bm = (ctypes.c_int32 * max(MAX_LEVELS, len(beam)))(*beam)
    n = ctypes.c_size_t()
    _raise(_lib.lsa_select_batched_workspace_bytes(ctypes.byref(desc), T, ctypes.cast(bm, ctypes.c_void_p),
                                                   ctypes.byref(n)), "lsa_select_batched_workspace_bytes")
    return int(n.value)


def lsa_select_batched(desc, tree_mem, Q, W, beam, q_pos, idx_out, leaves_out=None, qlat_out=None, beam_out=None,
                       workspace=None, status=None, stream=None):
    """As lsa_select, scheduled for large batches; workspace: device bytes of
    lsa_select_batched_workspace_bytes(desc, T, beam)."""
    bm = (ctypes.c_int32 * max(MAX_LEVELS, len(beam)))(*beam)
    T, Hq, d = Q.shape
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _raise(_lib.lsa_select_batched(ctypes.byref(desc), _ptr(tree_mem), _ptr(Q), T, Hq, d, _dtype(Q), _ptr(W),
                                   ctypes.cast(bm, ctypes.c_void_p), _ptr(q_pos), _ptr(idx_out), _ptr(leaves_out),
                                   _ptr(qlat_out), _ptr(beam_out), _ptr(workspace), ws_n, _ptr(status),
                                   _stream(stream, Q)), "lsa_select_batched")


def lsa_tree_attn_workspace_bytes(desc, T, Hq, d, dtype, n_leaves) -> int:
    n = ctypes.c_size_t()
    _raise(_lib.lsa_tree_attn_workspace_bytes(ctypes.byref(desc), T, Hq, d, _DTYPE[dtype], n_leaves,
                                              ctypes.byref(n)), "lsa_tree_attn_workspace_bytes")
    return int(n.value)


def lsa_tree_attn(desc, tree_mem, Q, K, V, leaves, q_pos, causal, scale, O, LSE, workspace, status=None,
                  stream=None):
    """leaves: int32 [n_heads, T, n_leaves] (kept leaf ids, -1 = none)."""
    T, Hq, d = Q.shape
    ws_n = workspace.numel() * workspace.element_size()
    _raise(_lib.lsa_tree_attn(ctypes.byref(desc), _ptr(tree_mem), _ptr(Q), T, Hq, _ptr(K), _ptr(V), K.shape[1], d,
                              _dtype(Q), _ptr(leaves), leaves.shape[-1], _ptr(q_pos), int(bool(causal)),
                              float(scale), _ptr(O), _ptr(LSE), _ptr(workspace), ws_n, _ptr(status),
                              _stream(stream, Q)), "lsa_tree_attn")


def lsa_attn_workspace_bytes(T, Hq, n_heads, d, K_sel, tail_len) -> int:
    n = ctypes.c_size_t()
    _raise(_lib.lsa_attn_workspace_bytes(T, Hq, n_heads, d, K_sel, tail_len, ctypes.byref(n)),
           "lsa_attn_workspace_bytes")
    return int(n.value)


def lsa_sparse_attn(Q, K, V, idx, q_pos, causal, tail_begin, tail_end, scale, O, LSE, workspace=None,
                    status=None, stream=None):
    T, Hq, d = Q.shape
    K_sel = 0 if idx is None else idx.shape[-1]
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _raise(_lib.lsa_sparse_attn(_ptr(Q), T, Hq, _ptr(K), _ptr(V), K.shape[0], K.shape[1], d, _dtype(Q), _ptr(idx),
                                K_sel, _ptr(q_pos), int(bool(causal)), tail_begin, tail_end, float(scale), _ptr(O),
                                _ptr(LSE), _ptr(workspace), ws_n, _ptr(status), _stream(stream, Q)),
           "lsa_sparse_attn")


def lsa_sparse_attn_noalloc(Q, K, V, idx, q_pos, causal, tail_begin, tail_end, scale, O, LSE, status=None,
                            stream=None):
    """lsa_sparse_attn without a workspace argument (split partials in the library's built-in array)."""
    T, Hq, d = Q.shape
    K_sel = 0 if idx is None else idx.shape[-1]
    _raise(_lib.lsa_sparse_attn_noalloc(_ptr(Q), T, Hq, _ptr(K), _ptr(V), K.shape[0], K.shape[1], d, _dtype(Q),
                                        _ptr(idx), K_sel, _ptr(q_pos), int(bool(causal)), tail_begin, tail_end,
                                        float(scale), _ptr(O), _ptr(LSE), _ptr(status), _stream(stream, Q)),
           "lsa_sparse_attn_noalloc")


def lsa_sparse_attn_bwd(Q, K, V, O, LSE, dO, idx, q_pos, causal, tail_begin, tail_end, scale, dQ, dK, dV,
                        status=None, stream=None):
    T, Hq, d = Q.shape
    K_sel = 0 if idx is None else idx.shape[-1]
    _raise(_lib.lsa_sparse_attn_bwd(_ptr(Q), T, Hq, _ptr(K), _ptr(V), K.shape[0], K.shape[1], d, _dtype(Q),
                                    _ptr(O), _ptr(LSE), _ptr(dO), _ptr(idx), K_sel, _ptr(q_pos),
                                    int(bool(causal)), tail_begin, tail_end, float(scale), _ptr(dQ), _ptr(dK),
                                    _ptr(dV), _ptr(status), _stream(stream, Q)), "lsa_sparse_attn_bwd")


def lsa_sparse_attn_sw_workspace_bytes(T, Hq, n_heads, d, K_sel, tail_len, n_sink, window) -> int:
    n = ctypes.c_size_t()
    _raise(_lib.lsa_sparse_attn_sw_workspace_bytes(T, Hq, n_heads, d, K_sel, int(tail_len), int(n_sink), int(window),
                                                   ctypes.byref(n)), "lsa_sparse_attn_sw_workspace_bytes")
    return int(n.value)


def lsa_sparse_attn_sw(Q, K, V, idx, q_pos, n_sink, window, tail_begin, tail_end, scale, O, LSE, workspace,
                       status=None, stream=None):
    T, Hq, d = Q.shape
    K_sel = 0 if idx is None else idx.shape[-1]
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _raise(_lib.lsa_sparse_attn_sw(_ptr(Q), T, Hq, _ptr(K), _ptr(V), K.shape[0], K.shape[1], d, _dtype(Q), _ptr(idx),
                                   K_sel, _ptr(q_pos), int(n_sink), int(window), tail_begin, tail_end, float(scale),
                                   _ptr(O), _ptr(LSE), _ptr(workspace), ws_n, _ptr(status), _stream(stream, Q)),
           "lsa_sparse_attn_sw")


def lsa_sparse_attn_sw_bwd(Q, K, V, O, LSE, dO, idx, q_pos, n_sink, window, tail_begin, tail_end, scale, dQ, dK, dV,
                           workspace, status=None, stream=None):
    T, Hq, d = Q.shape
    K_sel = 0 if idx is None else idx.shape[-1]
    ws_n = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _raise(_lib.lsa_sparse_attn_sw_bwd(_ptr(Q), T, Hq, _ptr(K), _ptr(V), K.shape[0], K.shape[1], d, _dtype(Q),
                                       _ptr(O), _ptr(LSE), _ptr(dO), _ptr(idx), K_sel, _ptr(q_pos), int(n_sink),
                                       int(window), tail_begin, tail_end, float(scale), _ptr(dQ), _ptr(dK), _ptr(dV),
                                       _ptr(workspace), ws_n, _ptr(status), _stream(stream, Q)),
           "lsa_sparse_attn_sw_bwd")


def lsa_project_keys(K, W, n, Z, status=None, stream=None):
    """K: [n_heads, n_cap, d]; W: [n_heads, d, r]; Z: [n_heads, n, r] fp32 (written)."""
    _raise(_lib.lsa_project_keys(_ptr(K), K.shape[0], K.shape[1], K.shape[2], _dtype(K), _ptr(W), W.shape[2],
                                 int(n), _ptr(Z), _ptr(status), _stream(stream, K)), "lsa_project_keys")


def lsa_balanced_assign_workspace_bytes(nseg, m, b) -> int:
    n = ctypes.c_size_t()
    _raise(_lib.lsa_balanced_assign_workspace_bytes(int(nseg), int(m), int(b), ctypes.byref(n)),
           "lsa_balanced_assign_workspace_bytes")
    return n.value


def lsa_balanced_assign(Z, mu, nseg, m, b, max_rounds, choice, workspace, status=None, stream=None):
    """Z: [nseg*m, r] fp32; mu: [nseg*b, r] fp32; choice: [nseg*m] uint8 (written)."""
    _raise(_lib.lsa_balanced_assign(_ptr(Z), _ptr(mu), int(nseg), int(m), int(b), Z.shape[1], int(max_rounds),
                                    _ptr(choice), _ptr(workspace), workspace.numel(), _ptr(status),
                                    _stream(stream, Z)), "lsa_balanced_assign")


def balanced_assign(Z, mu, nseg, m, b, max_rounds=0, status=None, check=True):
    """Centroid index (uint8) of every row of every segment; see lsa_balanced_assign."""
    choice = torch.empty(nseg * m, dtype=torch.uint8, device=Z.device)
    ws = torch.empty(lsa_balanced_assign_workspace_bytes(nseg, m, b), dtype=torch.uint8, device=Z.device)
    st = _new_status(Z.device) if status is None else status
    lsa_balanced_assign(Z, mu, nseg, m, b, max_rounds, choice, ws, st)
    if check:
        check_status(st, "lsa_balanced_assign")
    return choice


def lsa_decode_step_workspace_bytes(desc, Hq, d, beam, tail_len_max) -> int:
    n = ctypes.c_size_t()
    bm = (ctypes.c_int32 * len(beam))(*beam)
    _raise(_lib.lsa_decode_step_workspace_bytes(ctypes.byref(desc), Hq, d, bm, int(tail_len_max), ctypes.byref(n)),
           "lsa_decode_step_workspace_bytes")
    return n.value


def lsa_decode_step(desc, tree_mem, W, beam, K, V, Q, K_row, V_row, pos, tail_begin, scale, O, LSE, workspace,
                    leaves_out=None, status=None, stream=None):
    """K, V: [n_heads, n_cap, d] caches; Q: [1, Hq, d]; K_row, V_row: [n_heads, d] or None;
    O: [1, Hq, d]; LSE: [1, Hq]; leaves_out: [n_heads, beam[-1]] int32 or None."""
    bm = (ctypes.c_int32 * len(beam))(*beam)
    _raise(_lib.lsa_decode_step(ctypes.byref(desc), _ptr(tree_mem), _ptr(W), bm, _ptr(K), _ptr(V), K.shape[1],
                                K.shape[2], _dtype(K), _ptr(Q), Q.shape[1], _ptr(K_row), _ptr(V_row), int(pos),
                                int(tail_begin), float(scale), _ptr(O), _ptr(LSE), _ptr(leaves_out),
                                _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream, K)),
           "lsa_decode_step")


class DecodeStep:
    """Buffers of a decode loop over one index: call step(...) once per token."""

    def __init__(self, tree, W, beam, K, Hq, tail_len_max, scale=None):
        d = K.shape[2]
        self.tree, self.W, self.beam = tree, W, list(beam)
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        need = lsa_decode_step_workspace_bytes(tree.desc, Hq, d, self.beam, tail_len_max)
        self.ws = torch.empty(need, dtype=torch.uint8, device=K.device)
        self.O = torch.empty(1, Hq, d, dtype=K.dtype, device=K.device)
        self.LSE = torch.empty(1, Hq, dtype=torch.float32, device=K.device)
        self.leaves = torch.empty(K.shape[0], self.beam[-1], dtype=torch.int32, device=K.device)
        self.status = _new_status(K.device)

    def step(self, K, V, Q, K_row, V_row, pos, tail_begin, stream=None):
        lsa_decode_step(self.tree.desc, self.tree.mem, self.W, self.beam, K, V, Q, K_row, V_row, pos, tail_begin,
                        self.scale, self.O, self.LSE, self.ws, self.leaves, self.status, stream)
        return self.O, self.LSE


def project_keys(K, W, n=None):
    """Latents Z [n_heads, n, r] fp32 of the first n keys of K (all of them by default)."""
    n = K.shape[1] if n is None else n
    Z = torch.empty(K.shape[0], n, W.shape[2], dtype=torch.float32, device=K.device)
    st = _new_status(K.device)
    lsa_project_keys(K, W, n, Z, st)
    check_status(st, "lsa_project_keys")
    return Z


def lsa_kv_append(K, V, pos, K_rows, V_rows, stream=None):
    """K, V: [n_heads, n_cap, d] caches; K_rows, V_rows: [n_heads, d] rows written at `pos`."""
    _raise(_lib.lsa_kv_append(_ptr(K), _ptr(V), K.shape[0], K.shape[1], K.shape[2], _dtype(K), int(pos),
                              _ptr(K_rows), _ptr(V_rows), _stream(stream, K)), "lsa_kv_append")


def lsa_status_clear(status, stream=None):
    _raise(_lib.lsa_status_clear(_ptr(status), _stream(stream, status)), "lsa_status_clear")


def lsa_status_check(status, stream=None) -> int:
    out = ctypes.c_int32()
    _raise(_lib.lsa_status_check(_ptr(status), _stream(stream, status), ctypes.byref(out)), "lsa_status_check")
    return int(out.value)


# --- helpers: torch-allocated outputs around the same entry points -----------------

def _new_status(device):
    return torch.zeros(1, dtype=torch.int32, device=device)


def check_status(status, what: str):
    code = lsa_status_check(status)
    if code != LSA_OK:
        raise LsaError(code, what, "reported by a kernel")


@dataclass
class Tree:
    desc: lsa_tree_desc
    mem: torch.Tensor          # uint8 [desc.bytes] on the device

    @property
    def levels(self) -> int:
        return self.desc.levels

    @property
    def branching(self):
        return tuple(self.desc.branching[l] for l in range(self.desc.levels))

    def centroids(self, level: int) -> torch.Tensor:
        d = self.desc
        n = d.n_heads * d.nodes[level] * d.r
        off = d.off_centroids[level]
        return self.mem[off:off + 4 * n].view(torch.float32).view(d.n_heads, d.nodes[level], d.r)

    def min_pos(self, level: int) -> torch.Tensor:
        d = self.desc
        n = d.n_heads * d.nodes[level]
        off = d.off_min_pos[level]
        return self.mem[off:off + 4 * n].view(torch.int32).view(d.n_heads, d.nodes[level])

    def leaf_index(self) -> torch.Tensor:
        d = self.desc
        n = d.n_heads * d.n_tree
        off = d.off_leaf_index
        return self.mem[off:off + 4 * n].view(torch.int32).view(d.n_heads, d.n_tree)


def build_tree(K, W, branching, leaf_size, iters, seed, trace=False, workspace=None, status=None, check=True,
               pool=1):
    """Build the index over positions [0, leaf_size * prod(branching)) of K; pool > 1 clusters
    blocks of `pool` consecutive keys (the trace is then by block)."""
    Hkv, n_cap, d = K.shape
    desc = lsa_tree_describe(Hkv, W.shape[2], branching, leaf_size)
    mem = torch.empty(desc.bytes, dtype=torch.uint8, device=K.device)
    need = lsa_build_workspace_bytes(desc, d)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=K.device)
    tr = (torch.empty(len(branching), iters, Hkv, desc.n_tree // pool, dtype=torch.int32, device=K.device)
          if trace else None)
    st = _new_status(K.device) if status is None else status
    if pool == 1:
        lsa_build_tree(desc, mem, K, W, iters, seed, workspace, tr, st)
    else:
        lsa_build_tree_pooled(desc, mem, K, W, pool, iters, seed, workspace, tr, st)
    if check:
        check_status(st, "lsa_build_tree")
    tree = Tree(desc, mem)
    return (tree, tr) if trace else tree


def tree_append(tree: Tree, K, W, iters, seed, trace=False, workspace=None, status=None, check=True):
    """The index grown by one top-level node over the next U = leaf * b_1 * ... keys of K
    (positions tree.n_tree ..); returns the new Tree (and the subtree's build trace)."""
    d0 = tree.desc
    Hkv, n_cap, d = K.shape
    levels = d0.levels
    br = [d0.branching[l] for l in range(levels)]
    grown = lsa_tree_describe(Hkv, d0.r, [br[0] + 1] + br[1:], d0.leaf_size)
    mem = torch.empty(grown.bytes, dtype=torch.uint8, device=K.device)
    need = lsa_tree_append_workspace_bytes(d0, d)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=K.device)
    U = grown.n_tree - d0.n_tree
    tr = torch.empty(levels - 1, iters, Hkv, U, dtype=torch.int32, device=K.device) if trace else None
    st = _new_status(K.device) if status is None else status
    lsa_tree_append(d0, tree.mem, grown, mem, K, W, iters, seed, workspace, tr, st)
    if check:
        check_status(st, "lsa_tree_append")
    t = Tree(grown, mem)
    return (t, tr) if trace else t


def select(tree: Tree, Q, W, beam, q_pos=None, qlat=False, beams=False, leaves=False, status=None, check=True,
           batched=False):
    """Returns idx (and, when asked, leaves, query latents, per-level beams, in that order).
    batched: run lsa_select_batched (same results, scheduled for large batches)."""
    T = Q.shape[0]
    d = tree.desc
    K_sel = beam[-1] * d.leaf_size
    idx = torch.empty(d.n_heads, T, K_sel, dtype=torch.int32, device=Q.device)
    lv = torch.empty(d.n_heads, T, beam[-1], dtype=torch.int32, device=Q.device) if leaves else None
    ql = torch.empty(T, d.n_heads, d.r, dtype=torch.float32, device=Q.device) if qlat else None
    bo = torch.empty(d.levels, d.n_heads, T, max(beam), dtype=torch.int32, device=Q.device) if beams else None
    st = _new_status(Q.device) if status is None else status
    if batched:
        n = lsa_select_batched_workspace_bytes(d, T, beam)
        ws = torch.empty(max(n, 1), dtype=torch.uint8, device=Q.device)
        lsa_select_batched(d, tree.mem, Q, W, beam, q_pos, idx, lv, ql, bo, ws, st)
    else:
        lsa_select(d, tree.mem, Q, W, beam, q_pos, idx, lv, ql, bo, st)
    if check:
        check_status(st, "lsa_select_batched" if batched else "lsa_select")
    out = [idx]
    if leaves:
        out.append(lv)
    if qlat:
        out.append(ql)
    if beams:
        out.append(bo)
    return out[0] if len(out) == 1 else tuple(out)


def lsa_select_flat(desc, tree_mem, Q, W, n_leaves, q_pos, idx_out, leaves_out=None, qlat_out=None, status=None,
                    stream=None):
    T, Hq, d = Q.shape
    _raise(_lib.lsa_select_flat(ctypes.byref(desc), _ptr(tree_mem), _ptr(Q), T, Hq, d, _dtype(Q), _ptr(W),
                                int(n_leaves), _ptr(q_pos), _ptr(idx_out), _ptr(leaves_out), _ptr(qlat_out),
                                _ptr(status), _stream(stream, Q)), "lsa_select_flat")


def select_flat(tree: Tree, Q, W, n_leaves, q_pos=None, qlat=False, leaves=False, status=None, check=True):
    """Flat search over every leaf; returns idx (and, when asked, leaves, query latents)."""
    T = Q.shape[0]
    d = tree.desc
    idx = torch.empty(d.n_heads, T, n_leaves * d.leaf_size, dtype=torch.int32, device=Q.device)
    lv = torch.empty(d.n_heads, T, n_leaves, dtype=torch.int32, device=Q.device) if leaves else None
    ql = torch.empty(T, d.n_heads, d.r, dtype=torch.float32, device=Q.device) if qlat else None
    st = _new_status(Q.device) if status is None else status
    lsa_select_flat(d, tree.mem, Q, W, n_leaves, q_pos, idx, lv, ql, st)
    if check:
        check_status(st, "lsa_select_flat")
    out = [idx]
    if leaves:
        out.append(lv)
    if qlat:
        out.append(ql)
    return out[0] if len(out) == 1 else tuple(out)


def sparse_attn(Q, K, V, idx, q_pos=None, causal=False, tail=(0, 0), scale=None, workspace=None, status=None,
                check=True, sink=0, window=0):
    """Key-list attention; sink / window > 0 add the first `sink` positions and the `window` positions up to
    q_pos to every query's keys (causal, lsa_sparse_attn_sw)."""
    T, Hq, d = Q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    K_sel = 0 if idx is None else idx.shape[-1]
    if sink or window:
        need = lsa_sparse_attn_sw_workspace_bytes(T, Hq, K.shape[0], d, K_sel, tail[1] - tail[0], sink, window)
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
        O = torch.empty_like(Q)
        LSE = torch.empty(T, Hq, dtype=torch.float32, device=Q.device)
        st = _new_status(Q.device) if status is None else status
        lsa_sparse_attn_sw(Q, K, V, idx, q_pos, sink, window, tail[0], tail[1], scale, O, LSE, workspace, st)
        if check:
            check_status(st, "lsa_sparse_attn_sw")
        return O, LSE
    need = lsa_attn_workspace_bytes(T, Hq, K.shape[0], d, K_sel, tail[1] - tail[0])
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    O = torch.empty_like(Q)
    LSE = torch.empty(T, Hq, dtype=torch.float32, device=Q.device)
    st = _new_status(Q.device) if status is None else status
    lsa_sparse_attn(Q, K, V, idx, q_pos, causal, tail[0], tail[1], scale, O, LSE, workspace if need else None, st)
    if check:
        check_status(st, "lsa_sparse_attn")
    return O, LSE


def lsa_tree_attn_sw_workspace_bytes(desc, T, Hq, d, dtype, n_leaves, n_sink, window) -> int:
    n = ctypes.c_size_t()
    _raise(_lib.lsa_tree_attn_sw_workspace_bytes(ctypes.byref(desc), T, Hq, d, _DTYPE[dtype], n_leaves, int(n_sink),
                                                 int(window), ctypes.byref(n)), "lsa_tree_attn_sw_workspace_bytes")
    return int(n.value)


def lsa_tree_attn_sw(desc, tree_mem, Q, K, V, leaves, q_pos, n_sink, window, scale, O, LSE, workspace, status=None,
                     stream=None):
    T, Hq, d = Q.shape
    ws_n = workspace.numel() * workspace.element_size()
    _raise(_lib.lsa_tree_attn_sw(ctypes.byref(desc), _ptr(tree_mem), _ptr(Q), T, Hq, _ptr(K), _ptr(V), K.shape[1], d,
                                 _dtype(Q), _ptr(leaves), leaves.shape[-1], _ptr(q_pos), int(n_sink), int(window),
                                 float(scale), _ptr(O), _ptr(LSE), _ptr(workspace), ws_n, _ptr(status),
                                 _stream(stream, Q)), "lsa_tree_attn_sw")


def tree_attn(tree: Tree, Q, K, V, leaves, q_pos=None, causal=False, scale=None, workspace=None, status=None,
              check=True, sink=0, window=0):
    T, Hq, d = Q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if sink or window:
        need = lsa_tree_attn_sw_workspace_bytes(tree.desc, T, Hq, d, Q.dtype, leaves.shape[-1], sink, window)
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
        O = torch.empty_like(Q)
        LSE = torch.empty(T, Hq, dtype=torch.float32, device=Q.device)
        st = _new_status(Q.device) if status is None else status
        lsa_tree_attn_sw(tree.desc, tree.mem, Q, K, V, leaves, q_pos, sink, window, scale, O, LSE, workspace, st)
        if check:
            check_status(st, "lsa_tree_attn_sw")
        return O, LSE
    need = lsa_tree_attn_workspace_bytes(tree.desc, T, Hq, d, Q.dtype, leaves.shape[-1])
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    O = torch.empty_like(Q)
    LSE = torch.empty(T, Hq, dtype=torch.float32, device=Q.device)
    st = _new_status(Q.device) if status is None else status
    lsa_tree_attn(tree.desc, tree.mem, Q, K, V, leaves, q_pos, causal, scale, O, LSE, workspace, st)
    if check:
        check_status(st, "lsa_tree_attn")
    return O, LSE


def lsa_tree_attn_bwd_workspace_bytes(desc, T, Hq, d, dtype, n_leaves) -> int:
    n = ctypes.c_size_t()
    _raise(_lib.lsa_tree_attn_bwd_workspace_bytes(ctypes.byref(desc), T, Hq, d, _DTYPE[dtype], n_leaves,
                                                  ctypes.byref(n)), "lsa_tree_attn_bwd_workspace_bytes")
    return int(n.value)


def lsa_tree_attn_bwd(desc, tree_mem, Q, K, V, O, LSE, dO, leaves, q_pos, causal, scale, dQ, dK, dV, workspace,
                      status=None, stream=None):
    T, Hq, d = Q.shape
    ws_n = workspace.numel() * workspace.element_size()
    _raise(_lib.lsa_tree_attn_bwd(ctypes.byref(desc), _ptr(tree_mem), _ptr(Q), T, Hq, _ptr(K), _ptr(V), K.shape[1],
                                  d, _dtype(Q), _ptr(O), _ptr(LSE), _ptr(dO), _ptr(leaves), leaves.shape[-1],
                                  _ptr(q_pos), int(bool(causal)), float(scale), _ptr(dQ), _ptr(dK), _ptr(dV),
                                  _ptr(workspace), ws_n, _ptr(status), _stream(stream, Q)), "lsa_tree_attn_bwd")


def tree_attn_bwd(tree: Tree, Q, K, V, O, LSE, dO, leaves, q_pos=None, causal=False, scale=None, workspace=None,
                  status=None, check=True):
    T, Hq, d = Q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    need = lsa_tree_attn_bwd_workspace_bytes(tree.desc, T, Hq, d, Q.dtype, leaves.shape[-1])
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    dQ = torch.empty(T, Hq, d, dtype=torch.float32, device=Q.device)
    dK = torch.empty(K.shape, dtype=torch.float32, device=Q.device)
    dV = torch.empty(V.shape, dtype=torch.float32, device=Q.device)
    st = _new_status(Q.device) if status is None else status
    lsa_tree_attn_bwd(tree.desc, tree.mem, Q, K, V, O, LSE, dO, leaves, q_pos, causal, scale, dQ, dK, dV,
                      workspace, st)
    if check:
        check_status(st, "lsa_tree_attn_bwd")
    return dQ, dK, dV


def sparse_attn_bwd(Q, K, V, O, LSE, dO, idx, q_pos=None, causal=False, tail=(0, 0), scale=None, status=None,
                    check=True, sink=0, window=0):
    T, Hq, d = Q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dQ = torch.empty(T, Hq, d, dtype=torch.float32, device=Q.device)
    dK = torch.empty(K.shape, dtype=torch.float32, device=Q.device)
    dV = torch.empty(V.shape, dtype=torch.float32, device=Q.device)
    st = _new_status(Q.device) if status is None else status
    if sink or window:
        K_sel = 0 if idx is None else idx.shape[-1]
        ws = torch.empty(max(K.shape[0] * T * (K_sel + sink + window) * 4 + 256, 1), dtype=torch.uint8,
                         device=Q.device)
        lsa_sparse_attn_sw_bwd(Q, K, V, O, LSE, dO, idx, q_pos, sink, window, tail[0], tail[1], scale, dQ, dK, dV, ws,
                               st)
        if check:
            check_status(st, "lsa_sparse_attn_sw_bwd")
        return dQ, dK, dV
    lsa_sparse_attn_bwd(Q, K, V, O, LSE, dO, idx, q_pos, causal, tail[0], tail[1], scale, dQ, dK, dV, st)
    if check:
        check_status(st, "lsa_sparse_attn_bwd")
    return dQ, dK, dV
