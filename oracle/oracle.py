"""Python face of the fp64 CPU oracle (``oracle/lsa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline / reference arm are the only callers.  The product path never
imports this module.

Every function widens its inputs to float64 (the stored bf16/fp32 values are
exactly representable), calls the plain C loops and returns numpy arrays.  The
arithmetic itself lives only in the C file; this module marshals arguments.

Parity status of each function (what pins it, in ``tests/test_oracle_pins.py``):
  init_hash / splitmix64    published SplitMix64 output vectors
  project, query_latent     numpy matmul on the same inputs
  balanced_assign           brute-force enumeration of all balanced assignments
                            (exactly one is stable, and it is the greedy one) and
                            an independent deferred-acceptance implementation
  build_tree                centroid == mean of members, parent == mean of
                            children, exact leaf sizes, permutation, init rule
  tree_append               old nodes unchanged; centroids == means of the keys
                            listed under each node (new top node included); the
                            full-beam walk == brute-force flat top-B
  pool_keys,                pool 1 == build_tree; centroids == means of the listed
  build_tree_pooled         keys' latents; leaves are whole aligned blocks; block
                            tree == build_tree on latents pooled by numpy
  select                    full beam == brute-force flat top-B over all leaves,
                            scored-node count, causal eligibility brute force
  attn_fwd                  torch SDPA (CPU, float64) with a boolean mask, one
                            visible key returns its value row, permutation
                            invariance
  attn_bwd                  torch autograd through dense masked attention and
                            central finite differences
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lsa_oracle.c")
_LIB = os.path.join(_HERE, "liblsa_oracle.so")
_lock = threading.Lock()
_lib = None

MAX_LEVELS = 8


class OracleError(RuntimeError):
    pass


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (plain IEEE double: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-ffp-contract=off", "-fno-fast-math", src, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building if needed) the oracle library; a path selects another build."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


@contextlib.contextmanager
def using(path: str):
    """Temporarily route every call of this module to another build of the oracle
    (the mutation tests load deliberately broken copies this way)."""
    global _lib
    load()
    with _lock:
        old, _lib = _lib, _declare(ctypes.CDLL(path))
    try:
        yield
    finally:
        with _lock:
            _lib = old


def _declare(lib):
    P = ctypes.c_void_p
    i32, i64, u64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
    sig = {
        "orc_splitmix64_mix": (u64, [u64]),
        "orc_splitmix64_at": (u64, [u64, u64]),
        "orc_init_hash": (u64, [u64, i32, i64]),
        "orc_project": (ctypes.c_int, [P, i64, i32, P, i32, P]),
        "orc_query_latent": (ctypes.c_int, [P, i64, i32, i32, P, i32, P]),
        "orc_balanced_assign": (ctypes.c_int, [P, P, i64, i32, P]),
        "orc_distances": (ctypes.c_int, [P, i64, i32, P, i32, P]),
        "orc_level_init": (ctypes.c_int, [P, P, i64, i32, i32, u64, i32, P]),
        "orc_means": (ctypes.c_int, [P, i64, i32, P, i32, P]),
        "orc_build_tree": (ctypes.c_int, [P, i64, i32, P, i32, i32, i32, u64, P, P, P, P]),
        "orc_pool_keys": (ctypes.c_int, [P, i64, i32, i32, P]),
        "orc_tree_append": (ctypes.c_int, [P, P, P, i64, P, i64, i32, P, i32, i32, i32, u64, P, P, P, P]),
        "orc_build_tree_pooled": (ctypes.c_int, [P, i64, i32, i32, P, i32, i32, i32, u64, P, P, P, P]),
        "orc_select": (ctypes.c_int, [P, i64, i32, P, i32, i32, P, P, P, P, P, P, P, P]),
        "orc_attn_fwd": (ctypes.c_int, [P, i64, i32, i32, P, P, i64, P, i32, P, i32, i64, i64,
                                        f64, P, P]),
        "orc_attn_bwd": (ctypes.c_int, [P, i64, i32, i32, P, P, i64, P, i32, P, i32, i64, i64,
                                        f64, P, P, P, P]),
        "orc_attn_fwd_sw": (ctypes.c_int, [P, i64, i32, i32, P, P, i64, P, i32, P, i64, i64, i32, i32,
                                           f64, P, P]),
        "orc_attn_bwd_sw": (ctypes.c_int, [P, i64, i32, i32, P, P, i64, P, i32, P, i64, i64, i32, i32,
                                           f64, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _i64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int64)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with status {rc}")


# --- generator ---------------------------------------------------------------

def splitmix64_mix(z: int) -> int:
    return int(load().orc_splitmix64_mix(z))


def splitmix64_at(state: int, i: int) -> int:
    return int(load().orc_splitmix64_at(state, i))


def init_hash(seed: int, level: int, pos: int) -> int:
    return int(load().orc_init_hash(seed, level, pos))


# --- projection ----------------------------------------------------------------

def project(X, W) -> np.ndarray:
    X, W = _f64(X), _f64(W)
    n, d = X.shape
    r = W.shape[1]
    Z = np.empty((n, r), np.float64)
    _check(load().orc_project(_p(X), n, d, _p(W), r, _p(Z)), "orc_project")
    return Z


def query_latent(Qg, W) -> np.ndarray:
    """Qg: [T, G, d] rows of one GQA group; W: [d, r] -> [T, r]."""
    Qg, W = _f64(Qg), _f64(W)
    T, G, d = Qg.shape
    r = W.shape[1]
    out = np.empty((T, r), np.float64)
    _check(load().orc_query_latent(_p(Qg), T, G, d, _p(W), r, _p(out)), "orc_query_latent")
    return out


# --- clustering ------------------------------------------------------------------

def balanced_assign(D, pos) -> np.ndarray:
    D, pos = _f64(D), _i64(pos)
    m, b = D.shape
    a = np.empty(m, np.int32)
    _check(load().orc_balanced_assign(_p(D), _p(pos), m, b, _p(a)), "orc_balanced_assign")
    return a


def distances(Zs, mu) -> np.ndarray:
    Zs, mu = _f64(Zs), _f64(mu)
    m, r = Zs.shape
    b = mu.shape[0]
    D = np.empty((m, b), np.float64)
    _check(load().orc_distances(_p(Zs), m, r, _p(mu), b, _p(D)), "orc_distances")
    return D


def level_init(Zs, pos, b: int, seed: int, level: int) -> np.ndarray:
    Zs, pos = _f64(Zs), _i64(pos)
    m, r = Zs.shape
    mu = np.empty((b, r), np.float64)
    _check(load().orc_level_init(_p(Zs), _p(pos), m, r, b, seed, level, _p(mu)), "orc_level_init")
    return mu


def means(Zs, assign, b: int) -> np.ndarray:
    Zs, assign = _f64(Zs), _i32(assign)
    m, r = Zs.shape
    mu = np.empty((b, r), np.float64)
    _check(load().orc_means(_p(Zs), m, r, _p(assign), b, _p(mu)), "orc_means")
    return mu


class Tree:
    """Oracle tree of one KV head: per-level centroids / min positions, leaf_index."""

    def __init__(self, branching, leaf_size, r, centroids, min_pos, leaf_index, trace=None):
        self.branching = tuple(int(b) for b in branching)
        self.leaf_size = int(leaf_size)
        self.r = int(r)
        self.nodes = list(np.cumprod(self.branching).astype(np.int64))
        self.centroids_flat = centroids
        self.min_pos_flat = min_pos
        self.leaf_index = leaf_index
        self.trace = trace
        offs = np.concatenate([[0], np.cumsum(self.nodes)]).astype(np.int64)
        self.centroids = [centroids[offs[l] * r:offs[l + 1] * r].reshape(-1, r) for l in range(len(self.nodes))]
        self.min_pos = [min_pos[offs[l]:offs[l + 1]] for l in range(len(self.nodes))]

    @classmethod
    def from_levels(cls, branching, leaf_size, centroids_levels, min_pos_levels, leaf_index):
        """Wrap per-level arrays (e.g. a tree exported by another implementation)."""
        r = np.asarray(centroids_levels[0]).shape[-1]
        c = np.concatenate([_f64(x).reshape(-1) for x in centroids_levels])
        m = np.concatenate([_i32(x).reshape(-1) for x in min_pos_levels])
        return cls(branching, leaf_size, r, c, m, _i32(leaf_index).reshape(-1))


def build_tree(Z, branching, leaf_size: int, iters: int, seed: int, trace: bool = False) -> Tree:
    Z = _f64(Z)
    n, r = Z.shape
    br = np.ascontiguousarray(branching, np.int32)
    L = len(br)
    total_nodes = int(np.sum(np.cumprod(br.astype(np.int64))))
    cent = np.empty(total_nodes * r, np.float64)
    mpos = np.empty(total_nodes, np.int32)
    leaf = np.empty(n, np.int32)
    tr = np.empty((L, iters, n), np.int32) if trace else None
    _check(load().orc_build_tree(_p(Z), n, r, _p(br), L, leaf_size, iters, seed,
                                 _p(cent), _p(mpos), _p(leaf), _p(tr)), "orc_build_tree")
    return Tree(br, leaf_size, r, cent, mpos, leaf, tr)


def pool_keys(Z, p: int) -> np.ndarray:
    """Mean latent row of every block of p consecutive keys: [n, r] -> [n / p, r]."""
    Z = _f64(Z)
    n, r = Z.shape
    out = np.empty((n // p, r), np.float64)
    _check(load().orc_pool_keys(_p(Z), n, r, p, _p(out)), "orc_pool_keys")
    return out


def build_tree_pooled(Z, p: int, branching, leaf_size: int, iters: int, seed: int, trace: bool = False) -> Tree:
    """Tree over blocks of p consecutive keys (leaf_size / p blocks per leaf); leaf_index and
    min_pos in key positions, trace (if asked) by block."""
    Z = _f64(Z)
    n, r = Z.shape
    br = np.ascontiguousarray(branching, np.int32)
    L = len(br)
    total_nodes = int(np.sum(np.cumprod(br.astype(np.int64))))
    cent = np.empty(total_nodes * r, np.float64)
    mpos = np.empty(total_nodes, np.int32)
    leaf = np.empty(n, np.int32)
    tr = np.empty((L, iters, n // p), np.int32) if trace else None
    _check(load().orc_build_tree_pooled(_p(Z), n, r, p, _p(br), L, leaf_size, iters, seed,
                                        _p(cent), _p(mpos), _p(leaf), _p(tr)), "orc_build_tree_pooled")
    return Tree(br, leaf_size, r, cent, mpos, leaf, tr)


def tree_append(tree: Tree, Znew, iters: int, seed: int, trace: bool = False) -> Tree:
    """Attach a subtree over the U = leaf * b_1 * ... * b_{L-1} appended keys (latent rows Znew,
    positions n_old ..) as top node b_0; returns the grown tree (trace: the subtree's build)."""
    Znew = _f64(Znew)
    U, r = Znew.shape
    br = np.ascontiguousarray(tree.branching, np.int32)
    L = len(br)
    n_old = int(len(tree.leaf_index))
    grown = br.copy()
    grown[0] += 1
    total_nodes = int(np.sum(np.cumprod(grown.astype(np.int64))))
    cent = np.empty(total_nodes * r, np.float64)
    mpos = np.empty(total_nodes, np.int32)
    leaf = np.empty(n_old + U, np.int32)
    tr = np.empty((L - 1, iters, U), np.int32) if trace else None
    _check(load().orc_tree_append(_p(_f64(tree.centroids_flat)), _p(_i32(tree.min_pos_flat)),
                                  _p(_i32(tree.leaf_index)), n_old, _p(Znew), U, r, _p(br), L, tree.leaf_size,
                                  iters, seed, _p(cent), _p(mpos), _p(leaf), _p(tr)), "orc_tree_append")
    return Tree(grown, tree.leaf_size, r, cent, mpos, leaf, tr)


def select(qlat, tree: Tree, beam, q_pos=None, trace: bool = False):
    """Returns (idx [T, K_sel], beam_trace [L, T, Bmax] or None, scored [T])."""
    qlat = _f64(qlat)
    T, r = qlat.shape
    beam = np.ascontiguousarray(beam, np.int32)
    L = len(tree.branching)
    K_sel = int(beam[-1]) * tree.leaf_size
    idx = np.empty((T, K_sel), np.int32)
    bt = np.empty((L, T, int(beam.max())), np.int32) if trace else None
    scored = np.empty(T, np.int64)
    qp = None if q_pos is None else _i32(q_pos)
    br = np.ascontiguousarray(tree.branching, np.int32)
    _check(load().orc_select(_p(qlat), T, r, _p(br), L, tree.leaf_size,
                             _p(tree.centroids_flat), _p(_i32(tree.min_pos_flat)),
                             _p(_i32(tree.leaf_index)), _p(beam), _p(qp), _p(idx), _p(bt),
                             _p(scored)), "orc_select")
    return idx, bt, scored


# --- attention -------------------------------------------------------------------

def select_flat(qlat, tree: Tree, n_leaves, q_pos=None):
    """Flat search (bdtechtalks.com, "Latent sparse attention", "How latent sparse attention
    works": the query is compared with every cluster centroid): the beam walk with every node
    kept above the leaf level scores every (eligible) leaf and keeps the n_leaves best.
    Returns (idx [T, n_leaves * leaf], kept leaf ids [T, n_leaves], -1 padded)."""
    full = [int(tree.nodes[l]) for l in range(len(tree.nodes) - 1)]
    idx, beams, _ = select(qlat, tree, full + [int(n_leaves)], q_pos=q_pos, trace=True)
    return idx, beams[-1][:, :int(n_leaves)]


def attn_fwd(Qg, K, V, idx, q_pos=None, causal=False, tail=(0, 0), scale=None, sink=0, window=0):
    """Qg: [T, G, d]; K, V: [n_cap, d]; idx: [T, K_sel] or None -> (O [T,G,d], LSE [T,G]).
    sink / window > 0 (causal only): the first `sink` positions and the `window` positions up to
    q_pos join every query's key set, each key counted once."""
    Qg, K, V = _f64(Qg), _f64(K), _f64(V)
    T, G, d = Qg.shape
    n_cap = K.shape[0]
    if idx is None:
        idx_a, K_sel = None, 0
    else:
        idx_a = _i32(idx)
        K_sel = idx_a.shape[1]
    qp = None if q_pos is None else _i32(q_pos)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    O = np.empty((T, G, d), np.float64)
    LSE = np.empty((T, G), np.float64)
    if sink or window:
        assert causal, "sink and window keys need query positions (causal)"
        _check(load().orc_attn_fwd_sw(_p(Qg), T, G, d, _p(K), _p(V), n_cap, _p(idx_a), K_sel, _p(qp),
                                      int(tail[0]), int(tail[1]), int(sink), int(window), scale,
                                      _p(O), _p(LSE)), "orc_attn_fwd_sw")
        return O, LSE
    _check(load().orc_attn_fwd(_p(Qg), T, G, d, _p(K), _p(V), n_cap, _p(idx_a), K_sel, _p(qp),
                               int(bool(causal)), int(tail[0]), int(tail[1]), scale,
                               _p(O), _p(LSE)), "orc_attn_fwd")
    return O, LSE


def attn_bwd(Qg, K, V, idx, dO, q_pos=None, causal=False, tail=(0, 0), scale=None, sink=0, window=0):
    """Returns (dQ [T,G,d], dK [n_cap,d], dV [n_cap,d]); sink / window as in attn_fwd."""
    Qg, K, V, dO = _f64(Qg), _f64(K), _f64(V), _f64(dO)
    T, G, d = Qg.shape
    n_cap = K.shape[0]
    if idx is None:
        idx_a, K_sel = None, 0
    else:
        idx_a = _i32(idx)
        K_sel = idx_a.shape[1]
    qp = None if q_pos is None else _i32(q_pos)
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    dQ = np.empty((T, G, d), np.float64)
    dK = np.empty((n_cap, d), np.float64)
    dV = np.empty((n_cap, d), np.float64)
    if sink or window:
        assert causal, "sink and window keys need query positions (causal)"
        _check(load().orc_attn_bwd_sw(_p(Qg), T, G, d, _p(K), _p(V), n_cap, _p(idx_a), K_sel, _p(qp),
                                      int(tail[0]), int(tail[1]), int(sink), int(window), scale, _p(dO),
                                      _p(dQ), _p(dK), _p(dV)), "orc_attn_bwd_sw")
        return dQ, dK, dV
    _check(load().orc_attn_bwd(_p(Qg), T, G, d, _p(K), _p(V), n_cap, _p(idx_a), K_sel, _p(qp),
                               int(bool(causal)), int(tail[0]), int(tail[1]), scale, _p(dO),
                               _p(dQ), _p(dK), _p(dV)), "orc_attn_bwd")
    return dQ, dK, dV
