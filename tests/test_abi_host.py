"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
declared symbol, and rejects bad arguments with status codes before touching a device."""
import ctypes
import os
import re

import pytest

from hierarchical_latent_key_b200 import build_ext, configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lsa():
    build_ext.build()
    from hierarchical_latent_key_b200 import lsa as mod
    return mod


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(lsa_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lsa):
    lib = ctypes.CDLL(lsa.LIBRARY_PATH)
    syms = declared_symbols()
    assert len(syms) >= 12
    for s in syms:
        assert hasattr(lib, s), s


def test_version_and_strerror(lsa):
    assert lsa.lsa_version() == 1
    for code in range(7):
        assert lsa.lsa_strerror(code)
    assert lsa.lsa_strerror(99) == "unknown status"


@pytest.mark.parametrize("kw,code", [
    (dict(n_heads=0), 2), (dict(r=48), 2), (dict(branching=(16, 1)), 2), (dict(branching=(513,)), 2), (dict(branching=(16, 17)), 2),
    (dict(leaf_size=4), 2), (dict(branching=(16,) * 9), 2), (dict(branching=(16,) * 7, leaf_size=64), 2), (dict(n_heads=4, branching=(16,) * 6), 2),
])
def test_describe_rejects(lsa, kw, code):
    args = dict(n_heads=2, r=64, branching=(16, 16), leaf_size=64)
    args.update(kw)
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_tree_describe(args["n_heads"], args["r"], args["branching"], args["leaf_size"])
    assert e.value.code == code


def test_describe_layout(lsa):
    d = lsa.lsa_tree_describe(8, 64, (8, 16, 16, 16, 5), 64)
    assert d.n_tree == 10485760
    assert [d.nodes[l] for l in range(5)] == [8, 128, 2048, 32768, 163840]
    offs = [d.off_centroids[l] for l in range(5)] + [d.off_min_pos[l] for l in range(5)] + [d.off_leaf_index]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    assert d.bytes >= d.off_leaf_index + 8 * d.n_tree * 4


@pytest.mark.parametrize("name", ["decode_128k", "prefill_1m", "decode_10m"])
def test_index_is_about_two_percent_of_kv(lsa, name):
    """The pages put the index at about 2% of the KV cache; the layout here lands near it."""
    c = configs.get(name)
    d = lsa.lsa_tree_describe(c.Hkv, c.r, c.branching, c.leaf)
    kv_bytes = 2 * c.Hkv * c.n * c.d * 2
    assert 0.005 <= d.bytes / kv_bytes <= 0.03, d.bytes / kv_bytes


def test_workspace_queries(lsa):
    d = lsa.lsa_tree_describe(2, 64, (16, 16, 8), 64)
    assert lsa.lsa_build_workspace_bytes(d, 128) > 2 * 2 * 131072 * 64 * 4
    with pytest.raises(lsa.LsaError):
        lsa.lsa_build_workspace_bytes(d, 96)
    assert lsa.lsa_attn_workspace_bytes(4096, 32, 8, 128, 2048, 0) == 0     # enough units: no split
    assert lsa.lsa_attn_workspace_bytes(1, 32, 8, 128, 2048, 64) > 0       # decode: split partials


def test_workspace_of_the_next_rows(lsa):
    """Sizes at the 1M prefill geometry: the sink/window pass adds only its per-(query, head)
    output and LSE; the partials are T * Hq * n_leaves * d bf16; an update on append needs the
    subtree's buffer and its build workspace."""
    import torch
    d = lsa.lsa_tree_describe(8, 64, (16, 16, 16, 4), 64)
    T, Hq, B = 4096, 32, 32
    base = lsa.lsa_tree_attn_workspace_bytes(d, T, Hq, 128, torch.bfloat16, B)
    sw = lsa.lsa_tree_attn_sw_workspace_bytes(d, T, Hq, 128, torch.bfloat16, B, 16, 512)
    assert base >= T * Hq * B * 128 * 2
    assert sw - base == T * Hq * (128 * 2 + 4)
    sub = lsa.lsa_tree_describe(8, 64, (16, 16, 4), 64)
    assert lsa.lsa_tree_append_workspace_bytes(d, 128) >= sub.bytes + lsa.lsa_build_workspace_bytes(sub, 128)


def test_calls_validate_before_launch(lsa):
    """Bad arguments come back as status codes; no device is needed to see them."""
    import torch
    L = lsa._lib
    d = lsa.lsa_tree_describe(1, 16, (16, 16), 16)
    bm = (ctypes.c_int32 * 8)(4, 65)
    rc = L.lsa_select(ctypes.byref(d), None, None, 4, 1, 64, 0, None, ctypes.cast(bm, ctypes.c_void_p),
                      None, None, None, None, None, None, None)
    assert rc == lsa.LSA_ERR_SHAPE and b"beam[1]" in L.lsa_last_error()
    bm = (ctypes.c_int32 * 8)(4, 8)
    rc = L.lsa_select(ctypes.byref(d), None, None, 4, 1, 64, 0, None, ctypes.cast(bm, ctypes.c_void_p),
                      None, None, None, None, None, None, None)
    assert rc == lsa.LSA_ERR_INVALID_ARG
    d2 = lsa.lsa_tree_describe(2, 16, (16, 16), 16)
    rc = L.lsa_select(ctypes.byref(d2), None, None, 4, 3, 64, 0, None, ctypes.cast(bm, ctypes.c_void_p),
                      None, None, None, None, None, None, None)
    assert rc == lsa.LSA_ERR_SHAPE
    for pool in (0, 3, 32):   # pool must be >= 1 and divide leaf_size (16)
        rc = L.lsa_build_tree_pooled(ctypes.byref(d), None, None, 4096, 64, 1, None, pool, 1, 0, None, 0, None,
                                     None, None)
        assert rc == lsa.LSA_ERR_SHAPE and b"pool" in L.lsa_last_error()
    # the top level may grow to 512 through lsa_tree_append; the k-means build splits <= 16 ways
    wide = lsa.lsa_tree_describe(1, 16, (17, 16), 16)
    assert wide.nodes[0] == 17 and wide.n_tree == 17 * 16 * 16
    with pytest.raises(lsa.LsaError):
        lsa.lsa_tree_describe(1, 16, (513, 2), 16)
    with pytest.raises(lsa.LsaError):
        lsa.lsa_tree_describe(1, 16, (16, 17), 16)
    rc = L.lsa_build_tree(ctypes.byref(wide), None, None, 1 << 20, 64, 1, None, 1, 0, None, 0, None, None, None)
    assert rc == lsa.LSA_ERR_SHAPE and b"16 ways" in L.lsa_last_error()
    # append: grown must be the same tree with branching[0] + 1, and levels >= 2
    grown = lsa.lsa_tree_describe(1, 16, (17, 16), 16)
    other = lsa.lsa_tree_describe(1, 16, (18, 16), 16)
    base = lsa.lsa_tree_describe(1, 16, (16, 16), 16)
    P16 = ctypes.c_void_p(16)
    rc = L.lsa_tree_append(ctypes.byref(base), P16, ctypes.byref(other), P16, P16, 1 << 20, 64, 1, P16, 1, 0, None,
                           0, None, None, None)
    assert rc == lsa.LSA_ERR_SHAPE and b"branching[0] + 1" in L.lsa_last_error()
    flat1 = lsa.lsa_tree_describe(1, 16, (16,), 16)
    n = ctypes.c_size_t()
    assert L.lsa_tree_append_workspace_bytes(ctypes.byref(flat1), 64, ctypes.byref(n)) == lsa.LSA_ERR_SHAPE
    assert L.lsa_tree_append_workspace_bytes(ctypes.byref(base), 64, ctypes.byref(n)) == lsa.LSA_OK
    P32 = ctypes.c_void_p(32)
    rc = L.lsa_tree_append(ctypes.byref(base), P16, ctypes.byref(grown), P16, P16, 1 << 20, 64, 1, P16, 1, 0, P16,
                           n.value, None, None, None)
    assert rc == lsa.LSA_ERR_INVALID_ARG and b"not be tree_mem" in L.lsa_last_error()
    rc = L.lsa_tree_append(ctypes.byref(base), P16, ctypes.byref(grown), P32, P16, 1 << 20, 64, 1, P16, 1, 0, P16,
                           n.value - 1, None, None, None)
    assert rc == lsa.LSA_ERR_WORKSPACE
    bad = lsa.lsa_tree_desc.from_buffer_copy(d)
    bad.off_leaf_index += 256
    n = ctypes.c_size_t()
    assert L.lsa_build_workspace_bytes(ctypes.byref(bad), 64, ctypes.byref(n)) == lsa.LSA_ERR_INVALID_ARG
    # attention: 3 query heads per group, bad tail, causal without positions, missing workspace
    args = lambda **kw: dict(dict(Q=1, T=2, Hq=8, K=1, V=1, H=2, n_cap=100, d=128, dt=1, idx=1, K_sel=16,
                                  qp=None, causal=0, tb=0, te=0), **kw)
    def call(a):
        P = lambda v: ctypes.c_void_p(16) if v else None
        return L.lsa_sparse_attn(P(a["Q"]), a["T"], a["Hq"], P(a["K"]), P(a["V"]), a["H"], a["n_cap"], a["d"],
                                 a["dt"], P(a["idx"]), a["K_sel"], P(a["qp"]), a["causal"], a["tb"], a["te"],
                                 0.1, ctypes.c_void_p(16), ctypes.c_void_p(16), None, 0, None, None)
    assert call(args(Hq=6)) == lsa.LSA_ERR_SHAPE
    assert call(args(tb=50, te=120)) == lsa.LSA_ERR_SHAPE
    assert call(args(causal=1)) == lsa.LSA_ERR_INVALID_ARG
    assert call(args(dt=7)) == lsa.LSA_ERR_INVALID_ARG
    assert call(args(d=96)) == lsa.LSA_ERR_SHAPE
    assert call(args(T=1, K_sel=2048)) == lsa.LSA_ERR_WORKSPACE
    assert call(args(T=0)) == lsa.LSA_OK


def test_attn_no_queries(lsa):
    """A call without queries needs no workspace and launches nothing, for every key count."""
    L = lsa._lib
    assert lsa.lsa_attn_workspace_bytes(0, 32, 8, 128, 2048, 0) == 0
    assert lsa.lsa_attn_workspace_bytes(0, 32, 8, 128, 2048, 256) == 0
    P = ctypes.c_void_p(16)
    rc = L.lsa_sparse_attn_noalloc(P, 0, 32, P, P, 8, 1 << 20, 128, 1, P, 2048, None, 0, 0, 0, 0.1, P, P, None, None)
    assert rc == lsa.LSA_OK
    # the same call with an invalid argument is still rejected before anything else
    rc = L.lsa_sparse_attn_noalloc(P, 0, 30, P, P, 8, 1 << 20, 128, 1, P, 2048, None, 0, 0, 0, 0.1, P, P, None, None)
    assert rc == lsa.LSA_ERR_SHAPE


def test_project_keys_rejects(lsa):
    L = lsa._lib
    P = ctypes.c_void_p(16)
    assert L.lsa_project_keys(None, 2, 100, 128, 1, P, 64, 10, P, None, None) == lsa.LSA_ERR_INVALID_ARG
    assert L.lsa_project_keys(P, 2, 100, 128, 9, P, 64, 10, P, None, None) == lsa.LSA_ERR_INVALID_ARG
    assert L.lsa_project_keys(P, 2, 100, 96, 1, P, 64, 10, P, None, None) == lsa.LSA_ERR_SHAPE
    assert L.lsa_project_keys(P, 2, 100, 128, 1, P, 48, 10, P, None, None) == lsa.LSA_ERR_SHAPE
    assert L.lsa_project_keys(P, 2, 100, 128, 1, P, 64, 101, P, None, None) == lsa.LSA_ERR_SHAPE
    assert L.lsa_project_keys(P, 0, 100, 128, 1, P, 64, 10, P, None, None) == lsa.LSA_ERR_SHAPE


def test_balanced_assign_rejects(lsa):
    L = lsa._lib
    P = ctypes.c_void_p(16)
    n = ctypes.c_size_t()
    assert L.lsa_balanced_assign_workspace_bytes(4, 64, 4, ctypes.byref(n)) == lsa.LSA_OK and n.value > 0
    assert L.lsa_balanced_assign_workspace_bytes(4, 66, 4, ctypes.byref(n)) == lsa.LSA_ERR_SHAPE
    assert L.lsa_balanced_assign_workspace_bytes(4, 64, 17, ctypes.byref(n)) == lsa.LSA_ERR_SHAPE
    assert L.lsa_balanced_assign_workspace_bytes(0, 64, 4, ctypes.byref(n)) == lsa.LSA_ERR_SHAPE
    assert L.lsa_balanced_assign(P, P, 4, 64, 4, 48, 0, P, P, 1 << 20, None, None) == lsa.LSA_ERR_SHAPE
    assert L.lsa_balanced_assign(P, P, 4, 64, 4, 64, -1, P, P, 1 << 20, None, None) == lsa.LSA_ERR_INVALID_ARG
    assert L.lsa_balanced_assign(None, P, 4, 64, 4, 64, 0, P, P, 1 << 20, None, None) == lsa.LSA_ERR_INVALID_ARG
    assert L.lsa_balanced_assign(P, P, 4, 64, 4, 64, 0, P, P, 16, None, None) == lsa.LSA_ERR_WORKSPACE


def test_decode_step_rejects(lsa):
    L = lsa._lib
    P = ctypes.c_void_p(16)
    d = lsa.lsa_tree_describe(2, 64, (16, 16, 8), 64)
    beam = (ctypes.c_int32 * 3)(8, 32, 32)
    n = ctypes.c_size_t()
    assert L.lsa_decode_step_workspace_bytes(ctypes.byref(d), 8, 128, beam, 256, ctypes.byref(n)) == lsa.LSA_OK
    need = n.value
    # 32 leaves + 4 tail splits of 64 keys, 2 heads x 4 query heads x 130 floats each
    assert need >= 2 * 36 * 4 * 130 * 4

    def call(pos, tail_begin, ws=need, Kr=P, Vr=P, Hq=8):
        return L.lsa_decode_step(ctypes.byref(d), P, P, beam, P, P, d.n_tree + 256, 128, 1, P, Hq, Kr, Vr, pos,
                                 tail_begin, 0.1, P, P, None, P, ws, None, None)
    nt = d.n_tree
    assert call(nt - 2, nt) == lsa.LSA_ERR_SHAPE            # token before the last indexed key
    assert call(nt + 3, nt - 1) == lsa.LSA_ERR_SHAPE        # tail overlapping the index
    assert call(nt + 3, nt + 5) == lsa.LSA_ERR_SHAPE        # tail past the token
    assert call(nt + 256, nt) == lsa.LSA_ERR_SHAPE          # pos outside the cache
    assert call(nt + 3, nt, Vr=None) == lsa.LSA_ERR_INVALID_ARG
    assert call(nt + 3, nt, Hq=12) == lsa.LSA_ERR_SHAPE
    assert call(nt + 3, nt, ws=16) == lsa.LSA_ERR_WORKSPACE


def test_select_batched_rejects(lsa):
    """Host-side checks of the batched search: workspace sizes (growing with T, 0 for no
    queries), the batch limit, a missing or short workspace, and a bad beam."""
    L = lsa._lib
    P = ctypes.c_void_p(16)
    d = lsa.lsa_tree_describe(8, 64, (16, 16, 16, 4), 64)
    beam = (ctypes.c_int32 * 4)(8, 32, 32, 32)
    n = ctypes.c_size_t()
    sizes = []
    for T in (0, 1, 4096, 1 << 26):
        assert L.lsa_select_batched_workspace_bytes(ctypes.byref(d), T, beam, ctypes.byref(n)) == lsa.LSA_OK
        sizes.append(n.value)
    assert sizes[0] == 0 and 0 < sizes[1] < sizes[2] < sizes[3]
    # 4096 queries x 8 groups: the candidate lists alone hold 512 keys of 8 bytes per walk
    assert sizes[2] >= 4096 * 8 * 512 * 8
    assert L.lsa_select_batched_workspace_bytes(ctypes.byref(d), (1 << 26) + 1, beam, ctypes.byref(n)) == \
        lsa.LSA_ERR_SHAPE
    assert L.lsa_select_batched_workspace_bytes(ctypes.byref(d), 16, beam, None) == lsa.LSA_ERR_INVALID_ARG
    bad = (ctypes.c_int32 * 4)(8, 32, 33, 32)
    assert L.lsa_select_batched_workspace_bytes(ctypes.byref(d), 16, bad, ctypes.byref(n)) == lsa.LSA_ERR_SHAPE

    def call(T, ws, ws_bytes):
        return L.lsa_select_batched(ctypes.byref(d), P, P, T, 32, 128, lsa.LSA_BF16, P, beam, None, P, None, None,
                                    None, ws, ws_bytes, None, None)
    assert L.lsa_select_batched_workspace_bytes(ctypes.byref(d), 64, beam, ctypes.byref(n)) == lsa.LSA_OK
    assert call(64, None, 0) == lsa.LSA_ERR_WORKSPACE
    assert call(64, P, n.value - 1) == lsa.LSA_ERR_WORKSPACE
    assert call((1 << 26) + 1, P, 1 << 40) == lsa.LSA_ERR_SHAPE
    assert call(0, None, 0) == lsa.LSA_OK
