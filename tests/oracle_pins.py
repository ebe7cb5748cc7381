"""Pins of the CPU oracle to things other than itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with an
external fact: published generator vectors, brute-force enumeration, closed forms,
library routines (numpy, torch SDPA and autograd) or finite differences.  They are
collected by ``test_oracle_pins.py`` and re-run against deliberately broken copies of
the oracle by ``test_oracle_mutants.py`` (every planted mistake must trip a pin).

Special cases used (from the method's statement on the pages):
  * flat search scores every cluster centroid, so a hierarchical walk whose beam keeps
    every node above the leaf level equals brute-force top-B over all leaves;
  * sparse attention over every key is full softmax attention;
  * a centroid is the mean of its members (k-means), and with balanced children a
    parent centroid is the mean of its children's centroids.
"""
from __future__ import annotations

import itertools
import os

import numpy as np
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------
# small deterministic fixtures
# ---------------------------------------------------------------------------

def _mixture(rng, n, d, comps, sigma=0.3):
    c = rng.standard_normal((comps, d))
    c /= np.linalg.norm(c, axis=1, keepdims=True)
    return c[rng.integers(0, comps, n)] + sigma * rng.standard_normal((n, d))


def tiny_tree_case(seed=0, n=1024, d=32, r=8, branching=(8, 8), leaf=16, iters=4):
    rng = np.random.default_rng(seed)
    K = _mixture(rng, n, d, 16)
    W = rng.standard_normal((d, r)) / np.sqrt(d)
    Z = K @ W
    tree = orc.build_tree(orc.project(K, W), branching, leaf, iters, seed=seed, trace=True)
    return K, W, Z, tree


# ---------------------------------------------------------------------------
# generator
# ---------------------------------------------------------------------------

def pin_splitmix64_published_vectors():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "splitmix64.txt")) if l[0] != "#"]
    assert rows
    for seed, i, val in rows:
        assert orc.splitmix64_at(int(seed), int(i)) == int(val), (seed, i)


def pin_init_rule():
    """Child j of a segment starts at the member with the j-th smallest init hash."""
    rng = np.random.default_rng(3)
    pos = np.sort(rng.choice(5000, 40, replace=False))
    Zs = rng.standard_normal((40, 5))
    for level, seed in ((0, 0), (2, 77)):
        h = np.array([orc.init_hash(seed, level, int(p)) for p in pos], dtype=np.uint64)
        want = Zs[np.argsort(h, kind="stable")[:6]]
        got = orc.level_init(Zs, pos, 6, seed, level)
        np.testing.assert_array_equal(got, want)
    # the hash of (seed, level, pos) is the generator output `pos` of the stream whose
    # state is output `level` of the stream seeded with `seed`
    assert orc.init_hash(0, 0, 0) == orc.splitmix64_at(orc.splitmix64_at(0, 0), 0)
    assert orc.init_hash(5, 3, 11) == orc.splitmix64_at(orc.splitmix64_at(5, 3), 11)


# ---------------------------------------------------------------------------
# projection
# ---------------------------------------------------------------------------

def pin_projection_matches_numpy():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((37, 24))
    W = rng.standard_normal((24, 7))
    np.testing.assert_allclose(orc.project(X, W), X @ W, rtol=1e-12, atol=1e-12)
    Qg = rng.standard_normal((9, 4, 24))
    np.testing.assert_allclose(orc.query_latent(Qg, W), Qg.mean(axis=1) @ W, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# balanced assignment
# ---------------------------------------------------------------------------

def _pair_key(D, pos, i, c):
    return (D[i, c], pos[i], c)


def _is_stable(D, pos, a, b):
    m = len(a)
    for i in range(m):
        for c in range(b):
            if c == a[i]:
                continue
            if _pair_key(D, pos, i, c) >= _pair_key(D, pos, i, a[i]):
                continue                          # i does not prefer c
            members = [j for j in range(m) if a[j] == c]
            if any((D[i, c], pos[i]) < (D[j, c], pos[j]) for j in members):
                return False                      # (i, c) blocks
    return True


def _all_balanced(m, b):
    cap = m // b
    for lab in itertools.product(range(b), repeat=m):
        if all(lab.count(c) == cap for c in range(b)):
            yield np.array(lab)


def pin_balanced_assign_bruteforce():
    rng = np.random.default_rng(7)
    for trial in range(24):
        b = (2, 3, 4)[trial % 3]
        m = b * (2 if b > 2 else 3 + trial % 2)
        if trial % 4 == 0:  # coarse integer distances: many exact ties
            D = rng.integers(0, 3, (m, b)).astype(float)
        else:
            D = rng.random((m, b))
        pos = np.sort(rng.choice(100, m, replace=False))
        stable = [a for a in _all_balanced(m, b) if _is_stable(D, pos, a, b)]
        assert len(stable) == 1, (trial, len(stable))
        np.testing.assert_array_equal(orc.balanced_assign(D, pos), stable[0])


def _deferred_acceptance(D, pos, b):
    """Key-proposing deferred acceptance, written independently of the oracle."""
    m = D.shape[0]
    cap = m // b
    pref = [sorted(range(b), key=lambda c, i=i: (D[i, c], c)) for i in range(m)]
    nxt = [0] * m
    held = {c: [] for c in range(b)}
    free = list(range(m))
    while free:
        i = free.pop()
        c = pref[i][nxt[i]]
        nxt[i] += 1
        held[c].append(i)
        if len(held[c]) > cap:
            held[c].sort(key=lambda j: (D[j, c], pos[j]))
            free.append(held[c].pop())
    a = np.empty(m, int)
    for c, js in held.items():
        a[js] = c
    return a


def pin_balanced_assign_vs_deferred_acceptance():
    rng = np.random.default_rng(11)
    for m, b in ((64, 4), (240, 8), (256, 16)):
        D = rng.random((m, b)) ** 2
        pos = np.sort(rng.choice(10 * m, m, replace=False))
        a = orc.balanced_assign(D, pos)
        np.testing.assert_array_equal(np.bincount(a, minlength=b), np.full(b, m // b))
        np.testing.assert_array_equal(a, _deferred_acceptance(D, pos, b))


def pin_distances_closed_form():
    rng = np.random.default_rng(5)
    Z, mu = rng.standard_normal((20, 6)), rng.standard_normal((3, 6))
    want = ((Z[:, None, :] - mu[None]) ** 2).sum(-1)
    np.testing.assert_allclose(orc.distances(Z, mu), want, rtol=1e-12)
    a = rng.integers(0, 3, 20)
    a[:3] = [0, 1, 2]
    want_mu = np.stack([Z[a == c].mean(0) for c in range(3)])
    np.testing.assert_allclose(orc.means(Z, a, 3), want_mu, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# tree build
# ---------------------------------------------------------------------------

def pin_tree_invariants():
    K, W, Z, tree = tiny_tree_case()
    n, L, leaf = Z.shape[0], len(tree.branching), tree.leaf_size
    li = tree.leaf_index.astype(np.int64)
    np.testing.assert_array_equal(np.sort(li), np.arange(n))            # permutation
    leaves = li.reshape(-1, leaf)
    assert np.all(np.diff(leaves, axis=1) > 0)                           # ascending in a leaf
    # members of every node at every level, from the leaf partition
    for l in range(L):
        per_node = n // tree.nodes[l]
        groups = li.reshape(tree.nodes[l], per_node)                     # node-major leaf order
        mu = Z[groups].mean(axis=1)
        np.testing.assert_allclose(tree.centroids[l], mu, rtol=1e-10, atol=1e-12)
        np.testing.assert_array_equal(tree.min_pos[l], groups.min(axis=1))
        if l > 0:
            b = tree.branching[l]
            parent = tree.centroids[l].reshape(-1, b, Z.shape[1]).mean(axis=1)
            np.testing.assert_allclose(parent, tree.centroids[l - 1], rtol=1e-10, atol=1e-12)
    # the trace's last assignment of each level is the partition above
    for l in range(L):
        per_node = n // tree.nodes[l]
        node_of = np.empty(n, np.int64)
        node_of[li] = np.repeat(np.arange(tree.nodes[l]), per_node)
        np.testing.assert_array_equal(tree.trace[l, -1], node_of)


def pin_tree_first_step_from_init():
    """Level 0's first assignment uses the seeded start and the stable balanced rule."""
    K, W, Z, tree = tiny_tree_case()
    n = Z.shape[0]
    b = tree.branching[0]
    pos = np.arange(n)
    h = np.array([orc.init_hash(0, 0, int(p)) for p in pos], dtype=np.uint64)
    mu0 = Z[np.argsort(h)[:b]]
    D = ((Z[:, None, :] - mu0[None]) ** 2).sum(-1)
    a = _deferred_acceptance_fast(D, pos, b)
    np.testing.assert_array_equal(tree.trace[0, 0], a)


def _deferred_acceptance_fast(D, pos, b):
    """Round-synchronous deferred acceptance (numpy), independent of the oracle."""
    m = D.shape[0]
    cap = m // b
    order = np.lexsort((np.broadcast_to(np.arange(b), D.shape), D), axis=1)
    ptr = np.zeros(m, np.int64)
    rows = np.arange(m)
    while True:
        ch = order[rows, ptr]
        moved = False
        for c in range(b):
            w = np.nonzero(ch == c)[0]
            if len(w) > cap:
                o = np.lexsort((pos[w], D[w, c]))
                ptr[w[o[cap:]]] += 1
                moved = True
        if not moved:
            return ch


def _numpy_build(Z, branching, leaf, iters, seed):
    """The whole top-down build restated in numpy: per level, every parent's members (in
    ascending position) start from the seeded picks, then `iters` rounds of (squared
    distances, stable balanced assignment by the independent deferred-acceptance solver,
    member means).  Returns (centroids per level, leaf_index, trace [L, iters, n])."""
    n, r = Z.shape
    L = len(branching)
    members = [np.arange(n)]
    trace = np.full((L, iters, n), -1, np.int64)
    cents = []
    for l, b in enumerate(branching):
        nxt, cl = [], []
        for s, pos in enumerate(members):
            Zs = Z[pos]
            h = np.array([orc.init_hash(seed, l, int(p)) for p in pos], dtype=np.uint64)
            mu = Zs[np.argsort(h, kind="stable")[:b]]
            for t in range(iters):
                D = ((Zs[:, None, :] - mu[None]) ** 2).sum(-1)
                a = _deferred_acceptance_fast(D, pos, b)
                trace[l, t, pos] = s * b + a
                mu = np.stack([Zs[a == c].mean(axis=0) for c in range(b)])
            cl.append(mu)
            nxt += [pos[a == c] for c in range(b)]
        members = nxt
        cents.append(np.concatenate(cl))
    return cents, np.concatenate(members), trace


def pin_tree_independent_rebuild():
    """The oracle's composite build equals the numpy restatement of the same steps
    (kongchang.com, "How LSA Sidesteps Per-Key Scoring with Hierarchical Clustering":
    the tree is built like hierarchical k-means, root = all keys), on two trees: the
    two-level tiny case and a three-level one, every round of every level compared."""
    for kw in (dict(), dict(seed=5, branching=(4, 4, 4), leaf=16, iters=5)):
        K, W, Z, tree = tiny_tree_case(**kw)
        seed = kw.get("seed", 0)
        iters = kw.get("iters", 4)
        cents, li, tr = _numpy_build(Z, tree.branching, tree.leaf_size, iters, seed)
        np.testing.assert_array_equal(tree.trace, tr)
        np.testing.assert_array_equal(tree.leaf_index, li)
        for l in range(len(tree.branching)):
            np.testing.assert_allclose(tree.centroids[l], cents[l], rtol=1e-10, atol=1e-12)


def pin_tree_rounds_from_trace():
    """Every k-means round of every level follows from the round before it: round 0 of
    level l from the seeded picks inside each level-(l-1) node, round t > 0 from the
    numpy means of round t-1's partition; each assignment is the stable balanced one
    (independent solver).  Also checks that exactly `iters` rounds ran per level."""
    K, W, Z, tree = tiny_tree_case(seed=7, branching=(4, 4, 4), leaf=16, iters=6)
    n, L, iters = Z.shape[0], len(tree.branching), tree.trace.shape[1]
    assert iters == 6
    parent = np.zeros(n, np.int64)
    for l in range(L):
        b = tree.branching[l]
        for t in range(iters):
            for s in np.unique(parent):
                pos = np.nonzero(parent == s)[0]
                Zs = Z[pos]
                if t == 0:
                    h = np.array([orc.init_hash(7, l, int(p)) for p in pos], dtype=np.uint64)
                    mu = Zs[np.argsort(h, kind="stable")[:b]]
                else:
                    prev = tree.trace[l, t - 1, pos] - s * b
                    assert prev.min() >= 0 and prev.max() < b
                    mu = np.stack([Zs[prev == c].mean(axis=0) for c in range(b)])
                D = ((Zs[:, None, :] - mu[None]) ** 2).sum(-1)
                a = _deferred_acceptance_fast(D, pos, b)
                np.testing.assert_array_equal(tree.trace[l, t, pos], s * b + a, err_msg=f"level {l} round {t}")
        parent = tree.trace[l, iters - 1].astype(np.int64)


def pin_tree_deterministic_and_seeded():
    _, _, Z, t1 = tiny_tree_case()
    t2 = orc.build_tree(Z, t1.branching, t1.leaf_size, 4, seed=0)
    np.testing.assert_array_equal(t1.leaf_index, t2.leaf_index)
    t3 = orc.build_tree(Z, t1.branching, t1.leaf_size, 4, seed=1)
    assert not np.array_equal(t1.leaf_index, t3.leaf_index)


# ---------------------------------------------------------------------------
# hierarchical search
# ---------------------------------------------------------------------------

def _flat_topB(qlat, tree, B, q_pos=None):
    """Brute force: score every leaf centroid, keep the B best (score desc, id asc)."""
    leafc = tree.centroids[-1]
    T = qlat.shape[0]
    out = np.full((T, B * tree.leaf_size), -1, np.int64)
    for t in range(T):
        s = leafc @ qlat[t]
        ids = np.arange(len(s))
        if q_pos is not None:
            keep = tree.min_pos[-1] <= q_pos[t]
            s, ids = s[keep], ids[keep]
        o = np.lexsort((ids, -s))[:B]
        keys = tree.leaf_index.reshape(-1, tree.leaf_size)[ids[o]].reshape(-1)
        out[t, :len(keys)] = keys
    return out


def pin_select_full_beam_equals_flat():
    K, W, Z, tree = tiny_tree_case()
    rng = np.random.default_rng(2)
    q = rng.standard_normal((20, 3, K.shape[1]))
    qlat = q.mean(axis=1) @ W
    full = [tree.nodes[l] for l in range(len(tree.nodes) - 1)]
    for B in (1, 5, 12):
        idx, bt, scored = orc.select(qlat, tree, full + [B], trace=True)
        np.testing.assert_array_equal(idx, _flat_topB(qlat, tree, B))
        assert np.all(scored == sum(tree.nodes))
    # causal: a leaf is reachable with a full beam iff its smallest position is visible
    q_pos = rng.integers(0, Z.shape[0], 20)
    idx, bt, _ = orc.select(qlat, tree, full + [7], q_pos=q_pos, trace=True)
    np.testing.assert_array_equal(idx, _flat_topB(qlat, tree, 7, q_pos))
    # the flat-search entry is that walk: same keys, and leaves in (score desc, id asc) order
    idx_f, lv = orc.select_flat(qlat, tree, 7, q_pos=q_pos)
    np.testing.assert_array_equal(idx_f, _flat_topB(qlat, tree, 7, q_pos))
    li = tree.leaf_index.reshape(-1, tree.leaf_size)
    for t in range(qlat.shape[0]):
        got = lv[t][lv[t] >= 0]
        np.testing.assert_array_equal(li[got].reshape(-1), idx_f[t][:len(got) * tree.leaf_size])
        s = tree.centroids[-1][got] @ qlat[t]
        assert np.all(np.diff(s) <= 0)


def pin_select_beam_walk():
    """Narrow beams: counts, ranking and parent/child structure of every kept node."""
    K, W, Z, tree = tiny_tree_case()
    rng = np.random.default_rng(4)
    qlat = rng.standard_normal((16, W.shape[1]))
    beam = [3, 5]
    idx, bt, scored = orc.select(qlat, tree, beam, trace=True)
    b1 = tree.branching[1]
    assert np.all(scored == tree.nodes[0] + beam[0] * b1)
    for t in range(16):
        s0 = tree.centroids[0] @ qlat[t]
        top0 = np.lexsort((np.arange(len(s0)), -s0))[:beam[0]]
        np.testing.assert_array_equal(bt[0, t, :beam[0]], top0)
        cand = (top0[:, None] * b1 + np.arange(b1)).reshape(-1)
        s1 = tree.centroids[1][cand] @ qlat[t]
        top1 = cand[np.lexsort((cand, -s1))[:beam[1]]]
        np.testing.assert_array_equal(bt[1, t, :beam[1]], top1)
        want = tree.leaf_index.reshape(-1, tree.leaf_size)[top1].reshape(-1)
        np.testing.assert_array_equal(idx[t], want)
    # causal eligibility, brute force: every kept node's smallest position is visible,
    # and no eligible child of a kept parent that scored higher was dropped
    q_pos = rng.integers(0, Z.shape[0] // 3, 16)
    idx, bt, _ = orc.select(qlat, tree, beam, q_pos=q_pos, trace=True)
    for t in range(16):
        for l in range(2):
            kept = bt[l, t][bt[l, t] >= 0]
            assert np.all(tree.min_pos[l][kept] <= q_pos[t])
        elig0 = np.nonzero(tree.min_pos[0] <= q_pos[t])[0]
        s0 = tree.centroids[0][elig0] @ qlat[t]
        top0 = elig0[np.lexsort((elig0, -s0))[:beam[0]]]
        np.testing.assert_array_equal(bt[0, t][bt[0, t] >= 0], top0)
        valid = idx[t][idx[t] >= 0]
        assert len(valid) % tree.leaf_size == 0 and len(valid) > 0


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _sdpa_dense(Qg, K, V, mask, scale):
    """torch SDPA in float64 on CPU: Qg [T,G,d], K/V [n,d], mask [T,n] bool (True=visible)."""
    q = torch.from_numpy(Qg).permute(1, 0, 2)[None]           # [1, G, T, d]
    k = torch.from_numpy(K)[None, None].expand(1, Qg.shape[1], -1, -1)
    v = torch.from_numpy(V)[None, None].expand(1, Qg.shape[1], -1, -1)
    m = torch.from_numpy(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def _attn_case(seed=0, T=6, G=3, d=16, n=40, K_sel=12):
    rng = np.random.default_rng(seed)
    Qg = rng.standard_normal((T, G, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    idx = np.stack([rng.choice(n - 8, K_sel, replace=False) for _ in range(T)]).astype(np.int32)
    idx[:, -2:] = -1
    return rng, Qg, K, V, idx


def _mask_from(idx, n, tail, q_pos, causal):
    T = idx.shape[0]
    mask = np.zeros((T, n), bool)
    for t in range(T):
        sel = idx[t][idx[t] >= 0]
        mask[t, sel] = True
        mask[t, tail[0]:tail[1]] = True
        if causal:
            mask[t, q_pos[t] + 1:] = False
    return mask


def pin_attention_equals_sdpa():
    rng, Qg, K, V, idx = _attn_case()
    n, d = K.shape
    scale = 1 / np.sqrt(d)
    # every key selected (through the index list and a tail) = full attention
    all_idx = np.tile(np.arange(n - 8, dtype=np.int32), (Qg.shape[0], 1))
    O, LSE = orc.attn_fwd(Qg, K, V, all_idx, tail=(n - 8, n), scale=scale)
    full = _sdpa_dense(Qg, K, V, np.ones((Qg.shape[0], n), bool), scale)
    np.testing.assert_allclose(O, full, rtol=1e-10, atol=1e-12)
    lse_want = np.log(np.exp(scale * np.einsum("tgd,nd->tgn", Qg, K)).sum(-1))
    np.testing.assert_allclose(LSE, lse_want, rtol=1e-10)
    # sparse + tail + causal against a boolean mask
    q_pos = rng.integers(n // 2, n, Qg.shape[0]).astype(np.int32)
    for causal in (False, True):
        O, _ = orc.attn_fwd(Qg, K, V, idx, q_pos=q_pos, causal=causal, tail=(n - 8, n), scale=scale)
        mask = _mask_from(idx, n, (n - 8, n), q_pos, causal)
        np.testing.assert_allclose(O, _sdpa_dense(Qg, K, V, mask, scale), rtol=1e-10, atol=1e-12)


def pin_attention_special_cases():
    rng, Qg, K, V, idx = _attn_case(1)
    T = Qg.shape[0]
    one = np.full((T, 3), -1, np.int32)
    one[:, 1] = np.arange(T) * 2
    O, LSE = orc.attn_fwd(Qg, K, V, one, scale=0.7)
    for t in range(T):
        np.testing.assert_allclose(O[t], np.broadcast_to(V[2 * t], O[t].shape), rtol=1e-12)
        np.testing.assert_allclose(LSE[t], 0.7 * Qg[t] @ K[2 * t], rtol=1e-12)
    perm = idx[:, rng.permutation(idx.shape[1])]
    a, _ = orc.attn_fwd(Qg, K, V, idx)
    b, _ = orc.attn_fwd(Qg, K, V, perm)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    none = np.full((T, 4), -1, np.int32)
    O, LSE = orc.attn_fwd(Qg, K, V, none)
    assert np.all(O == 0) and np.all(np.isneginf(LSE))


def pin_backward_autograd():
    rng, Qg, K, V, idx = _attn_case(2)
    n, d = K.shape
    q_pos = rng.integers(n // 2, n, Qg.shape[0]).astype(np.int32)
    dO = rng.standard_normal(Qg.shape)
    scale = 0.3
    dQ, dK, dV = orc.attn_bwd(Qg, K, V, idx, dO, q_pos=q_pos, causal=True, tail=(n - 8, n), scale=scale)
    mask = torch.from_numpy(_mask_from(idx, n, (n - 8, n), q_pos, True))
    q = torch.from_numpy(Qg).requires_grad_()
    k = torch.from_numpy(K).requires_grad_()
    v = torch.from_numpy(V).requires_grad_()
    s = scale * torch.einsum("tgd,nd->tgn", q, k)
    s = s.masked_fill(~mask[:, None, :], float("-inf"))
    o = torch.einsum("tgn,nd->tgd", torch.softmax(s, -1), v)
    o.backward(torch.from_numpy(dO))
    np.testing.assert_allclose(dQ, q.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dK, k.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dV, v.grad.numpy(), rtol=1e-9, atol=1e-12)


def pin_backward_finite_differences():
    rng, Qg, K, V, idx = _attn_case(3, T=3, G=2, d=6, n=20, K_sel=6)
    dO = rng.standard_normal(Qg.shape)
    dQ, dK, dV = orc.attn_bwd(Qg, K, V, idx, dO)

    def loss(Qx, Kx, Vx):
        O, _ = orc.attn_fwd(Qx, Kx, Vx, idx)
        return float((O * dO).sum())

    eps = 1e-6
    for arr, grad, pick in ((Qg, dQ, (1, 1, 2)), (K, dK, (int(idx[0, 0]), 3)), (V, dV, (int(idx[2, 1]), 0))):
        plus, minus = arr.copy(), arr.copy()
        plus[pick] += eps
        minus[pick] -= eps
        args_p = [Qg, K, V]
        args_m = [Qg, K, V]
        which = 0 if arr is Qg else (1 if arr is K else 2)
        args_p[which], args_m[which] = plus, minus
        fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert abs(fd - grad[pick]) < 1e-6 * max(1.0, abs(fd)), (which, fd, grad[pick])



def _sink_window_mask(idx, n, tail, q_pos, sink, window):
    """Union of the index list, the tail, the first `sink` positions and the `window`
    positions up to q_pos, then the causal cut (bdtechtalks.com, "Latent sparse attention",
    section "How latent sparse attention works": chosen keys plus recent and sink tokens)."""
    m = _mask_from(idx, n, tail, q_pos, True)
    for t in range(idx.shape[0]):
        m[t, :sink] = True
        m[t, max(0, int(q_pos[t]) - window + 1):int(q_pos[t]) + 1] = True
        m[t, int(q_pos[t]) + 1:] = False
    return m


def pin_attention_sink_window():
    rng, Qg, K, V, idx = _attn_case(4)
    T = Qg.shape[0]
    n, d = K.shape
    scale = 1 / np.sqrt(d)
    q_pos = rng.integers(n // 2, n, T).astype(np.int32)
    q_pos[0] = 1                                   # a query before the end of the sink range
    # a window reaching position 0 is full causal attention, whatever the index list says
    O, _ = orc.attn_fwd(Qg, K, V, idx, q_pos=q_pos, causal=True, scale=scale, window=n)
    full = _sdpa_dense(Qg, K, V, np.arange(n)[None, :] <= q_pos[:, None], scale)
    np.testing.assert_allclose(O, full, rtol=1e-10, atol=1e-12)
    # index list + tail + sink + window = SDPA over the union mask
    sink, window = 3, 5
    O, LSE = orc.attn_fwd(Qg, K, V, idx, q_pos=q_pos, causal=True, tail=(n - 8, n), scale=scale, sink=sink,
                          window=window)
    m = _sink_window_mask(idx, n, (n - 8, n), q_pos, sink, window)
    np.testing.assert_allclose(O, _sdpa_dense(Qg, K, V, m, scale), rtol=1e-10, atol=1e-12)
    s = scale * np.einsum("tgd,nd->tgn", Qg, K)
    lse = np.log(np.where(m[:, None, :], np.exp(s), 0.0).sum(-1))
    np.testing.assert_allclose(LSE, lse, rtol=1e-10)
    # a key listed again in the index list (inside the window or the sink) counts once
    extra = np.stack([np.r_[np.arange(q_pos[t] - 2, q_pos[t] + 1).clip(0), [0, 1]] for t in range(T)]).astype(np.int32)
    dup = np.concatenate([idx, extra], 1)
    a, la = orc.attn_fwd(Qg, K, V, idx, q_pos=q_pos, causal=True, scale=scale, sink=sink, window=window)
    b, lb = orc.attn_fwd(Qg, K, V, dup, q_pos=q_pos, causal=True, scale=scale, sink=sink, window=window)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def pin_backward_sink_window_autograd():
    rng, Qg, K, V, idx = _attn_case(5)
    n, d = K.shape
    q_pos = rng.integers(n // 2, n, Qg.shape[0]).astype(np.int32)
    q_pos[1] = 2
    dO = rng.standard_normal(Qg.shape)
    scale, sink, window = 0.4, 2, 6
    dQ, dK, dV = orc.attn_bwd(Qg, K, V, idx, dO, q_pos=q_pos, causal=True, tail=(n - 8, n), scale=scale,
                              sink=sink, window=window)
    mask = torch.from_numpy(_sink_window_mask(idx, n, (n - 8, n), q_pos, sink, window))
    q = torch.from_numpy(Qg).requires_grad_()
    k = torch.from_numpy(K).requires_grad_()
    v = torch.from_numpy(V).requires_grad_()
    sc = (scale * torch.einsum("tgd,nd->tgn", q, k)).masked_fill(~mask[:, None, :], float("-inf"))
    o = torch.einsum("tgn,nd->tgd", torch.softmax(sc, -1), v)
    o.backward(torch.from_numpy(dO))
    np.testing.assert_allclose(dQ, q.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dK, k.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dV, v.grad.numpy(), rtol=1e-9, atol=1e-12)

def pin_tree_pooled():
    """Pooling then clustering (bdtechtalks.com, "How latent sparse attention works"): pool 1 is
    the plain build; with pool p the tree over blocks is the plain build over block means taken
    by numpy; every stored centroid is the mean of the latent rows of the keys its node lists,
    min_pos is a key position, and a leaf is a union of whole aligned blocks."""
    rng = np.random.default_rng(5)
    n, d, r, p, br, leaf = 1024, 32, 8, 4, (8, 8), 16
    K = _mixture(rng, n, d, 16)
    W = rng.standard_normal((d, r)) / np.sqrt(d)
    Z = K @ W
    Zo = orc.project(K, W)
    t0 = orc.build_tree(Zo, br, leaf, 3, seed=2, trace=True)
    t1 = orc.build_tree_pooled(Zo, 1, br, leaf, 3, seed=2, trace=True)
    np.testing.assert_array_equal(t1.leaf_index, t0.leaf_index)
    np.testing.assert_array_equal(t1.centroids_flat, t0.centroids_flat)
    np.testing.assert_array_equal(t1.min_pos_flat, t0.min_pos_flat)
    np.testing.assert_array_equal(t1.trace, t0.trace)
    tp = orc.build_tree_pooled(Zo, p, br, leaf, 3, seed=2, trace=True)
    li = tp.leaf_index.astype(np.int64)
    np.testing.assert_array_equal(np.sort(li), np.arange(n))
    blk = li.reshape(-1, p)
    assert np.all(blk[:, 0] % p == 0) and np.all(blk == blk[:, :1] + np.arange(p))
    assert np.all(np.diff(li.reshape(-1, leaf), axis=1) > 0)
    tb = orc.build_tree(Z.reshape(n // p, p, r).mean(axis=1), br, leaf // p, 3, seed=2, trace=True)
    np.testing.assert_array_equal(blk[:, 0] // p, tb.leaf_index)
    np.testing.assert_array_equal(tp.trace, tb.trace)
    for l in range(len(br)):
        groups = li.reshape(tp.nodes[l], -1)
        np.testing.assert_allclose(tp.centroids[l], Z[groups].mean(axis=1), rtol=1e-10, atol=1e-12)
        np.testing.assert_array_equal(tp.min_pos[l], groups.min(axis=1))


def pin_tree_append():
    """Update on append (kongchang.com, "How LSA Sidesteps Per-Key Scoring with Hierarchical
    Clustering": the tree can be precomputed and updated): two subtrees attached in turn.  Old
    nodes keep ids and values; every centroid of the grown tree (the new top nodes included) is
    the mean of the latent rows of the keys listed under it; min_pos is their smallest position;
    leaves stay ascending; the full-beam walk over the grown tree is brute-force flat top-B."""
    rng = np.random.default_rng(9)
    br, leaf, d, r = (4, 4, 2), 8, 16, 8
    n_old, U = 4 * 4 * 2 * leaf, 4 * 2 * leaf
    K = _mixture(rng, n_old + 2 * U, d, 12)
    W = rng.standard_normal((d, r)) / np.sqrt(d)
    Z = K @ W
    Zo = orc.project(K, W)
    tree = orc.build_tree(Zo[:n_old], br, leaf, 3, seed=4)
    for step in range(2):
        n = len(tree.leaf_index)
        grown = orc.tree_append(tree, Zo[n:n + U], 3, seed=4)
        assert grown.branching == (tree.branching[0] + 1,) + tree.branching[1:]
        for l in range(len(br)):
            k = tree.nodes[l]
            np.testing.assert_array_equal(grown.centroids[l][:k], tree.centroids[l])
            np.testing.assert_array_equal(grown.min_pos[l][:k], tree.min_pos[l])
        np.testing.assert_array_equal(grown.leaf_index[:n], tree.leaf_index)
        li = grown.leaf_index.astype(np.int64)
        np.testing.assert_array_equal(np.sort(li), np.arange(n + U))
        assert np.all(np.diff(li.reshape(-1, leaf), axis=1) > 0)
        for l in range(len(br)):
            groups = li.reshape(grown.nodes[l], -1)
            np.testing.assert_allclose(grown.centroids[l], Z[groups].mean(axis=1), rtol=1e-10, atol=1e-12)
            np.testing.assert_array_equal(grown.min_pos[l], groups.min(axis=1))
        tree = grown
    qlat = rng.standard_normal((12, d)) @ W
    full = [tree.nodes[l] for l in range(len(tree.nodes) - 1)]
    idx, _, _ = orc.select(qlat, tree, full + [5])
    np.testing.assert_array_equal(idx, _flat_topB(qlat, tree, 5))
    q_pos = rng.integers(0, n_old + 2 * U, 12)
    idx, _, _ = orc.select(qlat, tree, full + [5], q_pos=q_pos)
    np.testing.assert_array_equal(idx, _flat_topB(qlat, tree, 5, q_pos))


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
