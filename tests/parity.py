"""GPU-vs-oracle comparison helpers (near-tie protocol).

Stage-wise checks feed the oracle the GPU's upstream state, so one rounding-order
difference cannot cascade:
  * build: for every level and k-means round, the oracle recomputes the round from
    the GPU's previous assignment (the seeded start on round 1) with float64
    distances; a GPU assignment that differs must still be stable up to a
    tolerance (no blocking pair beyond eps), otherwise the check fails;
  * selection: for every level the oracle scores the candidates implied by the
    GPU's previous beam; a kept set that differs from the exact top-B may only
    differ inside the near-tie band around the cut-off score;
  * attention: the oracle evaluates on the GPU's key index lists.
"""
from __future__ import annotations

import numpy as np

from oracle import oracle as orc

NEAR_TIE_REL = 1e-5      # selection: relative band around the cut-off score
STABLE_EPS_REL = 1e-5    # build: eps = 1e-5 * (|z|^2 + |mu|^2) for a blocking pair


def _eps_stable(D, a, Zs, mu, rel=STABLE_EPS_REL):
    m, b = D.shape
    rows = np.arange(m)
    own = D[rows, a]
    worst = np.array([D[a == c, c].max() for c in range(b)])
    E = rel * ((Zs ** 2).sum(1)[:, None] + (mu ** 2).sum(1)[None, :])
    block = (D < own[:, None] - E) & (D < worst[None, :] - E)
    block[rows, a] = False
    return not block.any()


def check_build_stagewise(Z, trace, branching, leaf, iters, seed, max_segments=None, rng=None, check=None):
    """Z: [n, r] float64 latents of one head (oracle projection), or a function that
    returns the oracle latents of the given positions (for indexes too large to project
    whole); trace: [L, iters, n] GPU node ids by position; check(level, round,
    segment_size) -> bool selects which rounds are recomputed (all by default).  Returns
    (rounds that differed, keys that differed)."""
    trace = np.asarray(trace)
    if callable(Z):
        rows_of = Z
    else:
        Zfull = np.asarray(Z, np.float64)
        rows_of = lambda pos: Zfull[pos]
    n = trace.shape[-1]
    L = len(branching)
    parent = np.zeros(n, np.int64)
    rounds_diff = keys_diff = 0
    S = 1
    for l in range(L):
        b = branching[l]
        m = n // S
        cap = m // b
        counts = np.bincount(parent, minlength=S)
        assert np.all(counts == m), f"level {l}: unbalanced parent partition"
        order = np.lexsort((np.arange(n), parent)).reshape(S, m)
        segs = range(S)
        if max_segments is not None and S > max_segments:
            segs = sorted((rng or np.random.default_rng(0)).choice(S, max_segments, replace=False))
        for s in segs:
            if check is not None and not any(check(l, t, m) for t in range(iters)):
                continue
            pos = order[s]
            Zs = rows_of(pos)
            for t in range(iters):
                if check is not None and not check(l, t, m):
                    continue
                if t == 0:
                    mu = orc.level_init(Zs, pos, b, seed, l)
                else:
                    prev = trace[l, t - 1][pos] - s * b
                    mu = orc.means(Zs, prev, b)
                D = orc.distances(Zs, mu)
                want = orc.balanced_assign(D, pos)
                got = trace[l, t][pos] - s * b
                assert got.min() >= 0 and got.max() < b, f"level {l} round {t}: child out of range"
                assert np.all(np.bincount(got, minlength=b) == cap), f"level {l} round {t}: unbalanced"
                if not np.array_equal(got, want):
                    assert _eps_stable(D, got, Zs, mu), f"level {l} seg {s} round {t}: unstable assignment"
                    rounds_diff += 1
                    keys_diff += int((got != want).sum())
        parent = trace[l, iters - 1].astype(np.int64)
        S *= b
    return rounds_diff, keys_diff


def check_tree_structure(tree_h, Z, leaf, rel=1e-5):
    """tree_h: dict(centroids=[levels], min_pos=[levels], leaf_index) of one head."""
    Z = np.asarray(Z, np.float64)
    n = Z.shape[0]
    li = np.asarray(tree_h["leaf_index"]).astype(np.int64)
    np.testing.assert_array_equal(np.sort(li), np.arange(n))
    assert np.all(np.diff(li.reshape(-1, leaf), axis=1) > 0)
    for l, (cent, mp) in enumerate(zip(tree_h["centroids"], tree_h["min_pos"])):
        nodes = cent.shape[0]
        groups = li.reshape(nodes, n // nodes)
        mu = Z[groups].mean(axis=1)
        err = np.abs(np.asarray(cent, np.float64) - mu)
        scale = np.abs(mu).max() + 1e-30
        assert err.max() <= rel * scale, f"level {l}: centroid off by {err.max():.3g} (scale {scale:.3g})"
        np.testing.assert_array_equal(np.asarray(mp), groups.min(axis=1))


def check_select_stagewise(qlat, tree_h, branching, leaf, beam, q_pos, gpu_beam, gpu_idx, rel=NEAR_TIE_REL):
    """qlat: [T, r] oracle latents; gpu_beam: [L, T, Bmax]; gpu_idx: [T, K_sel].
    Returns the number of (query, level) kept sets that differed inside the band."""
    qlat = np.asarray(qlat, np.float64)
    cents = [np.asarray(c, np.float64) for c in tree_h["centroids"]]
    mpos = [np.asarray(m) for m in tree_h["min_pos"]]
    li = np.asarray(tree_h["leaf_index"])
    gpu_beam = np.asarray(gpu_beam)
    gpu_idx = np.asarray(gpu_idx)
    L = len(branching)
    near = 0
    for t in range(qlat.shape[0]):
        got = None
        for l in range(L):
            if l == 0:
                cand = np.arange(cents[0].shape[0])
            else:
                cand = (got[:, None] * branching[l] + np.arange(branching[l])).reshape(-1)
            if q_pos is not None:
                cand = cand[mpos[l][cand] <= q_pos[t]]
            B = beam[l]
            s = cents[l][cand] @ qlat[t]
            o = np.lexsort((cand, -s))
            k = min(B, len(cand))
            want = cand[o[:k]]
            row = gpu_beam[l, t]
            got = row[row >= 0].astype(np.int64)
            assert len(got) == k, f"t={t} level {l}: kept {len(got)} of {k}"
            assert np.all(row[k:] == -1)
            if set(got.tolist()) != set(want.tolist()):
                cutoff = s[o[k - 1]]
                floor = 1e-6 * np.linalg.norm(qlat[t]) * np.linalg.norm(cents[l][cand], axis=1).max()
                tol = rel * abs(cutoff) + floor
                score = dict(zip(cand.tolist(), s.tolist()))
                for node in set(got.tolist()) ^ set(want.tolist()):
                    assert abs(score[node] - cutoff) <= tol, \
                        f"t={t} level {l}: node {node} score {score[node]:.9g} outside band around {cutoff:.9g}"
                near += 1
        expect = np.full(gpu_idx.shape[1], -1, np.int64)
        keys = li.reshape(-1, leaf)[got].reshape(-1)
        expect[:len(keys)] = keys
        np.testing.assert_array_equal(gpu_idx[t], expect)
    return near


GRAD_RMS_REL = 1e-2     # rms(error) <= 1e-2 * rms(reference), over the touched rows
GRAD_ELEM_REL = 2 ** -5  # |error| <= 2^-5 |reference| + GRAD_ELEM_ABS * rms(reference), per element
GRAD_ELEM_ABS = 1e-1


def check_grad(name, got, want, zero_untouched=True, report=None):
    """Gradient tolerance (the pages give none).  The kernels round P, dS and the stored
    forward output O to bf16 (unit roundoff u = 2^-8) before their products, so a
    gradient element carries a few u of relative error in each of its terms; summed over
    hundreds of terms of either sign this stays near u of the gradient's own scale.  The
    bound is taken over the rows a selection touches (with zero_untouched, for dK and dV,
    rows no query sees must be exactly zero): rms(error) <= 1e-2 rms(ref), and per element
    |error| <= 2^-5 |ref| + 0.1 rms(ref) (measured: rms ratio ~2e-3, per-element
    excess up to ~0.045 rms(ref) on the tiny and scaled training shapes)."""
    got = np.asarray(got, np.float64).reshape(-1, np.shape(got)[-1])
    want = np.asarray(want, np.float64).reshape(-1, np.shape(want)[-1])
    touched = np.abs(want).max(axis=1) > 0
    if zero_untouched:
        assert np.all(got[~touched] == 0), (name, "nonzero gradient on an untouched row")
    else:
        touched[:] = True
    g, w = got[touched], want[touched]
    if w.size == 0:
        return
    err = np.abs(g - w)
    rms = np.sqrt((w ** 2).mean())
    rel_rms = np.sqrt((err ** 2).mean()) / rms
    elem = (err - GRAD_ELEM_REL * np.abs(w)).max() / rms
    if report is not None:
        report[name] = (float(rel_rms), float(elem))
    print(f"{name}: rms(err)/rms(ref) {rel_rms:.3g}, max(|err| - 2^-5|ref|)/rms(ref) {elem:.3g}")
    assert rel_rms <= GRAD_RMS_REL, (name, rel_rms)
    assert elem <= GRAD_ELEM_ABS, (name, elem)


def attn_errors(O_gpu, O_ref):
    d = np.abs(np.asarray(O_gpu, np.float64) - np.asarray(O_ref, np.float64))
    return float(d.max()), float(d.mean())


def export_tree(tree, h):
    """Per-level numpy copies of head h of a GPU tree (lsa.Tree)."""
    return dict(
        centroids=[tree.centroids(l)[h].cpu().numpy() for l in range(tree.levels)],
        min_pos=[tree.min_pos(l)[h].cpu().numpy() for l in range(tree.levels)],
        leaf_index=tree.leaf_index()[h].cpu().numpy(),
    )
