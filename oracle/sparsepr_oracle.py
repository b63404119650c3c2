"""SparsePR oracle: a plain, slow, fp64 numpy restatement of the per-call path.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference legs of ``bench.py`` may import
it.  It shares no code, constant generator or helper with the CUDA library; the
only thing both sides share is the seeded input generator in ``synth/``, which
holds none of the method's arithmetic.

Sources: web pages about "Partition the Support, Reconstruct the Residual"
(SparsePR, arXiv 2608.18484).  Cited by page and section:

  [abstract]    chatpaper.ai summary page -- the paper's English abstract.
  [gist 2.A]    gist.science "Resumen Tecnico: SparsePR", section 2.A (Particion
                Acoplada de Respuesta): the metric M_K = Q_s^T Q_s / M_s, k-means
                of keys on the eigenvectors of M_K into paired K/V groups, then
                query clustering on pre-softmax logit profiles against the K/V
                group centroids; one asymmetric pass, no alternating refinement.
  [gist 2.B]    same page, section 2.B (Reconstruccion de Residuales Ajustada por
                Sondas): exact probe rows, R = O_dense - O_sparse, R ~ b + xB,
                ridge, projection onto the top singular vectors of the probe
                residuals, correction of unprobed rows.
  [gist 2.C]    same page, section 2.C (Ejecucion Dispersa): group-contiguous
                permutation, variable-block sparse attention, rho_exec counts the
                routed cells plus the exact probe rows.
  [hs residual] huashangw.com article, section on retained mass versus output
                error: residual = omitted mass x (omitted output - retained output).
  [hs method]   huashangw.com article, method walkthrough: key-response
                coordinates are logit profiles under sampled queries; 64 probe
                rows per head drawn evenly from every query group; ridge
                regression; correction restricted to the top singular directions
                of the probe residuals (16 in the article); Fig. 2 (alpha is the
                target retained mass).
  [hs exec]     huashangw.com article, section on sparse execution: permuted
                group-contiguous Q/K/V; cells budgeted by the product of group
                token counts; rho_route; probe rows counted in the density.
  [hs support]  huashangw.com article, section on per-query versus grouped
                support: 6.2% of keys hold 90% of one query's weight, 22.9% once
                8 queries share one key set.
  [hs semantic] huashangw.com article, comparison of grouping strategies:
                "semantic" grouping clusters queries and keys separately; under
                the same sparse execution the coupled grouping raises the share
                of the residual an affine function explains and lowers the
                unexplained energy; the advantage holds over densities 12-35%.

Where the pages are silent the oracle takes the plainest reading and marks it
READING.  Every function is pinned by ``tests/test_oracle_*.py`` against brute
force, closed forms, library routines or the pages' identities.  One choice is
"parity unpinned": the pages give no cell-selection rule, so ``route_select``'s
rule itself (mass estimate + one shared alpha by bisection) is a reading; only its
invariants are pinned.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------------------
# Counter-based generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable
# pseudorandom number generators", OOPSLA 2014; public-domain definition by
# S. Vigna).  state += 0x9E3779B97F4A7C15; output = mix(state).
# The random draws of the method (query sample, k-means seeds, probe draws) are
# specified through this generator so that the CUDA side can implement the same
# definition independently.
# ---------------------------------------------------------------------------
_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15
_STREAM_MUL = 0xD1B54A32D192ED03

STREAM_QUERY_SAMPLE = 0
STREAM_KEY_KMEANS = 1
STREAM_QUERY_KMEANS = 2
STREAM_PROBES = 3


def splitmix64_mix(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


class SplitMix64:
    def __init__(self, state: int):
        self.state = state & _M64

    def next(self) -> int:
        self.state = (self.state + _GAMMA) & _M64
        return splitmix64_mix(self.state)


def stream_state(seed: int, bh: int, stream: int) -> int:
    """READING: one independent stream per (head, purpose):
    state0 = mix(seed + 0xD1B54A32D192ED03 * (8*bh + stream + 1))."""
    return splitmix64_mix((seed + _STREAM_MUL * (8 * bh + stream + 1)) & _M64)


def draw_without_replacement(rng: SplitMix64, n: int, m: int) -> list[int]:
    """m distinct values of range(n), uniformly, by a partial Fisher-Yates shuffle:
    for i < m, j = i + (next() mod (n - i)), swap slots i and j, emit slot i."""
    if m > n:
        raise ValueError("cannot draw more than n items")
    slot: dict[int, int] = {}
    out = []
    for i in range(m):
        j = i + rng.next() % (n - i)
        vi = slot.get(i, i)
        vj = slot.get(j, j)
        slot[i] = vj
        slot[j] = vi
        out.append(vj)
    return out


# ---------------------------------------------------------------------------
# Attention (textbook softmax attention, fp64).  The pages never state the
# scale; READING: 1/sqrt(d), the standard scaled-dot-product attention that
# SparsePR replaces ([ai-feeds] integration paragraph).
# ---------------------------------------------------------------------------
def attention(q, k, v, scale, mask=None, chunk=1024):
    """Softmax attention of rows q over keys k / values v.

    mask: optional bool [len(q), len(k)] (True = pair kept).  A row with no kept
    key gets O = 0 and LSE = -inf.  Returns (O [nq, dv], LSE [nq]) with LSE the
    natural-log partition function ln sum_k exp(scale q.k) over kept keys."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq = q.shape[0]
    out = np.zeros((nq, v.shape[1]))
    lse = np.full(nq, -np.inf)
    for s0 in range(0, nq, chunk):
        s1 = min(nq, s0 + chunk)
        s = scale * (q[s0:s1] @ k.T)
        if mask is not None:
            s = np.where(mask[s0:s1], s, -np.inf)
        mx = s.max(axis=1)
        ok = np.isfinite(mx)
        if not ok.any():
            continue
        p = np.exp(s[ok] - mx[ok, None])
        l = p.sum(axis=1)
        out[s0:s1][ok] = (p @ v) / l[:, None]
        lse[s0:s1][ok] = mx[ok] + np.log(l)
    return out, lse


# ---------------------------------------------------------------------------
# Frame-causal masking (the world-model rollout workload: queries in frame f see the
# keys of frames <= f, intersected with the route).  The pages' sources describe the
# per-call path without causality; READING: causality enters only where pairs are
# counted or attended -- the masks, the cell mass (visible keys only), the cell cost
# and the budget (visible pairs) -- and the grouping itself is unchanged.
# ---------------------------------------------------------------------------
def causal_mask(frames, rows=None) -> np.ndarray:
    """bool [len(rows), N]: key k is visible to query q iff frame(k) <= frame(q)."""
    f = np.asarray(frames)
    fq = f if rows is None else f[np.asarray(rows)]
    return f[None, :] <= fq[:, None]


def visible_counts(labels, frames, n_groups: int, n_frames: int) -> np.ndarray:
    """int64 [n_groups, n_frames]: tokens of group g in frames <= f (cumulative in f)."""
    c = np.zeros((n_groups, n_frames), np.int64)
    np.add.at(c, (np.asarray(labels), np.asarray(frames)), 1)
    return np.cumsum(c, axis=1)


def frame_histogram(labels, frames, n_groups: int, n_frames: int) -> np.ndarray:
    """int64 [n_groups, n_frames]: tokens of group a in frame f."""
    c = np.zeros((n_groups, n_frames), np.int64)
    np.add.at(c, (np.asarray(labels), np.asarray(frames)), 1)
    return c


# ---------------------------------------------------------------------------
# Response-coupled partitioning  [gist 2.A], [hs method], [abstract]
# ---------------------------------------------------------------------------
def sample_queries(n: int, m_s: int, seed: int, bh: int) -> np.ndarray:
    """M_s sampled query rows.  READING: uniform without replacement (stream 0)."""
    rng = SplitMix64(stream_state(seed, bh, STREAM_QUERY_SAMPLE))
    return np.array(draw_without_replacement(rng, n, m_s), dtype=np.int64)


def key_metric(q_s) -> np.ndarray:
    """M_K = Q_s^T Q_s / M_s  (gist 2.A, the only formula for it; uncentred)."""
    q_s = np.asarray(q_s, np.float64)
    return q_s.T @ q_s / q_s.shape[0]


def top_eigenpairs(m_k, r: int):
    """Leading r eigenpairs of the symmetric metric, eigenvalues descending.
    Tiny negative eigenvalues from rounding are clipped to 0 (M_K is PSD)."""
    w, u = np.linalg.eigh(np.asarray(m_k, np.float64))
    order = np.argsort(-w, kind="stable")[:r]
    return np.clip(w[order], 0.0, None), u[:, order]


def key_coords(k, lam, u) -> np.ndarray:
    """Key-response coordinates y = Lambda_r^{1/2} U_r^T k  (one row per key).

    READING of "k-means on the eigenvectors of M_K" (gist 2.A) together with
    "each key's logit distribution under the sampled queries" (hs method):
    at full rank ||y1 - y2||^2 = ||Q_s (k1 - k2)||^2 / M_s, the mean squared
    difference of the two keys' logits under the sampled queries."""
    return np.asarray(k, np.float64) @ (np.asarray(u, np.float64) * np.sqrt(lam)[None, :])


def kmeans_assign(x, mu, chunk=2048) -> np.ndarray:
    """argmin_j sum_c (x_c - mu_jc)^2, ties to the lowest j (np.argmin keeps the
    first minimum)."""
    x = np.asarray(x, np.float64)
    mu = np.asarray(mu, np.float64)
    lab = np.empty(x.shape[0], np.int64)
    for s0 in range(0, x.shape[0], chunk):
        d = ((x[s0:s0 + chunk, None, :] - mu[None, :, :]) ** 2).sum(axis=2)
        lab[s0:s0 + chunk] = np.argmin(d, axis=1)
    return lab


def kmeans_distances(x, mu) -> np.ndarray:
    x = np.asarray(x, np.float64)
    mu = np.asarray(mu, np.float64)
    return ((x[:, None, :] - mu[None, :, :]) ** 2).sum(axis=2)


def kmeans_update(x, labels, mu_prev) -> np.ndarray:
    """Centroid = mean of its members (fp64).  READING: an empty cluster keeps its
    previous centroid."""
    x = np.asarray(x, np.float64)
    mu = np.array(mu_prev, np.float64, copy=True)
    for g in range(mu.shape[0]):
        sel = labels == g
        if sel.any():
            mu[g] = x[sel].mean(axis=0)
    return mu


def kmeans(x, n_groups: int, iters: int, seed: int, bh: int, stream: int,
           label_history=None):
    """Lloyd's k-means.  READINGS: seeds = n_groups distinct rows drawn by the
    stream's generator (cluster j starts at the j-th drawn row); ``iters``
    assignment steps with a centroid update between consecutive ones (no early
    stop); ties to the lowest cluster index; empty clusters keep their centroid.

    label_history: optional list receiving the labels of every assignment step.
    ``teacher`` forcing for parity runs is available through kmeans_step."""
    x = np.asarray(x, np.float64)
    rng = SplitMix64(stream_state(seed, bh, stream))
    init = draw_without_replacement(rng, x.shape[0], n_groups)
    mu = x[init].copy()
    labels = None
    for t in range(iters):
        labels = kmeans_assign(x, mu)
        if label_history is not None:
            label_history.append(labels.copy())
        if t + 1 < iters:
            mu = kmeans_update(x, labels, mu)
    return labels, mu, np.array(init, np.int64)


def kmeans_init(n: int, n_groups: int, seed: int, bh: int, stream: int) -> np.ndarray:
    rng = SplitMix64(stream_state(seed, bh, stream))
    return np.array(draw_without_replacement(rng, n, n_groups), np.int64)


def group_means(k, labels, n_groups: int):
    """K/V group centroids = mean raw key of each group, and group sizes n_g.
    READING: the centroid of a K/V group (gist 2.A) is the mean of its raw keys,
    so q.c_g is q's mean logit over the group.  Empty group -> zero vector."""
    k = np.asarray(k, np.float64)
    n = np.bincount(labels, minlength=n_groups).astype(np.int64)
    c = np.zeros((n_groups, k.shape[1]))
    for g in range(n_groups):
        if n[g]:
            c[g] = k[labels == g].mean(axis=0)
    return c, n


def query_coords(q, c, scale) -> np.ndarray:
    """Query-response coordinates: pre-softmax logits of each query against the
    K/V group centroids, z_q = scale * C q  (gist 2.A).  READING: no centring."""
    return scale * (np.asarray(q, np.float64) @ np.asarray(c, np.float64).T)


def group_permutation(labels, n_groups: int):
    """Group-contiguous layout (gist 2.C, hs exec): perm[i] = original index of the
    token at permuted position i; offsets[g] = first position of group g.
    READING: stable, i.e. ascending original index inside a group."""
    labels = np.asarray(labels)
    perm = np.argsort(labels, kind="stable").astype(np.int64)
    offsets = np.zeros(n_groups + 1, np.int64)
    offsets[1:] = np.cumsum(np.bincount(labels, minlength=n_groups))
    return perm, offsets


# ---------------------------------------------------------------------------
# Route  [hs exec] budget by product of group sizes; [hs method] Fig. 2 alpha
# ---------------------------------------------------------------------------
def cell_mass(z, label_q, n_k, n_qgroups: int, frames=None, vis_k=None) -> np.ndarray:
    """Estimated attention mass of query group a on K/V group g.

    READING: a query's mass on group g is estimated from its centroid logit,
    sum_{k in g} exp(s q.k) ~ n_g exp(z_q[g]), normalised over groups:
    p_q(g) = softmax_g(z_q[g] + ln n_g) (empty groups excluded); the cell mass
    p(a, g) is the mean of p_q(g) over the queries of group a (0 for empty a).
    Frame-causal (frames = frame per token, vis_k = visible_counts of the keys):
    n_g is the number of keys of g the query can see, vis_k[g, frame(q)]."""
    z = np.asarray(z, np.float64)
    if frames is None:
        n_vis = np.broadcast_to(np.asarray(n_k)[None, :], z.shape)
    else:
        n_vis = np.asarray(vis_k)[:, np.asarray(frames)].T       # [N, Gk]
    logit = np.where(n_vis > 0, z + np.log(np.maximum(n_vis, 1)), -np.inf)
    mx = logit.max(axis=1, keepdims=True)
    p = np.exp(logit - mx)
    p /= p.sum(axis=1, keepdims=True)
    out = np.zeros((n_qgroups, z.shape[1]))
    for a in range(n_qgroups):
        sel = label_q == a
        if sel.any():
            out[a] = p[sel].mean(axis=0)
    return out


def cell_cost(n_q, n_k, hist_q=None, vis_k=None) -> np.ndarray:
    """Executed token pairs of cell (a, g): n_a * n_g  [hs exec].  Frame-causal
    (hist_q = frame_histogram of the queries, vis_k = visible_counts of the keys):
    the visible pairs sum_f hist_q[a, f] * vis_k[g, f]."""
    if hist_q is None:
        return np.outer(np.asarray(n_q, np.int64), np.asarray(n_k, np.int64))
    return np.asarray(hist_q, np.int64) @ np.asarray(vis_k, np.int64).T


@dataclass
class RouteResult:
    route: np.ndarray          # uint8 [Gq, Gk]
    alpha: float
    routed_pairs: int
    budget: float
    rho_exec: float
    rho_route: float


def _route_prefix(mass, cost, n_q, n_k):
    """Per query group: groups sorted by mass descending (ties -> lower g) among
    non-empty K/V groups, sequential fp64 cumulative mass and int cumulative cost."""
    rows = []
    for a in range(mass.shape[0]):
        if n_q[a] == 0:
            rows.append(None)
            continue
        cand = np.nonzero(n_k > 0)[0]
        order = cand[np.argsort(-mass[a, cand], kind="stable")]
        cm = np.cumsum(mass[a, order].astype(np.float64))
        cc = np.cumsum(cost[a, order].astype(np.int64))
        rows.append((order, cm, cc))
    return rows


def _prefix_len(cm, alpha):
    """Shortest prefix whose cumulative mass reaches alpha, at least one cell; all
    cells if rounding keeps the total below alpha."""
    idx = np.nonzero(cm >= alpha)[0]
    n = (idx[0] + 1) if idx.size else cm.size
    return max(1, int(n))


def _route_cost(rows, alpha):
    tot = 0
    for r in rows:
        if r is None:
            continue
        order, cm, cc = r
        tot += int(cc[_prefix_len(cm, alpha) - 1])
    return tot


def route_select(mass, n_q, n_k, density: float, n_probes: int, n_tokens: int,
                 bisect_steps: int = 60, cost=None, visible=None) -> RouteResult:
    """Pick the (query group, K/V group) cells to execute.

    READING (parity unpinned as a rule -- the pages fix only its ingredients):
    every query group keeps the shortest mass-sorted prefix of K/V groups whose
    estimated retained mass reaches one shared target alpha (Fig. 2's alpha,
    hs method), at least one cell; the cost of a cell is the product of the two
    group sizes (hs exec); the probe rows' exact pairs are charged first
    (gist 2.C: rho_exec includes the probe rows); alpha is the largest value in
    [0, 1] whose cost fits the budget, found by bisection in fp64.  density >= 1
    routes every non-empty cell.  Frame-causal: cost = the visible pairs per cell and
    visible = all visible pairs; READING: the probe rows are charged their expected
    visible keys, n_probes * visible / n_tokens (= n_probes * n_tokens without
    causality), since they are drawn after the route."""
    mass = np.asarray(mass, np.float64)
    n_q = np.asarray(n_q, np.int64)
    n_k = np.asarray(n_k, np.int64)
    cost = cell_cost(n_q, n_k) if cost is None else np.asarray(cost, np.int64)
    visible = float(n_tokens) * float(n_tokens) if visible is None else float(visible)
    probe_pairs = float(n_probes) * visible / float(n_tokens)
    budget = density * visible - probe_pairs
    rows = _route_prefix(mass, cost, n_q, n_k)
    route = np.zeros(mass.shape, np.uint8)
    if density >= 1.0:
        alpha = 1.0
        for a, r in enumerate(rows):
            if r is not None:
                route[a, r[0]] = 1
    else:
        lo, hi = 0.0, 1.0
        if _route_cost(rows, lo) <= budget:
            for _ in range(bisect_steps):
                mid = 0.5 * (lo + hi)
                if _route_cost(rows, mid) <= budget:
                    lo = mid
                else:
                    hi = mid
        alpha = lo
        for a, r in enumerate(rows):
            if r is None:
                continue
            order, cm, cc = r
            route[a, order[:_prefix_len(cm, alpha)]] = 1
    routed = int((cost * route).sum())
    return RouteResult(route=route, alpha=alpha, routed_pairs=routed, budget=budget,
                       rho_exec=(routed + probe_pairs) / visible,
                       rho_route=routed / visible)


def block_mask(route, label_q, perm_q, label_k, perm_k, block: int) -> np.ndarray:
    """Tile-level mask of the permuted layout: tile (i, j) is set when any query at
    permuted positions [i*block, (i+1)*block) and any key at permuted positions
    [j*block, (j+1)*block) form a routed pair."""
    n = len(perm_q)
    lq = np.asarray(label_q)[perm_q]
    lk = np.asarray(label_k)[perm_k]
    t = (n + block - 1) // block
    out = np.zeros((t, t), np.uint8)
    for i in range(t):
        qa = np.unique(lq[i * block:(i + 1) * block])
        sub = route[qa]
        for j in range(t):
            kg = np.unique(lk[j * block:(j + 1) * block])
            out[i, j] = 1 if sub[:, kg].any() else 0
    return out


# ---------------------------------------------------------------------------
# Sparse attention over the route  [gist 2.C]
# ---------------------------------------------------------------------------
def pair_mask(route, label_q, label_k, rows=None, frames=None) -> np.ndarray:
    """Token-pair mask: query q may see key k iff route[label_q[q], label_k[k]]
    (and, frame-causal, frame(k) <= frame(q))."""
    lq = np.asarray(label_q) if rows is None else np.asarray(label_q)[rows]
    m = np.asarray(route, bool)[lq][:, np.asarray(label_k)]
    if frames is not None:
        m &= causal_mask(frames, rows)
    return m


def sparse_attention(q, k, v, scale, route, label_q, label_k, rows=None, frames=None):
    """O_sparse and LSE for rows (all rows by default), original token order."""
    rows = np.arange(len(q)) if rows is None else np.asarray(rows)
    m = pair_mask(route, label_q, label_k, rows, frames)
    return attention(np.asarray(q)[rows], k, v, scale, mask=m)


# ---------------------------------------------------------------------------
# Probes and the residual fit  [gist 2.B], [hs method]
# ---------------------------------------------------------------------------
def probe_allocation(sizes, n_probes: int) -> np.ndarray:
    """Probes per query group, "drawn evenly from every group" (hs method).

    READING: water-filling.  While probes remain and some group has unprobed
    members: every such group receives min(floor(remaining / #groups), spare);
    when the even share is 0, the leftover probes go one each to the groups with
    spare members in order of decreasing group size (ties -> lower index)."""
    sizes = np.asarray(sizes, np.int64)
    alloc = np.zeros_like(sizes)
    remaining = int(n_probes)
    while remaining > 0:
        open_ = np.nonzero(alloc < sizes)[0]
        if open_.size == 0:
            break
        share = remaining // open_.size
        if share == 0:
            order = open_[np.argsort(-sizes[open_], kind="stable")]
            for a in order[:remaining]:
                alloc[a] += 1
            remaining = 0
            break
        for a in open_:
            add = min(share, int(sizes[a] - alloc[a]))
            alloc[a] += add
            remaining -= add
    return alloc


def pick_probes(perm_q, q_offsets, n_probes: int, seed: int, bh: int) -> np.ndarray:
    """Query-group-stratified probe rows (64 per head in the article).

    READING: group a's members are its tokens in permuted (ascending original)
    order; alloc_a of them are drawn without replacement with the probe stream,
    groups visited in ascending order; output = original token indices, group
    order then draw order."""
    sizes = np.diff(np.asarray(q_offsets))
    alloc = probe_allocation(sizes, n_probes)
    rng = SplitMix64(stream_state(seed, bh, STREAM_PROBES))
    out = []
    for a in range(len(sizes)):
        if alloc[a] == 0:
            continue
        members = np.asarray(perm_q)[q_offsets[a]:q_offsets[a + 1]]
        for p in draw_without_replacement(rng, len(members), int(alloc[a])):
            out.append(int(members[p]))
    return np.array(out, np.int64)


def probe_weights(q_offsets, n_probes: int) -> np.ndarray:
    """Weights of the probe rows for the weighted fit (ai-feeds: a "weighted" affine fit).

    READING: inverse inclusion probability: a probe of query group a stands for the
    n_a / alloc_a tokens of its group (alloc_a = its group's probe count), in the probe
    order of pick_probes (group order); normalised to mean 1 so lam keeps its scale."""
    sizes = np.diff(np.asarray(q_offsets))
    alloc = probe_allocation(sizes, n_probes)
    w = np.concatenate([np.full(int(alloc[a]), sizes[a] / alloc[a]) for a in range(len(sizes)) if alloc[a] > 0])
    return w * (w.size / w.sum())


def omitted_mass(lse_sparse, lse_dense) -> np.ndarray:
    """Share of the dense softmax mass that falls on skipped keys: 1 - Z_ret/Z."""
    return 1.0 - np.exp(np.asarray(lse_sparse) - np.asarray(lse_dense))


def probe_subspace(r_p, rank: int, rel_tol: float = 1e-6):
    """Top `rank` right singular vectors of the (uncentred) probe residual matrix
    (gist 2.B; hs method: 16 leading directions).  READING: directions whose
    singular value is <= rel_tol * sigma_max are zero columns (they carry no
    residual, so they contribute nothing to the correction)."""
    _, s, vt = np.linalg.svd(np.asarray(r_p, np.float64), full_matrices=False)
    v = np.zeros((r_p.shape[1], rank))
    sig = np.zeros(rank)
    k = min(rank, s.size)
    smax = s[0] if s.size else 0.0
    for i in range(k):
        if s[i] > rel_tol * smax and smax > 0:
            v[:, i] = vt[i]
            sig[i] = s[i]
    return v, sig


def ridge_fit(x, y, lam: float, weights=None):
    """Ridge-regularised affine fit y ~ b + x W (gist 2.B: R ~ b + xB, ridge).

    READINGS: the intercept is not penalised (solve on probe-centred x and y,
    b = mean(y) - mean(x) W); lam is absolute; uniform probe weights unless
    ``weights`` are given (then weighted means and rows scaled by sqrt(weight): the
    minimiser of sum_i w_i ||y_i - b - x_i W||^2 + lam ||W||^2).  Dual form
    W = Xc^T (Xc Xc^T + lam I)^-1 Yc, identical to the primal
    (Xc^T Xc + lam I)^-1 Xc^T Yc."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    wt = np.ones(x.shape[0]) if weights is None else np.asarray(weights, np.float64)
    xm = (wt[:, None] * x).sum(axis=0) / wt.sum()
    ym = (wt[:, None] * y).sum(axis=0) / wt.sum()
    sq = np.sqrt(wt)[:, None]
    xc = (x - xm) * sq
    yc = (y - ym) * sq
    w = xc.T @ np.linalg.solve(xc @ xc.T + lam * np.eye(x.shape[0]), yc)
    b = ym - xm @ w
    return w, b


@dataclass
class ProbeFit:
    probe_idx: np.ndarray      # [P] original query indices
    o_dense: np.ndarray        # [P, d]
    o_sparse: np.ndarray       # [P, d]
    lse_dense: np.ndarray
    lse_sparse: np.ndarray
    residual: np.ndarray       # [P, d] = o_dense - o_sparse
    vr: np.ndarray             # [d, r] subspace basis
    sigma: np.ndarray          # [r]
    w: np.ndarray              # [d, r]
    b: np.ndarray              # [r]  intercept in subspace coordinates
    b_full: np.ndarray         # [d]  = vr @ b
    bmat: np.ndarray           # [d, d] = w @ vr^T  (the pages' B)


FIT_INPUTS = ("full", "subspace")


def fit_from_probes(probe_idx, o_dense, o_sparse, lse_dense, lse_sparse, rank: int,
                    lam: float, weights=None, fit_input: str = "full") -> ProbeFit:
    """R_P = O_dense - O_sparse on the probes; V_r = top singular subspace of R_P;
    Y = R_P V_r; ridge fit of Y ~ b + (input) W with x = the probe rows' sparse output.

    The pages write the residual as an affine function of the sparse output, R ~ b + xB,
    fitted by ridge, with the *correction* projected onto the subspace of the probe
    residuals' leading singular vectors (gist 2.B, subspace restriction; hs method: the
    corrected result may only fall in the residual directions the probes observed).
    READINGS of the map's input:
      fit_input="full" (default): x is the whole d-dimensional sparse output row, the
        pages' R ~ b + xB taken literally; only the output side is restricted, so
        B = W V_r^T with W (d x r) the ridge slope onto the residual coordinates Y.
      fit_input="subspace": x projected on V_r as well (the abstract's "affine correction
        from the sparse output within the output subspace" read as applying to both
        sides): Y ~ b + (x V_r) W_sub, r + 1 parameters per direction, returned as
        w = V_r W_sub so that a row's residual coordinates are x w in both readings."""
    if fit_input not in FIT_INPUTS:
        raise ValueError(f"fit_input must be one of {FIT_INPUTS}")
    r_p = np.asarray(o_dense, np.float64) - np.asarray(o_sparse, np.float64)
    vr, sig = probe_subspace(r_p, rank)
    y = r_p @ vr
    xs = np.asarray(o_sparse, np.float64)
    if fit_input == "full":
        w, b = ridge_fit(xs, y, lam, weights)
    else:
        w_sub, b = ridge_fit(xs @ vr, y, lam, weights)
        w = vr @ w_sub
    return ProbeFit(probe_idx=np.asarray(probe_idx), o_dense=np.asarray(o_dense, np.float64),
                    o_sparse=xs, lse_dense=np.asarray(lse_dense),
                    lse_sparse=np.asarray(lse_sparse), residual=r_p, vr=vr, sigma=sig, w=w, b=b,
                    b_full=vr @ b, bmat=w @ vr.T)


def correct(o_sparse, fit: ProbeFit) -> np.ndarray:
    """O = x + b V_r^T + (x W) V_r^T for every row (gist 2.B: the predicted residual
    is added to the sparse output), then probe rows take their exact dense output
    (READING: the probes were computed exactly, so their final value is exact)."""
    x = np.asarray(o_sparse, np.float64)
    out = x + fit.b_full[None, :] + (x @ fit.w) @ fit.vr.T
    out[fit.probe_idx] = fit.o_dense
    return out


# ---------------------------------------------------------------------------
# One head, end to end
# ---------------------------------------------------------------------------
@dataclass
class Params:
    n_kgroups: int
    n_qgroups: int
    n_samples: int
    n_probes: int
    eig_rank: int
    sub_rank: int
    kmeans_iters: int
    density: float
    ridge_lambda: float = 1e-2
    scale: float = 0.0          # 0 -> 1/sqrt(d)
    seed: int = 0
    block: int = 64
    fit_weighted: bool = False   # probe weights n_a / alloc_a in the ridge (probe_weights)
    fit_input: str = "full"      # input of the affine map: "full" sparse output or "subspace" (fit_from_probes)

    def eff_scale(self, d: int) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(d)


@dataclass
class HeadPartition:
    sample_idx: np.ndarray
    metric: np.ndarray
    eigval: np.ndarray
    eigvec: np.ndarray
    key_coords: np.ndarray
    key_init: np.ndarray
    label_k: np.ndarray
    key_label_history: list
    centroids: np.ndarray      # raw-key group means [Gk, d]
    n_k: np.ndarray
    query_coords: np.ndarray
    query_init: np.ndarray
    label_q: np.ndarray
    query_label_history: list
    n_q: np.ndarray
    perm_q: np.ndarray
    q_offsets: np.ndarray
    perm_k: np.ndarray
    k_offsets: np.ndarray
    mass: np.ndarray
    route: RouteResult
    block_mask: np.ndarray = field(default=None)


def partition_head(q, k, p: Params, bh: int, key_coords_override=None,
                   query_coords_override=None, mass_override=None, frames=None) -> HeadPartition:
    """Response-coupled partition of one head: Q -> K grouping, then K -> Q grouping,
    a single asymmetric pass (gist 2.A; hs method), followed by the route.

    The *_override arguments let parity tests feed the CUDA path's fp32
    coordinates / cell masses into the oracle's k-means and route selection."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    n, d = q.shape
    s = p.eff_scale(d)
    idx = sample_queries(n, p.n_samples, p.seed, bh)
    m_k = key_metric(q[idx])
    lam, u = top_eigenpairs(m_k, p.eig_rank)
    y = key_coords(k, lam, u) if key_coords_override is None else np.asarray(key_coords_override, np.float64)
    hist_k: list = []
    label_k, _, kinit = kmeans(y, p.n_kgroups, p.kmeans_iters, p.seed, bh, STREAM_KEY_KMEANS, hist_k)
    c, n_k = group_means(k, label_k, p.n_kgroups)
    z = query_coords(q, c, s) if query_coords_override is None else np.asarray(query_coords_override, np.float64)
    hist_q: list = []
    label_q, _, qinit = kmeans(z, p.n_qgroups, p.kmeans_iters, p.seed, bh, STREAM_QUERY_KMEANS, hist_q)
    n_q = np.bincount(label_q, minlength=p.n_qgroups).astype(np.int64)
    perm_q, qoff = group_permutation(label_q, p.n_qgroups)
    perm_k, koff = group_permutation(label_k, p.n_kgroups)
    if frames is None:
        mass = cell_mass(z, label_q, n_k, p.n_qgroups) if mass_override is None else np.asarray(mass_override, np.float64)
        rr = route_select(mass, n_q, n_k, p.density, p.n_probes, n)
    else:
        nf = int(np.max(frames)) + 1
        vis_k = visible_counts(label_k, frames, p.n_kgroups, nf)
        hist_q = frame_histogram(label_q, frames, p.n_qgroups, nf)
        mass = (cell_mass(z, label_q, n_k, p.n_qgroups, frames, vis_k) if mass_override is None
                else np.asarray(mass_override, np.float64))
        cost = cell_cost(n_q, n_k, hist_q, vis_k)
        visible = float(hist_q.sum(axis=0) @ vis_k.sum(axis=0))
        rr = route_select(mass, n_q, n_k, p.density, p.n_probes, n, cost=cost, visible=visible)
    bm = block_mask(rr.route, label_q, perm_q, label_k, perm_k, p.block)
    return HeadPartition(sample_idx=idx, metric=m_k, eigval=lam, eigvec=u, key_coords=y,
                         key_init=kinit, label_k=label_k, key_label_history=hist_k,
                         centroids=c, n_k=n_k, query_coords=z, query_init=qinit,
                         label_q=label_q, query_label_history=hist_q, n_q=n_q,
                         perm_q=perm_q, q_offsets=qoff, perm_k=perm_k, k_offsets=koff,
                         mass=mass, route=rr, block_mask=bm)


def semantic_partition_head(q, k, p: Params, bh: int, frames=None) -> HeadPartition:
    """The semantic-grouping baseline [hs semantic]: keys and queries are clustered
    separately on their raw vectors (same k-means rules and seed streams as the
    coupled partition), then the same centroids, cell mass, route and layout.
    READING: "cluster queries and keys separately, similar tokens together" is
    Lloyd k-means on the raw d-dimensional rows."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    n, d = q.shape
    s = p.eff_scale(d)
    hist_k: list = []
    label_k, _, kinit = kmeans(k, p.n_kgroups, p.kmeans_iters, p.seed, bh, STREAM_KEY_KMEANS, hist_k)
    c, n_k = group_means(k, label_k, p.n_kgroups)
    z = query_coords(q, c, s)
    hist_q: list = []
    label_q, _, qinit = kmeans(q, p.n_qgroups, p.kmeans_iters, p.seed, bh, STREAM_QUERY_KMEANS, hist_q)
    n_q = np.bincount(label_q, minlength=p.n_qgroups).astype(np.int64)
    perm_q, qoff = group_permutation(label_q, p.n_qgroups)
    perm_k, koff = group_permutation(label_k, p.n_kgroups)
    if frames is None:
        mass = cell_mass(z, label_q, n_k, p.n_qgroups)
        rr = route_select(mass, n_q, n_k, p.density, p.n_probes, n)
    else:
        nf = int(np.max(frames)) + 1
        vis_k = visible_counts(label_k, frames, p.n_kgroups, nf)
        fh = frame_histogram(label_q, frames, p.n_qgroups, nf)
        mass = cell_mass(z, label_q, n_k, p.n_qgroups, frames, vis_k)
        rr = route_select(mass, n_q, n_k, p.density, p.n_probes, n, cost=cell_cost(n_q, n_k, fh, vis_k),
                          visible=float(fh.sum(axis=0) @ vis_k.sum(axis=0)))
    bm = block_mask(rr.route, label_q, perm_q, label_k, perm_k, p.block)
    return HeadPartition(sample_idx=np.zeros(0, np.int64), metric=np.zeros((d, d)), eigval=np.zeros(0),
                         eigvec=np.zeros((d, 0)), key_coords=k, key_init=kinit, label_k=label_k,
                         key_label_history=hist_k, centroids=c, n_k=n_k, query_coords=z, query_init=qinit,
                         label_q=label_q, query_label_history=hist_q, n_q=n_q, perm_q=perm_q, q_offsets=qoff,
                         perm_k=perm_k, k_offsets=koff, mass=mass, route=rr, block_mask=bm)


# ---------------------------------------------------------------------------
# Diagnostics of a partition [hs support], [hs semantic] (measurements, not steps of the path)
# ---------------------------------------------------------------------------
def support_fraction(prob, mass: float = 0.9) -> float:
    """Smallest fraction of the keys whose probabilities (one distribution, summing
    to 1) reach ``mass``: keys taken in decreasing probability."""
    pr = np.sort(np.asarray(prob, np.float64))[::-1]
    n_keep = int(np.searchsorted(np.cumsum(pr), mass * pr.sum() * (1.0 - 1e-12)) + 1)
    return min(n_keep, pr.size) / pr.size


def grouped_support(q, k, scale, label_q, groups, mass: float = 0.9, frames=None):
    """Per-query versus grouped support [hs support] over the given query groups.

    Returns (mean over the groups' queries of the per-query support fraction,
    mean over the groups of the pooled support fraction).  READING: the queries of a
    group share one key set, so the grouped support is the support of the group's
    pooled distribution, the mean of its members' softmax rows."""
    q = np.asarray(q, np.float64)
    per_q, pooled = [], []
    for a in groups:
        rows = np.nonzero(np.asarray(label_q) == a)[0]
        if rows.size == 0:
            continue
        logits = scale * (q[rows] @ np.asarray(k, np.float64).T)
        if frames is not None:
            logits = np.where(causal_mask(frames, rows), logits, -np.inf)
        pr = np.exp(logits - logits.max(axis=1, keepdims=True))
        pr /= pr.sum(axis=1, keepdims=True)
        per_q.extend(support_fraction(r, mass) for r in pr)
        pooled.append(support_fraction(pr.mean(axis=0), mass))
    return float(np.mean(per_q)), float(np.mean(pooled))


def affine_explainable(x, r):
    """How much of the residual R an affine function of the sparse output x explains
    [abstract: "predictability of the remaining residual from the sparse output"]:
    least-squares fit R ~ b + x B over the given rows (no penalty, full rank).
    Returns (explained fraction 1 - ||R - fit||^2 / ||R||^2, unexplained energy
    ||R - fit||^2)."""
    x = np.asarray(x, np.float64)
    r = np.asarray(r, np.float64)
    xa = np.hstack([np.ones((x.shape[0], 1)), x])
    coef, *_ = np.linalg.lstsq(xa, r, rcond=None)
    un = float(((r - xa @ coef) ** 2).sum())
    tot = float((r ** 2).sum())
    return (1.0 - un / tot if tot > 0 else 1.0), un


def probe_fit_head(q, k, v, part_label_q, part_label_k, route, perm_q, q_offsets,
                   p: Params, bh: int, frames=None) -> ProbeFit:
    """Exact probe rows (dense and routed attention), residual, subspace, ridge."""
    q = np.asarray(q, np.float64)
    d = q.shape[1]
    s = p.eff_scale(d)
    pidx = pick_probes(perm_q, q_offsets, p.n_probes, p.seed, bh)
    o_d, l_d = attention(q[pidx], k, v, s, mask=None if frames is None else causal_mask(frames, pidx))
    o_s, l_s = sparse_attention(q, k, v, s, route, part_label_q, part_label_k, rows=pidx, frames=frames)
    wts = probe_weights(q_offsets, p.n_probes) if p.fit_weighted else None
    return fit_from_probes(pidx, o_d, o_s, l_d, l_s, p.sub_rank, p.ridge_lambda, wts, p.fit_input)


@dataclass
class HeadResult:
    part: HeadPartition
    o_sparse: np.ndarray
    lse_sparse: np.ndarray
    fit: ProbeFit
    o: np.ndarray


def sparsepr_head(q, k, v, p: Params, bh: int, frames=None) -> HeadResult:
    """The whole per-call path for one head (huashangw sparse-execution section's
    stage list: grouping, route, permutation, sparse attention, exact probes,
    residual fit, correction, output restoration)."""
    q = np.asarray(q, np.float64)
    d = q.shape[1]
    s = p.eff_scale(d)
    part = partition_head(q, k, p, bh, frames=frames)
    route = part.route.route
    o_s, l_s = sparse_attention(q, k, v, s, route, part.label_q, part.label_k, frames=frames)
    fit = probe_fit_head(q, k, v, part.label_q, part.label_k, route, part.perm_q,
                         part.q_offsets, p, bh, frames=frames)
    o = correct(o_s, fit)
    return HeadResult(part=part, o_sparse=o_s, lse_sparse=l_s, fit=fit, o=o)


def rel_l2(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


__all__ = [n for n in dir() if not n.startswith("_")]
