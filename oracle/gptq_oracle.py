"""Plain fp64 CPU oracle for Hessian-aware layer-wise weight quantization (GPTQ / Babai).

TEST INFRASTRUCTURE ONLY.  This module is the checker the CUDA path is compared against; it is
called by ``tests/``, by ``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``
and by nothing else.  It shares no code with the CUDA library and imports nothing from the
package; it is slow on purpose (unblocked, column by column, numpy fp64).

Sources, by page title and section:

* [GEOM] "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane Algorithm"
  - section 2.1: the layer objective is a closest-vector problem; the basis comes from the
    calibration inputs and the per-column scales, the target from the float weights; Theorem 1:
    any factor of the Hessian X^T X gives an equivalent instance, so a square Cholesky factor
    may replace the tall input matrix.
  - section 2.2: GPTQ's error propagation is Babai's nearest-plane step; Theorem 4: GPTQ run
    back to front is exactly Babai; one more propagation after the projection changes nothing.
  - section 2.3: Theorem 5: without clipping, the error is at most one quarter of
    (T^-1 s)^T D (T^-1 s), D the diagonal of the LDL factorisation of the order-permuted
    Hessian, T the quantization order.
* [WSIC] "WaterSIC: information-theoretically (near) optimal linear layer quantization",
  section 2: Cholesky Sigma = L L^T, columns decided from the last to the first with the
  already-decided ones cancelled (successive interference cancellation); "dead feature
  erasure" of zero-variance inputs.
* [INIT] "Initialisation Determines the Basin", OA-EM section: the per-layer Hessian is the
  input Gram matrix plus a lambda-multiple of the identity.
* [RDQ] "RDQ: Residual Distribution Quantization", setup: group-128 asymmetric integer format.

The pages do not print GPTQ's update, its min-max quantizer or its Cholesky trick; where they
are silent the plainest reading is taken and flagged ``reading:`` below.

Pins (tests/test_oracle_pins.py, with tests/golden/gptq_two_column_hand.json): every public
function here is pinned against a closed form, a hand-derived example, an independent textbook
construction (Gram-Schmidt Babai, brute-force CVP) or an invariant.  No function is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "hessian",
    "fix_dead_features",
    "dampen",
    "hinv_upper_factor",
    "act_order",
    "min_pivot_order",
    "minmax_grid",
    "clipfree_grid",
    "gptq_columns",
    "babai_sic_reverse",
    "ssqr_columns",
    "ssqr_search",
    "hptq_rate",
    "hptq_search",
    "zsic_spacing",
    "pack_codes",
    "huffman_lengths",
    "canonical_codewords",
    "huffman_encode",
    "huffman_decode",
    "proxy_loss",
    "quadratic_loss",
    "babai_bound",
    "quantize_layer",
]


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor: bf16/fp32 -> fp64 is exact
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------------------------
# Hessian, dead features, damping, the factor
# ---------------------------------------------------------------------------------------------

def hessian(X) -> np.ndarray:
    """H = 2 X^T X for X stored tokens x features ([GEOM] 2.1, Hessian X^T X; [INIT] OA-EM).

    reading: the factor 2 is the second derivative of the squared output error; H is not
    divided by the token count (codes do not depend on a positive scale of H).
    """
    x = _f64(X)
    return 2.0 * (x.T @ x)


def fix_dead_features(H, W):
    """Zero-variance inputs: H_ii == 0 -> H_ii = 1 and W[:, i] = 0 ([WSIC] dead feature erasure).

    Returns (H', W', dead mask).
    """
    h = _f64(H).copy()
    w = _f64(W).copy()
    dead = np.diag(h) == 0.0
    idx = np.nonzero(dead)[0]
    h[idx, idx] = 1.0
    w[:, idx] = 0.0
    return h, w, dead


def dampen(H, damp: float):
    """H_d = H + damp * mean(diag H) * I, applied after the dead-feature fix ([INIT] +lambda I).

    reading: lambda is relative to the mean diagonal, damp = 0.01.  Returns (H_d, delta).
    """
    h = _f64(H)
    delta = damp * float(np.mean(np.diag(h)))
    return h + delta * np.eye(h.shape[0]), delta


def hinv_upper_factor(Hd) -> np.ndarray:
    """U upper triangular, positive diagonal, with U^T U = H_d^-1.

    Literal three-step route: Cholesky H_d = L L^T; inverse H_d^-1 = L^-T L^-1; then the
    upper Cholesky factor of that inverse (the transpose of its lower factor).  A non-positive
    pivot raises numpy's LinAlgError.
    """
    h = _f64(Hd)
    L = np.linalg.cholesky(h)
    Linv = np.linalg.inv(L)
    hinv = Linv.T @ Linv
    hinv = 0.5 * (hinv + hinv.T)
    return np.linalg.cholesky(hinv).T


# ---------------------------------------------------------------------------------------------
# Quantization order
# ---------------------------------------------------------------------------------------------

def act_order(H) -> np.ndarray:
    """Columns by descending Hessian diagonal ([GEOM] 2.3, the role of the order: "act-order",
    named there as the cheap approximation of the min-pivot order).

    reading: the diagonal of H after the dead-feature fix (damping adds the same amount to every
    entry and changes nothing); equal values keep ascending column index.  Returns perm with
    perm[k] = the original column processed k-th.
    """
    d = np.diag(_f64(H))
    return np.array(sorted(range(d.shape[0]), key=lambda i: (-d[i], i)), dtype=np.int64)


def min_pivot_order(Hd) -> np.ndarray:
    """Greedy min-pivot order ([GEOM] 2.3: Theorem 5's D is the LDL diagonal of the permuted
    Hessian; the bound is tightened by taking, at each LDL step, the smallest diagonal entry).

    The LDL factorisation eliminates columns one at a time; a column's pivot is its variance
    given the columns eliminated before it.  Babai decides them in the opposite order (the
    column eliminated last, conditioned on all others, is decided first), so the processing
    order is the elimination order reversed.  At each step the remaining column with the
    smallest current Schur-complement diagonal is eliminated (ties: lowest column index); a
    non-positive pivot raises LinAlgError.  Returns perm, perm[k] = column processed k-th.
    """
    S = _f64(Hd).copy()
    n = S.shape[0]
    remaining = list(range(n))
    elim = []
    for _ in range(n):
        k = int(np.argmin([S[i, i] for i in remaining]))  # first minimum = lowest index
        i = remaining.pop(k)
        p = S[i, i]
        if not p > 0.0:
            raise np.linalg.LinAlgError("non-positive pivot")
        col = S[:, i].copy()
        S -= np.outer(col, col) / p  # Schur complement; eliminated rows/columns stay zero
        elim.append(i)
    return np.array(elim[::-1], dtype=np.int64)


# ---------------------------------------------------------------------------------------------
# The quantization grid
# ---------------------------------------------------------------------------------------------

def minmax_grid(w, bits: int):
    """Asymmetric min-max grid per row of ``w`` (rows x k) ([RDQ] group-128 asymmetric format).

    reading: the range always contains 0 (lo = min(min w, 0), hi = max(max w, 0)); an all-zero
    range becomes [-1, 1]; scale s = (hi - lo) / (2^b - 1); zero point z = rint(-lo / s), so
    z lies in [0, 2^b - 1].  rint is round-half-to-even.  Returns (s, z) as fp64 vectors.
    """
    s, zt = _minmax_unrounded(w, bits)
    return s, np.rint(zt)


def _minmax_unrounded(w, bits: int):
    """``minmax_grid``'s scale and its zero point before rounding, -lo / s."""
    w = _f64(w)
    maxq = float(2 ** bits - 1)
    lo = np.minimum(w.min(axis=1), 0.0)
    hi = np.maximum(w.max(axis=1), 0.0)
    flat = (lo == 0.0) & (hi == 0.0)
    lo = np.where(flat, -1.0, lo)
    hi = np.where(flat, 1.0, hi)
    s = (hi - lo) / maxq
    return s, -lo / s


def clipfree_grid(w, bits: int, alpha):
    """Per-row uniform grid for the clip-free variant ([GEOM] 2.3, no-clipping setting).

    reading: the step is alpha * (hi - lo) / (2^b - 1) with [lo, hi] as in ``minmax_grid`` and
    alpha >= 1 a per-row widening factor; the zero point centres the row's range on the code
    range, z = rint((2^b - 1)/2 - (hi + lo) / (2 s)) (equal to rint(-lo/s) when alpha = 1).
    """
    w = _f64(w)
    maxq = float(2 ** bits - 1)
    lo = np.minimum(w.min(axis=1), 0.0)
    hi = np.maximum(w.max(axis=1), 0.0)
    flat = (lo == 0.0) & (hi == 0.0)
    lo = np.where(flat, -1.0, lo)
    hi = np.where(flat, 1.0, hi)
    s = np.asarray(alpha, dtype=np.float64) * (hi - lo) / maxq
    z = np.rint(maxq / 2.0 - (hi + lo) / (2.0 * s))
    return s, z


def zsic_spacing(pivots) -> np.ndarray:
    """Per-column grid spacing of ZSIC ([WSIC] 2: alpha_i proportional to 1 / |l_ii|).

    ``pivots`` are the LDL pivots D_jj = l_jj^2 of the Hessian in the processing order.
    reading: the factors are normalised to geometric mean 1, kappa_j = g / |l_jj| with g the
    geometric mean of |l_jj|, so that a row's steps s kappa_j have the same geometric mean (the
    same log-volume of the lattice cell, i.e. the same entropy-coded rate) as the uniform step s.
    """
    l = np.sqrt(_f64(pivots))
    g = float(np.exp(np.mean(np.log(l))))
    return g / l


# ---------------------------------------------------------------------------------------------
# Column loops
# ---------------------------------------------------------------------------------------------

def gptq_columns(W, U, bits: int, group: int = 0, clip: bool = True, alpha=None, grid=None,
                 col_scale=None, follow=None, tie_tol: float = 1e-3):
    """GPTQ error-feedback loop, columns 0..n-1 in order ([GEOM] 2.2).

    For each column j: quantize the current column on the row's grid, error
    e = (w_j - q_j) / U_jj, and feed it forward, w_k -= e U_jk for k > j.  U is the upper
    factor of the inverse damped Hessian in this processing order.

    Grid (reading): per row (group == 0) from the row as given; per group of ``group`` columns,
    recomputed at the group's first column from the current, error-fed weights of the group.
    clip=False: codes are unconstrained integers (no clamp) on the ``clipfree_grid`` with the
    per-row factor ``alpha`` (group must be 0).  clip="unbounded" (HPTQ reading, [GEOM]
    section 3: one unconstrained integer grid for normal and outlier weights): the lattice
    s Z with the min-max step of the row (times ``alpha`` when given), zero point 0, no clamp.  ``grid`` = (s, z) fixes the per-row grid
    instead (a fixed lattice).  ``col_scale`` (per-row grids only) multiplies the step of
    column j by col_scale[j]: the grid of column j is s col_scale[j] (c - z).

    ``follow`` is a harness for comparing an implementation that carries the weights in
    lower precision: dict(codes = m x n, zeros = m x ngroups for group grids) of its decisions
    in processing order.  Where its code (or group zero point) differs from this loop's by one
    and this loop's unrounded value lies within ``tie_tol`` grid steps of the rounding boundary
    between the two, the loop takes the other decision and carries on from it, so that one
    near-tie does not change every later decision of the row; any other difference is counted
    and the loop keeps its own.  The result then also holds ``followed`` (decisions taken over)
    and ``disagree`` (differences beyond the tolerance).  The arithmetic is unchanged.

    Returns dict(codes, scales, zeros, Q, e) in processing order; e is the m x n matrix of
    scaled errors, whose squares sum to tr(D H_d D^T).
    """
    w = _f64(W).copy()
    u = _f64(U)
    m, n = w.shape
    maxq = 2 ** bits - 1
    if (not clip or clip == "unbounded") and group:
        raise ValueError("the clip-free and unbounded variants use a per-row grid")
    if col_scale is not None and group:
        raise ValueError("per-column spacing uses a per-row grid")
    kap = np.ones(n) if col_scale is None else _f64(col_scale)
    ngroups = 1 if group == 0 else -(-n // group)
    scales = np.zeros((m, ngroups))
    zeros = np.zeros((m, ngroups))
    codes = np.zeros((m, n), dtype=np.int64)
    Q = np.zeros((m, n))
    E = np.zeros((m, n))
    unbounded = clip == "unbounded"
    if unbounded:
        clip = False
    followed = disagree = 0

    def take(own, unrounded, other):
        """own decision, or the followed one where the two sit on either side of a near-tie
        (unrounded: this loop's value in the units the decision rounds)"""
        nonlocal followed, disagree
        diff = other != own
        tie = diff & (np.abs(other - own) == 1) & (np.abs(unrounded - (own + other) / 2) <= tie_tol)
        followed += int(np.count_nonzero(tie))
        disagree += int(np.count_nonzero(diff & ~tie))
        return np.where(tie, other, own)
    if group == 0:
        if grid is not None:
            s, z = (np.asarray(g, dtype=np.float64).copy() for g in grid)
        elif unbounded:
            s, _ = minmax_grid(w, bits)
            if alpha is not None:
                s = s * _f64(alpha)
            z = np.zeros(m)
        elif clip:
            s, z = minmax_grid(w, bits)
        else:
            s, z = clipfree_grid(w, bits, np.ones(m) if alpha is None else alpha)
        scales[:, 0], zeros[:, 0] = s, z
    for j in range(n):
        if group and j % group == 0:
            s, zt = _minmax_unrounded(w[:, j:j + group], bits)
            z = np.rint(zt)
            if follow is not None and follow.get("zeros") is not None:
                z = take(z, zt, np.asarray(follow["zeros"], dtype=np.float64)[:, j // group])
            scales[:, j // group], zeros[:, j // group] = s, z
        sj = s * kap[j]
        c = np.rint(w[:, j] / sj) + z
        if clip:
            c = np.clip(c, 0, maxq)
        if follow is not None:
            # boundary between codes c and c' in units of w / sj: (c + c') / 2 - z
            c = take(c, w[:, j] / sj + z, np.asarray(follow["codes"], dtype=np.float64)[:, j])
        q = sj * (c - z)
        e = (w[:, j] - q) / u[j, j]
        w[:, j + 1:] -= np.outer(e, u[j, j + 1:])
        codes[:, j] = c.astype(np.int64)
        Q[:, j] = q
        E[:, j] = e
    out = dict(codes=codes, scales=scales, zeros=zeros, Q=Q, e=E)
    if follow is not None:
        out.update(followed=followed, disagree=disagree)
    return out


def ssqr_columns(W, U, bits: int, alpha):
    """GPTQ with SSQR outliers ([GEOM] section 3, SSQR: weights that do not fit the low-bit
    grid are kept in full precision as sparse floating-point values).

    reading: the clip-free centred grid of ``clipfree_grid`` with the per-row factor ``alpha``;
    an entry whose code falls outside [0, 2^b - 1] is an outlier: it keeps its current
    (error-fed) value exactly, q = w, so its error e is 0 and nothing is fed forward.
    Returns dict(codes (outliers 0), outlier (bool mask), Q, e, scales, zeros).
    """
    w = _f64(W).copy()
    u = _f64(U)
    m, n = w.shape
    maxq = 2 ** bits - 1
    s, z = clipfree_grid(w, bits, alpha)
    codes = np.zeros((m, n), dtype=np.int64)
    mask = np.zeros((m, n), dtype=bool)
    Q = np.zeros((m, n))
    E = np.zeros((m, n))
    for j in range(n):
        c = np.rint(w[:, j] / s) + z
        out = (c < 0) | (c > maxq)
        q = np.where(out, w[:, j], s * (c - z))
        e = (w[:, j] - q) / u[j, j]
        w[:, j + 1:] -= np.outer(e, u[j, j + 1:])
        codes[:, j] = np.where(out, 0, c).astype(np.int64)
        mask[:, j] = out
        Q[:, j] = q
        E[:, j] = e
    return dict(codes=codes, outlier=mask, Q=Q, e=E, scales=s[:, None], zeros=z[:, None])


def ssqr_search(W, U, bits: int, density: float, steps: int = 20, max_doublings: int = 12):
    """Per-row scale search of SSQR ([GEOM] section 3: a binary search adjusts the scale to
    meet a target outlier density).

    reading: the smallest factor alpha (finest grid) whose outlier count is at most
    density * n.  alpha starts at 1 and doubles until the row is feasible (at most
    ``max_doublings`` times); then ``steps`` bisection steps in log2(alpha) between the last
    infeasible value (alpha / 2, or 2^-8 when alpha = 1 is already feasible) and the feasible
    one.  The result is always a feasible alpha.  Returns (result of ``ssqr_columns`` at the
    chosen alphas, alphas, the last infeasible log2 alphas).
    """
    w = _f64(W)
    m, n = w.shape
    limit = np.floor(density * n + 1e-9)
    hi = np.zeros(m)                       # log2 alpha, feasible once the doubling stops
    feas = ssqr_columns(w, U, bits, 2.0 ** hi)["outlier"].sum(axis=1) <= limit
    lo = np.where(feas, -8.0, np.nan)
    for _ in range(max_doublings):
        if feas.all():
            break
        bad = ~feas
        lo[bad] = hi[bad]
        hi[bad] += 1.0
        feas = ssqr_columns(w, U, bits, 2.0 ** hi)["outlier"].sum(axis=1) <= limit
    if not feas.all():
        raise ValueError("some rows exceed the outlier density even at the widest grid")
    for _ in range(steps):
        mid = 0.5 * (lo + hi)
        ok = ssqr_columns(w, U, bits, 2.0 ** mid)["outlier"].sum(axis=1) <= limit
        hi = np.where(ok, mid, hi)
        lo = np.where(ok, lo, mid)
    alpha = 2.0 ** hi
    return ssqr_columns(w, U, bits, alpha), alpha, lo


def hptq_rate(codes) -> float:
    """Bits per weight of the canonical Huffman code of integer codes ([GEOM] section 3, HPTQ):
    the symbols are the codes minus their minimum, counted over the whole array; the size is
    sum over symbols of count x code length (``huffman_lengths``), divided by the number of
    codes."""
    c = np.asarray(codes, dtype=np.int64)
    counts = np.bincount((c - c.min()).ravel())
    ln = huffman_lengths(counts)
    return float(np.sum(counts * ln[:counts.size])) / c.size


def hptq_search(W, U, bits: int, budget: float, steps: int = 12, max_doublings: int = 12):
    """HPTQ's rate control ([GEOM] section 3, HPTQ: one unconstrained integer lattice for normal
    and outlier weights, Huffman-coded so that a variable bit width meets a compression budget).

    reading: one factor alpha for the whole layer multiplies every row's min-max step (the
    unbounded lattice of ``gptq_columns``); the budget counts the Huffman-coded integers alone
    (``hptq_rate``), in bits per weight; alpha is the smallest factor (finest lattice) whose
    coded size, sum of count x length, is at most budget x (number of weights) bits.  The search
    is the one ``ssqr_search`` runs per row, here for the layer: alpha = 2^t from t = 0, t += 1
    until the layer fits (at most ``max_doublings`` times), then ``steps`` bisection steps in t
    between the last value that did not fit (t - 1, or -8 when t = 0 fits) and the one that
    does.  alpha = 2.0 ** t.  Returns (gptq_columns result at the chosen alpha, alpha, coded
    bits at alpha, the last t that did not fit).
    """
    w = _f64(W)
    m, n = w.shape
    limit = budget * float(m * n)

    def coded_bits(t):
        r = gptq_columns(w, U, bits, clip="unbounded", alpha=np.full(m, 2.0 ** t))
        c = r["codes"]
        counts = np.bincount((c - c.min()).ravel())
        return r, int(np.sum(counts * huffman_lengths(counts)[:counts.size]))

    hi = 0.0
    r, b = coded_bits(hi)
    lo = -8.0
    doublings = 0
    while b > limit:
        if doublings == max_doublings:
            raise ValueError("the layer exceeds the budget even at the widest lattice")
        lo, hi = hi, hi + 1.0
        r, b = coded_bits(hi)
        doublings += 1
    for _ in range(steps):
        mid = 0.5 * (lo + hi)
        _, bm = coded_bits(mid)
        if bm <= limit:
            hi = mid
        else:
            lo = mid
    r, b = coded_bits(hi)
    return r, 2.0 ** hi, b, lo


def babai_sic_reverse(W, L, bits: int, clip: bool = False, alpha=None):
    """Last-to-first successive interference cancellation ([WSIC] 2; [GEOM] 2.2 Theorem 4).

    With H_d = L L^T (L lower), column j (from n-1 down to 0) is rounded on the row grid at the
    target w_j + sum_{k>j} (L_kj / L_jj) (w_k - q_k), i.e. the decided columns' residuals are
    cancelled through the Cholesky factor.  Per-row grid (``clipfree_grid`` with ``alpha`` when
    clip=False, ``minmax_grid`` when clip=True).  Returns dict(codes, scales, zeros, Q, D).
    """
    w = _f64(W)
    l = _f64(L)
    m, n = w.shape
    maxq = 2 ** bits - 1
    if clip:
        s, z = minmax_grid(w, bits)
    else:
        s, z = clipfree_grid(w, bits, np.ones(m) if alpha is None else alpha)
    D = np.zeros((m, n))
    codes = np.zeros((m, n), dtype=np.int64)
    Q = np.zeros((m, n))
    for j in range(n - 1, -1, -1):
        target = w[:, j] + D[:, j + 1:] @ (l[j + 1:, j] / l[j, j])
        c = np.rint(target / s) + z
        if clip:
            c = np.clip(c, 0, maxq)
        q = s * (c - z)
        D[:, j] = w[:, j] - q
        codes[:, j] = c.astype(np.int64)
        Q[:, j] = q
    return dict(codes=codes, scales=s[:, None].copy(), zeros=z[:, None].copy(), Q=Q, D=D)


# ---------------------------------------------------------------------------------------------
# Packing, losses, bound
# ---------------------------------------------------------------------------------------------

def pack_codes(codes, bits: int) -> np.ndarray:
    """Per row, an LSB-first bitstream of b-bit codes in uint32 words.

    reading: code of column c occupies bits [b c, b c + b) of the row's stream; the row stride is
    ceil(n b / 32) words; unused high bits of the last word are 0.
    """
    codes = np.asarray(codes, dtype=np.uint64)
    m, n = codes.shape
    nwords = -(-n * bits // 32)
    out = np.zeros((m, nwords), dtype=np.uint64)
    for col in range(n):
        pos = col * bits
        wi, off = divmod(pos, 32)
        out[:, wi] |= (codes[:, col] << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            out[:, wi + 1] |= codes[:, col] >> np.uint64(32 - off)
    return out.astype(np.uint32)


# ---------------------------------------------------------------------------------------------
# Entropy coding of unconstrained integer codes
# ---------------------------------------------------------------------------------------------

def huffman_lengths(counts) -> np.ndarray:
    """Huffman code lengths for symbol counts ([GEOM] section 3, HPTQ: the integers of a single
    unconstrained grid are Huffman-coded).  Textbook construction: repeatedly merge the two
    least frequent trees; a symbol's length is its depth.  Symbols with count 0 get length 0;
    a lone symbol gets length 1.  Ties may be broken either way: every optimal code has the same
    total length sum(count * length), the quantity the tests compare.
    """
    import heapq
    counts = [int(c) for c in counts]
    live = [i for i, c in enumerate(counts) if c > 0]
    lengths = np.zeros(len(counts), dtype=np.int64)
    if len(live) == 1:
        lengths[live[0]] = 1
        return lengths
    heap = [(counts[i], k, [i]) for k, i in enumerate(live)]
    heapq.heapify(heap)
    uid = len(live)
    while len(heap) > 1:
        c1, _, s1 = heapq.heappop(heap)
        c2, _, s2 = heapq.heappop(heap)
        for i in s1 + s2:
            lengths[i] += 1
        heapq.heappush(heap, (c1 + c2, uid, s1 + s2))
        uid += 1
    return lengths


def canonical_codewords(lengths) -> np.ndarray:
    """Canonical prefix code for given lengths: symbols ordered by (length, symbol) receive
    consecutive codewords, shifted left by one at each increase of the length."""
    lengths = [int(x) for x in lengths]
    words = np.zeros(len(lengths), dtype=np.uint64)
    code, prev = 0, 0
    for ln, sym in sorted((ln, i) for i, ln in enumerate(lengths) if ln > 0):
        code <<= ln - prev
        words[sym] = code
        code += 1
        prev = ln
    return words


def huffman_encode(symbols, lengths) -> tuple[np.ndarray, int]:
    """Concatenate the canonical codewords of ``symbols`` MSB first into 64-bit words (stream
    bit i is bit 63 - i % 64 of word i // 64).  Returns (words, total bits)."""
    words = canonical_codewords(lengths)
    out = []
    for sym in np.asarray(symbols).ravel():
        ln = int(lengths[sym])
        out.append(format(int(words[sym]), f"0{ln}b"))
    bits = "".join(out)
    nw = -(-len(bits) // 64)
    padded = bits.ljust(64 * max(nw, 1), "0")
    arr = np.array([int(padded[64 * k:64 * k + 64], 2) for k in range(max(nw, 1))],
                   dtype=np.uint64)
    return arr, len(bits)


def huffman_decode(words, total_bits: int, lengths, count: int) -> np.ndarray:
    """Inverse of ``huffman_encode``: read ``count`` symbols of the canonical code."""
    cw = canonical_codewords(lengths)
    table = {(int(lengths[i]), int(cw[i])): i for i in range(len(lengths)) if lengths[i] > 0}
    bits = "".join(format(int(w), "064b") for w in np.asarray(words, dtype=np.uint64))[:total_bits]
    out, pos = [], 0
    for _ in range(count):
        ln, val = 0, 0
        while True:
            val = (val << 1) | (bits[pos] == "1")
            pos += 1
            ln += 1
            if (ln, val) in table:
                out.append(table[(ln, val)])
                break
    return np.array(out, dtype=np.int64)


def proxy_loss(W0, Q, X) -> float:
    """||(W0 - Q) X^T||_F^2: squared output error over the calibration tokens ([GEOM] 2.1)."""
    d = _f64(W0) - _f64(Q)
    y = d @ _f64(X).T
    return float(np.sum(y * y))


def quadratic_loss(W0, Q, H) -> float:
    """tr(D H D^T) with D = W0 - Q ([GEOM] 2.1 objective in Hessian form)."""
    d = _f64(W0) - _f64(Q)
    return float(np.sum((d @ _f64(H)) * d))


def babai_bound(scales_per_col, pivots) -> float:
    """Theorem 5 ([GEOM] 2.3): sum over rows of (1/4) sum_p s_{r,p}^2 D_pp.

    ``scales_per_col`` is rows x n (the step of each entry, in processing order); ``pivots`` is
    the diagonal D of the LDL factorisation of the processing-order Hessian, i.e. the squared
    Cholesky pivots.
    """
    s = _f64(scales_per_col)
    return float(0.25 * np.sum((s * s) @ _f64(pivots)))


# ---------------------------------------------------------------------------------------------
# The whole layer
# ---------------------------------------------------------------------------------------------

def quantize_layer(W, X, bits: int, group: int = 0, reverse: bool = False, clip: bool = True,
                   damp: float = 0.01, ladder: float = 1.25, ladder_max: int = 8,
                   rows=None, H=None, order=None, spacing: str = "uniform", follow=None,
                   tie_tol: float = 1e-3):
    """Quantize one linear layer: H, dead fix, damping, factor, column loop, losses.

    ``W`` is m x n (output rows x input features), ``X`` is T x n.  ``rows`` restricts the
    column loop to a subset of rows (rows are independent once the factor is known).  ``H``
    may be passed precomputed (2 X^T X) to share it across layers.

    Forward order uses the GPTQ form with U (``gptq_columns``).  Reverse order uses the SIC
    form with the lower Cholesky factor of H_d (``babai_sic_reverse``); per-row grids only.
    ``order`` = "act", "min_pivot" or an explicit permutation (perm[k] = column processed
    k-th) runs the GPTQ form on the columns in that order, with U the factor of the permuted
    H_d; group grids then cover consecutive columns of the processing order (reading: the pages
    do not combine groups with an order), so scales / zeros are indexed by processing group.

    spacing="zsic" (per-row grids, forward or an explicit order): column j's step is the row
    step times ``zsic_spacing`` of the processing order's pivots.

    clip="unbounded": codes are any integers on the per-row lattice s Z (see gptq_columns), no
    ladder; they are meant for entropy coding (``huffman_lengths``).

    clip=False (reading of "per-row step set so that no entry needs clipping"): run unclamped;
    a row whose codes leave [0, 2^b - 1] is rerun with alpha multiplied by ``ladder``, at most
    ``ladder_max`` times; rows still outside raise ValueError.

    ``follow`` (GPTQ form, clipped or unbounded grids): another implementation's decisions for
    the selected rows, dict(codes in the original column order, zeros by processing group),
    taken over at near-ties as ``gptq_columns`` describes; the result adds ``followed`` and
    ``disagree``.

    Returns a dict; codes / scales / zeros / Q are in the original column order.
    """
    w_in = _f64(W)
    m, n = w_in.shape
    if H is None:
        H = hessian(X)
    h_fix, w0, dead = fix_dead_features(H, w_in)
    hd, delta = dampen(h_fix, damp)
    sel = np.arange(m) if rows is None else np.asarray(rows)
    w_sel = w0[sel]
    maxq = 2 ** bits - 1
    if reverse and group:
        raise ValueError("the last-to-first variant uses a per-row grid")
    if reverse and clip == "unbounded":
        raise ValueError("the unbounded lattice takes the forward or ordered form")
    perm = None
    if order is not None:
        if reverse:
            raise ValueError("an order replaces the reverse flag")
        if isinstance(order, str):
            perm = act_order(h_fix) if order == "act" else min_pivot_order(hd) if order == "min_pivot" else None
            if perm is None:
                raise ValueError(f"unknown order {order!r}")
        else:
            perm = np.asarray(order, dtype=np.int64)
            if sorted(perm.tolist()) != list(range(n)):
                raise ValueError("order is not a permutation of the columns")

    if follow is not None and (reverse or clip is False):
        raise ValueError("follow takes the GPTQ form without the scale ladder")
    if spacing not in ("uniform", "zsic"):
        raise ValueError(f"unknown spacing {spacing!r}")
    if spacing == "zsic" and (reverse or group):
        raise ValueError("ZSIC spacing here takes a per-row grid and the forward / ordered form")
    kap = None
    if perm is not None:
        U = hinv_upper_factor(hd[np.ix_(perm, perm)])
        pivots = 1.0 / np.diag(U) ** 2  # in processing order
        if spacing == "zsic":
            kap = zsic_spacing(pivots)

        fol = None if follow is None else dict(codes=np.asarray(follow["codes"])[:, perm],
                                               zeros=follow.get("zeros"))

        def run(rows_w, alpha):
            r = gptq_columns(rows_w[:, perm], U, bits, group=group, clip=clip, alpha=alpha,
                             col_scale=kap, follow=fol, tie_tol=tie_tol)
            for key in ("codes", "Q"):
                back = np.empty_like(r[key])
                back[:, perm] = r[key]
                r[key] = back
            return r
    elif reverse:
        L = np.linalg.cholesky(hd)
        pivots = np.diag(L) ** 2

        def run(rows_w, alpha):
            return babai_sic_reverse(rows_w, L, bits, clip=clip, alpha=alpha)
    else:
        U = hinv_upper_factor(hd)
        pivots = 1.0 / np.diag(U) ** 2
        if spacing == "zsic":
            kap = zsic_spacing(pivots)

        def run(rows_w, alpha):
            return gptq_columns(rows_w, U, bits, group=group, clip=clip, alpha=alpha,
                                col_scale=kap, follow=follow, tie_tol=tie_tol)

    alpha = np.ones(len(sel))
    res = run(w_sel, alpha)
    retries = 0
    if clip is False:
        for _ in range(ladder_max):
            bad = np.nonzero((res["codes"] < 0).any(axis=1) | (res["codes"] > maxq).any(axis=1))[0]
            if bad.size == 0:
                break
            retries += 1
            alpha[bad] *= ladder
            sub = run(w_sel[bad], alpha[bad])
            for key in ("codes", "scales", "zeros", "Q"):
                res[key][bad] = sub[key]
        bad = (res["codes"] < 0).any(axis=1) | (res["codes"] > maxq).any(axis=1)
        if bad.any():
            raise ValueError(f"{int(bad.sum())} rows still overflow after the scale ladder")

    Q = res["Q"]
    g = group if group else n
    s_cols = np.repeat(res["scales"], g, axis=1)[:, :n]  # processing order
    if kap is not None:
        s_cols = s_cols * kap[None, :]
    out = dict(H=H, dead=dead, delta=delta, Hd=hd, codes=res["codes"], scales=res["scales"],
               zeros=res["zeros"], Q=Q, alpha=alpha, ladder_rounds=retries, perm=perm,
               col_scale=kap)
    if follow is not None:
        out["followed"], out["disagree"] = res["followed"], res["disagree"]
    if reverse:
        out["L"] = L
    else:
        out["U"] = U
        out["sum_e2"] = float(np.sum(res["e"] ** 2))
    w0_sel = w0[sel]
    out["loss_damped"] = quadratic_loss(w0_sel, Q, hd)
    if X is not None:
        out["loss_proxy"] = proxy_loss(w0_sel, Q, X)
    out["loss_proxy_h"] = 0.5 * quadratic_loss(w0_sel, Q, h_fix)
    # pivots: 1/U_jj^2 in processing order (forward, or an explicit order), L_jj^2 (reverse,
    # per-row grid, so the column order of s_cols does not matter)
    out["bound"] = babai_bound(s_cols, pivots)
    out["packed"] = pack_codes(np.clip(res["codes"], 0, maxq), bits)
    if clip == "unbounded":
        sym = res["codes"] - res["codes"].min()
        ln = huffman_lengths(np.bincount(sym.ravel()))
        out["huffman_bits"] = int(np.sum(np.bincount(sym.ravel()) * ln[:sym.max() + 1]))
        out["rate"] = out["huffman_bits"] / sym.size
    return out
