"""Pins that tie the CPU oracle to the pages and to mathematics, not to itself.

Each function takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with something the method or arithmetic fixes:

* exact-rational brute force of the top-k over all N outer sums (Python
  ``fractions``), which shares nothing with the oracle's TwoSum ordering;
* the product-key identity topk(s1 (+) s2) = topk(topk(s1) (+) topk(s2))
  (SDM explainer section 3.1 step 1; technical summary Core Mechanism 2);
* hand-worked fixtures under ``tests/golden``;
* closed forms and invariants of the write/read recurrence (SDM explainer
  section 3.1 steps 2-3; technical summary Core Mechanism 3-4);
* round-to-nearest-even to bf16 checked with exact rationals.

``ALL_PINS`` is used both by the ordinary tests and by the planted-mistake
tests, which rebuild the oracle with one known error and require that at least
one pin fails.
"""

from __future__ import annotations

import json
import math
from fractions import Fraction
from pathlib import Path

import numpy as np

GOLDEN = Path(__file__).resolve().parent / "golden"


# ---------------------------------------------------------------- selection --

def brute_force_topk(s1, s2, K):
    """All N = len(s1)*len(s2) slots ordered by (exact sum desc, slot asc)."""
    n = len(s1)
    cells = []
    for a in range(n):
        for b in range(n):
            cells.append((-(Fraction(float(s1[a])) + Fraction(float(s2[b]))), a * n + b))
    cells.sort()
    return [slot for _, slot in cells[:K]], [-key for key, _ in cells[:K]]


def product_key_topk(s1, s2, K):
    """topk(topk(s1) (+) topk(s2)): per-half top-min(K, n), then the merge."""
    n = len(s1)
    kh = min(K, n)

    def half_top(s):
        order = sorted(range(n), key=lambda i: (-Fraction(float(s[i])), i))
        return order[:kh]

    cand = []
    for a in half_top(s1):
        for b in half_top(s2):
            cand.append((-(Fraction(float(s1[a])) + Fraction(float(s2[b]))), a * n + b))
    cand.sort()
    return [slot for _, slot in cand[:K]]


def _selection_inputs(rng, sqrt_n):
    """Random, tie-heavy, signed-zero and rounding-tie score vectors."""
    cases = []
    cases.append(rng.standard_normal(2 * sqrt_n).astype(np.float32))
    cases.append(rng.integers(-1, 2, size=2 * sqrt_n).astype(np.float32))
    z = np.zeros(2 * sqrt_n, dtype=np.float32)
    z[rng.integers(0, 2, size=2 * sqrt_n).astype(bool)] = -0.0
    cases.append(z)
    # s2 = 1 everywhere and tiny distinct s1: the sums differ only below
    # double precision, so only an exact comparison orders them correctly.
    rt = np.empty(2 * sqrt_n, dtype=np.float32)
    rt[:sqrt_n] = [2.0 ** (-60 - (i % 7)) for i in range(sqrt_n)]
    rt[sqrt_n:] = 1.0
    cases.append(rt)
    return cases


def pin_selection_brute_force(o, sizes=(1, 2, 3, 4, 8, 16)):
    rng = np.random.default_rng(1234)
    for sqrt_n in sizes:
        n = sqrt_n * sqrt_n
        ks = range(1, n + 1) if n <= 16 else sorted({1, 2, 3, 7, 8, n // 4, n // 2, n - 1, n})
        for x in _selection_inputs(rng, sqrt_n):
            for K in ks:
                idx, w = o.pkm_topk(x[None], K)
                want, _ = brute_force_topk(x[:sqrt_n], x[sqrt_n:], K)
                assert list(idx[0]) == want, (sqrt_n, K, x.tolist(), list(idx[0]), want)


def pin_selection_identity(o):
    """The product-key identity holds under the (exact sum, lowest slot) order,
    and the oracle (which never uses it) agrees with it."""
    rng = np.random.default_rng(99)
    for sqrt_n in (2, 4, 5, 8):
        for x in _selection_inputs(rng, sqrt_n):
            for K in (1, 2, sqrt_n, 2 * sqrt_n if 2 * sqrt_n <= sqrt_n * sqrt_n else 1):
                bf, _ = brute_force_topk(x[:sqrt_n], x[sqrt_n:], K)
                assert product_key_topk(x[:sqrt_n], x[sqrt_n:], K) == bf
                idx, _ = o.pkm_topk(x[None], K)
                assert list(idx[0]) == bf


def pin_selection_golden(o):
    data = json.loads((GOLDEN / "pkm_topk_worked.json").read_text())
    for case in data["cases"]:
        x = np.asarray(case["s1"] + case["s2"], dtype=np.float32)
        idx, w = o.pkm_topk(x[None], case["K"])
        assert list(idx[0]) == case["idx"], (case["name"], list(idx[0]))
        sc = np.asarray(case["scores"], dtype=np.float64)
        assert abs(w[0].sum() - 1.0) < 1e-12
        assert np.allclose(w[0] / w[0, 0], np.exp(sc - sc[0]), rtol=1e-12, atol=0), (case["name"], w[0])


def pin_weights(o):
    """Softmax weights: sum to one, K = 1 gives exactly 1, equal scores give
    equal weights, and w_i / w_j = exp(score_i - score_j) (exact scores)."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((20, 16)).astype(np.float32)
    for K in (1, 3, 8, 64):
        idx, w = o.pkm_topk(x, K)
        assert np.all(np.abs(w.sum(-1) - 1.0) < 1e-12)
        if K == 1:
            assert np.all(w == 1.0)
        for u in range(x.shape[0]):
            s1, s2 = x[u, :8], x[u, 8:]
            _, sums = brute_force_topk(s1, s2, K)
            sc = np.array([float(s) for s in sums])
            assert np.all(np.diff(w[u]) <= 1e-15)  # non-increasing along selection order
            ratio = w[u] / w[u, 0]
            assert np.allclose(ratio, np.exp(sc - sc[0]), rtol=1e-12, atol=0)
    ties = np.zeros((1, 8), dtype=np.float32)
    _, w = o.pkm_topk(ties, 5)
    assert np.all(w[0] == w[0, 0]) and abs(w[0, 0] - 0.2) < 1e-15


# ---------------------------------------------------------------- recurrence --

def random_selection(rng, B, T, H, N, K):
    """Distinct random slots per token-head with random positive weights."""
    idx = np.empty((B, T, H, K), dtype=np.int32)
    for i in np.ndindex(B, T, H):
        idx[i] = rng.choice(N, size=K, replace=False)
    w = rng.random((B, T, H, K)) + 0.05
    w /= w.sum(-1, keepdims=True)
    return idx, w


def _scan_inputs(rng, B=2, T=17, H=3, N=37, d_v=5, W=4, R=3):
    idx_w, w_w = random_selection(rng, B, T, H, N, W)
    idx_r, w_r = random_selection(rng, B, T, H, N, R)
    v = rng.standard_normal((B, T, H, d_v)).astype(np.float32)
    alpha = np.exp(-np.log1p(np.exp(rng.standard_normal((B, T, H))))).astype(np.float32)
    beta = rng.random((B, T, H)).astype(np.float32)
    M = (0.02 * rng.standard_normal((B, H, N, d_v))).astype(np.float32)
    return dict(idx_w=idx_w, w_w=w_w, idx_r=idx_r, w_r=w_r, v=v, alpha=alpha, beta=beta, M=M)


def pin_scan_golden(o):
    data = json.loads((GOLDEN / "scan_worked.json").read_text())
    for case in data["cases"]:
        arr = lambda k, dt: np.asarray(case[k], dtype=dt)
        y, M_T, _ = o.scan(arr("idx_w", np.int32), arr("w_w", np.float64), arr("idx_r", np.int32),
                           arr("w_r", np.float64), arr("v", np.float32), arr("alpha", np.float32),
                           arr("beta", np.float32), arr("M0", np.float32))
        assert np.array_equal(y, np.asarray(case["y"], dtype=np.float64)), (case["name"], y)
        assert np.array_equal(M_T, np.asarray(case["M_T"], dtype=np.float32)), (case["name"], M_T)


def pin_scan_identity_gates(o):
    """alpha = 1, beta = 0: the write is the identity, so M_T == M0 bit for bit
    and every read is the weighted gather of M0 (np.einsum)."""
    rng = np.random.default_rng(7)
    d = _scan_inputs(rng)
    d["alpha"][:] = 1.0
    d["beta"][:] = 0.0
    y, M_T, _ = o.scan(**d)
    assert np.array_equal(M_T, d["M"])
    B, T, H, R = d["idx_r"].shape
    for b, t, h in np.ndindex(B, T, H):
        rows = d["M"][b, h, d["idx_r"][b, t, h]].astype(np.float64)
        want = np.einsum("r,rc->c", d["w_r"][b, t, h], rows)
        assert np.allclose(y[b, t, h], want, rtol=1e-14, atol=1e-15)


def pin_scan_beta_one_overwrites(o, state_bf16=False):
    """beta = 1 with one write slot of weight 1 overwrites that slot with v
    exactly; a read of the same slot after the write returns v (read after
    write), not the previous token's value."""
    rng = np.random.default_rng(11)
    B, T, H, N, d_v = 1, 9, 2, 6, 4
    idx = rng.integers(0, N, size=(B, T, H, 1)).astype(np.int32)
    one = np.ones((B, T, H, 1))
    v = rng.standard_normal((B, T, H, d_v)).astype(np.float32)
    if state_bf16:
        v = np.vectorize(o.round_to_bf16)(v).astype(np.float32)
    alpha = rng.random((B, T, H)).astype(np.float32)
    beta = np.ones((B, T, H), dtype=np.float32)
    M = (0.02 * rng.standard_normal((B, H, N, d_v))).astype(np.float32)
    if state_bf16:
        M = np.vectorize(o.round_to_bf16)(M).astype(np.float32)
    y, M_T, _ = o.scan(idx, one, idx, one, v, alpha, beta, M, state_bf16=state_bf16)
    assert np.array_equal(y.astype(np.float32), v)
    for h in range(H):
        last = {}
        for t in range(T):
            last[int(idx[0, t, h, 0])] = v[0, t, h]
        for i in range(N):
            want = last.get(i, M[0, h, i])
            assert np.array_equal(M_T[0, h, i], want)


def pin_scan_unselected_untouched(o):
    rng = np.random.default_rng(13)
    d = _scan_inputs(rng, N=64, T=9)
    y, M_T, _ = o.scan(**d)
    B, T, H, _ = d["idx_w"].shape
    for b, h in np.ndindex(B, H):
        written = set(d["idx_w"][b, :, h].ravel().tolist())
        for i in range(64):
            if i not in written:
                assert np.array_equal(M_T[b, h, i], d["M"][b, h, i])
            else:
                assert not np.array_equal(M_T[b, h, i], d["M"][b, h, i])


def pin_scan_closed_form(o):
    """One slot written every token with weight 1, constant gates:
    m_T = a^T m_0 + c * sum_t a^(T-1-t) v_t with a = alpha(1 - beta), c = beta
    (geometric series of the per-slot delta rule)."""
    rng = np.random.default_rng(17)
    B, T, H, N, d_v = 1, 40, 1, 5, 3
    slot = 3
    idx = np.full((B, T, H, 1), slot, dtype=np.int32)
    one = np.ones((B, T, H, 1))
    al, be = 0.8125, 0.375  # exact binary fractions
    v = rng.standard_normal((B, T, H, d_v)).astype(np.float32)
    alpha = np.full((B, T, H), al, dtype=np.float32)
    beta = np.full((B, T, H), be, dtype=np.float32)
    M = rng.standard_normal((B, H, N, d_v)).astype(np.float32)
    y, M_T, _ = o.scan(idx, one, idx, one, v, alpha, beta, M)
    a, c = al * (1 - be), be
    m = M[0, 0, slot].astype(np.float64) * a ** T
    for t in range(T):
        m = m + c * a ** (T - 1 - t) * v[0, t, 0].astype(np.float64)
    # fp32 rounding of each of T stores, contracted by a < 1 each step
    assert np.allclose(M_T[0, 0, slot], m, rtol=0, atol=4 * 2.0 ** -24 * (1 + np.abs(m).max()) / (1 - a))
    # reads follow the same series token by token
    mt = M[0, 0, slot].astype(np.float64)
    for t in range(T):
        mt = a * mt + c * v[0, t, 0].astype(np.float64)
        assert np.allclose(y[0, t, 0], mt, rtol=0, atol=4 * 2.0 ** -24 * (1 + np.abs(mt).max()) / (1 - a))


def pin_scan_convex_bound(o):
    """With 0 < alpha <= 1, 0 <= beta <= 1 and softmax weights the write is a
    convex combination of the old row and v, and the read a convex combination
    of rows: |M_T| <= max(|M0|, |v|) and |y| <= that bound."""
    rng = np.random.default_rng(19)
    d = _scan_inputs(rng, N=20, T=30)
    y, M_T, _ = o.scan(**d)
    bound = max(np.abs(d["M"]).max(), np.abs(d["v"]).max())
    assert np.abs(M_T).max() <= bound * (1 + 1e-6)
    assert np.abs(y).max() <= bound * (1 + 1e-6)


def pin_scan_chunking(o):
    """The state carries the recurrence: scanning [0, T1) then [T1, T) from the
    intermediate state equals one scan over [0, T), bit for bit."""
    rng = np.random.default_rng(23)
    d = _scan_inputs(rng, T=21)
    y, M_T, _ = o.scan(**d)
    T1 = 8
    part = lambda a, lo, hi: a[:, lo:hi]
    keys = ["idx_w", "w_w", "idx_r", "w_r", "v", "alpha", "beta"]
    y1, M1, _ = o.scan(**{k: part(d[k], 0, T1) for k in keys}, M=d["M"])
    y2, M2, _ = o.scan(**{k: part(d[k], T1, 21) for k in keys}, M=M1)
    assert np.array_equal(np.concatenate([y1, y2], axis=1), y)
    assert np.array_equal(M2, M_T)


def pin_scan_ops_independent_of_n(o):
    """Per-token work is (4W + 2R) d_v operations whatever N is (SDM explainer
    section 3.2; technical summary IsoFLOP Design)."""
    rng = np.random.default_rng(29)
    B, T, H, d_v, W, R = 1, 3, 1, 4, 4, 2
    counts = []
    for N in (1 << 10, 1 << 14, 1 << 18):
        d = _scan_inputs(rng, B=B, T=T, H=H, N=N, d_v=d_v, W=W, R=R)
        _, _, ops = o.scan(**d)
        counts.append(ops)
    assert counts == [B * T * H * (4 * W + 2 * R) * d_v] * 3, counts


def pin_scan_bf16_state(o):
    """With a bf16 state every stored value is exactly representable in bf16,
    and the update stays within bf16 rounding of the fp32-state result."""
    rng = np.random.default_rng(31)
    d = _scan_inputs(rng, N=16, T=12)
    d["M"] = np.vectorize(o.round_to_bf16)(d["M"]).astype(np.float32)
    _, M16, _ = o.scan(**d, state_bf16=True)
    _, M32, _ = o.scan(**d, state_bf16=False)
    bits = M16.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)
    assert np.abs(M16 - M32).max() <= 2.0 ** -8 * 12 * max(1.0, np.abs(M32).max())
    assert not np.array_equal(M16, M32)


def pin_epilogue(o):
    """RMS-norm then gate: with g = 1 the output's mean square is
    ms / (ms + eps) of the ungated read; g scales element-wise; a constant
    factor on the state cancels up to eps."""
    rng = np.random.default_rng(37)
    d = _scan_inputs(rng, N=16, T=6, d_v=8)
    eps = 1e-6
    y0, _, _ = o.scan(**d)
    ones = np.ones_like(d["v"])
    y1, _, _ = o.scan(**d, g=ones, eps=eps)
    ms = (y0 ** 2).mean(-1)
    assert np.allclose((y1 ** 2).mean(-1), ms / (ms + eps), rtol=1e-12)
    assert np.allclose(y1 * np.sqrt(ms + eps)[..., None], y0, rtol=1e-12, atol=1e-15)
    g = rng.standard_normal(d["v"].shape).astype(np.float32)
    yg, _, _ = o.scan(**d, g=g, eps=eps)
    assert np.allclose(yg, y1 * g, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- rounding --

def _bf16_rne(x: float) -> float:
    """Round-to-nearest-even onto the bf16 grid with exact rationals."""
    if x == 0 or not math.isfinite(x):
        return x
    fx = Fraction(x)
    e = math.floor(math.log2(abs(x)))
    while Fraction(2) ** e > abs(fx):
        e -= 1
    while Fraction(2) ** (e + 1) <= abs(fx):
        e += 1
    q = max(e - 7, -133)
    scaled = fx / Fraction(2) ** q
    lo = math.floor(scaled)
    rem = scaled - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return float(lo * Fraction(2) ** q)


def pin_round_to_bf16(o):
    rng = np.random.default_rng(41)
    vals = list(rng.standard_normal(300)) + list(rng.standard_normal(100) * 1e-39)
    vals += [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -30, 2 ** -133,
             3 * 2 ** -134, 2 ** -134, 1.0, -2.5, 0.1, 65504.0]
    for x in vals:
        assert o.round_to_bf16(float(x)) == _bf16_rne(float(x)), x


# ----------------------------------------------------------------- backward --
# The backward (training derivatives) of the write/read recurrence and of the
# selection weights. The SDM explainer's section 3.4 says only that a
# memory-efficient backward exists; its derivatives follow from the forward
# formulas by the chain rule, so the forward itself (pinned above) is the
# reference: central finite differences of the double-precision forward.


def _scan_loss(o, inp, dy, dM_T):
    y, M_T = o.scan_f64(inp["idx_w"], inp["w_w"], inp["idx_r"], inp["w_r"], inp["v"], inp["alpha"],
                        inp["beta"], inp["M"])
    return float(np.sum(dy * y) + np.sum(dM_T * M_T))


def _backward_case(seed, T=6, N=11, W=3, R=2):
    rng = np.random.default_rng(seed)
    inp = _scan_inputs(rng, B=1, T=T, H=2, N=N, d_v=3, W=W, R=R)
    inp = {k: (v.astype(np.float64) if v.dtype == np.float32 else v) for k, v in inp.items()}
    inp["M"] = rng.standard_normal(inp["M"].shape)  # O(1) state so every term matters
    dy = rng.standard_normal(inp["v"].shape)
    dM_T = rng.standard_normal(inp["M"].shape)
    return rng, inp, dy, dM_T


def pin_backward_finite_differences(o):
    """<grad, D> equals the central difference (L(x + hD) - L(x - hD)) / 2h of
    L = sum <dy, y> + <dM_T, M_T> for a random direction D in each input, and
    for single coordinates of each input."""
    for seed in (0, 1):
        rng, inp, dy, dM_T = _backward_case(seed)
        g = o.scan_backward(inp["idx_w"], inp["w_w"], inp["idx_r"], inp["w_r"], inp["v"], inp["alpha"],
                            inp["beta"], inp["M"], dy, dM_T)
        grads = {"v": g["dv"], "alpha": g["dalpha"], "beta": g["dbeta"], "w_w": g["dw_w"], "w_r": g["dw_r"],
                 "M": g["dM0"]}
        h = 1e-6
        for name, grad in grads.items():
            dirs = [rng.standard_normal(grad.shape)]
            for _ in range(3):
                e = np.zeros(grad.shape)
                e[tuple(int(rng.integers(0, n)) for n in grad.shape)] = 1.0
                dirs.append(e)
            for D in dirs:
                plus = dict(inp, **{name: inp[name] + h * D})
                minus = dict(inp, **{name: inp[name] - h * D})
                fd = (_scan_loss(o, plus, dy, dM_T) - _scan_loss(o, minus, dy, dM_T)) / (2 * h)
                an = float(np.sum(grad * D))
                assert abs(fd - an) <= 1e-6 * (1.0 + abs(an)), (name, seed, fd, an)


def pin_backward_one_slot_golden(o):
    """Hand-derived derivatives of one write and one read of one slot
    (tests/golden/backward_one_slot.json), exact binary fractions."""
    data = json.loads((GOLDEN / "backward_one_slot.json").read_text())
    x = data["inputs"]
    one = lambda val, dt=np.float64: np.full((1, 1, 1, 1), val, dtype=dt)
    for case in data["cases"]:
        g = o.scan_backward(one(0, np.int32), one(x["k"]), one(0, np.int32), one(x["q"]), one(x["v"]),
                            np.full((1, 1, 1), x["alpha"]), np.full((1, 1, 1), x["beta"]), one(x["M0"]),
                            one(case["dy"]), one(case["dM_T"]))
        got = {"dw_r": g["dw_r"], "dM0": g["dM0"], "dv": g["dv"], "dalpha": g["dalpha"], "dbeta": g["dbeta"],
               "dw_w": g["dw_w"]}
        for k, arr in got.items():
            assert float(arr.ravel()[0]) == case[k], (case["name"], k, float(arr.ravel()[0]), case[k])


def pin_backward_unselected_pass_through(o):
    """Slots that no token writes pass dL/dM_T to dL/dM_0 unchanged, plus the
    read contributions sum_t q dy_t for slots that are only read."""
    rng, inp, dy, dM_T = _backward_case(3, T=5, N=40)
    g = o.scan_backward(inp["idx_w"], inp["w_w"], inp["idx_r"], inp["w_r"], inp["v"], inp["alpha"],
                        inp["beta"], inp["M"], dy, dM_T)
    written = set(inp["idx_w"].ravel().tolist())
    for h in range(inp["M"].shape[1]):
        for s in range(inp["M"].shape[2]):
            if s in written:
                continue
            want = dM_T[0, h, s].copy()
            for t in range(inp["idx_r"].shape[1]):
                for r in range(inp["idx_r"].shape[3]):
                    if inp["idx_r"][0, t, h, r] == s:
                        want += inp["w_r"][0, t, h, r] * dy[0, t, h]
            assert np.allclose(g["dM0"][0, h, s], want, rtol=0, atol=1e-12), (h, s)


def _softmax_loss(o, x, dw, K):
    idx, w = o.pkm_topk(x, K)
    return idx, float(np.sum(dw * w))


def pin_topk_backward(o):
    """d/dscores of <dw, w(scores)> for a fixed selection: central differences
    in fp32 scores with a power-of-two step (exact in fp32), and the invariant
    that each half's derivatives sum to zero (softmax is shift invariant)."""
    rng = np.random.default_rng(7)
    sqrt_n, K = 6, 5
    x = rng.standard_normal((3, 2 * sqrt_n)).astype(np.float32)
    dw = rng.standard_normal((3, K))
    idx, w = o.pkm_topk(x, K)
    ds = o.pkm_topk_backward(idx, w, dw, sqrt_n)
    assert np.allclose(ds[:, :sqrt_n].sum(-1), 0.0, atol=1e-12) and np.allclose(ds[:, sqrt_n:].sum(-1), 0.0,
                                                                                 atol=1e-12)
    h = np.float32(2.0 ** -12)
    for u in range(x.shape[0]):
        for j in range(2 * sqrt_n):
            xp, xm = x.copy(), x.copy()
            xp[u, j] += h
            xm[u, j] -= h
            ip, lp = _softmax_loss(o, xp[u:u + 1], dw[u:u + 1], K)
            im, lm = _softmax_loss(o, xm[u:u + 1], dw[u:u + 1], K)
            if not (np.array_equal(ip[0], idx[u]) and np.array_equal(im[0], idx[u])):
                continue  # the step moved the selection; the derivative is not defined there
            fd = (lp - lm) / (2 * float(h))
            assert abs(fd - ds[u, j]) <= 1e-5 * (1.0 + abs(ds[u, j])), (u, j, fd, ds[u, j])


def pin_epilogue_backward(o):
    """The epilogue's derivatives: a hand-worked row (tests/golden/epilogue_backward.json) and central
    differences of the double-precision epilogue along random directions in x and g."""
    data = json.loads((GOLDEN / "epilogue_backward.json").read_text())
    dx, dg = o.rmsnorm_gate_backward(np.array([data["x"]]), np.array([data["g"]]), np.array([data["dout"]]),
                                     eps=data["eps"])
    assert np.array_equal(dx[0], np.array(data["dx"])) and np.array_equal(dg[0], np.array(data["dg"])), (dx, dg)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((3, 5))
    g = rng.standard_normal((3, 5))
    dout = rng.standard_normal((3, 5))
    dx, dg = o.rmsnorm_gate_backward(x, g, dout, eps=1e-3)
    loss = lambda xx, gg: float(np.sum(dout * o.rmsnorm_gate(xx, gg, eps=1e-3)))
    h = 1e-6
    for _ in range(4):
        D = rng.standard_normal(x.shape)
        fd = (loss(x + h * D, g) - loss(x - h * D, g)) / (2 * h)
        assert abs(fd - np.sum(dx * D)) <= 1e-6 * (1 + abs(fd)), ("dx", fd, np.sum(dx * D))
        fd = (loss(x, g + h * D) - loss(x, g - h * D)) / (2 * h)
        assert abs(fd - np.sum(dg * D)) <= 1e-6 * (1 + abs(fd)), ("dg", fd, np.sum(dg * D))


# --------------------------------------------------- block-scaled fp8 state --

def _e4m3_grid():
    """All non-negative finite E4M3 values, from the format's definition
    (bias 7, 3 mantissa bits, subnormals m * 2^-9, largest 1.75 * 2^8), as
    exact fractions with their codes."""
    grid = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # NaN
            val = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
            grid.append((val, (e << 3) | m))
    return sorted(grid)


def _rne_e4m3(x: Fraction) -> int:
    """Exact round-to-nearest-even onto the E4M3 grid, clamped to 448."""
    grid = _e4m3_grid()
    sign = 0x80 if x < 0 else 0
    a = abs(x)
    if a >= grid[-1][0]:
        return sign | grid[-1][1]
    for (lo, cl), (hi, ch) in zip(grid, grid[1:]):
        if lo <= a <= hi:
            if a - lo < hi - a:
                return sign | cl
            if a - lo > hi - a:
                return sign | ch
            return sign | (cl if cl % 2 == 0 else ch)
    raise AssertionError(x)


def pin_e4m3_rounding(o):
    """Decoding of every finite code and round-to-nearest-even (with
    saturation) against an exact-rational reference of the format: at every
    representable value, every midpoint, beyond 448 and at random values."""
    grid = _e4m3_grid()
    for val, code in grid:
        assert o.decode_e4m3(code) == float(val) and o.decode_e4m3(0x80 | code) == -float(val), code
    probes = [v for v, _ in grid] + [(a + b) / 2 for (a, _), (b, _) in zip(grid, grid[1:])]
    probes += [Fraction(449), Fraction(464), Fraction(480), Fraction(10 ** 6), Fraction(1, 2 ** 11)]
    rng = np.random.default_rng(3)
    probes += [Fraction(float(x)) for x in np.exp(rng.uniform(-9, 6.5, 400))]
    for p in probes:
        for x in (p, -p):
            got = o.round_e4m3(float(x))
            want = _rne_e4m3(x)
            if x == 0:
                continue  # the sign of zero follows the input's sign bit
            assert got == want, (float(x), got, want)


def pin_fp8blk_blocks(o):
    """Each block's exponent is the smallest e for which the nearest-even
    E4M3 rounding of max|x| / 2^e is at most 448, i.e. max|x| <= 464 * 2^e
    (464 is the midpoint of 448 and the next step 480 and rounds to the even
    448), so the largest magnitude lands in (232, 464] and nothing is clipped;
    an all-zero block gets exponent 0. Codes are the exact rounding of
    x / 2^e, and quantising a dequantised block gives it back."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((40, 16)).astype(np.float32)
    x *= np.float32(2.0) ** rng.integers(-20, 20, (40, 1)).astype(np.float32)
    x[3] = 0.0
    x[5, :15] = 0.0
    x[7, 2] = np.float32(479.0 * 2.0 ** -3)  # maximum between 464 and 512 times a power of two
    x[8, :] = np.float32(464.0 * 2.0 ** 5)   # maximum exactly on 464 * 2^e: stays in that binade
    x[9, 4] = np.float32(450.0 * 2.0 ** -7)  # maximum between 448 and 464: rounds to 448, not clipped
    codes, exps = o.quantize_fp8blk(x)
    for i in range(x.shape[0]):
        m = Fraction(float(np.abs(x[i]).max()))
        if m == 0:
            assert exps[i, 0] == 0 and not (codes[i] & 0x7F).any()
            continue
        e = int(exps[i, 0])
        assert Fraction(232) < m / Fraction(2) ** e <= Fraction(464), (i, e, float(m))
        assert _rne_e4m3(m / Fraction(2) ** e) & 0x7F == 0x7E or m / Fraction(2) ** e < 448, (i, e)
        for j in range(16):
            assert codes[i, j] == _rne_e4m3(Fraction(float(x[i, j])) / Fraction(2) ** e), (i, j)
    deq = o.dequantize_fp8blk(codes, exps).astype(np.float32)
    c2, e2 = o.quantize_fp8blk(deq)
    assert np.array_equal(c2, codes) and np.array_equal(e2, exps)


def pin_fp8blk_scan(o):
    """The recurrence on the fp8 state: alpha = 1, beta = 0 leaves every code
    and scale unchanged; beta = 1 with one write slot of weight 1 stores
    exactly the quantised v; a read of that slot with weight 1 returns its
    decoded value."""
    rng = np.random.default_rng(6)
    B, T, H, N, d_v = 1, 5, 2, 16, 32
    M = rng.standard_normal((B, H, N, d_v)).astype(np.float32)
    codes, exps = o.quantize_fp8blk(M)
    idx_w, w_w = random_selection(rng, B, T, H, N, 3)
    idx_r, w_r = random_selection(rng, B, T, H, N, 2)
    v = rng.standard_normal((B, T, H, d_v)).astype(np.float32)
    ones, zeros = np.ones((B, T, H), np.float32), np.zeros((B, T, H), np.float32)
    _, C, X = o.scan_fp8blk(idx_w, w_w, idx_r, w_r, v, ones, zeros, codes, exps)
    assert np.array_equal(C, codes) and np.array_equal(X, exps)
    iw = idx_w[..., :1].copy()
    y, C, X = o.scan_fp8blk(iw, np.ones_like(iw, dtype=np.float32), iw, np.ones_like(iw, dtype=np.float32), v, ones,
                            ones, codes, exps)
    for t in range(T):
        for h in range(H):
            vc, ve = o.quantize_fp8blk(v[0, t, h])
            deq = o.dequantize_fp8blk(vc, ve)
            assert np.array_equal(y[0, t, h], deq), (t, h)
    last = {}
    for t in range(T):
        for h in range(H):
            last[(h, int(iw[0, t, h, 0]))] = t
    for (h, slot), t in last.items():
        vc, ve = o.quantize_fp8blk(v[0, t, h])
        assert np.array_equal(C[0, h, slot], vc) and np.array_equal(X[0, h, slot], ve)


ALL_PINS = {
    "selection_brute_force": pin_selection_brute_force,
    "selection_identity": pin_selection_identity,
    "selection_golden": pin_selection_golden,
    "weights": pin_weights,
    "scan_golden": pin_scan_golden,
    "scan_identity_gates": pin_scan_identity_gates,
    "scan_beta_one_overwrites": pin_scan_beta_one_overwrites,
    "scan_beta_one_overwrites_bf16": lambda o: pin_scan_beta_one_overwrites(o, state_bf16=True),
    "scan_unselected_untouched": pin_scan_unselected_untouched,
    "scan_closed_form": pin_scan_closed_form,
    "scan_convex_bound": pin_scan_convex_bound,
    "scan_chunking": pin_scan_chunking,
    "scan_ops_independent_of_n": pin_scan_ops_independent_of_n,
    "scan_bf16_state": pin_scan_bf16_state,
    "epilogue": pin_epilogue,
    "round_to_bf16": pin_round_to_bf16,
    "backward_finite_differences": pin_backward_finite_differences,
    "backward_one_slot_golden": pin_backward_one_slot_golden,
    "backward_unselected_pass_through": pin_backward_unselected_pass_through,
    "topk_backward": pin_topk_backward,
    "epilogue_backward": pin_epilogue_backward,
    "e4m3_rounding": pin_e4m3_rounding,
    "fp8blk_blocks": pin_fp8blk_blocks,
    "fp8blk_scan": pin_fp8blk_scan,
}


def failing_pins(o) -> list:
    """Names of the pins the given oracle fails."""
    failed = []
    for name, fn in ALL_PINS.items():
        try:
            fn(o)
        except AssertionError:
            failed.append(name)
    return failed
