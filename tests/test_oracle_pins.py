"""Pins of the CPU oracle to things other than itself.

Each test fixes part of the oracle against an independent source: hand-worked
groups (tests/golden/quant_groups.txt), torch's bfloat16 / float8_e4m3fn
conversions, exact rational arithmetic on tiny problems, brute-force nearest
search over the formats' value sets, and invariants the method must satisfy
(r = 0 and lambda = 1 reduce to plain W4A4; W = L1 L2 gives a zero residual;
inputs on the 4-bit grid quantise without error). The tests are sized so a
dropped term, a wrong sign, a transposed operand or a wrong rounding mode in
the oracle makes at least one of them fail.
"""

from fractions import Fraction
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_groups.txt")

E2M1_MAG = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e4m3_values_bruteforce():
    """Every non-negative finite E4M3 value with its code, from the bit layout."""
    vals = []
    for code in range(0x7F):  # 0x7F is NaN
        e, m = code >> 3, code & 7
        v = Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        vals.append((v, code))
    return vals


E4M3_TABLE = _e4m3_values_bruteforce()


def _nearest_even(a: Fraction, table):
    """Nearest entry of (value, code) table to a, ties to the even code."""
    best = None
    for v, c in table:
        d = abs(v - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0 and best[1] % 2 == 1):
            best = (d, c)
    return best[1]


def _e2m1_bruteforce(x: float) -> int:
    a = Fraction(abs(x)) if np.isfinite(x) else Fraction(100)
    if a >= 6:
        code = 7
    else:
        code = _nearest_even(a, [(Fraction(v), i) for i, v in enumerate(E2M1_MAG)])
    return code | (8 if np.signbit(x) else 0)


def _e4m3_bruteforce(x: float) -> int:
    a = Fraction(abs(x)) if np.isfinite(x) else Fraction(1000)
    code = 0x7E if a >= 448 else _nearest_even(a, E4M3_TABLE)
    return code | (0x80 if np.signbit(x) else 0)


# ----------------------------------------------------------------- bfloat16
def test_bf16_matches_torch_on_random_bit_patterns():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    ours = oracle.bf16_rn(v.astype(np.float64))
    ref = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_ties_and_neighbours_match_torch():
    rng = np.random.default_rng(2)
    hi = rng.integers(0, 0x7F7F, size=1 << 16, dtype=np.uint32)
    out = []
    for low in (0x7FFF, 0x8000, 0x8001, 0x0000, 0xFFFF):
        out.append(((hi << 16) | low).astype(np.uint32))
    bits = np.concatenate(out)
    v = bits.view(np.float32)
    for sign in (1.0, -1.0):
        vv = (v * sign).astype(np.float32)
        ours = oracle.bf16_rn(vv.astype(np.float64))
        ref = torch.from_numpy(vv.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(ours, ref)


def test_bf16_from_double_rounds_once():
    # A double just above a bf16 midpoint must round up; rounding through
    # float32 first would land on the midpoint and round to even (down).
    lo = 1.0
    ulp = 2.0 ** -7
    mid = lo + ulp / 2
    just_above = mid + 2.0 ** -40
    assert oracle.bf16_rn(np.array([just_above]))[0] == 0x3F81
    assert oracle.bf16_rn(np.array([mid]))[0] == 0x3F80          # tie -> even
    assert oracle.bf16_rn(np.array([lo + 1.5 * ulp]))[0] == 0x3F82  # tie -> even (up)


# ----------------------------------------------------------------- E4M3
def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    ours = oracle.e4m3_to_f32(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def _e4m3_probe_values():
    vals = np.array([float(v) for v, _ in E4M3_TABLE], np.float64)
    mids = (vals[:-1] + vals[1:]) / 2
    probes = [vals, mids]
    for m in (mids, vals):
        probes.append(np.nextafter(m.astype(np.float32), np.float32(np.inf)).astype(np.float64))
        probes.append(np.nextafter(m.astype(np.float32), np.float32(0)).astype(np.float64))
    rng = np.random.default_rng(3)
    probes.append(np.exp2(rng.uniform(-14, 8.8, 20000)))
    p = np.concatenate(probes).astype(np.float32)
    return np.concatenate([p, -p])


def test_e4m3_encode_matches_torch_in_range():
    v = _e4m3_probe_values()
    v = v[np.abs(v) <= 448]
    ours = oracle.e4m3_rn(v)
    ref = torch.from_numpy(v.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_matches_bruteforce_and_saturates():
    v = _e4m3_probe_values()[::7]
    extra = np.array([448.0, 449.0, 464.0, 480.0, 1e6, np.inf, -np.inf, -500.0], np.float32)
    v = np.concatenate([v, extra])
    ours = oracle.e4m3_rn(v)
    ref = np.array([_e4m3_bruteforce(float(x)) for x in v], np.uint8)
    assert np.array_equal(ours, ref)
    assert oracle.e4m3_rn(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


# ----------------------------------------------------------------- E2M1
def test_e2m1_listed_ties_and_signs():
    cases = [(0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4), (3.5, 0x6),
             (5.0, 0x6), (6.0, 0x7), (7.0, 0x7), (1e30, 0x7), (0.2, 0x0), (0.26, 0x1),
             (-0.0, 0x8), (-0.1, 0x8), (-6.5, 0xF), (-2.9, 0xD), (0.0, 0x0)]
    v = np.array([c[0] for c in cases], np.float32)
    assert [int(c) for c in oracle.e2m1_rn(v)] == [c[1] for c in cases]


def test_e2m1_matches_bruteforce():
    mags = np.array(E2M1_MAG)
    mids = (mags[:-1] + mags[1:]) / 2
    rng = np.random.default_rng(4)
    base = np.concatenate([mags, mids, rng.uniform(0, 8, 5000), np.exp2(rng.uniform(-30, 4, 2000))])
    b32 = base.astype(np.float32)
    v = np.concatenate([b32, np.nextafter(b32, np.float32(np.inf)), np.nextafter(b32, np.float32(0))])
    v = np.concatenate([v, -v])
    ours = oracle.e2m1_rn(v)
    ref = np.array([_e2m1_bruteforce(float(x)) for x in v], np.uint8)
    assert np.array_equal(ours, ref)


def test_e2m1_decode_table():
    for c in range(16):
        e, m = (c >> 1) & 3, c & 1
        mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
        want = -mag if c & 8 else mag
        got = float(oracle.e2m1_to_f32(np.array([c]))[0])
        assert got == want and np.signbit(got) == bool(c & 8)


# ----------------------------------------------------------------- golden groups
def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


@pytest.mark.parametrize("line", _golden())
def test_golden_group(line):
    head, *rest = [p.strip() for p in line.split("|")]
    kind, *args = head.split()
    if kind == "nvfp4":
        t = float(args[0])
        vals = [float(x) for x in args[1].split(",")]
        v = np.zeros(16, np.float32)
        v[:len(vals)] = vals
        codes, sf = oracle.nvfp4_group(v, t)
        assert sf == int(rest[0], 16)
        want = [int(c, 16) for c in rest[1].split(",")]
        assert list(codes[:len(want)]) == want
        assert all(c in (0, 8) for c in codes[len(vals):])
    elif kind == "int4":
        vals = [float(x) for x in args[0].split(",")]
        v = np.zeros(64, np.float32)
        v[:len(vals)] = vals
        q, s = oracle.int4_group(v)
        assert s == int(rest[0], 16)
        assert list(q[:len(vals)]) == [int(c) for c in rest[1].split(",")]
        assert not q[len(vals):].any()
    elif kind == "awq":
        vals = [float(x) for x in args[0].split(",")]
        W = np.zeros((64, 1), np.float32)
        W[:len(vals), 0] = vals
        pk = oracle.awq_pack_weight(W)
        assert int(pk["s"][0, 0]) == int(rest[0], 16)
        assert float(oracle.bf16_to_f32(pk["z"][0, 0])) == float(rest[1])
        q = oracle.unpack_nibbles(pk["q"])[0]
        assert list(q[:len(vals)]) == [int(c) for c in rest[2].split(",")]
        assert (q[len(vals):] == int(rest[1])).all()
    else:
        raise AssertionError(kind)


# ----------------------------------------------------------------- layouts
def test_pack_layout_single_element():
    """One non-zero weight lands in exactly one nibble at [n, k/2], low nibble
    for even k; this catches a transposed [K,N] -> [N,K] or a swapped nibble."""
    K, N = 64, 8
    for (k, n) in [(0, 0), (1, 0), (17, 5), (62, 7), (63, 3)]:
        W = np.zeros((K, N), np.float32)
        W[k, n] = 1.0
        pk = oracle.pack_weight("nvfp4", W, np.ones(K, np.float32), np.zeros((K, 0), np.uint16),
                                np.zeros((0, N), np.uint16))
        nz = np.argwhere(pk["codes"])
        assert nz.tolist() == [[n, k // 2]]
        byte = int(pk["codes"][n, k // 2])
        assert (byte & 0xF if k % 2 == 0 else byte >> 4) == 0x7  # 1.0 is the group max -> 6
        assert np.argwhere(pk["scales"]).tolist() == [[n, k // 16]]
        # amax(R) = 1 -> s_tw = 1/2688; block scale = e4m3(1/(6 s_tw)) = 448
        assert pk["scales"][n, k // 16] == 0x7E


def test_quantize_layout_single_element():
    M, K = 3, 64
    for (m, k) in [(0, 0), (2, 33), (1, 63)]:
        x = np.zeros((M, K), np.uint16)
        x[m, k] = 0x3F80  # 1.0
        aq = oracle.quantize_act("nvfp4", x, np.ones(K, np.float32), 1.0, np.zeros((K, 0), np.uint16))
        assert np.argwhere(aq["codes"]).tolist() == [[m, k // 2]]
        byte = int(aq["codes"][m, k // 2])
        assert (byte & 0xF if k % 2 == 0 else byte >> 4) == 0x7
        assert np.argwhere(aq["scales"]).tolist() == [[m, k // 16]]


# ----------------------------------------------------------------- exact small problems
def _deq_rows(prec, codes, scales):
    nib = oracle.unpack_nibbles(codes).astype(np.int64)
    if prec == "nvfp4":
        table = [Fraction(v) for v in E2M1_MAG]
        vals = [[(-table[c & 7] if c & 8 else table[c & 7]) for c in row] for row in nib]
        sc = [[Fraction(float(oracle.e4m3_to_f32(np.array([s]))[0])) for s in row] for row in scales]
        G = 16
    else:
        vals = [[Fraction(int(c) - 16 if c & 8 else int(c)) for c in row] for row in nib]
        sc = [[Fraction(float(oracle.bf16_to_f32(np.array([s]))[0])) for s in row] for row in scales]
        G = 64
    return [[v * sc[i][k // G] for k, v in enumerate(row)] for i, row in enumerate(vals)]


def _bf16_exact(q: Fraction) -> int:
    """Nearest bf16 of an exact rational, ties to even (brute force over the
    two neighbours)."""
    f = float(q)
    b = int(torch.tensor([f], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF
    cands = set()
    for d in (-2, -1, 0, 1, 2):
        c = (b + d) & 0xFFFF
        if (c & 0x7F80) != 0x7F80:
            cands.add(c)
    best = None
    for c in cands:
        v = Fraction(float(oracle.bf16_to_f32(np.array([c], np.uint16))[0]))
        d = abs(v - q)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


@pytest.mark.parametrize("prec,s_tx", [("nvfp4", 1.0), ("nvfp4", 0.25), ("nvfp4", 0.7), ("int4", 1.0)])
def test_linear_exact_on_tiny_problem(prec, s_tx):
    """y = s_tx s_tw sum_b sx sw sum qx qw + P L2 + b, exactly in rationals from
    the packed codes and scales. With s_tx != 1 an oracle that dropped s_tx
    from the output scale (or applied it twice) fails here."""
    M, K, N, r = 4, 128, 8, 16
    d = synth.svdq_layer(7, M, K, N, r, x_out_frac=0.05, x_out_scale=10.0)
    w = oracle.pack_weight(prec, d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act(prec, d["x"], w["inv_lam"], s_tx, d["L1"])
    y = oracle.linear(prec, a, w, s_tx, d["L2"], d["b"])

    xd = _deq_rows(prec, a["codes"], a["scales"])
    wd = _deq_rows(prec, w["codes"], w["scales"])
    # s_tx is an fp32 value at every interface (the tensor-scale buffer)
    alpha = Fraction(float(np.float32(s_tx))) * Fraction(w["s_tw"]) if prec == "nvfp4" else Fraction(1)
    P = [[Fraction(float(v)) for v in row] for row in oracle.bf16_to_f32(a["P"])]
    L2 = [[Fraction(float(v)) for v in row] for row in oracle.bf16_to_f32(d["L2"])]
    b = [Fraction(float(v)) for v in oracle.bf16_to_f32(d["b"])]
    for m in range(M):
        for n in range(N):
            exact = alpha * sum(xd[m][k] * wd[n][k] for k in range(K))
            exact += sum(P[m][j] * L2[j][n] for j in range(r)) + b[n]
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2**50) + Fraction(1, 2**80)
            assert int(oracle.bf16_rn(np.array([y[m, n]]))[0]) == _bf16_exact(exact)


def test_P_is_bf16_of_exact_sum():
    M, K, r = 3, 64, 16
    d = synth.svdq_layer(8, M, K, 8, r)
    inv = (1.0 / d["lam"].astype(np.float64)).astype(np.float32)
    a = oracle.quantize_act("nvfp4", d["x"], inv, 1.0, d["L1"])
    xf = oracle.bf16_to_f32(d["x"])
    L1 = oracle.bf16_to_f32(d["L1"])
    for m in range(M):
        xh = [Fraction(float(oracle.bf16_to_f32(oracle.bf16_rn(np.array([np.float32(xf[m, k] * inv[k])]))[0])))
              for k in range(K)]
        for j in range(r):
            exact = sum(xh[k] * Fraction(float(L1[k, j])) for k in range(K))
            assert int(a["P"][m, j]) == _bf16_exact(exact)


# ----------------------------------------------------------------- invariants
def _grid_weight(K, N, s_tw, rng):
    """W with every 16-group = scale * (E2M1 grid values), each group holding a
    +-6, and one group at the top scale 448 so that amax(W) = 6 * 448 * s_tw."""
    grid = np.array(E2M1_MAG + [-v for v in E2M1_MAG[1:]])
    e4 = np.array([float(v) for v, c in E4M3_TABLE if v >= Fraction(1, 64)])
    W = np.zeros((K, N))
    for n in range(N):
        for b in range(K // 16):
            s = 448.0 if (n == 0 and b == 0) else rng.choice(e4[e4 <= 448])
            g = rng.choice(grid, 16)
            g[rng.integers(16)] = 6.0 * rng.choice([-1, 1])
            W[b * 16:(b + 1) * 16, n] = g * s * s_tw
    return W.astype(np.float32)


def test_fp4_grid_weight_packs_without_error():
    rng = np.random.default_rng(5)
    K, N, s_tw = 128, 16, 2.0 ** -12
    W = _grid_weight(K, N, s_tw, rng)
    w = oracle.pack_weight("nvfp4", W, np.ones(K, np.float32), np.zeros((K, 0), np.uint16),
                           np.zeros((0, N), np.uint16), want_R=True)
    assert w["s_tw"] == s_tw
    deq = np.array(_deq_rows("nvfp4", w["codes"], w["scales"]), dtype=np.float64) * w["s_tw"]
    assert np.array_equal(deq.T, W.astype(np.float64))


def test_fp4_grid_activation_quantises_without_error():
    rng = np.random.default_rng(6)
    M, K = 8, 128
    Wg = _grid_weight(K, M, 1.0, rng)  # reuse the construction: columns -> rows
    x = Wg.T.astype(np.float32)
    xb = synth.bf16_bits(x)
    assert np.array_equal(oracle.bf16_to_f32(xb), x)  # grid values are bf16-exact
    a = oracle.quantize_act("nvfp4", xb, np.ones(K, np.float32), 1.0, np.zeros((K, 0), np.uint16))
    deq = np.array(_deq_rows("nvfp4", a["codes"], a["scales"]), dtype=np.float64)
    assert np.array_equal(deq, x.astype(np.float64))


def test_int4_grid_round_trip():
    rng = np.random.default_rng(7)
    K, N = 128, 8
    W = np.zeros((K, N), np.float32)
    for n in range(N):
        for g in range(K // 64):
            s = 2.0 ** rng.integers(-8, 2)
            q = rng.integers(-7, 8, 64).astype(np.float64)
            q[rng.integers(64)] = 7 * rng.choice([-1, 1])
            W[g * 64:(g + 1) * 64, n] = q * s
    w = oracle.pack_weight("int4", W, np.ones(K, np.float32), np.zeros((K, 0), np.uint16),
                           np.zeros((0, N), np.uint16))
    deq = np.array(_deq_rows("int4", w["codes"], w["scales"]), dtype=np.float64)
    assert np.array_equal(deq.T, W.astype(np.float64))


def test_r0_lambda1_reduces_to_plain_w4a4():
    """With no low-rank branch and lambda = 1 the layer is plain W4A4: the
    output equals the product of the two grid-built operands plus bias."""
    rng = np.random.default_rng(8)
    M, K, N = 8, 128, 16
    W = _grid_weight(K, N, 2.0 ** -10, rng)
    X = _grid_weight(K, M, 1.0, rng).T.astype(np.float32)
    xb = synth.bf16_bits(X)
    b = synth.bf16_bits(rng.normal(0, 0.01, N))
    w = oracle.pack_weight("nvfp4", W, np.ones(K, np.float32), np.zeros((K, 0), np.uint16),
                           np.zeros((0, N), np.uint16))
    a = oracle.quantize_act("nvfp4", xb, w["inv_lam"], 1.0, np.zeros((K, 0), np.uint16))
    y = oracle.linear("nvfp4", a, w, 1.0, np.zeros((0, N), np.uint16), b)
    want = X.astype(np.float64) @ W.astype(np.float64) + oracle.bf16_to_f32(b)
    assert np.allclose(y, want, rtol=1e-13, atol=1e-15)


def test_zero_residual_when_weight_is_low_rank():
    """W = L1 L2 exactly (small-integer factors, lambda = 1): the residual is
    zero, every weight code and scale is zero, s_tw falls back to 1, and the
    output is the low-rank branch plus bias."""
    rng = np.random.default_rng(9)
    M, K, N, r = 4, 64, 16, 16
    L1f = rng.integers(-3, 4, (K, r)) * 0.25
    L2f = rng.integers(-3, 4, (r, N)) * 0.125
    L1, L2 = synth.bf16_bits(L1f), synth.bf16_bits(L2f)
    W = (L1f @ L2f).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), L1f @ L2f)
    for prec in ("nvfp4", "int4"):
        w = oracle.pack_weight(prec, W, np.ones(K, np.float32), L1, L2, want_R=True)
        assert not w["R"].any() and not w["codes"].any() and not w["scales"].any()
        if prec == "nvfp4":
            assert w["s_tw"] == 1.0
        x = synth.bf16_bits(rng.normal(0, 1, (M, K)))
        bias = synth.bf16_bits(rng.normal(0, 0.01, N))
        a = oracle.quantize_act(prec, x, w["inv_lam"], 1.0, L1)
        y = oracle.linear(prec, a, w, 1.0, L2, bias)
        Pf = oracle.bf16_to_f32(a["P"]).astype(np.float64)
        want = Pf @ L2f + oracle.bf16_to_f32(bias)
        assert np.allclose(y, want, rtol=1e-14, atol=1e-14)


def test_smoothing_is_applied_to_weight_and_activation():
    """Scaling channel k of x by c and row k of W by 1/c (with lambda scaled by
    c) leaves the smoothed operands unchanged when c is a power of two."""
    M, K, N, r = 4, 64, 8, 16
    d = synth.svdq_layer(10, M, K, N, r)
    w1 = oracle.pack_weight("nvfp4", d["W"], d["lam"], d["L1"], d["L2"], want_R=True)
    a1 = oracle.quantize_act("nvfp4", d["x"], w1["inv_lam"], 1.0, d["L1"])
    c = np.ones(K, np.float32)
    c[::3] = 4.0
    x2 = synth.bf16_bits(oracle.bf16_to_f32(d["x"]) * c)
    W2 = (d["W"] / c[:, None]).astype(np.float32)
    w2 = oracle.pack_weight("nvfp4", W2, d["lam"] * c, d["L1"], d["L2"], want_R=True)
    a2 = oracle.quantize_act("nvfp4", x2, w2["inv_lam"], 1.0, d["L1"])
    assert np.array_equal(w1["R"], w2["R"])
    assert np.array_equal(a1["codes"], a2["codes"]) and np.array_equal(a1["P"], a2["P"])


def test_int4_group_sums_match_integer_matmul():
    M, K, N = 5, 192, 7
    d = synth.svdq_layer(11, M, K, N, 0)
    w = oracle.pack_weight("int4", d["W"], d["lam"], d["L1"], d["L2"])
    a = oracle.quantize_act("int4", d["x"], w["inv_lam"], 1.0, d["L1"])
    sums = oracle.int4_group_sums(a["codes"], w["codes"])

    def signed(c):
        n = oracle.unpack_nibbles(c).astype(np.int64)
        return np.where(n >= 8, n - 16, n)

    xs, ws = signed(a["codes"]), signed(w["codes"])
    for g in range(K // 64):
        want = xs[:, g * 64:(g + 1) * 64] @ ws[:, g * 64:(g + 1) * 64].T
        assert np.array_equal(sums[:, :, g], want)


def test_residual_matches_definition_small():
    """R = fp32(lambda*W) - L1 L2, checked in exact rational arithmetic."""
    K, N, r = 16, 4, 16
    d = synth.svdq_layer(12, 2, K, N, r)
    w = oracle.pack_weight("nvfp4", d["W"], d["lam"], d["L1"], d["L2"], want_R=True)
    L1 = oracle.bf16_to_f32(d["L1"])
    L2 = oracle.bf16_to_f32(d["L2"])
    for k in range(K):
        for n in range(N):
            what = Fraction(float(np.float32(d["lam"][k] * d["W"][k, n])))
            exact = what - sum(Fraction(float(L1[k, j])) * Fraction(float(L2[j, n])) for j in range(r))
            assert w["R"][k, n] == np.float32(float(exact))


# ----------------------------------------------------------------- AWQ
def test_awq_reconstruction_error_bound():
    K, N = 256, 32
    W = (np.random.default_rng(13).normal(0, 0.02, (K, N))).astype(np.float32)
    pk = oracle.awq_pack_weight(W)
    q = oracle.unpack_nibbles(pk["q"]).astype(np.float64)
    s = oracle.bf16_to_f32(pk["s"]).astype(np.float64)
    z = oracle.bf16_to_f32(pk["z"]).astype(np.float64)
    deq = (q - np.repeat(z, 64, axis=1)) * np.repeat(s, 64, axis=1)
    err = np.abs(deq.T - W)
    # Inside the grid the error is at most half a step. The zero point is an
    # integer and s = bf16(range / 15) is rounded (relative error <= 2^-9), so
    # the extreme values can fall outside the grid by at most 15 * 2^-8 steps
    # more, where they are clamped.
    assert (err <= np.repeat(s, 64, axis=1).T * (0.5 + 15 / 256) + 1e-9).all()
    assert (q >= 0).all() and (q <= 15).all() and (z == np.round(z)).all()


def test_awq_linear_exact_on_tiny_problem():
    d = synth.awq_inputs(14, 2, 128, 6)
    pk = oracle.awq_pack_weight(d["W"])
    b = synth.bf16_bits(np.linspace(-0.02, 0.02, 6))
    y = oracle.awq_linear(d["x"], pk, b)
    q = oracle.unpack_nibbles(pk["q"])
    s = oracle.bf16_to_f32(pk["s"])
    z = oracle.bf16_to_f32(pk["z"])
    x = oracle.bf16_to_f32(d["x"])
    bf = oracle.bf16_to_f32(b)
    for m in range(2):
        for n in range(6):
            exact = sum(Fraction(float(x[m, k])) * (int(q[n, k]) - Fraction(float(z[n, k // 64])))
                        * Fraction(float(s[n, k // 64])) for k in range(128)) + Fraction(float(bf[n]))
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2**48) + Fraction(1, 2**70)


# ------------------------------------------------------------------ fused QKV epilogue (RMSNorm + rotary)
# Pins of oracle.qkv_norm_rope: invariants of a norm followed by a rotation,
# and relations between oracle calls with different rotation tables; none
# re-derives the oracle's arithmetic.
H_Q, D_Q, M_Q = 3, 8, 5


def _qkv_case(seed):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((M_Q, 3 * H_Q * D_Q)) * np.exp(rng.uniform(-3, 3, (M_Q, 1)))
    wq = oracle.bf16_rn(rng.uniform(0.5, 1.5, D_Q))
    wk = oracle.bf16_rn(rng.uniform(0.5, 1.5, D_Q))
    theta = rng.uniform(-np.pi, np.pi, (M_Q, D_Q // 2))
    return y, wq, wk, theta


def _rot(theta, sign=1.0):
    return np.cos(theta).astype(np.float32), (sign * np.sin(theta)).astype(np.float32)


def _heads(a, sec):
    """Section sec (0 Q, 1 K, 2 V) of a [M, 3 H D] array as [M, H, D]."""
    return a[:, sec * H_Q * D_Q:(sec + 1) * H_Q * D_Q].reshape(a.shape[0], H_Q, D_Q)


ONES = oracle.bf16_rn(np.ones(D_Q))
ZEROS_T = np.zeros((M_Q, D_Q // 2))


def test_qkv_unit_weights_no_eps_give_unit_rms_heads():
    # with w = 1, eps = 0 and no rotation every Q/K head comes out with RMS 1
    # and points the same way as its input; V is passed through bit for bit
    y, _, _, _ = _qkv_case(1)
    c, s = _rot(ZEROS_T)
    o = oracle.qkv_norm_rope(y, H_Q, D_Q, ONES, ONES, 0.0, c, s)
    for sec in (0, 1):
        oh, yh = _heads(o, sec), _heads(y, sec)
        assert np.allclose(np.sqrt(np.mean(oh ** 2, axis=2)), 1.0, rtol=1e-13)
        ratio = oh / yh
        assert np.allclose(ratio, ratio[:, :, :1], rtol=1e-12) and (ratio > 0).all()
    assert np.array_equal(_heads(o, 2), _heads(y, 2))


def test_qkv_quarter_turn_maps_pairs():
    # a rotation by +90 degrees sends the pair (a, b) to (-b, a)
    y, wq, wk, _ = _qkv_case(2)
    c0, s0 = _rot(ZEROS_T)
    u = oracle.qkv_norm_rope(y, H_Q, D_Q, wq, wk, 1e-6, c0, s0)
    c, s = np.zeros_like(c0), np.ones_like(s0)
    o = oracle.qkv_norm_rope(y, H_Q, D_Q, wq, wk, 1e-6, c, s)
    for sec in (0, 1):
        uh, oh = _heads(u, sec), _heads(o, sec)
        assert np.allclose(oh[:, :, 0::2], -uh[:, :, 1::2], rtol=1e-14, atol=0)
        assert np.allclose(oh[:, :, 1::2], uh[:, :, 0::2], rtol=1e-14, atol=0)


def test_qkv_rotation_preserves_pair_norms_and_undoes():
    # each (2i, 2i+1) pair keeps its length; rotating the (unit-RMS) result by
    # the opposite angles with w = 1, eps = 0 gives back the unrotated heads
    y, _, _, theta = _qkv_case(3)
    c0, s0 = _rot(ZEROS_T)
    u = oracle.qkv_norm_rope(y, H_Q, D_Q, ONES, ONES, 0.0, c0, s0)
    c, s = _rot(theta)
    o = oracle.qkv_norm_rope(y, H_Q, D_Q, ONES, ONES, 0.0, c, s)
    for sec in (0, 1):
        uh, oh = _heads(u, sec), _heads(o, sec)
        nu = np.hypot(uh[:, :, 0::2], uh[:, :, 1::2])
        no = np.hypot(oh[:, :, 0::2], oh[:, :, 1::2])
        # cos and sin are given in fp32: cos^2 + sin^2 = 1 to within a few ulp
        assert np.allclose(no, nu, rtol=1e-6)
    cb, sb = _rot(theta, -1.0)
    back = oracle.qkv_norm_rope(o, H_Q, D_Q, ONES, ONES, 0.0, cb, sb)
    for sec in (0, 1):
        assert np.allclose(_heads(back, sec), _heads(u, sec), rtol=0, atol=1e-6)


def test_qkv_norm_scale_invariant_without_eps():
    y, wq, wk, theta = _qkv_case(4)
    c, s = _rot(theta)
    o1 = oracle.qkv_norm_rope(y, H_Q, D_Q, wq, wk, 0.0, c, s)
    o2 = oracle.qkv_norm_rope(7.5 * y, H_Q, D_Q, wq, wk, 0.0, c, s)
    for sec in (0, 1):
        assert np.allclose(_heads(o2, sec), _heads(o1, sec), rtol=1e-13, atol=1e-15)
    assert np.array_equal(_heads(o2, 2), 7.5 * _heads(y, 2))


def test_qkv_constant_head_closed_form():
    # a head whose D entries all equal c has mean square c^2, so its output
    # (no rotation) is c / sqrt(c^2 + eps) * w: eps sits under the root, next to
    # the mean, not the sum
    cval, eps = 1e-3, 1e-6
    y = np.zeros((1, 3 * H_Q * D_Q))
    y[0, :D_Q] = cval
    wq = oracle.bf16_rn(np.linspace(0.5, 2.0, D_Q))
    c, s = _rot(np.zeros((1, D_Q // 2)))
    o = oracle.qkv_norm_rope(y, H_Q, D_Q, wq, ONES, eps, c, s)
    expect = cval / np.sqrt(cval ** 2 + eps) * oracle.bf16_to_f32(wq).astype(np.float64)
    assert np.allclose(o[0, :D_Q], expect, rtol=1e-14)
    # an all-zero head stays zero
    assert not o[0, D_Q:2 * H_Q * D_Q].any()


def test_qkv_heads_and_sections_are_independent():
    # changing one head of Q changes only that head; K uses wk and Q uses wq
    y, wq, wk, theta = _qkv_case(5)
    c, s = _rot(theta)
    o = oracle.qkv_norm_rope(y, H_Q, D_Q, wq, wk, 1e-6, c, s)
    y2 = y.copy()
    y2[:, 1 * D_Q:2 * D_Q] *= -3.0  # Q head 1
    o2 = oracle.qkv_norm_rope(y2, H_Q, D_Q, wq, wk, 1e-6, c, s)
    changed = np.abs(o2 - o).max(axis=0) > 0
    assert changed[D_Q:2 * D_Q].all() and not changed[:D_Q].any() and not changed[2 * D_Q:].any()
    o3 = oracle.qkv_norm_rope(y, H_Q, D_Q, wq, ONES, 1e-6, c, s)
    assert np.array_equal(_heads(o3, 0), _heads(o, 0)) and not np.array_equal(_heads(o3, 1), _heads(o, 1))
    o4 = oracle.qkv_norm_rope(y, H_Q, D_Q, ONES, wk, 1e-6, c, s)
    assert np.array_equal(_heads(o4, 1), _heads(o, 1)) and not np.array_equal(_heads(o4, 0), _heads(o, 0))


# ------------------------------------------------------------------ fused GELU-MLP epilogue
def test_gelu_bf16_matches_scipy_erf_and_torch_rounding():
    # an independent GELU (scipy's erf) rounded by torch's bfloat16 conversion
    import scipy.special
    rng = np.random.default_rng(21)
    y = np.concatenate([rng.standard_normal(20000) * 3, rng.uniform(-12, 12, 5000), [0.0, 1e-30, -1e-30]])
    ref = 0.5 * y * (1.0 + scipy.special.erf(y / np.sqrt(2.0)))
    ref_bits = torch.from_numpy(ref).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.gelu_bf16(y)
    # torch may round float64 -> bfloat16 through float32; that can only differ
    # from one rounding where the float32 value sits exactly on a bf16 tie
    low = ref.astype(np.float32).view(np.uint32) & 0xFFFF
    safe = low != 0x8000
    assert safe.mean() > 0.99
    assert np.array_equal(got[safe], ref_bits[safe])


def test_gelu_bf16_odd_part_identity_and_limits():
    # GELU(x) - GELU(-x) = x for the Gaussian CDF; each side carries one bf16 rounding
    x = np.random.default_rng(22).uniform(-8, 8, 4000)
    gp = oracle.bf16_to_f32(oracle.gelu_bf16(x)).astype(np.float64)
    gm = oracle.bf16_to_f32(oracle.gelu_bf16(-x)).astype(np.float64)
    tol = (np.abs(gp) + np.abs(gm)) * 2.0 ** -8 + 1e-30
    assert (np.abs(gp - gm - x) <= tol).all()
    assert oracle.gelu_bf16(np.array([0.0]))[0] == 0
    big = np.array([8.0, 20.0, 100.0])
    assert np.array_equal(oracle.gelu_bf16(big), oracle.bf16_rn(big))
    assert (np.abs(oracle.bf16_to_f32(oracle.gelu_bf16(-big))) < 1e-13).all()


def test_mlp_epilogue_reduces_to_the_activation_pass_where_gelu_is_identity():
    # for y >= 8, GELU(y) = y to well below a bf16 ulp, so the fused epilogue's
    # down-projection inputs are those of the plain activation pass on bf16(y)
    d = synth.svdq_layer(23, 6, 128, 8, 16)
    y = 8.0 + np.abs(np.random.default_rng(23).standard_normal((6, 128))) * 4
    for prec in ("nvfp4", "int4"):
        a = oracle.mlp_gelu_down_act(prec, y, d["lam"] * 0 + 1.0, 1.0, d["L1"])
        b = oracle.quantize_act(prec, oracle.bf16_rn(y), d["lam"] * 0 + 1.0, 1.0, d["L1"])
        for k in ("codes", "scales", "P"):
            assert np.array_equal(a[k], b[k])
