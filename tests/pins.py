"""Pins for the CPU oracle: checks against facts that do not come from the oracle.

Every check takes an ``oracle.Oracle`` (the committed build, or a deliberately
altered one in test_oracle_mutants.py) and raises AssertionError when the
oracle disagrees with:

* the E2M1 bit-field definition (sign, 2 exponent bits with bias 1, 1 mantissa
  bit, subnormal at exponent 0) and the table in golden/e2m1_values.txt;
* brute-force nearest-value encoding over all 16 codes, with the tie rule
  "exact midpoints go to the value whose mantissa bit is 0";
* the rounding bound of a nearest-value quantiser and the storage layout
  (two codes per byte, low nibble = even k; one scale per 32 along K);
* the router's hand-worked cases (golden/router_cases.txt), numpy's stable
  sort, the full softmax at k = E, and sum_j w = 1;
* numpy's stable argsort for the grouping;
* the closed form of a layer whose codes are all equal;
* a dense, unpermuted brute-force layer written here with numpy;
* for the router GEMM: the closed form of all-equal weights (an exact sum by
  math.fsum), one-hot rows (a permutation of x's columns, exactly), numpy's
  dot product, and a router whose expert ranking is built in;
* for the INT2 codec: the symmetry and spacing of the four levels, brute-force
  nearest-level encoding with the stated tie rule, single-element layout probes
  (two bits per code, four codes per byte, one scale max|w|/1.5 per 32 along
  K), the rounding bound, and a dense brute-force layer whose experts mix
  E2M1 and INT2;
* for the block-scaled FP4 (NVFP4) variant: the E4M3 bit-field definition and
  the table in golden/e4m3_values.txt, brute-force nearest E4M3 encoding in
  exact arithmetic (ties to the even code, saturation at 448), the row
  encoding redone with numpy float32 steps and exact nearest searches,
  single-element layout probes (two codes per byte, one scale factor per 16,
  one row scale), the closed form of a constant row, the rounding bound, sign
  symmetry, and a dense brute-force variant layer; the variant stays within a
  loose distance of the exact layer.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# -- independent decoders ------------------------------------------------------

def e2m1_from_bits(code: int) -> float:
    """E2M1 value from its bit fields (OCP MX v1.0 FP4 element definition)."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return -mag if s else mag


E2M1_TABLE = np.array([e2m1_from_bits(c) for c in range(16)], dtype=np.float64)


def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def dequant_dense(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """codes [..., K/2, N], scales [..., K/32, N] -> float64 [..., K, N]."""
    lo = E2M1_TABLE[codes & 0x0F]
    hi = E2M1_TABLE[codes >> 4]
    K2, N = codes.shape[-2:]
    vals = np.empty(codes.shape[:-2] + (2 * K2, N), dtype=np.float64)
    vals[..., 0::2, :] = lo
    vals[..., 1::2, :] = hi
    s = np.repeat(bf16_to_f64(scales), 32, axis=-2)
    return vals * s


def brute_force_code(r: float) -> int:
    """Nearest E2M1 code to r: minimum |r - value|; ties to mantissa bit 0; zero is code 0."""
    best, best_d = None, None
    for c in range(16):
        d = abs(Fraction(float(r)) - Fraction(E2M1_TABLE[c]))
        if best is None or d < best_d or (d == best_d and (best & 1) and not (c & 1)):
            best, best_d = c, d
    if E2M1_TABLE[best] == 0.0:
        return 0
    return best


def nearest_bf16_bits(v: np.float32) -> int:
    """bf16 pattern nearest to float32 v (ties to even), by enumerating neighbours."""
    b = int(np.float32(v).view(np.uint32))
    lo = b >> 16
    cands = [lo, lo + 1]
    fv = Fraction(float(v))

    def val(p):
        return Fraction(float(np.uint32(p << 16).view(np.float32)))
    d0, d1 = abs(fv - val(cands[0])), abs(fv - val(cands[1]))
    if d0 < d1:
        return cands[0]
    if d1 < d0:
        return cands[1]
    return cands[0] if cands[0] % 2 == 0 else cands[1]


# -- checks ----------------------------------------------------------------------

def check_e2m1_table(o):
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "e2m1_values.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 16
    for code_s, val_s in rows:
        code = int(code_s)
        assert float(val_s) == e2m1_from_bits(code)
        assert o.e2m1_decode(code) == float(val_s), f"code {code}"


def encode_probe_values(rng) -> np.ndarray:
    grid = np.unique(np.abs(E2M1_TABLE))
    mids = (grid[1:] + grid[:-1]) / 2
    base = np.concatenate([grid, mids, [6.5, 7.0, 100.0, 1e-3, 0.0]])
    near = np.concatenate([np.nextafter(base.astype(np.float32), np.float32(np.inf)),
                           np.nextafter(base.astype(np.float32), np.float32(-np.inf))])
    rnd = rng.uniform(-7.0, 7.0, 400).astype(np.float32)
    v = np.concatenate([base.astype(np.float32), near, rnd])
    return np.concatenate([v, -v]).astype(np.float32)


def check_encode_bruteforce(o, rng):
    for r in encode_probe_values(rng):
        exp = brute_force_code(float(r))
        got = o.e2m1_encode(float(r))
        assert got == exp, f"encode({float(r)!r}) = {got}, brute force {exp}"


def check_quantize_layout(o):
    E, K, N = 2, 64, 3
    for (e, k, n, v) in [(0, 0, 0, 0.3), (1, 37, 2, -1.7), (0, 63, 1, 5.0), (1, 32, 0, -0.02)]:
        W = np.zeros((E, K, N), dtype=np.float32)
        W[e, k, n] = v
        codes, scales = o.quantize(W)
        nz = np.argwhere(codes != 0)
        assert nz.tolist() == [[e, k // 2, n]], nz
        byte = int(codes[e, k // 2, n])
        code = (byte & 0xF) if k % 2 == 0 else (byte >> 4)
        other = (byte >> 4) if k % 2 == 0 else (byte & 0xF)
        assert other == 0
        # the one element is the group max: |v| / s is 6 up to bf16 rounding of s
        assert code == (15 if v < 0 else 7), code
        snz = np.argwhere(scales != 0)
        assert snz.tolist() == [[e, k // 32, n]], snz
        assert int(scales[e, k // 32, n]) == nearest_bf16_bits(np.float32(abs(np.float32(v))) / np.float32(6))


def check_quantize_roundtrip(o, rng):
    E, K, N = 3, 128, 40
    W = (rng.standard_normal((E, K, N)) * 0.02).astype(np.float32)
    W[0, 0:32, 0] = 0.0                        # an all-zero group
    W[1, 32:64, 1] = np.float32(0.01)          # a constant group
    codes, scales = o.quantize(W)
    assert codes.shape == (E, K // 2, N) and scales.shape == (E, K // 32, N)
    deq = dequant_dense(codes, scales)
    s = np.repeat(bf16_to_f64(scales), 32, axis=1)
    # scale = nearest bf16 to float32(max|w| / 6), per group and column
    gmax = np.abs(W).reshape(E, K // 32, 32, N).max(axis=2)
    for idx in [(0, 0, 0), (1, 1, 1), (2, 3, 39), (0, 2, 17)]:
        q = np.float32(gmax[idx]) / np.float32(6)
        assert int(scales[idx]) == nearest_bf16_bits(q)
    assert np.all(scales[0, 0, 0] == 0) and np.all(deq[0, 0:32, 0] == 0)
    # nearest-value rounding: |deq - w| <= s * (half the local grid gap), ratios within [-6, 6]
    grid = np.unique(E2M1_TABLE)
    r = W.astype(np.float64) / np.where(s == 0, 1, s)
    inside = np.abs(r) <= 6
    hi_idx = np.clip(np.searchsorted(grid, r, side="left"), 1, len(grid) - 1)
    gap = grid[hi_idx] - grid[hi_idx - 1]
    err = np.abs(deq - W.astype(np.float64))
    bound = s * gap / 2 * (1 + 1e-6) + 1e-30
    assert np.all(err[inside] <= bound[inside])
    assert np.all(np.abs(r) <= 6.0 * (1 + 2.0 ** -7))   # bf16 rounding of s may push past 6
    # spot-check codes against brute force
    for (e, k, n) in [(0, 5, 3), (2, 77, 10), (1, 127, 39), (1, 40, 1)]:
        byte = int(codes[e, k // 2, n])
        code = (byte & 0xF) if k % 2 == 0 else (byte >> 4)
        sv = float(bf16_to_f64(scales[e, k // 32, n]))
        exp = 0 if sv == 0 else brute_force_code(float(np.float32(W[e, k, n]) / np.float32(sv)))
        assert code == exp


def check_router_golden(o):
    for ln in open(os.path.join(GOLDEN, "router_cases.txt")):
        if not ln.strip() or ln.startswith("#"):
            continue
        k_s, l_s, i_s, w_s = [p.strip() for p in ln.split("|")]
        k = int(k_s)
        logits = np.array([[float(v) for v in l_s.split()]], dtype=np.float32)
        idx, w = o.route(logits, k)
        assert idx[0].tolist() == [int(v) for v in i_s.split()], (ln, idx)
        np.testing.assert_allclose(w[0], [float(v) for v in w_s.split()], rtol=2e-7, atol=0)


def check_router_random(o, rng):
    for (T, E, k) in [(7, 16, 3), (5, 128, 8), (3, 512, 10), (4, 9, 9), (6, 33, 1)]:
        logits = rng.standard_normal((T, E)).astype(np.float32)
        logits[0, 3] = logits[0, 5]                       # a deliberate tie
        logits[1 % T, :] = np.round(logits[1 % T, :])     # many ties
        idx, w = o.route(logits, k)
        for t in range(T):
            order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))
            assert idx[t].tolist() == order[:k].tolist()
            sel = logits[t, idx[t]].astype(np.float64)
            ref = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()
            np.testing.assert_allclose(w[t], ref, rtol=1e-6)
            assert abs(float(w[t].astype(np.float64).sum()) - 1.0) <= 1e-6
            assert np.all(np.diff(w[t].astype(np.float64)) <= 0)
        if k == 1:
            assert np.all(w == 1.0)
        if k == E:   # full softmax of the row
            for t in range(T):
                full = np.exp(logits[t] - logits[t].max()) / np.exp(logits[t] - logits[t].max()).sum()
                np.testing.assert_allclose(w[t], full[idx[t]], rtol=1e-6)


def check_group(o, rng):
    for (T, E, k) in [(1, 128, 8), (9, 16, 4), (64, 128, 8), (5, 4, 4)]:
        idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, sp, pr = o.group(idx, E)
        flat = idx.reshape(-1)
        assert counts.tolist() == np.bincount(flat, minlength=E).tolist()
        assert offsets.tolist() == [0] + np.cumsum(np.bincount(flat, minlength=E)).tolist()
        assert sp.tolist() == np.argsort(flat, kind="stable").tolist()
        assert np.all(pr[sp] == np.arange(T * k))


def _layer_inputs(rng, E, H, I, T, random_codes):
    if random_codes:
        gu_c = rng.integers(0, 256, (E, H // 2, 2 * I), dtype=np.uint8)
        dn_c = rng.integers(0, 256, (E, I // 2, H), dtype=np.uint8)
        # scales: bf16 patterns of magnitudes around 0.002..0.01
        gu_s = (np.abs(rng.standard_normal((E, H // 32, 2 * I))) * 0.004 + 0.001).astype(np.float32)
        dn_s = (np.abs(rng.standard_normal((E, I // 32, H))) * 0.004 + 0.001).astype(np.float32)
        gu_s = (gu_s.view(np.uint32) >> 16).astype(np.uint16)
        dn_s = (dn_s.view(np.uint32) >> 16).astype(np.uint16)
    else:
        Wgu = (rng.standard_normal((E, H, 2 * I)) * 0.02).astype(np.float32)
        Wdn = (rng.standard_normal((E, I, H)) * 0.02).astype(np.float32)
        return Wgu, Wdn
    return gu_c, gu_s, dn_c, dn_s


def _expert_weights(E, H, I, gu_c, gu_s, dn_c, dn_s):
    import oracle as _oracle_pkg
    ew = _oracle_pkg.ExpertWeights(E, H, I)
    for e in range(E):
        ew.set(e, gu_c[e], gu_s[e], dn_c[e], dn_s[e])
    return ew


def dense_layer_reference(x_bf16, logits, k, gu_c, gu_s, dn_c, dn_s):
    """Unpermuted brute force: every token through every expert, weighted by the routing mask."""
    T, H = x_bf16.shape
    E = logits.shape[1]
    I = dn_c.shape[1] * 2
    x = bf16_to_f64(x_bf16)
    Wgu = dequant_dense(gu_c, gu_s)       # [E, H, 2I]
    Wdn = dequant_dense(dn_c, dn_s)       # [E, I, H]
    y = np.zeros((T, H))
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))
        sel = order[:k]
        ls = logits[t, sel].astype(np.float64)
        wsel = (np.exp(ls - ls[0]) / np.exp(ls - ls[0]).sum()).astype(np.float32).astype(np.float64)
        mask = np.zeros(E)
        mask[sel] = wsel
        for e in range(E):
            h = x[t] @ Wgu[e]
            g, u = h[:I], h[I:]
            a = g / (1.0 + np.exp(-g)) * u
            y[t] += mask[e] * (a @ Wdn[e])
    return y


def check_dense_bruteforce(o, rng):
    for (E, H, I, T, k) in [(4, 64, 32, 3, 2), (6, 32, 64, 2, 6), (8, 256, 128, 4, 2)]:
        gu_c, gu_s, dn_c, dn_s = _layer_inputs(rng, E, H, I, T, random_codes=True)
        x = rng.standard_normal((T, H)).astype(np.float32)
        x_bf16 = (x.view(np.uint32) >> 16).astype(np.uint16)
        logits = rng.standard_normal((T, E)).astype(np.float32)
        ew = _expert_weights(E, H, I, gu_c, gu_s, dn_c, dn_s)
        y64, yb = o.moe_forward(ew, x_bf16, logits, k)
        ref = dense_layer_reference(x_bf16, logits, k, gu_c, gu_s, dn_c, dn_s)
        scale = np.abs(ref).max()
        assert np.abs(y64 - ref).max() <= 1e-10 * scale, np.abs(y64 - ref).max() / scale


def check_closed_form(o, rng):
    E, H, I, T, k = 5, 96, 64, 3, 3
    x = rng.standard_normal((T, H)).astype(np.float32)
    x_bf16 = (x.view(np.uint32) >> 16).astype(np.uint16)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    for c, cd, s_bits, sd_bits in [(2, 9, 0x3B80, 0x3C00), (7, 4, 0x3A00, 0x3B00), (13, 3, 0x3C80, 0x3A80)]:
        gu_c = np.full((E, H // 2, 2 * I), c | (c << 4), dtype=np.uint8)
        dn_c = np.full((E, I // 2, H), cd | (cd << 4), dtype=np.uint8)
        gu_s = np.full((E, H // 32, 2 * I), s_bits, dtype=np.uint16)
        dn_s = np.full((E, I // 32, H), sd_bits, dtype=np.uint16)
        ew = _expert_weights(E, H, I, gu_c, gu_s, dn_c, dn_s)
        y64, yb, act = o.moe_forward(ew, x_bf16, logits, k, want_act=True)
        s = float(bf16_to_f64(s_bits))
        sd = float(bf16_to_f64(sd_bits))
        vc, vd = e2m1_from_bits(c), e2m1_from_bits(cd)
        for t in range(T):
            sx = math.fsum(bf16_to_f64(x_bf16[t]))
            g = vc * s * sx
            a = g / (1.0 + math.exp(-g)) * g
            np.testing.assert_allclose(act[t * k:(t + 1) * k], a, rtol=1e-12, atol=1e-300)
            np.testing.assert_allclose(y64[t], vd * sd * I * a, rtol=1e-6)


def check_bf16_output_rounding(o, rng):
    vals = [1.0, 1.0 + 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -40, 1.0 + 3 * 2.0 ** -8,
            -(1.0 + 2.0 ** -8 - 2.0 ** -40), 3.14159, -2.5e-3, 1e-38, 0.0]
    vals += list(rng.standard_normal(200) * 10.0)
    for v in vals:
        got = o.f64_to_bf16(v)
        # exact: nearest bf16 (ties even) to the real number v
        fv = Fraction(v)
        f32 = np.float32(v)
        b = int(f32.view(np.uint32)) >> 16
        cands = {(b + d) & 0xFFFF for d in (-1, 0, 1, 2)}
        best = None
        for cnd in cands:
            cf = float(np.uint32(cnd << 16).view(np.float32))
            if not math.isfinite(cf):
                continue
            cv = Fraction(cf)
            d = abs(fv - cv)
            if best is None or d < best[0] or (d == best[0] and cnd % 2 == 0):
                best = (d, cnd)
        assert got == best[1], (v, hex(got), hex(best[1]))


def _bf16_bits(v) -> np.ndarray:
    """float64 values that are exact in bfloat16 -> their bit patterns."""
    f = np.asarray(v, dtype=np.float32)
    bits = (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    assert np.array_equal(bf16_to_f64(bits), np.asarray(v, dtype=np.float64)), "value not exact in bf16"
    return bits


def _random_bf16(rng, shape, scale=1.0) -> np.ndarray:
    """Random bfloat16 bit patterns (float32 normal values truncated to bf16)."""
    f = (rng.standard_normal(shape) * scale).astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def check_router_gemm_equal_weights(o, rng):
    """W_r[e][h] = c for all e, h: every logit of token t is c * sum_h x[t][h] (the sum
    exact by math.fsum, then one rounding)."""
    T, H, E = 3, 256, 5
    x = _random_bf16(rng, (T, H))
    c = 0.375
    w = np.full((E, H), _bf16_bits([c])[0], dtype=np.uint16)
    got = o.router_logits(x, w)
    xs = bf16_to_f64(x)
    for t in range(T):
        ref = c * math.fsum(xs[t].tolist())
        bound = 1e-15 * c * float(np.abs(xs[t]).sum())
        assert np.all(np.abs(got[t] - ref) <= bound), (t, got[t], ref)


def check_router_gemm_onehot(o, rng):
    """W_r row e = the unit vector of column perm[e]: logit[t][e] = x[t][perm[e]] exactly
    (a transposed operand or a wrong row/column index moves the values)."""
    T, H, E = 4, 64, 7
    x = _random_bf16(rng, (T, H))
    perm = rng.permutation(H)[:E]
    wv = np.zeros((E, H))
    wv[np.arange(E), perm] = 1.0
    got = o.router_logits(x, _bf16_bits(wv))
    assert np.array_equal(got, bf16_to_f64(x)[:, perm]), (got, perm)


def check_router_gemm_numpy(o, rng):
    """Random bf16 x and W_r against numpy's float64 dot product."""
    T, H, E = 5, 512, 9
    x = _random_bf16(rng, (T, H))
    w = _random_bf16(rng, (E, H), 0.05)
    got = o.router_logits(x, w)
    xs, ws = bf16_to_f64(x), bf16_to_f64(w)
    ref = xs @ ws.T
    bound = 1e-13 * (np.abs(xs) @ np.abs(ws).T)
    assert np.all(np.abs(got - ref) <= bound)


def check_router_gemm_ranking(o, rng):
    """x = all ones, W_r row e = r_e (a constant row): logit e = H r_e, so the top-k
    are the k largest r_e, largest first, with equal r broken by the lower index."""
    H, E, k = 128, 10, 4
    r = np.array([0.5, 2.0, -1.0, 3.0, 2.0, 0.25, 3.0, -2.0, 1.0, 0.0])
    x = _bf16_bits(np.ones((2, H)))
    w = _bf16_bits(np.repeat(r[:, None], H, axis=1))
    lg = o.router_logits(x, w)
    assert np.array_equal(lg, np.tile(H * r, (2, 1)))
    idx, _ = o.route(lg.astype(np.float32), k)
    assert idx[0].tolist() == [3, 6, 1, 4] and idx[1].tolist() == [3, 6, 1, 4], idx


# -- INT2 -------------------------------------------------------------------------

INT2_LEVELS = np.array([-1.5, -0.5, 0.5, 1.5])


def int2_dequant_dense(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """INT2 codes [..., K/4, N] (code of k = 4r + i in bits 2i, 2i+1), scales [..., K/32, N]
    -> float64 [..., K, N]."""
    K4, N = codes.shape[-2:]
    vals = np.empty(codes.shape[:-2] + (4 * K4, N), dtype=np.float64)
    for i in range(4):
        vals[..., i::4, :] = INT2_LEVELS[(codes >> (2 * i)) & 3]
    return vals * np.repeat(bf16_to_f64(scales), 32, axis=-2)


def check_int2_table(o):
    """Four levels, equally spaced by 1, symmetric about 0, the largest 1.5."""
    v = np.array([o.int2_decode(q) for q in range(4)])
    assert np.array_equal(v, INT2_LEVELS), v
    assert np.all(np.diff(v) == 1.0) and np.all(v == -v[::-1])


def check_int2_encode_bruteforce(o, rng):
    """Nearest level; an exact midpoint (-1, 0, 1) goes to the level above."""
    probes = np.concatenate([rng.standard_normal(400) * 1.2, [-1.0, 0.0, 1.0, -2.0, 2.0, 1.5, -1.5, 7.0, -7.0],
                             np.nextafter(np.float32([-1, 0, 1]), np.float32(-9)),
                             np.nextafter(np.float32([-1, 0, 1]), np.float32(9))]).astype(np.float32)
    levels = [Fraction(float(v)) for v in INT2_LEVELS]
    for r in probes:
        d = [abs(Fraction(float(r)) - lv) for lv in levels]   # exact distances
        best = max(q for q in range(4) if d[q] == min(d))      # ties: the higher level
        assert o.int2_encode(float(r)) == best, (float(r), o.int2_encode(float(r)), best)


def check_int2_quantize_layout(o):
    """One nonzero weight per group: its code lands in bits 2(k % 4) of byte row k // 4,
    the group's scale is bf16(|w| / 1.5), and the other (zero) weights take code 2."""
    E, K, N = 2, 64, 3
    for (e, k, n, wv) in [(0, 0, 0, 0.75), (1, 5, 2, -0.3), (0, 38, 1, 1.0), (1, 63, 0, -2.5)]:
        W = np.zeros((E, K, N), dtype=np.float32)
        W[e, k, n] = wv
        codes, scales = o.quantize_int2(W)
        s = float(bf16_to_f64(scales[e, k // 32, n]))
        assert scales[e, k // 32, n] == nearest_bf16_bits(np.float32(np.float32(abs(wv)) / np.float32(1.5)))
        q = (int(codes[e, k // 4, n]) >> (2 * (k % 4))) & 3
        assert q == (3 if wv > 0 else 0), (q, wv)
        assert abs(INT2_LEVELS[q] * s - wv) <= 0.01 * abs(wv)
        # every other weight of the group is 0: r = 0 takes the level 0.5 (code 2)
        for kk in range(32 * (k // 32), 32 * (k // 32) + 32):
            if kk != k:
                assert (int(codes[e, kk // 4, n]) >> (2 * (kk % 4))) & 3 == 2
        # other columns and groups: all-zero groups (scale 0)
        assert scales[e, (k // 32) ^ 1, n] == 0 and scales[1 - e].max() == 0


def check_int2_roundtrip(o, rng):
    """|w - dequant(w)| <= s/2 (+ the bf16 rounding of s), with s = bf16(max|w| / 1.5)."""
    W = (rng.standard_normal((2, 128, 24)) * 0.02).astype(np.float32)
    codes, scales = o.quantize_int2(W)
    deq = int2_dequant_dense(codes, scales)
    s = np.repeat(bf16_to_f64(scales), 32, axis=-2)
    assert np.all(np.abs(W - deq) <= 0.5 * s * (1 + 2.0 ** -7) + 1e-30)
    for (e, k, n) in [(0, 3, 5), (1, 100, 0), (1, 31, 23)]:
        assert o.dequant_int2(codes[e], scales[e], k, n) == np.float32(deq[e, k, n])


def check_mixed_dense_bruteforce(o, rng):
    """A layer whose experts mix E2M1 and INT2, against an unpermuted dense brute force."""
    import oracle as _oracle_pkg
    E, H, I, T, k = 6, 64, 32, 3, 3
    fmt = [1, 0, 1, 1, 0, 1]
    gu_c, gu_s, dn_c, dn_s = _layer_inputs(rng, E, H, I, T, random_codes=True)
    gu_c2 = rng.integers(0, 256, (E, H // 4, 2 * I), dtype=np.uint8)
    dn_c2 = rng.integers(0, 256, (E, I // 4, H), dtype=np.uint8)
    ew = _oracle_pkg.ExpertWeights(E, H, I)
    Wgu = np.empty((E, H, 2 * I))
    Wdn = np.empty((E, I, H))
    for e in range(E):
        if fmt[e]:
            ew.set(e, gu_c2[e], gu_s[e], dn_c2[e], dn_s[e], fmt=1)
            Wgu[e] = int2_dequant_dense(gu_c2[e], gu_s[e])
            Wdn[e] = int2_dequant_dense(dn_c2[e], dn_s[e])
        else:
            ew.set(e, gu_c[e], gu_s[e], dn_c[e], dn_s[e])
            Wgu[e] = dequant_dense(gu_c[e], gu_s[e])
            Wdn[e] = dequant_dense(dn_c[e], dn_s[e])
    x = rng.standard_normal((T, H)).astype(np.float32)
    x_bf16 = (x.view(np.uint32) >> 16).astype(np.uint16)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    y64, _ = o.moe_forward(ew, x_bf16, logits, k)
    xs = bf16_to_f64(x_bf16)
    ref = np.zeros((T, H))
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))
        sel = order[:k]
        ls = logits[t, sel].astype(np.float64)
        wsel = (np.exp(ls - ls[0]) / np.exp(ls - ls[0]).sum()).astype(np.float32).astype(np.float64)
        for j, e in enumerate(sel):
            h = xs[t] @ Wgu[e]
            a = h[:I] / (1.0 + np.exp(-h[:I])) * h[I:]
            ref[t] += wsel[j] * (a @ Wdn[e])
    assert np.abs(y64 - ref).max() <= 1e-10 * np.abs(ref).max()


# -- the NVFP4 variant -------------------------------------------------------------

def e4m3_from_bits(b: int) -> float:
    """E4M3 value from its bit fields (OCP OFP8 E4M3: bias 7, no infinities, S.1111.111 NaN)."""
    s, e, m = (b >> 7) & 1, (b >> 3) & 15, b & 7
    if e == 15 and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


E4M3_POS = [Fraction(e4m3_from_bits(c)) for c in range(0x7F)]   # the non-negative finite values


def brute_e4m3(t) -> int:
    """Nearest non-negative finite E4M3 code to t >= 0 in exact arithmetic, ties to the even
    code, values above the largest (448) to 448."""
    t = Fraction(float(t))
    if t >= E4M3_POS[-1]:
        return 0x7E
    best, bd = 0, None
    for c, v in enumerate(E4M3_POS):
        d = abs(t - v)
        if bd is None or d < bd or (d == bd and c % 2 == 0):
            best, bd = c, d
    return best


def nvfp4_row_reference(v: np.ndarray):
    """The NVFP4 row encoding, each rounding step done by numpy float32 and each nearest-value
    choice by exact search: (codes [K/2], sf [K/16], g)."""
    v = np.asarray(v, dtype=np.float32)
    K = v.shape[0]
    amax = np.float32(np.abs(v).max()) if K else np.float32(0)
    g = np.float32(amax / np.float32(2688.0))
    d6 = np.float32(np.float32(6.0) * g)
    codes = np.zeros(K // 2, dtype=np.uint8)
    sf = np.zeros(K // 16, dtype=np.uint8)
    for b in range(K // 16):
        blk = v[16 * b:16 * b + 16]
        ab = np.float32(np.abs(blk).max())
        sb = brute_e4m3(np.float32(ab / d6)) if d6 > 0 else 0
        sf[b] = sb
        dq = np.float32(np.float32(e4m3_from_bits(sb)) * g)
        rq = np.float32(np.float32(1.0) / dq) if dq > 0 else np.float32(0)
        for kk in range(16):
            k = 16 * b + kk
            c = brute_force_code(float(np.float32(blk[kk] * rq))) if dq > 0 else 0
            codes[k // 2] |= np.uint8(c << (4 * (k % 2)))
    return codes, sf, g


def nvfp4_decode_rows(codes: np.ndarray, sf: np.ndarray, g: np.ndarray) -> np.ndarray:
    """codes [R, K/2], sf [R, K/16], g [R] -> float64 [R, K]."""
    R, K2 = codes.shape
    vals = np.empty((R, 2 * K2))
    vals[:, 0::2] = E2M1_TABLE[codes & 0x0F]
    vals[:, 1::2] = E2M1_TABLE[codes >> 4]
    s = np.repeat(np.array([[e4m3_from_bits(int(b)) for b in row] for row in sf]), 16, axis=1)
    return vals * s * g.astype(np.float64)[:, None]


def check_e4m3_table(o):
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "e4m3_values.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 12
    for b_s, v_s in rows:
        b, v = int(b_s, 16), float(v_s)
        got, ref = o.e4m3_decode(b), e4m3_from_bits(b)
        if math.isnan(v):
            assert math.isnan(got) and math.isnan(ref), f"byte {b:#x}"
        else:
            assert ref == v and got == v and math.copysign(1, got) == math.copysign(1, v), f"byte {b:#x}"
    for b in range(256):
        got, ref = o.e4m3_decode(b), e4m3_from_bits(b)
        assert (math.isnan(got) and math.isnan(ref)) or got == ref, f"byte {b:#x}"
    pos = [o.e4m3_decode(b) for b in range(0x7F)]
    assert all(a < b for a, b in zip(pos, pos[1:]))


def check_e4m3_encode(o, rng):
    vals = [float(v) for v in E4M3_POS]
    mids = [(a + b) / 2 for a, b in zip(E4M3_POS, E4M3_POS[1:])]
    base = np.array(vals + [float(m) for m in mids] + [448.0, 464.0, 480.0, 1e6, 2.0 ** -10, 2.0 ** -11, 0.0],
                    dtype=np.float32)
    near = np.concatenate([np.nextafter(base, np.float32(np.inf)), np.nextafter(base, np.float32(0))])
    rnd = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(600.0), 600)).astype(np.float32)
    for t in np.concatenate([base, near, rnd]):
        assert o.e4m3_encode(float(t)) == brute_e4m3(t), f"e4m3({float(t)!r})"


def _nvfp4_probe_rows(rng) -> np.ndarray:
    K = 64
    rows = [rng.standard_normal(K) * 0.02, rng.standard_normal(K) * 30.0, rng.standard_normal(K) * 1e-5,
            np.where(rng.random(K) < 0.3, rng.standard_normal(K), 0.0), np.zeros(K),
            rng.standard_normal(K) * np.repeat(10.0 ** rng.uniform(-6, 2, K // 16), 16)]
    # values on the E2M1 decision points of their block
    r = rng.standard_normal(K) * 0.1
    r[0] = 1.0
    r[1:8] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]) / 6.0
    rows.append(r)
    return np.array(rows, dtype=np.float32)


def check_nvfp4_row_bruteforce(o, rng):
    V = _nvfp4_probe_rows(rng)
    codes, sf, g = o.nvfp4_quantize(V)
    for r in range(V.shape[0]):
        c_ref, s_ref, g_ref = nvfp4_row_reference(V[r])
        assert g[r] == g_ref, f"row {r}: g {g[r]!r} vs {g_ref!r}"
        assert np.array_equal(sf[r], s_ref), f"row {r}: scale factors"
        assert np.array_equal(codes[r], c_ref), f"row {r}: codes"


def check_nvfp4_layout(o):
    K = 48
    for (k, v) in [(0, 0.3), (17, -2.5), (47, 1e-3), (32, 7.0)]:
        V = np.zeros((1, K), dtype=np.float32)
        V[0, k] = v
        codes, sf, g = o.nvfp4_quantize(V)
        # the single value is its row's and its block's maximum: scale factor 448, code 6
        assert g[0] == np.float32(np.float32(abs(v)) / np.float32(2688.0))
        exp_sf = np.zeros(K // 16, dtype=np.uint8)
        exp_sf[k // 16] = 0x7E
        assert np.array_equal(sf[0], exp_sf), (k, sf[0])
        exp_c = np.zeros(K // 2, dtype=np.uint8)
        exp_c[k // 2] = (0xF if v < 0 else 0x7) << (4 * (k % 2))
        assert np.array_equal(codes[0], exp_c), (k, codes[0])


def check_nvfp4_closed_form_and_bounds(o, rng):
    # a constant row decodes to itself exactly: g = c / 2688, scale factor 448, code 6
    for c in [0.37, 1.0, 3e-4, 250.0]:
        V = np.full((1, 32), c, dtype=np.float32)
        codes, sf, g = o.nvfp4_quantize(V)
        assert np.all(codes == 0x77) and np.all(sf == 0x7E)
        assert np.allclose(nvfp4_decode_rows(codes, sf, g), np.float32(c), rtol=2e-7, atol=0)
    V = _nvfp4_probe_rows(rng)
    codes, sf, g = o.nvfp4_quantize(V)
    dec = nvfp4_decode_rows(codes, sf, g)
    for r in range(V.shape[0]):
        for b in range(V.shape[1] // 16):
            s = e4m3_from_bits(int(sf[r, b])) * float(g[r])
            blk = V[r, 16 * b:16 * b + 16].astype(np.float64)
            if s == 0.0:
                assert np.all(dec[r, 16 * b:16 * b + 16] == 0.0)
                continue
            # the block maximum fits below 6 s up to the scale factor's rounding (3 mantissa bits)
            assert np.abs(blk).max() <= 6.0 * s * (1.0 + 2.0 ** -4) * (1 + 1e-6)
            # nearest-value rounding: within half of the widest E2M1 gap (2 s) unless saturated
            err = np.abs(blk - dec[r, 16 * b:16 * b + 16])
            assert np.all(err <= np.maximum(1.0 * s, np.abs(blk) - 6.0 * s) * (1 + 1e-6) + 1e-300)
    # sign symmetry
    c2, s2, g2 = o.nvfp4_quantize(-V)
    assert np.array_equal(s2, sf) and np.array_equal(g2, g)
    nz_lo, nz_hi = (codes & 0x07) != 0, (codes & 0x70) != 0
    flip = (nz_lo * 0x08 + nz_hi * 0x80).astype(np.uint8)
    assert np.array_equal(c2, codes ^ flip)


def nvfp4_dense_layer_reference(o, x_bf16, logits, k, gu_c, gu_s, dn_c, dn_s):
    """The NVFP4 variant, unpermuted: every operand encoded with the (pinned) row encoder,
    every token through every expert as dense float64 matmuls, act rounded to bf16 by
    enumeration of its neighbours, the routing mask applied at the end."""
    T, H = x_bf16.shape
    E = logits.shape[1]
    I = dn_c.shape[1] * 2
    xq = nvfp4_decode_rows(*o.nvfp4_quantize(bf16_to_f64(x_bf16).astype(np.float32)))
    Wgu = dequant_dense(gu_c, gu_s)       # [E, H, 2I]
    Wdn = dequant_dense(dn_c, dn_s)       # [E, I, H]
    y = np.zeros((T, H))
    for e in range(E):
        wg = nvfp4_decode_rows(*o.nvfp4_quantize(Wgu[e].T.astype(np.float32))).T   # columns along K
        wd = nvfp4_decode_rows(*o.nvfp4_quantize(Wdn[e].T.astype(np.float32))).T
        for t in range(T):
            order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))
            sel = list(order[:k])
            if e not in sel:
                continue
            ls = logits[t, order[:k]].astype(np.float64)
            wsel = (np.exp(ls - ls[0]) / np.exp(ls - ls[0]).sum()).astype(np.float32).astype(np.float64)
            h = xq[t] @ wg
            a = h[:I] / (1.0 + np.exp(-h[:I])) * h[I:]
            a16 = np.array([nearest_bf16_bits(np.float32(v)) if abs(v) < 3e38 else 0 for v in a], dtype=np.uint16)
            aq = nvfp4_decode_rows(*o.nvfp4_quantize(bf16_to_f64(a16)[None, :].astype(np.float32)))[0]
            y[t] += wsel[sel.index(e)] * (aq @ wd)
    return y


def check_nvfp4_dense_bruteforce(o, rng):
    for (E, H, I, T, k) in [(4, 64, 32, 3, 2), (6, 32, 64, 2, 3)]:
        gu_c, gu_s, dn_c, dn_s = _layer_inputs(rng, E, H, I, T, random_codes=True)
        x = rng.standard_normal((T, H)).astype(np.float32)
        x_bf16 = (x.view(np.uint32) >> 16).astype(np.uint16)
        logits = rng.standard_normal((T, E)).astype(np.float32)
        ew = _expert_weights(E, H, I, gu_c, gu_s, dn_c, dn_s)
        y64, _ = o.moe_forward_nvfp4(ew, x_bf16, logits, k)
        ref = nvfp4_dense_layer_reference(o, x_bf16, logits, k, gu_c, gu_s, dn_c, dn_s)
        scale = np.abs(ref).max()
        assert np.abs(y64 - ref).max() <= 1e-10 * scale, np.abs(y64 - ref).max() / scale
        # the variant approximates the exact layer (a swapped operand or a lost scale would not)
        exact, _ = o.moe_forward(ew, x_bf16, logits, k)
        assert np.linalg.norm(y64 - exact) <= 0.3 * np.linalg.norm(exact)


ALL_CHECKS = [
    ("e2m1_table", lambda o, rng: check_e2m1_table(o)),
    ("encode_bruteforce", check_encode_bruteforce),
    ("quantize_layout", lambda o, rng: check_quantize_layout(o)),
    ("quantize_roundtrip", check_quantize_roundtrip),
    ("router_golden", lambda o, rng: check_router_golden(o)),
    ("router_random", check_router_random),
    ("group", check_group),
    ("closed_form", check_closed_form),
    ("dense_bruteforce", check_dense_bruteforce),
    ("bf16_output_rounding", check_bf16_output_rounding),
    ("router_gemm_equal_weights", check_router_gemm_equal_weights),
    ("router_gemm_onehot", check_router_gemm_onehot),
    ("router_gemm_numpy", check_router_gemm_numpy),
    ("router_gemm_ranking", check_router_gemm_ranking),
    ("int2_table", lambda o, rng: check_int2_table(o)),
    ("int2_encode_bruteforce", check_int2_encode_bruteforce),
    ("int2_quantize_layout", lambda o, rng: check_int2_quantize_layout(o)),
    ("int2_roundtrip", check_int2_roundtrip),
    ("mixed_dense_bruteforce", check_mixed_dense_bruteforce),
    ("e4m3_table", lambda o, rng: check_e4m3_table(o)),
    ("e4m3_encode", check_e4m3_encode),
    ("nvfp4_row_bruteforce", check_nvfp4_row_bruteforce),
    ("nvfp4_layout", lambda o, rng: check_nvfp4_layout(o)),
    ("nvfp4_closed_form_and_bounds", check_nvfp4_closed_form_and_bounds),
    ("nvfp4_dense_bruteforce", check_nvfp4_dense_bruteforce),
]
