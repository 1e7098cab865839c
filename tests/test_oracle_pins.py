"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test ties the oracle to a fact the source pages fix (page "Paired-count
resident layout": 512-scan blocks, pairs, 1024-state tANS, 32 Poisson pair
models, four alternative forms, grouped offsets, exact integer sums, uint64
promotion, malformed streams raise, block_stride touches ceil(blocks/k)
blocks), to a closed form or library routine (scipy's Poisson pmf, Shannon
code lengths, brute-force dense sums), or to hand-derived golden bytes.
"""
import math
import os

import numpy as np
import pytest
from scipy import stats

import oracle as O
import workloads as W
from golden_io import frozen_tables

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LAM = lambda m: 0.005 * (16.0 / 0.005) ** (m / 31.0)


def _contract():
    out = {}
    for line in open(os.path.join(GOLDEN, "contract.txt")):
        line = line.split("|")[0].strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            out[k] = v
    return out


# ----------------------------------------------------------------------------
# constants the pages fix
# ----------------------------------------------------------------------------
def test_contract_constants():
    c = _contract()
    f, a, cost = O.models()
    assert f.shape[0] == int(c["pair_models"])
    assert int(f[0].sum()) == int(c["tans_states"])
    sym, nb, nbase = O.decode_table(0)
    assert sym.size == int(c["tans_states"])
    # a pair symbol carries two counts
    assert f.shape[1] == 16 ** int(c["pair_length"])
    # 512-scan blocks: one stream is 512 counts; a constant u8 stream is header + 1 byte
    s = O.encode_stream(np.full(int(c["scans_per_block"]), 3, np.uint16), 1)
    assert len(s) == int(c["header_bytes"]) + 1
    # grouped offsets: one 32-bit base and 32 16-bit relative offsets per 32 streams
    x = np.random.default_rng(0).poisson(1.0, (512, 70)).astype(np.uint8)
    g, p = O.encode_block(x, 8)
    assert g.shape == (math.ceil(70 / int(c["group_streams"])), 1 + 32 * int(c["group_rel_bits"]) // 32)
    assert g.dtype.itemsize * 8 == int(c["group_base_bits"])


def _golden_bytes(text):
    """Hex bytes with XX*n (a repeated byte) and (XX YY ..)*n (a repeated group)."""
    import re

    out = bytearray()
    for grp, reps, tok in re.findall(r"\(([0-9A-Fa-f ]+)\)\*(\d+)|(\S+)", text):
        if grp:
            out += bytes(int(t, 16) for t in grp.split()) * int(reps)
        elif "*" in tok:
            b, n = tok.split("*")
            out += bytes([int(b, 16)]) * int(n)
        else:
            out.append(int(tok, 16))
    return bytes(out)


def _golden_values(spec, w):
    v = np.zeros(512, np.uint16)
    kind, *args = spec.split()
    if kind == "zeros":
        pass
    elif kind == "const":
        v[:] = int(args[0])
    elif kind == "sparse":
        for t in args:
            pos, val = t.split(":")
            v[int(pos)] = int(val)
    elif kind == "affine":
        v[:] = (int(args[0]) * np.arange(512) + int(args[1])) % (1 << (8 * w))
    elif kind == "based":
        base, shift, mod = int(args[0]), int(args[1]), int(args[2])
        hi = np.zeros(512, np.int64)
        hi[[int(t) for t in args[3].split(",")]] = 1
        v[:] = base + ((hi << shift) | (np.arange(512) % mod))
    else:
        raise AssertionError(kind)
    return v


def test_golden_forms():
    """Hand-derived byte images of every form (tests/golden/forms.txt, derivations in
    its comments): encode gives the bytes and decode gives the values back; dec_* rows
    are decoder-only images (raw low bits beside the tANS section)."""
    seen = set()
    for line in open(os.path.join(GOLDEN, "forms.txt")):
        if line.startswith("#") or not line.strip():
            continue
        name, w, spec, expected = (t.strip() for t in line.split("|"))
        w = int(w)
        v = _golden_values(spec, w)
        if expected == "-":
            want = b""
        elif expected == "literal":
            want = bytes([4, 0]) + v.astype("<u2" if w == 2 else "u1").tobytes()
        else:
            want = _golden_bytes(expected)
        rc, back = O.decode_stream(want, w)
        assert rc == 0 and (back == v).all(), name
        got = O.encode_stream(v, w)
        if name.startswith("dec_"):
            assert got != want, name                      # the encoder picks shift 0 for these
            assert O.stream_header(got)[2] == 0, name
            rc, back = O.decode_stream(got, w)
            assert rc == 0 and (back == v).all(), name
        else:
            assert got == want, name
        seen.add(name.split("_")[0])
    assert {"empty", "const", "sparse", "literal", "paired", "based", "dec"} <= seen


# ----------------------------------------------------------------------------
# model tables against scipy's Poisson pmf
# ----------------------------------------------------------------------------
def _box_pmf(m):
    lam = LAM(m)
    q = stats.poisson.pmf(np.arange(15), lam)
    q = np.append(q, stats.poisson.sf(14, lam))          # tail folded into 15
    return q


def test_model_lambda_endpoints():
    assert LAM(0) == pytest.approx(0.005)
    assert LAM(31) == pytest.approx(16.0)


def test_model_tables_against_poisson():
    f, amax, cost = O.models()
    for m in range(32):
        q = _box_pmf(m)
        A = int(amax[m])
        # box: smallest A whose tail beyond A is below 2^-20
        tails = [q[a + 1:].sum() for a in range(16)]
        first = next(a for a in range(16) if tails[a] < 2.0 ** -20)
        assert A == first, m
        t = q[: A + 1] / q[: A + 1].sum()
        F = f[m].reshape(16, 16)                          # F[b][a], symbol a + 16 b
        assert int(F.sum()) == 1024
        inside = np.zeros((16, 16), bool)
        inside[: A + 1, : A + 1] = True
        assert (F[inside] >= 1).all() and (F[~inside] == 0).all()
        assert (np.abs(F.astype(int) - F.T.astype(int)) <= 1).all()   # ties split by symbol order
        K = 1024 - (A + 1) ** 2
        raw = np.outer(t, t) * K                          # raw[b][a]
        extra = F[: A + 1, : A + 1].astype(float) - 1.0 - np.floor(raw)
        assert np.isin(extra, [0.0, 1.0]).all(), m        # floor, plus at most one
        fr = raw - np.floor(raw)
        if (extra == 1).any() and (extra == 0).any():     # largest remainders got the +1
            assert fr[extra == 1].min() >= fr[extra == 0].max() - 1e-9, m
        # selection costs: round(256 * -log2 t)
        want = -256.0 * np.log2(t)
        assert np.all(np.abs(cost[m, : A + 1] - want) <= 0.5 + 1e-6), m


def test_decode_table_structure():
    f, amax, _ = O.models()
    for m in range(32):
        sym, nb, nbase = O.decode_table(m)
        counts = np.bincount(sym, minlength=256)
        assert (counts == f[m]).all()
        # spread: the k-th slot visited by the odd step holds non-decreasing symbols
        order = (643 * np.arange(1024)) % 1024
        assert len(set(order.tolist())) == 1024
        assert (np.diff(sym[order].astype(int)) >= 0).all()
        for s in np.nonzero(f[m])[0]:
            slots = np.nonzero(sym == s)[0]
            y = ((nbase[slots].astype(int) + 1024) >> nb[slots].astype(int))
            assert (y == np.arange(f[m][s], 2 * f[m][s])).all()
            top = (y << nb[slots].astype(int))
            assert ((top >= 1024) & (top < 2048)).all()
            assert (((y + 1) << nb[slots].astype(int)) <= 2048).all()


# ----------------------------------------------------------------------------
# the coder
# ----------------------------------------------------------------------------
def _streams(rng, n, w):
    dmax = (1 << (8 * w)) - 1
    out = []
    for i in range(n):
        kind = i % 8
        if kind == 0:
            v = rng.poisson(rng.uniform(0, 0.05), 512)
        elif kind == 1:
            v = rng.poisson(rng.uniform(0.05, 4), 512)
        elif kind == 2:
            v = rng.poisson(rng.uniform(4, 40), 512)
        elif kind == 3:
            v = rng.poisson(rng.uniform(40, 2000 if w == 2 else 200), 512)
        elif kind == 4:
            v = rng.integers(0, dmax + 1, 512)
        elif kind == 5:
            v = np.zeros(512, int)
            k = rng.integers(1, 300)
            v[rng.choice(512, k, replace=False)] = rng.integers(1, dmax + 1, k)
        elif kind == 6:
            v = np.full(512, rng.integers(0, dmax + 1))
        else:
            v = np.full(512, dmax)
            v[rng.integers(0, 512)] = rng.integers(0, dmax)
        out.append(np.minimum(v, dmax).astype(np.uint16))
    return out


@pytest.mark.parametrize("w", [1, 2])
def test_roundtrip_brute(w):
    """Page: every original count is retained exactly."""
    rng = np.random.default_rng(10 + w)
    for v in _streams(rng, 400, w):
        s = O.encode_stream(v, w)
        assert len(s) <= 2 + 512 * w
        rc, back = O.decode_stream(s, w)
        assert rc == 0 and (back == v).all()


def test_tans_cost_matches_shannon():
    """Paired length tracks the ideal code length sum(log2(1024/f)) of its model."""
    f, amax, _ = O.models()
    rng = np.random.default_rng(3)
    for lam in [0.02, 0.3, 1.5, 3.0, 7.0]:
        for _ in range(6):
            v = np.minimum(rng.poisson(lam, 512), 15).astype(np.uint16)
            v[0] = 0                                      # no base: hi == v, shift 0
            for m in range(32):
                n = O.paired_size(v, 1, m)
                if n < 0:
                    assert v.max() > amax[m]
                    continue
                hdr = O.stream_header(O.encode_stream(v, 1))
                shift = 0
                states = 2 if m >= 8 else 1              # spec S3: models 8-31 use two states
                ideal = 10 * states + sum(math.log2(1024 / f[m][int(v[2 * j] + 16 * v[2 * j + 1])])
                                          for j in range(256))
                bits_hi = 8 * (n - 2 - 64 * shift)
                # tANS tracks the Shannon length of its quantised model to within
                # the initial state plus a few percent (slot-position error)
                assert bits_hi - 8 < ideal + 12 + 0.03 * ideal, (lam, m)
                assert bits_hi >= ideal - 12 - 0.03 * ideal, (lam, m)
                del hdr


def test_model_choice_near_best():
    """The fixed-point selection lands within 4 % of the best model's exact size."""
    rng = np.random.default_rng(4)
    tot_sel = tot_best = 0
    for lam in [0.02, 0.1, 0.5, 1, 2, 3, 5, 9]:
        for _ in range(8):
            v = rng.poisson(lam, 512).astype(np.uint16)
            sizes = [O.paired_size(v, 1, m) for m in range(32)]
            best = min(s for s in sizes if s > 0)
            sel = O.stream_sizes(v, 1)[1]
            assert sel <= 1.04 * best + 2
            tot_sel += sel
            tot_best += best
    assert tot_sel <= 1.01 * tot_best


def _brute_model(hist, box, cost):
    """Spec S6 by enumeration: among the models whose box holds the largest hi,
    the lowest total fixed-point cost sum_v h[v] * cost[m][v]; ties to the lowest m."""
    top = max(v for v in range(16) if hist[v])
    best_m, best_c = None, None
    for m in range(32):
        if box[m] < top:
            continue
        total = sum(int(hist[v]) * int(cost[m][v]) for v in range(16) if hist[v])
        if best_c is None or total < best_c:
            best_m, best_c = m, total
    return best_m


def _tie_histograms(box, cost):
    """Histograms over hi in {0, 1, 2} (512 counts) on which two models reach the
    lowest total exactly: the rule must pick the lower model number."""
    out = []
    for h1 in range(0, 513, 3):
        for h2 in range(1, 513 - h1):
            h0 = 512 - h1 - h2
            if h0 < 1:
                continue
            tot = {m: h0 * int(cost[m][0]) + h1 * int(cost[m][1]) + h2 * int(cost[m][2])
                   for m in range(32) if box[m] >= 2}
            low = min(tot.values())
            if sum(1 for t in tot.values() if t == low) > 1:
                out.append((h0, h1, h2))
    return out


def test_model_choice_exact():
    """Spec S6 model selection against enumeration over all 32 frozen models: random
    hi histograms (with and without base and raw low bits) and constructed exact ties,
    which must go to the lowest model number."""
    _, _, box, cost = frozen_tables()
    rng = np.random.default_rng(31)
    cases = []
    for lam in [0.01, 0.05, 0.2, 0.7, 1.5, 3, 6, 10, 14]:
        for _ in range(6):
            v = np.minimum(rng.poisson(lam, 512), 15)
            v[rng.integers(0, 512)] = 0                 # min 0: no base, shift 0
            if v.max() > 0:
                cases.append(("plain", v.astype(np.uint16), 1))
    for _ in range(20):                                 # base and raw low bits (uint16)
        base = int(rng.integers(1, 3000))
        shift = int(rng.integers(1, 9))
        hi = np.minimum(rng.poisson(rng.uniform(0.2, 9), 512), 15)
        hi[rng.integers(0, 512)] = 0
        hi[rng.integers(0, 512)] = max(8, int(hi.max()))   # top hi >= 8 keeps the shift
        lo = rng.integers(0, 1 << shift, 512)
        lo[hi.argmin()] = 0                             # one element equals the base
        cases.append(("shifted", (base + (hi << shift) + lo).astype(np.uint16), 2))
    ties = _tie_histograms(box, cost)
    assert len(ties) >= 20
    for h0, h1, h2 in ties[:: max(1, len(ties) // 24)]:
        v = np.array([0] * h0 + [1] * h1 + [2] * h2, np.uint16)
        cases.append(("tie", rng.permutation(v), 1))
    n_ties = 0
    for kind, v, w in cases:
        vv = v.astype(np.int64)
        base = int(vv.min())
        shift = max(0, int(vv.max() - base).bit_length() - 4)
        hist = np.bincount((vv - base) >> shift, minlength=16)
        want = _brute_model(hist, box, cost)
        got = O.stream_sizes(v, w)[3]
        assert got == want, (kind, hist.tolist(), got, want)
        if kind == "tie":
            top = max(t for t in range(16) if hist[t])
            lows = [m for m in range(32) if box[m] >= top and
                    sum(int(hist[t]) * int(cost[m][t]) for t in range(16)) ==
                    sum(int(hist[t]) * int(cost[want][t]) for t in range(16))]
            assert len(lows) > 1 and want == min(lows)
            n_ties += 1
        s = O.encode_stream(v, w)
        hdr = O.stream_header(s)
        if hdr[0] == 3:
            assert hdr[1] == want and hdr[2] == shift and hdr[3] == int(base > 0)
    assert n_ties >= 20


@pytest.mark.parametrize("w", [1, 2])
def test_form_rule(w):
    """Contract: sparse preferred unless the paired stream saves at least two bytes."""
    rng = np.random.default_rng(20 + w)
    seen_tie = set()
    extra = [_sparse_near_boundary(rng, w) for _ in range(3000)]
    for v in _streams(rng, 400, w) + extra:
        s = O.encode_stream(v, w)
        if not v.any():
            assert s == b""
            continue
        if (v == v[0]).all():
            assert O.stream_header(s)[0] == 1
            continue
        sp, pa, lit, _ = O.stream_sizes(v, w)
        form = O.stream_header(s)[0]
        if sp <= pa + 1:
            want, size = 2, sp
        else:
            want, size = 3, pa
        if size >= lit:
            want, size = 4, lit
        assert form == want and len(s) == size
        if sp - pa in (1, 2) and size < lit:
            seen_tie.add(sp - pa)
    assert seen_tie == {1, 2}, "boundary of the two-byte rule not exercised"


def _sparse_near_boundary(rng, w):
    v = np.zeros(512, np.uint16)
    k = int(rng.integers(1, 120))
    v[rng.choice(512, k, replace=False)] = rng.integers(1, 1 << int(rng.integers(1, 9)), k)
    return v


def test_group_bound_worst_case():
    """32 literal uint16 streams still fit a group's 16-bit relative offsets."""
    x = np.random.default_rng(5).integers(0, 65536, (512, 32)).astype(np.uint16)
    g, p = O.encode_block(x, 16)
    ends = [(g[0, 1 + j // 2] >> (16 * (j & 1))) & 0xFFFF for j in range(32)]
    assert ends[-1] == 32 * 1026 and ends[-1] < 65536


def test_group_layout_invariants():
    w = W.workload("s19")
    x = w.host_counts()
    g, p = O.encode_block(x[:512], 16)
    P = w.n_pixels
    G = g.shape[0]
    prev_end = 0
    for gi in range(G):
        ends = [int((g[gi, 1 + j // 2] >> (16 * (j & 1))) & 0xFFFF) for j in range(32)]
        assert g[gi, 0] == prev_end
        assert all(b >= a for a, b in zip([0] + ends, ends))
        for j in range(32):
            if 32 * gi + j >= P:
                assert ends[j] == ends[j - 1]
        prev_end = int(g[gi, 0]) + ends[31]
    assert prev_end == p.size


# ----------------------------------------------------------------------------
# queries against brute force
# ----------------------------------------------------------------------------
def test_u8_mixed_fixture_mixes_stream_kinds():
    """The uint8 fixture for mixed warps: every block has 32-pixel groups holding
    plain paired streams beside paired streams with raw low bits (shift > 0),
    and low-dose run-model streams as well."""
    w = W.workload("u19")
    enc = O.encode(w.host_counts(), 8)
    for b in range(w.n_blocks):
        g, pay = enc.groups[b], enc.payloads[b]
        mixed = runs = 0
        for gi in range(g.shape[0]):
            ends = [0] + [(int(g[gi, 1 + j // 2]) >> (16 * (j & 1))) & 0xFFFF for j in range(32)]
            kinds = set()
            for j in range(32):
                a, e = int(g[gi, 0]) + ends[j], int(g[gi, 0]) + ends[j + 1]
                if e > a:
                    h = int(pay[a]) | (int(pay[a + 1]) << 8)
                    if h & 7 == 3:
                        kinds.add("shifted" if (h >> 8) & 15 else ("runs" if (h >> 3) & 31 < 8 else "plain"))
            mixed += {"plain", "shifted"} <= kinds
            runs += "runs" in kinds
        assert mixed >= 5 and runs >= 5, (b, mixed, runs)


@pytest.mark.parametrize("name", ["c1", "c2", "s17", "s19", "u19"])
def test_masked_sum_equals_dense(name):
    w = W.workload(name)
    x = w.host_counts()
    enc = O.encode(x, w.dtype_bits)
    valid = W.invalid_mask(w, 1) if name.startswith("s") else None
    dec = O.resident_decode_blocks(enc, 0, w.n_blocks)
    assert (dec == x).all()
    for k in (1, 2, 3):
        for mname, m in w.masks.items():
            d = O.dense_masked_sum(x, m, valid, k)
            r = O.resident_masked_sum(enc, m, valid, k)
            assert d.shape[0] == math.ceil(w.n_blocks / k)
            assert (d == r).all(), (name, mname, k)
    if valid is not None:
        frames = O.resident_decode_blocks(enc, 0, 1, valid)
        assert (frames[:, valid == 0] == 0).all()
        assert (frames[:, valid == 1] == x[:512][:, valid == 1]).all()


def test_dense_block_sums_is_the_masked_sum():
    """The many-mask form of the plain definition equals the per-mask one, on random
    masks and counts, with invalid pixels, and at the largest sums it is used for
    (a full 192x192 detector of 65535)."""
    rng = np.random.default_rng(12)
    for P, w in [(97, 8), (1000, 16)]:
        x = rng.integers(0, 1 << w, size=(512, P)).astype(np.uint8 if w == 8 else np.uint16)
        masks = (rng.random((7, P)) < rng.random((7, 1))).astype(np.uint8)
        valid = (rng.random(P) < 0.9).astype(np.uint8)
        got = O.dense_block_sums(x, masks, valid)
        for m in range(7):
            assert (got[m] == O.dense_masked_sum(x, masks[m], valid)[0]).all()
    x = np.full((512, 192 * 192), 65535, np.uint16)
    x[::5, ::7] = 1
    full = np.ones((1, 192 * 192), np.uint8)
    assert (O.dense_block_sums(x, full)[0] == x.astype(np.uint64).sum(axis=1)).all()


def test_uint64_promotion_257():
    """Contract: uint64 when a full-detector sum could exceed 2**32 (257x257 uint16)."""
    c = _contract()
    P = 257 * 257
    assert 257 in [int(t) for t in c["detector_sizes"].split(",")]
    assert O.out_bits_auto(P, 16) == 64
    assert O.out_bits_auto(192 * 192, 16) == 32
    assert O.out_bits_auto(P, 8) == 32
    x = np.full((512, P), 65535, np.uint16)
    x[::7, ::3] = 65534
    enc = O.encode(x, 16)
    full = np.ones(P, np.uint8)
    r = O.resident_masked_sum(enc, full)
    closed = P * 65535 - np.array([len(range(0, P, 3)) if i % 7 == 0 else 0 for i in range(512)])
    assert (r[0] == closed.astype(np.uint64)).all()
    assert int(r.max()) > int(c["u32_limit"])


# ----------------------------------------------------------------------------
# malformed streams raise (page: "ValueError from the query; the result is not returned")
# ----------------------------------------------------------------------------
def _fixture_block():
    w = W.workload("s17")
    x = w.host_counts()[:512]
    g, p = O.encode_block(x, 16)
    return w, x, g, p


def _extent(g, p_idx):
    gi, j = divmod(p_idx, 32)
    e = lambda j: int((g[gi, 1 + j // 2] >> (16 * (j & 1))) & 0xFFFF)
    return int(g[gi, 0]) + (e(j - 1) if j else 0), int(g[gi, 0]) + e(j)


def _first_of_form(g, p, P, form):
    for q in range(P):
        a, b = _extent(g, q)
        if b > a and (p[a] & 7) == form:
            return q, a, b
    raise AssertionError(form)


@pytest.mark.parametrize("bit", [13, 14, 15])
def test_reserved_bit_rejected(bit):
    w, x, g, p = _fixture_block()
    q, a, b = _first_of_form(g, p, w.n_pixels, 3)
    bad = p.copy()
    bad[a + 1] |= 1 << (bit - 8)
    with pytest.raises(O.MalformedStream):
        O.block_masked_sum(g, bad, 16, w.n_pixels, np.array([q]), np.array([1]))
    assert O.block_masked_sum(g, p, 16, w.n_pixels, np.array([q]), np.array([1])).sum() == x[:, q].sum()


def test_shortened_extent_rejected():
    """Verification: a shortened stream extent is rejected, for every form it can hit."""
    w, x, g, p = _fixture_block()
    for form in (1, 2, 3, 4):
        try:
            q, a, b = _first_of_form(g, p, w.n_pixels, form)
        except AssertionError:
            continue
        gi, j = divmod(q, 32)
        bad = g.copy()
        word = int(bad[gi, 1 + j // 2])
        sh = 16 * (j & 1)
        bad[gi, 1 + j // 2] = np.uint32(word - (1 << sh))
        with pytest.raises(O.MalformedStream):
            O.block_masked_sum(bad, p, 16, w.n_pixels, np.array([q]), np.array([1]))


def test_bad_forms_rejected():
    v = np.random.default_rng(6).poisson(2.0, 512).astype(np.uint16)
    s = bytearray(O.encode_stream(v, 1))
    assert s[0] & 7 == 3
    for form in (0, 5, 6, 7):
        t = bytearray(s)
        t[0] = (t[0] & ~7) | form
        assert O.decode_stream(bytes(t), 1)[0] != 0
    # constant zero
    assert O.decode_stream(bytes([1, 0, 0]), 1)[0] == 6
    # model/shift on a constant
    assert O.decode_stream(bytes([1 | 8, 0, 3]), 1)[0] == 3
    # sparse non-ascending positions: 5 then 5
    assert O.decode_stream(bytes([2, 0, 1, 5, 10, 0, 1, 1]), 1)[0] == 5
    # sparse nonzero pad bit (n=1: 9 bits in 2 bytes, bit 15 set)
    assert O.decode_stream(bytes([2, 0, 0, 5, 0x80, 1]), 1)[0] == 8
    # sparse zero value
    assert O.decode_stream(bytes([2, 0, 0, 5, 0, 0]), 1)[0] == 5
    # paired with a flipped bit in the tANS section is caught (state, length or pad)
    caught = 0
    for pos in range(2, len(s)):
        for bit in range(8):
            t = bytearray(s)
            t[pos] ^= 1 << bit
            rc, back = O.decode_stream(bytes(t), 1)
            caught += rc != 0 or not (back == v).all()
    assert caught == 8 * (len(s) - 2)
    # extra trailing byte
    assert O.decode_stream(bytes(s) + b"\0", 1)[0] == 4


def test_stride_touches_ceil_blocks():
    for B in range(1, 40):
        for k in range(1, 20):
            assert len(O.touched_blocks(B, k)) == math.ceil(B / k)
    w = W.workload("c2")
    x = w.host_counts()
    enc = O.encode(x, 16)
    bf = w.masks["bf"]
    q = int(np.nonzero(bf)[0][0])
    a, b = _extent(enc.groups[1], q)
    enc.payloads[1] = enc.payloads[1].copy()
    enc.payloads[1][a + 1] |= 0x80                   # reserved bit in block 1
    r = O.resident_masked_sum(enc, bf, None, 2)      # blocks 0,2,4,6: no error
    assert (r == O.dense_masked_sum(x, bf, None, 2)).all()
    with pytest.raises(O.MalformedStream):
        O.resident_masked_sum(enc, bf, None, 1)


def test_delta_chain_equals_full():
    w = W.workload("c2")
    x = w.host_counts()
    enc = O.encode(x, 16)
    for k in (1, 3):
        img = O.resident_masked_sum(enc, w.drag[0], None, k)
        for t in range(1, len(w.drag)):
            img = O.resident_delta(enc, img, w.drag[t - 1], w.drag[t], None, k)
            assert (img == O.dense_masked_sum(x, w.drag[t], None, k)).all(), (k, t)


def test_moments_pins():
    """The moment definition against closed forms: unit weights give the masked sum; one lit
    pixel per scan puts the centre of mass exactly on it; weights are linear; a pattern mirrored
    about the centre has zero first moment; strides take the touched blocks."""
    rng = np.random.default_rng(11)
    R, C, scans = 9, 11, 1024
    P = R * C
    x = rng.integers(0, 300, size=(scans, P)).astype(np.uint16)
    mask = (rng.random(P) < 0.6).astype(np.uint8)
    valid = (rng.random(P) < 0.9).astype(np.uint8)
    ones = np.ones((2, P), np.int32)
    m = O.dense_masked_moments(x, mask, ones, valid, 1)
    s = O.dense_masked_sum(x, mask, valid, 1).astype(np.int64)
    assert (m[0] == s).all() and (m[1] == s).all() and (m[2] == s).all()
    # one lit pixel per scan: CoM = its (row - r0, col - c0) exactly
    r0, c0 = 4, 5
    rr, cc = np.divmod(np.arange(P), C)
    w = np.stack([rr - r0, cc - c0]).astype(np.int32)
    lit = rng.integers(0, P, size=scans)
    y = np.zeros((scans, P), np.uint16)
    y[np.arange(scans), lit] = rng.integers(1, 60000, size=scans)
    full = np.ones(P, np.uint8)
    m = O.dense_masked_moments(y, full, w)
    assert (m[2].reshape(-1) == y.sum(axis=1)).all()
    assert (m[0].reshape(-1) == y.sum(axis=1).astype(np.int64) * (lit // C - r0)).all()
    assert (m[1].reshape(-1) == y.sum(axis=1).astype(np.int64) * (lit % C - c0)).all()
    # linear in the weights
    w2 = rng.integers(-1000, 1000, size=(2, P)).astype(np.int32)
    a = O.dense_masked_moments(x, mask, w, valid, 2)
    b = O.dense_masked_moments(x, mask, w2, valid, 2)
    c = O.dense_masked_moments(x, mask, (w + w2).astype(np.int32), valid, 2)
    assert (c[:2] == a[:2] + b[:2]).all() and (c[2] == a[2]).all()
    # a pattern mirrored about the centre row has zero row moment
    z = rng.integers(0, 50, size=(scans, R, C)).astype(np.uint16)
    z = (z + z[:, ::-1, :]).reshape(scans, P)
    assert (O.dense_masked_moments(z, full, w)[0] == 0).all()
    # stride k: rows of the touched blocks
    assert (O.dense_masked_moments(x, mask, w, valid, 2)[:, 0] == O.dense_masked_moments(x, mask, w, valid, 1)[:, 0]).all()
    assert O.dense_masked_moments(x, mask, w, valid, 3).shape == (3, 1, 512)
