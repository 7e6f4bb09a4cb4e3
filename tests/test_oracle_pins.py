"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against a closed form, an invariant the pages state,
a brute-force computation on small inputs, or the page's formula evaluated by
hand (tests/golden).  A plausible mistake in the oracle -- a dropped term, a
wrong sign or index, a transposed operand, the wrong RoPE/rotation order, the
wrong max in the P codes -- fails at least one of them.

Pages: RotateAttention (arXiv 2607.02584), papernotes.org page, sections
"key design 1" (RoPE-aware rotation), "key design 2" (range-rectified P),
"overall framework" (smoothing, quantised V, INT4 QK and PV), and the gecl
reading notes ("Method", "Key Insight").
"""
import math
import os

import numpy as np
import pytest

from synth import inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

SPLITS = [
    dict(D=64, seg=(24, 20, 20), grid=(2, 4, 4)),
    dict(D=128, seg=(44, 42, 42), grid=(3, 5, 7)),
    dict(D=128, seg=(16, 56, 56), grid=(2, 3, 4)),
]


def _prob(orc, rot, sp, **kw):
    return orc.problem(D=sp["D"], seg=sp["seg"], grid=sp["grid"], rot=rot, **kw)


# --- rotation: orthogonality and QK^T equivalence (key design 1: R must be in O(D)) ---

@pytest.mark.parametrize("rot", [1, 2, 3])
@pytest.mark.parametrize("sp", SPLITS)
def test_rotation_is_orthogonal(orc, rot, sp):
    R = orc.rotation_matrix(_prob(orc, rot, sp))
    err = np.abs(R @ R.T - np.eye(sp["D"])).max()
    assert err <= 1e-15


@pytest.mark.parametrize("rot", [1, 2, 3])
@pytest.mark.parametrize("sp", SPLITS)
def test_rotation_preserves_qk(orc, rot, sp):
    rng = np.random.default_rng(7)
    R = orc.rotation_matrix(_prob(orc, rot, sp))
    Q = rng.standard_normal((33, sp["D"]))
    K = rng.standard_normal((29, sp["D"]))
    diff = np.abs(Q @ K.T - (Q @ R) @ (K @ R).T).max()
    assert diff <= 1e-12 * np.linalg.norm(Q) * np.linalg.norm(K)


def test_non_orthogonal_rotation_breaks_qk(orc):
    """Sanity check of the test above: a scaled (non-orthogonal) R fails it."""
    sp = SPLITS[1]
    rng = np.random.default_rng(8)
    R = orc.rotation_matrix(_prob(orc, 2, sp)) * np.diag(rng.uniform(0.5, 2.0, sp["D"]))
    Q = rng.standard_normal((8, sp["D"]))
    K = rng.standard_normal((8, sp["D"]))
    assert np.abs(Q @ K.T - (Q @ R) @ (K @ R).T).max() > 1e-2


@pytest.mark.parametrize("rot", [1, 2])
def test_rotation_mixes_only_within_segments(orc, rot):
    """R is block-diagonal over the frame/height/width segments (key design 1)."""
    sp = SPLITS[1]
    R = orc.rotation_matrix(_prob(orc, rot, sp))
    o = np.cumsum((0,) + sp["seg"])
    for a in range(3):
        for b in range(3):
            if a != b:
                assert np.all(R[o[a]:o[a + 1], o[b]:o[b + 1]] == 0.0)


def test_half_rotation_pairs_dims_half_a_segment_apart(orc):
    """Half rotation mixes channel i with i + Dj/2 of each segment (key design 1)."""
    sp = SPLITS[1]
    R = orc.rotation_matrix(_prob(orc, 2, sp))
    o = 0
    for dj in sp["seg"]:
        h = dj // 2
        for i in range(h):
            nz_rows = set(np.nonzero(R[:, o + 2 * i])[0]) | set(np.nonzero(R[:, o + 2 * i + 1])[0])
            assert nz_rows == {o + i, o + i + h}
        o += dj


# --- RoPE: closed-form properties of rotary embeddings --------------------

@pytest.mark.parametrize("sp", SPLITS)
def test_rope_is_identity_at_origin_and_orthogonal(orc, sp):
    p = _prob(orc, 0, sp)
    assert np.array_equal(orc.rope_matrix(p, [0, 0, 0]), np.eye(sp["D"]))
    M = orc.rope_matrix(p, [1, 2, 3])
    assert np.abs(M @ M.T - np.eye(sp["D"])).max() <= 1e-15


@pytest.mark.parametrize("sp", SPLITS)
def test_rope_depends_on_relative_position_only(orc, sp):
    """<q M_a, k M_b> depends only on a - b along each axis."""
    p = _prob(orc, 0, sp)
    rng = np.random.default_rng(3)
    q = rng.standard_normal(sp["D"])
    k = rng.standard_normal(sp["D"])
    a, b = np.array([1, 3, 5]), np.array([0, 1, 2])
    shift = np.array([1, 1, 1])
    s1 = (q @ orc.rope_matrix(p, a)) @ (k @ orc.rope_matrix(p, b))
    s2 = (q @ orc.rope_matrix(p, a + shift)) @ (k @ orc.rope_matrix(p, b + shift))
    assert abs(s1 - s2) <= 1e-12 * np.linalg.norm(q) * np.linalg.norm(k)
    s3 = (q @ orc.rope_matrix(p, a)) @ (k @ orc.rope_matrix(p, b + shift))
    assert abs(s1 - s3) > 1e-6


def test_rope_frequency_layout(orc):
    """Pair k of segment j rotates by angle pos_j * theta^(-2k/Dj): the first pair
    of each segment turns by exactly pos_j radians, the others slower."""
    sp = SPLITS[1]
    p = _prob(orc, 0, sp)
    M = orc.rope_matrix(p, [1, 2, 3])
    o = 0
    for j, dj in enumerate(sp["seg"]):
        ang = math.atan2(M[o, o + 1], M[o, o])
        assert abs(ang - math.remainder([1, 2, 3][j], 2 * math.pi)) < 1e-12
        last = math.atan2(M[o + dj - 2, o + dj - 1], M[o + dj - 2, o + dj - 2])
        expect = [1, 2, 3][j] * 10000.0 ** (-(dj - 2) / dj)
        assert abs(last - expect) < 1e-12
        o += dj


@pytest.mark.parametrize("rot", [1, 2])
def test_fused_interleaved_stays_block_diagonal(orc, rot):
    """M' = M R keeps the 2x2 block-diagonal pattern for interleaved rotation
    (so it can be pre-stored in the RoPE tables); half rotation does not."""
    sp = SPLITS[1]
    p = _prob(orc, rot, sp)
    Mp = orc.rope_matrix(p, [1, 2, 3]) @ orc.rotation_matrix(p)
    D = sp["D"]
    mask = np.zeros((D, D), bool)
    for i in range(0, D, 2):
        mask[i:i + 2, i:i + 2] = True
    if rot == 1:
        assert np.all(Mp[~mask] == 0.0)
    else:
        assert np.any(Mp[~mask] != 0.0)


@pytest.mark.parametrize("rot", [0, 1, 2, 3])
@pytest.mark.parametrize("sp", SPLITS)
def test_elementwise_prologue_equals_matrix_form(orc, rot, sp):
    """The fp32 elementwise RoPE+rotation equals x M_n R in fp64 up to fp32 rounding."""
    p = _prob(orc, rot, sp)
    rng = np.random.default_rng(11)
    pos = si.positions(sp["grid"])
    x = rng.standard_normal((len(pos), sp["D"])).astype(np.float32)
    got = orc.rope_rotate(p, x, pos).astype(np.float64)
    R = orc.rotation_matrix(p)
    for n in range(len(pos)):
        ref = x[n].astype(np.float64) @ orc.rope_matrix(p, pos[n]) @ R
        assert np.abs(got[n] - ref).max() <= 4e-6 * np.abs(x[n]).max()


def test_rotation_before_rope_breaks_relative_logits(orc):
    """RoPE first, then R: only this order keeps (q M_a R)(k M_b R)^T = q M_a M_b^T k^T."""
    sp = SPLITS[1]
    pos = si.positions(sp["grid"])
    rng = np.random.default_rng(12)
    q = rng.standard_normal((len(pos), sp["D"])).astype(np.float32)
    k = rng.standard_normal((len(pos), sp["D"])).astype(np.float32)
    plain = orc.problem(D=sp["D"], seg=sp["seg"], grid=sp["grid"], rot=0)
    half = orc.problem(D=sp["D"], seg=sp["seg"], grid=sp["grid"], rot=2)
    ref = orc.rope_rotate(plain, q, pos).astype(np.float64) @ orc.rope_rotate(plain, k, pos).astype(np.float64).T
    good = orc.rope_rotate(half, q, pos).astype(np.float64) @ orc.rope_rotate(half, k, pos).astype(np.float64).T
    bad = orc.rope_rotate(half, q, pos, True).astype(np.float64) @ orc.rope_rotate(half, k, pos, True).astype(np.float64).T
    assert np.abs(good - ref).max() < 1e-3
    assert np.abs(bad - ref).max() > 1.0


# --- quantisation ----------------------------------------------------------

def _head(orc, name, head=0):
    wl = si.WORKLOADS[name]
    x = si.make_inputs(wl, heads=(head,))
    p = orc.problem(wl)
    h = orc.prologue_head(p, x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], x["pos"], want_rot=True)
    return wl, p, x, h


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_qk_quantisation_round_trip(orc, name):
    """Per-token symmetric INT4: codes in [-7, 7], |x - s c| <= s/2, the largest
    magnitude maps to +-7 (gecl notes: per-token INT4 for Q and K)."""
    wl, p, x, h = _head(orc, name)
    for codes4, s, xr in ((h["q4"], h["sq"], h["q_rot"]),
                          (h["k4"], h["sk"], h["k_rot"] - h["kmean"][None, :])):
        c = orc.unpack_codes(codes4).astype(np.float64)
        assert c.min() >= -7 and c.max() <= 7
        err = np.abs(xr - s[:, None] * c)
        assert np.all(err <= s[:, None] * 0.5 * (1 + 1e-5) + 1e-7)
        amax_idx = np.abs(xr).argmax(axis=1)
        assert np.all(np.abs(c[np.arange(len(c)), amax_idx]) == 7)
        assert np.allclose(s, np.abs(xr).max(axis=1) / 7.0, rtol=1e-6)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_v_quantisation_round_trip(orc, name):
    """Per-channel symmetric INT4 of V (papernotes page, overall framework:
    quantised V; the same symmetric rule as Q and K, taken over the tokens of a
    channel): codes in [-7, 7], |v - s_v c| <= s_v/2 for every element, the
    largest magnitude of each channel maps to +-7 with the value's sign, and
    s_v = amax/7 of its own channel.  Floor instead of rint, a missing clamp
    or a scale taken from another channel each breaks one of these."""
    wl, p, x, h = _head(orc, name)
    v = x["v"][0, 0].astype(np.float64)
    c = orc.unpack_codes(h["v4"]).astype(np.float64)
    s = h["sv"].astype(np.float64)
    assert c.min() >= -7 and c.max() <= 7
    err = np.abs(v - s[None, :] * c)
    assert np.all(err <= s[None, :] * 0.5 * (1 + 1e-5) + 1e-7)
    amax_idx = np.abs(v).argmax(axis=0)
    top = c[amax_idx, np.arange(wl.D)]
    assert np.all(top == 7 * np.sign(v[amax_idx, np.arange(wl.D)]))
    assert np.allclose(s, np.abs(v).max(axis=0) / 7.0, rtol=1e-6)
    # channels are quantised independently: scaling one channel of V by 2
    # doubles its scale and leaves every code unchanged
    v2 = x["v"][0, 0].copy()
    v2[:, 3] *= 2.0
    h2 = orc.prologue_head(p, x["q"][0, 0], x["k"][0, 0], v2, x["pos"])
    assert np.array_equal(h2["v4"], h["v4"])
    assert h2["sv"][3] == 2 * h["sv"][3]
    assert np.array_equal(np.delete(h2["sv"], 3), np.delete(h["sv"], 3))


def test_quantisation_rounds_the_exact_product_ties_to_even(orc):
    """The INT4 decision is rint, ties to even, of the exact product
    x * fl(7/amax) (a reading: the pages give code = round(x / s) without the
    floating-point steps).  Expected codes come from exact rational arithmetic
    here, not from the oracle: with amax = 7 the reciprocal is 1 and
    2.5, 3.5, -0.5, 1.5, -2.5 are exact ties (to 2, 4, 0, 2, -2; rounding
    half away from zero gives 3, 4, -1, 2, -3); with amax = 2.953125 the
    exact product of 1.0546875 and fl(7/amax) is 2.50000002 (code 3), where
    an fp32-rounded product would be the tie 2.5 (code 2)."""
    from fractions import Fraction
    sp = SPLITS[0]
    p = orc.problem(D=sp["D"], seg=sp["seg"], grid=sp["grid"], rot=1, block_k=16)
    pos = si.positions(sp["grid"])
    N = len(pos)
    v = np.zeros((N, sp["D"]), np.float32)
    col0 = [2.953125, 1.0546875, -1.0546875]
    col1 = [7.0, 2.5, 3.5, -0.5, 1.5, -2.5]
    v[:len(col0), 0] = col0
    v[:len(col1), 1] = col1
    q = np.zeros((N, sp["D"]), np.float32)
    h = orc.prologue_head(p, q, q, v, pos)
    c = orc.unpack_codes(h["v4"]).astype(int)

    def code(x, amax):
        inv = np.float32(7.0) / np.float32(amax)          # fl(7/amax)
        y = Fraction(float(np.float32(x))) * Fraction(float(inv))
        r = round(y)                                        # Python rounds ties to even
        return max(-7, min(7, r))

    assert [code(x, col0[0]) for x in col0] == [7, 3, -3]
    assert [code(x, 7.0) for x in col1] == [7, 2, 4, 0, 2, -2]
    assert list(c[:len(col0), 0]) == [7, 3, -3]
    assert list(c[:len(col1), 1]) == [7, 2, 4, 0, 2, -2]


def test_k_mean_and_colsum(orc):
    wl, p, x, h = _head(orc, "small")
    mean = h["k_rot"].astype(np.float64).mean(axis=0)
    assert np.allclose(h["kmean"], mean, rtol=1e-6, atol=1e-7)
    v = orc.unpack_codes(h["v4"]).astype(np.int64)
    nb = -(-wl.N // wl.block_k)
    ref = np.stack([v[t * wl.block_k:(t + 1) * wl.block_k].sum(axis=0) for t in range(nb)])
    assert np.array_equal(h["colsum"], ref)
    sv_ref = np.abs(x["v"][0, 0]).max(axis=0) / 7.0
    assert np.allclose(h["sv"], sv_ref, rtol=1e-6)


def test_zero_rows_quantise_to_zero(orc):
    sp = SPLITS[0]
    p = orc.problem(D=sp["D"], seg=sp["seg"], grid=sp["grid"], rot=1, block_k=16)
    pos = si.positions(sp["grid"])
    N = len(pos)
    rng = np.random.default_rng(2)
    q = rng.standard_normal((N, sp["D"])).astype(np.float32)
    q[3] = 0.0
    v = rng.standard_normal((N, sp["D"])).astype(np.float32)
    v[:, 5] = 0.0
    h = orc.prologue_head(p, q, q, v, pos)
    assert h["sq"][3] == 0.0 and not h["q4"][3].any()
    assert h["sv"][5] == 0.0 and not orc.unpack_codes(h["v4"])[:, 5].any()


# --- P codes (key design 2) --------------------------------------------------

def test_p_code_golden_table(orc):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "p_codes.txt")) if l.strip() and l[0] != "#"]
    for P, code in rows:
        P = float(P)
        S = np.float32(-np.inf) if P == 0.0 else np.float32(math.log(P))
        assert orc.p_code(float(S), 0.0) == int(code), (P, code)


def test_p_code_extremes(orc):
    assert orc.p_code(1.5, 1.5) == 7           # P = 1 -> 7
    assert orc.p_code(-40.0, 0.0) == -8        # P -> 0 -> -8
    assert orc.p_code(float("-inf"), 0.0) == -8


def test_all_sixteen_p_levels_used(orc):
    wl, p, x, h = _head(orc, "small")
    r = orc.attention_int4_rows(p, h, 0, wl.N, dumps=True)
    assert np.unique(r["codes"]).tolist() == list(range(-8, 8))


# --- attention: integer accumulators, recurrence, brute force ---------------

def test_s_int_and_acc_are_exact_integer_products(orc):
    wl, p, x, h = _head(orc, "small")
    r = orc.attention_int4_rows(p, h, 0, 64, dumps=True)
    q = orc.unpack_codes(h["q4"]).astype(np.int64)
    k = orc.unpack_codes(h["k4"]).astype(np.int64)
    v = orc.unpack_codes(h["v4"]).astype(np.int64)
    assert np.array_equal(r["s_int"], q[:64] @ k.T)
    c = r["codes"].astype(np.int64)
    Bk = wl.block_k
    for t in range(-(-wl.N // Bk)):
        sl = slice(t * Bk, (t + 1) * Bk)
        assert np.array_equal(r["acc"][:, t], (c[:, sl] + 8) @ v[sl])


@pytest.mark.parametrize("N,Bk", [(37, 8), (64, 16), (100, 64), (129, 128)])
def test_blocked_recurrence_equals_softmax(orc, N, Bk):
    """With quantisation off, the blocked online softmax equals softmax attention."""
    rng = np.random.default_rng(N)
    D = 64
    p = orc.problem(N=N, D=D, seg=(24, 20, 20), grid=(1, 1, N), rot=0, block_k=Bk)
    q = rng.standard_normal((N, D)) * 2
    k = rng.standard_normal((N, D)) * 2
    v = rng.standard_normal((N, D))
    out, lse = orc.attention_exact_blocked_rows(p, q, k, v)
    s = q @ k.T / math.sqrt(D)
    ref = orc.reference_attention_fp64(q, k, v)
    assert np.abs(out - ref).max() <= 1e-12
    lse_ref = s.max(1) + np.log(np.exp(s - s.max(1, keepdims=True)).sum(1))
    assert np.abs(lse - lse_ref).max() <= 1e-12


def _brute_force_quantised(wl, h, rows):
    """Unblocked closed form of the INT4 path: every key j of block t(j) gets
    code c_ij = rint(15 exp(S_ij - M_i(t))) - 8 against the running maximum
    M_i(t) = max over blocks <= t, and weight exp(M_i(t) - M_i(last)); the output
    is sum_j w_ij (c_ij + 8) s_v v_j / sum_j w_ij (c_ij + 8)."""
    from oracle import unpack_codes
    N, D, Bk = wl.N, wl.D, wl.block_k
    q = unpack_codes(h["q4"]).astype(np.int64)
    k = unpack_codes(h["k4"]).astype(np.int64)
    v = unpack_codes(h["v4"]).astype(np.float64) * h["sv"].astype(np.float64)
    S_int = q[rows] @ k.T
    ci = np.float32(h["sq"][rows]) * np.float32(1.0 / math.sqrt(D))
    S = (S_int.astype(np.float32) * h["sk"][None, :].astype(np.float32)) * ci[:, None]
    nb = -(-N // Bk)
    bmax = np.stack([S[:, t * Bk:(t + 1) * Bk].max(axis=1) for t in range(nb)], axis=1)
    run = np.maximum.accumulate(bmax, axis=1)
    M = np.repeat(run, Bk, axis=1)[:, :N]
    codes = np.rint(15.0 * np.exp(S.astype(np.float64) - M.astype(np.float64))) - 8
    w = np.exp(M.astype(np.float64) - run[:, -1:].astype(np.float64)) * (codes + 8)
    return (w @ v) / w.sum(axis=1, keepdims=True), codes


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_blocked_int4_equals_unblocked_brute_force(orc, name):
    wl, p, x, h = _head(orc, name)
    rows = np.arange(min(wl.N, 96))
    r = orc.attention_int4_rows(p, h, 0, len(rows), dumps=True)
    ref, codes = _brute_force_quantised(wl, h, rows)
    assert np.array_equal(r["codes"], codes.astype(np.int8))
    assert np.abs(r["out"] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_block_local_max_would_differ(orc):
    """The running maximum matters: codes against each block's own maximum differ."""
    wl, p, x, h = _head(orc, "small")
    r = orc.attention_int4_rows(p, h, 0, 32, dumps=True)
    from oracle import unpack_codes
    q = unpack_codes(h["q4"]).astype(np.int64)[:32]
    k = unpack_codes(h["k4"]).astype(np.int64)
    S = ((q @ k.T).astype(np.float32) * h["sk"][None, :]) * (h["sq"][:32] * np.float32(1 / math.sqrt(wl.D)))[:, None]
    Bk = wl.block_k
    local = np.concatenate([np.rint(15 * np.exp(S[:, t:t + Bk] - S[:, t:t + Bk].max(1, keepdims=True))) - 8
                            for t in range(0, wl.N, Bk)], axis=1)
    assert not np.array_equal(local.astype(np.int8), r["codes"])


def test_k_smoothing_leaves_softmax_unchanged(orc):
    wl, p, x, h = _head(orc, "small")
    q = h["q_rot"].astype(np.float64)
    k = h["k_rot"].astype(np.float64)
    v = x["v"][0, 0].astype(np.float64)
    a = orc.reference_attention_fp64(q, k, v)
    b = orc.reference_attention_fp64(q, k - h["kmean"][None, :].astype(np.float64), v)
    assert np.abs(a - b).max() <= 1e-12


# --- method accuracy (a property of the method, established by the oracle) ---

def _cosine(a, b):
    return float((a * b).sum() / np.linalg.norm(a) / np.linalg.norm(b))


@pytest.mark.parametrize("name,floor", [("tiny", 0.96), ("small", 0.95)])
def test_method_cosine_against_fp64(orc, name, floor):
    """Cosine of the INT4 output against unquantised fp64 attention.  The floors
    are what the method reaches on these inputs (each INT4 stage alone costs
    1-2%); the 0.99 target is not reached at the attention level."""
    wl, p, x, h = _head(orc, name)
    r = orc.attention_int4_rows(p, h, 0, wl.N)
    ref = orc.reference_attention_fp64(h["q_rot"], h["k_rot"], x["v"][0, 0])
    assert _cosine(r["out"], ref) >= floor


def test_half_rotation_beats_no_rotation(orc):
    """Papernotes page, main table: with outliers in the first half of each
    segment, half rotation gives the better INT4 accuracy."""
    wl = si.WORKLOADS["small"]
    x = si.make_inputs(wl, heads=(0,))
    cos = {}
    for rot in (0, 2):
        p = orc.problem(wl.with_(rot=rot))
        h = orc.prologue_head(p, x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], x["pos"], want_rot=True)
        r = orc.attention_int4_rows(p, h, 0, wl.N)
        ref = orc.reference_attention_fp64(h["q_rot"], h["k_rot"], x["v"][0, 0])
        cos[rot] = _cosine(r["out"], ref)
    assert cos[2] > cos[0]


def test_rotation_ranking_at_the_wan_shape(orc):
    """At the Wan-like shape (N = 32760, segments 44/42/42), sampled query rows
    of one head: half rotation beats no rotation and the full D x D Hadamard
    beats both (papernotes page, main table and ablation on rotation
    granularity), for the method's P codes and denominator."""
    wl = si.WORKLOADS["wan"]
    x = si.make_inputs(wl, heads=(0,))
    q, k, v, pos = x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], x["pos"]
    p0 = orc.problem(wl.with_(rot=0))
    rows = np.r_[0:128, wl.N - 128:wl.N]
    ref = orc.reference_attention_fp64(orc.rope_rotate(p0, q, pos)[rows], orc.rope_rotate(p0, k, pos), v)
    cos = {}
    for rot in (0, 2, 3):
        p = orc.problem(wl.with_(rot=rot))
        h = orc.prologue_head(p, q, k, v, pos)
        out = np.concatenate([orc.attention_int4_rows(p, h, 0, 128)["out"],
                              orc.attention_int4_rows(p, h, wl.N - 128, wl.N)["out"]])
        cos[rot] = _cosine(out, ref)
    assert cos[2] > cos[0] and cos[3] > cos[2], cos


def test_given_codes_entry(orc):
    """Attention on supplied P codes: its own codes reproduce it exactly; a
    flipped code changes the output as the unblocked closed form says."""
    wl, p, x, h = _head(orc, "small")
    R = 64
    r = orc.attention_int4_rows(p, h, 0, R, dumps=True)
    same = orc.attention_int4_rows_given_codes(p, h, r["codes"], 0, R)
    assert np.array_equal(same["out"], r["out"]) and np.array_equal(same["lse"], r["lse"])
    codes = r["codes"].copy()
    i, j = 5, int(np.nonzero(codes[5] < 7)[0][0])
    codes[i, j] += 1
    flipped = orc.attention_int4_rows_given_codes(p, h, codes, 0, R)["out"]
    # closed form with the flipped code
    ref, ref_codes = _brute_force_quantised(wl, h, np.arange(R))
    from oracle import unpack_codes
    v = unpack_codes(h["v4"]).astype(np.float64) * h["sv"].astype(np.float64)
    q = unpack_codes(h["q4"]).astype(np.int64)
    k = unpack_codes(h["k4"]).astype(np.int64)
    ci = np.float32(h["sq"][i]) * np.float32(1.0 / math.sqrt(wl.D))
    S = ((q[i] @ k.T).astype(np.float32) * h["sk"].astype(np.float32)) * ci
    Bk = wl.block_k
    nb = -(-wl.N // Bk)
    run = np.maximum.accumulate(np.array([S[t * Bk:(t + 1) * Bk].max() for t in range(nb)]))
    M = np.repeat(run, Bk)[:wl.N].astype(np.float64)
    w = np.exp(M - run[-1]) * (codes[i].astype(np.float64) + 8)
    expect = (w @ v) / w.sum()
    assert np.abs(flipped[i] - expect).max() <= 1e-12 * np.abs(expect).max()
    others = np.arange(R) != i
    assert np.array_equal(flipped[others], r["out"][others])


# --- ablation switches (reading R11): block-local max, symmetric P, fp32 l ---

def _brute_force_modes(wl, h, rows, p_mode, l_mode):
    """Unblocked closed form of the INT4 path under the ablation switches.

    Key j of block t(j) is coded against M_c = the block's own maximum (LOCAL)
    or the running maximum after its block (otherwise); its weight relative to
    the final maximum is exp(M_c - M_final).  Range codes are rint(15 e) - 8
    dequantised as (c + 8) / 15, symmetric codes rint(7 e) dequantised as c / 7,
    e = exp(S - M_c).  Output = sum_j w_j P_j s_v v_j / sum_j w_j L_j with
    P_j the dequantised code and L_j = P_j (code denominator) or e_j (fp32)."""
    from oracle import P_LOCAL, P_SYMMETRIC, L_FP32, unpack_codes
    N, D, Bk = wl.N, wl.D, wl.block_k
    q = unpack_codes(h["q4"]).astype(np.int64)
    k = unpack_codes(h["k4"]).astype(np.int64)
    v = unpack_codes(h["v4"]).astype(np.float64) * h["sv"].astype(np.float64)
    ci = np.float32(h["sq"][rows]) * np.float32(1.0 / math.sqrt(D))
    S = ((q[rows] @ k.T).astype(np.float32) * h["sk"][None, :].astype(np.float32)) * ci[:, None]
    nb = -(-N // Bk)
    bmax = np.stack([S[:, t * Bk:(t + 1) * Bk].max(axis=1) for t in range(nb)], axis=1)
    run = np.maximum.accumulate(bmax, axis=1)
    Mc = np.repeat(bmax if p_mode == P_LOCAL else run, Bk, axis=1)[:, :N].astype(np.float64)
    e = np.exp(S.astype(np.float64) - Mc)
    if p_mode == P_SYMMETRIC:
        codes = np.rint(7.0 * e)
        deq = codes / 7.0
    else:
        codes = np.rint(15.0 * e) - 8
        deq = (codes + 8) / 15.0
    w = np.exp(Mc - run[:, -1:].astype(np.float64))
    den = (w * (e if l_mode == L_FP32 else deq)).sum(axis=1, keepdims=True)
    return ((w * deq) @ v) / den, codes


@pytest.mark.parametrize("name", ["tiny", "small"])
@pytest.mark.parametrize("p_mode,l_mode", [(0, 1), (1, 0), (1, 1), (2, 0), (2, 1)])
def test_ablation_switches_equal_unblocked_brute_force(orc, name, p_mode, l_mode):
    wl, _, x, h = _head(orc, name)
    p = orc.problem(wl, p_mode=p_mode, l_mode=l_mode)
    rows = np.arange(min(wl.N, 96))
    r = orc.attention_int4_rows(p, h, 0, len(rows), dumps=True)
    ref, codes = _brute_force_modes(wl, h, rows, p_mode, l_mode)
    assert np.array_equal(r["codes"], codes.astype(np.int8))
    assert np.abs(r["out"] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_brute_force_modes_reduce_to_the_range_path(orc):
    """The generalised closed form, switches off, is the range-rectified one."""
    wl, p, x, h = _head(orc, "small")
    rows = np.arange(64)
    a, ca = _brute_force_modes(wl, h, rows, 0, 0)
    b, cb = _brute_force_quantised(wl, h, rows)
    assert np.array_equal(ca, cb) and np.abs(a - b).max() <= 1e-14 * np.abs(b).max()


def test_local_max_with_one_block_is_the_running_max(orc):
    """With a single key block the block maximum is the running maximum."""
    wl, _, x, h = _head(orc, "tiny")
    for l_mode in (0, 1):
        pb, pl = orc.problem(wl, l_mode=l_mode), orc.problem(wl, p_mode=1, l_mode=l_mode)
        pb.block_k = pl.block_k = wl.N
        base = orc.attention_int4_rows(pb, h, 0, wl.N, dumps=True)
        loc = orc.attention_int4_rows(pl, h, 0, wl.N, dumps=True)
        assert np.array_equal(base["codes"], loc["codes"])
        assert np.array_equal(base["out"], loc["out"]) and np.array_equal(base["lse"], loc["lse"])


def test_local_max_codes_differ_and_reach_seven_in_every_block(orc):
    """Against its own maximum every block has a key with P = 1 (code 7)."""
    wl, _, x, h = _head(orc, "small")
    r = orc.attention_int4_rows(orc.problem(wl, p_mode=1), h, 0, 32, dumps=True)
    base = orc.attention_int4_rows(orc.problem(wl), h, 0, 32, dumps=True)
    assert not np.array_equal(r["codes"], base["codes"])
    Bk = wl.block_k
    for t in range(0, wl.N, Bk):
        assert (r["codes"][:, t:t + Bk].max(axis=1) == 7).all()


def test_symmetric_codes_use_levels_zero_to_seven(orc):
    """SageAttention-style P: rint(7 P), levels 0..7 only, P = 1 -> 7, P -> 0 -> 0."""
    assert orc.p_code_sym(2.0, 2.0) == 7
    assert orc.p_code_sym(-40.0, 0.0) == 0 and orc.p_code_sym(float("-inf"), 0.0) == 0
    for seven_p, code in ((3.6, 4), (3.4, 3), (1.4, 1), (0.55, 1), (0.45, 0), (6.6, 7)):
        assert orc.p_code_sym(float(np.float32(math.log(seven_p / 7))), 0.0) == code, seven_p
    wl, _, x, h = _head(orc, "small")
    r = orc.attention_int4_rows(orc.problem(wl, p_mode=2), h, 0, wl.N, dumps=True)
    assert np.unique(r["codes"]).tolist() == list(range(0, 8))


def test_symmetric_acc_has_no_zero_point(orc):
    wl, _, x, h = _head(orc, "small")
    r = orc.attention_int4_rows(orc.problem(wl, p_mode=2), h, 0, 64, dumps=True)
    v = orc.unpack_codes(h["v4"]).astype(np.int64)
    c = r["codes"].astype(np.int64)
    Bk = wl.block_k
    for t in range(-(-wl.N // Bk)):
        sl = slice(t * Bk, (t + 1) * Bk)
        assert np.array_equal(r["acc"][:, t], c[:, sl] @ v[sl])


def test_uniform_row_gives_the_mean_of_v_in_every_mode(orc):
    """A zero query row has S = 0 for every key: every mode gives the mean of
    the dequantised V and lse = ln N (fp32 l) or ln(N * 15 / 15) = ln N."""
    wl, _, x, h = _head(orc, "small")
    h = dict(h)
    h["q4"] = h["q4"].copy()
    h["sq"] = h["sq"].copy()
    h["q4"][3] = 0          # what the prologue emits for an all-zero query token
    h["sq"][3] = 0.0
    mean = (orc.unpack_codes(h["v4"]).astype(np.float64) * h["sv"].astype(np.float64)).mean(axis=0)
    for p_mode in (0, 1, 2):
        for l_mode in (0, 1):
            r = orc.attention_int4_rows(orc.problem(wl, p_mode=p_mode, l_mode=l_mode), h, 3, 4)
            assert np.abs(r["out"][0] - mean).max() <= 1e-12 * np.abs(mean).max(), (p_mode, l_mode)
            assert abs(r["lse"][0] - math.log(wl.N)) <= 1e-12, (p_mode, l_mode)


def test_fp32_l_changes_only_the_denominator(orc):
    """Same codes and numerator: the two outputs of a row differ by one factor."""
    wl, _, x, h = _head(orc, "small")
    for p_mode in (0, 1, 2):
        a = orc.attention_int4_rows(orc.problem(wl, p_mode=p_mode), h, 0, 64, dumps=True)
        b = orc.attention_int4_rows(orc.problem(wl, p_mode=p_mode, l_mode=1), h, 0, 64, dumps=True)
        assert np.array_equal(a["codes"], b["codes"])
        ratio = np.exp(a["lse"] - b["lse"])          # l_codes / l_fp32
        assert np.abs(b["out"] - a["out"] * ratio[:, None]).max() <= 1e-12 * np.abs(a["out"]).max()
        assert np.all(ratio > 0) and not np.allclose(ratio, 1.0)


# --- full D x D Hadamard rotation (the pages' ablation; a third rotation mode) ---

@pytest.mark.parametrize("D", [64, 128])
def test_full_rotation_is_the_normalised_sylvester_hadamard(orc, D):
    """The oracle's matrix equals scipy's Sylvester Hadamard matrix / sqrt(D)."""
    from scipy.linalg import hadamard
    sp = SPLITS[0] if D == 64 else SPLITS[1]
    R = orc.rotation_matrix(_prob(orc, 3, sp))
    assert np.array_equal(R, hadamard(D).astype(np.float64) / math.sqrt(D))


def test_full_rotation_mixes_every_channel(orc):
    """Unlike the 2x2 rotations, every output channel depends on every input."""
    sp = SPLITS[1]
    p = _prob(orc, 3, sp, N=1)
    pos = si.positions(sp["grid"])[:1]
    for d in (0, 63, 127):
        x = np.zeros((1, sp["D"]), np.float32)
        x[0, d] = 1.0
        y = orc.rope_rotate(p, x, pos)   # position (0, 0, 0): RoPE is the identity
        assert np.all(np.abs(np.abs(y) - 1 / math.sqrt(sp["D"])) <= 1e-7)


def test_full_rotation_butterflies_follow_the_stated_order(orc):
    """fp32 transform equals the same butterfly sequence written out in numpy
    float32 (stage distances 1, 2, ..., D/2, then one scaling)."""
    sp = SPLITS[1]
    p = _prob(orc, 3, sp, N=1)
    pos = si.positions(sp["grid"])[:1]
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, sp["D"])).astype(np.float32) * np.float32(20)
    y = orc.rope_rotate(p, x, pos)[0]
    z = x[0].copy()
    d = 1
    while d < sp["D"]:
        idx = np.array([i for i in range(sp["D"]) if not i & d])
        a, b = z[idx].copy(), z[idx + d].copy()
        z[idx], z[idx + d] = a + b, a - b
        d *= 2
    z = z * np.float32(1 / math.sqrt(sp["D"]))
    assert np.array_equal(y, z)


def test_full_rotation_flattens_outlier_channels(orc):
    """Hadamard spreads the outlier channels over all channels: the per-token
    amax relative to the RMS falls (what makes INT4 codes finer)."""
    wl = si.WORKLOADS["small"]
    x = si.make_inputs(wl, heads=(0,))
    ratio = {}
    for rot in (0, 3):
        p = orc.problem(wl.with_(rot=rot))
        y = orc.rope_rotate(p, x["q"][0, 0], x["pos"]).astype(np.float64)
        ratio[rot] = np.mean(np.abs(y).max(1) / np.sqrt((y ** 2).mean(1)))
    assert ratio[3] < 0.6 * ratio[0]
