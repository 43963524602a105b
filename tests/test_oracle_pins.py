"""Pins of the CPU oracle to things other than itself (no GPU).

Each test checks the oracle against what the pages print, a closed form, an
invariant, a library routine the step reduces to, or brute force on tiny inputs.
"""
import itertools
import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synthetic as syn

H, I = 2816, 704


def f32(x):
    return struct.unpack("<f", struct.pack("<f", x))[0]


def ulp_dist(a: float, b: float) -> int:
    ia = struct.unpack("<i", struct.pack("<f", a))[0]
    ib = struct.unpack("<i", struct.pack("<f", b))[0]
    if ia < 0:
        ia = -(ia & 0x7FFFFFFF)
    if ib < 0:
        ib = -(ib & 0x7FFFFFFF)
    return abs(ia - ib)


# ----------------------------------------------------------------- expert sizes

def test_expert_bytes_match_the_pages(golden_dir):
    """prain README, 'Expert formats': 11.34 / 5.69 / 3.01 MiB per expert and
    42.5 / 21.3 / 11.3 GiB for all 30 x 128 experts."""
    g = json.load(open(os.path.join(golden_dir, "expert_sizes.json")))
    n = g["layers"] * g["experts_per_layer"]
    for name, fmt in oracle.FMT_NAMES.items():
        b = oracle.expert_bytes(fmt, H, I)
        assert round(b / 2**20, 2) == g["formats"][name]["expert_mib"], name
        assert round(b * n / 2**30, 1) == g["formats"][name]["all_gib"], name


def test_expert_bytes_closed_form():
    """3*H*I weights per expert; bf16 2 B each; int8 1 B + fp32 per row (2I + H rows);
    int4 half a byte + one bf16 scale per 64 weights."""
    for h, i in [(2816, 704), (256, 128), (64, 64), (1024, 192)]:
        w = 3 * h * i
        assert oracle.expert_bytes(oracle.BF16, h, i) == 2 * w
        assert oracle.expert_bytes(oracle.INT8, h, i) == w + 4 * (2 * i + h)
        assert oracle.expert_bytes(oracle.INT4, h, i) == w // 2 + 2 * (w // 64)
    assert oracle.expert_bytes(oracle.BF16, H, I) == 11894784
    assert oracle.expert_bytes(oracle.INT8, H, I) == 5964288
    assert oracle.expert_bytes(oracle.INT4, H, I) == 3159552


def test_blob_pieces_are_contiguous_and_16_byte_aligned():
    for fmt in (0, 1, 2):
        off = oracle.blob_offsets(fmt, H, I)
        assert off[0] == 0 and off == sorted(off)
        assert all(o % 256 == 0 for o in off)
        assert oracle.expert_bytes(fmt, H, I) % 256 == 0


# ------------------------------------------------------------------------ exp_p

def test_exp_p_within_two_ulp_of_libm():
    xs = np.concatenate([
        np.linspace(-103.0, 88.0, 20001, dtype=np.float32),
        -np.abs(np.random.default_rng(1).standard_normal(20000).astype(np.float32)) * 8,
        np.float32([0.0, -0.0, -1e-30, 1e-30, -0.5 * math.log(2), 0.5 * math.log(2), -87.3, -86.0]),
    ])
    worst = 0
    for x in xs:
        ref = f32(math.exp(float(x)))
        got = oracle.exp_p(float(x))
        if ref == 0.0:
            assert got == 0.0 or got < 2e-45
            continue
        worst = max(worst, ulp_dist(got, ref))
    assert worst <= 2, worst


def test_exp_p_special_values_and_monotone():
    assert oracle.exp_p(0.0) == 1.0
    assert oracle.exp_p(-0.0) == 1.0
    assert oracle.exp_p(float("-inf")) == 0.0
    assert oracle.exp_p(-200.0) == 0.0
    assert math.isinf(oracle.exp_p(100.0))
    assert math.isnan(oracle.exp_p(float("nan")))
    xs = np.linspace(-20, 0, 40001, dtype=np.float32)
    ys = oracle.exp_p_array(xs)
    assert np.all(np.diff(ys.astype(np.float64)) >= 0)


# ------------------------------------------------------------------------- gelu

def test_gelu_tanh_matches_torch():
    v = np.linspace(-8, 8, 4001)
    ref = torch.nn.functional.gelu(torch.tensor(v, dtype=torch.float64), approximate="tanh").numpy()
    got = np.array([oracle.gelu_tanh(x) for x in v])
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-15)
    assert oracle.gelu_tanh(0.0) == 0.0
    assert abs(oracle.gelu_tanh(30.0) - 30.0) < 1e-12
    assert abs(oracle.gelu_tanh(-30.0)) < 1e-12


# ---------------------------------------------------------------------- routing

def test_route_k1_weight_is_one_and_id_is_argmax():
    lg = syn.router_logits(64, 128, "normal", seed=3)
    ids, w = oracle.route_topk(lg, 1)
    assert np.all(w == 1.0)
    assert np.array_equal(ids[:, 0], np.argmax(lg, axis=1))


def test_route_ids_equal_stable_descending_sort():
    """Ties to the lower expert id: the order of a stable sort of -logit."""
    rng = np.random.default_rng(5)
    lg = rng.integers(-3, 4, size=(200, 16)).astype(np.float32)  # many ties
    for k in (1, 2, 5, 16):
        ids, _ = oracle.route_topk(lg, k)
        ref = np.argsort(-lg, axis=1, kind="stable")[:, :k]
        assert np.array_equal(ids, ref)


def test_route_all_equal_logits():
    ids, w = oracle.route_topk(np.zeros((3, 8), np.float32), 4)
    assert np.array_equal(ids, np.tile(np.arange(4), (3, 1)))
    assert np.all(w == 0.25)


def test_route_brute_force_subsets():
    """E=8: the chosen set maximises the summed logit over every k-subset."""
    lg = syn.router_logits(50, 8, "normal", seed=11)
    for k in (2, 3):
        ids, _ = oracle.route_topk(lg, k)
        for t in range(lg.shape[0]):
            best = max(itertools.combinations(range(8), k), key=lambda s: (sum(lg[t, list(s)]),
                                                                            [-e for e in s]))
            assert sorted(ids[t]) == sorted(best)


def test_route_full_k_is_softmax():
    lg = syn.router_logits(32, 64, "normal", seed=2)
    ids, w = oracle.route_topk(lg, 64)
    z = lg.astype(np.float64)
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ref = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    np.testing.assert_allclose(w, ref, rtol=2e-6, atol=1e-9)
    np.testing.assert_allclose(w.astype(np.float64).sum(axis=1), 1.0, atol=1e-5)


def test_route_topk_renormalised_softmax_fp64():
    """Weights equal softmax over all E, kept to the top k and renormalised (fp64)."""
    lg = syn.router_logits(64, 128, "biased", seed=4)
    ids, w = oracle.route_topk(lg, 8)
    z = lg.astype(np.float64)
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    top = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    ref = top / top.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(w, ref, rtol=3e-6, atol=0)
    assert np.all(np.diff(w, axis=1) <= 0)  # rank order: non-increasing weights


def test_route_nan_ranks_last():
    lg = np.array([[np.nan, 1.0, 0.5, np.nan]], np.float32)
    ids, _ = oracle.route_topk(lg, 4)
    assert ids.tolist() == [[1, 2, 0, 3]]


# ---------------------------------------------------------------------- permute

def test_permute_equals_stable_argsort_and_bincount():
    rng = np.random.default_rng(7)
    for T, k, E in [(37, 3, 11), (1, 8, 128), (64, 8, 128), (5, 1, 2)]:
        ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
        counts, offsets, sr, rp = oracle.permute(ids, E)
        flat = ids.ravel()
        assert np.array_equal(counts, np.bincount(flat, minlength=E))
        assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
        assert np.array_equal(sr, np.argsort(flat, kind="stable"))
        assert np.array_equal(rp[sr], np.arange(T * k))
        # token of a sorted row is route // k (remote_experts.cpp, begin)
        assert np.array_equal(flat[sr], np.repeat(np.arange(E), counts))


def test_permute_drops_out_of_range_ids():
    ids = np.array([[0, 5], [-1, 1], [1, 9]], np.int32)
    counts, offsets, sr, rp = oracle.permute(ids, 3)
    assert counts.tolist() == [1, 2, 0]
    assert offsets.tolist() == [0, 1, 3, 3]
    assert sr.tolist() == [0, 3, 4, -1, -1, -1]
    assert rp.tolist() == [0, -1, -1, 1, 2, -1]


# ------------------------------------------------------------------------- hits

def test_hits_page_vector(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "expert_pool_vectors.json")))["count_hits_matches_bincount"]
    assert oracle.hits(np.array(g["ids"]), g["E"]).tolist() == g["hits"]


def test_hits_is_bincount_ignoring_out_of_range_and_accumulates():
    rng = np.random.default_rng(9)
    ids = rng.integers(-5, 140, size=5000).astype(np.int32)
    ok = ids[(ids >= 0) & (ids < 128)]
    h = oracle.hits(ids, 128)
    assert np.array_equal(h, np.bincount(ok, minlength=128))
    assert np.array_equal(oracle.hits(ids, 128, h), 2 * h)


# ------------------------------------------------------------------- quantisers

def test_int8_exact_on_representable_rows():
    rng = np.random.default_rng(1)
    rows = []
    for j in range(6):
        m = rng.integers(-127, 128, size=256)
        m[rng.integers(0, 256)] = 127 * (1 if j % 2 else -1)
        rows.append(m * 2.0 ** (-3 - j))
    w = syn.bf16_bits(np.array(rows, np.float32))
    q, s = oracle.quantize_int8(w)
    for j in range(6):
        assert s[j] == np.float32(2.0 ** (-3 - j))
        assert np.array_equal(q[j].astype(np.int64) * 1.0 * 2.0 ** (-3 - j), syn.bf16_to_f32(w[j]))


def test_int8_zero_row_and_error_bound():
    w = syn.normal_bf16((64, 512), 0.02, 3, 0)
    w[5] = 0
    q, s = oracle.quantize_int8(w)
    assert s[5] == 0 and np.all(q[5] == 0)
    wf = syn.bf16_to_f32(w).astype(np.float64)
    err = np.abs(wf - q.astype(np.float64) * s[:, None].astype(np.float64))
    # |w/s| <= 127, so the fp32 quotient carries at most 127 * 2^-24 of rounding
    assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 127 * 2.0**-24) + 1e-30)
    assert np.all(np.abs(q) <= 127)
    assert np.all(np.abs(q).max(axis=1)[s > 0] == 127)


def _unpack_int4(qb: np.ndarray) -> np.ndarray:
    lo = (qb & 15).astype(np.int64) - 8
    hi = (qb >> 4).astype(np.int64) - 8
    out = np.empty(qb.shape[:-1] + (qb.shape[-1] * 2,), np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def test_int4_nibble_layout_and_exact_groups():
    """Groups that are m * s with |m| <= 7 (some |m| = 7) and s a bf16 value come
    back exactly; byte j carries weight 2j low and 2j+1 high."""
    rng = np.random.default_rng(2)
    rows = []
    scales = []
    for r in range(8):
        # a 5-bit mantissa keeps every m * s (|m| <= 7) exact in bf16
        s = float(rng.integers(16, 32)) * 2.0 ** -int(rng.integers(8, 14))
        m = rng.integers(-7, 8, size=128)
        m[3] = 7
        m[64 + 5] = -7
        rows.append(m * s)
        scales.append(s)
    w = syn.bf16_bits(np.array(rows, np.float32))
    assert np.array_equal(syn.bf16_to_f32(w).astype(np.float64), np.array(rows))
    q, sb = oracle.quantize_int4(w)
    sf = syn.bf16_to_f32(sb)
    for r in range(8):
        assert sf[r, 0] == np.float32(scales[r]) and sf[r, 1] == np.float32(scales[r])
        deq = _unpack_int4(q[r]) * float(scales[r])
        assert np.array_equal(deq, np.array(rows[r]))
    # explicit nibble order on a hand example
    s = 2.0 ** -6
    m = np.array([(c % 15) - 7 for c in range(64)])
    q1, _ = oracle.quantize_int4(syn.bf16_bits(np.float32(m * s))[None, :])
    assert q1[0, 0] == ((m[0] + 8) | ((m[1] + 8) << 4))
    assert q1[0, 31] == ((m[62] + 8) | ((m[63] + 8) << 4))


def _exact_err(w64: np.ndarray, s: float) -> Fraction:
    """Exact sum of squared residuals with the best codes in [-8, 7] for scale s."""
    tot = Fraction(0)
    sF = Fraction(s)
    for v in w64:
        vF = Fraction(float(v))
        best = min((abs(vF - m * sF) for m in range(-8, 8)))
        tot += best * best
    return tot


def test_int4_clip_search_is_the_mse_argmin():
    """For each group: every candidate error is the exact error of the best codes
    for its scale (to fp64 rounding), candidate scales are r * absmax / 7 for
    ratios running 0.70 .. 1.00, and the stored scale is the strict argmin with
    ties kept at the larger ratio."""
    w = syn.normal_bf16((3, 64 * 6), 0.02, 9, 1)
    q, sb = oracle.quantize_int4(w)
    sf = syn.bf16_to_f32(sb)
    for r in range(3):
        for g in range(6):
            w64 = w[r, g * 64:(g + 1) * 64]
            wf = syn.bf16_to_f32(w64).astype(np.float64)
            amax = np.abs(wf).max()
            s_c, e_c = oracle.int4_candidates(w64)
            ratios = s_c / (amax / 7.0)
            assert np.all(np.diff(s_c) >= 0)
            assert abs(ratios[0] - 0.70) < 0.01 and abs(ratios[15] - 1.0) < 0.01
            for i in range(16):
                ex = float(_exact_err(wf, float(s_c[i])))
                assert abs(e_c[i] - ex) <= 1e-12 * max(ex, 1e-30) + 1e-300
            best = min(range(15, -1, -1), key=lambda i: (e_c[i], -i))
            assert sf[r, g] == s_c[best]
            # stored codes are the nearest codes for the stored scale
            deq = _unpack_int4(q[r, g * 32:(g + 1) * 32]) * float(sf[r, g])
            assert float(sum(Fraction(float(a)) ** 2 for a in (wf - deq))) == pytest.approx(
                float(_exact_err(wf, float(sf[r, g]))), rel=1e-12, abs=1e-300)
    # on Gaussian weights clipping usually pays: most groups keep a ratio below 1.0,
    # and no chosen error exceeds the unclipped (ratio 1.0) candidate's
    wg = syn.normal_bf16((8, 64 * 44), 0.02, 9, 2)
    _, sbg = oracle.quantize_int4(wg)
    sfg = syn.bf16_to_f32(sbg)
    clipped = 0
    for r in range(8):
        for g in range(44):
            s_c, e_c = oracle.int4_candidates(wg[r, g * 64:(g + 1) * 64])
            i = int(np.nonzero(s_c == sfg[r, g])[0][-1])
            assert e_c[i] <= e_c[15]
            clipped += sfg[r, g] < s_c[15]
    assert clipped > 0.5 * 8 * 44


def test_int4_zero_group():
    w = np.zeros((1, 64), np.uint16)
    q, s = oracle.quantize_int4(w)
    assert s[0, 0] == 0 and np.all(q == 0x88)


def _torch_bf16_bits(u32: np.ndarray) -> np.ndarray:
    """fp32 bit patterns -> bf16 bit patterns by torch's own conversion."""
    f = torch.from_numpy(np.ascontiguousarray(u32, np.uint32).view(np.float32).copy())
    return f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_rounding_matches_torch_conversion():
    """The oracle's fp32 -> bf16 rounding (it fixes every int4 scale: prain README,
    'Expert formats', bf16 scale per 64 weights) equals torch's float32 ->
    bfloat16 conversion bit for bit: exact ties with an even and an odd kept
    part, one ulp either side of a tie, subnormals, values that round up to
    +-inf, +-0, +-inf, the largest finite values, and random patterns.  NaN stays
    NaN.  A truncating or ties-away rounding fails here."""
    pats = []
    rng = np.random.default_rng(7)
    hi = rng.integers(0, 1 << 16, size=3000, dtype=np.uint32)
    for lo in (0x8000, 0x7FFF, 0x8001, 0x0000, 0xFFFF, 0x0001):
        pats.append((hi << 16) | lo)                      # ties, both parities of hi; one ulp around them
    pats.append(rng.integers(0, 1 << 32, size=20000, dtype=np.uint64).astype(np.uint32))
    sub = rng.integers(1, 0x00800000, size=2000, dtype=np.uint32)
    pats.append(sub)                                      # positive subnormals
    pats.append(sub | 0x80000000)                         # negative subnormals
    pats.append(np.array([0x00008000, 0x00018000, 0x007F8000, 0x007FFFFF, 0x00800000, 0x80008000,
                          0x7F7F7FFF, 0x7F7F8000, 0x7F7FFFFF, 0x7F7E8000, 0xFF7F8000, 0xFF7FFFFF,
                          0x7F800000, 0xFF800000, 0x00000000, 0x80000000, 0x3F808000, 0x3F818000],
                         np.uint32))
    u = np.concatenate(pats).astype(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    f = u.view(np.float32)
    got = np.array([oracle.bf16_rne(float(v)) for v in f], np.uint16)
    ref = _torch_bf16_bits(u)
    assert np.array_equal(got[~nan], ref[~nan])
    # the overflow cases really reach infinity, and ties really go to even
    assert oracle.bf16_rne(struct.unpack("<f", struct.pack("<I", 0x7F7F8000))[0]) == 0x7F80
    assert oracle.bf16_rne(struct.unpack("<f", struct.pack("<I", 0x3F808000))[0]) == 0x3F80
    assert oracle.bf16_rne(struct.unpack("<f", struct.pack("<I", 0x3F818000))[0]) == 0x3F82
    qn = np.array([0x7FC00000, 0xFFC00001, 0x7F800001, 0xFF812345], np.uint32)
    for v in qn.view(np.float32):
        b = oracle.bf16_rne(float(v))
        assert (b & 0x7F80) == 0x7F80 and (b & 0x007F) != 0      # still a NaN


def test_int4_candidate_scales_are_torch_rounded():
    """Every candidate scale of the clip search is the bf16 rounding of the fp32
    r_i * absmax / 7 (ratios r_i = 0.70, 0.72, ..., 1.00; fp32 multiply, then
    fp32 divide), recomputed here with torch's float32 arithmetic and its
    bfloat16 conversion."""
    for seed in range(6):
        w64 = syn.normal_bf16((64,), 0.02 * (1 + seed), 41, seed)
        amax = torch.tensor(float(np.abs(syn.bf16_to_f32(w64)).max()), dtype=torch.float32)
        s_c, _ = oracle.int4_candidates(w64)
        for i in range(16):
            r = torch.tensor((70 + 2 * i) / 100, dtype=torch.float32)
            t = (r * amax) / torch.tensor(7.0, dtype=torch.float32)
            want = t.to(torch.bfloat16).to(torch.float32).item()
            assert struct.pack("<f", float(s_c[i])) == struct.pack("<f", want), (seed, i)


# ------------------------------------------------------------------ expert FFN

def _tiny_layer(fmt, E=4, h=128, i=64, seed=0):
    w13, w2 = syn.expert_weights(E, h, i, seed=seed)
    blobs = []
    deq13, deq2 = [], []
    for e in range(E):
        if fmt == oracle.BF16:
            blobs.append(oracle.pack_expert(fmt, h, i, w13[e], None, w2[e], None))
            deq13.append(syn.bf16_to_f32(w13[e]).astype(np.float64))
            deq2.append(syn.bf16_to_f32(w2[e]).astype(np.float64))
        elif fmt == oracle.INT8:
            q13, s13 = oracle.quantize_int8(w13[e])
            q2, s2 = oracle.quantize_int8(w2[e])
            blobs.append(oracle.pack_expert(fmt, h, i, q13, s13, q2, s2))
            deq13.append(q13.astype(np.float64) * s13[:, None].astype(np.float64))
            deq2.append(q2.astype(np.float64) * s2[:, None].astype(np.float64))
        else:
            q13, s13 = oracle.quantize_int4(w13[e])
            q2, s2 = oracle.quantize_int4(w2[e])
            blobs.append(oracle.pack_expert(fmt, h, i, q13, s13, q2, s2))
            deq13.append(_unpack_int4(q13) * np.repeat(syn.bf16_to_f32(s13).astype(np.float64), 64, axis=1))
            deq2.append(_unpack_int4(q2) * np.repeat(syn.bf16_to_f32(s2).astype(np.float64), 64, axis=1))
    home = np.concatenate(blobs)
    return oracle.Layer(fmt, E, h, i, home), deq13, deq2


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_single_expert_ffn_is_the_textbook_gemm_gelu_gemm(fmt):
    """One expert, k = 1: GEMM -> GELU-tanh gate * up -> GEMM in torch fp64, from
    weights dequantised independently here (q * s with the page's scale layout)."""
    L, d13, d2 = _tiny_layer(fmt)
    x = syn.activations(5, L.H, seed=1)
    xf = torch.tensor(syn.bf16_to_f32(x).astype(np.float64))
    for e in range(L.E):
        g = xf @ torch.tensor(d13[e]).T
        hh = torch.nn.functional.gelu(g[:, :L.I], approximate="tanh") * g[:, L.I:]
        ref = (hh @ torch.tensor(d2[e]).T).numpy()
        for t in range(5):
            y = oracle.expert_ffn(L, e, x[t])
            np.testing.assert_allclose(y, ref[t], rtol=1e-10, atol=1e-12)


def test_weight_accessor_matches_independent_dequant():
    for fmt in (0, 1, 2):
        L, d13, d2 = _tiny_layer(fmt, E=1)
        rng = np.random.default_rng(fmt)
        for _ in range(50):
            r, c = rng.integers(0, 2 * L.I), rng.integers(0, L.H)
            assert oracle.weight(fmt, L.home, L.H, L.I, 13, r, c) == d13[0][r, c]
            r, c = rng.integers(0, L.H), rng.integers(0, L.I)
            assert oracle.weight(fmt, L.home, L.H, L.I, 2, r, c) == d2[0][r, c]


def test_zero_activation_gives_zero_output():
    L, _, _ = _tiny_layer(0)
    assert np.all(oracle.expert_ffn(L, 1, np.zeros(L.H, np.uint16)) == 0.0)


def test_dense_all_experts_then_mask_equals_routed():
    """Tiny layer (8 experts, hidden 256, intermediate 128, top-2, 16 tokens): every
    expert on every token, then a dense [T, E] weight matrix that is zero off the
    top-k, equals the routed layer."""
    E, h, i, k, T = 8, 256, 128, 2, 16
    L, _, _ = _tiny_layer(0, E=E, h=h, i=i)
    x = syn.activations(T, h, seed=0)
    lg = syn.router_logits(T, E, "normal", seed=0)
    ids, w, rows, y = oracle.moe_layer(L, lg, x, k)
    dense_w = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            dense_w[t, ids[t, j]] = w[t, j]
    allx = np.zeros((T, E, h))
    for t in range(T):
        for e in range(E):
            allx[t, e] = oracle.expert_ffn(L, e, x[t])
    for t in range(T):
        for j in range(k):
            assert np.array_equal(rows[t * k + j], allx[t, ids[t, j]])
    ydense = np.einsum("te,teh->th", dense_w, allx)
    np.testing.assert_allclose(y, ydense, rtol=1e-12, atol=1e-14)


def test_combine_k1_unit_weight_is_identity():
    rows = np.random.default_rng(0).standard_normal((7, 33))
    ids = np.arange(7, dtype=np.int32)[:, None] % 3
    y = oracle.combine(rows, ids, np.ones((7, 1), np.float32), 3)
    assert np.array_equal(y, rows)


def test_slot_table_only_moves_where_blobs_are_read():
    """Router logits and expert ids are untouched by placement (expert_pool.rs,
    module doc): a layer whose experts are served from cache slots gives the same
    rows as the same layer served from home."""
    E, h, i, k, T = 8, 128, 64, 2, 6
    L, _, _ = _tiny_layer(2, E=E, h=h, i=i)
    eb = L.expert_bytes
    slot_of = np.full(E, -1, np.int32)
    slot_of[[5, 1, 6]] = [0, 2, 1]
    pool = np.zeros(3 * eb, np.uint8)
    for e in (5, 1, 6):
        pool[slot_of[e] * eb:(slot_of[e] + 1) * eb] = L.home[e * eb:(e + 1) * eb]
    Ls = oracle.Layer(2, E, h, i, L.home, pool=pool, slot_table=slot_of)
    x = syn.activations(T, h, seed=3)
    lg = syn.router_logits(T, E, "normal", seed=3)
    a = oracle.moe_layer(L, lg, x, k)
    b = oracle.moe_layer(Ls, lg, x, k)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    # and the slot really is what is read: corrupt home of a slotted expert
    home2 = L.home.copy()
    home2[5 * eb:6 * eb] = 0
    Lc = oracle.Layer(2, E, h, i, home2, pool=pool, slot_table=slot_of)
    assert np.array_equal(oracle.moe_layer(Lc, lg, x, k)[3], a[3])


# -------------------------------------------------------------------- placement

def test_placement_page_vectors(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "expert_pool_vectors.json")))
    c = g["target_gpu_picks_top_by_count"]
    assert oracle.refresh_target(np.array(c["counts"], np.uint32), c["budget"]).tolist() == c["target"]

    c = g["paired_swap_limits_demotions"]
    so = np.full(c["E"], -1, np.int32)
    so[c["resident"]] = np.arange(len(c["resident"]))
    so2, pr, de = oracle.apply_placement(so, c["budget"], np.array(c["target"]))
    assert len(pr) == c["promotions"] and len(de) == c["demotions"]
    assert sorted(np.nonzero(so2 >= 0)[0].tolist()) == c["resident_after"]

    c = g["paired_swap_keeps_extra_residents"]
    so = np.full(c["E"], -1, np.int32)
    so[c["resident"]] = np.arange(len(c["resident"]))
    so2, pr, de = oracle.apply_placement(so, c["budget"], np.array(c["target"]))
    assert len(pr) == c["promotions"] and len(de) == c["demotions"]
    assert int((so2 >= 0).sum()) == c["resident_count_after"]
    assert all(so2[e] >= 0 for e in c["must_be_resident"])
    assert all(so2[e] < 0 for e in c["must_not_be_resident"])

    c = g["jump_steps_refresh_schedule"]
    offload = c["budget"] < c["E"]
    for step, prefill, want in c["cases"]:
        assert oracle.should_refresh(offload, False, step, prefill, c["interval"]) == want

    c = g["vram_budget_formula"]
    b = oracle.budget_from_vram(c["free_bytes"], c["reserve_bytes"], c["expert_bytes"], c["layers"],
                                c["max_per_layer"], c["E"])
    assert 0 < b <= 128
    assert b == min((c["free_bytes"] - c["reserve_bytes"]) // (c["expert_bytes"] * c["layers"]), 128)

    c = g["per_layer_masks_differ_from_merged_union"]
    masks = []
    for ids in c["refresh_ids"]:
        so = np.full(c["E"], -1, np.int32)
        so[: c["budget"]] = np.arange(c["budget"])  # initial residents 0..budget
        t = oracle.refresh_target(oracle.hits(np.array(ids), c["E"]), c["budget"])
        so2, _, _ = oracle.apply_placement(so, c["budget"], t)
        masks.append((so2 >= 0).tolist())
    assert masks == c["per_layer"]
    assert np.logical_or.reduce(np.array(masks)).tolist() == c["merged"]


def test_placement_invariants_under_random_refreshes():
    rng = np.random.default_rng(4)
    E, n_slots = 128, 18
    so = np.full(E, -1, np.int32)
    so[:n_slots] = np.arange(n_slots)
    for step in range(200):
        ids = rng.zipf(1.3, size=64 * 8) % E
        t = oracle.refresh_target(oracle.hits(ids.astype(np.int32), E), n_slots)
        before = so.copy()
        so, pr, de = oracle.apply_placement(so, n_slots, t)
        res = np.nonzero(so >= 0)[0]
        assert len(res) == n_slots                        # residency size stays the budget
        assert sorted(so[res].tolist()) == list(range(n_slots))  # slots are a permutation
        assert all(so[e] >= 0 for e in t)                 # the target is resident
        assert len(pr) == len(de)                         # paired swaps
        assert all(before[e] < 0 for e in pr) and all(before[e] >= 0 for e in de)
        for p, d in zip(pr, de):
            assert so[p] == before[d]                     # promoted takes the demoted slot


# ------------------------------------------------------------ [miss] min_weight

def _mw_case(seed, T=200, E=32, k=8, resident_frac=0.4):
    rng = np.random.default_rng(seed)
    lg = syn.router_logits(T, E, "zipf", seed=seed)
    ids, w = oracle.route_topk(lg, k)
    slot = np.where(rng.random(E) < resident_frac, np.arange(E), -1).astype(np.int32)
    return ids, w, slot


def test_min_weight_one_or_all_resident_changes_nothing():
    ids, w, slot = _mw_case(1)
    for mw in (1.0, 1.5):
        i2, w2 = oracle.route_min_weight(ids, w, slot, 32, mw)
        assert np.array_equal(i2, ids) and np.array_equal(w2, w)
    i3, w3 = oracle.route_min_weight(ids, w, np.arange(32, dtype=np.int32), 32, 0.3)
    assert np.array_equal(i3, ids) and np.array_equal(w3, w)


def test_min_weight_keeps_the_share_and_the_full_weight():
    """Kept share before rescaling >= min_weight (or every route kept); dropped
    routes are non-resident and lighter than every kept non-resident route; kept
    weights sum back to the token's full weight."""
    ids, w, slot = _mw_case(2)
    for mw in (0.2, 0.5, 0.8, 0.95):
        i2, w2 = oracle.route_min_weight(ids, w, slot, 32, mw)
        for t in range(ids.shape[0]):
            kept = i2[t] >= 0
            dropped = ~kept
            if dropped.any():
                assert w[t][kept].astype(np.float64).sum() >= mw - 1e-6
                assert all(slot[e] < 0 for e in ids[t][dropped])
                nonres_kept = [j for j in np.nonzero(kept)[0] if slot[ids[t][j]] < 0]
                if nonres_kept:
                    assert w[t][dropped].max() <= w[t][nonres_kept].min()
            assert abs(w2[t].astype(np.float64).sum() - w[t].astype(np.float64).sum()) < 1e-5
            assert np.all(w2[t][dropped] == 0)


def test_min_weight_is_monotone_and_zero_keeps_only_resident():
    ids, w, slot = _mw_case(3)
    prev = None
    for mw in (0.95, 0.7, 0.4, 0.1):
        i2, _ = oracle.route_min_weight(ids, w, slot, 32, mw)
        drops = i2 < 0
        if prev is not None:
            assert np.all(drops[prev])   # lowering min_weight never brings a route back
        prev = drops
    i0, w0 = oracle.route_min_weight(ids, w, slot, 32, 0.0)
    res = slot[ids] >= 0
    assert np.array_equal(i0 >= 0, res)
    none = ~res.any(axis=1)
    assert np.all(w0[none] == 0)


def test_min_weight_hand_example():
    ids = np.array([[3, 0, 2, 1]], np.int32)
    w = np.array([[0.5, 0.25, 0.125, 0.125]], np.float32)
    slot = np.array([-1, 0, -1, -1], np.int32)   # only expert 1 is resident
    i2, w2 = oracle.route_min_weight(ids, w, slot, 4, 0.6)
    # 0.5 kept (share 0.5 < 0.6), 0.25 kept (share 0.75), expert 2 dropped (non-resident,
    # share reached), expert 1 kept (resident); scale 1 / 0.875
    assert i2.tolist() == [[3, 0, -1, 1]]
    np.testing.assert_array_equal(w2, np.float32([[0.5 * np.float32(1 / 0.875), 0.25 * np.float32(1 / 0.875), 0,
                                                   0.125 * np.float32(1 / 0.875)]]))


# ------------------------------------------------------ router projection (f3)

def _bf16_bits(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_router_logits_equal_a_library_matmul():
    """The projection is a plain matrix product: numpy's fp64 matmul of the same
    bf16 x and fp32 router weights agrees to fp64 rounding of the sums."""
    rng = np.random.default_rng(3)
    T, Hh, E = 9, 2816, 128
    x = syn.activations(T, Hh, seed=4)
    wr = (rng.standard_normal((E, Hh)) * 0.02).astype(np.float32)
    got = oracle.router_logits(x, wr)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
    want = xf @ wr.astype(np.float64).T
    scale = np.abs(xf) @ np.abs(wr.astype(np.float64)).T
    assert np.all(np.abs(got - want) <= 1e-12 * scale)


def test_router_logits_one_hot_rows_pick_weight_columns():
    """x = c * e_h (c a power of two) gives logits = c * w_router[:, h] exactly;
    a transposed operand or a wrong row index fails this."""
    rng = np.random.default_rng(5)
    Hh, E = 96, 24
    wr = rng.standard_normal((E, Hh)).astype(np.float32)
    xs = np.zeros((Hh, Hh), np.float32)
    for h in range(Hh):
        xs[h, h] = 2.0 ** (h % 5 - 2)
    got = oracle.router_logits(_bf16_bits(xs), wr)
    for h in range(Hh):
        assert np.array_equal(got[h], (2.0 ** (h % 5 - 2)) * wr[:, h].astype(np.float64))


def test_router_then_topk_with_identity_weights_is_topk_of_x():
    """With w_router = [I_E | 0] the logits are x's first E values, so routing
    them reduces to top-k of those values (exact: each logit is one product)."""
    T, Hh, E, k = 7, 64, 16, 4
    x = syn.activations(T, Hh, seed=8)
    wr = np.zeros((E, Hh), np.float32)
    wr[:, :E] = np.eye(E, dtype=np.float32)
    lg = oracle.router_logits(x, wr)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(lg, xf[:, :E].astype(np.float64))
    ids, _ = oracle.route_topk(lg.astype(np.float32), k)
    want = np.argsort(-xf[:, :E], axis=1, kind="stable")[:, :k]
    assert np.array_equal(ids, want)


# ------------------------------------------------- windowed hit counts (f3)

def test_hits_window_equals_bincount_over_the_window():
    """The sum of W per-step histograms is the bincount of all W steps' ids
    (numpy's bincount over the concatenation)."""
    rng = np.random.default_rng(11)
    E, W = 128, 8
    steps = [rng.integers(0, E, size=(rng.integers(1, 200),), dtype=np.int32) for _ in range(W)]
    ring = np.stack([oracle.hits(s, E) for s in steps])
    got = oracle.hits_window(ring)
    want = np.bincount(np.concatenate(steps), minlength=E).astype(np.uint32)
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.hits_window(ring[:1]), ring[0])
    assert not oracle.hits_window(np.zeros((W, E), np.uint32)).any()
