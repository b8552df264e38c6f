"""Pins for the CPU oracle (runs without a GPU).

Each test checks the oracle against something other than itself: the
closed-form E4M3 bit formula, a brute-force argmin rounding, golden spot
values with citations, a dense NumPy fp64 attention, and invariants that hold
for any correct softmax attention (single token, identical keys, zero query,
split-count and page-permutation invariance, LSE additivity, causal prefix
reduction, scale folding).
"""
import math
import os

import numpy as np
import pytest

import np_reference as npr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_spot.txt")


# --------------------------------------------------------------------------- E4M3

def test_e4m3_value_map_matches_bit_formula(oracle_lib):
    codes = np.arange(256)
    ref = npr.e4m3_values(codes)
    got = np.array([oracle_lib.e4m3_value(c) for c in codes])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert got[0x7E] == 448.0 and got[0xFE] == -448.0
    assert np.nanmax(np.abs(got)) == 448.0


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows.append((float(parts[0]), int(parts[1], 16), " ".join(parts[2:])))
    return rows


@pytest.mark.parametrize("x,code,note", _golden_rows())
def test_e4m3_golden_spot_values(oracle_lib, x, code, note):
    assert oracle_lib.e4m3_encode(x) == code, note
    assert int(npr.e4m3_round(np.array([x]))[0]) == code, note


ALL_BF16 = np.arange(65536, dtype=np.uint32).astype(np.uint16)


@pytest.mark.parametrize("scale", [1.0, 2.0 ** -3, 6.0 / 448.0, 1.0 / 3.0, 3.7 / 448.0, 4096.0])
def test_quantize_exhaustive_bf16_against_bruteforce(oracle_lib, scale):
    inv = np.float32(1.0) / np.float32(scale)
    got = oracle_lib.quantize(ALL_BF16, float(inv))
    x = (ALL_BF16.astype(np.uint32) << 16).view(np.float32)
    with np.errstate(invalid="ignore"):
        prod = (x * inv).astype(np.float32)  # one fp32 RN multiply
    ref = np.concatenate([npr.e4m3_round(prod[i:i + 8192]) for i in range(0, prod.size, 8192)])
    nan_in = np.isnan(prod)
    assert np.all(got[nan_in] == 0x7F)
    assert np.array_equal(got[~nan_in], ref[~nan_in])
    # saturation: nothing finite becomes NaN
    assert not np.any(((got & 0x7F) == 0x7F) & ~nan_in)


def test_quantize_round_trip_all_finite_codes(oracle_lib):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    for k in (-4, 0, 3):
        scale = 2.0 ** k
        vals = npr.e4m3_values(codes) * scale
        bits = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal(npr.bf16_bits_to_f64(bits), vals)  # exact in bf16
        got = oracle_lib.quantize(bits, float(np.float32(1.0) / np.float32(scale)))
        assert np.array_equal(got, codes)


def test_quantize_monotone(oracle_lib):
    x = np.linspace(-600, 600, 20001).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    xv = npr.bf16_bits_to_f64(bits)
    order = np.argsort(xv, kind="stable")
    codes = oracle_lib.quantize(bits, 1.0)
    vals = npr.e4m3_values(codes)[order]
    assert np.all(np.diff(vals) >= 0)


# --------------------------------------------------------------------------- attention helpers

def _case(rng, B, q_len, H, lens, fp8, shuffle=True, kv_std=1.0, scale=0.05):
    pages = [-(-L // 64) for L in lens]
    npg = sum(pages) + 2
    perm = rng.permutation(npg) if shuffle else np.arange(npg)
    maxp = max(pages)
    bt = np.full((B, maxp), perm[-1], dtype=np.int32)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    vals = (rng.standard_normal((npg, 64, 576)) * kv_std).astype(np.float32)
    if fp8:
        import oracle  # inputs only: the quantiser itself is pinned by the tests above
        bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
        kv = oracle.quantize(bits, float(np.float32(1.0) / np.float32(scale)))
        kv_scale = float(np.float32(scale))  # the API carries kv_scale as fp32
    else:
        kv = (vals.view(np.uint32) >> 16).astype(np.uint16)
        kv_scale = 1.0
    qn = (rng.standard_normal((B, q_len, H, 512)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    qr = (rng.standard_normal((B, q_len, H, 64)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return dict(q_nope=qn, q_rope=qr, kv_pages=kv, kv_scale=kv_scale, block_table=bt,
                seq_lens=np.array(lens, dtype=np.int32), q_len=q_len, H=H,
                softmax_scale=float(np.float32(1.0 / math.sqrt(192.0))))  # fp32 in the API


def _all_rows(c):
    return np.arange(len(c["seq_lens"]) * c["q_len"] * c["H"], dtype=np.int64)


def _oracle_decode(oracle_lib, c, rows=None):
    rows = _all_rows(c) if rows is None else rows
    return oracle_lib.decode_rows(c["q_nope"], c["q_rope"], c["kv_pages"], c["kv_scale"],
                                  c["block_table"], c["seq_lens"], c["q_len"], c["H"],
                                  c["softmax_scale"], rows)


# --------------------------------------------------------------------------- attention pins

@pytest.mark.parametrize("fp8", [True, False])
@pytest.mark.parametrize("B,q_len,H,lens", [
    (1, 1, 1, [1]), (1, 1, 4, [5]), (2, 2, 2, [64, 70]), (1, 4, 3, [130]), (3, 1, 2, [8, 1, 200]),
])
def test_decode_matches_dense_numpy(oracle_lib, fp8, B, q_len, H, lens):
    rng = np.random.default_rng(B * 100 + q_len * 10 + H + (7 if fp8 else 0))
    c = _case(rng, B, q_len, H, lens, fp8)
    o, lse = _oracle_decode(oracle_lib, c)
    O, LSE = npr.attend(**c)
    np.testing.assert_allclose(o, O.reshape(-1, 512), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, LSE.reshape(-1), rtol=1e-11, atol=1e-12)


def test_single_token_returns_its_value(oracle_lib):
    rng = np.random.default_rng(1)
    c = _case(rng, 1, 1, 3, [1], fp8=True)
    o, lse = _oracle_decode(oracle_lib, c)
    row = c["kv_pages"][c["block_table"][0, 0], 0]
    v = npr.e4m3_values(row) * c["kv_scale"]
    for h in range(3):
        assert np.array_equal(o[h], v[:512])
        q = np.concatenate([npr.bf16_bits_to_f64(c["q_nope"][0, 0, h]), npr.bf16_bits_to_f64(c["q_rope"][0, 0, h])])
        assert lse[h] == pytest.approx(c["softmax_scale"] * float(q @ v), rel=1e-12)


def test_identical_keys_give_mean_and_log_length(oracle_lib):
    rng = np.random.default_rng(2)
    c = _case(rng, 1, 1, 2, [150], fp8=False, shuffle=True)
    row = c["kv_pages"][c["block_table"][0, 0], 0].copy()
    c["kv_pages"][:, :, :] = row[None, None, :]
    o, lse = _oracle_decode(oracle_lib, c)
    v = npr.bf16_bits_to_f64(row)
    for h in range(2):
        np.testing.assert_allclose(o[h], v[:512], rtol=0, atol=1e-14)
        q = np.concatenate([npr.bf16_bits_to_f64(c["q_nope"][0, 0, h]), npr.bf16_bits_to_f64(c["q_rope"][0, 0, h])])
        s = c["softmax_scale"] * float(q @ v)
        assert lse[h] == pytest.approx(s + math.log(150), rel=1e-12)


def test_common_rope_key_shifts_lse_only(oracle_lib):
    # When every token has the same RoPE key r, changing the RoPE query by d
    # moves every score by softmax_scale * (d . r): the weights, and so O, do
    # not change, and the LSE moves by exactly that amount.
    rng = np.random.default_rng(5)
    c = _case(rng, 1, 1, 2, [300], fp8=False)
    r = c["kv_pages"][c["block_table"][0, 0], 0, 512:].copy()
    c["kv_pages"][:, :, 512:] = r[None, None, :]
    o, lse = _oracle_decode(oracle_lib, c)
    c2 = dict(c)
    qr2 = c["q_rope"].copy()
    qr2[0, 0, :, 3] = np.float32(0.75).view(np.uint32) >> 16       # exact in bf16
    qr2[0, 0, :, 40] = np.float32(-2.5).view(np.uint32) >> 16
    c2["q_rope"] = qr2
    o2, lse2 = _oracle_decode(oracle_lib, c2)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    rv = npr.bf16_bits_to_f64(r)
    for h in range(2):
        d = npr.bf16_bits_to_f64(qr2[0, 0, h]) - npr.bf16_bits_to_f64(c["q_rope"][0, 0, h])
        assert lse2[h] - lse[h] == pytest.approx(c["softmax_scale"] * float(d @ rv), rel=1e-10, abs=1e-12)


def test_zero_query_gives_mean_of_values(oracle_lib):
    rng = np.random.default_rng(3)
    c = _case(rng, 1, 1, 1, [97], fp8=True)
    c["q_nope"][:] = 0
    c["q_rope"][:] = 0
    o, lse = _oracle_decode(oracle_lib, c)
    t = np.arange(97)
    vals = npr.e4m3_values(c["kv_pages"][c["block_table"][0][t // 64], t % 64]) * c["kv_scale"]
    np.testing.assert_allclose(o[0], vals[:, :512].mean(axis=0), rtol=1e-12, atol=1e-14)
    assert lse[0] == pytest.approx(math.log(97), rel=1e-13)


@pytest.mark.parametrize("S", [1, 2, 4, 7, 64])
def test_split_count_invariance_and_lse_additivity(oracle_lib, S):
    rng = np.random.default_rng(10 + S)
    c = _case(rng, 2, 2, 2, [300, 1000], fp8=True)
    rows = _all_rows(c)
    o, lse = _oracle_decode(oracle_lib, c)
    ns = np.full(2, S, dtype=np.int32)
    po, pl = oracle_lib.partials_rows(c["q_nope"], c["q_rope"], c["kv_pages"], c["kv_scale"],
                                      c["block_table"], c["seq_lens"], ns, S, c["q_len"], c["H"],
                                      c["softmax_scale"], rows)
    # LSE additivity: LSE(all) = logsumexp over splits, computed here in fp64
    finite = np.isfinite(pl)
    m = np.where(finite, pl, -np.inf).max(axis=1)
    lse_sum = m + np.log(np.where(finite, np.exp(pl - m[:, None]), 0.0).sum(axis=1))
    np.testing.assert_allclose(lse_sum, lse, rtol=1e-12)
    # the merge (fp32 partials as the GPU stores them) reproduces the unsplit result
    n_per_row = ns[(rows // (c["H"] * c["q_len"]))]
    co, cl = oracle_lib.combine(po.astype(np.float32), pl.astype(np.float32), n_per_row)
    np.testing.assert_allclose(co, o, rtol=0, atol=2e-6)
    np.testing.assert_allclose(cl, lse, rtol=1e-6)


def test_split_range_partition(oracle_lib):
    for L in (1, 63, 64, 65, 1000, 4096, 131072):
        for S in (1, 2, 3, 7, 32, 64, 200):
            vis = L
            got = [oracle_lib.split_range(L, S, s, vis) for s in range(S)]
            n_pages = -(-L // 64)
            c = -(-n_pages // S)
            pos = 0
            for s, (t0, t1) in enumerate(got):
                assert t0 == pos or t1 == t0
                assert t0 % 64 == 0 or t1 == t0
                assert t1 - t0 <= c * 64
                pos = max(pos, t1)
            assert pos == L
            assert sum(t1 - t0 for t0, t1 in got) == L
    # causal clip: a shorter visible length truncates the last non-empty split
    assert oracle_lib.split_range(1000, 4, 3, 900) == (768, 900)
    assert oracle_lib.split_range(1000, 4, 3, 700) == (700, 700)


def test_page_permutation_invariance(oracle_lib):
    rng = np.random.default_rng(4)
    c = _case(rng, 2, 1, 2, [200, 130], fp8=True, shuffle=False)
    o1, l1 = _oracle_decode(oracle_lib, c)
    npg = c["kv_pages"].shape[0]
    perm = rng.permutation(npg)
    inv = np.argsort(perm)
    c2 = dict(c)
    c2["kv_pages"] = c["kv_pages"][perm]          # physical page p moves to slot inv[p]
    c2["block_table"] = inv[c["block_table"]].astype(np.int32)
    o2, l2 = _oracle_decode(oracle_lib, c2)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_causal_rows_equal_prefix_decode(oracle_lib):
    rng = np.random.default_rng(5)
    c = _case(rng, 1, 4, 2, [141], fp8=True)
    o, lse = _oracle_decode(oracle_lib, c)
    for q in range(4):
        c1 = dict(c)
        c1["q_len"] = 1
        c1["q_nope"] = c["q_nope"][:, q:q + 1].copy()
        c1["q_rope"] = c["q_rope"][:, q:q + 1].copy()
        c1["seq_lens"] = np.array([141 - 3 + q], dtype=np.int32)
        o1, l1 = _oracle_decode(oracle_lib, c1)
        for h in range(2):
            assert np.array_equal(o[q * 2 + h], o1[h])
            assert lse[q * 2 + h] == l1[h]


def test_fp8_scale_folding_equals_bf16_of_dequantised_values(oracle_lib):
    rng = np.random.default_rng(6)
    c = _case(rng, 1, 1, 2, [77], fp8=True, scale=0.125)
    vals = npr.e4m3_values(c["kv_pages"]) * 0.125
    vals = np.nan_to_num(vals, nan=0.0)
    bits = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(npr.bf16_bits_to_f64(bits), vals)
    o1, l1 = _oracle_decode(oracle_lib, c)
    c2 = dict(c)
    c2["kv_pages"] = bits
    c2["kv_scale"] = 1.0
    o2, l2 = _oracle_decode(oracle_lib, c2)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)


def test_combine_closed_forms(oracle_lib):
    rng = np.random.default_rng(7)
    po = rng.standard_normal((3, 4, 512)).astype(np.float32)
    pl = np.array([[0.5, -1.0, -np.inf, -np.inf],
                   [-np.inf, -np.inf, -np.inf, -np.inf],
                   [2.0, 0, 0, 0]], dtype=np.float32)
    ns = np.array([3, 4, 1], dtype=np.int32)
    o, lse = oracle_lib.combine(po, pl, ns)
    a, b = 0.5, -1.0
    p64 = po.astype(np.float64)
    want = (math.exp(a) * p64[0, 0] + math.exp(b) * p64[0, 1]) / (math.exp(a) + math.exp(b))
    np.testing.assert_allclose(o[0], want, rtol=1e-12)
    assert lse[0] == pytest.approx(math.log(math.exp(a) + math.exp(b)), rel=1e-12)
    assert np.all(o[1] == 0) and lse[1] == -np.inf
    np.testing.assert_allclose(o[2], po[2, 0].astype(np.float64), rtol=0, atol=0)
    assert lse[2] == pytest.approx(2.0)


# --------------------------------------------------------------------------- KV append
# The step before the path: RoPE on the 64-wide key, saturating E4M3, paged
# write ("Muse Spark Open" article, section "内核优化：解码吞吐 3 倍", bullet
# "RoPE 与 KV 缓存写入融合"; "SGLang & Miles ... Vera Rubin" article, bullet
# "原生 FP8 转换").  Reading: the original rotary embedding, pairs (2i, 2i+1),
# theta_i = 10000^(-2i/64).

def test_rope_position_zero_is_identity_and_norm_is_kept(oracle_lib):
    rng = np.random.default_rng(11)
    x = rng.standard_normal(64)
    assert np.array_equal(oracle_lib.rope_f64(x, 0), x)
    for pos in (1, 7, 4095, 131071, 262143):
        y = oracle_lib.rope_f64(x, pos)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12
        # each pair keeps its own length (a rotation acts within the pair)
        assert np.allclose(np.hypot(y[0::2], y[1::2]), np.hypot(x[0::2], x[1::2]), rtol=0, atol=1e-12)


def test_rope_closed_form_pairs(oracle_lib):
    # pair 0 has theta = 1: a rotation by pos radians; pair 16 has theta = 10000^-0.5 = 0.01
    x = np.zeros(64)
    x[0], x[1] = 1.0, 0.0
    x[32], x[33] = 0.0, 2.0
    y = oracle_lib.rope_f64(x, 3)
    assert abs(y[0] - math.cos(3.0)) < 1e-15 and abs(y[1] - math.sin(3.0)) < 1e-15
    assert abs(y[32] - (-2.0 * math.sin(0.03))) < 1e-15 and abs(y[33] - 2.0 * math.cos(0.03)) < 1e-15


def test_rope_composes_and_relative_positions(oracle_lib):
    # R(a) R(b) = R(a + b), and <R(m) q, R(n) k> depends only on m - n
    rng = np.random.default_rng(12)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    a, b = 37, 1000
    # rotating by a then by b: apply the pairwise rotation of b to R(a) x
    ra = oracle_lib.rope_f64(q, a)
    rab = oracle_lib.rope_f64(ra, b)
    assert np.allclose(rab, oracle_lib.rope_f64(q, a + b), rtol=0, atol=1e-11)
    d1 = oracle_lib.rope_f64(q, 500) @ oracle_lib.rope_f64(k, 480)
    d2 = oracle_lib.rope_f64(q, 20) @ oracle_lib.rope_f64(k, 0)
    assert abs(d1 - d2) < 1e-11


def test_rope_table_is_the_rounded_angles(oracle_lib):
    t = oracle_lib.rope_table(300)
    pos = np.arange(300)[:, None]
    theta = 10000.0 ** (-2.0 * np.arange(32) / 64.0)
    ang = pos * theta[None, :]
    assert np.array_equal(t[..., 0], np.cos(ang).astype(np.float32))
    assert np.array_equal(t[..., 1], np.sin(ang).astype(np.float32))
    assert np.all(t[0, :, 0] == 1.0) and np.all(t[0, :, 1] == 0.0)


def _append_case(seed=13, B=3, n_new=2, lens=(5, 64, 130), spare=3):
    rng = np.random.default_rng(seed)
    pages = [(L + 63) // 64 for L in lens]
    num_pages = sum(pages) + spare
    perm = rng.permutation(num_pages).astype(np.int32)
    bt = np.full((B, max(pages)), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    c = rng.standard_normal((B, n_new, 512)).astype(np.float32)
    r = (3.0 * rng.standard_normal((B, n_new, 64))).astype(np.float32)
    bits = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)  # truncate to bf16 bits
    return bits(c), bits(r), bt, np.array(lens, dtype=np.int32), num_pages


def test_append_places_rows_and_quantises_the_latent_like_the_prep_step(oracle_lib):
    c, r, bt, sl, num_pages = _append_case()
    B, n_new = c.shape[:2]
    inv = float(np.float32(448.0 / 8.0))
    table = oracle_lib.rope_table(256)
    kv = np.full((num_pages, 64, 576), 0xAA, dtype=np.uint8)
    assert oracle_lib.append_kv(c, r, table, bt, sl, n_new, inv, kv) == 0
    written = np.zeros((num_pages, 64), dtype=bool)
    for b in range(B):
        for j in range(n_new):
            pos = sl[b] - n_new + j
            page, row = bt[b, pos // 64], pos % 64
            written[page, row] = True
            # latent: the same codes as the (independently pinned) quantiser
            assert np.array_equal(kv[page, row, :512], oracle_lib.quantize(c[b, j], inv))
    # nothing else was touched
    assert np.all(kv[~written] == 0xAA)


def test_append_rope_codes_follow_the_fp64_rotation(oracle_lib):
    # the fp32 rotation rounds a few times; its codes equal the E4M3 rounding of
    # the exact fp64 rotation except where y * inv_scale lies within a few fp32
    # ulps of a rounding boundary, and then they are neighbours
    rng = np.random.default_rng(14)
    B, n_new, L = 1, 64, 100000
    c = np.zeros((B, n_new, 512), dtype=np.uint16)
    rf = (4.0 * rng.standard_normal((B, n_new, 64))).astype(np.float32)
    r = (rf.view(np.uint32) >> 16).astype(np.uint16)
    bt = np.arange((L + 63) // 64, dtype=np.int32)[None, :]
    kv = np.zeros((bt.shape[1], 64, 576), dtype=np.uint8)
    inv = float(np.float32(448.0 / 16.0))
    table = oracle_lib.rope_table(L)
    assert oracle_lib.append_kv(c, r, table, bt, np.array([L], np.int32), n_new, inv, kv) == 0
    vals = lambda codes: np.array([oracle_lib.e4m3_value(int(v)) for v in codes])
    diffs = 0
    for j in range(n_new):
        pos = L - n_new + j
        x = (r[0, j].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        y = oracle_lib.rope_f64(x, pos) * inv
        got = kv[pos // 64, pos % 64, 512:]
        want = npr.e4m3_round(y.astype(np.float32))
        mism = got != want
        diffs += int(mism.sum())
        if mism.any():
            # neighbouring codes only, and only near a rounding boundary
            assert np.all(np.abs(vals(got[mism]) - vals(want[mism])) <=
                          2 * np.abs(vals(want[mism])) * 2.0 ** -3 + 2.0 ** -9)
    assert diffs <= n_new * 64 // 100


def test_append_skips_out_of_range_tokens(oracle_lib):
    c, r, bt, sl, num_pages = _append_case()
    kv = np.zeros((num_pages, 64, 576), dtype=np.uint8)
    table = oracle_lib.rope_table(100)  # request 2 ends at position 129: beyond the table
    skipped = oracle_lib.append_kv(c, r, table, bt, sl, 2, 1.0, kv)
    assert skipped == 2
    bt2 = bt.copy()
    bt2[0, 0] = num_pages + 5  # page id outside the pool
    kv2 = np.zeros_like(kv)
    assert oracle_lib.append_kv(c, r, oracle_lib.rope_table(256), bt2, sl, 2, 1.0, kv2) == 2


def test_fp8_query_partials_equal_the_bf16_path_on_the_dequantised_query(oracle_lib):
    # The FP8-query entry point reads 576 E4M3 codes per row with one scale.
    # With a power-of-two scale the dequantised query is exactly bf16, so the
    # bf16 entry point (pinned against dense NumPy above) on those values must
    # give the same partials; with one split it must match dense NumPy too.
    rng = np.random.default_rng(11)
    c = _case(rng, 2, 2, 3, [130, 70], fp8=True)
    q_scale = 0.0625
    qbits = np.concatenate([c["q_nope"], c["q_rope"]], axis=-1)       # [B][q][H][576] bf16
    q8 = oracle_lib.quantize(qbits, float(np.float32(1.0) / np.float32(q_scale)))
    qv = npr.e4m3_values(q8) * q_scale
    assert np.all(np.isfinite(qv))
    vbits = (qv.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(npr.bf16_bits_to_f64(vbits), qv)
    rows = _all_rows(c)
    ns = np.array([3, 2], dtype=np.int32)
    args = (c["kv_pages"], c["kv_scale"], c["block_table"], c["seq_lens"], ns, 3, c["q_len"], c["H"],
            c["softmax_scale"], rows)
    o8, l8 = oracle_lib.partials_rows_q8(q8, q_scale, *args)
    ob, lb = oracle_lib.partials_rows(np.ascontiguousarray(vbits[..., :512]),
                                      np.ascontiguousarray(vbits[..., 512:]), *args)
    np.testing.assert_allclose(o8, ob, rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(np.isneginf(l8), np.isneginf(lb))
    fin = np.isfinite(lb)
    np.testing.assert_allclose(l8[fin], lb[fin], rtol=1e-13)
    # one split: the unsplit decode, against dense NumPy on the dequantised query
    o1, l1 = oracle_lib.partials_rows_q8(q8, q_scale, c["kv_pages"], c["kv_scale"], c["block_table"],
                                         c["seq_lens"], np.ones(2, np.int32), 1, c["q_len"], c["H"],
                                         c["softmax_scale"], rows)
    c2 = dict(c)
    c2["q_nope"] = np.ascontiguousarray(vbits[..., :512])
    c2["q_rope"] = np.ascontiguousarray(vbits[..., 512:])
    O, LSE = npr.attend(**c2)
    np.testing.assert_allclose(o1[:, 0], O.reshape(-1, 512), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(l1[:, 0], LSE.reshape(-1), rtol=1e-11, atol=1e-12)
