"""Pins of the CPU oracle against facts fixed outside it: IEEE binary16,
closed forms, library routines (scipy Hadamard, scipy softmax), invariants of
orthogonal rotations, hand-derived worked values (tests/golden) and a second,
independently written numpy oracle.  CPU only."""
import json
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special

from oracle import np_mini
from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantizer_worked.json")
D = 128


def rand_orth(rng):
    q, r = np.linalg.qr(rng.standard_normal((D, D)))
    return (q * np.sign(np.diag(r))[None, :]).astype(np.float32)


# --- binary16 ----------------------------------------------------------------------------

def test_f16_to_f32_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = orc.f16_bits_to_f32(bits)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_matches_numpy():
    rng = np.random.default_rng(0)
    parts = [
        rng.standard_normal(200000).astype(np.float32) * 10,
        (rng.standard_normal(100000) * 1e-5).astype(np.float32),      # subnormal halves
        (rng.standard_normal(50000) * 1e-7).astype(np.float32),       # underflow region
        rng.uniform(6e4, 7e4, 20000).astype(np.float32),               # overflow edge
        np.array([65504, 65519.99, 65520, -65520, 2**-25, 2**-24, 3 * 2**-26, 0.0, -0.0,
                  np.inf, -np.inf], np.float32),
    ]
    # exact midpoints between consecutive halves (ties), normal and subnormal
    h = np.arange(0, 0x7bff, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    parts.append(((lo + hi) / 2).astype(np.float32))
    parts.append(-((lo + hi) / 2).astype(np.float32))
    x = np.concatenate(parts)
    got = orc.f32_to_f16_bits(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


# --- FWHT and rotations -------------------------------------------------------------------

@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128])
def test_fwht_equals_sylvester_matrix(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal((5, n))
    H = scipy.linalg.hadamard(n).astype(np.float64)
    for r in range(5):
        assert np.allclose(orc.fwht_f64(x[r]), H @ x[r], rtol=0, atol=1e-12)


def test_fwht_orthogonality_and_involution():
    I = np.eye(D)
    H = np.stack([orc.fwht_f64(I[i]) for i in range(D)])
    assert np.array_equal(H @ H.T, D * np.eye(D))
    x = np.random.default_rng(1).standard_normal(D)
    assert np.allclose(orc.fwht_f64(orc.fwht_f64(x)) / D, x, atol=1e-13)


def test_dense_rotation_is_row_vector_convention():
    """x_rot = x . R: the basis vector e_i must rotate to row i of R."""
    R = rand_orth(np.random.default_rng(2))
    out = orc.rotate_f64(np.eye(D), 0, R=R)
    assert np.array_equal(out, R.astype(np.float64))
    back = orc.unrotate_f64(np.eye(D), 0, R=R)          # e_j . R^T = column j of R
    assert np.array_equal(back, R.astype(np.float64).T)


def test_perm_fwht_equals_explicit_matrix():
    """FWHT mode equals the dense rotation R[perm[i], :] = H[i, :]/sqrt(128),
    which is orthogonal; its inverse undoes it."""
    rng = np.random.default_rng(3)
    perm = rng.permutation(D).astype(np.int32)
    H = scipy.linalg.hadamard(D) / np.sqrt(D)
    R = np.zeros((D, D))
    R[perm, :] = H
    assert np.allclose(R @ R.T, np.eye(D), atol=1e-14)
    x = rng.standard_normal((7, D))
    got = orc.rotate_f64(x, 1, perm=perm)
    assert np.allclose(got, x @ R, atol=1e-12)
    assert np.allclose(orc.unrotate_f64(got, 1, perm=perm), x, atol=1e-12)
    dense = orc.rotate_f64(x, 0, R=R.astype(np.float32))
    assert np.allclose(dense, got, rtol=0, atol=1e-6)


@pytest.mark.parametrize("mode", [0, 1])
def test_rotation_invariance_of_attention(mode):
    """Attention over (qR, KR, VR) followed by R_v^T equals attention over
    (q, K, V) in fp64: the rotation applied before quantization and removed
    after attention changes nothing but the quantization error."""
    rng = np.random.default_rng(4 + mode)
    L = 37
    q = rng.standard_normal(D)
    K = rng.standard_normal((L, D)) * 2
    V = rng.standard_normal((L, D))
    if mode == 0:
        kw = dict(R=rand_orth(rng))
        vw = dict(R=rand_orth(rng))
    else:
        kw = dict(perm=rng.permutation(D).astype(np.int32))
        vw = dict(perm=rng.permutation(D).astype(np.int32))
    ref = orc.attention_f64(q, K, V)
    rot = orc.attention_f64(orc.rotate_f64(q, mode, **kw)[0], orc.rotate_f64(K, mode, **kw),
                            orc.rotate_f64(V, mode, **vw))
    back = orc.unrotate_f64(rot, mode, **vw)[0]
    assert np.max(np.abs(back - ref)) <= 1e-5 * np.linalg.norm(ref)
    # a dense fp32 R is orthogonal only to fp32 precision; FWHT is exact
    assert np.max(np.abs(back - ref)) <= (1e-6 if mode == 0 else 1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rotation_lowers_int2_error_on_outlier_channels(seed):
    """The pages' reason for rotating (KVLinC abstract: the Hadamard rotation
    reduces quantization error; RotateKV abstract item (i): outlier-aware
    rotation; OptR introduction): keys with a few channels 20x larger than
    the rest, quantized to INT2 in groups of 32, come back closer to the
    input when they are rotated first (dense orthogonal R or perm + FWHT)
    and the rotation is removed after dequantisation than when they are
    quantized as they are."""
    rng = np.random.default_rng(100 + seed)
    K = rng.standard_normal((256, D))
    K[:, rng.choice(D, 8, replace=False)] *= 20
    kb = orc.f32_to_f16_bits(K.astype(np.float32))
    Kh = orc.f16_bits_to_f32(kb).astype(np.float64)

    def rel_error(mode, **kw):
        c, s, z = orc.quantize_rows(orc.rotate_rows_f32(kb, mode, **kw))
        back = orc.unrotate_f64(np_mini.dequant(c, s, z), mode, **kw)
        return np.linalg.norm(back - Kh) / np.linalg.norm(Kh)

    plain = rel_error(0, R=np.eye(D, dtype=np.float32))
    dense = rel_error(0, R=rand_orth(rng).astype(np.float32))
    fwht = rel_error(1, perm=rng.permutation(D).astype(np.int32))
    assert dense < 0.85 * plain and fwht < 0.85 * plain, (plain, dense, fwht)


def test_attention_f64_against_scipy_softmax():
    rng = np.random.default_rng(5)
    L = 9
    q, K, V = rng.standard_normal(D), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    p = scipy.special.softmax(K @ q / np.sqrt(D))
    assert np.allclose(orc.attention_f64(q, K, V), p @ V, atol=1e-13)


# --- quantizer ----------------------------------------------------------------------------

def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_quantizer_worked_groups():
    for case in golden()["groups"]:
        row = np.zeros(D, np.float32)
        for g in range(4):            # same group in all 4 slots
            row[g * 32:(g + 1) * 32] = np.array(case["x"], np.float32)
        codes, s, z = orc.quantize_rows(row)
        for g in range(4):
            assert list(codes[0, g * 32:(g + 1) * 32]) == case["codes"], case["name"]
            assert s[0, g] == case["s_bits"] and z[0, g] == case["z_bits"], case["name"]


def test_quantizer_grid_round_trip():
    """x = z + c*s with z an fp16 value, s a power of two and c covering all
    four levels: codes recover c exactly and dequantisation returns x."""
    rng = np.random.default_rng(6)
    for _ in range(200):
        row = np.zeros(D, np.float32)
        want = np.zeros(D, np.uint8)
        zs, ss = [], []
        for g in range(4):
            s = np.float32(2.0 ** rng.integers(-8, 4))
            z = np.float32(np.float16(rng.uniform(-4, 4)))
            c = rng.integers(0, 4, 32)
            c[:4] = [0, 1, 2, 3]
            rng.shuffle(c)
            row[g * 32:(g + 1) * 32] = z + c.astype(np.float32) * s
            want[g * 32:(g + 1) * 32] = c
            zs.append(z)
            ss.append(s)
        codes, s_bits, z_bits = orc.quantize_rows(row)
        assert np.array_equal(codes[0], want)
        assert np.array_equal(orc.f16_bits_to_f32(s_bits[0]), np.array(ss, np.float32))
        assert np.array_equal(orc.f16_bits_to_f32(z_bits[0]), np.array(zs, np.float32))
        deq = np_mini.dequant(codes[0], s_bits[0], z_bits[0])
        assert np.array_equal(deq, row.astype(np.float64))


def test_quantizer_error_bound():
    """Every element that is not clamped lies within half a step of its
    dequantised value; clamped ones only spill by the fp16 rounding of z/s."""
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((500, D)) * rng.uniform(0.1, 30, (500, 1))).astype(np.float32)
    codes, s_bits, z_bits = orc.quantize_rows(x)
    s = orc.f16_bits_to_f32(s_bits).astype(np.float64)
    z = orc.f16_bits_to_f32(z_bits).astype(np.float64)
    g = np.arange(D) // 32
    xhat = codes * s[:, g] + z[:, g]
    err = np.abs(x - xhat)
    t = (x - z[:, g]) / s[:, g]
    inner = (t >= -0.5) & (t <= 3.5)
    assert np.all(err[inner] <= 0.5 * s[:, g][inner] * (1 + 2e-6) + 1e-30)
    # outside the grid only by the rounding of z and s (far below one step)
    assert np.all(np.abs(t[~inner] - np.clip(t[~inner], -0.5, 3.5)) < 0.01)
    # every level is used and the extremes land on 0 and 3
    assert set(np.unique(codes)) == {0, 1, 2, 3}


def test_quantizer_matches_numpy_mini_oracle():
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((300, D)) * rng.uniform(0.01, 50, (300, 1))).astype(np.float32)
    x[0, :32] = 1.5                       # constant group
    x[1, :32] = np.linspace(0, 3, 32)     # exact grid with ties
    a = orc.quantize_rows(x)
    b = np_mini.quantize_rows(x)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


# --- packing and the cache block format -------------------------------------------------------

def test_pack_worked_bytes():
    for case in golden()["pack"]:
        codes = np.zeros(D, np.uint8)
        for g, c in enumerate(case["codes_g0_g1_g2_g3"]):
            codes[g * 32 + 5] = c                      # element 5 of each group
        b = orc.pack_row(codes)
        assert b[5] == case["byte"] and b.sum() == case["byte"]


def test_pack_unpack_round_trip():
    rng = np.random.default_rng(9)
    for _ in range(50):
        c = rng.integers(0, 4, D).astype(np.uint8)
        assert np.array_equal(orc.unpack_row(orc.pack_row(c)), c)


def test_block_layout_is_a_bijection():
    """The 16 tokens' fields tile the 1536-byte block exactly once."""
    owner = np.full(orc.BLK_BYTES, -1)
    for tau in range(16):
        block = np.zeros(orc.BLK_BYTES, np.uint8)
        ff = np.full(32, 0xFF, np.uint8)
        f16 = np.full(4, 0xFFFF, np.uint16)
        orc.store_token(block, tau, ff, ff, f16, f16, f16, f16)
        hit = np.nonzero(block)[0]
        assert len(hit) == 96                        # 32 + 32 + 16 + 16 bytes per token
        assert np.all(owner[hit] == -1)
        owner[hit] = tau
    assert np.all(owner >= 0)


def test_block_layout_worked_offsets():
    lay = golden()["layout"]
    for c in lay["k_word"]:
        block = np.zeros(orc.BLK_BYTES, np.uint8)
        kb = np.zeros(32, np.uint8)
        kb[4 * c["wi"]:4 * c["wi"] + 4] = [1, 2, 3, 4]
        z32, z4 = np.zeros(32, np.uint8), np.zeros(4, np.uint16)
        orc.store_token(block, c["tau"], kb, z32, z4, z4, z4, z4)
        assert list(block[c["offset"]:c["offset"] + 4]) == [1, 2, 3, 4]
    for c in lay["v_piece"]:
        block = np.zeros(orc.BLK_BYTES, np.uint8)
        vb = np.zeros(32, np.uint8)
        vb[2 * c["w"]:2 * c["w"] + 2] = [7, 9]
        z32, z4 = np.zeros(32, np.uint8), np.zeros(4, np.uint16)
        orc.store_token(block, c["tau"], z32, vb, z4, z4, z4, z4)
        assert list(block[c["offset"]:c["offset"] + 2]) == [7, 9]
    for c in lay["k_meta"]:
        block = np.zeros(orc.BLK_BYTES, np.uint8)
        ks, kz = np.zeros(4, np.uint16), np.zeros(4, np.uint16)
        ks[c["g"]], kz[c["g"]] = 0x1234, 0x5678
        z32, z4 = np.zeros(32, np.uint8), np.zeros(4, np.uint16)
        orc.store_token(block, c["tau"], z32, z32, ks, kz, z4, z4)
        assert list(block[c["offset"]:c["offset"] + 4]) == [0x34, 0x12, 0x78, 0x56]
    for c in lay["v_scale"]:
        block = np.zeros(orc.BLK_BYTES, np.uint8)
        vs, vz = np.zeros(4, np.uint16), np.zeros(4, np.uint16)
        vs[c["g"]], vz[c["g"]] = 0x1111, 0x2222
        z32, z4 = np.zeros(32, np.uint8), np.zeros(4, np.uint16)
        orc.store_token(block, c["tau"], z32, z32, z4, z4, vs, vz)
        assert list(block[c["offset"]:c["offset"] + 4]) == [0x11, 0x11, 0x22, 0x22]


# --- append / decode ----------------------------------------------------------------------------

def f16(x):
    return np.asarray(x, np.float16).view(np.uint16)


def grid_rows(rng, n):
    """fp16 rows whose every group of 32 is an exact 4-level grid z + c*s."""
    rows = np.zeros((n, D), np.float32)
    for r in range(n):
        for g in range(4):
            s = np.float32(2.0 ** rng.integers(-3, 1))
            z = np.float32(rng.integers(-16, 16) / 8.0)     # multiples of 1/8: fp16-exact
            c = rng.integers(0, 4, 32)
            c[:4] = [0, 1, 2, 3]
            rng.shuffle(c)
            rows[r, g * 32:(g + 1) * 32] = z + c * s
    assert np.array_equal(rows.astype(np.float16).astype(np.float32), rows)
    return rows


def test_decode_exact_on_grid_values_with_identity_rotation():
    """With R = I and K/V on exact 4-level grids, quantization is lossless and
    the decode equals exact fp64 attention (scipy softmax)."""
    rng = np.random.default_rng(10)
    L, Hkv = 37, 2
    K = grid_rows(rng, L * Hkv).reshape(1, L, Hkv, D)
    V = grid_rows(rng, L * Hkv).reshape(1, L, Hkv, D)
    I = np.stack([np.eye(D, dtype=np.float32)] * Hkv)
    cache = orc.Cache(1, Hkv, 48, 0)
    sl = np.zeros(1, np.int32)
    assert orc.append(cache, f16(K), f16(V), 0, I, I, None, sl) == 0
    assert sl[0] == L
    Q = rng.standard_normal((1, 2 * Hkv, D)).astype(np.float16)
    out, st = orc.decode(cache, Q.view(np.uint16), 0, I, I, None, sl)
    assert st == 0
    for hq in range(2 * Hkv):
        h = hq // 2
        q = Q[0, hq].astype(np.float64)
        Kh, Vh = K[0, :, h].astype(np.float64), V[0, :, h].astype(np.float64)
        p = scipy.special.softmax(Kh @ q / np.sqrt(D))
        assert np.allclose(out[0, hq], p @ Vh, rtol=0, atol=1e-12)


def test_decode_zero_query_is_mean_of_values():
    """q = 0 gives equal scores: the output is the mean of the dequantised V
    rows (decoded here by the numpy mini-oracle), rotated back."""
    rng = np.random.default_rng(11)
    L = 21
    R = np.stack([rand_orth(rng)])
    K = rng.standard_normal((1, L, 1, D)).astype(np.float16)
    V = rng.standard_normal((1, L, 1, D)).astype(np.float16)
    cache = orc.Cache(1, 1, 32, 0)
    sl = np.zeros(1, np.int32)
    orc.append(cache, K.view(np.uint16), V.view(np.uint16), 0, R, R, None, sl)
    out, _ = orc.decode(cache, np.zeros((1, 1, D), np.uint16), 0, R, R, None, sl)
    vrows = []
    for t in range(L):
        _, vb, _, _, vs, vz = orc.load_token(cache.blocks[0, 0, t // 16], t % 16)
        vrows.append(np_mini.dequant(orc.unpack_row(vb), vs, vz))
    ref = np.mean(vrows, axis=0) @ R[0].astype(np.float64).T
    assert np.allclose(out[0, 0], ref, atol=1e-12)


@pytest.mark.parametrize("mode,S,G", [(0, 0, 1), (0, 4, 4), (1, 0, 2), (1, 3, 1)])
def test_c_oracle_matches_numpy_mini_oracle(mode, S, G):
    """Two independent oracles: bit-exact codes and metadata from the same
    rotated fp32 rows, <= 1e-12 on the decoded output."""
    rng = np.random.default_rng(12 + mode + S)
    B, T, Hkv = 2, 41, 2
    Hq = Hkv * G
    K = (rng.standard_normal((B, T, Hkv, D)) * 3).astype(np.float16)
    V = rng.standard_normal((B, T, Hkv, D)).astype(np.float16)
    if mode == 0:
        Rk = np.stack([rand_orth(rng) for _ in range(Hkv)])
        Rv = np.stack([rand_orth(rng) for _ in range(Hkv)])
        perm = None
        kw = lambda h, kind: dict(R=(Rk if kind == 0 else Rv)[h])
    else:
        Rk = Rv = None
        perm = np.stack([np.stack([rng.permutation(D) for _ in range(Hkv)])
                         for _ in range(2)]).astype(np.int32)
        kw = lambda h, kind: dict(perm=perm[kind, h])
    cache = orc.Cache(B, Hkv, 48, S)
    sl = np.array([0, 5], np.int32)
    assert orc.append(cache, K.view(np.uint16), V.view(np.uint16), mode, Rk, Rv, perm, sl) == 0
    Q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    out, st = orc.decode(cache, Q.view(np.uint16), mode, Rk, Rv, perm, sl)
    assert st == 0
    for b in range(B):
        L0 = [0, 5][b]
        for h in range(Hkv):
            khat, vhat = [], []
            for kind, X in ((0, K), (1, V)):
                xr_c = orc.rotate_rows_f32(X[b, :, h].view(np.uint16), mode, **kw(h, kind))
                xr_n = np_mini.rotate_rows_f32(X[b, :, h], mode, **kw(h, kind))
                assert np.max(np.abs(xr_c - xr_n) / (np.abs(xr_n) + 1e-3)) < 1e-6
                codes, s, z = np_mini.quantize_rows(xr_c)
                rows = []
                for t in range(L0 + T):
                    p = t
                    if p < L0:                      # never written: zero block -> value 0
                        rows.append(np.zeros(D))
                        continue
                    if p < S:
                        rows.append(xr_c[p - L0].astype(np.float16).astype(np.float64))
                        continue
                    blk = cache.blocks[b, h, p // 16]
                    kb, vb, ks, kz, vs, vz = orc.load_token(blk, p % 16)
                    bb, ss, zz = (kb, ks, kz) if kind == 0 else (vb, vs, vz)
                    assert np.array_equal(orc.unpack_row(bb), codes[p - L0])
                    assert np.array_equal(ss, s[p - L0]) and np.array_equal(zz, z[p - L0])
                    rows.append(np_mini.dequant(codes[p - L0], s[p - L0], z[p - L0]))
                (khat if kind == 0 else vhat).append(np.array(rows))
            for hq in range(h * G, (h + 1) * G):
                ref = np_mini.decode_one(Q[b, hq], khat[0], vhat[0], mode,
                                         Rk[h] if mode == 0 else None,
                                         Rv[h] if mode == 0 else None,
                                         perm[0, h] if mode == 1 else None,
                                         perm[1, h] if mode == 1 else None)
                assert np.allclose(out[b, hq], ref, rtol=0, atol=1e-12)


def test_sinks_are_rotated_fp16_rows_and_leave_slots_zero():
    rng = np.random.default_rng(13)
    S, T = 4, 6
    R = np.stack([rand_orth(rng)])
    K = rng.standard_normal((1, T, 1, D)).astype(np.float16)
    V = rng.standard_normal((1, T, 1, D)).astype(np.float16)
    cache = orc.Cache(1, 1, 16, S)
    cache.blocks[:] = 0xAB
    sl = np.zeros(1, np.int32)
    orc.append(cache, K.view(np.uint16), V.view(np.uint16), 0, R, R, None, sl)
    kr = np_mini.rotate_rows_f32(K[0, :, 0], 0, R=R[0])
    assert np.array_equal(cache.k_sink[0, 0], kr[:S].astype(np.float16).view(np.uint16))
    for tau in range(S):
        fields = orc.load_token(cache.blocks[0, 0, 0], tau)
        assert all(not np.any(f) for f in fields)
    kb = orc.load_token(cache.blocks[0, 0, 0], S)[0]
    assert np.array_equal(orc.unpack_row(kb), np_mini.quantize_rows(kr[S:S + 1])[0][0])


def test_capacity_overflow_skips_sequence():
    rng = np.random.default_rng(14)
    cache = orc.Cache(2, 1, 16, 0)
    K = rng.standard_normal((2, 5, 1, D)).astype(np.float16)
    R = np.stack([np.eye(D, dtype=np.float32)])
    sl = np.array([12, 3], np.int32)
    st = orc.append(cache, K.view(np.uint16), K.view(np.uint16), 0, R, R, None, sl)
    assert st == orc.ST_CAPACITY
    assert list(sl) == [12, 8]
    assert not cache.blocks[0].any() and cache.blocks[1].any()


def test_decode_bad_length_gives_zero_and_status():
    cache = orc.Cache(2, 1, 16, 0)
    R = np.stack([np.eye(D, dtype=np.float32)])
    Q = np.ones((2, 1, D), np.float16).view(np.uint16)
    out, st = orc.decode(cache, Q, 0, R, R, None, np.array([0, 17], np.int32))
    assert st == orc.ST_BAD_LEN and not out.any()


# --- identified sinks (RotateKV abstract, item (iii)) -----------------------------------------

def _rot_inputs(rng, mode, Hkv):
    if mode == 0:
        Rk = np.stack([rand_orth(rng) for _ in range(Hkv)])
        Rv = np.stack([rand_orth(rng) for _ in range(Hkv)])
        return Rk, Rv, None
    perm = np.stack([np.stack([rng.permutation(D) for _ in range(Hkv)])
                     for _ in range(2)]).astype(np.int32)
    return None, None, perm


@pytest.mark.parametrize("mode,G", [(0, 2), (1, 1)])
def test_identified_sinks_equal_leading_sinks_of_the_reordered_sequence(mode, G):
    """Attention does not depend on the order of the positions and the
    quantizer works token by token, so a sequence whose identified sinks sit
    anywhere must give what the leading-sink layout gives for the same
    tokens reordered with the sinks first: the same fp16 rows, the same
    bytes for every INT2 token, and the same output up to the order of the
    fp64 sums.  Appended in three calls, so the position bookkeeping across
    calls is exercised; sequence 0 has more massive tokens than rows."""
    rng = np.random.default_rng(41 + mode)
    B, Hkv, S, cap = 3, 2, 3, 64
    Hq = Hkv * G
    chunks = [17, 1, 22]
    Ttot = sum(chunks)
    massive = [[2, 18, 30, 35], [0, 39], []]
    picks = [[2, 18, 30], [0, 39], []]
    K = (rng.standard_normal((B, Ttot, Hkv, D)) * 3).astype(np.float32)
    V = rng.standard_normal((B, Ttot, Hkv, D)).astype(np.float32)
    act = np.abs(rng.standard_normal((B, Ttot))).astype(np.float32)
    for b, ts in enumerate(massive):
        K[b, ts] *= 50
        act[b, ts] = 1000.0
    K = K.astype(np.float16)
    V = V.astype(np.float16)
    Rk, Rv, perm = _rot_inputs(rng, mode, Hkv)
    ic = orc.Cache(B, Hkv, cap, S, identified=True)
    sl = np.zeros(B, np.int32)
    t0 = 0
    for T in chunks:
        orc.identify_sinks(ic, act[:, t0:t0 + T], 100.0, sl)
        assert orc.append(ic, K[:, t0:t0 + T].view(np.uint16), V[:, t0:t0 + T].view(np.uint16),
                          mode, Rk, Rv, perm, sl) == 0
        t0 += T
    assert list(sl) == [Ttot] * B
    assert list(ic.sink_count) == [len(p) for p in picks]
    for b in range(B):
        assert list(ic.sink_pos[b, :len(picks[b])]) == picks[b]
    Q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    out, st = orc.decode(ic, Q.view(np.uint16), mode, Rk, Rv, perm, sl)
    assert st == 0
    for b in range(B):
        order = picks[b] + [t for t in range(Ttot) if t not in picks[b]]
        n = len(picks[b])
        lc = orc.Cache(1, Hkv, cap, n)
        sl1 = np.zeros(1, np.int32)
        assert orc.append(lc, K[b:b + 1, order].view(np.uint16), V[b:b + 1, order].view(np.uint16),
                          mode, Rk, Rv, perm, sl1) == 0
        assert np.array_equal(ic.k_sink[b, :, :n], lc.k_sink[0])
        assert np.array_equal(ic.v_sink[b, :, :n], lc.v_sink[0])
        assert not ic.k_sink[b, :, n:].any() and not ic.v_sink[b, :, n:].any()
        for h in range(Hkv):
            for pnew, p in enumerate(order):
                got = orc.load_token(ic.blocks[b, h, p // 16], p % 16)
                if pnew < n:
                    kb, vb, ks, kz, vs, vz = got
                    assert not kb.any() and not vb.any() and not kz.any()
                    assert not vs.any() and not vz.any()
                    assert list(ks) == [0x7E00] * 4          # the INT2 path's marker
                else:
                    exp = orc.load_token(lc.blocks[0, h, pnew // 16], pnew % 16)
                    assert all(np.array_equal(x, y) for x, y in zip(got, exp))
        ref, st1 = orc.decode(lc, Q[b:b + 1].view(np.uint16), mode, Rk, Rv, perm, sl1)
        assert st1 == 0
        assert np.allclose(out[b], ref[0], rtol=0, atol=1e-12)


def test_identified_sinks_with_threshold_minus_inf_are_the_leading_sinks():
    """tau = -inf marks every token: the first S positions get the rows, which
    is the leading-sink layout exactly (same rows, same INT2 bytes, same
    decode bit for bit); only the marker in the sinks' K meta differs."""
    rng = np.random.default_rng(43)
    B, Hkv, S, cap, T = 2, 1, 4, 48, 37
    K = rng.standard_normal((B, T, Hkv, D)).astype(np.float16)
    V = rng.standard_normal((B, T, Hkv, D)).astype(np.float16)
    Rk, Rv, _ = _rot_inputs(rng, 0, Hkv)
    ic = orc.Cache(B, Hkv, cap, S, identified=True)
    lc = orc.Cache(B, Hkv, cap, S)
    sl_i = np.zeros(B, np.int32)
    sl_l = np.zeros(B, np.int32)
    orc.identify_sinks(ic, np.zeros((B, T), np.float32), -np.inf, sl_i)
    orc.append(ic, K.view(np.uint16), V.view(np.uint16), 0, Rk, Rv, None, sl_i)
    orc.append(lc, K.view(np.uint16), V.view(np.uint16), 0, Rk, Rv, None, sl_l)
    assert list(ic.sink_count) == [S] * B
    assert np.array_equal(ic.sink_pos, np.tile(np.arange(S, dtype=np.int32), (B, 1)))
    assert np.array_equal(ic.k_sink, lc.k_sink) and np.array_equal(ic.v_sink, lc.v_sink)
    diff = ic.blocks != lc.blocks
    # the differing bytes are exactly the K-meta scale fields of the S sink slots
    exp = np.zeros_like(diff)
    for tau in range(S):
        r, th = tau % 8, tau // 8
        for g in range(4):
            off = 1024 + 8 * (4 * r + g) + 4 * th
            exp[:, :, 0, off + 1] = True                  # 0x7E00: high byte 0x7E, low byte 0
    assert np.array_equal(diff, exp)
    Q = rng.standard_normal((B, Hkv, D)).astype(np.float16).view(np.uint16)
    o_i, _ = orc.decode(ic, Q, 0, Rk, Rv, None, sl_i)
    o_l, _ = orc.decode(lc, Q, 0, Rk, Rv, None, sl_l)
    assert np.array_equal(o_i, o_l)


def test_identify_sinks_threshold_order_and_skips():
    """Ties count (act == tau), NaN never does, rows go to the earliest
    positions, the list continues across calls, and a sequence that the
    append would skip (no room for T tokens, or a negative length) gets no
    sink."""
    cache = orc.Cache(4, 1, 32, 2, identified=True)
    act = np.array([[1, 5, 5, 9],                   # tie at 5 counts: rows -> 1, 2
                    [np.nan, 4.99, 5, 7],           # NaN and 4.99 do not: rows -> 2, 3
                    [9, 9, 9, 9],                   # no room: 30 + 4 > 32
                    [9, 9, 9, 9]], np.float32)      # negative length
    sl = np.array([0, 0, 30, -1], np.int32)
    orc.identify_sinks(cache, act, 5.0, sl)
    assert list(cache.sink_count) == [2, 2, 0, 0]
    assert list(cache.sink_pos[0]) == [1, 2] and list(cache.sink_pos[1]) == [2, 3]
    assert list(sl) == [0, 0, 30, -1]                # lengths are the append's business
    # a later call continues at the current length and stops at S rows
    cache2 = orc.Cache(1, 1, 32, 3, identified=True)
    orc.identify_sinks(cache2, np.array([[0, 7, 0]], np.float32), 5.0, np.array([0], np.int32))
    orc.identify_sinks(cache2, np.array([[7, 7, 7]], np.float32), 5.0, np.array([3], np.int32))
    assert cache2.sink_count[0] == 3 and list(cache2.sink_pos[0]) == [1, 3, 4]


# --- pre-RoPE grouped-head rotation (RotateKV abstract, item (ii)) ----------------------------

@pytest.mark.parametrize("base", [10000.0, 500000.0])
def test_rope_is_the_complex_rotation(base):
    """RoPE against an independent complex-exponential formulation, plus two
    facts of any rotary embedding: it keeps norms, and q.k after RoPE at
    positions p and t depends on p - t only."""
    rng = np.random.default_rng(50)
    for t in (0, 1, 7, 4095, 131071):
        x = rng.standard_normal(D)
        got = orc.rope_f64(x, t, base)
        # theta_c from two pow() implementations may differ in the last bit,
        # which the angle t*theta_c scales by t
        assert np.allclose(got, np_mini.rope_complex(x, t, base), rtol=0, atol=1e-13 * (1 + t))
        assert abs(np.linalg.norm(got) - np.linalg.norm(x)) < 1e-12
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    for p, t in ((10, 3), (5000, 4990), (70000, 12)):
        lhs = orc.rope_f64(q, p, base) @ orc.rope_f64(k, t, base)
        assert abs(lhs - orc.rope_f64(q, p - t, base) @ k) < 1e-9
    # a pair is turned by exactly t*theta_c: channel 0 pairs with channel 64 at theta_0 = 1
    e0 = np.zeros(D)
    e0[0] = 1.0
    r = orc.rope_f64(e0, 3, base)
    assert abs(r[0] - np.cos(3.0)) < 1e-15 and abs(r[64] - np.sin(3.0)) < 1e-15
    assert np.count_nonzero(r) == 2


@pytest.mark.parametrize("gh", [1, 4])
def test_prerope_score_has_a_query_side_form(gh):
    """The pre-RoPE score needs no per-position un-rotation of the key: with
    k_hat the cached (group-rotated) key row, M the group rotation and x the
    head's slice of k_hat M^T, the RoPE'd score q . RoPE_t(x) equals
    sum_c cos(t theta_c) (k_hat . a_c) + sin(t theta_c) (k_hat . b_c), where
    a_c = q_c M[c] + q_{c+64} M[c+64] and b_c = q_{c+64} M[c] - q_c M[c+64]
    (rows of M at the head's offset) are fixed per query: RoPE's pairs
    (c, c+64) turn by t theta_c, and M is orthogonal."""
    rng = np.random.default_rng(31 + gh)
    n = D * gh
    M = np_mini.group_rotation_matrix(rng.permutation(n))
    j, base = gh - 1, 10000.0
    q = rng.standard_normal(D)
    khat = rng.standard_normal((6, n))
    ts = np.array([0, 1, 2, 17, 4096, 131071])
    direct = np.array([q @ np_mini.rope_complex((khat[i] @ M.T)[j * D:(j + 1) * D], t, base)
                       for i, t in enumerate(ts)])
    Mj = M[j * D:(j + 1) * D]                   # rows of the head's channels
    h = D // 2
    a = q[:h, None] * Mj[:h] + q[h:, None] * Mj[h:]
    b = q[h:, None] * Mj[:h] - q[:h, None] * Mj[h:]
    theta = np.power(base, -2.0 * np.arange(h) / D)
    query_side = np.array([np.cos(t * theta) @ (a @ khat[i]) + np.sin(t * theta) @ (b @ khat[i])
                           for i, t in enumerate(ts)])
    assert np.allclose(query_side, direct, rtol=1e-10, atol=1e-10)



@pytest.mark.parametrize("gh", [1, 2, 4, 8])
def test_group_rotation_is_the_permuted_hadamard_matrix(gh):
    n = D * gh
    rng = np.random.default_rng(51 + gh)
    perm = rng.permutation(n).astype(np.int32)
    x = rng.standard_normal(n)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    exp = H @ x[perm] / np.sqrt(n)
    got = orc.rotate_group_f64(x, perm)
    assert np.allclose(got, exp, rtol=0, atol=1e-12)
    assert np.allclose(orc.unrotate_group_f64(got, perm), x, rtol=0, atol=1e-12)


@pytest.mark.parametrize("gh,G", [(1, 1), (2, 2), (4, 1)])
def test_prerope_c_oracle_matches_numpy_mini_oracle(gh, G):
    """Append (pre-RoPE keys rotated per group of gh heads, values per head)
    and decode against the independent numpy oracle: codes and metadata
    bit-exact on the same rotated fp32 rows, outputs within 1e-12."""
    rng = np.random.default_rng(60 + gh + G)
    B, T, Hkv, base = 2, 41, 4, 10000.0
    Hq = Hkv * G
    n = D * gh
    K = (rng.standard_normal((B, T, Hkv, D)) * 3).astype(np.float16)
    V = rng.standard_normal((B, T, Hkv, D)).astype(np.float16)
    perm = np.concatenate([np.concatenate([rng.permutation(n) for _ in range(Hkv // gh)]),
                           np.concatenate([rng.permutation(D) for _ in range(Hkv)])]
                          ).astype(np.int32).reshape(2, Hkv * D)
    cache = orc.Cache(B, Hkv, 48, 0)
    L0 = [0, 5]
    sl = np.array(L0, np.int32)
    assert orc.append_prerope(cache, K.view(np.uint16), V.view(np.uint16), gh, perm, sl) == 0
    assert list(sl) == [T, 5 + T]
    Q = rng.standard_normal((B, Hq, D)).astype(np.float16)
    out, st = orc.decode_prerope(cache, Q.view(np.uint16), gh, perm, base, sl)
    assert st == 0
    for b in range(B):
        for q in range(Hkv // gh):
            pg = perm[0, q * n:(q + 1) * n]
            # rotated fp32 group rows of every appended token, numpy and C
            xg = K[b, :, q * gh:(q + 1) * gh].astype(np.float64).reshape(T, n)
            rot_n = (xg @ np_mini.group_rotation_matrix(pg)).astype(np.float32)
            rot_c = np.stack([orc.rotate_group_f64(xg[t], pg) for t in range(T)]).astype(np.float32)
            assert np.max(np.abs(rot_c - rot_n) / (np.abs(rot_n) + 1e-3)) < 1e-6
            khat = np.zeros((L0[b] + T, n))        # never-written positions decode to 0
            for jj in range(gh):
                h = q * gh + jj
                codes, s, z = np_mini.quantize_rows(rot_c[:, jj * D:(jj + 1) * D])
                vr = np_mini.rotate_rows_f32(V[b, :, h], 1, perm=perm[1, h * D:(h + 1) * D])
                vcodes = np_mini.quantize_rows(vr)[0]
                for t in range(T):
                    p = L0[b] + t
                    kb, vb, ks, kz, _, _ = orc.load_token(cache.blocks[b, h, p // 16], p % 16)
                    assert np.array_equal(orc.unpack_row(kb), codes[t])
                    assert np.array_equal(ks, s[t]) and np.array_equal(kz, z[t])
                    assert np.array_equal(orc.unpack_row(vb), vcodes[t])
                    khat[p, jj * D:(jj + 1) * D] = np_mini.dequant(codes[t], s[t], z[t])
            for jj in range(gh):
                h = q * gh + jj
                vhat = np.zeros((L0[b] + T, D))
                vr = np_mini.rotate_rows_f32(V[b, :, h], 1, perm=perm[1, h * D:(h + 1) * D])
                vcodes, vs, vz = np_mini.quantize_rows(vr)
                for t in range(T):
                    vhat[L0[b] + t] = np_mini.dequant(vcodes[t], vs[t], vz[t])
                for hq in range(h * G, (h + 1) * G):
                    ref = np_mini.decode_prerope_one(Q[b, hq], khat, jj, pg, base, vhat,
                                                     perm[1, h * D:(h + 1) * D])
                    assert np.allclose(out[b, hq], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("gh", [1, 2])
def test_prerope_all_sinks_is_fp16_attention_with_rope(gh):
    """With every position a sink nothing is quantized: the decode must be
    the attention over the stored fp16 rows, keys RoPE'd at their positions
    (complex-exponential formulation), softmax from scipy, values rotated
    back through the explicit permuted Hadamard matrix.  The sink rows must
    hold the pre-RoPE keys exactly as given."""
    rng = np.random.default_rng(70 + gh)
    B, T, Hkv, G, base = 2, 13, 2 * gh, 2, 10000.0
    n = D * gh
    K = (rng.standard_normal((B, T, Hkv, D)) * 2).astype(np.float16)
    V = rng.standard_normal((B, T, Hkv, D)).astype(np.float16)
    perm = np.concatenate([np.concatenate([rng.permutation(n) for _ in range(Hkv // gh)]),
                           np.concatenate([rng.permutation(D) for _ in range(Hkv)])]
                          ).astype(np.int32).reshape(2, Hkv * D)
    cache = orc.Cache(B, Hkv, 32, 16)
    sl = np.zeros(B, np.int32)
    assert orc.append_prerope(cache, K.view(np.uint16), V.view(np.uint16), gh, perm, sl) == 0
    assert np.array_equal(cache.k_sink[:, :, :T], K.transpose(0, 2, 1, 3).view(np.uint16))
    assert not cache.blocks.any()                         # no INT2 token, nothing written there
    Q = rng.standard_normal((B, Hkv * G, D)).astype(np.float16)
    out, st = orc.decode_prerope(cache, Q.view(np.uint16), gh, perm, base, sl)
    assert st == 0
    for b in range(B):
        for h in range(Hkv):
            pv = perm[1, h * D:(h + 1) * D]
            vr = np_mini.rotate_rows_f32(V[b, :, h], 1, perm=pv)
            # the stored value rows are the fp16 rounding of the rotated rows
            vs = cache.v_sink[b, h, :T].view(np.float16).astype(np.float64)
            assert np.max(np.abs(vs - vr.astype(np.float16).astype(np.float64))) <= \
                np.max(np.abs(vs)) * 2.0 ** -10
            k = np.stack([np_mini.rope_complex(K[b, t, h].astype(np.float64), t, base)
                          for t in range(T)])
            for hq in range(h * G, (h + 1) * G):
                sc = k @ Q[b, hq].astype(np.float64) / np.sqrt(D)
                p = scipy.special.softmax(sc)
                ref = (p @ vs) @ np_mini.rotation_matrix(1, perm=pv).T
                assert np.allclose(out[b, hq], ref, rtol=0, atol=1e-12)


def test_prerope_identified_sinks_threshold_minus_inf_are_the_leading_sinks():
    rng = np.random.default_rng(75)
    B, T, Hkv, gh, S = 2, 40, 2, 2, 4
    K = (rng.standard_normal((B, T, Hkv, D)) * 2).astype(np.float16)
    V = rng.standard_normal((B, T, Hkv, D)).astype(np.float16)
    perm = np.concatenate([rng.permutation(D * gh), np.concatenate(
        [rng.permutation(D) for _ in range(Hkv)])]).astype(np.int32).reshape(2, Hkv * D)
    ic = orc.Cache(B, Hkv, 48, S, identified=True)
    lc = orc.Cache(B, Hkv, 48, S)
    sl_i = np.zeros(B, np.int32)
    sl_l = np.zeros(B, np.int32)
    orc.identify_sinks(ic, np.zeros((B, T), np.float32), -np.inf, sl_i)
    orc.append_prerope(ic, K.view(np.uint16), V.view(np.uint16), gh, perm, sl_i)
    orc.append_prerope(lc, K.view(np.uint16), V.view(np.uint16), gh, perm, sl_l)
    assert np.array_equal(ic.k_sink, lc.k_sink) and np.array_equal(ic.v_sink, lc.v_sink)
    Q = rng.standard_normal((B, Hkv, D)).astype(np.float16).view(np.uint16)
    o_i, _ = orc.decode_prerope(ic, Q, gh, perm, 10000.0, sl_i)
    o_l, _ = orc.decode_prerope(lc, Q, gh, perm, 10000.0, sl_l)
    assert np.array_equal(o_i, o_l)


def test_prerope_identified_sinks_match_numpy_mini_oracle():
    """Identified sinks at positions that are not their row numbers, in a
    pre-RoPE cache: every sink is RoPE'd at its own position from its stored
    pre-RoPE key, every other position from its dequantised, un-rotated
    group row (independent numpy oracle), to 1e-12."""
    rng = np.random.default_rng(77)
    B, T, Hkv, gh, G, S, base = 1, 30, 2, 2, 1, 3, 10000.0
    n = D * gh
    K = (rng.standard_normal((B, T, Hkv, D)) * 2).astype(np.float16)
    V = rng.standard_normal((B, T, Hkv, D)).astype(np.float16)
    perm = np.concatenate([rng.permutation(n), np.concatenate(
        [rng.permutation(D) for _ in range(Hkv)])]).astype(np.int32).reshape(2, Hkv * D)
    cache = orc.Cache(B, Hkv, 32, S, identified=True)
    act = np.zeros((B, T), np.float32)
    act[0, [4, 17, 23, 29]] = 1.0                   # four massive tokens, three rows
    sl = np.zeros(B, np.int32)
    orc.identify_sinks(cache, act, 0.5, sl)
    assert list(cache.sink_pos[0]) == [4, 17, 23]
    assert orc.append_prerope(cache, K.view(np.uint16), V.view(np.uint16), gh, perm, sl) == 0
    Q = rng.standard_normal((B, Hkv * G, D)).astype(np.float16)
    out, st = orc.decode_prerope(cache, Q.view(np.uint16), gh, perm, base, sl)
    assert st == 0
    sinks = [4, 17, 23]
    khat = np.zeros((T, n))
    for t in range(T):
        if t in sinks:
            continue
        for jj in range(gh):
            kb, vb, ks, kz, vs, vz = orc.load_token(cache.blocks[0, jj, t // 16], t % 16)
            khat[t, jj * D:(jj + 1) * D] = np_mini.dequant(orc.unpack_row(kb), ks, kz)
    for h in range(Hkv):
        pv = perm[1, h * D:(h + 1) * D]
        vhat = np.zeros((T, D))
        for t in range(T):
            kb, vb, ks, kz, vs, vz = orc.load_token(cache.blocks[0, h, t // 16], t % 16)
            if t in sinks:
                vhat[t] = cache.v_sink[0, h, sinks.index(t)].view(np.float16).astype(np.float64)
                assert list(ks) == [0x7E00] * 4 and not kb.any()
            else:
                vhat[t] = np_mini.dequant(orc.unpack_row(vb), vs, vz)
        keys = {t: K[0, t, h].astype(np.float64) for t in sinks}
        ref = np_mini.decode_prerope_one(Q[0, h], khat, h, perm[0], base, vhat, pv, keys)
        assert np.allclose(out[0, h], ref, rtol=0, atol=1e-12)


# --- KVLinC key correction adapters --------------------------------------------------------

def _adapter_case(mode, S, G, r, seed, T=45):
    rng = np.random.default_rng(seed)
    B, Hkv = 2, 2
    K = (rng.standard_normal((B, T, Hkv, D)) * 2).astype(np.float16)
    V = rng.standard_normal((B, T, Hkv, D)).astype(np.float16)
    if mode == 0:
        Rk = np.stack([rand_orth(rng) for _ in range(Hkv)])
        Rv = np.stack([rand_orth(rng) for _ in range(Hkv)])
        perm = None
    else:
        Rk = Rv = None
        perm = np.stack([np.stack([rng.permutation(D) for _ in range(Hkv)])
                         for _ in range(2)]).astype(np.int32)
    cache = orc.Cache(B, Hkv, 48, S)
    sl = np.zeros(B, np.int32)
    assert orc.append(cache, K.view(np.uint16), V.view(np.uint16), mode, Rk, Rv, perm, sl) == 0
    lens = np.array([T, T - 7], np.int32)
    Q = rng.standard_normal((B, Hkv * G, D)).astype(np.float16)
    U = (rng.standard_normal((Hkv, D, r)) * 0.1).astype(np.float32)
    Vd = (rng.standard_normal((Hkv, D, r)) * 0.1).astype(np.float32)
    return K, V, Q, cache, lens, Rk, Rv, perm, U, Vd


@pytest.mark.parametrize("mode,S,G,r", [(0, 0, 1, 8), (0, 4, 2, 128), (1, 0, 1, 1), (1, 3, 4, 16)])
def test_adapter_decode_equals_attention_with_corrected_keys(mode, S, G, r):
    """The key correction adapter, written out with explicit matrices in
    numpy: every INT2 key, dequantised (numpy mini-oracle) and taken back to
    the model's basis, becomes k^ + (k^ . U) . V^T; fp16 sink keys stay as
    stored; then plain softmax attention and the value rotation removed.  A
    swapped U and V, a correction in the rotated basis or one applied to the
    sinks would each fail this."""
    K, V, Q, cache, lens, Rk, Rv, perm, U, Vd = _adapter_case(mode, S, G, r, 60 + r + S)
    out, st = orc.decode_adapter(cache, Q.view(np.uint16), mode, Rk, Rv, perm, lens, U, Vd)
    assert st == 0
    B, T, Hkv = K.shape[:3]
    for b in range(B):
        L = int(lens[b])
        for h in range(Hkv):
            kw = (lambda kind: dict(R=(Rk if kind == 0 else Rv)[h])) if mode == 0 else \
                (lambda kind: dict(perm=perm[kind, h]))
            Mk = np_mini.rotation_matrix(mode, **kw(0))
            Mv = np_mini.rotation_matrix(mode, **kw(1))
            kr = np_mini.rotate_rows_f32(K[b, :L, h], mode, **kw(0))
            vr = np_mini.rotate_rows_f32(V[b, :L, h], mode, **kw(1))
            kc, ks, kz = np_mini.quantize_rows(kr)
            vc, vs, vz = np_mini.quantize_rows(vr)
            khat = np_mini.dequant(kc, ks, kz)
            vhat = np_mini.dequant(vc, vs, vz)
            sink = np.arange(L) < S
            khat[sink] = kr[sink].astype(np.float16).astype(np.float64)
            vhat[sink] = vr[sink].astype(np.float16).astype(np.float64)
            kmodel = khat @ Mk.T                           # back to the model's basis
            kcorr = kmodel + (kmodel @ U[h].astype(np.float64)) @ Vd[h].astype(np.float64).T
            kcorr[sink] = kmodel[sink]
            for hq in range(h * G, (h + 1) * G):
                q = Q[b, hq].astype(np.float64)
                s = kcorr @ q / np.sqrt(D)
                p = np.exp(s - s.max())
                ref = (p / p.sum()) @ vhat @ Mv.T
                assert np.allclose(out[b, hq], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", [0, 1])
def test_zero_adapter_is_the_plain_decode(mode):
    K, V, Q, cache, lens, Rk, Rv, perm, U, Vd = _adapter_case(mode, 4, 2, 8, 71)
    plain, _ = orc.decode(cache, Q.view(np.uint16), mode, Rk, Rv, perm, lens)
    for zu, zv in ((np.zeros_like(U), Vd), (U, np.zeros_like(Vd))):
        out, st = orc.decode_adapter(cache, Q.view(np.uint16), mode, Rk, Rv, perm, lens, zu, zv)
        assert st == 0
        assert np.allclose(out, plain, rtol=0, atol=1e-12)
    # a context made of fp16 sinks only has no quantized key to correct
    short = np.array([3, 2], np.int32)
    plain, _ = orc.decode(cache, Q.view(np.uint16), mode, Rk, Rv, perm, short)
    out, _ = orc.decode_adapter(cache, Q.view(np.uint16), mode, Rk, Rv, perm, short, U, Vd)
    assert np.array_equal(out, plain)
