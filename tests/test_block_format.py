"""The oracle's block layout against the documented block format, read and
written by tests/block_format.py (a vectorised implementation of the format
as include/kvq.h states it, sharing no code with the oracle or the kernels).
CPU only; the GPU side is in test_gpu_parity.py
(test_gpu_cache_reads_as_documented)."""
import numpy as np

import workloads as W
from oracle import oracle as orc
from tests import block_format as bf

D = 128


def test_format_offsets_are_a_bijection_onto_the_block():
    used = np.concatenate([bf.K_IDX.ravel(), bf.V_IDX.ravel(), bf.KM_IDX.ravel(), bf.VM_IDX.ravel()])
    assert used.size == bf.BLK_BYTES
    assert np.array_equal(np.sort(used), np.arange(bf.BLK_BYTES))


def test_documented_writer_reads_back_through_the_oracle():
    """Random logical content written by the documented format is what the
    oracle's token reader returns, token by token."""
    rng = np.random.default_rng(11)
    for _ in range(20):
        k = rng.integers(0, 4, (16, D))
        v = rng.integers(0, 4, (16, D))
        ks, kz, vs, vz = (rng.integers(0, 1 << 16, (16, 4)).astype(np.uint16) for _ in range(4))
        blk = bf.write_block(k, v, ks, kz, vs, vz)
        for tau in range(16):
            kb, vb, oks, okz, ovs, ovz = orc.load_token(blk, tau)
            assert np.array_equal(orc.unpack_row(kb), k[tau])
            assert np.array_equal(orc.unpack_row(vb), v[tau])
            for a, b in ((oks, ks), (okz, kz), (ovs, vs), (ovz, vz)):
                assert np.array_equal(a, b[tau])


def test_oracle_writer_reads_back_through_the_documented_format():
    """Tokens the oracle stores (orc_store_token) read back unchanged through
    the documented format."""
    rng = np.random.default_rng(12)
    blk = np.zeros(bf.BLK_BYTES, np.uint8)
    k = rng.integers(0, 4, (16, D))
    v = rng.integers(0, 4, (16, D))
    ks, kz, vs, vz = (rng.integers(0, 1 << 16, (16, 4)).astype(np.uint16) for _ in range(4))
    for tau in rng.permutation(16):
        orc.store_token(blk, int(tau), orc.pack_row(k[tau]), orc.pack_row(v[tau]), ks[tau], kz[tau],
                        vs[tau], vz[tau])
    got = bf.read_blocks(blk)
    assert np.array_equal(got["k"], k) and np.array_equal(got["v"], v)
    for name, ref in (("ks", ks), ("kz", kz), ("vs", vs), ("vz", vz)):
        assert np.array_equal(got[name], ref)


def test_logical_packing_matches_the_oracle():
    rng = np.random.default_rng(13)
    codes = rng.integers(0, 4, (64, D))
    for row in codes:
        assert np.array_equal(bf.pack_codes(row), orc.pack_row(row))
        assert np.array_equal(bf.unpack_codes(orc.pack_row(row)), row)


def test_oracle_append_reads_as_documented():
    """A whole cache appended by the oracle (dense and FWHT rotations, a
    ragged batch across block boundaries): every token read through the
    documented format equals the oracle's own logical view of it."""
    for mode in (0, 1):
        w = W.custom(name="fmt", seed=40 + mode, B=2, Hq=2, Hkv=2, mode=mode, context=70,
                     k_outliers=2)
        Rk, Rv, perm = W.rotations(w)
        oc = orc.Cache(w.B, w.Hkv, 80, 0)
        sl = np.array([0, 5], np.int32)
        K, V = W.kv_batch(w, 0, 70, "cpu")
        assert orc.append(oc, W.f16_bits(K), W.f16_bits(V), mode, Rk, Rv, perm, sl) == 0
        got = bf.read_blocks(oc.blocks)          # [B][Hkv][nblk][16] ...
        for b in range(w.B):
            for h in range(w.Hkv):
                for p in range(int(sl[b])):
                    kb, vb, ks, kz, vs, vz = orc.load_token(oc.blocks[b, h, p // 16], p % 16)
                    blk, tau = p // 16, p % 16
                    assert np.array_equal(got["k"][b, h, blk, tau], orc.unpack_row(kb))
                    assert np.array_equal(got["v"][b, h, blk, tau], orc.unpack_row(vb))
                    assert np.array_equal(got["ks"][b, h, blk, tau], ks)
                    assert np.array_equal(got["kz"][b, h, blk, tau], kz)
                    assert np.array_equal(got["vs"][b, h, blk, tau], vs)
                    assert np.array_equal(got["vz"][b, h, blk, tau], vz)
