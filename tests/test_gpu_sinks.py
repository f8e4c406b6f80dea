"""Identified attention sinks ("RotateKV", abstract item (iii): the sinks are
singled out by their massive activations and kept out of the 2-bit code):
the CUDA path through the C ABI against the CPU oracle.
  - sink lists (positions, counts): bit-exact;
  - cache bytes: every INT2 token bit-exact with the same token appended to a
    cache without sinks (same kernels, same rotated rows); every sink row the
    fp16 rounding of the kernel's rotated row, its INT2 slot the marker;
  - decode: max-abs error <= 2e-3 * ||o_ref||_2 per (sequence, head), as for
    the leading sinks.
"""
import numpy as np
import pytest
import torch

import rotated_int2_kv_head_b200 as kvq
import workloads as W
from oracle import oracle as orc

from kvq_testlib import (D, append_variant, f16bits, gpu_append, gpu_decode, rel_err, rot_tensors,
                         upload_oracle_cache)

pytestmark = pytest.mark.gpu
DEC_TOL = 2e-3
TAU = W.MASSIVE_TAU


@pytest.fixture(scope="module", autouse=True)
def built():
    from rotated_int2_kv_head_b200 import build
    build.build()
    torch.cuda.init()


def _act(rng, B, T, rate, extra=()):
    a = np.abs(rng.standard_normal((B, T))).astype(np.float32)
    a[rng.random((B, T)) < rate] = 1000.0
    for b, t in extra:
        a[b, t] = 1000.0
    return a


# --- identification ------------------------------------------------------------------------

def test_identify_sinks_matches_oracle():
    """Several calls of different sizes, including one of 40000 tokens (two
    passes of the kernel) whose only massive tokens sit in the second pass,
    ties at tau, NaN, a sequence without room for the tokens and one with a
    negative length."""
    rng = np.random.default_rng(5)
    B, S, cap = 6, 8, 45056
    gc = kvq.KVCache(B, 1, cap, S, identified_sinks=True)
    oc = orc.Cache(B, 1, cap, S, identified=True)
    lens = np.array([0, 3, 0, 44000, -1, 0], np.int32)
    for T in (1, 37, 300, 1, 2500, 40000):
        act = _act(rng, B, T, 2e-3 if T < 40000 else 0.0)
        act[5] = 0.5                             # sequence 5: massive tokens only at the end
        if T == 37:
            act[0, 5] = TAU                      # a tie counts
            act[1, 6] = np.nan                   # NaN never does
        if T == 40000:
            act[5, 33000] = act[5, 39999] = 1000.0   # second pass only
        if lens[0] + T > cap:
            break
        sl = torch.from_numpy(lens).cuda()
        kvq.kvq_identify_sinks(torch.from_numpy(act).cuda(), TAU, gc, sl)
        orc.identify_sinks(oc, act, TAU, lens)
        torch.cuda.synchronize()
        assert np.array_equal(gc.sink_count.cpu().numpy(), oc.sink_count), T
        assert np.array_equal(gc.sink_pos.cpu().numpy(), oc.sink_pos), T
        # the lengths move with the append, not here; advance them by hand
        ok = (lens >= 0) & (lens + T <= cap)
        lens = np.where(ok, lens + T, lens).astype(np.int32)
    assert oc.sink_count[4] == 0
    assert list(oc.sink_pos[5][:oc.sink_count[5]]) == [2839 + 33000, 2839 + 39999]


# --- append -----------------------------------------------------------------------------------

def _grot(w, rt, X, h, kind, variant):
    rows = X[:, :, h].reshape(-1, D).cuda()
    if w.mode == 0:
        R = (rt[0] if kind == 0 else rt[1])[h].contiguous()
        return kvq.kvq_debug_rotate_f32(rows, 0, R=R, variant=variant).cpu().numpy()
    return kvq.kvq_debug_rotate_f32(rows, 1, perm=rt[2][kind, h].contiguous(),
                                    variant=variant).cpu().numpy()


@pytest.mark.parametrize("mode,chunks,paged", [
    (0, [37, 1, 70], False),           # CUDA-core dense kernel
    (0, [300, 1, 520], False),         # tensor-core bulk kernel
    (1, [37, 1, 130], False),          # permutation + FWHT: CUDA-core, then tensor-core kernel
    (0, [300, 37, 1], True),           # both dense kernels on a paged cache
])
def test_append_identified_sinks(mode, chunks, paged):
    B, Hkv, S = 3, 2, 4
    cap = ((sum(chunks) + 15) // 16) * 16 + 32
    w = W.custom(seed=120 + mode + len(chunks) + 7 * paged, B=B, Hq=2 * Hkv, Hkv=Hkv, mode=mode,
                 sink=S, k_outliers=4, sink_key_scale=50.0, massive_rate=0.02,
                 channel_scale=(0.5, 20.0) if mode == 1 else None)
    rt, rn = rot_tensors(w)
    if paged:
        nblk = cap // 16
        num_blocks = B * nblk + 5
        perm = torch.randperm(num_blocks, generator=torch.Generator().manual_seed(4))[:B * nblk]
        table = perm.view(B, nblk).to(torch.int32).cuda()
        ic = kvq.PagedKVCache(B, Hkv, cap, num_blocks, table, S, identified_sinks=True)
        plain = kvq.PagedKVCache(B, Hkv, cap, num_blocks, table, 0)
    else:
        ic = kvq.KVCache(B, Hkv, cap, S, identified_sinks=True)
        plain = kvq.KVCache(B, Hkv, cap, 0)
    oc = orc.Cache(B, Hkv, cap, S, identified=True)
    L0 = [0, 3, 16]
    sl_i = torch.tensor(L0, dtype=torch.int32, device="cuda")
    sl_p = sl_i.clone()
    osl = np.array(L0, np.int32)
    pos = list(L0)
    rows = []                              # (chunk start per b, K, V, variant) per call
    for T in chunks:
        K = torch.stack([W.kv_rows(w, b, pos[b], pos[b] + T, "cpu")[0] for b in range(B)])
        V = torch.stack([W.kv_rows(w, b, pos[b], pos[b] + T, "cpu")[1] for b in range(B)])
        act = np.stack([W.activations(w, b, pos[b], pos[b] + T) for b in range(B)])
        kvq.kvq_identify_sinks(torch.from_numpy(act).cuda(), TAU, ic, sl_i)
        gpu_append(ic, K.cuda(), V.cuda(), w, rt, sl_i)
        gpu_append(plain, K.cuda(), V.cuda(), w, rt, sl_p)
        orc.identify_sinks(oc, act, TAU, osl)
        assert orc.append(oc, f16bits(K), f16bits(V), w.mode, rn[0], rn[1], rn[2], osl) == 0
        rows.append((list(pos), K, V, append_variant(mode, T, B)))
        pos = [p + T for p in pos]
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(ic) == 0 and kvq.kvq_get_status(plain) == 0
    assert list(sl_i.cpu().numpy()) == list(osl) == pos
    assert np.array_equal(ic.sink_count.cpu().numpy(), oc.sink_count)
    assert np.array_equal(ic.sink_pos.cpu().numpy(), oc.sink_pos)
    assert (oc.sink_count >= 1).all() and (oc.sink_count == S).any()
    gi = ic.logical_view().cpu().numpy() if paged else ic.block_view().cpu().numpy()
    gp = plain.logical_view().cpu().numpy() if paged else plain.block_view().cpu().numpy()
    gks, gvs = f16bits(ic.k_sink), f16bits(ic.v_sink)
    n_sink = 0
    for starts, K, V, variant in rows:
        T = K.shape[1]
        for kind, X in ((0, K), (1, V)):
            for h in range(Hkv):
                grot = _grot(w, rt, X, h, kind, variant).reshape(B, T, D)
                for b in range(B):
                    plist = list(oc.sink_pos[b, :oc.sink_count[b]])
                    for t in range(T):
                        p = starts[b] + t
                        blk_i = gi[b, h, p // 16]
                        if p in plist:
                            j = plist.index(p)
                            sink = (gks if kind == 0 else gvs)[b, h, j]
                            assert np.array_equal(sink, orc.f32_to_f16_bits(grot[b, t]))
                            kb, vb, ks, kz, vs, vz = orc.load_token(blk_i, p % 16)
                            assert not kb.any() and not vb.any() and not kz.any()
                            assert not vs.any() and not vz.any()
                            assert list(ks) == [0x7E00] * 4
                            n_sink += 1
                        else:
                            got = orc.load_token(blk_i, p % 16)
                            exp = orc.load_token(gp[b, h, p // 16], p % 16)
                            assert all(np.array_equal(x, y) for x, y in zip(got, exp))
    assert n_sink > 0
    # the decode over this cache against the oracle's decode over its own cache
    Q = W.queries(w, "cpu")
    ref, st = orc.decode(oc, f16bits(Q), mode, rn[0], rn[1], rn[2], osl, n_threads=8)
    assert st == 0
    out = gpu_decode(ic, Q.cuda(), w, rt, sl_i, max(pos))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(ic) == 0
    err = rel_err(out.cpu().numpy(), ref)
    assert err.max() <= DEC_TOL, err.max()


# --- decode -----------------------------------------------------------------------------------

def oracle_identified_cache(w, lens, cap, chunk=700):
    """The oracle identifies and appends every sequence's tokens [0, lens[b])
    in chunks, so that the sink list builds up across calls."""
    _, rn = rot_tensors(w)
    oc = orc.Cache(w.B, w.Hkv, cap, w.sink, identified=True)
    for b in range(w.B):
        sub = orc.Cache(1, w.Hkv, cap, w.sink, identified=True)
        sl = np.zeros(1, np.int32)
        for t0 in range(0, lens[b], chunk):
            t1 = min(lens[b], t0 + chunk)
            k, v = W.kv_rows(w, b, t0, t1, "cpu")
            orc.identify_sinks(sub, W.activations(w, b, t0, t1)[None], TAU, sl)
            orc.append(sub, f16bits(k[None]), f16bits(v[None]), w.mode, rn[0], rn[1], rn[2], sl)
        oc.blocks[b] = sub.blocks[0]
        oc.k_sink[b] = sub.k_sink[0]
        oc.v_sink[b] = sub.v_sink[0]
        oc.sink_pos[b] = sub.sink_pos[0]
        oc.sink_count[b] = sub.sink_count[0]
    return oc


ID_DECODE_CASES = [
    # G, mode, S, rate, lengths
    (1, 0, 4, 0.01, [1, 2, 17, 300, 1500]),
    (4, 0, 4, 0.003, [16, 33, 257, 2100]),
    (2, 1, 8, 0.01, [5, 100, 1024]),
    (8, 0, 2, 0.05, [3, 64, 800]),
]


@pytest.mark.parametrize("G,mode,S,rate,lens", ID_DECODE_CASES)
def test_decode_identified_sinks_matches_oracle(G, mode, S, rate, lens):
    Hkv = 2
    w = W.custom(seed=140 + G + S, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=mode, sink=S,
                 k_outliers=6, sink_key_scale=50.0, massive_rate=rate)
    cap = ((max(lens) + 15) // 16) * 16
    oc = oracle_identified_cache(w, lens, cap)
    assert (oc.sink_count >= 1).all()
    rt, rn = rot_tensors(w)
    Q = W.queries(w, "cpu")
    sl = np.array(lens, np.int32)
    ref, st = orc.decode(oc, f16bits(Q), mode, rn[0], rn[1], rn[2], sl, n_threads=8)
    assert st == 0
    cache = upload_oracle_cache(oc)
    out = gpu_decode(cache, Q.cuda(), w, rt, torch.from_numpy(sl).cuda(), max(lens))
    err = rel_err(out.cpu().numpy(), ref)
    assert err.max() <= DEC_TOL, err.max()
    assert kvq.kvq_get_status(cache) == 0


def test_multi_query_decode_identified_sinks():
    """q_len = 4 new tokens per sequence with sinks among the new tokens:
    query i must see the sinks at positions <= L - 4 + i only."""
    Hkv, G, q_len, S = 2, 1, 4, 4
    lens = [6, 40, 515]
    w = W.custom(seed=151, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=0, sink=S, k_outliers=4,
                 sink_key_scale=50.0, massive_rate=0.0)
    cap = ((max(lens) + 15) // 16) * 16
    rt, rn = rot_tensors(w)
    oc = orc.Cache(w.B, Hkv, cap, S, identified=True)
    for b, L in enumerate(lens):
        sub = orc.Cache(1, Hkv, cap, S, identified=True)
        sl1 = np.zeros(1, np.int32)
        k, v = W.kv_rows(w, b, 0, L, "cpu")
        act = np.zeros((1, L), np.float32)
        act[0, [0, L - 3, L - 1]] = 1000.0       # sinks: first token and two of the new ones
        orc.identify_sinks(sub, act, TAU, sl1)
        orc.append(sub, f16bits(k[None]), f16bits(v[None]), 0, rn[0], rn[1], None, sl1)
        oc.blocks[b], oc.k_sink[b], oc.v_sink[b] = sub.blocks[0], sub.k_sink[0], sub.v_sink[0]
        oc.sink_pos[b], oc.sink_count[b] = sub.sink_pos[0], sub.sink_count[0]
    cache = upload_oracle_cache(oc)
    g = torch.Generator().manual_seed(77)
    Q = torch.randn((w.B, w.Hq, q_len, D), generator=g).to(torch.float16)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = kvq.decode_workspace(w.B, w.Hq * q_len, Hkv, max(lens))
    ws.fill_(0xFF)
    out = torch.empty_like(Q).cuda()
    kvq.kvq_decode_attention_ex(Q.cuda(), cache, 0, rt[0], rt[1], None, sl, S, max(lens), ws, out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    got = out.cpu().numpy()
    for i in range(q_len):
        li = np.array(lens, np.int32) - (q_len - 1 - i)
        ref, st = orc.decode(oc, f16bits(Q[:, :, i].contiguous()), 0, rn[0], rn[1], None, li,
                             n_threads=8)
        assert st == 0
        err = rel_err(got[:, :, i], ref)
        assert err.max() <= DEC_TOL, (i, err.max())
