"""Pre-RoPE grouped-head key rotation ("RotateKV", abstract item (ii)): the
CUDA path through the C ABI against the CPU oracle.
  - group rotation: max-abs error <= 1e-5 of the row's largest value;
  - cache bytes: bit-exact when both sides quantize the same rotated fp32 rows
    (the kernel's own rotation, from the test export); against the oracle's
    own fp64 rotation, <= 1e-4 of the code elements differ, each at a near tie;
  - decode output: max-abs error <= 2e-3 * ||o_ref||_2 per (sequence, head).
"""
import numpy as np
import pytest
import torch

import rotated_int2_kv_head_b200 as kvq
import workloads as W
from oracle import oracle as orc

from kvq_testlib import D, f16bits, logical, near_tie_ok, rel_err

pytestmark = pytest.mark.gpu
DEC_TOL = 2e-3
BASE = 10000.0


@pytest.fixture(scope="module", autouse=True)
def built():
    from rotated_int2_kv_head_b200 import build
    build.build()
    torch.cuda.init()


def _wl(seed, B, Hkv, G, k_outliers=6):
    return W.custom(seed=seed, B=B, Hq=Hkv * G, Hkv=Hkv, mode=1, k_outliers=k_outliers)


@pytest.mark.parametrize("gh", [1, 2, 4, 8])
def test_group_rotation_matches_oracle(gh):
    n = D * gh
    rng = np.random.default_rng(200 + gh)
    X = (rng.standard_normal((300, n)) * rng.uniform(0.1, 30, (1, n))).astype(np.float16)
    perm = rng.permutation(n).astype(np.int32)
    got = kvq.kvq_debug_rotate_group_f32(torch.from_numpy(X).cuda(), gh,
                                         torch.from_numpy(perm).cuda()).cpu().numpy()
    for r in range(X.shape[0]):
        ref = orc.rotate_group_f64(X[r].astype(np.float64), perm)
        assert np.max(np.abs(got[r] - ref)) <= 1e-5 * np.max(np.abs(ref)), r


@pytest.mark.parametrize("gh,T,L0,paged", [
    (1, 1, [0, 5, 16], False),
    (2, 37, [0, 3, 29], False),
    (4, 300, [0, 7, 16], False),
    (8, 20, [1, 0, 40], False),
    (2, 37, [0, 3, 29], True),
])
def test_prerope_append_matches_oracle(gh, T, L0, paged):
    Hkv = 8 if gh == 8 else 4
    B = 3
    w = _wl(210 + gh + T, B, Hkv, 1)
    perm = W.prerope_perm(w, gh)
    K = torch.stack([W.kv_rows(w, b, L0[b], L0[b] + T, "cpu")[0] for b in range(B)])
    V = torch.stack([W.kv_rows(w, b, L0[b], L0[b] + T, "cpu")[1] for b in range(B)])
    cap = ((max(L0) + T + 15) // 16) * 16 + 16
    nblk = cap // 16
    if paged:
        num_blocks = B * nblk + 3
        tperm = torch.randperm(num_blocks, generator=torch.Generator().manual_seed(9))[:B * nblk]
        table = tperm.view(B, nblk).to(torch.int32).cuda()
        cache = kvq.PagedKVCache(B, Hkv, cap, num_blocks, table)
    else:
        cache = kvq.KVCache(B, Hkv, cap)
    sl = torch.tensor(L0, dtype=torch.int32, device="cuda")
    pt = torch.from_numpy(perm).cuda()
    kvq.kvq_prerope_append(K.cuda(), V.cuda(), gh, pt, cache, sl)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    assert list(sl.cpu().numpy()) == [l + T for l in L0]
    gblocks = (cache.logical_view() if paged else cache.block_view()).cpu().numpy()
    gc = orc.Cache(B, Hkv, cap, 0)
    gc.blocks[:] = gblocks
    oc = orc.Cache(B, Hkv, cap, 0)
    osl = np.array(L0, np.int32)
    assert orc.append_prerope(oc, f16bits(K), f16bits(V), gh, perm, osl) == 0
    n_codes = n_diff = 0
    for q in range(Hkv // gh):
        pg = perm[0, q * D * gh:(q + 1) * D * gh]
        rows = K[:, :, q * gh:(q + 1) * gh].reshape(B * T, D * gh).contiguous()
        grot = kvq.kvq_debug_rotate_group_f32(rows.cuda(), gh, torch.from_numpy(pg).cuda())
        grot = grot.cpu().numpy().reshape(B, T, D * gh)
        for b in range(B):
            for t in range(T):
                p = L0[b] + t
                orot = orc.rotate_group_f64(K[b, t, q * gh:(q + 1) * gh].reshape(-1).float().numpy()
                                            .astype(np.float64), pg)
                for j in range(gh):
                    h = q * gh + j
                    c, s, z = orc.quantize_rows(grot[b, t, j * D:(j + 1) * D])
                    lg = logical(gc, b, h, p)
                    assert np.array_equal(lg[0], c[0]) and np.array_equal(lg[2], s[0])
                    assert np.array_equal(lg[3], z[0])
                    lo = logical(oc, b, h, p)
                    n_codes += D
                    n_diff += int((lo[0] != lg[0]).sum())
                    if np.array_equal(lo[2], lg[2]) and np.array_equal(lo[3], lg[3]):
                        assert near_tie_ok(orot[j * D:(j + 1) * D], lo[0], lg[0], lo[2], lo[3])
    for h in range(Hkv):
        rows = V[:, :, h].reshape(-1, D).cuda()
        vrot = kvq.kvq_debug_rotate_f32(rows, 1, perm=torch.from_numpy(
            np.ascontiguousarray(perm[1, h * D:(h + 1) * D])).cuda()).cpu().numpy().reshape(B, T, D)
        for b in range(B):
            for t in range(T):
                c, s, z = orc.quantize_rows(vrot[b, t])
                lg = logical(gc, b, h, L0[b] + t)
                assert np.array_equal(lg[1], c[0]) and np.array_equal(lg[4], s[0])
                assert np.array_equal(lg[5], z[0])
    # each differing key code above is a near tie; their rate is measured
    # over more than a million codes in test_gpu_parity.py
    assert n_diff < n_codes
    for b in range(B):
        last = (L0[b] + T + 15) // 16
        assert not gc.blocks[b, :, last:].any()


def oracle_prerope_cache(w, gh, perm, lens, cap):
    oc = orc.Cache(w.B, w.Hkv, cap, 0)
    for b in range(w.B):
        k, v = W.kv_rows(w, b, 0, lens[b], "cpu")
        sub = orc.Cache(1, w.Hkv, cap, 0)
        sl = np.zeros(1, np.int32)
        assert orc.append_prerope(sub, f16bits(k[None]), f16bits(v[None]), gh, perm, sl) == 0
        oc.blocks[b] = sub.blocks[0]
    return oc


def gpu_prerope_decode(cache, Q, gh, perm_t, lens_t, max_ctx):
    ws = kvq.prerope_workspace(cache.B, Q.shape[1], cache.Hkv, gh, max_ctx)
    ws.fill_(0xFF)
    out = torch.empty_like(Q)
    kvq.kvq_prerope_decode(Q.contiguous(), cache, gh, perm_t, BASE, lens_t, max_ctx, ws, out)
    return out


PR_DECODE_CASES = [
    # gh, G, Hkv, lengths (gh = G = 1 runs the four-positions-per-step kernel)
    (1, 1, 2, [1, 15, 16, 17, 300, 1000]),
    (1, 1, 3, [2, 3, 4, 5, 7, 64, 65, 259, 4099]),
    (1, 1, 1, [8191]),
    (2, 1, 4, [33, 512, 2047]),
    (2, 2, 2, [5, 19, 800]),
    (4, 2, 4, [4, 257, 1500]),
    (8, 1, 8, [16, 600]),
    (1, 8, 2, [64, 999]),
    (2, 4, 2, [129, 3]),
]


@pytest.mark.parametrize("gh,G,Hkv,lens", PR_DECODE_CASES)
def test_prerope_decode_matches_oracle(gh, G, Hkv, lens):
    w = _wl(230 + gh * 10 + G, len(lens), Hkv, G)
    perm = W.prerope_perm(w, gh)
    cap = ((max(lens) + 15) // 16) * 16
    oc = oracle_prerope_cache(w, gh, perm, lens, cap)
    Q = W.queries(w, "cpu")
    sl = np.array(lens, np.int32)
    ref, st = orc.decode_prerope(oc, f16bits(Q), gh, perm, BASE, sl, n_threads=8)
    assert st == 0
    cache = kvq.KVCache(w.B, Hkv, cap)
    cache.blocks.copy_(torch.from_numpy(oc.blocks.reshape(-1)))
    out = gpu_prerope_decode(cache, Q.cuda(), gh, torch.from_numpy(perm).cuda(),
                             torch.from_numpy(sl).cuda(), max(lens))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    err = rel_err(out.cpu().numpy(), ref)
    assert err.max() <= DEC_TOL, err.max()


@pytest.mark.parametrize("gh", [2, 1])
def test_prerope_decode_long_context(gh):
    """Positions up to 131071: the RoPE angles are reduced in fp64 (per block,
    or every 64 steps of four positions for gh = 1) and advanced in fp32 in
    between."""
    L = 131072
    w = _wl(251, 1, 2, 1)
    perm = W.prerope_perm(w, gh)
    oc = oracle_prerope_cache(w, gh, perm, [L], L)
    Q = W.queries(w, "cpu")
    sl = np.array([L], np.int32)
    ref, st = orc.decode_prerope(oc, f16bits(Q), gh, perm, BASE, sl, n_threads=8)
    assert st == 0
    cache = kvq.KVCache(1, 2, L)
    cache.blocks.copy_(torch.from_numpy(oc.blocks.reshape(-1)))
    out = gpu_prerope_decode(cache, Q.cuda(), gh, torch.from_numpy(perm).cuda(),
                             torch.from_numpy(sl).cuda(), L)
    err = rel_err(out.cpu().numpy(), ref)
    assert err.max() <= DEC_TOL, err.max()


@pytest.mark.parametrize("gh,G", [(2, 2), (1, 1)])
@pytest.mark.parametrize("paged", [False, True])
def test_prerope_append_then_decode(paged, gh, G):
    """GPU appends (37, 300 and single tokens) then the GPU decode, against the
    oracle's append + decode of the same tokens."""
    Hkv, B = 4, 3
    w = _wl(260 + paged + 10 * gh, B, Hkv, G)
    perm = W.prerope_perm(w, gh)
    pt = torch.from_numpy(perm).cuda()
    L0 = [0, 5, 16]
    chunks = [37, 300, 1, 1]
    cap = ((max(L0) + sum(chunks) + 15) // 16) * 16
    nblk = cap // 16
    if paged:
        num_blocks = B * nblk + 5
        tperm = torch.randperm(num_blocks, generator=torch.Generator().manual_seed(8))[:B * nblk]
        cache = kvq.PagedKVCache(B, Hkv, cap, num_blocks, tperm.view(B, nblk).to(torch.int32).cuda())
    else:
        cache = kvq.KVCache(B, Hkv, cap)
    oc = orc.Cache(B, Hkv, cap, 0)
    sl = torch.tensor(L0, dtype=torch.int32, device="cuda")
    osl = np.array(L0, np.int32)
    pos = list(L0)
    for T in chunks:
        K = torch.stack([W.kv_rows(w, b, pos[b], pos[b] + T, "cpu")[0] for b in range(B)])
        V = torch.stack([W.kv_rows(w, b, pos[b], pos[b] + T, "cpu")[1] for b in range(B)])
        kvq.kvq_prerope_append(K.cuda(), V.cuda(), gh, pt, cache, sl)
        assert orc.append_prerope(oc, f16bits(K), f16bits(V), gh, perm, osl) == 0
        pos = [p + T for p in pos]
    Q = W.queries(w, "cpu")
    ref, st = orc.decode_prerope(oc, f16bits(Q), gh, perm, BASE, osl, n_threads=8)
    assert st == 0
    out = gpu_prerope_decode(cache, Q.cuda(), gh, pt, sl, max(pos))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    assert list(sl.cpu().numpy()) == pos
    err = rel_err(out.cpu().numpy(), ref)
    assert err.max() <= DEC_TOL, err.max()


def test_prerope_bad_length_and_unsupported():
    w = _wl(270, 2, 2, 1)
    perm = torch.from_numpy(W.prerope_perm(w, 1)).cuda()
    cache = kvq.KVCache(2, 2, 64)
    Q = torch.randn((2, 2, D), device="cuda").half()
    sl = torch.tensor([0, 65], dtype=torch.int32, device="cuda")
    out = gpu_prerope_decode(cache, Q, 1, perm, sl, 64)
    torch.cuda.synchronize()
    assert not out.float().abs().sum().item()
    assert kvq.kvq_get_status(cache) == kvq.KVQ_DEV_BAD_LEN
    with pytest.raises(kvq.KvqError) as e:                       # G * gh > 8
        Q8 = torch.randn((2, 16, D), device="cuda").half()
        kvq.kvq_prerope_decode(Q8, cache, 2, perm, BASE, sl, 64,
                               kvq.prerope_workspace(2, 16, 2, 2, 64), torch.empty_like(Q8))
    assert e.value.code == 2


# --- with fp16 sinks (RotateKV items ii and iii together) -----------------------------------------

@pytest.mark.parametrize("gh,G", [(2, 2), (1, 1)])
@pytest.mark.parametrize("identified", [False, True])
def test_prerope_sinks_append_and_decode(identified, gh, G):
    """Leading sinks (the first 4 positions) or identified ones (massive
    tokens): sink rows hold the pre-RoPE key exactly as given and the fp16
    of the kernel's rotated value; INT2 slots zero (identified: the K-scale
    marker); the decode against the oracle over appends of 37, 300 and 1
    tokens."""
    Hkv, B, S = 4, 3, 4
    w = W.custom(seed=280 + identified + 10 * gh, B=B, Hq=Hkv * G, Hkv=Hkv, mode=1, sink=S, k_outliers=4,
                 sink_key_scale=50.0, massive_rate=0.01 if identified else 0.0)
    perm = W.prerope_perm(w, gh)
    pt = torch.from_numpy(perm).cuda()
    L0 = [0, 2, 16]
    chunks = [37, 300, 1]
    cap = ((max(L0) + sum(chunks) + 15) // 16) * 16
    cache = kvq.KVCache(B, Hkv, cap, S, identified_sinks=identified)
    oc = orc.Cache(B, Hkv, cap, S, identified=identified)
    sl = torch.tensor(L0, dtype=torch.int32, device="cuda")
    osl = np.array(L0, np.int32)
    pos = list(L0)
    Ks, Vs = [], []
    for T in chunks:
        K = torch.stack([W.kv_rows(w, b, pos[b], pos[b] + T, "cpu")[0] for b in range(B)])
        V = torch.stack([W.kv_rows(w, b, pos[b], pos[b] + T, "cpu")[1] for b in range(B)])
        if identified:
            act = np.stack([W.activations(w, b, pos[b], pos[b] + T) for b in range(B)])
            kvq.kvq_identify_sinks(torch.from_numpy(act).cuda(), W.MASSIVE_TAU, cache, sl)
            orc.identify_sinks(oc, act, W.MASSIVE_TAU, osl)
        kvq.kvq_prerope_append(K.cuda(), V.cuda(), gh, pt, cache, sl)
        assert orc.append_prerope(oc, f16bits(K), f16bits(V), gh, perm, osl) == 0
        Ks.append((list(pos), K, V))
        pos = [p + T for p in pos]
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    if identified:
        assert np.array_equal(cache.sink_count.cpu().numpy(), oc.sink_count)
        assert np.array_equal(cache.sink_pos.cpu().numpy(), oc.sink_pos)
        assert (oc.sink_count >= 1).all()
    gks, gvs = f16bits(cache.k_sink), f16bits(cache.v_sink)
    gb = cache.block_view().cpu().numpy()
    n_sink = 0
    for starts, K, V in Ks:
        T = K.shape[1]
        for h in range(Hkv):
            vrot = kvq.kvq_debug_rotate_f32(V[:, :, h].reshape(-1, D).cuda(), 1, perm=torch.from_numpy(
                np.ascontiguousarray(perm[1, h * D:(h + 1) * D])).cuda()).cpu().numpy().reshape(B, T, D)
            for b in range(B):
                plist = (list(oc.sink_pos[b, :oc.sink_count[b]]) if identified
                         else list(range(S)))
                for t in range(T):
                    p = starts[b] + t
                    if p not in plist:
                        continue
                    j = plist.index(p)
                    assert np.array_equal(gks[b, h, j], f16bits(K[b, t, h]))
                    assert np.array_equal(gvs[b, h, j], orc.f32_to_f16_bits(vrot[b, t]))
                    kb, vb, ks, kz, vs, vz = orc.load_token(gb[b, h, p // 16], p % 16)
                    assert not kb.any() and not vb.any() and not kz.any() and not vs.any()
                    assert list(ks) == ([0x7E00] * 4 if identified else [0] * 4)
                    n_sink += 1
    assert n_sink > 0
    Q = W.queries(w, "cpu")
    ref, st = orc.decode_prerope(oc, f16bits(Q), gh, perm, BASE, osl, n_threads=8)
    assert st == 0
    out = gpu_prerope_decode(cache, Q.cuda(), gh, pt, sl, max(pos))
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    err = rel_err(out.cpu().numpy(), ref)
    assert err.max() <= DEC_TOL, err.max()
