"""KVLinC on the GPU ("KVLinC : KV Cache Quantization with Hadamard Rotation
and Linear Correction", abstract): values Hadamard-rotated, keys corrected by
lightweight linear adapters at decode.  kvq_decode_attention_adapter against
the oracle's adapter decode (orc_decode_adapter) over the same cache bytes,
within 2e-3 * ||o|| per (sequence, query head); a zero adapter is the plain
decode bit for bit; bad adapter arguments are refused on the host."""
import numpy as np
import pytest
import torch

import rotated_int2_kv_head_b200 as kvq
import workloads as W
from oracle import oracle as orc
from oracle import np_mini

from kvq_testlib import D, f16bits, rel_err, rot_tensors, upload_oracle_cache

pytestmark = pytest.mark.gpu
DEC_TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def built():
    from rotated_int2_kv_head_b200 import build
    build.build()
    torch.cuda.init()


def oracle_cache(w, lens, cap, Rk, Rv, perm):
    oc = orc.Cache(w.B, w.Hkv, cap, w.sink)
    for b in range(w.B):
        k, v = W.kv_rows(w, b, 0, lens[b], "cpu")
        sub = orc.Cache(1, w.Hkv, cap, w.sink)
        sl = np.zeros(1, np.int32)
        orc.append(sub, f16bits(k[None]), f16bits(v[None]), w.mode, Rk, Rv, perm, sl)
        oc.blocks[b] = sub.blocks[0]
        if w.sink:
            oc.k_sink[b] = sub.k_sink[0]
            oc.v_sink[b] = sub.v_sink[0]
    return oc


def adapters(Hkv, r, seed, scale=0.15):
    g = torch.Generator().manual_seed(seed)
    U = (torch.randn((Hkv, D, r), generator=g) * scale).float()
    V = (torch.randn((Hkv, D, r), generator=g) * scale).float()
    return U, V


CASES = [
    # G, mode, S, rank, q_len, rotation
    (1, 0, 0, 16, 1, "random"),
    (4, 0, 4, 128, 1, "random"),
    (2, 1, 0, 1, 1, "fwht"),
    (1, 0, 4, 32, 1, "kvlinc"),        # keys unrotated, values Hadamard-rotated
    (2, 0, 0, 8, 2, "kvlinc"),         # two new tokens per sequence, causal
]


@pytest.mark.parametrize("G,mode,S,r,q_len,rot", CASES)
def test_adapter_decode_matches_oracle(G, mode, S, r, q_len, rot):
    Hkv = 2
    lens = [q_len, 17, 300, 1100]              # the shortest holds its q_len new tokens
    # sink keys at the scale of the others, so that the INT2 keys (which the
    # adapter corrects) carry the attention
    w = W.custom(seed=400 + G + r, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=mode, sink=S,
                 k_outliers=4)
    cap = ((max(lens) + 15) // 16) * 16
    Rk, Rv, perm = W.rotations(w)
    if rot == "kvlinc":
        Rk = np.stack([np.eye(D, dtype=np.float32)] * Hkv)
        Rv = np.stack([(np_mini.hadamard(D) / np.sqrt(D)).astype(np.float32)] * Hkv)
    oc = oracle_cache(w, lens, cap, Rk, Rv, perm)
    cache = upload_oracle_cache(oc)
    rk = torch.from_numpy(Rk).cuda() if Rk is not None else None
    rv = torch.from_numpy(Rv).cuda() if Rv is not None else None
    pm = torch.from_numpy(perm).cuda() if perm is not None else None
    U, V = adapters(Hkv, r, 7 + r)
    g = torch.Generator().manual_seed(33 + q_len)
    shape = (w.B, w.Hq, D) if q_len == 1 else (w.B, w.Hq, q_len, D)
    Q = torch.randn(shape, generator=g).to(torch.float16)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = kvq.decode_workspace(w.B, w.Hq * q_len, Hkv, max(lens))
    ws.fill_(0xFF)
    out = torch.full(shape, float("nan"), dtype=torch.float16, device="cuda")
    kvq.kvq_decode_attention_adapter(Q.cuda(), cache, mode, rk, rv, pm, U.cuda(), V.cuda(), sl,
                                     S, max(lens), ws, out)
    torch.cuda.synchronize()
    assert kvq.kvq_get_status(cache) == 0
    got = out.cpu().numpy()
    for i in range(q_len):
        li = np.array(lens, np.int32) - (q_len - 1 - i)
        Qi = Q if q_len == 1 else Q[:, :, i].contiguous()
        ref, st = orc.decode_adapter(oc, f16bits(Qi), mode, Rk, Rv, perm, li, U.numpy(),
                                     V.numpy(), n_threads=8)
        assert st == 0
        err = rel_err(got if q_len == 1 else got[:, :, i], ref)
        assert err.max() <= DEC_TOL, (i, err.max())
        # the adapter changes the result (it is not a no-op at this size)
        plain, _ = orc.decode(oc, f16bits(Qi), mode, Rk, Rv, perm, li, n_threads=8)
        assert rel_err(plain.astype(np.float32), ref).max() > 10 * DEC_TOL


@pytest.mark.parametrize("mode", [0, 1])
def test_zero_adapter_is_the_plain_decode_bit_for_bit(mode):
    Hkv, G = 2, 2
    lens = [40, 333]
    w = W.custom(seed=450 + mode, B=2, Hq=Hkv * G, Hkv=Hkv, mode=mode, sink=4, k_outliers=4)
    cap = 336
    rt, rn = rot_tensors(w)
    oc = oracle_cache(w, lens, cap, *rn)
    cache = upload_oracle_cache(oc)
    Q = W.queries(w, "cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = kvq.decode_workspace(2, w.Hq, Hkv, max(lens))
    plain = torch.empty_like(Q)
    kvq.kvq_decode_attention(Q, cache, mode, *rt, sl, 4, max(lens), ws, plain)
    Z = torch.zeros((Hkv, D, 3), dtype=torch.float32, device="cuda")
    out = torch.empty_like(Q)
    kvq.kvq_decode_attention_adapter(Q, cache, mode, *rt, Z, Z, sl, 4, max(lens), ws, out)
    torch.cuda.synchronize()
    assert torch.equal(out, plain)


def test_adapter_rejects_bad_arguments():
    cache = kvq.KVCache(1, 2, 64)
    L = kvq.lib()
    Q = torch.zeros((1, 2, D), dtype=torch.float16, device="cuda")
    R = torch.zeros((2, D, D), dtype=torch.float32, device="cuda")
    U = torch.zeros((2, D, 4), dtype=torch.float32, device="cuda")
    sl = torch.ones(1, dtype=torch.int32, device="cuda")
    ws = kvq.decode_workspace(1, 2, 2, 64)
    import ctypes as C
    args = lambda u, v, r: (Q.data_ptr(), 2, 1, 0, C.byref(cache.desc), 0, R.data_ptr(),
                            R.data_ptr(), None, u, v, r, sl.data_ptr(), 0, 64, ws.data_ptr(),
                            ws.numel(), Q.data_ptr(), None)
    assert L.kvq_decode_attention_adapter(*args(U.data_ptr(), U.data_ptr(), 0)) == 1
    assert L.kvq_decode_attention_adapter(*args(U.data_ptr(), U.data_ptr(), 129)) == 1
    assert L.kvq_decode_attention_adapter(*args(None, U.data_ptr(), 4)) == 1
    assert L.kvq_decode_attention_adapter(*args(U.data_ptr() + 2, U.data_ptr(), 4)) == 2
    torch.cuda.synchronize()
