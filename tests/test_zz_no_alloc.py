"""The allocation-free decode entry point (kvq_decode_attention_noalloc).

It exists for callers that cannot allocate device memory: it takes no
workspace and uses a fixed device array inside the library instead.  These
tests call it through the C ABI, twice in a row on the same inputs, and
check each result against the regular entry point (caller workspace) and
against the CPU oracle, within the decode tolerance the other tests use.
They also check that a shape too large for the fixed array is refused on
the host.  The file is named so that
pytest collects it last, and it builds its own inputs, so it passes both on
its own in a fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import rotated_int2_kv_head_b200 as kvq
import workloads as W

pytestmark = pytest.mark.gpu
DEC_TOL = 2e-3


def rows_close(a, b):
    a = a.float().cpu().numpy().astype(np.float64).reshape(-1, 128)
    b = b.double().cpu().numpy().reshape(-1, 128)
    err = np.abs(a - b).max(axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-30)
    return err.max()


@pytest.mark.parametrize("G,mode,S", [(1, 0, 0), (4, 0, 4), (2, 1, 0)])
def test_noalloc_matches_workspace_decode_twice(G, mode, S):
    from rotated_int2_kv_head_b200 import build
    build.build()
    Hkv = 2
    lens = [1, 37, 300, 1025]
    w = W.custom(seed=77 + G, B=len(lens), Hq=Hkv * G, Hkv=Hkv, mode=mode, sink=S,
                 k_outliers=4, sink_key_scale=50.0 if S else 1.0)
    cap = ((max(lens) + 15) // 16) * 16
    Rk, Rv, perm = W.rotations(w)
    rk = torch.from_numpy(Rk).cuda() if Rk is not None else None
    rv = torch.from_numpy(Rv).cuda() if Rv is not None else None
    pm = torch.from_numpy(perm).cuda() if perm is not None else None
    cache = kvq.KVCache(w.B, Hkv, cap, S)
    K, V = W.kv_batch(w, 0, max(lens), "cpu")
    sl = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    kvq.kvq_rotate_quantize_append(K.cuda(), V.cuda(), mode, rk, rv, pm, cache, sl)
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    Q = W.queries(w, "cpu").cuda()

    ws = kvq.decode_workspace(w.B, w.Hq, Hkv, max(lens))
    ref = torch.empty_like(Q)
    kvq.kvq_decode_attention(Q, cache, mode, rk, rv, pm, lens_t, S, max(lens), ws, ref)

    # the CPU oracle's decode over the same cache bytes, as a check
    # independent of the library (the bytes, not the oracle's own append: a
    # near-tie code that differs would move a one-token context by a whole
    # quantization step)
    from oracle import oracle as orc
    oc = orc.Cache(w.B, Hkv, cap, S)
    oc.blocks[:] = cache.block_view().cpu().numpy()
    if S:
        oc.k_sink[:] = W.f16_bits(cache.k_sink)
        oc.v_sink[:] = W.f16_bits(cache.v_sink)
    ref_o, _ = orc.decode(oc, W.f16_bits(Q), mode, Rk, Rv, perm, np.array(lens, np.int32))
    ref_o = torch.from_numpy(ref_o)

    for _ in range(2):                      # two calls in a row share the array
        out = torch.full_like(Q, float("nan"))
        kvq.kvq_decode_attention_noalloc(Q, cache, mode, rk, rv, pm, lens_t, S, max(lens), out)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert rows_close(out, ref) <= DEC_TOL
        assert rows_close(out, ref_o) <= DEC_TOL
    assert kvq.kvq_get_status(cache) == 0


def test_noalloc_refuses_shapes_beyond_its_array():
    from rotated_int2_kv_head_b200 import build
    build.build()
    B, H = 256, 32
    need = kvq.kvq_decode_workspace_size(B, H, H, 16)
    assert need > (4 << 20)
    cache = kvq.KVCache(B, H, 16, 0)
    Q = torch.zeros((B, H, 128), dtype=torch.float16, device="cuda")
    out = torch.empty_like(Q)
    R = torch.zeros((H, 128, 128), dtype=torch.float32, device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attention_noalloc(Q, cache, 0, R, R, None, lens, 0, 16, out)
    assert e.value.code == 5                # KVQ_ERR_WORKSPACE
